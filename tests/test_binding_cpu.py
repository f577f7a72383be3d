"""The Python binding refuses host tensors: there is no CPU path to fall back to.

Every public call that takes tensors must raise before anything reaches the
library when handed CPU tensors, so a caller without a GPU (or with its data
on the host) gets an error, never a silently computed result.  Runs without a
GPU: the checks are host-side argument marshalling.
"""
import pytest
import torch

import uncertainty_routed_heterogeneous_b200 as heta

GRID, WIN = (2, 4, 4), (1, 3, 3)
N = GRID[0] * GRID[1] * GRID[2]


def _qkv():
    return [torch.zeros((1, 2, N, 64), dtype=torch.bfloat16) for _ in range(3)]


CALLS = {
    "route": lambda: heta.route(torch.zeros((1, N)), 4),
    "route_threshold": lambda: heta.route_threshold(torch.zeros((1, N)), 0.9),
    "route_swap": lambda: heta.route_swap(torch.zeros((1, 4), dtype=torch.int32), N, 1, 7, 0),
    "route_swap_blocks": lambda: heta.route_swap_blocks(torch.zeros((1, 4), dtype=torch.int32),
                                                        N, 1, 7, 0, 2),
    "attention": lambda: heta.attention(*_qkv(), GRID, WIN,
                                        torch.zeros((1, 4), dtype=torch.int32)),
    "attention_noalloc": lambda: heta.attention_noalloc(*_qkv(), GRID, WIN,
                                                        torch.zeros((1, 4), dtype=torch.int32)),
    "attention_counts": lambda: heta.attention_counts(*_qkv(), GRID, WIN,
                                                      torch.zeros((1, 4), dtype=torch.int32),
                                                      torch.zeros(1, dtype=torch.int32)),
    "uncertainty": lambda: heta.uncertainty(torch.zeros((1, N, 64), dtype=torch.bfloat16),
                                            torch.zeros(64)),
}


@pytest.mark.parametrize("name", sorted(CALLS))
def test_host_tensors_are_refused(name):
    with pytest.raises(TypeError, match="CUDA tensor"):
        CALLS[name]()


def test_every_tensor_call_is_covered():
    tensor_calls = {"route", "route_threshold", "route_swap", "route_swap_blocks", "attention",
                    "attention_noalloc", "attention_counts", "uncertainty"}
    assert tensor_calls <= set(heta.__all__)
    assert tensor_calls == set(CALLS)
