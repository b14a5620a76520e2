"""The staging copy entry point (jssa_copy_mapped) on the GPU: pinned host memory to the device
and back, interior rows of a pinned buffer, and rejection of pageable host memory."""
import pytest
import torch

import token_level_sparse_jssa_b200 as jssa

pytestmark = pytest.mark.gpu


def test_pinned_host_to_device_and_back():
    g = torch.Generator().manual_seed(7)
    n_rows, row = 6, 3072  # bf16 elements per row (6 KB, whole 16-byte words)
    host = torch.randn(n_rows, row, generator=g).to(torch.bfloat16).pin_memory()
    dev = torch.empty(row, dtype=torch.bfloat16, device="cuda")
    back = torch.zeros(n_rows, row, dtype=torch.bfloat16).pin_memory()
    for i in range(n_rows):  # interior rows of the pinned buffer, in and out
        jssa.copy_mapped(dev, host[i])
        assert torch.equal(dev.cpu(), host[i])
        jssa.copy_mapped(back[i], dev)
    torch.cuda.synchronize()
    assert torch.equal(back, host)


def test_device_to_device_and_partial_length():
    src = torch.arange(4096, dtype=torch.int32, device="cuda")
    dst = torch.full((4096,), -1, dtype=torch.int32, device="cuda")
    jssa.copy_mapped(dst, src, nbytes=1024 * 4)
    torch.cuda.synchronize()
    assert torch.equal(dst[:1024], src[:1024])
    assert bool((dst[1024:] == -1).all())


def test_pageable_host_memory_is_rejected():
    host = torch.ones(1024, dtype=torch.float32)  # not pinned
    dev = torch.empty(1024, dtype=torch.float32, device="cuda")
    with pytest.raises(jssa.JssaError) as e:
        jssa.copy_mapped(dev, host)
    assert e.value.code == 1
    torch.cuda.synchronize()
