"""The no-allocation entry point, sagesla_forward_no_alloc, through the C ABI.

Callers that cannot allocate device memory (a host integration that only passes input and
output buffers, a memory pool that may not grow, a process that must not call cudaMalloc once
loaded) use this entry point: the forward's scratch lives in a device array built into the
library. These tests check that it rejects problems larger than that array, that the array's size in
the Python binding is the header's, and that two consecutive calls on different problems (the
larger first, so that the second runs on the first one's leftover scratch) give exactly the
outputs of the ordinary sagesla_forward with a caller workspace: the forward is deterministic,
so any difference would be stale scratch showing through.
"""
import ctypes
import os
import re

import pytest
import torch

import sparse_bit_attention_b200 as sba
from sparse_bit_attention_b200 import binding, inputs
from sparse_bit_attention_b200.build import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    build()
    return binding.load_library()


def _no_alloc(lib, q, k, v, out, ratio, stream=None):
    vq, vk, vv, vo = (binding._view(x) for x in (q, k, v, out))
    return lib.sagesla_forward_no_alloc(ctypes.byref(vq), ctypes.byref(vk), ctypes.byref(vv),
                                        ratio, 64, ctypes.byref(vo), stream)


def test_rejects_problems_larger_than_the_scratch_area(lib):
    # 8 heads x 32768 tokens need ~0.3 GB of scratch; refused before any CUDA call.
    shape = (1, 8, 32768, 128)
    assert sba.sagesla_workspace_size(*shape, 0.1) > binding.NO_ALLOC_SCRATCH_BYTES
    q = torch.empty(shape, dtype=torch.bfloat16)
    out = torch.empty(shape, dtype=torch.float32)
    assert _no_alloc(lib, q, q, q, out, 0.1) == 3          # SAGESLA_ERR_WORKSPACE
    assert _no_alloc(lib, q, q, q, out, 0.0) == 1          # invalid ratio


def test_scratch_size_matches_the_header():
    text = open(os.path.join(ROOT, "include", "sagesla.h")).read()
    m = re.search(r"#define SAGESLA_NO_ALLOC_SCRATCH_BYTES \((\d+)ull << (\d+)\)", text)
    assert m, "SAGESLA_NO_ALLOC_SCRATCH_BYTES not found"
    assert binding.NO_ALLOC_SCRATCH_BYTES == int(m.group(1)) << int(m.group(2))


@pytest.mark.gpu
def test_no_alloc_matches_forward_on_two_calls_in_a_row(lib):
    dev = torch.device("cuda:0")
    stream = ctypes.c_void_p(torch.cuda.current_stream(dev).cuda_stream)
    for n, ratio, seed in [(1000, 0.25, 31), (700, 0.1, 32)]:
        q, k, v = (x.to(dev) for x in inputs.make_random(1, 2, n, seed, k_offset_std=1.0))
        ref = sba.sagesla_forward(q, k, v, ratio)
        out = torch.full(q.shape, float("nan"), dtype=torch.float32, device=dev)
        assert _no_alloc(lib, q, k, v, out, ratio, stream) == 0
        torch.cuda.synchronize()
        assert torch.equal(out, ref)
