"""w8a8_linear_fused_noalloc: the whole-layer entry point for callers that
cannot allocate device memory (a plugin inside a runtime that reserved all
device memory up front, or code with a fixed memory budget, and so no
workspace to hand over).  It must give the same output as w8a8_linear_fused
with a caller workspace, call after call, although every call reuses the one
static scratch array inside the library.

This file is named to be collected last, so a run that stops at the first
failure has already run every other test; it also passes on its own in a
fresh process.
"""
from __future__ import annotations

import ctypes

import numpy as np
import pytest
import torch

import oracle
import synth
import w8a8_int8_dynamic_token_b200 as w8a8
from w8a8_int8_dynamic_token_b200 import binding as B

from gpu_util import bits_of, check_y, sample_rows, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from w8a8_int8_dynamic_token_b200 import build
    build.build()
    torch.cuda.set_device(0)
    yield
    assert w8a8.last_device_error() == B.W8A8_OK


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _noalloc(x, Wq, s_w, bias, y):
    M, K = x.shape
    N = Wq.shape[0]
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return B.w8a8_linear_fused_noalloc(_p(x), M, K, x.stride(0), _p(Wq), _p(s_w), _p(bias), N,
                                       _p(y), y.stride(0), stream)


# (M, N, K): a ragged multi-tile GEMM case, the GEMV path (M = 2), and the
# fused-QKV projection at full size (M * K = 13.4 MB, inside the 16 MiB limit).
@pytest.mark.parametrize("M,N,K", [(300, 520, 3072), (2, 1032, 3072), (4352, 9216, 3072)])
def test_noalloc_matches_workspace_entry_point_on_consecutive_calls(M, N, K):
    w = synth.make_w(N, K, seed=11)
    wq_ref, sw_ref = oracle.quantize_weights(w)
    Wq, s_w = torch.from_numpy(wq_ref).cuda(), torch.from_numpy(sw_ref).cuda()
    b_bits = synth.make_bias(N, 11)
    b = to_dev(b_bits)
    for call in range(2):   # two calls in a row, different activations each time
        x_bits = synth.make_x(M, K, "studentt", seed=100 + call)
        x = to_dev(x_bits)
        y_static = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
        assert _noalloc(x, Wq, s_w, b, y_static) == B.W8A8_OK
        y_ws = w8a8.linear_fused(x, Wq, s_w, b)          # existing entry point, caller workspace
        torch.cuda.synchronize()
        assert np.array_equal(bits_of(y_static), bits_of(y_ws)), f"call {call}"
        rows = sample_rows(M, seed=call, n_random=32)
        q_ref, s_ref = oracle.quant_rows(x_bits[rows])
        y32, y_ref = oracle.epilogue(oracle.gemm_i32(q_ref, wq_ref), s_ref, sw_ref, b_bits)
        assert check_y(bits_of(y_static)[rows], y_ref, y32, f"noalloc call {call}") == 0


def test_noalloc_rejects_sizes_beyond_its_scratch():
    dev = "cuda"
    # M * K = 53.5 MB > 16 MiB
    x = torch.zeros((4352, 12288), dtype=torch.bfloat16, device=dev)
    Wq = torch.zeros((8, 12288), dtype=torch.int8, device=dev)
    s_w = torch.ones(8, device=dev)
    y = torch.empty((4352, 8), dtype=torch.bfloat16, device=dev)
    assert _noalloc(x, Wq, s_w, None, y) == B.W8A8_ERR_WORKSPACE
    # more than 16384 rows
    x = torch.zeros((16385, 16), dtype=torch.bfloat16, device=dev)
    Wq = torch.zeros((8, 16), dtype=torch.int8, device=dev)
    y = torch.empty((16385, 8), dtype=torch.bfloat16, device=dev)
    assert _noalloc(x, Wq, s_w, None, y) == B.W8A8_ERR_WORKSPACE
