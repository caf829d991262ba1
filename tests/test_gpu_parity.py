"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle,
element by element, on seeded inputs.

The bar: s_a bit-equal, q byte-equal, int32 accumulators equal, every bf16
output within 1 bf16 ulp of the oracle's fp32 epilogue value (bit-equal
expected, and counted), all outputs finite.  Small cases are compared in full;
the full-size workloads compare s_a and q in full and y on sampled rows (seeded
random rows plus both sides of every 128-row tile boundary), which the oracle
computes row by row.
"""
from __future__ import annotations

import functools

import numpy as np
import pytest
import torch

import oracle
import synth
import w8a8_int8_dynamic_token_b200 as w8a8
from w8a8_int8_dynamic_token_b200 import binding as B

from gpu_util import bf16_to_f64, bits_of, check_y, f32_bits, sample_rows, to_dev

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


def _quant_check(x_bits, q_dev, s_dev):
    q_ref, s_ref = oracle.quant_rows(x_bits)
    s = s_dev.cpu().numpy()
    assert np.array_equal(f32_bits(s), f32_bits(s_ref)), "s differs"
    q = q_dev.cpu().numpy()
    assert np.array_equal(q, q_ref), f"q differs at {np.argwhere(q != q_ref)[:5].tolist()}"
    return q_ref, s_ref


# ----------------------------------------------------------------- quantization

@pytest.mark.parametrize("M,K,kind", [
    (64, 256, "outlier20"), (300, 3072, "studentt"), (17, 12288, "gelu"), (5, 16, "normal"),
    (1000, 4096, "normal"), (3, 133120, "normal"), (7, 2064, "studentt"), (33, 24576, "gelu"),
])
def test_quant_act_bitexact(M, K, kind):
    x = synth.make_x(M, K, kind, seed=M)
    q, s = w8a8.quant_act(to_dev(x))
    torch.cuda.synchronize()
    _quant_check(x, q, s)


def test_quant_act_strided_rows():
    M, K, ld = 50, 1024, 1056
    full = synth.make_x(M, ld, "studentt", seed=9)
    xd = to_dev(full)[:, :K]
    assert xd.stride(0) == ld
    q, s = w8a8.quant_act(xd)
    torch.cuda.synchronize()
    _quant_check(np.ascontiguousarray(full[:, :K]), q, s)


def _edge_rows(K):
    rows = []
    rows.append(np.zeros(K))                                   # zero row
    r = np.zeros(K); r[K // 3] = -3.0; rows.append(r)          # single nonzero
    r = np.zeros(K); r[0] = 127.0; r[1:254] = np.arange(-126.5, 126.5, 1.0)[:253]; rows.append(r)
    r = np.zeros(K); r[0] = 254.0; r[1:10] = [5, 7, -3, 1, 3, -1, 63.5, -63.5, 0.5]; rows.append(r)
    rows.append(np.full(K, 2.0 ** -130))                       # subnormal bf16 everywhere
    r = np.full(K, 2.0 ** -133); r[5] = 2.0 ** -127; rows.append(r)  # subnormal, one larger
    r = np.linspace(-1e30, 1e30, K); rows.append(r)            # huge magnitudes
    r = np.full(K, -7.0); rows.append(r)                       # constant negative row
    rng = np.random.default_rng(4)
    rows.append(rng.standard_normal(K) * 1e-20)                # tiny normal values
    return synth.to_bf16_bits(np.stack(rows))


@pytest.mark.parametrize("K", [256, 3072])
def test_quant_edge_rows(K):
    x = _edge_rows(K)
    q, s = w8a8.quant_act(to_dev(x))
    torch.cuda.synchronize()
    q_ref, s_ref = _quant_check(x, q, s)
    assert s_ref[0] == 0 and not q_ref[0].any()
    assert q_ref[4].min() == 127                                # all-equal subnormal row


def test_division_free_quant_step_exhaustive():
    # every positive finite bf16 row maximum a with every bf16 x, |x| <= a
    checked, bad = w8a8.binding.selftest_quant_exhaustive()
    assert bad == 0
    # pairs on the fast step: all maxima except the tiniest (whose scale is
    # below 2^-100 and which take the IEEE-division path)
    assert checked > 900_000_000


@pytest.mark.parametrize("N,K", [(264, 3072), (128, 256), (8, 16), (520, 12288)])
def test_quantize_weights_bitexact(N, K):
    w = synth.make_w(N, K, seed=N)
    Wq, s_w = w8a8.quantize_weights(to_dev(w))
    torch.cuda.synchronize()
    _quant_check(w, Wq, s_w)


# ----------------------------------------------------------------- int32 GEMM

GEMM_SHAPES = [(64, 128, 256), (300, 520, 400), (129, 264, 272), (1, 8, 16), (257, 1032, 3072),
               (128, 256, 128), (640, 768, 1024), (200, 136, 12288)]
VARIANTS = [B.VARIANT_GEMM_BN128, B.VARIANT_GEMM_BN256, B.VARIANT_GEMM_PAIR]


@pytest.mark.parametrize("variant", VARIANTS)
@pytest.mark.parametrize("M,N,K", GEMM_SHAPES)
def test_gemm_int32_exact(M, N, K, variant):
    rng = np.random.default_rng(M * 7 + N * 3 + K)
    q = rng.integers(-127, 128, size=(M, K), dtype=np.int8)
    wq = rng.integers(-127, 128, size=(N, K), dtype=np.int8)
    s_a = torch.ones(M, device="cuda")
    s_w = torch.ones(N, device="cuda")
    acc = w8a8.linear(torch.from_numpy(q).cuda(), s_a, torch.from_numpy(wq).cuda(), s_w,
                      acc_debug=True, variant=variant)
    torch.cuda.synchronize()
    assert np.array_equal(acc.cpu().numpy(), oracle.gemm_i32(q, wq))


@pytest.mark.parametrize("variant", VARIANTS + [B.VARIANT_GEMV])
def test_gemm_int32_extremes_at_max_k(variant):
    K = 133120
    rows = 1 if variant == B.VARIANT_GEMV else 2   # GEMV keeps M*K bytes in shared memory
    q = np.full((rows, K), 127, np.int8)
    q[rows - 1] = -127 if rows == 2 else 127
    wq = np.full((8, K), 127, np.int8)
    wq[3, ::2] = -127
    acc = w8a8.linear(torch.from_numpy(q).cuda(), torch.ones(rows, device="cuda"),
                      torch.from_numpy(wq).cuda(), torch.ones(8, device="cuda"),
                      acc_debug=True, variant=variant)
    torch.cuda.synchronize()
    ref = oracle.gemm_i32(q, wq)
    assert ref[0, 0] == 127 * 127 * K and ref[0, 3] == 0
    assert np.array_equal(acc.cpu().numpy(), ref)


# ----------------------------------------------------------------- epilogue

@pytest.mark.parametrize("variant", VARIANTS)
@pytest.mark.parametrize("M,N,K,bias", [(300, 520, 400, True), (300, 520, 400, False),
                                        (129, 1032, 3072, True), (64, 128, 256, True)])
def test_linear_y_vs_oracle(M, N, K, bias, variant):
    x = synth.make_x(M, K, "studentt", seed=1)
    w = synth.make_w(N, K, seed=1)
    b = synth.make_bias(N, seed=1) if bias else None
    q_ref, s_ref = oracle.quant_rows(x)
    wq_ref, sw_ref = oracle.quantize_weights(w)
    acc = oracle.gemm_i32(q_ref, wq_ref)
    y32, y_ref = oracle.epilogue(acc, s_ref, sw_ref, b)
    y = w8a8.linear(torch.from_numpy(q_ref).cuda(), torch.from_numpy(s_ref).cuda(),
                    torch.from_numpy(wq_ref).cuda(), torch.from_numpy(sw_ref).cuda(),
                    to_dev(b) if b is not None else None, variant=variant)
    torch.cuda.synchronize()
    assert check_y(bits_of(y), y_ref, y32, "linear") == 0


def test_linear_strided_output():
    M, N, K, ldy = 130, 136, 256, 200
    x, w, b = synth.make_x(M, K, "normal", 2), synth.make_w(N, K, 2), synth.make_bias(N, 2)
    q_ref, s_ref = oracle.quant_rows(x)
    wq_ref, sw_ref = oracle.quantize_weights(w)
    y32, y_ref = oracle.epilogue(oracle.gemm_i32(q_ref, wq_ref), s_ref, sw_ref, b)
    big = torch.full((M, ldy), float("nan"), dtype=torch.bfloat16, device="cuda")
    out = big[:, :N]
    w8a8.linear(torch.from_numpy(q_ref).cuda(), torch.from_numpy(s_ref).cuda(),
                torch.from_numpy(wq_ref).cuda(), torch.from_numpy(sw_ref).cuda(), to_dev(b),
                out=out)
    torch.cuda.synchronize()
    assert check_y(bits_of(out), y_ref, y32, "strided") == 0
    assert torch.isnan(big[:, N:]).all()          # nothing written past N


# ----------------------------------------------------------------- GEMV (M <= 16)

@pytest.mark.parametrize("M", [1, 2, 3, 5, 8, 16])
@pytest.mark.parametrize("N,K", [(128, 256), (1032, 3072), (64, 12288)])
def test_gemv_fused_and_unfused(M, N, K):
    x, w, b = synth.make_x(M, K, "normal", M), synth.make_w(N, K, M), synth.make_bias(N, M)
    wq_ref, sw_ref = oracle.quantize_weights(w)
    ref = oracle.linear(x, wq_ref, sw_ref, b)
    Wq, s_w = torch.from_numpy(wq_ref).cuda(), torch.from_numpy(sw_ref).cuda()
    assert w8a8.select(M, N, K)["variant_name"] == "gemv"
    y, q, s_a = w8a8.linear_fused(to_dev(x), Wq, s_w, to_dev(b), return_intermediates=True)
    y2 = w8a8.linear_fused(to_dev(x), Wq, s_w, to_dev(b))
    y3 = w8a8.linear(torch.from_numpy(ref["q"]).cuda(), torch.from_numpy(ref["s_a"]).cuda(), Wq,
                     s_w, to_dev(b), variant=B.VARIANT_GEMV)
    acc = w8a8.linear(torch.from_numpy(ref["q"]).cuda(), torch.from_numpy(ref["s_a"]).cuda(), Wq,
                      s_w, acc_debug=True, variant=B.VARIANT_GEMV)
    torch.cuda.synchronize()
    assert np.array_equal(q.cpu().numpy(), ref["q"])
    assert np.array_equal(f32_bits(s_a.cpu().numpy()), f32_bits(ref["s_a"]))
    assert np.array_equal(acc.cpu().numpy(), ref["acc"])
    for yy in (y, y2, y3):
        assert check_y(bits_of(yy), ref["y"], ref["y32"], "gemv") == 0


def test_gemm_variant_at_tiny_m_matches_gemv():
    M, N, K = 3, 264, 512
    x, w, b = synth.make_x(M, K, "normal", 5), synth.make_w(N, K, 5), synth.make_bias(N, 5)
    wq_ref, sw_ref = oracle.quantize_weights(w)
    ref = oracle.linear(x, wq_ref, sw_ref, b)
    args = (torch.from_numpy(ref["q"]).cuda(), torch.from_numpy(ref["s_a"]).cuda(),
            torch.from_numpy(wq_ref).cuda(), torch.from_numpy(sw_ref).cuda(), to_dev(b))
    for v in (B.VARIANT_GEMV, B.VARIANT_GEMM_BN128, B.VARIANT_GEMM_BN256, B.VARIANT_GEMM_PAIR):
        y = w8a8.linear(*args, variant=v)
        torch.cuda.synchronize()
        assert check_y(bits_of(y), ref["y"], ref["y32"], f"variant {v}") == 0


# ----------------------------------------------------------------- whole layer

def test_tiny_config_bitexact():
    c = synth.TINY
    x, w, b = c.x(), c.w(), c.b()
    wq_ref, sw_ref = oracle.quantize_weights(w)
    ref = oracle.linear(x, wq_ref, sw_ref, b)
    Wq, s_w = w8a8.quantize_weights(to_dev(w))
    y, q, s_a = w8a8.linear_fused(to_dev(x), Wq, s_w, to_dev(b), return_intermediates=True)
    torch.cuda.synchronize()
    assert np.array_equal(Wq.cpu().numpy(), wq_ref)
    assert np.array_equal(q.cpu().numpy(), ref["q"])
    assert np.array_equal(f32_bits(s_a.cpu().numpy()), f32_bits(ref["s_a"]))
    assert np.array_equal(bits_of(y), ref["y"])
    # instrument self-check: output/reference norm ratio ~1 (not ~E[s_a])
    r = np.linalg.norm(bf16_to_f64(bits_of(y))) / np.linalg.norm(ref["y32"].astype(np.float64))
    assert abs(r - 1) < 1e-3


@functools.lru_cache(maxsize=8)
def _weights(N, K, seed):
    w = synth.make_w(N, K, seed)
    wq, sw = oracle.quantize_weights(w)
    return w, wq, sw


def _run_layer_sampled(case: synth.LayerCase, check_weights=False):
    """Full-size layer through w8a8_linear_fused; s_a and q compared in full,
    y on sampled rows.  Returns the number of non-bit-equal sampled outputs."""
    x = case.x()
    w, wq_ref, sw_ref = _weights(case.N, case.K, case.seed)
    b = case.b()
    if check_weights:
        Wq, s_w = w8a8.quantize_weights(to_dev(w))
        torch.cuda.synchronize()
        assert np.array_equal(Wq.cpu().numpy(), wq_ref)
        assert np.array_equal(f32_bits(s_w.cpu().numpy()), f32_bits(sw_ref))
    else:
        Wq, s_w = torch.from_numpy(wq_ref).cuda(), torch.from_numpy(sw_ref).cuda()
    y, q, s_a = w8a8.linear_fused(to_dev(x), Wq, s_w, to_dev(b), return_intermediates=True)
    y_plain = w8a8.linear_fused(to_dev(x), Wq, s_w, to_dev(b))   # workspace path
    torch.cuda.synchronize()
    q_ref, s_ref = _quant_check(x, q, s_a)
    rows = sample_rows(case.M, seed=case.seed)
    acc = oracle.gemm_i32(q_ref[rows], wq_ref)
    y32, y_ref = oracle.epilogue(acc, s_ref[rows], sw_ref, b)
    yb = bits_of(y)[rows]
    mism = check_y(yb, y_ref, y32, case.name)
    assert np.array_equal(bits_of(y_plain)[rows], yb)
    return mism


@pytest.mark.parametrize("case", [synth.QKV, synth.FFN_UP, synth.FFN_DOWN, synth.ADALN_M1,
                                  synth.ADALN_M2], ids=lambda c: c.name)
def test_full_size_configs(case):
    assert _run_layer_sampled(case, check_weights=True) == 0


def test_ffn_pair_back_to_back():
    up, down = synth.FFN_UP, synth.FFN_DOWN
    xu, xd = up.x(), down.x()
    _, wqu, swu = _weights(up.N, up.K, up.seed)
    _, wqd, swd = _weights(down.N, down.K, down.seed)
    bu, bd = up.b(), down.b()
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        yu, qu, sau = w8a8.linear_fused(to_dev(xu), torch.from_numpy(wqu).cuda(),
                                        torch.from_numpy(swu).cuda(), to_dev(bu),
                                        return_intermediates=True)
        yd, qd, sad = w8a8.linear_fused(to_dev(xd), torch.from_numpy(wqd).cuda(),
                                        torch.from_numpy(swd).cuda(), to_dev(bd),
                                        return_intermediates=True)
    s.synchronize()
    for x, y, q, sa, wq, sw, b, M in ((xu, yu, qu, sau, wqu, swu, bu, up.M),
                                      (xd, yd, qd, sad, wqd, swd, bd, down.M)):
        q_ref, s_ref = _quant_check(x, q, sa)
        rows = sample_rows(M, seed=3, n_random=32)
        y32, y_ref = oracle.epilogue(oracle.gemm_i32(q_ref[rows], wq), s_ref[rows], sw, b)
        assert check_y(bits_of(y)[rows], y_ref, y32, "ffn pair") == 0


SWEEP = [c for c in synth.sweep_cases() if c.seed == 0 or c.M <= 4352]


@pytest.mark.parametrize("case", SWEEP, ids=lambda c: c.name)
def test_sweep_point(case):
    assert _run_layer_sampled(case) == 0


# ----------------------------------------------------------------- host buffers

@pytest.mark.parametrize("M,N,K", [(64, 128, 256), (300, 520, 3072), (2, 1032, 3072)])
def test_linear_fused_host_buffers(M, N, K):
    x, w, b = synth.make_x(M, K, "studentt", 4), synth.make_w(N, K, 4), synth.make_bias(N, 4)
    wq_ref, sw_ref = oracle.quantize_weights(w)
    ref = oracle.linear(x, wq_ref, sw_ref, b)
    x_host = torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).pin_memory()
    y_host = torch.empty((M, N), dtype=torch.bfloat16).pin_memory()
    x_dev = torch.empty((M, K), dtype=torch.bfloat16, device="cuda")
    y_dev = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    nws = w8a8.workspace_size(M, N, K)
    ws = torch.empty((max(nws, 1),), dtype=torch.uint8, device="cuda")
    w8a8.linear_fused_host(x_host, torch.from_numpy(wq_ref).cuda(),
                           torch.from_numpy(sw_ref).cuda(), to_dev(b), y_host, x_dev, y_dev, ws)
    torch.cuda.current_stream().synchronize()
    assert check_y(bits_of(y_host), ref["y"], ref["y32"], "host buffers") == 0


# ----------------------------------------------------------------- failure detection

def test_bounded_wait_times_out_and_context_survives():
    assert w8a8.last_device_error() == B.W8A8_OK
    assert w8a8.selftest_bounded_wait(20_000_000) == B.W8A8_OK      # 20 ms limit
    assert w8a8.last_device_error() == B.W8A8_ERR_DEVICE_TIMEOUT
    assert w8a8.last_device_error() == B.W8A8_OK                    # cleared on read
    # the context is still usable
    test_tiny_config_bitexact()
    assert w8a8.last_device_error() == B.W8A8_OK


def test_errors_are_returned_not_raised_in_c():
    st = B.w8a8_quant_act(None, 4, 16, 16, None, None, None)
    assert st == B.W8A8_ERR_INVALID_ARG
    x = torch.zeros((4, 24), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(w8a8.W8A8Error) as e:
        w8a8.quant_act(x)
    assert e.value.status == B.W8A8_ERR_UNSUPPORTED_SHAPE
