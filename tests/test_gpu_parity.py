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

from gpu_util import bf16_to_f64, bf16_ulp, bits_of, check_y, f32_bits, sample_rows, to_dev

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
    # more rows than one pass of every warp's slots: the slot rings are refilled
    (20000, 256, "normal"), (9000, 4096, "studentt"), (2000, 12288, "gelu"), (4353, 3072, "studentt"),
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


def test_int8_peak_loop_runs_clean():
    """The tensor-core ceiling measurement: every CTA pair issues MMAs from
    shared memory; the launch must complete with no device error."""
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    for pairs, iters in ((1, 10), (sms // 2, 1000)):
        B.bench_mma_i8_peak(iters, pairs)
    torch.cuda.synchronize()
    assert w8a8.last_device_error() == B.W8A8_OK
    with pytest.raises(w8a8.W8A8Error):
        B.bench_mma_i8_peak(500001, 1)          # beyond the bounded length


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
VARIANTS = [B.VARIANT_GEMM_BN64, B.VARIANT_GEMM_BN128, B.VARIANT_GEMM_BN256, B.VARIANT_GEMM_PAIR]


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

@pytest.mark.parametrize("M", [1, 2, 3, 4, 5, 8, 16])
@pytest.mark.parametrize("N,K", [(128, 256), (1032, 3072), (64, 12288), (18432, 3072), (136, 16),
                                 (520, 2064)])
def test_gemv_fused_and_unfused(M, N, K):
    x, w, b = synth.make_x(M, K, "normal", M), synth.make_w(N, K, M), synth.make_bias(N, M)
    wq_ref, sw_ref = oracle.quantize_weights(w)
    ref = oracle.linear(x, wq_ref, sw_ref, b)
    Wq, s_w = torch.from_numpy(wq_ref).cuda(), torch.from_numpy(sw_ref).cuda()
    # the selector takes the CUDA-core GEMV (quantizing its rows in the same
    # launch at M = 1, 2) unless the tensor-core variant streams a wide or deep
    # weight faster; the CUDA-core GEMV is also checked through its explicit
    # (unfused) variant
    p = w8a8.select(M, N, K)
    wide = ((M >= 5 and (N >= 6144 or K >= 8192)) or
            (M >= 4 and (N >= 12288 or N * K >= 6144 * 12288)) or (M >= 12 and N >= 3072))
    assert p["variant_name"] == ("gemv_tc" if wide else "gemv")
    assert p["quant_in_gemm_launch"] == (0 if wide else int(M == 1 or (M == 2 and K <= 8192)))
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


# (M, N, K): activation rows padded to 16 / 32 / 64 / 128; one tile
# (128 x 256, K shared by up to 8 CTAs), ragged N (1032, K in eight parts), K
# not a multiple of 128 (2064), the AdaLN shape (144 tiles, no split), the QKV
# weight (72 tiles, K in two halves), N = 3072 (24 tiles, K in four parts),
# 16 tiles with K in six parts, 14 tiles with K in seven, and 3 tiles in five.
GEMV_TC_CASES = [(1, 128, 256), (2, 18432, 3072), (5, 1032, 2064), (16, 9216, 3072),
                 (17, 3072, 3072), (31, 3072, 12288), (64, 264, 3072), (100, 9216, 3072),
                 (128, 1032, 12288), (3, 128, 16), (16, 2048, 8192), (8, 1792, 4096)]


@pytest.mark.parametrize("M,N,K", GEMV_TC_CASES)
def test_gemv_tc_int32_exact_and_y(M, N, K):
    """The tensor-core small-M variant (weights on the MMA's 128-row side,
    K split among the CTAs of a cluster, partial sums added in distributed
    shared memory): raw int32 equal to the oracle, y bit-equal."""
    plan = w8a8.select(M, N, K, variant=B.VARIANT_GEMV_TC)
    assert plan["k_split"] >= 1 and plan["grid"] == plan["num_tiles"] * plan["k_split"]
    x, w, b = synth.make_x(M, K, "studentt", M + 3), synth.make_w(N, K, M + 3), synth.make_bias(N, M + 3)
    wq_ref, sw_ref = oracle.quantize_weights(w)
    ref = oracle.linear(x, wq_ref, sw_ref, b)
    args = (torch.from_numpy(ref["q"]).cuda(), torch.from_numpy(ref["s_a"]).cuda(),
            torch.from_numpy(wq_ref).cuda(), torch.from_numpy(sw_ref).cuda())
    acc = w8a8.linear(*args, acc_debug=True, variant=B.VARIANT_GEMV_TC)
    y = w8a8.linear(*args, to_dev(b), variant=B.VARIANT_GEMV_TC)
    y_nobias = w8a8.linear(*args, variant=B.VARIANT_GEMV_TC)
    torch.cuda.synchronize()
    assert np.array_equal(acc.cpu().numpy(), ref["acc"])
    assert check_y(bits_of(y), ref["y"], ref["y32"], "gemv_tc") == 0
    y32n, yn = oracle.epilogue(ref["acc"], ref["s_a"], sw_ref, None)
    assert check_y(bits_of(y_nobias), yn, y32n, "gemv_tc no bias") == 0


@pytest.mark.parametrize("M,N,K", [(6, 136, 40000), (16, 3072, 12288), (11, 9216, 3072)])
def test_small_m_whole_layer_with_intermediates(M, N, K):
    """linear_fused at 5 <= M <= 16 against a deep or wide weight: the
    quantization kernel, then the tensor-core small-M variant reading q (K
    shared among up to 8 CTAs of a cluster): y, q and s_a against the oracle
    in full."""
    x, w, b = synth.make_x(M, K, "studentt", M + 40), synth.make_w(N, K, M + 40), synth.make_bias(N, M + 40)
    wq_ref, sw_ref = oracle.quantize_weights(w)
    ref = oracle.linear(x, wq_ref, sw_ref, b)
    Wq, s_w = torch.from_numpy(wq_ref).cuda(), torch.from_numpy(sw_ref).cuda()
    assert w8a8.select(M, N, K)["variant_name"] == "gemv_tc"
    y, q, s_a = w8a8.linear_fused(to_dev(x), Wq, s_w, to_dev(b), return_intermediates=True)
    y2 = w8a8.linear_fused(to_dev(x), Wq, s_w, None)
    torch.cuda.synchronize()
    assert np.array_equal(q.cpu().numpy(), ref["q"])
    assert np.array_equal(f32_bits(s_a.cpu().numpy()), f32_bits(ref["s_a"]))
    assert check_y(bits_of(y), ref["y"], ref["y32"], "small-M layer") == 0
    y32n, yn = oracle.epilogue(ref["acc"], ref["s_a"], sw_ref, None)
    assert check_y(bits_of(y2), yn, y32n, "small-M layer, no bias") == 0


def test_gemv_tc_extremes_at_max_k():
    K = 133120
    q = np.full((3, K), 127, np.int8)
    q[1] = -127
    q[2, ::2] = -127
    wq = np.full((136, K), 127, np.int8)
    wq[5, ::2] = -127
    acc = w8a8.linear(torch.from_numpy(q).cuda(), torch.ones(3, device="cuda"),
                      torch.from_numpy(wq).cuda(), torch.ones(136, device="cuda"),
                      acc_debug=True, variant=B.VARIANT_GEMV_TC)
    torch.cuda.synchronize()
    ref = oracle.gemm_i32(q, wq)
    assert ref[0, 0] == 127 * 127 * K and ref[1, 0] == -127 * 127 * K
    assert np.array_equal(acc.cpu().numpy(), ref)


def test_gemm_variant_at_tiny_m_matches_gemv():
    M, N, K = 3, 264, 512
    x, w, b = synth.make_x(M, K, "normal", 5), synth.make_w(N, K, 5), synth.make_bias(N, 5)
    wq_ref, sw_ref = oracle.quantize_weights(w)
    ref = oracle.linear(x, wq_ref, sw_ref, b)
    args = (torch.from_numpy(ref["q"]).cuda(), torch.from_numpy(ref["s_a"]).cuda(),
            torch.from_numpy(wq_ref).cuda(), torch.from_numpy(sw_ref).cuda(), to_dev(b))
    for v in (B.VARIANT_GEMV, B.VARIANT_GEMM_BN128, B.VARIANT_GEMM_BN256, B.VARIANT_GEMM_PAIR,
              B.VARIANT_GEMV_TC):
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
                                  synth.ADALN_M2, synth.ADALN_M16], ids=lambda c: c.name)
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


SWEEP = synth.sweep_cases()


@pytest.mark.parametrize("case", SWEEP, ids=lambda c: c.name)
def test_sweep_point(case):
    assert _run_layer_sampled(case) == 0


# ----------------------------------------------------------------- host buffers

# (M, N, K): one chunk; 256 + 44 rows; two rows; six chunks of 384 rows
@pytest.mark.parametrize("M,N,K", [(64, 128, 256), (300, 520, 3072), (2, 1032, 3072),
                                   (2304, 1032, 1024)])
def test_linear_fused_host_buffers(M, N, K):
    """Host buffers in and out, the rows in chunks whose copies and layer
    calls run on three streams: y against the oracle in full.  The staging
    buffers start out holding other values, so a chunk computed before its
    copy in, or copied out before its layer, shows."""
    x, w, b = synth.make_x(M, K, "studentt", 4), synth.make_w(N, K, 4), synth.make_bias(N, 4)
    wq_ref, sw_ref = oracle.quantize_weights(w)
    ref = oracle.linear(x, wq_ref, sw_ref, b)
    x_host = torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).pin_memory()
    y_host = torch.empty((M, N), dtype=torch.bfloat16).pin_memory()
    x_dev = torch.full((M, K), 3.0, dtype=torch.bfloat16, device="cuda")
    y_dev = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
    nws = w8a8.workspace_size(M, N, K)
    ws = torch.empty((max(nws, 1),), dtype=torch.uint8, device="cuda")
    w8a8.linear_fused_host(x_host, torch.from_numpy(wq_ref).cuda(),
                           torch.from_numpy(sw_ref).cuda(), to_dev(b), y_host, x_dev, y_dev, ws)
    torch.cuda.current_stream().synchronize()
    assert check_y(bits_of(y_host), ref["y"], ref["y32"], "host buffers") == 0


def test_linear_fused_host_buffers_in_a_cuda_graph():
    """The chunked host-buffer call captured once (its internal streams fork
    from and join back into the capturing stream) and replayed on new host
    inputs: each replay's y_host matches the oracle for that input."""
    M, N, K = 1100, 264, 512
    w, b = synth.make_w(N, K, 6), synth.make_bias(N, 6)
    wq_ref, sw_ref = oracle.quantize_weights(w)
    Wq, s_w, bd = torch.from_numpy(wq_ref).cuda(), torch.from_numpy(sw_ref).cuda(), to_dev(b)
    x_host = torch.empty((M, K), dtype=torch.bfloat16).pin_memory()
    y_host = torch.empty((M, N), dtype=torch.bfloat16).pin_memory()
    x_dev = torch.zeros((M, K), dtype=torch.bfloat16, device="cuda")
    y_dev = torch.zeros((M, N), dtype=torch.bfloat16, device="cuda")
    ws = torch.empty((w8a8.workspace_size(M, N, K),), dtype=torch.uint8, device="cuda")
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            w8a8.linear_fused_host(x_host, Wq, s_w, bd, y_host, x_dev, y_dev, ws, stream=s)
    torch.cuda.synchronize()
    for seed in (7, 8):
        x = synth.make_x(M, K, "normal", seed)
        x_host.copy_(torch.from_numpy(x.view(np.int16)).view(torch.bfloat16))
        g.replay()
        torch.cuda.synchronize()
        ref = oracle.linear(x, wq_ref, sw_ref, b)
        assert check_y(bits_of(y_host), ref["y"], ref["y32"], f"graph replay {seed}") == 0
    del g


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


# ----------------------------------------------------------------- chained calls

@pytest.mark.parametrize("M,N,K", [(4352, 9216, 3072), (64, 9216, 3072), (3, 18432, 3072),
                                   (16, 18432, 3072)])
def test_layer_right_after_quantize_weights(M, N, K):
    """Weight quantization into a buffer holding other values, then at once
    on the same stream a layer on precomputed q reading that Wq (the pair
    GEMM, the one-CTA GEMM, the GEMV, the tensor-core small-M kernel: each
    prefetches weights before its dependency wait).  The weight kernel must
    release its dependents only when it has completed, so the layer sees the
    finished weights: y must equal the layer run after a full synchronize."""
    dev = torch.device("cuda")
    W = to_dev(synth.make_w(N, K, 11))
    q, s_a = w8a8.quant_act(to_dev(synth.make_x(M, K, "normal", 11)))
    Wq, s_w = torch.empty((N, K), dtype=torch.int8, device=dev), torch.empty(N, device=dev)
    y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
    ws = torch.empty((max(1, w8a8.workspace_size(M, N, K)),), dtype=torch.uint8, device=dev)
    s = B._stream()

    def run():
        assert B.w8a8_quantize_weights(B._ptr(W), N, K, K, B._ptr(Wq), B._ptr(s_w), s) == 0
        assert B.w8a8_linear(B._ptr(q), B._ptr(s_a), M, K, B._ptr(Wq), B._ptr(s_w), None, N,
                             B._ptr(y), N, None, B._ptr(ws), ws.numel(), s) == 0

    run()
    torch.cuda.synchronize()
    ref = y.clone()
    for fill in (7, -100, 0):
        Wq.fill_(fill)
        s_w.fill_(float(fill))
        y.fill_(float("nan"))
        run()
        torch.cuda.synchronize()
        assert torch.equal(y.view(torch.int16), ref.view(torch.int16)), f"fill {fill}"


def test_chained_layers_share_buffers_under_dependent_launch():
    """Consecutive layer calls are launched as programmatic dependents: each
    kernel starts before the previous one finishes and waits for it before
    touching its data.  A chain whose every input is the previous output, with
    one workspace reused by every call and GEMV and GEMM layers interleaved,
    must equal the oracle run step by step."""
    K = 1024
    dims = [(384, K), (2, K), (300, K), (1, K), (384, K)]   # (M, N=K) per step: GEMM/GEMV mix
    rng_seed = 21
    ws = torch.empty((w8a8.workspace_size(384, K, K) + 256,), dtype=torch.uint8, device="cuda")
    x_bits = synth.make_x(384, K, "studentt", rng_seed)
    weights = []
    for i in range(len(dims)):
        w = synth.make_w(K, K, rng_seed + i)
        wq, sw = oracle.quantize_weights(w)
        weights.append((wq, sw, synth.make_bias(K, rng_seed + i)))
    # GPU: one stream, no synchronization between the calls
    cur = to_dev(x_bits)
    outs = []
    for (M, _), (wq, sw, b) in zip(dims, weights):
        y = w8a8.linear_fused(cur[:M], torch.from_numpy(wq).cuda(), torch.from_numpy(sw).cuda(),
                              to_dev(b), workspace=ws)
        outs.append(y)
        nxt = torch.zeros((384, K), dtype=torch.bfloat16, device="cuda")
        nxt[:M] = y
        cur = nxt
    torch.cuda.synchronize()
    # oracle, step by step
    ref_in = x_bits
    for step, ((M, _), (wq, sw, b), y) in enumerate(zip(dims, weights, outs)):
        r = oracle.linear(np.ascontiguousarray(ref_in[:M]), wq, sw, b)
        assert check_y(bits_of(y), r["y"], r["y32"], f"chain step {step}") == 0
        nxt = np.zeros((384, K), np.uint16)
        nxt[:M] = r["y"]
        ref_in = nxt


def test_back_to_back_calls_reuse_one_workspace():
    """Many fused calls on one workspace, no synchronization in between: the
    quantization of call i+1 overwrites q / s_a that the GEMM of call i reads,
    and must wait for it."""
    M, N, K = 640, 1024, 3072
    ws = torch.empty((w8a8.workspace_size(M, N, K),), dtype=torch.uint8, device="cuda")
    w = synth.make_w(N, K, 31)
    wq, sw = oracle.quantize_weights(w)
    b = synth.make_bias(N, 31)
    Wq, s_w, bd = torch.from_numpy(wq).cuda(), torch.from_numpy(sw).cuda(), to_dev(b)
    xs = [synth.make_x(M, K, "studentt", 40 + i) for i in range(4)]
    xs_dev = [to_dev(x) for x in xs]
    outs = [torch.empty((M, N), dtype=torch.bfloat16, device="cuda") for _ in xs]
    torch.cuda.synchronize()
    for xd, o in zip(xs_dev, outs):   # nothing but these calls between the launches
        w8a8.linear_fused(xd, Wq, s_w, bd, out=o, workspace=ws)
    ys = outs
    torch.cuda.synchronize()
    for i, (x, y) in enumerate(zip(xs, ys)):
        rows = sample_rows(M, seed=i, n_random=32)
        r = oracle.linear(np.ascontiguousarray(x[rows]), wq, sw, b)
        assert check_y(bits_of(y)[rows], r["y"], r["y32"], f"call {i}") == 0


# ----------------------------------------------------------------- K-split tail

# (M, N, K): under one wave, every tile shared by four pairs (512 x 1024 x
# 12288), ragged edges in M and N with tiles shared by two or three pairs
# (600 x 2056 x 12288), four full waves of whole tiles and then 112 tiles
# shared out at 146 k-blocks per pair (8704 x 3072 x 12288).
SPLIT_CASES = [(512, 1024, 12288), (600, 2056, 12288), (8704, 3072, 12288)]


@pytest.mark.parametrize("M,N,K", SPLIT_CASES)
def test_pair_k_split_matches_unsplit_and_oracle(M, N, K):
    """The pair kernel with its last tiles shared out along K (partial int32
    sums, last-arriver reduction) against the same kernel unsplit -- raw
    accumulators and y, in full -- and against the oracle on sampled rows."""
    plan = w8a8.select(M, N, K, variant=B.VARIANT_GEMM_PAIR)
    assert plan["split_tiles"] > 0
    # the binding sizes the workspace for the forced plan, K-split region included
    assert w8a8.workspace_size(M, N, K, B.VARIANT_GEMM_PAIR) >= M * K + 4 * M + 16 * 4096 * 4 * (
        plan["split_tiles"] + plan["grid"] // 2 - 1)
    rng = np.random.default_rng(M + N + K)
    q = rng.integers(-127, 128, size=(M, K), dtype=np.int8)
    wq = rng.integers(-127, 128, size=(N, K), dtype=np.int8)
    s_a = (rng.random(M, dtype=np.float32) * 0.05 + 1e-3).astype(np.float32)
    s_w = (rng.random(N, dtype=np.float32) * 0.002 + 1e-4).astype(np.float32)
    b = synth.make_bias(N, seed=5)
    args = (torch.from_numpy(q).cuda(), torch.from_numpy(s_a).cuda(), torch.from_numpy(wq).cuda(),
            torch.from_numpy(s_w).cuda(), to_dev(b))
    acc_split = w8a8.linear(*args, acc_debug=True, variant=B.VARIANT_GEMM_PAIR)
    acc_plain = w8a8.linear(*args, acc_debug=True, variant=B.VARIANT_GEMM_PAIR, split=False)
    y_split = w8a8.linear(*args, variant=B.VARIANT_GEMM_PAIR)
    y_plain = w8a8.linear(*args, variant=B.VARIANT_GEMM_PAIR, split=False)
    torch.cuda.synchronize()
    assert torch.equal(acc_split, acc_plain)
    assert torch.equal(y_split, y_plain)
    rows = sample_rows(M, seed=7, n_random=24, tile=256)
    ref = oracle.gemm_i32(q[rows], wq)
    assert np.array_equal(acc_split.cpu().numpy()[rows], ref)
    y32, y_ref = oracle.epilogue(ref, s_a[rows], s_w, b)
    assert check_y(bits_of(y_split)[rows], y_ref, y32, "k-split") == 0


def test_pair_k_split_repeated_calls_on_one_workspace():
    """Back-to-back split launches on one workspace: each call's counters are
    cleared before its GEMM and no call reads another's partial sums."""
    M, N, K = 512, 1024, 12288
    assert w8a8.select(M, N, K, variant=B.VARIANT_GEMM_PAIR)["split_tiles"] > 0
    rng = np.random.default_rng(99)
    wq = rng.integers(-127, 128, size=(N, K), dtype=np.int8)
    Wq = torch.from_numpy(wq).cuda()
    ones_n = torch.ones(N, device="cuda")
    ws = torch.empty((w8a8.workspace_size(M, N, K, B.VARIANT_GEMM_PAIR),), dtype=torch.uint8,
                     device="cuda")
    qs = [rng.integers(-127, 128, size=(M, K), dtype=np.int8) for _ in range(3)]
    accs = [w8a8.linear(torch.from_numpy(q).cuda(), torch.ones(M, device="cuda"), Wq, ones_n,
                        acc_debug=True, variant=B.VARIANT_GEMM_PAIR, workspace=ws) for q in qs]
    torch.cuda.synchronize()
    for i, (q, acc) in enumerate(zip(qs, accs)):
        rows = sample_rows(M, seed=i, n_random=16, tile=256)
        assert np.array_equal(acc.cpu().numpy()[rows], oracle.gemm_i32(q[rows], wq)), i


def test_pair_k_split_ignores_counter_words_planted_with_the_live_tag():
    """A workspace whose every 64-bit word reads as a counter of the very
    launch about to run, with all but one contribution already arrived
    ((tag << 8) | 3 for tiles shared by four pairs): without the clearing
    before the launch, the first contribution to arrive would finish its tile
    from partial sums nobody wrote.  The result must still equal the unsplit
    kernel and the oracle."""
    M, N, K = 512, 1024, 12288
    assert w8a8.select(M, N, K, variant=B.VARIANT_GEMM_PAIR)["split_tiles"] > 0
    rng = np.random.default_rng(123)
    q = rng.integers(-127, 128, size=(M, K), dtype=np.int8)
    wq = rng.integers(-127, 128, size=(N, K), dtype=np.int8)
    args = (torch.from_numpy(q).cuda(), torch.ones(M, device="cuda"), torch.from_numpy(wq).cuda(),
            torch.ones(N, device="cuda"))
    ref_plain = w8a8.linear(*args, acc_debug=True, variant=B.VARIANT_GEMM_PAIR, split=False)
    ws = torch.empty((w8a8.workspace_size(M, N, K, B.VARIANT_GEMM_PAIR),), dtype=torch.uint8,
                     device="cuda")
    for _ in range(2):
        torch.cuda.synchronize()
        word = np.array([(B.debug_peek_tag() << 8) | 3], dtype=np.uint64).view(np.int64)[0]
        ws.view(torch.int64).fill_(int(word))
        acc = w8a8.linear(*args, acc_debug=True, variant=B.VARIANT_GEMM_PAIR, workspace=ws)
        torch.cuda.synchronize()
        assert torch.equal(acc, ref_plain)
    rows = sample_rows(M, seed=5, n_random=16, tile=256)
    assert np.array_equal(acc.cpu().numpy()[rows], oracle.gemm_i32(q[rows], wq))


# ----------------------------------------------------------------- packed weights

@pytest.mark.parametrize("N,K", [(8, 16), (264, 3072), (18432, 3072), (3072, 12288)])
def test_unpack_int32_weights_bitexact(N, K):
    """Packed int32 storage (written by the oracle's packer) -> int8 codes on
    the GPU, byte-equal to the oracle's unpacking; every code including -128."""
    rng = np.random.default_rng(N + K)
    wq = rng.integers(-128, 128, size=(N, K), dtype=np.int8)
    wq[0, :min(K, 256)] = np.arange(-128, 128, dtype=np.int16).astype(np.int8)[:min(K, 256)]
    packed = oracle.pack_int32(wq)
    got = w8a8.unpack_int32_weights(torch.from_numpy(packed).cuda())
    torch.cuda.synchronize()
    assert np.array_equal(got.cpu().numpy(), oracle.unpack_int32(packed, K))


def test_unpacked_weights_drive_the_layer():
    """A layer whose weights come from packed storage equals the layer with
    the oracle's codes (the scales are stored beside the codes)."""
    M, N, K = 300, 520, 3072
    x, w, b = synth.make_x(M, K, "studentt", 8), synth.make_w(N, K, 8), synth.make_bias(N, 8)
    wq, sw = oracle.quantize_weights(w)
    Wq = w8a8.unpack_int32_weights(torch.from_numpy(oracle.pack_int32(wq)).cuda())
    y = w8a8.linear_fused(to_dev(x), Wq, torch.from_numpy(sw).cuda(), to_dev(b))
    torch.cuda.synchronize()
    r = oracle.linear(x, wq, sw, b)
    assert check_y(bits_of(y), r["y"], r["y32"], "packed weights") == 0


# ----------------------------------------------------------------- DiT block

def test_dit_block_linears_back_to_back():
    """One DiT block's linear set at CFG batch 2 (fused q|k|v, to_out, fused
    proj|gate, FFN out, AdaLN GEMV), launched back to back on one stream with
    one shared workspace; every output against the oracle on sampled rows."""
    cases = synth.DIT_BLOCK
    ws = torch.empty((max(w8a8.workspace_size(c.M, c.N, c.K) for c in cases),),
                     dtype=torch.uint8, device="cuda")
    host, outs = [], []
    for c in cases:
        x, b = c.x(), c.b()
        wq, sw = oracle.quantize_weights(c.w())
        host.append((x, wq, sw, b))
        outs.append((to_dev(x), torch.from_numpy(wq).cuda(), torch.from_numpy(sw).cuda(),
                     to_dev(b)))
    torch.cuda.synchronize()
    ys = [w8a8.linear_fused(xd, Wq, s_w, bd, workspace=ws) for xd, Wq, s_w, bd in outs]
    torch.cuda.synchronize()
    for c, (x, wq, sw, b), y in zip(cases, host, ys):
        rows = sample_rows(c.M, seed=c.seed, n_random=32, tile=256)
        r = oracle.linear(np.ascontiguousarray(x[rows]), wq, sw, b)
        assert check_y(bits_of(y)[rows], r["y"], r["y32"], c.name) == 0


# ----------------------------------------------------------------- N-split tail

# (M, N, K): 76 tiles = one round + 2, ragged M and a ragged last column
# block (500 x 9720); 94 tiles = one round + 20 (512 x 12032).
NSPLIT_CASES = [(500, 9720, 512, 2), (512, 12032, 512, 2)]


@pytest.mark.parametrize("M,N,K,nsplit", NSPLIT_CASES)
def test_pair_n_split_tail_exact(M, N, K, nsplit):
    """The pair kernel with the tiles of its last round cut along N into
    narrower tiles: raw int32 accumulators and y against the oracle, in full."""
    assert w8a8.select(M, N, K, variant=B.VARIANT_GEMM_PAIR)["tail_tiles_nsplit"] == nsplit
    rng = np.random.default_rng(M * 3 + N + K)
    q = rng.integers(-127, 128, size=(M, K), dtype=np.int8)
    wq = rng.integers(-127, 128, size=(N, K), dtype=np.int8)
    s_a = (rng.random(M, dtype=np.float32) * 0.05 + 1e-3).astype(np.float32)
    s_w = (rng.random(N, dtype=np.float32) * 0.002 + 1e-4).astype(np.float32)
    b = synth.make_bias(N, seed=6)
    args = (torch.from_numpy(q).cuda(), torch.from_numpy(s_a).cuda(), torch.from_numpy(wq).cuda(),
            torch.from_numpy(s_w).cuda(), to_dev(b))
    acc = w8a8.linear(*args, acc_debug=True, variant=B.VARIANT_GEMM_PAIR)
    y = w8a8.linear(*args, variant=B.VARIANT_GEMM_PAIR)
    torch.cuda.synchronize()
    ref = oracle.gemm_i32(q, wq)
    assert np.array_equal(acc.cpu().numpy(), ref)
    y32, y_ref = oracle.epilogue(ref, s_a, s_w, b)
    assert check_y(bits_of(y), y_ref, y32, "n-split") == 0


# ----------------------------------------------------------------- quantization fused into the GEMM launch

def _fused_call(x, Wq, s_w, b, y, ws, ws_bytes, q_out=None, s_a_out=None, options=0):
    st = B.w8a8_linear_fused_ex(B._ptr(x), x.shape[0], x.shape[1], x.stride(0), B._ptr(Wq),
                                B._ptr(s_w), B._ptr(b), Wq.shape[0], B._ptr(y), y.stride(0),
                                B._ptr(q_out), B._ptr(s_a_out), B._ptr(ws), ws_bytes, options,
                                B._stream())
    assert st == 0, B.status_string(st)


# (M, N, K, ldx): the QKV shape, a ragged M (last row block of 67 rows, last
# pass of 3 rows per CTA group) with K = 3072, a short K (single-vector lanes),
# a strided x (ldx > K), the FFN down-projection (K = 12288: one bulk-path
# row per warp, longer register-path rows read twice), eight passes of rows
# (8704 x 3072 x 3072, the first round's rows through the ring, the rest
# interleaved with epilogues), a ragged 12288-wide K with two bulk rows per
# warp, and K = 6144 (two rows in flight per warp's share of the ring).
FUSED_CASES = [(4352, 9216, 3072, 3072), (1091, 6144, 3072, 3072), (1537, 4096, 3072, 3200),
               (2048, 4096, 512, 512), (4352, 3072, 12288, 12288), (8704, 3072, 3072, 3072),
               (2600, 2048, 12288, 12296), (3000, 4096, 6144, 6144)]


@pytest.mark.parametrize("M,N,K,ldx", FUSED_CASES)
def test_quantization_fused_into_pair_launch(M, N, K, ldx):
    """With the one-launch option and room for the row-block counters, the
    pair plan quantizes x inside the GEMM launch; the result must be bit-equal
    to the two-launch path and q, s_a must equal the oracle's; y against the
    oracle on sampled rows."""
    plan = w8a8.select(M, N, K)
    assert plan["variant_name"] == "gemm_pair" and plan["quant_in_gemm_launch"] == 1
    xb = synth.make_x(M, K, "gelu" if K > 3072 else "studentt", 17)
    x_full = np.zeros((M, ldx), np.uint16)
    x_full[:, :K] = xb
    x = to_dev(x_full)[:, :K]
    w = synth.make_w(N, K, 17)
    wq, sw = oracle.quantize_weights(w)
    b = synth.make_bias(N, 17)
    Wq, s_w, bd = torch.from_numpy(wq).cuda(), torch.from_numpy(sw).cuda(), to_dev(b)
    need = w8a8.workspace_size(M, N, K)
    ws = torch.empty((need,), dtype=torch.uint8, device="cuda")
    q_head = ((M * K + 255) // 256) * 256 + ((4 * M + 255) // 256) * 256   # q and s_a only
    y1 = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    y2 = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    y3 = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    q = torch.empty((M, K), dtype=torch.int8, device="cuda")
    s_a = torch.empty((M,), dtype=torch.float32, device="cuda")
    one = B.FUSED_ONE_LAUNCH
    _fused_call(x, Wq, s_w, bd, y1, ws, need, options=one)       # one launch
    _fused_call(x, Wq, s_w, bd, y2, ws, q_head, options=one)     # no counters: two launches
    _fused_call(x, Wq, s_w, bd, y3, ws, need, q_out=q, s_a_out=s_a, options=one)
    torch.cuda.synchronize()
    assert torch.equal(y1.view(torch.int16), y2.view(torch.int16))
    assert torch.equal(y1.view(torch.int16), y3.view(torch.int16))
    q_ref, s_ref = _quant_check(xb, q, s_a)
    rows = sample_rows(M, seed=17, n_random=32)
    y32, y_ref = oracle.epilogue(oracle.gemm_i32(q_ref[rows], wq), s_ref[rows], sw, b)
    assert check_y(bits_of(y1)[rows], y_ref, y32, "fused launch") == 0


def test_quantization_fused_into_pair_launch_replayed_in_a_cuda_graph():
    """The one-launch layer captured in a CUDA graph (its row-block counters
    are cleared by a memset node of the same graph) and replayed on new
    activations each time: every replay must equal the oracle."""
    M, N, K = 2304, 4096, 3072
    plan = w8a8.select(M, N, K)
    assert plan["variant_name"] == "gemm_pair" and plan["quant_in_gemm_launch"] == 1
    w = synth.make_w(N, K, 23)
    wq, sw = oracle.quantize_weights(w)
    b = synth.make_bias(N, 23)
    Wq, s_w, bd = torch.from_numpy(wq).cuda(), torch.from_numpy(sw).cuda(), to_dev(b)
    need = w8a8.workspace_size(M, N, K)
    ws = torch.empty((need,), dtype=torch.uint8, device="cuda")
    x = torch.empty((M, K), dtype=torch.bfloat16, device="cuda")
    y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            st = B.w8a8_linear_fused_ex(B._ptr(x), M, K, K, B._ptr(Wq), B._ptr(s_w), B._ptr(bd), N,
                                        B._ptr(y), N, None, None, B._ptr(ws), need,
                                        B.FUSED_ONE_LAUNCH, B._stream(s))
            assert st == 0, B.status_string(st)
    torch.cuda.current_stream().wait_stream(s)
    for seed in (31, 32, 33):
        xb = synth.make_x(M, K, "studentt", seed)
        x.copy_(to_dev(xb))
        g.replay()
        torch.cuda.synchronize()
        rows = sample_rows(M, seed=seed, n_random=24)
        r = oracle.linear(np.ascontiguousarray(xb[rows]), wq, sw, b)
        assert check_y(bits_of(y)[rows], r["y"], r["y32"], f"graph replay {seed}") == 0
    del g


# ----------------------------------------------------------------- W8A16 (weight-only)

# ragged N (520, 1032, 264, 4104, 9000), ragged M and K tails (400, 2064 by
# 16 below a k-block), one tile to many rounds of tiles
W8A16_CASES = [(64, 128, 256, True), (300, 520, 400, True), (129, 1032, 3072, False),
               (17, 264, 12288, True), (4352, 9216, 3072, True), (1000, 4104, 1024, True),
               (2000, 9000, 400, False)]


@pytest.mark.parametrize("M,N,K,bias", W8A16_CASES)
def test_w8a16_vs_oracle(M, N, K, bias):
    """y = bf16((x @ Wq^T) * s_w + bias) with fp32 tensor-core accumulation in
    an unspecified order: each output must lie within one bf16 ulp of the
    oracle's fp32 value plus the bound on any fp32 summation order,
    |s_w| * gamma_K * sum_k |x q| (gamma_K = K u / (1 - K u), u = 2^-24), plus
    the two fp32 roundings of the epilogue."""
    x = synth.make_x(M, K, "studentt", 21)
    w = synth.make_w(N, K, 21)
    wq, sw = oracle.quantize_weights(w)
    b = synth.make_bias(N, 21) if bias else None
    y = w8a8.w8a16_linear(to_dev(x), torch.from_numpy(wq).cuda(), torch.from_numpy(sw).cuda(),
                          to_dev(b) if b is not None else None)
    torch.cuda.synchronize()
    rows = np.arange(M) if M <= 512 else sample_rows(M, seed=21, n_random=32)
    r = oracle.w8a16_linear(np.ascontiguousarray(x[rows]), wq, sw, b)
    got = bf16_to_f64(bits_of(y)[rows])
    ref = r["y32"].astype(np.float64)
    u = 2.0 ** -24
    gamma = K * u / (1 - K * u)
    tol = (bf16_ulp(ref) + np.abs(sw.astype(np.float64))[None, :] * gamma * r["abs_sum"]
           + 4 * u * np.abs(ref) + 1e-30)
    assert np.isfinite(got).all()
    bad = np.abs(got - ref) > tol
    assert not bad.any(), f"{int(bad.sum())} outputs outside the bound, first {np.argwhere(bad)[:3].tolist()}"
    # most outputs round to the oracle's bf16 value exactly
    assert np.mean(bits_of(y)[rows] == r["y"]) > 0.9
