"""Host-side tests of libw8a8.so that need no GPU: exported symbols, status
codes, argument checking (which happens before any CUDA call) and the
selector's decisions."""
from __future__ import annotations

import ctypes
import os
import subprocess

import pytest

import w8a8_int8_dynamic_token_b200 as w8a8
from w8a8_int8_dynamic_token_b200 import binding as B

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


@pytest.fixture(scope="module", autouse=True)
def built():
    from w8a8_int8_dynamic_token_b200 import build
    build.build()
    yield


def test_library_exports_every_header_symbol():
    names = B.header_functions()
    assert len(names) >= 10
    lib = ctypes.CDLL(B.LIB_PATH)
    for n in names:
        assert hasattr(lib, n), n
    out = subprocess.run(["nm", "-D", "--defined-only", B.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if " T " in line}
    assert set(names) <= exported
    # only the declared API is exported
    assert {e for e in exported if e.startswith(("w8a8_", "w8a16_"))} == set(names)


def test_binding_covers_every_header_symbol():
    assert set(B.header_functions()) == set(B._SIGNATURES)


def test_status_strings():
    for st in range(8):
        assert w8a8.status_string(st) not in ("", "unknown status")
    assert w8a8.status_string(99) == "unknown status"
    assert "sm_100a" in w8a8.version()


P = ctypes.c_void_p(256)  # never dereferenced: argument errors come first


@pytest.mark.parametrize("M,K,ld,expect", [
    (0, 16, 16, B.W8A8_ERR_INVALID_ARG),
    (4, 0, 16, B.W8A8_ERR_INVALID_ARG),
    (4, 32, 16, B.W8A8_ERR_INVALID_ARG),          # ld < K
    (4, 24, 24, B.W8A8_ERR_UNSUPPORTED_SHAPE),    # K % 16
    (4, 16, 20, B.W8A8_ERR_UNSUPPORTED_SHAPE),    # ld % 8
    (4, 133152, 133152, B.W8A8_ERR_UNSUPPORTED_SHAPE),  # K > 133144
])
def test_quant_act_argument_errors(M, K, ld, expect):
    assert B.w8a8_quant_act(P, M, K, ld, P, P, None) == expect
    assert B.w8a8_quantize_weights(P, M, K, ld, P, P, None) == expect


def test_null_and_misaligned_pointers():
    assert B.w8a8_quant_act(None, 4, 16, 16, P, P, None) == B.W8A8_ERR_INVALID_ARG
    bad = ctypes.c_void_p(258)
    assert B.w8a8_quant_act(bad, 4, 16, 16, P, P, None) == B.W8A8_ERR_MISALIGNED
    assert B.w8a8_linear(P, P, 4, 16, P, P, None, 8, bad, 8, None, None, 0, None) == \
        B.W8A8_ERR_MISALIGNED
    assert B.w8a8_linear(P, P, 4, 16, P, P, None, 12, P, 12, None, None, 0, None) == \
        B.W8A8_ERR_UNSUPPORTED_SHAPE   # N % 8
    assert B.w8a8_linear_ex(P, P, 4, 16, P, P, None, 8, P, 8, None, 9, None, 0, None) == \
        B.W8A8_ERR_INVALID_ARG         # unknown variant


def test_valid_arguments_reach_the_device_query():
    # With valid arguments the call proceeds to the CUDA device query; without
    # a GPU that reports a CUDA error (on a B200 it would launch).
    st = B.w8a8_quant_act(P, 4, 16, 16, P, P, None)
    try:
        import torch
        has_gpu = torch.cuda.is_available()
    except Exception:
        has_gpu = False
    if not has_gpu:
        assert st == B.W8A8_ERR_CUDA


def _golden(name):
    out = {}
    for line in open(os.path.join(GOLDEN, name)):
        line = line.split("#", 1)[0].split()
        if line:
            out[line[0]] = int(line[1])
    return out


def test_selector_small_m_goes_to_gemv():
    # The AdaLN modulation layer runs at M = batch (1, or 2 with CFG), below
    # the 16 rows a torch._int_mm path cannot serve: every such M is served
    # here, by the GEMV (quantizing its rows in the same launch at M = 1, 2),
    # from 4 rows to 24 on this 18432-wide weight by the tensor-core small-M
    # variant (measured crossovers), and by the tcgen05 GEMM above.
    g = _golden("int_mm_min_rows.txt")
    lim, K, N = g["int_mm_min_rows_exclusive"], g["adaln_in_features"], g["adaln_out_features"]
    for M in (1, 2, 3):
        p = w8a8.select(M, N, K)
        assert p["variant_name"] == "gemv" and p["quant_in_gemm_launch"] == int(M <= 2)
    for M in (4, 5, lim, lim + 1, 20, 24):
        assert w8a8.select(M, N, K)["variant_name"] == "gemv_tc"
    assert w8a8.select(25, N, K)["variant_name"].startswith("gemm")
    assert w8a8.select(lim, N, K, variant=B.VARIANT_GEMV)["variant_name"] == "gemv"
    assert w8a8.workspace_size(1, N, K) == 0
    assert w8a8.workspace_size(3, N, K) >= 3 * K + 3 * 4   # q and s_a for the quantization kernel


def test_selector_narrow_weights_keep_the_gemv_to_11_rows():
    # 3072 x 3072: the GEMV's dot products stay cheaper than the tensor-core
    # variant up to 11 rows (8 rows: 7.4 vs 8.8 us; 12 rows: 10.0 vs 9.3);
    # 3072 x 12288: the tensor-core variant from 5 rows (4 rows: 14.8 vs 15.2;
    # 5 rows: 16.1 vs 13.9)
    for M in (3, 8, 11):
        p = w8a8.select(M, 3072, 3072)
        assert p["variant_name"] == "gemv" and p["quant_in_gemm_launch"] == 0
    for M in (12, 16):
        assert w8a8.select(M, 3072, 3072)["variant_name"] == "gemv_tc"
    assert w8a8.select(2, 3072, 12288)["quant_in_gemm_launch"] == 0   # K > 8192: two launches
    assert w8a8.select(4, 3072, 12288)["variant_name"] == "gemv"
    assert w8a8.select(5, 3072, 12288)["variant_name"] == "gemv_tc"
    assert w8a8.select(11, 1024, 3072)["variant_name"] == "gemv"


def test_selector_one_row_block_narrow_n_takes_64_column_tiles():
    assert w8a8.select(17, 3072, 3072)["variant_name"] == "gemm_bn64"
    assert w8a8.select(64, 9216, 3072)["variant_name"] == "gemm_bn128"   # 72 tiles already
    p = w8a8.select(100, 3072, 12288)
    assert p["variant_name"] == "gemm_bn64" and p["tile_n"] == 64 and p["num_tiles"] == 48


def test_selector_gemm_plans():
    p = w8a8.select(4352, 9216, 3072)
    assert p["variant_name"] == "gemm_pair" and p["num_tiles"] == 17 * 36 and p["grid"] == 148
    p = w8a8.select(4352, 9216, 3072, variant=B.VARIANT_GEMM_BN256)
    assert p["num_tiles"] == 34 * 36 and p["grid"] == 148
    p = w8a8.select(4352, 3072, 12288)
    assert p["num_tiles"] == 17 * 12 and p["grid"] == 148
    # tiny output: few tiles, grid = tiles
    p = w8a8.select(64, 128, 256)
    assert p["grid"] == p["num_tiles"] <= 2
    # too deep for the GEMV's shared-memory rows: the tensor-core small-M
    # variant to 48 rows, the GEMM above
    assert w8a8.select(16, 64, 16384)["variant_name"] == "gemv_tc"
    assert w8a8.select(48, 64, 16384)["variant_name"] == "gemv_tc"
    assert w8a8.select(49, 64, 16384)["variant_name"].startswith("gemm")
    assert w8a8.select(33, 64, 8192)["variant_name"].startswith("gemm")
    # forced variants
    assert w8a8.select(1, 64, 256, variant=B.VARIANT_GEMM_BN128)["tile_n"] == 128
    with pytest.raises(w8a8.W8A8Error):
        w8a8.select(17, 64, 256, variant=B.VARIANT_GEMV)


def test_workspace_size_covers_q_and_scales():
    M, N, K = 4352, 9216, 3072
    n = w8a8.workspace_size(M, N, K)
    assert n >= M * K + 4 * M and n % 256 == 0


# The pair kernel's schedule: whole tiles in full waves, then the last one to
# two waves' tiles shared out along K in equal runs of k-blocks per pair.  A
# model of the device-side partition (work items, contributor counts, partial
# slots) checks that every (tile, k-block) is computed exactly once and that
# the partial-sum slots of different contributions never collide.
def _pair_items(tiles, split_tiles, per, kb, pairs, pair, nsplit=0):
    if nsplit > 1:   # whole tiles in full rounds, then one narrow tail tile per pair
        tile0 = tiles - tiles % pairs
        items = [(t, 0, kb, 1, 0, 0, 256) for t in range(pair, tile0, pairs)]
        if pair < (tiles - tile0) * nsplit:
            w = 256 // nsplit
            items.append((tile0 + pair // nsplit, 0, kb, 1, 0, (pair % nsplit) * w, w))
        return items
    tile0 = tiles - split_tiles
    items = [(t, 0, kb, 1, 0, 0, 256) for t in range(pair, tile0, pairs)]
    if split_tiles:
        units = split_tiles * kb
        u0, u1 = pair * per, min(pair * per + per, units)
        t = u0 // kb if u0 < u1 else None
        while t is not None and t * kb < u1:
            first, last = (t * kb) // per, ((t + 1) * kb - 1) // per
            items.append((tile0 + t, max(u0 - t * kb, 0), min(u1 - t * kb, kb),
                          last - first + 1, pair - first, 0, 256))
            t += 1
    return items


SPLIT_SHAPES = [(4352, 9216, 3072), (4352, 12288, 3072), (4352, 3072, 12288), (512, 1024, 12288),
                (640, 768, 1024), (200, 136, 12288), (1280, 4096, 1024), (2560, 8192, 512),
                (8704, 9216, 3072), (16384, 3072, 12288), (512, 9472, 3072), (8704, 3072, 12288),
                (600, 2056, 12288), (768, 1024, 133120), (2, 8, 133120)]


@pytest.mark.parametrize("M,N,K", SPLIT_SHAPES)
def test_pair_k_split_partition(M, N, K):
    p = w8a8.select(M, N, K, variant=B.VARIANT_GEMM_PAIR)
    tiles, pairs, kb = p["num_tiles"], p["grid"] // 2, -(-K // 128)
    st, per = p["split_tiles"], p["split_kblocks_per_pair"]
    if tiles % 74 == 0:
        assert st == 0
    if st:
        assert per >= 24 and per * pairs >= st * kb
        assert st <= tiles and (tiles - st) % pairs == 0 and st < 2 * pairs
    ns = p["tail_tiles_nsplit"]
    assert not (ns and st)
    covered = {}
    slots = set()
    for pair in range(pairs):
        for t, b, e, nparts, part, n0, w in _pair_items(tiles, st, per, kb, pairs, pair, ns):
            assert 0 <= b < e <= kb and 0 <= part < nparts
            for k in range(b, e):
                for c in range(n0 // 64, (n0 + w) // 64):   # 64-column granules
                    assert (t, k, c) not in covered
                    covered[(t, k, c)] = pair
                covered.setdefault((t, k), pair)
            if nparts > 1:
                slot = (t - (tiles - st)) + pair
                assert slot not in slots and slot < st + pairs - 1
                slots.add(slot)
    assert sum(1 for key in covered if len(key) == 3) == tiles * kb * 4
    # contributor counts agree with who actually covers each tile
    for t in range(tiles - st, tiles):
        owners = sorted({covered[(t, k)] for k in range(kb)})
        assert owners == list(range(owners[0], owners[-1] + 1))


def test_pair_n_split_tail_plans():
    # QKV: 612 tiles = 8 rounds of 74 + 20; the 20 are cut in halves (40 <= 74)
    p = w8a8.select(4352, 9216, 3072)
    assert p["tail_tiles_nsplit"] == 2 and p["split_tiles"] == 0 and p["waves_x100"] == 850
    # FFN up: 816 = 11 x 74 + 2 -> halves
    p = w8a8.select(4352, 12288, 3072)
    assert p["tail_tiles_nsplit"] == 2 and p["waves_x100"] == 1150
    # a last round more than half full cannot be shortened by cutting along N
    assert w8a8.select(4352, 3072, 12288)["tail_tiles_nsplit"] == 0    # 204 = 2 x 74 + 56
    assert w8a8.select(8704, 3072, 12288)["tail_tiles_nsplit"] == 0    # 408 = 5 x 74 + 38
    # under one round there is no tail to cut
    assert w8a8.select(512, 9216, 3072, variant=B.VARIANT_GEMM_PAIR)["tail_tiles_nsplit"] == 0


def test_pair_k_split_plans():
    # 408 tiles of 96 k-blocks: 4 full waves whole, 112 tiles shared out at
    # 146 k-blocks per pair instead of a 6th wave of 96 (saves 46 >= 24)
    p = w8a8.select(8704, 3072, 12288)
    assert p["variant_name"] == "gemm_pair"
    assert p["split_tiles"] == 408 - 4 * 74 and p["split_kblocks_per_pair"] == -(-112 * 96 // 74)
    assert p["waves_x100"] == 400 + -(-100 * 146 // 96)
    # short tiles: shared-out pieces would be epilogue-bound -> no K split
    for M, N, K in ((4352, 9216, 3072), (4352, 12288, 3072), (8704, 3072, 3072)):
        assert w8a8.select(M, N, K)["split_tiles"] == 0
    # a tail that is already three quarters full: the split saves too little
    assert w8a8.select(4352, 3072, 12288)["split_tiles"] == 0
    # under one wave with long K: shared out entirely in pieces of >= 24 k-blocks
    p = w8a8.select(512, 1024, 12288, variant=B.VARIANT_GEMM_PAIR)
    assert p["split_tiles"] == 8 and p["split_kblocks_per_pair"] == 24
    p = w8a8.select(512, 9472, 3072, variant=B.VARIANT_GEMM_PAIR)   # exactly one wave
    assert p["split_tiles"] == 0 and p["num_tiles"] == 74
    # the workspace covers the K-split region: counters + (split + pairs - 1) slots of 256 KiB
    n = w8a8.workspace_size(8704, 3072, 12288)
    assert n >= 8704 * 12288 + 4 * 8704 + (112 + 73) * 256 * 1024
    # a forced pair plan gets its own K-split region even where the automatic
    # plan (one round of 128 x 128 tiles here) has none
    auto = w8a8.workspace_size(512, 1024, 12288)
    assert w8a8.workspace_size(512, 1024, 12288, B.VARIANT_GEMM_PAIR) >= auto + (8 + 73) * 256 * 1024
    assert w8a8.workspace_size(512, 1024, 12288, B.VARIANT_AUTO) == auto
    assert w8a8.workspace_size(512, 1024, 12288, B.VARIANT_GEMM_BN256) == auto
    with pytest.raises(w8a8.W8A8Error):
        w8a8.workspace_size(17, 64, 256, B.VARIANT_GEMV_TC + 1)


def test_small_m_split_keeps_every_cluster_resident():
    # clusters of s CTAs a 148-SM B200 holds at once (one CTA per SM), from
    # the device's occupancy query for this kernel
    held = {1: 148, 2: 74, 3: 45, 4: 33, 5: 26, 6: 22, 7: 15, 8: 15}
    for N in range(128, 18433, 128):
        for K in (256, 3072, 8192, 12288):
            p = w8a8.select(16, N, K, variant=B.VARIANT_GEMV_TC)
            tiles, s = p["num_tiles"], p["k_split"]
            assert tiles <= held[s] or s == 1, (N, K, s)
            assert tiles * s <= 148 or s == 1
    # measured best split per tile count (M = 16): 24 tiles of 3072 x 12288 in
    # fours (12.9 us; clusters of 6, of which only 22 fit: 20.1 us), 48 tiles
    # in twos (9.2 us; threes: 13.7), 16 tiles in sixes, 8 in eights
    for N, want in ((3072, 4), (6144, 2), (2048, 6), (1024, 8), (9216, 2), (18432, 1)):
        assert w8a8.select(16, N, 12288, variant=B.VARIANT_GEMV_TC)["k_split"] == want, N


def test_selector_tile_width_and_pairs_follow_the_measured_rounds():
    # 128-wide tiles only where they fill the rounds 1.4x better than 256-wide
    # ones: 768 x 9216 x 3072 takes 3 rounds of 128-wide tiles, 2 of 256-wide
    # ones or 1.5 of pairs (measured 29.5 / 25.3 / 24.1 us)
    assert w8a8.select(768, 9216, 3072)["variant_name"] == "gemm_pair"
    assert w8a8.select(384, 9216, 3072)["variant_name"] == "gemm_bn256"
    assert w8a8.select(256, 9216, 3072)["variant_name"] == "gemm_bn128"   # one round either way
    assert w8a8.select(768, 3072, 3072)["variant_name"] == "gemm_bn128"
    # pairs from 256 rows when they fill the rounds as well (300 x 18432: 144
    # pair tiles, 26.4 us against 26.6 for 256-wide tiles, 29.4 for 128-wide)
    assert w8a8.select(300, 18432, 3072)["variant_name"] == "gemm_pair"
    # under one round of pair tiles that one round of single-CTA tiles holds:
    # the single-CTA tiles at K = 3072 (512 x 9216: 18.0 vs 18.9 us) and where
    # the pair plan would share K out (1024 x 3072 x 12288: 47.9 vs 51.7) ...
    assert w8a8.select(512, 9216, 3072)["variant_name"] == "gemm_bn256"
    assert w8a8.select(1024, 3072, 12288)["variant_name"] == "gemm_bn256"
    assert w8a8.select(1024, 3072, 12288, variant=B.VARIANT_GEMM_PAIR)["split_tiles"] == 48
    # ... the pairs, unsplit, on deep K (512 x 9216 x 12288: 47.1 vs 52.0)
    p = w8a8.select(512, 9216, 12288)
    assert p["variant_name"] == "gemm_pair" and p["split_tiles"] == 0 and p["num_tiles"] == 72
    # the full-size layers keep the pair kernel
    for M, N, K in ((4352, 9216, 3072), (4352, 3072, 12288), (8704, 3072, 3072),
                    (8704, 24576, 3072), (16384, 3072, 12288)):
        assert w8a8.select(M, N, K)["variant_name"] == "gemm_pair", (M, N, K)


def test_selector_at_17_rows_follows_the_measured_crossovers():
    # 17 rows, the first above torch._int_mm's limit: the tensor-core small-M
    # variant on weights at least 9216 wide or 8192 deep, the GEMM otherwise
    assert w8a8.select(17, 9216, 3072)["variant_name"] == "gemv_tc"
    assert w8a8.select(17, 12288, 3072)["variant_name"] == "gemv_tc"
    assert w8a8.select(17, 3072, 12288)["variant_name"] == "gemv_tc"
    assert w8a8.select(17, 6144, 3072)["variant_name"].startswith("gemm")
    assert w8a8.select(17, 3072, 3072)["variant_name"].startswith("gemm")
    assert w8a8.select(24, 9216, 3072)["variant_name"].startswith("gemm")
    assert w8a8.select(24, 12288, 3072)["variant_name"] == "gemv_tc"
    assert w8a8.select(25, 12288, 3072)["variant_name"].startswith("gemm")
    # 64-column tiles for one row block only up to 37 tiles of 128 columns
    assert w8a8.select(17, 6144, 3072)["variant_name"] == "gemm_bn128"
    assert w8a8.select(17, 4096, 3072)["variant_name"] == "gemm_bn64"


@pytest.mark.parametrize("M", [49, 100, 4352, 16384])
@pytest.mark.parametrize("KN", [(3072, 9216), (3072, 3072), (3072, 12288), (12288, 3072)])
def test_selector_is_total_and_consistent(M, KN):
    K, N = KN
    p = w8a8.select(M, N, K)
    assert p["variant_name"] in ("gemm_bn64", "gemm_bn128", "gemm_bn256", "gemm_pair")
    tm, tn = p["tile_m"], p["tile_n"]
    assert p["num_tiles"] == -(-M // tm) * -(-N // tn)
    assert 1 <= p["grid"] <= 148
    if p["variant_name"] == "gemm_pair":
        assert tm == tn == 256 and p["grid"] % 2 == 0


def test_quantization_inside_the_gemm_launch_plan():
    # rows whose bf16 fit one epilogue warp's 24 KB share of the operand ring
    assert w8a8.select(4352, 9216, 3072)["quant_in_gemm_launch"] == 1
    assert w8a8.select(4352, 12288, 3072)["quant_in_gemm_launch"] == 1
    assert w8a8.select(4352, 3072, 12288)["quant_in_gemm_launch"] == 1
    assert w8a8.select(8704, 3072, 3072)["quant_in_gemm_launch"] == 1    # any number of passes
    assert w8a8.select(4352, 3072, 12304)["quant_in_gemm_launch"] == 0   # K > 12288
    assert w8a8.select(100, 3072, 3072)["quant_in_gemm_launch"] == 0     # not the pair kernel


# Property check of the selector over random shapes (host only): every plan
# covers the output exactly once with tiles the launch can hold.
from hypothesis import given, settings, strategies as hst  # noqa: E402


def _cdiv(a, b):
    return -(-a // b)


@settings(max_examples=400, deadline=None)
@given(M=hst.integers(1, 20000), n8=hst.integers(1, 4000), k16=hst.integers(1, 2000))
def test_selector_plans_are_valid_for_random_shapes(M, n8, k16):
    N, K = 8 * n8, 16 * k16
    p = w8a8.select(M, N, K)
    v = p["variant_name"]
    assert p["grid"] >= 1
    if v == "gemv":
        assert M <= 16 and M * K + 1024 <= 232448
        assert not ((M >= 5 and (N >= 6144 or K >= 8192)) or
                    (M >= 4 and (N >= 12288 or N * K >= 6144 * 12288)) or (M >= 12 and N >= 3072))
        assert p["quant_in_gemm_launch"] == int(M == 1 or (M == 2 and K <= 8192))
        return
    tm, tn, tiles = p["tile_m"], p["tile_n"], p["num_tiles"]
    if v == "gemv_tc":
        assert 4 <= M <= 48
        assert ((M <= 16 and (N >= 3072 or K >= 8192)) or (M <= 20 and N >= 9216)
                or (M <= 24 and N >= 12288) or (M <= 32 and K >= 8192) or K >= 12288)
        assert tm == 128 and tn == (16 if M <= 16 else (32 if M <= 32 else 64))
        assert tiles == _cdiv(N, 128)
        ks = p["k_split"]
        assert 1 <= ks <= 8 and ks <= _cdiv(K, 128) and p["grid"] == tiles * ks
        return
    assert tiles == _cdiv(M, tm) * _cdiv(N, tn)
    assert p["grid"] <= 148
    if v != "gemm_pair":
        assert p["grid"] == min(tiles, 148)
        assert not (p["split_tiles"] or p["tail_tiles_nsplit"])
        return
    assert tm == tn == 256 and p["grid"] % 2 == 0
    pairs, kb = p["grid"] // 2, _cdiv(K, 128)
    ns, st, per = p["tail_tiles_nsplit"], p["split_tiles"], p["split_kblocks_per_pair"]
    assert not (ns and st)
    if ns:
        rem = tiles % pairs
        assert tiles >= pairs and 0 < rem and 2 * rem <= pairs and ns == 2
    if st:
        assert per >= 24 and per * pairs >= st * kb and st < 2 * pairs
        assert (tiles - st) % pairs == 0
    if p["quant_in_gemm_launch"]:
        assert K <= 12288


# --------------------------------------------------------------------------
# The torch binding checks shapes before anything reaches the library: a
# short bias or output would otherwise let a kernel read or write past the
# end of a buffer.
# --------------------------------------------------------------------------

def _cpu_layer(M=8, N=16, K=32):
    import torch
    return (torch.zeros((M, K), dtype=torch.bfloat16), torch.zeros((N, K), dtype=torch.int8),
            torch.ones(N, dtype=torch.float32))


@pytest.mark.parametrize("fn", ["linear_fused", "w8a16_linear"])
def test_binding_rejects_short_bias_and_output(fn):
    import torch
    x, Wq, s_w = _cpu_layer()
    call = getattr(w8a8, fn)
    with pytest.raises(ValueError, match="bias must have shape"):
        call(x, Wq, s_w, torch.zeros(15, dtype=torch.bfloat16))
    with pytest.raises(ValueError, match="out must have shape"):
        call(x, Wq, s_w, None, out=torch.zeros((7, 16), dtype=torch.bfloat16))
    with pytest.raises(ValueError, match="out must have shape"):
        # fewer rows than M, however wide its row stride
        call(x, Wq, s_w, None, out=torch.zeros((7, 64), dtype=torch.bfloat16)[:, :16])
    with pytest.raises(ValueError, match="must be a CUDA tensor"):
        call(x, Wq, s_w, torch.zeros(16, dtype=torch.bfloat16))   # shapes fine: device next


def test_binding_linear_rejects_short_bias_and_output():
    import torch
    q = torch.zeros((8, 32), dtype=torch.int8)
    s_a = torch.ones(8, dtype=torch.float32)
    _, Wq, s_w = _cpu_layer()
    with pytest.raises(ValueError, match="bias must have shape"):
        w8a8.linear(q, s_a, Wq, s_w, torch.zeros(8, dtype=torch.bfloat16))
    with pytest.raises(ValueError, match="out must have shape"):
        w8a8.linear(q, s_a, Wq, s_w, out=torch.zeros((8, 8), dtype=torch.bfloat16))


def test_debug_peek_tag_is_stable_without_launches():
    a = B.debug_peek_tag()
    b = B.debug_peek_tag()
    assert a == b and 0 < a < 2 ** 56
