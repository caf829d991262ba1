// w8a8_capi.cu -- the C ABI of libw8a8.so (declared in include/w8a8.h):
// argument checks, the (M, N, K) -> kernel selector, TMA descriptor encoding
// and kernel launches.  The library allocates no memory; all scratch memory
// is the caller's workspace.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <atomic>
#include <chrono>
#include <cstdint>
#include <cstring>
#include <mutex>
#include <random>

#include "../../include/w8a8.h"
#include "w8a8_gemm.cuh"
#include "w8a8_gemv.cuh"
#include "w8a8_pack.cuh"
#include "w8a8_peak.cuh"
#include "w8a16_tmem.cuh"
#include "w8a8_ptx.cuh"
#include "w8a8_quant.cuh"
#include "w8a8_swapab.cuh"

namespace w8a8 {

constexpr int64_t kMaxK = 133144;  // 127 * 127 * K <= 2^31 - 1
constexpr int kMaxDevices = 64;
constexpr int kGemmStages256 = 4;  // 4 x 48 KB ring for 128x256 tiles
constexpr int kGemmStages128 = 6;  // 6 x 32 KB ring for 128x128 tiles
constexpr int kGemmStages64 = 8;   // 8 x 24 KB ring for 128x64 tiles
constexpr int kGemmStagesPair = 6; // 6 x 32 KB ring per CTA for 256x256 pair tiles
constexpr int kGemmGroupM = 8;
// K-split tail of the pair kernel (in 128-deep k-blocks): shortest piece a
// pair takes, and the least tail time the split must save per pair.
constexpr int64_t kSplitMinPiece = 24;
constexpr int64_t kSplitMinGain = 24;
constexpr int64_t kQuantMaxV = 12;  // 16-byte vectors per thread in the quant kernel
constexpr int kGemvMaxSmem = 232448 - 1024;   // q rows of the GEMV (M * K bytes)

// ---------------------------------------------------------------- device info

struct DeviceInfo {
  std::atomic<int> state{0};  // 0 unknown, 1 ready
  int cc_major = 0, cc_minor = 0, sms = 0, max_smem_optin = 0;
};
DeviceInfo g_dev[kMaxDevices];

int query_device(const DeviceInfo **out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    cudaGetLastError();
    return W8A8_ERR_CUDA;
  }
  DeviceInfo &d = g_dev[dev];
  if (d.state.load(std::memory_order_acquire) != 1) {
    int maj = 0, min = 0, sms = 0, smem = 0;
    if (cudaDeviceGetAttribute(&maj, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&min, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&smem, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) !=
            cudaSuccess) {
      cudaGetLastError();
      return W8A8_ERR_CUDA;
    }
    d.cc_major = maj;
    d.cc_minor = min;
    d.sms = sms;
    d.max_smem_optin = smem;
    d.state.store(1, std::memory_order_release);
  }
  if (d.cc_major != 10 || d.cc_minor != 0) return W8A8_ERR_UNSUPPORTED_DEVICE;
  *out = &d;
  return W8A8_OK;
}

// ---------------------------------------------------------------- checks

inline bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int check_mk(int64_t M, int64_t K, int64_t ld) {
  if (M < 1 || K < 1 || ld < K) return W8A8_ERR_INVALID_ARG;
  if (K % 16 != 0 || K > kMaxK || ld % 8 != 0) return W8A8_ERR_UNSUPPORTED_SHAPE;
  if (M > INT32_MAX / 2) return W8A8_ERR_UNSUPPORTED_SHAPE;
  return W8A8_OK;
}

int check_n(int64_t N, int64_t ldy) {
  if (N < 1 || ldy < N) return W8A8_ERR_INVALID_ARG;
  if (N % 8 != 0 || ldy % 8 != 0 || N > INT32_MAX / 2) return W8A8_ERR_UNSUPPORTED_SHAPE;
  return W8A8_OK;
}

// ---------------------------------------------------------------- selector

// The fused pair launch quantizes x with its epilogue warps (8 per CTA), one
// row per warp per pass; the rows the first round of tiles reads come through
// the operand ring, one row per warp's share of it at least, hence the bound
// on K (24 KB per warp: 12288 bf16).
constexpr int64_t kFuseMaxK = 12288;


inline int64_t cdiv(int64_t a, int64_t b) { return (a + b - 1) / b; }

inline bool gemv_fits(int64_t M, int64_t K, int max_smem) {
  return M <= kGemvMaxM && M * K + 1024 <= static_cast<int64_t>(max_smem);
}

// The tensor-core small-M variant serves up to this many activation rows.
constexpr int64_t kSwapMaxM = 128;

// Small-M selection, from whole-layer times on a B200 (quantization
// included, CUDA graphs of back-to-back calls, weights rotated over more than
// 2x L2; us):
//
//   N x K          M:   1     2     4     5     8    12    16
//   18432 x 3072  gemv 10.3* 11.9* 15.2  17.7  21.4  29.2  33.3
//                 tc               14.4  14.0  14.5  15.3  16.0   GEMM 18.6-20.4
//   9216 x 3072   gemv  6.3*  7.5*  9.5  10.4  12.7  16.7  19.2
//                 tc               10.4   9.9  10.3  11.4  12.5   GEMM 14.3-16.5
//   3072 x 3072   gemv  3.6*  4.1*  6.4   6.1   7.4  10.0  11.0
//                 tc                9.0   8.3   8.8   9.3   9.9   GEMM 10.9-11.7
//   3072 x 12288  gemv  9.2*  11.3  14.8  16.1  20.1  35.9  42.4
//                 tc               15.2  13.9  14.3  14.9  15.5   GEMM 30.3-32.4
//
// (* the GEMV with the quantization in its own launch; elsewhere the
// quantization kernel runs first.)  The GEMV's dot products cost 1-2 us per
// row on wide weights (and more on deep ones, whose rows fill its shared
// memory); the tensor-core variant is nearly flat in M.  Measured on 110
// shapes of 4-48 rows (N 1024-18432, K 3072-12288), these rules pick the
// fastest variant or one within 3% of it.
inline bool gemv_quantizes_itself(int64_t M, int64_t K) { return M == 1 || (M == 2 && K <= 8192); }
inline bool swap_beats_gemv(int64_t M, int64_t N, int64_t K) {
  return (M >= 5 && (N >= 6144 || K >= 8192)) ||
         (M >= 4 && (N >= 12288 || N * K >= int64_t{6144} * 12288)) || (M >= 12 && N >= 3072);
}
// Above 16 rows (or where the GEMV's rows do not fit), the tensor-core
// variant still beats the GEMM's one row block: to 20 rows from 9216 wide
// (17 rows at 9216 x 3072: 13.5 vs 14.6 us; even at 20; behind from 24), to
// 24 rows from 12288 wide (18432 x 3072 at 24 rows: 17.9 vs 18.3), to 32 rows
// from 8192 deep (3072 x 12288 at 32 rows: 20.6 vs 30.4; 4096 x 8192: 19.0 vs
// 22.3) and to 48 rows from 12288 deep (28.0 vs 30.5 at 3072 x 12288; 8192
// deep at 48 rows: behind, 24.9 vs 21.9).
inline bool swap_beats_gemm(int64_t M, int64_t N, int64_t K) {
  return (M <= 16 && (N >= 3072 || K >= 8192)) || (M <= 20 && N >= 9216) ||
         (M <= 24 && N >= 12288) || (M <= 32 && K >= 8192) || (M <= 48 && K >= 12288);
}

inline int swap_mpad(int64_t M) { return M <= 16 ? 16 : (M <= 32 ? 32 : (M <= 64 ? 64 : 128)); }

inline int swap_max_split(int mpad) {
  switch (mpad) {
    case 16: return SwapLayout<16>::kMaxSplit;
    case 32: return SwapLayout<32>::kMaxSplit;
    case 64: return SwapLayout<64>::kMaxSplit;
    default: return SwapLayout<128>::kMaxSplit;
  }
}

// Clusters of s CTAs (one CTA per SM) that a 148-SM B200 holds at once, as
// CTAs: a cluster must fit within one GPC, so sizes that do not divide the
// GPCs' SM counts leave SMs idle (cudaOccupancyMaxActiveClusters for the
// small-M kernel: 148, 148, 135, 132, 130, 132, 105, 120 CTAs for s = 1..8).
// Scaled to other SM counts.
constexpr int kClusterCTAs148[9] = {0, 148, 148, 135, 132, 130, 132, 105, 120};
inline int64_t max_active_clusters(int64_t s, int32_t sms) {
  return static_cast<int64_t>(kClusterCTAs148[s]) * sms / 148 / s;
}

// CTAs per tile (the cluster size) of the small-M kernel: K shared among up
// to 4 CTAs, or more while the grid stays within 2/3 of the SMs, and never
// more clusters than fit at once (a second wave of clusters doubles the time:
// 24 tiles of 3072 x 12288 at M = 16 took 20.1 us in clusters of 6, of which
// 22 fit, against 12.9 us in clusters of 4).  Measured best per tile count at
// M = 16-32: 8 tiles 4-8, 12 tiles 6, 16 tiles 4-6, 24 tiles 4, 32 tiles 3-4,
// 48 tiles 2, 72 tiles 2, 144 tiles 1.
inline int64_t swap_split(int64_t tiles, int64_t kb, int mpad, int32_t sms) {
  int64_t want = (2 * static_cast<int64_t>(sms) / 3) / tiles;
  if (want < 4) want = 4;
  int64_t split = sms / tiles;
  if (split > want) split = want;
  if (split > swap_max_split(mpad)) split = swap_max_split(mpad);
  if (split > kb) split = kb;
  while (split > 1 && tiles > max_active_clusters(split, sms)) --split;
  return split < 1 ? 1 : split;
}

// How the pair kernel runs its last round(s) of 256 x 256 tiles on `pairs`
// CTA pairs: whole tiles in full rounds, then -- when it pays -- either the
// last round's tiles cut along N into two 128-column tiles (nsplit = 2), or
// the last one to two rounds' tiles shared out along K so that every pair gets
// the same number of k-blocks (a problem of less than one round is shared out
// entirely).  Every shared-out piece costs about two epilogues (its partial
// sums written, or read back and added), some 24 k-blocks of MMA time, so
// pieces are at least that long and the split must save at least that much
// per pair on the tail.
struct PairTail {
  int64_t tile0;   // tiles run whole before the shared-out ones
  int64_t per;     // k-blocks per pair of the shared-out tiles (0: none)
  int64_t nsplit;  // 2: the last round's tiles cut along N
};

inline PairTail pair_tail(int64_t tiles, int64_t kb, int64_t pairs) {
  PairTail t{tiles, 0, 1};
  const int64_t full = tiles / pairs, rem = tiles % pairs;
  if (full >= 1 && rem > 0 && 2 * rem <= pairs) {
    // A last round of rem tiles on `pairs` pairs costs as much as a full
    // round: cut each of its tiles along N into two 128-column tiles, one per
    // pair.  (Narrow tiles read more operand bytes per MMA; at 64 columns the
    // round becomes bandwidth-bound and gains nothing.)
    t.nsplit = 2;
    t.tile0 = full * pairs;
  } else if (rem != 0) {
    const int64_t t0 = full >= 1 ? (full - 1) * pairs : 0;
    const int64_t units = (tiles - t0) * kb;
    int64_t pp = cdiv(units, pairs);
    if (pp < kSplitMinPiece) pp = kSplitMinPiece;
    const int64_t tail_unsplit = (cdiv(tiles, pairs) - t0 / pairs) * kb;
    if (tail_unsplit - pp >= kSplitMinGain && units <= INT32_MAX / 2) {
      t.tile0 = t0;
      t.per = pp;
    }
  }
  return t;
}

// Tile width and pair selection for the GEMM, from whole-layer times on a
// B200 (quantization included, CUDA graphs; 104 shapes of 48-8704 rows, N
// 1024-18432, K 3072 and 12288).  Per round of 148 CTAs, 128-wide tiles take
// 0.67-0.75x the time of 256-wide ones for half the work, so they must fill
// the rounds 1.4x better to win (768 x 9216 x 3072: 29.5 us against 25.3 for
// 256-wide tiles and 24.1 for pairs).  Pair tiles win from 256 rows where
// they fill the rounds about as well -- except under one round of pair tiles
// that one round of single-CTA tiles holds, where the pair kernel either
// shares K out (1024 x 3072 x 12288: 51.7 us against 47.9) or, at K = 3072,
// loses its fill and drain (512 x 9216 x 3072: 18.9 against 18.0); on deep K
// unsplit pairs still win (512 x 9216 x 12288: 47.1 against 52.0).
constexpr double kBn128MinFillGain = 1.4;
constexpr int64_t kPairMinM = 256;
constexpr int64_t kPairOneRoundMinK = 6144;

int select_plan(int64_t M, int64_t N, int64_t K, int32_t sms, int variant, int max_smem,
                w8a8_plan *plan) {
  if (sms < 1) return W8A8_ERR_INVALID_ARG;
  int v = variant;
  if (v == W8A8_VARIANT_AUTO) {
    if (gemv_fits(M, K, max_smem) && !swap_beats_gemv(M, N, K)) {
      v = W8A8_VARIANT_GEMV;
    } else if (swap_beats_gemm(M, N, K)) {
      // a handful of rows against a wide or deep weight: the tensor-core
      // small-M variant (its K shared among the CTAs of a cluster) streams
      // the weight faster than the GEMV's dot products or one row block of
      // the GEMM
      v = W8A8_VARIANT_GEMV_TC;
    } else if (M <= kBM && cdiv(N, 128) * 4 <= sms) {
      // one row block and few 128-column tiles: 64-column tiles put twice as
      // many CTAs on the weight stream (measured ~4% faster at N = 3072; at
      // N = 6144, 96 tiles of 64 columns, 8-18% slower than 48 of 128)
      v = W8A8_VARIANT_GEMM_BN64;
    } else {
      // wave efficiency of each tile width; 256-wide tiles move half the
      // activation bytes per op, so 128-wide tiles must win clearly
      const int64_t t256 = cdiv(M, kBM) * cdiv(N, 256);
      const int64_t t128 = cdiv(M, kBM) * cdiv(N, 128);
      const double e256 = static_cast<double>(t256) / (cdiv(t256, sms) * sms) *
                          (static_cast<double>(N) / (cdiv(N, 256) * 256));
      const double e128 = static_cast<double>(t128) / (cdiv(t128, sms) * sms) *
                          (static_cast<double>(N) / (cdiv(N, 128) * 128));
      v = (e128 > kBn128MinFillGain * e256) ? W8A8_VARIANT_GEMM_BN128 : W8A8_VARIANT_GEMM_BN256;
      // CTA pairs (256 x 256 tiles) halve each CTA's operand traffic; use
      // them when the problem has enough rows that pair tiles fill the GPU
      // about as well as single-CTA tiles do.
      const int64_t pairs = sms / 2;
      const int64_t tp = cdiv(M, 256) * cdiv(N, 256);
      const double ep = static_cast<double>(tp) / (cdiv(tp, pairs) * pairs) *
                        (static_cast<double>(M) / (cdiv(M, 256) * 256)) *
                        (static_cast<double>(N) / (cdiv(N, 256) * 256));
      const double e1 = (v == W8A8_VARIANT_GEMM_BN128 ? e128 : e256) *
                        (static_cast<double>(M) / (cdiv(M, kBM) * kBM));
      const int64_t t1 = v == W8A8_VARIANT_GEMM_BN128 ? t128 : t256;
      const bool one_round = pairs >= 1 && tp < pairs && t1 <= sms;
      const bool pair_loses_one_round =
          one_round && (K < kPairOneRoundMinK || pair_tail(tp, cdiv(K, kBK), pairs).per > 0);
      if (M >= kPairMinM && sms >= 2 && ep >= 0.95 * e1 && !pair_loses_one_round)
        v = W8A8_VARIANT_GEMM_PAIR;
    }
  }
  std::memset(plan, 0, sizeof(*plan));
  plan->variant = v;
  if (v == W8A8_VARIANT_GEMV_TC) {
    if (M > kSwapMaxM) return W8A8_ERR_UNSUPPORTED_SHAPE;
    const int mpad = swap_mpad(M);
    const int64_t tiles = cdiv(N, kBM);
    const int64_t kb = cdiv(K, kBK);
    const int64_t split = swap_split(tiles, kb, mpad, sms);
    if (tiles * split > INT32_MAX) return W8A8_ERR_UNSUPPORTED_SHAPE;
    plan->tile_m = kBM;
    plan->tile_n = mpad;
    plan->num_tiles = static_cast<int32_t>(tiles);
    plan->k_split = static_cast<int32_t>(split);
    plan->grid = static_cast<int32_t>(tiles * split);
    plan->waves_x100 = static_cast<int32_t>(cdiv(100 * tiles * split, sms));
    return W8A8_OK;
  }
  if (v == W8A8_VARIANT_GEMV) {
    if (!gemv_fits(M, K, max_smem)) return W8A8_ERR_UNSUPPORTED_SHAPE;
    const int64_t smem = M * K;
    int per_sm = static_cast<int>((max_smem) / (smem + 1024));
    per_sm = per_sm < 1 ? 1 : (per_sm > 2 ? 2 : per_sm);  // one resident wave
    const int64_t rows_per_cta = kGemvWarps * kGemvRows;
    int64_t grid = cdiv(N, rows_per_cta);
    const int64_t cap = static_cast<int64_t>(sms) * per_sm;
    plan->num_tiles = static_cast<int32_t>(N);
    plan->grid = static_cast<int32_t>(grid < cap ? grid : cap);
    plan->quant_in_gemm_launch = gemv_quantizes_itself(M, K) ? 1 : 0;
    return W8A8_OK;
  }
  if (v == W8A8_VARIANT_GEMM_PAIR) {
    if (sms < 2) return W8A8_ERR_UNSUPPORTED_SHAPE;
    const int64_t tiles = cdiv(M, 256) * cdiv(N, 256);
    if (tiles > INT32_MAX) return W8A8_ERR_UNSUPPORTED_SHAPE;
    const int64_t kb = cdiv(K, kBK);
    int64_t pairs = sms / 2;
    const int64_t full = tiles / pairs;
    const PairTail tail = pair_tail(tiles, kb, pairs);
    const int64_t tile0 = tail.tile0, per = tail.per, nsplit = tail.nsplit;
    if (tile0 == tiles && tiles < pairs) pairs = tiles;
    plan->tile_m = 256;
    plan->tile_n = 256;
    plan->num_tiles = static_cast<int32_t>(tiles);
    plan->grid = static_cast<int32_t>(2 * pairs);
    plan->quant_in_gemm_launch = K <= kFuseMaxK ? 1 : 0;
    if (nsplit > 1) {
      plan->tail_tiles_nsplit = static_cast<int32_t>(nsplit);
      plan->waves_x100 = static_cast<int32_t>(100 * full + 100 / nsplit);
    } else if (tile0 < tiles) {
      plan->split_tiles = static_cast<int32_t>(tiles - tile0);
      plan->split_kblocks_per_pair = static_cast<int32_t>(per);
      plan->waves_x100 = static_cast<int32_t>(100 * tile0 / pairs + cdiv(100 * per, kb));
    } else {
      plan->waves_x100 = static_cast<int32_t>(100 * tiles / pairs);
    }
    return W8A8_OK;
  }
  if (v != W8A8_VARIANT_GEMM_BN64 && v != W8A8_VARIANT_GEMM_BN128 && v != W8A8_VARIANT_GEMM_BN256)
    return W8A8_ERR_INVALID_ARG;
  const int bn = v == W8A8_VARIANT_GEMM_BN64 ? 64 : (v == W8A8_VARIANT_GEMM_BN128 ? 128 : 256);
  const int64_t tiles = cdiv(M, kBM) * cdiv(N, bn);
  if (tiles > INT32_MAX) return W8A8_ERR_UNSUPPORTED_SHAPE;
  plan->tile_m = kBM;
  plan->tile_n = bn;
  plan->num_tiles = static_cast<int32_t>(tiles);
  plan->grid = static_cast<int32_t>(tiles < sms ? tiles : sms);
  plan->waves_x100 = static_cast<int32_t>(100 * tiles / plan->grid);
  return W8A8_OK;
}

// ---------------------------------------------------------------- workspace

size_t align256(size_t b) { return (b + 255) & ~static_cast<size_t>(255); }

// Per-128-row-block "rows quantized" counters of the fused pair launch.
size_t ready_counter_bytes(int64_t M) {
  return align256(static_cast<size_t>(cdiv(M, kBM)) * sizeof(unsigned long long));
}


size_t fused_workspace_bytes(int64_t M, int64_t K) {
  return align256(static_cast<size_t>(M) * static_cast<size_t>(K)) +
         align256(static_cast<size_t>(M) * sizeof(float));
}

// The pair kernel's K-split region: arrival counters (16 per shared-out
// tile, 64-bit), then the partial-sum slots (split_tiles + pairs - 1 of them,
// 16 slices of 32 x 128 int32 each).  The counters are cleared on the stream
// before each launch that uses them; the partial sums need no initializing.
size_t split_counter_bytes(const w8a8_plan &plan) {
  return align256(static_cast<size_t>(plan.split_tiles) * kSlicesPerTile *
                  sizeof(unsigned long long));
}
size_t split_workspace_bytes(const w8a8_plan &plan) {
  if (plan.variant != W8A8_VARIANT_GEMM_PAIR || plan.split_tiles == 0) return 0;
  const size_t slots = static_cast<size_t>(plan.split_tiles) + plan.grid / 2 - 1;
  return split_counter_bytes(plan) + slots * kSlicesPerTile * kSlotInts * sizeof(int32_t);
}

// The K-split region handed to the pair kernel; counters == nullptr runs it
// unsplit.
struct SplitRegion {
  unsigned long long *counters = nullptr;
  int32_t *partials = nullptr;
};

// Launch tags of the arrival counters (K-split tail, fused quantization).
// The host clears a launch's counter region (cudaMemsetAsync, which
// allocates nothing) before the launch, and every counter also carries the
// launch's tag, so a word that some other launch left counts as zero.  Tags
// count up from a random start drawn once per process: memory written by
// other code (another layer's activations, another process's counters) is
// not mistaken for a live counter except by a 2^-48 chance.
unsigned long long initial_tag() {
  unsigned long long t = 0;
  try {
    std::random_device rd;
    t = (static_cast<unsigned long long>(rd()) << 32) ^ rd();
  } catch (...) {
    t = static_cast<unsigned long long>(
        std::chrono::high_resolution_clock::now().time_since_epoch().count());
  }
  return t;
}
std::atomic<unsigned long long> g_tag{initial_tag()};

// The next launch tag, `bits` wide and never 0.
unsigned long long next_tag(int bits) {
  const unsigned long long mask = (1ull << bits) - 1;
  const unsigned long long t = g_tag.fetch_add(1, std::memory_order_relaxed) & mask;
  return t != 0 ? t : 1;
}

// Clears `bytes` of counters on `stream` before the launch that uses them.
int clear_counters(void *p, size_t bytes, cudaStream_t stream) {
  if (p == nullptr || bytes == 0) return W8A8_OK;
  if (cudaMemsetAsync(p, 0, bytes, stream) != cudaSuccess) {
    cudaGetLastError();
    return W8A8_ERR_CUDA;
  }
  return W8A8_OK;
}

SplitRegion split_region(const w8a8_plan &plan, void *base, size_t bytes) {
  SplitRegion r;
  const size_t need = split_workspace_bytes(plan);
  if (need == 0 || base == nullptr || bytes < need || !aligned16(base)) return r;
  r.counters = static_cast<unsigned long long *>(base);
  r.partials = reinterpret_cast<int32_t *>(static_cast<uint8_t *>(base) + split_counter_bytes(plan));
  return r;
}

// ---------------------------------------------------------------- TMA maps

PFN_cuTensorMapEncodeTiled_v12000 get_encoder() {
  static std::atomic<PFN_cuTensorMapEncodeTiled_v12000> fn{nullptr};
  PFN_cuTensorMapEncodeTiled_v12000 f = fn.load(std::memory_order_acquire);
  if (f == nullptr) {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) !=
            cudaSuccess ||
        q != cudaDriverEntryPointSuccess || p == nullptr) {
      cudaGetLastError();
      return nullptr;
    }
    f = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    fn.store(f, std::memory_order_release);
  }
  return f;
}

// int8 matrix [rows, K] dense, box = 128 (K) x box_rows, 128-byte swizzle.
// Tensor maps encoded earlier on this thread, keyed by everything that goes
// into them (which map form, base address, extents, row stride, box rows): a
// map holds addresses and shapes only, so a hit is the map a new encoding
// would produce.  Encoding costs host time on every layer call otherwise.
struct MapKey {
  int kind;
  const void *base;
  int64_t rows, cols, ld;
  int box;
  bool operator==(const MapKey &o) const {
    return kind == o.kind && base == o.base && rows == o.rows && cols == o.cols && ld == o.ld &&
           box == o.box;
  }
};
struct MapEntry {
  MapKey key;
  bool valid;
  CUtensorMap map;
};
constexpr int kMapCacheSize = 64;
thread_local MapEntry t_map_cache[kMapCacheSize];

MapEntry &map_slot(const MapKey &k) {
  uint64_t h = reinterpret_cast<uintptr_t>(k.base) * 0x9E3779B97F4A7C15ull;
  h ^= static_cast<uint64_t>(k.kind) * 0xC2B2AE3D27D4EB4Full + static_cast<uint64_t>(k.rows) * 31u +
       static_cast<uint64_t>(k.cols) * 131u + static_cast<uint64_t>(k.ld) * 7u +
       static_cast<uint64_t>(k.box);
  return t_map_cache[(h >> 32) % kMapCacheSize];
}

bool map_lookup(const MapKey &k, CUtensorMap *out) {
  const MapEntry &e = map_slot(k);
  if (!e.valid || !(e.key == k)) return false;
  *out = e.map;
  return true;
}

void map_store(const MapKey &k, const CUtensorMap &m) {
  MapEntry &e = map_slot(k);
  e.key = k;
  e.map = m;
  e.valid = true;
}

int encode_i8_map(CUtensorMap *map, const void *base, int64_t rows, int64_t K, int box_rows) {
  const MapKey key{1, base, rows, K, K, box_rows};
  if (map_lookup(key, map)) return W8A8_OK;
  PFN_cuTensorMapEncodeTiled_v12000 enc = get_encoder();
  if (enc == nullptr) return W8A8_ERR_CUDA;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(K)};
  cuuint32_t box[2] = {static_cast<cuuint32_t>(kBK), static_cast<cuuint32_t>(box_rows)};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void *>(base), dims,
                   strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return W8A8_ERR_CUDA;
  map_store(key, *map);
  return W8A8_OK;
}

// bf16 matrix [rows, cols] with row stride ld elements, box 64 (cols) x
// box_rows, 128-byte swizzle (the W8A16 GEMM's activation operand).
int encode_bf16_load_map(CUtensorMap *map, const void *base, int64_t rows, int64_t cols,
                         int64_t ld, int box_rows) {
  const MapKey key{2, base, rows, cols, ld, box_rows};
  if (map_lookup(key, map)) return W8A8_OK;
  PFN_cuTensorMapEncodeTiled_v12000 enc = get_encoder();
  if (enc == nullptr) return W8A8_ERR_CUDA;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(ld * 2)};
  cuuint32_t box[2] = {static_cast<cuuint32_t>(kWtBK), static_cast<cuuint32_t>(box_rows)};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims,
                   strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return W8A8_ERR_CUDA;
  map_store(key, *map);
  return W8A8_OK;
}

// int8 matrix [rows, K] dense, box 64 (K) x box_rows, 64-byte swizzle (the
// tensor-memory W8A16 GEMM's weights: a converter lane reads one row's four
// 16-byte chunks without bank conflicts).
int encode_i8_sw64_map(CUtensorMap *map, const void *base, int64_t rows, int64_t K,
                       int box_rows) {
  const MapKey key{3, base, rows, K, K, box_rows};
  if (map_lookup(key, map)) return W8A8_OK;
  PFN_cuTensorMapEncodeTiled_v12000 enc = get_encoder();
  if (enc == nullptr) return W8A8_ERR_CUDA;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(K)};
  cuuint32_t box[2] = {static_cast<cuuint32_t>(kWtBK), static_cast<cuuint32_t>(box_rows)};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void *>(base), dims, strides,
                   box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return W8A8_ERR_CUDA;
  map_store(key, *map);
  return W8A8_OK;
}

// bf16 matrix [rows, cols] with row stride ld elements, box 32 x 32, 64-byte
// swizzle (the epilogue's staging layout).
int encode_bf16_store_map(CUtensorMap *map, const void *base, int64_t rows, int64_t cols,
                          int64_t ld) {
  const MapKey key{4, base, rows, cols, ld, 0};
  if (map_lookup(key, map)) return W8A8_OK;
  PFN_cuTensorMapEncodeTiled_v12000 enc = get_encoder();
  if (enc == nullptr) return W8A8_ERR_CUDA;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(ld * 2)};
  cuuint32_t box[2] = {static_cast<cuuint32_t>(kEpiChunk), 32u};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims,
                   strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B,
                   CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return W8A8_ERR_CUDA;
  map_store(key, *map);
  return W8A8_OK;
}

// ---------------------------------------------------------------- launches

// Launch with cudaLaunchKernelEx.  dependent = programmatic dependent launch:
// the kernel may start before the preceding work on the stream completes and
// must call griddepcontrol.wait before touching anything that work produces
// (the GEMM kernels do, before their first q / s_a read and any store).
template <typename... KArgs, typename... Args>
int launch_cl(bool dependent, unsigned cluster_x, void (*kernel)(KArgs...), dim3 grid, dim3 block,
              size_t smem, cudaStream_t stream, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[2];
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = 0;
  if (dependent) {
    attr[cfg.numAttrs].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[cfg.numAttrs].val.programmaticStreamSerializationAllowed = 1;
    ++cfg.numAttrs;
  }
  if (cluster_x > 1) {  // a cluster of cluster_x CTAs along x (no multicast loads)
    attr[cfg.numAttrs].id = cudaLaunchAttributeClusterDimension;
    attr[cfg.numAttrs].val.clusterDim.x = cluster_x;
    attr[cfg.numAttrs].val.clusterDim.y = 1;
    attr[cfg.numAttrs].val.clusterDim.z = 1;
    ++cfg.numAttrs;
  }
  if (cfg.numAttrs == 0) cfg.attrs = nullptr;
  cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, args...);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return W8A8_ERR_CUDA;
  }
  return W8A8_OK;
}

template <typename... KArgs, typename... Args>
int launch_ex(bool dependent, void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
              cudaStream_t stream, Args... args) {
  return launch_cl(dependent, 1u, kernel, grid, block, smem, stream, args...);
}

template <typename... KArgs, typename... Args>
int launch(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
           Args... args) {
  return launch_ex(false, kernel, grid, block, smem, stream, args...);
}

// Raise a kernel's dynamic shared memory limit to `bytes`, once per device
// (the attribute is per function and device; setting it costs microseconds,
// so it is not repeated on every call).  Each kernel asks for its largest
// possible footprint.
template <auto Kernel>
int ensure_smem_limit(int bytes) {
  static std::atomic<uint64_t> done{0};  // one bit per device
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    cudaGetLastError();
    return W8A8_ERR_CUDA;
  }
  const uint64_t bit = 1ull << dev;
  if (done.load(std::memory_order_acquire) & bit) return W8A8_OK;
  if (cudaFuncSetAttribute(reinterpret_cast<const void *>(Kernel),
                           cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) != cudaSuccess) {
    cudaGetLastError();
    return W8A8_ERR_CUDA;
  }
  done.fetch_or(bit, std::memory_order_acq_rel);
  return W8A8_OK;
}

// Warps per row and row slots per group of quant_rows_bulk_kernel for rows of
// K elements: at most 3072 elements per warp (1, 2 or 4 warps per row), then
// as many slots (up to 4) as the slot storage holds for the 16 / G groups.
void quant_bulk_shape(int64_t K, int *group_warps, int *slots) {
  const int64_t row_bytes = 2 * K;
  int g = 1;
  while (g < 4 && g * kQuantBulkWarpElems < K) g *= 2;
  const int64_t groups = kQuantBulkWarps / g;
  int64_t sl = kQuantBulkSmem / (groups * row_bytes);
  if (sl > kQuantBulkMaxSlots) sl = kQuantBulkMaxSlots;
  *group_warps = g;
  *slots = static_cast<int>(sl);
}

// release_early: let the kernel that follows be launched as soon as this one
// starts (activations; never for weights, see quant_rows_kernel).
int launch_quant(const void *x, int64_t rows, int64_t K, int64_t ldx, int8_t *q, float *s,
                 bool release_early, cudaStream_t stream) {
  const int rel = release_early ? 1 : 0;
  const uint16_t *xp = static_cast<const uint16_t *>(x);
  if (rows > INT32_MAX / 2) return W8A8_ERR_UNSUPPORTED_SHAPE;
  const DeviceInfo *d = nullptr;
  int st = query_device(&d);
  if (st != W8A8_OK) return st;
  int gw = 0, slots = 0;
  quant_bulk_shape(K, &gw, &slots);
  // The bulk kernel gives each CTA 16 / gw rows at a time; with 5 or more
  // rows but fewer than that fills the SMs with, the register kernel below
  // spreads them wider (up to one row per CTA).  Measured on a B200 with the
  // layer that follows: 16 rows x 3072, 3.7 -> 1.9 us alone, 17.3 -> 16.8 us
  // for the 18432-wide layer; at 2-4 rows the bulk kernel's single CTA was
  // 0.3-0.5 us faster inside the layer.
  if (K <= kQuantBulkMaxK && (rows < 5 || cdiv(rows, kQuantBulkWarps / gw) >= d->sms)) {
    const int groups = kQuantBulkWarps / gw;
    const int smem = groups * slots * static_cast<int>(2 * K);
    st = ensure_smem_limit<quant_rows_bulk_kernel>(kQuantBulkSmem);
    if (st != W8A8_OK) return st;
    int64_t grid = cdiv(rows, groups);
    if (grid > d->sms) grid = d->sms;
    return launch_ex(true, quant_rows_bulk_kernel, dim3(static_cast<unsigned>(grid)),
                     dim3(kQuantBulkWarps * 32), static_cast<size_t>(smem), stream, xp,
                     static_cast<int>(rows), static_cast<int>(K), ldx, q, s, gw, slots, rel);
  }
  // G threads per row (32 .. 256), each holding V <= kQuantMaxV vectors of
  // 8 bf16 in registers, and G widened until the rows fill the SMs (or one
  // row per CTA); longer rows take the two-pass kernel.
  const int64_t nvec = K / 8;
  int G = 32;
  int64_t V = cdiv(nvec, G);
  while (G < 256 && (V > kQuantMaxV || cdiv(rows, 256 / G) < d->sms)) {
    G *= 2;
    V = cdiv(nvec, G);
  }
  if (V > kQuantMaxV) {  // rows longer than 256 x 12 x 8 = 24576 elements
    return launch_ex(true, quant_rows_long_kernel, dim3(static_cast<unsigned>(rows)), dim3(256), 0,
                     stream, xp, K, ldx, q, s, rel);
  }
  const int rows_per_block = 256 / G;
  const int64_t grid = cdiv(rows, rows_per_block);
  const int r32 = static_cast<int>(rows), k32 = static_cast<int>(K);
#define W8A8_QUANT_CASE(VV)                                                                \
  return launch_ex(true, quant_rows_kernel<VV>, dim3(static_cast<unsigned>(grid)), dim3(256), \
                   0, stream, xp, r32, k32, ldx, q, s, G, rel)
  switch (V) {
    case 1: W8A8_QUANT_CASE(1);
    case 2: W8A8_QUANT_CASE(2);
    case 3: W8A8_QUANT_CASE(3);
    case 4: W8A8_QUANT_CASE(4);
    case 5: case 6: W8A8_QUANT_CASE(6);
    case 7: case 8: W8A8_QUANT_CASE(8);
    default: W8A8_QUANT_CASE(12);
  }
#undef W8A8_QUANT_CASE
}

template <int BN, int STAGES, bool RAW>
int launch_gemm_t(const w8a8_plan &plan, const int8_t *q, const float *s_a, int64_t M,
                  int64_t K, const int8_t *wq, const float *s_w, const void *bias, int64_t N,
                  void *y, int64_t ldy, int32_t *acc, cudaStream_t stream) {
  using L = GemmLayout<BN, STAGES>;
  CUtensorMap ma, mb, my;
  int st = encode_i8_map(&ma, q, M, K, kBM);
  if (st != W8A8_OK) return st;
  st = encode_i8_map(&mb, wq, N, K, BN);
  if (st != W8A8_OK) return st;
  if (RAW) {
    std::memset(&my, 0, sizeof(my));  // the raw-int32 variant stores directly
  } else {
    st = encode_bf16_store_map(&my, y, M, N, ldy);
    if (st != W8A8_OK) return st;
  }
  GemmParams p;
  p.M = static_cast<int32_t>(M);
  p.N = static_cast<int32_t>(N);
  p.K = static_cast<int32_t>(K);
  p.num_m_blk = static_cast<int32_t>(cdiv(M, kBM));
  p.num_n_blk = static_cast<int32_t>(cdiv(N, BN));
  p.num_tiles = plan.num_tiles;
  p.k_blocks = static_cast<int32_t>(cdiv(K, kBK));
  p.group_m = kGemmGroupM;
  p.s_a = s_a;
  p.s_w = s_w;
  p.bias = static_cast<const uint16_t *>(bias);
  p.y = static_cast<uint16_t *>(y);
  p.ldy = ldy;
  p.acc_out = acc;
  constexpr auto kernel = gemm_i8_tcgen05_kernel<BN, STAGES, RAW>;
  st = ensure_smem_limit<kernel>(L::kSmemBytes);
  if (st != W8A8_OK) return st;
  return launch_ex(true, kernel, dim3(plan.grid), dim3(kGemmThreads), L::kSmemBytes, stream, ma,
                   mb, my, p);
}

// Rows of x that the pair kernel's first round of work items reads: every
// pair's first item is a tile below min(tiles, pairs) in the banded order
// (or a K-piece of one), so the row blocks of those tiles, rounded to whole
// 128-row counter blocks and capped at M.
int64_t pair_first_round_rows(const w8a8_plan &plan, int64_t M, int64_t N) {
  const int64_t num_m = cdiv(M, 256), num_n = cdiv(N, kPairBN);
  const int64_t group_m = kGemmGroupM / 2;
  const int64_t pairs = plan.grid / 2;
  const int64_t upto = plan.num_tiles < pairs ? plan.num_tiles : pairs;
  int64_t max_mb = 0;
  for (int64_t t = 0; t < upto; ++t) {
    const int64_t band = group_m * num_n;
    const int64_t g = t / band, first_m = g * group_m;
    const int64_t rows_in_band = num_m - first_m < group_m ? num_m - first_m : group_m;
    const int64_t mb = first_m + (t - g * band) % rows_in_band;
    if (mb > max_mb) max_mb = mb;
  }
  const int64_t rows = (max_mb + 1) * 256;
  return rows < M ? rows : M;
}

// The per-token quantization fused into the pair launch: x is quantized into
// q / s_a (the GEMM's operands) by the kernel itself.
struct FuseArgs {
  const void *x;
  int64_t ldx;
  unsigned long long *row_ready;  // cdiv(M, 128) counters
};

template <bool RAW, bool FUSE>
int launch_gemm_pair(const w8a8_plan &plan, const int8_t *q, const float *s_a, int64_t M,
                     int64_t K, const int8_t *wq, const float *s_w, const void *bias, int64_t N,
                     void *y, int64_t ldy, int32_t *acc, const SplitRegion &split,
                     const FuseArgs *fuse, cudaStream_t stream) {
  using L = PairLayout<kGemmStagesPair>;
  CUtensorMap ma, mb, mbt, my;
  int st = encode_i8_map(&ma, q, M, K, kBM);
  if (st != W8A8_OK) return st;
  st = encode_i8_map(&mb, wq, N, K, kPairBN / 2);
  if (st != W8A8_OK) return st;
  // narrow tail tiles: each CTA loads (256 / nsplit) / 2 rows of Wq per stage
  const int nsplit = plan.tail_tiles_nsplit > 1 ? plan.tail_tiles_nsplit : 1;
  if (nsplit > 1) {
    st = encode_i8_map(&mbt, wq, N, K, kPairBN / 2 / nsplit);
    if (st != W8A8_OK) return st;
  } else {
    mbt = mb;
  }
  if (RAW) {
    std::memset(&my, 0, sizeof(my));
  } else {
    st = encode_bf16_store_map(&my, y, M, N, ldy);
    if (st != W8A8_OK) return st;
  }
  GemmParams p;
  p.M = static_cast<int32_t>(M);
  p.N = static_cast<int32_t>(N);
  p.K = static_cast<int32_t>(K);
  p.num_m_blk = static_cast<int32_t>(cdiv(M, 256));
  p.num_n_blk = static_cast<int32_t>(cdiv(N, kPairBN));
  p.num_tiles = plan.num_tiles;
  p.k_blocks = static_cast<int32_t>(cdiv(K, kBK));
  p.group_m = kGemmGroupM / 2;
  p.s_a = s_a;
  p.s_w = s_w;
  p.bias = static_cast<const uint16_t *>(bias);
  p.y = static_cast<uint16_t *>(y);
  p.ldy = ldy;
  p.acc_out = acc;
  p.dp_tiles = plan.num_tiles;
  p.tail_nsplit = 1;
  p.sk_per = 0;
  p.sk_units = 0;
  p.split_partials = nullptr;
  p.split_counters = nullptr;
  p.split_epoch = 0;
  int grid = plan.grid;
  if (nsplit > 1) {
    p.tail_nsplit = nsplit;
    p.dp_tiles = plan.num_tiles - plan.num_tiles % (plan.grid / 2);
  } else if (plan.split_tiles > 0 && split.counters != nullptr) {
    p.dp_tiles = plan.num_tiles - plan.split_tiles;
    p.sk_per = plan.split_kblocks_per_pair;
    p.sk_units = plan.split_tiles * p.k_blocks;
    p.split_partials = split.partials;
    p.split_counters = split.counters;
    p.split_epoch = next_tag(56);
  } else if (plan.split_tiles > 0 && plan.num_tiles < plan.grid / 2) {
    grid = 2 * plan.num_tiles;  // unsplit and under one wave: one pair per tile
  }
  p.x = nullptr;
  p.ldx = 0;
  p.q_w = nullptr;
  p.s_a_w = nullptr;
  p.row_ready = nullptr;
  p.fuse_tag = 0;
  p.fuse_bulk_rows = 0;
  if (FUSE) {
    p.x = static_cast<const uint16_t *>(fuse->x);
    p.ldx = fuse->ldx;
    p.q_w = const_cast<int8_t *>(q);
    p.s_a_w = const_cast<float *>(s_a);
    p.row_ready = fuse->row_ready;
    p.fuse_tag = next_tag(48);
    p.fuse_bulk_rows = static_cast<int32_t>(pair_first_round_rows(plan, M, N));
  }
  constexpr auto kernel = gemm_i8_tcgen05_pair_kernel<kGemmStagesPair, RAW, FUSE>;
  st = ensure_smem_limit<kernel>(L::kSmemBytes);
  if (st != W8A8_OK) return st;
  return launch_ex(true, kernel, dim3(grid), dim3(kGemmThreads), L::kSmemBytes, stream, ma, mb,
                   mbt, my, p);
}

template <int MPAD, bool RAW>
int launch_swapab_t(const w8a8_plan &plan, const int8_t *q, const float *s_a, int64_t M, int64_t K,
                    const int8_t *wq, const float *s_w, const void *bias, int64_t N, void *y,
                    int64_t ldy, int32_t *acc, cudaStream_t stream) {
  using L = SwapLayout<MPAD>;
  CUtensorMap mw, mq;
  int st = encode_i8_map(&mw, wq, N, K, kBM);
  if (st != W8A8_OK) return st;
  st = encode_i8_map(&mq, q, M, K, MPAD);
  if (st != W8A8_OK) return st;
  SwapParams p;
  p.M = static_cast<int32_t>(M);
  p.N = static_cast<int32_t>(N);
  p.K = static_cast<int32_t>(K);
  p.k_blocks = static_cast<int32_t>(cdiv(K, kBK));
  p.split = plan.k_split;
  p.s_a = s_a;
  p.s_w = s_w;
  p.bias = static_cast<const uint16_t *>(bias);
  p.y = static_cast<uint16_t *>(y);
  p.ldy = ldy;
  p.acc_out = acc;
  constexpr auto kernel = gemm_i8_swapab_kernel<MPAD, RAW>;
  st = ensure_smem_limit<kernel>(L::kSmemBytes);
  if (st != W8A8_OK) return st;
  return launch_cl(true, static_cast<unsigned>(plan.k_split), kernel, dim3(plan.grid),
                   dim3(kSwThreads), L::kSmemBytes, stream, mw, mq, p);
}

template <bool RAW>
int launch_swapab(const w8a8_plan &plan, const int8_t *q, const float *s_a, int64_t M, int64_t K,
                  const int8_t *wq, const float *s_w, const void *bias, int64_t N, void *y,
                  int64_t ldy, int32_t *acc, cudaStream_t stream) {
  switch (plan.tile_n) {
    case 16: return launch_swapab_t<16, RAW>(plan, q, s_a, M, K, wq, s_w, bias, N, y, ldy, acc, stream);
    case 32: return launch_swapab_t<32, RAW>(plan, q, s_a, M, K, wq, s_w, bias, N, y, ldy, acc, stream);
    case 64: return launch_swapab_t<64, RAW>(plan, q, s_a, M, K, wq, s_w, bias, N, y, ldy, acc, stream);
    default: return launch_swapab_t<128, RAW>(plan, q, s_a, M, K, wq, s_w, bias, N, y, ldy, acc, stream);
  }
}

template <bool FUSED, bool RAW>
int launch_gemv_m(const w8a8_plan &plan, const GemvParams &p, cudaStream_t stream) {
  const int smem = p.M * p.K;
#define W8A8_GEMV_CASE(MT)                                                              \
  {                                                                                     \
    constexpr auto kernel = gemv_i8_kernel<MT, FUSED, RAW>;                             \
    int st = ensure_smem_limit<kernel>(kGemvMaxSmem);                                   \
    if (st != W8A8_OK) return st;                                                       \
    return launch_ex(true, kernel, dim3(plan.grid), dim3(kGemvThreads), smem, stream, p); \
  }
  if (p.M <= 1) W8A8_GEMV_CASE(1)
  if (p.M <= 2) W8A8_GEMV_CASE(2)
  if (p.M <= 4) W8A8_GEMV_CASE(4)
  if (p.M <= 8) W8A8_GEMV_CASE(8)
  W8A8_GEMV_CASE(16)
#undef W8A8_GEMV_CASE
}

__global__ void bounded_wait_selftest_kernel(uint64_t limit_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_mbarrier_init();
  }
  __syncthreads();
  // nothing ever arrives on `bar`: the wait must give up after limit_ns
  if (threadIdx.x == 0) mbar_wait(&bar, 0u, &abort_flag, limit_ns);
}

// Every positive finite bf16 maximum a (blockIdx.x + 1) against every bf16
// value x with |x| <= a: the fast step's result -- scalar, and in the packed
// fp32x2 form the bulk quantization kernel uses -- must equal the
// IEEE-division path's, bit for bit.
__global__ void __launch_bounds__(256) quant_exhaustive_kernel(unsigned long long *counts) {
  const uint32_t abits = blockIdx.x + 1u;  // 0x0001 .. 0x7F7F
  const float a = __uint_as_float(abits << 16);
  const float s = __fdiv_rn(a, 127.0f);
  if (!quant_fast_ok(s)) return;
  const float y = __frcp_rn(s);
  const float2 neg_s = make_float2(-s, -s), y2 = make_float2(y, y);
  unsigned long long checked = 0, bad = 0;
  for (uint32_t xb = threadIdx.x; xb < 65536u; xb += blockDim.x) {
    if ((xb & 0x7FFFu) > abits) continue;  // |x| > a (also skips Inf and NaN)
    const float x = __uint_as_float(xb << 16);
    ++checked;
    const uint32_t want = quant_exact(x, s);
    if (quant_fast(x, s, y) != want) ++bad;
    // the packed form: x in every one of the 8 positions of a vector
    const uint32_t w = xb | (xb << 16);
    const uint2 codes = quant_vec8_x2(make_uint4(w, w, w, w), neg_s, y2);
    const uint32_t b = want & 0xFFu;
    if (codes.x != b * 0x01010101u || codes.y != b * 0x01010101u) ++bad;
  }
  atomicAdd(&counts[0], checked);
  if (bad) atomicAdd(&counts[1], bad);
}

// split_ws / split_ws_bytes: room for the pair kernel's K-split region, or
// nullptr / 0 (the pair kernel then runs unsplit).  counters_cleared: the
// caller has already cleared the region's counters on `stream` (before an
// earlier launch of the same call), so none is issued here.
int linear_impl(const int8_t *q, const float *s_a, int64_t M, int64_t K, const int8_t *Wq,
                const float *s_w, const void *bias, int64_t N, void *y, int64_t ldy,
                int32_t *acc, int variant, void *split_ws, size_t split_ws_bytes,
                bool counters_cleared, cudaStream_t stream) {
  if (!q || !s_a || !Wq || !s_w || (!y && !acc)) return W8A8_ERR_INVALID_ARG;
  int st = check_mk(M, K, K);
  if (st != W8A8_OK) return st;
  st = check_n(N, acc ? (ldy >= N ? ldy : N) : ldy);
  if (st != W8A8_OK) return st;
  if (!aligned16(q) || !aligned16(Wq) || !aligned16(s_w) || (bias && !aligned16(bias)) ||
      (y && !aligned16(y)) || (acc && !aligned16(acc)) ||
      (reinterpret_cast<uintptr_t>(s_a) & 3u))
    return W8A8_ERR_MISALIGNED;
  const DeviceInfo *d = nullptr;
  st = query_device(&d);
  if (st != W8A8_OK) return st;
  w8a8_plan plan;
  st = select_plan(M, N, K, d->sms, variant, d->max_smem_optin, &plan);
  if (st != W8A8_OK) return st;
  if (plan.variant == W8A8_VARIANT_GEMV) {
    GemvParams p = {};
    p.M = static_cast<int32_t>(M);
    p.N = static_cast<int32_t>(N);
    p.K = static_cast<int32_t>(K);
    p.q = q;
    p.s_a = s_a;
    p.wq = Wq;
    p.s_w = s_w;
    p.bias = static_cast<const uint16_t *>(bias);
    p.y = static_cast<uint16_t *>(y);
    p.ldy = ldy;
    p.acc_out = acc;
    return acc ? launch_gemv_m<false, true>(plan, p, stream)
               : launch_gemv_m<false, false>(plan, p, stream);
  }
  if (plan.variant == W8A8_VARIANT_GEMV_TC) {
    return acc ? launch_swapab<true>(plan, q, s_a, M, K, Wq, s_w, bias, N, y, ldy, acc, stream)
               : launch_swapab<false>(plan, q, s_a, M, K, Wq, s_w, bias, N, y, ldy, acc, stream);
  }
  if (plan.variant == W8A8_VARIANT_GEMM_PAIR) {
    const SplitRegion split = split_region(plan, split_ws, split_ws_bytes);
    if (!counters_cleared) {
      st = clear_counters(split.counters, split.counters ? split_counter_bytes(plan) : 0, stream);
      if (st != W8A8_OK) return st;
    }
    return acc ? launch_gemm_pair<true, false>(plan, q, s_a, M, K, Wq, s_w, bias, N, y, ldy, acc,
                                               split, nullptr, stream)
               : launch_gemm_pair<false, false>(plan, q, s_a, M, K, Wq, s_w, bias, N, y, ldy, acc,
                                                split, nullptr, stream);
  }
  if (plan.variant == W8A8_VARIANT_GEMM_BN64) {
    return acc ? launch_gemm_t<64, kGemmStages64, true>(plan, q, s_a, M, K, Wq, s_w, bias, N, y,
                                                         ldy, acc, stream)
               : launch_gemm_t<64, kGemmStages64, false>(plan, q, s_a, M, K, Wq, s_w, bias, N,
                                                          y, ldy, acc, stream);
  }
  if (plan.variant == W8A8_VARIANT_GEMM_BN128) {
    return acc ? launch_gemm_t<128, kGemmStages128, true>(plan, q, s_a, M, K, Wq, s_w, bias, N,
                                                           y, ldy, acc, stream)
               : launch_gemm_t<128, kGemmStages128, false>(plan, q, s_a, M, K, Wq, s_w, bias,
                                                            N, y, ldy, acc, stream);
  }
  return acc ? launch_gemm_t<256, kGemmStages256, true>(plan, q, s_a, M, K, Wq, s_w, bias, N, y,
                                                         ldy, acc, stream)
             : launch_gemm_t<256, kGemmStages256, false>(plan, q, s_a, M, K, Wq, s_w, bias, N,
                                                          y, ldy, acc, stream);
}

// ---------------------------------------------------------------- static scratch
// Scratch for w8a8_linear_fused_noalloc: the int8 activations (up to 16 MiB)
// followed by their fp32 row scales (up to 16384 rows) and 4 KiB for the
// fused launch's row-block counters.  In host code the
// array's name only stands in for the device object; its device address is
// looked up once per device with cudaGetSymbolAddress.
constexpr size_t kNoAllocMaxQBytes = static_cast<size_t>(16) << 20;
constexpr int64_t kNoAllocMaxRows = 16384;
constexpr size_t kNoAllocScratchBytes =
    kNoAllocMaxQBytes + static_cast<size_t>(kNoAllocMaxRows) * sizeof(float) + 4096;
static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];

struct NoAllocScratch {
  std::atomic<int> state{0};  // 1 once ptr holds this device's address
  void *ptr = nullptr;
  std::mutex mu;
};
NoAllocScratch g_noalloc[kMaxDevices];

// Device address of the scratch array on the current device (looked up on
// the first call per device).
int noalloc_scratch(void **out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    cudaGetLastError();
    return W8A8_ERR_CUDA;
  }
  NoAllocScratch &s = g_noalloc[dev];
  if (s.state.load(std::memory_order_acquire) != 1) {
    std::lock_guard<std::mutex> lock(s.mu);
    if (s.state.load(std::memory_order_relaxed) != 1) {
      void *p = nullptr;
      if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) {
        cudaGetLastError();
        return W8A8_ERR_CUDA;
      }
      s.ptr = p;
      s.state.store(1, std::memory_order_release);
    }
  }
  *out = s.ptr;
  return W8A8_OK;
}

}  // namespace w8a8

using namespace w8a8;

extern "C" {

const char *w8a8_status_string(int status) {
  switch (status) {
    case W8A8_OK: return "ok";
    case W8A8_ERR_INVALID_ARG: return "invalid argument (null pointer, size < 1 or stride too small)";
    case W8A8_ERR_UNSUPPORTED_SHAPE: return "unsupported shape (need K % 16 == 0, N % 8 == 0, K <= 133144, strides % 8 == 0)";
    case W8A8_ERR_MISALIGNED: return "misaligned pointer (16-byte alignment required)";
    case W8A8_ERR_WORKSPACE: return "workspace missing or too small";
    case W8A8_ERR_CUDA: return "CUDA runtime or driver call failed";
    case W8A8_ERR_DEVICE_TIMEOUT: return "a bounded device-side wait timed out";
    case W8A8_ERR_UNSUPPORTED_DEVICE: return "unsupported device (sm_100 required)";
    default: return "unknown status";
  }
}

const char *w8a8_version(void) { return "w8a8 1.1 sm_100a"; }

int w8a8_bench_mma_i8_peak(int64_t iterations, int32_t pairs, w8a8_stream_t stream) {
  if (iterations < 1 || iterations > 500000 || pairs < 1) return W8A8_ERR_INVALID_ARG;
  const DeviceInfo *d = nullptr;
  int st = query_device(&d);
  if (st != W8A8_OK) return st;
  if (pairs > d->sms / 2) return W8A8_ERR_INVALID_ARG;
  return launch(mma_i8_peak_kernel, dim3(static_cast<unsigned>(2 * pairs)), dim3(kPeakThreads),
                kPeakSmemBytes, reinterpret_cast<cudaStream_t>(stream), iterations);
}

int w8a8_debug_peek_tag(uint64_t *tag) {
  if (!tag) return W8A8_ERR_INVALID_ARG;
  const unsigned long long t = g_tag.load(std::memory_order_relaxed) & ((1ull << 56) - 1);
  *tag = t != 0 ? t : 1;
  return W8A8_OK;
}

int w8a8_quantize_weights(const void *W, int64_t N, int64_t K, int64_t ldw, int8_t *Wq,
                          float *s_w, w8a8_stream_t stream) {
  if (!W || !Wq || !s_w) return W8A8_ERR_INVALID_ARG;
  int st = check_mk(N, K, ldw);
  if (st != W8A8_OK) return st;
  if (!aligned16(W) || !aligned16(Wq) || (reinterpret_cast<uintptr_t>(s_w) & 3u))
    return W8A8_ERR_MISALIGNED;
  const DeviceInfo *d = nullptr;
  st = query_device(&d);
  if (st != W8A8_OK) return st;
  return launch_quant(W, N, K, ldw, Wq, s_w, false, reinterpret_cast<cudaStream_t>(stream));
}

int w8a8_unpack_int32_weights(const int32_t *packed, int64_t N, int64_t K, int8_t *Wq,
                              w8a8_stream_t stream) {
  if (!packed || !Wq) return W8A8_ERR_INVALID_ARG;
  int st = check_mk(N, K, K);
  if (st != W8A8_OK) return st;
  if (!aligned16(packed) || !aligned16(Wq)) return W8A8_ERR_MISALIGNED;
  const DeviceInfo *d = nullptr;
  st = query_device(&d);
  if (st != W8A8_OK) return st;
  const int64_t n16 = N * K / 16;
  const int64_t cap = static_cast<int64_t>(d->sms) * 8;
  const int64_t grid = cdiv(n16, 256) < cap ? cdiv(n16, 256) : cap;
  return launch(unpack_int32_weights_kernel, dim3(static_cast<unsigned>(grid)), dim3(256), 0,
                reinterpret_cast<cudaStream_t>(stream), reinterpret_cast<const uint4 *>(packed),
                reinterpret_cast<uint4 *>(Wq), n16);
}

int w8a8_quant_act(const void *x, int64_t M, int64_t K, int64_t ldx, int8_t *q, float *s_a,
                   w8a8_stream_t stream) {
  if (!x || !q || !s_a) return W8A8_ERR_INVALID_ARG;
  int st = check_mk(M, K, ldx);
  if (st != W8A8_OK) return st;
  if (!aligned16(x) || !aligned16(q) || (reinterpret_cast<uintptr_t>(s_a) & 3u))
    return W8A8_ERR_MISALIGNED;
  const DeviceInfo *d = nullptr;
  st = query_device(&d);
  if (st != W8A8_OK) return st;
  return launch_quant(x, M, K, ldx, q, s_a, true, reinterpret_cast<cudaStream_t>(stream));
}

int w8a8_select(int64_t M, int64_t N, int64_t K, int32_t num_sms, int variant,
                w8a8_plan *plan) {
  if (!plan) return W8A8_ERR_INVALID_ARG;
  int st = check_mk(M, K, K);
  if (st != W8A8_OK) return st;
  st = check_n(N, N);
  if (st != W8A8_OK) return st;
  // B200: 227 KB of opt-in shared memory per block
  return select_plan(M, N, K, num_sms, variant, 232448, plan);
}

int w8a8_workspace_size(int64_t M, int64_t N, int64_t K, size_t *bytes) {
  return w8a8_workspace_size_ex(M, N, K, W8A8_VARIANT_AUTO, bytes);
}

int w8a8_workspace_size_ex(int64_t M, int64_t N, int64_t K, int variant, size_t *bytes) {
  if (!bytes) return W8A8_ERR_INVALID_ARG;
  int st = check_mk(M, K, K);
  if (st != W8A8_OK) return st;
  st = check_n(N, N);
  if (st != W8A8_OK) return st;
  w8a8_plan plan;
  st = select_plan(M, N, K, 148, variant, 232448, &plan);
  if (st != W8A8_OK) return st;
  *bytes = plan.variant == W8A8_VARIANT_GEMV && plan.quant_in_gemm_launch
               ? 0
               : fused_workspace_bytes(M, K) + ready_counter_bytes(M) +
                     split_workspace_bytes(plan);
  return W8A8_OK;
}

int w8a8_linear(const int8_t *q, const float *s_a, int64_t M, int64_t K, const int8_t *Wq,
                const float *s_w, const void *bias, int64_t N, void *y, int64_t ldy,
                int32_t *acc_debug, void *workspace, size_t ws_bytes, w8a8_stream_t stream) {
  return linear_impl(q, s_a, M, K, Wq, s_w, bias, N, y, ldy, acc_debug, W8A8_VARIANT_AUTO,
                     workspace, ws_bytes, false, reinterpret_cast<cudaStream_t>(stream));
}

int w8a8_linear_ex(const int8_t *q, const float *s_a, int64_t M, int64_t K, const int8_t *Wq,
                   const float *s_w, const void *bias, int64_t N, void *y, int64_t ldy,
                   int32_t *acc_debug, int variant, void *workspace, size_t ws_bytes,
                   w8a8_stream_t stream) {
  if (variant < W8A8_VARIANT_AUTO || variant > W8A8_VARIANT_GEMV_TC) return W8A8_ERR_INVALID_ARG;
  return linear_impl(q, s_a, M, K, Wq, s_w, bias, N, y, ldy, acc_debug, variant, workspace,
                     ws_bytes, false, reinterpret_cast<cudaStream_t>(stream));
}

int w8a8_linear_fused(const void *x, int64_t M, int64_t K, int64_t ldx, const int8_t *Wq,
                      const float *s_w, const void *bias, int64_t N, void *y, int64_t ldy,
                      int8_t *q_out, float *s_a_out, void *workspace, size_t ws_bytes,
                      w8a8_stream_t stream_) {
  return w8a8_linear_fused_ex(x, M, K, ldx, Wq, s_w, bias, N, y, ldy, q_out, s_a_out, workspace,
                              ws_bytes, 0, stream_);
}

int w8a8_linear_fused_ex(const void *x, int64_t M, int64_t K, int64_t ldx, const int8_t *Wq,
                         const float *s_w, const void *bias, int64_t N, void *y, int64_t ldy,
                         int8_t *q_out, float *s_a_out, void *workspace, size_t ws_bytes,
                         int options, w8a8_stream_t stream_) {
  if (options & ~W8A8_FUSED_ONE_LAUNCH) return W8A8_ERR_INVALID_ARG;
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  if (!x || !Wq || !s_w || !y) return W8A8_ERR_INVALID_ARG;
  int st = check_mk(M, K, ldx);
  if (st != W8A8_OK) return st;
  st = check_n(N, ldy);
  if (st != W8A8_OK) return st;
  if (!aligned16(x) || !aligned16(Wq) || !aligned16(s_w) || !aligned16(y) ||
      (bias && !aligned16(bias)) || (q_out && !aligned16(q_out)) ||
      (s_a_out && (reinterpret_cast<uintptr_t>(s_a_out) & 3u)))
    return W8A8_ERR_MISALIGNED;
  const DeviceInfo *d = nullptr;
  st = query_device(&d);
  if (st != W8A8_OK) return st;
  w8a8_plan plan;
  st = select_plan(M, N, K, d->sms, W8A8_VARIANT_AUTO, d->max_smem_optin, &plan);
  if (st != W8A8_OK) return st;

  if (plan.variant == W8A8_VARIANT_GEMV && plan.quant_in_gemm_launch) {
    GemvParams p = {};
    p.M = static_cast<int32_t>(M);
    p.N = static_cast<int32_t>(N);
    p.K = static_cast<int32_t>(K);
    p.x = static_cast<const uint16_t *>(x);
    p.ldx = ldx;
    p.wq = Wq;
    p.s_w = s_w;
    p.bias = static_cast<const uint16_t *>(bias);
    p.y = static_cast<uint16_t *>(y);
    p.ldy = ldy;
    p.q_out = q_out;
    p.s_a_out = s_a_out;
    return launch_gemv_m<true, false>(plan, p, stream);
  }

  // workspace layout: [q (M*K) | s_a (M floats) | row-ready counters | K-split region]
  int8_t *q = q_out;
  float *s_a = s_a_out;
  const size_t qs_bytes = fused_workspace_bytes(M, K);
  if (!q || !s_a) {
    if (!workspace || ws_bytes < qs_bytes || !aligned16(workspace)) return W8A8_ERR_WORKSPACE;
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    if (!q) q = reinterpret_cast<int8_t *>(ws);
    if (!s_a) s_a = reinterpret_cast<float *>(ws + align256(static_cast<size_t>(M * K)));
  }
  const size_t head = qs_bytes + ready_counter_bytes(M);
  const bool have_ready = workspace && aligned16(workspace) && ws_bytes >= head;
  void *split_ws = nullptr;
  size_t split_bytes = 0;
  if (have_ready && ws_bytes > head) {
    split_ws = static_cast<uint8_t *>(workspace) + head;
    split_bytes = ws_bytes - head;
  }
  // One launch on request.  Its row-block counters are cleared on the stream
  // before the launch (a captured graph clears them on every replay).
  if ((options & W8A8_FUSED_ONE_LAUNCH) && plan.variant == W8A8_VARIANT_GEMM_PAIR &&
      plan.quant_in_gemm_launch && have_ready) {
    // one launch: the pair kernel quantizes x itself, its producers waiting
    // only for the 128-row blocks they load
    FuseArgs f;
    f.x = x;
    f.ldx = ldx;
    f.row_ready = reinterpret_cast<unsigned long long *>(static_cast<uint8_t *>(workspace) +
                                                         qs_bytes);
    const SplitRegion split = split_region(plan, split_ws, split_bytes);
    st = clear_counters(f.row_ready, ready_counter_bytes(M), stream);
    if (st != W8A8_OK) return st;
    st = clear_counters(split.counters, split.counters ? split_counter_bytes(plan) : 0, stream);
    if (st != W8A8_OK) return st;
    return launch_gemm_pair<false, true>(plan, q, s_a, M, K, Wq, s_w, bias, N, y, ldy, nullptr,
                                         split, &f, stream);
  }
  // the K-split counters are cleared before the quantization kernel, so
  // that the GEMM stays its programmatic dependent
  if (plan.variant == W8A8_VARIANT_GEMM_PAIR) {
    const SplitRegion split = split_region(plan, split_ws, split_bytes);
    st = clear_counters(split.counters, split.counters ? split_counter_bytes(plan) : 0, stream);
    if (st != W8A8_OK) return st;
  }
  st = launch_quant(x, M, K, ldx, q, s_a, true, stream);
  if (st != W8A8_OK) return st;
  return linear_impl(q, s_a, M, K, Wq, s_w, bias, N, y, ldy, nullptr, plan.variant, split_ws,
                     split_bytes, true, stream);
}

int w8a8_linear_fused_noalloc(const void *x, int64_t M, int64_t K, int64_t ldx, const int8_t *Wq,
                              const float *s_w, const void *bias, int64_t N, void *y, int64_t ldy,
                              w8a8_stream_t stream) {
  if (!x || !Wq || !s_w || !y) return W8A8_ERR_INVALID_ARG;
  int st = check_mk(M, K, ldx);
  if (st != W8A8_OK) return st;
  st = check_n(N, ldy);
  if (st != W8A8_OK) return st;
  if (M > kNoAllocMaxRows || M * K > static_cast<int64_t>(kNoAllocMaxQBytes))
    return W8A8_ERR_WORKSPACE;  // beyond the static scratch limits
  const DeviceInfo *d = nullptr;
  st = query_device(&d);
  if (st != W8A8_OK) return st;
  void *scratch = nullptr;
  st = noalloc_scratch(&scratch);
  if (st != W8A8_OK) return st;
  return w8a8_linear_fused(x, M, K, ldx, Wq, s_w, bias, N, y, ldy, nullptr, nullptr, scratch,
                           kNoAllocScratchBytes, stream);
}

// The end-to-end call splits the rows into up to kHostChunks chunks: chunk
// c's copy in (on the caller's stream), its layer (on an internal stream) and
// its copy out (on another) overlap the other chunks' work, so the copies in
// and out -- PCIe carries both directions at once -- run side by side with
// the layer.  Every output depends on its own row only, so the result is the
// same as one call over all rows.  The internal streams and events are made
// once per device and reused; a mutex orders the calls that enqueue on them.
constexpr int kHostChunks = 8;
constexpr int64_t kHostChunkMinRows = 256;

struct HostPipe {
  std::mutex mu;
  bool ready = false;
  cudaStream_t compute = nullptr, d2h = nullptr;
  cudaEvent_t fork = nullptr, done = nullptr;
  cudaEvent_t in[kHostChunks] = {}, out[kHostChunks] = {};
};
HostPipe g_pipe[kMaxDevices];

int host_pipe_ready(HostPipe &hp) {
  if (hp.ready) return W8A8_OK;
  bool ok = cudaStreamCreateWithFlags(&hp.compute, cudaStreamNonBlocking) == cudaSuccess &&
            cudaStreamCreateWithFlags(&hp.d2h, cudaStreamNonBlocking) == cudaSuccess &&
            cudaEventCreateWithFlags(&hp.fork, cudaEventDisableTiming) == cudaSuccess &&
            cudaEventCreateWithFlags(&hp.done, cudaEventDisableTiming) == cudaSuccess;
  for (int c = 0; ok && c < kHostChunks; ++c)
    ok = cudaEventCreateWithFlags(&hp.in[c], cudaEventDisableTiming) == cudaSuccess &&
         cudaEventCreateWithFlags(&hp.out[c], cudaEventDisableTiming) == cudaSuccess;
  if (!ok) {
    cudaGetLastError();
    return W8A8_ERR_CUDA;
  }
  hp.ready = true;
  return W8A8_OK;
}

int w8a8_linear_fused_host(const void *x_host, int64_t M, int64_t K, const int8_t *Wq,
                           const float *s_w, const void *bias, int64_t N, void *y_host,
                           void *x_dev, void *y_dev, void *workspace, size_t ws_bytes,
                           w8a8_stream_t stream_) {
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  if (!x_host || !y_host || !x_dev || !y_dev) return W8A8_ERR_INVALID_ARG;
  int st = check_mk(M, K, K);
  if (st != W8A8_OK) return st;
  st = check_n(N, N);
  if (st != W8A8_OK) return st;
  const DeviceInfo *d = nullptr;
  st = query_device(&d);
  if (st != W8A8_OK) return st;
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    cudaGetLastError();
    return W8A8_ERR_CUDA;
  }
  HostPipe &hp = g_pipe[dev];
  std::lock_guard<std::mutex> lock(hp.mu);
  st = host_pipe_ready(hp);
  if (st != W8A8_OK) return st;
  // chunks of at least kHostChunkMinRows rows, a multiple of 128
  int64_t rows_per = cdiv(M, kHostChunks);
  if (rows_per < kHostChunkMinRows) rows_per = kHostChunkMinRows;
  rows_per = cdiv(rows_per, 128) * 128;
  const int64_t nch = cdiv(M, rows_per);  // <= kHostChunks
  const uint8_t *xh = static_cast<const uint8_t *>(x_host);
  uint8_t *yh = static_cast<uint8_t *>(y_host);
  uint8_t *xd = static_cast<uint8_t *>(x_dev);
  uint8_t *yd = static_cast<uint8_t *>(y_dev);
  // fork: the internal streams start after the work already on `stream`
  bool cuda_ok = cudaEventRecord(hp.fork, stream) == cudaSuccess &&
                 cudaStreamWaitEvent(hp.compute, hp.fork, 0) == cudaSuccess &&
                 cudaStreamWaitEvent(hp.d2h, hp.fork, 0) == cudaSuccess;
  st = W8A8_OK;
  for (int64_t c = 0; cuda_ok && st == W8A8_OK && c < nch; ++c) {
    const int64_t r0 = c * rows_per;
    const int64_t rows = M - r0 < rows_per ? M - r0 : rows_per;
    const size_t xoff = static_cast<size_t>(r0 * K) * 2, xbytes = static_cast<size_t>(rows * K) * 2;
    const size_t yoff = static_cast<size_t>(r0 * N) * 2, ybytes = static_cast<size_t>(rows * N) * 2;
    cuda_ok = cudaMemcpyAsync(xd + xoff, xh + xoff, xbytes, cudaMemcpyHostToDevice, stream) ==
                  cudaSuccess &&
              cudaEventRecord(hp.in[c], stream) == cudaSuccess &&
              cudaStreamWaitEvent(hp.compute, hp.in[c], 0) == cudaSuccess;
    if (!cuda_ok) break;
    st = w8a8_linear_fused(xd + xoff, rows, K, K, Wq, s_w, bias, N, yd + yoff, N, nullptr, nullptr,
                           workspace, ws_bytes, reinterpret_cast<w8a8_stream_t>(hp.compute));
    if (st != W8A8_OK) break;
    cuda_ok = cudaEventRecord(hp.out[c], hp.compute) == cudaSuccess &&
              cudaStreamWaitEvent(hp.d2h, hp.out[c], 0) == cudaSuccess &&
              cudaMemcpyAsync(yh + yoff, yd + yoff, ybytes, cudaMemcpyDeviceToHost, hp.d2h) ==
                  cudaSuccess;
  }
  // join: `stream` continues once the last copy out (and, through the
  // events, every chunk's layer) is done -- also after an error, so that
  // the streams stay ordered
  const bool joined = cudaEventRecord(hp.out[0], hp.compute) == cudaSuccess &&
                      cudaStreamWaitEvent(hp.d2h, hp.out[0], 0) == cudaSuccess &&
                      cudaEventRecord(hp.done, hp.d2h) == cudaSuccess &&
                      cudaStreamWaitEvent(stream, hp.done, 0) == cudaSuccess;
  if (!cuda_ok || !joined) {
    cudaGetLastError();
    return W8A8_ERR_CUDA;
  }
  return st;
}

int w8a16_linear(const void *x, int64_t M, int64_t K, int64_t ldx, const int8_t *Wq,
                 const float *s_w, const void *bias, int64_t N, void *y, int64_t ldy,
                 w8a8_stream_t stream) {
  if (!x || !Wq || !s_w || !y) return W8A8_ERR_INVALID_ARG;
  int st = check_mk(M, K, ldx);
  if (st != W8A8_OK) return st;
  st = check_n(N, ldy);
  if (st != W8A8_OK) return st;
  if (!aligned16(x) || !aligned16(Wq) || !aligned16(s_w) || !aligned16(y) ||
      (bias && !aligned16(bias)))
    return W8A8_ERR_MISALIGNED;
  const DeviceInfo *d = nullptr;
  st = query_device(&d);
  if (st != W8A8_OK) return st;
  using L = WtLayout;
  CUtensorMap mx, mw;
  st = encode_bf16_load_map(&mx, x, M, K, ldx, kWtBN);
  if (st != W8A8_OK) return st;
  st = encode_i8_sw64_map(&mw, Wq, N, K, kBM);
  if (st != W8A8_OK) return st;
  WtParams p;
  std::memset(&p, 0, sizeof(p));
  p.M = static_cast<int32_t>(M);
  p.N = static_cast<int32_t>(N);
  p.K = static_cast<int32_t>(K);
  p.num_n_blk = static_cast<int32_t>(cdiv(N, kBM));
  p.num_m_blk = static_cast<int32_t>(cdiv(M, kWtBN));
  const int64_t tiles = static_cast<int64_t>(p.num_m_blk) * p.num_n_blk;
  if (tiles > INT32_MAX) return W8A8_ERR_UNSUPPORTED_SHAPE;
  p.num_tiles = static_cast<int32_t>(tiles);
  p.k_blocks = static_cast<int32_t>(cdiv(K, kWtBK));
  p.s_w = s_w;
  p.bias = static_cast<const uint16_t *>(bias);
  p.y = static_cast<uint16_t *>(y);
  p.ldy = ldy;
  constexpr auto kernel = gemm_w8a16_tmem_kernel;
  st = ensure_smem_limit<kernel>(L::kSmemBytes);
  if (st != W8A8_OK) return st;
  const int64_t grid = tiles < d->sms ? tiles : d->sms;
  return launch_ex(true, kernel, dim3(static_cast<unsigned>(grid)), dim3(kWtThreads),
                   L::kSmemBytes, reinterpret_cast<cudaStream_t>(stream), mx, mw, p);
}

int w8a8_last_device_error(w8a8_stream_t stream) {
  if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess) {
    cudaGetLastError();
    return W8A8_ERR_CUDA;
  }
  unsigned int word = 0, zero = 0;
  if (cudaMemcpyFromSymbol(&word, g_device_error, sizeof(word)) != cudaSuccess ||
      cudaMemcpyToSymbol(g_device_error, &zero, sizeof(zero)) != cudaSuccess) {
    cudaGetLastError();
    return W8A8_ERR_CUDA;
  }
  return (word & W8A8_DEVERR_TIMEOUT) ? W8A8_ERR_DEVICE_TIMEOUT : W8A8_OK;
}

int w8a8_selftest_quant_exhaustive(unsigned long long *counts_dev, w8a8_stream_t stream_) {
  if (!counts_dev) return W8A8_ERR_INVALID_ARG;
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  const DeviceInfo *d = nullptr;
  int st = query_device(&d);
  if (st != W8A8_OK) return st;
  if (cudaMemsetAsync(counts_dev, 0, 2 * sizeof(unsigned long long), stream) != cudaSuccess) {
    cudaGetLastError();
    return W8A8_ERR_CUDA;
  }
  return launch(quant_exhaustive_kernel, dim3(0x7F7F), dim3(256), 0, stream, counts_dev);
}

int w8a8_selftest_bounded_wait(int64_t limit_ns, w8a8_stream_t stream) {
  if (limit_ns < 1000 || limit_ns > 10000000000LL) return W8A8_ERR_INVALID_ARG;
  const DeviceInfo *d = nullptr;
  int st = query_device(&d);
  if (st != W8A8_OK) return st;
  return launch(bounded_wait_selftest_kernel, dim3(1), dim3(32), 0,
                reinterpret_cast<cudaStream_t>(stream), static_cast<uint64_t>(limit_ns));
}

}  // extern "C"
