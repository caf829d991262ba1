// w8a8_swapab.cuh -- the W8A8 layer for few activation rows (M <= 128) on
// the tensor cores, with the roles of the operands swapped.
//
// At small M the layer is a stream of the int8 weight matrix from HBM (the
// AdaLN modulation and conditioning linears at M = batch; unsloth commit
// history of test_diffusion_transformer_quant.py, the commit on torch._int_mm
// requiring more than 16 rows).  A tcgen05 MMA needs M = 128 rows on its A
// side, so the weights take that side: each CTA owns 128 rows of Wq (128
// output columns of y) and computes the transposed tile
//     D[n, m] = sum_k Wq[n, k] * q[m, k]        (exact int32, in TMEM)
// with N = MPAD >= M activation rows (16, 32, 64 or 128; rows past M are
// zero-filled by the tensor-memory-accelerator load).  With few tiles the K
// range is split among the CTAs of a cluster (up to 8); the partial int32
// sums are added exactly in the first CTA's shared memory (distributed
// shared memory stores, no global workspace), which then runs the epilogue
//     y[m, n] = bf16_rne( ((float)acc * s_a[m]) * s_w[n] + (float)bias[n] ).
//
// Warp roles: warps 0 and 6 producers (TMA loads of the Wq box and the q box
// of each 128-deep k-block into a STAGES-deep ring, alternate k-blocks each;
// the first ring of Wq boxes is issued before the programmatic-dependency
// wait, since the weights do not depend on the preceding kernel), warp 1 TMEM
// allocation and the single MMA thread, warps 2..5 the epilogue (one TMEM
// lane quarter each: lane = weight row n, column = activation row m).  Every
// wait is bounded.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cstdint>

#include "w8a8_gemm.cuh"
#include "w8a8_ptx.cuh"

namespace w8a8 {

constexpr int kSwThreads = 224;  // 7 warps
constexpr int kSwLoadWarp2 = 6;  // the second load-issuing warp
constexpr int kSwMaxSplit = 8;   // CTAs of a cluster sharing one tile along K

template <int MPAD>
struct SwapLayout {
  static constexpr int kStages = MPAD <= 32 ? 8 : (MPAD == 64 ? 6 : 4);
  static constexpr int kABytes = kBM * kBK;    // 128 weight rows x 128 bytes of K
  static constexpr int kBBytes = MPAD * kBK;   // MPAD activation rows x 128 bytes
  static constexpr int kStageBytes = kABytes + kBBytes;
  static constexpr int kRingBytes = kStages * kStageBytes;
  // partial sums of the other CTAs of the cluster land in the first CTA's
  // ring once every MMA of the cluster has completed: [rank - 1][row][MPAD]
  static constexpr int kPartialBytes = kBM * MPAD * 4;
  static constexpr int kMaxSplit =
      1 + (kRingBytes / kPartialBytes < kSwMaxSplit - 1 ? kRingBytes / kPartialBytes
                                                         : kSwMaxSplit - 1);
  static constexpr int kBarOffset = kRingBytes;  // 1024-aligned
  static constexpr int kBarBytes = (2 * kStages + 2) * 8 + 8;
  static constexpr int kSmemBytes = kBarOffset + kBarBytes + 1024;
  static constexpr int kTmemCols = MPAD < 32 ? 32 : MPAD;
  static_assert(kSmemBytes <= 232448, "shared memory budget");
  static_assert(kStages % 2 == 0, "the two load threads own alternate stages");
};

struct SwapParams {
  int32_t M, N, K;
  int32_t k_blocks;       // cdiv(K, 128)
  int32_t split;          // CTAs of a cluster along K (the cluster size)
  const float *s_a;
  const float *s_w;
  const uint16_t *bias;   // bf16 bits or nullptr
  uint16_t *y;            // bf16 [M, N], row stride ldy
  int64_t ldy;
  int32_t *acc_out;       // raw int32 [M, N] dense instead of y (debug), or nullptr
};

// Store 16 bytes into the shared memory of CTA `rank` of the cluster, at the
// address that `local` has in this CTA.
__device__ __forceinline__ void st_cluster_v4(uint32_t local, uint32_t rank, uint4 v) {
  const uint32_t remote = map_to_cta(local, rank);
  asm volatile("st.shared::cluster.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(remote), "r"(v.x),
               "r"(v.y), "r"(v.z), "r"(v.w)
               : "memory");
}

// The epilogue of both kernels (warps 2..5, TMEM lane quarter warp & 3, i.e.
// 32 weight rows n of the tile each), after the MMAs of every CTA of the
// cluster: the other CTAs store their int32 partial sums into the first
// CTA's idle ring (distributed shared memory), which adds them exactly and
// writes y[m, n] = bf16_rne(((float)acc * s_a[m]) * s_w[n] + (float)bias[n]).
// s_a: the row scales, written by the preceding kernel.  All threads of the
// CTA call it.
template <int MPAD, bool RAW_OUT>
__device__ __forceinline__ void swap_epilogue(const SwapParams &p, uint32_t tmem_base,
                                              uint64_t *tfull, volatile int *abort_flag,
                                              uint8_t *ring, int warp, int lane, int tile,
                                              int rank, int split, const float *s_a) {
  const bool epi = warp >= 2 && warp < 6;
  const int quarter = warp & 3;
  const int row_local = quarter * 32 + lane;          // 0..127 within the tile
  const int n = tile * kBM + row_local;
  int ok = 1;
  if (epi) {
    ok = mbar_wait(tfull, 0u, abort_flag) ? 1 : 0;
    tc_fence_after();
  }
  // every CTA's MMAs have completed: the first CTA's ring may take partials
  __syncwarp();
  if (split > 1) cluster_sync();
  const uint32_t t_row = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16);
  uint8_t *partials = ring;  // [rank - 1][row_local][MPAD] int32, in the first CTA
  // columns per TMEM load: 32, or MPAD when it is 16 (32 are allocated)
  constexpr int CW = MPAD < 32 ? MPAD : 32;
  if (split > 1 && epi && rank > 0 && ok) {
#pragma unroll 1
    for (int c = 0; c < MPAD; c += CW) {
      uint32_t r[32];
      tmem_ld_32x32b_x32(t_row + c, r);
      tmem_ld_wait();
      const uint32_t base = smem_addr(partials + (static_cast<size_t>(rank - 1) * kBM + row_local) *
                                                     MPAD * 4 + c * 4);
#pragma unroll
      for (int g = 0; g < CW / 4; ++g)
        st_cluster_v4(base + 16u * g, 0u,
                      make_uint4(r[4 * g], r[4 * g + 1], r[4 * g + 2], r[4 * g + 3]));
    }
  }
  if (split > 1) cluster_sync();  // partials visible in the first CTA
  if (epi && rank == 0 && ok) {
    grid_dependency_wait();  // s_a comes from the preceding kernel
    const bool n_ok = n < p.N;
    const float sw = n_ok ? __ldg(p.s_w + n) : 0.0f;
    const float bv = (n_ok && p.bias != nullptr)
                         ? __uint_as_float(static_cast<uint32_t>(__ldg(p.bias + n)) << 16)
                         : 0.0f;
#pragma unroll 1
    for (int c = 0; c < MPAD; c += CW) {
      uint32_t r[32];
      tmem_ld_32x32b_x32(t_row + c, r);
      tmem_ld_wait();
      for (int j = 1; j < split; ++j) {
        const uint4 *src = reinterpret_cast<const uint4 *>(
            partials + (static_cast<size_t>(j - 1) * kBM + row_local) * MPAD * 4 + c * 4);
#pragma unroll
        for (int g = 0; g < CW / 4; ++g) {
          const uint4 a = src[g];
          r[4 * g] += a.x; r[4 * g + 1] += a.y; r[4 * g + 2] += a.z; r[4 * g + 3] += a.w;
        }
      }
      if (!n_ok) continue;
#pragma unroll
      for (int j = 0; j < CW; ++j) {
        const int m = c + j;
        if (m >= p.M) break;
        if constexpr (RAW_OUT) {
          p.acc_out[static_cast<int64_t>(m) * p.N + n] = static_cast<int32_t>(r[j]);
        } else {
          float v = __int2float_rn(static_cast<int32_t>(r[j]));
          v = __fmul_rn(__fmul_rn(v, __ldcg(s_a + m)), sw);
          if (p.bias != nullptr) v = __fadd_rn(v, bv);
          const __nv_bfloat16 h = __float2bfloat16_rn(v);
          p.y[static_cast<int64_t>(m) * p.ldy + n] = *reinterpret_cast<const uint16_t *>(&h);
        }
      }
    }
  }
}

template <int MPAD, bool RAW_OUT>
__global__ void __launch_bounds__(kSwThreads, 1)
    gemm_i8_swapab_kernel(const __grid_constant__ CUtensorMap tmap_w,
                          const __grid_constant__ CUtensorMap tmap_q, const SwapParams p) {
  using L = SwapLayout<MPAD>;
  constexpr int S = L::kStages;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_addr(smem_raw);
  uint8_t *smem = smem_raw + ((1024u - (raw_addr & 1023u)) & 1023u);
  uint64_t *full = reinterpret_cast<uint64_t *>(smem + L::kBarOffset);
  uint64_t *empty = full + S;
  uint64_t *tfull = empty + S;
  uint64_t *drain = tfull + 1;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(drain + 1);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int split = p.split;
  const int rank = static_cast<int>(blockIdx.x) % split;  // == cluster rank
  const int tile = static_cast<int>(blockIdx.x) / split;
  // this CTA's k-blocks: an even share, the first (k_blocks % split) CTAs one more
  const int per = p.k_blocks / split, extra = p.k_blocks % split;
  const int kb0 = rank * per + (rank < extra ? rank : extra);
  const int kb1 = kb0 + per + (rank < extra ? 1 : 0);

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(tfull, 1);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbarrier_init();
    tma_prefetch_desc(&tmap_w);
    tma_prefetch_desc(&tmap_q);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, L::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0 || warp == kSwLoadWarp2) {
    // ------------------------------------------------------------ producers
    // Two threads issue the loads, thread u the k-blocks i with i % 2 == u
    // (so each owns every other stage of the even-sized ring): one thread
    // waiting on each stage before refilling it sustains about half the TMA
    // box throughput per SM that two do.
    if (lane == 0) {
      const int u = warp == 0 ? 0 : 1;
      const int nkb = kb1 - kb0;
      const int pre = nkb < S ? nkb : S;
      for (int i = u; i < pre; i += 2) {
        mbar_arrive_expect_tx(&full[i], L::kStageBytes);
        tma_load_2d(&tmap_w, &full[i], smem + i * L::kStageBytes, (kb0 + i) * kBK, tile * kBM);
      }
      grid_dependency_wait();  // q is written by the preceding kernel
      int last = 0;            // one past the last k-block this thread issued
      for (int i = u; i < nkb; i += 2) {
        const int stage = i % S;
        uint8_t *sa = smem + stage * L::kStageBytes;
        if (i >= S) {
          if (!mbar_wait(&empty[stage], static_cast<uint32_t>((i / S) & 1) ^ 1u, abort_flag)) break;
          mbar_arrive_expect_tx(&full[stage], L::kStageBytes);
          tma_load_2d(&tmap_w, &full[stage], sa, (kb0 + i) * kBK, tile * kBM);
        }
        tma_load_2d(&tmap_q, &full[stage], sa + L::kABytes, (kb0 + i) * kBK, 0);
        last = i + 1;
      }
      if (u == 0) grid_dependents_launch();
      // every load this thread issued has been consumed by an MMA (or, after
      // an abort, is waited for here) before the CTA leaves
      for (int i = (last > S ? last - S : 0); i < last; ++i) {
        if ((i & 1) != u) continue;
        volatile int never = 0;
        mbar_wait(&full[i % S], static_cast<uint32_t>((i / S) & 1), &never);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_i8(kBM, MPAD);
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true, any = false;
      for (int kb = kb0; kb < kb1; ++kb) {
        if (!mbar_wait(&full[stage], phase, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t sa = smem_addr(smem + stage * L::kStageBytes);
        const uint64_t adesc = smem_desc_k_sw128(sa);
        const uint64_t bdesc = smem_desc_k_sw128(sa + L::kABytes);
#pragma unroll
        for (int k = 0; k < kBK / kMmaK; ++k)
          mma_i8(tmem_base, adesc + 2u * k, bdesc + 2u * k, idesc, (kb != kb0 || k != 0) ? 1u : 0u);
        any = true;
        mma_commit(&empty[stage]);
        if (++stage == S) {
          stage = 0;
          phase ^= 1u;
        }
      }
      if (ok) {
        mma_commit(tfull);  // arrives once every MMA above has completed
      } else if (any) {
        mma_commit(drain);
        volatile int never = 0;
        mbar_wait(drain, 0u, &never);
      }
    }
  }

  // ---------------------------------------------------------------- epilogue
  swap_epilogue<MPAD, RAW_OUT>(p, tmem_base, tfull, abort_flag, smem, warp, lane, tile, rank, split,
                               p.s_a);
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, L::kTmemCols);
  }
}

}  // namespace w8a8
