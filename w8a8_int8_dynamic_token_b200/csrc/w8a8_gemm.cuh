// w8a8_gemm.cuh -- int8 x int8 -> int32 GEMM on the sm_100a tensor cores
// (tcgen05.mma kind::i8) with the dequantization epilogue fused:
//
//   acc[m,n] = sum_k q[m,k] * Wq[n,k]                         (exact int32)
//   y[m,n]   = bf16_rne( ((float)acc * s_a[m]) * s_w[n] + (float)bias[n] )
//
// This is the "int8 scaled matmul" step of the W8A8 int8-dynamic layer
// ("Issue 5 probe: int8 quantized DiT serve paths on the RTX 3090 (24 GB)",
// section "Round two ... W8A8 int8-dynamic": the cutlass int8 scaled-MM; "Qwen-
// Image-2.1: TE AutoRound-AWQ on GPU + all-resident single-3090 stack",
// section "Whole-pipeline follow-up": int8 GEMMs with per-token / per-channel
// scales).  The epilogue keeps the x s_a factor the "Round two" section singles
// out, and evaluates it as separately rounded fp32 operations in a fixed order.
//
// Structure (one CTA per SM, persistent over output tiles of 128 x BN):
//   warp 0      one thread issues TMA tile loads of q and Wq (128-byte swizzle,
//               K-major, 128 int8 of K per stage) into a STAGES-deep ring;
//   warp 1      allocates TMEM and one thread issues tcgen05.mma (M=128, N=BN,
//               K=32 per instruction) into one of two TMEM accumulators, then
//               commits to the ring's "empty" barriers and the accumulator's
//               "full" barrier;
//   warps 2..5  the epilogue: tcgen05.ld of the accumulator (each warp owns
//               the 32 TMEM lanes = rows its warp index selects), the fp32
//               scale/bias math, bf16 packing and 16-byte stores; then they
//               release the accumulator so the next tile's MMAs overlap them.
// Ragged edges: TMA zero-fills rows/columns outside the tensors (zeros add
// nothing to an integer dot product); the epilogue masks its stores.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cstdint>

#include "w8a8_ptx.cuh"

namespace w8a8 {

constexpr int kGemmThreads = 192;
constexpr int kBM = 128;   // rows of y per tile (TMEM lanes)
constexpr int kBK = 128;   // int8 K elements per stage = one 128-byte swizzle row
constexpr int kMmaK = 32;  // K per tcgen05.mma kind::i8

template <int BN, int STAGES>
struct GemmLayout {
  static constexpr int kABytes = kBM * kBK;
  static constexpr int kBBytes = BN * kBK;
  static constexpr int kStageBytes = kABytes + kBBytes;
  static constexpr int kTileBytes = STAGES * kStageBytes;
  // full[STAGES], empty[STAGES], tfull[2], tempty[2], drain, then two words
  static constexpr int kBarBytes = (2 * STAGES + 5) * 8 + 8;
  static constexpr int kSmemBytes = kTileBytes + kBarBytes + 1024;  // + alignment slack
  static constexpr int kTmemCols = 2 * BN;                          // two accumulators
};

struct GemmParams {
  int32_t M, N, K;
  int32_t num_m_blk, num_n_blk, num_tiles, k_blocks, group_m;
  const float *s_a;
  const float *s_w;
  const uint16_t *bias;  // bf16 bits or nullptr
  uint16_t *y;           // bf16 bits
  int64_t ldy;
  int32_t *acc_out;      // raw int32 [M, N] dense (debug variant)
};

// Tile t -> (row block, column block).  Row blocks are walked in bands of
// group_m so the tiles in flight at one time share their q and Wq slices in L2.
__device__ __forceinline__ void gemm_tile_coords(int t, const GemmParams &p, int &mb, int &nb) {
  const int band = p.group_m * p.num_n_blk;
  const int g = t / band;
  const int first_m = g * p.group_m;
  const int rows_in_band = min(p.num_m_blk - first_m, p.group_m);
  const int r = t - g * band;
  mb = first_m + r % rows_in_band;
  nb = r / rows_in_band;
}

// Wait without looking at the abort flag (used to drain work in flight after
// an abort).  Bounded like every other wait.
__device__ __forceinline__ bool mbar_wait_drain(uint64_t *bar, uint32_t parity) {
  volatile int never = 0;
  return mbar_wait(bar, parity, &never, kWaitLimitNs);
}

template <int BN, int STAGES, bool RAW_OUT>
__global__ void __launch_bounds__(kGemmThreads, 1)
    gemm_i8_tcgen05_kernel(const __grid_constant__ CUtensorMap tmap_a,
                           const __grid_constant__ CUtensorMap tmap_b, const GemmParams p) {
  using L = GemmLayout<BN, STAGES>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_addr(smem_raw);
  uint8_t *smem = smem_raw + ((1024u - (raw_addr & 1023u)) & 1023u);
  uint64_t *full = reinterpret_cast<uint64_t *>(smem + L::kTileBytes);
  uint64_t *empty = full + STAGES;
  uint64_t *tfull = empty + STAGES;
  uint64_t *tempty = tfull + 2;
  uint64_t *drain = tempty + 2;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(drain + 1);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 4);  // one arrival per epilogue warp
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbarrier_init();
    tma_prefetch_desc(&tmap_a);
    tma_prefetch_desc(&tmap_b);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, L::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued = 0;
      bool ok = true;
      for (int t = blockIdx.x; ok && t < p.num_tiles; t += gridDim.x) {
        int mb, nb;
        gemm_tile_coords(t, p, mb, nb);
        for (int kb = 0; kb < p.k_blocks; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag)) {
            ok = false;
            break;
          }
          uint8_t *sa = smem + stage * L::kStageBytes;
          uint8_t *sb = sa + L::kABytes;
          mbar_arrive_expect_tx(&full[stage], L::kStageBytes);
          tma_load_2d(&tmap_a, &full[stage], sa, kb * kBK, mb * kBM);
          tma_load_2d(&tmap_b, &full[stage], sb, kb * kBK, nb * BN);
          ++issued;
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (!ok) {
        // let the last loads land before the block's shared memory goes away
        const uint32_t n = issued < static_cast<uint32_t>(STAGES) ? issued : STAGES;
        for (uint32_t i = issued - n; i < issued; ++i)
          mbar_wait_drain(&full[i % STAGES], (i / STAGES) & 1u);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_i8(kBM, BN);
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      bool any_mma = false;
      for (int t = blockIdx.x; ok && t < p.num_tiles; t += gridDim.x) {
        if (!mbar_wait(&tempty[acc], acc_phase ^ 1u, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * BN);
        for (int kb = 0; kb < p.k_blocks; ++kb) {
          if (!mbar_wait(&full[stage], phase, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sa = smem_addr(smem + stage * L::kStageBytes);
          const uint64_t adesc = smem_desc_k_sw128(sa);
          const uint64_t bdesc = smem_desc_k_sw128(sa + L::kABytes);
#pragma unroll
          for (int k = 0; k < kBK / kMmaK; ++k) {
            // +32 bytes along K inside the swizzled row = +2 in the address field
            mma_i8(d_tmem, adesc + 2u * k, bdesc + 2u * k, idesc, (kb | k) != 0 ? 1u : 0u);
          }
          any_mma = true;
          mma_commit(&empty[stage]);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        mma_commit(&tfull[acc]);
        if (++acc == 2) {
          acc = 0;
          acc_phase ^= 1u;
        }
      }
      if (!ok && any_mma) {
        // no tensor-core work may still be writing TMEM when it is freed
        mma_commit(drain);
        mbar_wait_drain(drain, 0);
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int quarter = warp & 3;  // TMEM lanes 32*quarter .. +31 = tile rows
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int t = blockIdx.x; t < p.num_tiles; t += gridDim.x) {
      int mb, nb;
      gemm_tile_coords(t, p, mb, nb);
      int ok = 1;
      if (lane == 0) ok = mbar_wait(&tfull[acc], acc_phase, abort_flag) ? 1 : 0;
      ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
      if (!ok) break;
      tc_fence_after();

      const int row = mb * kBM + quarter * 32 + lane;
      const bool row_ok = row < p.M;
      const float sa = row_ok ? __ldg(p.s_a + row) : 0.0f;
      const uint32_t t_row = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) +
                             static_cast<uint32_t>(acc * BN);
#pragma unroll 1
      for (int c = 0; c < BN; c += 32) {
        uint32_t r[32];
        tmem_ld_32x32b_x32(t_row + c, r);
        tmem_ld_wait();
        const int col0 = nb * BN + c;
        if constexpr (RAW_OUT) {
          if (row_ok) {
            int32_t *dst = p.acc_out + static_cast<int64_t>(row) * p.N + col0;
#pragma unroll
            for (int g = 0; g < 8; ++g) {
              if (col0 + 4 * g < p.N) {
                reinterpret_cast<uint4 *>(dst)[g] =
                    make_uint4(r[4 * g], r[4 * g + 1], r[4 * g + 2], r[4 * g + 3]);
              }
            }
          }
        } else {
          uint16_t *dst = p.y + static_cast<int64_t>(row) * p.ldy + col0;
#pragma unroll
          for (int g = 0; g < 4; ++g) {  // 8 columns per group; N % 8 == 0
            const int cg = col0 + 8 * g;
            if (cg >= p.N) break;
            const float4 w0 = __ldg(reinterpret_cast<const float4 *>(p.s_w + cg));
            const float4 w1 = __ldg(reinterpret_cast<const float4 *>(p.s_w + cg) + 1);
            const float sw[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
            float bb[8];
            if (p.bias != nullptr) {
              const uint4 braw = __ldg(reinterpret_cast<const uint4 *>(p.bias + cg));
              const uint32_t bw[4] = {braw.x, braw.y, braw.z, braw.w};
#pragma unroll
              for (int i = 0; i < 4; ++i) {
                bb[2 * i] = __uint_as_float(bw[i] << 16);
                bb[2 * i + 1] = __uint_as_float(bw[i] & 0xFFFF0000u);
              }
            }
            uint32_t packed[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              float v0 = __int2float_rn(static_cast<int32_t>(r[8 * g + 2 * i]));
              float v1 = __int2float_rn(static_cast<int32_t>(r[8 * g + 2 * i + 1]));
              v0 = __fmul_rn(__fmul_rn(v0, sa), sw[2 * i]);
              v1 = __fmul_rn(__fmul_rn(v1, sa), sw[2 * i + 1]);
              if (p.bias != nullptr) {
                v0 = __fadd_rn(v0, bb[2 * i]);
                v1 = __fadd_rn(v1, bb[2 * i + 1]);
              }
              const __nv_bfloat162 h = __floats2bfloat162_rn(v0, v1);
              packed[i] = *reinterpret_cast<const uint32_t *>(&h);
            }
            if (row_ok) {
              reinterpret_cast<uint4 *>(dst)[g] =
                  make_uint4(packed[0], packed[1], packed[2], packed[3]);
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty[acc]);
      if (++acc == 2) {
        acc = 0;
        acc_phase ^= 1u;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, L::kTmemCols);
  }
}

}  // namespace w8a8
