// w8a16_gemm.cuh -- the weight-only variant: int8 weights, bf16 activations,
// on the sm_100a tensor cores (tcgen05.mma kind::f16, fp32 accumulators):
//
//   y[m,n] = bf16( (sum_k x[m,k] * q[n,k]) * s_w[n] + bias[n] )
//
// ("Issue 5 probe: int8 quantized DiT serve paths on the RTX 3090 (24 GB)",
// section "Round one: int8 weight-only via compressed-tensors": int8
// weight-only, per-output-channel symmetric, activations kept in bf16.)  With
// one scale per output channel the scale factors out of the sum, so it is
// applied once in the epilogue; every product x * q is exact in fp32 and the
// tensor core accumulates them in fp32.
//
// A kind::f16 MMA takes A and B of the same 16-bit type, so the int8 weights
// are widened to bf16 in shared memory inside the main loop (exact: |q| <= 128
// has an 8-bit significand).  One CTA per SM, persistent over 128 x BN tiles:
//   warp 0       TMA: x (bf16, 128 rows x 64 K, 128-byte swizzle) and Wq
//                (int8, BN rows x 64 K, unswizzled) into a STAGES-deep ring;
//   warp 1       TMEM owner; one thread issues tcgen05.mma (M = 128, N = BN,
//                K = 16) once a stage's weights are widened;
//   warps 2..9   the epilogue, as in the int8 GEMM (fp32 accumulators);
//   warps 10..13 widen each stage's BN x 64 int8 weights to bf16, writing the
//                128-byte-swizzled K-major layout the MMA reads.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cstdint>

#include "w8a8_gemm.cuh"
#include "w8a8_ptx.cuh"

namespace w8a8 {

// D (fp32, TMEM) (+)= A (bf16, smem) x B (bf16, smem)^T, one CTA, K = 16.
__device__ __forceinline__ void mma_bf16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                         uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Instruction descriptor, kind::f16: D f32 (bits 4-5 = 1), A and B bf16
// (bits 7-9 = 1, 10-12 = 1), both K-major, N >> 3 at bits 17-22, M >> 4 at
// bits 24-28.
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N) {
  return (1u << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>(N >> 3) << 17) |
         (static_cast<uint32_t>(M >> 4) << 24);
}

// One epilogue warp's share of an fp32 accumulator (its 32 TMEM lanes, COLS
// columns from col_base, in 32-column chunks): y = bf16(acc * s_w + bias), the
// multiply and the add separately rounded fp32 operations, stored through the
// same 64-byte-swizzled staging buffers and TMA stores as the int8 GEMM's
// epilogue.
template <int COLS>
__device__ __forceinline__ void w16_epilogue_warp_slice(const GemmParams &p,
                                                        const CUtensorMap *tmap_y, uint32_t t_row,
                                                        int row0, int col_base,
                                                        uint8_t *stage_buf,
                                                        uint32_t &chunk_count, int lane) {
  if (row0 >= p.M) return;  // all 32 rows past M: nothing to store
#pragma unroll 1
  for (int c = 0; c < COLS; c += kEpiChunk) {
    const int col0 = col_base + c;
    if (col0 >= p.N) break;  // warp-uniform
    float sw[32];
    uint32_t bw[16];
#pragma unroll
    for (int g = 0; g < 4; ++g) {
      const int cg = col0 + 8 * g;
      if (cg < p.N) {
        const float4 w0 = __ldg(reinterpret_cast<const float4 *>(p.s_w + cg));
        const float4 w1 = __ldg(reinterpret_cast<const float4 *>(p.s_w + cg) + 1);
        sw[8 * g + 0] = w0.x; sw[8 * g + 1] = w0.y; sw[8 * g + 2] = w0.z; sw[8 * g + 3] = w0.w;
        sw[8 * g + 4] = w1.x; sw[8 * g + 5] = w1.y; sw[8 * g + 6] = w1.z; sw[8 * g + 7] = w1.w;
        if (p.bias != nullptr) {
          const uint4 braw = __ldg(reinterpret_cast<const uint4 *>(p.bias + cg));
          bw[4 * g + 0] = braw.x; bw[4 * g + 1] = braw.y;
          bw[4 * g + 2] = braw.z; bw[4 * g + 3] = braw.w;
        } else {
          bw[4 * g + 0] = bw[4 * g + 1] = bw[4 * g + 2] = bw[4 * g + 3] = 0u;
        }
      } else {
#pragma unroll
        for (int i = 0; i < 8; ++i) sw[8 * g + i] = 0.0f;
        bw[4 * g + 0] = bw[4 * g + 1] = bw[4 * g + 2] = bw[4 * g + 3] = 0u;
      }
    }
    uint32_t r[32];
    tmem_ld_32x32b_x32(t_row + c, r);
    tmem_ld_wait();
    uint32_t packed[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      float2 v = make_float2(__uint_as_float(r[2 * i]), __uint_as_float(r[2 * i + 1]));
      v = mul2_rn(v, make_float2(sw[2 * i], sw[2 * i + 1]));
      if (p.bias != nullptr)
        v = add2_rn(v, make_float2(__uint_as_float(bw[i] << 16),
                                   __uint_as_float(bw[i] & 0xFFFF0000u)));
      const __nv_bfloat162 h = __floats2bfloat162_rn(v.x, v.y);
      packed[i] = *reinterpret_cast<const uint32_t *>(&h);
    }
    uint8_t *buf = stage_buf + (chunk_count & 1u) * kEpiBufBytes;
    if (lane == 0) bulk_wait_group_read<1>();
    __syncwarp();
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int pos = j ^ ((lane >> 1) & 3);
      *reinterpret_cast<uint4 *>(buf + lane * 64 + pos * 16) =
          make_uint4(packed[4 * j], packed[4 * j + 1], packed[4 * j + 2], packed[4 * j + 3]);
    }
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) {
      tma_store_2d(tmap_y, buf, col0, row0);
      bulk_commit_group();
    }
    ++chunk_count;
  }
}

constexpr int kW16ConvWarps = 4;
constexpr int kW16Threads = (2 + kEpiWarps + kW16ConvWarps) * 32;  // 448
constexpr int kW16BK = 64;  // bf16 elements of K per stage = one 128-byte swizzle row

template <int BN, int STAGES>
struct W16Layout {
  static constexpr int kABytes = kBM * kW16BK * 2;   // x tile, bf16
  static constexpr int kBBytes = BN * kW16BK * 2;    // widened weights, bf16
  static constexpr int kB8Bytes = BN * kW16BK;       // int8 weights as loaded
  static constexpr int kStageBytes = kABytes + kBBytes + kB8Bytes;
  static constexpr int kTileBytes = STAGES * kStageBytes;
  static constexpr int kEpiOffset = kTileBytes;
  static constexpr int kEpiBytes = kEpiWarps * 2 * kEpiBufBytes;
  static constexpr int kBarOffset = kEpiOffset + kEpiBytes;
  // full[STAGES], conv[STAGES], empty[STAGES], tfull[2], tempty[2], drain, two words
  static constexpr int kBarBytes = (3 * STAGES + 5) * 8 + 8;
  static constexpr int kSmemBytes = kBarOffset + kBarBytes + 1024;
  static constexpr int kTmemCols = 2 * BN;
  static_assert(kStageBytes % 1024 == 0, "stage buffers stay 1024-byte aligned");
  static_assert(kSmemBytes <= 232448, "shared memory budget");
};

// Two int8 lanes of a word -> a bf16x2 word, exactly and with full-rate
// integer/float operations only: sign-extend the byte (a byte permute with
// the sign-replicate selector), add it to the bit pattern of 1.5 * 2^23 --
// giving the float 1.5 * 2^23 + v exactly -- subtract 1.5 * 2^23 (exact,
// = (float)v), and keep the upper halves: (float)v has at most 8 significant
// bits, so its low 16 bits are zero and its upper half is bf16(v).
__device__ __forceinline__ uint32_t prmt_b32(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t r;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(sel));
  return r;
}

__device__ __forceinline__ uint32_t widen2(uint32_t w, uint32_t sel_lo, uint32_t sel_hi) {
  const float magic = 12582912.0f;  // 1.5 * 2^23
  // selector 0xNNNn, N = 8 + n: result byte 0 = byte n of w, bytes 1..3 =
  // that byte's sign (prmt's sign-replicate selectors)
  const uint32_t e0 = prmt_b32(w, 0u, sel_lo);
  const uint32_t e1 = prmt_b32(w, 0u, sel_hi);
  const float f0 = __fsub_rn(__uint_as_float(__float_as_uint(magic) + e0), magic);
  const float f1 = __fsub_rn(__uint_as_float(__float_as_uint(magic) + e1), magic);
  return prmt_b32(__float_as_uint(f0), __float_as_uint(f1), 0x7632u);
}

// int8 weights of one stage -> bf16 in the 128-byte-swizzled K-major layout:
// row r (128 bytes = 64 bf16) holds its 16-byte chunk j at position j ^ (r & 7).
// Thread `t` of the converter warps takes rows t, t + 128, ...
template <int BN>
__device__ __forceinline__ void widen_stage(const uint8_t *b8, uint8_t *b16, int t) {
  for (int r = t; r < BN; r += kW16ConvWarps * 32) {
    const uint4 *src = reinterpret_cast<const uint4 *>(b8 + r * kW16BK);
#pragma unroll
    for (int h = 0; h < 4; ++h) {  // 16 int8 -> two 16-byte bf16 chunks
      const uint4 v = src[h];
      const uint32_t w[4] = {v.x, v.y, v.z, v.w};
      uint32_t o[8];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        o[2 * i] = widen2(w[i], 0x8880u, 0x9991u);
        o[2 * i + 1] = widen2(w[i], 0xAAA2u, 0xBBB3u);
      }
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        const int j = 2 * h + c;  // 16-byte chunk = bf16 elements 8j .. 8j + 7
        *reinterpret_cast<uint4 *>(b16 + r * 128 + ((j ^ (r & 7)) << 4)) =
            make_uint4(o[4 * c], o[4 * c + 1], o[4 * c + 2], o[4 * c + 3]);
      }
    }
  }
}

template <int BN, int STAGES>
__global__ void __launch_bounds__(kW16Threads, 1)
    gemm_w8a16_tcgen05_kernel(const __grid_constant__ CUtensorMap tmap_x,
                              const __grid_constant__ CUtensorMap tmap_w,
                              const __grid_constant__ CUtensorMap tmap_y, const GemmParams p) {
  using L = W16Layout<BN, STAGES>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_addr(smem_raw);
  uint8_t *smem = smem_raw + ((1024u - (raw_addr & 1023u)) & 1023u);
  uint64_t *full = reinterpret_cast<uint64_t *>(smem + L::kBarOffset);
  uint64_t *conv = full + STAGES;
  uint64_t *empty = conv + STAGES;
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
      mbar_init(&conv[s], kW16ConvWarps);  // one arrival per converter warp
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], kEpiWarps);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbarrier_init();
    tma_prefetch_desc(&tmap_x);
    tma_prefetch_desc(&tmap_w);
    tma_prefetch_desc(&tmap_y);
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
      grid_dependency_wait();  // x may come from the preceding kernel
      for (int t = blockIdx.x; ok && t < p.num_tiles; t += gridDim.x) {
        int mb, nb;
        gemm_tile_coords(t, p, mb, nb);
        for (int kb = 0; kb < p.k_blocks; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag)) {
            ok = false;
            break;
          }
          uint8_t *sa = smem + stage * L::kStageBytes;
          uint8_t *s8 = sa + L::kABytes + L::kBBytes;
          mbar_arrive_expect_tx(&full[stage], L::kABytes + L::kB8Bytes);
          tma_load_2d(&tmap_w, &full[stage], s8, kb * kW16BK, nb * BN);
          tma_load_2d(&tmap_x, &full[stage], sa, kb * kW16BK, mb * kBM);
          ++issued;
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      grid_dependents_launch();
      if (!ok) {
        const uint32_t n = issued < static_cast<uint32_t>(STAGES) ? issued : STAGES;
        for (uint32_t i = issued - n; i < issued; ++i)
          mbar_wait_drain(&full[i % STAGES], (i / STAGES) & 1u);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16(kBM, BN);
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
          if (!mbar_wait(&full[stage], phase, abort_flag) ||
              !mbar_wait(&conv[stage], phase, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sa = smem_addr(smem + stage * L::kStageBytes);
          const uint64_t adesc = smem_desc_k_sw128(sa);
          const uint64_t bdesc = smem_desc_k_sw128(sa + L::kABytes);
#pragma unroll
          for (int k = 0; k < kW16BK / 16; ++k)  // K = 16 bf16 = 32 bytes per MMA
            mma_bf16(d_tmem, adesc + 2u * k, bdesc + 2u * k, idesc, (kb | k) != 0 ? 1u : 0u);
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
        mma_commit(drain);
        mbar_wait_drain(drain, 0);
      }
    }
  } else if (warp < 2 + kEpiWarps) {
    // ------------------------------------------------------------ epilogue
    const int e = warp - 2;
    const int quarter = warp & 3;
    const int half = e >> 2;
    uint8_t *stage_buf = smem + L::kEpiOffset + e * 2 * kEpiBufBytes;
    uint32_t chunk_count = 0;
    int acc = 0;
    uint32_t acc_phase = 0;
    grid_dependency_wait();
    for (int t = blockIdx.x; t < p.num_tiles; t += gridDim.x) {
      int mb, nb;
      gemm_tile_coords(t, p, mb, nb);
      int ok = 1;
      if (lane == 0) ok = mbar_wait(&tfull[acc], acc_phase, abort_flag) ? 1 : 0;
      ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
      if (!ok) break;
      tc_fence_after();
      const uint32_t t_row = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) +
                             static_cast<uint32_t>(acc * BN + half * (BN / 2));
      w16_epilogue_warp_slice<BN / 2>(p, &tmap_y, t_row, mb * kBM + quarter * 32,
                                      nb * BN + half * (BN / 2), stage_buf, chunk_count, lane);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty[acc]);
      if (++acc == 2) {
        acc = 0;
        acc_phase ^= 1u;
      }
    }
    if (lane == 0) bulk_wait_all();
    __syncwarp();
  } else {
    // ------------------------------------------------------------ weight widening
    const int ct = threadIdx.x - (2 + kEpiWarps) * 32;  // 0 .. 127
    int stage = 0;
    uint32_t phase = 0;
    for (int t = blockIdx.x; t < p.num_tiles; t += gridDim.x) {
      bool ok = true;
      for (int kb = 0; kb < p.k_blocks; ++kb) {
        int got = 1;
        if (lane == 0) got = mbar_wait(&full[stage], phase, abort_flag) ? 1 : 0;
        got = __shfl_sync(0xFFFFFFFFu, got, 0);
        if (!got) {
          ok = false;
          break;
        }
        uint8_t *sa = smem + stage * L::kStageBytes;
        widen_stage<BN>(sa + L::kABytes + L::kBBytes, sa + L::kABytes, ct);
        fence_proxy_async_smem();  // the MMA reads these bytes through the async proxy
        __syncwarp();
        if (lane == 0) mbar_arrive(&conv[stage]);
        if (++stage == STAGES) {
          stage = 0;
          phase ^= 1u;
        }
      }
      if (!ok) break;
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
