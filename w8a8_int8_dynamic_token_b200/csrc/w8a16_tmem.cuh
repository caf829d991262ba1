// w8a16_tmem.cuh -- the weight-only variant with the widened weights in tensor
// memory:
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
// must be widened to bf16 (exact: |q| <= 128 has an 8-bit significand).
// Widening them into shared memory costs more shared-memory bandwidth than the
// MMAs themselves (16 KB written and 16 KB read again per stage; measured at
// 26% of the bf16 peak on a B200, against 55% for this design).  Here the
// weights take the MMA's A side, which tcgen05.mma may read from tensor
// memory: converter warps read each stage's int8 weights from shared memory
// once and write the widened rows straight into TMEM with tcgen05.st, so
// shared memory carries only the TMA-loaded x and int8 weights and the MMA's
// reads of x.  Each CTA computes the transposed tile
//     D[n, m] = sum_k q[n, k] * x[m, k]      (fp32 in TMEM)
// for 128 weight rows n and 192 tokens m (two accumulators of 192 columns plus
// four 32-column A stages fill the 512 TMEM columns), persistent over tiles.
//   warp 0       TMA: x (bf16, 192 rows x 64 K, 128-byte swizzle) and Wq
//                (int8, 128 rows x 64 K, 64-byte swizzle) into a 6-deep ring;
//   warp 1       TMEM owner; one thread issues tcgen05.mma (M = 128 from TMEM,
//                N = 192, K = 16) once a stage's x and widened weights are in;
//   warps 2..5   converters: lane = weight row, 64 int8 from shared memory ->
//                64 bf16 -> 32 TMEM columns of the A stage;
//   warps 6..9   epilogue: lane = weight row n, columns = tokens m:
//                y[m, n] = bf16(acc * s_w[n] + bias[n]), stored as 32 lanes x
//                2 bytes = 64 contiguous bytes per token row.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cstdint>

#include "w8a8_gemm.cuh"
#include "w8a8_ptx.cuh"

namespace w8a8 {

constexpr int kWtThreads = 320;    // 10 warps
constexpr int kWtBN = 192;         // tokens per tile (the MMA's N)
constexpr int kWtStages = 6;
constexpr int kWtAStages = 4;      // A (widened weights) stages in TMEM, 32 columns each
constexpr int kWtBK = 64;          // K elements per stage

struct WtLayout {
  static constexpr int kXBytes = kWtBN * kWtBK * 2;    // 24 KB
  static constexpr int kWBytes = kBM * kWtBK;          // 8 KB
  static constexpr int kStageBytes = kXBytes + kWBytes;
  static constexpr int kRingBytes = kWtStages * kStageBytes;
  static constexpr int kBarOffset = kRingBytes;
  // full[S], empty[S], afull[A], aempty[A], tfull[2], tempty[2], drain, two words
  static constexpr int kBarBytes = (2 * kWtStages + 2 * kWtAStages + 5) * 8 + 8;
  static constexpr int kSmemBytes = kBarOffset + kBarBytes + 1024;
  static constexpr int kTmemCols = 512;
  static constexpr int kAccCols = kWtBN;                 // per accumulator
  static constexpr int kACol0 = 2 * kWtBN;               // first A-stage column
  static_assert(kStageBytes % 1024 == 0, "stage buffers stay 1024-byte aligned");
  static_assert(kACol0 + kWtAStages * 32 <= kTmemCols, "tensor memory budget");
  static_assert(kSmemBytes <= 232448, "shared memory budget");
};

// Instruction descriptor, kind::f16: D f32 (bits 4-5 = 1), A and B bf16
// (bits 7-9 = 1, 10-12 = 1), both K-major, N >> 3 at bits 17-22, M >> 4 at
// bits 24-28.
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N) {
  return (1u << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>(N >> 3) << 17) |
         (static_cast<uint32_t>(M >> 4) << 24);
}

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

// D (fp32, TMEM) (+)= A (bf16, TMEM) x B (bf16, smem)^T, one CTA, K = 16.
__device__ __forceinline__ void mma_bf16_ta(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                            uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Warp-collective store of 32 consecutive 32-bit columns of the warp's 32
// TMEM lanes: thread t writes lane (base lane + t), columns col .. col+31.
__device__ __forceinline__ void tmem_st_32x32b_x32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, "
      "%17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
      "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]),
      "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]),
      "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}

__device__ __forceinline__ void tmem_st_wait() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

struct WtParams {
  int32_t M, N, K;
  int32_t num_n_blk, num_m_blk, num_tiles, k_blocks;
  const float *s_w;
  const uint16_t *bias;  // bf16 bits or nullptr
  uint16_t *y;           // bf16 [M, N], row stride ldy
  int64_t ldy;
};

__global__ void __launch_bounds__(kWtThreads, 1)
    gemm_w8a16_tmem_kernel(const __grid_constant__ CUtensorMap tmap_x,
                           const __grid_constant__ CUtensorMap tmap_w, const WtParams p) {
  using L = WtLayout;
  constexpr int S = kWtStages, SA = kWtAStages;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_addr(smem_raw);
  uint8_t *smem = smem_raw + ((1024u - (raw_addr & 1023u)) & 1023u);
  uint64_t *full = reinterpret_cast<uint64_t *>(smem + L::kBarOffset);
  uint64_t *empty = full + S;
  uint64_t *afull = empty + S;
  uint64_t *aempty = afull + SA;
  uint64_t *tfull = aempty + SA;
  uint64_t *tempty = tfull + 2;
  uint64_t *drain = tempty + 2;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(drain + 1);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < SA; ++a) {
      mbar_init(&afull[a], 4);   // the four converter warps
      mbar_init(&aempty[a], 1);  // the MMA commit
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 4);  // the four epilogue warps
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbarrier_init();
    tma_prefetch_desc(&tmap_x);
    tma_prefetch_desc(&tmap_w);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, L::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  // tile t: weight block t / num_m_blk (consecutive CTAs share it), token block t % num_m_blk
  auto coords = [&](int t, int &nb, int &mb) {
    nb = t / p.num_m_blk;
    mb = t - nb * p.num_m_blk;
  };

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      grid_dependency_wait();  // x may come from the preceding kernel
      int stage = 0;
      uint32_t phase = 0, issued = 0;
      bool ok = true;
      for (int t = blockIdx.x; ok && t < p.num_tiles; t += gridDim.x) {
        int nb, mb;
        coords(t, nb, mb);
        for (int kb = 0; kb < p.k_blocks; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag)) {
            ok = false;
            break;
          }
          uint8_t *sx = smem + stage * L::kStageBytes;
          mbar_arrive_expect_tx(&full[stage], L::kStageBytes);
          tma_load_2d(&tmap_x, &full[stage], sx, kb * kWtBK, mb * kWtBN);
          tma_load_2d(&tmap_w, &full[stage], sx + L::kXBytes, kb * kWtBK, nb * kBM);
          ++issued;
          if (++stage == S) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      grid_dependents_launch();
      const uint32_t n = issued < static_cast<uint32_t>(S) ? issued : S;
      for (uint32_t i = issued - n; i < issued; ++i) {
        volatile int never = 0;
        mbar_wait(&full[i % S], (i / S) & 1u, &never);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16(kBM, kWtBN);
      int stage = 0, astage = 0, acc = 0;
      uint32_t phase = 0, aphase = 0, acc_phase = 0;
      bool ok = true, any = false;
      for (int t = blockIdx.x; ok && t < p.num_tiles; t += gridDim.x) {
        if (!mbar_wait(&tempty[acc], acc_phase ^ 1u, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * L::kAccCols);
        for (int kb = 0; kb < p.k_blocks; ++kb) {
          if (!mbar_wait(&full[stage], phase, abort_flag) ||
              !mbar_wait(&afull[astage], aphase, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t bdesc = smem_desc_k_sw128(smem_addr(smem + stage * L::kStageBytes));
          const uint32_t a_tmem = tmem_base + static_cast<uint32_t>(L::kACol0 + astage * 32);
#pragma unroll
          for (int k = 0; k < kWtBK / 16; ++k)  // 16 bf16 = 8 TMEM columns, 32 bytes of x
            mma_bf16_ta(d_tmem, a_tmem + 8u * k, bdesc + 2u * k, idesc, (kb | k) != 0 ? 1u : 0u);
          any = true;
          mma_commit(&empty[stage]);
          mma_commit(&aempty[astage]);
          if (++stage == S) {
            stage = 0;
            phase ^= 1u;
          }
          if (++astage == SA) {
            astage = 0;
            aphase ^= 1u;
          }
        }
        if (!ok) break;
        mma_commit(&tfull[acc]);
        if (++acc == 2) {
          acc = 0;
          acc_phase ^= 1u;
        }
      }
      if (!ok && any) {
        mma_commit(drain);
        volatile int never = 0;
        mbar_wait(drain, 0u, &never);
      }
    }
  } else if (warp < 6) {
    // ------------------------------------------------------------ converters
    const int quarter = warp & 3;                  // TMEM lanes 32 quarter .. + 31
    const int row = quarter * 32 + lane;           // weight row within the tile
    int stage = 0, astage = 0;
    uint32_t phase = 0, aphase = 0;
    bool ok = true;
    for (int t = blockIdx.x; ok && t < p.num_tiles; t += gridDim.x) {
      for (int kb = 0; kb < p.k_blocks; ++kb) {
        int w1 = mbar_wait(&full[stage], phase, abort_flag) ? 1 : 0;
        int w2 = mbar_wait(&aempty[astage], aphase ^ 1u, abort_flag) ? 1 : 0;
        if (!__all_sync(0xFFFFFFFFu, w1 & w2)) {
          ok = false;
          break;
        }
        tc_fence_after();
        // this row's 64 int8: four 16-byte chunks, laid out by the TMA's
        // 64-byte swizzle (chunk c of row r at position c ^ ((r >> 1) & 3)),
        // so the 32 lanes' reads of one chunk hit distinct banks
        const uint4 *src = reinterpret_cast<const uint4 *>(smem + stage * L::kStageBytes +
                                                           L::kXBytes + row * kWtBK);
        uint32_t o[32];
#pragma unroll
        for (int h = 0; h < 4; ++h) {
          const uint4 v = src[h ^ ((row >> 1) & 3)];
          const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            // bf16 elements 16 h + 4 i .. + 3 -> columns 8 h + 2 i, 8 h + 2 i + 1
            o[8 * h + 2 * i] = widen2(w[i], 0x8880u, 0x9991u);
            o[8 * h + 2 * i + 1] = widen2(w[i], 0xAAA2u, 0xBBB3u);
          }
        }
        tmem_st_32x32b_x32(tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) +
                               static_cast<uint32_t>(L::kACol0 + astage * 32),
                           o);
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&afull[astage]);
        if (++stage == S) {
          stage = 0;
          phase ^= 1u;
        }
        if (++astage == SA) {
          astage = 0;
          aphase ^= 1u;
        }
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int quarter = warp & 3;
    int acc = 0;
    uint32_t acc_phase = 0;
    grid_dependency_wait();  // y may still be read by the preceding kernel
    for (int t = blockIdx.x; t < p.num_tiles; t += gridDim.x) {
      int nb, mb;
      coords(t, nb, mb);
      int ok = 1;
      if (lane == 0) ok = mbar_wait(&tfull[acc], acc_phase, abort_flag) ? 1 : 0;
      ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
      if (!ok) break;
      tc_fence_after();
      const int n = nb * kBM + quarter * 32 + lane;
      const bool n_ok = n < p.N;
      const float sw = n_ok ? __ldg(p.s_w + n) : 0.0f;
      const float bv = (n_ok && p.bias != nullptr)
                           ? __uint_as_float(static_cast<uint32_t>(__ldg(p.bias + n)) << 16)
                           : 0.0f;
      const uint32_t t_row = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) +
                             static_cast<uint32_t>(acc * L::kAccCols);
#pragma unroll 1
      for (int c = 0; c < kWtBN; c += 32) {
        const int m0 = mb * kWtBN + c;
        if (m0 >= p.M) break;  // warp-uniform
        uint32_t r[32];
        tmem_ld_32x32b_x32(t_row + c, r);
        tmem_ld_wait();
        if (!n_ok) continue;
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          if (m0 + j >= p.M) break;
          float v = __fmul_rn(__uint_as_float(r[j]), sw);
          if (p.bias != nullptr) v = __fadd_rn(v, bv);
          const __nv_bfloat16 h = __float2bfloat16_rn(v);
          p.y[static_cast<int64_t>(m0 + j) * p.ldy + n] = *reinterpret_cast<const uint16_t *>(&h);
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
