// w8a8_gemv.cuh -- the W8A8 layer for M <= 16 activation rows.
//
// At M = batch (1, or 2 under classifier-free guidance) the AdaLN modulation
// and conditioning-embedder linears are matrix-vector products (unsloth commit
// history of test_diffusion_transformer_quant.py: the commit on torch._int_mm
// needing more than 16 rows, e.g. Flux norm1.linear 3072 -> 18432 at M = 1).
// Their cost is streaming the int8 weight matrix from HBM once, so this kernel
// is built around that stream:
//   1. (fused variant) every CTA quantizes the M activation rows into shared
//      memory with the per-token rule of the quantization kernel;
//      (unfused variant) every CTA copies the given q rows into shared memory;
//   2. each warp walks pairs of weight rows, every lane holding 8 16-byte
//      vectors of each row in flight (evict-first loads; the first pair's
//      loads are issued before step 1 so the prologue hides under them, and
//      before waiting on the preceding kernel when launched as a programmatic
//      dependent; the warp's next pair is prefetched into L2 by two bulk
//      prefetches while it works on the current one),
//      accumulating M int32 dot products with dp4a (exact: every partial sum
//      is bounded by 127*127*K < 2^31);
//   3. a warp reduction, then lane m writes
//      y[m,n] = bf16_rne(((float)acc * s_a[m]) * s_w[n] + (float)bias[n]).
#pragma once

#include <cuda_bf16.h>
#include <cstdint>

#include "w8a8_prefetch.cuh"
#include "w8a8_ptx.cuh"
#include "w8a8_quant.cuh"

namespace w8a8 {

constexpr int kGemvThreads = 256;
constexpr int kGemvMaxM = 16;

struct GemvParams {
  int32_t M, N, K;
  const uint16_t *x;  // bf16 [M, K], row stride ldx (fused variant)
  int64_t ldx;
  const int8_t *q;    // int8 [M, K] dense (unfused variant)
  const float *s_a;   // [M] (unfused variant)
  const int8_t *wq;   // [N, K] dense
  const float *s_w;
  const uint16_t *bias;  // or nullptr
  uint16_t *y;
  int64_t ldy;
  int32_t *acc_out;   // raw int32 [M, N] dense instead of y (debug), or nullptr
  int8_t *q_out;      // fused variant: optional copy of q (written by CTA 0)
  float *s_a_out;     // fused variant: optional copy of s_a
};

// Block-wide max of bit patterns of non-negative floats.
__device__ __forceinline__ uint32_t block_max_u32(uint32_t v, uint32_t *red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = max(v, __shfl_xor_sync(0xFFFFFFFFu, v, o));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  __syncthreads();  // red[] may still be read from the previous call
  if (lane == 0) red[warp] = v;
  __syncthreads();
  v = 0u;
#pragma unroll
  for (int w = 0; w < kGemvThreads / 32; ++w) v = max(v, red[w]);
  return v;
}

constexpr int kGemvWarps = kGemvThreads / 32;
constexpr int kGemvRows = 2;  // weight rows per warp step
constexpr int kGemvVec = 8;   // 16-byte weight vectors per lane per row per step

// Loads kGemvVec 16-byte vectors per row for the rows n0, n0+1, starting at
// vector index kb + lane (stride 32); rows past N and vectors past K read 0.
__device__ __forceinline__ void gemv_load(const int8_t *__restrict__ wq, int N, int nvec16,
                                          int n0, int kb, int lane,
                                          uint4 (&wv)[kGemvRows][kGemvVec]) {
#pragma unroll
  for (int r = 0; r < kGemvRows; ++r) {
    const int n = n0 + r;
    const uint4 *wr = reinterpret_cast<const uint4 *>(wq + static_cast<int64_t>(n) * nvec16 * 16);
#pragma unroll
    for (int u = 0; u < kGemvVec; ++u) {
      const int vi = kb + lane + 32 * u;
      wv[r][u] = (n < N && vi < nvec16) ? __ldcs(wr + vi) : make_uint4(0u, 0u, 0u, 0u);
    }
  }
}

template <int MT, bool FUSED, bool RAW_OUT>
__global__ void __launch_bounds__(kGemvThreads, 2) gemv_i8_kernel(const GemvParams p) {
  extern __shared__ __align__(16) uint8_t gemv_smem[];
  int8_t *qs = reinterpret_cast<int8_t *>(gemv_smem);  // [M][K]
  __shared__ float sas[kGemvMaxM];
  __shared__ uint32_t red[4][kGemvWarps];

  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int K = p.K;
  const int nvec16 = K >> 4;   // 16-byte int8 vectors per row
  const int npairs = (p.N + kGemvRows - 1) / kGemvRows;
  const int warps_total = gridDim.x * kGemvWarps;
  int pi = blockIdx.x * kGemvWarps + warp;

  // The weight stream is what this kernel waits on: start it before the
  // activation prologue -- and, under programmatic dependent launch, before
  // waiting for the preceding kernel (the weights do not depend on it; x, q
  // and s_a may, so they are read only after the wait).
  uint4 wv[kGemvRows][kGemvVec];
  if (pi < npairs) gemv_load(p.wq, p.N, nvec16, pi * kGemvRows, 0, lane, wv);
  grid_dependency_wait();

  // ---- 1. activation rows -> shared memory (int8) + scales.  Fused, up to
  // 4 rows of up to 4096 elements: the whole block loads every row at once
  // into registers and reduces all their maxima in one block reduction (the
  // latency of one row, whatever M); longer rows: one row at a time; more
  // rows: one warp per row, 8 rows at once.
  if constexpr (FUSED && MT <= 4) {
    const int nvec8 = K >> 3;
    if (nvec8 <= 2 * kGemvThreads) {
      uint4 xv[MT][2];
      uint32_t mb[MT];
#pragma unroll
      for (int m = 0; m < MT; ++m) {
        const uint4 *xr = reinterpret_cast<const uint4 *>(p.x + static_cast<int64_t>(m) * p.ldx);
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          const int v = tid + j * kGemvThreads;
          xv[m][j] = (m < p.M && v < nvec8) ? __ldg(xr + v) : make_uint4(0u, 0u, 0u, 0u);
        }
      }
#pragma unroll
      for (int m = 0; m < MT; ++m) {
        mb[m] = __float_as_uint(absmax_vec8(xv[m][1], absmax_vec8(xv[m][0], 0.0f)));
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) mb[m] = max(mb[m], __shfl_xor_sync(0xFFFFFFFFu, mb[m], o));
        if (lane == 0) red[m][warp] = mb[m];
      }
      __syncthreads();
#pragma unroll
      for (int m = 0; m < MT; ++m) {
        if (m >= p.M) break;
        uint32_t a = 0u;
#pragma unroll
        for (int w = 0; w < kGemvWarps; ++w) a = max(a, red[m][w]);
        const float amax = __uint_as_float(a);
        const float sc = (amax == 0.0f) ? 0.0f : __fdiv_rn(amax, 127.0f);
        const bool fast = quant_fast_ok(sc);
        const float rc = fast ? __frcp_rn(sc) : 0.0f;
        if (tid == 0) sas[m] = sc;
        uint2 *qrow = reinterpret_cast<uint2 *>(qs + m * K);
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          const int v = tid + j * kGemvThreads;
          if (v < nvec8)
            qrow[v] = (sc == 0.0f) ? make_uint2(0u, 0u) : quant_vec8(xv[m][j], sc, rc, fast);
        }
      }
    } else {
      for (int m = 0; m < p.M; ++m) {
        const uint4 *xr = reinterpret_cast<const uint4 *>(p.x + static_cast<int64_t>(m) * p.ldx);
        float mm = 0.0f;
        for (int v = tid; v < nvec8; v += kGemvThreads) mm = absmax_vec8(__ldg(xr + v), mm);
        const float amax = __uint_as_float(block_max_u32(__float_as_uint(mm), red[0]));
        const float sc = (amax == 0.0f) ? 0.0f : __fdiv_rn(amax, 127.0f);
        const bool fast = quant_fast_ok(sc);
        const float rc = fast ? __frcp_rn(sc) : 0.0f;
        if (tid == 0) sas[m] = sc;
        uint2 *qrow = reinterpret_cast<uint2 *>(qs + m * K);
        for (int v = tid; v < nvec8; v += kGemvThreads)
          qrow[v] = (sc == 0.0f) ? make_uint2(0u, 0u) : quant_vec8(__ldg(xr + v), sc, rc, fast);
      }
    }
  } else if constexpr (FUSED) {
    for (int m = warp; m < p.M; m += kGemvWarps)
      quant_row_by_warp<12>(p.x + static_cast<int64_t>(m) * p.ldx, K, qs + m * K, &sas[m], lane);
  } else {
    const uint4 *src = reinterpret_cast<const uint4 *>(p.q);
    uint4 *dst = reinterpret_cast<uint4 *>(qs);
    for (int v = tid; v < p.M * nvec16; v += kGemvThreads) dst[v] = __ldg(src + v);
    if (tid < p.M) sas[tid] = __ldg(p.s_a + tid);
  }
  __syncthreads();
  grid_dependents_launch();  // every CTA is resident; the next kernel may be scheduled
  if constexpr (FUSED) {
    if (blockIdx.x == 0) {
      if (p.q_out != nullptr) {
        const uint4 *src = reinterpret_cast<const uint4 *>(qs);
        uint4 *dst = reinterpret_cast<uint4 *>(p.q_out);
        for (int v = tid; v < p.M * nvec16; v += kGemvThreads) dst[v] = src[v];
      }
      if (p.s_a_out != nullptr && tid < p.M) p.s_a_out[tid] = sas[tid];
    }
  }

  // ---- 2. stream weight rows, two rows per warp step.  Before working on a
  // pair, lanes 0 and 1 ask for the warp's next pair of rows to be brought
  // into L2 (one bulk prefetch per row), so the weight stream from HBM goes
  // on while the warp computes and reduces; the register loads of the next
  // pair then come from L2.
  bool loaded = true;  // wv already holds (pi, kb = 0)
  for (; pi < npairs; pi += warps_total) {
    const int n0 = pi * kGemvRows;
    {
      const int nn = n0 + warps_total * kGemvRows + lane;
      if (lane < kGemvRows && nn < p.N)
        bulk_prefetch_l2(p.wq + static_cast<int64_t>(nn) * K, static_cast<uint32_t>(K));
    }
    int acc[kGemvRows][MT];
#pragma unroll
    for (int r = 0; r < kGemvRows; ++r)
#pragma unroll
      for (int m = 0; m < MT; ++m) acc[r][m] = 0;
    for (int kb = 0; kb < nvec16; kb += 32 * kGemvVec) {
      if (!loaded) gemv_load(p.wq, p.N, nvec16, n0, kb, lane, wv);
      loaded = false;
#pragma unroll
      for (int u = 0; u < kGemvVec; ++u) {
        const int vi = kb + lane + 32 * u;
        if (vi < nvec16) {
#pragma unroll
          for (int m = 0; m < MT; ++m) {
            if (m < p.M) {
              const int4 qv = reinterpret_cast<const int4 *>(qs + m * K)[vi];
#pragma unroll
              for (int r = 0; r < kGemvRows; ++r) {
                acc[r][m] = __dp4a(static_cast<int>(wv[r][u].x), qv.x, acc[r][m]);
                acc[r][m] = __dp4a(static_cast<int>(wv[r][u].y), qv.y, acc[r][m]);
                acc[r][m] = __dp4a(static_cast<int>(wv[r][u].z), qv.z, acc[r][m]);
                acc[r][m] = __dp4a(static_cast<int>(wv[r][u].w), qv.w, acc[r][m]);
              }
            }
          }
        }
      }
    }
    // ---- 3. reduce across the warp; lane m finishes row m of each weight row
#pragma unroll
    for (int r = 0; r < kGemvRows; ++r) {
      const int n = n0 + r;
#pragma unroll
      for (int m = 0; m < MT; ++m) {
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) acc[r][m] += __shfl_xor_sync(0xFFFFFFFFu, acc[r][m], o);
      }
      int mine = 0;
#pragma unroll
      for (int m = 0; m < MT; ++m)
        if (lane == m) mine = acc[r][m];
      if (lane < p.M && n < p.N) {
        if constexpr (RAW_OUT) {
          p.acc_out[static_cast<int64_t>(lane) * p.N + n] = mine;
        } else {
          float v = __int2float_rn(mine);
          v = __fmul_rn(__fmul_rn(v, sas[lane]), __ldg(p.s_w + n));
          if (p.bias != nullptr)
            v = __fadd_rn(v, __uint_as_float(static_cast<uint32_t>(__ldg(p.bias + n)) << 16));
          const __nv_bfloat16 h = __float2bfloat16_rn(v);
          p.y[static_cast<int64_t>(lane) * p.ldy + n] = *reinterpret_cast<const uint16_t *>(&h);
        }
      }
    }
  }
}

}  // namespace w8a8
