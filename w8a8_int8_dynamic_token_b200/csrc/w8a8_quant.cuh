// w8a8_quant.cuh -- per-row symmetric int8 quantization (activations per
// token, weights per output channel).
//
// Definition (the W8A8 int8-dynamic scheme of "Issue 5 probe: int8 quantized
// DiT serve paths on the RTX 3090 (24 GB)", section "Round two ... W8A8
// int8-dynamic"; dynamic activation scaling per "Int8 Quantization",
// "Parameters" table):
//   s = max_k |x[k]| / 127         fp32, IEEE division, round to nearest even
//   q[k] = clamp(rint(x[k] / s), -127, 127)   quotient: IEEE fp32 division;
//                                             rint: nearest, ties to even
//   max |x| == 0  ->  s = 0, q = 0
//
// Layout of the work (quant_rows_kernel): a group of G threads owns one row,
// keeps its vectors (8 bf16 each) in registers, reduces max |x| (fmaxf on the
// widened values, then an integer max of the non-negative bit patterns across
// lanes and, for G > 32, across warps through shared memory), then quantizes
// its registers and writes 8 int8 per vector.  Each row is read from HBM
// exactly once.
//
// Rounding: rint(t) for |t| <= 127.0001 is formed exactly by adding
// 1.5 * 2^23 in round-to-nearest-even fp32 arithmetic; the low byte of the
// sum's bit pattern is then the two's-complement int8.  The quotient x / s is
// not divided out element by element: the row's correctly rounded reciprocal
// and one correction step give the same correctly rounded quotient as an IEEE
// division, without a branch (see quant_fast).
#pragma once

#include <cuda_bf16.h>
#include <cstdint>

#include "w8a8_ptx.cuh"

namespace w8a8 {

constexpr float kRintMagic = 12582912.0f;  // 1.5 * 2^23

// Exact path: q = clamp(rint(x / s), -127, 127) with an IEEE division.
// Returns the bit pattern of rint(t) + 1.5 * 2^23, whose low byte is the code.
__device__ __forceinline__ uint32_t quant_exact(float v, float s) {
  float t = __fdiv_rn(v, s);
  t = fminf(fmaxf(t, -127.0f), 127.0f);
  return __float_as_uint(__fadd_rn(t, kRintMagic));
}

// Fast path without a division: Markstein's correction step (P. Markstein,
// "Computation of elementary functions on the IBM RISC System/6000
// processor", IBM J. Res. Develop. 34(1), 1990).  With y = RN(1/s), the
// correctly rounded reciprocal, q0 = RN(x * y) is within one ulp of x/s, the
// remainder e = x - q0 * s is exact in one fused multiply-add, and
// q1 = RN(q0 + e * y) is the correctly rounded quotient RN(x/s) -- the same
// value an IEEE division returns -- provided nothing overflows or underflows,
// which quant_fast_ok guarantees for the row's scale.  Then rint(q1) is formed
// by adding 1.5 * 2^23 (exact, ties to even), and |rint(q1)| <= 127 (the clamp
// is inactive).  The step is checked exhaustively against the IEEE division
// on the GPU (w8a8_selftest_quant_exhaustive: every positive bf16 row
// maximum with every bf16 value of the row).
__device__ __forceinline__ uint32_t quant_fast(float x, float s, float y) {
  const float q0 = __fmul_rn(x, y);
  const float e = __fmaf_rn(-q0, s, x);
  const float q1 = __fmaf_rn(e, y, q0);
  return __float_as_uint(__fadd_rn(q1, kRintMagic));
}

__device__ __forceinline__ uint2 pack_codes(const uint32_t (&c)[8]) {
  uint2 out;
  out.x = __byte_perm(__byte_perm(c[0], c[1], 0x0040), __byte_perm(c[2], c[3], 0x0040), 0x5410);
  out.y = __byte_perm(__byte_perm(c[4], c[5], 0x0040), __byte_perm(c[6], c[7], 0x0040), 0x5410);
  return out;
}

// One 16-byte vector of 8 bf16 -> 8 fp32 (exact widening).
__device__ __forceinline__ void unpack8(uint4 v, float (&x)[8]) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    x[2 * i] = __uint_as_float(w[i] << 16);
    x[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}

// max(m, |x_i|): fmaxf returns one of its operands unchanged, so the maximum
// is exact (subnormals included: nothing is compiled with flush-to-zero).
__device__ __forceinline__ float absmax8(const float (&x)[8], float m) {
#pragma unroll
  for (int i = 0; i < 8; ++i) m = fmaxf(m, fabsf(x[i]));
  return m;
}

// 8 bf16 (one 16-byte vector) -> 8 int8 codes (8 bytes).  s > 0; y = RN(1/s);
// fast = the row's scale is in the range where quant_fast is exact (a
// row-uniform choice, so there is no divergence inside a row).
__device__ __forceinline__ uint2 quant_vec8(uint4 v, float s, float y, bool fast) {
  float x[8];
  unpack8(v, x);
  uint32_t c[8];
  if (fast) {
#pragma unroll
    for (int i = 0; i < 8; ++i) c[i] = quant_fast(x[i], s, y);
  } else {
#pragma unroll
    for (int i = 0; i < 8; ++i) c[i] = quant_exact(x[i], s);
  }
  return pack_codes(c);
}

// Per-row constants of the fast path.
__device__ __forceinline__ bool quant_fast_ok(float s) {
  return s >= 7.8886090522101181e-31f /* 2^-100 */ && s <= 2.6584559915698317e+36f /* 2^121 */;
}

// Largest |x| of a 16-byte vector of 8 bf16, accumulated into m.
__device__ __forceinline__ float absmax_vec8(uint4 v, float m) {
  float x[8];
  unpack8(v, x);
  return absmax8(x, m);
}

// Non-negative floats order like their bit patterns: reductions across lanes
// run on the bits.
__device__ __forceinline__ uint32_t warp_max_u32(uint32_t v, int width) {
  for (int o = width >> 1; o > 0; o >>= 1) v = max(v, __shfl_xor_sync(0xFFFFFFFFu, v, o));
  return v;
}

// One warp quantizes one row of K elements (K % 8 == 0) into qr / *s_out.
// Rows of up to 32 x V vectors of 8 stay in registers (x read once); longer
// rows take two passes, max |x| first, then the codes (the second pass reading
// the row back from L2).  All 32 lanes must call it.
template <int V>
__device__ __forceinline__ void quant_row_by_warp(const uint16_t *__restrict__ xr, int K,
                                                  int8_t *__restrict__ qr, float *s_out,
                                                  int lane) {
  const int nvec = K >> 3;
  const uint4 *xv = reinterpret_cast<const uint4 *>(xr);
  uint2 *qv = reinterpret_cast<uint2 *>(qr);
  if (nvec <= 32 * V) {
    uint4 v[V];
#pragma unroll
    for (int j = 0; j < V; ++j) {
      const int vi = lane + 32 * j;
      v[j] = vi < nvec ? __ldcs(xv + vi) : make_uint4(0u, 0u, 0u, 0u);
    }
    float m0 = 0.0f, m1 = 0.0f;
#pragma unroll
    for (int j = 0; j < V; ++j) {
      if (j & 1) m1 = absmax_vec8(v[j], m1); else m0 = absmax_vec8(v[j], m0);
    }
    const float amax = __uint_as_float(warp_max_u32(__float_as_uint(fmaxf(m0, m1)), 32));
    const float sc = (amax == 0.0f) ? 0.0f : __fdiv_rn(amax, 127.0f);
    const bool fast = quant_fast_ok(sc);
    const float rc = fast ? __frcp_rn(sc) : 0.0f;
    if (lane == 0) *s_out = sc;
#pragma unroll
    for (int j = 0; j < V; ++j) {
      const int vi = lane + 32 * j;
      if (vi < nvec) qv[vi] = (sc == 0.0f) ? make_uint2(0u, 0u) : quant_vec8(v[j], sc, rc, fast);
    }
  } else {
    float m = 0.0f;
    for (int vi = lane; vi < nvec; vi += 32) m = absmax_vec8(__ldg(xv + vi), m);
    const float amax = __uint_as_float(warp_max_u32(__float_as_uint(m), 32));
    const float sc = (amax == 0.0f) ? 0.0f : __fdiv_rn(amax, 127.0f);
    const bool fast = quant_fast_ok(sc);
    const float rc = fast ? __frcp_rn(sc) : 0.0f;
    if (lane == 0) *s_out = sc;
    for (int vi = lane; vi < nvec; vi += 32)
      qv[vi] = (sc == 0.0f) ? make_uint2(0u, 0u) : quant_vec8(__ldcs(xv + vi), sc, rc, fast);
  }
}

// Very long rows (K > 24576): one block of 256 threads per row, two passes
// over the row -- max |x| first, then quantize -- the second pass reading the
// row back from L2.
__global__ void __launch_bounds__(256) quant_rows_long_kernel(const uint16_t *__restrict__ x,
                                                              int64_t K, int64_t ldx,
                                                              int8_t *__restrict__ q,
                                                              float *__restrict__ s,
                                                              int release_early) {
  __shared__ uint32_t red[8];
  const int64_t row = blockIdx.x;
  const int tid = threadIdx.x;
  const int64_t nvec = K >> 3;
  const uint4 *xr = reinterpret_cast<const uint4 *>(x + row * ldx);
  if (release_early) grid_dependents_launch();  // see quant_rows_kernel
  grid_dependency_wait();
  float m = 0.0f;
  for (int64_t vi = tid; vi < nvec; vi += 256) m = absmax_vec8(__ldg(xr + vi), m);
  uint32_t mb = warp_max_u32(__float_as_uint(m), 32);
  if ((tid & 31) == 0) red[tid >> 5] = mb;
  __syncthreads();
  mb = 0u;
#pragma unroll
  for (int w = 0; w < 8; ++w) mb = max(mb, red[w]);
  const float amax = __uint_as_float(mb);
  const float sc = (amax == 0.0f) ? 0.0f : __fdiv_rn(amax, 127.0f);
  const bool fast = quant_fast_ok(sc);
  const float rc = fast ? __frcp_rn(sc) : 0.0f;
  if (tid == 0) s[row] = sc;
  uint2 *qr = reinterpret_cast<uint2 *>(q + row * K);
  for (int64_t vi = tid; vi < nvec; vi += 256) {
    const uint4 v = __ldcs(xr + vi);
    qr[vi] = (sc == 0.0f) ? make_uint2(0u, 0u) : quant_vec8(v, sc, rc, fast);
  }
}

// ---------------------------------------------------------------------------
// The hot-path kernel for rows of up to kQuantBulkMaxK elements: one CTA of 16
// warps per SM, persistent.  A group of G warps (G = 1, 2 or 4: at most 3072
// elements per warp) owns one row at a time; rows reach shared memory by bulk
// copies (one cp.async.bulk per row), S slots per group, so each group has S
// rows in flight and the CTA 16 / G * S * 2K bytes -- the whole CTA's share of
// a 4352 x 3072 layer is requested at once.  Group g of CTA c takes rows
// c * groups + g + i * gridDim.x * groups, i = 0, 1, ..., so rows complete
// roughly in order across the GPU.  Per row: max |x| on bf16 bit patterns
// (sign cleared, 16x2 integer maxima), across the group's lanes and warps;
// the scale and its reciprocal; then the codes with the division-free step in
// packed fp32x2 arithmetic, 8 bytes per lane per store.  Every slot wait is
// bounded; on expiry the group waits for its copies in flight and the kernel
// returns with the device error word set.
constexpr int kQuantBulkMaxK = 12288;
constexpr int kQuantBulkSmem = 196608;   // slot storage per CTA
constexpr int kQuantBulkWarps = 16;
constexpr int kQuantBulkMaxSlots = 4;
constexpr int kQuantBulkWarpElems = 3072;  // elements of a row per warp, at most

__device__ __forceinline__ uint32_t max_u16x2(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("max.u16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

__device__ __forceinline__ float2 fma2_rn(float2 a, float2 b, float2 c) {
  float2 d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;"
      : "=l"(reinterpret_cast<uint64_t &>(d))
      : "l"(reinterpret_cast<const uint64_t &>(a)), "l"(reinterpret_cast<const uint64_t &>(b)),
        "l"(reinterpret_cast<const uint64_t &>(c)));
  return d;
}

__device__ __forceinline__ float2 mul2_rn_q(float2 a, float2 b) {
  float2 d;
  asm("mul.rn.f32x2 %0, %1, %2;"
      : "=l"(reinterpret_cast<uint64_t &>(d))
      : "l"(reinterpret_cast<const uint64_t &>(a)), "l"(reinterpret_cast<const uint64_t &>(b)));
  return d;
}

__device__ __forceinline__ float2 add2_rn_q(float2 a, float2 b) {
  float2 d;
  asm("add.rn.f32x2 %0, %1, %2;"
      : "=l"(reinterpret_cast<uint64_t &>(d))
      : "l"(reinterpret_cast<const uint64_t &>(a)), "l"(reinterpret_cast<const uint64_t &>(b)));
  return d;
}

// max |x| of 8 bf16 as packed 16x2 bit patterns, accumulated into m.
__device__ __forceinline__ uint32_t absmax_bits8(uint4 v, uint32_t m) {
  m = max_u16x2(m, v.x & 0x7FFF7FFFu);
  m = max_u16x2(m, v.y & 0x7FFF7FFFu);
  m = max_u16x2(m, v.z & 0x7FFF7FFFu);
  return max_u16x2(m, v.w & 0x7FFF7FFFu);
}

// The division-free step (quant_fast) on two values at once: each lane of
// every packed operation is the same separately rounded operation.  neg_s =
// (-s, -s): x - q0 * s == fma(q0, -s, x), exactly.
__device__ __forceinline__ uint2 quant_vec8_x2(uint4 v, float2 neg_s, float2 y) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  const float2 magic = make_float2(kRintMagic, kRintMagic);
  uint32_t c[8];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 x = make_float2(__uint_as_float(w[i] << 16), __uint_as_float(w[i] & 0xFFFF0000u));
    const float2 q0 = mul2_rn_q(x, y);
    const float2 e = fma2_rn(q0, neg_s, x);
    const float2 q1 = fma2_rn(e, y, q0);
    const float2 r = add2_rn_q(q1, magic);
    c[2 * i] = __float_as_uint(r.x);
    c[2 * i + 1] = __float_as_uint(r.y);
  }
  return pack_codes(c);
}

// One warp quantizes one row of K elements held in shared memory (16-byte
// aligned) into qr / *s_out: the bulk kernel's per-row step for one warp.
__device__ __forceinline__ void quant_row_from_smem(const uint4 *xs, int K, int8_t *qr,
                                                    float *s_out, int lane) {
  const int nvec = K >> 3;
  uint32_t m0 = 0u, m1 = 0u;
  int vi = lane;
  for (; vi + 32 < nvec; vi += 64) {
    m0 = absmax_bits8(xs[vi], m0);
    m1 = absmax_bits8(xs[vi + 32], m1);
  }
  if (vi < nvec) m0 = absmax_bits8(xs[vi], m0);
  uint32_t mb = max_u16x2(m0, m1);
  mb = warp_max_u32(max(mb & 0xFFFFu, mb >> 16), 32);
  const float amax = __uint_as_float(mb << 16);
  const float sc = (amax == 0.0f) ? 0.0f : __fdiv_rn(amax, 127.0f);
  const bool fast = quant_fast_ok(sc);
  const float rc = fast ? __frcp_rn(sc) : 0.0f;
  if (lane == 0) *s_out = sc;
  uint2 *qv = reinterpret_cast<uint2 *>(qr);
  if (sc == 0.0f) {
    for (int v = lane; v < nvec; v += 32) qv[v] = make_uint2(0u, 0u);
  } else if (fast) {
    const float2 neg_s = make_float2(-sc, -sc), y2 = make_float2(rc, rc);
#pragma unroll 2
    for (int v = lane; v < nvec; v += 32) qv[v] = quant_vec8_x2(xs[v], neg_s, y2);
  } else {
    for (int v = lane; v < nvec; v += 32) qv[v] = quant_vec8(xs[v], sc, rc, false);
  }
}

__global__ void __launch_bounds__(kQuantBulkWarps * 32, 1)
    quant_rows_bulk_kernel(const uint16_t *__restrict__ x, int rows, int K, int64_t ldx,
                           int8_t *__restrict__ q, float *__restrict__ s, int group_warps,
                           int slots, int release_early) {
  extern __shared__ __align__(128) uint8_t quant_slots[];
  __shared__ uint64_t bars[kQuantBulkWarps * kQuantBulkMaxSlots];
  __shared__ uint32_t red[kQuantBulkWarps];
  __shared__ int okf[kQuantBulkWarps];
  __shared__ int abort_flag;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = group_warps;
  const int groups = kQuantBulkWarps / G;
  const int group = warp / G, gw = warp % G;    // gw: this warp's index in its group
  const bool leader = gw == 0 && lane == 0;
  const uint32_t row_bytes = static_cast<uint32_t>(K) * 2u;
  uint8_t *mine = quant_slots + static_cast<size_t>(group) * slots * row_bytes;
  uint64_t *bar = bars + group * kQuantBulkMaxSlots;
  const int stride = static_cast<int>(gridDim.x) * groups;
  const int first = static_cast<int>(blockIdx.x) * groups + group;
  const int n_rows = first < rows ? (rows - first + stride - 1) / stride : 0;
  if (threadIdx.x == 0) abort_flag = 0;
  if (leader)
    for (int j = 0; j < slots; ++j) mbar_init(&bar[j], 1);
  fence_mbarrier_init();
  __syncthreads();
  // see quant_rows_kernel
  if (release_early) grid_dependents_launch();
  grid_dependency_wait();
  int issued = 0;
  if (leader) {
    for (; issued < slots && issued < n_rows; ++issued) {
      const int64_t row = first + static_cast<int64_t>(issued) * stride;
      mbar_arrive_expect_tx(&bar[issued], row_bytes);
      bulk_load_g2s(mine + issued * row_bytes, x + row * ldx, row_bytes, &bar[issued]);
    }
  }
  const int nvec = K >> 3;
  const int gthreads = G * 32;
  const int t = gw * 32 + lane;   // thread index within the group
  int i = 0;
  for (; i < n_rows; ++i) {
    const int slot = i % slots;
    int ok = mbar_wait(&bar[slot], static_cast<uint32_t>(i / slots) & 1u, &abort_flag) ? 1 : 0;
    ok = __all_sync(0xFFFFFFFFu, ok);
    if (G > 1) {  // the group's warps leave together or not at all
      if (lane == 0) okf[warp] = ok;
      named_barrier_sync(1 + group, gthreads);
      for (int w = 0; w < G; ++w) ok &= okf[group * G + w];
    }
    if (!ok) break;
    const int64_t row = first + static_cast<int64_t>(i) * stride;
    const uint4 *xs = reinterpret_cast<const uint4 *>(mine + slot * row_bytes);
    uint32_t m0 = 0u, m1 = 0u;
    int vi = t;
    for (; vi + gthreads < nvec; vi += 2 * gthreads) {
      m0 = absmax_bits8(xs[vi], m0);
      m1 = absmax_bits8(xs[vi + gthreads], m1);
    }
    if (vi < nvec) m0 = absmax_bits8(xs[vi], m0);
    uint32_t mb = max_u16x2(m0, m1);
    mb = warp_max_u32(max(mb & 0xFFFFu, mb >> 16), 32);
    if (G > 1) {  // across the group's warps
      if (lane == 0) red[warp] = mb;
      named_barrier_sync(1 + group, gthreads);
      mb = 0u;
      for (int w = 0; w < G; ++w) mb = max(mb, red[group * G + w]);
    }
    const float amax = __uint_as_float(mb << 16);
    const float sc = (amax == 0.0f) ? 0.0f : __fdiv_rn(amax, 127.0f);
    const bool fast = quant_fast_ok(sc);
    const float rc = fast ? __frcp_rn(sc) : 0.0f;
    if (t == 0) s[row] = sc;
    uint2 *qr = reinterpret_cast<uint2 *>(q + row * K);
    if (sc == 0.0f) {
      for (int v = t; v < nvec; v += gthreads) qr[v] = make_uint2(0u, 0u);
    } else if (fast) {
      const float2 neg_s = make_float2(-sc, -sc), y2 = make_float2(rc, rc);
#pragma unroll 2
      for (int v = t; v < nvec; v += gthreads) qr[v] = quant_vec8_x2(xs[v], neg_s, y2);
    } else {
      for (int v = t; v < nvec; v += gthreads) qr[v] = quant_vec8(xs[v], sc, rc, false);
    }
    // every thread of the group is done with the slot (and with red[])
    // before the slot is refilled
    if (G > 1) named_barrier_sync(1 + group, gthreads); else __syncwarp();
    if (leader && issued < n_rows) {
      const int64_t nrow = first + static_cast<int64_t>(issued) * stride;
      mbar_arrive_expect_tx(&bar[slot], row_bytes);
      bulk_load_g2s(mine + slot * row_bytes, x + nrow * ldx, row_bytes, &bar[slot]);
      ++issued;
    }
  }
  if (i < n_rows && leader) {
    // gave up: let the copies still in flight land before the CTA leaves
    volatile int never = 0;
    for (int j = i; j < issued; ++j)
      mbar_wait(&bar[j % slots], static_cast<uint32_t>(j / slots) & 1u, &never);
  }
}

// Rows longer than kQuantBulkMaxK: a group of G threads owns one row (G = 32,
// one warp, whenever the row fits in 12 vectors per lane).  Each
// thread issues all of its V 16-byte loads at once (evict-first: the
// activations are read exactly once), reduces max |x| in registers and across
// the group (shuffles; shared memory when G > 32), then quantizes its
// registers with the division-free step and writes 8 int8 per vector.  The
// row's scale needs one IEEE division and one reciprocal per warp.
template <int V>
__global__ void __launch_bounds__(256) quant_rows_kernel(const uint16_t *__restrict__ x,
                                                         int rows, int K, int64_t ldx,
                                                         int8_t *__restrict__ q,
                                                         float *__restrict__ s, int G,
                                                         int release_early) {
  __shared__ uint32_t red[8];
  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int group = tid / G;       // row within the block
  const int t = tid % G;           // thread within the row group
  const int rows_per_block = blockDim.x / G;
  const int row = blockIdx.x * rows_per_block + group;
  const bool row_ok = row < rows;
  const int nvec = K >> 3;

  const uint4 *xr = reinterpret_cast<const uint4 *>(x + (row_ok ? row : 0) * ldx);
  // Launched as a programmatic dependent: x may come from the preceding
  // kernel, and q / s may still be read by it -- wait before either.  With
  // release_early (activations), the kernel that follows may be launched at
  // once: the library's GEMM, GEMV and small-M kernels read only the weights
  // before their own dependency wait, which completes after this kernel (and,
  // through this kernel's wait, the one before it).  Without (weights: the
  // kernel that follows prefetches the very Wq written here), dependents
  // start only when this grid has completed.
  if (release_early) grid_dependents_launch();
  grid_dependency_wait();
  uint4 v[V];
#pragma unroll
  for (int j = 0; j < V; ++j) {
    const int vi = t + j * G;
    v[j] = (row_ok && vi < nvec) ? __ldcs(xr + vi) : make_uint4(0u, 0u, 0u, 0u);
  }
  float m0 = 0.0f, m1 = 0.0f;
#pragma unroll
  for (int j = 0; j < V; ++j) {
    if (j & 1) m1 = absmax_vec8(v[j], m1); else m0 = absmax_vec8(v[j], m0);
  }
  uint32_t mb = warp_max_u32(__float_as_uint(fmaxf(m0, m1)), 32);
  if (G > 32) {  // G is uniform in the block
    if (lane == 0) red[warp] = mb;
    __syncthreads();
    const int wpg = G >> 5;
    mb = 0u;
    for (int w = 0; w < wpg; ++w) mb = max(mb, red[group * wpg + w]);
  }
  if (!row_ok) return;
  const float amax = __uint_as_float(mb);
  const float sc = (amax == 0.0f) ? 0.0f : __fdiv_rn(amax, 127.0f);
  const bool fast = quant_fast_ok(sc);
  const float rc = fast ? __frcp_rn(sc) : 0.0f;
  if (t == 0) s[row] = sc;
  uint2 *qr = reinterpret_cast<uint2 *>(q + static_cast<int64_t>(row) * K);
#pragma unroll
  for (int j = 0; j < V; ++j) {
    const int vi = t + j * G;
    if (vi < nvec) qr[vi] = (sc == 0.0f) ? make_uint2(0u, 0u) : quant_vec8(v[j], sc, rc, fast);
  }
}

}  // namespace w8a8
