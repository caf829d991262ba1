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
// Layout of the work: a group of G threads owns one row.  Each thread loads V
// 16-byte vectors (8 bf16 each) of the row into registers with streaming
// loads, so the row is read from HBM exactly once; the group reduces max |x|
// as an integer max of bit patterns (packed 16-bit max, warp shuffles and,
// for G > 32, shared memory); then every
// thread quantizes its registers and writes 8 int8 per vector.
//
// Rounding: rint(t) for |t| <= 127.0001 is formed exactly by adding and
// subtracting 1.5 * 2^23 in round-to-nearest-even fp32 arithmetic; the low
// byte of (t + 1.5 * 2^23)'s bit pattern is then the two's-complement int8.
#pragma once

#include <cuda_bf16.h>
#include <cstdint>

namespace w8a8 {

constexpr float kRintMagic = 12582912.0f;  // 1.5 * 2^23

// Quantize two bf16 (packed in one 32-bit word) with scale s; returns the two
// int8 codes in the low bytes of two words (as bit patterns of t + magic).
__device__ __forceinline__ void quant_pair(uint32_t packed, float s, uint32_t &c0, uint32_t &c1) {
  const float v0 = __uint_as_float(packed << 16);
  const float v1 = __uint_as_float(packed & 0xFFFF0000u);
  float t0 = __fdiv_rn(v0, s);
  float t1 = __fdiv_rn(v1, s);
  t0 = fminf(fmaxf(t0, -127.0f), 127.0f);
  t1 = fminf(fmaxf(t1, -127.0f), 127.0f);
  c0 = __float_as_uint(__fadd_rn(t0, kRintMagic));
  c1 = __float_as_uint(__fadd_rn(t1, kRintMagic));
}

// 8 bf16 (one 16-byte vector) -> 8 int8 (8 bytes).
__device__ __forceinline__ uint2 quant_vec8(uint4 v, float s) {
  uint32_t c[8];
  quant_pair(v.x, s, c[0], c[1]);
  quant_pair(v.y, s, c[2], c[3]);
  quant_pair(v.z, s, c[4], c[5]);
  quant_pair(v.w, s, c[6], c[7]);
  uint2 out;
  out.x = __byte_perm(__byte_perm(c[0], c[1], 0x0040), __byte_perm(c[2], c[3], 0x0040), 0x5410);
  out.y = __byte_perm(__byte_perm(c[4], c[5], 0x0040), __byte_perm(c[6], c[7], 0x0040), 0x5410);
  return out;
}

// max |x| on packed bf16 pairs, exactly: with the sign bit cleared, the
// order of IEEE bit patterns is the order of the values, so a per-half
// unsigned 16-bit max of (bits & 0x7FFF) is the max of |x| (subnormals too).
__device__ __forceinline__ uint32_t bf16x2_absmax(uint32_t acc, uint32_t v) {
  return __vmaxu2(acc, v & 0x7FFF7FFFu);
}

__device__ __forceinline__ uint32_t bf16x2_max_halves(uint32_t m) {
  const uint32_t hi = m >> 16, lo = m & 0xFFFFu;
  return hi > lo ? hi : lo;
}

// x: [rows, K] bf16 (row stride ldx elements); q: [rows, K] int8 dense;
// s: [rows] fp32.  Block = rows_per_block groups of G threads.
template <int V>
__global__ void __launch_bounds__(256) quant_rows_kernel(const uint16_t *__restrict__ x,
                                                         int64_t rows, int64_t K, int64_t ldx,
                                                         int8_t *__restrict__ q,
                                                         float *__restrict__ s, int G) {
  __shared__ uint32_t red[32];
  const int tid = threadIdx.x;
  const int group = tid / G;  // row within the block
  const int t = tid % G;      // thread within the row group
  const int rows_per_block = blockDim.x / G;
  const int64_t row = static_cast<int64_t>(blockIdx.x) * rows_per_block + group;
  const bool row_ok = row < rows;
  const int64_t nvec = K >> 3;

  const uint4 *xr = reinterpret_cast<const uint4 *>(x + (row_ok ? row : 0) * ldx);
  uint4 v[V];
  uint32_t m = 0u;
#pragma unroll
  for (int j = 0; j < V; ++j) {
    const int64_t vi = t + static_cast<int64_t>(j) * G;
    if (row_ok && vi < nvec) {
      v[j] = __ldcs(xr + vi);
    } else {
      v[j] = make_uint4(0u, 0u, 0u, 0u);
    }
    m = bf16x2_absmax(m, v[j].x);
    m = bf16x2_absmax(m, v[j].y);
    m = bf16x2_absmax(m, v[j].z);
    m = bf16x2_absmax(m, v[j].w);
  }
  // the reduction runs on the bit patterns of |x| (unsigned order = value order)
  uint32_t mb = bf16x2_max_halves(m);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) mb = max(mb, __shfl_xor_sync(0xFFFFFFFFu, mb, o));
  if (G > 32) {
    const int warp = tid >> 5, lane = tid & 31;
    if (lane == 0) red[warp] = mb;
    __syncthreads();
    const int wpg = G >> 5;  // warps per group
    const int first = group * wpg;
    mb = 0u;
    for (int w = 0; w < wpg; ++w) mb = max(mb, red[first + w]);
  }
  if (!row_ok) return;
  const float amax = __uint_as_float(mb << 16);

  const float sc = (amax == 0.0f) ? 0.0f : __fdiv_rn(amax, 127.0f);
  if (t == 0) s[row] = sc;
  uint2 *qr = reinterpret_cast<uint2 *>(q + row * K);
#pragma unroll
  for (int j = 0; j < V; ++j) {
    const int64_t vi = t + static_cast<int64_t>(j) * G;
    if (vi < nvec) {
      uint2 o = (sc == 0.0f) ? make_uint2(0u, 0u) : quant_vec8(v[j], sc);
      qr[vi] = o;
    }
  }
}

// Long rows (more than 256 threads x 8 vectors): one block of 256 threads per
// row, two passes over the row -- max |x| first, then quantize -- the second
// pass reading the row back from L2.
__global__ void __launch_bounds__(256) quant_rows_long_kernel(const uint16_t *__restrict__ x,
                                                              int64_t K, int64_t ldx,
                                                              int8_t *__restrict__ q,
                                                              float *__restrict__ s) {
  __shared__ uint32_t red[8];
  const int64_t row = blockIdx.x;
  const int tid = threadIdx.x;
  const int64_t nvec = K >> 3;
  const uint4 *xr = reinterpret_cast<const uint4 *>(x + row * ldx);
  uint32_t m = 0u;
  for (int64_t vi = tid; vi < nvec; vi += 256) {
    const uint4 v = __ldg(xr + vi);
    m = bf16x2_absmax(m, v.x);
    m = bf16x2_absmax(m, v.y);
    m = bf16x2_absmax(m, v.z);
    m = bf16x2_absmax(m, v.w);
  }
  uint32_t mb = bf16x2_max_halves(m);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) mb = max(mb, __shfl_xor_sync(0xFFFFFFFFu, mb, o));
  if ((tid & 31) == 0) red[tid >> 5] = mb;
  __syncthreads();
  mb = 0u;
#pragma unroll
  for (int w = 0; w < 8; ++w) mb = max(mb, red[w]);
  const float amax = __uint_as_float(mb << 16);
  const float sc = (amax == 0.0f) ? 0.0f : __fdiv_rn(amax, 127.0f);
  if (tid == 0) s[row] = sc;
  uint2 *qr = reinterpret_cast<uint2 *>(q + row * K);
  for (int64_t vi = tid; vi < nvec; vi += 256) {
    const uint4 v = __ldcs(xr + vi);
    qr[vi] = (sc == 0.0f) ? make_uint2(0u, 0u) : quant_vec8(v, sc);
  }
}

}  // namespace w8a8
