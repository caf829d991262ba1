// w8a8_peak.cuh -- the int8 tensor-core ceiling of the device, measured.
//
// The GEMM's roofline needs the dense kind::i8 rate this B200 actually
// delivers, at the clock it holds under that load.  This kernel issues the
// GEMM's own instruction -- tcgen05.mma.cta_group::2.kind::i8, M = 256,
// N = 256, K = 32 -- back to back on every CTA pair, from operands that stay
// in shared memory (filled once with pseudo-random bytes, so the datapath
// switches as it does on real data), into one TMEM accumulator.  There is no
// global-memory traffic and no epilogue: the time is the tensor pipe's alone.
// Each instruction is 2 * 256 * 256 * 32 = 4,194,304 int8 operations per pair.
#pragma once

#include <cstdint>

#include "w8a8_gemm.cuh"
#include "w8a8_ptx.cuh"

namespace w8a8 {

constexpr int kPeakThreads = 128;
constexpr int kPeakOperandBytes = 2 * kBM * kBK;  // A (128 rows) + B (128 rows), per CTA
constexpr int kPeakSmemBytes = kPeakOperandBytes + 1024;
constexpr double kPeakOpsPerMma = 2.0 * 256 * 256 * kMmaK;

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kPeakThreads, 1)
    mma_i8_peak_kernel(int64_t iterations) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ uint64_t done;
  __shared__ uint32_t tmem_slot;
  __shared__ int abort_flag;
  const uint32_t raw_addr = smem_addr(smem_raw);
  uint8_t *smem = smem_raw + ((1024u - (raw_addr & 1023u)) & 1023u);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();

  // operands: a 32-bit integer hash of the byte offset and the block
  uint32_t *words = reinterpret_cast<uint32_t *>(smem);
  for (int i = threadIdx.x; i < kPeakOperandBytes / 4; i += kPeakThreads) {
    uint32_t h = static_cast<uint32_t>(i) * 0x9E3779B1u + blockIdx.x * 0x85EBCA77u;
    h ^= h >> 15;
    h *= 0x2C1B3C6Du;
    h ^= h >> 12;
    words[i] = h;
  }
  fence_proxy_async_smem();  // generic writes -> visible to the tensor core
  if (threadIdx.x == 0) {
    mbar_init(&done, 1);
    abort_flag = 0;
    fence_mbarrier_init();
  }
  if (warp == 0) {
    tmem_alloc_pair(&tmem_slot, 256);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync();
  tc_fence_after();
  const uint32_t tmem_base = tmem_slot;

  if (warp == 1 && lane == 0) {
    if (rank == 0) {
      constexpr uint32_t idesc = idesc_i8(2 * kBM, 256);
      const uint32_t sa = smem_addr(smem);
      const uint64_t adesc = smem_desc_k_sw128(sa);
      const uint64_t bdesc = smem_desc_k_sw128(sa + kBM * kBK);
      for (int64_t it = 0; it < iterations; ++it) {
#pragma unroll
        for (int k = 0; k < kBK / kMmaK; ++k)
          mma_i8_pair(tmem_base, adesc + 2u * k, bdesc + 2u * k, idesc, (it | k) != 0 ? 1u : 0u);
      }
      mma_commit_pair(&done, 0x3);  // arrives in both CTAs once every MMA has completed
    }
    // bounded: a wait that gives up records the timeout in the error word
    mbar_wait(&done, 0u, &abort_flag);
  }
  tc_fence_before();
  cluster_sync();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, 256);
  }
}

}  // namespace w8a8
