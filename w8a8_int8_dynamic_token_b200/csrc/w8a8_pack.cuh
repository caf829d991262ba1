// w8a8_pack.cuh -- loading int8 weights from their packed int32 storage.
//
// A serialized W8A8 checkpoint stores each int8 weight code as an unsigned
// byte biased by 128, four per int32 word ("Issue 5 probe: int8 quantized DiT
// serve paths on the RTX 3090 (24 GB)", section "Artifact (outside Git, under
// the helper state root)": the quantized transformer is built with
// compressed-tensors' pack_to_int32).  Codes run along K,
// the first of each group of four in the least significant byte, so on a
// little-endian device the packed array's bytes, in memory order, are
// (code + 128) mod 256 = code XOR 0x80: unpacking is a byte-wise XOR that
// leaves the layout as it is (int8 [N, K], K-major, the GEMM's B operand).
//
// HBM-bound: N*K bytes read, N*K bytes written.
#pragma once

#include <cstdint>

namespace w8a8 {

__global__ void __launch_bounds__(256) unpack_int32_weights_kernel(const uint4 *__restrict__ packed,
                                                                   uint4 *__restrict__ wq,
                                                                   int64_t n16) {
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n16;
       i += stride) {
    uint4 v = __ldcs(packed + i);
    v.x ^= 0x80808080u;
    v.y ^= 0x80808080u;
    v.z ^= 0x80808080u;
    v.w ^= 0x80808080u;
    __stcs(wq + i, v);
  }
}

}  // namespace w8a8
