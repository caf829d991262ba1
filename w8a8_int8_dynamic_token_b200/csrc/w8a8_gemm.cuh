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
//   warps 2..9  the epilogue, two warps per 32-lane TMEM quarter (a warp may
//               only read the quarter its index selects), each taking half of
//               the tile's columns in chunks of 32: tcgen05.ld, the fp32
//               scale/bias math, bf16 packing into a 64-byte-swizzled staging
//               buffer in shared memory, and a TMA store of the 32 x 32 box
//               (two staging buffers per warp, so the store of one chunk
//               overlaps the math of the next).  After its last chunk a warp
//               releases the accumulator, so the next tile's MMAs overlap the
//               epilogue of this one.
// Ragged edges: TMA zero-fills rows/columns outside the tensors on load (zeros
// add nothing to an integer dot product) and clips them on store.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cstdint>

#include "w8a8_ptx.cuh"
#include "w8a8_quant.cuh"

namespace w8a8 {

constexpr int kGemmThreads = 320;   // 2 + 8 warps
constexpr int kEpiWarps = 8;
constexpr int kEpiChunk = 32;        // columns per epilogue step
constexpr int kEpiBufBytes = 32 * kEpiChunk * 2;  // 32 rows x 32 bf16
constexpr int kBM = 128;   // rows of y per tile (TMEM lanes)
constexpr int kBK = 128;   // int8 K elements per stage = one 128-byte swizzle row
constexpr int kMmaK = 32;  // K per tcgen05.mma kind::i8
constexpr int kPairBN = 256;  // columns of a CTA-pair tile

template <int BN, int STAGES>
struct GemmLayout {
  static constexpr int kABytes = kBM * kBK;
  static constexpr int kBBytes = BN * kBK;
  static constexpr int kStageBytes = kABytes + kBBytes;
  static constexpr int kTileBytes = STAGES * kStageBytes;
  static constexpr int kEpiOffset = kTileBytes;  // 1024-aligned
  static constexpr int kEpiBytes = kEpiWarps * 2 * kEpiBufBytes;
  static constexpr int kBarOffset = kEpiOffset + kEpiBytes;
  // full[STAGES], empty[STAGES], tfull[2], tempty[2], drain, then two words
  static constexpr int kBarBytes = (2 * STAGES + 5) * 8 + 8;
  static constexpr int kSmemBytes = kBarOffset + kBarBytes + 1024;  // + alignment slack
  static constexpr int kTmemCols = 2 * BN;                          // two accumulators
  static_assert(kSmemBytes <= 232448, "shared memory budget");
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
  // CTA-pair kernel only.  Tiles [0, dp_tiles) are whole-tile work in full
  // rounds (pair j takes tiles j, j + pairs, ...).  The remaining tiles, when
  // there are any, form the tail, handled in one of two ways:
  //  - split along N (tail_nsplit = 2 or 4): each tail tile becomes
  //    tail_nsplit tiles 256/tail_nsplit columns wide, one per pair;
  //  - split along K (sk_per > 0): their k-blocks, in (tile, k-block) order,
  //    form sk_units units and pair j takes the units [j * sk_per,
  //    (j + 1) * sk_per).  A tile worked on by several pairs is finished by
  //    the last of them to arrive (per epilogue warp slice, elected by an
  //    arrival counter), which adds the others' int32 partial sums from
  //    split_partials.
  int32_t dp_tiles;        // == num_tiles: no tail
  int32_t tail_nsplit;     // 1 (no N split), 2 or 4
  int32_t sk_per;          // K split: units per pair, 0 = no K split
  int32_t sk_units;        // (num_tiles - dp_tiles) * k_blocks
  int32_t *split_partials; // (num_tiles - dp_tiles + pairs - 1) slots of 16 slices
  // (num_tiles - dp_tiles) x 16 counters, each (tag << 8) | arrivals,
  // cleared by the host before the launch.  A counter whose tag is not this
  // launch's split_epoch counts as 0 as well; the electing contribution
  // resets it to 0.
  unsigned long long *split_counters;
  unsigned long long split_epoch;  // 1 .. 2^56 - 1
  // CTA-pair kernel with the per-token quantization fused in (K <= 12288):
  // the epilogue warps of all CTAs quantize the rows of x (bf16 [M, K], row
  // stride ldx) into q_w / s_a_w -- the buffers the GEMM then reads through
  // tmap_a and s_a.  In pass j, CTA c takes rows 8 c .. 8 c + 7 + j * 8 *
  // gridDim.x (one per epilogue warp), so the 128-row blocks complete in
  // order; after each pass one thread of the CTA adds its rows to the block's
  // counter, (fuse_tag << 16) | rows (the host clears the counters before the
  // launch, and a counter holding another launch's tag counts as 0).  A
  // producer waits for its block's count before loading q.  Rows below
  // fuse_bulk_rows (those the first round of tiles reads) are brought into
  // the still unused operand ring by bulk copies, every warp's rows at once;
  // the producer starts filling the ring once every epilogue warp is done
  // with it.  Later rows are read into registers while the first tiles' MMAs
  // run, and between passes the warps take the epilogue of any tile whose
  // accumulator is ready.
  const uint16_t *x;
  int64_t ldx;
  int8_t *q_w;
  float *s_a_w;
  unsigned long long *row_ready;   // cdiv(M, 128) counters
  unsigned long long fuse_tag;     // 1 .. 2^48 - 1
  int32_t fuse_bulk_rows;          // rows [0, fuse_bulk_rows) take the bulk path
};

// One epilogue warp slice of a 256 x 256 pair tile: 32 rows x 128 columns.
constexpr int kSlotInts = 32 * 128;
constexpr int kSlicesPerTile = 16;  // 2 CTAs x 8 epilogue warps

// The i-th work item of a CTA pair: a whole tile, a narrow tail tile (a
// column range of a tile), or a run of k-blocks of a tile shared out along K.
// Returns false past the pair's last item.
struct WorkItem {
  int tile;        // tile index (row/column block via pair_tile_coords)
  int kb_begin, kb_end;
  int n_off;       // first column of the item within the tile
  int ncols;       // columns of the item: 256, or 256 / tail_nsplit
  int t_rel;       // tile - dp_tiles (K-split tiles only)
  int nparts;      // pairs contributing to this tile along K (1: all of K)
  int part;        // this pair's index among them, in k order
};

__device__ __forceinline__ bool pair_work_item(const GemmParams &p, int pair_id, int num_pairs,
                                               int i, WorkItem &w) {
  const int n_dp =
      pair_id < p.dp_tiles ? (p.dp_tiles - pair_id + num_pairs - 1) / num_pairs : 0;
  w.n_off = 0;
  w.ncols = kPairBN;
  w.t_rel = -1;
  w.nparts = 1;
  w.part = 0;
  if (i < n_dp) {
    w.tile = pair_id + i * num_pairs;
    w.kb_begin = 0;
    w.kb_end = p.k_blocks;
    return true;
  }
  if (p.dp_tiles >= p.num_tiles) return false;
  if (p.tail_nsplit > 1) {  // one narrow tail tile per pair, pairs 0 .. R * nsplit - 1
    if (i != n_dp || pair_id >= (p.num_tiles - p.dp_tiles) * p.tail_nsplit) return false;
    w.tile = p.dp_tiles + pair_id / p.tail_nsplit;
    w.ncols = kPairBN / p.tail_nsplit;
    w.n_off = (pair_id % p.tail_nsplit) * w.ncols;
    w.kb_begin = 0;
    w.kb_end = p.k_blocks;
    return true;
  }
  if (p.sk_per <= 0) return false;
  const int kb = p.k_blocks;
  const int u0 = pair_id * p.sk_per;
  const int u1 = min(u0 + p.sk_per, p.sk_units);
  if (u0 >= u1) return false;
  const int t_rel = u0 / kb + (i - n_dp);
  if (t_rel * kb >= u1) return false;
  w.t_rel = t_rel;
  w.tile = p.dp_tiles + t_rel;
  w.kb_begin = max(u0 - t_rel * kb, 0);
  w.kb_end = min(u1 - t_rel * kb, kb);
  const int first = (t_rel * kb) / p.sk_per;
  const int last = ((t_rel + 1) * kb - 1) / p.sk_per;
  w.nparts = last - first + 1;
  w.part = pair_id - first;
  return true;
}

// Registers one arrival on a tagged counter, (tag << BITS) | arrivals, for
// launch tag `tag` (a counter holding another tag counts as 0); returns how
// many arrivals came before (-1 if the retry bound ran out, which also sets
// the device error word).
template <int BITS>
__device__ __forceinline__ int tagged_arrive(unsigned long long *counter, unsigned long long tag,
                                             unsigned long long add = 1) {
  constexpr unsigned long long kMask = (1ull << BITS) - 1;
  unsigned long long cur = *reinterpret_cast<volatile unsigned long long *>(counter);
  for (int i = 0; i < (1 << 20); ++i) {
    const unsigned long long before = (cur >> BITS) == tag ? (cur & kMask) : 0ull;
    const unsigned long long prev = atomicCAS(counter, cur, (tag << BITS) | (before + add));
    if (prev == cur) return static_cast<int>(before);
    cur = prev;
  }
  atomicOr(&g_device_error, W8A8_DEVERR_TIMEOUT);
  return -1;
}

__device__ __forceinline__ int split_arrive(unsigned long long *counter, unsigned long long epoch) {
  return tagged_arrive<8>(counter, epoch);
}

// Waits (acquire, bounded like every other wait) until the rows of 128-row
// block b of q are quantized; then their q and s_a may be read (the TMA
// loads that follow included).
__device__ __forceinline__ bool rows_block_wait(const GemmParams &p, int b,
                                                volatile int *abort_flag) {
  const int r0 = b * kBM;
  const int n = p.M - r0 < kBM ? p.M - r0 : kBM;
  const unsigned long long want = (p.fuse_tag << 16) | static_cast<unsigned long long>(n);
  const unsigned long long *c = p.row_ready + b;
  if (ld_acquire_gpu_u64(c) != want) {
    const uint64_t t0 = global_timer_ns();
    for (uint32_t i = 1; ld_acquire_gpu_u64(c) != want; ++i) {
      if ((i & 15u) == 0u) {
        if (*abort_flag) return false;
        if (global_timer_ns() - t0 > kWaitLimitNs) {
          *abort_flag = 1;
          atomicOr(&g_device_error, W8A8_DEVERR_TIMEOUT);
          return false;
        }
      }
    }
  }
  fence_proxy_async_global();  // order the TMA reads after the acquire
  return true;
}

// Partial-sum slice of pair `pair` on shared-out tile t_rel.  Slot t_rel +
// pair is unique: two contributions (t, j) and (t + d, j - d), d >= 1, cannot
// both exist, since pair j - d ends at or before unit j * sk_per, which is
// below (t + 1) * k_blocks, where tile t + d starts at the earliest.
__device__ __forceinline__ int32_t *split_slice(const GemmParams &p, int t_rel, int pair,
                                                int slice) {
  return p.split_partials +
         (static_cast<int64_t>(t_rel + pair) * kSlicesPerTile + slice) * kSlotInts;
}

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

// One epilogue warp's share of an accumulator: its 32 TMEM lanes (tile rows
// row0 .. row0+31) and COLS columns starting at output column col_base, in
// chunks of 32 columns.  t_row addresses (first lane, first column).
// Modes: kEpiNormal -- the epilogue proper; kEpiWritePartial -- store the
// raw int32 accumulators to the slice at `slot` and nothing else;
// kEpiAddPartials -- add the slices at slot + j * part_stride, j < nparts,
// j != own_part, to the accumulators (exact int32 sums), then the epilogue
// proper.
constexpr int kEpiNormal = 0, kEpiWritePartial = 1, kEpiAddPartials = 2;

template <int COLS, bool RAW_OUT>
__device__ __forceinline__ void epilogue_warp_slice(const GemmParams &p, const CUtensorMap *tmap_y,
                                                    uint32_t t_row, int row0, int col_base,
                                                    uint8_t *stage_buf, uint32_t &chunk_count,
                                                    int lane, int mode = kEpiNormal,
                                                    int32_t *slot = nullptr, int nparts = 0,
                                                    int own_part = 0, int64_t part_stride = 0,
                                                    int ncols = COLS) {
  const int row = row0 + lane;
  const bool row_ok = row < p.M;
  // s_a may have been written earlier in this same launch (fused
  // quantization): read it through L2, never the non-coherent path
  const float sa = row_ok ? __ldcg(p.s_a + row) : 0.0f;
  // a warp whose 32 rows all lie past M has nothing to store; a narrow tile
  // (ncols < COLS, a multiple of 32) has fewer chunks
  const int cols_here = row0 < p.M ? (ncols < COLS ? ncols : COLS) : 0;
#pragma unroll 1
  for (int c = 0; c < cols_here; c += kEpiChunk) {
    const int col0 = col_base + c;
    if (col0 >= p.N) break;  // warp-uniform
    if (mode == kEpiWritePartial) {
      uint32_t r[32];
      tmem_ld_32x32b_x32(t_row + c, r);
      tmem_ld_wait();
      // slice layout: uint4 index ((c / 32) * 8 + g) * 32 + lane (coalesced)
      uint4 *dst = reinterpret_cast<uint4 *>(slot) + (c / 32) * 256 + lane;
#pragma unroll
      for (int g = 0; g < 8; ++g)
        __stcg(dst + 32 * g, make_uint4(r[4 * g], r[4 * g + 1], r[4 * g + 2], r[4 * g + 3]));
      continue;
    }
    if constexpr (RAW_OUT) {
      uint32_t r[32];
      tmem_ld_32x32b_x32(t_row + c, r);
      tmem_ld_wait();
      if (mode == kEpiAddPartials) {
        for (int j = 0; j < nparts; ++j) {
          if (j == own_part) continue;
          const uint4 *src =
              reinterpret_cast<const uint4 *>(slot + j * part_stride) + (c / 32) * 256 + lane;
#pragma unroll
          for (int g = 0; g < 8; ++g) {
            const uint4 a = __ldcg(src + 32 * g);
            r[4 * g] += a.x; r[4 * g + 1] += a.y; r[4 * g + 2] += a.z; r[4 * g + 3] += a.w;
          }
        }
      }
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
      // per-column scale and bias of this chunk (warp-uniform addresses);
      // issued before the TMEM load so the two latencies overlap
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
      if (mode == kEpiAddPartials) {  // exact int32 sum of the K-parts
        for (int j = 0; j < nparts; ++j) {
          if (j == own_part) continue;
          const uint4 *src =
              reinterpret_cast<const uint4 *>(slot + j * part_stride) + (c / 32) * 256 + lane;
#pragma unroll
          for (int g = 0; g < 8; ++g) {
            const uint4 a = __ldcg(src + 32 * g);
            r[4 * g] += a.x; r[4 * g + 1] += a.y; r[4 * g + 2] += a.z; r[4 * g + 3] += a.w;
          }
        }
      }
      // two adjacent columns at a time in packed fp32: each lane of every
      // packed operation is the same separately rounded operation as before
      uint32_t packed[16];
      const float2 sa2 = make_float2(sa, sa);
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        float2 v = make_float2(__int2float_rn(static_cast<int32_t>(r[2 * i])),
                               __int2float_rn(static_cast<int32_t>(r[2 * i + 1])));
        v = mul2_rn(v, sa2);
        v = mul2_rn(v, make_float2(sw[2 * i], sw[2 * i + 1]));
        if (p.bias != nullptr)
          v = add2_rn(v, make_float2(__uint_as_float(bw[i] << 16),
                                     __uint_as_float(bw[i] & 0xFFFF0000u)));
        const __nv_bfloat162 h = __floats2bfloat162_rn(v.x, v.y);
        packed[i] = *reinterpret_cast<const uint32_t *>(&h);
      }
      // staging buffer of this chunk: free once the store issued two
      // chunks ago has finished reading it
      uint8_t *buf = stage_buf + (chunk_count & 1u) * kEpiBufBytes;
      if (lane == 0) bulk_wait_group_read<1>();
      __syncwarp();
      // row `lane` = 64 bytes = four 16-byte pieces; 64-byte swizzle:
      // piece j of row r sits at position j ^ ((r >> 1) & 3)
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
}

template <int BN, int STAGES, bool RAW_OUT>
__global__ void __launch_bounds__(kGemmThreads, 1)
    gemm_i8_tcgen05_kernel(const __grid_constant__ CUtensorMap tmap_a,
                           const __grid_constant__ CUtensorMap tmap_b,
                           const __grid_constant__ CUtensorMap tmap_y, const GemmParams p) {
  using L = GemmLayout<BN, STAGES>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_addr(smem_raw);
  uint8_t *smem = smem_raw + ((1024u - (raw_addr & 1023u)) & 1023u);
  uint64_t *full = reinterpret_cast<uint64_t *>(smem + L::kBarOffset);
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
      mbar_init(&tempty[a], kEpiWarps);  // one arrival per epilogue warp
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbarrier_init();
    tma_prefetch_desc(&tmap_a);
    tma_prefetch_desc(&tmap_b);
    if constexpr (!RAW_OUT) tma_prefetch_desc(&tmap_y);
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
      // The weights do not depend on the preceding kernel: the first ring's
      // worth of Wq loads is issued before waiting for it (programmatic
      // dependent launch); q is loaded only after the wait.
      int prefetched = 0;
      if (static_cast<int>(blockIdx.x) < p.num_tiles) {
        int mb0, nb0;
        gemm_tile_coords(blockIdx.x, p, mb0, nb0);
        prefetched = p.k_blocks < STAGES ? p.k_blocks : STAGES;
        for (int kb = 0; kb < prefetched; ++kb) {
          uint8_t *sb = smem + kb * L::kStageBytes + L::kABytes;
          mbar_arrive_expect_tx(&full[kb], L::kStageBytes);
          tma_load_2d(&tmap_b, &full[kb], sb, kb * kBK, nb0 * BN);
        }
      }
      grid_dependency_wait();
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
          if (prefetched > 0) {
            --prefetched;  // this stage's barrier is armed and its Wq tile is in flight
          } else {
            mbar_arrive_expect_tx(&full[stage], L::kStageBytes);
            tma_load_2d(&tmap_b, &full[stage], sb, kb * kBK, nb * BN);
          }
          tma_load_2d(&tmap_a, &full[stage], sa, kb * kBK, mb * kBM);
          ++issued;
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      grid_dependents_launch();  // all loads issued: the next kernel may start its prologue
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
    const int e = warp - 2;            // 0..7
    const int quarter = warp & 3;      // TMEM lanes 32*quarter .. +31 = tile rows
    const int half = e >> 2;           // which half of the tile's columns
    uint8_t *stage_buf = smem + L::kEpiOffset + e * 2 * kEpiBufBytes;
    uint32_t chunk_count = 0;          // TMA stores issued by this warp
    int acc = 0;
    uint32_t acc_phase = 0;
    grid_dependency_wait();            // s_a comes from the preceding kernel
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
      epilogue_warp_slice<BN / 2, RAW_OUT>(p, &tmap_y, t_row, mb * kBM + quarter * 32,
                                           nb * BN + half * (BN / 2), stage_buf, chunk_count,
                                           lane);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty[acc]);
      if (++acc == 2) {
        acc = 0;
        acc_phase ^= 1u;
      }
    }
    if constexpr (!RAW_OUT) {
      if (lane == 0) bulk_wait_all();  // staging buffers stay valid until stored
      __syncwarp();
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, L::kTmemCols);
  }
}

// ------------------------------------------------------------------------
// CTA-pair variant (tcgen05 .cta_group::2): a cluster of two CTAs on two SMs
// computes 256 x 256 output tiles.  CTA r of the pair loads rows
// [128 r, 128 r + 128) of the tile's q block and rows [128 r, 128 r + 128) of
// its Wq block (no multicast: each CTA loads its own halves), so a stage is
// 32 KB per CTA instead of 48 KB and the ring is 6 deep; the leader CTA
// (rank 0) issues M = 256, N = 256 MMAs that read both CTAs' shared memory
// and accumulate into both CTAs' TMEM (CTA r holds rows 128 r .. 128 r + 127
// of the tile, all 256 columns).  Both CTAs' TMA loads report to the
// leader's "full" barrier; the leader's commits arrive on "empty" and
// accumulator-"full" barriers in both CTAs; both CTAs' epilogue warps arrive
// on the leader's accumulator-"empty" barrier.

template <int STAGES>
struct PairLayout {
  static constexpr int kABytes = kBM * kBK;              // this CTA's 128 rows of q
  static constexpr int kBBytes = (kPairBN / 2) * kBK;    // this CTA's 128 rows of Wq
  static constexpr int kStageBytes = kABytes + kBBytes;
  static constexpr int kTileBytes = STAGES * kStageBytes;
  static constexpr int kEpiOffset = kTileBytes;  // 1024-aligned
  static constexpr int kEpiBytes = kEpiWarps * 2 * kEpiBufBytes;
  static constexpr int kBarOffset = kEpiOffset + kEpiBytes;
  // full[S], empty[S], tfull[2], tempty[2], drain, then two words; then the
  // fused quantization's barriers: kQuantSlots per epilogue warp, ring_free,
  // and two decision words
  static constexpr int kQuantSlots = 4;
  static constexpr int kBarBytes = (2 * STAGES + 5) * 8 + 8 + (kEpiWarps * kQuantSlots + 1) * 8 + 8;
  static constexpr int kSmemBytes = kBarOffset + kBarBytes + 1024;
  static constexpr int kTmemCols = 2 * kPairBN;
  // each epilogue warp's share of the ring for the bulk-path rows
  static constexpr int kQuantWarpBytes = STAGES * kStageBytes / kEpiWarps;
  static_assert(kSmemBytes <= 232448, "shared memory budget");
};

// Pair tile t -> (256-row block, 256-column block), banded like gemm_tile_coords.
__device__ __forceinline__ void pair_tile_coords(int t, const GemmParams &p, int &mb, int &nb) {
  gemm_tile_coords(t, p, mb, nb);  // p.num_m_blk counts 256-row blocks here
}

template <int STAGES, bool RAW_OUT, bool FUSE_QUANT>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kGemmThreads, 1)
    gemm_i8_tcgen05_pair_kernel(const __grid_constant__ CUtensorMap tmap_a,
                                const __grid_constant__ CUtensorMap tmap_b,
                                const __grid_constant__ CUtensorMap tmap_b_tail,
                                const __grid_constant__ CUtensorMap tmap_y, const GemmParams p) {
  using L = PairLayout<STAGES>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_addr(smem_raw);
  uint8_t *smem = smem_raw + ((1024u - (raw_addr & 1023u)) & 1023u);
  uint64_t *full = reinterpret_cast<uint64_t *>(smem + L::kBarOffset);
  uint64_t *empty = full + STAGES;
  uint64_t *tfull = empty + STAGES;
  uint64_t *tempty = tfull + 2;
  uint64_t *drain = tempty + 2;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(drain + 1);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
  uint64_t *qbar = drain + 2;                         // [kEpiWarps][kQuantSlots]
  uint64_t *ring_free = qbar + kEpiWarps * L::kQuantSlots;
  volatile int *epi_go = reinterpret_cast<volatile int *>(ring_free + 1);  // [2]

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();  // 0 = leader
  const int pair_id = blockIdx.x >> 1;
  const int num_pairs = gridDim.x >> 1;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);   // the leader's expect-tx arrival; bytes from both CTAs
      mbar_init(&empty[s], 1);  // the leader's MMA commit
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 2 * kEpiWarps);  // epilogue warps of both CTAs
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    if constexpr (FUSE_QUANT) {
      for (int i = 0; i < kEpiWarps * L::kQuantSlots; ++i) mbar_init(&qbar[i], 1);
      mbar_init(ring_free, kEpiWarps);
      epi_go[0] = epi_go[1] = 0;
    }
    fence_mbarrier_init();
    tma_prefetch_desc(&tmap_a);
    tma_prefetch_desc(&tmap_b);
    if (p.tail_nsplit > 1) tma_prefetch_desc(&tmap_b_tail);
    if constexpr (!RAW_OUT) tma_prefetch_desc(&tmap_y);
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_slot, L::kTmemCols);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync();  // barriers of both CTAs initialized, TMEM allocated
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ producer (both CTAs)
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued = 0;
      bool ok = true;
      // Wq loads of the first ring's worth of stages before waiting for the
      // preceding kernel (programmatic dependent launch); q after the wait.
      int prefetched = 0;
      WorkItem w;
      // An item of ncols columns loads this CTA's ncols / 2 rows of Wq (the
      // narrow tail tiles through their own, narrower TMA box).
      auto b_map = [&](const WorkItem &it) { return it.ncols == kPairBN ? &tmap_b : &tmap_b_tail; };
      auto b_row = [&](const WorkItem &it, int nb) {
        return nb * kPairBN + it.n_off + static_cast<int>(rank) * (it.ncols / 2);
      };
      auto stage_tx = [&](const WorkItem &it) {
        return 2u * static_cast<uint32_t>(L::kABytes + (it.ncols / 2) * kBK);
      };
      // fused quantization: the epilogue warps use the ring for their first
      // rows; nothing is loaded into it before they are all done with it
      if (FUSE_QUANT && !mbar_wait(ring_free, 0u, abort_flag)) ok = false;
      if (ok && pair_work_item(p, pair_id, num_pairs, 0, w)) {
        int mb0, nb0;
        pair_tile_coords(w.tile, p, mb0, nb0);
        const int nkb = w.kb_end - w.kb_begin;
        prefetched = nkb < STAGES ? nkb : STAGES;
        for (int i = 0; i < prefetched; ++i) {
          uint8_t *sb = smem + i * L::kStageBytes + L::kABytes;
          if (rank == 0) mbar_arrive_expect_tx(&full[i], stage_tx(w));
          tma_load_2d_pair(b_map(w), map_to_cta(smem_addr(&full[i]), 0), sb,
                           (w.kb_begin + i) * kBK, b_row(w, nb0));
        }
      }
      grid_dependency_wait();
      int ready_blk = -1;  // fused quantization: the q block known to be complete
      for (int it = 0; ok && pair_work_item(p, pair_id, num_pairs, it, w); ++it) {
        int mb, nb;
        pair_tile_coords(w.tile, p, mb, nb);
        if constexpr (FUSE_QUANT) {
          const int blk = mb * 2 + static_cast<int>(rank);
          if (blk != ready_blk && blk * kBM < p.M) {
            if (!rows_block_wait(p, blk, abort_flag)) {
              ok = false;
              break;
            }
            ready_blk = blk;
          }
        }
        for (int kb = w.kb_begin; kb < w.kb_end; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag)) {
            ok = false;
            break;
          }
          uint8_t *sa = smem + stage * L::kStageBytes;
          uint8_t *sb = sa + L::kABytes;
          const uint32_t leader_full = map_to_cta(smem_addr(&full[stage]), 0);
          if (prefetched > 0) {
            --prefetched;  // armed and Wq in flight already
          } else {
            if (rank == 0) mbar_arrive_expect_tx(&full[stage], stage_tx(w));
            tma_load_2d_pair(b_map(w), leader_full, sb, kb * kBK, b_row(w, nb));
          }
          tma_load_2d_pair(&tmap_a, leader_full, sa, kb * kBK, mb * 256 + static_cast<int>(rank) * 128);
          ++issued;
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      grid_dependents_launch();  // all loads issued: the next kernel may start its prologue
      // The leader's last commits still arrive on this CTA's "empty"
      // barriers: wait for them before the CTA may leave (bounded).
      const uint32_t n = issued < static_cast<uint32_t>(STAGES) ? issued : STAGES;
      for (uint32_t i = issued - n; i < issued; ++i)
        mbar_wait_drain(&empty[i % STAGES], (i / STAGES) & 1u);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (leader only)
    if (lane == 0 && rank == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      bool any_mma = false;
      WorkItem w;
      for (int it = 0; ok && pair_work_item(p, pair_id, num_pairs, it, w); ++it) {
        if (!mbar_wait(&tempty[acc], acc_phase ^ 1u, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * kPairBN);
        const uint32_t idesc = idesc_i8(2 * kBM, w.ncols);
        for (int kb = w.kb_begin; kb < w.kb_end; ++kb) {
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
            mma_i8_pair(d_tmem, adesc + 2u * k, bdesc + 2u * k, idesc,
                        (kb != w.kb_begin || k != 0) ? 1u : 0u);
          any_mma = true;
          mma_commit_pair(&empty[stage], 0x3);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        mma_commit_pair(&tfull[acc], 0x3);
        if (++acc == 2) {
          acc = 0;
          acc_phase ^= 1u;
        }
      }
      if (!ok && any_mma) {
        mma_commit_pair(drain, 0x1);
        mbar_wait_drain(drain, 0);
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue (both CTAs)
    const int e = warp - 2;
    const int quarter = warp & 3;
    const int half = e >> 2;
    uint8_t *stage_buf = smem + L::kEpiOffset + e * 2 * kEpiBufBytes;
    uint32_t chunk_count = 0;
    int acc = 0;
    uint32_t acc_phase = 0;
    const int slice = static_cast<int>(rank) * kEpiWarps + e;
    grid_dependency_wait();  // s_a (or, fused, x) comes from the preceding kernel
    int it = 0;
    bool more = true;
    // The epilogue of this pair's next work item (this warp's slice); false
    // once the pair has none left or a wait gave up.
    auto do_item = [&]() -> bool {
      WorkItem w;
      if (!pair_work_item(p, pair_id, num_pairs, it, w)) return false;
      int mb, nb;
      pair_tile_coords(w.tile, p, mb, nb);
      if constexpr (FUSE_QUANT) {  // acquire this slice's rows (their s_a)
        const int blk = mb * 2 + static_cast<int>(rank);
        if (lane == 0 && blk * kBM < p.M) rows_block_wait(p, blk, abort_flag);
        __syncwarp();
      }
      int ok = 1;
      if (lane == 0) ok = mbar_wait(&tfull[acc], acc_phase, abort_flag) ? 1 : 0;
      ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
      if (!ok) return false;
      tc_fence_after();
      // this warp: TMEM lane quarter `quarter`, columns [half * ncols / 2, +ncols / 2)
      const int wcols = w.ncols / 2;
      const uint32_t t_row = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) +
                             static_cast<uint32_t>(acc * kPairBN + half * wcols);
      const int row0 = mb * 256 + static_cast<int>(rank) * 128 + quarter * 32;
      const int col_base = nb * kPairBN + w.n_off + half * wcols;
      if (w.nparts == 1) {
        epilogue_warp_slice<kPairBN / 2, RAW_OUT>(p, &tmap_y, t_row, row0, col_base, stage_buf,
                                                  chunk_count, lane, kEpiNormal, nullptr, 0, 0, 0,
                                                  wcols);
      } else {
        // Shared-out tile: the last contribution to arrive finishes it.  The
        // part holding k-block 0 is this pair's last item and usually the
        // last to arrive: if all the others are in already it skips writing
        // its own partial sums.
        unsigned long long *counter = p.split_counters + w.t_rel * kSlicesPerTile + slice;
        int32_t *first_slice = split_slice(p, w.t_rel, pair_id - w.part, slice);
        const unsigned long long all_others =
            (p.split_epoch << 8) | static_cast<unsigned long long>(w.nparts - 1);
        int last = 0;
        if (w.part == 0 && lane == 0) last = ld_acquire_gpu_u64(counter) == all_others ? 1 : 0;
        __syncwarp();  // orders the lanes' partial-sum reads after lane 0's acquire
        last = __shfl_sync(0xFFFFFFFFu, last, 0);
        if (!last) {
          epilogue_warp_slice<kPairBN / 2, RAW_OUT>(
              p, &tmap_y, t_row, row0, col_base, stage_buf, chunk_count, lane, kEpiWritePartial,
              first_slice + static_cast<int64_t>(w.part) * kSlicesPerTile * kSlotInts);
          __threadfence();
          __syncwarp();
          if (lane == 0) last = split_arrive(counter, p.split_epoch) == w.nparts - 1 ? 1 : 0;
          __syncwarp();
          last = __shfl_sync(0xFFFFFFFFu, last, 0);
        }
        if (last) {
          __threadfence();
          if (lane == 0) *reinterpret_cast<volatile unsigned long long *>(counter) = 0ull;
          epilogue_warp_slice<kPairBN / 2, RAW_OUT>(
              p, &tmap_y, t_row, row0, col_base, stage_buf, chunk_count, lane, kEpiAddPartials,
              first_slice, w.nparts, w.part, static_cast<int64_t>(kSlicesPerTile) * kSlotInts);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(map_to_cta(smem_addr(&tempty[acc]), 0));
      if (++acc == 2) {
        acc = 0;
        acc_phase ^= 1u;
      }
      ++it;
      return true;
    };
    if constexpr (FUSE_QUANT) {
      // pass j: this CTA's 8 rows 8 c + j * 8 * gridDim.x + e (one 128-row
      // block: 8 divides 128), then one arrival for all of them.  Rows below
      // fuse_bulk_rows come through this warp's share of the ring (bulk
      // copies, up to kQuantSlots rows in flight); later rows through
      // registers.  Between passes, one thread looks whether the next tile's
      // accumulator is ready, and if so the warps take its epilogue first.
      const int stride = static_cast<int>(gridDim.x) * kEpiWarps;
      const int cbase = static_cast<int>(blockIdx.x) * kEpiWarps;
      const int npass = cbase < p.M ? (p.M - cbase + stride - 1) / stride : 0;
      const uint32_t row_bytes = static_cast<uint32_t>(p.K) * 2u;
      int nslots = static_cast<int>(L::kQuantWarpBytes / row_bytes);
      if (nslots > L::kQuantSlots) nslots = L::kQuantSlots;
      uint8_t *qslot = smem + e * L::kQuantWarpBytes;
      uint64_t *wbar = qbar + e * L::kQuantSlots;
      const int bulk_end = p.fuse_bulk_rows < p.M ? p.fuse_bulk_rows : p.M;
      const int nbulk =
          cbase + e < bulk_end ? (bulk_end - cbase - e + stride - 1) / stride : 0;
      int issued = 0;
      auto issue = [&]() {
        const int64_t row = cbase + e + static_cast<int64_t>(issued) * stride;
        const int sl = issued % nslots;
        mbar_arrive_expect_tx(&wbar[sl], row_bytes);
        bulk_load_g2s(qslot + sl * row_bytes, p.x + row * p.ldx, row_bytes, &wbar[sl]);
        ++issued;
      };
      if (lane == 0) {
        while (issued < nslots && issued < nbulk) issue();
        if (nbulk == 0) mbar_arrive(ring_free);
      }
      for (int j = 0; j < npass; ++j) {
        const int base = cbase + j * stride;
        const int row = base + e;
        if (j < nbulk) {
          const int sl = j % nslots;
          int ok = mbar_wait(&wbar[sl], static_cast<uint32_t>(j / nslots) & 1u, abort_flag) ? 1 : 0;
          ok = __all_sync(0xFFFFFFFFu, ok);
          if (ok)
            quant_row_from_smem(reinterpret_cast<const uint4 *>(qslot + sl * row_bytes), p.K,
                                p.q_w + static_cast<int64_t>(row) * p.K, p.s_a_w + row, lane);
          __syncwarp();  // every lane is done with the slot
          if (lane == 0) {
            if (ok && issued < nbulk) issue();
            if (j == nbulk - 1) mbar_arrive(ring_free);  // this warp is done with the ring
          }
        } else if (row < p.M) {
          quant_row_by_warp<12>(p.x + static_cast<int64_t>(row) * p.ldx, p.K,
                                p.q_w + static_cast<int64_t>(row) * p.K, p.s_a_w + row, lane);
        }
        fence_proxy_async_global();
        __threadfence();  // release: every lane's q and s_a stores before the count
        if (e == 0 && lane == 0) epi_go[j & 1] = (more && mbar_try_wait(&tfull[acc], acc_phase)) ? 1 : 0;
        named_barrier_sync(1, kEpiWarps * 32);
        if (e == 0 && lane == 0) {
          const int rows = p.M - base < kEpiWarps ? p.M - base : kEpiWarps;
          tagged_arrive<16>(&p.row_ready[base / kBM], p.fuse_tag,
                            static_cast<unsigned long long>(rows));
        }
        if (epi_go[j & 1]) more = do_item();
      }
      if (lane == 0) {  // after a wait that gave up: let the copies in flight land
        for (int j = issued > nslots ? issued - nslots : 0; j < issued; ++j) {
          volatile int never = 0;
          mbar_wait(&wbar[j % nslots], static_cast<uint32_t>(j / nslots) & 1u, &never);
        }
      }
    }
    while (more) more = do_item();
    if constexpr (!RAW_OUT) {
      if (lane == 0) bulk_wait_all();
      __syncwarp();
    }
  }

  // Both CTAs finish (the leader's MMAs write the follower's TMEM, the
  // follower's epilogue reads it) before either frees the pair's TMEM.
  tc_fence_before();
  cluster_sync();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, L::kTmemCols);
  }
}

}  // namespace w8a8
