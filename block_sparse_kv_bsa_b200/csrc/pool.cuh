// pool.cuh - one warp's column sums of one 128-row KV block.
//
// Shared by the router (which pools history blocks while it streams them)
// and by the pooled-key cache written at append time (which pools the rows
// while it moves them into the cache), so both produce the same block means
// bit for bit.  Block = 128 rows x D bf16, contiguous, read
// as VPR = D/8 sixteen-byte vectors per row.  Lane (c = lane % VPR,
// g = lane / VPR) reads vector column c of rows g, g + RPI, ... (RPI = 32 /
// VPR rows per warp-wide load), 16 independent loads in flight per batch;
// rows at or past `valid` read as zero.  The RPI lanes holding the same
// columns are then combined by shuffles in a fixed order, so every lane ends
// with the sums of its 8 columns c*8 .. c*8+7.
#pragma once

#include "common.cuh"

namespace bsa {

// The summation itself, for any source of rows: `load(row)` returns this
// lane's vector of a row below `valid`, and `seen(row, x)` is called once for
// every row 0..127 with the vector that was added (zeros at and past
// `valid`), so a caller can move the rows while it pools them.
// NB rows per lane are loaded before any is added (more loads in flight for
// a larger NB); the rows are still added in the same order, so the sums do
// not depend on NB.
template <int VPR, class Load, class Seen, int NB = 16>
__device__ __forceinline__ void warp_colsum_rows(Load load, Seen seen, int valid, int g,
                                                 float (&acc)[8]) {
  constexpr int RPI = 32 / VPR;
  constexpr int kBatches = kBlk / (RPI * NB);
  static_assert(kBlk % (RPI * NB) == 0, "batches must cover the 128 rows exactly");
#pragma unroll
  for (int e = 0; e < 8; ++e) acc[e] = 0.f;
#pragma unroll
  for (int bt = 0; bt < kBatches; ++bt) {
    uint4 x[NB];
#pragma unroll
    for (int i = 0; i < NB; ++i) {
      const int row = (bt * NB + i) * RPI + g;
      x[i] = row < valid ? load(row) : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int i = 0; i < NB; ++i) {
      seen((bt * NB + i) * RPI + g, x[i]);
      acc[0] += bf16lo(x[i].x); acc[1] += bf16hi(x[i].x);
      acc[2] += bf16lo(x[i].y); acc[3] += bf16hi(x[i].y);
      acc[4] += bf16lo(x[i].z); acc[5] += bf16hi(x[i].z);
      acc[6] += bf16lo(x[i].w); acc[7] += bf16hi(x[i].w);
    }
  }
#pragma unroll
  for (int off = VPR; off < 32; off <<= 1) {
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] += __shfl_xor_sync(0xffffffffu, acc[e], off);
  }
}

template <int VPR>
__device__ __forceinline__ void warp_block_colsum(const uint4* blk, int valid, int c, int g,
                                                  float (&acc)[8]) {
  warp_colsum_rows<VPR>([&](int row) { return ld_nc_v4(blk + row * VPR + c); },
                        [](int, uint4) {}, valid, g, acc);
}

// The block mean of this lane's 8 columns: sums / valid (fp32).
template <int VPR>
__device__ __forceinline__ void warp_block_mean(const uint4* blk, int valid, int c, int g,
                                                float (&km)[8]) {
  float acc[8];
  warp_block_colsum<VPR>(blk, valid, c, g, acc);
#pragma unroll
  for (int e = 0; e < 8; ++e) km[e] = acc[e] / static_cast<float>(valid);
}

}  // namespace bsa
