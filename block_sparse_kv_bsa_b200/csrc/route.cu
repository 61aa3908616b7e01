// route.cu - bsa_route: per-query-block KV block selection.
//
// "Velox: Spatial Memory Makes World Models Efficient", Methodology Step 4
// (a block importance computed from the mean query and mean key of each
// block, softly boosted by geometric overlap: at most a 1 + lambda boost, none
// without overlap) and Step 5 (a bounded top-K route with reserved blocks
// added outside the budget).  The additive form used here is
//   s'[j, n] = sm_scale * <qmean_j, kmean_n> + lambda * min(g[j, n] / g_ref, 1).
//
// Up to three launches, all stream-ordered, no host round trip:
//   1. pool_q      mean of each query block's valid rows -> qm (workspace);
//                  skipped when the caller passes the query means
//   2. scores      from the pooled-key cache (the key means written at
//                  append): the product of query means and key means, on the
//                  tensor core for up to 64 query blocks (score_tc.cu), else
//                  on the FMA pipes; without the cache, pool_score streams
//                  every history K block once (one warp per block), pools it
//                  in registers and scores it against all query means of its
//                  head (the HBM-bound form of routing)
//   3. topk        add the prior (g read row by row), then an exact top-K per
//                  row by radix select on order-preserving score keys held in
//                  shared memory, ties to the lower index, emitted in ascending
//                  index order by a block-wide ordered compaction, followed by
//                  the own-chunk blocks.
// All sums run in fp32 in a fixed order, so results are deterministic.
#include <cuda.h>

#include <algorithm>
#include <mutex>

#include "common.cuh"
#include "pool.cuh"

namespace bsa {

// Threads of the block-wide selections (the long-row top-K and the page's
// route): 128 measured faster than 256 (fewer warps paying each barrier,
// scan and reduction) and than 64.
constexpr int kTopkThreads = 128;

struct RouteArgs {
  const uint4* q;          // [B, Hh, n_own*128, D] bf16
  const uint4* kc;         // [B, Hh, max_blocks, 128, D] bf16
  const int32_t* block_valid;
  const int32_t* q_valid;  // [n_own] or null
  const float* g;          // [B, n_own, n_hist] or null
  const float* kmean;      // [B, Hh, max_blocks, D] pooled keys, or null
  float* qm;               // [B, Hh, n_own, D]
  float* s;                // [B, Hh, n_own, s_ld]: row (b, h, j) holds its n_hist scores
  int32_t* idx;
  int32_t* cnt;
  int32_t* d_err;
  int B, Hh, n_own, n_hist, own_first, max_blocks, top_k, max_sel;
  int s_ld;                // score row stride: n_hist rounded up to 32 (128-byte rows)
  float sm_scale, lam, g_ref;
};

__device__ __forceinline__ int clamp_valid(int v, int32_t* d_err) {
  if (v < 1 || v > kBlk) {
    report(d_err, BSA_DEV_BAD_VALID);
    return v < 1 ? 1 : kBlk;
  }
  return v;
}

// Query-block means: one warp per (b, h, query block), with pool.cuh's
// summation, the same as bsa_tokens_to_blocks_mean's and the pooled-key
// cache's, so every block mean in the library comes from one summation.
constexpr int kPoolQWarps = 8;

template <int VPR>
__global__ void __launch_bounds__(kPoolQWarps * 32) pool_q_kernel(RouteArgs a) {
  pdl_wait();     // global memory only after the predecessor grid completed
  pdl_trigger();
  constexpr int D = VPR * 8;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int j = blockIdx.x * kPoolQWarps + warp;
  if (j >= a.n_own) return;
  const int h = blockIdx.y, b = blockIdx.z;
  int valid = a.q_valid != nullptr ? a.q_valid[j] : a.block_valid[a.own_first + j];
  valid = clamp_valid(valid, a.d_err);
  const long long blk = (static_cast<long long>(b) * a.Hh + h) * a.n_own + j;
  const int c = lane % VPR, g = lane / VPR;
  float m[8];
  warp_block_mean<VPR>(a.q + blk * kBlk * VPR, valid, c, g, m);
  if (g == 0) {
    float4* out = reinterpret_cast<float4*>(a.qm + blk * D + c * 8);
    out[0] = make_float4(m[0], m[1], m[2], m[3]);
    out[1] = make_float4(m[4], m[5], m[6], m[7]);
  }
}

// K-stream kernel: one warp reduces one history block at a time.  A CTA of
// 8 warps covers kScoreBlocksPerWarp consecutive blocks per warp of one
// (b, h), with that head's query means in shared memory (the only CTA-wide
// barrier).  Per block, each lane issues 16 independent 16-byte loads per
// batch (rows past the valid count read as 0), accumulates 8 fp32 column sums,
// the lanes holding the same columns are combined by shuffles, and the block
// mean is scored against every query mean (four independent shuffle chains
// per pass).  Many warps per SM and no per-block barrier keep HBM busy.
// The prior is added by the top-K kernel, which reads g row by row.
constexpr int kScoreWarps = 8;
constexpr int kScoreBlocksPerWarp = 8;

template <int VPR>
__global__ void __launch_bounds__(kScoreWarps * 32)
pool_score_kernel(RouteArgs a) {
  pdl_wait();     // global memory only after the predecessor grid completed
  pdl_trigger();
  constexpr int D = VPR * 8;
  constexpr int LPR = VPR;              // lanes per row (one 16-byte chunk each)
  constexpr int RPI = 32 / LPR;         // rows per warp-wide load (2 or 4)
  extern __shared__ float qm[];         // [n_own][D] of this head
  const int h = blockIdx.y, b = blockIdx.z;
  const long long bh = static_cast<long long>(b) * a.Hh + h;
  for (int i = threadIdx.x; i < a.n_own * D; i += kScoreWarps * 32) qm[i] = a.qm[bh * a.n_own * D + i];
  __syncthreads();
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int c = lane % LPR;             // 16-byte column chunk of this lane
  const int g = lane / LPR;             // row phase within a load / query-block phase
  const int n_base = (blockIdx.x * kScoreWarps + warp) * kScoreBlocksPerWarp;
  // Score one block mean (this lane's 8 columns in km) against every query
  // mean: lane group g takes query blocks j = g, g + RPI, ...; the LPR lanes
  // of a group are reduced by shuffles.  The loop bound is the same for every
  // lane (the shuffles are warp-wide); out-of-range query blocks only skip
  // their arithmetic.
  auto score_block = [&](int n, const float (&km)[8]) {
    for (int jb = 0; jb < a.n_own; jb += 4 * RPI) {
      const int j0 = jb + g;
      float d[4];
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        d[t] = 0.f;
        const int j = j0 + t * RPI;
        if (j < a.n_own) {
          const float4* q4 = reinterpret_cast<const float4*>(qm + j * D + c * 8);
          const float4 q0 = q4[0], q1 = q4[1];
          d[t] = fmaf(q0.x, km[0], d[t]); d[t] = fmaf(q0.y, km[1], d[t]);
          d[t] = fmaf(q0.z, km[2], d[t]); d[t] = fmaf(q0.w, km[3], d[t]);
          d[t] = fmaf(q1.x, km[4], d[t]); d[t] = fmaf(q1.y, km[5], d[t]);
          d[t] = fmaf(q1.z, km[6], d[t]); d[t] = fmaf(q1.w, km[7], d[t]);
        }
      }
#pragma unroll
      for (int off = 1; off < LPR; off <<= 1) {
#pragma unroll
        for (int t = 0; t < 4; ++t) d[t] += __shfl_xor_sync(0xffffffffu, d[t], off);
      }
      if (c < 4) {
        float dv = d[0];
#pragma unroll
        for (int t = 1; t < 4; ++t) dv = c == t ? d[t] : dv;
        const int j = j0 + c * RPI;
        if (j < a.n_own) a.s[(bh * a.n_own + j) * a.s_ld + n] = a.sm_scale * dv;
      }
    }
  };
  {
    for (int u = 0; u < kScoreBlocksPerWarp; ++u) {
      const int n = n_base + u;
      if (n >= a.n_hist) break;
      const int valid = clamp_valid(a.block_valid[n], a.d_err);
      float km[8];
      warp_block_mean<VPR>(a.kc + (bh * a.max_blocks + n) * kBlk * VPR, valid, c, g, km);
      score_block(n, km);
    }
  }
}

// Scores from the pooled-key cache: s[j, n] = sm_scale * <qmean_j, kmean_n>
// for all query blocks j of a head and a tile of 64 history blocks, as a
// register-blocked CUDA-core product (the whole step is ~0.7 GFLOP at chunk
// 48, far too small for the tensor cores to matter).  Both operands go to
// shared memory with a 4-float row pad; each thread owns up to 8 query
// blocks x 4 history blocks and accumulates over D, 4 dimensions per step
// in two-wide FMAs.
constexpr int kMeanTileN = 64;
constexpr int kMeanThreads = 128;

// Query blocks jb + tq + 8x (x < X) against history blocks n0 + tk + 16y
// (y < 4) of the staged tile; X is the number of 8-row groups the tile's
// query blocks need, so padded rows cost nothing.  Each dot product keeps
// two running sums, over the even and over the odd dimensions (in order),
// as one f32x2 accumulator: the two halves of a 16-byte load are already
// the operand pairs, so one fma.f32x2 does two dimensions.
template <int D, int X>
__device__ __forceinline__ void score_means_tile(const RouteArgs& a, const float* qs,
                                                 const float* ks, long long bh, int n0, int jb) {
  constexpr int P = D + 4;
  // With rows P = D+4 floats apart (an odd number of 16-byte units), the 16
  // history rows a warp reads per step sit in distinct bank groups; the two
  // query rows of a warp are broadcasts.
  const int tk = threadIdx.x % 16, tq = threadIdx.x / 16;
  uint64_t acc[X][4];
#pragma unroll
  for (int x = 0; x < X; ++x)
#pragma unroll
    for (int y = 0; y < 4; ++y) acc[x][y] = 0ull;   // {+0.f, +0.f}
#pragma unroll 2
  for (int d = 0; d < D; d += 4) {
    ulonglong2 q[X], k[4];
#pragma unroll
    for (int x = 0; x < X; ++x)
      q[x] = *reinterpret_cast<const ulonglong2*>(qs + (jb + tq + 8 * x) * P + d);
#pragma unroll
    for (int y = 0; y < 4; ++y)
      k[y] = *reinterpret_cast<const ulonglong2*>(ks + (tk + 16 * y) * P + d);
    // All first halves, then all second halves: 4X independent FMAs
    // between the two that update one accumulator.
#pragma unroll
    for (int x = 0; x < X; ++x)
#pragma unroll
      for (int y = 0; y < 4; ++y) acc[x][y] = f2_fma(q[x].x, k[y].x, acc[x][y]);
#pragma unroll
    for (int x = 0; x < X; ++x)
#pragma unroll
      for (int y = 0; y < 4; ++y) acc[x][y] = f2_fma(q[x].y, k[y].y, acc[x][y]);
  }
#pragma unroll
  for (int x = 0; x < X; ++x) {
    const int j = jb + tq + 8 * x;
    if (j >= a.n_own) continue;
#pragma unroll
    for (int y = 0; y < 4; ++y) {
      const int n = n0 + tk + 16 * y;
      float even, odd;
      f2_unpack(acc[x][y], even, odd);
      if (n < a.n_hist) a.s[(bh * a.n_own + j) * a.s_ld + n] = a.sm_scale * (even + odd);
    }
  }
}

template <int D>
__global__ void __launch_bounds__(kMeanThreads, 1)
score_means_kernel(RouteArgs a) {
  pdl_wait();     // global memory only after the predecessor grid completed
  pdl_trigger();
  constexpr int P = D + 4;                       // padded row (floats)
  extern __shared__ float sm[];
  const int nq = (a.n_own + 15) & ~15;           // query rows, rounded up to 16
  float* qs = sm;                                // [nq][P]
  float* ks = qs + nq * P;                       // [64][P]
  const int h = blockIdx.y, b = blockIdx.z;
  const long long bh = static_cast<long long>(b) * a.Hh + h;
  const int n0 = blockIdx.x * kMeanTileN;
  // Stage the query means and this tile's key means, kLoads independent
  // 16-byte loads per thread in flight before any is stored.
  constexpr int kLoads = 16;
  const int n_q4 = nq * (D / 4), n_k4 = kMeanTileN * (D / 4);
  for (int base = 0; base < n_q4 + n_k4; base += kLoads * kMeanThreads) {
    float4 v[kLoads];
#pragma unroll
    for (int u = 0; u < kLoads; ++u) {
      const int i = base + u * kMeanThreads + threadIdx.x;
      v[u] = make_float4(0.f, 0.f, 0.f, 0.f);
      if (i < n_q4) {
        const int r = i / (D / 4), c4 = i % (D / 4);
        if (r < a.n_own) v[u] = ld_nc_f4(a.qm + (bh * a.n_own + r) * D + c4 * 4);
      } else if (i < n_q4 + n_k4) {
        const int r = (i - n_q4) / (D / 4), c4 = (i - n_q4) % (D / 4);
        if (n0 + r < a.n_hist) v[u] = ld_nc_f4(a.kmean + (bh * a.max_blocks + n0 + r) * D + c4 * 4);
      }
    }
#pragma unroll
    for (int u = 0; u < kLoads; ++u) {
      const int i = base + u * kMeanThreads + threadIdx.x;
      if (i < n_q4) {
        const int r = i / (D / 4), c4 = i % (D / 4);
        *reinterpret_cast<float4*>(qs + r * P + c4 * 4) = v[u];
      } else if (i < n_q4 + n_k4) {
        const int r = (i - n_q4) / (D / 4), c4 = (i - n_q4) % (D / 4);
        *reinterpret_cast<float4*>(ks + r * P + c4 * 4) = v[u];
      }
    }
  }
  __syncthreads();
  // Query rows in tiles of 64; a tile's last row read is round8(n_own) - 1,
  // inside the nq staged (zero-filled) rows.
  for (int jb = 0; jb < a.n_own; jb += 64) {
    const int groups = min(8, (a.n_own - jb + 7) / 8);
    switch (groups) {
      case 1: score_means_tile<D, 1>(a, qs, ks, bh, n0, jb); break;
      case 2: score_means_tile<D, 2>(a, qs, ks, bh, n0, jb); break;
      case 3: score_means_tile<D, 3>(a, qs, ks, bh, n0, jb); break;
      case 4: score_means_tile<D, 4>(a, qs, ks, bh, n0, jb); break;
      case 5: score_means_tile<D, 5>(a, qs, ks, bh, n0, jb); break;
      case 6: score_means_tile<D, 6>(a, qs, ks, bh, n0, jb); break;
      case 7: score_means_tile<D, 7>(a, qs, ks, bh, n0, jb); break;
      default: score_means_tile<D, 8>(a, qs, ks, bh, n0, jb); break;
    }
  }
}

// For up to 64 query blocks the same product runs on the tensor core
// (score_tc.cu: three tf32 passes over hi/lo splits of both means).
bool score_means_tc_fits(int n_own, int D);
bsa_status launch_score_means_tc(const float* qm, const float* kmean, float* s, int s_ld, int BH,
                                 int n_own, int n_hist, int max_blocks, int D, float sm_scale,
                                 int sms, int32_t* d_err, cudaStream_t st);

// Streaming multiprocessors of the current device (cached per device).
static int device_sms() {
  static int cache[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
  if (cache[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
    cache[dev] = n;
  }
  return cache[dev];
}

// Order-preserving map of a float onto uint32 (larger float -> larger key).
__device__ __forceinline__ uint32_t score_key(float x) {
  uint32_t u = __float_as_uint(x);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
// Its inverse: the float a key came from, bit for bit.
__device__ __forceinline__ float key_score(uint32_t k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7fffffffu) : ~k);
}

// Block-wide exclusive prefix of a per-thread flag (threads in index order).
// Returns this thread's exclusive count; *total gets the block total.
__device__ __forceinline__ int block_excl_count(bool flag, int* warp_tot, int* total) {
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  unsigned m = __ballot_sync(0xffffffffu, flag);
  int in_warp = __popc(m & ((1u << lane) - 1u));
  if (lane == 0) warp_tot[warp] = __popc(m);
  __syncthreads();
  int before = 0, all = 0;
#pragma unroll
  for (int w = 0; w < kTopkThreads / 32; ++w) {
    int c = warp_tot[w];
    before += (w < warp) ? c : 0;
    all += c;
  }
  __syncthreads();
  *total = all;
  return before + in_warp;
}

// Keys of a row at most this long are staged in shared memory.
constexpr int kTopkSmemKeys = 40960;

// Fused score of history block n of row (b, j): the model score plus the
// prior boost lam * min(g / g_ref, 1) (g shared by all heads).
__device__ __forceinline__ float fuse_prior(const RouteArgs& a, float sc, float gv) {
  return sc + a.lam * fminf(gv / a.g_ref, 1.0f);
}
__device__ __forceinline__ float fused_score(const RouteArgs& a, const float* sr, const float* gr,
                                             int n) {
  float sc = sr[n];
  if (gr != nullptr) sc = fuse_prior(a, sc, gr[n]);
  return sc;
}

__global__ void __launch_bounds__(kTopkThreads) topk_kernel(RouteArgs a) {
  pdl_wait();     // global memory only after the predecessor grid completed
  pdl_trigger();
  extern __shared__ uint32_t keys[];   // [n_hist] when staged
  __shared__ int hist[256];
  __shared__ int warp_tot[kTopkThreads / 32];
  __shared__ uint32_t s_prefix;
  __shared__ int s_remaining;
  const int j = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const long long row = (static_cast<long long>(b) * a.Hh + h) * a.n_own + j;
  int32_t* out = a.idx + row * a.max_sel;
  const float* sr = a.s + row * a.s_ld;
  const float* gr = a.g != nullptr ? a.g + (static_cast<long long>(b) * a.n_own + j) * a.n_hist
                                   : nullptr;
  const int K = a.top_k < a.n_hist ? a.top_k : a.n_hist;
  const bool staged = a.n_hist <= kTopkSmemKeys;
  auto key_at = [&](int n) -> uint32_t {
    return staged ? keys[n] : score_key(fused_score(a, sr, gr, n));
  };

  if (K == a.n_hist) {
    for (int n = threadIdx.x; n < a.n_hist; n += kTopkThreads) out[n] = n;
  } else if (K > 0) {
    if (staged) {
#pragma unroll 4
      for (int n = threadIdx.x; n < a.n_hist; n += kTopkThreads)
        keys[n] = score_key(fused_score(a, sr, gr, n));
      __syncthreads();
    }
    uint32_t prefix = 0, pmask = 0;
    int remaining = K;
    for (int shift = 24; shift >= 0; shift -= 8) {
      for (int i = threadIdx.x; i < 256; i += kTopkThreads) hist[i] = 0;
      __syncthreads();
      for (int n = threadIdx.x; n < a.n_hist; n += kTopkThreads) {
        uint32_t k = key_at(n);
        if ((k & pmask) == prefix) atomicAdd(&hist[(k >> shift) & 255u], 1);
      }
      __syncthreads();
      if (threadIdx.x < 32) {
        // Lane l holds bins 255 - 8l .. 248 - 8l (highest first); a suffix
        // count over lanes finds the bin that holds the remaining-th key.
        const int l = threadIdx.x;
        int cnts[8], tot = 0;
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          cnts[q] = hist[255 - (8 * l + q)];
          tot += cnts[q];
        }
        int incl = tot;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
          const int t = __shfl_up_sync(0xffffffffu, incl, off);
          if (l >= off) incl += t;
        }
        const int excl = incl - tot;
        if (excl < remaining && remaining <= incl) {
          int above = excl, d = 255 - 8 * l;
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            d = 255 - (8 * l + q);
            if (above + cnts[q] >= remaining) break;
            above += cnts[q];
          }
          s_prefix = prefix | (static_cast<uint32_t>(d) << shift);
          s_remaining = remaining - above;
        }
      }
      __syncthreads();
      prefix = s_prefix;
      remaining = s_remaining;
      pmask |= 255u << shift;
      __syncthreads();
    }
    const uint32_t thr = prefix;   // key of the K-th largest score
    const int need_eq = remaining; // how many keys equal to thr are taken
    int pos = 0, eq_seen = 0;
    for (int base = 0; base < a.n_hist; base += kTopkThreads) {
      const int n = base + threadIdx.x;
      uint32_t k = n < a.n_hist ? key_at(n) : 0u;
      bool gt = n < a.n_hist && k > thr;
      bool eq = n < a.n_hist && k == thr;
      int eq_tot, sel_tot;
      int eq_rank = eq_seen + block_excl_count(eq, warp_tot, &eq_tot);
      bool sel = gt || (eq && eq_rank < need_eq);
      int at = pos + block_excl_count(sel, warp_tot, &sel_tot);
      if (sel) out[at] = n;
      pos += sel_tot;
      eq_seen += eq_tot;
    }
  }
  for (int i = threadIdx.x; i < a.n_own; i += kTopkThreads) out[K + i] = a.own_first + i;
  for (int i = K + a.n_own + threadIdx.x; i < a.max_sel; i += kTopkThreads) out[i] = -1;
  if (threadIdx.x == 0) a.cnt[row] = K + a.n_own;
}

// ---------------------------------------------------------------------------
// The page's full route (Methodology Steps 4-5): coverage split, tau-gated
// multiplicative fusion, previous-chunk reservation, mass prefix, window.
// ---------------------------------------------------------------------------
constexpr int kVeloxMaxHist = 32768;   // keys + flags staged in shared memory
constexpr int kVeloxSortMax = 1024;    // largest uncovered budget (K_unc)

struct VeloxArgs {
  const float* coverage;  // [B, n_own] or null
  float eta_cov, tau, mass;
  int k_cov, k_unc, prev_first, n_prev, window_half, ref_first, n_ref;
};

// Radix select over keys[0..n) staged in shared memory: after it, keys above
// *thr are taken, plus the *need_eq lowest-index keys equal to *thr (K total).
__device__ void radix_threshold(const uint32_t* keys, int n, int K, int* hist, uint32_t* s_prefix,
                                int* s_remaining, uint32_t* thr, int* need_eq) {
  uint32_t prefix = 0, pmask = 0;
  int remaining = K;
  for (int shift = 24; shift >= 0; shift -= 8) {
    for (int i = threadIdx.x; i < 256; i += blockDim.x) hist[i] = 0;
    __syncthreads();
    for (int i = threadIdx.x; i < n; i += blockDim.x) {
      const uint32_t k = keys[i];
      if ((k & pmask) == prefix) atomicAdd(&hist[(k >> shift) & 255u], 1);
    }
    __syncthreads();
    if (threadIdx.x < 32) {
      const int l = threadIdx.x;
      int cnts[8], tot = 0;
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        cnts[q] = hist[255 - (8 * l + q)];
        tot += cnts[q];
      }
      int incl = tot;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const int t = __shfl_up_sync(0xffffffffu, incl, off);
        if (l >= off) incl += t;
      }
      const int excl = incl - tot;
      if (excl < remaining && remaining <= incl) {
        int above = excl, d = 255 - 8 * l;
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          d = 255 - (8 * l + q);
          if (above + cnts[q] >= remaining) break;
          above += cnts[q];
        }
        *s_prefix = prefix | (static_cast<uint32_t>(d) << shift);
        *s_remaining = remaining - above;
      }
    }
    __syncthreads();
    prefix = *s_prefix;
    remaining = *s_remaining;
    pmask |= 255u << shift;
    __syncthreads();
  }
  *thr = prefix;
  *need_eq = remaining;
}

// Warp-wide search for the m-th largest of the keys the lanes hold (v, 0 =
// no key): the largest t with #{v >= t} >= m, bit by bit from the top.  The
// caller passes lo <= answer <= hi; the bits above the highest bit where lo
// and hi differ are the answer's too, so the search starts below them.  It
// stops early once a count is exactly m (*exact: #{v >= t} == m).
template <int NV>
__device__ __forceinline__ uint32_t warp_kth_key(const uint32_t (&v)[NV], int m, uint32_t lo,
                                                 uint32_t hi, bool* exact) {
  const int top = lo == hi ? -1 : 31 - __clz(lo ^ hi);
  uint32_t thr = top < 0 ? lo : lo & ~((2u << top) - 1u);
  bool ex = false;
#pragma unroll 1
  for (int bit = top; bit >= 0; --bit) {
    const uint32_t cand = thr | (1u << bit);
    int c = 0;
#pragma unroll
    for (int i = 0; i < NV; ++i) c += v[i] >= cand;
    const int tot = static_cast<int>(__reduce_add_sync(0xffffffffu, static_cast<unsigned>(c)));
    if (tot >= m) {
      thr = cand;
      if (tot == m) {
        ex = true;
        break;
      }
    }
  }
  if (!ex) {
    int c = 0;
#pragma unroll
    for (int i = 0; i < NV; ++i) c += v[i] >= thr;
    ex = static_cast<int>(__reduce_add_sync(0xffffffffu, static_cast<unsigned>(c))) == m;
  }
  *exact = ex;
  return thr;
}

// Candidates of the pivot pass of topk_row_kernel (shared memory, in block
// index order).
constexpr int kTopkCandCap = 512;

// Top K of the n_cand candidate keys ckey[] (blocks cidx[], in ascending
// block order, all >= lo), by one warp holding NV per lane: the K-th
// largest key as in warp_kth_key, then every larger key and the first
// K - #{larger} keys equal to it, written to out[] in block order.
template <int NV>
__device__ __forceinline__ void warp_select_candidates(const uint32_t* ckey, const uint16_t* cidx,
                                                       int n_cand, int K, uint32_t lo,
                                                       int32_t* out) {
  const int lane = threadIdx.x & 31;
  const unsigned below = (1u << lane) - 1u;
  uint32_t v[NV];
  uint32_t hi = 0u;
#pragma unroll
  for (int i = 0; i < NV; ++i) {
    v[i] = i * 32 + lane < n_cand ? ckey[i * 32 + lane] : 0u;
    hi = max(hi, v[i]);
  }
  hi = __reduce_max_sync(0xffffffffu, hi);
  bool ex;
  const uint32_t th = warp_kth_key(v, K, lo, hi, &ex);
  int need_eq = 0;
  if (!ex) {
    int gt = 0;
#pragma unroll
    for (int i = 0; i < NV; ++i) gt += v[i] > th;
    need_eq = K - static_cast<int>(__reduce_add_sync(0xffffffffu, static_cast<unsigned>(gt)));
  }
  int at = 0, eq_before = 0;
#pragma unroll
  for (int i = 0; i < NV; ++i) {
    if (i * 32 >= n_cand) break;
    const bool valid = i * 32 + lane < n_cand;
    const bool is_eq = valid && v[i] == th;
    const unsigned em = __ballot_sync(0xffffffffu, is_eq);
    const int r_eq = eq_before + __popc(em & below);
    const bool sel = valid && (ex ? v[i] >= th : (v[i] > th || (is_eq && r_eq < need_eq)));
    const unsigned sm = __ballot_sync(0xffffffffu, sel);
    if (sel) out[at + __popc(sm & below)] = cidx[i * 32 + lane];
    at += __popc(sm);
    eq_before += __popc(em);
  }
}

// Top-K of a row of at most 128 * KPL history blocks: one CTA of 128
// threads per row, thread t holding the keys of blocks c * 128 + t (c < KPL)
// in registers.
//   1. Search, bit by bit from the top, for the largest t with
//      #{key >= t} >= K (the K-th largest key), one block-wide count per
//      bit.  It stops early once a count is exactly K: those keys are then
//      the top K and no key equal to the K-th is left out.
//   2. Otherwise take the keys > t and the lowest-indexed K - #{key > t}
//      keys equal to t.
//   3. Write the selected blocks in ascending order: one ballot per
//      32-block group, the group totals in shared memory, one barrier.
// For a long row and a small K a pivot pass runs first and usually settles
// the row with far fewer comparisons: warp 0 takes the keys of every 8th
// block as a sample and finds a pivot P, the sample's m-th largest key, m
// chosen so that about 2K keys of the row lie at or above P; one block-wide
// count checks that between K and kTopkCandCap keys do (then P <= the K-th
// largest key, so every key of the top K is a candidate), the candidates are
// compacted in block order into shared memory, and warp 0 selects the top K
// among them as in 1-3 (ties to the lower block).  Otherwise 1-3 run on the
// whole row.
// The selected set and its order are those of topk_kernel.
constexpr int kTopkRowThreads = 128;

template <int KPL>
__global__ void __launch_bounds__(kTopkRowThreads, KPL <= 18 ? 8 : 6) topk_row_kernel(RouteArgs a) {
  pdl_wait();     // global memory only after the predecessor grid completed
  pdl_trigger();
  constexpr int kWarps = kTopkRowThreads / 32;
  __shared__ unsigned part[2][kWarps];
  __shared__ unsigned grp[2][KPL][kWarps];     // per-(group, warp) ballot counts: eq, sel
  constexpr int kSamp = (16 * KPL + 31) / 32;   // sample keys per lane of warp 0
  __shared__ uint32_t samp[32 * kSamp];
  __shared__ uint32_t ckey[kTopkCandCap];
  __shared__ uint16_t cidx[kTopkCandCap];
  __shared__ uint32_t cmask[KPL * kWarps];        // candidate flags, word = 32 blocks
  __shared__ uint32_t kbuf[KPL * kTopkRowThreads];  // candidate keys by block
  __shared__ uint32_t s_pivot;
  const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
  const int j = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const long long row = (static_cast<long long>(b) * a.Hh + h) * a.n_own + j;
  int32_t* out = a.idx + row * a.max_sel;
  const float* sr = a.s + row * a.s_ld;
  const float* gr = a.g != nullptr ? a.g + (static_cast<long long>(b) * a.n_own + j) * a.n_hist
                                   : nullptr;
  const int nh = a.n_hist;
  const int K = a.top_k < nh ? a.top_k : nh;
  if (K == nh) {
    for (int n = t; n < nh; n += kTopkRowThreads) out[n] = n;
  } else if (K > 0) {
    float f[KPL], gv[KPL];
#pragma unroll
    for (int c = 0; c < KPL; ++c) {
      const int n = c * kTopkRowThreads + t;
      f[c] = n < nh ? sr[n] : 0.f;
      gv[c] = (gr != nullptr && n < nh) ? gr[n] : 0.f;
    }
    uint32_t key[KPL];
#pragma unroll
    for (int c = 0; c < KPL; ++c) {
      const int n = c * kTopkRowThreads + t;
      key[c] = n < nh ? score_key(gr != nullptr ? fuse_prior(a, f[c], gv[c]) : f[c]) : 0u;
    }
    // Padding keys are 0: they count only toward t = 0, which every row
    // satisfies anyway, and the selection below skips them by index.
    auto block_count = [&](uint32_t cand, bool strict, int parity) -> int {
      unsigned c0 = 0, c1 = 0;
#pragma unroll
      for (int c = 0; c < KPL; c += 2) {
        c0 += strict ? key[c] > cand : key[c] >= cand;
        if (c + 1 < KPL) c1 += strict ? key[c + 1] > cand : key[c + 1] >= cand;
      }
      const unsigned w = __reduce_add_sync(0xffffffffu, c0 + c1);
      if (lane == 0) part[parity][warp] = w;
      __syncthreads();
      unsigned tot = 0;
#pragma unroll
      for (int i = 0; i < kWarps; ++i) tot += part[parity][i];
      return static_cast<int>(tot);
    };
    // part[] alternates between two buffers: a warp can only overwrite a
    // buffer after the next barrier, which every warp reaches only after
    // reading it.
    int parity = 0;
    const unsigned below = (1u << lane) - 1u;
    bool done = false;
    if (K <= kTopkCandCap / 4 && nh >= 6 * K) {
      // ---- pivot pass ----
      if ((t & 7) == 0) {
#pragma unroll
        for (int c = 0; c < KPL; ++c) samp[(t >> 3) * KPL + c] = key[c];
      }
      for (int i = 16 * KPL + t; i < 32 * kSamp; i += kTopkRowThreads) samp[i] = 0u;
      __syncthreads();
      if (warp == 0) {
        uint32_t v[kSamp];
        int nv = 0;
        uint32_t lo = 0xffffffffu, hi = 0u;
#pragma unroll
        for (int i = 0; i < kSamp; ++i) {
          v[i] = samp[i * 32 + lane];
          nv += v[i] != 0u;
          lo = v[i] != 0u ? min(lo, v[i]) : lo;
          hi = max(hi, v[i]);
        }
        nv = static_cast<int>(__reduce_add_sync(0xffffffffu, static_cast<unsigned>(nv)));
        lo = __reduce_min_sync(0xffffffffu, lo);
        hi = __reduce_max_sync(0xffffffffu, hi);
        // About 2K keys of the row at or above the sample's m-th largest.
        int m = static_cast<int>((2LL * K * nv + nh - 1) / nh);
        m = max(1, min(m, nv));
        bool ex;
        const uint32_t p = warp_kth_key(v, m, lo, hi, &ex);
        if (lane == 0) s_pivot = p;
      }
      __syncthreads();
      const uint32_t piv = s_pivot;
      const int n_cand = block_count(piv, false, parity);
      parity ^= 1;
      if (n_cand >= K && n_cand <= kTopkCandCap) {
        // Candidates in block order through a bitmask: word c * 4 + warp
        // holds the flags of blocks (c * 4 + warp) * 32 + lane, so words
        // ascend with the block; each candidate's key goes to kbuf[block].
#pragma unroll
        for (int c = 0; c < KPL; ++c) {
          const bool cand = key[c] >= piv;
          const unsigned m = __ballot_sync(0xffffffffu, cand);
          if (lane == 0) cmask[c * kWarps + warp] = m;
          if (cand) kbuf[c * kTopkRowThreads + t] = key[c];
        }
        __syncthreads();
        if (warp == 0) {
          // Lane l takes words l, l + 32, ...: one warp scan of the word
          // counts per round places each word's blocks after the earlier
          // words' ones.
          constexpr int kWords = KPL * kWarps;
          int at = 0;
#pragma unroll 1
          for (int w0 = 0; w0 < kWords; w0 += 32) {
            const int w = w0 + lane;
            unsigned m = w < kWords ? cmask[w] : 0u;
            const int cnt = __popc(m);
            int incl = cnt;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
              const int x = __shfl_up_sync(0xffffffffu, incl, off);
              if (lane >= off) incl += x;
            }
            int p = at + incl - cnt;
            while (m != 0u) {
              const int n = w * 32 + __ffs(m) - 1;
              m &= m - 1u;
              ckey[p] = kbuf[n];
              cidx[p] = static_cast<uint16_t>(n);
              ++p;
            }
            at += __shfl_sync(0xffffffffu, incl, 31);
          }
          __syncwarp();
          if (n_cand <= 128)
            warp_select_candidates<4>(ckey, cidx, n_cand, K, piv, out);
          else if (n_cand <= 256)
            warp_select_candidates<8>(ckey, cidx, n_cand, K, piv, out);
          else
            warp_select_candidates<16>(ckey, cidx, n_cand, K, piv, out);
        }
        done = true;
      }
    }
    if (!done) {
      uint32_t thr = 0;
      bool exact = false;
#pragma unroll 1
      for (int bit = 31; bit >= 0; --bit) {
        const uint32_t cand = thr | (1u << bit);
        const int cnt = block_count(cand, false, parity);
        parity ^= 1;
        if (cnt >= K) {
          thr = cand;
          if (cnt == K) { exact = true; break; }
        }
      }
      // exact: take key >= thr (K of them); else key > thr plus the first
      // need_eq keys == thr.
      const int need_eq = exact ? 0 : K - block_count(thr, true, parity);
      bool eq[KPL];
#pragma unroll
      for (int c = 0; c < KPL; ++c) {
        eq[c] = !exact && c * kTopkRowThreads + t < nh && key[c] == thr;
        const unsigned m = __ballot_sync(0xffffffffu, eq[c]);
        if (lane == 0) grp[0][c][warp] = __popc(m);
      }
      __syncthreads();
      bool sel[KPL];
      int before = 0;   // equal keys in earlier groups
#pragma unroll
      for (int c = 0; c < KPL; ++c) {
        const int n = c * kTopkRowThreads + t;
        int rank = before + __popc(__ballot_sync(0xffffffffu, eq[c]) & below);
#pragma unroll
        for (int w = 0; w < kWarps; ++w) {
          const int e = static_cast<int>(grp[0][c][w]);
          rank += w < warp ? e : 0;
          before += e;
        }
        sel[c] = n < nh && (exact ? key[c] >= thr : (key[c] > thr || (eq[c] && rank < need_eq)));
        const unsigned m = __ballot_sync(0xffffffffu, sel[c]);
        if (lane == 0) grp[1][c][warp] = __popc(m);
      }
      __syncthreads();
      int pos = 0;      // selected blocks in earlier groups
#pragma unroll
      for (int c = 0; c < KPL; ++c) {
        int at = pos + __popc(__ballot_sync(0xffffffffu, sel[c]) & below);
#pragma unroll
        for (int w = 0; w < kWarps; ++w) {
          const int e = static_cast<int>(grp[1][c][w]);
          at += w < warp ? e : 0;
          pos += e;
        }
        if (sel[c]) out[at] = c * kTopkRowThreads + t;
      }
    }
  }
  for (int i = t; i < a.n_own; i += kTopkRowThreads) out[K + i] = a.own_first + i;
  for (int i = K + a.n_own + t; i < a.max_sel; i += kTopkRowThreads) out[i] = -1;
  if (t == 0) a.cnt[row] = K + a.n_own;
}

// Block-wide exclusive prefix, over threads in index order, of a per-thread
// count; *total gets the block total.  Two barriers.
__device__ __forceinline__ int block_excl_scan(int v, int* warp_tot, int* total) {
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  int incl = v;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int t = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl += t;
  }
  if (lane == 31) warp_tot[warp] = incl;
  __syncthreads();
  int before = 0, all = 0;
#pragma unroll
  for (int w = 0; w < kTopkThreads / 32; ++w) {
    const int c = warp_tot[w];
    before += (w < warp) ? c : 0;
    all += c;
  }
  __syncthreads();
  *total = all;
  return before + incl - v;
}

// Tree reduction of red[0..255] (already written and synchronised): level w
// combines red[t] and red[t + w] for t < w, w = 128, 64, ..., 1.  The levels
// below 32 run in warp 0 with shuffles, which pair the same operands in the
// same order.  Returns the result to every thread.
template <typename Op>
__device__ __forceinline__ float block_tree(float* red, Op op) {
#pragma unroll
  for (int w = kTopkThreads / 2; w >= 32; w >>= 1) {
    if (threadIdx.x < w) red[threadIdx.x] = op(red[threadIdx.x], red[threadIdx.x + w]);
    __syncthreads();
  }
  if (threadIdx.x < 32) {
    float x = red[threadIdx.x];
#pragma unroll
    for (int w = 16; w > 0; w >>= 1) x = op(x, __shfl_down_sync(0xffffffffu, x, w));
    if (threadIdx.x == 0) red[0] = x;
  }
  __syncthreads();
  const float r = red[0];
  __syncthreads();
  return r;
}

// Each thread owns the contiguous blocks [t * run, min((t+1) * run, nh)), so
// a block scan of per-thread counts orders everything by block index.
constexpr int kVeloxRankMax = 256;   // budgets up to this are ranked by counting

__global__ void __launch_bounds__(kTopkThreads) velox_select_kernel(RouteArgs a, VeloxArgs v) {
  pdl_wait();     // global memory only after the predecessor grid completed
  pdl_trigger();
  extern __shared__ __align__(16) uint8_t vsm[];
  const int nh = a.n_hist;
  uint64_t* sortbuf = reinterpret_cast<uint64_t*>(vsm);                 // [kVeloxSortMax]
  uint32_t* keys = reinterpret_cast<uint32_t*>(sortbuf + kVeloxSortMax); // [nh]
  uint8_t* flag = reinterpret_cast<uint8_t*>(keys + nh);                // [nh]
  __shared__ int hist[256];
  __shared__ int warp_tot[kTopkThreads / 32];
  __shared__ uint32_t s_prefix;
  __shared__ int s_remaining, s_m;
  __shared__ float red[kTopkThreads];
  __shared__ int nidx[kVeloxRankMax];     // sorted position -> block
  __shared__ float pr[kVeloxRankMax];     // sorted position -> softmax probability
  const int t = threadIdx.x;
  const int j = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const long long row = (static_cast<long long>(b) * a.Hh + h) * a.n_own + j;
  int32_t* out = a.idx + row * a.max_sel;
  const float* sr = a.s + row * a.s_ld;
  const float* gr = a.g != nullptr ? a.g + (static_cast<long long>(b) * a.n_own + j) * nh : nullptr;
  const bool covered = v.coverage != nullptr && v.coverage[b * a.n_own + j] >= v.eta_cov;
  const int p0 = min(max(v.prev_first, 0), nh);
  const int p1 = min(max(v.prev_first + v.n_prev, p0), nh);
  const int run = (nh + kTopkThreads - 1) / kTopkThreads;
  const int r0 = min(t * run, nh), r1 = min(r0 + run, nh);

  // Keys > thr, and the need_eq lowest-indexed keys == thr (key 0 never
  // taken): calls take(n) for each, in ascending n within this thread's run.
  // Returns this thread's count before the run and the block total.
  auto select_run = [&](uint32_t thr, int need_eq, auto take) {
    int eq_local = 0;
    for (int n = r0; n < r1; ++n) eq_local += (keys[n] == thr && keys[n] != 0u);
    int eq_tot;
    int eq_rank = block_excl_scan(eq_local, warp_tot, &eq_tot);
    for (int n = r0; n < r1; ++n) {
      const uint32_t k = keys[n];
      if (k == 0u) continue;
      if (k > thr) {
        take(n);
      } else if (k == thr) {
        if (eq_rank < need_eq) take(n);
        ++eq_rank;
      }
    }
  };

  if (covered) {
    // s + log(1 + lam * g_hat) ranks like the renormalised product of the
    // importance distribution and 1 + lam * g_hat; the previous chunk is
    // reserved (key 0 keeps it out of the selection).
    for (int n = t; n < nh; n += kTopkThreads) {
      const bool res = n >= p0 && n < p1;
      float f = sr[n];
      if (gr != nullptr) {
        const float gv = gr[n];
        const float gh = gv > v.tau ? fminf(gv / a.g_ref, 1.0f) : 0.0f;
        f += log1pf(a.lam * gh);
      }
      keys[n] = res ? 0u : score_key(f);
      flag[n] = res ? 1 : 0;
    }
    __syncthreads();
    const int n_res = p1 - p0;
    const int K = max(0, min(v.k_cov - n_res, nh - n_res));
    if (K > 0) {
      uint32_t thr;
      int need_eq;
      radix_threshold(keys, nh, K, hist, &s_prefix, &s_remaining, &thr, &need_eq);
      select_run(thr, need_eq, [&](int n) { flag[n] = 1; });
    }
  } else {
    // The scores are read from global memory once, here; later passes take
    // them back from the keys (key_score inverts score_key exactly).
    float mx = -INFINITY;
    for (int n = t; n < nh; n += kTopkThreads) {
      const float f = sr[n];
      keys[n] = score_key(f);
      flag[n] = 0;
      mx = fmaxf(mx, f);
    }
    const int K = min(v.k_unc, nh);
    if (K > 0) {
      // Row maximum and normaliser of softmax(s), in a fixed order.
      red[t] = mx;
      __syncthreads();
      const float smax = block_tree(red, [](float x, float y) { return fmaxf(x, y); });
      // exp(s - smax) as 2^((s - smax) log2 e) on the MUFU: relative error
      // about 1e-6 for the exponents that matter (s - smax > -20), far
      // inside the route's 1e-4 tolerance on the mass cut.  Every term below
      // (the normaliser, the mass, the ranked probabilities) uses it.
      auto ex = [&](uint32_t k) { return ex2_approx((key_score(k) - smax) * 1.4426950408889634f); };
      float z = 0.f;
      for (int n = t; n < nh; n += kTopkThreads) z += ex(keys[n]);
      red[t] = z;
      __syncthreads();
      const float zsum = block_tree(red, [](float x, float y) { return x + y; });
      const float inv_z = 1.0f / zsum;
      // The K best blocks, then their order by (score descending, index
      // ascending) so the mass prefix can be walked.
      uint32_t thr;
      int need_eq;
      radix_threshold(keys, nh, K, hist, &s_prefix, &s_remaining, &thr, &need_eq);
      // Mass of the K best.  Two fp32 sums of the same K positive terms, in
      // any two orders, differ by at most 2 (K - 1) 2^-24 W, W <= 1 (up to
      // rounding) being the exact total; so when this sum is below the mass
      // cut by more than 1.2e-7 (K + 1), the walk below, whose running sum
      // only grows, stays below the cut to the end and takes all K: their
      // order is not needed.  The K terms are those of the keys above thr
      // plus need_eq copies of the term of thr (equal keys, equal scores),
      // added last.
      float mass_local = 0.f;
      for (int n = r0; n < r1; ++n)
        if (keys[n] > thr) mass_local += ex(keys[n]) * inv_z;
      red[t] = mass_local;
      __syncthreads();
      float mass_k = block_tree(red, [](float x, float y) { return x + y; });
      if (need_eq > 0) {
        const float e_thr = ex(thr) * inv_z;
        for (int i = 0; i < need_eq; ++i) mass_k += e_thr;
      }
      if (mass_k < v.mass - 1.2e-7f * static_cast<float>(K + 1)) {
        select_run(thr, need_eq, [&](int n) { flag[n] = 1; });
      } else {
        int sel_local = 0;
        select_run(thr, need_eq, [&](int) { ++sel_local; });
        int sel_tot;
        int at = block_excl_scan(sel_local, warp_tot, &sel_tot);
        // ascending order of ~((key << 32) | ~n) = descending key, ascending n
        select_run(thr, need_eq, [&](int n) {
          sortbuf[at++] = ~((static_cast<uint64_t>(keys[n]) << 32) |
                            (0xFFFFFFFFu - static_cast<uint32_t>(n)));
        });
        __syncthreads();
        if (K <= kVeloxRankMax) {
          // Rank by counting (the values are distinct): one barrier instead of
          // a sorting network.
          for (int u = t; u < K; u += kTopkThreads) {
            const uint64_t x = sortbuf[u];
            int rank = 0;
            for (int i = 0; i < K; ++i) rank += sortbuf[i] < x;
            const int n = static_cast<int>(0xFFFFFFFFu - static_cast<uint32_t>(~x));
            nidx[rank] = n;
            pr[rank] = ex(keys[n]) * inv_z;
          }
          __syncthreads();
          if (t == 0) {
            float acc = 0.f;
            int m = K;
            for (int r = 0; r < K; ++r) {
              acc += pr[r];
              if (acc >= v.mass) {
                m = r + 1;
                break;
              }
            }
            s_m = m;
          }
          __syncthreads();
          for (int r = t; r < s_m; r += kTopkThreads) flag[nidx[r]] = 1;
        } else {
          int P = 2;
          while (P < K) P <<= 1;
          for (int i = K + t; i < P; i += kTopkThreads) sortbuf[i] = ~0ull;
          __syncthreads();
          for (int kk = 2; kk <= P; kk <<= 1) {
            for (int jj = kk >> 1; jj > 0; jj >>= 1) {
              for (int i = t; i < P; i += kTopkThreads) {
                const int ixj = i ^ jj;
                if (ixj > i) {
                  const uint64_t x = sortbuf[i], y = sortbuf[ixj];
                  const bool up = (i & kk) == 0;
                  if (up ? (x > y) : (x < y)) {
                    sortbuf[i] = y;
                    sortbuf[ixj] = x;
                  }
                }
              }
              __syncthreads();
            }
          }
          if (t == 0) {
            float acc = 0.f;
            int m = K;
            for (int r = 0; r < K; ++r) {
              const int n = static_cast<int>(0xFFFFFFFFu - static_cast<uint32_t>(~sortbuf[r]));
              acc += ex(keys[n]) * inv_z;
              if (acc >= v.mass) {
                m = r + 1;
                break;
              }
            }
            s_m = m;
          }
          __syncthreads();
          for (int r = t; r < s_m; r += kTopkThreads)
            flag[static_cast<int>(0xFFFFFFFFu - static_cast<uint32_t>(~sortbuf[r]))] = 1;
        }
      }
    }
  }
  __syncthreads();
  // Window of previous-chunk blocks around this query block's position, and
  // the reference blocks, outside the budget.
  for (int pos = j - v.window_half + t; pos <= j + v.window_half; pos += kTopkThreads) {
    const int n = v.prev_first + pos;
    if (pos >= 0 && pos < v.n_prev && n >= 0 && n < nh) flag[n] = 1;
  }
  for (int r = t; r < v.n_ref; r += kTopkThreads) {
    const int n = v.ref_first + r;
    if (n >= 0 && n < nh) flag[n] = 1;
  }
  __syncthreads();
  int mine = 0;
  for (int n = r0; n < r1; ++n) mine += flag[n];
  int pos;
  int at = block_excl_scan(mine, warp_tot, &pos);
  for (int n = r0; n < r1; ++n)
    if (flag[n]) {
      if (at < a.max_sel) out[at] = n;
      ++at;
    }
  const int c = min(pos, a.max_sel - a.n_own);
  if (pos + a.n_own > a.max_sel && t == 0) report(a.d_err, BSA_DEV_BAD_COUNT);
  for (int i = t; i < a.n_own; i += kTopkThreads) out[c + i] = a.own_first + i;
  for (int i = c + a.n_own + t; i < a.max_sel; i += kTopkThreads) out[i] = -1;
  if (t == 0) a.cnt[row] = c + a.n_own;
}

static size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

static void route_ws_layout(int B, int Hh, int D, int n_own, int n_hist, size_t* qm_bytes,
                            size_t* s_bytes) {
  *qm_bytes = align256(sizeof(float) * static_cast<size_t>(B) * Hh * n_own * D);
  *s_bytes = align256(sizeof(float) * static_cast<size_t>(B) * Hh * n_own *
                      static_cast<size_t>(n_hist > 0 ? (n_hist + 31) & ~31 : 0));
}

}  // namespace bsa

using namespace bsa;

extern "C" bsa_status bsa_route_workspace_size(int B, int Hh, int D, int n_q_blocks, int n_hist,
                                               size_t* bytes) {
  if (bytes == nullptr || B <= 0 || Hh <= 0 || n_q_blocks <= 0 || n_hist < 0)
    return BSA_ERR_INVALID_ARG;
  if (D != 64 && D != 128) return BSA_ERR_UNSUPPORTED;
  size_t a, b;
  route_ws_layout(B, Hh, D, n_q_blocks, n_hist, &a, &b);
  *bytes = a + b;
  return BSA_OK;
}

namespace bsa {

// Validation shared by both routes, the query means and the model scores
// (from the pooled-key cache or by streaming the history keys).  Fills `a`
// for the selection kernel the caller launches next.
// The query means come from q_blk (pooled here, by pool_q_kernel) or, when
// q_mean is given, from the caller (q_blk is then not read).
static bsa_status route_scores(const void* q_blk, const float* q_mean, const bsa_kv_cache* c,
                               const int32_t* q_valid, int n_hist, int own_first, int n_own,
                               const float* g, float lambda, float g_ref, float sm_scale,
                               int32_t* idx, int32_t* cnt, int max_sel, void* workspace,
                               size_t ws_bytes, int32_t* d_err, cudaStream_t s, RouteArgs* out) {
  if ((q_blk == nullptr && q_mean == nullptr) || c == nullptr || idx == nullptr ||
      cnt == nullptr || workspace == nullptr || c->k == nullptr || c->block_valid == nullptr)
    return BSA_ERR_INVALID_ARG;
  if (q_mean != nullptr && !aligned16(q_mean)) return BSA_ERR_INVALID_ARG;
  if (q_mean != nullptr) q_blk = c->k;  // not read; keeps the alignment check below uniform
  if (c->B <= 0 || c->Hh <= 0 || n_own <= 0 || n_hist < 0 || max_sel <= 0)
    return BSA_ERR_INVALID_ARG;
  if (c->D != 64 && c->D != 128) return BSA_ERR_UNSUPPORTED;
  if (!(sm_scale == sm_scale) || (g != nullptr && !(g_ref > 0.f)) || !(lambda == lambda))
    return BSA_ERR_INVALID_ARG;
  if (!aligned16(q_blk) || !aligned16(c->k) || (reinterpret_cast<uintptr_t>(workspace) & 255u) ||
      (c->kmean != nullptr && !aligned16(c->kmean)))
    return BSA_ERR_INVALID_ARG;
  if (own_first < n_hist || own_first < 0 || own_first + n_own > c->n_blocks ||
      c->n_blocks > c->max_blocks || c->B > 65535 || c->Hh > 65535 || n_own > 65535)
    return BSA_ERR_SHAPE;
  size_t qm_b, s_b;
  route_ws_layout(c->B, c->Hh, c->D, n_own, n_hist, &qm_b, &s_b);
  if (ws_bytes < qm_b + s_b) return BSA_ERR_CAPACITY;
  const size_t qm_smem = sizeof(float) * static_cast<size_t>(n_own) * c->D;
  if (qm_smem > 200 * 1024) return BSA_ERR_UNSUPPORTED;
  const int nq16 = (n_own + 15) & ~15;
  const size_t mean_smem = sizeof(float) * static_cast<size_t>(nq16 + kMeanTileN) * (c->D + 4);
  if (c->kmean != nullptr && mean_smem > 200 * 1024) return BSA_ERR_UNSUPPORTED;

  RouteArgs& a = *out;
  a = RouteArgs{};
  a.q = static_cast<const uint4*>(q_blk);
  a.kc = static_cast<const uint4*>(c->k);
  a.block_valid = c->block_valid;
  a.q_valid = q_valid;
  a.g = g;
  a.kmean = c->kmean;
  a.qm = q_mean != nullptr ? const_cast<float*>(q_mean) : static_cast<float*>(workspace);
  a.s = reinterpret_cast<float*>(static_cast<char*>(workspace) + qm_b);
  a.idx = idx;
  a.cnt = cnt;
  a.d_err = d_err;
  a.B = c->B;
  a.Hh = c->Hh;
  a.n_own = n_own;
  a.n_hist = n_hist;
  a.own_first = own_first;
  a.max_blocks = c->max_blocks;
  a.max_sel = max_sel;
  a.s_ld = (n_hist + 31) & ~31;
  a.sm_scale = sm_scale;
  a.lam = lambda;
  a.g_ref = g_ref;

  dim3 pgrid((n_own + kPoolQWarps - 1) / kPoolQWarps, c->Hh, c->B);
  const int per_cta = kScoreWarps * kScoreBlocksPerWarp;
  dim3 sgrid((n_hist + per_cta - 1) / per_cta, c->Hh, c->B);
  dim3 mgrid((n_hist + kMeanTileN - 1) / kMeanTileN, c->Hh, c->B);
  const bool tc = n_hist > 0 && c->kmean != nullptr && score_means_tc_fits(n_own, c->D) &&
                  static_cast<long long>(c->B) * c->Hh <= (1 << 24);
  if (c->D == 128) {
    if (q_mean == nullptr)
      BSA_TRY(launch_pdl(pool_q_kernel<16>, pgrid, dim3(kPoolQWarps * 32), 0, s, a));
    if (tc) {
      BSA_TRY(launch_score_means_tc(a.qm, c->kmean, a.s, a.s_ld, c->B * c->Hh, n_own, n_hist,
                                    c->max_blocks, c->D, sm_scale, device_sms(), d_err, s));
    } else if (n_hist > 0 && c->kmean != nullptr) {
      if (cudaFuncSetAttribute(score_means_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               static_cast<int>(mean_smem)) != cudaSuccess)
        return BSA_ERR_CUDA;
      BSA_TRY(launch_pdl(score_means_kernel<128>, mgrid, dim3(kMeanThreads), mean_smem, s, a));
    } else if (n_hist > 0) {
      if (cudaFuncSetAttribute(pool_score_kernel<16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               static_cast<int>(qm_smem)) != cudaSuccess)
        return BSA_ERR_CUDA;
      BSA_TRY(launch_pdl(pool_score_kernel<16>, sgrid, dim3(kScoreWarps * 32), qm_smem, s, a));
    }
  } else {
    if (q_mean == nullptr)
      BSA_TRY(launch_pdl(pool_q_kernel<8>, pgrid, dim3(kPoolQWarps * 32), 0, s, a));
    if (tc) {
      BSA_TRY(launch_score_means_tc(a.qm, c->kmean, a.s, a.s_ld, c->B * c->Hh, n_own, n_hist,
                                    c->max_blocks, c->D, sm_scale, device_sms(), d_err, s));
    } else if (n_hist > 0 && c->kmean != nullptr) {
      if (cudaFuncSetAttribute(score_means_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               static_cast<int>(mean_smem)) != cudaSuccess)
        return BSA_ERR_CUDA;
      BSA_TRY(launch_pdl(score_means_kernel<64>, mgrid, dim3(kMeanThreads), mean_smem, s, a));
    } else if (n_hist > 0) {
      if (cudaFuncSetAttribute(pool_score_kernel<8>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               static_cast<int>(qm_smem)) != cudaSuccess)
        return BSA_ERR_CUDA;
      BSA_TRY(launch_pdl(pool_score_kernel<8>, sgrid, dim3(kScoreWarps * 32), qm_smem, s, a));
    }
  }
  return launch_status();
}

}  // namespace bsa

using namespace bsa;

namespace bsa {

// bsa_route and bsa_route_qmean: scores (query means from q_blk or given),
// then the top-K of every row.
static bsa_status route_topk(const void* q_blk, const float* q_mean, const bsa_kv_cache* c,
                             const int32_t* q_valid, int n_hist, int own_first, int n_own,
                             const float* g, float lambda, float g_ref, float sm_scale, int top_k,
                             int32_t* idx, int32_t* cnt, int max_sel, void* workspace,
                             size_t ws_bytes, int32_t* d_err, void* stream) {
  if (top_k < 0) return BSA_ERR_INVALID_ARG;
  const int K = top_k < n_hist ? top_k : n_hist;
  if (n_hist >= 0 && n_own > 0 && max_sel > 0 && max_sel < K + n_own) return BSA_ERR_CAPACITY;
  cudaStream_t s = as_stream(stream);
  RouteArgs a;
  bsa_status st = route_scores(q_blk, q_mean, c, q_valid, n_hist, own_first, n_own, g, lambda,
                               g_ref, sm_scale, idx, cnt, max_sel, workspace, ws_bytes, d_err, s,
                               &a);
  if (st != BSA_OK) return st;
  a.top_k = top_k;
  // Rows of up to 3072 history blocks: keys in registers (their count per
  // thread follows the row length); longer rows: a radix select over keys
  // staged in shared memory.  One CTA per row either way.
  dim3 qgrid(n_own, c->Hh, c->B);
  if (n_hist <= kTopkRowThreads * 24) {
    if (n_hist <= kTopkRowThreads * 4)
      BSA_TRY(launch_pdl(topk_row_kernel<4>, qgrid, dim3(kTopkRowThreads), 0, s, a));
    else if (n_hist <= kTopkRowThreads * 10)
      BSA_TRY(launch_pdl(topk_row_kernel<10>, qgrid, dim3(kTopkRowThreads), 0, s, a));
    else if (n_hist <= kTopkRowThreads * 18)
      BSA_TRY(launch_pdl(topk_row_kernel<18>, qgrid, dim3(kTopkRowThreads), 0, s, a));
    else
      BSA_TRY(launch_pdl(topk_row_kernel<24>, qgrid, dim3(kTopkRowThreads), 0, s, a));
    return launch_status();
  }
  const size_t topk_smem =
      n_hist <= kTopkSmemKeys ? sizeof(uint32_t) * static_cast<size_t>(n_hist > 0 ? n_hist : 1) : 0;
  if (cudaFuncSetAttribute(topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(topk_smem)) != cudaSuccess)
    return BSA_ERR_CUDA;
  BSA_TRY(launch_pdl(topk_kernel, qgrid, dim3(kTopkThreads), topk_smem, s, a));
  return launch_status();
}

}  // namespace bsa

extern "C" bsa_status bsa_route(const void* q_blk, const bsa_kv_cache* c, const int32_t* q_valid,
                                int n_hist, int own_first, int n_own, const float* g,
                                float lambda, float g_ref, float sm_scale, int top_k, int32_t* idx,
                                int32_t* cnt, int max_sel, void* workspace, size_t ws_bytes,
                                int32_t* d_err, void* stream) {
  if (q_blk == nullptr) return BSA_ERR_INVALID_ARG;
  return route_topk(q_blk, nullptr, c, q_valid, n_hist, own_first, n_own, g, lambda, g_ref,
                    sm_scale, top_k, idx, cnt, max_sel, workspace, ws_bytes, d_err, stream);
}

extern "C" bsa_status bsa_route_qmean(const float* q_mean, const bsa_kv_cache* c, int n_hist,
                                      int own_first, int n_own, const float* g, float lambda,
                                      float g_ref, float sm_scale, int top_k, int32_t* idx,
                                      int32_t* cnt, int max_sel, void* workspace, size_t ws_bytes,
                                      int32_t* d_err, void* stream) {
  if (q_mean == nullptr) return BSA_ERR_INVALID_ARG;
  return route_topk(nullptr, q_mean, c, nullptr, n_hist, own_first, n_own, g, lambda, g_ref,
                    sm_scale, top_k, idx, cnt, max_sel, workspace, ws_bytes, d_err, stream);
}

// bsa_route_velox and bsa_route_velox_qmean: the scores (query means from
// q_blk or given), then the page's selection.
static bsa_status route_velox(const void* q_blk, const float* q_mean, const bsa_kv_cache* c,
                              const int32_t* q_valid, int n_hist, int own_first, int n_own,
                              const float* g, float lambda, float g_ref, float sm_scale,
                              const bsa_velox_route* opts, int32_t* idx, int32_t* cnt,
                              int max_sel, void* workspace, size_t ws_bytes, int32_t* d_err,
                              void* stream) {
  if (opts == nullptr) return BSA_ERR_INVALID_ARG;
  const bsa_velox_route& o = *opts;
  if (o.k_cov < 0 || o.k_unc < 0 || o.n_prev < 0 || o.window_half < 0 || o.n_ref < 0 ||
      !(o.mass == o.mass) || !(o.tau == o.tau) || !(o.eta_cov == o.eta_cov))
    return BSA_ERR_INVALID_ARG;
  if (o.k_unc > kVeloxSortMax || n_hist > kVeloxMaxHist) return BSA_ERR_UNSUPPORTED;
  // Largest route a query block can get: its budgeted part, the window and
  // the reference blocks (all history), then its own chunk.
  const int p0 = std::min(std::max(o.prev_first, 0), std::max(n_hist, 0));
  const int p1 = std::min(std::max(o.prev_first + o.n_prev, p0), std::max(n_hist, 0));
  const long long budget = std::max<long long>(std::max(o.k_cov, p1 - p0), o.k_unc);
  const long long bound =
      std::min<long long>(n_hist, budget + 2LL * o.window_half + 1 + o.n_ref) + n_own;
  if (max_sel < bound) return BSA_ERR_CAPACITY;
  cudaStream_t s = as_stream(stream);
  RouteArgs a;
  bsa_status st = route_scores(q_blk, q_mean, c, q_valid, n_hist, own_first, n_own, g, lambda,
                               g_ref, sm_scale, idx, cnt, max_sel, workspace, ws_bytes, d_err, s,
                               &a);
  if (st != BSA_OK) return st;
  VeloxArgs v{o.coverage, o.eta_cov, o.tau, o.mass, o.k_cov, o.k_unc, o.prev_first, o.n_prev,
              o.window_half, o.ref_first, o.n_ref};
  const size_t smem = sizeof(uint64_t) * kVeloxSortMax +
                      static_cast<size_t>(std::max(n_hist, 1)) * (sizeof(uint32_t) + 1) + 16;
  if (cudaFuncSetAttribute(velox_select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(smem)) != cudaSuccess)
    return BSA_ERR_CUDA;
  dim3 qgrid(n_own, c->Hh, c->B);
  BSA_TRY(launch_pdl(velox_select_kernel, qgrid, dim3(kTopkThreads), smem, s, a, v));
  return launch_status();
}

extern "C" bsa_status bsa_route_velox(const void* q_blk, const bsa_kv_cache* c,
                                      const int32_t* q_valid, int n_hist, int own_first,
                                      int n_own, const float* g, float lambda, float g_ref,
                                      float sm_scale, const bsa_velox_route* opts, int32_t* idx,
                                      int32_t* cnt, int max_sel, void* workspace, size_t ws_bytes,
                                      int32_t* d_err, void* stream) {
  if (q_blk == nullptr) return BSA_ERR_INVALID_ARG;
  return route_velox(q_blk, nullptr, c, q_valid, n_hist, own_first, n_own, g, lambda, g_ref,
                     sm_scale, opts, idx, cnt, max_sel, workspace, ws_bytes, d_err, stream);
}

extern "C" bsa_status bsa_route_velox_qmean(const float* q_mean, const bsa_kv_cache* c,
                                            int n_hist, int own_first, int n_own, const float* g,
                                            float lambda, float g_ref, float sm_scale,
                                            const bsa_velox_route* opts, int32_t* idx,
                                            int32_t* cnt, int max_sel, void* workspace,
                                            size_t ws_bytes, int32_t* d_err, void* stream) {
  if (q_mean == nullptr) return BSA_ERR_INVALID_ARG;
  return route_velox(nullptr, q_mean, c, nullptr, n_hist, own_first, n_own, g, lambda, g_ref,
                     sm_scale, opts, idx, cnt, max_sel, workspace, ws_bytes, d_err, stream);
}

// ---------------------------------------------------------------------------
// bsa_route_noalloc: routing for callers that must not allocate device memory
// ---------------------------------------------------------------------------
// The router needs scratch for the query-block means and the fused scores.
// bsa_route takes it from the caller; this variant keeps it in one fixed
// array that lives in the library's own device image, so a caller never has
// to obtain device memory for it.  The array exists once per GPU that loads
// the library and stays resident until the process exits.
namespace bsa {

constexpr size_t kNoAllocScratchBytes = BSA_ROUTE_NOALLOC_SCRATCH_BYTES;
static __device__ __align__(256) unsigned char g_route_scratch[kNoAllocScratchBytes];

constexpr int kMaxScratchDevices = 64;
struct ScratchEntry {
  unsigned long long ctx_id;  // unique id of the context the address belongs to
  void* addr;
};
static ScratchEntry g_scratch[kMaxScratchDevices];
static std::mutex g_scratch_mutex;

using CtxGetCurrentFn = CUresult (*)(CUcontext*);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long*);

// Driver entry points for the current context and its process-unique id,
// found through the runtime (the library does not link the driver library).
static bool context_id(unsigned long long* id) {
  static CtxGetCurrentFn get_current = nullptr;
  static CtxGetIdFn get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<CtxGetCurrentFn>(p);
    p = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<CtxGetIdFn>(p);
  });
  if (get_current == nullptr || get_id == nullptr) return false;
  CUcontext ctx = nullptr;
  if (get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr) return false;
  return get_id(ctx, id) == CUDA_SUCCESS;
}

// Device address of g_route_scratch in the current context.  Host code cannot
// use the symbol itself (on the host it names a shadow object, not device
// memory), so the address is looked up with the device current.  It belongs
// to the context that loaded the library's module, so it is cached per device
// together with that context's process-unique id: a device reset or another
// context on the device has a new id, and the address is looked up again
// instead of reusing one that is no longer mapped.
static bsa_status noalloc_scratch(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return BSA_ERR_CUDA;
  if (dev < 0 || dev >= kMaxScratchDevices) return BSA_ERR_UNSUPPORTED;
  // When no context is current on this thread yet, cudaSetDevice makes the
  // device's primary context current (it allocates nothing).
  unsigned long long id = 0;
  if (!context_id(&id)) {
    if (cudaSetDevice(dev) != cudaSuccess || !context_id(&id)) return BSA_ERR_CUDA;
  }
  std::lock_guard<std::mutex> lock(g_scratch_mutex);
  ScratchEntry& e = g_scratch[dev];
  if (e.addr == nullptr || e.ctx_id != id) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_route_scratch) != cudaSuccess || p == nullptr)
      return BSA_ERR_CUDA;
    e.addr = p;
    e.ctx_id = id;
  }
  *out = e.addr;
  return BSA_OK;
}

}  // namespace bsa

extern "C" bsa_status bsa_route_noalloc(const void* q_blk, const bsa_kv_cache* c,
                                        const int32_t* q_valid, int n_hist, int own_first,
                                        int n_own, const float* g, float lambda, float g_ref,
                                        float sm_scale, int top_k, int32_t* idx, int32_t* cnt,
                                        int max_sel, int32_t* d_err, void* stream) {
  if (c == nullptr) return BSA_ERR_INVALID_ARG;
  size_t need = 0;
  bsa_status st = bsa_route_workspace_size(c->B, c->Hh, c->D, n_own, n_hist, &need);
  if (st != BSA_OK) return st;
  if (need > bsa::kNoAllocScratchBytes) return BSA_ERR_CAPACITY;
  void* scratch = nullptr;
  st = bsa::noalloc_scratch(&scratch);
  if (st != BSA_OK) return st;
  return bsa_route(q_blk, c, q_valid, n_hist, own_first, n_own, g, lambda, g_ref, sm_scale, top_k,
                   idx, cnt, max_sel, scratch, bsa::kNoAllocScratchBytes, d_err, stream);
}
