// reorder.cu - Gilbert-ordered block storage: bsa_kv_append,
// bsa_tokens_to_blocks, bsa_blocks_to_tokens and bsa_gilbert_perm.
//
// "Velox: Spatial Memory Makes World Models Efficient", Key Contributions 3
// and Methodology Step 6: KV is stored as 128-token blocks along a
// global-aligned Gilbert curve, so a block is a compact patch of latent
// cells and skipping a block skips one contiguous tile load.
//
// The move is a pure HBM stream: every (token, head) row of D bf16 values is
// read once and written once.  A CTA takes 32 curve slots x 8 heads; thread
// t moves 16-byte vectors so that a warp reads 2 KB of consecutive heads of
// one token and writes whole 256-byte cache rows.  Each thread keeps eight
// vectors in flight per tensor.
#include <stdio.h>

#include "common.cuh"
#include "gilbert.cuh"
#include "pool.cuh"

namespace bsa {

// The curve walk kept out of line: the kernels' table path stays compact.
__device__ __noinline__ int curve_token_call(int T, int H, int W, int p) {
  return curve_token(T, H, W, p);
}

constexpr int kRowsPerCta = 32;
constexpr int kHeadsPerCta = 8;
constexpr int kReorderThreads = 256;
constexpr int kInflight = 8;

struct ReorderArgs {
  const uint4* src0;
  uint4* dst0;
  const uint4* src1;  // optional second tensor (V of an append)
  uint4* dst1;
  const int32_t* perm;  // [N] token -> curve slot
  int32_t* block_valid; // optional: written for the chunk's blocks
  int32_t* d_err;
  int N;                // tokens in the chunk
  int nb;               // blocks of the chunk
  int B, Hh;
  long long blk_stride; // blocks per (b, h) in the block tensor
  int base_block;       // first block of the chunk in the block tensor
  int T, H, W;          // chunk grid (used when perm is NULL)
};

// kToBlocks: raster tokens -> block slots (scatter, zero pads).
// !kToBlocks: block slots -> raster tokens (gather).
template <int VPR, bool kToBlocks>
__global__ void __launch_bounds__(kReorderThreads)
reorder_kernel(ReorderArgs a) {
  pdl_wait();     // global memory only after the predecessor grid completed
  pdl_trigger();
  // Row rr of the CTA moves token s_tk[rr] to curve slot s_slot[rr].  With a
  // table, rows are tokens (slot = perm[token]; a scatter into blocks also
  // covers the chunk's pad slots as rows past N).  Without one (perm ==
  // NULL), rows are curve slots and each locates its token on the curve.
  __shared__ int s_slot[kRowsPerCta];
  __shared__ int s_tk[kRowsPerCta];
  const int r0 = blockIdx.x * kRowsPerCta;
  const int h0 = blockIdx.y * kHeadsPerCta;
  const int b = blockIdx.z;
  const bool by_slot = a.perm == nullptr;
  const int rows_total = (kToBlocks || by_slot) ? a.nb * kBlk : a.N;

  if (threadIdx.x < kRowsPerCta) {
    const int r = r0 + threadIdx.x;
    int slot = -1, tk = -1;
    if (by_slot) {
      if (r < rows_total) {
        slot = r;
        tk = r < a.N ? curve_token_call(a.T, a.H, a.W, r) : -1;
      }
    } else if (r < a.N) {
      const int p = __ldg(a.perm + r);
      if (p < 0 || p >= a.N) {
        report(a.d_err, BSA_DEV_BAD_PERM);
      } else {
        slot = p;
        tk = r;
      }
    } else if (kToBlocks && r < rows_total) {
      slot = r;  // pad slot: zero-filled
    }
    if (!kToBlocks && tk < 0) slot = -1;   // nothing to write for a pad slot
    s_slot[threadIdx.x] = slot;
    s_tk[threadIdx.x] = tk;
    if (kToBlocks && a.block_valid != nullptr && blockIdx.y == 0 && b == 0 && r < rows_total &&
        (r % kBlk) == 0) {
      int blk = r / kBlk;
      int v = a.N - blk * kBlk;
      a.block_valid[a.base_block + blk] = v < kBlk ? v : kBlk;
    }
  }
  __syncthreads();

  constexpr int kVecPerRow = VPR;
  constexpr int kWork = kRowsPerCta * kHeadsPerCta * kVecPerRow;
  const long long tok_row_vecs = static_cast<long long>(a.Hh) * kVecPerRow;

  for (int base = threadIdx.x; base < kWork; base += kReorderThreads * kInflight) {
    uint4 v0[kInflight], v1[kInflight];
    long long dsto[kInflight];
    bool live[kInflight];
#pragma unroll
    for (int u = 0; u < kInflight; ++u) {
      int e = base + u * kReorderThreads;
      live[u] = false;
      dsto[u] = 0;
      if (e >= kWork) continue;
      int v = e % kVecPerRow;
      int hh = (e / kVecPerRow) % kHeadsPerCta;
      int rr = e / (kVecPerRow * kHeadsPerCta);
      int h = h0 + hh;
      int r = r0 + rr;
      const int slot = s_slot[rr];
      if (h >= a.Hh || r >= rows_total || slot < 0) continue;
      const int tk = s_tk[rr];
      long long blk_row = (static_cast<long long>(b) * a.Hh + h) * a.blk_stride * kBlk +
                          static_cast<long long>(a.base_block) * kBlk + slot;
      long long tok_row = (static_cast<long long>(b) * a.N + (tk < 0 ? 0 : tk)) * tok_row_vecs +
                          static_cast<long long>(h) * kVecPerRow;
      live[u] = true;
      if (kToBlocks) {
        dsto[u] = blk_row * kVecPerRow + v;
        if (tk >= 0) {
          v0[u] = ld_nc_v4(a.src0 + tok_row + v);
          if (a.src1 != nullptr) v1[u] = ld_nc_v4(a.src1 + tok_row + v);
        } else {
          v0[u] = make_uint4(0, 0, 0, 0);
          v1[u] = make_uint4(0, 0, 0, 0);
        }
      } else {
        dsto[u] = tok_row + v;
        v0[u] = ld_nc_v4(a.src0 + blk_row * kVecPerRow + v);
      }
    }
#pragma unroll
    for (int u = 0; u < kInflight; ++u) {
      if (!live[u]) continue;
      st_v4(a.dst0 + dsto[u], v0[u]);
      if (kToBlocks && a.dst1 != nullptr) st_v4(a.dst1 + dsto[u], v1[u]);
    }
  }
}

template <bool kToBlocks>
static bsa_status launch_reorder(const ReorderArgs& a, int D, cudaStream_t s) {
  const int rows = (kToBlocks || a.perm == nullptr) ? a.nb * kBlk : a.N;
  dim3 grid((rows + kRowsPerCta - 1) / kRowsPerCta, (a.Hh + kHeadsPerCta - 1) / kHeadsPerCta,
            a.B);
  if (D == 128) {
    return launch_pdl(reorder_kernel<16, kToBlocks>, grid, dim3(kReorderThreads), 0, s, a);
  }
  return launch_pdl(reorder_kernel<8, kToBlocks>, grid, dim3(kReorderThreads), 0, s, a);
}

// Pooled-key cache: one warp per (b, h, block) writes the fp32 mean of the
// block's valid key rows (the router's own pooling code, pool.cuh).
constexpr int kMeanWarps = 8;

template <int VPR>
__global__ void __launch_bounds__(kMeanWarps * 32)
block_mean_kernel(const uint4* kc, const int32_t* block_valid, float* kmean, int Hh,
                  int max_blocks, int first, int count, int32_t* d_err) {
  constexpr int D = VPR * 8;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int i = blockIdx.x * kMeanWarps + warp;
  if (i >= count) return;
  const int n = first + i;
  const long long bh = static_cast<long long>(blockIdx.z) * Hh + blockIdx.y;
  int valid = block_valid[n];
  if (valid < 1 || valid > kBlk) {
    report(d_err, BSA_DEV_BAD_VALID);
    valid = valid < 1 ? 1 : kBlk;
  }
  const int c = lane % VPR, g = lane / VPR;
  float km[8];
  warp_block_mean<VPR>(kc + (bh * max_blocks + n) * kBlk * VPR, valid, c, g, km);
  if (g == 0) {
    float4* out = reinterpret_cast<float4*>(kmean + (bh * max_blocks + n) * D + c * 8);
    out[0] = make_float4(km[0], km[1], km[2], km[3]);
    out[1] = make_float4(km[4], km[5], km[6], km[7]);
  }
}

static bsa_status launch_block_means(const bsa_kv_cache* c, int first, int count, int32_t* d_err,
                                     cudaStream_t s) {
  if (count <= 0) return BSA_OK;
  dim3 grid((count + kMeanWarps - 1) / kMeanWarps, c->Hh, c->B);
  const uint4* kc = static_cast<const uint4*>(c->k);
  if (c->D == 128)
    block_mean_kernel<16><<<grid, kMeanWarps * 32, 0, s>>>(kc, c->block_valid, c->kmean, c->Hh,
                                                           c->max_blocks, first, count, d_err);
  else
    block_mean_kernel<8><<<grid, kMeanWarps * 32, 0, s>>>(kc, c->block_valid, c->kmean, c->Hh,
                                                          c->max_blocks, first, count, d_err);
  return launch_status();
}

// Slot -> token for the 128 curve slots [slot0, slot0 + 128) of one block:
// s_tok[d] is the raster token whose perm entry is slot0 + d, or -1.  The
// CTA's NT threads (NT >= 128) scan perm in rounds of kScan independent loads
// per thread (one L2 round trip per round); entries outside [0, N) are
// skipped, and reported when `report_bad`.  Ends with a CTA barrier.
// s_tok[d] = the token at curve slot slot0 + d (d < 128), or -1 for a pad
// slot.  With a table, the CTA scans perm (token -> slot); without one
// (perm == NULL), each thread locates its slot on the curve.
template <int NT>
__device__ __forceinline__ void invert_block_slots(const int32_t* perm, int N, int slot0,
                                                   int* s_tok, bool report_bad, int32_t* d_err,
                                                   int T, int H, int W) {
  static_assert(NT >= kBlk, "one thread per slot clears the table");
  if (perm == nullptr) {
    if (threadIdx.x < kBlk) {
      const int p = slot0 + static_cast<int>(threadIdx.x);
      s_tok[threadIdx.x] = p < N ? curve_token_call(T, H, W, p) : -1;
    }
    __syncthreads();
    return;
  }
  if (threadIdx.x < kBlk) s_tok[threadIdx.x] = -1;
  __syncthreads();
  auto take = [&](int r, int p) {
    if (p < 0 || p >= N) {
      if (report_bad) report(d_err, BSA_DEV_BAD_PERM);
      return;
    }
    const unsigned d = static_cast<unsigned>(p - slot0);
    if (d < static_cast<unsigned>(kBlk)) s_tok[d] = r;
  };
  constexpr int kScan = 16;
  // Four entries per load when perm is 16-byte aligned: one round of loads
  // covers 64 * NT tokens, so a chunk's scan costs one memory latency.
  int done = 0;
  if ((reinterpret_cast<uintptr_t>(perm) & 15u) == 0) {
    const int n4 = N / 4;
    const int4* perm4 = reinterpret_cast<const int4*>(perm);
    for (int base = 0; base < n4; base += kScan * NT) {
      int4 pv[kScan];
#pragma unroll
      for (int k = 0; k < kScan; ++k) {
        const int i = base + threadIdx.x + k * NT;
        pv[k] = i < n4 ? __ldg(perm4 + i) : make_int4(0, 0, 0, 0);
      }
#pragma unroll
      for (int k = 0; k < kScan; ++k) {
        const int i = base + threadIdx.x + k * NT;
        if (i >= n4) break;
        take(4 * i, pv[k].x);
        take(4 * i + 1, pv[k].y);
        take(4 * i + 2, pv[k].z);
        take(4 * i + 3, pv[k].w);
      }
    }
    done = 4 * n4;
  }
  for (int base = done; base < N; base += kScan * NT) {
    int pv[kScan];
#pragma unroll
    for (int k = 0; k < kScan; ++k) {
      const int r = base + threadIdx.x + k * NT;
      pv[k] = r < N ? __ldg(perm + r) : 0;
    }
#pragma unroll
    for (int k = 0; k < kScan; ++k) {
      const int r = base + threadIdx.x + k * NT;
      if (r >= N) break;
      take(r, pv[k]);
    }
  }
  __syncthreads();
}

// Fused append for chunks of up to kGatherMaxTokens tokens: one CTA per
// (chunk block, group of kAppendHeads heads, batch) gathers the block's 128
// curve slots from the token-major K and V and writes whole cache rows; each
// K warp owns one head and pools the block's key rows with the router's
// summation (pool.cuh) while it moves them, so the pooled-key cache costs
// no second pass over K.  The CTA inverts the caller's permutation for its
// own slots by scanning it (perm is small and L2-resident at these sizes).
constexpr int kAppendHeads = 4;
constexpr int kAppendThreads = 2 * kAppendHeads * 32;  // K warps, then V warps
constexpr int kGatherMaxTokens = 1 << 14;

struct AppendArgs {
  const uint4* k_tok;
  const uint4* v_tok;
  uint4* kc;
  uint4* vc;
  float* kmean;         // optional
  const int32_t* perm;
  int32_t* block_valid;
  int32_t* d_err;
  int N, Hh, max_blocks, base_block;
  int T, H, W;          // chunk grid (used when perm is NULL)
};

template <int VPR>
__global__ void __launch_bounds__(kAppendThreads)
append_gather_kernel(AppendArgs a) {
  pdl_wait();     // global memory only after the predecessor grid completed
  pdl_trigger();
  constexpr int D = VPR * 8;
  __shared__ int s_tok[kBlk];
  const int j = blockIdx.x;
  const int b = blockIdx.z;
  const int slot0 = j * kBlk;
  const int valid = min(kBlk, a.N - slot0);
  const bool first_cta = blockIdx.y == 0 && b == 0;
  invert_block_slots<kAppendThreads>(a.perm, a.N, slot0, s_tok, j == 0 && first_cta, a.d_err,
                                     a.T, a.H, a.W);
  if (first_cta && threadIdx.x == 0) a.block_valid[a.base_block + j] = valid;
  // A slot of the chunk that no token maps to: perm is not a permutation.
  if (first_cta && threadIdx.x < valid && s_tok[threadIdx.x] < 0) report(a.d_err, BSA_DEV_BAD_PERM);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const bool is_k = warp < kAppendHeads;
  const int h = blockIdx.y * kAppendHeads + (is_k ? warp : warp - kAppendHeads);
  if (h >= a.Hh) return;
  const int c = lane % VPR, g = lane / VPR;
  const long long tok_stride = static_cast<long long>(a.Hh) * VPR;  // vectors per token
  const long long tok_base = static_cast<long long>(b) * a.N * tok_stride +
                             static_cast<long long>(h) * VPR + c;
  const long long bh = static_cast<long long>(b) * a.Hh + h;
  const long long blk = bh * a.max_blocks + a.base_block + j;
  const uint4* src = is_k ? a.k_tok : a.v_tok;
  uint4* dst = (is_k ? a.kc : a.vc) + blk * kBlk * VPR + c;
  // Rows at or past `valid` are the block's zero pad rows.
  auto load = [&](int row) {
    const int tok = s_tok[row];
    return tok >= 0 ? ld_nc_v4(src + tok_base + static_cast<long long>(tok) * tok_stride)
                    : make_uint4(0, 0, 0, 0);
  };
  auto store = [&](int row, uint4 x) { st_v4(dst + row * VPR, x); };
  float acc[8];
  warp_colsum_rows<VPR>(load, store, valid, g, acc);
  if (is_k && a.kmean != nullptr && g == 0) {
    float4* out = reinterpret_cast<float4*>(a.kmean + blk * D + c * 8);
    const float inv = static_cast<float>(valid);
    out[0] = make_float4(acc[0] / inv, acc[1] / inv, acc[2] / inv, acc[3] / inv);
    out[1] = make_float4(acc[4] / inv, acc[5] / inv, acc[6] / inv, acc[7] / inv);
  }
}

static bsa_status launch_append_gather(const AppendArgs& a, int B, int D, int nb, cudaStream_t s) {
  dim3 grid(nb, (a.Hh + kAppendHeads - 1) / kAppendHeads, B);
  if (D == 128) return launch_pdl(append_gather_kernel<16>, grid, dim3(kAppendThreads), 0, s, a);
  return launch_pdl(append_gather_kernel<8>, grid, dim3(kAppendThreads), 0, s, a);
}

// One tensor (the query chunk) into blocks together with the fp32 mean of
// each block's valid rows: one CTA per (chunk block, kMeanHeads heads,
// batch); warp w moves head w of the group, writing whole block rows (pads as
// zeros), and pools the rows while it moves them with pool.cuh's summation,
// the one every block mean of the library uses, so the router can score from
// these means without reading the blocks again.
constexpr int kMeanHeads = 4;
constexpr int kMeanGatherThreads = kMeanHeads * 32;

struct GatherMeanArgs {
  const uint4* x_tok;
  uint4* x_blk;
  float* x_mean;
  const int32_t* perm;
  int32_t* d_err;
  int N, Hh, nb;
  int T, H, W;          // chunk grid (used when perm is NULL)
};

template <int VPR>
__global__ void __launch_bounds__(kMeanGatherThreads)
gather_mean_kernel(GatherMeanArgs a) {
  pdl_wait();     // global memory only after the predecessor grid completed
  pdl_trigger();
  constexpr int D = VPR * 8;
  __shared__ int s_tok[kBlk];
  const int j = blockIdx.x;
  const int b = blockIdx.z;
  const int slot0 = j * kBlk;
  const int valid = min(kBlk, a.N - slot0);
  const bool first_cta = blockIdx.y == 0 && b == 0;
  invert_block_slots<kMeanGatherThreads>(a.perm, a.N, slot0, s_tok, j == 0 && first_cta,
                                         a.d_err, a.T, a.H, a.W);
  if (first_cta && threadIdx.x < valid && s_tok[threadIdx.x] < 0) report(a.d_err, BSA_DEV_BAD_PERM);
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int h = blockIdx.y * kMeanHeads + warp;
  if (h >= a.Hh) return;
  const int c = lane % VPR, g = lane / VPR;
  const long long tok_stride = static_cast<long long>(a.Hh) * VPR;  // vectors per token
  const long long tok_base = static_cast<long long>(b) * a.N * tok_stride +
                             static_cast<long long>(h) * VPR + c;
  const long long blk = (static_cast<long long>(b) * a.Hh + h) * a.nb + j;
  uint4* dst = a.x_blk + blk * kBlk * VPR + c;
  auto load = [&](int row) {
    const int tok = s_tok[row];
    return tok >= 0 ? ld_nc_v4(a.x_tok + tok_base + static_cast<long long>(tok) * tok_stride)
                    : make_uint4(0, 0, 0, 0);
  };
  auto store = [&](int row, uint4 x) { st_v4(dst + row * VPR, x); };
  float acc[8];
  // 32 rows in flight per lane: this kernel has one warp per (block, head),
  // only 8 warps per SM.
  warp_colsum_rows<VPR, decltype(load), decltype(store), 32>(load, store, valid, g, acc);
  if (g == 0) {
    float4* out = reinterpret_cast<float4*>(a.x_mean + blk * D + c * 8);
    const float inv = static_cast<float>(valid);
    out[0] = make_float4(acc[0] / inv, acc[1] / inv, acc[2] / inv, acc[3] / inv);
    out[1] = make_float4(acc[4] / inv, acc[5] / inv, acc[6] / inv, acc[7] / inv);
  }
}

static bsa_status check_chunk(int B, int Hh, int D, int T, int H, int W) {
  if (B <= 0 || Hh <= 0 || T <= 0 || H <= 0 || W <= 0) return BSA_ERR_INVALID_ARG;
  if (D != 64 && D != 128) return BSA_ERR_UNSUPPORTED;
  long long n = static_cast<long long>(T) * H * W;
  if (n > (1LL << 24)) return BSA_ERR_SHAPE;
  if (B > 65535) return BSA_ERR_SHAPE;
  return BSA_OK;
}

}  // namespace bsa

using namespace bsa;

extern "C" int bsa_abi_version(void) { return BSA_ABI_VERSION; }

extern "C" const char* bsa_status_string(bsa_status s) {
  switch (s) {
    case BSA_OK: return "BSA_OK";
    case BSA_ERR_INVALID_ARG: return "BSA_ERR_INVALID_ARG";
    case BSA_ERR_SHAPE: return "BSA_ERR_SHAPE";
    case BSA_ERR_CAPACITY: return "BSA_ERR_CAPACITY";
    case BSA_ERR_UNSUPPORTED: return "BSA_ERR_UNSUPPORTED";
    case BSA_ERR_CUDA: return "BSA_ERR_CUDA";
    case BSA_ERR_DEVICE_FAULT: return "BSA_ERR_DEVICE_FAULT";
    case BSA_ERR_TIMEOUT: return "BSA_ERR_TIMEOUT";
  }
  return "BSA_UNKNOWN_STATUS";
}

extern "C" bsa_status bsa_gilbert_perm(int T, int H, int W, int32_t* host_perm) {
  if (host_perm == nullptr || T <= 0 || H <= 0 || W <= 0) return BSA_ERR_INVALID_ARG;
  long long n = static_cast<long long>(T) * H * W;
  if (n > (1LL << 24)) return BSA_ERR_SHAPE;
  for (int p = 0; p < static_cast<int>(n); ++p) {
    V3 c = gilbert_cell(T, H, W, p);
    if (c.t < 0 || c.t >= T || c.h < 0 || c.h >= H || c.w < 0 || c.w >= W) return BSA_ERR_SHAPE;
    host_perm[(static_cast<long long>(c.t) * H + c.h) * W + c.w] = p;
  }
  return BSA_OK;
}

extern "C" bsa_status bsa_kv_append(bsa_kv_cache* c, const void* k_tok, const void* v_tok, int T,
                                    int H, int W, const int32_t* d_perm, int32_t* d_err,
                                    void* stream) {
  if (c == nullptr || k_tok == nullptr || v_tok == nullptr ||
      c->k == nullptr || c->v == nullptr || c->block_valid == nullptr)
    return BSA_ERR_INVALID_ARG;
  bsa_status st = check_chunk(c->B, c->Hh, c->D, T, H, W);
  if (st != BSA_OK) return st;
  if (!aligned16(k_tok) || !aligned16(v_tok) || !aligned16(c->k) || !aligned16(c->v))
    return BSA_ERR_INVALID_ARG;
  if (c->max_blocks <= 0 || c->n_blocks < 0 || c->n_blocks > c->max_blocks)
    return BSA_ERR_INVALID_ARG;
  const int n = T * H * W;
  const int nb = (n + kBlk - 1) / kBlk;
  if (c->n_blocks + nb > c->max_blocks) return BSA_ERR_CAPACITY;
  if (c->kmean != nullptr && !aligned16(c->kmean)) return BSA_ERR_INVALID_ARG;
  if (n <= kGatherMaxTokens) {
    // One pass: gather into whole cache rows, pooling the keys on the way.
    AppendArgs g{};
    g.k_tok = static_cast<const uint4*>(k_tok);
    g.v_tok = static_cast<const uint4*>(v_tok);
    g.kc = static_cast<uint4*>(c->k);
    g.vc = static_cast<uint4*>(c->v);
    g.kmean = c->kmean;
    g.perm = d_perm;
    g.T = T;
    g.H = H;
    g.W = W;
    g.block_valid = c->block_valid;
    g.d_err = d_err;
    g.N = n;
    g.Hh = c->Hh;
    g.max_blocks = c->max_blocks;
    g.base_block = c->n_blocks;
    st = launch_append_gather(g, c->B, c->D, nb, as_stream(stream));
  } else {
    // Large chunks: scatter K and V, then pool the new blocks.
    ReorderArgs a{};
    a.src0 = static_cast<const uint4*>(k_tok);
    a.dst0 = static_cast<uint4*>(c->k);
    a.src1 = static_cast<const uint4*>(v_tok);
    a.dst1 = static_cast<uint4*>(c->v);
    a.perm = d_perm;
    a.T = T;
    a.H = H;
    a.W = W;
    a.block_valid = c->block_valid;
    a.d_err = d_err;
    a.N = n;
    a.nb = nb;
    a.B = c->B;
    a.Hh = c->Hh;
    a.blk_stride = c->max_blocks;
    a.base_block = c->n_blocks;
    st = launch_reorder<true>(a, c->D, as_stream(stream));
    if (st == BSA_OK && c->kmean != nullptr)
      st = launch_block_means(c, c->n_blocks, nb, d_err, as_stream(stream));
  }
  if (st == BSA_OK) c->n_blocks += nb;
  return st;
}

extern "C" bsa_status bsa_kv_pool_means(const bsa_kv_cache* c, int first, int count,
                                        int32_t* d_err, void* stream) {
  if (c == nullptr || c->k == nullptr || c->kmean == nullptr || c->block_valid == nullptr)
    return BSA_ERR_INVALID_ARG;
  if (c->D != 64 && c->D != 128) return BSA_ERR_UNSUPPORTED;
  if (c->B <= 0 || c->Hh <= 0 || c->B > 65535 || c->Hh > 65535 || first < 0 || count < 0 ||
      first + count > c->max_blocks || !aligned16(c->k) || !aligned16(c->kmean))
    return BSA_ERR_INVALID_ARG;
  return launch_block_means(c, first, count, d_err, as_stream(stream));
}

extern "C" bsa_status bsa_tokens_to_blocks(const void* x_tok, void* x_blk, int B, int Hh, int D,
                                           int T, int H, int W, const int32_t* d_perm,
                                           int32_t* d_err, void* stream) {
  if (x_tok == nullptr || x_blk == nullptr) return BSA_ERR_INVALID_ARG;
  bsa_status st = check_chunk(B, Hh, D, T, H, W);
  if (st != BSA_OK) return st;
  if (!aligned16(x_tok) || !aligned16(x_blk)) return BSA_ERR_INVALID_ARG;
  const int n = T * H * W;
  ReorderArgs a{};
  a.src0 = static_cast<const uint4*>(x_tok);
  a.dst0 = static_cast<uint4*>(x_blk);
  a.perm = d_perm;
  a.T = T;
  a.H = H;
  a.W = W;
  a.d_err = d_err;
  a.N = n;
  a.nb = (n + kBlk - 1) / kBlk;
  a.B = B;
  a.Hh = Hh;
  a.blk_stride = a.nb;
  a.base_block = 0;
  return launch_reorder<true>(a, D, as_stream(stream));
}

extern "C" bsa_status bsa_tokens_to_blocks_mean(const void* x_tok, void* x_blk, float* x_mean,
                                                int B, int Hh, int D, int T, int H, int W,
                                                const int32_t* d_perm, int32_t* d_err,
                                                void* stream) {
  if (x_tok == nullptr || x_blk == nullptr || x_mean == nullptr)
    return BSA_ERR_INVALID_ARG;
  bsa_status st = check_chunk(B, Hh, D, T, H, W);
  if (st != BSA_OK) return st;
  if (!aligned16(x_tok) || !aligned16(x_blk) || !aligned16(x_mean)) return BSA_ERR_INVALID_ARG;
  const int n = T * H * W;
  if (n > kGatherMaxTokens) return BSA_ERR_UNSUPPORTED;
  GatherMeanArgs a{};
  a.x_tok = static_cast<const uint4*>(x_tok);
  a.x_blk = static_cast<uint4*>(x_blk);
  a.x_mean = x_mean;
  a.perm = d_perm;
  a.T = T;
  a.H = H;
  a.W = W;
  a.d_err = d_err;
  a.N = n;
  a.Hh = Hh;
  a.nb = (n + kBlk - 1) / kBlk;
  dim3 grid(a.nb, (Hh + kMeanHeads - 1) / kMeanHeads, B);
  cudaStream_t s = as_stream(stream);
  if (D == 128) return launch_pdl(gather_mean_kernel<16>, grid, dim3(kMeanGatherThreads), 0, s, a);
  return launch_pdl(gather_mean_kernel<8>, grid, dim3(kMeanGatherThreads), 0, s, a);
}

extern "C" bsa_status bsa_blocks_to_tokens(const void* x_blk, void* x_tok, int B, int Hh, int D,
                                           int T, int H, int W, const int32_t* d_perm,
                                           int32_t* d_err, void* stream) {
  if (x_tok == nullptr || x_blk == nullptr) return BSA_ERR_INVALID_ARG;
  bsa_status st = check_chunk(B, Hh, D, T, H, W);
  if (st != BSA_OK) return st;
  if (!aligned16(x_tok) || !aligned16(x_blk)) return BSA_ERR_INVALID_ARG;
  const int n = T * H * W;
  ReorderArgs a{};
  a.src0 = static_cast<const uint4*>(x_blk);
  a.dst0 = static_cast<uint4*>(x_tok);
  a.perm = d_perm;
  a.T = T;
  a.H = H;
  a.W = W;
  a.d_err = d_err;
  a.N = n;
  a.nb = (n + kBlk - 1) / kBlk;
  a.B = B;
  a.Hh = Hh;
  a.blk_stride = a.nb;
  a.base_block = 0;
  return launch_reorder<false>(a, D, as_stream(stream));
}

extern "C" bsa_status bsa_check_device_error(int32_t* d_err, void* stream, int32_t* code_out) {
  if (d_err == nullptr) return BSA_ERR_INVALID_ARG;
  cudaStream_t s = as_stream(stream);
  int32_t code = 0;
  if (cudaMemcpyAsync(&code, d_err, sizeof(int32_t), cudaMemcpyDeviceToHost, s) != cudaSuccess)
    return BSA_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return BSA_ERR_CUDA;
  if (code != 0) {
    if (cudaMemsetAsync(d_err, 0, sizeof(int32_t), s) != cudaSuccess) return BSA_ERR_CUDA;
    if (cudaStreamSynchronize(s) != cudaSuccess) return BSA_ERR_CUDA;
  }
  if (code_out != nullptr) *code_out = code;
  if (code == 0) return BSA_OK;
  return code == BSA_DEV_WAIT_TIMEOUT ? BSA_ERR_TIMEOUT : BSA_ERR_DEVICE_FAULT;
}
