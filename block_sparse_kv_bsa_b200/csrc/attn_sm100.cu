// attn_sm100.cu - bsa_attn: indexed block-sparse attention on tcgen05.
//
// "Velox: Spatial Memory Makes World Models Efficient", Methodology Step 6:
// each query block attends only to the KV blocks of its route, and because
// a block is exactly one 128-row attention tile, a skipped block costs
// neither its QK^T tile product nor its K/V tile load.
//
// One CTA computes one (batch, head, query block) work item; CTAs are
// numbered head-major so that the query blocks of a head run together and
// share that head's own-chunk K/V tiles through L2.
//
// Tensor memory (512 columns x 128 lanes, lane = query row):
//   [0,128) [128,256)  two S = Q K^T buffers (fp32)
//   [256, 256+D)       O accumulator (fp32)
//   [384, 384+D/2)     Q (bf16 pairs, the A operand of Q K^T)
//   [448, 512)         P (bf16 pairs, the A operand of P V)
// Both products take A from tensor memory and only B (a K or V tile) from
// shared memory: with M = 128 an operand read from shared memory costs as
// much bandwidth as the tensor core consumes, so keeping Q and P out of
// shared memory is what leaves room for the K/V tile stream.
//
// Warp roles:
//   warp 0      TMA producer: the K and V tiles of each selected block
//               (128 rows x D bf16, 128-byte swizzled boxes of 64 columns)
//               into a three-stage ring; one full and one empty mbarrier per
//               stage cover both tiles.  Tile row = ((b*Hh + h)*max_blocks +
//               blk)*128.
//   warp 1      allocates tensor memory; one lane issues tcgen05.mma:
//               S_i = Q K_i^T and O += P_i V_i, committing each group to an
//               mbarrier.  It waits only twice per tile (next stage loaded;
//               this tile's P stored): a wait in the issuing thread leaves the
//               tensor pipe without queued work, and measured ~170 SM cycles of
//               lost tensor time per wait.
//   warps 2-9   softmax: two warpgroups split every row (half 0: S/P columns
//               0-63 and O columns [0, D/2); half 1 the rest).  They put Q
//               into tensor memory, then per tile load S, mask the pad keys
//               of a tail block, exchange the row maximum through shared
//               memory, exponentiate in base 2 with a stale-maximum rule (O
//               and the running sums are rescaled only when the row maximum
//               grows by more than 2^8, so O/l stays exact), store P (bf16)
//               into tensor memory, and finally normalise O and write O, LSE.
// Every wait is bounded; a wait that gives up records
// BSA_DEV_WAIT_TIMEOUT, stops the other roles through a shared flag, lets
// in-flight copies and MMAs finish (bounded) and frees tensor memory.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <mutex>

#include "common.cuh"

namespace bsa {

constexpr int kSoftmaxThreads = 256;  // two warpgroups, one per 64-column half
constexpr int kAttnThreads = 64 + kSoftmaxThreads;
constexpr int kStages = 3;            // K/V ring depth (one K and one V tile per stage)
constexpr int kSBufs = 2;
constexpr uint32_t kColS = 0;
constexpr uint32_t kColO = 256;
constexpr uint32_t kColQ = 384;
constexpr uint32_t kColP = 448;
constexpr long long kWaitLimit = 1LL << 31;  // SM clocks (about a second)
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kRescaleThreshold = 8.0f;    // log2 units

// mbarrier slots
enum {
  B_Q_FULL = 0,
  B_KV_FULL = 1,                      // + stage: K and V tile of one route entry landed
  B_KV_EMPTY = B_KV_FULL + kStages,   // + stage: both products that read the stage are done
  B_S_FULL = B_KV_EMPTY + kStages,    // + buffer
  B_P_FULL = B_S_FULL + kSBufs,
  B_O_READY,
  B_MMA_DONE,
  B_COUNT
};

template <int D>
struct AttnLayout {
  static constexpr int kTileBytes = kBlk * D * 2;      // 128 rows x D bf16
  static constexpr int kK = 0;
  static constexpr int kV = kK + kStages * kTileBytes;
  static constexpr int kBars = kV + kStages * kTileBytes;
  static constexpr int kMisc = kBars + B_COUNT * 8;
  static constexpr int kRed = (kMisc + 64 + 15) & ~15;  // float [3 slots][2 halves][128 rows]
  static constexpr int kTotal = kRed + 3 * 2 * kBlk * 4;
  static constexpr int kAlloc = kTotal + 1024;          // room to align to 1024
};

struct AttnArgs {
  const __nv_bfloat16* q;
  const int32_t* idx;
  const int32_t* cnt;
  const int32_t* block_valid;
  const int32_t* q_valid;
  __nv_bfloat16* o;
  float* lse;
  int32_t* d_err;
  int Hh, n_q_blocks, max_sel, max_blocks, n_blocks;
  float scale_log2;
};

__device__ __forceinline__ int route_count(const AttnArgs& a, long long item) {
  int n = a.cnt[item];
  if (n < 0 || n > a.max_sel) {
    report(a.d_err, BSA_DEV_BAD_COUNT);
    n = n < 0 ? 0 : a.max_sel;
  }
  return n;
}

__device__ __forceinline__ int route_block(const AttnArgs& a, long long item, int i) {
  int blk = a.idx[item * a.max_sel + i];
  if (blk < 0 || blk >= a.n_blocks) {
    report(a.d_err, BSA_DEV_BAD_INDEX);
    blk = 0;
  }
  return blk;
}

__device__ __forceinline__ int block_rows(const AttnArgs& a, int blk) {
  int v = a.block_valid[blk];
  if (v < 1 || v > kBlk) {
    report(a.d_err, BSA_DEV_BAD_VALID);
    v = v < 1 ? 1 : kBlk;
  }
  return v;
}

__device__ __forceinline__ void named_bar_sync_softmax() {
  asm volatile("bar.sync 1, %0;" ::"n"(kSoftmaxThreads) : "memory");
}

template <int D>
__global__ void __launch_bounds__(kAttnThreads, 1)
bsa_attn_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                AttnArgs a) {
  using L = AttnLayout<D>;
  constexpr int kBoxes = D / 64;
  constexpr uint32_t kTileBytes = L::kTileBytes;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                           ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + L::kBars);
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(sm + L::kMisc);
  volatile int* s_abort = reinterpret_cast<volatile int*>(sm + L::kMisc + 4);

  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  const long long item = blockIdx.x;  // ((b*Hh + h)*n_q_blocks + j)
  const long long bh = item / a.n_q_blocks;
  const int j = static_cast<int>(item % a.n_q_blocks);

  if (threadIdx.x == 0) {
    for (int i = 0; i < B_COUNT; ++i) {
      uint32_t count = 1;
      if (i == B_Q_FULL || i == B_P_FULL) count = kSoftmaxThreads;
      mbar_init(&bars[i], count);
    }
    *s_abort = 0;
    fence_mbar_init();
  }
  if (warp == 1) tmem_alloc(s_tmem, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *s_tmem;
  const int n = route_count(a, item);

  if (warp == 0) {
    // ---------------- TMA producer ----------------
    if (lane == 0 && n > 0) {
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      int issued = 0;
      for (int i = 0; i < n; ++i) {
        const int st = i % kStages;
        const int blk = route_block(a, item, i);
        const int row = static_cast<int>((bh * a.max_blocks + blk) * kBlk);
        if (i >= kStages && !mbar_wait_bounded(&bars[B_KV_EMPTY + st], ((i / kStages) - 1) & 1,
                                               s_abort, kWaitLimit))
          break;
        mbar_expect_tx(&bars[B_KV_FULL + st], 2 * kTileBytes);
        for (int bx = 0; bx < kBoxes; ++bx) {
          tma_load_2d(sm + L::kK + st * kTileBytes + bx * (kBlk * 128), &tm_k, bx * 64, row,
                      &bars[B_KV_FULL + st]);
          tma_load_2d(sm + L::kV + st * kTileBytes + bx * (kBlk * 128), &tm_v, bx * 64, row,
                      &bars[B_KV_FULL + st]);
        }
        issued = i + 1;
      }
      if (issued < n) {
        report(a.d_err, BSA_DEV_WAIT_TIMEOUT);
        *s_abort = 1;
      }
      // Drain: every copy this thread issued must land before the CTA exits.
      for (int st = 0; st < kStages; ++st) {
        int last = -1;
        for (int i = st; i < issued; i += kStages) last = i;
        if (last >= 0)
          mbar_wait_bounded(&bars[B_KV_FULL + st], (last / kStages) & 1, nullptr, kWaitLimit);
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    // Every mbarrier wait of this thread leaves the tensor pipe without new
    // work for a while, so there are only two per tile: the K/V stage of the
    // next tile (before its Q K^T) and this tile's P (before its P V).  The S
    // buffer that Q K^T_{t} overwrites held S_{t-2}; the softmax read it
    // before storing P_{t-2}, which this thread already waited for.
    if (lane == 0 && n > 0) {
      constexpr uint32_t kIdQK = idesc_bf16(128, 128, 0);
      constexpr uint32_t kIdPV = idesc_bf16(128, D, 1);
      bool ok = mbar_wait_bounded(&bars[B_Q_FULL], 0, s_abort, kWaitLimit);
      auto issue_qk = [&](int t) {
        const int st = t % kStages, sb = t % kSBufs;
        const uint32_t k_addr = smem_u32(sm + L::kK + st * kTileBytes);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk / 4) * (kBlk * 128) + (kk % 4) * 32;
          tc_mma_ts(tmem + kColS + sb * 128, tmem + kColQ + kk * 8,
                    smem_desc(k_addr + off, 16, 1024), kIdQK, kk > 0 ? 1u : 0u);
        }
        tc_commit(&bars[B_S_FULL + sb]);
      };
      if (ok) ok = mbar_wait_bounded(&bars[B_KV_FULL + 0], 0, s_abort, kWaitLimit);
      if (ok) {
        tc_fence_after();
        issue_qk(0);
      }
      for (int i = 0; ok && i < n; ++i) {
        if (i + 1 < n) {
          const int t = i + 1;
          ok = mbar_wait_bounded(&bars[B_KV_FULL + t % kStages], (t / kStages) & 1, s_abort,
                                 kWaitLimit);
          if (!ok) break;
          tc_fence_after();
          issue_qk(t);
        }
        const int st = i % kStages;
        ok = mbar_wait_bounded(&bars[B_P_FULL], i & 1, s_abort, kWaitLimit);
        if (!ok) break;
        tc_fence_after();
        const uint32_t v_addr = smem_u32(sm + L::kV + st * kTileBytes);
#pragma unroll
        for (int kk = 0; kk < kBlk / 16; ++kk) {
          tc_mma_ts(tmem + kColO, tmem + kColP + kk * 8,
                    smem_desc(v_addr + kk * 2048, kBlk * 128, 1024), kIdPV,
                    (i > 0 || kk > 0) ? 1u : 0u);
        }
        tc_commit(&bars[B_KV_EMPTY + st]);
        tc_commit(&bars[B_O_READY]);
      }
      if (!ok) {
        report(a.d_err, BSA_DEV_WAIT_TIMEOUT);
        *s_abort = 1;
      }
      // Drain: all MMAs issued by this thread complete before TMEM is freed.
      tc_commit(&bars[B_MMA_DONE]);
      mbar_wait_bounded(&bars[B_MMA_DONE], 0, nullptr, kWaitLimit);
    }
  } else {
    // ---------------- softmax / epilogue (warps 2..9) ----------------
    // Two warpgroups split every row: half 0 owns S/P columns 0-63 and O
    // columns [0, D/2), half 1 the rest.  The row maximum is exchanged through
    // shared memory once per tile; the running sums stay per half (both halves
    // use the same reference maximum) and are added in the epilogue.
    const int half = (warp - 2) >> 2;        // 0 or 1
    const int wq = warp & 3;                 // TMEM lane window of this warp
    const int r = wq * 32 + lane;            // query row owned by this thread
    const uint32_t lane_base = static_cast<uint32_t>(wq * 32) << 16;
    constexpr int kHalfCols = kBlk / 2;      // S / P columns per thread
    constexpr int kHalfD = D / 2;            // O columns per thread
    const int c0 = half * kHalfCols;
    const uint32_t o_col = kColO + half * kHalfD;
    float* red = reinterpret_cast<float*>(sm + L::kRed);  // [3][2][128]

    // Q row r -> tensor memory as bf16 pairs (the A operand of Q K^T).  With
    // D = 128 each half stores its 64 elements; with D = 64 half 0 stores the
    // whole row.
    if (n > 0) {
      const uint4* qrow = reinterpret_cast<const uint4*>(a.q + (item * kBlk + r) * D);
      if (D == 128 || half == 0) {
        const int e0 = (D == 128) ? half * 64 : 0;   // first element stored
        uint32_t qw[32];
#pragma unroll
        for (int v = 0; v < 8; ++v) {
          uint4 x = ld_nc_v4(qrow + e0 / 8 + v);
          qw[4 * v + 0] = x.x; qw[4 * v + 1] = x.y; qw[4 * v + 2] = x.z; qw[4 * v + 3] = x.w;
        }
        tmem_st32u(tmem + lane_base + kColQ + e0 / 2, qw);
        tc_wait_st();
      }
      tc_fence_before();
      mbar_arrive(&bars[B_Q_FULL]);
    }

    float m_ref = -INFINITY, l = 0.f;
    bool ok = true;
    // Route lookahead: the block index two tiles ahead and the valid-row
    // count one tile ahead are loaded early and first used a tile later, so
    // these dependent global loads never stall the softmax.  Indices are
    // validated (and reported) by the producer; here they are only clamped.
    const int32_t* route = a.idx + item * a.max_sel;
    auto clamp_blk = [&](int b_) { return static_cast<unsigned>(b_) < static_cast<unsigned>(a.n_blocks) ? b_ : 0; };
    int blk_ahead = n > 1 ? route[1] : 0;
    int valid_raw = n > 0 ? a.block_valid[clamp_blk(route[0])] : kBlk;
    for (int i = 0; i < n; ++i) {
      const int sb = i % kSBufs;
      int valid = valid_raw;
      if (valid < 1 || valid > kBlk) {
        report(a.d_err, BSA_DEV_BAD_VALID);
        valid = valid < 1 ? 1 : kBlk;
      }
      const int blk_ahead2 = (i + 2 < n) ? route[i + 2] : 0;
      valid_raw = (i + 1 < n) ? a.block_valid[clamp_blk(blk_ahead)] : kBlk;
      blk_ahead = blk_ahead2;
      ok = __all_sync(0xffffffffu, mbar_wait_bounded(&bars[B_S_FULL + sb], (i / kSBufs) & 1,
                                                     s_abort, kWaitLimit));
      if (!ok) break;
      tc_fence_after();
      float s[kHalfCols];
      tmem_ld_cols<kHalfCols>(tmem + lane_base + kColS + sb * 128 + c0, s);
      if (valid < kBlk) {  // tail block of a chunk: mask its pad keys
#pragma unroll
        for (int c = 0; c < kHalfCols; ++c)
          if (c0 + c >= valid) s[c] = -INFINITY;
      }
      float mq[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
      for (int c = 0; c < kHalfCols; ++c) mq[c & 3] = fmaxf(mq[c & 3], s[c]);
      const float pm = fmaxf(fmaxf(mq[0], mq[1]), fmaxf(mq[2], mq[3]));
      float* red_t = red + (i & 1) * (2 * kBlk);
      red_t[half * kBlk + r] = pm;
      named_bar_sync_softmax();
      const float mx = fmaxf(pm, red_t[(half ^ 1) * kBlk + r]);
      const float mx2 = mx * a.scale_log2;
      float m_new = m_ref;
      if (i == 0 || mx2 > m_ref + kRescaleThreshold) m_new = mx2;
      float rq[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int c = 0; c < kHalfCols; ++c) {
        s[c] = ex2_approx(fmaf(s[c], a.scale_log2, -m_new));
        rq[c & 3] += s[c];
      }
      const float rs = (rq[0] + rq[1]) + (rq[2] + rq[3]);
      uint32_t pk[kHalfCols / 2];
#pragma unroll
      for (int c = 0; c < kHalfCols / 2; ++c) pk[c] = pack_bf16x2(s[2 * c], s[2 * c + 1]);
      if (i > 0) {
        // P V of the previous tile must be done: it reads the P columns this
        // tile overwrites and accumulates into the O that may be rescaled.
        // tcgen05.ld/st are warp-collective: the branch is warp-uniform and a
        // lane whose maximum did not move scales by exactly 1.
        ok = __all_sync(0xffffffffu, mbar_wait_bounded(&bars[B_O_READY], (i - 1) & 1, s_abort,
                                                       kWaitLimit));
        if (!ok) break;
        tc_fence_after();
        const bool grow = m_new != m_ref;
        if (__any_sync(0xffffffffu, grow)) {
          const float alpha = grow ? ex2_approx(m_ref - m_new) : 1.0f;
          l *= alpha;
#pragma unroll
          for (int c = 0; c < kHalfD / 32; ++c) {
            float o[32];
            tmem_ld_cols<32>(tmem + lane_base + o_col + c * 32, o);
#pragma unroll
            for (int e = 0; e < 32; ++e) o[e] *= alpha;
            tmem_st32(tmem + lane_base + o_col + c * 32, o);
          }
        }
      }
      l += rs;
      m_ref = m_new;
      // P row r, this half's 64 keys -> 32 TMEM columns of bf16 pairs.
      tmem_st32u(tmem + lane_base + kColP + half * (kHalfCols / 2), pk);
      tc_wait_st();
      tc_fence_before();
      mbar_arrive(&bars[B_P_FULL]);
    }
    if (!ok) {
      report(a.d_err, BSA_DEV_WAIT_TIMEOUT);
      *s_abort = 1;
    }
    // Epilogue: total row sum from both halves, then each half writes its
    // D/2 output columns; half 0 writes the LSE.
    const int q_valid = a.q_valid != nullptr ? a.q_valid[j] : kBlk;
    const long long grow_idx = item * kBlk + r;
    __nv_bfloat16* orow = a.o + grow_idx * D + half * kHalfD;
    bool have = ok && n > 0 && r < q_valid;
    if (ok && n > 0) {
      ok = __all_sync(0xffffffffu,
                      mbar_wait_bounded(&bars[B_O_READY], (n - 1) & 1, s_abort, kWaitLimit));
      if (!ok) {
        report(a.d_err, BSA_DEV_WAIT_TIMEOUT);
        *s_abort = 1;
        have = false;
      }
      tc_fence_after();
    }
    // Slot 2 is never used by the per-tile exchange (slots 0 and 1), so the
    // other half may still be reading its last tile's maximum.
    float* red_e = red + 2 * (2 * kBlk);
    red_e[half * kBlk + r] = l;
    named_bar_sync_softmax();
    const float l_tot = red_e[r] + red_e[kBlk + r];
    const float inv_l = have ? 1.0f / l_tot : 0.f;
#pragma unroll
    for (int c = 0; c < kHalfD / 32; ++c) {
      float o[32];
#pragma unroll
      for (int e = 0; e < 32; ++e) o[e] = 0.f;
      if (ok && n > 0) tmem_ld_cols<32>(tmem + lane_base + o_col + c * 32, o);
#pragma unroll
      for (int e = 0; e < 32; e += 8) {
        uint4 v;
        v.x = pack_bf16x2(have ? o[e + 0] * inv_l : 0.f, have ? o[e + 1] * inv_l : 0.f);
        v.y = pack_bf16x2(have ? o[e + 2] * inv_l : 0.f, have ? o[e + 3] * inv_l : 0.f);
        v.z = pack_bf16x2(have ? o[e + 4] * inv_l : 0.f, have ? o[e + 5] * inv_l : 0.f);
        v.w = pack_bf16x2(have ? o[e + 6] * inv_l : 0.f, have ? o[e + 7] * inv_l : 0.f);
        *reinterpret_cast<uint4*>(orow + c * 32 + e) = v;
      }
    }
    if (half == 0)
      a.lse[grow_idx] = have ? (m_ref + __log2f(l_tot)) * 0.6931471805599453f : -INFINITY;
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ---------------------------------------------------------------------------
// Host side: tensor maps and launch
// ---------------------------------------------------------------------------
static PFN_cuTensorMapEncodeTiled_v12000 get_encode() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// 2D map over a bf16 matrix [rows, D]: boxes of 128 rows x 64 columns, 128B swizzle.
static bool make_map(CUtensorMap* m, const void* base, long long rows, int D) {
  auto enc = get_encode();
  if (enc == nullptr) return false;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(D) * 2};
  cuuint32_t box[2] = {64, 128};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides,
                   box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

static bool device_is_sm100() {
  int dev = 0, major = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return false;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess)
    return false;
  return major == 10;
}

template <int D>
static bsa_status launch_attn(const void* q, const bsa_kv_cache* c, const AttnArgs& a,
                              long long items, cudaStream_t s) {
  CUtensorMap tk, tv;
  const long long crows = static_cast<long long>(c->B) * c->Hh * c->max_blocks * kBlk;
  if (!make_map(&tk, c->k, crows, D) || !make_map(&tv, c->v, crows, D)) return BSA_ERR_CUDA;
  const int smem = AttnLayout<D>::kAlloc;
  if (cudaFuncSetAttribute(bsa_attn_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) !=
      cudaSuccess)
    return BSA_ERR_CUDA;
  bsa_attn_kernel<D><<<static_cast<unsigned>(items), kAttnThreads, smem, s>>>(tk, tv, a);
  return launch_status();
}

}  // namespace bsa

using namespace bsa;

extern "C" bsa_status bsa_attn(const void* q_blk, const bsa_kv_cache* c, const int32_t* q_valid,
                               const int32_t* idx, const int32_t* cnt, int n_q_blocks, int max_sel,
                               float sm_scale, void* o_blk, float* lse, int32_t* d_err,
                               void* stream) {
  if (q_blk == nullptr || c == nullptr || idx == nullptr || cnt == nullptr || o_blk == nullptr ||
      lse == nullptr || c->k == nullptr || c->v == nullptr || c->block_valid == nullptr)
    return BSA_ERR_INVALID_ARG;
  if (c->B <= 0 || c->Hh <= 0 || n_q_blocks <= 0 || max_sel <= 0 || c->max_blocks <= 0 ||
      c->n_blocks < 0 || c->n_blocks > c->max_blocks || !(sm_scale == sm_scale))
    return BSA_ERR_INVALID_ARG;
  if (c->D != 64 && c->D != 128) return BSA_ERR_UNSUPPORTED;
  if (!aligned16(q_blk) || !aligned16(o_blk) || !aligned16(c->k) || !aligned16(c->v))
    return BSA_ERR_INVALID_ARG;
  const long long items = static_cast<long long>(c->B) * c->Hh * n_q_blocks;
  const long long crows = static_cast<long long>(c->B) * c->Hh * c->max_blocks * kBlk;
  if (items * kBlk >= (1LL << 31) || crows >= (1LL << 31)) return BSA_ERR_SHAPE;
  if (!device_is_sm100()) return BSA_ERR_UNSUPPORTED;
  AttnArgs a{};
  a.q = static_cast<const __nv_bfloat16*>(q_blk);
  a.idx = idx;
  a.cnt = cnt;
  a.block_valid = c->block_valid;
  a.q_valid = q_valid;
  a.o = static_cast<__nv_bfloat16*>(o_blk);
  a.lse = lse;
  a.d_err = d_err;
  a.Hh = c->Hh;
  a.n_q_blocks = n_q_blocks;
  a.max_sel = max_sel;
  a.max_blocks = c->max_blocks;
  a.n_blocks = c->n_blocks;
  a.scale_log2 = sm_scale * kLog2e;
  cudaStream_t s = as_stream(stream);
  return c->D == 128 ? launch_attn<128>(q_blk, c, a, items, s)
                     : launch_attn<64>(q_blk, c, a, items, s);
}
