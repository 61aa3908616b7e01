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
//   [0,128) [128,256) [256,384)  three S = Q K^T buffers (fp32); tile t uses
//                                buffer t % 3, and P_t (bf16 pairs, the A
//                                operand of P V) is written over columns
//                                [0, 64) of that buffer
//   [384, 384+D)                 O accumulator (fp32)
// Q (128 x D bf16) stays in shared memory for the whole work item and is the
// A operand of Q K^T; V is the B operand of P V (A from tensor memory).
// Three S buffers let the Q K^T of tile t + 3 run as soon as the P V of
// tile t has read P_t, so S_t is ready well before the tensor core needs
// P_t, and the softmax of one tile overlaps the products of the next two.
//
// Warp roles (384 threads):
//   warp 0      TMA producer: Q once, then the K tile (three-slot K ring) and
//               the V tile (three-slot V ring) of each selected block, 128
//               rows x D bf16 in 128-byte swizzled boxes of 64 columns; K runs
//               two tiles ahead of V, the order in which the products consume
//               them.  Tile row = ((b*Hh + h)*max_blocks + blk)*128.
//   warp 1      allocates tensor memory; one elected lane issues O += P_t V_t once
//               the softmax warpgroup has stored P_t and seen V_t land (one
//               barrier per tile).
//   warp 2      one elected lane issues S_t = Q K_t^T once K_t has landed and the
//               P V of tile t - 3 (which read P from the same buffer) is done.
//               The tensor pipe is fed only as fast as its issuing threads
//               issue: a wait in an issuing thread, and every instruction it
//               shares issue slots with, costs tensor time (measured: ~190
//               SM cycles per wait per tile, and as much again from busy
//               warps on the same SM).  Two issuers on two SM sub-partitions
//               keep work queued while one of them waits.  Operand
//               descriptors are built once per CTA.
//   warp 3      idle (keeps the softmax warpgroups aligned to lane windows).
//   warps 4-11  softmax: warpgroup g (warps 4-7, 8-11) takes every other tile
//               t = g, g + 2, ...; a thread owns one query row.  Per tile it
//               loads S, masks the pad keys of a tail block, takes the row
//               maximum, receives the reference maximum of tile t - 1 from
//               the other warpgroup and passes on its own (stale-maximum
//               rule: the reference moves only when the row maximum exceeds
//               it by more than 2^8, and O is then rescaled, so O/l stays
//               exact), exponentiates in base 2 and stores P.  Finally the
//               two warpgroups merge their running sums and write O and LSE.
// Every wait is bounded; a wait that gives up records
// BSA_DEV_WAIT_TIMEOUT, stops the other roles through a shared flag, lets
// in-flight copies and MMAs finish (bounded) and frees tensor memory.  Every
// warp runs the same sequence of named-barrier operations whether or not a
// wait gave up, so an abort never leaves a partner waiting at a barrier.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <mutex>

#include "common.cuh"
#include "gilbert.cuh"

namespace bsa {

constexpr int kSoftmaxThreads = 256;  // two warpgroups, one per tile parity
constexpr int kAttnThreads = 128 + kSoftmaxThreads;  // producer, PV issuer, QK issuer, spare
constexpr int kKSlots = 3;            // K ring
constexpr int kVSlots = 3;            // V ring
constexpr int kSBufs = 3;             // S / P buffers in tensor memory
constexpr int kKLead = 2;             // K tiles issued ahead of the V tile
constexpr uint32_t kColO = 384;
constexpr long long kWaitLimit = 1LL << 31;  // SM clocks (about a second)
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kRescaleThreshold = 8.0f;    // log2 units
// Token-order output: the row -> token table is built by one warp scanning
// the permutation while the tiles run, which stays hidden up to this size.
constexpr int kTokOutMaxTokens = 1 << 14;

// mbarrier slots
enum {
  B_Q_FULL = 0,                       // Q landed (producer arrive + bytes)
  B_K_FULL = 1,                       // + K slot: K tile landed
  B_K_EMPTY = B_K_FULL + kKSlots,     // + K slot: its Q K^T is done
  B_V_FULL = B_K_EMPTY + kKSlots,     // + V slot: V tile landed
  B_V_EMPTY = B_V_FULL + kVSlots,     // + V slot: its P V is done
  B_PV_READY = B_V_EMPTY + kVSlots,   // + slot t % 3: P_t stored, V_t and K_{t+3} landed
  B_S_FULL = B_PV_READY + kVSlots,    // + S buffer: the S of its tile is ready
  B_MMA_DONE = B_S_FULL + kSBufs,     // + issuer (0: P V thread, 1: Q K^T thread)
  B_MMA_DONE_END = B_MMA_DONE + 2,
  B_COUNT = B_MMA_DONE_END
};

template <int D>
struct AttnLayout {
  static constexpr int kTileBytes = kBlk * D * 2;      // 128 rows x D bf16
  static constexpr int kQ = 0;
  static constexpr int kK = kQ + kTileBytes;
  static constexpr int kV = kK + kKSlots * kTileBytes;
  static constexpr int kBars = kV + kVSlots * kTileBytes;
  static constexpr int kMisc = kBars + B_COUNT * 8;
  static constexpr int kTok = (kMisc + 64 + 15) & ~15;  // float [2 warpgroups][128 rows]
  static constexpr int kSlotTok = kTok + 2 * kBlk * 4;  // int [128]: raster token of each row
  static constexpr int kTotal = kSlotTok + kBlk * 4;
  static constexpr int kAlloc = kTotal + 1024;          // room to align to 1024
  // The epilogue's [2][2][128] floats reuse K slot 0: by then every Q K^T
  // has completed and no K copy is in flight.
  static constexpr int kFin = kK;
  static_assert(kAlloc <= 227 * 1024, "shared memory per CTA");
  static_assert(kTileBytes >= 4 * kBlk * 4, "epilogue scratch fits in one K slot");
};

struct AttnArgs {
  const int32_t* idx;
  const int32_t* cnt;
  const int32_t* block_valid;
  const int32_t* q_valid;
  __nv_bfloat16* o;
  float* lse;
  int32_t* d_err;
  const int32_t* perm;      // token -> curve slot (token-order output only)
  int n_tok;                // tokens of the chunk (token-order output only)
  int T, H, W;              // chunk grid (token-order output without perm)
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

__device__ __forceinline__ int checked_block(const AttnArgs& a, int blk) {
  if (blk < 0 || blk >= a.n_blocks) {
    report(a.d_err, BSA_DEV_BAD_INDEX);
    blk = 0;
  }
  return blk;
}
__device__ __forceinline__ int route_block(const AttnArgs& a, long long item, int i) {
  return checked_block(a, a.idx[item * a.max_sel + i]);
}

// Named barriers 1-8 carry the row-maximum tokens between the two softmax
// warpgroups (one per direction and TMEM lane window, 64 threads each);
// barrier 9 joins all softmax threads in the epilogue.
__device__ __forceinline__ void named_bar_sync(int id, int count) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}
__device__ __forceinline__ void named_bar_arrive(int id, int count) {
  asm volatile("bar.arrive %0, %1;" ::"r"(id), "r"(count) : "memory");
}

// Maximum of three floats in one instruction (sm_100).
__device__ __forceinline__ float fmax3(float x, float y, float z) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(x), "f"(y), "f"(z));
  return d;
}

// kTokOut: O and LSE go straight to raster token order ([B, N, Hh, D] and
// [B, N, Hh]) through the chunk's permutation, instead of block order; the
// otherwise idle warp 3 inverts the permutation for the CTA's 128 rows while
// the tiles are computed.
template <int D, bool kTokOut>
__global__ void __launch_bounds__(kAttnThreads, 1)
bsa_attn_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o,
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
      // The 128 threads of the warpgroup that owns the tile.
      if (i >= B_PV_READY && i < B_PV_READY + kVSlots) count = kSoftmaxThreads / 2;
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
  // Barriers and tensor memory are set up while the predecessor grid (the
  // router) finishes; the route and Q are read only after it completed.
  pdl_wait();
  pdl_trigger();
  // The producer starts Q's copy and reads the first route entry before the
  // route count arrives (every row of idx has max_sel >= 1 entries).
  int first_blk = 0;
  if (warp == 0) {
    if (elect_one()) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      mbar_expect_tx(&bars[B_Q_FULL], kTileBytes);
      for (int bx = 0; bx < kBoxes; ++bx)
        tma_load_2d(sm + L::kQ + bx * (kBlk * 128), &tm_q, bx * 64, static_cast<int>(item * kBlk),
                    &bars[B_Q_FULL]);
    }
    __syncwarp();
    first_blk = a.idx[item * a.max_sel];
  }
  const int n = route_count(a, item);

  if (warp == 0) {
    // ---------------- TMA producer ----------------
    if (lane == 0) {
      int k_issued = 0, v_issued = 0;
      bool ok = true;
      // Step s issues K_s (while s < n), then V_{s - kKLead}.
      for (int step = 0; ok && step < n + kKLead; ++step) {
        if (step < n) {
          const int t = step, sl = t % kKSlots;
          const int blk = t == 0 ? checked_block(a, first_blk) : route_block(a, item, t);
          const int row = static_cast<int>((bh * a.max_blocks + blk) * kBlk);
          if (t >= kKSlots)
            ok = mbar_wait_bounded(&bars[B_K_EMPTY + sl], ((t / kKSlots) - 1) & 1, s_abort,
                                   kWaitLimit);
          if (!ok) break;
          mbar_expect_tx(&bars[B_K_FULL + sl], kTileBytes);
          for (int bx = 0; bx < kBoxes; ++bx)
            tma_load_2d(sm + L::kK + sl * kTileBytes + bx * (kBlk * 128), &tm_k, bx * 64, row,
                        &bars[B_K_FULL + sl]);
          k_issued = t + 1;
        }
        const int t = step - kKLead;
        if (t >= 0 && t < n) {
          const int sl = t % kVSlots;
          const int row = static_cast<int>((bh * a.max_blocks + route_block(a, item, t)) * kBlk);
          if (t >= kVSlots)
            ok = mbar_wait_bounded(&bars[B_V_EMPTY + sl], ((t / kVSlots) - 1) & 1, s_abort,
                                   kWaitLimit);
          if (!ok) break;
          mbar_expect_tx(&bars[B_V_FULL + sl], kTileBytes);
          for (int bx = 0; bx < kBoxes; ++bx)
            tma_load_2d(sm + L::kV + sl * kTileBytes + bx * (kBlk * 128), &tm_v, bx * 64, row,
                        &bars[B_V_FULL + sl]);
          v_issued = t + 1;
        }
      }
      if (!ok) {
        report(a.d_err, BSA_DEV_WAIT_TIMEOUT);
        *s_abort = 1;
      }
      // Drain: every copy this warp issued (Q's too, issued whatever n is)
      // must land before the CTA exits.
      mbar_wait_bounded(&bars[B_Q_FULL], 0, nullptr, kWaitLimit);
      for (int sl = 0; sl < kKSlots; ++sl) {
        int last = -1;
        for (int t = sl; t < k_issued; t += kKSlots) last = t;
        if (last >= 0)
          mbar_wait_bounded(&bars[B_K_FULL + sl], (last / kKSlots) & 1, nullptr, kWaitLimit);
      }
      for (int sl = 0; sl < kVSlots; ++sl) {
        int last = -1;
        for (int t = sl; t < v_issued; t += kVSlots) last = t;
        if (last >= 0)
          mbar_wait_bounded(&bars[B_V_FULL + sl], (last / kVSlots) & 1, nullptr, kWaitLimit);
      }
    }
  } else if (warp == 1 || warp == 2) {
    // ---------------- MMA issuers ----------------
    // Warp 1 issues O += P_t V_t, warp 2 issues S_t = Q K_t^T: two threads on
    // two SM sub-partitions, so that one's waits do not leave the tensor pipe
    // without queued work.  Q K^T_t overwrites the S buffer whose P the
    // P V of tile t - 3 read, so it waits for that P V to complete.  The
    // whole warp runs the loop and the waits and one elected lane issues
    // (measured 1-1.5 % faster than a loop run by lane 0 alone).
    if (n > 0) {
      constexpr uint32_t kSlot16 = kTileBytes >> 4;
      bool ok = true;
      if (warp == 2) {
        constexpr uint32_t kIdQK = idesc_bf16(128, 128, 0);
        const uint64_t q_desc = smem_desc(smem_u32(sm + L::kQ), 16, 1024);
        const uint64_t k_desc0 = smem_desc(smem_u32(sm + L::kK), 16, 1024);
        ok = __all_sync(0xffffffffu, mbar_wait_bounded(&bars[B_Q_FULL], 0, s_abort, kWaitLimit));
        for (int t = 0; ok && t < n; ++t) {
          const int sl = t % kKSlots;
          ok = __all_sync(0xffffffffu, mbar_wait_bounded(&bars[B_K_FULL + sl], (t / kKSlots) & 1,
                                                         s_abort, kWaitLimit));
          if (ok && t >= kSBufs)
            ok = __all_sync(0xffffffffu,
                            mbar_wait_bounded(&bars[B_V_EMPTY + t % kVSlots],
                                              ((t / kVSlots) - 1) & 1, s_abort, kWaitLimit));
          if (!ok) break;
          tc_fence_after();
          const uint64_t k_desc = desc_add(k_desc0, sl * kSlot16);
          if (elect_one()) {
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
              const uint32_t off = ((kk / 4) * (kBlk * 128) + (kk % 4) * 32) >> 4;
              tc_mma_ss(tmem + (t % kSBufs) * 128, desc_add(q_desc, off), desc_add(k_desc, off),
                        kIdQK, kk > 0 ? 1u : 0u);
            }
            tc_commit(&bars[B_K_EMPTY + sl]);
            tc_commit(&bars[B_S_FULL + t % kSBufs]);
          }
          __syncwarp();
        }
      } else {
        constexpr uint32_t kIdPV = idesc_bf16(128, D, 1);
        const uint64_t v_desc0 = smem_desc(smem_u32(sm + L::kV), kBlk * 128, 1024);
        for (int i = 0; ok && i < n; ++i) {
          const int sl = i % kVSlots;
          ok = __all_sync(0xffffffffu, mbar_wait_bounded(&bars[B_PV_READY + sl], (i / kVSlots) & 1,
                                                         s_abort, kWaitLimit));
          if (!ok) break;
          tc_fence_after();
          const uint32_t p_col = tmem + (i % kSBufs) * 128;
          const uint64_t v_desc = desc_add(v_desc0, sl * kSlot16);
          if (elect_one()) {
#pragma unroll
            for (int kk = 0; kk < kBlk / 16; ++kk) {
              tc_mma_ts(tmem + kColO, p_col + kk * 8, desc_add(v_desc, (kk * 2048) >> 4), kIdPV,
                        (i > 0 || kk > 0) ? 1u : 0u);
            }
            tc_commit(&bars[B_V_EMPTY + sl]);
          }
          __syncwarp();
        }
      }
      if (!ok && lane == 0) {
        report(a.d_err, BSA_DEV_WAIT_TIMEOUT);
        *s_abort = 1;
      }
      // Drain: all MMAs issued by lane 0 complete before TMEM is freed.
      if (lane == 0) {
        tc_commit(&bars[B_MMA_DONE + (warp - 1)]);
        mbar_wait_bounded(&bars[B_MMA_DONE + (warp - 1)], 0, nullptr, kWaitLimit);
      }
      __syncwarp();
    }
  } else if (warp == 3) {
    // ---------------- row -> raster token table (token-order output) ----------------
    // s_tok[r] = the token whose curve slot is j*128 + r, or -1 (pad row):
    // the lanes scan perm with 16 loads in flight each, or, without a table,
    // locate the slots on the Gilbert curve themselves.  Released to the
    // softmax warps through named barrier 10 (arrive; they sync before
    // their stores).
    if (kTokOut) {
      int* s_tok = reinterpret_cast<int*>(sm + L::kSlotTok);
      const int slot0 = j * kBlk;
      if (a.perm == nullptr) {
        // No table: each lane locates its slots on the Gilbert curve.
        for (int i = lane; i < kBlk; i += 32)
          s_tok[i] = slot0 + i < a.n_tok ? curve_token(a.T, a.H, a.W, slot0 + i) : -1;
        __syncwarp();
      } else {
        for (int i = lane; i < kBlk; i += 32) s_tok[i] = -1;
        __syncwarp();
        constexpr int kScan = 16;
        for (int base = 0; base < a.n_tok; base += kScan * 32) {
          int pv[kScan];
#pragma unroll
          for (int k = 0; k < kScan; ++k) {
            const int t = base + lane + k * 32;
            pv[k] = t < a.n_tok ? __ldg(a.perm + t) : -1;
          }
#pragma unroll
          for (int k = 0; k < kScan; ++k) {
            const int t = base + lane + k * 32;
            if (t >= a.n_tok) break;
            if (pv[k] < 0 || pv[k] >= a.n_tok) {
              report(a.d_err, BSA_DEV_BAD_PERM);
              continue;
            }
            const unsigned d = static_cast<unsigned>(pv[k] - slot0);
            if (d < static_cast<unsigned>(kBlk)) s_tok[d] = t;
          }
        }
        __syncwarp();
      }
      // A slot of a token row that no token maps to: perm is no permutation.
      const int rows = min(kBlk, a.n_tok - slot0);
      for (int i = lane; i < rows; i += 32)
        if (s_tok[i] < 0) report(a.d_err, BSA_DEV_BAD_PERM);
      named_bar_arrive(10, kSoftmaxThreads + 32);
    }
  } else if (warp >= 4) {
    // ---------------- softmax / epilogue (warps 4..11) ----------------
    // The reference maximum m_t of tile t is decided in tile order: the
    // thread of row r in the warpgroup of tile t - 1 hands m_{t-1} to the
    // thread of row r in the other warpgroup through shared memory and a
    // named barrier per TMEM lane window (producer bar.arrive, consumer
    // bar.sync).  Both warpgroups thus exponentiate against the same
    // reference as O.  Each keeps its own running sum, expressed in the last
    // reference it used; the two are merged in the epilogue.
    const int g = (warp - 4) >> 2;           // warpgroup: 0 or 1
    const int wq = warp & 3;                 // TMEM lane window of this warp
    const int r = wq * 32 + lane;            // query row owned by this thread
    const uint32_t lane_base = static_cast<uint32_t>(wq * 32) << 16;
    float* tok = reinterpret_cast<float*>(sm + L::kTok);  // [2 warpgroups][128 rows]
    const int bar_in = 1 + (g ^ 1) * 4 + wq;              // token from the other warpgroup
    const int bar_out = 1 + g * 4 + wq;                   // token to the other warpgroup

    float m_last = -INFINITY;  // reference of this warpgroup's running sum
    float l = 0.f;
    bool ok = true;
    // Route lookahead: the valid-row count of this warpgroup's next tile and
    // the block index of the one after it are loaded a tile early, so these
    // dependent global loads never stall the softmax.  Indices are validated
    // (and reported) by the producer; here they are only clamped.
    const int32_t* route = a.idx + item * a.max_sel;
    auto clamp_blk = [&](int b_) {
      return static_cast<unsigned>(b_) < static_cast<unsigned>(a.n_blocks) ? b_ : 0;
    };
    int blk_ahead = (g + 2 < n) ? route[g + 2] : 0;
    int valid_raw = (g < n) ? a.block_valid[clamp_blk(route[g])] : kBlk;
    for (int t = g; t < n; t += 2) {
      int valid = valid_raw;
      if (valid < 1 || valid > kBlk) {
        report(a.d_err, BSA_DEV_BAD_VALID);
        valid = valid < 1 ? 1 : kBlk;
      }
      const int blk_ahead2 = (t + 4 < n) ? route[t + 4] : 0;
      valid_raw = (t + 2 < n) ? a.block_valid[clamp_blk(blk_ahead)] : kBlk;
      blk_ahead = blk_ahead2;
      const uint32_t s_col = static_cast<uint32_t>(t % kSBufs) * 128;

      // One barrier per S buffer: its next completion (S_{t+3}) needs the
      // P V of this tile, which needs this warpgroup's P_t, so it cannot run
      // two phases ahead of this wait; and S_{t-3} completed before the
      // token reached this warpgroup, so it is not behind either: the parity
      // is exact.  (A barrier per warpgroup could take S_t and S_{t+2} before
      // its warpgroup looked, since S_{t+2} depends only on the other
      // warpgroup.)
      float s[kBlk];
      if (ok)
        ok = __all_sync(0xffffffffu, mbar_wait_bounded(&bars[B_S_FULL + t % kSBufs],
                                                       (t / kSBufs) & 1, s_abort, kWaitLimit));
      if (ok) {
        tc_fence_after();
        tmem_ld_cols<kBlk>(tmem + lane_base + s_col, s);
      } else {
#pragma unroll
        for (int c = 0; c < kBlk; ++c) s[c] = 0.f;
      }
      if (valid < kBlk) {  // tail block of a chunk: mask its pad keys
#pragma unroll
        for (int c = 0; c < kBlk; ++c)
          if (c >= valid) s[c] = -INFINITY;
      }
      // Row maximum: four chains over columns 0-11, 12-123 (pairs), 124-127.
      static_assert(kBlk == 128, "the maximum below covers exactly 128 columns");
      float mq[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) mq[k] = fmax3(s[k], s[k + 4], s[k + 8]);
#pragma unroll
      for (int c = 12; c + 4 < kBlk; c += 8) {
#pragma unroll
        for (int k = 0; k < 4; ++k) mq[k] = fmax3(mq[k], s[c + k], s[c + 4 + k]);
      }
#pragma unroll
      for (int k = 0; k < 4; ++k) mq[k] = fmaxf(mq[k], s[kBlk - 4 + k]);
      const float mx = fmaxf(fmaxf(mq[0], mq[1]), fmaxf(mq[2], mq[3])) * a.scale_log2;

      // Reference maximum of tile t, decided in tile order.
      float m_prev = -INFINITY;
      if (t > 0) {
        named_bar_sync(bar_in, 64);
        m_prev = tok[(g ^ 1) * kBlk + r];
      }
      const float m_t = (t == 0 || mx > m_prev + kRescaleThreshold) ? mx : m_prev;
      if (t + 1 < n) {
        tok[g * kBlk + r] = m_t;
        named_bar_arrive(bar_out, 64);
      }

      // P (bf16 pairs) overwrites the S buffer it was computed from, 64 keys
      // at a time: TMEM columns s_col + [0, 64) then hold P row r.
      // Pairs of columns go through two-wide FMA / add; the running sums
      // are the four partial sums of columns = 0, 1, 2, 3 (mod 4).
      const uint64_t scale2 = f2_pack(a.scale_log2, a.scale_log2);
      const uint64_t neg_m2 = f2_pack(-m_t, -m_t);
      uint64_t acc2[2] = {0ull, 0ull};
#pragma unroll
      for (int q = 0; q < kBlk / 64; ++q) {
        uint32_t pk[32];
#pragma unroll
        for (int c = 0; c < 32; ++c) {
          float x0, x1;
          f2_unpack(f2_fma(f2_pack(s[64 * q + 2 * c], s[64 * q + 2 * c + 1]), scale2, neg_m2), x0,
                    x1);
          const float e0 = ex2_approx(x0), e1 = ex2_approx(x1);
          acc2[c & 1] = f2_add(acc2[c & 1], f2_pack(e0, e1));
          pk[c] = pack_bf16x2(e0, e1);
        }
        if (ok) tmem_st32u(tmem + lane_base + s_col + 32 * q, pk);
      }
      float rq[4];
      f2_unpack(acc2[0], rq[0], rq[1]);
      f2_unpack(acc2[1], rq[2], rq[3]);
      const float rs = (rq[0] + rq[1]) + (rq[2] + rq[3]);
      if (m_t != m_last) {  // m_last = -inf scales the empty sum 0 by 0
        l *= ex2_approx(m_last - m_t);
        m_last = m_t;
      }
      l += rs;

      // A row whose reference moved (rare under the stale-maximum rule)
      // rescales O after the P V of tile t - 1 has completed and before this
      // tile's P is released; a warp with no such row releases at once.
      // That completion is V_EMPTY of slot (t - 1) % 3, phase (t - 1) / 3.
      // The wait is exact: the previous phase (P V of tile t - 4) completed
      // before Q K^T of tile t - 1 was issued, whose S the other warpgroup
      // saw before handing over the token this warpgroup holds; and the next
      // phase (P V of tile t + 2) needs this tile's P V first, which needs
      // this release.  tcgen05.ld/st are warp-collective: the branch is
      // warp-uniform and a lane whose reference did not move scales by 1.
      if (ok && t > 0 && __any_sync(0xffffffffu, m_t != m_prev)) {
        ok = __all_sync(0xffffffffu,
                        mbar_wait_bounded(&bars[B_V_EMPTY + (t - 1) % kVSlots],
                                          ((t - 1) / kVSlots) & 1, s_abort, kWaitLimit));
        const bool grow = m_t != m_prev;
        if (ok) {
          tc_fence_after();
          const float alpha = grow ? ex2_approx(m_prev - m_t) : 1.0f;
#pragma unroll
          for (int c = 0; c < D / 32; ++c) {
            float o[32];
            tmem_ld_cols<32>(tmem + lane_base + kColO + c * 32, o);
#pragma unroll
            for (int e = 0; e < 32; ++e) o[e] *= alpha;
            tmem_st32(tmem + lane_base + kColO + c * 32, o);
          }
        }
      }
      // Before releasing the tile to the MMA thread: V_t and K_{t+3} (the
      // next product into this S buffer) have landed.  This warpgroup waits
      // for K slot t % 3 and V slot t % 3 only at tiles t, t + 6, ..., and the
      // tile three earlier on the same slots was released (by the other
      // warpgroup) only after its own copies landed, so each parity is exact.
      if (ok) {
        ok = __all_sync(0xffffffffu, mbar_wait_bounded(&bars[B_V_FULL + t % kVSlots],
                                                       (t / kVSlots) & 1, s_abort, kWaitLimit));
      }
      tc_wait_st();
      tc_fence_before();
      mbar_arrive(&bars[B_PV_READY + t % kVSlots]);
    }
    if (!ok) {
      report(a.d_err, BSA_DEV_WAIT_TIMEOUT);
      *s_abort = 1;
    }
    // Epilogue: merge the two running sums against the final reference (the
    // larger of the two: references never decrease), then each warpgroup
    // normalises D/2 output columns; warpgroup 0 writes the LSE.
    const int q_valid = a.q_valid != nullptr ? a.q_valid[j] : kBlk;
    const long long grow_idx = item * kBlk + r;
    // The last P V (tile n - 1) is awaited by the warpgroup that processed
    // tile n - 1 (it saw S_{n-1}, issued after the P V of tile n - 4 had
    // completed, so the phase of V_EMPTY is exact); that completion covers
    // every earlier MMA of the issuer, and every Q K^T completed before
    // S_{n-1}.  The named barrier then releases both warpgroups: K slot 0 is
    // free for the merge and O is final.
    if (ok && n > 0 && g == ((n - 1) & 1)) {
      ok = __all_sync(0xffffffffu,
                      mbar_wait_bounded(&bars[B_V_EMPTY + (n - 1) % kVSlots],
                                        ((n - 1) / kVSlots) & 1, s_abort, kWaitLimit));
      if (!ok) {
        report(a.d_err, BSA_DEV_WAIT_TIMEOUT);
        *s_abort = 1;
      }
    }
    tc_fence_before();
    named_bar_sync(9, kSoftmaxThreads);
    float* fin = reinterpret_cast<float*>(sm + L::kFin);  // [m, l][warpgroup][128 rows]
    fin[(0 * 2 + g) * kBlk + r] = m_last;
    fin[(1 * 2 + g) * kBlk + r] = l;
    named_bar_sync(9, kSoftmaxThreads);
    tc_fence_after();
    ok = __all_sync(0xffffffffu, ok && *s_abort == 0);
    const float m0 = fin[0 * kBlk + r], m1 = fin[1 * kBlk + r];
    const float m_fin = fmaxf(m0, m1);
    const bool have = ok && n > 0 && r < q_valid && m_fin > -INFINITY;
    float l_tot = 0.f;
    if (have) {
      l_tot = fin[2 * kBlk + r] * ex2_approx(m0 - m_fin) + fin[3 * kBlk + r] * ex2_approx(m1 - m_fin);
    }
    const float inv_l = have ? 1.0f / l_tot : 0.f;
    // Destination of this row: block order, or the raster token of the row
    // (a pad row has none and writes nothing).
    long long out_row = grow_idx;  // in units of D (O) and of 1 (LSE)
    bool write_row = true;
    if (kTokOut) {
      named_bar_sync(10, kSoftmaxThreads + 32);
      const int tok = reinterpret_cast<const int*>(sm + L::kSlotTok)[r];
      const long long b = bh / a.Hh, h = bh % a.Hh;
      out_row = (b * a.n_tok + tok) * a.Hh + h;
      write_row = tok >= 0;
    }
    __nv_bfloat16* orow = a.o + out_row * D + g * (D / 2);
#pragma unroll
    for (int c = 0; c < D / 64; ++c) {
      float o[32];
#pragma unroll
      for (int e = 0; e < 32; ++e) o[e] = 0.f;
      if (ok && n > 0) tmem_ld_cols<32>(tmem + lane_base + kColO + g * (D / 2) + c * 32, o);
#pragma unroll
      for (int e = 0; e < 32; e += 8) {
        uint4 v;
        v.x = pack_bf16x2(have ? o[e + 0] * inv_l : 0.f, have ? o[e + 1] * inv_l : 0.f);
        v.y = pack_bf16x2(have ? o[e + 2] * inv_l : 0.f, have ? o[e + 3] * inv_l : 0.f);
        v.z = pack_bf16x2(have ? o[e + 4] * inv_l : 0.f, have ? o[e + 5] * inv_l : 0.f);
        v.w = pack_bf16x2(have ? o[e + 6] * inv_l : 0.f, have ? o[e + 7] * inv_l : 0.f);
        if (kTokOut) {
          if (write_row) *reinterpret_cast<uint4*>(orow + c * 32 + e) = v;
        } else {
          // Block order: staged in K slot 1 (free: every Q K^T has
          // completed) in the layout of a loaded tile -- 64-column boxes
          // of 128 rows x 128 bytes, 16-byte chunk j of row r at chunk
          // j ^ (r % 8) -- and written by TMA below.
          const int col = g * (D / 2) + c * 32 + e;
          uint8_t* stage = sm + L::kK + kTileBytes + (col / 64) * (kBlk * 128);
          *reinterpret_cast<uint4*>(stage + r * 128 + ((((col % 64) / 8) ^ (r & 7)) * 16)) = v;
        }
      }
    }
    if (g == 0 && write_row)
      a.lse[out_row] = have ? (m_fin + __log2f(l_tot)) * 0.6931471805599453f : -INFINITY;
    if (!kTokOut) {
      // Both warpgroups' halves are staged; one thread writes the tile
      // (coalesced, where 128 threads writing their own rows would each
      // touch a different 256-byte row per store) and waits until the
      // copy has read shared memory, before the CTA can exit.
      fence_proxy_async_smem();
      named_bar_sync(9, kSoftmaxThreads);
      if (warp == 4 && elect_one()) {
        for (int bx = 0; bx < kBoxes; ++bx)
          tma_store_2d(&tm_o, bx * 64, static_cast<int>(item * kBlk),
                       sm + L::kK + kTileBytes + bx * (kBlk * 128));
        bulk_commit_group();
        bulk_wait_read_all();
      }
    }
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

template <int D, bool kTokOut>
static bsa_status launch_attn(const void* q, const bsa_kv_cache* c, const AttnArgs& a,
                              long long items, cudaStream_t s) {
  CUtensorMap tq, tk, tv, to;
  const long long crows = static_cast<long long>(c->B) * c->Hh * c->max_blocks * kBlk;
  if (!make_map(&tq, q, items * kBlk, D) || !make_map(&tk, c->k, crows, D) ||
      !make_map(&tv, c->v, crows, D))
    return BSA_ERR_CUDA;
  // O in block order has Q's layout; the token-order kernel stores O itself.
  if (kTokOut) {
    to = tq;
  } else if (!make_map(&to, a.o, items * kBlk, D)) {
    return BSA_ERR_CUDA;
  }
  const int smem = AttnLayout<D>::kAlloc;
  if (cudaFuncSetAttribute(bsa_attn_kernel<D, kTokOut>,
                           cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
    return BSA_ERR_CUDA;
  return launch_pdl(bsa_attn_kernel<D, kTokOut>, dim3(static_cast<unsigned>(items)),
                    dim3(kAttnThreads), static_cast<size_t>(smem), s, tq, tk, tv, to, a);
}

}  // namespace bsa

using namespace bsa;

namespace bsa {

// bsa_attn and bsa_attn_tokens: argument checks, then one launch.  perm is
// NULL for block-order output.
static bsa_status attn_call(const void* q_blk, const bsa_kv_cache* c, const int32_t* q_valid,
                            const int32_t* idx, const int32_t* cnt, int n_q_blocks, int max_sel,
                            float sm_scale, bool tok_out, const int32_t* perm, int T, int H,
                            int W, void* o, float* lse, int32_t* d_err, void* stream) {
  if (q_blk == nullptr || c == nullptr || idx == nullptr || cnt == nullptr || o == nullptr ||
      lse == nullptr || c->k == nullptr || c->v == nullptr || c->block_valid == nullptr)
    return BSA_ERR_INVALID_ARG;
  if (c->B <= 0 || c->Hh <= 0 || n_q_blocks <= 0 || max_sel <= 0 || c->max_blocks <= 0 ||
      c->n_blocks < 0 || c->n_blocks > c->max_blocks || !(sm_scale == sm_scale))
    return BSA_ERR_INVALID_ARG;
  if (c->D != 64 && c->D != 128) return BSA_ERR_UNSUPPORTED;
  if (!aligned16(q_blk) || !aligned16(o) || !aligned16(c->k) || !aligned16(c->v))
    return BSA_ERR_INVALID_ARG;
  const long long items = static_cast<long long>(c->B) * c->Hh * n_q_blocks;
  const long long crows = static_cast<long long>(c->B) * c->Hh * c->max_blocks * kBlk;
  if (items * kBlk >= (1LL << 31) || crows >= (1LL << 31)) return BSA_ERR_SHAPE;
  if (!device_is_sm100()) return BSA_ERR_UNSUPPORTED;
  AttnArgs a{};
  a.idx = idx;
  a.cnt = cnt;
  a.block_valid = c->block_valid;
  a.q_valid = q_valid;
  a.o = static_cast<__nv_bfloat16*>(o);
  a.lse = lse;
  a.d_err = d_err;
  a.perm = perm;
  a.n_tok = T * H * W;
  a.T = T;
  a.H = H;
  a.W = W;
  a.Hh = c->Hh;
  a.n_q_blocks = n_q_blocks;
  a.max_sel = max_sel;
  a.max_blocks = c->max_blocks;
  a.n_blocks = c->n_blocks;
  a.scale_log2 = sm_scale * kLog2e;
  cudaStream_t s = as_stream(stream);
  if (tok_out)
    return c->D == 128 ? launch_attn<128, true>(q_blk, c, a, items, s)
                       : launch_attn<64, true>(q_blk, c, a, items, s);
  return c->D == 128 ? launch_attn<128, false>(q_blk, c, a, items, s)
                     : launch_attn<64, false>(q_blk, c, a, items, s);
}

}  // namespace bsa

extern "C" bsa_status bsa_attn(const void* q_blk, const bsa_kv_cache* c, const int32_t* q_valid,
                               const int32_t* idx, const int32_t* cnt, int n_q_blocks, int max_sel,
                               float sm_scale, void* o_blk, float* lse, int32_t* d_err,
                               void* stream) {
  return attn_call(q_blk, c, q_valid, idx, cnt, n_q_blocks, max_sel, sm_scale, false, nullptr, 0,
                   0, 0, o_blk, lse, d_err, stream);
}

extern "C" bsa_status bsa_attn_tokens(const void* q_blk, const bsa_kv_cache* c,
                                      const int32_t* q_valid, const int32_t* idx,
                                      const int32_t* cnt, int max_sel, float sm_scale, int T,
                                      int H, int W, const int32_t* d_perm, void* o_tok,
                                      float* lse_tok, int32_t* d_err, void* stream) {
  if (T <= 0 || H <= 0 || W <= 0) return BSA_ERR_INVALID_ARG;
  const long long n = static_cast<long long>(T) * H * W;
  if (n > kTokOutMaxTokens) return BSA_ERR_UNSUPPORTED;
  const int nb = static_cast<int>((n + kBlk - 1) / kBlk);
  return attn_call(q_blk, c, q_valid, idx, cnt, nb, max_sel, sm_scale, true, d_perm, T, H, W,
                   o_tok, lse_tok, d_err, stream);
}
