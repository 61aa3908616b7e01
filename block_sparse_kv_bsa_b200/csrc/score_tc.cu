// score_tc.cu - the pooled product of routing on the tensor core.
//
// "Velox: Spatial Memory Makes World Models Efficient", Methodology Step 4:
// the model part of a history block's importance for a query block is the
// scaled dot product of the query block's mean query with the history
// block's mean key,
//   s[j, n] = sm_scale * <qmean_j, kmean_n>,
// for every query block j of a head and every history block n of the same
// head: per head a [n_own x D] by [D x n_hist] product of fp32 means.
//
// The scores decide an exact top-K, so they need about fp32's precision, not
// tf32's.  Each mean x is split as x = hi + lo, hi = x with its 13 low
// mantissa bits cleared (exact in tf32) and lo = x - hi (exact in fp32), and
// the product runs as three tcgen05.mma kind::tf32 passes into one fp32
// accumulator:
//   <q, k> = <q_lo, k_hi> + <q_hi, k_lo> + <q_hi, k_hi>   (+ <q_lo, k_lo>)
// The dropped term and lo's own rounding to tf32 are each below 2^-20 of
// |q_d k_d| per term, far inside the route's near-tie tolerance.
//
// One CTA takes a contiguous run of 128-key tiles of one (batch, head), so it
// loads and splits that head's query means once:
//   A  = 128 pooled keys (lane = history block) in tensor memory: a tile
//        arrives by TMA in 128-byte slices of 32 dims (a four-stage ring in
//        shared memory); the thread of each key row reads its 32 values,
//        splits them and stores hi and lo into a four-stage ring of 64
//        tensor-memory columns, so the MMAs read only B from shared memory;
//   B  = the head's query means, rows 0..63 (N = n_own rounded up to 16;
//        rows past n_own only feed accumulator columns that are never
//        read), split once in shared memory, K-major 128-byte slices;
//   D  = two 64-column fp32 accumulators in tensor memory, lane = history
//        block, column = query block.
// The accumulator's lanes are consecutive history blocks, so each store of
// the epilogue writes 32 consecutive scores of one query block's row.
// Tensor memory (512 columns): [0, 128) the accumulators, [128, 384) the
// key ring (stage s: hi at 128 + 64 s, lo 32 columns further).
// Warp roles (320 threads):
//   warps 0-3  split the query means once, then every key slice, one key
//              row per thread (TMEM lane window = warp);
//   warps 4-7  epilogue: one TMEM lane window each (32 history blocks),
//              scale, store one row segment per query block;
//   warp 8     TMA producer (query means once, key slices into the ring);
//   warp 9     allocates tensor memory; one elected lane issues the MMAs.
// Every wait is bounded; a wait that gives up records BSA_DEV_WAIT_TIMEOUT,
// stops the other roles through a shared flag, lets in-flight copies and
// MMAs finish (bounded) and frees tensor memory.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <mutex>

#include "common.cuh"

namespace bsa {

constexpr int kTcKeys = 128;          // history blocks per tile (MMA M)
constexpr int kTcMaxOwn = 64;         // query blocks of a head held in B
constexpr int kTcThreads = 320;
constexpr int kTcSplitThreads = 128;  // warps 0-3
constexpr int kTcEpiThreads = 128;    // warps 4-7
constexpr int kTcTmaWarp = 8;
constexpr int kTcMmaWarp = 9;
constexpr int kTcStages = 4;          // key slices in flight (shared and tensor memory)
constexpr uint32_t kTcColA = 128;     // first column of the key ring
constexpr int kTcTrStride = 36;       // floats per query row of an epilogue transpose
constexpr long long kTcWaitLimit = 1LL << 31;  // SM clocks (about a second)

enum : int {
  TB_Q_FULL = 0,
  TB_Q_SPLIT = 1,
  TB_K_FULL = 2,                         // kTcStages: slice landed in shared memory
  TB_K_FREE = TB_K_FULL + kTcStages,     // slice read out of shared memory
  TB_A_READY = TB_K_FREE + kTcStages,    // hi / lo stored in tensor memory
  TB_A_EMPTY = TB_A_READY + kTcStages,   // MMAs that read them completed
  TB_ACC_FULL = TB_A_EMPTY + kTcStages,  // 2 accumulators
  TB_ACC_EMPTY = TB_ACC_FULL + 2,
  TB_MMA_DONE = TB_ACC_EMPTY + 2,
  TB_COUNT = TB_MMA_DONE + 1
};

template <int D>
struct TcLayout {
  static constexpr int kSlices = D / 32;                   // 128-byte slices of 32 dims
  static constexpr int kQSlice = 64 * 128;                 // 64 query-mean rows
  static constexpr int kQBytes = kSlices * kQSlice;        // one half (hi or lo)
  static constexpr int kKSlice = kTcKeys * 128;            // 128 key rows
  static constexpr int kQHi = 0;
  static constexpr int kQLo = kQHi + kQBytes;
  static constexpr int kK = kQLo + kQBytes;                // stage s at kK + s * kKSlice
  static constexpr int kTr = kK + kTcStages * kKSlice;     // epilogue transposes
  static constexpr int kBars = kTr + 4 * kTcMaxOwn * kTcTrStride * 4;
  static constexpr int kMisc = kBars + TB_COUNT * 8;
  static constexpr int kBytes = kMisc + 16;
  static constexpr int kAlloc = kBytes + 1024;             // 1024-byte alignment slack
};
static_assert(TcLayout<128>::kAlloc <= 227 * 1024, "shared memory");

struct TcScoreArgs {
  float* s;          // [BH, n_own, s_ld]
  long long s_ld;    // score row stride (a multiple of 32: rows start 128-byte aligned)
  int32_t* d_err;
  int n_own, n_hist, splits;
  long long q_rows_per_head;  // n_own
  long long k_rows_per_head;  // max_blocks
  float sm_scale;
};

// Instruction descriptor of tcgen05.mma kind::tf32: tf32 x tf32 -> fp32,
// A and B K-major, M x N.
__host__ __device__ constexpr uint32_t idesc_tf32(int M, int N) {
  return (1u << 4)                                  // D format: f32
         | (2u << 7)                                // A format: tf32
         | (2u << 10)                               // B format: tf32
         | (static_cast<uint32_t>(N >> 3) << 17)    // N / 8
         | (static_cast<uint32_t>(M >> 4) << 24);   // M / 16
}

// D[tmem] (+)= A[tmem] * B[smem]^T, kind::tf32: A is M = 128 rows, one per
// TMEM lane, K-major with one tf32 element per 32-bit column.
__device__ __forceinline__ void tc_mma_tf32_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                               uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::tf32 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

__device__ __forceinline__ uint32_t tf32_hi(uint32_t x) { return x & 0xffffe000u; }
__device__ __forceinline__ uint32_t tf32_lo(uint32_t x) {
  return __float_as_uint(__fsub_rn(__uint_as_float(x), __uint_as_float(tf32_hi(x))));
}

// Split `bytes` of fp32 at `hi` in place into hi (13 low mantissa bits
// cleared) and lo = x - hi at the same offset from `lo`.  Both buffers have
// the same 1024-byte-aligned swizzled layout, so a value keeps its place.
__device__ __forceinline__ void split_tf32(uint8_t* hi, uint8_t* lo, int bytes, int tid) {
#pragma unroll 4
  for (int o = tid * 16; o < bytes; o += kTcSplitThreads * 16) {
    const uint4 x = *reinterpret_cast<const uint4*>(hi + o);
    *reinterpret_cast<uint4*>(hi + o) =
        make_uint4(tf32_hi(x.x), tf32_hi(x.y), tf32_hi(x.z), tf32_hi(x.w));
    *reinterpret_cast<uint4*>(lo + o) =
        make_uint4(tf32_lo(x.x), tf32_lo(x.y), tf32_lo(x.z), tf32_lo(x.w));
  }
}

template <int D>
__global__ void __launch_bounds__(kTcThreads, 1)
score_means_tc_kernel(const __grid_constant__ CUtensorMap tm_q,
                      const __grid_constant__ CUtensorMap tm_k, TcScoreArgs a) {
  using L = TcLayout<D>;
  constexpr int S = L::kSlices;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                           ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + L::kBars);
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(sm + L::kMisc);
  volatile int* s_abort = reinterpret_cast<volatile int*>(sm + L::kMisc + 4);

  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  const long long bh = blockIdx.x / a.splits;
  const int part = blockIdx.x % a.splits;
  const int per_head = (a.n_hist + kTcKeys - 1) / kTcKeys;
  const int t_first = static_cast<int>(static_cast<long long>(part) * per_head / a.splits);
  const int nt = static_cast<int>(static_cast<long long>(part + 1) * per_head / a.splits) - t_first;
  const int n_slices = nt * S;  // key slices of this CTA, slice f in stage f % kTcStages

  if (threadIdx.x == 0) {
    for (int i = 0; i < TB_COUNT; ++i) {
      uint32_t count = 1;
      if (i == TB_Q_SPLIT || (i >= TB_K_FREE && i < TB_A_EMPTY)) count = kTcSplitThreads;
      if (i == TB_ACC_EMPTY || i == TB_ACC_EMPTY + 1) count = kTcEpiThreads;
      mbar_init(&bars[i], count);
    }
    *s_abort = 0;
    fence_mbar_init();
  }
  if (warp == kTcMmaWarp) tmem_alloc(s_tmem, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *s_tmem;
  // The query means are written by the kernel before this one.
  pdl_wait();
  pdl_trigger();

  if (warp == kTcTmaWarp) {
    // ---------------- TMA producer ----------------
    if (lane == 0 && nt > 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      mbar_expect_tx(&bars[TB_Q_FULL], L::kQBytes);
      for (int sl = 0; sl < S; ++sl)
        tma_load_2d(sm + L::kQHi + sl * L::kQSlice, &tm_q, sl * 32,
                    static_cast<int>(bh * a.q_rows_per_head), &bars[TB_Q_FULL]);
      int issued = 0;
      bool ok = true;
      for (int f = 0; f < n_slices; ++f) {
        const int st = f % kTcStages;
        if (f >= kTcStages) {
          ok = mbar_wait_bounded(&bars[TB_K_FREE + st], ((f / kTcStages) - 1) & 1, s_abort,
                                 kTcWaitLimit);
          if (!ok) break;
        }
        const int row = static_cast<int>(bh * a.k_rows_per_head + (t_first + f / S) * kTcKeys);
        mbar_expect_tx(&bars[TB_K_FULL + st], L::kKSlice);
        tma_load_2d(sm + L::kK + st * L::kKSlice, &tm_k, (f % S) * 32, row,
                    &bars[TB_K_FULL + st]);
        issued = f + 1;
      }
      if (!ok) {
        report(a.d_err, BSA_DEV_WAIT_TIMEOUT);
        *s_abort = 1;
      }
      // Drain: every copy issued must land before the CTA exits.
      mbar_wait_bounded(&bars[TB_Q_FULL], 0, nullptr, kTcWaitLimit);
      for (int st = 0; st < kTcStages; ++st) {
        int last = -1;
        for (int f = st; f < issued; f += kTcStages) last = f;
        if (last >= 0)
          mbar_wait_bounded(&bars[TB_K_FULL + st], (last / kTcStages) & 1, nullptr,
                            kTcWaitLimit);
      }
    }
  } else if (warp == kTcMmaWarp) {
    // ---------------- MMA issuer ----------------
    // Per key slice, small terms first: k_lo q_hi, k_hi q_lo, then k_hi q_hi.
    if (nt > 0) {
      const uint32_t id = idesc_tf32(kTcKeys, (a.n_own + 15) & ~15);
      const uint64_t q_hi = smem_desc(smem_u32(sm + L::kQHi), 16, 1024);
      const uint64_t q_lo = smem_desc(smem_u32(sm + L::kQLo), 16, 1024);
      constexpr uint32_t kQSlice16 = L::kQSlice >> 4;
      bool ok = __all_sync(0xffffffffu,
                           mbar_wait_bounded(&bars[TB_Q_SPLIT], 0, s_abort, kTcWaitLimit));
      for (int f = 0; ok && f < n_slices; ++f) {
        const int t = f / S, sl = f % S, st = f % kTcStages, acc = t & 1;
        if (sl == 0 && t >= 2)
          ok = __all_sync(0xffffffffu,
                          mbar_wait_bounded(&bars[TB_ACC_EMPTY + acc], ((t >> 1) - 1) & 1,
                                            s_abort, kTcWaitLimit));
        if (ok)
          ok = __all_sync(0xffffffffu, mbar_wait_bounded(&bars[TB_A_READY + st],
                                                         (f / kTcStages) & 1, s_abort,
                                                         kTcWaitLimit));
        if (!ok) break;
        tc_fence_after();
        const uint32_t k_hi = tmem + kTcColA + st * 64, k_lo = k_hi + 32;
        const uint64_t qh = desc_add(q_hi, sl * kQSlice16);
        const uint64_t ql = desc_add(q_lo, sl * kQSlice16);
        if (elect_one()) {
#pragma unroll
          for (int pass = 0; pass < 3; ++pass) {
            const uint32_t ka = pass == 0 ? k_lo : k_hi;
            const uint64_t bd = pass == 1 ? ql : qh;
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              tc_mma_tf32_ts(tmem + acc * 64, ka + kk * 8, desc_add(bd, kk * 2), id,
                             (sl > 0 || pass > 0 || kk > 0) ? 1u : 0u);
          }
          tc_commit(&bars[TB_A_EMPTY + st]);
          if (sl == S - 1) tc_commit(&bars[TB_ACC_FULL + acc]);
        }
        __syncwarp();
      }
      if (!ok && lane == 0) {
        report(a.d_err, BSA_DEV_WAIT_TIMEOUT);
        *s_abort = 1;
      }
      // Drain: every MMA issued completes before tensor memory is freed.
      if (lane == 0) {
        tc_commit(&bars[TB_MMA_DONE]);
        mbar_wait_bounded(&bars[TB_MMA_DONE], 0, nullptr, kTcWaitLimit);
      }
      __syncwarp();
    }
  } else if (warp < 4) {
    // ---------------- hi / lo split ----------------
    if (nt > 0) {
      const int tid = threadIdx.x;
      // Every wait is warp-uniform: tcgen05.st below needs whole warps.
      bool ok = __all_sync(0xffffffffu,
                           mbar_wait_bounded(&bars[TB_Q_FULL], 0, s_abort, kTcWaitLimit));
      if (ok) {
        split_tf32(sm + L::kQHi, sm + L::kQLo, L::kQBytes, tid);
        fence_proxy_async_smem();
        mbar_arrive(&bars[TB_Q_SPLIT]);
      }
      // Key slices: the thread of key row r (TMEM lane r) reads the row's
      // 32 values (16-byte chunk c of row r sits at chunk c ^ (r % 8) of the
      // 128-byte swizzled row), releases the shared-memory stage, and
      // stores hi and lo into the stage's tensor-memory columns once the
      // MMAs that read them last have completed.
      const int r = tid;                       // warps 0-3: TMEM lanes 0..127
      const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
      for (int f = 0; ok && f < n_slices; ++f) {
        const int st = f % kTcStages;
        ok = __all_sync(0xffffffffu, mbar_wait_bounded(&bars[TB_K_FULL + st],
                                                       (f / kTcStages) & 1, s_abort,
                                                       kTcWaitLimit));
        if (!ok) break;
        const uint8_t* row = sm + L::kK + st * L::kKSlice + r * 128;
        uint32_t hi[32], lo[32];
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          const uint4 x = *reinterpret_cast<const uint4*>(row + ((c ^ (r & 7)) * 16));
          hi[4 * c + 0] = x.x;
          hi[4 * c + 1] = x.y;
          hi[4 * c + 2] = x.z;
          hi[4 * c + 3] = x.w;
        }
        mbar_arrive(&bars[TB_K_FREE + st]);
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          lo[e] = tf32_lo(hi[e]);
          hi[e] = tf32_hi(hi[e]);
        }
        if (f >= kTcStages)
          ok = __all_sync(0xffffffffu,
                          mbar_wait_bounded(&bars[TB_A_EMPTY + st], ((f / kTcStages) - 1) & 1,
                                            s_abort, kTcWaitLimit));
        if (!ok) break;
        tc_fence_after();
        const uint32_t col = tmem + lane_base + kTcColA + st * 64;
        tmem_st32u(col, hi);
        tmem_st32u(col + 32, lo);
        tc_wait_st();
        tc_fence_before();
        mbar_arrive(&bars[TB_A_READY + st]);
      }
      if (!ok) {
        report(a.d_err, BSA_DEV_WAIT_TIMEOUT);
        *s_abort = 1;
      }
    }
  } else if (warp < 8) {
    // ---------------- epilogue ----------------
    // Thread (warp w, lane l) holds history block n0 + 32 (w - 4) + l: its
    // scores against query blocks 0..63 are its accumulator row.  Each warp
    // transposes its 32 x 64 scores through shared memory ([query][key],
    // 36 floats per query row: conflict-free both ways) and writes every
    // query row's 32 scores as 8 16-byte pieces, four rows per store.
    // Score rows are 128-byte aligned (s_ld a multiple of 32), so a warp's
    // 32 blocks lie in one row whenever the first does; scores of blocks
    // past n_hist land in the row's padding, which nothing reads.
    if (nt > 0) {
      const int wq = warp - 4;               // TMEM lanes 32*wq .. 32*wq + 31
      const uint32_t lane_base = static_cast<uint32_t>(wq * 32) << 16;
      float* tr = reinterpret_cast<float*>(sm + L::kTr) + wq * kTcMaxOwn * kTcTrStride;
      float* row0 = a.s + bh * a.q_rows_per_head * a.s_ld;
      const int rows = a.n_own;
      bool ok = true;
      for (int t = 0; t < nt; ++t) {
        const int acc = t & 1;
        ok = __all_sync(0xffffffffu, mbar_wait_bounded(&bars[TB_ACC_FULL + acc], (t >> 1) & 1,
                                                       s_abort, kTcWaitLimit));
        if (!ok) break;
        tc_fence_after();
#pragma unroll
        for (int h = 0; h < kTcMaxOwn; h += 32) {
          float v[32];
          tmem_ld_cols<32>(tmem + lane_base + acc * 64 + h, v);
          if (h + 32 == kTcMaxOwn) {
            tc_fence_before();
            mbar_arrive(&bars[TB_ACC_EMPTY + acc]);
          }
#pragma unroll
          for (int e = 0; e < 32; ++e) tr[(h + e) * kTcTrStride + lane] = a.sm_scale * v[e];
        }
        __syncwarp();
        const int n0 = (t_first + t) * kTcKeys + wq * 32;
        if (n0 < a.s_ld) {
          float* dst = row0 + n0 + (lane & 7) * 4;
          for (int i = lane; i < rows * 8; i += 32) {
            const int j = i >> 3;
            const float4 x = *reinterpret_cast<const float4*>(tr + j * kTcTrStride + (lane & 7) * 4);
            *reinterpret_cast<float4*>(dst + static_cast<long long>(j) * a.s_ld) = x;
          }
        }
        __syncwarp();
      }
      if (!ok && lane == 0) {
        report(a.d_err, BSA_DEV_WAIT_TIMEOUT);
        *s_abort = 1;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kTcMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

static PFN_cuTensorMapEncodeTiled_v12000 tc_encode_fn() {
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

// 2D map over an fp32 matrix [rows, D]: boxes of `box_rows` rows x 32
// columns (128 bytes), 128-byte swizzle; rows past the end read as zeros.
static bool make_map_f32(CUtensorMap* m, const float* base, long long rows, int D, int box_rows) {
  auto enc = tc_encode_fn();
  if (enc == nullptr) return false;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(D) * 4};
  cuuint32_t box[2] = {32, static_cast<cuuint32_t>(box_rows)};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<float*>(base), dims, strides,
                   box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool score_means_tc_fits(int n_own, int D) {
  return n_own >= 1 && n_own <= kTcMaxOwn && (D == 64 || D == 128);
}

// s[(bh * n_own + j) * s_ld + n] = sm_scale * <qm[bh, j], kmean[bh, n]> for
// bh < BH, j < n_own, n < n_hist; qm is [BH, n_own, D], kmean [BH,
// max_blocks, D], both fp32 and 16-byte aligned.  `sms` sets how many CTAs
// share a head's tiles.
bsa_status launch_score_means_tc(const float* qm, const float* kmean, float* s, int s_ld, int BH,
                                 int n_own, int n_hist, int max_blocks, int D, float sm_scale,
                                 int sms, int32_t* d_err, cudaStream_t st) {
  if (!score_means_tc_fits(n_own, D) || n_hist <= 0 || BH <= 0 || n_hist > max_blocks ||
      s_ld < n_hist)
    return BSA_ERR_UNSUPPORTED;
  if (static_cast<long long>(BH) * max_blocks + kTcKeys > (1LL << 31) - 1)
    return BSA_ERR_SHAPE;
  CUtensorMap tq, tk;
  if (!make_map_f32(&tq, qm, static_cast<long long>(BH) * n_own, D, kTcMaxOwn) ||
      !make_map_f32(&tk, kmean, static_cast<long long>(BH) * max_blocks, D, kTcKeys))
    return BSA_ERR_CUDA;
  const int per_head = (n_hist + kTcKeys - 1) / kTcKeys;
  int splits = sms > 0 ? sms / BH : 1;
  splits = std::max(1, std::min(splits, per_head));
  if (static_cast<long long>(BH) * splits > (1LL << 31) - 1) return BSA_ERR_SHAPE;
  TcScoreArgs a{};
  a.s = s;
  a.s_ld = s_ld;
  a.d_err = d_err;
  a.n_own = n_own;
  a.n_hist = n_hist;
  a.splits = splits;
  a.q_rows_per_head = n_own;
  a.k_rows_per_head = max_blocks;
  a.sm_scale = sm_scale;
  const dim3 grid(static_cast<unsigned>(BH * splits));
  if (D == 128) {
    constexpr int smem = TcLayout<128>::kAlloc;
    if (cudaFuncSetAttribute(score_means_tc_kernel<128>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
      return BSA_ERR_CUDA;
    return launch_pdl(score_means_tc_kernel<128>, grid, dim3(kTcThreads),
                      static_cast<size_t>(smem), st, tq, tk, a);
  }
  constexpr int smem = TcLayout<64>::kAlloc;
  if (cudaFuncSetAttribute(score_means_tc_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           smem) != cudaSuccess)
    return BSA_ERR_CUDA;
  return launch_pdl(score_means_tc_kernel<64>, grid, dim3(kTcThreads), static_cast<size_t>(smem),
                    st, tq, tk, a);
}

}  // namespace bsa
