/*
 * bsa.h - C ABI of the block-sparse KV attention library (libbsa.so).
 *
 * The library implements, for one NVIDIA B200 (sm_100a), the attention
 * path described in "Velox: Spatial Memory Makes World Models Efficient":
 *
 *   - a KV cache stored as 128-token blocks in a global-aligned
 *     generalised Hilbert ("Gilbert") order (Key Contributions 3;
 *     Methodology Step 6),                                 bsa_kv_append
 *   - a per-query-block router that scores KV blocks from the mean query and
 *     mean key of each block, adds a geometric overlap prior and keeps a
 *     bounded top-K route plus the query block's own chunk (Methodology
 *     Steps 4 and 5),                                      bsa_route
 *   - an indexed block-sparse attention that touches only the selected
 *     128-token blocks, skipping both the QK^T tile and the KV load of every
 *     other block (Methodology Step 6),                    bsa_attn
 *
 * Conventions shared by every call
 * --------------------------------
 *   Ownership  The caller allocates and frees all device memory and passes
 *              raw device pointers.  The library keeps no device state and
 *              allocates nothing on the device; workspaces are passed in.
 *   Streams    `stream` is a cudaStream_t passed as void* (NULL = the legacy
 *              default stream).  All device work is asynchronous on it.
 *   Types      Q, K, V and O are bf16; g and LSE are fp32; indices int32.
 *   Layout     Dense, row-major, no strides:
 *                token layout  [B, T*H*W, Hh, D]   raster (t, h, w) order
 *                block layout  [B, Hh, n_blocks, 128, D]
 *   Errors     Every call returns a bsa_status and never aborts.  Arguments
 *              are checked before anything is launched (nothing is launched
 *              when a check fails).  A launch failure maps to BSA_ERR_CUDA.
 *              Problems only the device can see (an index outside the cache,
 *              a count above max_sel, a bounded wait that gave up) are
 *              written as a BSA_DEV_* code into the caller's int32 word
 *              `d_err` (first error wins; the kernel then finishes without
 *              touching memory outside its arguments) and are read back
 *              with bsa_check_device_error.  d_err may be NULL to skip that
 *              reporting.
 *   Threads    Calls are thread-safe: the only global mutable state is a
 *              few small host-side caches (driver entry points, the
 *              bsa_route_noalloc scratch address), each guarded by a lock.
 */
#ifndef BSA_H_
#define BSA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define BSA_ABI_VERSION 2
#define BSA_BLOCK 128 /* tokens per KV block = attention tile height */

typedef enum bsa_status {
  BSA_OK = 0,
  BSA_ERR_INVALID_ARG = 1,  /* null pointer, non-positive size, bad scalar */
  BSA_ERR_SHAPE = 2,        /* sizes inconsistent with each other */
  BSA_ERR_CAPACITY = 3,     /* cache or output buffer too small */
  BSA_ERR_UNSUPPORTED = 4,  /* e.g. head_dim not 64 or 128, device not sm_100 */
  BSA_ERR_CUDA = 5,         /* a CUDA runtime call or launch failed */
  BSA_ERR_DEVICE_FAULT = 6, /* d_err held a BSA_DEV_* code */
  BSA_ERR_TIMEOUT = 7       /* d_err held BSA_DEV_WAIT_TIMEOUT */
} bsa_status;

/* Codes a kernel writes into d_err (0 = no error). */
#define BSA_DEV_OK 0
#define BSA_DEV_BAD_INDEX 1    /* a route index outside [0, n_blocks) */
#define BSA_DEV_BAD_COUNT 2    /* a route count outside [0, max_sel] */
#define BSA_DEV_BAD_VALID 3    /* a block_valid entry outside [1, 128] */
#define BSA_DEV_BAD_PERM 4     /* a permutation entry outside the chunk */
#define BSA_DEV_WAIT_TIMEOUT 5 /* a bounded pipeline wait gave up */

/*
 * Caller-owned view of the block KV cache.
 *   k, v         device bf16 [B, Hh, max_blocks, 128, D]
 *   block_valid  device int32 [max_blocks]: valid rows of each block (128, or
 *                the tail count of a chunk's last block); pad rows are zero.
 *   n_blocks     blocks in use, [0, max_blocks]; bsa_kv_append writes at
 *                [n_blocks, n_blocks + nb) and then advances it (host side).
 *   D            64 or 128.
 *   kmean        optional pooled-key cache, device fp32 [B, Hh, max_blocks, D]
 *                (16-byte aligned), or NULL.  When present, bsa_kv_append
 *                also writes the mean of the valid key rows of every block it
 *                appends, and bsa_route reads these means instead of streaming
 *                the history keys (Velox, Methodology Step 4: block importance
 *                from mean key vectors; pooling once per block at append time
 *                gives the same fp32 means as pooling during routing).  Blocks
 *                written into k directly need bsa_kv_pool_means.
 */
typedef struct bsa_kv_cache {
  void *k;
  void *v;
  int32_t *block_valid;
  int32_t B, Hh, D;
  int32_t max_blocks;
  int32_t n_blocks;
  float *kmean;
} bsa_kv_cache;

/* Returns BSA_ABI_VERSION of the loaded library. */
int bsa_abi_version(void);

/* Static, NUL-terminated name of a status code. */
const char *bsa_status_string(bsa_status status);

/*
 * Gilbert order of a T x H x W latent chunk (host only, no device work).
 * Velox, Key Contributions 3 and Methodology Step 6: neighbouring latent
 * cells are stored contiguously, and every chunk of one shape shares one
 * order ("global-aligned"), so block n of any chunk covers the same cells.
 *   host_perm  host int32 [T*H*W], written: host_perm[i] is the curve
 *              position of raster token i = (t*H + h)*W + w.  Consecutive
 *              positions are grid neighbours (unit steps).
 * Errors: BSA_ERR_INVALID_ARG (null pointer, non-positive extent),
 *         BSA_ERR_SHAPE (T*H*W above 2^24).
 */
bsa_status bsa_gilbert_perm(int T, int H, int W, int32_t *host_perm);

/*
 * Append one chunk to the cache (Velox, Key Contributions 3): token i of the
 * chunk goes to row perm[i] % 128 of block n_blocks + perm[i] / 128 for every
 * head; the tail pad rows of the last block are zeroed; block_valid is set
 * for the nb = ceil(T*H*W / 128) new blocks; cache->n_blocks += nb.
 *   k_tok, v_tok  device bf16 [B, T*H*W, Hh, D] (cache's B, Hh, D)
 *   d_perm        device int32 [T*H*W], the table from bsa_gilbert_perm
 *                 (any permutation of [0, T*H*W) is accepted; entries
 *                 outside that range raise BSA_DEV_BAD_PERM and are
 *                 skipped), or NULL: the kernels then locate every slot on
 *                 the Gilbert curve of (T, H, W) themselves (the order
 *                 bsa_gilbert_perm tabulates), with no table and nothing
 *                 allocated.  The same for every call below taking d_perm.
 * Errors: BSA_ERR_INVALID_ARG, BSA_ERR_CAPACITY (n_blocks + nb > max_blocks,
 *         cache unchanged), BSA_ERR_UNSUPPORTED, BSA_ERR_CUDA.
 */
bsa_status bsa_kv_append(bsa_kv_cache *cache, const void *k_tok, const void *v_tok,
                         int T, int H, int W, const int32_t *d_perm,
                         int32_t *d_err, void *stream);

/*
 * (Re)compute cache->kmean for blocks [first, first + count) of every
 * (batch, head) from cache->k and cache->block_valid: the mean of each
 * block's valid key rows in fp32, exactly as bsa_kv_append writes them.  For
 * blocks the caller wrote into the cache directly.
 * Errors: BSA_ERR_INVALID_ARG (kmean NULL, range outside [0, max_blocks)),
 *         BSA_ERR_UNSUPPORTED, BSA_ERR_CUDA; BSA_DEV_BAD_VALID on the device.
 */
bsa_status bsa_kv_pool_means(const bsa_kv_cache *cache, int first, int count,
                             int32_t *d_err, void *stream);

/*
 * The same scatter for a single tensor, e.g. the query chunk before routing:
 *   x_tok [B, T*H*W, Hh, D]  ->  x_blk [B, Hh, nb*128, D] (pad rows zeroed).
 * The pages do not state how Q is ordered; it shares the KV order so a query
 * block and a KV block of the same chunk cover the same cells.
 */
bsa_status bsa_tokens_to_blocks(const void *x_tok, void *x_blk, int B, int Hh, int D,
                                int T, int H, int W, const int32_t *d_perm,
                                int32_t *d_err, void *stream);

/*
 * bsa_tokens_to_blocks that also pools (Velox, Methodology Step 4: the block
 * importance uses the mean query of each block): besides x_blk it writes
 *   x_mean  device fp32 [B, Hh, nb, D], 16-byte aligned: the mean of the
 *           valid rows of every block (rows 0 .. min(128, T*H*W - 128*j) - 1
 *           of block j), summed in fp32 in the same fixed order as every
 *           other block mean of the library (bsa_route's own pooling, the
 *           pooled-key cache), so bsa_route_qmean on these means selects
 *           exactly what bsa_route on x_blk selects.
 * One pass over the tokens: the route then needs no second read of the
 * query blocks.  Chunks of up to 16384 tokens.
 * Errors: those of bsa_tokens_to_blocks; BSA_ERR_UNSUPPORTED above 16384
 *         tokens.
 */
bsa_status bsa_tokens_to_blocks_mean(const void *x_tok, void *x_blk, float *x_mean, int B,
                                     int Hh, int D, int T, int H, int W,
                                     const int32_t *d_perm, int32_t *d_err, void *stream);

/* Inverse gather, e.g. the attention output back to raster tokens:
 *   x_blk [B, Hh, nb*128, D]  ->  x_tok [B, T*H*W, Hh, D]. */
bsa_status bsa_blocks_to_tokens(const void *x_blk, void *x_tok, int B, int Hh, int D,
                                int T, int H, int W, const int32_t *d_perm,
                                int32_t *d_err, void *stream);

/* Device workspace bsa_route needs, in bytes (256-byte aligned pieces). */
bsa_status bsa_route_workspace_size(int B, int Hh, int D, int n_q_blocks, int n_hist,
                                    size_t *bytes);

/*
 * Route every (batch, head, query block) (Velox, Methodology Steps 4-5):
 *   qm[j] = mean of the valid rows of query block j,
 *   km[n] = mean of the valid rows of history block n (n < n_hist),
 *   s[j,n] = sm_scale * <qm[j], km[n]>  (+ lambda * min(g[b,j,n] / g_ref, 1)
 *            when g is given; g is shared by all heads),
 *   route = the top_k largest s over the history (ties to the lower block
 *           index; every history block when top_k >= n_hist), sorted
 *           ascending, followed by the own chunk [own_first, own_first+n_own).
 * Arithmetic is fp32 with a fixed reduction order; with the pooled-key
 * cache and at most 64 query blocks, <qm, km> runs on the tensor core as
 * three tf32 products of hi/lo splits of both means (about fp32's
 * precision, fixed order), so results are deterministic either way.
 *   q_blk      device bf16 [B, Hh, n_own*128, D] (block order)
 *   q_valid    device int32 [n_own] valid rows per query block, or NULL to
 *              use cache->block_valid[own_first + j]
 *   g          device fp32 [B, n_own, n_hist] or NULL
 *   idx        device int32 [B, Hh, n_own, max_sel]; entries past cnt are -1
 *   cnt        device int32 [B, Hh, n_own] = min(top_k, n_hist) + n_own
 *   workspace  device, at least bsa_route_workspace_size bytes, 256-aligned
 * Errors: BSA_ERR_INVALID_ARG, BSA_ERR_SHAPE (e.g. own chunk outside the
 *         cache, history overlapping it), BSA_ERR_CAPACITY (max_sel too
 *         small, workspace too small), BSA_ERR_UNSUPPORTED, BSA_ERR_CUDA.
 */
bsa_status bsa_route(const void *q_blk, const bsa_kv_cache *cache, const int32_t *q_valid,
                     int n_hist, int own_first, int n_own, const float *g,
                     float lambda, float g_ref, float sm_scale, int top_k,
                     int32_t *idx, int32_t *cnt, int max_sel,
                     void *workspace, size_t ws_bytes, int32_t *d_err, void *stream);

/*
 * bsa_route with the query-block means given instead of the query blocks
 * (Velox, Methodology Steps 4-5), e.g. from bsa_tokens_to_blocks_mean:
 *   q_mean  device fp32 [B, Hh, n_own, D], 16-byte aligned
 * Everything else, the result and the errors are those of bsa_route (the
 * workspace is sized by bsa_route_workspace_size as there).  With the means
 * of bsa_tokens_to_blocks_mean the routes equal bsa_route's bit for bit.
 */
bsa_status bsa_route_qmean(const float *q_mean, const bsa_kv_cache *cache, int n_hist,
                           int own_first, int n_own, const float *g, float lambda, float g_ref,
                           float sm_scale, int top_k, int32_t *idx, int32_t *cnt, int max_sel,
                           void *workspace, size_t ws_bytes, int32_t *d_err, void *stream);

/*
 * Indexed block-sparse attention (Velox, Methodology Step 6).  For query row
 * r of block j of head (b, h), over the valid rows k of the blocks
 * idx[b,h,j,0:cnt[b,h,j]] (order irrelevant, no causal mask):
 *   O_r   = sum_k softmax_k(sm_scale * q_r . k_k) v_k      (bf16 out)
 *   LSE_r = log sum_k exp(sm_scale * q_r . k_k)            (fp32, natural log)
 * Rows r >= q_valid[j], and every row of a query block with an empty route,
 * get O = 0 and LSE = -inf.  bf16 tensor-core products, fp32 accumulation.
 *   q_blk   device bf16 [B, Hh, n_q_blocks*128, D]
 *   q_valid device int32 [n_q_blocks] or NULL (all 128)
 *   idx,cnt device int32 as produced by bsa_route
 *   o_blk   device bf16 [B, Hh, n_q_blocks*128, D]
 *   lse     device fp32 [B, Hh, n_q_blocks*128]
 * Errors: BSA_ERR_INVALID_ARG, BSA_ERR_UNSUPPORTED (D not 64/128, no sm_100
 *         device), BSA_ERR_CUDA; on the device BSA_DEV_BAD_INDEX,
 *         BSA_DEV_BAD_COUNT, BSA_DEV_BAD_VALID, BSA_DEV_WAIT_TIMEOUT.
 */
bsa_status bsa_attn(const void *q_blk, const bsa_kv_cache *cache, const int32_t *q_valid,
                    const int32_t *idx, const int32_t *cnt, int n_q_blocks, int max_sel,
                    float sm_scale, void *o_blk, float *lse, int32_t *d_err, void *stream);

/*
 * bsa_attn with O and LSE written straight to raster token order (Velox,
 * Methodology Step 6, followed by the inverse of the query reordering):
 * row r of query block j is the token t with d_perm[t] = 128*j + r (the
 * Gilbert order of (T, H, W) when d_perm is NULL), so
 *   o_tok[b, t, h, :] = O of that row           device bf16 [B, T*H*W, Hh, D]
 *   lse_tok[b, t, h]  = LSE of that row          device fp32 [B, T*H*W, Hh]
 * and pad rows (slots no token maps to) are not written.  This saves the
 * separate bsa_blocks_to_tokens pass over O.  The query chunk has
 * ceil(T*H*W / 128) blocks; q_blk, q_valid, idx, cnt, max_sel and sm_scale
 * are those of bsa_attn, and d_perm is the table the query was reordered
 * with (bsa_tokens_to_blocks).  Chunks of up to 16384 tokens.
 * Errors: those of bsa_attn; BSA_ERR_UNSUPPORTED above 16384 tokens; on the
 *         device BSA_DEV_BAD_PERM for a d_perm that is not a permutation
 *         (rows without a token are then not written).
 */
bsa_status bsa_attn_tokens(const void *q_blk, const bsa_kv_cache *cache, const int32_t *q_valid,
                           const int32_t *idx, const int32_t *cnt, int max_sel, float sm_scale,
                           int T, int H, int W, const int32_t *d_perm, void *o_tok,
                           float *lse_tok, int32_t *d_err, void *stream);

/*
 * Self-test of the bounded-wait failure path used by every pipeline wait in
 * the library (there is no counterpart in the Velox page).  Launches one
 * thread that waits on an mbarrier nobody arrives on; after limit_cycles SM
 * clocks (1 .. 2^34) the wait gives up, BSA_DEV_WAIT_TIMEOUT is written to
 * d_err, and the kernel returns normally: bsa_check_device_error then
 * reports BSA_ERR_TIMEOUT and the CUDA context stays usable.
 * Errors: BSA_ERR_INVALID_ARG (null d_err, limit out of range), BSA_ERR_CUDA.
 */
bsa_status bsa_selftest_bounded_wait(int32_t *d_err, long long limit_cycles, void *stream);

/*
 * Options of the page's own route (Velox, Methodology Steps 4-5).
 *   coverage     device fp32 [B, n_own]: fraction of each query block's
 *                tokens inside a valid historical slab, or NULL (no query
 *                block is well covered)
 *   eta_cov      a query block is well covered when coverage >= eta_cov (0.9)
 *   tau          overlap at or below tau counts as none (0.1)
 *   k_cov        covered route size: the previous chunk is reserved first,
 *                then the best other history blocks up to k_cov in all (80)
 *   k_unc        cap of the uncovered route (150, at most 1024)
 *   mass         uncovered route: smallest prefix of softmax(s), in order of
 *                decreasing s (ties to the lower index), whose mass reaches
 *                this value (the page does not state it; 0.9 is a choice)
 *   prev_first, n_prev   the previous chunk's blocks [prev_first, +n_prev)
 *   window_half  window of previous-chunk blocks at Gilbert positions
 *                j - window_half .. j + window_half around query block j,
 *                added outside the budget (13)
 *   ref_first, n_ref     reference blocks always added (n_ref may be 0)
 */
typedef struct bsa_velox_route {
  const float *coverage;
  float eta_cov, tau;
  int32_t k_cov, k_unc;
  float mass;
  int32_t prev_first, n_prev;
  int32_t window_half;
  int32_t ref_first, n_ref;
} bsa_velox_route;

/*
 * The page's full route for every (batch, head, query block).  Scores s are
 * those of bsa_route (sm_scale * <mean q, mean k>, from the pooled-key cache
 * when present).  A well-covered query block ranks history blocks by
 * s + log(1 + lambda * g_hat), g_hat = min(g / g_ref, 1) where g > tau and 0
 * elsewhere, which is the order of the importance distribution multiplied by
 * (1 + lambda * g_hat) and renormalised; it takes the previous chunk, then
 * the best remaining blocks up to k_cov.  Other query blocks take the
 * smallest mass prefix of the unfused distribution, at most k_unc blocks.
 * Every route is joined with the window and reference blocks, sorted
 * ascending without repeats, and followed by the own chunk; cnt varies per
 * query block and unused idx entries are -1.
 *   max_sel   at least min(n_hist, max(k_cov, n_prev, k_unc) + 2 *
 *             window_half + 1 + n_ref) + n_own, else BSA_ERR_CAPACITY
 * Errors: those of bsa_route; BSA_ERR_UNSUPPORTED when n_hist > 32768 or
 *         k_unc > 1024.
 */
bsa_status bsa_route_velox(const void *q_blk, const bsa_kv_cache *cache, const int32_t *q_valid,
                           int n_hist, int own_first, int n_own, const float *g,
                           float lambda, float g_ref, float sm_scale,
                           const bsa_velox_route *opts, int32_t *idx, int32_t *cnt, int max_sel,
                           void *workspace, size_t ws_bytes, int32_t *d_err, void *stream);

/*
 * bsa_route_velox with the query-block means given instead of the query
 * blocks (Velox, Methodology Steps 4-5), e.g. from bsa_tokens_to_blocks_mean:
 *   q_mean  device fp32 [B, Hh, n_own, D], 16-byte aligned
 * Everything else, the result and the errors are those of bsa_route_velox.
 * With the means of bsa_tokens_to_blocks_mean the routes equal
 * bsa_route_velox's bit for bit.
 */
bsa_status bsa_route_velox_qmean(const float *q_mean, const bsa_kv_cache *cache, int n_hist,
                                 int own_first, int n_own, const float *g, float lambda,
                                 float g_ref, float sm_scale, const bsa_velox_route *opts,
                                 int32_t *idx, int32_t *cnt, int max_sel, void *workspace,
                                 size_t ws_bytes, int32_t *d_err, void *stream);

/*
 * Geometric overlap prior g and coverage from slabs (Velox, Methodology
 * Step 3; slabs as in Step 1).  Each slab (a source-camera token rectangle
 * [u0, u1] x [v0, v1] in pixel-edge coordinates plus a depth interval
 * [d0, d1]) becomes the smallest box with its camera's axes that holds its
 * frustum segment.  g[b, j, m] is the largest IoU between a valid slab box
 * of query block j and one of history block m, each IoU estimated on an
 * n x n x n grid of cell centres of the query box after a separating-axis
 * test (0 when separated); the intersection is capped at the smaller box
 * volume, so g is in [0, 1].  coverage[b, j] is the fraction of query block
 * j's valid tokens (q_valid[j] of 128) whose back-projected point lies in a
 * valid slab of any history block: depth in that slab's camera within
 * [d0, d1], projection within its rectangle.  Tokens without depth count as
 * uncovered.  All decisions are float32 with one rounding per operation in
 * a fixed order, so the counts are reproducible.  g and coverage are the
 * inputs bsa_route and bsa_route_velox take.
 *   cams       device float32 [B, n_cams, 12]: R (3x3 row-major, world from
 *              camera; camera axes x right, y down, z forward) then the
 *              camera centre; pinhole intrinsics fx, fy, cx, cy (latent
 *              pixels) shared by all cameras
 *   q_cam      device int32 [B, n_q, S]: camera of each query slab, -1 = none
 *   q_rect     device float32 [B, n_q, S, 6]: u0, u1, v0, v1, d0, d1
 *   h_cam      device int32 [B, n_hist, S], h_rect [B, n_hist, S, 6]: history
 *   S          slabs per block, 1..4;  grid_n  grid points per axis, 1..16
 *   tok_cam    device int32 [B, n_q, 128]: camera of each query token, -1 =
 *              no depth;  tok_uvd  device float32 [B, n_q, 128, 3]: u, v, d
 *   q_valid    device int32 [n_q] valid tokens per query block, or NULL (128)
 *   g          device float32 [B, n_q, n_hist] written, or NULL (skipped)
 *   coverage   device float32 [B, n_q] written, or NULL (skipped)
 * Errors: BSA_ERR_INVALID_ARG (null input for a requested output, both
 *         outputs NULL, S or grid_n out of range, fx or fy not positive),
 *         BSA_ERR_SHAPE, BSA_ERR_CUDA; on the device a camera index outside
 *         [-1, n_cams) raises BSA_DEV_BAD_INDEX (the slab or token is then
 *         absent) and a q_valid entry outside [0, 128] BSA_DEV_BAD_VALID.
 */
bsa_status bsa_geometry_prior(const float *cams, int n_cams, float fx, float fy, float cx,
                              float cy, const int32_t *q_cam, const float *q_rect, int n_q,
                              const int32_t *h_cam, const float *h_rect, int n_hist,
                              int slabs_per_block, int grid_n, const int32_t *tok_cam,
                              const float *tok_uvd, const int32_t *q_valid, int B, float *g,
                              float *coverage, int32_t *d_err, void *stream);

/*
 * bsa_route without a workspace argument, for callers that cannot allocate
 * device memory themselves: for example code running inside another
 * runtime's plugin or enqueue hook, where the host framework owns every
 * device allocation and forbids new ones, or a latency-bound loop that cannot
 * afford cudaMalloc's implicit device synchronisation.  There is no
 * counterpart in the Velox page; it only changes where bsa_route's scratch
 * lives.
 *   Scratch   a fixed array of BSA_ROUTE_NOALLOC_SCRATCH_BYTES (16 MiB) in
 *             the library's device image, present on every GPU that loads the
 *             library until the process exits.  The call allocates nothing
 *             (no cudaMalloc, no allocating library routine).
 *   Set-up    the first call on a device looks up that device's address of
 *             the array (cudaGetSymbolAddress, with the device current) and
 *             caches it together with the process-unique id of the current
 *             CUDA context; make that first call before any stream capture.
 *             The address is only valid in that context: after a device
 *             reset, or from another context on the device, the id differs
 *             and the next call looks the address up again (that call is
 *             then a first call again).
 *   Sharing   every call on a device uses the same array.  Nothing in it has
 *             to start at zero (each call writes every entry it reads), but
 *             calls that overlap on the GPU (different streams, or threads
 *             without ordering) race on it and must be serialised by the
 *             caller.
 * Arguments, results and errors are those of bsa_route; in addition a
 * problem whose workspace (bsa_route_workspace_size) exceeds the scratch size
 * returns BSA_ERR_CAPACITY without launching anything.
 */
#define BSA_ROUTE_NOALLOC_SCRATCH_BYTES (16u << 20)
bsa_status bsa_route_noalloc(const void *q_blk, const bsa_kv_cache *cache, const int32_t *q_valid,
                             int n_hist, int own_first, int n_own, const float *g,
                             float lambda, float g_ref, float sm_scale, int top_k,
                             int32_t *idx, int32_t *cnt, int max_sel, int32_t *d_err,
                             void *stream);

/*
 * Synchronise `stream`, read d_err, clear it, and map it to a status:
 * BSA_OK, BSA_ERR_TIMEOUT (BSA_DEV_WAIT_TIMEOUT) or BSA_ERR_DEVICE_FAULT.
 * The raw code is stored in *code_out when code_out is not NULL.
 */
bsa_status bsa_check_device_error(int32_t *d_err, void *stream, int32_t *code_out);

#ifdef __cplusplus
}
#endif

#endif /* BSA_H_ */
