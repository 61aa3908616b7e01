// geometry.cu - bsa_geometry_prior: the geometric overlap prior g and the
// coverage score from slabs.
//
// "Velox: Spatial Memory Makes World Models Efficient", Methodology Step 3:
// each query slab and historical slab (Step 1: a source-camera token
// rectangle plus a depth interval) is approximated by a camera-facing
// oriented bounding box; the score of a (query block, KV block) pair is the
// IoU of the query box with the best-matching historical box, estimated on
// a deterministic grid after a separating-axis test; the coverage of a query
// block is the fraction of its tokens that fall inside a valid historical
// slab both spatially and in depth.
//
// Every quantity that decides an integer (inside or not, separated or not)
// is computed in float32 with one rounding per operation, in a fixed order
// (explicit __fmul_rn / __fadd_rn / __fdiv_rn, so nothing is contracted into
// an FMA), so that the counts are reproducible operation by operation:
//   box: tan-space edges (u - cx) / fx, the frustum segment's extremes over
//        the two depths, centre c + ((R0 l0 + R1 l1) + R2 l2);
//   separating axes: in box A's frame, M = A^T B, t = A^T (C_b - C_a);
//   grid: cell centres s_i = (2i+1)/n - 1 of A, coordinates in B's frame
//        ((t_k + N_k0 x) + N_k1 y) + N_k2 z with N = B^T A;
//   IoU = I / ((va + vb) - I), I = min(va * count / n^3, vb);
//   coverage: X = c + ((R0 x + R1 y) + R2 d), then R_s^T (X - c_s), the depth
//        window and the projection (fx * xs) / zs + cx into the rectangle.
//
// prior_g_kernel: one thread per (history block, query block, batch); the
//   query block's boxes are built once per CTA in shared memory.
// coverage_kernel: a cluster of 4 CTAs per (query block, batch), each
//   taking a quarter of the history slabs; per CTA 128 tokens x 4 slab
//   groups test 512-slab tiles staged through shared memory (the next tile
//   prefetched into registers); a CTA stops once every token with depth has
//   found a slab; the first CTA ORs the token flags of the cluster through
//   distributed shared memory.
#include <cooperative_groups.h>

#include "common.cuh"

namespace cg = cooperative_groups;

namespace bsa {

constexpr int kGeoMaxSlabs = 4;      // slabs per block
constexpr int kGeoMaxGrid = 16;      // grid points per axis
constexpr int kPriorThreads = 128;
constexpr int kCovGroups = 4;
constexpr int kCovThreads = kBlk * kCovGroups;
constexpr int kCovTile = kCovThreads;  // history slabs per shared-memory tile (one per thread)
constexpr int kCovSplit = 4;           // CTAs (one cluster) per query block
constexpr float kSatEps = 1e-6f;

struct Box {
  float c[3];
  float a[3][3];   // a[k] = axis k (world)
  float h[3];
};

struct GeoArgs {
  const float* cams;      // [B, n_cams, 12]
  const int32_t* q_cam;   // [B, n_q, S]
  const float* q_rect;    // [B, n_q, S, 6]
  const int32_t* h_cam;   // [B, n_hist, S]
  const float* h_rect;    // [B, n_hist, S, 6]
  const int32_t* tok_cam; // [B, n_q, 128]
  const float* tok_uvd;   // [B, n_q, 128, 3]
  const int32_t* q_valid; // [n_q] or null
  float* g;               // [B, n_q, n_hist] or null
  float* cov;             // [B, n_q] or null
  int32_t* d_err;
  int n_cams, n_q, n_hist, S, n;
  float fx, fy, cx, cy;
};

__device__ __forceinline__ float fm(float x, float y) { return __fmul_rn(x, y); }
__device__ __forceinline__ float fa(float x, float y) { return __fadd_rn(x, y); }
__device__ __forceinline__ float fs(float x, float y) { return __fsub_rn(x, y); }
__device__ __forceinline__ float fd(float x, float y) { return __fdiv_rn(x, y); }
__device__ __forceinline__ float dot3(const float* x, const float* y) {
  return fa(fa(fm(x[0], y[0]), fm(x[1], y[1])), fm(x[2], y[2]));
}

// A camera index, checked: -1 (absent) stays -1; out of range is reported
// and treated as absent.
__device__ __forceinline__ int check_cam(const GeoArgs& a, int cam) {
  if (cam < -1 || cam >= a.n_cams) {
    report(a.d_err, BSA_DEV_BAD_INDEX);
    return -1;
  }
  return cam;
}

__device__ void slab_box(const float* cam, const GeoArgs& g, const float* rect, Box& b) {
  const float u0 = rect[0], u1 = rect[1], v0 = rect[2], v1 = rect[3], d0 = rect[4], d1 = rect[5];
  const float ax0 = fd(fs(u0, g.cx), g.fx), ax1 = fd(fs(u1, g.cx), g.fx);
  const float ay0 = fd(fs(v0, g.cy), g.fy), ay1 = fd(fs(v1, g.cy), g.fy);
  const float x_lo = fminf(fm(ax0, d0), fm(ax0, d1)), x_hi = fmaxf(fm(ax1, d0), fm(ax1, d1));
  const float y_lo = fminf(fm(ay0, d0), fm(ay0, d1)), y_hi = fmaxf(fm(ay1, d0), fm(ay1, d1));
  const float lc[3] = {fm(fa(x_lo, x_hi), 0.5f), fm(fa(y_lo, y_hi), 0.5f), fm(fa(d0, d1), 0.5f)};
  b.h[0] = fm(fs(x_hi, x_lo), 0.5f);
  b.h[1] = fm(fs(y_hi, y_lo), 0.5f);
  b.h[2] = fm(fs(d1, d0), 0.5f);
#pragma unroll
  for (int i = 0; i < 3; ++i) {
    b.c[i] = fa(cam[9 + i], fa(fa(fm(cam[3 * i + 0], lc[0]), fm(cam[3 * i + 1], lc[1])),
                               fm(cam[3 * i + 2], lc[2])));
#pragma unroll
    for (int k = 0; k < 3; ++k) b.a[k][i] = cam[3 * i + k];   // column k of R
  }
}

__device__ bool sat_separated(const Box& A, const Box& B) {
  float T[3], t[3], M[3][3], aM[3][3];
#pragma unroll
  for (int i = 0; i < 3; ++i) T[i] = fs(B.c[i], A.c[i]);
#pragma unroll
  for (int i = 0; i < 3; ++i) {
    t[i] = dot3(A.a[i], T);
#pragma unroll
    for (int j = 0; j < 3; ++j) {
      M[i][j] = dot3(A.a[i], B.a[j]);
      aM[i][j] = fabsf(M[i][j]);
    }
  }
#pragma unroll
  for (int i = 0; i < 3; ++i) {
    const float rb = fa(fa(fm(B.h[0], aM[i][0]), fm(B.h[1], aM[i][1])), fm(B.h[2], aM[i][2]));
    if (fabsf(t[i]) > fa(A.h[i], rb)) return true;
  }
#pragma unroll
  for (int j = 0; j < 3; ++j) {
    const float ra = fa(fa(fm(A.h[0], aM[0][j]), fm(A.h[1], aM[1][j])), fm(A.h[2], aM[2][j]));
    const float tj = fa(fa(fm(t[0], M[0][j]), fm(t[1], M[1][j])), fm(t[2], M[2][j]));
    if (fabsf(tj) > fa(ra, B.h[j])) return true;
  }
#pragma unroll
  for (int i = 0; i < 3; ++i) {
    const int i1 = (i + 1) % 3, i2 = (i + 2) % 3;
#pragma unroll
    for (int j = 0; j < 3; ++j) {
      const int j1 = (j + 1) % 3, j2 = (j + 2) % 3;
      const float lhs = fabsf(fs(fm(t[i2], M[i1][j]), fm(t[i1], M[i2][j])));
      const float ra = fa(fm(A.h[i1], fa(aM[i2][j], kSatEps)), fm(A.h[i2], fa(aM[i1][j], kSatEps)));
      const float rb = fa(fm(B.h[j1], fa(aM[i][j2], kSatEps)), fm(B.h[j2], fa(aM[i][j1], kSatEps)));
      if (lhs > fa(ra, rb)) return true;
    }
  }
  return false;
}

// Grid IoU of A (the query box) with B; s[] holds the n cell-centre
// coordinates (2i+1)/n - 1.
__device__ float box_iou(const Box& A, const Box& B, const float* s, int n) {
  if (sat_separated(A, B)) return 0.f;
  float D[3], t[3], N[3][3];
#pragma unroll
  for (int i = 0; i < 3; ++i) D[i] = fs(A.c[i], B.c[i]);
#pragma unroll
  for (int k = 0; k < 3; ++k) {
    t[k] = dot3(B.a[k], D);
#pragma unroll
    for (int l = 0; l < 3; ++l) N[k][l] = dot3(B.a[k], A.a[l]);
  }
  int cnt = 0;
  for (int i = 0; i < n; ++i) {
    const float x = fm(s[i], A.h[0]);
    float P[3];
#pragma unroll
    for (int k = 0; k < 3; ++k) P[k] = fa(t[k], fm(N[k][0], x));
    for (int j = 0; j < n; ++j) {
      const float y = fm(s[j], A.h[1]);
      float Q[3];
#pragma unroll
      for (int k = 0; k < 3; ++k) Q[k] = fa(P[k], fm(N[k][1], y));
      for (int l = 0; l < n; ++l) {
        const float z = fm(s[l], A.h[2]);
        const bool in = fabsf(fa(Q[0], fm(N[0][2], z))) <= B.h[0] &&
                        fabsf(fa(Q[1], fm(N[1][2], z))) <= B.h[1] &&
                        fabsf(fa(Q[2], fm(N[2][2], z))) <= B.h[2];
        cnt += in ? 1 : 0;
      }
    }
  }
  const float va = fm(fm(fm(8.f, A.h[0]), A.h[1]), A.h[2]);
  const float vb = fm(fm(fm(8.f, B.h[0]), B.h[1]), B.h[2]);
  const float inter = fminf(fm(va, fd(static_cast<float>(cnt), static_cast<float>(n * n * n))), vb);
  const float uni = fs(fa(va, vb), inter);
  if (!(uni > 0.f)) return 0.f;
  return fd(inter, uni);
}

__global__ void __launch_bounds__(kPriorThreads)
prior_g_kernel(GeoArgs a) {
  __shared__ Box s_q[kGeoMaxSlabs];
  __shared__ int s_qv[kGeoMaxSlabs];
  __shared__ float s_pts[kGeoMaxGrid];
  const int j = blockIdx.y, b = blockIdx.z;
  const int m = blockIdx.x * kPriorThreads + threadIdx.x;
  const float* cams = a.cams + static_cast<long long>(b) * a.n_cams * 12;
  if (threadIdx.x < a.S) {
    const long long qi = (static_cast<long long>(b) * a.n_q + j) * a.S + threadIdx.x;
    const int cam = check_cam(a, a.q_cam[qi]);
    s_qv[threadIdx.x] = cam >= 0;
    if (cam >= 0) slab_box(cams + cam * 12, a, a.q_rect + qi * 6, s_q[threadIdx.x]);
  }
  if (threadIdx.x < a.n)
    s_pts[threadIdx.x] = fs(fd(static_cast<float>(2 * threadIdx.x + 1), static_cast<float>(a.n)), 1.f);
  __syncthreads();
  if (m >= a.n_hist) return;
  float best = 0.f;
  for (int sh = 0; sh < a.S; ++sh) {
    const long long hi = (static_cast<long long>(b) * a.n_hist + m) * a.S + sh;
    const int cam = check_cam(a, a.h_cam[hi]);
    if (cam < 0) continue;
    Box hb;
    slab_box(cams + cam * 12, a, a.h_rect + hi * 6, hb);
    for (int sq = 0; sq < a.S; ++sq) {
      if (!s_qv[sq]) continue;
      const float v = box_iou(s_q[sq], hb, s_pts, a.n);
      best = v > best ? v : best;
    }
  }
  a.g[(static_cast<long long>(b) * a.n_q + j) * a.n_hist + m] = best;
}

struct CovSlab {
  float R[9];
  float c[3];
  float rect[6];
};

// One history slab, fetched through its camera (invalid -> ok = 0).
__device__ __forceinline__ int load_slab(const GeoArgs& a, const float* cams, long long hi, int cam,
                                         CovSlab& out) {
  if (cam < 0) return 0;
  const float* C = cams + cam * 12;
#pragma unroll
  for (int e = 0; e < 9; ++e) out.R[e] = C[e];
#pragma unroll
  for (int e = 0; e < 3; ++e) out.c[e] = C[9 + e];
#pragma unroll
  for (int e = 0; e < 6; ++e) out.rect[e] = a.h_rect[hi * 6 + e];
  return 1;
}

__global__ void __cluster_dims__(kCovSplit, 1, 1) __launch_bounds__(kCovThreads)
coverage_kernel(GeoArgs a) {
  __shared__ CovSlab s_slab[kCovTile];
  __shared__ int s_ok[kCovTile];
  __shared__ int s_hit[kBlk];
  cg::cluster_group cluster = cg::this_cluster();
  const int part = static_cast<int>(cluster.block_rank());
  const int j = blockIdx.x / kCovSplit, b = blockIdx.y;
  const int r = threadIdx.x % kBlk, grp = threadIdx.x / kBlk;
  const float* cams = a.cams + static_cast<long long>(b) * a.n_cams * 12;
  int nv = a.q_valid != nullptr ? a.q_valid[j] : kBlk;
  if (nv < 0 || nv > kBlk) {
    if (part == 0 && threadIdx.x == 0) report(a.d_err, BSA_DEV_BAD_VALID);
    nv = nv < 0 ? 0 : kBlk;
  }
  // This thread's token as a world point (if it has depth).
  const long long ti = (static_cast<long long>(b) * a.n_q + j) * kBlk + r;
  bool live = false;
  float X[3] = {0.f, 0.f, 0.f};
  if (r < nv) {
    const int cam = check_cam(a, a.tok_cam[ti]);
    if (cam >= 0) {
      const float* C = cams + cam * 12;
      const float u = a.tok_uvd[ti * 3 + 0], v = a.tok_uvd[ti * 3 + 1], d = a.tok_uvd[ti * 3 + 2];
      const float x = fm(fd(fs(u, a.cx), a.fx), d);
      const float y = fm(fd(fs(v, a.cy), a.fy), d);
#pragma unroll
      for (int i = 0; i < 3; ++i)
        X[i] = fa(C[9 + i], fa(fa(fm(C[3 * i + 0], x), fm(C[3 * i + 1], y)), fm(C[3 * i + 2], d)));
      live = true;
    }
  }
  if (grp == 0) s_hit[r] = 0;

  // This CTA's share of the history slabs; one slab per thread per tile,
  // the next tile fetched into registers while this one is tested (camera
  // indices one tile further ahead).
  const int n_slabs = a.n_hist * a.S;
  const int per = (n_slabs + kCovSplit - 1) / kCovSplit;
  const int lo = min(n_slabs, part * per), hi = min(n_slabs, lo + per);
  const long long hbase = static_cast<long long>(b) * n_slabs;
  auto cam_at = [&](int si) { return si < hi ? check_cam(a, a.h_cam[hbase + si]) : -1; };
  CovSlab next;
  int next_ok = load_slab(a, cams, hbase + lo + threadIdx.x, cam_at(lo + threadIdx.x), next);
  int cam_ahead = cam_at(lo + kCovTile + threadIdx.x);
  bool hit = false;
  for (int base = lo; base < hi; base += kCovTile) {
    // Stop once no token with depth is left uncovered; also fences the
    // previous tile's readers.
    if (!__syncthreads_or(live && !hit)) break;
    s_slab[threadIdx.x] = next;
    s_ok[threadIdx.x] = next_ok;
    __syncthreads();
    const int nb = base + kCovTile;
    next_ok = load_slab(a, cams, hbase + nb + threadIdx.x, cam_ahead, next);
    cam_ahead = cam_at(nb + kCovTile + threadIdx.x);
    if (live && !hit) {
      const int nt = min(kCovTile, hi - base);
      for (int k = grp; k < nt; k += kCovGroups) {
        if (!s_ok[k]) continue;
        const CovSlab& sl = s_slab[k];
        const float D[3] = {fs(X[0], sl.c[0]), fs(X[1], sl.c[1]), fs(X[2], sl.c[2])};
        const float col2[3] = {sl.R[2], sl.R[5], sl.R[8]};
        const float zs = dot3(col2, D);
        if (!(zs > 0.f && zs >= sl.rect[4] && zs <= sl.rect[5])) continue;
        const float col0[3] = {sl.R[0], sl.R[3], sl.R[6]};
        const float col1[3] = {sl.R[1], sl.R[4], sl.R[7]};
        const float us = fa(fd(fm(a.fx, dot3(col0, D)), zs), a.cx);
        const float vs = fa(fd(fm(a.fy, dot3(col1, D)), zs), a.cy);
        if (us >= sl.rect[0] && us <= sl.rect[1] && vs >= sl.rect[2] && vs <= sl.rect[3]) {
          hit = true;
          break;
        }
      }
    }
  }
  __syncthreads();
  if (hit) s_hit[r] = 1;   // any group; benign same-value writes
  // The cluster's CTAs covered disjoint slab ranges: CTA 0 ORs their token
  // flags through distributed shared memory and writes the fraction.
  cluster.sync();
  if (part == 0 && threadIdx.x < kBlk) {
    int any = s_hit[threadIdx.x];
#pragma unroll
    for (int q = 1; q < kCovSplit; ++q) any |= cluster.map_shared_rank(s_hit, q)[threadIdx.x];
    int cnt = any;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) cnt += __shfl_xor_sync(0xffffffffu, cnt, off);
    if ((threadIdx.x & 31) == 0) s_ok[threadIdx.x / 32] = cnt;   // reuse: per-warp counts
  }
  __syncthreads();
  if (part == 0 && threadIdx.x == 0) {
    const int total = s_ok[0] + s_ok[1] + s_ok[2] + s_ok[3];
    a.cov[static_cast<long long>(b) * a.n_q + j] =
        nv > 0 ? fd(static_cast<float>(total), static_cast<float>(nv)) : 0.f;
  }
  cluster.sync();   // the other CTAs stay resident until their flags were read
}

}  // namespace bsa

using namespace bsa;

extern "C" bsa_status bsa_geometry_prior(const float* cams, int n_cams, float fx, float fy, float cx,
                                         float cy, const int32_t* q_cam, const float* q_rect,
                                         int n_q, const int32_t* h_cam, const float* h_rect,
                                         int n_hist, int slabs_per_block, int grid_n,
                                         const int32_t* tok_cam, const float* tok_uvd,
                                         const int32_t* q_valid, int B, float* g, float* coverage,
                                         int32_t* d_err, void* stream) {
  if (cams == nullptr || (g == nullptr && coverage == nullptr)) return BSA_ERR_INVALID_ARG;
  if (B <= 0 || n_cams <= 0 || n_q <= 0 || n_hist < 0 || slabs_per_block < 1 ||
      slabs_per_block > kGeoMaxSlabs || grid_n < 1 || grid_n > kGeoMaxGrid)
    return BSA_ERR_INVALID_ARG;
  if (!(fx > 0.f) || !(fy > 0.f) || !(cx == cx) || !(cy == cy)) return BSA_ERR_INVALID_ARG;
  if (h_cam == nullptr || h_rect == nullptr) {
    if (n_hist > 0) return BSA_ERR_INVALID_ARG;
  }
  if (g != nullptr && (q_cam == nullptr || q_rect == nullptr)) return BSA_ERR_INVALID_ARG;
  if (coverage != nullptr && (tok_cam == nullptr || tok_uvd == nullptr)) return BSA_ERR_INVALID_ARG;
  if (B > 65535 || n_q > 65535 || static_cast<long long>(n_q) * kCovSplit >= (1LL << 31) ||
      static_cast<long long>(n_hist) * slabs_per_block >= (1LL << 31))
    return BSA_ERR_SHAPE;
  GeoArgs a{};
  a.cams = cams;
  a.q_cam = q_cam;
  a.q_rect = q_rect;
  a.h_cam = h_cam;
  a.h_rect = h_rect;
  a.tok_cam = tok_cam;
  a.tok_uvd = tok_uvd;
  a.q_valid = q_valid;
  a.g = g;
  a.cov = coverage;
  a.d_err = d_err;
  a.n_cams = n_cams;
  a.n_q = n_q;
  a.n_hist = n_hist;
  a.S = slabs_per_block;
  a.n = grid_n;
  a.fx = fx;
  a.fy = fy;
  a.cx = cx;
  a.cy = cy;
  cudaStream_t s = as_stream(stream);
  if (g != nullptr && n_hist > 0) {
    dim3 grid((n_hist + kPriorThreads - 1) / kPriorThreads, n_q, B);
    prior_g_kernel<<<grid, kPriorThreads, 0, s>>>(a);
  }
  if (coverage != nullptr) {
    dim3 grid(n_q * kCovSplit, B);
    coverage_kernel<<<grid, kCovThreads, 0, s>>>(a);
  }
  return launch_status();
}
