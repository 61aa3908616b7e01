// gilbert.cuh - generalised Hilbert ("Gilbert") order of a T x H x W grid.
//
// "Velox: Spatial Memory Makes World Models Efficient", Key Contributions 3
// and Methodology Step 6 store the KV cache along a global-aligned Gilbert
// curve.  The page does not define the curve, so this library fixes one
// generalised Hilbert recursion (described below) and locates a curve
// position by descending it: no table and no recursion stack, usable on the
// host and on the device.
//
// A frame is an entry cell o, a travel axis A and two side axes B, C (signed
// unit vectors in (t, h, w)), with extents a, b, c.  The frame's curve runs
// from o to o + (a-1)A.  One level of the descent splits a frame into
// ordered sub-frames:
//   line    b = c = 1: cells o + i*A.
//   split   2a > 3*max(b, c) (and a >= 4 even or a >= 5 odd): A is cut into
//           an even first part (largest even number <= a/2) and the rest.
//   octant  a even >= 4, one side even >= 4 (it plays C), the other >= 3
//           (it plays B), 2*short >= long; or the 2x2x2 frame.  The eight
//           octants are visited in the Gray order 000 010 011 001 101 111 110
//           100 of (A, B, C) upper-half bits; each octant's frame is chosen
//           so that it starts next to where the previous one ended.
//   u-turn  otherwise, along the longer side L (ties: B): up L through the
//           first half of A, across the far part of L along A, back down L
//           through the rest of A; the short side is carried whole.  L's
//           first part is even (>= 2), or 1 for the 2x2 square of a unit
//           thick frame.
// Every sub-frame keeps "a even, or a, b, c all odd", so every step of the
// curve is a unit step.  The top frame's travel axis is the longest even
// extent (all extents if none is even), ties to w, then h, then t; the two
// side axes follow in the same order.
#pragma once

#ifndef __CUDACC__
#define __host__
#define __device__
#endif

namespace bsa {

struct V3 {
  int t, h, w;
};

__host__ __device__ inline V3 v3(int t, int h, int w) { return V3{t, h, w}; }
__host__ __device__ inline V3 vadd(V3 x, V3 y) { return V3{x.t + y.t, x.h + y.h, x.w + y.w}; }
__host__ __device__ inline V3 vscale(int k, V3 x) { return V3{k * x.t, k * x.h, k * x.w}; }
__host__ __device__ inline V3 vneg(V3 x) { return V3{-x.t, -x.h, -x.w}; }

struct GFrame {
  V3 o, A, B, C;
  int a, b, c;
};

enum GRule { kLine = 0, kSplit = 1, kOctant = 2, kOctantSwapped = 3, kUTurnB = 4, kUTurnC = 5 };

__host__ __device__ inline GFrame gframe(V3 o, V3 A, V3 B, V3 C, int a, int b, int c) {
  GFrame f;
  f.o = o; f.A = A; f.B = B; f.C = C; f.a = a; f.b = b; f.c = c;
  return f;
}

// Largest even number not above n/2 (n >= 4).
__host__ __device__ inline int g_even_floor_half(int n) {
  int h = n / 2;
  return h - (h & 1);
}

// Even first part >= 2 leaving at least one, closest to n/2 rounding up (n >= 3).
__host__ __device__ inline int g_even_part(int n) {
  int h = n / 2;
  if ((h & 1) == 0 && h >= 2) return h;
  return (h + 1 < n) ? h + 1 : h - 1;
}

__host__ __device__ inline int g_rule(const GFrame& f) {
  if (f.b == 1 && f.c == 1) return kLine;
  int lng = f.b > f.c ? f.b : f.c;
  bool a_long_enough = (f.a % 2 == 0) ? (f.a >= 4) : (f.a >= 5);
  if (2 * f.a > 3 * lng && a_long_enough) return kSplit;
  bool turn_b = f.b >= f.c;
  int shrt = turn_b ? f.c : f.b;
  if (2 * shrt >= lng) {
    if (f.a == 2 && f.b == 2 && f.c == 2) return kOctant;
    if (f.a % 2 == 0 && f.a >= 4) {
      if (f.c % 2 == 0 && f.c >= 4 && f.b >= 3) return kOctant;
      if (f.b % 2 == 0 && f.b >= 4 && f.c >= 3) return kOctantSwapped;
    }
  }
  return turn_b ? kUTurnB : kUTurnC;
}

__host__ __device__ inline int g_pieces(int rule) {
  switch (rule) {
    case kLine: return 0;
    case kSplit: return 2;
    case kOctant:
    case kOctantSwapped: return 8;
    default: return 3;
  }
}

// Sub-frame k of frame f under `rule`.
__host__ __device__ inline GFrame g_sub(const GFrame& f, int rule, int k) {
  if (rule == kSplit) {
    int a0 = g_even_floor_half(f.a);
    if (k == 0) return gframe(f.o, f.A, f.B, f.C, a0, f.b, f.c);
    return gframe(vadd(f.o, vscale(a0, f.A)), f.A, f.B, f.C, f.a - a0, f.b, f.c);
  }
  if (rule == kUTurnB || rule == kUTurnC) {
    bool tb = (rule == kUTurnB);
    V3 L = tb ? f.B : f.C;
    V3 S = tb ? f.C : f.B;
    int l = tb ? f.b : f.c;
    int s = tb ? f.c : f.b;
    int l0, a0;
    if (l >= 3) {
      l0 = g_even_part(l);
      a0 = f.a / 2;
    } else {  // 2 x 2 square, unit third side
      l0 = 1;
      a0 = 1;
    }
    if (k == 0) return gframe(f.o, L, f.A, S, l0, a0, s);
    if (k == 1) return gframe(vadd(f.o, vscale(l0, L)), f.A, L, S, f.a, l - l0, s);
    V3 o2 = vadd(vadd(f.o, vscale(f.a - 1, f.A)), vscale(l0 - 1, L));
    return gframe(o2, vneg(L), vneg(f.A), S, l0, f.a - a0, s);
  }
  // Octant split.  In the swapped form B and C exchange roles.
  bool sw = (rule == kOctantSwapped);
  V3 A = f.A;
  V3 Bv = sw ? f.C : f.B;
  V3 Cv = sw ? f.B : f.C;
  int a = f.a;
  int b = sw ? f.c : f.b;
  int c = sw ? f.b : f.c;
  int a0, b0, c0;
  if (a == 2 && b == 2 && c == 2) {
    a0 = b0 = c0 = 1;
  } else {
    a0 = g_even_floor_half(a);
    c0 = g_even_floor_half(c);
    b0 = g_even_part(b);
  }
  int a1 = a - a0, b1 = b - b0, c1 = c - c0;
  // Corner helper: o + i*A + j*B + k*C.
  auto at = [&](int i, int j, int kk) {
    return vadd(vadd(vadd(f.o, vscale(i, A)), vscale(j, Bv)), vscale(kk, Cv));
  };
  switch (k) {
    case 0: return gframe(at(0, 0, 0), Bv, A, Cv, b0, a0, c0);
    case 1: return gframe(at(0, b0, 0), Cv, A, Bv, c0, a0, b1);
    case 2: return gframe(at(0, b0, c0), Cv, A, Bv, c1, a0, b1);
    case 3: return gframe(at(0, b0 - 1, c - 1), A, vneg(Bv), vneg(Cv), a0, b0, c1);
    case 4: return gframe(at(a0, b0 - 1, c - 1), vneg(Cv), A, vneg(Bv), c1, a1, b0);
    case 5: return gframe(at(a0, b0, c0), A, Bv, Cv, a1, b1, c1);
    case 6: return gframe(at(a - 1, b0, c0 - 1), vneg(Cv), vneg(A), Bv, c0, a1, b1);
    default: return gframe(at(a - 1, b0 - 1, 0), vneg(Bv), vneg(A), Cv, b0, a1, c0);
  }
}

// Top-level frame of a T x H x W grid.
__host__ __device__ inline GFrame g_top(int T, int H, int W) {
  // Axis order by (extent descending, then w before h before t).
  int ext[3] = {W, H, T};  // index 0 = w, 1 = h, 2 = t (priority order)
  int ord[3] = {0, 1, 2};
  for (int i = 0; i < 3; ++i)
    for (int j = i + 1; j < 3; ++j)
      if (ext[ord[j]] > ext[ord[i]] || (ext[ord[j]] == ext[ord[i]] && ord[j] < ord[i])) {
        int tmp = ord[i]; ord[i] = ord[j]; ord[j] = tmp;
      }
  int travel = -1;
  for (int i = 0; i < 3 && travel < 0; ++i)
    if (ext[ord[i]] % 2 == 0) travel = ord[i];
  if (travel < 0) travel = ord[0];
  int side[2], ns = 0;
  for (int i = 0; i < 3; ++i)
    if (ord[i] != travel) side[ns++] = ord[i];
  V3 unit[3] = {v3(0, 0, 1), v3(0, 1, 0), v3(1, 0, 0)};
  return gframe(v3(0, 0, 0), unit[travel], unit[side[0]], unit[side[1]],
                ext[travel], ext[side[0]], ext[side[1]]);
}

// Cell at curve position p (0 <= p < T*H*W).
__host__ __device__ inline V3 gilbert_cell(int T, int H, int W, int p) {
  GFrame f = g_top(T, H, W);
  for (int depth = 0; depth < 64; ++depth) {
    int rule = g_rule(f);
    if (rule == kLine) return vadd(f.o, vscale(p, f.A));
    int n = g_pieces(rule);
    for (int k = 0; k < n; ++k) {
      GFrame s = g_sub(f, rule, k);
      int vol = s.a * s.b * s.c;
      if (p < vol || k == n - 1) {
        f = s;
        break;
      }
      p -= vol;
    }
  }
  return v3(-1, -1, -1);  // unreachable for valid input
}

// Raster index (t*H + h)*W + w of the cell at curve position p.
__host__ __device__ inline int curve_token(int T, int H, int W, int p) {
  const V3 c = gilbert_cell(T, H, W, p);
  return (c.t * H + c.h) * W + c.w;
}

}  // namespace bsa
