"""Oracle: generalised Hilbert ("Gilbert") order of a T x H x W latent grid.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path may import this
module: only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline
leg of ``bench.py`` use it.  It shares no code with the CUDA library.

What it follows
---------------
"Velox: Spatial Memory Makes World Models Efficient", Key Contributions
item 3 and Methodology Steps 5-6: the KV cache is stored in a
"global-aligned Gilbert" order, a generalised Hilbert space-filling curve,
so that neighbouring latent regions are contiguous in memory and a
128-token KV block covers a compact patch of the scene.  The page names the
curve but does not define it, so the construction below is this project's
own generalised Hilbert recursion, fixed once and written out so a reader
can check it by hand:

* A *box* is an entry cell ``o`` plus three signed unit axes ``A`` (the
  travel axis), ``B`` and ``C`` with extents ``a, b, c``.  Its curve starts
  at ``o`` and ends at ``o + (a-1) A``, the corner next to the entry along
  ``A``.  On a grid coloured like a chess board such a unit-step path exists
  only when ``a`` is even or all three extents are odd ("feasible");
  every piece produced below is feasible, which is what makes every step of
  the whole curve a unit step.
* LINE: ``b == c == 1`` - walk along ``A``.
* SPLIT: the box is long in ``A`` (``2a > 3 max(b, c)``): cut ``A`` into an
  even first part and the rest, walk both along ``A``.
* OCTANT: ``a`` and one side are even (>= 4), the other side >= 3 and the
  sides are comparable (``2 short >= long``): cut all three axes and visit the
  eight octants in the reflected-Gray order 000, 010, 011, 001, 101, 111,
  110, 100 (bits = upper half of A, B, C), each octant entered and left at
  the cells that touch its neighbours in that order.  On a 2^k cube this is
  a 3D Hilbert curve: every dyadic sub-cube is one contiguous run.
* UTURN: otherwise turn along the longer side ``L`` (the 2D Hilbert move):
  up ``L`` in the first part of ``A``, across the far part of ``L`` along
  ``A``, back down ``L`` in the last part of ``A``; the short side is
  carried whole.
* Top level: the travel axis is the longest axis of (t, h, w) whose extent
  is even (all axes if none is even); ties go to w, then h, then t.  The
  curve starts at (0, 0, 0).  Every chunk with the same T x H x W uses the
  same order, which is the "global-aligned" property: block n of one chunk
  covers the same latent cells as block n of any other chunk of that shape.

The result is returned as ``perm[i] = p``: raster token ``i = (t*H + h)*W + w``
sits at curve position ``p``.
"""
from __future__ import annotations

import sys
from dataclasses import dataclass
from typing import Iterator, List, Tuple

import numpy as np

Vec = Tuple[int, int, int]


def _add(u: Vec, v: Vec) -> Vec:
    return (u[0] + v[0], u[1] + v[1], u[2] + v[2])


def _mul(k: int, u: Vec) -> Vec:
    return (k * u[0], k * u[1], k * u[2])


def _neg(u: Vec) -> Vec:
    return (-u[0], -u[1], -u[2])


@dataclass(frozen=True)
class Box:
    """A sub-box of the grid with its own traversal frame (see module doc)."""

    o: Vec          # entry cell, in (t, h, w) grid coordinates
    A: Vec          # travel axis (unit, signed)
    B: Vec
    C: Vec
    a: int          # extent along A
    b: int          # extent along B
    c: int          # extent along C


def feasible(a: int, b: int, c: int) -> bool:
    """Whether a unit-step path from o to o+(a-1)A through all a*b*c cells can exist.

    Parity argument on the chequerboard colouring: the two ends differ in
    colour iff a-1 is odd; a path through N cells has ends of different
    colour iff N is even.  A travel extent of 1 only works for one cell.
    """
    if a == 1:
        return b == 1 and c == 1
    return a % 2 == 0 or (a % 2 == 1 and b % 2 == 1 and c % 2 == 1)


def _even_half_down(n: int) -> int:
    """Largest even number <= n/2 (n >= 4)."""
    h = n // 2
    return h - (h & 1)


def _even_part_with_rest(n: int) -> int:
    """An even first part n0 >= 2 with n - n0 >= 1, as close to n/2 as possible
    rounding up (n >= 3)."""
    h = n // 2
    if h % 2 == 0 and h >= 2:
        return h
    return h + 1 if h + 1 < n else h - 1


def _split_a(bx: Box) -> List[Box]:
    a0 = _even_half_down(bx.a)
    return [
        Box(bx.o, bx.A, bx.B, bx.C, a0, bx.b, bx.c),
        Box(_add(bx.o, _mul(a0, bx.A)), bx.A, bx.B, bx.C, bx.a - a0, bx.b, bx.c),
    ]


def _uturn(bx: Box, turn_is_b: bool) -> List[Box]:
    """Turn along side L (B if turn_is_b else C), carrying the other side S whole."""
    if turn_is_b:
        L, l, S, s = bx.B, bx.b, bx.C, bx.c
    else:
        L, l, S, s = bx.C, bx.c, bx.B, bx.b
    a = bx.a
    if l >= 3:
        l0 = _even_part_with_rest(l)
        a0 = a // 2
    else:  # the 2 x 2 square with a unit-thick third side
        assert l == 2 and a == 2 and s == 1, (bx,)
        l0, a0 = 1, 1
    o, A = bx.o, bx.A
    first = Box(o, L, A, S, l0, a0, s)
    middle = Box(_add(o, _mul(l0, L)), A, L, S, a, l - l0, s)
    last_o = _add(_add(o, _mul(a - 1, A)), _mul(l0 - 1, L))
    last = Box(last_o, _neg(L), _neg(A), S, l0, a - a0, s)
    return [first, middle, last]


def _octant(bx: Box, swap: bool) -> List[Box]:
    """Eight-octant Gray-order split; ``swap`` exchanges the roles of B and C so
    that the C role always has an even extent."""
    o, A = bx.o, bx.A
    if swap:
        Bv, b, Cv, c = bx.C, bx.c, bx.B, bx.b
    else:
        Bv, b, Cv, c = bx.B, bx.b, bx.C, bx.c
    a = bx.a
    if (a, b, c) == (2, 2, 2):
        a0 = b0 = c0 = 1
    else:
        a0 = _even_half_down(a)
        c0 = _even_half_down(c)
        b0 = _even_part_with_rest(b)
    a1, b1, c1 = a - a0, b - b0, c - c0

    def at(i: int, j: int, k: int) -> Vec:
        return _add(_add(_add(o, _mul(i, A)), _mul(j, Bv)), _mul(k, Cv))

    nA, nB, nC = _neg(A), _neg(Bv), _neg(Cv)
    return [
        Box(at(0, 0, 0), Bv, A, Cv, b0, a0, c0),                 # octant 000
        Box(at(0, b0, 0), Cv, A, Bv, c0, a0, b1),                # octant 010
        Box(at(0, b0, c0), Cv, A, Bv, c1, a0, b1),               # octant 011
        Box(at(0, b0 - 1, c - 1), A, nB, nC, a0, b0, c1),        # octant 001
        Box(at(a0, b0 - 1, c - 1), nC, A, nB, c1, a1, b0),       # octant 101
        Box(at(a0, b0, c0), A, Bv, Cv, a1, b1, c1),              # octant 111
        Box(at(a - 1, b0, c0 - 1), nC, nA, Bv, c0, a1, b1),      # octant 110
        Box(at(a - 1, b0 - 1, 0), nB, nA, Cv, b0, a1, c0),       # octant 100
    ]


def _octant_roles(a: int, b: int, c: int):
    """Return the B/C role swap flag when the octant split applies, else None."""
    if (a, b, c) == (2, 2, 2):
        return False
    if a % 2 or a < 4:
        return None
    if c % 2 == 0 and c >= 4 and b >= 3:
        return False
    if b % 2 == 0 and b >= 4 and c >= 3:
        return True
    return None


def pieces(bx: Box) -> List[Box]:
    """One level of the recursion: the ordered sub-boxes of a non-line box."""
    a, b, c = bx.a, bx.b, bx.c
    long_side = max(b, c)
    if 2 * a > 3 * long_side and (a >= 4 if a % 2 == 0 else a >= 5):
        return _split_a(bx)
    turn_is_b = b >= c
    short_side = c if turn_is_b else b
    swap = _octant_roles(a, b, c)
    if swap is not None and 2 * short_side >= long_side:
        return _octant(bx, swap)
    return _uturn(bx, turn_is_b)


def walk(bx: Box) -> Iterator[Vec]:
    """Yield the cells of ``bx`` in curve order."""
    if bx.b == 1 and bx.c == 1:
        for i in range(bx.a):
            yield _add(bx.o, _mul(i, bx.A))
        return
    for sub in pieces(bx):
        assert feasible(sub.a, sub.b, sub.c), (bx, sub)
        yield from walk(sub)


def top_box(T: int, H: int, W: int) -> Box:
    """The top-level frame for a T x H x W grid (axes in (t, h, w) order)."""
    dims = {"t": T, "h": H, "w": W}
    unit = {"t": (1, 0, 0), "h": (0, 1, 0), "w": (0, 0, 1)}
    prio = {"w": 0, "h": 1, "t": 2}
    names = sorted(dims, key=lambda n: (-dims[n], prio[n]))
    even = [n for n in names if dims[n] % 2 == 0]
    travel = even[0] if even else names[0]
    rest = [n for n in names if n != travel]
    nb, nc = rest[0], rest[1]
    return Box((0, 0, 0), unit[travel], unit[nb], unit[nc],
               dims[travel], dims[nb], dims[nc])


def gilbert_cells(T: int, H: int, W: int) -> List[Vec]:
    """The (t, h, w) cells of the grid in curve order."""
    if T <= 0 or H <= 0 or W <= 0:
        raise ValueError("grid extents must be positive")
    old = sys.getrecursionlimit()
    sys.setrecursionlimit(max(old, 10000))
    try:
        return list(walk(top_box(T, H, W)))
    finally:
        sys.setrecursionlimit(old)


def gilbert_perm(T: int, H: int, W: int) -> np.ndarray:
    """perm[i] = curve position of raster token i = (t*H + h)*W + w (int32)."""
    cells = gilbert_cells(T, H, W)
    perm = np.full(T * H * W, -1, dtype=np.int64)
    for p, (t, h, w) in enumerate(cells):
        perm[(t * H + h) * W + w] = p
    return perm.astype(np.int32)
