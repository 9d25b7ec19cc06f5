// Compile-time structure of the real-basis Clebsch-Gordan tensors and of the path sets the
// kernels are specialised for.  Shared by the host table generator (host.cpp) and the
// kernels (kernels.cuh) so that both agree on where each coefficient lives in the packed table.
//
// Sparsity pattern (selection rules of the real basis).  With real harmonics whose m > 0
// components vary as cos(m phi) and m < 0 as sin(|m| phi) (e3nn course, "Curriculum at a
// glance", lesson 02b), invariance of the coupling tensor under rotations about z forces
//     |m3| in { |m1| + |m2| , ||m1| - |m2|| },
// and its behaviour under the reflection y -> -y (which flips the sign of every sin-type
// component and multiplies the l1 (x) l2 -> l3 coupling by (-1)^(l1+l2+l3)) forces
//     #{ i : m_i < 0 } = l1 + l2 + l3  (mod 2).
// Entries outside this pattern are exactly zero; entries inside may still vanish for
// particular (l1, l2, l3).  The packed table stores every pattern entry, lexicographic in
// (m1, m2, m3) with m ascending from -l, blocks ordered by (l1, l2, l3) lexicographically
// over all triangle-valid triples with every l <= E3_LMAX.
#pragma once

#if defined(__CUDACC__)
#define E3_HD __host__ __device__
#else
#define E3_HD
#endif

namespace e3b {

constexpr int E3_LMAX = 3;

E3_HD constexpr int iabs(int a) { return a < 0 ? -a : a; }

E3_HD constexpr bool triangle(int l1, int l2, int l3) {
  return iabs(l1 - l2) <= l3 && l3 <= l1 + l2;
}

E3_HD constexpr bool cg_nz(int l1, int l2, int l3, int m1, int m2, int m3) {
  const int a1 = iabs(m1), a2 = iabs(m2), a3 = iabs(m3);
  if (a3 != a1 + a2 && a3 != iabs(a1 - a2)) return false;
  const int nsin = (m1 < 0) + (m2 < 0) + (m3 < 0);
  return (nsin & 1) == ((l1 + l2 + l3) & 1);
}

// Pattern entries of one (l1, l2, l3) block.
E3_HD constexpr int cg_block_nnz(int l1, int l2, int l3) {
  int n = 0;
  for (int m1 = -l1; m1 <= l1; ++m1)
    for (int m2 = -l2; m2 <= l2; ++m2)
      for (int m3 = -l3; m3 <= l3; ++m3) n += cg_nz(l1, l2, l3, m1, m2, m3) ? 1 : 0;
  return n;
}

// Offsets of every block in the packed table, computed once (blocks in lexicographic
// (l1, l2, l3) order over triangle-valid triples; `total` is the table size).
struct CGOffsetTable {
  int off[E3_LMAX + 1][E3_LMAX + 1][E3_LMAX + 1];
  int total;
};
E3_HD constexpr CGOffsetTable make_cg_offsets() {
  CGOffsetTable t{};
  int off = 0;
  for (int a = 0; a <= E3_LMAX; ++a)
    for (int b = 0; b <= E3_LMAX; ++b)
      for (int c = 0; c <= E3_LMAX; ++c) {
        t.off[a][b][c] = off;
        if (triangle(a, b, c)) off += cg_block_nnz(a, b, c);
      }
  t.total = off;
  return t;
}
constexpr CGOffsetTable kCGOffsets = make_cg_offsets();

// Offset of block (l1, l2, l3) in the packed table; (E3_LMAX+1, 0, 0) gives the table size.
E3_HD constexpr int cg_block_offset(int l1, int l2, int l3) {
  return l1 > E3_LMAX ? kCGOffsets.total : kCGOffsets.off[l1][l2][l3];
}

constexpr int CG_TABLE_SIZE = cg_block_offset(E3_LMAX + 1, 0, 0);

// Index of pattern entry (m1, m2, m3) of block (l1, l2, l3) in the packed table (-1 if the
// entry is outside the pattern).
E3_HD constexpr int cg_index(int l1, int l2, int l3, int m1, int m2, int m3) {
  if (!cg_nz(l1, l2, l3, m1, m2, m3)) return -1;
  int n = cg_block_offset(l1, l2, l3);
  for (int a = -l1; a <= l1; ++a)
    for (int b = -l2; b <= l2; ++b)
      for (int c = -l3; c <= l3; ++c) {
        if (a == m1 && b == m2 && c == m3) return n;
        n += cg_nz(l1, l2, l3, a, b, c) ? 1 : 0;
      }
  return -1;
}

// A^p[m1, m3] = sum_m2 C[m1, m2, m3] Y[m2] has a structural zero unless some m2 is in the
// pattern.
E3_HD constexpr bool a_nz(int l1, int l2, int l3, int m1, int m3) {
  for (int m2 = -l2; m2 <= l2; ++m2)
    if (cg_nz(l1, l2, l3, m1, m2, m3)) return true;
  return false;
}

E3_HD constexpr int a_block_nnz(int l1, int l2, int l3) {
  int n = 0;
  for (int m1 = -l1; m1 <= l1; ++m1)
    for (int m3 = -l3; m3 <= l3; ++m3) n += a_nz(l1, l2, l3, m1, m3) ? 1 : 0;
  return n;
}

// ------------------------------------------------------------------------ path sets ---
// The full enumeration for x irreps l = 0..LX (one block each), y irreps l = 0..LY (one
// each) and output degrees <= LO: for l1, for l2, for l3 = |l1-l2| .. min(l1+l2, LO).
// Parities never change the arithmetic (p3 = p1 p2 only labels the output), so a path set
// depends on (LX, LY, LO) alone.

E3_HD constexpr int n_paths(int LX, int LY, int LO) {
  int n = 0;
  for (int l1 = 0; l1 <= LX; ++l1)
    for (int l2 = 0; l2 <= LY; ++l2)
      for (int l3 = iabs(l1 - l2); l3 <= l1 + l2 && l3 <= LO; ++l3) ++n;
  return n;
}

// which = 0: l1, 1: l2, 2: l3 of path p.
E3_HD constexpr int path_l(int LX, int LY, int LO, int p, int which) {
  int n = 0;
  for (int l1 = 0; l1 <= LX; ++l1)
    for (int l2 = 0; l2 <= LY; ++l2)
      for (int l3 = iabs(l1 - l2); l3 <= l1 + l2 && l3 <= LO; ++l3) {
        if (n == p) return which == 0 ? l1 : (which == 1 ? l2 : l3);
        ++n;
      }
  return -1;
}

// Per-channel output offset of path p (uncollapsed: blocks in path order).
E3_HD constexpr int path_out_off(int LX, int LY, int LO, int p) {
  int off = 0;
  for (int q = 0; q < p; ++q) off += 2 * path_l(LX, LY, LO, q, 2) + 1;
  return off;
}

E3_HD constexpr int out_dim_per_channel(int LX, int LY, int LO) {
  return path_out_off(LX, LY, LO, n_paths(LX, LY, LO));
}

// Cost model of the forward inner loop per edge and channel for path p: structural nonzeros
// of A plus the weight scaling on the smaller side.
E3_HD constexpr int path_cost(int LX, int LY, int LO, int p) {
  const int l1 = path_l(LX, LY, LO, p, 0), l2 = path_l(LX, LY, LO, p, 1),
            l3 = path_l(LX, LY, LO, p, 2);
  const int d1 = 2 * l1 + 1, d3 = 2 * l3 + 1;
  return a_block_nnz(l1, l2, l3) + (d1 < d3 ? d1 : d3);
}

// Path groups.  Each thread accumulates 4 channels x the outputs of one group of paths in
// registers, so a group is capped at a number of outputs per channel.  Groups are contiguous runs
// of paths in enumeration order, cut greedily when the next path would exceed the cap or would
// make the group's x components per channel (its degree span l1) exceed 7: a backward thread holds
// x and grad_x of that span in registers, and the merged kernel's register need is its largest
// group's (measured on the l <= 3 set: the span 2..3, 12 components, made the backward spill).
constexpr int GROUP_OUT_CAP = 20;

// Everything the kernels need to know about a path set, computed once per (LX, LY, LO).
constexpr int MAX_PATHS = 64;
struct PathTable {
  int n, ngroups, out_dim;
  int l1[MAX_PATHS], l2[MAX_PATHS], l3[MAX_PATHS];
  int out_off[MAX_PATHS + 1];
  int gbegin[MAX_PATHS + 1];
};
E3_HD constexpr PathTable make_path_table(int LX, int LY, int LO, int cap) {
  PathTable t{};
  for (int l1 = 0; l1 <= LX; ++l1)
    for (int l2 = 0; l2 <= LY; ++l2)
      for (int l3 = iabs(l1 - l2); l3 <= l1 + l2 && l3 <= LO; ++l3) {
        t.l1[t.n] = l1;
        t.l2[t.n] = l2;
        t.l3[t.n] = l3;
        t.out_off[t.n + 1] = t.out_off[t.n] + 2 * l3 + 1;
        ++t.n;
      }
  t.out_dim = t.out_off[t.n];
  int outs = 0;
  t.gbegin[0] = 0;
  t.ngroups = 1;
  int l1_first = 0;  // lowest x degree of the current group
  for (int p = 0; p < t.n; ++p) {
    const int d = 2 * t.l3[p] + 1;
    const int nx = (t.l1[p] + 1) * (t.l1[p] + 1) - l1_first * l1_first;  // x components if p joins
    if (outs > 0 && (outs + d > cap || nx > 7)) {
      t.gbegin[t.ngroups++] = p;
      outs = 0;
    }
    if (outs == 0) l1_first = t.l1[p];
    outs += d;
  }
  t.gbegin[t.ngroups] = t.n;
  return t;
}

}  // namespace e3b
