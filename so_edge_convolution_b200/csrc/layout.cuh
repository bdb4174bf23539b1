// layout.cuh -- how the edge-frame features are grouped and laid out.
//
// Edge-frame rows (l, m) with |m| <= min(l, mmax) are grouped by |m| = g:
//   g = 0:  (l, 0)              for l = 0..L          (L+1 rows)
//   g >= 1: (l, +g) for l = g..L, then (l, -g) for l = g..L   (2(L+1-g) rows)
// so that the per-m mixing is one dense product per group:
//   g = 0:  v0 = W0 u0
//   g >= 1: [v+; v-] = [[W1, -W2], [W2, W1]] [u+; u-]
// ("TrimSO(2): Fast and Memory-Efficient Training of Equivariant Interatomic
// Potentials", Abstract: dense matrix multiplications between the
// representation transformations; the +-m pair map is the recombination).
//
// A group's features are the row-major (row-in-group, channel) pairs.  Every
// group's column range is padded with zeros to a multiple of 64 so that a
// product over the padded range equals the product over the true range.
#pragma once

#include "common.cuh"

namespace so2 {

constexpr int MAX_GROUPS = 7;  // mmax <= 6

struct Layout {
  int L, mmax, ci, co, nr, S, T, ng;
  int dsz;                        // floats of Wigner-D per edge (full blocks)
  int rows[MAX_GROUPS];           // rows in group g
  int row0[MAX_GROUPS];           // first edge-frame row of group g
  int Kin[MAX_GROUPS], Kin_pad[MAX_GROUPS], kin_off[MAX_GROUPS];     // input side
  int Kout[MAX_GROUPS], Kout_pad[MAX_GROUPS], kout_off[MAX_GROUPS];  // output side
  int KA, KG;                     // padded widths of the input / output feature rows
  int wr_off[MAX_GROUPS], WR, WK; // stacked weights [WR x WK] (rows out, cols in)
  int wt_off[MAX_GROUPS], WTR, WTK; // transposed stacked weights [WTR x WTK]
};

__host__ __device__ inline int round_up(int a, int b) { return (a + b - 1) / b * b; }

inline Layout make_layout(int L, int mmax, int ci, int co, int nr) {
  Layout y{};
  y.L = L;
  y.mmax = mmax;
  y.ci = ci;
  y.co = co;
  y.nr = nr;
  y.S = (L + 1) * (L + 1);
  y.ng = mmax + 1;
  y.dsz = (L + 1) * (4 * (L + 1) * (L + 1) - 1) / 3;
  int t = 0, ka = 0, kg = 0, wr = 0, wt = 0, wk = 0, wtk = 0;
  for (int g = 0; g < y.ng; ++g) {
    y.rows[g] = (g == 0) ? (L + 1) : 2 * (L + 1 - g);
    y.row0[g] = t;
    t += y.rows[g];
    y.Kin[g] = y.rows[g] * ci;
    y.Kin_pad[g] = round_up(y.Kin[g], 64);
    y.kin_off[g] = ka;
    ka += y.Kin_pad[g];
    y.Kout[g] = y.rows[g] * co;
    y.Kout_pad[g] = round_up(y.Kout[g], 64);
    y.kout_off[g] = kg;
    kg += y.Kout_pad[g];
    y.wr_off[g] = wr;
    wr += y.Kout[g];
    y.wt_off[g] = wt;
    wt += y.Kin[g];
    wk = wk > y.Kin_pad[g] ? wk : y.Kin_pad[g];
    wtk = wtk > y.Kout_pad[g] ? wtk : y.Kout_pad[g];
  }
  y.T = t;
  y.KA = ka;
  y.KG = kg;
  y.WR = wr;
  y.WK = wk;
  y.WTR = wt;
  y.WTK = wtk;
  return y;
}

// Row j of group g -> (l, m).
__host__ __device__ inline void group_row_lm(const Layout &y, int g, int j, int &l, int &m) {
  if (g == 0) {
    l = j;
    m = 0;
    return;
  }
  const int half = y.L + 1 - g;
  if (j < half) {
    l = g + j;
    m = g;
  } else {
    l = g + (j - half);
    m = -g;
  }
}

// (l, m) with |m| <= min(l, mmax) -> (group, row within group).
__host__ __device__ inline void lm_group_row(const Layout &y, int l, int m, int &g, int &j) {
  if (m == 0) {
    g = 0;
    j = l;
    return;
  }
  g = m > 0 ? m : -m;
  const int half = y.L + 1 - g;
  j = (m > 0) ? (l - g) : (half + l - g);
}

// Kept Wigner-D rows.  Row (g, j) of the grouped edge-frame layout, i.e.
// (l, m) with |m| <= mmax, needs the row D^l[m][:] (2l + 1 entries).  The
// kept rows of one edge, concatenated in grouped row order, take
// kept_d_size(L, mmax) floats; kept_d_prefix gives where row (g, j) starts.
// Group 0 holds rows l = 0..L (sum of widths (L+1)^2), group g >= 1 rows
// (l, +g) then (l, -g) for l = g..L (each half (L+1)^2 - g^2).
__host__ __device__ inline int kept_d_prefix(int L, int g, int j) {
  const int S = (L + 1) * (L + 1);
  int base = 0;
  for (int q = 0; q < g; ++q) base += (q == 0) ? S : 2 * (S - q * q);
  if (g == 0) return base + j * j;
  const int half = L + 1 - g;
  if (j < half) {
    const int l = g + j;
    return base + l * l - g * g;
  }
  const int l = g + (j - half);
  return base + (S - g * g) + (l * l - g * g);
}
__host__ __device__ inline int kept_d_size(int L, int mmax) {
  const int S = (L + 1) * (L + 1);
  int t = S;
  for (int g = 1; g <= mmax; ++g) t += 2 * (S - g * g);
  return t;
}

}  // namespace so2
