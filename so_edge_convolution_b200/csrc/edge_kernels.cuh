// edge_kernels.cuh -- CUDA-core stages around the tensor-core mixing.
//
// Graph preparation (integer counting sort), per-edge geometry / Wigner-D /
// radial gate, rotation on gather into the grouped edge-frame operand,
// node-centric inverse rotation on reduction, the weight packing and the
// small per-edge gradient terms.  Stage names follow "TrimSO(2): Fast and
// Memory-Efficient Training of Equivariant Interatomic Potentials"
// (Abstract).
#pragma once

#include "layout.cuh"
#include "wigner.cuh"

namespace so2 {

// ---------------------------------------------------------------------------
// Graph preparation: stable counting sort of edges by one endpoint.
// ---------------------------------------------------------------------------

// counts[key]++ for every edge; keys outside [0, N) raise SO2_ERR_INDEX and
// are counted as node 0 so that every later access stays in bounds.
__global__ void k_count_keys(const int64_t *__restrict__ keys, int64_t E, int64_t N,
                             int *__restrict__ counts, DevStatus *st) {
  for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < E;
       e += (int64_t)gridDim.x * blockDim.x) {
    int64_t k = keys[e];
    if (k < 0 || k >= N) {
      raise_error(st, SO2_ERR_INDEX, static_cast<int>(e & 0x7fffffff));
      k = 0;
    }
    atomicAdd(&counts[k], 1);
  }
}

// Exclusive scan of counts[0..N) into offsets[0..N] with one block.
__global__ void k_scan_offsets(const int *__restrict__ counts, int64_t N, int *__restrict__ offsets) {
  __shared__ int partial[1024];
  const int t = threadIdx.x;
  const int64_t per = (N + blockDim.x - 1) / blockDim.x;
  const int64_t b = t * per, e = (b + per < N) ? b + per : N;
  int s = 0;
  for (int64_t i = b; i < e; ++i) s += counts[i];
  partial[t] = s;
  __syncthreads();
  for (int off = 1; off < (int)blockDim.x; off <<= 1) {
    const int v = (t >= off) ? partial[t - off] : 0;
    __syncthreads();
    partial[t] += v;
    __syncthreads();
  }
  int run = (t == 0) ? 0 : partial[t - 1];
  for (int64_t i = b; i < e; ++i) {
    offsets[i] = run;
    run += counts[i];
  }
  if (t == blockDim.x - 1) offsets[N] = partial[t];
}

__global__ void k_place(const int64_t *__restrict__ keys, int64_t E, int64_t N,
                        const int *__restrict__ offsets, int *__restrict__ cursor,
                        int *__restrict__ perm) {
  for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < E;
       e += (int64_t)gridDim.x * blockDim.x) {
    int64_t k = keys[e];
    if (k < 0 || k >= N) k = 0;
    const int pos = offsets[k] + atomicAdd(&cursor[k], 1);
    perm[pos] = static_cast<int>(e);
  }
}

// Within each key's segment, order the edge ids ascending (insertion sort by
// one thread per segment), which makes the sort stable and deterministic.
__global__ void k_sort_segments(const int *__restrict__ offsets, int64_t N, int *__restrict__ perm) {
  for (int64_t n = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; n < N;
       n += (int64_t)gridDim.x * blockDim.x) {
    const int b = offsets[n], e = offsets[n + 1];
    for (int i = b + 1; i < e; ++i) {
      const int v = perm[i];
      int j = i - 1;
      while (j >= b && perm[j] > v) {
        perm[j + 1] = perm[j];
        --j;
      }
      perm[j + 1] = v;
    }
  }
}

// ---------------------------------------------------------------------------
// Per-edge records for one chunk of sorted positions [e0, e0 + M).
// ---------------------------------------------------------------------------
struct EdgeRec {
  int eid, src, dst, key;  // key = the endpoint this order is sorted by
};

// Geometry record: d, r_hat[3], R[9] (row-major), 3 spare.
constexpr int GEO = 16;

__global__ void k_edge_prep(Layout y, const int *__restrict__ perm, int64_t e0, int M,
                            const int64_t *__restrict__ ei, int64_t E, int64_t N, int key_row,
                            const float *__restrict__ edge_vec, EdgeRec *__restrict__ rec,
                            float *__restrict__ geo, float *__restrict__ D, DevStatus *st) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= M) return;
  const int e = perm[e0 + i];
  int64_t s = ei[e], d = ei[E + e];
  if (s < 0 || s >= N) s = 0;  // already reported by the sort
  if (d < 0 || d >= N) d = 0;
  EdgeRec r;
  r.eid = e;
  r.src = static_cast<int>(s);
  r.dst = static_cast<int>(d);
  r.key = key_row == 0 ? r.src : r.dst;
  rec[i] = r;
  Frame f;
  if (!make_frame(edge_vec[3 * (int64_t)e], edge_vec[3 * (int64_t)e + 1],
                  edge_vec[3 * (int64_t)e + 2], f))
    raise_error(st, SO2_ERR_DEGENERATE, e);
  float *gr = geo + (int64_t)i * GEO;
  gr[0] = f.d;
  gr[1] = f.rh[0];
  gr[2] = f.rh[1];
  gr[3] = f.rh[2];
  for (int k = 0; k < 9; ++k) gr[4 + k] = f.R[k];
  float Dl[dsize(LMAX_SUPPORTED)];
  wigner_blocks(f.R, y.L, Dl);
  float *Dg = D + (int64_t)i * y.dsz;
  for (int k = 0; k < y.dsz; ++k) Dg[k] = Dl[k];
}

__device__ __forceinline__ float rbf_val(float d, int k, const Layout &y, float cutoff) {
  const float sig = cutoff / static_cast<float>(y.nr - 1);
  const float mu = sig * static_cast<float>(k);
  const float t = (d - mu) / sig;
  return __expf(-0.5f * t * t);
}

// g[i][c'] = b[c'] + sum_k w_rad[k][c'] phi_k(d_i)
__global__ void k_edge_gate(Layout y, float cutoff, int M, const float *__restrict__ geo,
                            const float *__restrict__ w_rad, const float *__restrict__ b_rad,
                            float *__restrict__ gate) {
  const int i = blockIdx.x;
  if (i >= M) return;
  const float d = geo[(int64_t)i * GEO];
  for (int c = threadIdx.x; c < y.co; c += blockDim.x) {
    float acc = b_rad[c];
    for (int k = 0; k < y.nr; ++k) acc += w_rad[k * y.co + c] * rbf_val(d, k, y, cutoff);
    gate[(int64_t)i * y.co + c] = acc;
  }
}

// ---------------------------------------------------------------------------
// Rotation on gather: row (l, m) of the edge frame = sum_m' D^l[m][m'] X[node][l, m'],
// optionally times the gate, written in the grouped layout as bf16 (hi, lo).
// One block per edge, threads over channels.
// ---------------------------------------------------------------------------
template <typename TX>
__global__ void k_rotate_gather(Layout y, int M, const EdgeRec *__restrict__ rec,
                                const float *__restrict__ D, const TX *__restrict__ X, int side,
                                int use_src, const float *__restrict__ gate,
                                __nv_bfloat16 *__restrict__ out_hi, __nv_bfloat16 *__restrict__ out_lo,
                                int ld) {
  const int i = blockIdx.x;
  if (i >= M) return;
  const int C = side ? y.co : y.ci;
  const int *col_off = side ? y.kout_off : y.kin_off;
  const int *col_pad = side ? y.Kout_pad : y.Kin_pad;
  const EdgeRec r = rec[i];
  const int node = use_src ? r.src : r.dst;
  const float *De = D + (int64_t)i * y.dsz;
  const TX *Xn = X + (int64_t)node * y.S * C;
  __nv_bfloat16 *oh = out_hi + (int64_t)i * ld;
  __nv_bfloat16 *ol = out_lo ? out_lo + (int64_t)i * ld : nullptr;
  for (int g = 0; g < y.ng; ++g) {
    const int base = col_off[g];
    const int width = y.rows[g] * C;
    for (int j = 0; j < y.rows[g]; ++j) {
      int l, m;
      group_row_lm(y, g, j, l, m);
      const float *Drow = De + dblock_off(l) + (m + l) * (2 * l + 1);
      for (int c = threadIdx.x; c < C; c += blockDim.x) {
        float acc = 0.f;
        for (int mp = -l; mp <= l; ++mp)
          acc += Drow[mp + l] * to_f32(Xn[(l * l + l + mp) * C + c]);
        if (gate) acc *= gate[(int64_t)i * C + c];
        __nv_bfloat16 h, lo;
        split_bf16(acc, h, lo);
        oh[base + j * C + c] = h;
        if (ol) ol[base + j * C + c] = lo;
      }
    }
    for (int k = width + threadIdx.x; k < col_pad[g]; k += blockDim.x) {
      oh[base + k] = __float2bfloat16_rn(0.f);
      if (ol) ol[base + k] = __float2bfloat16_rn(0.f);
    }
  }
}

// [M x K] bf16 row-major -> [K x Mp] (Mp = ld of the output), columns >= M zero.
__global__ void k_transpose_bf16(const __nv_bfloat16 *__restrict__ in, int M, int K, int ld_in,
                                 __nv_bfloat16 *__restrict__ out, int Mp) {
  __shared__ __nv_bfloat16 tile[32][33];
  const int k0 = blockIdx.x * 32, m0 = blockIdx.y * 32;
  for (int r = threadIdx.y; r < 32; r += blockDim.y) {
    const int m = m0 + r, k = k0 + threadIdx.x;
    tile[r][threadIdx.x] = (m < M && k < K) ? in[(int64_t)m * ld_in + k] : __float2bfloat16_rn(0.f);
  }
  __syncthreads();
  for (int r = threadIdx.y; r < 32; r += blockDim.y) {
    const int k = k0 + r, m = m0 + threadIdx.x;
    if (k < K && m < Mp) out[(int64_t)k * Mp + m] = tile[threadIdx.x][r];
  }
}

// ---------------------------------------------------------------------------
// Inverse rotation on reduction, node-centric.  For every node whose sorted
// segment meets this chunk, out[n][(l,m')][c] += sum over its chunk edges of
// sum_m D^l[m][m'] * F[i][row(l,m)][c] (* gate).  One block per node, threads
// over channels; the chunks run in stream order, so every output element is
// updated by one thread at a time and the sum order is fixed.
// ---------------------------------------------------------------------------
__global__ void k_scatter_nodes(Layout y, int64_t e0, int M, const EdgeRec *__restrict__ rec,
                                const int *__restrict__ offsets, const float *__restrict__ D,
                                const float *__restrict__ F, int ldf, int side,
                                const float *__restrict__ gate, float *__restrict__ out) {
  if (M <= 0) return;
  const int C = side ? y.co : y.ci;
  const int *col_off = side ? y.kout_off : y.kin_off;
  const int n_first = rec[0].key, n_last = rec[M - 1].key;
  float acc[(LMAX_SUPPORTED + 1) * (LMAX_SUPPORTED + 1)];
  for (int n = n_first + blockIdx.x; n <= n_last; n += gridDim.x) {
    int b = offsets[n] - static_cast<int>(e0), e = offsets[n + 1] - static_cast<int>(e0);
    b = b < 0 ? 0 : b;
    e = e > M ? M : e;
    if (b >= e) continue;
    for (int c = threadIdx.x; c < C; c += blockDim.x) {
      for (int s = 0; s < y.S; ++s) acc[s] = 0.f;
      for (int i = b; i < e; ++i) {
        const float *De = D + (int64_t)i * y.dsz;
        const float *Fi = F + (int64_t)i * ldf;
        const float gv = gate ? gate[(int64_t)i * C + c] : 1.f;
        for (int l = 0; l <= y.L; ++l) {
          const int mm = l < y.mmax ? l : y.mmax;
          const float *Dl = De + dblock_off(l);
          for (int m = -mm; m <= mm; ++m) {
            int g, j;
            lm_group_row(y, l, m, g, j);
            const float v = gv * Fi[col_off[g] + j * C + c];
            const float *Drow = Dl + (m + l) * (2 * l + 1);
            for (int mp = -l; mp <= l; ++mp) acc[l * l + l + mp] += Drow[mp + l] * v;
          }
        }
      }
      float *o = out + (int64_t)n * y.S * C + c;
      for (int s = 0; s < y.S; ++s) o[s * C] += acc[s];
    }
  }
}

// ---------------------------------------------------------------------------
// Weights: packed blocks -> stacked per-group matrices (bf16 hi/lo) and their
// transposes; zero padding outside each group's true extent.
// ---------------------------------------------------------------------------
template <typename TW>
__device__ __forceinline__ float stacked_w(const Layout &y, const TW *w, const long long *blk_off,
                                           int g, int n, int k) {
  // value of the stacked group-g matrix at (out row n, in col k)
  if (g == 0) return to_f32(w[blk_off[0] + (long long)n * y.Kin[0] + k]);
  const int ho = (y.L + 1 - g) * y.co, hi = (y.L + 1 - g) * y.ci;
  const int rb = n >= ho, cb = k >= hi;
  const int nn = n - rb * ho, kk = k - cb * hi;
  const long long w1 = blk_off[2 * g - 1], w2 = blk_off[2 * g];
  const long long idx = (long long)nn * hi + kk;
  if (rb == cb) return to_f32(w[w1 + idx]);
  const float v2 = to_f32(w[w2 + idx]);
  return (rb == 0) ? -v2 : v2;  // [[W1, -W2], [W2, W1]]
}

struct BlockOffsets {
  long long off[2 * MAX_GROUPS];
};

template <typename TW>
__global__ void k_pack_weights(Layout y, BlockOffsets bo, const TW *__restrict__ w,
                               __nv_bfloat16 *__restrict__ wst_hi, __nv_bfloat16 *__restrict__ wst_lo,
                               __nv_bfloat16 *__restrict__ wtr_hi, __nv_bfloat16 *__restrict__ wtr_lo) {
  const int g = blockIdx.y;
  if (g >= y.ng) return;
  const int64_t total = (int64_t)y.Kout[g] * y.Kin[g];
  for (int64_t t = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; t < total;
       t += (int64_t)gridDim.x * blockDim.x) {
    const int n = static_cast<int>(t / y.Kin[g]), k = static_cast<int>(t % y.Kin[g]);
    const float v = stacked_w(y, w, bo.off, g, n, k);
    __nv_bfloat16 h, l;
    split_bf16(v, h, l);
    const int64_t a = (int64_t)(y.wr_off[g] + n) * y.WK + k;
    const int64_t b = (int64_t)(y.wt_off[g] + k) * y.WTK + n;
    wst_hi[a] = h;
    wtr_hi[b] = h;
    if (wst_lo) {
      wst_lo[a] = l;
      wtr_lo[b] = l;
    }
  }
}

// d(stacked) -> packed gradient blocks: W0 directly; for g >= 1
// grad W1 = A + D, grad W2 = C - B where d(stacked) = [[A, B], [C, D]].
__global__ void k_unstack_grad(Layout y, BlockOffsets bo, const float *__restrict__ dws,
                               float *__restrict__ grad_w) {
  const int g = blockIdx.y;
  if (g >= y.ng) return;
  if (g == 0) {
    const int64_t total = (int64_t)y.Kout[0] * y.Kin[0];
    for (int64_t t = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; t < total;
         t += (int64_t)gridDim.x * blockDim.x) {
      const int n = static_cast<int>(t / y.Kin[0]), k = static_cast<int>(t % y.Kin[0]);
      grad_w[bo.off[0] + t] = dws[(int64_t)(y.wr_off[0] + n) * y.WK + k];
    }
    return;
  }
  const int ho = (y.L + 1 - g) * y.co, hi = (y.L + 1 - g) * y.ci;
  const int64_t total = (int64_t)ho * hi;
  for (int64_t t = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; t < total;
       t += (int64_t)gridDim.x * blockDim.x) {
    const int n = static_cast<int>(t / hi), k = static_cast<int>(t % hi);
    const float *r0 = dws + (int64_t)(y.wr_off[g] + n) * y.WK;
    const float *r1 = dws + (int64_t)(y.wr_off[g] + ho + n) * y.WK;
    grad_w[bo.off[2 * g - 1] + t] = r0[k] + r1[hi + k];
    grad_w[bo.off[2 * g] + t] = r1[k] - r0[hi + k];
  }
}

// ---------------------------------------------------------------------------
// Backward per-edge terms.  For one edge (block) and all channels:
//   Gy~ = D G[dst] on rows |m| <= mmax+1,   a = D x[src] on the same rows,
//   Gg[c'] = sum_{kept rows} Gy~ * v,
//   h_k   = sum_{kept rows, c'} (g v) (J_k Gy~) + sum_{kept rows, c} Ga (J_k a),
// where v (mixing output) and Ga (gradient of the rotated input) come from
// the two products.  h_x, h_y give the frame part of dL/dr.
// ---------------------------------------------------------------------------
template <typename TX>
__global__ void k_edge_terms(Layout y, int M, const EdgeRec *__restrict__ rec,
                             const float *__restrict__ D, const float *__restrict__ gate,
                             const float *__restrict__ G, const TX *__restrict__ X,
                             const float *__restrict__ V, const float *__restrict__ Ga,
                             float *__restrict__ Gg, float *__restrict__ h) {
  const int i = blockIdx.x;
  if (i >= M) return;
  const int *kout_off = y.kout_off;
  const int *kin_off = y.kin_off;
  const EdgeRec r = rec[i];
  const float *De = D + (int64_t)i * y.dsz;
  float hx = 0.f, hy = 0.f;
  const int wide = y.mmax + 1;
  float buf[2 * LMAX_SUPPORTED + 1];
  // output side
  for (int c = threadIdx.x; c < y.co; c += blockDim.x) {
    const float gv = gate[(int64_t)i * y.co + c];
    const float *Gn = G + (int64_t)r.dst * y.S * y.co;
    const float *Vi = V + (int64_t)i * y.KG;
    float gg = 0.f;
    for (int l = 0; l <= y.L; ++l) {
      const int mw = l < wide ? l : wide;
      const float *Dl = De + dblock_off(l);
      for (int m = -mw; m <= mw; ++m) {
        float acc = 0.f;
        for (int mp = -l; mp <= l; ++mp) acc += Dl[(m + l) * (2 * l + 1) + mp + l] * Gn[(l * l + l + mp) * y.co + c];
        buf[m + mw] = acc;
      }
      const int mm = l < y.mmax ? l : y.mmax;
      for (int m = -mm; m <= mm; ++m) {
        int g, j;
        lm_group_row(y, l, m, g, j);
        const float v = Vi[kout_off[g] + j * y.co + c];
        gg += buf[m + mw] * v;
        float jx, jy;
        gen_xy(l, m, [&](int q) { return buf[q + mw]; }, jx, jy);
        hx += gv * v * jx;
        hy += gv * v * jy;
      }
    }
    Gg[(int64_t)i * y.co + c] = gg;
  }
  // input side
  for (int c = threadIdx.x; c < y.ci; c += blockDim.x) {
    const TX *Xn = X + (int64_t)r.src * y.S * y.ci;
    const float *Gai = Ga + (int64_t)i * y.KA;
    for (int l = 0; l <= y.L; ++l) {
      const int mw = l < wide ? l : wide;
      const float *Dl = De + dblock_off(l);
      for (int m = -mw; m <= mw; ++m) {
        float acc = 0.f;
        for (int mp = -l; mp <= l; ++mp) acc += Dl[(m + l) * (2 * l + 1) + mp + l] * to_f32(Xn[(l * l + l + mp) * y.ci + c]);
        buf[m + mw] = acc;
      }
      const int mm = l < y.mmax ? l : y.mmax;
      for (int m = -mm; m <= mm; ++m) {
        int g, j;
        lm_group_row(y, l, m, g, j);
        const float ga = Gai[kin_off[g] + j * y.ci + c];
        float jx, jy;
        gen_xy(l, m, [&](int q) { return buf[q + mw]; }, jx, jy);
        hx += ga * jx;
        hy += ga * jy;
      }
    }
  }
  // block reduction of (hx, hy) in a fixed order
  __shared__ float red[2][32];
  for (int o = 16; o > 0; o >>= 1) {
    hx += __shfl_xor_sync(0xffffffffu, hx, o);
    hy += __shfl_xor_sync(0xffffffffu, hy, o);
  }
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) {
    red[0][w] = hx;
    red[1][w] = hy;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    float sx = 0.f, sy = 0.f;
    for (int k = 0; k < (int)(blockDim.x >> 5); ++k) {
      sx += red[0][k];
      sy += red[1][k];
    }
    h[2 * (int64_t)i] = sx;
    h[2 * (int64_t)i + 1] = sy;
  }
}

// grad_r[eid] = R^T (-h_y, h_x, 0) / d + (sum_c' Gg[c'] sum_k W_rad[k][c'] phi'_k(d)) r_hat.
// One warp per edge.
__global__ void k_edge_final(Layout y, float cutoff, int M, const EdgeRec *__restrict__ rec,
                             const float *__restrict__ geo, const float *__restrict__ Gg,
                             const float *__restrict__ h, const float *__restrict__ w_rad,
                             float *__restrict__ grad_r) {
  const int i = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (i >= M) return;
  const float *gr = geo + (int64_t)i * GEO;
  const float d = gr[0];
  const float sig = cutoff / static_cast<float>(y.nr - 1);
  float dd = 0.f;
  for (int c = lane; c < y.co; c += 32) {
    float dg = 0.f;
    for (int k = 0; k < y.nr; ++k) {
      const float mu = sig * static_cast<float>(k);
      const float t = (d - mu) / sig;
      dg += w_rad[k * y.co + c] * (-t / sig) * __expf(-0.5f * t * t);
    }
    dd += Gg[(int64_t)i * y.co + c] * dg;
  }
  for (int o = 16; o > 0; o >>= 1) dd += __shfl_xor_sync(0xffffffffu, dd, o);
  if (lane == 0) {
    const float hx = h[2 * (int64_t)i], hy = h[2 * (int64_t)i + 1];
    const float inv = d > 0.f ? 1.f / d : 0.f;
    const float *R = gr + 4;
    const int e = rec[i].eid;
    for (int a = 0; a < 3; ++a)
      grad_r[3 * (int64_t)e + a] = (R[0 * 3 + a] * (-hy) + R[1 * 3 + a] * hx) * inv + dd * gr[1 + a];
  }
}

// grad_w_rad[k][c'] += sum_i phi_k(d_i) Gg[i][c'];  grad_b[c'] += sum_i Gg[i][c'].
// Block (32 channels, 8 edge lanes); fixed-order reduction.
__global__ void k_rad_grad(Layout y, float cutoff, int M, const float *__restrict__ geo,
                           const float *__restrict__ Gg, float *__restrict__ grad_w_rad,
                           float *__restrict__ grad_b) {
  const int c = blockIdx.x * 32 + threadIdx.x;
  const int k = blockIdx.y;  // 0..nr-1 for w_rad, nr for the bias
  __shared__ float red[8][32];
  float acc = 0.f;
  if (c < y.co) {
    for (int i = threadIdx.y; i < M; i += blockDim.y) {
      const float phi = (k < y.nr) ? rbf_val(geo[(int64_t)i * GEO], k, y, cutoff) : 1.f;
      acc += phi * Gg[(int64_t)i * y.co + c];
    }
  }
  red[threadIdx.y][threadIdx.x] = acc;
  __syncthreads();
  if (threadIdx.y == 0 && c < y.co) {
    float s = 0.f;
    for (int t = 0; t < (int)blockDim.y; ++t) s += red[t][threadIdx.x];
    if (k < y.nr) {
      if (grad_w_rad) grad_w_rad[k * y.co + c] += s;
    } else if (grad_b) {
      grad_b[c] += s;
    }
  }
}

// Frames and full Wigner-D for inspection.
__global__ void k_frames(int lmax, int64_t E, const float *__restrict__ edge_vec, float *__restrict__ Rout,
                         float *__restrict__ Dout) {
  const int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
  if (e >= E) return;
  Frame f;
  make_frame(edge_vec[3 * e], edge_vec[3 * e + 1], edge_vec[3 * e + 2], f);
  if (Rout)
    for (int k = 0; k < 9; ++k) Rout[9 * e + k] = f.R[k];
  if (Dout) {
    float Dl[dsize(LMAX_SUPPORTED)];
    wigner_blocks(f.R, lmax, Dl);
    const int n = dsize(lmax);
    for (int k = 0; k < n; ++k) Dout[e * n + k] = Dl[k];
  }
}

}  // namespace so2
