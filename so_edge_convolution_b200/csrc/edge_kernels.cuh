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

// One thread per edge; the Wigner-D recursion runs in this thread's slice of
// dynamic shared memory (blockDim.x * dsz floats) and is then copied out
// with coalesced stores.
__global__ void k_edge_prep(Layout y, const int *__restrict__ perm, int64_t e0, int M,
                            const int64_t *__restrict__ ei, int64_t E, int64_t N, int key_row,
                            const float *__restrict__ edge_vec, EdgeRec *__restrict__ rec,
                            float *__restrict__ geo, float *__restrict__ D, DevStatus *st) {
  extern __shared__ float sD[];
  const int i0 = blockIdx.x * blockDim.x;
  const int i = i0 + threadIdx.x;
  float *mine = sD + threadIdx.x * y.dsz;
  if (i < M) {
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
    wigner_blocks(f.R, y.L, mine);
  }
  __syncthreads();
  const int n_here = (M - i0) < (int)blockDim.x ? (M - i0) : (int)blockDim.x;
  const int total = n_here * y.dsz;
  float *dst = D + (int64_t)i0 * y.dsz;
  for (int k = threadIdx.x; k < total; k += blockDim.x) dst[k] = sD[k];
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
// One warp per edge, lanes over channel pairs; |m| <= MM is unrolled at
// compile time so the per-row accumulators stay in registers.
// ---------------------------------------------------------------------------
__device__ __forceinline__ float2 load2(const float *p) { return *reinterpret_cast<const float2 *>(p); }
__device__ __forceinline__ float2 load2(const __nv_bfloat16 *p) {
  return __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(p));
}
__device__ __forceinline__ void store_split2(__nv_bfloat16 *hi, __nv_bfloat16 *lo, float a, float b) {
  __nv_bfloat16 h0, l0, h1, l1;
  split_bf16(a, h0, l0);
  split_bf16(b, h1, l1);
  *reinterpret_cast<__nv_bfloat162 *>(hi) = __halves2bfloat162(h0, h1);
  if (lo) *reinterpret_cast<__nv_bfloat162 *>(lo) = __halves2bfloat162(l0, l1);
}

// Per-channel coefficient: 0 (absent), 1, or an [edge][channel] array.
struct Coef {
  const float *p;
  int mode;  // 0 zero, 1 one, 2 array
};
__device__ __forceinline__ float2 coef2(const Coef &k, int64_t i, int C, int c) {
  if (k.mode == 0) return make_float2(0.f, 0.f);
  if (k.mode == 1) return make_float2(1.f, 1.f);
  return load2(k.p + i * C + c);
}

// out[row (l,m)] = A * b[m] + B * (Omega b)[m],  b = D^l X[node][l, :],
// Omega = w_x J_x + w_y J_y with (w_x, w_y) = omega[i][0..1].  With B absent
// this is plain rotation on gather (A = 1) or gated rotation (A = g).
template <typename TX, int MM>
__global__ void k_rotate_gather(Layout y, int M, const EdgeRec *__restrict__ rec,
                                const float *__restrict__ D, const TX *__restrict__ X, int side,
                                int use_src, Coef A, Coef B, const float *__restrict__ omega,
                                __nv_bfloat16 *__restrict__ out_hi, __nv_bfloat16 *__restrict__ out_lo,
                                int ld) {
  constexpr int W = MM + 1;
  const int C = side ? y.co : y.ci;
  const int *col_off = side ? y.kout_off : y.kin_off;
  const int *col_pad = side ? y.Kout_pad : y.Kin_pad;
  const int lane = threadIdx.x & 31, wpb = blockDim.x >> 5;
  const bool wide = B.mode != 0;
  for (int i = blockIdx.x * wpb + (threadIdx.x >> 5); i < M; i += gridDim.x * wpb) {
    const EdgeRec r = rec[i];
    const int node = use_src ? r.src : r.dst;
    const float *De = D + (int64_t)i * y.dsz;
    const TX *Xn = X + (int64_t)node * y.S * C;
    __nv_bfloat16 *oh = out_hi + (int64_t)i * ld;
    __nv_bfloat16 *ol = out_lo ? out_lo + (int64_t)i * ld : nullptr;
    float wx = 0.f, wy = 0.f;
    if (wide) {
      wx = omega[4 * (int64_t)i];
      wy = omega[4 * (int64_t)i + 1];
    }
    for (int c = 2 * lane; c < C; c += 64) {
      const float2 ca = coef2(A, i, C, c), cb = coef2(B, i, C, c);
      for (int l = 0; l <= y.L; ++l) {
        float a0[2 * W + 1], a1[2 * W + 1];
#pragma unroll
        for (int k = 0; k < 2 * W + 1; ++k) a0[k] = a1[k] = 0.f;
        const float *Dl = De + dblock_off(l);
        const int w = 2 * l + 1;
        const int top = wide ? W : MM;
        for (int mp = -l; mp <= l; ++mp) {
          const float2 xv = load2(Xn + (l * l + l + mp) * C + c);
#pragma unroll
          for (int m = -W; m <= W; ++m) {
            if (m < -l || m > l || m < -top || m > top) continue;
            const float dv = Dl[(m + l) * w + mp + l];
            a0[m + W] += dv * xv.x;
            a1[m + W] += dv * xv.y;
          }
        }
#pragma unroll
        for (int m = -MM; m <= MM; ++m) {
          if (m < -l || m > l) continue;
          int g, j;
          lm_group_row(y, l, m, g, j);
          const int col = col_off[g] + j * C + c;
          float o0 = ca.x * a0[m + W], o1 = ca.y * a1[m + W];
          if (wide) {
            float jx0, jy0, jx1, jy1;
            gen_xy(l, m, [&](int q) { return a0[q + W]; }, jx0, jy0);
            gen_xy(l, m, [&](int q) { return a1[q + W]; }, jx1, jy1);
            o0 += cb.x * (wx * jx0 + wy * jy0);
            o1 += cb.y * (wx * jx1 + wy * jy1);
          }
          store_split2(oh + col, ol ? ol + col : nullptr, o0, o1);
        }
      }
    }
    for (int g = 0; g < y.ng; ++g) {
      const int width = y.rows[g] * C;
      for (int k = width + 2 * lane; k < col_pad[g]; k += 64)
        store_split2(oh + col_off[g] + k, ol ? ol + col_off[g] + k : nullptr, 0.f, 0.f);
    }
  }
}

// [M x K] bf16 row-major -> [K x Mp] (row stride ld_out), columns in [M, Mp) zero.
// 64 x 64 tiles through shared memory, 32-bit accesses.
__global__ void k_transpose_bf16(const __nv_bfloat16 *__restrict__ in, int M, int K, int ld_in,
                                 __nv_bfloat16 *__restrict__ out, int Mp, int ld_out) {
  __shared__ __nv_bfloat16 tile[64][66];
  const int k0 = blockIdx.x * 64, m0 = blockIdx.y * 64;
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;  // 32 x 8
  for (int r = ty; r < 64; r += 8) {
    const int m = m0 + r, k = k0 + 2 * tx;
    __nv_bfloat162 v = __floats2bfloat162_rn(0.f, 0.f);
    if (m < M && k < K) v = *reinterpret_cast<const __nv_bfloat162 *>(in + (int64_t)m * ld_in + k);
    tile[r][2 * tx] = v.x;
    tile[r][2 * tx + 1] = v.y;
  }
  __syncthreads();
  for (int r = ty; r < 64; r += 8) {
    const int k = k0 + r, m = m0 + 2 * tx;
    if (k < K && m < Mp) {
      __nv_bfloat162 v;
      v.x = tile[2 * tx][r];
      v.y = tile[2 * tx + 1][r];
      *reinterpret_cast<__nv_bfloat162 *>(out + (int64_t)k * ld_out + m) = v;
    }
  }
}

// Up to three per-edge row sets F_u (grouped layout, row stride ld[u]) and
// their per-channel coefficients: the reduced rows are
//   Z = sum_u A_u F_u - Omega (sum_{u<2} B_u F_u)      (|m| up to mmax + 1)
struct ScatterTerms {
  const float *F[3];
  int ld[3];
  Coef A[3];
  Coef B[2];
};

// ---------------------------------------------------------------------------
// Inverse rotation on reduction, node-centric.  For every node whose sorted
// segment meets this chunk, out[n][(l,m')][c] += sum over its chunk edges of
// sum_m D^l[m][m'] Z[i][(l,m)][c], Z as described by ScatterTerms.  One block per node,
// threads over channel pairs, the node's sums in shared memory; the chunks
// run in stream order, so every output element is updated by one thread at
// a time and the sum order is fixed.
// ---------------------------------------------------------------------------
template <int MM>
__global__ void k_scatter_nodes(Layout y, int64_t e0, int M, const EdgeRec *__restrict__ rec,
                                const int *__restrict__ offsets, const float *__restrict__ D,
                                ScatterTerms t, int side, const float *__restrict__ omega,
                                float *__restrict__ out) {
  extern __shared__ float acc[];  // [S][C]
  if (M <= 0) return;
  constexpr int W = MM + 1;
  const int C = side ? y.co : y.ci;
  const int *col_off = side ? y.kout_off : y.kin_off;
  const bool wide = t.B[0].mode != 0 || t.B[1].mode != 0;
  const int n_first = rec[0].key, n_last = rec[M - 1].key;
  for (int n = n_first + blockIdx.x; n <= n_last; n += gridDim.x) {
    int b = offsets[n] - static_cast<int>(e0), e = offsets[n + 1] - static_cast<int>(e0);
    b = b < 0 ? 0 : b;
    e = e > M ? M : e;
    if (b >= e) continue;
    for (int k = threadIdx.x; k < y.S * C; k += blockDim.x) acc[k] = 0.f;
    __syncthreads();
    for (int c = 2 * threadIdx.x; c < C; c += 2 * blockDim.x) {
      for (int i = b; i < e; ++i) {
        const float *De = D + (int64_t)i * y.dsz;
        float2 ka[3], kb[2];
#pragma unroll
        for (int u = 0; u < 3; ++u) ka[u] = t.F[u] ? coef2(t.A[u], i, C, c) : make_float2(0.f, 0.f);
#pragma unroll
        for (int u = 0; u < 2; ++u) kb[u] = t.F[u] ? coef2(t.B[u], i, C, c) : make_float2(0.f, 0.f);
        float wx = 0.f, wy = 0.f;
        if (wide) {
          wx = omega[4 * (int64_t)i];
          wy = omega[4 * (int64_t)i + 1];
        }
        for (int l = 0; l <= y.L; ++l) {
          float z0[2 * W + 1], z1[2 * W + 1], q0[2 * W + 1], q1[2 * W + 1];
#pragma unroll
          for (int m = -W; m <= W; ++m) {
            z0[m + W] = z1[m + W] = q0[m + W] = q1[m + W] = 0.f;
            if (m < -l || m > l || m < -MM || m > MM) continue;
            int g, j;
            lm_group_row(y, l, m, g, j);
#pragma unroll
            for (int u = 0; u < 3; ++u) {
              if (!t.F[u]) continue;
              const float2 f = load2(t.F[u] + (int64_t)i * t.ld[u] + col_off[g] + j * C + c);
              z0[m + W] += ka[u].x * f.x;
              z1[m + W] += ka[u].y * f.y;
              if (u < 2) {
                q0[m + W] += kb[u].x * f.x;
                q1[m + W] += kb[u].y * f.y;
              }
            }
          }
          const int top = wide ? W : MM;
          if (wide) {
            float r0[2 * W + 1], r1[2 * W + 1];
#pragma unroll
            for (int m = -W; m <= W; ++m) {
              r0[m + W] = r1[m + W] = 0.f;
              if (m < -l || m > l) continue;
              float jx0, jy0, jx1, jy1;
              gen_xy(l, m, [&](int qq) { return (qq < -MM || qq > MM) ? 0.f : q0[qq + W]; }, jx0, jy0);
              gen_xy(l, m, [&](int qq) { return (qq < -MM || qq > MM) ? 0.f : q1[qq + W]; }, jx1, jy1);
              r0[m + W] = wx * jx0 + wy * jy0;
              r1[m + W] = wx * jx1 + wy * jy1;
            }
#pragma unroll
            for (int m = -W; m <= W; ++m) {
              z0[m + W] -= r0[m + W];
              z1[m + W] -= r1[m + W];
            }
          }
          const float *Dl = De + dblock_off(l);
          const int w = 2 * l + 1;
          for (int mp = -l; mp <= l; ++mp) {
            float t0 = 0.f, t1 = 0.f;
#pragma unroll
            for (int m = -W; m <= W; ++m) {
              if (m < -l || m > l || m < -top || m > top) continue;
              const float dv = Dl[(m + l) * w + mp + l];
              t0 += dv * z0[m + W];
              t1 += dv * z1[m + W];
            }
            float *a = acc + (l * l + l + mp) * C + c;
            a[0] += t0;
            a[1] += t1;
          }
        }
      }
    }
    __syncthreads();
    float *o = out + (int64_t)n * y.S * C;
    for (int k = threadIdx.x; k < y.S * C; k += blockDim.x) o[k] += acc[k];
    __syncthreads();
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
// Backward per-edge terms.  For one edge (warp) and all channels:
//   Gy~ = D G[dst] on rows |m| <= mmax+1,   a = D x[src] on the same rows,
//   Gg[c'] = sum_{kept rows} Gy~ * v,
//   h_k   = sum_{kept rows, c'} (g v) (J_k Gy~) + sum_{kept rows, c} Ga (J_k a),
// where v (mixing output) and Ga (gradient of the rotated input) come from
// the two products.  h_x, h_y give the frame part of dL/dr.
// ---------------------------------------------------------------------------
template <typename TX, int MM>
__global__ void k_edge_terms(Layout y, int M, const EdgeRec *__restrict__ rec,
                             const float *__restrict__ D, const float *__restrict__ gate,
                             const float *__restrict__ G, const TX *__restrict__ X,
                             const float *__restrict__ V, const float *__restrict__ Ga,
                             float *__restrict__ Gg, float *__restrict__ h) {
  constexpr int W = MM + 1;  // widest |m| needed by the generators
  const int lane = threadIdx.x & 31, wpb = blockDim.x >> 5;
  for (int i = blockIdx.x * wpb + (threadIdx.x >> 5); i < M; i += gridDim.x * wpb) {
    const EdgeRec r = rec[i];
    const float *De = D + (int64_t)i * y.dsz;
    float hx = 0.f, hy = 0.f;
    // output side
    const float *Gn = G + (int64_t)r.dst * y.S * y.co;
    const float *Vi = V + (int64_t)i * y.KG;
    for (int c = 2 * lane; c < y.co; c += 64) {
      const float2 gv = load2(gate + (int64_t)i * y.co + c);
      float gg0 = 0.f, gg1 = 0.f;
      for (int l = 0; l <= y.L; ++l) {
        float b0[2 * W + 1], b1[2 * W + 1];
#pragma unroll
        for (int k = 0; k < 2 * W + 1; ++k) b0[k] = b1[k] = 0.f;
        const float *Dl = De + dblock_off(l);
        const int w = 2 * l + 1;
        for (int mp = -l; mp <= l; ++mp) {
          const float2 gx = load2(Gn + (l * l + l + mp) * y.co + c);
#pragma unroll
          for (int m = -W; m <= W; ++m) {
            if (m < -l || m > l) continue;
            const float dv = Dl[(m + l) * w + mp + l];
            b0[m + W] += dv * gx.x;
            b1[m + W] += dv * gx.y;
          }
        }
#pragma unroll
        for (int m = -MM; m <= MM; ++m) {
          if (m < -l || m > l) continue;
          int g, j;
          lm_group_row(y, l, m, g, j);
          const float2 v = load2(Vi + y.kout_off[g] + j * y.co + c);
          gg0 += b0[m + W] * v.x;
          gg1 += b1[m + W] * v.y;
          float jx0, jy0, jx1, jy1;
          gen_xy(l, m, [&](int q) { return b0[q + W]; }, jx0, jy0);
          gen_xy(l, m, [&](int q) { return b1[q + W]; }, jx1, jy1);
          hx += gv.x * v.x * jx0 + gv.y * v.y * jx1;
          hy += gv.x * v.x * jy0 + gv.y * v.y * jy1;
        }
      }
      *reinterpret_cast<float2 *>(Gg + (int64_t)i * y.co + c) = make_float2(gg0, gg1);
    }
    // input side
    const TX *Xn = X + (int64_t)r.src * y.S * y.ci;
    const float *Gai = Ga + (int64_t)i * y.KA;
    for (int c = 2 * lane; c < y.ci; c += 64) {
      for (int l = 0; l <= y.L; ++l) {
        float b0[2 * W + 1], b1[2 * W + 1];
#pragma unroll
        for (int k = 0; k < 2 * W + 1; ++k) b0[k] = b1[k] = 0.f;
        const float *Dl = De + dblock_off(l);
        const int w = 2 * l + 1;
        for (int mp = -l; mp <= l; ++mp) {
          const float2 xv = load2(Xn + (l * l + l + mp) * y.ci + c);
#pragma unroll
          for (int m = -W; m <= W; ++m) {
            if (m < -l || m > l) continue;
            const float dv = Dl[(m + l) * w + mp + l];
            b0[m + W] += dv * xv.x;
            b1[m + W] += dv * xv.y;
          }
        }
#pragma unroll
        for (int m = -MM; m <= MM; ++m) {
          if (m < -l || m > l) continue;
          int g, j;
          lm_group_row(y, l, m, g, j);
          const float2 ga = load2(Gai + y.kin_off[g] + j * y.ci + c);
          float jx0, jy0, jx1, jy1;
          gen_xy(l, m, [&](int q) { return b0[q + W]; }, jx0, jy0);
          gen_xy(l, m, [&](int q) { return b1[q + W]; }, jx1, jy1);
          hx += ga.x * jx0 + ga.y * jx1;
          hy += ga.x * jy0 + ga.y * jy1;
        }
      }
    }
    for (int o = 16; o > 0; o >>= 1) {
      hx += __shfl_xor_sync(0xffffffffu, hx, o);
      hy += __shfl_xor_sync(0xffffffffu, hy, o);
    }
    if (lane == 0) {
      h[2 * (int64_t)i] = hx;
      h[2 * (int64_t)i + 1] = hy;
    }
  }
}

// grad_r[eid] = R^T (-h_y, h_x, 0) / d + (sum_c' Gg[c'] sum_k W_rad[k][c'] phi'_k(d)) r_hat.
// One warp per edge; phi'_k(d) is computed once per edge (lanes over k).
__global__ void k_edge_final(Layout y, float cutoff, int M, const EdgeRec *__restrict__ rec,
                             const float *__restrict__ geo, const float *__restrict__ Gg,
                             const float *__restrict__ h, const float *__restrict__ w_rad,
                             float *__restrict__ grad_r) {
  const int lane = threadIdx.x & 31, wpb = blockDim.x >> 5;
  const float sig = cutoff / static_cast<float>(y.nr - 1);
  for (int i = blockIdx.x * wpb + (threadIdx.x >> 5); i < M; i += gridDim.x * wpb) {
    const float *gr = geo + (int64_t)i * GEO;
    const float d = gr[0];
    float dphi[2];  // k = lane, lane + 32
    for (int u = 0; u < 2; ++u) {
      const int k = lane + 32 * u;
      const float t = (d - sig * static_cast<float>(k)) / sig;
      dphi[u] = (k < y.nr) ? (-t / sig) * __expf(-0.5f * t * t) : 0.f;
    }
    float dd = 0.f;
    // every lane runs every shuffle: the channel loop is warp-uniform
    for (int c0 = 0; c0 < y.co; c0 += 32) {
      const int c = c0 + lane;
      float dg = 0.f;
      for (int k = 0; k < y.nr; ++k) {
        const float dk = __shfl_sync(0xffffffffu, dphi[k >> 5], k & 31);
        if (c < y.co) dg += w_rad[k * y.co + c] * dk;
      }
      if (c < y.co) dd += Gg[(int64_t)i * y.co + c] * dg;
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
}

// Radial-gate gradients, stage 1: each block sums, over a tile of RAD_TILE
// edges, phi_k(d_i) A[i][c'] + phi'_k(d_i) dd_i B[i][c'] (rows k < nr) and
// A[i][c'] (bias row k = nr) into part[block][k][c'].  B (and dd_i =
// omega[i][2]) is optional.  Stage 2 adds the blocks in order.
constexpr int RAD_TILE = 256;
__global__ void k_rad_partial(Layout y, float cutoff, int M, const float *__restrict__ geo,
                              const float *__restrict__ Ag, const float *__restrict__ Bg,
                              const float *__restrict__ omega, float *__restrict__ part) {
  extern __shared__ float phi[];  // [2][RAD_TILE][nr]
  const int i0 = blockIdx.x * RAD_TILE;
  const int n = (M - i0) < RAD_TILE ? (M - i0) : RAD_TILE;
  float *dphi = phi + RAD_TILE * y.nr;
  const float sig = cutoff / static_cast<float>(y.nr - 1);
  for (int t = threadIdx.x; t < n * y.nr; t += blockDim.x) {
    const int i = t / y.nr, k = t % y.nr;
    const float d = geo[(int64_t)(i0 + i) * GEO];
    phi[t] = rbf_val(d, k, y, cutoff);
    if (Bg) {
      const float u = (d - sig * static_cast<float>(k)) / sig;
      dphi[t] = (-u / sig) * phi[t] * omega[4 * (int64_t)(i0 + i) + 2];
    }
  }
  __syncthreads();
  const int P = (y.nr + 1) * y.co;
  for (int pidx = threadIdx.x; pidx < P; pidx += blockDim.x) {
    const int k = pidx / y.co, c = pidx % y.co;
    float s = 0.f;
    if (k < y.nr) {
      for (int i = 0; i < n; ++i) s += phi[i * y.nr + k] * Ag[(int64_t)(i0 + i) * y.co + c];
      if (Bg)
        for (int i = 0; i < n; ++i) s += dphi[i * y.nr + k] * Bg[(int64_t)(i0 + i) * y.co + c];
    } else {
      for (int i = 0; i < n; ++i) s += Ag[(int64_t)(i0 + i) * y.co + c];
    }
    part[(int64_t)blockIdx.x * P + pidx] = s;
  }
}

__global__ void k_rad_reduce(Layout y, int nblk, const float *__restrict__ part,
                             float *__restrict__ grad_w_rad, float *__restrict__ grad_b) {
  const int P = (y.nr + 1) * y.co;
  const int pidx = blockIdx.x * blockDim.x + threadIdx.x;
  if (pidx >= P) return;
  float s = 0.f;
  for (int b = 0; b < nblk; ++b) s += part[(int64_t)b * P + pidx];
  const int k = pidx / y.co, c = pidx % y.co;
  if (k < y.nr) {
    if (grad_w_rad) grad_w_rad[k * y.co + c] += s;
  } else if (grad_b) {
    grad_b[c] += s;
  }
}

// ---------------------------------------------------------------------------
// Double backward, per edge: the frame turn and gate change that the edge
// cotangent gg_r induces.  With u = R gg_r / d: omega = (u_y, -u_x) (the
// z component, a roll of the frame, does not change the output),
// dd = r_hat . gg_r and dg[c'] = dd * sum_k W_rad[k][c'] phi'_k(d).
// omega[i] = (w_x, w_y, dd, 0).  One warp per edge.
// ---------------------------------------------------------------------------
__global__ void k_edge_omega(Layout y, float cutoff, int M, const EdgeRec *__restrict__ rec,
                             const float *__restrict__ geo, const float *__restrict__ gg_r,
                             const float *__restrict__ w_rad, float *__restrict__ omega,
                             float *__restrict__ dgate) {
  const int lane = threadIdx.x & 31, wpb = blockDim.x >> 5;
  const float sig = cutoff / static_cast<float>(y.nr - 1);
  for (int i = blockIdx.x * wpb + (threadIdx.x >> 5); i < M; i += gridDim.x * wpb) {
    const float *gr = geo + (int64_t)i * GEO;
    const float d = gr[0];
    const int e = rec[i].eid;
    const float g0 = gg_r[3 * (int64_t)e], g1 = gg_r[3 * (int64_t)e + 1], g2 = gg_r[3 * (int64_t)e + 2];
    const float *R = gr + 4;
    const float inv = d > 0.f ? 1.f / d : 0.f;
    const float ux = (R[0] * g0 + R[1] * g1 + R[2] * g2) * inv;
    const float uy = (R[3] * g0 + R[4] * g1 + R[5] * g2) * inv;
    const float dd = gr[1] * g0 + gr[2] * g1 + gr[3] * g2;
    if (lane == 0) {
      omega[4 * (int64_t)i] = uy;
      omega[4 * (int64_t)i + 1] = -ux;
      omega[4 * (int64_t)i + 2] = dd;
      omega[4 * (int64_t)i + 3] = 0.f;
    }
    float dphi[2];
    for (int u = 0; u < 2; ++u) {
      const int k = lane + 32 * u;
      const float t = (d - sig * static_cast<float>(k)) / sig;
      dphi[u] = (k < y.nr) ? (-t / sig) * __expf(-0.5f * t * t) : 0.f;
    }
    for (int c0 = 0; c0 < y.co; c0 += 32) {
      const int c = c0 + lane;
      float dg = 0.f;
      for (int k = 0; k < y.nr; ++k) {
        const float dk = __shfl_sync(0xffffffffu, dphi[k >> 5], k & 31);
        if (c < y.co) dg += w_rad[k * y.co + c] * dk;
      }
      if (c < y.co) dgate[(int64_t)i * y.co + c] = dd * dg;
    }
  }
}

// Double backward, per edge and output channel:
//   A[c'] = sum_{kept rows} (Omega Gy~)(V) + Gy~ dV + Gy~ V~    (d Q / d g)
//   B[c'] = sum_{kept rows} Gy~ V                              (d Q / d dg)
// with Gy~ = D G[dst] (rows up to mmax + 1 for Omega), V = M a, dV = M(Omega a),
// V~ = M(D gg_x[src]) (optional).  One warp per edge, lanes over channels.
template <int MM>
__global__ void k_edge_terms2(Layout y, int M, const EdgeRec *__restrict__ rec,
                              const float *__restrict__ D, const float *__restrict__ G,
                              const float *__restrict__ omega, const float *__restrict__ V,
                              const float *__restrict__ dV, const float *__restrict__ Vt,
                              float *__restrict__ Aout, float *__restrict__ Bout) {
  constexpr int W = MM + 1;
  const int lane = threadIdx.x & 31, wpb = blockDim.x >> 5;
  for (int i = blockIdx.x * wpb + (threadIdx.x >> 5); i < M; i += gridDim.x * wpb) {
    const EdgeRec r = rec[i];
    const float *De = D + (int64_t)i * y.dsz;
    const float *Gn = G + (int64_t)r.dst * y.S * y.co;
    const float wx = omega ? omega[4 * (int64_t)i] : 0.f;
    const float wy = omega ? omega[4 * (int64_t)i + 1] : 0.f;
    const int64_t ro = (int64_t)i * y.KG;
    for (int c = 2 * lane; c < y.co; c += 64) {
      float A0 = 0.f, A1 = 0.f, B0 = 0.f, B1 = 0.f;
      for (int l = 0; l <= y.L; ++l) {
        float b0[2 * W + 1], b1[2 * W + 1];
#pragma unroll
        for (int k = 0; k < 2 * W + 1; ++k) b0[k] = b1[k] = 0.f;
        const float *Dl = De + dblock_off(l);
        const int w = 2 * l + 1;
        for (int mp = -l; mp <= l; ++mp) {
          const float2 gx = load2(Gn + (l * l + l + mp) * y.co + c);
#pragma unroll
          for (int m = -W; m <= W; ++m) {
            if (m < -l || m > l) continue;
            const float dv = Dl[(m + l) * w + mp + l];
            b0[m + W] += dv * gx.x;
            b1[m + W] += dv * gx.y;
          }
        }
#pragma unroll
        for (int m = -MM; m <= MM; ++m) {
          if (m < -l || m > l) continue;
          int g, j;
          lm_group_row(y, l, m, g, j);
          const int64_t col = ro + y.kout_off[g] + j * y.co + c;
          const float2 v = load2(V + col);
          const float2 dv = dV ? load2(dV + col) : make_float2(0.f, 0.f);
          float jx0, jy0, jx1, jy1;
          gen_xy(l, m, [&](int q) { return b0[q + W]; }, jx0, jy0);
          gen_xy(l, m, [&](int q) { return b1[q + W]; }, jx1, jy1);
          const float og0 = wx * jx0 + wy * jy0, og1 = wx * jx1 + wy * jy1;
          A0 += og0 * v.x + b0[m + W] * dv.x;
          A1 += og1 * v.y + b1[m + W] * dv.y;
          if (Vt) {
            const float2 vt = load2(Vt + col);
            A0 += b0[m + W] * vt.x;
            A1 += b1[m + W] * vt.y;
          }
          B0 += b0[m + W] * v.x;
          B1 += b1[m + W] * v.y;
        }
      }
      *reinterpret_cast<float2 *>(Aout + (int64_t)i * y.co + c) = make_float2(A0, A1);
      *reinterpret_cast<float2 *>(Bout + (int64_t)i * y.co + c) = make_float2(B0, B1);
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
