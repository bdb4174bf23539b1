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

// Occupancy and load-batching of the per-edge gather kernels (rotation on
// gather, edge terms).  They are latency bound, so each is compiled for a
// number of resident 256-thread blocks per SM (which caps its registers),
// and the edge-term kernels may fence every few rows so that the compiler
// does not hoist a whole level's loads into registers.  Defaults are the
// fastest measured on B200 for lmax 4 and 6, mmax 2, C 128.
#ifndef SO2_GATHER_MINB  // runtime-degree kernels
#define SO2_GATHER_MINB 2
#endif
#ifndef SO2_ET_BATCH  // rows per load batch, runtime-degree edge terms (0: no fence)
#define SO2_ET_BATCH 2
#endif
#ifndef SO2_ET_MINB_LC  // compile-time-degree edge terms
#define SO2_ET_MINB_LC 2
#endif
#ifndef SO2_ET_BATCH_LC
#define SO2_ET_BATCH_LC 2
#endif
#ifndef SO2_ROT_MINB  // compile-time-degree rotation, lmax < 6
#define SO2_ROT_MINB 2
#endif
#ifndef SO2_ROT_MINB_L6  // compile-time-degree rotation, lmax 6
#define SO2_ROT_MINB_L6 3
#endif

// Largest number of radial basis functions (the ABI allows 2..64).
constexpr int RAD_MAX_NR = 64;

// Keeps the compiler from moving loads across this point.
__device__ __forceinline__ void load_fence() { asm volatile("" ::: "memory"); }

// Whether the edge-term kernels fence before row mp of degree l.
template <int LC>
__device__ __forceinline__ constexpr bool et_fence(int l, int mp) {
  constexpr int b = LC < 0 ? SO2_ET_BATCH : SO2_ET_BATCH_LC;
  return b > 0 && mp > -l && (mp + l) % b == 0;
}

// Degree l as a compile-time value.
template <int N>
struct Lv {
  static constexpr int value = N;
};

template <int I, int N, typename F>
__device__ __forceinline__ void static_levels(F &f) {
  if constexpr (I < N) {
    f(Lv<I>{});
    static_levels<I + 1, N>(f);
  }
}

// f(Lv<l>{}) for l = 0..L.  LC >= 0 (then L = LC): every level inlined in
// sequence, so loads of one level can be scheduled early in the previous
// one.  LC = -1: a runtime loop whose body switches to the level's
// compile-time instance, so no level keeps registers live in another.
template <int LC, typename F>
__device__ __forceinline__ void each_level(int L, F &&f) {
  if constexpr (LC >= 0) {
    static_levels<0, LC + 1>(f);
  } else {
#pragma unroll 1
    for (int l = 0; l <= L; ++l) {
      switch (l) {
        case 0: f(Lv<0>{}); break;
        case 1: f(Lv<1>{}); break;
        case 2: f(Lv<2>{}); break;
        case 3: f(Lv<3>{}); break;
        case 4: f(Lv<4>{}); break;
        case 5: f(Lv<5>{}); break;
        default: f(Lv<6>{}); break;
      }
    }
  }
}
static_assert(LMAX_SUPPORTED == 6, "each_level instantiates degrees 0..6");

// The library is built from more than one translation unit that include this
// header: its kernels that are not templates have internal linkage (static).

// ---------------------------------------------------------------------------
// Graph preparation: stable counting sort of edges by one endpoint.
// ---------------------------------------------------------------------------

// counts[key]++ for every edge; keys outside [0, N) raise SO2_ERR_INDEX and
// are counted as node 0 so that every later access stays in bounds.
static __global__ void k_count_keys(const int64_t *__restrict__ keys, int64_t E, int64_t N,
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
static __global__ void k_scan_offsets(const int *__restrict__ counts, int64_t N, int *__restrict__ offsets) {
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

static __global__ void k_place(const int64_t *__restrict__ keys, int64_t E, int64_t N,
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

// Within each key's segment, order the edge ids ascending, which makes the
// sort stable and deterministic.  One warp per segment: segments of up to
// 128 edges are placed by rank (each lane holds up to four ids and counts,
// for each, the smaller ids of the segment; ids are distinct, so the ranks
// are a permutation); longer ones fall back to an insertion sort by lane 0.
static __global__ void k_sort_segments(const int *__restrict__ offsets, int64_t N, int *__restrict__ perm) {
  const int lane = threadIdx.x & 31, wpb = blockDim.x >> 5;
  constexpr int PER = 4;
  for (int64_t n = blockIdx.x * (int64_t)wpb + (threadIdx.x >> 5); n < N;
       n += (int64_t)gridDim.x * wpb) {
    const int b = offsets[n], e = offsets[n + 1], len = e - b;
    if (len <= 1) continue;
    if (len <= 32 * PER) {
      int v[PER], rank[PER];
#pragma unroll
      for (int q = 0; q < PER; ++q) {
        const int k = lane + 32 * q;
        v[q] = k < len ? perm[b + k] : 0x7fffffff;
        rank[q] = 0;
      }
      const int nq = (len + 31) / 32;  // warp-uniform
      for (int q2 = 0; q2 < nq; ++q2) {
        for (int j = 0; j < 32; ++j) {
          int u = v[0];
#pragma unroll
          for (int q = 1; q < PER; ++q) u = (q2 == q) ? v[q] : u;
          const int w = __shfl_sync(0xffffffffu, u, j);
#pragma unroll
          for (int q = 0; q < PER; ++q) rank[q] += (w < v[q]);
        }
      }
      __syncwarp();
#pragma unroll
      for (int q = 0; q < PER; ++q)
        if (lane + 32 * q < len) perm[b + rank[q]] = v[q];
    } else if (lane == 0) {
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
}

// ---------------------------------------------------------------------------
// Per-edge records for one chunk of sorted positions [e0, e0 + M).
// ---------------------------------------------------------------------------
struct EdgeRec {
  int eid, src, dst, key;  // key = the endpoint this order is sorted by
};
static_assert(sizeof(EdgeRec) == sizeof(int4), "EdgeRec is read as int4 by the fused epilogue");

// Geometry record: d, r_hat[3], R[9] (row-major), 3 spare.
constexpr int GEO = 16;

// One thread per edge: the record, the frame and the Wigner-D blocks, the
// blocks into this warp's shared tile sD[k][33] (entry-major, so each
// thread's writes and the copy-out below are free of bank conflicts), then
// copied out edge by edge with coalesced stores.  Block = one warp.
//
// With DT, the kept rows D^l[m][:] (|m| <= mmax) are also written row-major
// by layout row: row t of all the chunk's edges is one contiguous run of
// M x (2l+1) floats at DT + kept_d_prefix(t) * dt_chunk, which is the layout
// the product's reduction epilogue stages 32 edges from with coalesced loads.
template <int L>
__global__ void __launch_bounds__(32) k_edge_prep(int64_t e0, int M, const int *__restrict__ perm,
                                                  const int64_t *__restrict__ ei, int64_t E,
                                                  int64_t N, int key_row,
                                                  const float *__restrict__ edge_vec,
                                                  EdgeRec *__restrict__ rec, float *__restrict__ geo,
                                                  float *__restrict__ D, DevStatus *st,
                                                  int mmax = 0, float *__restrict__ DT = nullptr,
                                                  int dt_chunk = 0) {
  constexpr int dsz = dsize(L);
  extern __shared__ float sD[];  // [dsz][33]
  const int lane = threadIdx.x;
  const int i0 = blockIdx.x * 32;
  const int i = i0 + lane;
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
#pragma unroll
    for (int k = 0; k < 9; ++k) gr[4 + k] = f.R[k];
    wigner_blocks_thread<L>(f.R, sD + lane, 33);
  }
  __syncwarp();
  const int nj = (M - i0) < 32 ? (M - i0) : 32;
  for (int j = 0; j < nj; ++j) {
    float *dst = D + (int64_t)(i0 + j) * dsz;
    for (int k = lane; k < dsz; k += 32) dst[k] = sD[k * 33 + j];
  }
  if (DT) {
    for (int g = 0; g <= mmax; ++g) {
      const int rows = g == 0 ? L + 1 : 2 * (L + 1 - g);
      for (int j = 0; j < rows; ++j) {
        const int l = g == 0 ? j : g + (j < L + 1 - g ? j : j - (L + 1 - g));
        const int m = g == 0 ? 0 : (j < L + 1 - g ? g : -g);
        const int w = 2 * l + 1;
        const int src = dblock_off(l) + (m + l) * w;  // entry (m, 0) of block l
        float *dst = DT + (int64_t)kept_d_prefix(L, g, j) * dt_chunk + (int64_t)i0 * w;
        for (int idx = lane; idx < nj * w; idx += 32) {
          const int el = idx / w, k = idx - el * w;
          dst[idx] = sD[(src + k) * 33 + el];
        }
      }
    }
  }
}

__device__ __forceinline__ float rbf_val(float d, int k, const Layout &y, float cutoff) {
  const float sig = cutoff / static_cast<float>(y.nr - 1);
  const float mu = sig * static_cast<float>(k);
  const float t = (d - mu) / sig;
  return __expf(-0.5f * t * t);
}

// g[i][c'] = b[c'] + sum_k w_rad[k][c'] phi_k(d_i).  A block takes
// GATE_EDGES edges: the basis values go to shared memory basis-major
// (phi[k][i]), then each thread keeps one channel's GATE_EDGES sums in
// registers, reading each w_rad[k][c'] once and four basis values per
// shared-memory load.
constexpr int GATE_EDGES = 32;
static __global__ void k_edge_gate(Layout y, float cutoff, int M, const float *__restrict__ geo,
                            const float *__restrict__ w_rad, const float *__restrict__ b_rad,
                            float *__restrict__ gate) {
  extern __shared__ float4 phi4[];  // [nr][GATE_EDGES / 4]
  float *phi = reinterpret_cast<float *>(phi4);
  const int i0 = blockIdx.x * GATE_EDGES;
  const int n = (M - i0) < GATE_EDGES ? (M - i0) : GATE_EDGES;
  for (int t = threadIdx.x; t < y.nr * GATE_EDGES; t += blockDim.x) {
    const int k = t / GATE_EDGES, i = t % GATE_EDGES;
    phi[t] = (i < n) ? rbf_val(geo[(int64_t)(i0 + i) * GEO], k, y, cutoff) : 0.f;
  }
  __syncthreads();
  for (int c = threadIdx.x; c < y.co; c += blockDim.x) {
    float acc[GATE_EDGES];
    const float b = b_rad[c];
#pragma unroll
    for (int i = 0; i < GATE_EDGES; ++i) acc[i] = b;
#pragma unroll 4
    for (int k = 0; k < y.nr; ++k) {
      const float w = w_rad[k * y.co + c];
#pragma unroll
      for (int q = 0; q < GATE_EDGES / 4; ++q) {
        const float4 f = phi4[k * (GATE_EDGES / 4) + q];
        acc[4 * q + 0] += f.x * w;
        acc[4 * q + 1] += f.y * w;
        acc[4 * q + 2] += f.z * w;
        acc[4 * q + 3] += f.w * w;
      }
    }
#pragma unroll
    for (int i = 0; i < GATE_EDGES; ++i)
      if (i < n) gate[(int64_t)(i0 + i) * y.co + c] = acc[i];
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
// this is plain rotation on gather (A = 1) or gated rotation (A = g).  With
// out2 the same rotation also gives out2 = A2 * b + B2 * (Omega b).
__device__ __forceinline__ float4 load4(const float *p) { return *reinterpret_cast<const float4 *>(p); }
// Read-only (non-coherent) loads, free to move across the kernel's stores.
__device__ __forceinline__ float4 load4_ro(const float *p) { return __ldg(reinterpret_cast<const float4 *>(p)); }
__device__ __forceinline__ float4 load4_ro(const __nv_bfloat16 *p) {
  const uint2 u = __ldg(reinterpret_cast<const uint2 *>(p));
  const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&u.x));
  const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&u.y));
  return make_float4(a.x, a.y, b.x, b.y);
}
__device__ __forceinline__ float4 load4(const __nv_bfloat16 *p) {
  const uint2 u = *reinterpret_cast<const uint2 *>(p);
  const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&u.x));
  const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&u.y));
  return make_float4(a.x, a.y, b.x, b.y);
}
// Four elements as loaded (raw), converted to f32 only where they are used,
// so that a load issued ahead of its use does not wait for the data.
template <typename T> struct Raw4;
template <> struct Raw4<float> { float4 v; };
template <> struct Raw4<__nv_bfloat16> { uint2 v; };
__device__ __forceinline__ Raw4<float> ld_raw4(const float *p) {
  return Raw4<float>{__ldg(reinterpret_cast<const float4 *>(p))};
}
__device__ __forceinline__ Raw4<__nv_bfloat16> ld_raw4(const __nv_bfloat16 *p) {
  return Raw4<__nv_bfloat16>{__ldg(reinterpret_cast<const uint2 *>(p))};
}
__device__ __forceinline__ float4 cvt4(const Raw4<float> &r) { return r.v; }
__device__ __forceinline__ float4 cvt4(const Raw4<__nv_bfloat16> &r) {
  const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&r.v.x));
  const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&r.v.y));
  return make_float4(a.x, a.y, b.x, b.y);
}
template <typename T> __device__ __forceinline__ Raw4<T> zero_raw4() { return Raw4<T>{}; }

__device__ __forceinline__ void store_split4(__nv_bfloat16 *hi, __nv_bfloat16 *lo, float4 v) {
  __nv_bfloat16 h[4], l[4];
  split_bf16(v.x, h[0], l[0]);
  split_bf16(v.y, h[1], l[1]);
  split_bf16(v.z, h[2], l[2]);
  split_bf16(v.w, h[3], l[3]);
  uint2 uh, ul;
  *reinterpret_cast<__nv_bfloat162 *>(&uh.x) = __halves2bfloat162(h[0], h[1]);
  *reinterpret_cast<__nv_bfloat162 *>(&uh.y) = __halves2bfloat162(h[2], h[3]);
  *reinterpret_cast<uint2 *>(hi) = uh;
  if (lo) {
    *reinterpret_cast<__nv_bfloat162 *>(&ul.x) = __halves2bfloat162(l[0], l[1]);
    *reinterpret_cast<__nv_bfloat162 *>(&ul.y) = __halves2bfloat162(l[2], l[3]);
    *reinterpret_cast<uint2 *>(lo) = ul;
  }
}
__device__ __forceinline__ float4 coef4(const Coef &k, int64_t i, int C, int c) {
  if (k.mode == 0) return make_float4(0.f, 0.f, 0.f, 0.f);
  if (k.mode == 1) return make_float4(1.f, 1.f, 1.f, 1.f);
  return load4(k.p + i * C + c);
}

// Copy one edge's Wigner-D blocks (dsz floats) into this warp's shared slice.
__device__ __forceinline__ void stage_d(const float *De, int dsz, float *sD) {
  const int lane = threadIdx.x & 31;
  for (int k = lane; k < dsz; k += 32) sD[k] = De[k];
  __syncwarp();
}

// LC >= 0 fixes lmax at compile time (loops fully unrolled); -1 reads it
// from the layout.
template <typename TX, int MM, int LC = -1, bool DUAL = false>
__global__ void __launch_bounds__(256, LC == 6 ? SO2_ROT_MINB_L6 : (LC >= 0 ? SO2_ROT_MINB : SO2_GATHER_MINB)) k_rotate_gather(Layout y, int M, const EdgeRec *__restrict__ rec,
                                const float *__restrict__ D, const TX *__restrict__ X, int side,
                                int use_src, Coef A, Coef B, const float *__restrict__ omega,
                                __nv_bfloat16 *__restrict__ out_hi, __nv_bfloat16 *__restrict__ out_lo,
                                int ld, Coef A2, Coef B2, __nv_bfloat16 *__restrict__ out2_hi,
                                __nv_bfloat16 *__restrict__ out2_lo) {
  constexpr int W = MM + 1;
  extern __shared__ float sDall[];  // [warps][dsz]
  const int C = side ? y.co : y.ci;
  const int *col_off = side ? y.kout_off : y.kin_off;
  const int *col_pad = side ? y.Kout_pad : y.Kin_pad;
  const int lane = threadIdx.x & 31, wpb = blockDim.x >> 5;
  float *sD = sDall + (threadIdx.x >> 5) * y.dsz;
  constexpr bool dual = DUAL;  // a second output from the same rotation
  const bool wide = B.mode != 0 || (dual && B2.mode != 0);
  for (int i = blockIdx.x * wpb + (threadIdx.x >> 5); i < M; i += gridDim.x * wpb) {
    const EdgeRec r = rec[i];
    const int node = use_src ? r.src : r.dst;
    __syncwarp();
    stage_d(D + (int64_t)i * y.dsz, y.dsz, sD);
    const TX *Xn = X + (int64_t)node * y.S * C;
    __nv_bfloat16 *oh = out_hi + (int64_t)i * ld;
    __nv_bfloat16 *ol = out_lo ? out_lo + (int64_t)i * ld : nullptr;
    __nv_bfloat16 *o2h = dual ? out2_hi + (int64_t)i * ld : nullptr;
    __nv_bfloat16 *o2l = dual && out2_lo ? out2_lo + (int64_t)i * ld : nullptr;
    float wx = 0.f, wy = 0.f;
    if (wide) {
      wx = omega[4 * (int64_t)i];
      wy = omega[4 * (int64_t)i + 1];
    }
    // Two schedules, each chosen by measurement for the degrees it serves:
    // lmax 6 runs every level inlined with plain loads; the others run
    // per-level bodies with read-only loads the compiler may hoist.
    if constexpr (LC == 6) {
      for (int c = 4 * lane; c < C; c += 128) {
        const float4 ca = coef4(A, i, C, c), cb = coef4(B, i, C, c);
        const float4 ca2 = dual ? coef4(A2, i, C, c) : make_float4(0.f, 0.f, 0.f, 0.f);
        const float4 cb2 = dual ? coef4(B2, i, C, c) : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int l = 0; l <= LC; ++l) {
          float4 a[2 * W + 1];
#pragma unroll
          for (int k = 0; k < 2 * W + 1; ++k) a[k] = make_float4(0.f, 0.f, 0.f, 0.f);
          const float *Dl = sD + dblock_off(l);
          const int w = 2 * l + 1;
          const int top = wide ? W : MM;
#pragma unroll
          for (int mp = -l; mp <= l; ++mp) {
            const float4 xv = load4(Xn + (l * l + l + mp) * C + c);
#pragma unroll
            for (int m = -W; m <= W; ++m) {
              if (m < -l || m > l || m < -top || m > top) continue;
              const float dv = Dl[(m + l) * w + mp + l];
              a[m + W].x += dv * xv.x;
              a[m + W].y += dv * xv.y;
              a[m + W].z += dv * xv.z;
              a[m + W].w += dv * xv.w;
            }
          }
#pragma unroll
          for (int m = -MM; m <= MM; ++m) {
            if (m < -l || m > l) continue;
            int g, j;
            lm_group_row(y, l, m, g, j);
            const int col = col_off[g] + j * C + c;
            float4 om = make_float4(0.f, 0.f, 0.f, 0.f);  // (Omega a)[m]
            if (wide) {
              float jx, jy;
              gen_xy(l, m, [&](int q) { return a[q + W].x; }, jx, jy);
              om.x = wx * jx + wy * jy;
              gen_xy(l, m, [&](int q) { return a[q + W].y; }, jx, jy);
              om.y = wx * jx + wy * jy;
              gen_xy(l, m, [&](int q) { return a[q + W].z; }, jx, jy);
              om.z = wx * jx + wy * jy;
              gen_xy(l, m, [&](int q) { return a[q + W].w; }, jx, jy);
              om.w = wx * jx + wy * jy;
            }
            const float4 av = a[m + W];
            store_split4(oh + col, ol ? ol + col : nullptr,
                         make_float4(ca.x * av.x + cb.x * om.x, ca.y * av.y + cb.y * om.y,
                                     ca.z * av.z + cb.z * om.z, ca.w * av.w + cb.w * om.w));
            if (dual)
              store_split4(o2h + col, o2l ? o2l + col : nullptr,
                           make_float4(ca2.x * av.x + cb2.x * om.x, ca2.y * av.y + cb2.y * om.y,
                                       ca2.z * av.z + cb2.z * om.z, ca2.w * av.w + cb2.w * om.w));
          }
        }
      }
    } else {
      for (int c = 4 * lane; c < C; c += 128) {
        const float4 ca = coef4(A, i, C, c), cb = coef4(B, i, C, c);
        const float4 ca2 = dual ? coef4(A2, i, C, c) : make_float4(0.f, 0.f, 0.f, 0.f);
        const float4 cb2 = dual ? coef4(B2, i, C, c) : make_float4(0.f, 0.f, 0.f, 0.f);
        each_level<LC>(y.L, [&](auto lv) {
          constexpr int l = decltype(lv)::value;
          constexpr int w = 2 * l + 1;
          constexpr int mlo = -(W < l ? W : l), mhi = (W < l ? W : l);
          float4 a[2 * W + 1];
#pragma unroll
          for (int k = 0; k < 2 * W + 1; ++k) a[k] = make_float4(0.f, 0.f, 0.f, 0.f);
          const float *Dl = sD + dblock_off(l);
          const int top = wide ? W : MM;
#pragma unroll
          for (int mp = -l; mp <= l; ++mp) {
            const float4 xv = load4_ro(Xn + (l * l + l + mp) * C + c);
#pragma unroll
            for (int m = mlo; m <= mhi; ++m) {
              if (m < -top || m > top) continue;
              const float dv = Dl[(m + l) * w + mp + l];
              a[m + W].x += dv * xv.x;
              a[m + W].y += dv * xv.y;
              a[m + W].z += dv * xv.z;
              a[m + W].w += dv * xv.w;
            }
          }
#pragma unroll
          for (int m = -(MM < l ? MM : l); m <= (MM < l ? MM : l); ++m) {
            int g, j;
            lm_group_row(y, l, m, g, j);
            const int col = col_off[g] + j * C + c;
            float4 om = make_float4(0.f, 0.f, 0.f, 0.f);  // (Omega a)[m]
            if (wide) {
              float jx, jy;
              gen_xy(l, m, [&](int q) { return a[q + W].x; }, jx, jy);
              om.x = wx * jx + wy * jy;
              gen_xy(l, m, [&](int q) { return a[q + W].y; }, jx, jy);
              om.y = wx * jx + wy * jy;
              gen_xy(l, m, [&](int q) { return a[q + W].z; }, jx, jy);
              om.z = wx * jx + wy * jy;
              gen_xy(l, m, [&](int q) { return a[q + W].w; }, jx, jy);
              om.w = wx * jx + wy * jy;
            }
            const float4 av = a[m + W];
            store_split4(oh + col, ol ? ol + col : nullptr,
                         make_float4(ca.x * av.x + cb.x * om.x, ca.y * av.y + cb.y * om.y,
                                     ca.z * av.z + cb.z * om.z, ca.w * av.w + cb.w * om.w));
            if (dual)
              store_split4(o2h + col, o2l ? o2l + col : nullptr,
                           make_float4(ca2.x * av.x + cb2.x * om.x, ca2.y * av.y + cb2.y * om.y,
                                       ca2.z * av.z + cb2.z * om.z, ca2.w * av.w + cb2.w * om.w));
          }
        });
      }
    }
    for (int g = 0; g < y.ng; ++g) {
      const int width = y.rows[g] * C;
      for (int k = width + 4 * lane; k < col_pad[g]; k += 128) {
        store_split4(oh + col_off[g] + k, ol ? ol + col_off[g] + k : nullptr,
                     make_float4(0.f, 0.f, 0.f, 0.f));
        if (dual)
          store_split4(o2h + col_off[g] + k, o2l ? o2l + col_off[g] + k : nullptr,
                       make_float4(0.f, 0.f, 0.f, 0.f));
      }
    }
  }
}

// Up to three per-edge row sets F_u (grouped layout, row stride ld[u]; f32,
// or bf16 where the kernel's TF says so) and their per-channel coefficients:
// the reduced rows are
//   Z = sum_u A_u F_u - Omega (sum_{u<2} B_u F_u)      (|m| up to mmax + 1)
struct ScatterTerms {
  const float *F[3];
  int ld[3];
  Coef A[3];
  Coef B[2];
};

// ---------------------------------------------------------------------------
// Inverse rotation on reduction, node-centric, one term: for every node n
// whose sorted segment meets this chunk and every degree l,
//   out[n][(l, m')][c] += sum_{chunk edges i of n} sum_m D_i^l[m][m'] k_i[c] F[i][(l, m)][c]
// with k the optional per-edge channel coefficient (the gate) and F the
// product rows (grouped layout, row stride ld).  One warp per (node, l),
// four channels per lane, the node's sums in registers; each output element
// has one writer per launch and the chunks run in stream order, so the sum
// order is fixed and no atomics are needed.
// ---------------------------------------------------------------------------
#ifndef SO2_RN_MINB  // resident 256-thread blocks per SM for k_reduce_nodes
#define SO2_RN_MINB 2
#endif
// Shared memory per warp of k_reduce_nodes: two buffers of the kept D rows
// of one edge, rows padded to a multiple of 4 floats (at most 13 x 16).
constexpr int RN_DBUF = 13 * 16;

template <int MM, int l, typename TF>
__device__ __forceinline__ void reduce_level(const Layout &y, int b, int e, int C,
                                             const int *col_off, const float *__restrict__ D,
                                             const TF *__restrict__ F, int ld,
                                             const float *__restrict__ coef, float *o, int c,
                                             bool act, float *dsm) {
  constexpr int w = 2 * l + 1;
  constexpr int wpad = (w + 3) / 4 * 4;
  constexpr int mm = MM < l ? MM : l;  // kept rows |m| <= mm
  constexpr int nm = 2 * mm + 1;
  constexpr int nd = nm * w;  // kept D entries of one edge
  constexpr int nu = (nd + 31) / 32;
  static_assert(nm * wpad <= RN_DBUF, "D staging buffer");
  const int lane = threadIdx.x & 31;
  float4 acc[w];
#pragma unroll
  for (int k = 0; k < w; ++k) acc[k] = make_float4(0.f, 0.f, 0.f, 0.f);
  int cols[nm];
#pragma unroll
  for (int m = -mm; m <= mm; ++m) {
    int g, j;
    lm_group_row(y, l, m, g, j);
    cols[m + mm] = col_off[g] + j * C + c;
  }
  // one edge's inputs: its kept D entries (one per lane), coefficient, rows
  float dreg[nu];
  float4 kc;
  Raw4<TF> fz[nm];
  auto load_edge = [&](int i) {
    const float *Dl = D + (int64_t)i * y.dsz + dblock_off(l) + (l - mm) * w;
#pragma unroll
    for (int u = 0; u < nu; ++u) dreg[u] = (lane + 32 * u < nd) ? __ldg(Dl + lane + 32 * u) : 0.f;
    kc = make_float4(1.f, 1.f, 1.f, 1.f);
    if (coef && act) kc = __ldg(reinterpret_cast<const float4 *>(coef + (int64_t)i * C + c));
#pragma unroll
    for (int m = 0; m < nm; ++m)
      fz[m] = act ? ld_raw4(F + (int64_t)i * ld + cols[m]) : zero_raw4<TF>();
  };
  if (b < e) load_edge(b);
  for (int i = b; i < e; ++i) {
    // stage this edge's D rows (buffer i & 1), scale its rows, fetch the next edge
    float *Ds = dsm + (i & 1) * RN_DBUF;
#pragma unroll
    for (int u = 0; u < nu; ++u) {
      const int k = lane + 32 * u;
      if (k < nd) Ds[(k / w) * wpad + k % w] = dreg[u];
    }
    float4 z[nm];
#pragma unroll
    for (int m = 0; m < nm; ++m) {
      const float4 f = cvt4(fz[m]);
      z[m] = make_float4(kc.x * f.x, kc.y * f.y, kc.z * f.z, kc.w * f.w);
    }
    __syncwarp();
    if (i + 1 < e) load_edge(i + 1);
#pragma unroll
    for (int m = 0; m < nm; ++m) {
#pragma unroll
      for (int q = 0; q < wpad / 4; ++q) {
        const float4 d = *reinterpret_cast<const float4 *>(Ds + m * wpad + 4 * q);
        const float dv[4] = {d.x, d.y, d.z, d.w};
#pragma unroll
        for (int t = 0; t < 4; ++t) {
          const int mp = 4 * q + t;
          if (mp < w) {
            acc[mp].x += dv[t] * z[m].x;
            acc[mp].y += dv[t] * z[m].y;
            acc[mp].z += dv[t] * z[m].z;
            acc[mp].w += dv[t] * z[m].w;
          }
        }
      }
    }
  }
  if (!act) return;
#pragma unroll
  for (int mp = 0; mp < w; ++mp) {
    float4 *dst = reinterpret_cast<float4 *>(o + (l * l + mp) * C + c);
    float4 v = *dst;
    v.x += acc[mp].x;
    v.y += acc[mp].y;
    v.z += acc[mp].z;
    v.w += acc[mp].w;
    *dst = v;
  }
}

// The general form of the node reduction (several product row sets and the
// frame-turn term of the double backward, see ScatterTerms):
//   Z = sum_u A_u F_u - Omega (sum_{u<2} B_u F_u),  rows |m| <= mmax + 1,
//   out[n][(l, m')][c] += sum_{chunk edges i of n} sum_m D_i^l[m][m'] Z_i[(l, m)][c].
// One warp per (node, l), four channels per lane, D rows staged per edge.
template <int MM, int l, typename TF>
__device__ __forceinline__ void reduce_level_terms(const Layout &y, int b, int e, int C,
                                                   const int *col_off, const float *__restrict__ D,
                                                   const ScatterTerms &t,
                                                   const float *__restrict__ omega, bool wide,
                                                   float *o, int c, bool act, float *dsm) {
  constexpr int W = MM + 1;
  constexpr int w = 2 * l + 1;
  constexpr int wpad = (w + 3) / 4 * 4;
  constexpr int mm = MM < l ? MM : l;  // rows of the products
  constexpr int mz = W < l ? W : l;    // rows of Z (the frame turn reaches one further)
  constexpr int nz = 2 * mz + 1;
  constexpr int nd = nz * w;
  constexpr int nu = (nd + 31) / 32;
  static_assert(nz * wpad <= RN_DBUF, "D staging buffer");
  const int lane = threadIdx.x & 31;
  float4 acc[w];
#pragma unroll
  for (int k = 0; k < w; ++k) acc[k] = make_float4(0.f, 0.f, 0.f, 0.f);
  int cols[2 * mm + 1];
#pragma unroll
  for (int m = -mm; m <= mm; ++m) {
    int g, j;
    lm_group_row(y, l, m, g, j);
    cols[m + mm] = col_off[g] + j * C + c;
  }
  for (int i = b; i < e; ++i) {
    const float *Dl = D + (int64_t)i * y.dsz + dblock_off(l) + (l - mz) * w;
    float dreg[nu];
#pragma unroll
    for (int u = 0; u < nu; ++u) dreg[u] = (lane + 32 * u < nd) ? __ldg(Dl + lane + 32 * u) : 0.f;
    float4 z[nz], q[2 * mm + 1];
#pragma unroll
    for (int m = 0; m < nz; ++m) z[m] = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int m = 0; m < 2 * mm + 1; ++m) q[m] = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int u = 0; u < 3; ++u) {
      if (!t.F[u]) continue;
      const float4 ka = act ? coef4(t.A[u], i, C, c) : make_float4(0.f, 0.f, 0.f, 0.f);
      const float4 kb =
          (u < 2 && act) ? coef4(t.B[u < 2 ? u : 0], i, C, c) : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int m = 0; m < 2 * mm + 1; ++m) {
        const float4 f = act ? load4(reinterpret_cast<const TF *>(t.F[u]) +
                                     (int64_t)i * t.ld[u] + cols[m])
                             : make_float4(0.f, 0.f, 0.f, 0.f);
        z[m - mm + mz].x += ka.x * f.x;
        z[m - mm + mz].y += ka.y * f.y;
        z[m - mm + mz].z += ka.z * f.z;
        z[m - mm + mz].w += ka.w * f.w;
        q[m].x += kb.x * f.x;
        q[m].y += kb.y * f.y;
        q[m].z += kb.z * f.z;
        q[m].w += kb.w * f.w;
      }
    }
    if (wide) {
      const float wx = omega[4 * (int64_t)i], wy = omega[4 * (int64_t)i + 1];
#pragma unroll
      for (int m = -mz; m <= mz; ++m) {
        auto qx = [&](int r) { return (r < -mm || r > mm) ? 0.f : q[r + mm].x; };
        auto qy = [&](int r) { return (r < -mm || r > mm) ? 0.f : q[r + mm].y; };
        auto qz = [&](int r) { return (r < -mm || r > mm) ? 0.f : q[r + mm].z; };
        auto qw = [&](int r) { return (r < -mm || r > mm) ? 0.f : q[r + mm].w; };
        float jx, jy;
        gen_xy(l, m, qx, jx, jy);
        z[m + mz].x -= wx * jx + wy * jy;
        gen_xy(l, m, qy, jx, jy);
        z[m + mz].y -= wx * jx + wy * jy;
        gen_xy(l, m, qz, jx, jy);
        z[m + mz].z -= wx * jx + wy * jy;
        gen_xy(l, m, qw, jx, jy);
        z[m + mz].w -= wx * jx + wy * jy;
      }
    }
    __syncwarp();  // every lane is done reading the previous edge's D rows
#pragma unroll
    for (int u = 0; u < nu; ++u) {
      const int k = lane + 32 * u;
      if (k < nd) dsm[(k / w) * wpad + k % w] = dreg[u];
    }
    __syncwarp();
#pragma unroll
    for (int m = 0; m < nz; ++m) {
#pragma unroll
      for (int q4 = 0; q4 < wpad / 4; ++q4) {
        const float4 d = *reinterpret_cast<const float4 *>(dsm + m * wpad + 4 * q4);
        const float dv[4] = {d.x, d.y, d.z, d.w};
#pragma unroll
        for (int tt = 0; tt < 4; ++tt) {
          const int mp = 4 * q4 + tt;
          if (mp < w) {
            acc[mp].x += dv[tt] * z[m].x;
            acc[mp].y += dv[tt] * z[m].y;
            acc[mp].z += dv[tt] * z[m].z;
            acc[mp].w += dv[tt] * z[m].w;
          }
        }
      }
    }
  }
  if (!act) return;
#pragma unroll
  for (int mp = 0; mp < w; ++mp) {
    float4 *dst = reinterpret_cast<float4 *>(o + (l * l + mp) * C + c);
    float4 v = *dst;
    v.x += acc[mp].x;
    v.y += acc[mp].y;
    v.z += acc[mp].z;
    v.w += acc[mp].w;
    *dst = v;
  }
}

template <int MM, typename TF = float>
__global__ void __launch_bounds__(256, SO2_RN_MINB) k_reduce_nodes_terms(
    Layout y, int64_t e0, int M, const EdgeRec *__restrict__ rec, const int *__restrict__ offsets,
    const float *__restrict__ D, ScatterTerms t, int side, const float *__restrict__ omega,
    float *__restrict__ out) {
  __shared__ __align__(16) float dbuf[8][RN_DBUF];
  if (M <= 0) return;
  const int C = side ? y.co : y.ci;
  const int *col_off = side ? y.kout_off : y.kin_off;
  const bool wide = t.B[0].mode != 0 || t.B[1].mode != 0;
  const int lane = threadIdx.x & 31, wpb = blockDim.x >> 5;
  float *dsm = dbuf[threadIdx.x >> 5];
  const int n_first = rec[0].key, n_last = rec[M - 1].key;
  const int nn = n_last - n_first + 1;
  const int items = nn * (y.L + 1);
  // degree-major item order, highest degree first (as in k_reduce_nodes)
  for (int it = blockIdx.x * wpb + (threadIdx.x >> 5); it < items; it += gridDim.x * wpb) {
    const int n = n_first + it % nn, l = y.L - it / nn;
    int b = offsets[n] - static_cast<int>(e0), e = offsets[n + 1] - static_cast<int>(e0);
    b = b < 0 ? 0 : b;
    e = e > M ? M : e;
    if (b >= e) continue;
    float *o = out + (int64_t)n * y.S * C;
    for (int c0 = 0; c0 < C; c0 += 128) {
      const int c = c0 + 4 * lane;
      const bool act = c < C;
      switch (l) {
        case 0: reduce_level_terms<MM, 0, TF>(y, b, e, C, col_off, D, t, omega, wide, o, c, act, dsm); break;
        case 1: reduce_level_terms<MM, 1, TF>(y, b, e, C, col_off, D, t, omega, wide, o, c, act, dsm); break;
        case 2: reduce_level_terms<MM, 2, TF>(y, b, e, C, col_off, D, t, omega, wide, o, c, act, dsm); break;
        case 3: reduce_level_terms<MM, 3, TF>(y, b, e, C, col_off, D, t, omega, wide, o, c, act, dsm); break;
        case 4: reduce_level_terms<MM, 4, TF>(y, b, e, C, col_off, D, t, omega, wide, o, c, act, dsm); break;
        case 5: reduce_level_terms<MM, 5, TF>(y, b, e, C, col_off, D, t, omega, wide, o, c, act, dsm); break;
        default: reduce_level_terms<MM, 6, TF>(y, b, e, C, col_off, D, t, omega, wide, o, c, act, dsm); break;
      }
    }
  }
}

template <int MM, typename TF = float>
__global__ void __launch_bounds__(256, SO2_RN_MINB) k_reduce_nodes(Layout y, int64_t e0, int M,
                                                      const EdgeRec *__restrict__ rec,
                                                      const int *__restrict__ offsets,
                                                      const float *__restrict__ D,
                                                      const TF *__restrict__ F, int ld,
                                                      const float *__restrict__ coef, int side,
                                                      float *__restrict__ out) {
  __shared__ __align__(16) float dbuf[8][2 * RN_DBUF];
  if (M <= 0) return;
  const int C = side ? y.co : y.ci;
  const int *col_off = side ? y.kout_off : y.kin_off;
  const int lane = threadIdx.x & 31, wpb = blockDim.x >> 5;
  float *dsm = dbuf[threadIdx.x >> 5];
  const int n_first = rec[0].key, n_last = rec[M - 1].key;
  const int nn = n_last - n_first + 1;
  const int items = nn * (y.L + 1);
  // degree-major item order, highest degree first: warps that run at the
  // same time mostly run the same degree's code (instruction cache), and the
  // heaviest items start first
  for (int it = blockIdx.x * wpb + (threadIdx.x >> 5); it < items; it += gridDim.x * wpb) {
    const int n = n_first + it % nn, l = y.L - it / nn;
    int b = offsets[n] - static_cast<int>(e0), e = offsets[n + 1] - static_cast<int>(e0);
    b = b < 0 ? 0 : b;
    e = e > M ? M : e;
    if (b >= e) continue;
    float *o = out + (int64_t)n * y.S * C;
    // warp-uniform channel loop (the level bodies shuffle across the warp)
    for (int c0 = 0; c0 < C; c0 += 128) {
      const int c = c0 + 4 * lane;
      const bool act = c < C;  // C is a multiple of 16, so c + 3 < C too
      switch (l) {
        case 0: reduce_level<MM, 0, TF>(y, b, e, C, col_off, D, F, ld, coef, o, c, act, dsm); break;
        case 1: reduce_level<MM, 1, TF>(y, b, e, C, col_off, D, F, ld, coef, o, c, act, dsm); break;
        case 2: reduce_level<MM, 2, TF>(y, b, e, C, col_off, D, F, ld, coef, o, c, act, dsm); break;
        case 3: reduce_level<MM, 3, TF>(y, b, e, C, col_off, D, F, ld, coef, o, c, act, dsm); break;
        case 4: reduce_level<MM, 4, TF>(y, b, e, C, col_off, D, F, ld, coef, o, c, act, dsm); break;
        case 5: reduce_level<MM, 5, TF>(y, b, e, C, col_off, D, F, ld, coef, o, c, act, dsm); break;
        default: reduce_level<MM, 6, TF>(y, b, e, C, col_off, D, F, ld, coef, o, c, act, dsm); break;
      }
    }
  }
}


// ---------------------------------------------------------------------------
// Inverse rotation on reduction, node-centric.  For every node whose sorted
// segment meets this chunk, out[n][(l,m')][c] += sum over its chunk edges of
// sum_m D^l[m][m'] Z[i][(l,m)][c], Z as described by ScatterTerms.  One block per node,
// threads over channel pairs, the node's sums in shared memory; the chunks
// run in stream order, so every output element is updated by one thread at
// a time and the sum order is fixed.
// ---------------------------------------------------------------------------
template <int MM, typename TF = float>
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
              const float2 f = load2(reinterpret_cast<const TF *>(t.F[u]) + (int64_t)i * t.ld[u] +
                                     col_off[g] + j * C + c);
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

// transposed = 0: stacked [n][k] planes (coalesced over k); transposed = 1:
// their transposes [k][n] (coalesced over n).
template <typename TW>
__global__ void k_pack_weights(Layout y, BlockOffsets bo, const TW *__restrict__ w, int transposed,
                               __nv_bfloat16 *__restrict__ hi, __nv_bfloat16 *__restrict__ lo) {
  const int g = blockIdx.y;
  if (g >= y.ng) return;
  const int64_t total = (int64_t)y.Kout[g] * y.Kin[g];
  for (int64_t t = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; t < total;
       t += (int64_t)gridDim.x * blockDim.x) {
    int n, k;
    if (transposed) {
      k = static_cast<int>(t / y.Kout[g]);
      n = static_cast<int>(t % y.Kout[g]);
    } else {
      n = static_cast<int>(t / y.Kin[g]);
      k = static_cast<int>(t % y.Kin[g]);
    }
    const float v = stacked_w(y, w, bo.off, g, n, k);
    __nv_bfloat16 h, l;
    split_bf16(v, h, l);
    const int64_t a = transposed ? (int64_t)(y.wt_off[g] + k) * y.WTK + n
                                 : (int64_t)(y.wr_off[g] + n) * y.WK + k;
    hi[a] = h;
    if (lo) lo[a] = l;
  }
}

// d(stacked) -> packed gradient blocks: W0 directly; for g >= 1
// grad W1 = A + D, grad W2 = C - B where d(stacked) = [[A, B], [C, D]].
static __global__ void k_unstack_grad(Layout y, BlockOffsets bo, const float *__restrict__ dws,
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
// PART: 3 = both sides in one pass; 1 = output side only (writes Gg and the
// record h); 2 = input side only (adds its share to h and finishes the edge's
// gradient).  With gv_hi, the output side also writes g * (D G[dst]) on the
// kept rows as the transposed product's operand planes (what rotation on
// gather of G would write).
//
// The record h[i] = (h_x, h_y, dd, -) carries the edge's sums from the output
// side to the input side, where
//   dL/dr = R^T (-h_y, h_x, 0) / d + dd r_hat,
//   dd = sum_c' Gg[c'] sum_k W_rad[k][c'] phi'_k(d)
// (the frame part through the rotation generators, the gate part through the
// derivative of the radial basis).  grad_r (indexed by the caller's edge id)
// is written when the input side runs and grad_r is given.
template <typename TX, int MM, int LC = -1, int PART = 3, typename TF = float>
__global__ void __launch_bounds__(256, LC >= 0 ? SO2_ET_MINB_LC : SO2_GATHER_MINB) k_edge_terms(Layout y, int M, const EdgeRec *__restrict__ rec,
                             const float *__restrict__ D, const float *__restrict__ gate,
                             const float *__restrict__ G, const TX *__restrict__ X,
                             const TF *__restrict__ V, const TF *__restrict__ Ga,
                             float *__restrict__ Gg, float4 *__restrict__ h,
                             __nv_bfloat16 *__restrict__ gv_hi, __nv_bfloat16 *__restrict__ gv_lo,
                             const float *__restrict__ geo, const float *__restrict__ w_rad,
                             float cutoff, float *__restrict__ grad_r) {
  constexpr int W = MM + 1;  // widest |m| needed by the generators
  extern __shared__ float sDall[];  // [warps][dsz + RAD_MAX_NR]
  const int lane = threadIdx.x & 31, wpb = blockDim.x >> 5;
  float *sD = sDall + (threadIdx.x >> 5) * (y.dsz + RAD_MAX_NR);
  float *sPhi = sD + y.dsz;  // phi'_k(d) of the warp's edge
  const float sig = cutoff / static_cast<float>(y.nr - 1);
  for (int i = blockIdx.x * wpb + (threadIdx.x >> 5); i < M; i += gridDim.x * wpb) {
    const EdgeRec r = rec[i];
    __syncwarp();
    stage_d(D + (int64_t)i * y.dsz, y.dsz, sD);
    float hx = 0.f, hy = 0.f, dd = 0.f;
    if (PART & 1) {  // phi'_k(d), for the output side's gate part
      const float d = geo[(int64_t)i * GEO];
      for (int k = lane; k < y.nr; k += 32) {
        const float t = (d - sig * static_cast<float>(k)) / sig;
        sPhi[k] = (-t / sig) * __expf(-0.5f * t * t);
      }
      __syncwarp();
    }
    // output side
    const float *Gn = G + (int64_t)r.dst * y.S * y.co;
    const TF *Vi = V + (int64_t)i * y.KG;
    for (int c = 4 * lane; (PART & 1) && c < y.co; c += 128) {
      const float4 gv = load4(gate + (int64_t)i * y.co + c);
      float4 gg = make_float4(0.f, 0.f, 0.f, 0.f);
      each_level<LC>(y.L, [&](auto lv) {
        constexpr int l = decltype(lv)::value;
        constexpr int w = 2 * l + 1;
        constexpr int mw = W < l ? W : l, mm = MM < l ? MM : l;
        float4 b[2 * W + 1];
#pragma unroll
        for (int k = 0; k < 2 * W + 1; ++k) b[k] = make_float4(0.f, 0.f, 0.f, 0.f);
        const float *Dl = sD + dblock_off(l);
#pragma unroll
        for (int mp = -l; mp <= l; ++mp) {
          if (et_fence<LC>(l, mp)) load_fence();
          const float4 gx = load4(Gn + (l * l + l + mp) * y.co + c);
#pragma unroll
          for (int m = -mw; m <= mw; ++m) {
            const float dv = Dl[(m + l) * w + mp + l];
            b[m + W].x += dv * gx.x;
            b[m + W].y += dv * gx.y;
            b[m + W].z += dv * gx.z;
            b[m + W].w += dv * gx.w;
          }
        }
#pragma unroll
        for (int m = -mm; m <= mm; ++m) {
          int g, j;
          lm_group_row(y, l, m, g, j);
          if (gv_hi) {  // the output-side operand g * (D G[dst]) of the transposed product
            const int64_t col = (int64_t)i * y.KG + y.kout_off[g] + j * y.co + c;
            store_split4(gv_hi + col, gv_lo ? gv_lo + col : nullptr,
                         make_float4(gv.x * b[m + W].x, gv.y * b[m + W].y, gv.z * b[m + W].z,
                                     gv.w * b[m + W].w));
          }
          const float4 v = load4(Vi + y.kout_off[g] + j * y.co + c);
          gg.x += b[m + W].x * v.x;
          gg.y += b[m + W].y * v.y;
          gg.z += b[m + W].z * v.z;
          gg.w += b[m + W].w * v.w;
          float jx, jy;
          gen_xy(l, m, [&](int q) { return b[q + W].x; }, jx, jy);
          hx += gv.x * v.x * jx;
          hy += gv.x * v.x * jy;
          gen_xy(l, m, [&](int q) { return b[q + W].y; }, jx, jy);
          hx += gv.y * v.y * jx;
          hy += gv.y * v.y * jy;
          gen_xy(l, m, [&](int q) { return b[q + W].z; }, jx, jy);
          hx += gv.z * v.z * jx;
          hy += gv.z * v.z * jy;
          gen_xy(l, m, [&](int q) { return b[q + W].w; }, jx, jy);
          hx += gv.w * v.w * jx;
          hy += gv.w * v.w * jy;
        }
      });
      *reinterpret_cast<float4 *>(Gg + (int64_t)i * y.co + c) = gg;
      // dd share of these four channels: Gg . (W_rad^T phi'(d))
      float4 dg = make_float4(0.f, 0.f, 0.f, 0.f);
      for (int k = 0; k < y.nr; ++k) {
        const float dk = sPhi[k];
        const float4 wk = __ldg(reinterpret_cast<const float4 *>(w_rad + (int64_t)k * y.co + c));
        dg.x += wk.x * dk;
        dg.y += wk.y * dk;
        dg.z += wk.z * dk;
        dg.w += wk.w * dk;
      }
      dd += gg.x * dg.x + gg.y * dg.y + gg.z * dg.z + gg.w * dg.w;
    }
    if ((PART & 1) && gv_hi) {
      for (int g = 0; g < y.ng; ++g)
        for (int k = y.rows[g] * y.co + 4 * lane; k < y.Kout_pad[g]; k += 128) {
          const int64_t col = (int64_t)i * y.KG + y.kout_off[g] + k;
          store_split4(gv_hi + col, gv_lo ? gv_lo + col : nullptr, make_float4(0.f, 0.f, 0.f, 0.f));
        }
    }
    // input side
    const TX *Xn = X + (int64_t)r.src * y.S * y.ci;
    const TF *Gai = Ga + (int64_t)i * y.KA;
    for (int c = 4 * lane; (PART & 2) && c < y.ci; c += 128) {
      each_level<LC>(y.L, [&](auto lv) {
        constexpr int l = decltype(lv)::value;
        constexpr int w = 2 * l + 1;
        constexpr int mw = W < l ? W : l, mm = MM < l ? MM : l;
        float4 b[2 * W + 1];
#pragma unroll
        for (int k = 0; k < 2 * W + 1; ++k) b[k] = make_float4(0.f, 0.f, 0.f, 0.f);
        const float *Dl = sD + dblock_off(l);
#pragma unroll
        for (int mp = -l; mp <= l; ++mp) {
          if (et_fence<LC>(l, mp)) load_fence();
          const float4 xv = load4(Xn + (l * l + l + mp) * y.ci + c);
#pragma unroll
          for (int m = -mw; m <= mw; ++m) {
            const float dv = Dl[(m + l) * w + mp + l];
            b[m + W].x += dv * xv.x;
            b[m + W].y += dv * xv.y;
            b[m + W].z += dv * xv.z;
            b[m + W].w += dv * xv.w;
          }
        }
#pragma unroll
        for (int m = -mm; m <= mm; ++m) {
          int g, j;
          lm_group_row(y, l, m, g, j);
          const float4 ga = load4(Gai + y.kin_off[g] + j * y.ci + c);
          float jx, jy;
          gen_xy(l, m, [&](int q) { return b[q + W].x; }, jx, jy);
          hx += ga.x * jx;
          hy += ga.x * jy;
          gen_xy(l, m, [&](int q) { return b[q + W].y; }, jx, jy);
          hx += ga.y * jx;
          hy += ga.y * jy;
          gen_xy(l, m, [&](int q) { return b[q + W].z; }, jx, jy);
          hx += ga.z * jx;
          hy += ga.z * jy;
          gen_xy(l, m, [&](int q) { return b[q + W].w; }, jx, jy);
          hx += ga.w * jx;
          hy += ga.w * jy;
        }
      });
    }
    for (int o = 16; o > 0; o >>= 1) {
      hx += __shfl_xor_sync(0xffffffffu, hx, o);
      hy += __shfl_xor_sync(0xffffffffu, hy, o);
      dd += __shfl_xor_sync(0xffffffffu, dd, o);
    }
    if (lane == 0) {
      if (!(PART & 1)) {  // the output side's sums
        const float4 ho = h[i];
        hx += ho.x;
        hy += ho.y;
        dd = ho.z;
      }
      if ((PART & 2) && grad_r) {
        const float *gr = geo + (int64_t)i * GEO;
        const float d = gr[0];
        const float inv = d > 0.f ? 1.f / d : 0.f;
        const float *R = gr + 4;
        for (int a = 0; a < 3; ++a)
          grad_r[3 * (int64_t)r.eid + a] =
              (R[0 * 3 + a] * (-hy) + R[1 * 3 + a] * hx) * inv + dd * gr[1 + a];
      } else {
        h[i] = make_float4(hx, hy, dd, 0.f);
      }
    }
  }
}

// Radial-gate gradients, stage 1: each block sums, over a tile of RAD_TILE
// edges, phi_k(d_i) A[i][c'] + phi'_k(d_i) dd_i B[i][c'] (rows k < nr) and
// A[i][c'] (bias row k = nr) into part[block][k][c'].  B (and dd_i =
// omega[i][2]) is optional.  One thread per channel keeps all nr + 1 sums
// in registers and reads each product once.  Stage 2 adds the blocks in
// order.
constexpr int RAD_TILE = 64;
static __global__ void k_rad_partial(Layout y, float cutoff, int M, const float *__restrict__ geo,
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
  for (int c = threadIdx.x; c < y.co; c += blockDim.x) {
    for (int k0 = 0; k0 < y.nr; k0 += 16) {  // 16 radial sums per pass
      float acc[16], bias = 0.f;
#pragma unroll
      for (int k = 0; k < 16; ++k) acc[k] = 0.f;
      auto add = [&](int i, float a, float b) {
        bias += a;
#pragma unroll
        for (int k = 0; k < 16; ++k) {
          if (k0 + k < y.nr) {
            acc[k] += phi[i * y.nr + k0 + k] * a;
            if (Bg) acc[k] += dphi[i * y.nr + k0 + k] * b;
          }
        }
      };
      // four edges' loads in flight before their (in-order) sums
      int i = 0;
      for (; i + 4 <= n; i += 4) {
        float a[4], b[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          a[u] = Ag[(int64_t)(i0 + i + u) * y.co + c];
          b[u] = Bg ? Bg[(int64_t)(i0 + i + u) * y.co + c] : 0.f;
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) add(i + u, a[u], b[u]);
      }
      for (; i < n; ++i)
        add(i, Ag[(int64_t)(i0 + i) * y.co + c], Bg ? Bg[(int64_t)(i0 + i) * y.co + c] : 0.f);
#pragma unroll
      for (int k = 0; k < 16; ++k)
        if (k0 + k < y.nr) part[(int64_t)blockIdx.x * P + (k0 + k) * y.co + c] = acc[k];
      if (k0 == 0) part[(int64_t)blockIdx.x * P + y.nr * y.co + c] = bias;
    }
  }
}

// Stage 2: block = 32 consecutive (k, c') entries x RAD_RED_WARPS warps; each
// warp sums a strided share of the blocks' partials (four loads in flight),
// then the shares are added in a fixed order.
constexpr int RAD_RED_WARPS = 32;
static __global__ void __launch_bounds__(32 * RAD_RED_WARPS)
    k_rad_reduce(Layout y, int nblk, const float *__restrict__ part,
                 float *__restrict__ grad_w_rad, float *__restrict__ grad_b) {
  __shared__ float red[RAD_RED_WARPS][32];
  const int P = (y.nr + 1) * y.co;
  const int pidx = blockIdx.x * 32 + (threadIdx.x & 31);
  const int w = threadIdx.x >> 5;
  float s = 0.f;
  if (pidx < P) {
#pragma unroll 4
    for (int b = w; b < nblk; b += RAD_RED_WARPS) s += part[(int64_t)b * P + pidx];
  }
  red[w][threadIdx.x & 31] = s;
  __syncthreads();
  if (w == 0 && pidx < P) {
    float t = 0.f;
    for (int u = 0; u < RAD_RED_WARPS; ++u) t += red[u][threadIdx.x];
    const int k = pidx / y.co, c = pidx % y.co;
    if (k < y.nr) {
      if (grad_w_rad) grad_w_rad[k * y.co + c] += t;
    } else if (grad_b) {
      grad_b[c] += t;
    }
  }
}

// ---------------------------------------------------------------------------
// Double backward, per edge: the frame turn and gate change that the edge
// cotangent gg_r induces.  With u = R gg_r / d: omega = (u_y, -u_x) (the
// z component, a roll of the frame, does not change the output),
// dd = r_hat . gg_r and dg[c'] = dd * sum_k W_rad[k][c'] phi'_k(d).
// omega[i] = (w_x, w_y, dd, 0).  One warp per edge.
// ---------------------------------------------------------------------------
static __global__ void k_edge_omega(Layout y, float cutoff, int M, const EdgeRec *__restrict__ rec,
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
// V~ = M(D gg_x[src]) (optional).  One warp per edge, four channels per lane,
// D staged in shared memory, degrees compile-time as in k_edge_terms.
template <int MM, int LC = -1, typename TF = float>
__global__ void __launch_bounds__(256, LC >= 0 ? SO2_ET_MINB_LC : SO2_GATHER_MINB)
    k_edge_terms2(Layout y, int M, const EdgeRec *__restrict__ rec, const float *__restrict__ D,
                  const float *__restrict__ G, const float *__restrict__ omega,
                  const TF *__restrict__ V, const TF *__restrict__ dV,
                  const TF *__restrict__ Vt, float *__restrict__ Aout,
                  float *__restrict__ Bout) {
  constexpr int W = MM + 1;
  extern __shared__ float sDall[];  // [warps][dsz]
  const int lane = threadIdx.x & 31, wpb = blockDim.x >> 5;
  float *sD = sDall + (threadIdx.x >> 5) * y.dsz;
  for (int i = blockIdx.x * wpb + (threadIdx.x >> 5); i < M; i += gridDim.x * wpb) {
    const EdgeRec r = rec[i];
    __syncwarp();
    stage_d(D + (int64_t)i * y.dsz, y.dsz, sD);
    const float *Gn = G + (int64_t)r.dst * y.S * y.co;
    const float wx = omega ? omega[4 * (int64_t)i] : 0.f;
    const float wy = omega ? omega[4 * (int64_t)i + 1] : 0.f;
    const int64_t ro = (int64_t)i * y.KG;
    for (int c = 4 * lane; c < y.co; c += 128) {
      float4 Aa = make_float4(0.f, 0.f, 0.f, 0.f), Bb = make_float4(0.f, 0.f, 0.f, 0.f);
      each_level<LC>(y.L, [&](auto lv) {
        constexpr int l = decltype(lv)::value;
        constexpr int w = 2 * l + 1;
        constexpr int mw = W < l ? W : l, mm = MM < l ? MM : l;
        float4 b[2 * W + 1];
#pragma unroll
        for (int k = 0; k < 2 * W + 1; ++k) b[k] = make_float4(0.f, 0.f, 0.f, 0.f);
        const float *Dl = sD + dblock_off(l);
#pragma unroll
        for (int mp = -l; mp <= l; ++mp) {
          if (et_fence<LC>(l, mp)) load_fence();
          const float4 gx = load4(Gn + (l * l + l + mp) * y.co + c);
#pragma unroll
          for (int m = -mw; m <= mw; ++m) {
            const float dv = Dl[(m + l) * w + mp + l];
            b[m + W].x += dv * gx.x;
            b[m + W].y += dv * gx.y;
            b[m + W].z += dv * gx.z;
            b[m + W].w += dv * gx.w;
          }
        }
#pragma unroll
        for (int m = -mm; m <= mm; ++m) {
          int g, j;
          lm_group_row(y, l, m, g, j);
          const int64_t col = ro + y.kout_off[g] + j * y.co + c;
          const float4 v = load4(V + col);
          const float4 dv = dV ? load4(dV + col) : make_float4(0.f, 0.f, 0.f, 0.f);
          const float4 vt = Vt ? load4(Vt + col) : make_float4(0.f, 0.f, 0.f, 0.f);
          float4 og;  // (Omega Gy~)[m]
          float jx, jy;
          gen_xy(l, m, [&](int q) { return b[q + W].x; }, jx, jy);
          og.x = wx * jx + wy * jy;
          gen_xy(l, m, [&](int q) { return b[q + W].y; }, jx, jy);
          og.y = wx * jx + wy * jy;
          gen_xy(l, m, [&](int q) { return b[q + W].z; }, jx, jy);
          og.z = wx * jx + wy * jy;
          gen_xy(l, m, [&](int q) { return b[q + W].w; }, jx, jy);
          og.w = wx * jx + wy * jy;
          const float4 bm = b[m + W];
          Aa.x += og.x * v.x + bm.x * (dv.x + vt.x);
          Aa.y += og.y * v.y + bm.y * (dv.y + vt.y);
          Aa.z += og.z * v.z + bm.z * (dv.z + vt.z);
          Aa.w += og.w * v.w + bm.w * (dv.w + vt.w);
          Bb.x += bm.x * v.x;
          Bb.y += bm.y * v.y;
          Bb.z += bm.z * v.z;
          Bb.w += bm.w * v.w;
        }
      });
      *reinterpret_cast<float4 *>(Aout + (int64_t)i * y.co + c) = Aa;
      *reinterpret_cast<float4 *>(Bout + (int64_t)i * y.co + c) = Bb;
    }
  }
}

// ---------------------------------------------------------------------------
// Second order in the edge vectors (d_edge_vec of the double backward).
//
// With u = gg_r (the cotangent on grad_edge_vec) and ~x = gg_x,
//   d_edge_vec_e = H_e u_e + dL_e/dr_e |_{x := ~x},
// H_e the Hessian of the edge's share L_e = <b, g * V> of <grad_out, out>
// (b = trunc(D G[dst]), V = M trunc(D x[src])).  In the edge frame (R r_hat =
// z_hat, U = R u) a second direction W turns the frame by
//   omega_W = (W_y, -W_x) / d,   and jointly with u by
//   omega_uW = -(W_z omega_u + U_z omega_W) / d,
// so d2D[u, W] = (Omega_uW + (Omega_u Omega_W + Omega_W Omega_u) / 2) D (the
// roll parts drop out: L_e does not depend on the roll), and the gate moves
// by g_W = g' W_z, g_uW = g'' U_z W_z + g' (U_perp . W_perp) / d.  For the
// edge-frame axes W = x, y, z this gives (with J_x, J_y the generators,
// Omega_u = alpha J_x + beta J_y, (alpha, beta) = omega_u):
//   X_x = (U_z/d^2) J_y - (alpha / 2d)(J_x J_y + J_y J_x) - (beta/d) J_y^2
//   X_y = -(U_z/d^2) J_x + (alpha/d) J_x^2 + (beta / 2d)(J_x J_y + J_y J_x)
//   q_z = -F_D[Omega_u]/d + <Omega_u b, g' V> + <g' b, dV> + U_z <g'', Gg>
//   q_x = F_D[X_x] + <g (-J_y b / d), dV> + U_z <(-J_y b / d), g' V>
//         + <M^T P, -J_y a / d> + (U_x / d) <g', Gg>
//   q_y = F_D[X_y] + <g (J_x b / d), dV> + U_z <(J_x b / d), g' V>
//         + <M^T P, J_x a / d> + (U_y / d) <g', Gg>
// where F_D[X] = <X b, g V> + <Ga, X a>, a = trunc(D x), dV = M trunc(Omega_u
// D x), Ga = M^T (g b), M^T P = M^T (g Omega_u b + g_u b) (the double
// backward's products) and Gg[c'] = sum_rows b V.  The ~x part is the first
// backward's edge gradient: (-h_y / d, h_x / d, <g', sum_rows b ~V>) with
// h_k = <g ~V, J_k b> + <Ga, J_k ~a>, ~a = trunc(D ~x), ~V = M ~a.
// H u = R^T q.  The terms split by what they read: the output side (b, V,
// dV, ~V; destination order) and the input side (a, ~a, Ga, M^T P; source
// order); each side adds R^T of its share onto d_edge_vec[eid].
// ---------------------------------------------------------------------------

// First- and second-order generator rows of one degree-l coefficient vector
// (zero outside |q| <= l): for |m| <= MM, jx = (J_x c)[m], jy = (J_y c)[m],
// xx = (J_x J_x c)[m], yy = (J_y J_y c)[m], sym = ((J_x J_y + J_y J_x) c)[m].
// c holds rows |q| <= MM + 2 (index q + MM + 2); the first-order rows at
// |q| <= MM + 1 are formed once and the second generator is applied to them.
template <int MM>
struct GenRows {
  float jx[2 * MM + 1], jy[2 * MM + 1], xx[2 * MM + 1], yy[2 * MM + 1], sym[2 * MM + 1];
};
template <int MM>
__device__ __forceinline__ void gen_rows2(int l, const float (&c)[2 * MM + 5], GenRows<MM> &o) {
  constexpr int W1 = MM + 1, W2 = MM + 2;
  auto cc = [&](int q) { return (q < -l || q > l || q < -W2 || q > W2) ? 0.f : c[q + W2]; };
  float fx[2 * W1 + 1], fy[2 * W1 + 1];
#pragma unroll
  for (int q = -W1; q <= W1; ++q) {
    fx[q + W1] = 0.f;
    fy[q + W1] = 0.f;
    if (q >= -l && q <= l) gen_xy(l, q, cc, fx[q + W1], fy[q + W1]);
  }
  auto ax = [&](int q) { return (q < -l || q > l || q < -W1 || q > W1) ? 0.f : fx[q + W1]; };
  auto ay = [&](int q) { return (q < -l || q > l || q < -W1 || q > W1) ? 0.f : fy[q + W1]; };
#pragma unroll
  for (int m = -MM; m <= MM; ++m) {
    o.jx[m + MM] = fx[m + W1];
    o.jy[m + MM] = fy[m + W1];
    float yx = 0.f, xy = 0.f;
    o.xx[m + MM] = 0.f;
    o.yy[m + MM] = 0.f;
    if (m >= -l && m <= l) {
      gen_xy(l, m, ax, o.xx[m + MM], yx);  // J_x J_x c, J_y J_x c
      gen_xy(l, m, ay, xy, o.yy[m + MM]);  // J_x J_y c, J_y J_y c
    }
    o.sym[m + MM] = xy + yx;
  }
}

__device__ __forceinline__ float comp4(const float4 &v, int k) {
  return k == 0 ? v.x : (k == 1 ? v.y : (k == 2 ? v.z : v.w));
}
__device__ __forceinline__ void acc4(float4 &v, int k, float a) {
  if (k == 0) v.x += a;
  else if (k == 1) v.y += a;
  else if (k == 2) v.z += a;
  else v.w += a;
}

// The edge-frame share q (3 floats, summed over the warp) rotated back and
// added onto d_edge_vec[eid] (one writer per edge per launch; launches run in
// stream order).
__device__ __forceinline__ void hess_flush(const float *gr, int eid, float qx, float qy, float qz,
                                           float *__restrict__ d_r) {
  const float *R = gr + 4;
#pragma unroll
  for (int a = 0; a < 3; ++a)
    d_r[3 * (int64_t)eid + a] += R[0 * 3 + a] * qx + R[1 * 3 + a] * qy + R[2 * 3 + a] * qz;
}

// Output side, destination order.  omega (w_x, w_y, U_z per edge) and dV are
// given with an edge-vector cotangent, Vt with gg_x.
template <int MM, int LC = -1, typename TF = float>
__global__ void __launch_bounds__(256, LC >= 0 ? SO2_ET_MINB_LC : SO2_GATHER_MINB)
    k_edge_hess_out(Layout y, float cutoff, int M, const EdgeRec *__restrict__ rec,
                    const float *__restrict__ D, const float *__restrict__ geo,
                    const float *__restrict__ gate, const float *__restrict__ G,
                    const float *__restrict__ omega, const TF *__restrict__ V,
                    const TF *__restrict__ dV, const TF *__restrict__ Vt,
                    const float *__restrict__ w_rad, float *__restrict__ d_r) {
  constexpr int W2 = MM + 2;
  extern __shared__ float sDall[];  // [warps][dsz + 2 RAD_MAX_NR]
  const int lane = threadIdx.x & 31, wpb = blockDim.x >> 5;
  float *sD = sDall + (threadIdx.x >> 5) * (y.dsz + 2 * RAD_MAX_NR);
  float *sP1 = sD + y.dsz, *sP2 = sP1 + RAD_MAX_NR;  // phi'_k(d), phi''_k(d)
  const float sig = cutoff / static_cast<float>(y.nr - 1);
  for (int i = blockIdx.x * wpb + (threadIdx.x >> 5); i < M; i += gridDim.x * wpb) {
    const EdgeRec r = rec[i];
    __syncwarp();
    stage_d(D + (int64_t)i * y.dsz, y.dsz, sD);
    const float *gr = geo + (int64_t)i * GEO;
    const float d = gr[0];
    const float inv = d > 0.f ? 1.f / d : 0.f;
    const float al = omega ? omega[4 * (int64_t)i] : 0.f;
    const float be = omega ? omega[4 * (int64_t)i + 1] : 0.f;
    const float Uz = omega ? omega[4 * (int64_t)i + 2] : 0.f;
    const float Ux = -be * d, Uy = al * d;
    for (int k = lane; k < y.nr; k += 32) {
      const float t = (d - sig * static_cast<float>(k)) / sig;
      const float ph = __expf(-0.5f * t * t);
      sP1[k] = (-t / sig) * ph;
      sP2[k] = ((t * t - 1.f) / (sig * sig)) * ph;
    }
    __syncwarp();
    const float *Gn = G + (int64_t)r.dst * y.S * y.co;
    const int64_t ro = (int64_t)i * y.KG;
    float qx = 0.f, qy = 0.f, qz = 0.f, hx = 0.f, hy = 0.f;
    for (int c = 4 * lane; c < y.co; c += 128) {
      const float4 g4 = load4(gate + (int64_t)i * y.co + c);
      float4 gp4 = make_float4(0.f, 0.f, 0.f, 0.f), gpp4 = gp4;
      for (int k = 0; k < y.nr; ++k) {
        const float4 wk = __ldg(reinterpret_cast<const float4 *>(w_rad + (int64_t)k * y.co + c));
        const float p1 = sP1[k], p2 = sP2[k];
        gp4.x += wk.x * p1;
        gp4.y += wk.y * p1;
        gp4.z += wk.z * p1;
        gp4.w += wk.w * p1;
        gpp4.x += wk.x * p2;
        gpp4.y += wk.y * p2;
        gpp4.z += wk.z * p2;
        gpp4.w += wk.w * p2;
      }
      float4 Gg = make_float4(0.f, 0.f, 0.f, 0.f), Ggt = Gg;
      each_level<LC>(y.L, [&](auto lv) {
        constexpr int l = decltype(lv)::value;
        constexpr int w = 2 * l + 1;
        constexpr int mb = W2 < l ? W2 : l, mm = MM < l ? MM : l;
        float4 b[2 * W2 + 1];
#pragma unroll
        for (int k = 0; k < 2 * W2 + 1; ++k) b[k] = make_float4(0.f, 0.f, 0.f, 0.f);
        const float *Dl = sD + dblock_off(l);
#pragma unroll
        for (int mp = -l; mp <= l; ++mp) {
          const float4 gx = load4(Gn + (l * l + l + mp) * y.co + c);
#pragma unroll
          for (int m = -mb; m <= mb; ++m) {
            const float dv = Dl[(m + l) * w + mp + l];
            b[m + W2].x += dv * gx.x;
            b[m + W2].y += dv * gx.y;
            b[m + W2].z += dv * gx.z;
            b[m + W2].w += dv * gx.w;
          }
        }
#pragma unroll 1
        for (int k = 0; k < 4; ++k) {
          float bk[2 * W2 + 1];
#pragma unroll
          for (int q = 0; q < 2 * W2 + 1; ++q) bk[q] = comp4(b[q], k);
          GenRows<MM> gr2;
          gen_rows2<MM>(l, bk, gr2);
          const float gk = comp4(g4, k), gpk = comp4(gp4, k);
#pragma unroll
          for (int m = -mm; m <= mm; ++m) {
            int g, j;
            lm_group_row(y, l, m, g, j);
            const int64_t col = ro + y.kout_off[g] + j * y.co + c;
            const float v = comp4(load4(V + col), k);
            const float dvv = dV ? comp4(load4(dV + col), k) : 0.f;
            const float vt = Vt ? comp4(load4(Vt + col), k) : 0.f;
            const float jx = gr2.jx[m + MM], jy = gr2.jy[m + MM];
            const float xx = gr2.xx[m + MM], yy = gr2.yy[m + MM], sym = gr2.sym[m + MM];
            const float bm = bk[m + W2];
            const float gv = gk * v, gpv = gpk * v;
            const float ob = al * jx + be * jy;  // (Omega_u b)[m]
            const float xxb = Uz * inv * inv * jy - 0.5f * al * inv * sym - be * inv * yy;
            const float xyb = -Uz * inv * inv * jx + al * inv * xx + 0.5f * be * inv * sym;
            qz += -inv * ob * gv + ob * gpv + gpk * bm * dvv;
            qx += xxb * gv - inv * jy * (gk * dvv + Uz * gpv);
            qy += xyb * gv + inv * jx * (gk * dvv + Uz * gpv);
            acc4(Gg, k, bm * v);
            acc4(Ggt, k, bm * vt);
            hx += gk * vt * jx;
            hy += gk * vt * jy;
          }
        }
      });
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const float gpk = comp4(gp4, k), gppk = comp4(gpp4, k), ggk = comp4(Gg, k);
        qz += Uz * gppk * ggk + gpk * comp4(Ggt, k);
        qx += Ux * inv * gpk * ggk;
        qy += Uy * inv * gpk * ggk;
      }
    }
    for (int o = 16; o > 0; o >>= 1) {
      qx += __shfl_xor_sync(0xffffffffu, qx, o);
      qy += __shfl_xor_sync(0xffffffffu, qy, o);
      qz += __shfl_xor_sync(0xffffffffu, qz, o);
      hx += __shfl_xor_sync(0xffffffffu, hx, o);
      hy += __shfl_xor_sync(0xffffffffu, hy, o);
    }
    if (lane == 0) hess_flush(gr, r.eid, qx - hy * inv, qy + hx * inv, qz, d_r);
  }
}

// Input side, source order.  omega and MP (= M^T P) are given with an
// edge-vector cotangent, GX (= gg_x) with a node cotangent; Ga = M^T (g b).
template <typename TX, int MM, int LC = -1, typename TF = float>
__global__ void __launch_bounds__(256, LC >= 0 ? SO2_ET_MINB_LC : SO2_GATHER_MINB)
    k_edge_hess_in(Layout y, int M, const EdgeRec *__restrict__ rec, const float *__restrict__ D,
                   const float *__restrict__ geo, const TX *__restrict__ X,
                   const float *__restrict__ GX, const float *__restrict__ omega,
                   const TF *__restrict__ Ga, const TF *__restrict__ MP,
                   float *__restrict__ d_r) {
  constexpr int W2 = MM + 2;
  extern __shared__ float sDall[];  // [warps][dsz]
  const int lane = threadIdx.x & 31, wpb = blockDim.x >> 5;
  float *sD = sDall + (threadIdx.x >> 5) * y.dsz;
  for (int i = blockIdx.x * wpb + (threadIdx.x >> 5); i < M; i += gridDim.x * wpb) {
    const EdgeRec r = rec[i];
    __syncwarp();
    stage_d(D + (int64_t)i * y.dsz, y.dsz, sD);
    const float *gr = geo + (int64_t)i * GEO;
    const float d = gr[0];
    const float inv = d > 0.f ? 1.f / d : 0.f;
    const float al = omega ? omega[4 * (int64_t)i] : 0.f;
    const float be = omega ? omega[4 * (int64_t)i + 1] : 0.f;
    const float Uz = omega ? omega[4 * (int64_t)i + 2] : 0.f;
    const TX *Xn = X + (int64_t)r.src * y.S * y.ci;
    const float *GXn = GX ? GX + (int64_t)r.src * y.S * y.ci : nullptr;
    const int64_t ro = (int64_t)i * y.KA;
    float qx = 0.f, qy = 0.f, qz = 0.f, hx = 0.f, hy = 0.f;
    for (int c = 4 * lane; c < y.ci; c += 128) {
      each_level<LC>(y.L, [&](auto lv) {
        constexpr int l = decltype(lv)::value;
        constexpr int w = 2 * l + 1;
        constexpr int mb = W2 < l ? W2 : l, mm = MM < l ? MM : l;
        float4 a[2 * W2 + 1], at[2 * W2 + 1];
#pragma unroll
        for (int k = 0; k < 2 * W2 + 1; ++k) {
          a[k] = make_float4(0.f, 0.f, 0.f, 0.f);
          at[k] = a[k];
        }
        const float *Dl = sD + dblock_off(l);
#pragma unroll
        for (int mp = -l; mp <= l; ++mp) {
          const float4 xv = load4(Xn + (l * l + l + mp) * y.ci + c);
          const float4 tv = GXn ? load4(GXn + (l * l + l + mp) * y.ci + c)
                                : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
          for (int m = -mb; m <= mb; ++m) {
            const float dv = Dl[(m + l) * w + mp + l];
            a[m + W2].x += dv * xv.x;
            a[m + W2].y += dv * xv.y;
            a[m + W2].z += dv * xv.z;
            a[m + W2].w += dv * xv.w;
            at[m + W2].x += dv * tv.x;
            at[m + W2].y += dv * tv.y;
            at[m + W2].z += dv * tv.z;
            at[m + W2].w += dv * tv.w;
          }
        }
#pragma unroll 1
        for (int k = 0; k < 4; ++k) {
          float ak[2 * W2 + 1], tk[2 * W2 + 1];
#pragma unroll
          for (int q = 0; q < 2 * W2 + 1; ++q) {
            ak[q] = comp4(a[q], k);
            tk[q] = comp4(at[q], k);
          }
          GenRows<MM> ga2;
          gen_rows2<MM>(l, ak, ga2);
          auto tq = [&](int q) { return (q < -mb || q > mb) ? 0.f : tk[q + W2]; };
#pragma unroll
          for (int m = -mm; m <= mm; ++m) {
            int g, j;
            lm_group_row(y, l, m, g, j);
            const int64_t col = ro + y.kin_off[g] + j * y.ci + c;
            const float ga = comp4(load4(Ga + col), k);
            const float mpv = MP ? comp4(load4(MP + col), k) : 0.f;
            float tx, ty;
            gen_xy(l, m, tq, tx, ty);
            const float jx = ga2.jx[m + MM], jy = ga2.jy[m + MM];
            const float xx = ga2.xx[m + MM], yy = ga2.yy[m + MM], sym = ga2.sym[m + MM];
            const float oa = al * jx + be * jy;  // (Omega_u a)[m]
            const float xxa = Uz * inv * inv * jy - 0.5f * al * inv * sym - be * inv * yy;
            const float xya = -Uz * inv * inv * jx + al * inv * xx + 0.5f * be * inv * sym;
            qz += -inv * ga * oa;
            qx += ga * xxa - inv * mpv * jy;
            qy += ga * xya + inv * mpv * jx;
            hx += ga * tx;
            hy += ga * ty;
          }
        }
      });
    }
    for (int o = 16; o > 0; o >>= 1) {
      qx += __shfl_xor_sync(0xffffffffu, qx, o);
      qy += __shfl_xor_sync(0xffffffffu, qy, o);
      qz += __shfl_xor_sync(0xffffffffu, qz, o);
      hx += __shfl_xor_sync(0xffffffffu, hx, o);
      hy += __shfl_xor_sync(0xffffffffu, hy, o);
    }
    if (lane == 0) hess_flush(gr, r.eid, qx - hy * inv, qy + hx * inv, qz, d_r);
  }
}

// ---------------------------------------------------------------------------
// Message block: the activation between the two SO(2) convolutions
// ("TrimSO(2): Fast and Memory-Efficient Training of Equivariant Interatomic
// Potentials", Abstract: recombination with activation).  In the edge frame,
// per channel c, with h = g1 * V1 (the first conv's gated product rows):
//   h'[row][c] = h[row][c] * s_c,  s_c = sigmoid(h[(0,0)][c])
// (SiLU on the (0,0) row; s_c does not change under a roll of the frame).
// The rows of both convs are the kept edge-frame rows in the grouped layout
// (the block keeps one channel count, so input and output layouts agree).
// One warp per edge, four channels per lane.
// ---------------------------------------------------------------------------
__device__ __forceinline__ float4 sigmoid4(float4 h) {
  return make_float4(1.f / (1.f + __expf(-h.x)), 1.f / (1.f + __expf(-h.y)),
                     1.f / (1.f + __expf(-h.z)), 1.f / (1.f + __expf(-h.w)));
}

// Forward: h' as the second product's operand planes (bf16 hi, and lo on the
// split path), zero on the padding columns.
template <typename TF>
__global__ void __launch_bounds__(256) k_block_act(Layout y, int M, const TF *__restrict__ V1,
                                                   const float *__restrict__ gate1,
                                                   __nv_bfloat16 *__restrict__ hp_hi,
                                                   __nv_bfloat16 *__restrict__ hp_lo) {
  const int lane = threadIdx.x & 31, wpb = blockDim.x >> 5;
  const int C = y.co;
  for (int i = blockIdx.x * wpb + (threadIdx.x >> 5); i < M; i += gridDim.x * wpb) {
    const TF *v = V1 + (int64_t)i * y.KG;
    __nv_bfloat16 *oh = hp_hi + (int64_t)i * y.KA;
    __nv_bfloat16 *ol = hp_lo ? hp_lo + (int64_t)i * y.KA : nullptr;
    for (int c = 4 * lane; c < C; c += 128) {
      const float4 g = load4(gate1 + (int64_t)i * C + c);
      const float4 v00 = load4(v + y.kout_off[0] + c);  // row (0, 0)
      const float4 sg = sigmoid4(make_float4(g.x * v00.x, g.y * v00.y, g.z * v00.z, g.w * v00.w));
      const float4 k = make_float4(g.x * sg.x, g.y * sg.y, g.z * sg.z, g.w * sg.w);
      for (int gi = 0; gi < y.ng; ++gi)
        for (int j = 0; j < y.rows[gi]; ++j) {
          const int col = y.kout_off[gi] + j * C + c;
          const float4 vr = load4(v + col);
          store_split4(oh + col, ol ? ol + col : nullptr,
                       make_float4(k.x * vr.x, k.y * vr.y, k.z * vr.z, k.w * vr.w));
        }
    }
    for (int gi = 0; gi < y.ng; ++gi)
      for (int kk = y.rows[gi] * C + 4 * lane; kk < y.Kin_pad[gi]; kk += 128)
        store_split4(oh + y.kin_off[gi] + kk, ol ? ol + y.kin_off[gi] + kk : nullptr,
                     make_float4(0.f, 0.f, 0.f, 0.f));
  }
}

// Backward through the activation.  With Gh = dL/dh' (= M2^T (g2 D G[dst]),
// the second conv's transposed product rows):
//   dh[row] = s Gh[row] + [row == (0,0)] s (1 - s) sum_rows h Gh,
// and through h = g1 V1: the first conv's output-side operand gv1 = g1 dh
// (planes, zero padding), Gg1[c] = sum_rows dh V1 (its gate's gradient), and
// the gate's share of dL/d|r|, dd1 = sum_c Gg1[c] sum_k W_rad1[k][c] phi'_k(d),
// added onto the edge record h_rec[i].z.
template <typename TF>
__global__ void __launch_bounds__(256) k_block_act_bwd(
    Layout y, float cutoff, int M, const float *__restrict__ geo, const TF *__restrict__ V1,
    const float *__restrict__ gate1, const TF *__restrict__ Gh, const float *__restrict__ w_rad1,
    __nv_bfloat16 *__restrict__ gv_hi, __nv_bfloat16 *__restrict__ gv_lo,
    float *__restrict__ Gg1, float4 *__restrict__ h_rec) {
  __shared__ float sphi[8][RAD_MAX_NR];
  const int lane = threadIdx.x & 31, wpb = blockDim.x >> 5;
  float *sP = sphi[threadIdx.x >> 5];
  const int C = y.co;
  const float sig = cutoff / static_cast<float>(y.nr - 1);
  for (int i = blockIdx.x * wpb + (threadIdx.x >> 5); i < M; i += gridDim.x * wpb) {
    const float d = geo[(int64_t)i * GEO];
    __syncwarp();
    for (int k = lane; k < y.nr; k += 32) {
      const float t = (d - sig * static_cast<float>(k)) / sig;
      sP[k] = (-t / sig) * __expf(-0.5f * t * t);
    }
    __syncwarp();
    const TF *v = V1 + (int64_t)i * y.KG;
    const TF *gh = Gh + (int64_t)i * y.KA;
    __nv_bfloat16 *oh = gv_hi + (int64_t)i * y.KG;
    __nv_bfloat16 *ol = gv_lo ? gv_lo + (int64_t)i * y.KG : nullptr;
    float dd = 0.f;
    for (int c = 4 * lane; c < C; c += 128) {
      const float4 g = load4(gate1 + (int64_t)i * C + c);
      const float4 v00 = load4(v + y.kout_off[0] + c);
      const float4 sg = sigmoid4(make_float4(g.x * v00.x, g.y * v00.y, g.z * v00.z, g.w * v00.w));
      // sum over rows of h Gh
      float4 hg = make_float4(0.f, 0.f, 0.f, 0.f);
      for (int gi = 0; gi < y.ng; ++gi)
        for (int j = 0; j < y.rows[gi]; ++j) {
          const float4 vr = load4(v + y.kout_off[gi] + j * C + c);
          const float4 gr = load4(gh + y.kin_off[gi] + j * C + c);
          hg.x += g.x * vr.x * gr.x;
          hg.y += g.y * vr.y * gr.y;
          hg.z += g.z * vr.z * gr.z;
          hg.w += g.w * vr.w * gr.w;
        }
      const float4 e00 = make_float4(sg.x * (1.f - sg.x) * hg.x, sg.y * (1.f - sg.y) * hg.y,
                                     sg.z * (1.f - sg.z) * hg.z, sg.w * (1.f - sg.w) * hg.w);
      float4 gg = make_float4(0.f, 0.f, 0.f, 0.f);
      for (int gi = 0; gi < y.ng; ++gi)
        for (int j = 0; j < y.rows[gi]; ++j) {
          const float4 vr = load4(v + y.kout_off[gi] + j * C + c);
          const float4 gr = load4(gh + y.kin_off[gi] + j * C + c);
          float4 dh = make_float4(sg.x * gr.x, sg.y * gr.y, sg.z * gr.z, sg.w * gr.w);
          if (gi == 0 && j == 0) {
            dh.x += e00.x;
            dh.y += e00.y;
            dh.z += e00.z;
            dh.w += e00.w;
          }
          const int col = y.kout_off[gi] + j * C + c;
          store_split4(oh + col, ol ? ol + col : nullptr,
                       make_float4(g.x * dh.x, g.y * dh.y, g.z * dh.z, g.w * dh.w));
          gg.x += dh.x * vr.x;
          gg.y += dh.y * vr.y;
          gg.z += dh.z * vr.z;
          gg.w += dh.w * vr.w;
        }
      *reinterpret_cast<float4 *>(Gg1 + (int64_t)i * C + c) = gg;
      float4 dg = make_float4(0.f, 0.f, 0.f, 0.f);
      for (int k = 0; k < y.nr; ++k) {
        const float4 wk = __ldg(reinterpret_cast<const float4 *>(w_rad1 + (int64_t)k * C + c));
        const float p = sP[k];
        dg.x += wk.x * p;
        dg.y += wk.y * p;
        dg.z += wk.z * p;
        dg.w += wk.w * p;
      }
      dd += gg.x * dg.x + gg.y * dg.y + gg.z * dg.z + gg.w * dg.w;
    }
    for (int gi = 0; gi < y.ng; ++gi)
      for (int kk = y.rows[gi] * C + 4 * lane; kk < y.Kout_pad[gi]; kk += 128)
        store_split4(oh + y.kout_off[gi] + kk, ol ? ol + y.kout_off[gi] + kk : nullptr,
                     make_float4(0.f, 0.f, 0.f, 0.f));
    for (int o = 16; o > 0; o >>= 1) dd += __shfl_xor_sync(0xffffffffu, dd, o);
    if (lane == 0) h_rec[i].z += dd;
  }
}

// Frames and full Wigner-D for inspection, with the same per-thread code the
// op uses.  Block = one warp, 32 edges.
template <int L>
__global__ void __launch_bounds__(32) k_frames(int64_t E, const float *__restrict__ edge_vec,
                                               float *__restrict__ Rout, float *__restrict__ Dout) {
  constexpr int dsz = dsize(L);
  extern __shared__ float sD[];  // [dsz][33]
  const int lane = threadIdx.x;
  for (int64_t e0 = blockIdx.x * 32ll; e0 < E; e0 += gridDim.x * 32ll) {
    const int64_t e = e0 + lane;
    __syncwarp();
    if (e < E) {
      Frame f;
      make_frame(edge_vec[3 * e], edge_vec[3 * e + 1], edge_vec[3 * e + 2], f);
      if (Rout)
        for (int k = 0; k < 9; ++k) Rout[9 * e + k] = f.R[k];
      wigner_blocks_thread<L>(f.R, sD + lane, 33);
    }
    __syncwarp();
    if (!Dout) continue;
    const int nj = (E - e0) < 32 ? static_cast<int>(E - e0) : 32;
    for (int j = 0; j < nj; ++j)
      for (int k = lane; k < dsz; k += 32) Dout[(e0 + j) * dsz + k] = sD[k * 33 + j];
  }
}

}  // namespace so2
