// gemm_tc.cuh -- grouped, persistent tcgen05 GEMM for the per-m mixing.
//
// C[M x N] (+)= A[M x K] * B[N x K]^T, A and B bf16 and K-major, f32
// accumulation in tensor memory.  With SPLIT, A and B are each given as a
// (hi, lo) pair of bf16 planes whose sum carries 16 significant bits, and the
// product is hi*hi + hi*lo + lo*hi (the lo*lo term is below the f32 path's
// tolerance).  This is how the f32 configurations reach ~1e-5 relative error
// on bf16 tensor cores.
//
// Several independent problems (one per m, the dense per-m multiplications
// named in "TrimSO(2): Fast and Memory-Efficient Training of Equivariant
// Interatomic Potentials", Abstract) share one launch: each group addresses
// its own rectangle of the same A and B tensors.
//
// Structure: one CTA per SM loops over 128 x 256 output tiles.  Warp 0 issues
// the TMA loads into a STAGES-deep shared-memory ring, warp 1 issues the MMAs
// (one thread) into one of two TMEM accumulators (2 x 256 columns), warps
// 2..(1 + SO2_EPI_WARPS) (one to four per TMEM lane quadrant) drain the other
// accumulator -- to global memory and/or through the fused reduction epilogue
// -- so a tile's epilogue overlaps the next tile's main loop.  Every wait is
// bounded (see mbar_wait); after a wait gives up, the producer and the MMA
// thread wait (bounded) for their copies and products still in flight before
// the CTA frees its tensor memory and exits.
#pragma once

#include "common.cuh"
#include "layout.cuh"

#ifndef SO2_EPI_WARPS
#define SO2_EPI_WARPS 12
#endif
#ifndef SO2_EPI_RELAXED_ARRIVE
#define SO2_EPI_RELAXED_ARRIVE 1
#endif

namespace so2 {

constexpr int GEMM_BM = 128;
constexpr int GEMM_BN = 256;
constexpr int GEMM_MAX_GROUPS = 8;
constexpr int GEMM_THREADS = 64 + 32 * SO2_EPI_WARPS;  // warp 0 TMA, warp 1 MMA, then epilogue

struct GemmGroup {
  int M, N, K;           // K is a multiple of the K block
  int a_row, a_col;      // origin of this group's A rectangle (rows, K cols)
  int b_row, b_col;      // origin of this group's B rectangle
  int tiles_n, tile_begin;
  long long c_off;       // element offset of C[0][0] for this group
  int ldc;               // row stride of C in elements
  int mgroup;            // |m| of this group (fused reduction epilogue)
  int tiles_mn;          // tiles per K split
  int klen;              // K per split (multiple of the K block); ksplit = ceil(K / klen)
};

// Fused epilogue "inverse rotation on reduction": instead of (or besides)
// storing a tile of the product, multiply it by the per-edge gate, rotate
// each edge-frame row (l, m) back with D^l[m][:] and add it onto the node
// key[edge] of out[node][(l, m')][c].  Requires rows = edges and C % 32 == 0.
struct GemmScatter {
  const int4 *rec;     // per edge: (eid, src, dst, key)
  const float *gate;   // [rows][C] or null
  const float *DT;     // kept D rows, row-major by layout row (see k_edge_prep)
  float *out;          // [N][S][C]
  int C, L, dt_chunk;
};

struct GemmParams {
  int n_groups;
  int total_tiles;
  GemmGroup g[GEMM_MAX_GROUPS];
  float *C;
  int beta;   // 0: C = AB^T, 1: C += AB^T
  int split;  // 1: hi/lo planes (3 products), 0: hi only
  int store;  // write C
  int cbf16;  // C is bf16 (plain stores only: beta 0, no K split); f32 otherwise
  int scatter;  // fused reduction epilogue (GemmScatter)
  GemmScatter sc;
  DevStatus *status;
};

constexpr int EPI_WARPS = SO2_EPI_WARPS;  // 4 to 16: one to four per TMEM lane quadrant
static_assert(EPI_WARPS % 4 == 0 && EPI_WARPS <= 16, "epilogue warps per TMEM quadrant");
constexpr int EPI_SMEM_PER_WARP = (32 * 33 + 32 * 16 + 32) * 4;  // multiple of 16 B
constexpr int EPI_SMEM = EPI_WARPS * EPI_SMEM_PER_WARP;
// Plain bf16 products: each epilogue warp writes its 32 x 32 chunk of f32
// results through a [32][33] shared-memory transpose so that every store
// instruction covers one 128-byte row segment instead of 32 rows.
#ifndef SO2_TSTORE
#define SO2_TSTORE 1
#endif
constexpr int EPI_TST_BYTES = EPI_WARPS * 32 * 33 * 4;
template <bool SPLIT, bool SCATTER, bool MN>
constexpr bool gemm_tstore() {
  return SO2_TSTORE && !SPLIT && !SCATTER && !MN;
}

// Row j of an m-group (|m| = g) of an lmax-L layout -> (l, m); rows of group
// g >= 1 are (l, +g) for l = g..L then (l, -g).
__device__ __forceinline__ void gemm_row_lm(int L, int g, int j, int &l, int &m) {
  if (g == 0) {
    l = j;
    m = 0;
    return;
  }
  const int half = L + 1 - g;
  if (j < half) {
    l = g + j;
    m = g;
  } else {
    l = g + (j - half);
    m = -g;
  }
}

// Per-warp scratch of the fused reduction epilogue.
struct EpiScratch {
  float *T;     // [32][33] product values, edge-major
  float *Dw;    // [32][16] D^l[m][:] of the warp's edges for the current row
  int *keys;    // [32] node of each edge (-1 past the end)
};

static_assert((32 * 33 * 4) % 16 == 0 && EPI_SMEM_PER_WARP % 16 == 0,
              "float4 reads of the staged D rows need 16-byte alignment");
__device__ __forceinline__ EpiScratch epi_scratch(float *base) {
  EpiScratch e;
  e.T = base;
  e.Dw = base + 32 * 33;  // 32 * 33 floats = 4224 B: rows of 16 stay 16-byte aligned
  e.keys = reinterpret_cast<int *>(base + 32 * 33 + 32 * 16);
  return e;
}

// Stage D^l[m][:] (W = 2l + 1 floats, row stride 16) of the warp's 32 edges
// (rows row_base..) into Dw; zero past the end of the chunk.  src is the
// first edge's row in the kept-row copy, where the 32 edges' rows are
// contiguous, so the loads are coalesced.
template <int W>
__device__ __forceinline__ void epi_stage_d(const float *__restrict__ src, int nrow,
                                            const EpiScratch &x) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int it = 0; it < W; ++it) {
    const int idx = lane + 32 * it;
    const int el = idx / W, k = idx - el * W;
    x.Dw[el * 16 + k] = (el < nrow) ? __ldg(src + idx) : 0.f;
  }
}

// One warp, one 32-column chunk (channels c0.. of edge-frame row (l, m)) of
// its 32 edges: adds sum_e D_e^l[m][m'] g_e[c] v_e[c] onto
// out[key_e][(l, m')][c], one coalesced atomic per (node run, m', c).
// r holds one edge's 32 values per lane (lane = edge); keys must be staged;
// with a non-null dsrc (the first edge's kept D row) the edges' D rows are
// staged into Dw first.  Each lane writes its edge's values into shared
// memory; read back with lane = channel, each lane scales its column by the
// gate (one 128-byte gate row segment per load); the warp's 32 edges split
// into runs of equal node (a ballot finds the run starts), each summed in
// registers and flushed with W coalesced atomics.
// With cst, the chunk's values (ungated: S.gate is null then) are also
// stored to rows cst + el * ldc, el < the chunk's valid rows, one 128-byte
// row segment per store instruction, from the transposed staging.
template <int W>
__device__ __forceinline__ void epi_scatter_w(const GemmScatter &S, int M, int row_base, int l,
                                              int c0, const uint32_t (&r)[32],
                                              const float *dsrc, const EpiScratch &x,
                                              float *cst, int ldc, bool cst_lane) {
  const int lane = threadIdx.x & 31;
  const int my_key = x.keys[lane];
  __syncwarp();  // the previous chunk's reads of T and Dw are done
#pragma unroll
  for (int k = 0; k < 32; ++k) x.T[lane * 33 + k] = __uint_as_float(r[k]);
  if (dsrc) epi_stage_d<W>(dsrc, M - row_base, x);
  __syncwarp();
  // lane = channel from here on
  const int c = c0 + lane;
  const int S_ = (S.L + 1) * (S.L + 1);
  const int prev_key = lane ? x.keys[lane - 1] : -2;
  const int nvalid = __popc(__ballot_sync(0xffffffffu, my_key >= 0));  // a prefix of the warp
  if (S.gate) {
    // each lane scales its own channel column: one 128-byte gate row segment
    // per load instruction
    const float *gp = S.gate + (int64_t)row_base * S.C + c;
#pragma unroll 8
    for (int el = 0; el < nvalid; ++el) x.T[el * 33 + lane] *= __ldg(gp + (int64_t)el * S.C);
  }
  if (cst && cst_lane) {
#pragma unroll 4
    for (int el = 0; el < nvalid; ++el) cst[(int64_t)el * ldc + lane] = x.T[el * 33 + lane];
  }
  unsigned starts = __ballot_sync(0xffffffffu, my_key != prev_key && my_key >= 0);
  while (starts) {
    const int s0 = __ffs(starts) - 1;
    starts &= starts - 1;
    const int s1 = starts ? __ffs(starts) - 1 : nvalid;
    const int key = x.keys[s0];
    float acc[W];
#pragma unroll
    for (int k = 0; k < W; ++k) acc[k] = 0.f;
#pragma unroll 4
    for (int el = s0; el < s1; ++el) {
      const float v = x.T[el * 33 + lane];
      const float4 *d4 = reinterpret_cast<const float4 *>(x.Dw + el * 16);
#pragma unroll
      for (int k4 = 0; k4 < (W + 3) / 4; ++k4) {
        const float4 d = d4[k4];
        if (4 * k4 + 0 < W) acc[4 * k4 + 0] += d.x * v;
        if (4 * k4 + 1 < W) acc[4 * k4 + 1] += d.y * v;
        if (4 * k4 + 2 < W) acc[4 * k4 + 2] += d.z * v;
        if (4 * k4 + 3 < W) acc[4 * k4 + 3] += d.w * v;
      }
    }
    float *o = S.out + ((int64_t)key * S_ + l * l) * S.C + c;
#pragma unroll
    for (int k = 0; k < W; ++k) atomicAdd(o + k * S.C, acc[k]);
  }
}

__device__ __forceinline__ void epi_scatter_chunk(const GemmScatter &S, int M, int row_base, int l,
                                                  int c0, const uint32_t (&r)[32],
                                                  const float *dsrc, const EpiScratch &x,
                                                  float *cst, int ldc, bool cst_lane) {
  switch (2 * l + 1) {
    case 1: epi_scatter_w<1>(S, M, row_base, l, c0, r, dsrc, x, cst, ldc, cst_lane); break;
    case 3: epi_scatter_w<3>(S, M, row_base, l, c0, r, dsrc, x, cst, ldc, cst_lane); break;
    case 5: epi_scatter_w<5>(S, M, row_base, l, c0, r, dsrc, x, cst, ldc, cst_lane); break;
    case 7: epi_scatter_w<7>(S, M, row_base, l, c0, r, dsrc, x, cst, ldc, cst_lane); break;
    case 9: epi_scatter_w<9>(S, M, row_base, l, c0, r, dsrc, x, cst, ldc, cst_lane); break;
    case 11: epi_scatter_w<11>(S, M, row_base, l, c0, r, dsrc, x, cst, ldc, cst_lane); break;
    default: epi_scatter_w<13>(S, M, row_base, l, c0, r, dsrc, x, cst, ldc, cst_lane); break;
  }
}

// BK = 32 uses the 64-byte swizzle, BK = 64 the 128-byte swizzle; a pair's
// stage with hi/lo planes is 64 KB per CTA at BK = 64.
// With PAIR, two CTAs (a cluster) share each 256 x 256 tile: each holds 128
// rows of A and of the output, and half (128 rows) of B.
template <int BK, int STAGES, bool SPLIT, bool SCATTER, bool PAIR = false, bool TST = false>
struct GemmCfg {
  static constexpr bool TSTORE = TST;
  static constexpr int NB = PAIR ? GEMM_BN / 2 : GEMM_BN;  // B rows held by this CTA
  static constexpr int TBM = PAIR ? 2 * GEMM_BM : GEMM_BM;  // output rows per tile
  static constexpr int A_BYTES = GEMM_BM * BK * 2;
  static constexpr int B_BYTES = NB * BK * 2;
  static constexpr int PLANES = SPLIT ? 2 : 1;
  static constexpr int STAGE_BYTES = (A_BYTES + B_BYTES) * PLANES;
  static constexpr int SMEM =
      STAGES * STAGE_BYTES + 1024 /*align*/ + 256 /*barriers*/ +
      (SCATTER ? EPI_SMEM : (TST ? EPI_TST_BYTES : 0));
  static constexpr int TMEM_COLS = 2 * GEMM_BN;
  static_assert(SMEM <= 232448, "shared memory per CTA");
};

__device__ __forceinline__ uint64_t sdesc_k(uint32_t saddr, int bk) {
  return bk == 32 ? sdesc_k_sw64(saddr) : sdesc_k_sw128(saddr);
}

// Tile -> group, output origin and K range [k0, k0 + klen_t).  K splits are
// outermost inside a group so that concurrent tiles share operand rows in L2.
// TBM: output rows per tile.
template <int TBM>
__device__ __forceinline__ void tile_coords(const GemmParams &p, int tile, int &gi, int &m0,
                                            int &n0, int &k0, int &kl) {
  gi = 0;
  while (gi + 1 < p.n_groups && tile >= p.g[gi + 1].tile_begin) ++gi;
  const GemmGroup &G = p.g[gi];
  const int local = tile - G.tile_begin;
  const int ks = local / G.tiles_mn, mn = local % G.tiles_mn;
  m0 = (mn / G.tiles_n) * TBM;
  n0 = (mn % G.tiles_n) * GEMM_BN;
  k0 = ks * G.klen;
  kl = (G.K - k0) < G.klen ? (G.K - k0) : G.klen;
}

// PAIR: launched in clusters of two CTAs; the even CTA issues the pair's
// MMAs, both load their operand halves and drain their own accumulator lanes.
template <int BK, int STAGES, bool SPLIT, bool SCATTER, bool MN, bool PAIR = false>
__global__ void __launch_bounds__(GEMM_THREADS, 1)
    k_gemm_tc(const __grid_constant__ CUtensorMap tA_hi, const __grid_constant__ CUtensorMap tA_lo,
              const __grid_constant__ CUtensorMap tB_hi, const __grid_constant__ CUtensorMap tB_lo,
              const __grid_constant__ GemmParams p) {
  using Cfg = GemmCfg<BK, STAGES, SPLIT, SCATTER, PAIR, gemm_tstore<SPLIT, SCATTER, MN>()>;
  constexpr int NB = Cfg::NB, TBM = Cfg::TBM;
  static_assert(!MN || BK % 16 == 0, "MN-major K block");
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t *full = reinterpret_cast<uint64_t *>(smem + STAGES * Cfg::STAGE_BYTES);
  uint64_t *empty = full + STAGES;
  uint64_t *tfull = empty + STAGES;  // [2]
  uint64_t *tempty = tfull + 2;      // [2]
  uint64_t *drain = tempty + 2;      // products in flight at an abort
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(drain + 1);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
  float *epi_smem = reinterpret_cast<float *>(smem + STAGES * Cfg::STAGE_BYTES + 256);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  // CTA pair: rank in the cluster, the cluster's index and count; the even
  // CTA's full[] and tempty[] barriers serve both CTAs
  const int rank = PAIR ? static_cast<int>(cluster_ctarank()) : 0;
  const int unit0 = PAIR ? static_cast<int>(blockIdx.x) / 2 : static_cast<int>(blockIdx.x);
  const int units = PAIR ? static_cast<int>(gridDim.x) / 2 : static_cast<int>(gridDim.x);
  const uint32_t full_c = PAIR ? mapa_shared(smem_u32(full), 0) : 0;
  const uint32_t tempty_c = PAIR ? mapa_shared(smem_u32(tempty), 0) : 0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], (PAIR ? 2 : 1) * EPI_WARPS);  // one arrive per epilogue warp
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    if (PAIR) {
      tmem_alloc_pair(tmem_slot, Cfg::TMEM_COLS);
      tmem_relinquish_pair();
    } else {
      tmem_alloc(tmem_slot, Cfg::TMEM_COLS);
      tmem_relinquish();
    }
  }
  tc_fence_before();
  __syncthreads();
  if (PAIR) cluster_sync();  // the peer's barriers are initialised before any remote use
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0 && lane == 0) {
    // ---------------- TMA producer ----------------
    int it = 0;
    bool ok = true;
    for (int tile = unit0; ok && tile < p.total_tiles; tile += units) {
      int gi, m0, n0, k0, kl;
      tile_coords<TBM>(p, tile, gi, m0, n0, k0, kl);
      const GemmGroup &G = p.g[gi];
      const int nk = kl / BK;
      const int am = G.a_row + m0 + rank * GEMM_BM;  // this CTA's A rows
      const int bn = G.b_row + n0 + rank * NB;       // this CTA's B rows
      for (int kb = 0; kb < nk; ++kb, ++it) {
        const int s = it % STAGES;
        const uint32_t ph = (it / STAGES) & 1;
        if (!mbar_wait(&empty[s], ph ^ 1, p.status, abort_flag)) {
          ok = false;
          break;
        }
        uint8_t *st = smem + s * Cfg::STAGE_BYTES;
        // the even CTA expects the bytes of both CTAs' loads
        if (rank == 0) mbar_arrive_expect_tx(&full[s], (PAIR ? 2 : 1) * Cfg::STAGE_BYTES);
        auto load = [&](void *dst, const CUtensorMap *map, int c0, int c1) {
          if (PAIR)
            tma_load_2d_pair(dst, map, full_c + 8u * s, c0, c1);
          else
            tma_load_2d(dst, map, &full[s], c0, c1);
        };
        const int kc = k0 + kb * BK;
        if (!MN) {
          load(st, &tA_hi, G.a_col + kc, am);
          load(st + Cfg::A_BYTES, &tB_hi, G.b_col + kc, bn);
          if (SPLIT) {
            load(st + Cfg::A_BYTES + Cfg::B_BYTES, &tA_lo, G.a_col + kc, am);
            load(st + 2 * Cfg::A_BYTES + Cfg::B_BYTES, &tB_lo, G.b_col + kc, bn);
          }
        } else {
          // MN-major operands: the inner TMA coordinate is the M / N index, the
          // outer one the K index; one box per 64 M / N elements
          constexpr int BOX = 64 * BK * 2;
          for (int h = 0; h < GEMM_BM / 64; ++h) load(st + h * BOX, &tA_hi, am + 64 * h, G.a_col + kc);
          for (int h = 0; h < NB / 64; ++h)
            load(st + Cfg::A_BYTES + h * BOX, &tB_hi, bn + 64 * h, G.b_col + kc);
          if (SPLIT) {
            for (int h = 0; h < GEMM_BM / 64; ++h)
              load(st + Cfg::A_BYTES + Cfg::B_BYTES + h * BOX, &tA_lo, am + 64 * h, G.a_col + kc);
            for (int h = 0; h < NB / 64; ++h)
              load(st + 2 * Cfg::A_BYTES + Cfg::B_BYTES + h * BOX, &tB_lo, bn + 64 * h,
                   G.b_col + kc);
          }
        }
      }
    }
    // After an abort the MMA thread may not consume the last stages: wait
    // (bounded) until their copies have landed before shared memory is
    // released.  The pair's full[] barriers live in the even CTA and count
    // both CTAs' bytes.
    if (*abort_flag && rank == 0) {
      for (int i = it > STAGES ? it - STAGES : 0; i < it; ++i)
        mbar_wait(&full[i % STAGES], (i / STAGES) & 1, p.status, nullptr, 200000000ull);
    }
  } else if (warp == 1 && lane == 0 && rank == 0) {
    // ---------------- MMA issuer (the even CTA of a pair) ----------------
    constexpr uint32_t idesc = idesc_bf16_f32(TBM, GEMM_BN, MN);
    constexpr uint32_t LBO = 64 * BK * 2;  // MN-major: bytes between 64-element MN chunks
    int it = 0, tcount = 0;
    bool ok = true;
    for (int tile = unit0; ok && tile < p.total_tiles; tile += units, ++tcount) {
      int gi, m0, n0, k0, kl;
      tile_coords<TBM>(p, tile, gi, m0, n0, k0, kl);
      const int nk = kl / BK;
      const int acc = tcount & 1;
      const uint32_t aph = (tcount >> 1) & 1;
      if (!mbar_wait(&tempty[acc], aph ^ 1, p.status, abort_flag)) break;
      tc_fence_after();
      const uint32_t d_tmem = tmem + acc * GEMM_BN;
      for (int kb = 0; kb < nk; ++kb, ++it) {
        const int s = it % STAGES;
        const uint32_t ph = (it / STAGES) & 1;
        if (!mbar_wait(&full[s], ph, p.status, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t base = smem_u32(smem + s * Cfg::STAGE_BYTES);
        const uint32_t oa = base, ob = base + Cfg::A_BYTES;
        const uint32_t oal = base + Cfg::A_BYTES + Cfg::B_BYTES;
        const uint32_t obl = base + 2 * Cfg::A_BYTES + Cfg::B_BYTES;
        const uint64_t a_hi = MN ? sdesc_mn_sw128(oa, LBO) : sdesc_k(oa, BK);
        const uint64_t b_hi = MN ? sdesc_mn_sw128(ob, LBO) : sdesc_k(ob, BK);
        const uint64_t a_lo = MN ? sdesc_mn_sw128(oal, LBO) : sdesc_k(oal, BK);
        const uint64_t b_lo = MN ? sdesc_mn_sw128(obl, LBO) : sdesc_k(obl, BK);
#pragma unroll
        for (int kk = 0; kk < BK / 16; ++kk) {
          // next 16 K: 32 bytes along a K-major row, or two 1024-byte atoms of
          // an MN-major tile (in 16-byte units)
          const uint64_t step = static_cast<uint64_t>(MN ? kk * 128 : kk * 2);
          if (PAIR) {
            umma_bf16_pair(d_tmem, a_hi + step, b_hi + step, idesc, (kb | kk) != 0);
            if (SPLIT) {
              umma_bf16_pair(d_tmem, a_hi + step, b_lo + step, idesc, 1);
              umma_bf16_pair(d_tmem, a_lo + step, b_hi + step, idesc, 1);
            }
          } else {
            umma_bf16(d_tmem, a_hi + step, b_hi + step, idesc, (kb | kk) != 0);
            if (SPLIT) {
              umma_bf16(d_tmem, a_hi + step, b_lo + step, idesc, 1);
              umma_bf16(d_tmem, a_lo + step, b_hi + step, idesc, 1);
            }
          }
        }
        if (PAIR)
          umma_commit_pair(&empty[s]);  // frees stage s in both CTAs
        else
          umma_commit(&empty[s]);
      }
      if (ok) {
        if (PAIR)
          umma_commit_pair(&tfull[acc]);
        else
          umma_commit(&tfull[acc]);
      }
    }
    // After an abort, products already issued may still be writing tensor
    // memory: wait (bounded) for all of them before it is freed.
    if (*abort_flag) {
      if (PAIR)
        umma_commit_pair(drain);
      else
        umma_commit(drain);
      mbar_wait(drain, 0, p.status, nullptr, 200000000ull);
    }
  } else if (warp >= 2) {
    // ---------------- epilogue: TMEM -> registers -> C and/or node sums ----------------
    const int q = warp & 3;           // TMEM lane quadrant this warp may read
    const int half = (warp - 2) >> 2;  // which share of the tile's column chunks
    const EpiScratch xs = epi_scratch(epi_smem + (warp - 2) * (EPI_SMEM_PER_WARP / 4));
    int tcount = 0;
    for (int tile = unit0; tile < p.total_tiles; tile += units, ++tcount) {
      int gi, m0, n0, k0, kl;
      tile_coords<TBM>(p, tile, gi, m0, n0, k0, kl);
      const GemmGroup &G = p.g[gi];
      const bool atomic_c = G.klen < G.K;  // split K: partial sums meet in C
      const int acc = tcount & 1;
      const uint32_t aph = (tcount >> 1) & 1;
      const int row_base = m0 + rank * GEMM_BM + q * 32;  // this CTA's accumulator lanes
      if (SCATTER && p.scatter) {
        const int e = row_base + lane;
        xs.keys[lane] = (e < G.M) ? p.sc.rec[e].w : -1;
      }
      if (!mbar_wait(&tfull[acc], aph, p.status, abort_flag)) break;
      tc_fence_after();
      const int row = row_base + lane;
      float *Cg = p.C + G.c_off;
      int staged = -1;  // edge-frame row whose D rows are in Dw
      // an ungated fused reduction that also stores the product (plain f32,
      // no accumulation into C) stores it from the reduction's transposed
      // staging, with coalesced row segments
      const bool store_staged = SCATTER && p.scatter && p.store && !p.sc.gate && !p.cbf16 &&
                                !p.beta && !atomic_c;
      for (int cc = half; cc < GEMM_BN / 32; cc += EPI_WARPS / 4) {
        const int col0 = n0 + cc * 32;
        if (col0 >= G.N) break;  // warp-uniform
        uint32_t r[32];
        tmem_ld32(tmem + (static_cast<uint32_t>(q * 32) << 16) + acc * GEMM_BN + cc * 32, r);
        // store first (when asked), so that r is dead before the reduction
        if (Cfg::TSTORE && p.store) {
          float *Tt = epi_smem + (warp - 2) * (32 * 33);
          __syncwarp();  // the previous chunk's reads of Tt are done
#pragma unroll
          for (int k = 0; k < 32; ++k) Tt[lane * 33 + k] = __uint_as_float(r[k]);
          __syncwarp();
          const int nrow = G.M - row_base;  // rows of this chunk inside the product
          if (p.cbf16) {
            // bf16 rows: lanes 0-15 write column pairs of row e, 16-31 of row e + 1
            __nv_bfloat16 *cb = reinterpret_cast<__nv_bfloat16 *>(p.C) + G.c_off;
            const int rh = lane >> 4, cp = 2 * (lane & 15);
            if (col0 + cp < G.N) {  // N is a multiple of 16: the pair is inside
#pragma unroll 4
              for (int e = 0; e < 32; e += 2) {
                const int er = e + rh;
                if (er >= nrow) break;
                *reinterpret_cast<__nv_bfloat162 *>(
                    cb + static_cast<long long>(row_base + er) * G.ldc + col0 + cp) =
                    __floats2bfloat162_rn(Tt[er * 33 + cp], Tt[er * 33 + cp + 1]);
              }
            }
          } else if (col0 + lane < G.N) {
            float *cp = Cg + static_cast<long long>(row_base) * G.ldc + col0 + lane;
#pragma unroll 4
            for (int e = 0; e < 32; ++e) {
              if (e >= nrow) break;
              float v = Tt[e * 33 + lane];
              float *d = cp + static_cast<long long>(e) * G.ldc;
              if (atomic_c) {
                atomicAdd(d, v);
              } else {
                if (p.beta) v += *d;
                *d = v;
              }
            }
          }
        } else if (p.store && p.cbf16 && row < G.M) {
          __nv_bfloat16 *cb = reinterpret_cast<__nv_bfloat16 *>(p.C) + G.c_off +
                              static_cast<long long>(row) * G.ldc + col0;
          if (col0 + 32 <= G.N) {
#pragma unroll
            for (int j = 0; j < 32; j += 8) {
              uint4 u;
              u.x = pack_bf16x2(__uint_as_float(r[j]), __uint_as_float(r[j + 1]));
              u.y = pack_bf16x2(__uint_as_float(r[j + 2]), __uint_as_float(r[j + 3]));
              u.z = pack_bf16x2(__uint_as_float(r[j + 4]), __uint_as_float(r[j + 5]));
              u.w = pack_bf16x2(__uint_as_float(r[j + 6]), __uint_as_float(r[j + 7]));
              *reinterpret_cast<uint4 *>(cb + j) = u;
            }
          } else {
            for (int j = 0; j < 32 && col0 + j < G.N; ++j)
              cb[j] = __float2bfloat16_rn(__uint_as_float(r[j]));
          }
        } else if (p.store && row < G.M && !store_staged) {
          float *crow = Cg + static_cast<long long>(row) * G.ldc + col0;
          const bool vec = (col0 + 32 <= G.N) && ((reinterpret_cast<uintptr_t>(crow) & 15) == 0);
          if (atomic_c && vec) {
#pragma unroll
            for (int j = 0; j < 32; j += 4)
              atomicAdd(reinterpret_cast<float4 *>(crow + j),
                        make_float4(__uint_as_float(r[j]), __uint_as_float(r[j + 1]),
                                    __uint_as_float(r[j + 2]), __uint_as_float(r[j + 3])));
          } else if (atomic_c) {
            for (int j = 0; j < 32 && col0 + j < G.N; ++j) atomicAdd(crow + j, __uint_as_float(r[j]));
          } else if (vec) {
#pragma unroll
            for (int j = 0; j < 32; j += 4) {
              float4 v = make_float4(__uint_as_float(r[j]), __uint_as_float(r[j + 1]),
                                     __uint_as_float(r[j + 2]), __uint_as_float(r[j + 3]));
              float4 *dst = reinterpret_cast<float4 *>(crow + j);
              if (p.beta) {
                const float4 o = *dst;
                v.x += o.x;
                v.y += o.y;
                v.z += o.z;
                v.w += o.w;
              }
              *dst = v;
            }
          } else {
            for (int j = 0; j < 32 && col0 + j < G.N; ++j) {
              const float v = __uint_as_float(r[j]);
              crow[j] = p.beta ? crow[j] + v : v;
            }
          }
        }
        if (SCATTER && p.scatter) {
          const int j = col0 / p.sc.C, c0 = col0 % p.sc.C;
          int l, m;
          gemm_row_lm(p.sc.L, G.mgroup, j, l, m);
          const float *dsrc =
              j != staged ? p.sc.DT + (int64_t)kept_d_prefix(p.sc.L, G.mgroup, j) * p.sc.dt_chunk +
                                (int64_t)row_base * (2 * l + 1)
                          : nullptr;
          epi_scatter_chunk(p.sc, G.M, row_base, l, c0, r, dsrc, xs,
                            store_staged ? Cg + static_cast<long long>(row_base) * G.ldc + col0
                                         : nullptr,
                            G.ldc, col0 + lane < G.N);
          staged = j;
        }
      }
      // The accumulator is free once this warp's tensor-memory loads are done
      // (tcgen05.wait::ld above); its global stores and atomics need no
      // ordering with the next tile's MMAs, so the arrive is relaxed.
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
#if SO2_EPI_RELAXED_ARRIVE
        if (PAIR)
          mbar_arrive_cluster_relaxed(tempty_c + 8u * acc);  // the even CTA's barrier
        else
          mbar_arrive_relaxed(&tempty[acc]);
#else
        if (PAIR)
          mbar_arrive_cluster(tempty_c + 8u * acc);
        else
          mbar_arrive(&tempty[acc]);
#endif
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  // a pair's MMAs read both CTAs' shared memory and write both CTAs' tensor
  // memory: neither CTA frees or leaves before the other is done
  if (PAIR) cluster_sync();
  if (warp == 1) {
    tc_fence_after();
    if (PAIR)
      tmem_dealloc_pair(tmem, Cfg::TMEM_COLS);
    else
      tmem_dealloc(tmem, Cfg::TMEM_COLS);
  }
}

}  // namespace so2
