// so2conv_api.cu -- host side of libso2conv: argument checks, workspace plan,
// tensor maps and the launch sequence of forward / backward / double
// backward and of the message block.  Every step runs in this library's own
// kernels (the double backward's per-edge terms in so2conv_dbl_terms.cu);
// the host only orchestrates on the caller's stream.
#include <cstdio>
#include <cstring>
#include <mutex>
#include <vector>

#include "dbl_terms.h"
#include "dispatch.cuh"
#include "edge_kernels.cuh"
#include "gemm_tc.cuh"

using namespace so2;

#ifndef SO2_SCATTER_PAIR_STAGES  // pipeline stages of the CTA-pair product with the fused epilogue
#define SO2_SCATTER_PAIR_STAGES 4
#endif
#ifndef SO2_SCATTER_STAGES
#define SO2_SCATTER_STAGES 3
#endif
// K block of the split (hi/lo) products: 64 (128-byte rows, 128-byte swizzle;
// by measurement the operands arrive faster in 128-byte rows, even with half as
// many, twice as large stages) or 32 (64-byte rows and swizzle)
#ifndef SO2_SPLIT_BK
#define SO2_SPLIT_BK 64
#endif
// plain bf16 products: the transposing store epilogue takes ~50 KB of shared memory
#if SO2_TSTORE
#define SO2_BF16_PLAIN_PAIR_STAGES 5
#define SO2_BF16_PLAIN_STAGES 3
#else
#define SO2_BF16_PLAIN_PAIR_STAGES 6
#define SO2_BF16_PLAIN_STAGES 4
#endif
#if SO2_SPLIT_BK == 64
#define SO2_SPLIT_PLAIN_PAIR_STAGES 3
#define SO2_SPLIT_MN_PAIR_STAGES 3
#define SO2_SPLIT_SCATTER_PAIR_STAGES 2
#define SO2_SPLIT_SCATTER_STAGES 1
#define SO2_SPLIT_PLAIN_STAGES 2
#else
#define SO2_SPLIT_PLAIN_PAIR_STAGES 6
#define SO2_SPLIT_MN_PAIR_STAGES 6
#define SO2_SPLIT_SCATTER_PAIR_STAGES SO2_SCATTER_PAIR_STAGES
#define SO2_SPLIT_SCATTER_STAGES SO2_SCATTER_STAGES
#define SO2_SPLIT_PLAIN_STAGES 4
#endif

// Whether the reduction onto nodes runs in the product's epilogue (see
// fusable()): f32 yes, bf16 no.
#ifndef SO2_FUSE_BF16
#define SO2_FUSE_BF16 0
#endif
#ifndef SO2_FUSE_F32
#define SO2_FUSE_F32 1
#endif

namespace {

// Edges per chunk of per-edge intermediates (the workspace grows with it);
// so2conv_set_max_chunk_edges changes it for the process.
#ifndef SO2_CHUNK_MAX
#define SO2_CHUNK_MAX 65536
#endif
int g_chunk_max = SO2_CHUNK_MAX;

// --------------------------------------------------------------------------
// cuTensorMapEncodeTiled through the runtime's driver entry point (no link
// against libcuda, so the library also loads on machines without a GPU).
// --------------------------------------------------------------------------
typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encode() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// bf16 matrix [rows x cols] with row stride ld (elements); box bk x box_rows
// with the swizzle that matches bk (32 -> 64 B rows, 64 -> 128 B rows), zero
// fill outside the matrix.
bool make_map(CUtensorMap *m, const void *base, int64_t rows, int64_t cols, int64_t ld,
              int box_rows, int bk) {
  EncodeTiledFn enc = get_encode();
  if (!enc) return false;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(ld * 2)};
  cuuint32_t box[2] = {static_cast<cuuint32_t>(bk), static_cast<cuuint32_t>(box_rows)};
  cuuint32_t estr[2] = {1u, 1u};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
             bk == 32 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// The same bf16 matrix read MN-major: box of 64 columns (inner, 128 B) by bk
// rows, 128-byte swizzle.
bool make_map_mn(CUtensorMap *m, const void *base, int64_t rows, int64_t cols, int64_t ld,
                 int bk) {
  EncodeTiledFn enc = get_encode();
  if (!enc) return false;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(ld * 2)};
  cuuint32_t box[2] = {64u, static_cast<cuuint32_t>(bk)};
  cuuint32_t estr[2] = {1u, 1u};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// K block of the product kernel (64 elements = 128-byte rows unless the split
// path is built with 32).
inline int gemm_bk(bool split) { return split ? SO2_SPLIT_BK : 64; }

int num_sms() {
  int dev = 0, n = 148;
  if (cudaGetDevice(&dev) == cudaSuccess &&
      cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess && n > 0)
    return n;
  return 148;
}

// --------------------------------------------------------------------------
// Workspace plan
// --------------------------------------------------------------------------
struct Plan {
  Layout y;
  int64_t N = 0, E = 0;
  int chunk = 0;
  bool split = true, xbf16 = false;
  size_t total = 0;
  // byte offsets
  int na = 1, ngv = 1;  // row-stacked operand sets (double backward uses 3 and 2)
  size_t DT = 0;  // kept D rows by layout row, for the fused reduction epilogue (f32 path)
  size_t status, counts, cursor, offsets, perm, rec, geo, D, gate, wst_hi, wst_lo, wtr_hi, wtr_lo,
      a_hi, a_lo, V, gv_hi, gv_lo, Ga, Gg, h, dws, radp, omega,
      dgate, tA, tB;
};

size_t take(size_t &cur, size_t bytes) {
  cur = (cur + 1023) & ~static_cast<size_t>(1023);
  const size_t at = cur;
  cur += bytes;
  return at;
}

bool desc_ok(const so2conv_desc *d) {
  if (!d) return false;
  if (d->lmax < 0 || d->lmax > LMAX_SUPPORTED) return false;
  if (d->mmax < 0 || d->mmax > d->lmax) return false;
  if (d->c_in < 16 || d->c_in > 512 || d->c_in % 16) return false;
  if (d->c_out < 16 || d->c_out > 512 || d->c_out % 16) return false;
  if (d->n_rbf < 2 || d->n_rbf > 64) return false;
  if (!(d->rbf_cutoff > 0.f)) return false;
  if (d->dtype != SO2_F32 && d->dtype != SO2_BF16) return false;
  return true;
}

Plan make_plan(const so2conv_desc *d, int64_t N, int64_t E, int which) {
  Plan p;
  p.y = make_layout(d->lmax, d->mmax, d->c_in, d->c_out, d->n_rbf);
  p.N = N;
  p.E = E;
  p.split = d->dtype == SO2_F32;
  p.xbf16 = d->dtype == SO2_BF16;
  const int64_t cap = which == SO2_WS_DOUBLE_BACKWARD ? g_chunk_max / 2 : g_chunk_max;
  const int64_t ch = E < cap ? E : cap;
  p.chunk = static_cast<int>(round_up(static_cast<int>(ch > 0 ? ch : 1), 128));
  const Layout &y = p.y;
  const bool bwd = which >= SO2_WS_BACKWARD;
  const bool dbl = which == SO2_WS_DOUBLE_BACKWARD;
  p.na = dbl ? 3 : 1;
  p.ngv = dbl ? 2 : 1;
  const int lo = p.split ? 1 : 0;
  const size_t na = p.na, ngv = p.ngv;
  size_t c = 0;
  p.status = take(c, 256);
  p.counts = take(c, sizeof(int) * (N + 1));
  p.cursor = take(c, sizeof(int) * (N + 1));
  p.offsets = take(c, sizeof(int) * (N + 1));
  p.perm = take(c, sizeof(int) * (E > 0 ? E : 1));
  p.rec = take(c, sizeof(EdgeRec) * p.chunk);
  p.geo = take(c, sizeof(float) * GEO * p.chunk);
  p.D = take(c, sizeof(float) * (size_t)y.dsz * p.chunk);
  p.gate = take(c, sizeof(float) * (size_t)y.co * p.chunk);
  if ((p.split ? SO2_FUSE_F32 : SO2_FUSE_BF16) && !dbl) p.DT = take(c, sizeof(float) * (size_t)kept_d_size(y.L, y.mmax) * p.chunk);
  p.wst_hi = take(c, 2ull * y.WR * y.WK);
  p.wst_lo = take(c, 2ull * y.WR * y.WK * lo);
  p.wtr_hi = take(c, 2ull * y.WTR * y.WTK);
  p.wtr_lo = take(c, 2ull * y.WTR * y.WTK * lo);
  p.a_hi = take(c, 2ull * na * p.chunk * y.KA);
  p.a_lo = take(c, 2ull * na * p.chunk * y.KA * lo);
  const size_t pe = p.split ? 4 : 2;  // bytes per product element (see prows)
  p.V = take(c, pe * na * p.chunk * y.KG);
  if (bwd) {
    p.gv_hi = take(c, 2ull * ngv * p.chunk * y.KG);
    p.gv_lo = take(c, 2ull * ngv * p.chunk * y.KG * lo);
    p.Ga = take(c, pe * ngv * p.chunk * y.KA);
    p.Gg = take(c, 4ull * p.chunk * y.co);
    p.h = take(c, 16ull * p.chunk);
    p.dws = take(c, 4ull * y.WR * y.WK);
    p.radp = take(c, 4ull * ((p.chunk + RAD_TILE - 1) / RAD_TILE) * (y.nr + 1) * y.co);
  }
  if (dbl) {
    p.omega = take(c, 16ull * p.chunk);
    p.dgate = take(c, 4ull * p.chunk * y.co);
    p.tA = take(c, 4ull * p.chunk * y.co);
    p.tB = take(c, 4ull * p.chunk * y.co);
  }
  p.total = (c + 1023) & ~static_cast<size_t>(1023);
  return p;
}

template <typename T>
T *at(void *ws, size_t off) {
  return reinterpret_cast<T *>(static_cast<char *>(ws) + off);
}

BlockOffsets block_offsets(const Layout &y) {
  BlockOffsets b{};
  long long off = 0;
  b.off[0] = 0;
  off += static_cast<long long>(y.Kout[0]) * y.Kin[0];
  for (int g = 1; g < y.ng; ++g) {
    const long long sz = static_cast<long long>((y.L + 1 - g) * y.co) * ((y.L + 1 - g) * y.ci);
    b.off[2 * g - 1] = off;
    off += sz;
    b.off[2 * g] = off;
    off += sz;
  }
  return b;
}

int64_t num_weights(const Layout &y) {
  BlockOffsets b = block_offsets(y);
  if (y.ng == 1) return static_cast<int64_t>(y.Kout[0]) * y.Kin[0];
  const int g = y.ng - 1;
  return b.off[2 * g] + static_cast<long long>((y.L + 1 - g) * y.co) * ((y.L + 1 - g) * y.ci);
}

#define CK(call)                                  \
  do {                                            \
    if ((call) != cudaSuccess) return SO2_ERR_CUDA; \
  } while (0)

// Every kernel launch of the library is counted (so2conv_launch_count).
long long g_launches = 0;

#define CKL()                                                      \
  do {                                                             \
    ++g_launches;                                                  \
    if (cudaPeekAtLastError() != cudaSuccess) return SO2_ERR_CUDA; \
  } while (0)

// Optional CUDA-event timing of the launches, by kind: 0 products with W,
// 1 with W^T, 2 weight gradients (the tensor-core kinds), 3 rotation on
// gather, 4 edge preparation (sort, records, frames, Wigner-D, gates),
// 5 per-edge gradient terms, 6 radial-weight sums, 7 weight packing and
// node-side scatter.
constexpr int PROF_KINDS = 8;
struct Prof {
  int on = 0;  // 0 off, 1 tensor-core launches, 2 every kind
  std::vector<cudaEvent_t> ev[PROF_KINDS];  // start/stop pairs
  int used[PROF_KINDS] = {};
};
Prof g_prof;

cudaEvent_t prof_event(int kind) {
  Prof &P = g_prof;
  if (P.used[kind] >= static_cast<int>(P.ev[kind].size())) {
    cudaEvent_t e;
    if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
    P.ev[kind].push_back(e);
  }
  return P.ev[kind][P.used[kind]++];
}

// Records a start/stop event pair around the launches of its lifetime.
struct ProfScope {
  cudaEvent_t e1 = nullptr;
  cudaStream_t s;
  ProfScope(int kind, cudaStream_t s_) : s(s_) {
    if (g_prof.on < 2) return;
    cudaEvent_t e0 = prof_event(kind);
    e1 = prof_event(kind);
    if (e0) cudaEventRecord(e0, s);
  }
  ~ProfScope() {
    if (e1) cudaEventRecord(e1, s);
  }
};

int grid_for(int64_t n, int block) {
  int64_t g = (n + block - 1) / block;
  if (g < 1) g = 1;
  if (g > 148 * 16) g = 148 * 16;
  return static_cast<int>(g);
}

// Raise the dynamic shared memory limit of a kernel (once per kernel).
template <typename K>
bool allow_smem(K kernel, int bytes) {
  if (bytes <= 48 * 1024) return true;
  return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) ==
         cudaSuccess;
}

// Which products run on CTA pairs (cta_group::2): plain, with the fused
// reduction epilogue, weight gradients (MN-major operands).
#ifndef SO2_PAIR_PLAIN
#define SO2_PAIR_PLAIN 1
#endif
#ifndef SO2_PAIR_SCATTER
#define SO2_PAIR_SCATTER 1
#endif
#ifndef SO2_PAIR_MN
#define SO2_PAIR_MN 1
#endif

// Blocks per weight group of the gradient unstacking: enough that each
// thread handles a few elements (its loop is load-latency bound).
constexpr int UNSTACK_BLOCKS = 512;

int warp_grid(int M, int warps_per_block) {
  int g = (M + warps_per_block - 1) / warps_per_block;
  if (g < 1) g = 1;
  if (g > 148 * 8) g = 148 * 8;
  return g;
}

// --------------------------------------------------------------------------
// GEMM launcher
// --------------------------------------------------------------------------
struct GemmLauncher {
  GemmParams p{};
  int bm = GEMM_BM;  // output rows per tile: 2 * GEMM_BM for CTA-pair launches
  // ksplit > 1 splits K into that many ranges (multiples of 64) whose
  // partial products are added into C atomically (C must hold the base).
  void add(int M, int N, int K, int a_row, int a_col, int b_row, int b_col, long long c_off,
           int ldc, int ksplit = 1) {
    if (M <= 0 || N <= 0) return;
    GemmGroup &g = p.g[p.n_groups++];
    g.M = M;
    g.N = N;
    g.K = K;
    g.a_row = a_row;
    g.a_col = a_col;
    g.b_row = b_row;
    g.b_col = b_col;
    g.c_off = c_off;
    g.ldc = ldc;
    g.mgroup = p.n_groups - 1;
    g.tiles_n = (N + GEMM_BN - 1) / GEMM_BN;
    g.tiles_mn = ((M + bm - 1) / bm) * g.tiles_n;
    if (ksplit < 1) ksplit = 1;
    g.klen = round_up((K + ksplit - 1) / ksplit, 64);
    if (g.klen > K) g.klen = K;
    const int nsplit = (K + g.klen - 1) / g.klen;
    g.tile_begin = p.total_tiles;
    p.total_tiles += g.tiles_mn * nsplit;
  }
};

template <int BK, int STAGES, bool SPLIT, bool SCATTER, bool MN, bool PAIR = false>
cudaError_t launch_gemm_t(const CUtensorMap &a_hi, const CUtensorMap &a_lo, const CUtensorMap &b_hi,
                          const CUtensorMap &b_lo, const GemmParams &p, cudaStream_t s) {
  using Cfg = GemmCfg<BK, STAGES, SPLIT, SCATTER, PAIR, gemm_tstore<SPLIT, SCATTER, MN>()>;
  auto kernel = k_gemm_tc<BK, STAGES, SPLIT, SCATTER, MN, PAIR>;
  // per device: the shared-memory attribute and the persistent grid size
  // (CTAs, or clusters for pairs)
  constexpr int MAX_DEV = 64;
  static bool configured_dev[MAX_DEV] = {};
  static int max_units_dev[MAX_DEV] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= MAX_DEV) return cudaErrorInvalidDevice;
  bool &configured = configured_dev[dev];
  int &max_units = max_units_dev[dev];
  if (!configured) {
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         Cfg::SMEM);
    if (e != cudaSuccess) return e;
    max_units = num_sms();
    if (PAIR) {
      // clusters of two CTAs that can be resident at once (both SMs of a TPC)
      cudaLaunchConfig_t cfg{};
      cudaLaunchAttribute attr[1];
      attr[0].id = cudaLaunchAttributeClusterDimension;
      attr[0].val.clusterDim.x = 2;
      attr[0].val.clusterDim.y = 1;
      attr[0].val.clusterDim.z = 1;
      cfg.gridDim = dim3(2 * max_units, 1, 1);
      cfg.blockDim = dim3(GEMM_THREADS, 1, 1);
      cfg.dynamicSmemBytes = Cfg::SMEM;
      cfg.attrs = attr;
      cfg.numAttrs = 1;
      int n = 0;
      e = cudaOccupancyMaxActiveClusters(&n, kernel, &cfg);
      if (e != cudaSuccess) return e;
      if (n < 1) return cudaErrorInvalidConfiguration;
      max_units = n;
    }
    configured = true;
  }
  const int units = p.total_tiles < max_units ? p.total_tiles : max_units;
  if (!PAIR) {
    kernel<<<units, GEMM_THREADS, Cfg::SMEM, s>>>(a_hi, a_lo, b_hi, b_lo, p);
    return cudaPeekAtLastError();
  }
  cudaLaunchConfig_t cfg{};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.gridDim = dim3(2 * units, 1, 1);
  cfg.blockDim = dim3(GEMM_THREADS, 1, 1);
  cfg.dynamicSmemBytes = Cfg::SMEM;
  cfg.stream = s;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, a_hi, a_lo, b_hi, b_lo, p);
}

cudaError_t launch_gemm(int kind, bool split, const CUtensorMap &a_hi, const CUtensorMap &a_lo,
                        const CUtensorMap &b_hi, const CUtensorMap &b_lo, GemmParams p,
                        float *C, int beta, DevStatus *st, cudaStream_t s,
                        const GemmScatter *sc = nullptr, bool store = true, bool mn = false,
                        bool pair = false, bool cbf16 = false) {
  if (p.total_tiles == 0) return cudaSuccess;
  p.C = C;
  p.cbf16 = cbf16 ? 1 : 0;
  p.beta = beta;
  p.split = split ? 1 : 0;
  p.status = st;
  p.store = store ? 1 : 0;
  p.scatter = sc ? 1 : 0;
  if (sc) p.sc = *sc;
  cudaEvent_t e0 = nullptr, e1 = nullptr;
  if (g_prof.on) {
    e0 = prof_event(kind);
    e1 = prof_event(kind);
    if (e0) cudaEventRecord(e0, s);
  }
  ++g_launches;
  // the fused reduction epilogue's scratch (6.4 KB per epilogue warp) can cost
  // a pipeline stage
  cudaError_t r;
  if (sc && pair)
    r = split ? launch_gemm_t<SO2_SPLIT_BK, SO2_SPLIT_SCATTER_PAIR_STAGES, true, true, false, true>(a_hi, a_lo, b_hi, b_lo, p, s)
              : launch_gemm_t<64, SO2_SCATTER_PAIR_STAGES, false, true, false, true>(a_hi, a_lo, b_hi, b_lo, p, s);
  else if (sc)
    r = split ? launch_gemm_t<SO2_SPLIT_BK, SO2_SPLIT_SCATTER_STAGES, true, true, false>(a_hi, a_lo, b_hi, b_lo, p, s)
              : launch_gemm_t<64, SO2_SCATTER_STAGES, false, true, false>(a_hi, a_lo, b_hi, b_lo, p, s);
  else if (mn && pair)
    r = split ? launch_gemm_t<SO2_SPLIT_BK, SO2_SPLIT_MN_PAIR_STAGES, true, false, true, true>(a_hi, a_lo, b_hi, b_lo, p, s)
              : launch_gemm_t<64, 6, false, false, true, true>(a_hi, a_lo, b_hi, b_lo, p, s);
  else if (mn)
    r = split ? launch_gemm_t<SO2_SPLIT_BK, SO2_SPLIT_PLAIN_STAGES, true, false, true>(a_hi, a_lo, b_hi, b_lo, p, s)
              : launch_gemm_t<64, 4, false, false, true>(a_hi, a_lo, b_hi, b_lo, p, s);
  else if (pair)
    r = split ? launch_gemm_t<SO2_SPLIT_BK, SO2_SPLIT_PLAIN_PAIR_STAGES, true, false, false, true>(a_hi, a_lo, b_hi, b_lo, p, s)
              : launch_gemm_t<64, SO2_BF16_PLAIN_PAIR_STAGES, false, false, false, true>(a_hi, a_lo, b_hi, b_lo, p, s);
  else
    r = split ? launch_gemm_t<SO2_SPLIT_BK, SO2_SPLIT_PLAIN_STAGES, true, false, false>(a_hi, a_lo, b_hi, b_lo, p, s)
              : launch_gemm_t<64, SO2_BF16_PLAIN_STAGES, false, false, false>(a_hi, a_lo, b_hi, b_lo, p, s);
  if (e1) cudaEventRecord(e1, s);
  return r;
}

// --------------------------------------------------------------------------
// Shared pieces of the three entry points
// --------------------------------------------------------------------------
struct Ctx {
  const so2conv_desc *d;
  Plan P;
  void *ws;
  cudaStream_t s;
  DevStatus *st;
  CUtensorMap m_a_hi, m_a_lo, m_v_hi, m_v_lo, m_wst_hi, m_wst_lo, m_wtr_hi, m_wtr_lo;
  CUtensorMap m_wst2_hi, m_wst2_lo;  // stacked weights, half-height boxes (CTA pairs)
  CUtensorMap m_wtr2_hi, m_wtr2_lo;  // their transposes, likewise
  CUtensorMap m_amn_hi, m_amn_lo, m_vmn_hi, m_vmn_lo;  // the same planes, MN-major boxes
};

inline bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

// Product rows (V, Ga) are f32 on the split path and bf16 on the bf16 path
// (their rounding, 2^-9 relative, is far inside that path's tolerance, and it
// halves the bytes every consumer reads).  Element `elems` of the rows at
// workspace offset `off`, type-erased; kernels read it as their TF.
inline const float *prows(const Ctx &c, size_t off, size_t elems) {
  return reinterpret_cast<const float *>(static_cast<const char *>(c.ws) + off +
                                         elems * (c.P.split ? 4 : 2));
}

so2_status common_checks(const so2conv_desc *d, int64_t N, int64_t E, const void *x,
                         const int64_t *ei, const float *ev, so2conv_params prm, void *ws,
                         size_t ws_bytes, int which, Plan &P) {
  if (!desc_ok(d)) return d ? SO2_ERR_UNSUPPORTED : SO2_ERR_INVALID_ARG;
  if (N < 0 || E < 0 || N > (1ll << 30) || E > (1ll << 30)) return SO2_ERR_INVALID_ARG;
  if (N == 0 && E > 0) return SO2_ERR_INVALID_ARG;
  if ((N > 0 && !x) || (E > 0 && (!ei || !ev)) || !prm.w || !prm.w_rad || !prm.b_rad)
    return SO2_ERR_INVALID_ARG;
  if (!aligned16(x)) return SO2_ERR_INVALID_ARG;  // read with 16-byte vector loads
  if (!ws) return SO2_ERR_WORKSPACE;
  if (reinterpret_cast<uintptr_t>(ws) & 255) return SO2_ERR_WORKSPACE;
  P = make_plan(d, N, E, which);
  if (ws_bytes < P.total) return SO2_ERR_WORKSPACE;
  return SO2_OK;
}

so2_status build_maps(Ctx &c, bool bwd) {
  const Plan &P = c.P;
  const Layout &y = P.y;
  void *ws = c.ws;
  const int bk = gemm_bk(P.split);
  bool ok = true;
  const int64_t ra = (int64_t)P.na * P.chunk, rg = (int64_t)P.ngv * P.chunk;
  ok &= make_map(&c.m_a_hi, at<void>(ws, P.a_hi), ra, y.KA, y.KA, GEMM_BM, bk);
  ok &= make_map(&c.m_a_lo, at<void>(ws, P.split ? P.a_lo : P.a_hi), ra, y.KA, y.KA, GEMM_BM, bk);
  ok &= make_map(&c.m_wst_hi, at<void>(ws, P.wst_hi), y.WR, y.WK, y.WK, GEMM_BN, bk);
  ok &= make_map(&c.m_wst_lo, at<void>(ws, P.split ? P.wst_lo : P.wst_hi), y.WR, y.WK, y.WK, GEMM_BN, bk);
  ok &= make_map(&c.m_wst2_hi, at<void>(ws, P.wst_hi), y.WR, y.WK, y.WK, GEMM_BN / 2, bk);
  ok &= make_map(&c.m_wst2_lo, at<void>(ws, P.split ? P.wst_lo : P.wst_hi), y.WR, y.WK, y.WK, GEMM_BN / 2, bk);
  if (bwd) {
    ok &= make_map(&c.m_v_hi, at<void>(ws, P.gv_hi), rg, y.KG, y.KG, GEMM_BM, bk);
    ok &= make_map(&c.m_v_lo, at<void>(ws, P.split ? P.gv_lo : P.gv_hi), rg, y.KG, y.KG, GEMM_BM, bk);
    ok &= make_map(&c.m_wtr_hi, at<void>(ws, P.wtr_hi), y.WTR, y.WTK, y.WTK, GEMM_BN, bk);
    ok &= make_map(&c.m_wtr_lo, at<void>(ws, P.split ? P.wtr_lo : P.wtr_hi), y.WTR, y.WTK, y.WTK, GEMM_BN, bk);
    ok &= make_map(&c.m_wtr2_hi, at<void>(ws, P.wtr_hi), y.WTR, y.WTK, y.WTK, GEMM_BN / 2, bk);
    ok &= make_map(&c.m_wtr2_lo, at<void>(ws, P.split ? P.wtr_lo : P.wtr_hi), y.WTR, y.WTK, y.WTK, GEMM_BN / 2, bk);
    ok &= make_map_mn(&c.m_amn_hi, at<void>(ws, P.a_hi), ra, y.KA, y.KA, bk);
    ok &= make_map_mn(&c.m_amn_lo, at<void>(ws, P.split ? P.a_lo : P.a_hi), ra, y.KA, y.KA, bk);
    ok &= make_map_mn(&c.m_vmn_hi, at<void>(ws, P.gv_hi), rg, y.KG, y.KG, bk);
    ok &= make_map_mn(&c.m_vmn_lo, at<void>(ws, P.split ? P.gv_lo : P.gv_hi), rg, y.KG, y.KG, bk);
  }
  return ok ? SO2_OK : SO2_ERR_CUDA;
}

// Stable sort of edges by edge_index[key_row]; fills offsets [N+1] and perm [E].
so2_status sort_edges(Ctx &c, const int64_t *ei, int key_row) {
  const Plan &P = c.P;
  int *counts = at<int>(c.ws, P.counts), *cursor = at<int>(c.ws, P.cursor);
  int *offsets = at<int>(c.ws, P.offsets), *perm = at<int>(c.ws, P.perm);
  ProfScope ps(4, c.s);
  CK(cudaMemsetAsync(counts, 0, sizeof(int) * (P.N + 1), c.s));
  CK(cudaMemsetAsync(cursor, 0, sizeof(int) * (P.N + 1), c.s));
  const int64_t *keys = ei + key_row * P.E;
  k_count_keys<<<grid_for(P.E, 256), 256, 0, c.s>>>(keys, P.E, P.N, counts, c.st);
  CKL();
  k_scan_offsets<<<1, 1024, 0, c.s>>>(counts, P.N, offsets);
  CKL();
  k_place<<<grid_for(P.E, 256), 256, 0, c.s>>>(keys, P.E, P.N, offsets, cursor, perm);
  CKL();
  k_sort_segments<<<warp_grid(static_cast<int>(P.N), 8), 256, 0, c.s>>>(offsets, P.N, perm);
  CKL();
  return SO2_OK;
}

// Stacked weight planes (and, when the call needs them, their transposes).
so2_status pack_weights(Ctx &c, const void *w, bool transposes) {
  const Plan &P = c.P;
  const Layout &y = P.y;
  __nv_bfloat16 *wh = at<__nv_bfloat16>(c.ws, P.wst_hi), *wl = P.split ? at<__nv_bfloat16>(c.ws, P.wst_lo) : nullptr;
  __nv_bfloat16 *th = at<__nv_bfloat16>(c.ws, P.wtr_hi), *tl = P.split ? at<__nv_bfloat16>(c.ws, P.wtr_lo) : nullptr;
  ProfScope ps(7, c.s);
  // zero padding first
  CK(cudaMemsetAsync(wh, 0, 2ull * y.WR * y.WK, c.s));
  if (wl) CK(cudaMemsetAsync(wl, 0, 2ull * y.WR * y.WK, c.s));
  if (transposes) {
    CK(cudaMemsetAsync(th, 0, 2ull * y.WTR * y.WTK, c.s));
    if (tl) CK(cudaMemsetAsync(tl, 0, 2ull * y.WTR * y.WTK, c.s));
  }
  dim3 grid(256, y.ng);
  BlockOffsets bo = block_offsets(y);
  for (int t = 0; t < (transposes ? 2 : 1); ++t) {
    __nv_bfloat16 *h = t ? th : wh, *l = t ? tl : wl;
    if (P.xbf16)
      k_pack_weights<__nv_bfloat16><<<grid, 256, 0, c.s>>>(y, bo, static_cast<const __nv_bfloat16 *>(w), t, h, l);
    else
      k_pack_weights<float><<<grid, 256, 0, c.s>>>(y, bo, static_cast<const float *>(w), t, h, l);
    CKL();
  }
  return SO2_OK;
}

// Per chunk: records, frames, Wigner-D, gate.
so2_status chunk_prep(Ctx &c, int64_t e0, int M, const int64_t *ei, const float *ev, int key_row,
                      so2conv_params prm) {
  const Plan &P = c.P;
  ProfScope ps(4, c.s);
  const int smem = P.y.dsz * 33 * static_cast<int>(sizeof(float));
  bool ok = true;
  SO2_DISPATCH_L(P.y.L, ok = allow_smem(k_edge_prep<L>, smem);
                 if (ok) k_edge_prep<L><<<(M + 31) / 32, 32, smem, c.s>>>(
                     e0, M, at<int>(c.ws, P.perm), ei, P.E, P.N, key_row, ev,
                     at<EdgeRec>(c.ws, P.rec), at<float>(c.ws, P.geo), at<float>(c.ws, P.D), c.st,
                     P.y.mmax, P.DT ? at<float>(c.ws, P.DT) : nullptr, P.chunk));
  if (!ok) return SO2_ERR_CUDA;
  CKL();
  k_edge_gate<<<(M + GATE_EDGES - 1) / GATE_EDGES, 128, GATE_EDGES * P.y.nr * sizeof(float),
                c.s>>>(P.y, c.d->rbf_cutoff, M, at<float>(c.ws, P.geo), prm.w_rad, prm.b_rad,
                       at<float>(c.ws, P.gate));
  CKL();
  return SO2_OK;
}

// Rotation on gather into the grouped layout (rows of `out_*`, stride ld):
// out = A * D X + B * Omega D X  (see k_rotate_gather).
so2_status rotate(Ctx &c, int M, const void *X, bool xbf16, int side, int use_src, Coef A, Coef B,
                  const float *omega, __nv_bfloat16 *hi, __nv_bfloat16 *lo, int ld,
                  Coef A2 = Coef{nullptr, 0}, Coef B2 = Coef{nullptr, 0},
                  __nv_bfloat16 *hi2 = nullptr, __nv_bfloat16 *lo2 = nullptr) {
  const Plan &P = c.P;
  const EdgeRec *rec = at<EdgeRec>(c.ws, P.rec);
  const float *D = at<float>(c.ws, P.D);
  const int dsm = 8 * P.y.dsz * static_cast<int>(sizeof(float));  // staged D per warp
  ProfScope ps(3, c.s);
#define SO2_ROT_LAUNCH(TX, DU)                                                                 \
  DISPATCH_LM(P.y.L, P.y.mmax,                                                                 \
              (k_rotate_gather<TX, MM, LC, DU><<<warp_grid(M, 8), 256, dsm, c.s>>>(             \
                  P.y, M, rec, D, static_cast<const TX *>(X), side, use_src, A, B, omega, hi, lo, \
                  ld, A2, B2, hi2, lo2)))
  if (xbf16) {
    if (hi2) {
      SO2_ROT_LAUNCH(__nv_bfloat16, true);
    } else {
      SO2_ROT_LAUNCH(__nv_bfloat16, false);
    }
  } else {
    if (hi2) {
      SO2_ROT_LAUNCH(float, true);
    } else {
      SO2_ROT_LAUNCH(float, false);
    }
  }
#undef SO2_ROT_LAUNCH
  CKL();
  return SO2_OK;
}

constexpr Coef ZERO{nullptr, 0};
constexpr Coef ONE{nullptr, 1};
inline Coef arr(const float *p) { return Coef{p, 2}; }

// x[src] rotated into rows [row0, row0 + M) of the a-operand planes.
so2_status rotate_x(Ctx &c, int M, const void *x, bool xbf16, int row0 = 0, Coef A = ONE,
                    Coef B = ZERO, const float *omega = nullptr) {
  const Plan &P = c.P;
  const size_t off = (size_t)row0 * P.y.KA;
  __nv_bfloat16 *hi = at<__nv_bfloat16>(c.ws, P.a_hi) + off;
  __nv_bfloat16 *lo = P.split ? at<__nv_bfloat16>(c.ws, P.a_lo) + off : nullptr;
  return rotate(c, M, x, xbf16, 0, 1, A, B, omega, hi, lo, P.y.KA);
}

// x[src] rotated once into two row sets of the a-operand planes:
// rows [row0, row0 + M) get A * D x + B * Omega D x, rows [row1, ...) A2, B2.
so2_status rotate_x2(Ctx &c, int M, const void *x, bool xbf16, int row0, Coef A, Coef B,
                     int row1, Coef A2, Coef B2, const float *omega) {
  const Plan &P = c.P;
  __nv_bfloat16 *hi = at<__nv_bfloat16>(c.ws, P.a_hi);
  __nv_bfloat16 *lo = P.split ? at<__nv_bfloat16>(c.ws, P.a_lo) : nullptr;
  const size_t o0 = (size_t)row0 * P.y.KA, o1 = (size_t)row1 * P.y.KA;
  return rotate(c, M, x, xbf16, 0, 1, A, B, omega, hi + o0, lo ? lo + o0 : nullptr, P.y.KA, A2,
                B2, hi + o1, lo ? lo + o1 : nullptr);
}

// G[dst] rotated once into two row sets of the output-side operand planes.
so2_status rotate_g2(Ctx &c, int M, const float *G, int row0, Coef A, Coef B, int row1, Coef A2,
                     Coef B2, const float *omega) {
  const Plan &P = c.P;
  __nv_bfloat16 *hi = at<__nv_bfloat16>(c.ws, P.gv_hi);
  __nv_bfloat16 *lo = P.split ? at<__nv_bfloat16>(c.ws, P.gv_lo) : nullptr;
  const size_t o0 = (size_t)row0 * P.y.KG, o1 = (size_t)row1 * P.y.KG;
  return rotate(c, M, G, false, 1, 0, A, B, omega, hi + o0, lo ? lo + o0 : nullptr, P.y.KG, A2,
                B2, hi + o1, lo ? lo + o1 : nullptr);
}

// G[dst] rotated (with coefficients) into rows [row0, row0 + M) of the
// output-side operand planes.
so2_status rotate_g(Ctx &c, int M, const float *G, int row0, Coef A, Coef B = ZERO,
                    const float *omega = nullptr) {
  const Plan &P = c.P;
  const size_t off = (size_t)row0 * P.y.KG;
  __nv_bfloat16 *hi = at<__nv_bfloat16>(c.ws, P.gv_hi) + off;
  __nv_bfloat16 *lo = P.split ? at<__nv_bfloat16>(c.ws, P.gv_lo) + off : nullptr;
  return rotate(c, M, G, false, 1, 0, A, B, omega, hi, lo, P.y.KG);
}

// Zero rows [row0 + M, row0 + roundup(M, 64)) of both planes of the input
// (out_side = false) or output side operand, so that a weight-gradient
// product over the padded edge range adds nothing for them.
so2_status zero_tail(Ctx &c, int M, bool out_side, int row0) {
  const Plan &P = c.P;
  const int K = out_side ? P.y.KG : P.y.KA;
  const int Kp = round_up(M, 64);
  if (Kp == M) return SO2_OK;
  const size_t off = (size_t)(row0 + M) * K * 2, bytes = (size_t)(Kp - M) * K * 2;
  char *hi = at<char>(c.ws, out_side ? P.gv_hi : P.a_hi);
  CK(cudaMemsetAsync(hi + off, 0, bytes, c.s));
  if (P.split) {
    char *lo = at<char>(c.ws, out_side ? P.gv_lo : P.a_lo);
    CK(cudaMemsetAsync(lo + off, 0, bytes, c.s));
  }
  return SO2_OK;
}

// dW (+)= (rows of segment seg_g of the output-side planes)^T x (rows of
// segment seg_a of the input-side planes): K = edges, both operands read
// MN-major straight from the edge-major planes.
so2_status gemm_dw(Ctx &c, int M, int seg_g, int seg_a) {
  const Plan &P = c.P;
  const Layout &y = P.y;
  const int Kp = round_up(M, 64);
  // The output is small (a few hundred tiles at most) and K long: split K.
  // Pick the split count that wastes least of the last wave (the time is
  // waves x K per split), keeping at least 2,048 edges per split so that the
  // atomic epilogue of a split stays hidden behind the next one's main loop.
  const bool pair = SO2_PAIR_MN;
  const int bm = pair ? 2 * GEMM_BM : GEMM_BM;
  int tiles = 0;
  for (int g = 0; g < y.ng; ++g)
    tiles += ((y.Kout[g] + bm - 1) / bm) * ((y.Kin[g] + GEMM_BN - 1) / GEMM_BN);
  const int sms = pair ? num_sms() / 2 : num_sms();  // concurrent tiles
  const int max_split = Kp / 2048 > 1 ? Kp / 2048 : 1;
  int ksplit = 1;
  long long best = -1;
  for (int ks = 1; ks <= max_split; ++ks) {
    const long long waves = (static_cast<long long>(tiles) * ks + sms - 1) / sms;
    const long long cost = waves * round_up((Kp + ks - 1) / ks, 64);
    if (best < 0 || cost < best) {
      best = cost;
      ksplit = ks;
    }
  }
  GemmLauncher L;
  L.bm = bm;
  for (int g = 0; g < y.ng; ++g)
    L.add(y.Kout[g], y.Kin[g], Kp, y.kout_off[g], seg_g * P.chunk, y.kin_off[g], seg_a * P.chunk,
          static_cast<long long>(y.wr_off[g]) * y.WK, y.WK, ksplit);
  CK(launch_gemm(2, P.split, c.m_vmn_hi, c.m_vmn_lo, c.m_amn_hi, c.m_amn_lo, L.p,
                 at<float>(c.ws, P.dws), 1, c.st, c.s, nullptr, true, true, pair));
  return SO2_OK;
}

// Ga rows = output-side operand rows times the transposed stacked weights
// (rows [row0, row0 + rows) of both).
so2_status gemm_ga(Ctx &c, int rows, const GemmScatter *sc = nullptr, bool store = true,
                   int row0 = 0) {
  const Plan &P = c.P;
  const Layout &y = P.y;
  const bool pair = sc ? SO2_PAIR_SCATTER : SO2_PAIR_PLAIN;
  GemmLauncher L;
  L.bm = pair ? 2 * GEMM_BM : GEMM_BM;
  for (int g = 0; g < y.ng; ++g)
    L.add(rows, y.Kin[g], y.Kout_pad[g], row0, y.kout_off[g], y.wt_off[g], 0,
          static_cast<long long>(row0) * y.KA + y.kin_off[g], y.KA);
  CK(launch_gemm(1, P.split, c.m_v_hi, c.m_v_lo, pair ? c.m_wtr2_hi : c.m_wtr_hi,
                 pair ? c.m_wtr2_lo : c.m_wtr_lo, L.p, at<float>(c.ws, P.Ga), 0, c.st, c.s, sc,
                 store, false, pair, !P.split));
  return SO2_OK;
}

// V = rotated features times stacked weights (one group per m).  The plain
// product runs on CTA pairs (256 x 256 tiles, half of B per CTA).
so2_status gemm_v(Ctx &c, int rows, const GemmScatter *sc = nullptr, bool store = true) {
  const Plan &P = c.P;
  const Layout &y = P.y;
  const bool pair = sc ? SO2_PAIR_SCATTER : SO2_PAIR_PLAIN;
  GemmLauncher L;
  L.bm = pair ? 2 * GEMM_BM : GEMM_BM;
  for (int g = 0; g < y.ng; ++g)
    L.add(rows, y.Kout[g], y.Kin_pad[g], 0, y.kin_off[g], y.wr_off[g], 0, y.kout_off[g], y.KG);
  CK(launch_gemm(0, P.split, c.m_a_hi, c.m_a_lo, pair ? c.m_wst2_hi : c.m_wst_hi,
                 pair ? c.m_wst2_lo : c.m_wst_lo, L.p, at<float>(c.ws, P.V), 0, c.st, c.s, sc,
                 store, false, pair, !P.split));
  return SO2_OK;
}

// The fused gate + inverse rotation + reduction epilogue needs whole 32-wide
// channel chunks inside one edge-frame row.
// Whether the reduction onto nodes runs in the product's epilogue.  The
// epilogue costs the same per tile on both paths, but the bf16 product's main
// loop is three times shorter, so there the epilogue would set the pace:
// bf16 products store their rows and k_reduce_nodes reduces them
// (measured 2-4 % faster per step); the split f32 path keeps the fusion.
bool fusable(int C, bool split) {
  return C % 32 == 0 && (split ? SO2_FUSE_F32 : SO2_FUSE_BF16);
}

GemmScatter make_scatter(Ctx &c, const float *gate, float *out, int C) {
  GemmScatter sc;
  sc.rec = at<int4>(c.ws, c.P.rec);
  sc.gate = gate;
  sc.DT = at<float>(c.ws, c.P.DT);
  sc.out = out;
  sc.C = C;
  sc.L = c.P.y.L;
  sc.dt_chunk = c.P.chunk;
  return sc;
}

// Node-centric inverse rotation on reduction (see k_scatter_nodes) for the
// chunk's nodes, on `side` (0: input channels, 1: output channels).
so2_status scatter(Ctx &c, int64_t e0, int M, const ScatterTerms &t, int side,
                   const float *omega, float *out) {
  const Plan &P = c.P;
  const Layout &y = P.y;
  const int C = side ? y.co : y.ci;
  int threads = C / 2;
  threads = threads < 32 ? 32 : (threads > 256 ? 256 : threads);
  const int smem = y.S * C * static_cast<int>(sizeof(float));
  const EdgeRec *rec = at<EdgeRec>(c.ws, P.rec);
  const int *off = at<int>(c.ws, P.offsets);
  const float *D = at<float>(c.ws, P.D);
  ProfScope ps(7, c.s);
  if (!(reinterpret_cast<uintptr_t>(out) & 15)) {  // node-centric kernel with vector RMW
    if (P.split) {
      DISPATCH_MM(y.mmax, k_reduce_nodes_terms<MM, float><<<warp_grid(M, 8), 256, 0, c.s>>>(
                              y, e0, M, rec, off, D, t, side, omega, out));
    } else {
      DISPATCH_MM(y.mmax, k_reduce_nodes_terms<MM, __nv_bfloat16><<<warp_grid(M, 8), 256, 0, c.s>>>(
                              y, e0, M, rec, off, D, t, side, omega, out));
    }
    CKL();
    return SO2_OK;
  }
  bool ok = true;
  if (P.split) {
    DISPATCH_MM(y.mmax, ok = allow_smem(k_scatter_nodes<MM, float>, smem);
                if (ok) k_scatter_nodes<MM, float><<<grid_for(M, 1), threads, smem, c.s>>>(
                    y, e0, M, rec, off, D, t, side, omega, out));
  } else {
    DISPATCH_MM(y.mmax, ok = allow_smem(k_scatter_nodes<MM, __nv_bfloat16>, smem);
                if (ok) k_scatter_nodes<MM, __nv_bfloat16><<<grid_for(M, 1), threads, smem, c.s>>>(
                    y, e0, M, rec, off, D, t, side, omega, out));
  }
  if (!ok) return SO2_ERR_CUDA;
  CKL();
  return SO2_OK;
}

// One-term node-centric reduction (see k_reduce_nodes): out += D^T (k * F)
// per node; falls back to the general kernel when out is not 16-byte aligned.
// F: product rows from prows() (element type of the path).
so2_status reduce_nodes(Ctx &c, int64_t e0, int M, const float *F, int ld, const float *coef,
                        int side, float *out) {
  const Plan &P = c.P;
  const Layout &y = P.y;
  if (reinterpret_cast<uintptr_t>(out) & 15) {
    ScatterTerms t{};
    t.F[0] = F;
    t.ld[0] = ld;
    t.A[0] = coef ? Coef{coef, 2} : Coef{nullptr, 1};
    return scatter(c, e0, M, t, side, nullptr, out);
  }
  ProfScope ps(7, c.s);
  if (P.split) {
    DISPATCH_MM(y.mmax, k_reduce_nodes<MM, float><<<warp_grid(M, 8), 256, 0, c.s>>>(
                            y, e0, M, at<EdgeRec>(c.ws, P.rec), at<int>(c.ws, P.offsets),
                            at<float>(c.ws, P.D), F, ld, coef, side, out));
  } else {
    DISPATCH_MM(y.mmax, k_reduce_nodes<MM, __nv_bfloat16><<<warp_grid(M, 8), 256, 0, c.s>>>(
                            y, e0, M, at<EdgeRec>(c.ws, P.rec), at<int>(c.ws, P.offsets),
                            at<float>(c.ws, P.D), reinterpret_cast<const __nv_bfloat16 *>(F),
                            ld, coef, side, out));
  }
  CKL();
  return SO2_OK;
}

so2_status rad_grads(Ctx &c, int M, const float *Ag, const float *Bg, const float *omega,
                     float *grad_w_rad, float *grad_b) {
  const Plan &P = c.P;
  const Layout &y = P.y;
  const int nblk = (M + RAD_TILE - 1) / RAD_TILE;
  const int sm = 2 * RAD_TILE * y.nr * static_cast<int>(sizeof(float));
  if (!allow_smem(k_rad_partial, sm)) return SO2_ERR_CUDA;
  ProfScope ps(6, c.s);
  k_rad_partial<<<nblk, 128, sm, c.s>>>(y, c.d->rbf_cutoff, M, at<float>(c.ws, P.geo), Ag, Bg,
                                        omega, at<float>(c.ws, P.radp));
  CKL();
  const int Pn = (y.nr + 1) * y.co;
  k_rad_reduce<<<(Pn + 31) / 32, 32 * RAD_RED_WARPS, 0, c.s>>>(y, nblk, at<float>(c.ws, P.radp),
                                                                grad_w_rad, grad_b);
  CKL();
  return SO2_OK;
}

// Per-edge gradient terms of the backward (see k_edge_terms): part 1 the
// output side (Gg, h; with write_gv also the transposed product's operand
// planes), part 2 the input side (adds to h and writes grad_r).
so2_status edge_terms(Ctx &c, int M, int part, const void *x, const float *grad_out,
                      bool write_gv, const float *w_rad = nullptr, float *grad_r = nullptr) {
  const Plan &P = c.P;
  const Layout &y = P.y;
  ProfScope ps(5, c.s);
  const int sm = 8 * (y.dsz + RAD_MAX_NR) * 4;
  const int g = warp_grid(M, 8);
  const EdgeRec *rec = at<EdgeRec>(c.ws, P.rec);
  const float *Dp = at<float>(c.ws, P.D), *gate = at<float>(c.ws, P.gate);
  const float *Vp = prows(c, P.V, 0), *Gap = prows(c, P.Ga, 0);
  float *Ggp = at<float>(c.ws, P.Gg);
  float4 *hp = at<float4>(c.ws, P.h);
  const float *geo = at<float>(c.ws, P.geo);
  const float cut = c.d->rbf_cutoff;
  __nv_bfloat16 *gh = write_gv ? at<__nv_bfloat16>(c.ws, P.gv_hi) : nullptr;
  __nv_bfloat16 *gl = write_gv && P.split ? at<__nv_bfloat16>(c.ws, P.gv_lo) : nullptr;
#define SO2_ET_LAUNCH(TX, TF)                                                                \
  DISPATCH_LM(y.L, y.mmax,                                                                   \
              /* all levels inlined spills at lmax 6: runtime-degree kernel there */          \
              constexpr int LE = (LC >= 0 && LC <= 4) ? LC : -1;                              \
              if (part == 1) k_edge_terms<TX, MM, LE, 1, TF><<<g, 256, sm, c.s>>>(             \
                  y, M, rec, Dp, gate, grad_out, static_cast<const TX *>(x),                  \
                  reinterpret_cast<const TF *>(Vp), reinterpret_cast<const TF *>(Gap), Ggp,   \
                  hp, gh, gl, geo, w_rad, cut, nullptr);                                      \
              else k_edge_terms<TX, MM, LE, 2, TF><<<g, 256, sm, c.s>>>(                       \
                  y, M, rec, Dp, gate, grad_out, static_cast<const TX *>(x),                  \
                  reinterpret_cast<const TF *>(Vp), reinterpret_cast<const TF *>(Gap), Ggp,   \
                  hp, nullptr, nullptr, geo, w_rad, cut, grad_r);)
  if (P.xbf16) {
    SO2_ET_LAUNCH(__nv_bfloat16, __nv_bfloat16)
  } else {
    SO2_ET_LAUNCH(float, float)
  }
#undef SO2_ET_LAUNCH
  CKL();
  return SO2_OK;
}

// --------------------------------------------------------------------------
// Message block (two SO(2) convolutions with the activation between them).
// Two contexts share one workspace: the per-edge records, frames, Wigner-D,
// sort, edge-gradient record and output-side operand planes are common; each
// conv has its own gate, packed weights, operand planes (conv 2's are the
// activation h'), product rows and weight-gradient accumulator.
// --------------------------------------------------------------------------
struct BlockPlan {
  Plan p1, p2;
  size_t total = 0;
};

BlockPlan make_block_plan(const so2conv_desc *d, int64_t N, int64_t E, int which) {
  BlockPlan b;
  b.p1 = make_plan(d, N, E, which ? SO2_WS_BACKWARD : SO2_WS_FORWARD);
  const Plan &p = b.p1;
  const Layout &y = p.y;
  size_t c = p.total;
  Plan q = p;
  const size_t lo = p.split ? 1 : 0, pe = p.split ? 4 : 2;
  q.gate = take(c, 4ull * y.co * p.chunk);
  q.wst_hi = take(c, 2ull * y.WR * y.WK);
  q.wst_lo = take(c, 2ull * y.WR * y.WK * lo);
  q.a_hi = take(c, 2ull * p.chunk * y.KA);
  q.a_lo = take(c, 2ull * p.chunk * y.KA * lo);
  if (which) {
    q.wtr_hi = take(c, 2ull * y.WTR * y.WTK);
    q.wtr_lo = take(c, 2ull * y.WTR * y.WTK * lo);
    q.V = take(c, pe * p.chunk * y.KG);
    q.Gg = take(c, 4ull * p.chunk * y.co);
    q.dws = take(c, 4ull * y.WR * y.WK);
  }
  b.p2 = q;
  b.total = (c + 1023) & ~static_cast<size_t>(1023);
  b.p1.total = b.p2.total = b.total;
  return b;
}

// The gate of a second conv for the chunk's edges (frames from chunk_prep).
so2_status gate_only(Ctx &c, int M, so2conv_params prm) {
  ProfScope ps(4, c.s);
  k_edge_gate<<<(M + GATE_EDGES - 1) / GATE_EDGES, 128, GATE_EDGES * c.P.y.nr * sizeof(float),
                c.s>>>(c.P.y, c.d->rbf_cutoff, M, at<float>(c.ws, c.P.geo), prm.w_rad, prm.b_rad,
                       at<float>(c.ws, c.P.gate));
  CKL();
  return SO2_OK;
}

so2_status block_setup(const so2conv_desc *d, int64_t N, int64_t E, const void *x,
                       const int64_t *ei, const float *ev, so2conv_params p1,
                       so2conv_params p2, void *ws, size_t ws_bytes, int which,
                       so2_stream_t stream, Ctx &c1, Ctx &c2) {
  if (!d) return SO2_ERR_INVALID_ARG;
  if (!desc_ok(d) || d->c_in != d->c_out) return SO2_ERR_UNSUPPORTED;
  if (!p2.w || !p2.w_rad || !p2.b_rad) return SO2_ERR_INVALID_ARG;
  Plan P;
  // argument checks of the single conv (the block's workspace is larger)
  so2_status r = common_checks(d, N, E, x, ei, ev, p1, ws, (size_t)-1,
                               which ? SO2_WS_BACKWARD : SO2_WS_FORWARD, P);
  if (r != SO2_OK) return r;
  const BlockPlan bp = make_block_plan(d, N, E, which);
  if (ws_bytes < bp.total) return SO2_ERR_WORKSPACE;
  for (Ctx *c : {&c1, &c2}) {
    c->d = d;
    c->ws = ws;
    c->s = reinterpret_cast<cudaStream_t>(stream);
    c->st = at<DevStatus>(ws, bp.p1.status);
  }
  c1.P = bp.p1;
  c2.P = bp.p2;
  CK(cudaMemsetAsync(c1.st, 0, sizeof(DevStatus), c1.s));
  return SO2_OK;
}

// h' = act(g1 * V1) as conv 2's operand planes.
so2_status block_act(Ctx &c1, Ctx &c2, int M) {
  const Plan &P = c1.P;
  ProfScope ps(5, c1.s);
  __nv_bfloat16 *hh = at<__nv_bfloat16>(c2.ws, c2.P.a_hi);
  __nv_bfloat16 *hl = P.split ? at<__nv_bfloat16>(c2.ws, c2.P.a_lo) : nullptr;
  if (P.split)
    k_block_act<float><<<warp_grid(M, 8), 256, 0, c1.s>>>(
        P.y, M, reinterpret_cast<const float *>(prows(c1, P.V, 0)), at<float>(c1.ws, P.gate), hh, hl);
  else
    k_block_act<__nv_bfloat16><<<warp_grid(M, 8), 256, 0, c1.s>>>(
        P.y, M, reinterpret_cast<const __nv_bfloat16 *>(prows(c1, P.V, 0)),
        at<float>(c1.ws, P.gate), hh, hl);
  CKL();
  return SO2_OK;
}

// Backward through the activation: conv 1's output-side planes, Gg1 and the
// gate's share of the edge gradient (k_block_act_bwd).
so2_status block_act_bwd(Ctx &c1, Ctx &c2, int M, const float *w_rad1) {
  const Plan &P = c1.P;
  ProfScope ps(5, c1.s);
  __nv_bfloat16 *gh = at<__nv_bfloat16>(c1.ws, P.gv_hi);
  __nv_bfloat16 *gl = P.split ? at<__nv_bfloat16>(c1.ws, P.gv_lo) : nullptr;
#define SO2_ABW(TF)                                                                            \
  k_block_act_bwd<TF><<<warp_grid(M, 8), 256, 0, c1.s>>>(                                      \
      P.y, c1.d->rbf_cutoff, M, at<float>(c1.ws, P.geo),                                       \
      reinterpret_cast<const TF *>(prows(c1, P.V, 0)), at<float>(c1.ws, P.gate),                \
      reinterpret_cast<const TF *>(prows(c2, c2.P.Ga, 0)), w_rad1, gh, gl, at<float>(c1.ws, P.Gg), \
      at<float4>(c1.ws, P.h))
  if (P.split) {
    SO2_ABW(float);
  } else {
    SO2_ABW(__nv_bfloat16);
  }
#undef SO2_ABW
  CKL();
  return SO2_OK;
}

// One thread waits, with the library's bounded wait, on an mbarrier phase
// that nothing completes; the wait gives up after limit_ns and records
// SO2_ERR_TIMEOUT (the path every tensor-core wait takes when a partner
// never arrives).
__global__ void k_wait_selftest(DevStatus *st, uint64_t limit_ns) {
  __shared__ uint64_t bar;
  if (threadIdx.x != 0) return;
  mbar_init(&bar, 1);
  fence_mbar_init();
  mbar_wait(&bar, 0, st, nullptr, limit_ns);
}

// Library-owned scratch for so2conv_forward_noalloc (see its declaration).
static __device__ __align__(256) unsigned char g_noalloc_ws[SO2_NOALLOC_WORKSPACE_BYTES];

// The array's device address differs per CUDA context (each context loads its
// own copy of this module), so it is cached per context, keyed by the
// driver's process-unique context id (a context created after
// cudaDeviceReset gets a new id, so a stale address is never reused).  The
// driver calls go through the runtime's entry-point query, so the library
// does not link libcuda.
typedef CUresult (*CtxGetCurrentFn)(CUcontext *);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long *);
struct NoallocSlot {
  unsigned long long ctx_id;
  void *ptr;
};
constexpr int NOALLOC_MAX_CONTEXTS = 64;
NoallocSlot g_noalloc_slots[NOALLOC_MAX_CONTEXTS];
int g_noalloc_used = 0;
std::mutex g_noalloc_mu;

bool current_context_id(unsigned long long &id) {
  static CtxGetCurrentFn get_cur = nullptr;
  static CtxGetIdFn get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_cur = reinterpret_cast<CtxGetCurrentFn>(p);
    p = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<CtxGetIdFn>(p);
  });
  if (!get_cur || !get_id) return false;
  CUcontext ctx = nullptr;
  if (get_cur(&ctx) != CUDA_SUCCESS) return false;
  if (!ctx) {  // no context current yet: make the device's primary context current
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || cudaSetDevice(dev) != cudaSuccess) return false;
    if (get_cur(&ctx) != CUDA_SUCCESS || !ctx) return false;
  }
  return get_id(ctx, &id) == CUDA_SUCCESS;
}

// Device address of g_noalloc_ws in the current context: looked up with
// cudaGetSymbolAddress (the host-side name of the array is not a device
// address) the first time a context asks, then cached.
void *noalloc_base() {
  unsigned long long id = 0;
  if (!current_context_id(id)) return nullptr;
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  for (int i = 0; i < g_noalloc_used; ++i)
    if (g_noalloc_slots[i].ctx_id == id) return g_noalloc_slots[i].ptr;
  void *p = nullptr;
  if (cudaGetSymbolAddress(&p, g_noalloc_ws) != cudaSuccess || !p) return nullptr;
  const int i = g_noalloc_used < NOALLOC_MAX_CONTEXTS ? g_noalloc_used++ : NOALLOC_MAX_CONTEXTS - 1;
  g_noalloc_slots[i] = NoallocSlot{id, p};
  return p;
}

}  // namespace

// ============================================================================
// C ABI
// ============================================================================
extern "C" {

size_t so2conv_workspace_size(const so2conv_desc *desc, int64_t n_nodes, int64_t n_edges,
                              int which) {
  if (!desc_ok(desc) || n_nodes < 0 || n_edges < 0) return 0;
  return make_plan(desc, n_nodes, n_edges, which).total;
}

int64_t so2conv_num_weights(const so2conv_desc *desc) {
  if (!desc_ok(desc)) return 0;
  return num_weights(make_layout(desc->lmax, desc->mmax, desc->c_in, desc->c_out, desc->n_rbf));
}

so2_status so2conv_forward(const so2conv_desc *desc, int64_t N, int64_t E, const void *x,
                           const int64_t *edge_index, const float *edge_vec,
                           so2conv_params prm, float *out, void *ws, size_t ws_bytes,
                           so2_stream_t stream) {
  Plan P;
  so2_status r = common_checks(desc, N, E, x, edge_index, edge_vec, prm, ws, ws_bytes,
                               SO2_WS_FORWARD, P);
  if (r != SO2_OK) return r;
  if (N > 0 && !out) return SO2_ERR_INVALID_ARG;
  Ctx c;
  c.d = desc;
  c.P = P;
  c.ws = ws;
  c.s = reinterpret_cast<cudaStream_t>(stream);
  c.st = at<DevStatus>(ws, P.status);
  CK(cudaMemsetAsync(c.st, 0, sizeof(DevStatus), c.s));
  const Layout &y = P.y;
  if (N > 0) CK(cudaMemsetAsync(out, 0, sizeof(float) * N * y.S * y.co, c.s));
  if (E == 0) return SO2_OK;
  if ((r = build_maps(c, false)) != SO2_OK) return r;
  if ((r = sort_edges(c, edge_index, 1)) != SO2_OK) return r;
  if ((r = pack_weights(c, prm.w, false)) != SO2_OK) return r;
  for (int64_t e0 = 0; e0 < E; e0 += P.chunk) {
    const int M = static_cast<int>((E - e0) < P.chunk ? (E - e0) : P.chunk);
    const bool fuse = fusable(y.co, P.split);
    if ((r = chunk_prep(c, e0, M, edge_index, edge_vec, 1, prm)) != SO2_OK) return r;
    if ((r = rotate_x(c, M, x, P.xbf16)) != SO2_OK) return r;
    if (fuse) {
      // product, gate, inverse rotation and reduction in one kernel
      const GemmScatter sc = make_scatter(c, at<float>(ws, P.gate), out, y.co);
      if ((r = gemm_v(c, M, &sc, false)) != SO2_OK) return r;
    } else {
      if ((r = gemm_v(c, M)) != SO2_OK) return r;
      if ((r = reduce_nodes(c, e0, M, prows(c, P.V, 0), y.KG, at<float>(ws, P.gate), 1, out)) !=
          SO2_OK)
        return r;
    }
  }
  return SO2_OK;
}

so2_status so2conv_backward(const so2conv_desc *desc, int64_t N, int64_t E, const void *x,
                            const int64_t *edge_index, const float *edge_vec,
                            so2conv_params prm, const float *grad_out, float *grad_x,
                            float *grad_w, float *grad_w_rad, float *grad_b_rad,
                            float *grad_edge_vec, void *ws, size_t ws_bytes,
                            so2_stream_t stream) {
  Plan P;
  so2_status r = common_checks(desc, N, E, x, edge_index, edge_vec, prm, ws, ws_bytes,
                               SO2_WS_BACKWARD, P);
  if (r != SO2_OK) return r;
  if ((N > 0 && !grad_out) || !aligned16(grad_out)) return SO2_ERR_INVALID_ARG;
  Ctx c;
  c.d = desc;
  c.P = P;
  c.ws = ws;
  c.s = reinterpret_cast<cudaStream_t>(stream);
  c.st = at<DevStatus>(ws, P.status);
  CK(cudaMemsetAsync(c.st, 0, sizeof(DevStatus), c.s));
  const Layout &y = P.y;
  const int64_t nw = num_weights(y);
  if (grad_x && N > 0) CK(cudaMemsetAsync(grad_x, 0, sizeof(float) * N * y.S * y.ci, c.s));
  if (grad_w) CK(cudaMemsetAsync(grad_w, 0, sizeof(float) * nw, c.s));
  if (grad_w_rad) CK(cudaMemsetAsync(grad_w_rad, 0, sizeof(float) * y.nr * y.co, c.s));
  if (grad_b_rad) CK(cudaMemsetAsync(grad_b_rad, 0, sizeof(float) * y.co, c.s));
  if (E == 0) return SO2_OK;
  const bool need_v = grad_edge_vec || grad_w_rad || grad_b_rad;
  const bool need_ga = grad_x || grad_edge_vec;
  if ((r = build_maps(c, true)) != SO2_OK) return r;
  if ((r = sort_edges(c, edge_index, 0)) != SO2_OK) return r;
  if ((r = pack_weights(c, prm.w, true)) != SO2_OK) return r;
  float *dws = at<float>(ws, P.dws);
  if (grad_w) CK(cudaMemsetAsync(dws, 0, 4ull * y.WR * y.WK, c.s));
  for (int64_t e0 = 0; e0 < E; e0 += P.chunk) {
    const int M = static_cast<int>((E - e0) < P.chunk ? (E - e0) : P.chunk);
    if ((r = chunk_prep(c, e0, M, edge_index, edge_vec, 0, prm)) != SO2_OK) return r;
    if ((r = rotate_x(c, M, x, P.xbf16)) != SO2_OK) return r;
    // Gv = g * (D G[dst]) on the kept rows: written by the output-side edge
    // terms when they run (they rotate G[dst] anyway), else by rotation on gather
    if (need_v) {
      if ((r = gemm_v(c, M)) != SO2_OK) return r;
      if ((r = edge_terms(c, M, 1, x, grad_out, true, prm.w_rad)) != SO2_OK) return r;
    } else if ((r = rotate_g(c, M, grad_out, 0, arr(at<float>(ws, P.gate)))) != SO2_OK) {
      return r;
    }
    const bool fuse_gx = grad_x && fusable(y.ci, P.split);
    if (need_ga) {
      const GemmScatter sc = make_scatter(c, nullptr, grad_x, y.ci);
      if ((r = gemm_ga(c, M, fuse_gx ? &sc : nullptr, grad_edge_vec != nullptr || !fuse_gx)) !=
          SO2_OK)
        return r;
    }
    if (grad_w) {
      if ((r = zero_tail(c, M, false, 0)) != SO2_OK) return r;
      if ((r = zero_tail(c, M, true, 0)) != SO2_OK) return r;
      if ((r = gemm_dw(c, M, 0, 0)) != SO2_OK) return r;
    }
    if (grad_x && !fuse_gx &&
        (r = reduce_nodes(c, e0, M, prows(c, P.Ga, 0), y.KA, nullptr, 0, grad_x)) != SO2_OK)
      return r;
    if (need_v) {
      if (grad_edge_vec &&
          (r = edge_terms(c, M, 2, x, grad_out, false, prm.w_rad, grad_edge_vec)) != SO2_OK)
        return r;
      if ((grad_w_rad || grad_b_rad) &&
          (r = rad_grads(c, M, at<float>(ws, P.Gg), nullptr, nullptr, grad_w_rad, grad_b_rad)) !=
              SO2_OK)
        return r;
    }
  }
  if (grad_w) {
    ProfScope ps(7, c.s);
    k_unstack_grad<<<dim3(UNSTACK_BLOCKS, y.ng), 256, 0, c.s>>>(y, block_offsets(y), dws,
                                                             grad_w);
    CKL();
  }
  return SO2_OK;
}

// Double backward.  With gg_r the cotangent on grad_edge_vec, each edge's
// frame turns by Omega = w_x J_x + w_y J_y (dD = Omega D) and its gate moves
// by dg; with gg_x the cotangent on grad_x.  Writing Gy~ = D G[dst] (kept
// rows), Gv = g Gy~, a = D x[src], da = trunc(Omega D x[src]),
// a~ = D gg_x[src], P = g trunc(Omega D G[dst]) + dg Gy~, V = M a,
// dV = M da, V~ = M a~:
//   Q = sum_e <P, M a> + <Gv, M da> + <Gv, M a~>
//   d_x[src]      += D^T (M^T P - Omega M^T Gv)
//   d_grad_out[d] += D^T (dg V + g dV + g V~ - Omega (g V))
//   d_W           += P (x) a + Gv (x) da + Gv (x) a~
//   dQ/dg  = sum_rows (Omega Gy~) V + Gy~ dV + Gy~ V~,  dQ/ddg = sum_rows Gy~ V
// Pass A runs in source order (d_x), pass B in destination order (the rest).
so2_status so2conv_double_backward(const so2conv_desc *desc, int64_t N, int64_t E, const void *x,
                                   const int64_t *edge_index, const float *edge_vec,
                                   so2conv_params prm, const float *grad_out, const float *gg_x,
                                   const float *gg_edge_vec, float *d_x, float *d_w,
                                   float *d_w_rad, float *d_b_rad, float *d_grad_out,
                                   float *d_edge_vec, void *ws, size_t ws_bytes,
                                   so2_stream_t stream) {
  if (!desc) return SO2_ERR_INVALID_ARG;
  Plan P;
  so2_status r = common_checks(desc, N, E, x, edge_index, edge_vec, prm, ws, ws_bytes,
                               SO2_WS_DOUBLE_BACKWARD, P);
  if (r != SO2_OK) return r;
  if ((N > 0 && !grad_out) || !aligned16(grad_out)) return SO2_ERR_INVALID_ARG;
  Ctx c;
  c.d = desc;
  c.P = P;
  c.ws = ws;
  c.s = reinterpret_cast<cudaStream_t>(stream);
  c.st = at<DevStatus>(ws, P.status);
  CK(cudaMemsetAsync(c.st, 0, sizeof(DevStatus), c.s));
  const Layout &y = P.y;
  const int64_t nw = num_weights(y);
  if (d_x && N > 0) CK(cudaMemsetAsync(d_x, 0, sizeof(float) * N * y.S * y.ci, c.s));
  if (d_grad_out && N > 0) CK(cudaMemsetAsync(d_grad_out, 0, sizeof(float) * N * y.S * y.co, c.s));
  if (d_w) CK(cudaMemsetAsync(d_w, 0, sizeof(float) * nw, c.s));
  if (d_w_rad) CK(cudaMemsetAsync(d_w_rad, 0, sizeof(float) * y.nr * y.co, c.s));
  if (d_b_rad) CK(cudaMemsetAsync(d_b_rad, 0, sizeof(float) * y.co, c.s));
  if (d_edge_vec && E > 0) CK(cudaMemsetAsync(d_edge_vec, 0, sizeof(float) * 3 * E, c.s));
  if (!aligned16(gg_x)) return SO2_ERR_INVALID_ARG;
  const bool has_r = gg_edge_vec != nullptr, has_x = gg_x != nullptr;
  if (E == 0 || (!has_r && !has_x)) return SO2_OK;
  if ((r = build_maps(c, true)) != SO2_OK) return r;
  if ((r = pack_weights(c, prm.w, true)) != SO2_OK) return r;
  const Coef gate = arr(at<float>(ws, P.gate));
  const Coef dgate = arr(at<float>(ws, P.dgate));
  const float *omega = at<float>(ws, P.omega);
  float *dws = at<float>(ws, P.dws);
  if (d_w) CK(cudaMemsetAsync(dws, 0, 4ull * y.WR * y.WK, c.s));
  const int ch = P.chunk;

  // ---- pass A (source order): d_x, and the input side of d_edge_vec ----
  if ((d_x && has_r) || d_edge_vec) {
    if ((r = sort_edges(c, edge_index, 0)) != SO2_OK) return r;
    for (int64_t e0 = 0; e0 < E; e0 += ch) {
      const int M = static_cast<int>((E - e0) < ch ? (E - e0) : ch);
      if ((r = chunk_prep(c, e0, M, edge_index, edge_vec, 0, prm)) != SO2_OK) return r;
      if (has_r) {
        {
          ProfScope ps(5, c.s);
          k_edge_omega<<<warp_grid(M, 8), 256, 0, c.s>>>(
              y, desc->rbf_cutoff, M, at<EdgeRec>(ws, P.rec), at<float>(ws, P.geo), gg_edge_vec,
              prm.w_rad, at<float>(ws, P.omega), at<float>(ws, P.dgate));
          CKL();
        }
        // P = dg * b + g * Omega b and Gv = g * b from one rotation b = D G[dst]
        if ((r = rotate_g2(c, M, grad_out, 0, dgate, gate, ch, gate, ZERO, omega)) != SO2_OK)
          return r;
        if ((r = gemm_ga(c, ch + M)) != SO2_OK) return r;  // [M^T P; M^T Gv]
      } else {
        if ((r = rotate_g(c, M, grad_out, ch, gate)) != SO2_OK) return r;  // Gv = g * b
        if ((r = gemm_ga(c, M, nullptr, true, ch)) != SO2_OK) return r;    // M^T Gv
      }
      if (d_x && has_r) {
        ScatterTerms t{};
        t.F[0] = prows(c, P.Ga, 0);
        t.ld[0] = y.KA;
        t.A[0] = ONE;
        t.F[1] = prows(c, P.Ga, (size_t)ch * y.KA);
        t.ld[1] = y.KA;
        t.B[1] = ONE;
        if ((r = scatter(c, e0, M, t, 0, omega, d_x)) != SO2_OK) return r;
      }
      if (d_edge_vec) {
        ProfScope ps(5, c.s);
        const float *Gap = prows(c, P.Ga, (size_t)ch * y.KA);
        const float *MPp = has_r ? prows(c, P.Ga, 0) : nullptr;
        CK(launch_hess_in(y, warp_grid(M, 8), M, at<EdgeRec>(ws, P.rec), at<float>(ws, P.D),
                          at<float>(ws, P.geo), x, P.xbf16, gg_x, has_r ? omega : nullptr, Gap,
                          MPp, !P.split, d_edge_vec, c.s));
        CKL();
      }
    }
  }

  // ---- pass B (destination order): d_grad_out, radial gate, d_W, the
  // output side of d_edge_vec ----
  if (d_grad_out || d_w || d_w_rad || d_b_rad || d_edge_vec) {
    if ((r = sort_edges(c, edge_index, 1)) != SO2_OK) return r;
    for (int64_t e0 = 0; e0 < E; e0 += ch) {
      const int M = static_cast<int>((E - e0) < ch ? (E - e0) : ch);
      if ((r = chunk_prep(c, e0, M, edge_index, edge_vec, 1, prm)) != SO2_OK) return r;
      if (has_r) {
        ProfScope ps(5, c.s);
        k_edge_omega<<<warp_grid(M, 8), 256, 0, c.s>>>(
            y, desc->rbf_cutoff, M, at<EdgeRec>(ws, P.rec), at<float>(ws, P.geo), gg_edge_vec,
            prm.w_rad, at<float>(ws, P.omega), at<float>(ws, P.dgate));
        CKL();
      }
      // a-operand rows: [a; da; a~]
      if (has_r) {  // a = D x and da = Omega D x from one rotation
        if ((r = rotate_x2(c, M, x, P.xbf16, 0, ONE, ZERO, ch, ZERO, ONE, omega)) != SO2_OK)
          return r;
      } else if ((r = rotate_x(c, M, x, P.xbf16, 0)) != SO2_OK) {
        return r;
      }
      if (has_x && (r = rotate_x(c, M, gg_x, false, 2 * ch)) != SO2_OK) return r;
      if ((r = gemm_v(c, has_x ? 2 * ch + M : (has_r ? ch + M : M))) != SO2_OK) return r;
      const float *V = prows(c, P.V, 0);
      const float *dV = prows(c, P.V, (size_t)ch * y.KG);
      const float *Vt = prows(c, P.V, (size_t)2 * ch * y.KG);
      if (d_grad_out && N > 0) {
        ScatterTerms t{};
        t.F[0] = V;
        t.ld[0] = y.KG;
        t.A[0] = has_r ? dgate : ZERO;
        t.B[0] = has_r ? gate : ZERO;
        if (has_r) {
          t.F[1] = dV;
          t.ld[1] = y.KG;
          t.A[1] = gate;
        }
        if (has_x) {
          t.F[2] = Vt;
          t.ld[2] = y.KG;
          t.A[2] = gate;
        }
        if ((r = scatter(c, e0, M, t, 1, has_r ? omega : nullptr, d_grad_out)) != SO2_OK) return r;
      }
      if (d_edge_vec) {
        ProfScope ps(5, c.s);
        CK(launch_hess_out(y, desc->rbf_cutoff, warp_grid(M, 8), M, at<EdgeRec>(ws, P.rec),
                           at<float>(ws, P.D), at<float>(ws, P.geo), at<float>(ws, P.gate),
                           grad_out, has_r ? omega : nullptr, V, has_r ? dV : nullptr,
                           has_x ? Vt : nullptr, !P.split, prm.w_rad, d_edge_vec, c.s));
        CKL();
      }
      if (d_w_rad || d_b_rad) {
        {
          ProfScope ps(5, c.s);
          CK(launch_edge_terms2(y, warp_grid(M, 8), M, at<EdgeRec>(ws, P.rec), at<float>(ws, P.D),
                              grad_out, has_r ? omega : nullptr, V, has_r ? dV : nullptr,
                              has_x ? Vt : nullptr, !P.split, at<float>(ws, P.tA),
                              at<float>(ws, P.tB), c.s));
          CKL();
        }
        if ((r = rad_grads(c, M, at<float>(ws, P.tA), has_r ? at<float>(ws, P.tB) : nullptr,
                           omega, d_w_rad, d_b_rad)) != SO2_OK)
          return r;
      }
      if (d_w) {
        if (has_r) {
          if ((r = rotate_g2(c, M, grad_out, 0, dgate, gate, ch, gate, ZERO, omega)) != SO2_OK)
            return r;
        } else if ((r = rotate_g(c, M, grad_out, ch, gate)) != SO2_OK) {
          return r;
        }
        if (has_r) {
          if ((r = zero_tail(c, M, true, 0)) != SO2_OK) return r;
          if ((r = zero_tail(c, M, false, 0)) != SO2_OK) return r;
          if ((r = zero_tail(c, M, false, ch)) != SO2_OK) return r;
        }
        if ((r = zero_tail(c, M, true, ch)) != SO2_OK) return r;
        if (has_x && (r = zero_tail(c, M, false, 2 * ch)) != SO2_OK) return r;
        if (has_r) {
          if ((r = gemm_dw(c, M, 0, 0)) != SO2_OK) return r;  // P (x) a
          if ((r = gemm_dw(c, M, 1, 1)) != SO2_OK) return r;  // Gv (x) da
        }
        if (has_x && (r = gemm_dw(c, M, 1, 2)) != SO2_OK) return r;  // Gv (x) a~
      }
    }
  }
  if (d_w) {
    ProfScope ps(7, c.s);
    k_unstack_grad<<<dim3(UNSTACK_BLOCKS, y.ng), 256, 0, c.s>>>(y, block_offsets(y), dws, d_w);
    CKL();
  }
  return SO2_OK;
}

so2_status so2conv_forward_noalloc(const so2conv_desc *desc, int64_t N, int64_t E,
                                   const void *x, const int64_t *edge_index,
                                   const float *edge_vec, so2conv_params prm, float *out,
                                   so2_stream_t stream) {
  if (!desc_ok(desc)) return desc ? SO2_ERR_UNSUPPORTED : SO2_ERR_INVALID_ARG;
  if (N < 0 || E < 0) return SO2_ERR_INVALID_ARG;
  const size_t need = make_plan(desc, N, E, SO2_WS_FORWARD).total;
  if (need > SO2_NOALLOC_WORKSPACE_BYTES) return SO2_ERR_WORKSPACE;
  void *base = noalloc_base();
  if (!base) return SO2_ERR_CUDA;
  return so2conv_forward(desc, N, E, x, edge_index, edge_vec, prm, out, base,
                         SO2_NOALLOC_WORKSPACE_BYTES, stream);
}

so2_status so2conv_noalloc_check(so2_stream_t stream) {
  void *base = noalloc_base();
  if (!base) return SO2_ERR_CUDA;
  return so2conv_check(base, stream);
}

size_t so2conv_block_workspace_size(const so2conv_desc *desc, int64_t n_nodes, int64_t n_edges,
                                    int which) {
  if (!desc_ok(desc) || desc->c_in != desc->c_out || n_nodes < 0 || n_edges < 0) return 0;
  if (which != 0 && which != 1) return 0;
  return make_block_plan(desc, n_nodes, n_edges, which).total;
}

so2_status so2conv_block_forward(const so2conv_desc *desc, int64_t N, int64_t E, const void *x,
                                 const int64_t *edge_index, const float *edge_vec,
                                 so2conv_params p1, so2conv_params p2, float *out, void *ws,
                                 size_t ws_bytes, so2_stream_t stream) {
  Ctx c1, c2;
  so2_status r = block_setup(desc, N, E, x, edge_index, edge_vec, p1, p2, ws, ws_bytes, 0,
                             stream, c1, c2);
  if (r != SO2_OK) return r;
  if (N > 0 && !out) return SO2_ERR_INVALID_ARG;
  const Plan &P = c1.P;
  const Layout &y = P.y;
  if (N > 0) CK(cudaMemsetAsync(out, 0, sizeof(float) * N * y.S * y.co, c1.s));
  if (E == 0) return SO2_OK;
  if ((r = build_maps(c1, false)) != SO2_OK) return r;
  if ((r = build_maps(c2, false)) != SO2_OK) return r;
  if ((r = sort_edges(c1, edge_index, 1)) != SO2_OK) return r;
  if ((r = pack_weights(c1, p1.w, false)) != SO2_OK) return r;
  if ((r = pack_weights(c2, p2.w, false)) != SO2_OK) return r;
  for (int64_t e0 = 0; e0 < E; e0 += P.chunk) {
    const int M = static_cast<int>((E - e0) < P.chunk ? (E - e0) : P.chunk);
    if ((r = chunk_prep(c1, e0, M, edge_index, edge_vec, 1, p1)) != SO2_OK) return r;
    if ((r = gate_only(c2, M, p2)) != SO2_OK) return r;
    if ((r = rotate_x(c1, M, x, P.xbf16)) != SO2_OK) return r;
    if ((r = gemm_v(c1, M)) != SO2_OK) return r;  // V1
    if ((r = block_act(c1, c2, M)) != SO2_OK) return r;
    if (fusable(y.co, P.split)) {
      const GemmScatter sc = make_scatter(c2, at<float>(ws, c2.P.gate), out, y.co);
      if ((r = gemm_v(c2, M, &sc, false)) != SO2_OK) return r;
    } else {
      if ((r = gemm_v(c2, M)) != SO2_OK) return r;
      if ((r = reduce_nodes(c2, e0, M, prows(c2, c2.P.V, 0), y.KG, at<float>(ws, c2.P.gate), 1,
                            out)) != SO2_OK)
        return r;
    }
  }
  return SO2_OK;
}

so2_status so2conv_block_backward(const so2conv_desc *desc, int64_t N, int64_t E, const void *x,
                                  const int64_t *edge_index, const float *edge_vec,
                                  so2conv_params p1, so2conv_params p2, const float *grad_out,
                                  float *grad_x, float *grad_w1, float *grad_w_rad1,
                                  float *grad_b_rad1, float *grad_w2, float *grad_w_rad2,
                                  float *grad_b_rad2, float *grad_edge_vec, void *ws,
                                  size_t ws_bytes, so2_stream_t stream) {
  Ctx c1, c2;
  so2_status r = block_setup(desc, N, E, x, edge_index, edge_vec, p1, p2, ws, ws_bytes, 1,
                             stream, c1, c2);
  if (r != SO2_OK) return r;
  if ((N > 0 && !grad_out) || !aligned16(grad_out)) return SO2_ERR_INVALID_ARG;
  const Plan &P = c1.P;
  const Layout &y = P.y;
  cudaStream_t s = c1.s;
  const int64_t nw = num_weights(y);
  if (grad_x && N > 0) CK(cudaMemsetAsync(grad_x, 0, sizeof(float) * N * y.S * y.ci, s));
  for (float *g : {grad_w1, grad_w2})
    if (g) CK(cudaMemsetAsync(g, 0, sizeof(float) * nw, s));
  for (float *g : {grad_w_rad1, grad_w_rad2})
    if (g) CK(cudaMemsetAsync(g, 0, sizeof(float) * y.nr * y.co, s));
  for (float *g : {grad_b_rad1, grad_b_rad2})
    if (g) CK(cudaMemsetAsync(g, 0, sizeof(float) * y.co, s));
  if (E == 0) return SO2_OK;
  if ((r = build_maps(c1, true)) != SO2_OK) return r;
  if ((r = build_maps(c2, true)) != SO2_OK) return r;
  if ((r = sort_edges(c1, edge_index, 0)) != SO2_OK) return r;
  if ((r = pack_weights(c1, p1.w, true)) != SO2_OK) return r;
  if ((r = pack_weights(c2, p2.w, true)) != SO2_OK) return r;
  if (grad_w1) CK(cudaMemsetAsync(at<float>(ws, c1.P.dws), 0, 4ull * y.WR * y.WK, s));
  if (grad_w2) CK(cudaMemsetAsync(at<float>(ws, c2.P.dws), 0, 4ull * y.WR * y.WK, s));
  const bool need_ga1 = grad_x || grad_edge_vec;
  const bool fuse_gx = grad_x && fusable(y.ci, P.split);
  for (int64_t e0 = 0; e0 < E; e0 += P.chunk) {
    const int M = static_cast<int>((E - e0) < P.chunk ? (E - e0) : P.chunk);
    if ((r = chunk_prep(c1, e0, M, edge_index, edge_vec, 0, p1)) != SO2_OK) return r;
    if ((r = gate_only(c2, M, p2)) != SO2_OK) return r;
    if ((r = rotate_x(c1, M, x, P.xbf16)) != SO2_OK) return r;
    if ((r = gemm_v(c1, M)) != SO2_OK) return r;  // V1
    if ((r = block_act(c1, c2, M)) != SO2_OK) return r;
    if ((r = gemm_v(c2, M)) != SO2_OK) return r;  // V2
    // conv 2's output side: Gg2, the edge record (frame terms of the output
    // rotation and the gate-2 part), gv2 = g2 * (D G[dst]) planes
    if ((r = edge_terms(c2, M, 1, x, grad_out, true, p2.w_rad)) != SO2_OK) return r;
    if ((r = gemm_ga(c2, M)) != SO2_OK) return r;  // dL/dh' = M2^T gv2
    if (grad_w2) {
      if ((r = zero_tail(c2, M, false, 0)) != SO2_OK) return r;
      if ((r = zero_tail(c2, M, true, 0)) != SO2_OK) return r;
      if ((r = gemm_dw(c2, M, 0, 0)) != SO2_OK) return r;  // gv2 (x) h'
    }
    if ((r = block_act_bwd(c1, c2, M, p1.w_rad)) != SO2_OK) return r;  // gv1, Gg1, dd1
    if (need_ga1) {
      const GemmScatter sc = make_scatter(c1, nullptr, grad_x, y.ci);
      if ((r = gemm_ga(c1, M, fuse_gx ? &sc : nullptr, grad_edge_vec != nullptr || !fuse_gx)) !=
          SO2_OK)
        return r;
    }
    if (grad_w1) {
      if ((r = zero_tail(c1, M, false, 0)) != SO2_OK) return r;
      if ((r = zero_tail(c1, M, true, 0)) != SO2_OK) return r;
      if ((r = gemm_dw(c1, M, 0, 0)) != SO2_OK) return r;  // gv1 (x) a
    }
    if (grad_x && !fuse_gx &&
        (r = reduce_nodes(c1, e0, M, prows(c1, P.Ga, 0), y.KA, nullptr, 0, grad_x)) != SO2_OK)
      return r;
    if (grad_edge_vec &&
        (r = edge_terms(c1, M, 2, x, grad_out, false, p1.w_rad, grad_edge_vec)) != SO2_OK)
      return r;
    if ((grad_w_rad2 || grad_b_rad2) &&
        (r = rad_grads(c2, M, at<float>(ws, c2.P.Gg), nullptr, nullptr, grad_w_rad2,
                       grad_b_rad2)) != SO2_OK)
      return r;
    if ((grad_w_rad1 || grad_b_rad1) &&
        (r = rad_grads(c1, M, at<float>(ws, c1.P.Gg), nullptr, nullptr, grad_w_rad1,
                       grad_b_rad1)) != SO2_OK)
      return r;
  }
  ProfScope ps(7, s);
  if (grad_w1) {
    k_unstack_grad<<<dim3(UNSTACK_BLOCKS, y.ng), 256, 0, s>>>(
        y, block_offsets(y), at<float>(ws, c1.P.dws), grad_w1);
    CKL();
  }
  if (grad_w2) {
    k_unstack_grad<<<dim3(UNSTACK_BLOCKS, y.ng), 256, 0, s>>>(
        y, block_offsets(y), at<float>(ws, c2.P.dws), grad_w2);
    CKL();
  }
  return SO2_OK;
}

so2_status so2conv_check(void *ws, so2_stream_t stream) {
  if (!ws) return SO2_ERR_WORKSPACE;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(s) != cudaSuccess) return SO2_ERR_CUDA;
  DevStatus h{};
  // the status word is the first thing in every workspace plan
  if (cudaMemcpy(&h, ws, sizeof(h), cudaMemcpyDeviceToHost) != cudaSuccess) return SO2_ERR_CUDA;
  if (h.code != 0) {
    DevStatus z{};
    if (cudaMemcpy(ws, &z, sizeof(z), cudaMemcpyHostToDevice) != cudaSuccess) return SO2_ERR_CUDA;
  }
  return static_cast<so2_status>(h.code);
}

long long so2conv_launch_count(void) { return g_launches; }

so2_status so2conv_wait_selftest(void *ws, size_t ws_bytes, int64_t limit_us,
                                 so2_stream_t stream) {
  if (!ws || ws_bytes < sizeof(DevStatus) || (reinterpret_cast<uintptr_t>(ws) & 255))
    return SO2_ERR_WORKSPACE;
  if (limit_us < 1 || limit_us > 10000000) return SO2_ERR_INVALID_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(ws, 0, sizeof(DevStatus), s) != cudaSuccess) return SO2_ERR_CUDA;
  k_wait_selftest<<<1, 32, 0, s>>>(static_cast<DevStatus *>(ws),
                                    static_cast<uint64_t>(limit_us) * 1000ull);
  ++g_launches;
  return cudaPeekAtLastError() == cudaSuccess ? SO2_OK : SO2_ERR_CUDA;
}

so2_status so2conv_set_max_chunk_edges(int64_t n) {
  if (n < 0 || n > (1 << 22)) return SO2_ERR_INVALID_ARG;
  g_chunk_max = n == 0 ? SO2_CHUNK_MAX : round_up(static_cast<int>(n) < 256 ? 256 : static_cast<int>(n), 256);
  return SO2_OK;
}

int64_t so2conv_max_chunk_edges(void) { return g_chunk_max; }

void so2conv_profile_enable(int on) {
  g_prof.on = on < 0 ? 0 : (on > 2 ? 2 : on);
  if (g_prof.on)
    for (int k = 0; k < PROF_KINDS; ++k) g_prof.used[k] = 0;
}

so2_status so2conv_profile_read(int kind, int *n_launches, double *total_ms) {
  if (kind < 0 || kind >= PROF_KINDS || !n_launches || !total_ms) return SO2_ERR_INVALID_ARG;
  double ms = 0.0;
  const int n = g_prof.used[kind] / 2;
  for (int i = 0; i < n; ++i) {
    float t = 0.f;
    if (cudaEventSynchronize(g_prof.ev[kind][2 * i + 1]) != cudaSuccess) return SO2_ERR_CUDA;
    if (cudaEventElapsedTime(&t, g_prof.ev[kind][2 * i], g_prof.ev[kind][2 * i + 1]) != cudaSuccess)
      return SO2_ERR_CUDA;
    ms += t;
  }
  *n_launches = n;
  *total_ms = ms;
  return SO2_OK;
}

const char *so2conv_status_string(so2_status s) {
  switch (s) {
    case SO2_OK: return "ok";
    case SO2_ERR_INVALID_ARG: return "invalid argument";
    case SO2_ERR_UNSUPPORTED: return "unsupported shape or option";
    case SO2_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
    case SO2_ERR_CUDA: return "CUDA runtime error";
    case SO2_ERR_INDEX: return "edge index outside [0, n_nodes)";
    case SO2_ERR_TIMEOUT: return "a bounded device wait gave up";
    case SO2_ERR_DEGENERATE: return "zero-length edge vector";
  }
  return "unknown status";
}

so2_status so2conv_edge_frames(int32_t lmax, int64_t E, const float *edge_vec, float *R_out,
                               float *D_out, so2_stream_t stream) {
  if (lmax < 0 || lmax > LMAX_SUPPORTED || E < 0) return SO2_ERR_UNSUPPORTED;
  if (E == 0) return SO2_OK;
  if (!edge_vec) return SO2_ERR_INVALID_ARG;
  const int smem = dsize(lmax) * 33 * static_cast<int>(sizeof(float));
  const int64_t nb = (E + 31) / 32;
  const int grid = static_cast<int>(nb < 148 * 64 ? nb : 148 * 64);
  bool ok = true;
  SO2_DISPATCH_L(lmax, ok = allow_smem(k_frames<L>, smem);
                 if (ok) k_frames<L><<<grid, 32, smem, reinterpret_cast<cudaStream_t>(stream)>>>(
                     E, edge_vec, R_out, D_out));
  if (!ok) return SO2_ERR_CUDA;
  return cudaPeekAtLastError() == cudaSuccess ? SO2_OK : SO2_ERR_CUDA;
}

}  // extern "C"
