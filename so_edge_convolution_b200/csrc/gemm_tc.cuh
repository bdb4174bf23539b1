// gemm_tc.cuh -- grouped tcgen05 GEMM for the per-m mixing.
//
// C[M x N] (+)= A[M x K] * B[N x K]^T, A and B bf16 and K-major, f32
// accumulation in tensor memory.  With `split`, A and B are each given as a
// (hi, lo) pair of bf16 planes whose sum carries 16 significant bits, and the
// product is hi*hi + hi*lo + lo*hi (the lo*lo term is below f32-level
// accuracy for the tolerances the f32 path is held to).  This is how the f32
// configurations reach ~1e-5 relative error on bf16 tensor cores.
//
// Several independent problems (one per m, for the dense per-m
// multiplications named in "TrimSO(2): Fast and Memory-Efficient Training of
// Equivariant Interatomic Potentials", Abstract) run in one launch: each
// group addresses its own rectangle of the same A and B tensors.
#pragma once

#include "common.cuh"

namespace so2 {

constexpr int GEMM_BM = 128;
constexpr int GEMM_BN = 128;
constexpr int GEMM_BK = 64;
constexpr int GEMM_MAX_GROUPS = 8;
constexpr int GEMM_THREADS = 192;  // warp 0 TMA, warp 1 MMA, warps 2..5 epilogue

struct GemmGroup {
  int M, N, K;           // K is a multiple of GEMM_BK
  int a_row, a_col;      // origin of this group's A rectangle (rows, K cols)
  int b_row, b_col;      // origin of this group's B rectangle
  int tiles_n, tile_begin;
  long long c_off;       // element offset of C[0][0] for this group
  int ldc;               // row stride of C in elements
};

struct GemmParams {
  int n_groups;
  int total_tiles;
  GemmGroup g[GEMM_MAX_GROUPS];
  float *C;
  int beta;   // 0: C = AB^T, 1: C += AB^T
  int split;  // 1: hi/lo planes (3 products), 0: hi only
  DevStatus *status;
};

template <int STAGES, bool SPLIT>
struct GemmSmem {
  static constexpr int A_BYTES = GEMM_BM * GEMM_BK * 2;
  static constexpr int B_BYTES = GEMM_BN * GEMM_BK * 2;
  static constexpr int PLANES = SPLIT ? 2 : 1;
  static constexpr int STAGE_BYTES = (A_BYTES + B_BYTES) * PLANES;
  static constexpr int TOTAL = STAGES * STAGE_BYTES + 1024 /*align*/ + 256 /*barriers*/;
};

template <int STAGES, bool SPLIT>
__global__ void __launch_bounds__(GEMM_THREADS, 1)
    k_gemm_tc(const __grid_constant__ CUtensorMap tA_hi, const __grid_constant__ CUtensorMap tA_lo,
              const __grid_constant__ CUtensorMap tB_hi, const __grid_constant__ CUtensorMap tB_lo,
              const __grid_constant__ GemmParams p) {
  using L = GemmSmem<STAGES, SPLIT>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t *full = reinterpret_cast<uint64_t *>(smem + STAGES * L::STAGE_BYTES);
  uint64_t *empty = full + STAGES;
  uint64_t *tmem_full = empty + STAGES;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(tmem_full + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // which group / tile
  int gi = 0;
  while (gi + 1 < p.n_groups && static_cast<int>(blockIdx.x) >= p.g[gi + 1].tile_begin) ++gi;
  const GemmGroup &G = p.g[gi];
  const int local = blockIdx.x - G.tile_begin;
  const int m0 = (local / G.tiles_n) * GEMM_BM;
  const int n0 = (local % G.tiles_n) * GEMM_BN;
  const int nk = G.K / GEMM_BK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(tmem_full, 1);
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, GEMM_BN);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0 && lane == 0) {
    // ---------------- TMA producer ----------------
    for (int kb = 0; kb < nk; ++kb) {
      const int s = kb % STAGES;
      const uint32_t ph = (kb / STAGES) & 1;
      if (!mbar_wait(&empty[s], ph ^ 1, p.status)) break;
      uint8_t *st = smem + s * L::STAGE_BYTES;
      mbar_arrive_expect_tx(&full[s], L::STAGE_BYTES);
      const int kc = kb * GEMM_BK;
      tma_load_2d(st, &tA_hi, &full[s], G.a_col + kc, G.a_row + m0);
      tma_load_2d(st + L::A_BYTES, &tB_hi, &full[s], G.b_col + kc, G.b_row + n0);
      if (SPLIT) {
        tma_load_2d(st + L::A_BYTES + L::B_BYTES, &tA_lo, &full[s], G.a_col + kc, G.a_row + m0);
        tma_load_2d(st + 2 * L::A_BYTES + L::B_BYTES, &tB_lo, &full[s], G.b_col + kc,
                    G.b_row + n0);
      }
    }
  } else if (warp == 1 && lane == 0) {
    // ---------------- MMA issuer ----------------
    constexpr uint32_t idesc = idesc_bf16_f32(GEMM_BM, GEMM_BN);
    bool ok = true;
    for (int kb = 0; kb < nk; ++kb) {
      const int s = kb % STAGES;
      const uint32_t ph = (kb / STAGES) & 1;
      if (!mbar_wait(&full[s], ph, p.status)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t base = smem_u32(smem + s * L::STAGE_BYTES);
      const uint64_t a_hi = sdesc_k_sw128(base);
      const uint64_t b_hi = sdesc_k_sw128(base + L::A_BYTES);
      const uint64_t a_lo = sdesc_k_sw128(base + L::A_BYTES + L::B_BYTES);
      const uint64_t b_lo = sdesc_k_sw128(base + 2 * L::A_BYTES + L::B_BYTES);
#pragma unroll
      for (int kk = 0; kk < GEMM_BK / 16; ++kk) {
        const uint64_t step = static_cast<uint64_t>(kk * 2);  // 32 bytes, in 16-byte units
        umma_bf16(tmem, a_hi + step, b_hi + step, idesc, (kb | kk) != 0);
        if (SPLIT) {
          umma_bf16(tmem, a_hi + step, b_lo + step, idesc, 1);
          umma_bf16(tmem, a_lo + step, b_hi + step, idesc, 1);
        }
      }
      umma_commit(&empty[s]);
    }
    if (ok) umma_commit(tmem_full);
  } else if (warp >= 2) {
    // ---------------- epilogue: TMEM -> registers -> C ----------------
    const int q = warp & 3;  // TMEM lane quadrant this warp may read
    const int row = m0 + q * 32 + lane;
    bool ready = (nk > 0) ? mbar_wait(tmem_full, 0, p.status) : true;
    tc_fence_after();
    if (ready) {
      float *Cg = p.C + G.c_off;
      for (int cc = 0; cc < GEMM_BN / 32; ++cc) {
        uint32_t r[32];
        if (nk > 0) {
          tmem_ld32(tmem + (static_cast<uint32_t>(q * 32) << 16) + cc * 32, r);
        } else {
#pragma unroll
          for (int j = 0; j < 32; ++j) r[j] = 0u;
        }
        const int col0 = n0 + cc * 32;
        if (row < G.M && col0 < G.N) {
          float *crow = Cg + static_cast<long long>(row) * G.ldc + col0;
          const bool full_vec = (col0 + 32 <= G.N) && ((reinterpret_cast<uintptr_t>(crow) & 15) == 0);
          if (full_vec) {
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
      }
    }
    tc_fence_before();
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, GEMM_BN);
  }
}

}  // namespace so2
