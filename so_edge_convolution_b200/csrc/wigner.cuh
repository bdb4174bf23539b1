// wigner.cuh -- per-edge frame, real Wigner-D and rotation generators.
//
// Frame: R = R_y(-theta) R_z(-phi) for the edge direction (polar angle
// theta, azimuth phi), so R r_hat = z_hat.  Any roll about z would do: the
// convolution's output does not depend on it.
//
// Wigner-D: D^1 = P R P^T (P maps (x, y, z) to the l = 1 order (y, z, x)),
// then D^l for l >= 2 by the Ivanic-Ruedenberg recursion (J. Phys. Chem.
// 1996, 100, 6342; corrections 1998, 102, 9099), which builds each D^l from
// D^1 and D^{l-1}.  This is the rotation of real spherical harmonics without
// the Condon-Shortley phase, with Y(R n) = D(R) Y(n).
//
// Generators: J_x, J_y are d/dtheta D(R_{x,y}(theta)) at theta = 0 in the
// same real basis; they couple |m| to |m| +- 1 with weights
// s_k = sqrt((l-k)(l+k+1)) / 2 (sqrt(2) s_0 where m = 0 is involved).  With
// them, a small turn (I + [w]x) R of the frame changes D by
// (w_x J_x + w_y J_y + w_z J_z) D.
#pragma once

#include "common.cuh"

namespace so2 {

constexpr int LMAX_SUPPORTED = 6;

__host__ __device__ constexpr int dblock_off(int l) { return l * (4 * l * l - 1) / 3; }
__host__ __device__ constexpr int dsize(int lmax) { return dblock_off(lmax + 1); }

struct Frame {
  float d;
  float rh[3];
  float R[9];  // row-major
};

// Returns false for a zero-length vector (the frame is then the identity).
__device__ __forceinline__ bool make_frame(float rx, float ry, float rz, Frame &f) {
  const float d = sqrtf(rx * rx + ry * ry + rz * rz);
  f.d = d;
  if (!(d > 0.f)) {
    f.rh[0] = 0.f;
    f.rh[1] = 0.f;
    f.rh[2] = 1.f;
    for (int i = 0; i < 9; ++i) f.R[i] = (i % 4 == 0) ? 1.f : 0.f;
    return false;
  }
  const float inv = 1.f / d;
  const float x = rx * inv, y = ry * inv, z = rz * inv;
  f.rh[0] = x;
  f.rh[1] = y;
  f.rh[2] = z;
  const float rho = sqrtf(x * x + y * y);
  float cp = 1.f, sp = 0.f;
  if (rho > 0.f) {
    cp = x / rho;
    sp = y / rho;
  }
  const float ct = z, st = rho;
  f.R[0] = ct * cp;
  f.R[1] = ct * sp;
  f.R[2] = -st;
  f.R[3] = -sp;
  f.R[4] = cp;
  f.R[5] = 0.f;
  f.R[6] = st * cp;
  f.R[7] = st * sp;
  f.R[8] = ct;
  return true;
}

// The Ivanic-Ruedenberg recursion writes entry (m, n) of D^l (l >= 2) as a
// sum of at most IR_TERMS products coef * D^1[i] * D^{l-1}[j], with D^1
// row-major 3x3 (index (a+1)*3+(b+1)) and D^{l-1} row-major (2l-1)^2.
// ir_terms lists them (unused slots have coef 0 and indices 0).
constexpr int IR_TERMS = 10;

__host__ __device__ inline int ir_terms(int l, int m, int n, float *coef, int *i1, int *i2) {
  const int wp = 2 * l - 1;
  int nt = 0;
  auto put = [&](float c, int i, int j, int a, int b) {
    coef[nt] = c;
    i1[nt] = (i + 1) * 3 + (j + 1);
    i2[nt] = (a + l - 1) * wp + (b + l - 1);
    ++nt;
  };
  // c * P(i, a, b)
  auto P = [&](float c, int i, int a, int b) {
    if (b == -l) {
      put(c, i, 1, a, -l + 1);
      put(c, i, -1, a, l - 1);
    } else if (b == l) {
      put(c, i, 1, a, l - 1);
      put(-c, i, -1, a, -l + 1);
    } else {
      put(c, i, 0, a, b);
    }
  };
  const int am = m < 0 ? -m : m;
  const int an = n < 0 ? -n : n;
  const int dm0 = (m == 0);
  const float den = (an == l) ? static_cast<float>((2 * l) * (2 * l - 1))
                              : static_cast<float>((l + n) * (l - n));
  const float u = sqrtf(static_cast<float>((l + m) * (l - m)) / den);
  const float v = 0.5f * sqrtf(static_cast<float>((1 + dm0) * (l + am - 1) * (l + am)) / den) *
                  static_cast<float>(1 - 2 * dm0);
  const float wc = -0.5f * sqrtf(static_cast<float>((l - am - 1) * (l - am)) / den) *
                   static_cast<float>(1 - dm0);
  const float r2 = 1.41421356237f;
  if (u != 0.f) P(u, 0, m, n);
  if (v != 0.f) {
    if (m == 0) {
      P(v, 1, 1, n);
      P(v, -1, -1, n);
    } else if (m > 0) {
      P(v * (m == 1 ? r2 : 1.f), 1, m - 1, n);
      if (m != 1) P(-v, -1, -m + 1, n);
    } else {
      if (m != -1) P(v, 1, m + 1, n);
      P(v * (m == -1 ? r2 : 1.f), -1, -m - 1, n);
    }
  }
  if (wc != 0.f) {
    if (m > 0) {
      P(wc, 1, m + 1, n);
      P(wc, -1, -m - 1, n);
    } else {
      P(wc, 1, m - 1, n);
      P(-wc, -1, -m + 1, n);
    }
  }
  for (int t = nt; t < IR_TERMS; ++t) {
    coef[t] = 0.f;
    i1[t] = 0;
    i2[t] = 0;
  }
  return nt;
}

// Entry (m, n) of D^l (l >= 2) evaluated directly from the term list.
__device__ __forceinline__ float ir_entry(int l, int m, int n, const float *D1, const float *Dp) {
  float c[IR_TERMS];
  int a[IR_TERMS], b[IR_TERMS];
  const int nt = ir_terms(l, m, n, c, a, b);
  float val = 0.f;
  for (int t = 0; t < nt; ++t) val += c[t] * D1[a[t]] * Dp[b[t]];
  return val;
}

// Number of tabulated entries for levels 2..lmax (entry index of (l, m, n)
// is dblock_off(l) - dblock_off(2) + (m+l)(2l+1) + (n+l)).
__host__ __device__ constexpr int ir_table_entries(int lmax) {
  return lmax < 2 ? 0 : dblock_off(lmax + 1) - dblock_off(2);
}

// Table layout (structure of arrays, NE = ir_table_entries(lmax)):
// coef[t * NE + e] floats, then idx[t * NE + e] ints with i1 | i2 << 8.
__global__ void k_ir_table(int lmax, float *table) {
  const int NE = ir_table_entries(lmax);
  const int e = blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= NE) return;
  int l = 2;
  while (l < lmax && e >= dblock_off(l + 1) - dblock_off(2)) ++l;
  const int local = e - (dblock_off(l) - dblock_off(2));
  const int w = 2 * l + 1;
  float c[IR_TERMS];
  int a[IR_TERMS], b[IR_TERMS];
  ir_terms(l, local / w - l, local % w - l, c, a, b);
  int *idx = reinterpret_cast<int *>(table + IR_TERMS * NE);
  for (int t = 0; t < IR_TERMS; ++t) {
    table[t * NE + e] = c[t];
    idx[t * NE + e] = a[t] | (b[t] << 8);
  }
}

// Full blocks D^0..D^lmax (each (2l+1)^2 row-major, concatenated) of the
// rotation R, computed by one warp into D (shared memory): the lanes share
// the entries of each level, levels one after another.  With a term table
// (k_ir_table) every entry is the same branch-free 10-term sum; without one
// the terms are enumerated per entry.
__device__ inline void wigner_blocks_warp(const float *R, int lmax, float *D,
                                          const float *table = nullptr) {
  const int lane = threadIdx.x & 31;
  if (lane == 0) D[0] = 1.f;
  if (lmax >= 1 && lane < 9) {
    // (y, z, x) ordering: sh index 0 <- y(1), 1 <- z(2), 2 <- x(0)
    const int pm[3] = {1, 2, 0};
    const int a = lane / 3, b = lane % 3;
    D[dblock_off(1) + lane] = R[pm[a] * 3 + pm[b]];
  }
  __syncwarp();
  const float *D1 = D + dblock_off(1);
  for (int l = 2; l <= lmax; ++l) {
    const float *Dp = D + dblock_off(l - 1);
    float *Dl = D + dblock_off(l);
    const int w = 2 * l + 1;
    if (table) {
      const int NE = ir_table_entries(lmax);
      const int *tidx = reinterpret_cast<const int *>(table + IR_TERMS * NE);
      const int base = dblock_off(l) - dblock_off(2);
      for (int idx = lane; idx < w * w; idx += 32) {
        float val = 0.f;
#pragma unroll
        for (int t = 0; t < IR_TERMS; ++t) {
          const int pk = __ldg(tidx + t * NE + base + idx);
          val += __ldg(table + t * NE + base + idx) * D1[pk & 0xff] * Dp[pk >> 8];
        }
        Dl[idx] = val;
      }
    } else {
      for (int idx = lane; idx < w * w; idx += 32)
        Dl[idx] = ir_entry(l, idx / w - l, idx % w - l, D1, Dp);
    }
    __syncwarp();
  }
}

__device__ __forceinline__ float gen_s(int l, int k) {
  return 0.5f * sqrtf(static_cast<float>((l - k) * (l + k + 1)));
}

// (J_x a)[m] and (J_y a)[m] for one l; `a(q)` returns the coefficient of
// order q (only |q| <= |m| + 1 is touched).
template <typename F>
__device__ __forceinline__ void gen_xy(int l, int m, F a, float &jx, float &jy) {
  const float r2 = 1.41421356237f;
  if (l == 0) {
    jx = 0.f;
    jy = 0.f;
    return;
  }
  if (m == 0) {
    const float s0 = r2 * gen_s(l, 0);
    jx = s0 * a(-1);
    jy = -s0 * a(1);
    return;
  }
  if (m > 0) {
    const int k = m;
    jx = (k < l ? gen_s(l, k) * a(-(k + 1)) : 0.f) + (k >= 2 ? gen_s(l, k - 1) * a(-(k - 1)) : 0.f);
    jy = (k == 1 ? r2 * gen_s(l, 0) * a(0) : gen_s(l, k - 1) * a(k - 1)) -
         (k < l ? gen_s(l, k) * a(k + 1) : 0.f);
    return;
  }
  const int k = -m;
  jx = (k == 1 ? -r2 * gen_s(l, 0) * a(0) : -gen_s(l, k - 1) * a(k - 1)) -
       (k < l ? gen_s(l, k) * a(k + 1) : 0.f);
  jy = (k >= 2 ? gen_s(l, k - 1) * a(-(k - 1)) : 0.f) - (k < l ? gen_s(l, k) * a(-(k + 1)) : 0.f);
}

}  // namespace so2
