// wigner.cuh -- per-edge frame, real Wigner-D and rotation generators.
//
// Frame: R = R_y(-theta) R_z(-phi) for the edge direction (polar angle
// theta, azimuth phi), so R r_hat = z_hat.  Any roll about z would do: the
// convolution's output does not depend on it.
//
// Wigner-D: D^1 = P R P^T (P maps (x, y, z) to the l = 1 order (y, z, x)),
// then D^l for l >= 2 by the Ivanic-Ruedenberg recursion (J. Phys. Chem.
// 1996, 100, 6342; corrections 1998, 102, 9099), which builds each D^l from
// D^1 and D^{l-1}.  One thread computes one edge's blocks, with every
// coefficient of the recursion a compile-time constant.  This is the rotation of real spherical harmonics without
// the Condon-Shortley phase, with Y(R n) = D(R) Y(n).
//
// Generators: J_x, J_y are d/dtheta D(R_{x,y}(theta)) at theta = 0 in the
// same real basis; they couple |m| to |m| +- 1 with weights
// s_k = sqrt((l-k)(l+k+1)) / 2 (sqrt(2) s_0 where m = 0 is involved).  With
// them, a small turn (I + [w]x) R of the frame changes D by
// (w_x J_x + w_y J_y + w_z J_z) D.
#pragma once

#include <utility>

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
// sum of at most IR_TERMS products coef * D^1[a] * D^{l-1}[b], with D^1
// row-major 3x3 (index (i+1)*3+(j+1) for orders i, j in -1..1) and D^{l-1}
// row-major (2l-1)^2.  ir_terms lists them; it is constexpr, so the kernels
// below get every coefficient and index as an immediate.
constexpr int IR_TERMS = 10;

struct IRTerm {
  float c;
  int a, b;
};
struct IREntry {
  IRTerm t[IR_TERMS];
  int n;
};

// Square root by Newton's method in double (compile-time coefficients).
__host__ __device__ constexpr double cx_sqrt(double v) {
  if (v <= 0.0) return 0.0;
  double x = v > 1.0 ? v : 1.0;
  for (int i = 0; i < 200; ++i) {
    const double nx = 0.5 * (x + v / x);
    if (nx == x) break;
    x = nx;
  }
  return x;
}

struct IRBuilder {
  IREntry e{};
  int l;
  __host__ __device__ constexpr void put(double c, int i, int j, int a, int b) {
    const int wp = 2 * l - 1;
    e.t[e.n].c = static_cast<float>(c);
    e.t[e.n].a = (i + 1) * 3 + (j + 1);
    e.t[e.n].b = (a + l - 1) * wp + (b + l - 1);
    ++e.n;
  }
  // c * P(i, a, b): the D^1 x D^{l-1} product of the recursion, with the
  // column of D^{l-1} folded back at the edges b = +-l.
  __host__ __device__ constexpr void P(double c, int i, int a, int b) {
    if (b == -l) {
      put(c, i, 1, a, -l + 1);
      put(c, i, -1, a, l - 1);
    } else if (b == l) {
      put(c, i, 1, a, l - 1);
      put(-c, i, -1, a, -l + 1);
    } else {
      put(c, i, 0, a, b);
    }
  }
};

__host__ __device__ constexpr IREntry ir_terms(int l, int m, int n) {
  IRBuilder B{};
  B.l = l;
  const int am = m < 0 ? -m : m;
  const int an = n < 0 ? -n : n;
  const int dm0 = (m == 0);
  const double den = (an == l) ? static_cast<double>((2 * l) * (2 * l - 1))
                               : static_cast<double>((l + n) * (l - n));
  const double u = cx_sqrt(static_cast<double>((l + m) * (l - m)) / den);
  const double v = 0.5 * cx_sqrt(static_cast<double>((1 + dm0) * (l + am - 1) * (l + am)) / den) *
                   static_cast<double>(1 - 2 * dm0);
  const double w = -0.5 * cx_sqrt(static_cast<double>((l - am - 1) * (l - am)) / den) *
                   static_cast<double>(1 - dm0);
  const double r2 = cx_sqrt(2.0);
  if (u != 0.0) B.P(u, 0, m, n);
  if (v != 0.0) {
    if (m == 0) {
      B.P(v, 1, 1, n);
      B.P(v, -1, -1, n);
    } else if (m > 0) {
      B.P(v * (m == 1 ? r2 : 1.0), 1, m - 1, n);
      if (m != 1) B.P(-v, -1, -m + 1, n);
    } else {
      if (m != -1) B.P(v, 1, m + 1, n);
      B.P(v * (m == -1 ? r2 : 1.0), -1, -m - 1, n);
    }
  }
  if (w != 0.0) {
    if (m > 0) {
      B.P(w, 1, m + 1, n);
      B.P(w, -1, -m - 1, n);
    } else {
      B.P(w, 1, m - 1, n);
      B.P(-w, -1, -m + 1, n);
    }
  }
  return B.e;
}

// Entry E (row-major) of D^l from D^1 (registers) and D^{l-1} (Dp[k * s]).
template <int l, int E, int... T>
__device__ __forceinline__ float ir_value(const float (&D1)[9], const float *Dp, int s,
                                          std::integer_sequence<int, T...>) {
  constexpr int w = 2 * l + 1;
  constexpr IREntry en = ir_terms(l, E / w - l, E % w - l);
  float v = 0.f;
  ((T < en.n ? (v += en.t[T].c * D1[en.t[T].a] * Dp[en.t[T].b * s]) : 0.f), ...);
  return v;
}

template <int l, int... E>
__device__ __forceinline__ void ir_level(const float (&D1)[9], const float *Dp, float *Dl, int s,
                                         std::integer_sequence<int, E...>) {
  ((Dl[E * s] = ir_value<l, E>(D1, Dp, s, std::make_integer_sequence<int, IR_TERMS>{})), ...);
}

template <int l, int L>
__device__ __forceinline__ void ir_levels(const float (&D1)[9], float *D, int s) {
  if constexpr (l <= L) {
    ir_level<l>(D1, D + dblock_off(l - 1) * s, D + dblock_off(l) * s, s,
                std::make_integer_sequence<int, (2 * l + 1) * (2 * l + 1)>{});
    ir_levels<l + 1, L>(D1, D, s);
  }
}

// Full blocks D^0..D^L of the rotation R (row-major 3x3), each (2l+1)^2
// row-major, concatenated, computed by one thread into D[k * s]
// (k < dsize(L)); s is the stride between a thread's consecutive entries.
template <int L>
__device__ __forceinline__ void wigner_blocks_thread(const float (&R)[9], float *D, int s) {
  D[0] = 1.f;
  if constexpr (L >= 1) {
    // (y, z, x) ordering of the l = 1 functions: index 0 <- y, 1 <- z, 2 <- x
    constexpr int pm[3] = {1, 2, 0};
    float D1[9];
#pragma unroll
    for (int k = 0; k < 9; ++k) {
      D1[k] = R[pm[k / 3] * 3 + pm[k % 3]];
      D[(dblock_off(1) + k) * s] = D1[k];
    }
    ir_levels<2, L>(D1, D, s);
  }
}

// Calls f with the compile-time lmax L (0..LMAX_SUPPORTED).
#define SO2_DISPATCH_L(lmax, ...)              \
  switch (lmax) {                              \
    case 0: { constexpr int L = 0; __VA_ARGS__; } break; \
    case 1: { constexpr int L = 1; __VA_ARGS__; } break; \
    case 2: { constexpr int L = 2; __VA_ARGS__; } break; \
    case 3: { constexpr int L = 3; __VA_ARGS__; } break; \
    case 4: { constexpr int L = 4; __VA_ARGS__; } break; \
    case 5: { constexpr int L = 5; __VA_ARGS__; } break; \
    default: { constexpr int L = 6; __VA_ARGS__; } break; \
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
