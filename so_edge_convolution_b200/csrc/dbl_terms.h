// dbl_terms.h -- launchers of the double backward's per-edge terms.
//
// The kernels (radial terms, and the two sides of the second order in the
// edge vectors) are compiled in their own translation unit,
// so2conv_dbl_terms.cu, so that the library's units build in parallel.
// Product rows (V, dV, Vt, Ga, MP) are f32, or bf16 when pbf16; X is bf16
// when xbf16.  All launches go to stream s with `grid` blocks of 256 threads.
#pragma once

#include "layout.cuh"

namespace so2 {

struct EdgeRec;

// Radial terms of the double backward (k_edge_terms2): Aout, Bout [M][c_out].
cudaError_t launch_edge_terms2(const Layout &y, int grid, int M, const EdgeRec *rec,
                               const float *D, const float *G, const float *omega,
                               const void *V, const void *dV, const void *Vt, bool pbf16,
                               float *Aout, float *Bout, cudaStream_t s);

// Input side of d_edge_vec (k_edge_hess_in), source order.
cudaError_t launch_hess_in(const Layout &y, int grid, int M, const EdgeRec *rec, const float *D,
                           const float *geo, const void *X, bool xbf16, const float *GX,
                           const float *omega, const void *Ga, const void *MP, bool pbf16,
                           float *d_r, cudaStream_t s);

// Output side of d_edge_vec (k_edge_hess_out), destination order.
cudaError_t launch_hess_out(const Layout &y, float cutoff, int grid, int M, const EdgeRec *rec,
                            const float *D, const float *geo, const float *gate, const float *G,
                            const float *omega, const void *V, const void *dV, const void *Vt,
                            bool pbf16, const float *w_rad, float *d_r, cudaStream_t s);

}  // namespace so2
