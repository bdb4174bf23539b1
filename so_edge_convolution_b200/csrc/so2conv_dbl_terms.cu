// so2conv_dbl_terms.cu -- the double backward's per-edge kernels and their
// launchers (see dbl_terms.h).  Same kernels and shapes as the rest of the
// library (edge_kernels.cuh); only the translation unit differs.
#include "dbl_terms.h"
#include "dispatch.cuh"
#include "edge_kernels.cuh"

namespace so2 {

cudaError_t launch_edge_terms2(const Layout &y, int grid, int M, const EdgeRec *rec,
                               const float *D, const float *G, const float *omega,
                               const void *V, const void *dV, const void *Vt, bool pbf16,
                               float *Aout, float *Bout, cudaStream_t s) {
  const int sm = 8 * y.dsz * 4;
#define SO2_ET2(TF)                                                                             \
  DISPATCH_LM(y.L, y.mmax,                                                                      \
              (k_edge_terms2<MM, ((LC >= 0 && LC <= 4) ? LC : -1), TF><<<grid, 256, sm, s>>>(   \
                  y, M, rec, D, G, omega, static_cast<const TF *>(V),                           \
                  static_cast<const TF *>(dV), static_cast<const TF *>(Vt), Aout, Bout)))
  if (pbf16) {
    SO2_ET2(__nv_bfloat16);
  } else {
    SO2_ET2(float);
  }
#undef SO2_ET2
  return cudaPeekAtLastError();
}

// The second-order kernels use their runtime-degree bodies only (compile
// time); the second order in r is not on the forward + backward path.
cudaError_t launch_hess_in(const Layout &y, int grid, int M, const EdgeRec *rec, const float *D,
                           const float *geo, const void *X, bool xbf16, const float *GX,
                           const float *omega, const void *Ga, const void *MP, bool pbf16,
                           float *d_r, cudaStream_t s) {
  const int sm = 8 * y.dsz * 4;
#define SO2_HIN(TX, TF)                                                                         \
  DISPATCH_MM(y.mmax, k_edge_hess_in<TX, MM, -1, TF><<<grid, 256, sm, s>>>(                     \
                          y, M, rec, D, geo, static_cast<const TX *>(X), GX, omega,             \
                          static_cast<const TF *>(Ga), static_cast<const TF *>(MP), d_r))
  if (xbf16) {
    SO2_HIN(__nv_bfloat16, __nv_bfloat16);
  } else {
    SO2_HIN(float, float);
  }
#undef SO2_HIN
  (void)pbf16;  // the bf16 path (xbf16) is the one whose product rows are bf16
  return cudaPeekAtLastError();
}

cudaError_t launch_hess_out(const Layout &y, float cutoff, int grid, int M, const EdgeRec *rec,
                            const float *D, const float *geo, const float *gate, const float *G,
                            const float *omega, const void *V, const void *dV, const void *Vt,
                            bool pbf16, const float *w_rad, float *d_r, cudaStream_t s) {
  const int sm = 8 * (y.dsz + 2 * RAD_MAX_NR) * 4;
#define SO2_HOUT(TF)                                                                            \
  DISPATCH_MM(y.mmax, k_edge_hess_out<MM, -1, TF><<<grid, 256, sm, s>>>(                        \
                          y, cutoff, M, rec, D, geo, gate, G, omega,                            \
                          static_cast<const TF *>(V), static_cast<const TF *>(dV),              \
                          static_cast<const TF *>(Vt), w_rad, d_r))
  if (pbf16) {
    SO2_HOUT(__nv_bfloat16);
  } else {
    SO2_HOUT(float);
  }
#undef SO2_HOUT
  return cudaPeekAtLastError();
}

}  // namespace so2
