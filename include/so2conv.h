/*
 * so2conv.h -- C ABI of libso2conv, a B200 (sm_100a) SO(2) edge convolution.
 *
 * The operation ("TrimSO(2): Fast and Memory-Efficient Training of
 * Equivariant Interatomic Potentials", Abstract: rotation on gather, dense
 * per-m matrix multiplication, recombination, inverse rotation on
 * reduction, with first and higher-order derivatives).  For every edge
 * e = (s -> d) with edge vector r_e:
 *
 *   R_e r_hat_e = z_hat                   an edge frame (its roll is free)
 *   a  = trunc(D(R_e) x[s])               real Wigner-D, rows |m| <= mmax kept
 *   v0 = W0 u0                            m = 0,  u0 = (a[l,0,:]) for l = 0..L
 *   v+ = W1_m u+ - W2_m u-                m >= 1, u+- = (a[l,+-m,:]) for l = m..L
 *   v- = W2_m u+ + W1_m u-
 *   y~ = g * v,  g = W_rad^T phi(|r_e|) + b_rad   (per output channel)
 *   out[d] += D(R_e)^T y~
 *
 * Conventions (readings; the pages print no formulas):
 *  - real spherical harmonics, orthonormal, no Condon-Shortley phase,
 *    flat index l*l + l + m (m = -l..l), so the l = 1 block is (y, z, x);
 *  - D(R) satisfies Y(R n) = D(R) Y(n);
 *  - phi_k(d) = exp(-(d - mu_k)^2 / (2 sigma^2)), mu_k = k * cutoff/(n_rbf-1),
 *    sigma = cutoff/(n_rbf-1), no envelope;
 *  - plain sum over incoming edges, no normalisation.
 *
 * Layouts (all row-major, C contiguous, caller-owned device memory):
 *  - x        [N, S, c_in]   S = (lmax+1)^2; f32 or bf16 (desc.dtype)
 *  - out      [N, S, c_out]  f32
 *  - edge_index int64 [2, E]: row 0 = source s, row 1 = destination d
 *  - edge_vec f32 [E, 3]:    r_e = pos[s] - pos[d] (+ periodic shift)
 *  - w        packed weight blocks, dtype as x: W0 [(L+1)c_out, (L+1)c_in],
 *             then for m = 1..mmax W1_m, W2_m [(L+1-m)c_out, (L+1-m)c_in];
 *             row index (l'-m)*c_out + c', column (l-m)*c_in + c
 *  - w_rad    f32 [n_rbf, c_out];  b_rad f32 [c_out]
 *  - every gradient is f32 and has the layout of the tensor it belongs to
 *    (grad_w: packed like w).
 *
 * Ownership: the caller owns every buffer and the stream.  The library
 * allocates nothing; it uses the workspace it is given (size from
 * so2conv_workspace_size).  All work is enqueued on `stream`, asynchronously;
 * no call synchronises except so2conv_check.  Outputs are overwritten, never
 * accumulated.  A NULL gradient pointer means "do not compute this one".
 *
 * Errors: argument problems are returned at once.  Problems only the device
 * can see (an index outside [0, N), a zero-length edge vector, a bounded
 * wait that ran out) are recorded in the workspace and reported by
 * so2conv_check; the device never traps.
 *
 * Supported: 0 <= mmax <= lmax <= 6, c_in and c_out multiples of 16 in
 * [16, 512], 2 <= n_rbf <= 64.  Anything else is SO2_ERR_UNSUPPORTED.
 *
 * Alignment: the node feature arrays read with vector loads (x, grad_out,
 * gg_x) must be 16-byte aligned, as cudaMalloc and PyTorch allocations are;
 * otherwise SO2_ERR_INVALID_ARG.  Other arrays need their element alignment.
 */
#ifndef SO2CONV_H
#define SO2CONV_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st *so2_stream_t; /* a cudaStream_t */

typedef enum {
  SO2_OK = 0,
  SO2_ERR_INVALID_ARG = 1,   /* NULL where a pointer is required, bad size */
  SO2_ERR_UNSUPPORTED = 2,   /* shape outside the supported range */
  SO2_ERR_WORKSPACE = 3,     /* workspace missing or smaller than required */
  SO2_ERR_CUDA = 4,          /* a CUDA runtime call failed */
  SO2_ERR_INDEX = 5,         /* device: edge_index entry outside [0, N) */
  SO2_ERR_TIMEOUT = 6,       /* device: a bounded wait gave up */
  SO2_ERR_DEGENERATE = 7     /* device: zero-length edge vector */
} so2_status;

typedef enum { SO2_F32 = 0, SO2_BF16 = 1 } so2_dtype;

typedef struct {
  int32_t lmax, mmax, c_in, c_out, n_rbf;
  float rbf_cutoff;
  int32_t dtype; /* so2_dtype of x and w; accumulation is always f32 */
} so2conv_desc;

typedef struct {
  const void *w;      /* packed mixing weights, dtype of desc */
  const float *w_rad; /* [n_rbf, c_out] */
  const float *b_rad; /* [c_out] */
} so2conv_params;

enum { SO2_WS_FORWARD = 0, SO2_WS_BACKWARD = 1, SO2_WS_DOUBLE_BACKWARD = 2 };

/* Bytes of workspace the given call needs (0 on unsupported shapes).  The
 * workspace must be 256-byte aligned device memory; contents need not be
 * initialised.  The same workspace may be reused by later calls on the same
 * stream. */
size_t so2conv_workspace_size(const so2conv_desc *desc, int64_t n_nodes,
                              int64_t n_edges, int which);

/* Number of packed weights (elements of w). */
int64_t so2conv_num_weights(const so2conv_desc *desc);

/* Forward: out = sum over edges of D^T (g * M_W(trunc(D x[src]))).
 * Defined by "TrimSO(2): Fast and Memory-Efficient Training of Equivariant
 * Interatomic Potentials", Abstract: rotation on gather, the dense per-m
 * mixing, recombination and inverse rotation on reduction, in that order.
 * Inputs as in the layout list above; `out` [N, S, c_out] f32 is
 * overwritten (nodes without incoming edges get 0).  Returns SO2_OK or an
 * argument / workspace status at once; device-detected problems go to
 * so2conv_check. */
so2_status so2conv_forward(const so2conv_desc *desc, int64_t n_nodes,
                           int64_t n_edges, const void *x,
                           const int64_t *edge_index, const float *edge_vec,
                           so2conv_params params, float *out, void *ws,
                           size_t ws_bytes, so2_stream_t stream);

/* Backward of <grad_out, out>: gradients w.r.t. x, w, w_rad, b_rad and the
 * edge vectors.  Any output pointer may be NULL (skipped).  Defined as the
 * exact first derivative of the forward map ("TrimSO(2): Fast and
 * Memory-Efficient Training of Equivariant Interatomic Potentials",
 * Abstract: the operator supports the differentiation that training needs).
 * grad_out [N, S, c_out] f32; grad_x [N, S, c_in], grad_w packed like w,
 * grad_w_rad [n_rbf, c_out], grad_b_rad [c_out], grad_edge_vec [E, 3], all f32
 * and overwritten.  Errors as for so2conv_forward. */
so2_status so2conv_backward(const so2conv_desc *desc, int64_t n_nodes,
                            int64_t n_edges, const void *x,
                            const int64_t *edge_index, const float *edge_vec,
                            so2conv_params params, const float *grad_out,
                            float *grad_x, float *grad_w, float *grad_w_rad,
                            float *grad_b_rad, float *grad_edge_vec, void *ws,
                            size_t ws_bytes, so2_stream_t stream);

/* Double backward: derivatives of
 *   Q = <gg_x, grad_x> + <gg_edge_vec, grad_edge_vec>
 * (grad_* from so2conv_backward with the same inputs) w.r.t. x, w, w_rad,
 * b_rad, grad_out and the edge vectors.  gg_x / gg_edge_vec may be NULL
 * (treated as zero).
 * Defined as the exact second derivative that force training takes
 * ("TrimSO(2): ...", Abstract: higher-order differentiation;
 * "Breaking the Training Barrier of Billion-Parameter Universal Machine
 * Learning Interatomic Potentials", Abstract: training needs second-order
 * derivatives).  gg_x [N, S, c_in], gg_edge_vec [E, 3]; outputs f32 with the
 * layouts of x, w, w_rad, b_rad, grad_out, edge_vec, overwritten; NULL skips
 * one.
 * d_edge_vec [E, 3] (may be NULL) is the derivative with respect to the
 * edge vectors: the Hessian of each edge's share of <grad_out, out> applied
 * to gg_edge_vec, plus the edge gradient of the first backward with x
 * replaced by gg_x.  Errors as for so2conv_forward. */
so2_status so2conv_double_backward(
    const so2conv_desc *desc, int64_t n_nodes, int64_t n_edges, const void *x,
    const int64_t *edge_index, const float *edge_vec, so2conv_params params,
    const float *grad_out, const float *gg_x, const float *gg_edge_vec,
    float *d_x, float *d_w, float *d_w_rad, float *d_b_rad, float *d_grad_out,
    float *d_edge_vec, void *ws, size_t ws_bytes, so2_stream_t stream);

/* Message block: two SO(2) convolutions with the activation between them,
 * in the edge frame ("TrimSO(2): Fast and Memory-Efficient Training of
 * Equivariant Interatomic Potentials", Abstract: rotation on gather,
 * recombination with activation, inverse rotation on reduction).  Per edge:
 *   a  = trunc(D x[s]);  h = g1 * M_W1(a);  h' = h * sigmoid(h[(0,0)])
 *   (per channel: SiLU on the (0,0) row, the other rows gated by the same
 *   sigmoid);  y~ = g2 * M_W2(h');  out[d] += D^T y~.
 * p1 and p2 are the two convolutions' packed weights and radial gates, laid
 * out as for so2conv_forward.  The block keeps one channel count: desc.c_in
 * must equal desc.c_out (SO2_ERR_UNSUPPORTED otherwise).  The workspace comes
 * from so2conv_block_workspace_size (which = 0 forward, 1 backward); other
 * rules (ownership, errors, alignment, so2conv_check) as for the single
 * convolution. */
size_t so2conv_block_workspace_size(const so2conv_desc *desc, int64_t n_nodes,
                                    int64_t n_edges, int which);
so2_status so2conv_block_forward(const so2conv_desc *desc, int64_t n_nodes,
                                 int64_t n_edges, const void *x,
                                 const int64_t *edge_index, const float *edge_vec,
                                 so2conv_params p1, so2conv_params p2, float *out,
                                 void *ws, size_t ws_bytes, so2_stream_t stream);
/* Backward of <grad_out, block output>: gradients w.r.t. x, both
 * convolutions' weights and radial gates, and the edge vectors (the exact
 * first derivative of the block).  Any output may be NULL (skipped); all are
 * f32 and overwritten. */
so2_status so2conv_block_backward(
    const so2conv_desc *desc, int64_t n_nodes, int64_t n_edges, const void *x,
    const int64_t *edge_index, const float *edge_vec, so2conv_params p1,
    so2conv_params p2, const float *grad_out, float *grad_x, float *grad_w1,
    float *grad_w_rad1, float *grad_b_rad1, float *grad_w2, float *grad_w_rad2,
    float *grad_b_rad2, float *grad_edge_vec, void *ws, size_t ws_bytes,
    so2_stream_t stream);

/* Synchronises `stream`, reads and clears the device error word kept in the
 * workspace, and returns it (SO2_OK if none).  Each forward / backward /
 * double backward call clears the word when it starts, so the result covers
 * the most recent call made with this workspace. */
so2_status so2conv_check(void *ws, so2_stream_t stream);

/* Static English text for a status code. */
const char *so2conv_status_string(so2_status status);

/* Edge frames and Wigner-D as the library computes them, for inspection:
 * R_out [E, 9] (row-major 3x3, R r_hat = z_hat) and D_out [E, Dsz] with the
 * blocks l = 0..lmax concatenated, each (2l+1)x(2l+1) row-major, Dsz =
 * sum_l (2l+1)^2.  Either output may be NULL. */
so2_status so2conv_edge_frames(int32_t lmax, int64_t n_edges,
                               const float *edge_vec, float *R_out,
                               float *D_out, so2_stream_t stream);

/* Size of the library-owned scratch array behind so2conv_forward_noalloc. */
#define SO2_NOALLOC_WORKSPACE_BYTES (96u << 20)

/* Forward that allocates nothing and needs no caller workspace.
 *
 * No counterpart on the pages: this exists for callers that cannot call
 * cudaMalloc (or any allocating routine) at the point where they run the
 * convolution -- for example code that executes inside another component's
 * stream capture, a plugin whose host application owns all device memory, or
 * a real-time loop that must not touch the allocator.  Such a caller still
 * passes its own inputs and `out`; the scratch memory comes from a fixed
 * device array of SO2_NOALLOC_WORKSPACE_BYTES inside this library, which
 * every GPU that loads the library holds until the process exits.
 *
 * Same arguments and results as so2conv_forward, without ws / ws_bytes.
 * Problems whose forward workspace (so2conv_workspace_size with
 * SO2_WS_FORWARD) exceeds the array are rejected with SO2_ERR_WORKSPACE
 * before anything is launched.  The workspace grows with both sizes: about
 * 4 E + 12 N bytes for the sort plus the per-chunk edge intermediates, so the
 * limit is near 3,800 edges at lmax 4, C 128, f32, and even the smallest
 * shapes stop near 20 M edges.
 *
 * Set-up: the array's device address belongs to the CUDA context that loaded
 * the library's module.  The first call in each context looks it up
 * (cudaGetSymbolAddress) and caches it under the driver's process-unique id
 * of that context, so a context created later, for example after
 * cudaDeviceReset, gets its own lookup.  Make that first call in each context
 * before any stream capture.
 *
 * All calls in a context share the one array, which keeps the last call's
 * contents (each call re-initialises what it reads), so calls that can
 * overlap on the GPU -- different streams, or different host threads -- race
 * and must be serialised by the caller.  Device-side input problems (bad
 * index, zero-length edge) are recorded at the head of the shared array:
 * read them with so2conv_noalloc_check. */
so2_status so2conv_forward_noalloc(const so2conv_desc *desc, int64_t n_nodes,
                                   int64_t n_edges, const void *x,
                                   const int64_t *edge_index,
                                   const float *edge_vec, so2conv_params params,
                                   float *out, so2_stream_t stream);

/* so2conv_check for the array behind so2conv_forward_noalloc in the current
 * context: synchronises `stream`, reads and clears the device status word of
 * the most recent no-alloc forward and returns it. */
so2_status so2conv_noalloc_check(so2_stream_t stream);

/* Self-test of failure detection without a fault: enqueues one kernel whose
 * thread waits, with the bounded wait every tensor-core kernel uses, on an
 * mbarrier phase that nothing completes.  The wait gives up after limit_us
 * microseconds (1 .. 10^7) and records SO2_ERR_TIMEOUT in the status word at
 * the head of ws (>= 256-byte aligned device memory of at least 8 bytes), so
 * so2conv_check(ws, stream) then returns SO2_ERR_TIMEOUT and the context stays
 * usable. */
so2_status so2conv_wait_selftest(void *ws, size_t ws_bytes, int64_t limit_us,
                                 so2_stream_t stream);

/* Number of kernels this library has launched in this process (all entry
 * points, all devices).  A plain counter, not thread safe. */
long long so2conv_launch_count(void);

/* Edges per chunk of per-edge intermediates (records, frames, Wigner-D,
 * operands and products live in the workspace for one chunk at a time; the
 * double backward uses half).  Larger chunks mean fewer, fuller launches and
 * a larger workspace.  n = 0 restores the default (65,536); otherwise n is
 * rounded up to a multiple of 256 (at least 256).  Returns
 * SO2_ERR_INVALID_ARG for n < 0 or n > 2^22.  Process-wide and not thread
 * safe: query so2conv_workspace_size after changing it, and do not change it
 * while a call is being issued. */
so2_status so2conv_set_max_chunk_edges(int64_t n);
int64_t so2conv_max_chunk_edges(void);

/* Live timing of the library's launches.  so2conv_profile_enable(1) clears
 * the record and starts recording a pair of CUDA events around every
 * tensor-core launch, on the stream it is launched on; (2) does the same and
 * also brackets each group of CUDA-core launches; (0) stops recording and
 * keeps the record for so2conv_profile_read.
 * so2conv_profile_read waits for the recorded events and returns, for one
 * kind, the number of recorded ranges and their summed duration in
 * milliseconds.  Kinds (SO2_PROFILE_KINDS of them): 0 products with the
 * stacked weights, 1 products with their transposes, 2 weight-gradient
 * products (0-2: the tcgen05 kernel, one range per launch), 3 rotation on
 * gather, 4 edge preparation (sort, records, frames, Wigner-D, gates),
 * 5 per-edge gradient terms, 6 radial-weight sums, 7 weight packing and
 * unpacking and the node-side scatter.  Process-wide state, not thread
 * safe. */
#define SO2_PROFILE_KINDS 8
void so2conv_profile_enable(int on);
so2_status so2conv_profile_read(int kind, int *n_launches, double *total_ms);

#ifdef __cplusplus
}
#endif

#endif /* SO2CONV_H */
