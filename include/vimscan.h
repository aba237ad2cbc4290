/*
 * vimscan.h -- C ABI of the B200 (sm_100a) selective-scan library libvimscan.so.
 *
 * The operations are those of the page "Vision Mamba Guide: Efficient Bidirectional
 * SSM & VMamba" (aifetchly-blog):
 *   - the S6 recurrence with input-dependent Delta, B, C (sections "Discretization
 *     via Zero-Order Hold (ZOH)" and "The Selective State Space (S6) Mechanism"):
 *         Delta_t = softplus(delta_raw_t + delta_bias)      (softplus(x) = x for x > 20)
 *         h_t     = exp(Delta_t * A) * h_{t-1} + Bbar_t * u_t            (h starts at 0)
 *         y_t     = C_t . h_t + D * u_t
 *     with the first-order Bbar_t = Delta_t * B_t, or on request (VIM_FLAG_ZOH_EXACT)
 *     the exact zero-order-hold form;
 *   - the Vim bidirectional block (section "2. The Bidirectional Mamba Block"): a
 *     forward pass over the tokens and a backward pass from the last token to the
 *     first, fused as (y^f + y^b) * silu(z), silu(z) = z / (1 + exp(-z));
 *   - the VMamba cross-scan (sections "1. Cross-Scan Traversal (CS-Traverse)",
 *     "2. Parallel S6 State Space Processing", "3. Cross-Merge Reversal
 *     (CS-Merge)"): four scans of an H x W grid (row-major, its reverse,
 *     column-major, its reverse), each mapped back to (h, w) and summed.
 *
 * Conventions for every entry point:
 *   - All tensor pointers are DEVICE pointers owned by the caller, contiguous and
 *     row-major, 16-byte aligned (vim_scan_bidir_host takes its activations from
 *     host memory; see there).  The library allocates no device memory and keeps
 *     no state between calls; scratch memory is the caller's workspace.
 *   - `dt` is the element type of u, delta, z, B, C, ys and y (fp32 or bf16).  A, D
 *     and delta_bias are always fp32.  Arithmetic is fp32 with the state h held in
 *     fp32 registers; bf16 outputs are rounded once, to nearest even.
 *   - Calls are asynchronous on `stream` (NULL = the legacy default stream) and
 *     return before the kernels finish.  Inputs must stay valid and unmodified, and
 *     outputs and workspace untouched, until the stream reaches that point.
 *   - Arguments are checked on the host before anything is launched.  A failed
 *     check returns VIM_ERR_INVALID_ARG, VIM_ERR_UNSUPPORTED or VIM_ERR_WORKSPACE and
 *     launches nothing.  A launch failure returns VIM_ERR_CUDA.  No call aborts,
 *     throws or prints.
 *   - Sizes of 0 (batch, tokens or channels) are valid and do nothing.
 *   - Supported: d_state in {2, 4, 8, 16}; channels a multiple of 8 (bf16) or of 4
 *     (fp32).  Anything else returns VIM_ERR_UNSUPPORTED.
 *   - Outputs must not overlap inputs or the workspace.
 */
#ifndef VIMSCAN_H
#define VIMSCAN_H

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    VIM_OK = 0,
    VIM_ERR_INVALID_ARG = 1,   /* null or misaligned pointer, negative size        */
    VIM_ERR_UNSUPPORTED = 2,   /* d_state or channel count outside the supported set */
    VIM_ERR_WORKSPACE = 3,     /* workspace missing, misaligned or too small        */
    VIM_ERR_CUDA = 4,          /* a CUDA launch failed                              */
    VIM_ERR_TIMEOUT = 5        /* reserved: a bounded device-side wait ran out      */
} vim_status;

typedef enum { VIM_F32 = 0, VIM_BF16 = 1 } vim_dtype;

/*
 * Vim bidirectional selective scan with gated fusion (section "2. The Bidirectional
 * Mamba Block"; its output projection is not part of this call):
 *
 *   y[b,t,d] = ( y^f[b,t,d] + y^b[b,t,d] ) * silu(z[b,t,d])
 *   y^f : forward S6 over t = 0 .. L-1 with A[0], D[0], delta_bias[0], B, C
 *   y^b : backward S6 over t = L-1 .. 0 with A[1], D[1], delta_bias[1],
 *         B + bc_dir_stride, C + bc_dir_stride; y^b is indexed by original position.
 *
 *   u, delta, z : [batch, L, d_inner] (dt).  delta holds the raw value; the call
 *                 applies softplus(delta + delta_bias[k][d]).  z may be NULL: no gate.
 *   B, C        : [batch, L, d_state] (dt), shared by all channels of a token.
 *   bc_dir_stride: element offset of the backward direction's B and C from B and C
 *                 (0 = both directions read the same B and C).  Must be >= 0.
 *   A           : [2, d_inner, d_state] fp32 (index 0 = forward, 1 = backward);
 *                 fastest when A[k][d][n] == (n+1) * A[k][d][0] (the S4D-real form).
 *   D, delta_bias : [2, d_inner] fp32.
 *   y           : [batch, L, d_inner] (dt), written once.
 *   workspace   : caller-owned device scratch of at least
 *                 vim_scan_workspace_bytes(0, batch, L, 0, d_inner, d_state) bytes,
 *                 256-byte aligned (may be NULL when that size is 0).
 */
vim_status vim_scan_bidir(const void *u, const void *delta, const void *z,
                          const void *B, const void *C, int64_t bc_dir_stride,
                          const float *A, const float *D, const float *delta_bias,
                          void *y, int batch, int L, int d_inner, int d_state, vim_dtype dt,
                          void *workspace, size_t workspace_bytes, cudaStream_t stream);

/*
 * vim_scan_bidir with the pathways' convolution front fused in (section "2. The
 * Bidirectional Mamba Block": each pathway runs "1D Conv -> SiLU" before its S6; the
 * page's block uses a depthwise Conv1d of kernel 3 and padding 1, the backward one on
 * the reversed sequence):
 *
 *   u_f[b,t,d] = silu(conv_b[0][d] + w[0][d][0] x[t-1] + w[0][d][1] x[t] + w[0][d][2] x[t+1])
 *   u_b[b,t,d] = silu(conv_b[1][d] + w[1][d][0] x[t+1] + w[1][d][1] x[t] + w[1][d][2] x[t-1])
 *   (x = 0 outside 0..L-1; silu(v) = v / (1 + exp(-v)))
 *
 * and then exactly vim_scan_bidir with the forward direction fed u_f and the backward
 * one u_b (each direction's D skip uses its own u).  The smoothed inputs are formed in
 * registers from the staged x and never written to memory.
 *
 *   x       : [batch, L, d_inner] (dt), the pathways' common input.
 *   conv_w  : [2, d_inner, 3] fp32 (index 0 = forward); conv_b : [2, d_inner] fp32.
 *   all other arguments and the workspace as in vim_scan_bidir.
 */
vim_status vim_scan_bidir_conv(const void *x, const float *conv_w, const float *conv_b,
                               const void *delta, const void *z, const void *B, const void *C,
                               int64_t bc_dir_stride, const float *A, const float *D,
                               const float *delta_bias, void *y, int batch, int L, int d_inner,
                               int d_state, vim_dtype dt, void *workspace, size_t workspace_bytes,
                               cudaStream_t stream);

/* vim_scan_bidir_conv with the per-kernel events of vim_scan_bidir_events. */
vim_status vim_scan_bidir_conv_events(const void *x, const float *conv_w, const float *conv_b,
                                      const void *delta, const void *z, const void *B, const void *C,
                                      int64_t bc_dir_stride, const float *A, const float *D,
                                      const float *delta_bias, void *y, int batch, int L, int d_inner,
                                      int d_state, vim_dtype dt, void *workspace, size_t workspace_bytes,
                                      cudaStream_t stream, cudaEvent_t *events);

/*
 * VMamba four-direction cross-scan with CS-Merge (sections "1. Cross-Scan
 * Traversal", "2. Parallel S6 State Space Processing", "3. Cross-Merge Reversal"):
 *
 *   y[b,h,w,c] = ( sum_{k=1..4} y_k[b,h,w,c] ) * silu(z[b,h,w,c])
 *   scan 1 visits p = h*W + w in increasing order, scan 2 in decreasing order,
 *   scan 3 visits the grid column by column (step t = w*H + h), scan 4 the reverse
 *   of scan 3; each y_k is written back at the grid position its step visited.
 *
 *   u, delta, z : [batch, H, W, channels] (dt), channels last.  z may be NULL.
 *   B, C        : [4, batch, H*W, d_state] (dt), per direction, stored by GRID
 *                 position: scan k reads B[k, b, p, :] when it visits position p.
 *   A           : [4, channels, d_state] fp32; D, delta_bias : [4, channels] fp32.
 *   y           : [batch, H, W, channels] (dt).
 *   workspace   : at least vim_scan_workspace_bytes(1, batch, H, W, channels,
 *                 d_state) bytes, 256-byte aligned.
 */
vim_status vmamba_cross_scan4(const void *u, const void *delta, const void *z,
                              const void *B, const void *C,
                              const float *A, const float *D, const float *delta_bias,
                              void *y, int batch, int H, int W, int channels, int d_state,
                              vim_dtype dt, void *workspace, size_t workspace_bytes,
                              cudaStream_t stream);

/*
 * CS-Merge alone (section "3. Cross-Merge Reversal (CS-Merge)"): maps each of four
 * scan-order outputs back to its grid position and sums them.
 *
 *   ys : [4, batch, H*W, channels] (dt); row t of ys[k] belongs to the grid position
 *        that scan k+1 visits at step t (orders as in vmamba_cross_scan4).
 *   z  : [batch, H, W, channels] (dt) or NULL; the sum is multiplied by silu(z).
 *   y  : [batch, H, W, channels] (dt).  Sums are formed in fp32.
 */
vim_status cross_merge4(const void *ys, const void *z, void *y, int batch, int H, int W,
                        int channels, vim_dtype dt, cudaStream_t stream);

/*
 * Instrumented variants for benchmarks: the same checks and the same launches as
 * vim_scan_bidir / vmamba_cross_scan4, plus cudaEventRecord(events[i], stream) at
 * each kernel boundary.  A scan runs, per pair of directions, up to three kernels:
 * chunk summaries, their fold, and the main pass (the first two only when the
 * sequence spans more than one chunk; a skipped kernel's two events are recorded back
 * to back).  events[0] is recorded before the first kernel and events[3*k+i+1] after
 * kernel i of pair k, so vim_scan_bidir_events needs 4 events and
 * vmamba_cross_scan4_events 7.  Events are created by the caller; a NULL `events`
 * behaves exactly like the plain entry point.
 */
vim_status vim_scan_bidir_events(const void *u, const void *delta, const void *z,
                                 const void *B, const void *C, int64_t bc_dir_stride,
                                 const float *A, const float *D, const float *delta_bias,
                                 void *y, int batch, int L, int d_inner, int d_state,
                                 vim_dtype dt, void *workspace, size_t workspace_bytes,
                                 cudaStream_t stream, cudaEvent_t *events);

vim_status vmamba_cross_scan4_events(const void *u, const void *delta, const void *z,
                                     const void *B, const void *C,
                                     const float *A, const float *D, const float *delta_bias,
                                     void *y, int batch, int H, int W, int channels,
                                     int d_state, vim_dtype dt, void *workspace,
                                     size_t workspace_bytes, cudaStream_t stream,
                                     cudaEvent_t *events);

/*
 * Derivative of vim_scan_bidir (first-order Bbar) for a loss with derivative `dout`
 * with respect to y: the chain rule through the gate and each direction's recurrence
 * in reverse visiting order (the adjoint g of h obeys g_t = C_t dy_t + Abar_(t+1)
 * g_(t+1), dy = dout * silu(z)); training through the scan is what the pages'
 * "efficient training" of the selective scan refers to.
 *
 *   u, delta, z, B, C, bc_dir_stride, A, D, delta_bias : the forward call's inputs.
 *   dout   : [batch, L, d_inner] (dt).
 *   du, ddelta, dz : [batch, L, d_inner] (dt), written.  ddelta is with respect to the
 *            raw delta (through softplus).  dz must be NULL exactly when z is NULL.
 *   dB, dC : fp32, shaped like B and C: [batch, L, d_state], and with bc_dir_stride > 0
 *            the backward direction's part bc_dir_stride elements further on (at least
 *            bc_dir_stride + batch*L*d_state floats); with 0 both directions' terms
 *            are summed into one.
 *   dA [2, d_inner, d_state], dD [2, d_inner], ddelta_bias [2, d_inner] : fp32, written.
 *   workspace : vim_scan_bwd_workspace_bytes(batch, L, d_inner, d_state,
 *            bc_dir_stride > 0) bytes, 256-byte aligned.
 * The same size limits as vim_scan_bidir.  Results are deterministic (no floating
 * point atomics in global memory).
 */
vim_status vim_scan_bidir_bwd(const void *u, const void *delta, const void *z,
                              const void *B, const void *C, int64_t bc_dir_stride,
                              const float *A, const float *D, const float *delta_bias,
                              const void *dout, void *du, void *ddelta, void *dz,
                              float *dB, float *dC, float *dA, float *dD, float *ddelta_bias,
                              int batch, int L, int d_inner, int d_state, vim_dtype dt,
                              void *workspace, size_t workspace_bytes, cudaStream_t stream);
size_t vim_scan_bwd_workspace_bytes(int batch, int L, int d_inner, int d_state, int separate_bc);
/*
 * Derivative of vmamba_cross_scan4 (first-order Bbar) for a loss with derivative `dout`
 * with respect to y: dl/dz = dout (sum_k y_k) silu'(z), and each CS-Traverse direction
 * runs the chain rule of its recurrence with dl/dy_k = dout silu(z) at the grid
 * positions it visits (sections "1. Cross-Scan Traversal" to "3. Cross-Merge
 * Reversal").
 *
 *   u, delta, z, B, C, A, D, delta_bias : the forward call's inputs and layouts.
 *   dout, du, ddelta, dz : [batch, H, W, channels] (dt); dz NULL exactly when z is.
 *   dB, dC : fp32 [4, batch, H*W, d_state], grid order like B and C.
 *   dA [4, channels, d_state], dD [4, channels], ddelta_bias [4, channels] : fp32.
 *   workspace : vmamba_cross_scan4_bwd_workspace_bytes(...) bytes, 256-byte aligned.
 */
vim_status vmamba_cross_scan4_bwd(const void *u, const void *delta, const void *z,
                                  const void *B, const void *C,
                                  const float *A, const float *D, const float *delta_bias,
                                  const void *dout, void *du, void *ddelta, void *dz,
                                  float *dB, float *dC, float *dA, float *dD, float *ddelta_bias,
                                  int batch, int H, int W, int channels, int d_state, vim_dtype dt,
                                  void *workspace, size_t workspace_bytes, cudaStream_t stream);
size_t vmamba_cross_scan4_bwd_workspace_bytes(int batch, int H, int W, int channels, int d_state);

/* vim_scan_bidir_bwd plus 4 CUDA events (caller-created, or NULL for none) recorded
 * before the chunk summaries, after them, after the main derivative kernel and at
 * the end, for per-phase times. */
vim_status vim_scan_bidir_bwd_events(const void *u, const void *delta, const void *z,
                                     const void *B, const void *C, int64_t bc_dir_stride,
                                     const float *A, const float *D, const float *delta_bias,
                                     const void *dout, void *du, void *ddelta, void *dz,
                                     float *dB, float *dC, float *dA, float *dD, float *ddelta_bias,
                                     int batch, int L, int d_inner, int d_state, vim_dtype dt,
                                     void *workspace, size_t workspace_bytes, cudaStream_t stream,
                                     cudaEvent_t *events);

/*
 * The Vim block's two S6 modules from their common input x, projections included
 * (page "Vision Mamba Guide": section "2. The Bidirectional Mamba Block" runs
 * "1D Conv -> SiLU -> SSM" per pathway; its SSM module, under "The Selective State
 * Space (S6) Mechanism", derives B, C and Delta from its own input):
 *
 *   u_k   = silu(conv_k(x)) as in vim_scan_bidir_conv (conv_w, conv_b non-NULL), else x
 *   P_k   = u_k Wx[k]   (x_proj, no bias; [batch*L, 2N+1])
 *   B_k   = P_k[:, 0:N],  C_k = P_k[:, N:2N],  s_k = P_k[:, 2N]
 *   delta_raw_k[t, d] = s_k[t] * Wdt[k][d]      (dt_proj; its bias is dt_bias, in softplus)
 *   y = (S6_f(u_f; B_f, C_f, delta_f) + S6_b(u_b; B_b, C_b, delta_b)) * silu(z)
 *
 *   x, z, y : [batch, L, d_inner] bf16 (z may be NULL).
 *   Wx      : [2, d_inner, 2*d_state + 1] bf16 (index 0 = forward pathway).
 *   Wdt, dt_bias, D : [2, d_inner] fp32;  A : [2, d_inner, d_state] fp32.
 *   conv_w [2, d_inner, 3], conv_b [2, d_inner] fp32, both or neither.
 *   events  : NULL, or 5 CUDA events: start, after the projection, then those of
 *             vim_scan_bidir_events.
 *   workspace : vim_block_workspace_bytes(...) bytes, 256-byte aligned; it holds B, C
 *             (bf16) and s (fp32) of both pathways between the two kernels, and with
 *             the convolution front both pathways' u_k (bf16).
 * x_proj runs on the tensor cores with u_k rounded to bf16 and fp32 accumulation; B and
 * C are rounded to bf16, s stays fp32; Delta is never written to memory.  With the
 * convolution front the scan reads u_k as the projection kernel rounded and stored it
 * (the front is formed once).  Only bf16 I/O
 * (VIM_F32 returns VIM_ERR_UNSUPPORTED), the first-order Bbar, and d_inner up to 2776
 * (one pathway's Wx, transposed, is held in one CTA's shared memory).
 */
vim_status vim_block_scan(const void *x, const float *conv_w, const float *conv_b, const void *Wx,
                          const float *Wdt, const float *dt_bias, const float *A, const float *D,
                          const void *z, void *y, int batch, int L, int d_inner, int d_state,
                          vim_dtype dt, void *workspace, size_t workspace_bytes, cudaStream_t stream,
                          cudaEvent_t *events);
size_t vim_block_workspace_bytes(int batch, int L, int d_inner, int d_state);

/*
 * Derivatives of vim_block_scan (first-order Bbar) for a loss whose derivative with
 * respect to y is dout: the scan's derivative per pathway, carried back through dt_proj
 * and x_proj (P_k = u_k Wx[k], delta_raw_k = s_k Wdt[k]) and the convolution fronts.
 *
 *   x, conv_w, conv_b, Wx, Wdt, dt_bias, A, D, z : as in vim_block_scan (bf16 x, z, Wx).
 *   dout      : [batch, L, d_inner] bf16.
 *   Outputs (overwritten): dx [batch, L, d_inner] bf16; dz (NULL exactly when z is);
 *             dWx [2, d_inner, 2*d_state + 1], dWdt and ddt_bias [2, d_inner], dA [2,
 *             d_inner, d_state], dD [2, d_inner] fp32; dconv_w [2, d_inner, 3] and
 *             dconv_b [2, d_inner] fp32 exactly when conv_w and conv_b are given.
 *   workspace : vim_block_bwd_workspace_bytes(batch, L, d_inner, d_state) bytes,
 *             256-byte aligned.
 * The projections are formed again as the forward call forms them (B, C rounded to
 * bf16, s in fp32); the pathways' inputs u_k are formed in fp32 for the derivative.
 * Every sum is taken in a fixed order.  Only bf16 I/O (VIM_ERR_UNSUPPORTED else) and
 * the d_inner limit of vim_block_scan.  Size 0 writes zero parameter derivatives.
 */
vim_status vim_block_scan_bwd(const void *x, const float *conv_w, const float *conv_b, const void *Wx,
                              const float *Wdt, const float *dt_bias, const float *A, const float *D, const void *z,
                              const void *dout, void *dx, float *dconv_w, float *dconv_b, float *dWx, float *dWdt,
                              float *ddt_bias, float *dA, float *dD, void *dz, int batch, int L, int d_inner,
                              int d_state, vim_dtype dt, void *workspace, size_t workspace_bytes, cudaStream_t stream);
size_t vim_block_bwd_workspace_bytes(int batch, int L, int d_inner, int d_state);

/*
 * Options of the _ex entry points, or-ed into `flags` (unknown bits return
 * VIM_ERR_INVALID_ARG).
 *
 * VIM_FLAG_ZOH_EXACT: the exact zero-order-hold input matrix of section
 * "Discretization via Zero-Order Hold (ZOH)", Bbar = (Delta A)^-1 (exp(Delta A) - I)
 * Delta B, which for the diagonal A is, per state,
 *     Bbar_n = (exp(Delta A_n) - 1) / A_n * B_n      (Delta B_n where A_n = 0),
 * in place of its first-order form Bbar = Delta B used otherwise.  exp(Delta A_n) - 1
 * is formed without cancellation for small Delta A_n.
 */
#define VIM_FLAG_ZOH_EXACT 1u

/*
 * vim_scan_bidir with every option: the convolution front when conv_w and conv_b are
 * both non-NULL (then u holds x, as in vim_scan_bidir_conv; one NULL and the other
 * not is VIM_ERR_INVALID_ARG), the options in `flags`, and the events of
 * vim_scan_bidir_events when `events` is non-NULL.  Other arguments as in
 * vim_scan_bidir.
 */
vim_status vim_scan_bidir_ex(const void *u, const float *conv_w, const float *conv_b,
                             const void *delta, const void *z, const void *B, const void *C,
                             int64_t bc_dir_stride, const float *A, const float *D,
                             const float *delta_bias, void *y, int batch, int L, int d_inner,
                             int d_state, vim_dtype dt, unsigned flags, void *workspace,
                             size_t workspace_bytes, cudaStream_t stream, cudaEvent_t *events);

/*
 * vim_scan_bidir_bwd_events with options in `flags` (unknown bits return
 * VIM_ERR_INVALID_ARG).  With VIM_FLAG_ZOH_EXACT it is the derivative of the scan with
 * the exact hold, Bbar_n = e_n B_n, e_n = (exp(Delta A_n) - 1) / A_n: e_n takes Delta's
 * place in du and dB; the Delta term has de_n/dDelta = exp(Delta A_n); dA_n gains
 * g B_n u de_n/dA_n with de_n/dA_n = (Delta exp(Delta A_n) - e_n) / A_n (its series
 * Delta^2 (1/2 + Delta A_n / 3 + ...) for small Delta A_n).  Other arguments, the
 * workspace and the events as in vim_scan_bidir_bwd_events.
 */
vim_status vim_scan_bidir_bwd_ex(const void *u, const void *delta, const void *z,
                                 const void *B, const void *C, int64_t bc_dir_stride,
                                 const float *A, const float *D, const float *delta_bias,
                                 const void *dout, void *du, void *ddelta, void *dz,
                                 float *dB, float *dC, float *dA, float *dD, float *ddelta_bias,
                                 int batch, int L, int d_inner, int d_state, vim_dtype dt,
                                 unsigned flags, void *workspace, size_t workspace_bytes,
                                 cudaStream_t stream, cudaEvent_t *events);

/*
 * vmamba_cross_scan4_bwd with options in `flags` (unknown bits return
 * VIM_ERR_INVALID_ARG): VIM_FLAG_ZOH_EXACT gives the derivative of the cross-scan with
 * the exact hold, each direction's terms as in vim_scan_bidir_bwd_ex.  Other arguments
 * and the workspace as in vmamba_cross_scan4_bwd.
 */
vim_status vmamba_cross_scan4_bwd_ex(const void *u, const void *delta, const void *z,
                                     const void *B, const void *C,
                                     const float *A, const float *D, const float *delta_bias,
                                     const void *dout, void *du, void *ddelta, void *dz,
                                     float *dB, float *dC, float *dA, float *dD, float *ddelta_bias,
                                     int batch, int H, int W, int channels, int d_state, vim_dtype dt,
                                     unsigned flags, void *workspace, size_t workspace_bytes,
                                     cudaStream_t stream);

/* vmamba_cross_scan4 with the options in `flags` and the events of
 * vmamba_cross_scan4_events when `events` is non-NULL. */
vim_status vmamba_cross_scan4_ex(const void *u, const void *delta, const void *z,
                                 const void *B, const void *C,
                                 const float *A, const float *D, const float *delta_bias,
                                 void *y, int batch, int H, int W, int channels, int d_state,
                                 vim_dtype dt, unsigned flags, void *workspace,
                                 size_t workspace_bytes, cudaStream_t stream, cudaEvent_t *events);

/*
 * vim_scan_bidir for callers that cannot allocate device memory.
 *
 * The pages have no counterpart to this call; it is a packaging variant.  Some
 * callers cannot hand the scan a workspace: code running where cudaMalloc is not
 * allowed or not wanted (inside a stream capture that must not allocate, under an
 * allocator that owns all device memory, or from a plugin with no allocator of its
 * own).  This entry point takes the same inputs and output as vim_scan_bidir, without
 * a workspace, and keeps the chunk carries in a buffer built into the library: a
 * file-scope device array of VIM_NOALLOC_SCRATCH_BYTES bytes, which every GPU that
 * loads the library holds until the process exits.  The call allocates nothing.
 *
 *   - Limit: the problem must need at most VIM_NOALLOC_SCRATCH_BYTES of scratch, that
 *     is vim_scan_workspace_bytes(0, batch, L, 0, d_inner, d_state) <= that size
 *     (sequences of up to 256 tokens need none).  Larger problems return
 *     VIM_ERR_WORKSPACE and launch nothing.
 *   - The first call on each device looks up the buffer's device address (with that
 *     device current) and remembers it for the rest of the process; make that first
 *     call before any stream capture.  A failed lookup returns VIM_ERR_CUDA.  The
 *     remembered address belongs to the device's primary context as it was then: after
 *     cudaDeviceReset (or anything else that destroys that context) this entry point
 *     must not be called again in the same process.
 *   - All calls share the one buffer, and it keeps whatever the last call left in it.
 *     Nothing in it needs to start at zero: every value a call reads from it was
 *     written earlier by the same call.  Calls whose work overlaps on the GPU (two streams,
 *     or two threads with the same device) race on the buffer and corrupt each
 *     other's results: serialise them.
 */
#define VIM_NOALLOC_SCRATCH_BYTES ((size_t)8 << 20)
vim_status vim_scan_bidir_noalloc(const void *u, const void *delta, const void *z,
                                  const void *B, const void *C, int64_t bc_dir_stride,
                                  const float *A, const float *D, const float *delta_bias,
                                  void *y, int batch, int L, int d_inner, int d_state,
                                  vim_dtype dt, cudaStream_t stream);

/*
 * Derivatives of vim_scan_bidir_conv (or, with VIM_FLAG_ZOH_EXACT in flags, of its
 * exact-hold form) for a loss whose derivative with respect to y is dout: the scan's
 * derivative carried through each pathway's convolution front (section "2. The
 * Bidirectional Mamba Block": the pathways' "1D Conv -> SiLU" in front of their SSMs).
 *
 *   x, conv_w, conv_b, delta, z, B, C, bc_dir_stride, A, D, delta_bias, dt : as in
 *                 vim_scan_bidir_conv (conv_w [2, d_inner, 3], conv_b [2, d_inner] fp32).
 *   dout        : [batch, L, d_inner] (dt).
 *   Outputs (overwritten): dx [batch, L, d_inner] (dt); dconv_w [2, d_inner, 3] and
 *                 dconv_b [2, d_inner] fp32; ddelta (w.r.t. the raw delta), dz, dB, dC,
 *                 dA, dD, ddelta_bias as in vim_scan_bidir_bwd (dz NULL exactly when z
 *                 is).
 *   workspace   : vim_scan_conv_bwd_workspace_bytes(batch, L, d_inner, d_state, dt,
 *                 bc_dir_stride > 0) bytes, 256-byte aligned.  It holds, besides the
 *                 scan derivative's scratch, both pathways' smoothed inputs u_k and
 *                 their dl/du_k, in fp32.
 *
 * Every sum (over tokens for the taps, biases and parameters, over channels for dB
 * and dC) is taken in a fixed order: results repeat bit for bit.  Errors as for
 * vim_scan_bidir_bwd; size 0 writes zero parameter derivatives.
 */
vim_status vim_scan_bidir_conv_bwd_ex(const void *x, const float *conv_w, const float *conv_b, const void *delta,
                                      const void *z, const void *B, const void *C, int64_t bc_dir_stride,
                                      const float *A, const float *D, const float *delta_bias, const void *dout,
                                      void *dx, float *dconv_w, float *dconv_b, void *ddelta, void *dz, float *dB,
                                      float *dC, float *dA, float *dD, float *ddelta_bias, int batch, int L,
                                      int d_inner, int d_state, vim_dtype dt, unsigned flags, void *workspace,
                                      size_t workspace_bytes, cudaStream_t stream);
/* vim_scan_bidir_conv_bwd_ex with flags 0 (the first-order Bbar). */
vim_status vim_scan_bidir_conv_bwd(const void *x, const float *conv_w, const float *conv_b, const void *delta,
                                   const void *z, const void *B, const void *C, int64_t bc_dir_stride,
                                   const float *A, const float *D, const float *delta_bias, const void *dout,
                                   void *dx, float *dconv_w, float *dconv_b, void *ddelta, void *dz, float *dB,
                                   float *dC, float *dA, float *dD, float *ddelta_bias, int batch, int L,
                                   int d_inner, int d_state, vim_dtype dt, void *workspace, size_t workspace_bytes,
                                   cudaStream_t stream);
/* Workspace bytes of vim_scan_bidir_conv_bwd (0 for invalid arguments or an empty problem). */
size_t vim_scan_conv_bwd_workspace_bytes(int batch, int L, int d_inner, int d_state, vim_dtype dt, int separate_bc);

/*
 * vim_scan_bidir for activations in HOST memory: the same operation, flags and
 * parameters as vim_scan_bidir_ex without the convolution front, with u, delta, z,
 * B, C read from the host and y written to the host.  The pages have no counterpart
 * to this call; it is a packaging variant for callers whose activations live on the
 * host, so that the transfers are part of the library's pipeline.
 *
 *   u, delta, z, B, C, y : HOST pointers, shaped as in vim_scan_bidir (z may be NULL;
 *                 bc_dir_stride as there, counted in elements of the host B and C).
 *                 Page-locked memory (cudaHostAlloc, cudaHostRegister) lets the copies
 *                 run asynchronously and overlap; pageable memory gives the same result
 *                 but the driver stages those copies and the call waits for them.
 *   A, D, delta_bias : DEVICE pointers (the module's parameters stay resident).
 *   slices      : the batch is cut into this many pieces (at most batch; >= 1).  Piece k
 *                 goes to the device on `upload`, is scanned on `stream` and its y comes
 *                 back on `download`, so that piece k+1's upload and piece k-1's
 *                 download run while piece k is scanned.  Results do not depend on
 *                 `slices` for sequences longer than 256 tokens; shorter ones may take
 *                 a different chunking per piece and differ in rounding.
 *   workspace   : DEVICE scratch of vim_scan_host_workspace_bytes(batch, L, d_inner,
 *                 d_state, dt, slices, bc_dir_stride > 0) bytes, 256-byte aligned: two
 *                 staging sets of one piece each, and the scan's summaries.
 *   upload, download : streams for the copies (NULL: `stream` itself, and no overlap).
 *                 Use two streams created with cudaStreamNonBlocking that nothing else
 *                 uses during the call.
 *
 * Ordering: the copies start after the work queued on `stream` before the call, and
 * `stream` reaches the end of the call when the last piece of y is on the host: wait
 * on `stream` (an event or a synchronize) before reading y.  The host buffers must
 * stay valid and unmodified until then.  The call creates and releases its own CUDA
 * events and allocates no memory.  A failed check launches and copies nothing; a CUDA
 * failure part-way (VIM_ERR_CUDA) may leave y partly written.
 */
vim_status vim_scan_bidir_host(const void *u, const void *delta, const void *z, const void *B,
                               const void *C, int64_t bc_dir_stride, const float *A, const float *D,
                               const float *delta_bias, void *y, int batch, int L, int d_inner,
                               int d_state, vim_dtype dt, unsigned flags, int slices, void *workspace,
                               size_t workspace_bytes, cudaStream_t stream, cudaStream_t upload,
                               cudaStream_t download);
/* Workspace bytes of vim_scan_bidir_host (0 for invalid arguments or an empty problem). */
size_t vim_scan_host_workspace_bytes(int batch, int L, int d_inner, int d_state, vim_dtype dt, int slices,
                                     int two_bc);

/*
 * Training pair: the forward scan that also keeps the states its derivative needs, and
 * the derivative that takes them.  Reverse mode needs h entering every 32-token chunk
 * of the derivative in each direction ("Vision Mamba Guide", "Discretization via
 * Zero-Order Hold (ZOH)": the recurrence h_t = Abar_t h_(t-1) + Bbar_t u_t, run by the
 * forward pass anyway).  vim_scan_bidir_bwd forms them with a summary pass and a fold of
 * its own; after vim_scan_bidir_ckpt the forward pass has written them as it went.
 *
 * vim_scan_bidir_ckpt: vim_scan_bidir_ex without the convolution front (same arguments,
 * same y, same workspace), and
 *   ckpt  : DEVICE, fp32 [batch][ceil(L / 32)][2][d_state][d_inner] (state-major, so that
 *           the forward kernels write whole lines), vim_scan_ckpt_bytes bytes, 8-byte
 *           aligned, written whole: entry [b][c][k] is the state of direction k (0 forward,
 *           1 backward) entering 32-token chunk c in that direction's visiting order (zeros
 *           for the chunk each direction visits first).
 * vim_scan_bidir_bwd_ckpt: vim_scan_bidir_bwd_ex (same arguments, outputs and workspace)
 *   with ckpt as written by vim_scan_bidir_ckpt on the same u, delta, B, C, A,
 *   delta_bias and flags.  The results equal vim_scan_bidir_bwd_ex's up to rounding (the
 *   states come from the forward kernels' arithmetic instead of the derivative's
 *   summaries).  Checkpoints from other inputs give a wrong derivative, not an error.
 * vim_scan_bidir_conv_ckpt / vim_scan_bidir_conv_bwd_ckpt: the same pair for the scan with
 *   the pathways' convolution front (the arguments of vim_scan_bidir_conv / _ex and of
 *   vim_scan_bidir_conv_bwd_ex, with ckpt as above: the states of the recurrence on each
 *   pathway's u_k = silu(conv_k(x))).
 * vmamba_cross_scan4_ckpt / vmamba_cross_scan4_bwd_ckpt: the pair for the cross-scan (the
 *   arguments of vmamba_cross_scan4_ex and vmamba_cross_scan4_bwd_ex), ckpt fp32
 *   [2][batch][ceil(H W / 32)][2][d_state][channels], vmamba_cross_ckpt_bytes bytes: per pair
 *   of scans (rows, then columns) the states above over that pair's steps.
 * All return VIM_ERR_INVALID_ARG for a NULL or misaligned ckpt on a non-empty problem.
 */
vim_status vim_scan_bidir_ckpt(const void *u, const void *delta, const void *z, const void *B, const void *C,
                               int64_t bc_dir_stride, const float *A, const float *D, const float *delta_bias,
                               void *y, float *ckpt, int batch, int L, int d_inner, int d_state, vim_dtype dt,
                               unsigned flags, void *workspace, size_t workspace_bytes, cudaStream_t stream,
                               cudaEvent_t *events);
vim_status vim_scan_bidir_bwd_ckpt(const void *u, const void *delta, const void *z, const void *B, const void *C,
                                   int64_t bc_dir_stride, const float *A, const float *D, const float *delta_bias,
                                   const float *ckpt, const void *dout, void *du, void *ddelta, void *dz, float *dB,
                                   float *dC, float *dA, float *dD, float *ddelta_bias, int batch, int L,
                                   int d_inner, int d_state, vim_dtype dt, unsigned flags, void *workspace,
                                   size_t workspace_bytes, cudaStream_t stream, cudaEvent_t *events);
vim_status vim_scan_bidir_conv_ckpt(const void *x, const float *conv_w, const float *conv_b, const void *delta,
                                    const void *z, const void *B, const void *C, int64_t bc_dir_stride,
                                    const float *A, const float *D, const float *delta_bias, void *y, float *ckpt,
                                    int batch, int L, int d_inner, int d_state, vim_dtype dt, unsigned flags,
                                    void *workspace, size_t workspace_bytes, cudaStream_t stream,
                                    cudaEvent_t *events);
vim_status vim_scan_bidir_conv_bwd_ckpt(const void *x, const float *conv_w, const float *conv_b, const void *delta,
                                        const void *z, const void *B, const void *C, int64_t bc_dir_stride,
                                        const float *A, const float *D, const float *delta_bias, const float *ckpt,
                                        const void *dout, void *dx, float *dconv_w, float *dconv_b, void *ddelta,
                                        void *dz, float *dB, float *dC, float *dA, float *dD, float *ddelta_bias,
                                        int batch, int L, int d_inner, int d_state, vim_dtype dt, unsigned flags,
                                        void *workspace, size_t workspace_bytes, cudaStream_t stream);
vim_status vmamba_cross_scan4_ckpt(const void *u, const void *delta, const void *z, const void *B, const void *C,
                                   const float *A, const float *D, const float *delta_bias, void *y, float *ckpt,
                                   int batch, int H, int W, int channels, int d_state, vim_dtype dt, unsigned flags,
                                   void *workspace, size_t workspace_bytes, cudaStream_t stream,
                                   cudaEvent_t *events);
vim_status vmamba_cross_scan4_bwd_ckpt(const void *u, const void *delta, const void *z, const void *B,
                                       const void *C, const float *A, const float *D, const float *delta_bias,
                                       const float *ckpt, const void *dout, void *du, void *ddelta, void *dz,
                                       float *dB, float *dC, float *dA, float *dD, float *ddelta_bias, int batch,
                                       int H, int W, int channels, int d_state, vim_dtype dt, unsigned flags,
                                       void *workspace, size_t workspace_bytes, cudaStream_t stream);
/* Bytes of the checkpoints (0 for invalid arguments or an empty problem). */
size_t vim_scan_ckpt_bytes(int batch, int L, int d_inner, int d_state);
size_t vmamba_cross_ckpt_bytes(int batch, int H, int W, int channels, int d_state);

/*
 * Workspace bytes the scan entry points need (0 when none).  which = 0 for
 * vim_scan_bidir (L_or_H = L, W ignored), 1 for vmamba_cross_scan4 (L_or_H = H).
 * Returns 0 for invalid arguments as well; the entry point then reports them.
 */
size_t vim_scan_workspace_bytes(int which, int batch, int L_or_H, int W, int channels,
                                int d_state);

/* Static, NUL-terminated description of a status code (never NULL). */
const char *vim_status_string(vim_status status);

#ifdef __cplusplus
}
#endif

#endif /* VIMSCAN_H */
