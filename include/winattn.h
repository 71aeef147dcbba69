/*
 * winattn — fused, exact windowed softmax attention (forward) for vision
 * transformers on NVIDIA B200 (sm_100a).
 *
 * The operation (from "FLASHSWIN: Unlocking Large Windows and Dense Tokens
 * in Swin Vision Transformers with Memory Efficient Attention", section
 * "어떻게 동작하나", and "Rank-Factorized Implicit Neural Bias: Scaling
 * Super-Resolution Transformer with FlashAttention", section 2.1):
 *
 *   For every image b, head h and M x M window (wy, wx) of the map rolled by
 *   -shift (rolled token (yr, xr) is original token ((yr + shift) mod H,
 *   (xr + shift) mod W)), with window-local token p = i*M + j:
 *
 *     q~_p = [ R(i, j) q_p , u_h(p) ]        k~_p = [ R(i, j) k_p , w_h(p) ]
 *     z(p, p') = d^-1/2 <R q_p, R k_p'> + <u_h(p), w_h(p')>
 *                + ( -inf if shift > 0 and L(p) != L(p') else 0 )
 *     o_p = sum_p' softmax_p'(z(p, .)) v_p'
 *
 *   and o_p is written back to the original position of token p.  A map
 *   whose sides are not multiples of M is padded at the bottom and right to
 *   Hp x Wp, the next multiples of M, before the roll (H and W above read
 *   Hp and Wp; Swin pads before its roll, and FlashSwin-T runs M = 16 and 32
 *   on its 56 x 56 map, "FLASHSWIN" page, section "무엇과 다른가"); pad
 *   positions hold no token: they are never attended to (-inf) and never
 *   written, and nothing is copied.  R(i, j)
 *   is window-local 2D RoPE: pair (2k, 2k+1) of the first half of the head
 *   dim turns counter-clockwise by i * theta_h[k], pair (d/2 + 2k,
 *   d/2 + 2k + 1) of the second half by j * theta_h[k], k < d/4.  L is the
 *   wrap label 2*[yr >= H - shift] + [xr >= W - shift] of the rolled map.
 *   The u/w bias terms are present only when bias_feats is given.
 *
 * The N x N score matrix of a window (N = M*M) is never stored: the kernel
 * streams key tiles with an online softmax, so device memory beyond the
 * caller's buffers does not grow with M.
 *
 * Threading: every call is asynchronous on the given CUDA stream.  Calls on
 * different streams may run concurrently; they share only the per-device
 * status word read by winattn_last_device_status().
 */
#ifndef WINATTN_H
#define WINATTN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Return codes.  0 is success; every error is negative. */
#define WINATTN_OK                  0
#define WINATTN_ERR_ARG            -1  /* null pointer, non-positive size, M > 256,
                                          shift outside [0, M), unsupported head dim d          */
#define WINATTN_ERR_RANK           -2  /* rank > 0 without bias_feats, bias_feats without rank,
                                          or rank outside the supported set                    */
#define WINATTN_ERR_ALIGN          -3  /* a device pointer is not 16-byte aligned              */
#define WINATTN_ERR_DTYPE          -4  /* dtype is neither WINATTN_BF16 nor WINATTN_FP32       */
#define WINATTN_ERR_ARCH           -5  /* the current device is not compute capability 10.0    */
#define WINATTN_ERR_CUDA           -6  /* a CUDA runtime call or kernel launch failed          */
#define WINATTN_ERR_DEVICE_TIMEOUT -7  /* a bounded wait inside a kernel gave up               */
#define WINATTN_ERR_ALIAS          -8  /* out overlaps q, k or v                               */
#define WINATTN_ERR_SIZE           -9  /* a size product overflows the kernel's index range,
                                          or a host workspace is too small                     */
#define WINATTN_ERR_DEVICE_BOUNDS -10  /* debug builds (-DWINATTN_DEBUG) only: a kernel formed a
                                          token index or TMA box origin outside the map (the
                                          access was clamped into the map instead)            */

/* Storage / arithmetic types of q, k, v, bias_feats and out. */
#define WINATTN_BF16 0  /* bf16 storage; tensor-core QK^T and PV (bf16 in, fp32 accumulate),
                           RoPE and softmax in fp32                                            */
#define WINATTN_FP32 1  /* fp32 storage; fp32 arithmetic throughout                            */

/*
 * winattn_fwd — the fused forward pass.
 *
 *   q, k, v     device, [B][H_img][W_img][heads][d] row-major (channel-last,
 *               C = heads*d contiguous per token), element type `dtype`.
 *               16-byte aligned.  Read only.
 *   theta       device, fp32 [heads][d/4] RoPE frequencies theta = exp(omega),
 *               or NULL for no rotation.  Read only.
 *   bias_feats  device, element type `dtype`, [heads][2][M*M][rank]: index 0
 *               holds u(p) (query side), index 1 holds w(p) (key side), for
 *               window-local p = i*M + j; or NULL when rank == 0.  16-byte
 *               aligned.  Read only.
 *   B, H_img, W_img, M, shift, heads, d, rank
 *               sizes: any H_img, W_img >= 1 (padded to multiples of M as
 *               above), 0 <= shift < M,
 *               d in {32, 64} for WINATTN_BF16, d in {16, 32, 64} for
 *               WINATTN_FP32; rank in {0, 16, 32}; M <= 256; the number of
 *               128-row query tiles must fit in a 31-bit grid.
 *   dtype       WINATTN_BF16 or WINATTN_FP32.
 *   out         device, same layout and type as q; caller-allocated, must not
 *               overlap q, k or v.  Every element is written.
 *   stream      a cudaStream_t (NULL = the legacy default stream).
 *
 * Ownership: the caller owns every buffer; the library keeps no pointer past
 * the call and allocates no device memory.  Errors found on the host return
 * before anything is enqueued (out is untouched).  A kernel that gives up a
 * bounded wait records WINATTN_ERR_DEVICE_TIMEOUT in the per-device status
 * word (see winattn_last_device_status) and leaves `out` unspecified.
 */
int winattn_fwd(const void *q, const void *k, const void *v,
                const float *theta, const void *bias_feats,
                int B, int H_img, int W_img, int M, int shift,
                int heads, int d, int rank, int dtype,
                void *out, void *stream);

/*
 * winattn_fwd_lse — winattn_fwd that also saves, for the backward pass, the
 * log-sum-exp of every row's scores: lse[b][y][x][h] = log sum_p' exp z(p, p')
 * over the allowed keys p' of token (y, x) of image b, head h (natural log,
 * fp32, device, [B][H_img][W_img][heads], 4-byte aligned, must not overlap
 * q, k, v or out; written for every token, never at pad positions).  The
 * backward recomputes P = exp(z - lse) from it instead of storing any N x N
 * matrix ("FLASHSWIN" page, section "무엇과 다른가": memory was what kept
 * windows small in training).  Same arguments, results and errors as
 * winattn_fwd otherwise (lse NULL: WINATTN_ERR_ARG).  Adds 4 bytes per token
 * and head of writes.
 */
int winattn_fwd_lse(const void *q, const void *k, const void *v,
                    const float *theta, const void *bias_feats,
                    int B, int H_img, int W_img, int M, int shift,
                    int heads, int d, int rank, int dtype,
                    void *out, float *lse, void *stream);

/*
 * winattn_fwd_sparse — window attention on a list of gated windows only, as
 * the residual refinement of a global linear attention ("HSMLA:
 * Hierarchical Softmax Multi-scale Linear Attention for Efficient Vision
 * Transformers", section 2, Hierarchical Block-Level Gating and Two-Path
 * Residual Kernel): every token keeps the global linear-attention output
 * O_lin, and the tokens of the gated windows add O_local - O_lin-local:
 *
 *   out_p <- out_p + o_p - ( sum_p' relu(q_p).relu(k_p') v_p' )
 *                          / ( sum_p' relu(q_p).relu(k_p') )
 *
 * with o_p the window attention above and both sums over the allowed keys
 * p' of p (same window, same wrap label, real tokens), on the raw q, k (no
 * rotation, no bias features; the fraction is 0 when its denominator is 0).
 *
 *   q, k, v, theta, bias_feats, sizes  as for winattn_fwd; dtype WINATTN_BF16.
 *   windows     device, int32 [n_windows], 4-byte aligned: window ids
 *               w = (b * nWy + wy) * nWx + wx of the (padded) grid of windows
 *               of the rolled map, nWy = ceil(H_img / M), nWx = ceil(W_img / M);
 *               each id at most once (a repeated id adds its residual twice,
 *               racing) and below B * nWy * nWx (not checked on the device:
 *               an id out of range reads and writes outside the maps).
 *   n_windows   0 .. B * nWy * nWx (0: nothing is enqueued).
 *   out         device, bf16 map like q, holding O_lin on entry; updated in
 *               place for the tokens of the listed windows, untouched
 *               elsewhere.  Must not overlap q, k or v.
 *
 * Stream-ordered and asynchronous; allocates nothing.  Errors as winattn_fwd;
 * WINATTN_ERR_DTYPE for fp32.
 */
int winattn_fwd_sparse(const void *q, const void *k, const void *v,
                       const float *theta, const void *bias_feats,
                       int B, int H_img, int W_img, int M, int shift,
                       int heads, int d, int rank, int dtype,
                       const int32_t *windows, int n_windows, void *out, void *stream);

/*
 * winattn_rib_features — the rank-r bias factors of "Rank-Factorized
 * Implicit Neural Bias: Scaling Super-Resolution Transformer with
 * FlashAttention" (section 2.1) on the GPU: for every head, side (0 = u,
 * queries; 1 = w, keys) and window position p = i*M + j, Fourier features of
 * the window-local coordinate (c = 2 i / (M - 1) - 1 per axis, 0 when M = 1;
 * [sin 2^k pi c_y]_k, [cos 2^k pi c_y]_k, [sin 2^k pi c_x]_k,
 * [cos 2^k pi c_x]_k, k < 8) through tanh(f w1) w2.
 *
 *   w1     device fp32 [heads][2][32][64], 16-byte aligned.
 *   w2     device fp32 [heads][2][64][rank], 16-byte aligned.
 *   rank   16 or 32 (WINATTN_ERR_RANK otherwise); M <= 256.
 *   table  device bf16 [heads][2][M*M][rank] (the bias_feats of winattn_fwd),
 *          16-byte aligned; overwritten.
 * Stream-ordered; allocates nothing.
 */
int winattn_rib_features(const float *w1, const float *w2, int M, int heads, int rank, void *table, void *stream);

/*
 * winattn_fwd_rib — winattn_fwd with rank-r bias features generated from the
 * MLP weights in the same call: winattn_rib_features into `table` (caller
 * owned, bf16 [heads][2][M*M][rank], 16-byte aligned, must not overlap the
 * maps), then the attention reading it.  The table depends only on the
 * window position and head, so it is built once per call (a few
 * microseconds even at M = 96) and read by every window from L2, rather
 * than recomputed by every CTA that loads a tile of it.  dtype WINATTN_BF16.
 */
int winattn_fwd_rib(const void *q, const void *k, const void *v, const float *theta,
                    const float *w1, const float *w2,
                    int B, int H_img, int W_img, int M, int shift,
                    int heads, int d, int rank, int dtype,
                    void *table, void *out, void *stream);

/*
 * winattn_cla_gate — the convolutional local attention gate of the same
 * page (section 2.2): out = o * sigmoid(PW(DW3x3(x))) per token and channel,
 * DW a depth-wise 3 x 3 convolution with zero padding and one bias per
 * channel, PW a C x C point-wise convolution with bias.
 *
 *   x      device bf16 [B][H_img][W_img][C]: the block input the gate is
 *          computed from.
 *   o      device bf16, same shape: the attention output to gate.
 *   dw     device fp32 [C][3][3];  dw_b  fp32 [C].
 *   pw     device fp32 [C][C] (output channel major);  pw_b  fp32 [C].
 *   C      16 .. 256, a multiple of 16 (heads * d of the attention).
 *   out    device bf16, same shape; may be o itself (in place), must not
 *          overlap x.
 * One fused kernel: the depth-wise convolution in fp32 on the CUDA cores,
 * rounded to bf16, the point-wise contraction on tcgen05 (fp32 accumulate),
 * bias, sigmoid and product in the epilogue.  Stream-ordered; allocates
 * nothing.
 */
int winattn_cla_gate(const void *x, const void *o, const float *dw, const float *dw_b,
                     const float *pw, const float *pw_b, int B, int H_img, int W_img, int C, int dtype,
                     void *out, void *stream);

/*
 * winattn_bwd — the backward pass: gradients of a scalar loss L with respect
 * to q, k, v, the RoPE frequencies theta and the bias features, given
 * dout = dL/dO, the forward's output `out` and its saved log-sum-exp `lse`
 * (winattn_fwd_lse).  The FLASHSWIN page trains with learned frequencies
 * theta = exp(omega) (section "어떻게 동작하나"; dL/domega = theta dL/dtheta)
 * and names training memory as what kept windows small (section "무엇과
 * 다른가"): no N x N matrix is stored, P is recomputed per tile as
 * exp(z - lse).  With dS = P o (dP - rowsum(dO o O)), dP = dO V^T:
 *   dv = P^T dO;  d(Rq) = d^-1/2 dS (Rk);  d(Rk) = d^-1/2 dS^T (Rq);
 *   dq = R(i, j)^T d(Rq), dk likewise;  du = dS w, dw = dS^T u;
 *   dtheta_k = sum over tokens of i (g_{2k+1} x~_{2k} - g_{2k} x~_{2k+1})
 *              + j (same over the second half) for x~ = Rq, g = d(Rq) and
 *              for x~ = Rk, g = d(Rk).
 *
 *   q, k, v, theta, bias_feats, sizes, dtype
 *               as for winattn_fwd (dtype must be WINATTN_BF16).
 *   out, dout   device, bf16 maps like q: the forward's output and dL/dO.
 *   lse         device, fp32 [B][H_img][W_img][heads], from winattn_fwd_lse
 *               with the same inputs.
 *   dq, dk, dv  device, bf16 maps like q; caller-allocated, written for every
 *               token; must not overlap each other or any input map.
 *   dtheta      device, fp32 [heads][d/4], or NULL to skip (must be NULL
 *               when theta is); overwritten (zeroed, then summed into).
 *   dbias       device, fp32 [heads][2][M*M][rank] (du at index 0, dw at 1),
 *               or NULL to skip (NULL when bias_feats is); 16-byte aligned;
 *               overwritten.
 *   workspace   device, at least winattn_bwd_workspace_bytes(...) bytes,
 *               16-byte aligned (NULL allowed when that is 0): fp32 sums of
 *               dQ over the key tiles of windows larger than one 128-row
 *               tile.  Caller-owned; its contents on entry do not matter.
 *
 * Stream-ordered and asynchronous; allocates nothing.  theta, dbias and the
 * workspace gradients are summed with fp32 atomics, so their last bits may
 * vary from run to run; dq, dk, dv of windows of at most 128 tokens are
 * written directly and are bit-reproducible.  Errors as winattn_fwd
 * (WINATTN_ERR_DTYPE for fp32, WINATTN_ERR_SIZE for a short workspace,
 * WINATTN_ERR_ALIAS for overlapping gradients).
 */
int winattn_bwd(const void *q, const void *k, const void *v,
                const float *theta, const void *bias_feats,
                const void *out, const void *dout, const float *lse,
                int B, int H_img, int W_img, int M, int shift,
                int heads, int d, int rank, int dtype,
                void *dq, void *dk, void *dv, float *dtheta, float *dbias,
                void *workspace, size_t workspace_bytes, void *stream);

/* Device workspace bytes winattn_bwd needs (0 when every window fits one
 * 128-row tile, M * M <= 128), or 0 for invalid sizes. */
size_t winattn_bwd_workspace_bytes(int B, int H_img, int W_img, int M, int heads, int d);

/*
 * winattn_check_args — the host-side argument checks of winattn_fwd alone:
 * returns the code winattn_fwd would return before enqueuing anything
 * (WINATTN_OK if the arguments are acceptable).  Touches no device and makes
 * no CUDA call; pointers are only compared and checked for alignment.
 */
int winattn_check_args(const void *q, const void *k, const void *v,
                       const float *theta, const void *bias_feats,
                       int B, int H_img, int W_img, int M, int shift,
                       int heads, int d, int rank, int dtype, const void *out);

/*
 * winattn_fwd_host — the same operation on HOST buffers q, k, v, out (pinned
 * memory gives asynchronous copies; pageable memory works but the copies
 * then block).  theta and bias_feats stay device pointers (resident
 * parameters).  `workspace` is a caller-owned device buffer of at least
 * winattn_host_workspace_bytes(...) bytes, 16-byte aligned, that holds the
 * device copies of q, k, v and out.  Enqueues the H2D copies, the kernels and
 * the D2H copy of out and returns; synchronise `stream` before reading out.
 * The work is stream-ordered on `stream` (it starts after the work already
 * enqueued there, and work enqueued there later starts after it), but runs on
 * library-owned streams ("lanes", created once per device by the first call,
 * which should therefore come before any stream capture): the batch is cut
 * into up to 8 chunks of whole images that take turns on 3 lanes, so that one
 * chunk's kernel and read-back overlap the next chunk's upload.  Concurrent
 * host-buffer calls on one device are serialised on those lanes.  Allocates
 * no device memory.
 */
int winattn_fwd_host(const void *q_host, const void *k_host, const void *v_host,
                     const float *theta, const void *bias_feats,
                     int B, int H_img, int W_img, int M, int shift,
                     int heads, int d, int rank, int dtype,
                     void *out_host, void *workspace, size_t workspace_bytes,
                     void *stream);

/* Bytes of device workspace winattn_fwd_host needs (4 maps, each rounded up to
 * 256 bytes), or 0 for invalid sizes. */
size_t winattn_host_workspace_bytes(int B, int H_img, int W_img, int heads, int d, int dtype);

/*
 * winattn_fwd_host_static — winattn_fwd_host for callers that cannot allocate
 * device memory: code that links this library into a process whose device
 * memory is owned by someone else (a host application that must not grow the
 * GPU's allocations, a plug-in without access to the owner's allocator), so
 * it can pass neither a workspace nor device buffers.  (There is no
 * counterpart on the pages: this is an interface convenience, not part of the
 * method.)
 *
 * Same arguments and result as winattn_fwd_host, without the workspace: the
 * device copies of q, k, v and out live in one library-owned static device
 * buffer of WINATTN_STATIC_WORKSPACE_BYTES (every GPU that loads the library
 * holds it until the process exits).  Problems whose four maps do not fit
 * (winattn_host_workspace_bytes(...) > WINATTN_STATIC_WORKSPACE_BYTES) return
 * WINATTN_ERR_SIZE before anything is enqueued.  Allocates nothing: no
 * cudaMalloc, cudaFree or allocating library call.
 *
 * Unlike winattn_fwd_host it enqueues its copies and kernel on `stream`
 * alone, one after the other (no lanes, no chunks).
 *
 * The first call on a device looks up the buffer's device address with that
 * device current; make that first call before any stream capture.  Every call
 * on a device shares the one buffer and leaves its contents behind (each call
 * overwrites all of what it reads), so calls whose work overlaps on the GPU
 * (other streams, or host threads) race on it: order them on one stream.
 */
#define WINATTN_STATIC_WORKSPACE_BYTES ((size_t)32 << 20)
int winattn_fwd_host_static(const void *q_host, const void *k_host, const void *v_host,
                            const float *theta, const void *bias_feats,
                            int B, int H_img, int W_img, int M, int shift,
                            int heads, int d, int rank, int dtype,
                            void *out_host, void *stream);

/* A static, human-readable description of a return code. */
const char *winattn_strerror(int code);

/*
 * winattn_last_device_status — synchronises `stream`, then reads and clears
 * the current device's status word.  Returns WINATTN_OK when no kernel has
 * given up a bounded wait since the last read, WINATTN_ERR_DEVICE_TIMEOUT
 * when one has, WINATTN_ERR_DEVICE_BOUNDS when a debug build found an index
 * outside the map, or WINATTN_ERR_CUDA if the synchronisation failed.
 */
int winattn_last_device_status(void *stream);

/*
 * winattn_launch_info — the launch plan winattn_fwd would use, for tests and
 * benchmarks: work items (128-row query tiles), grid size (persistent kernels:
 * one CTA per SM of a 148-SM B200, capped by the work items), threads per CTA,
 * dynamic shared memory bytes, windows packed per tile and the kernel chosen
 * (0 = generic tensor-core kernel, 1 = persistent small-window kernel,
 * 2 = persistent large-window kernel, 3 = fp32 SIMT kernel, 4 = pipelined
 * kernel for 8 x 8 windows, 5 = pipelined kernel for 16 x 16 windows).  Any output pointer may be NULL.  Makes no CUDA
 * call.  Returns the winattn_check_args code for the sizes (pointers are not
 * checked).
 */
int winattn_launch_info(int B, int H_img, int W_img, int M, int shift, int heads, int d,
                        int rank, int dtype, int64_t *work_items, int *grid, int *threads,
                        int *smem_bytes, int *windows_per_tile, int *kernel);

/*
 * winattn_selftest_wait_timeout — failure-detection self-test (the pages
 * have no counterpart): enqueues on `stream` a one-warp kernel that waits on
 * an mbarrier nothing arrives at, through the bounded wait the attention
 * kernels use.  The wait gives up after its limit (2 s of %globaltimer), the
 * kernel records WINATTN_ERR_DEVICE_TIMEOUT in the status word and returns;
 * a following winattn_last_device_status(stream) returns that code and the
 * device stays usable.  Returns WINATTN_OK once enqueued, WINATTN_ERR_ARCH
 * off sm_100, WINATTN_ERR_CUDA if the launch failed.  Touches no caller
 * memory.
 */
int winattn_selftest_wait_timeout(void *stream);

/*
 * winattn_set_kernel_enabled — process-wide switch of a specialised kernel
 * (the kernel ids of winattn_launch_info: 1 = persistent small-window,
 * 2 = persistent large-window, 4 = pipelined 8 x 8 kernel, 5 = pipelined
 * 16 x 16 kernel).  While a kernel is
 * disabled, winattn_fwd and winattn_launch_info route its problems to the
 * next kernel that serves them (in the end the generic tensor-core kernel,
 * which serves every bf16 problem); the results agree within the bf16
 * tolerance.  For testing the fallbacks and for isolating a kernel; the
 * generic and fp32 kernels cannot be disabled.  Returns the previous state
 * (1 enabled, 0 disabled) or WINATTN_ERR_ARG for another id.  Makes no CUDA
 * call.  The large-window kernel is also bypassed, without this switch, when
 * its build does not have the register count its warpgroup split assumes.
 */
int winattn_set_kernel_enabled(int kernel, int enabled);

#ifdef __cplusplus
}
#endif
#endif /* WINATTN_H */
