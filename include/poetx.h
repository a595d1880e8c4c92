/*
 * poetx.h - C ABI of the POET-X orthogonal-equivalence linear layer for
 * NVIDIA B200 (sm_100a).
 *
 * The layer (POET-X write-up, zhichai.net, "POET-X：单卡H100训练130亿参数模型",
 * sections 1-3):
 *   z = P^T (W0^T (R^T x))                       section 1, input-centric form
 *   R = Psi_R^T Diag(G_R1..G_R,m/b) Psi_R        section 2, block-stochastic R
 *   P = Psi_P^T Diag(G_P1..G_P,n/b) Psi_P        (the same construction on the n side)
 *   G = (I + Q)(I + Q + Q^2 + Q^3), Q = -Q^T     section 3, Cayley-Neumann
 *   Q stored as its b(b-1)/2 upper triangle      section 3
 * W0 (m x n) is frozen between merges; every few hundred steps the training
 * loop folds R and P into it (W0 <- R W0 P), resets Q = 0 and draws new
 * permutations (merge_if_needed in the write-up's API snippet).
 *
 * Batched row form: X is T x m (one token per row), Z = X R W0 P is T x n.
 *
 * Conventions shared by every call:
 *  - Every pointer argument is a DEVICE pointer unless stated otherwise, owned
 *    and allocated by the caller, 16-byte aligned.  The library allocates no
 *    memory; scratch comes from the caller's workspace (`ws`, `ws_bytes`,
 *    sized by the matching *_workspace_bytes call).
 *  - Work is queued asynchronously on `stream` (a cudaStream_t; NULL = the
 *    legacy default stream).  Nothing synchronises the host.
 *  - Arguments are validated before anything is queued; on error the call
 *    returns a non-zero poetx_status and queues nothing.  A failure reported
 *    by the CUDA runtime while queueing returns POETX_E_CUDA.
 *  - Kernels never trap: a wait that times out inside a kernel or an index
 *    out of range sets a sticky device error word, read with
 *    poetx_device_error().
 *  - Layout of the stored weight (the "Psi frame"): W is [n][m] row-major,
 *    W[j'][i'] = W0[permR[i']][permP[j']], i.e. the nn.Linear weight W0^T with
 *    rows permuted by Psi_P and columns by Psi_R.  Permutations: perm[i'] is
 *    the natural index at frame position i', (Psi v)[i'] = v[perm[i']].
 *  - Packed triangle: row-major over i < j, k(i,j) = i(b-1) - i(i-1)/2 +
 *    (j-i-1), Q[i][j] = +q[k], Q[j][i] = -q[k].
 *  - dtype POETX_BF16: x, z, W, G, y_save, dz, dx are bf16, accumulation is
 *    fp32 on tcgen05 tensor cores; b must be a multiple of 64.  dtype
 *    POETX_FP32: everything fp32 (FFMA; tcgen05 has no fp32 kind).
 *  - Requirements: b >= 2 divides m and n; m <= 51200 and n <= 102400 (bf16)
 *    or 51200 (fp32), the widest rows the row-staging kernels hold in shared
 *    memory; T <= 2^31 - 257 token rows; the device is compute capability
 *    10.0 (B200).
 */
#ifndef POETX_H
#define POETX_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  POETX_OK = 0,
  POETX_E_ARG = 1,       /* null pointer, negative size, bad flag */
  POETX_E_SHAPE = 2,     /* b does not divide m or n, b unsupported for the dtype, m, n or T above its limit */
  POETX_E_DTYPE = 3,     /* unknown dtype */
  POETX_E_ALIGN = 4,     /* a pointer is not 16-byte aligned */
  POETX_E_WORKSPACE = 5, /* ws too small or NULL */
  POETX_E_ARCH = 6,      /* current device is not compute capability 10.0 */
  POETX_E_CUDA = 7       /* the CUDA runtime reported an error while queueing */
} poetx_status;

typedef enum { POETX_FP32 = 0, POETX_BF16 = 1 } poetx_dtype;

/* Evaluation order of a bf16 layer (poetx_layer.fold).  0, the default, is
 * the write-up's input-centric form (section 1): every block product acts on
 * token rows and no transformed weight is ever formed.  The bits below let
 * the library apply a block product to the n x m weight instead when that
 * moves fewer bytes; each forms a weight-sized TRANSIENT copy in the caller's
 * workspace (never kept between calls) and gives the same product rounded at
 * a different point.  fp32 layers ignore them.
 *   POETX_FOLD_R: forward with T > n: W_R = W Diag(G_R)^T, Y = Xg W_R^T.
 *   POETX_FOLD_P: backward with T > m: W_P = Diag(G_P)^T W, dU = dV W_P.
 *   POETX_FOLD_WEIGHT_CENTRIC: a forward that saves nothing (y_save ==
 *     xg_save == NULL) with T > 6nm/(2m+4n) forms the whole transformed
 *     weight Psi_P^T Diag(G_P)^T W Diag(G_R)^T Psi_R and runs one GEMM (the
 *     write-up's weight-centric form). */
enum {
  POETX_FOLD_R = 1,
  POETX_FOLD_P = 2,
  POETX_FOLD_WEIGHT_CENTRIC = 4,
  POETX_FOLD_ALL = 7
};

/* One layer.  All pointers are device pointers owned by the caller. */
typedef struct {
  int32_t m, n, b;      /* W0 is m x n; blocks of b x b */
  int32_t dtype;        /* poetx_dtype */
  void* W;              /* [n][m] frame-ordered frozen weight (see above) */
  const int32_t* permR; /* [m] Psi_R */
  const int32_t* permP; /* [n] Psi_P */
  float* qR;            /* [m/b][b(b-1)/2] packed triangles of Q_R (fp32) */
  float* qP;            /* [n/b][b(b-1)/2] packed triangles of Q_P (fp32) */
  void* GR;             /* [m/b][b][b] G_R blocks in dtype, written by poetx_cnp_build */
  void* GP;             /* [n/b][b][b] G_P blocks in dtype */
  int32_t fold;         /* POETX_FOLD_* bits; 0 = input-centric (other bits: POETX_E_ARG) */
} poetx_layer;

/* Human-readable name of a status code (static string, never NULL). */
const char* poetx_status_string(int status);

/* ABI version (major*10000 + minor*100 + patch). */
int32_t poetx_version(void);

/* Reads the sticky device error word (bit 1: a bounded wait inside a GEMM
 * timed out; bit 2: a bounded wait inside a copy kernel timed out; bit 4: a
 * permutation index was out of range; bit 8, builds with -DPOETX_DEBUG only:
 * a TMA or bulk copy broke an alignment or coordinate rule and was skipped)
 * into *code (HOST pointer) and clears it.  Synchronises the current device. */
poetx_status poetx_device_error(uint32_t* code);

/* Workspace sizes in bytes (host-side arithmetic only, no device access);
 * 0 for an invalid layer or T. */
size_t poetx_cnp_workspace_bytes(int32_t nblk, int32_t b, int32_t dtype);
size_t poetx_forward_workspace_bytes(const poetx_layer* layer, int64_t T);
size_t poetx_backward_workspace_bytes(const poetx_layer* layer, int64_t T);
size_t poetx_backward_recompute_workspace_bytes(const poetx_layer* layer, int64_t T);
size_t poetx_merge_workspace_bytes(const poetx_layer* layer);
size_t poetx_check_perm_workspace_bytes(int32_t len);

/* Stored-weight frame.  import: W = frame(W0lin) with W0lin the natural
 * nn.Linear weight W0^T ([n][m], dtype); export is the inverse.  Bit-exact
 * permutations (section 2's Psi folded into W0's row/column order). */
poetx_status poetx_frame_import(const poetx_layer* layer, const void* W0lin, void* stream);
poetx_status poetx_frame_export(const poetx_layer* layer, void* W0lin, void* stream);

/* Cayley-Neumann build (section 3): for each of nblk packed triangles
 * q[nblk][b(b-1)/2] (fp32) writes G[nblk][b][b] (dtype) with
 * G = (I+Q)(I+Q+Q^2+Q^3), evaluated as S = Q Q, G = I + 2Q + 2S + (2Q+S) S
 * (every power of Q is built from Q and S = Q^2).  POETX_FP32: fp32 FFMA;
 * POETX_BF16 with b = 256: one block per pair of SMs, every product on
 * tcgen05 tensor cores (cta_group::2) with bf16 operands and fp32
 * accumulation, S and H = 2Q + S kept in shared memory as bf16 operands,
 * G = I + H + S + H S^T rounded once to bf16; POETX_BF16 with other b: a chain
 * of tcgen05 GEMMs with tf32 operands over the whole batch. */
poetx_status poetx_cnp_build(int32_t nblk, int32_t b, const float* q, int32_t dtype, void* G, void* ws,
                             size_t ws_bytes, void* stream);

/* Both Cayley-Neumann builds of a layer in one batch: GR from qR and GP
 * from qP (same arithmetic as poetx_cnp_build on each side).  Workspace:
 * poetx_layer_cnp_workspace_bytes(layer). */
size_t poetx_layer_cnp_workspace_bytes(const poetx_layer* layer);
poetx_status poetx_layer_cnp_build(const poetx_layer* layer, void* ws, size_t ws_bytes, void* stream);

/* poetx_cnp_build without a caller workspace, for callers that cannot
 * allocate device memory (for example a host program with no device
 * allocator of its own, or a process that fixes its memory budget at
 * start-up).  The write-up has no counterpart: this is a deployment variant of
 * poetx_cnp_build with the same arguments (minus ws) and the same result.
 * Scratch is a 24 MiB device array inside the library, held by every GPU
 * that loads it until the process exits.  It fits the build that runs:
 * POETX_BF16 with b = 256 (one block per pair of SMs) takes 128 KiB per block
 * (its bf16 Q), so nblk <= 191; the other
 * builds take Q, S and H in fp32, nblk*b*b <= ~2.09e6 elements (b = 512:
 * nblk <= 7; fp32 b = 64: nblk <= 511).  Larger requests return
 * POETX_E_WORKSPACE without queueing anything.  The
 * first call on a device looks up the array's device address
 * (cudaGetSymbolAddress) with that device current; make that first call
 * before any stream capture.  All calls share the one array and its contents
 * persist between calls (nothing in it needs to start at zero): calls whose
 * work overlaps on the GPU (other streams, other threads) race on it, so
 * order them on one stream or synchronise between them. */
poetx_status poetx_cnp_build_fixed(int32_t nblk, int32_t b, const float* q, int32_t dtype, void* G, void* stream);

/* The Cayley-Neumann builds of several layers (1 <= nlayers <= 16, all with
 * the same b and dtype; `layers` is a HOST array of layer structs) in one
 * batch: GR and GP of every layer.  Workspace:
 * poetx_layers_cnp_workspace_bytes(nlayers, layers) (0 for an invalid set). */
size_t poetx_layers_cnp_workspace_bytes(int32_t nlayers, const poetx_layer* layers);
poetx_status poetx_layers_cnp_build(int32_t nlayers, const poetx_layer* layers, void* ws, size_t ws_bytes,
                                    void* stream);

/* Backward of poetx_cnp_build: given dG = dL/dG [nblk][b][b] (fp32), writes
 * dq = dL/dq [nblk][b(b-1)/2] (fp32), dq_k = dL/dQ[i][j] - dL/dQ[j][i].
 * accumulate != 0 adds to dq instead of overwriting it.  dtype names the
 * layer precision the gradient serves: POETX_FP32 multiplies in fp32 FFMA;
 * POETX_BF16 on tcgen05 tensor cores with fp32 accumulation, bf16 operands
 * for b = 256 (one block per pair of SMs; the terms of dq that need no
 * product, 2 (dG[i][j] - dG[j][i]), are added in fp32) and tf32 operands for
 * other b.  Results are identical for every nblk and block order. */
poetx_status poetx_cnp_backward(int32_t nblk, int32_t b, const float* q, const float* dG, float* dq,
                                int32_t accumulate, int32_t dtype, void* ws, size_t ws_bytes, void* stream);

/* Forward (section 1, input-centric): z = x R W0 P for T token rows.
 * x [T][m], z [T][n] in natural feature order (dtype).  y_save [T][n] (dtype)
 * receives Y = (x Psi_R^T Diag(G_R)) W (the P-side input, in the Psi_P
 * frame) for the backward; pass NULL for inference.  xg_save [T][m] (dtype,
 * nullable) receives Xg = x Psi_R^T, which spares the backward a gather of x.
 * Uses layer->GR/GP as last built by poetx_cnp_build.  T = 0 is a no-op.
 * With layer->fold == 0 every step acts on the token rows.  With
 * POETX_FOLD_R, bf16 layers with T > n apply Diag(G_R) to the weight rows
 * instead (Y = Xg (W Diag(G_R)^T)^T, same product, rounded once at W_R
 * instead of at U).  With POETX_FOLD_WEIGHT_CENTRIC, y_save == xg_save ==
 * NULL (inference) and T > 6nm/(2m+4n), bf16 layers fold the whole layer into
 * one natural-frame weight and compute z = x W_eff^T as a single GEMM (same
 * product, rounded at the folded weights instead of at the activations). */
poetx_status poetx_forward(const poetx_layer* layer, int64_t T, const void* x, void* z, void* y_save,
                           void* xg_save, void* ws, size_t ws_bytes, void* stream);

/* Backward of L = <dz, z>: dx [T][m] (dtype; NULL skips it) and the packed
 * gradients dqR [m/b][b(b-1)/2], dqP [n/b][b(b-1)/2] (fp32; overwritten, or
 * added to when accumulate != 0).  Needs either the xg_save of the matching
 * forward or (xg_save == NULL) the input x, which is then gathered again, and
 * the forward's y_save.  With y_save == NULL the backward recomputes Y from
 * Xg (one more block product and W0 product; the "POET-X mem" variant of the
 * write-up's section "三种变体", which keeps no [T][n] activation); its
 * workspace is then poetx_backward_recompute_workspace_bytes.  W0 is frozen,
 * so no dW0.  The dq sums over tokens use a fixed split and order
 * (deterministic for a given shape).  With POETX_FOLD_P, bf16 layers with
 * T > m form dU = dV (Diag(G_P)^T W) instead of (dV Diag(G_P)^T) W (same
 * product, rounded once at the folded weight instead of at dY).  The
 * recomputing backward takes the forward's fold decisions, so its Y is the
 * forward's bit for bit. */
poetx_status poetx_backward(const poetx_layer* layer, int64_t T, const void* x, const void* y_save,
                            const void* xg_save, const void* dz, void* dx, float* dqR, float* dqP,
                            int32_t accumulate, void* ws, size_t ws_bytes, void* stream);

/* poetx_backward with the Cayley-Neumann backward left out: instead of the
 * packed dq it writes the token sums dGR = dL/dG_R [m/b][b][b] and dGP =
 * dL/dG_P [n/b][b][b] (fp32, 16-byte aligned; overwritten, or added to when
 * accumulate != 0), the same fixed-order sums poetx_backward feeds its CNP
 * backward.  The CNP backward is linear in dG and per block, so one
 * poetx_cnp_backward over the dG of many layers (blocks back to back in the
 * order of their packed triangles: qR then qP of each layer) gives all their
 * dq in one batch.  Same arguments, checks and workspace as poetx_backward. */
poetx_status poetx_backward_dG(const poetx_layer* layer, int64_t T, const void* x, const void* y_save,
                               const void* xg_save, const void* dz, void* dx, float* dGR, float* dGP,
                               int32_t accumulate, void* ws, size_t ws_bytes, void* stream);

/* Merge (merge_if_needed in the write-up's API snippet): writes into W_out
 * ([n][m], dtype, must not overlap layer->W) the weight R W0 P expressed in
 * the frame of new_permR [m], new_permP [n] (device), with R and P built from
 * the layer's current G blocks; then sets qR = qP = 0 and GR = GP = I.  The
 * intermediate W Diag(G_R)^T is kept in fp32 (bf16 layers: the second block
 * product reads it at tf32 precision) and rounded to dtype once at the end.
 * The caller swaps W_out and the permutations into the layer afterwards. */
poetx_status poetx_merge(const poetx_layer* layer, const int32_t* new_permR, const int32_t* new_permP,
                         void* W_out, void* ws, size_t ws_bytes, void* stream);

/* Debug check: *d_ok (device int32) = 1 if perm [len] is a bijection of
 * 0..len-1, else 0. */
poetx_status poetx_check_perm(const int32_t* perm, int32_t len, int32_t* d_ok, void* ws, size_t ws_bytes,
                              void* stream);

/* Self-test of the failure path (no counterpart in the write-up): queues one
 * warp that waits on an mbarrier no thread arrives on, through the bounded
 * wait every kernel of the library uses, but with a limit of limit_us
 * microseconds (1..1000000) instead of 4 s.  The wait gives up, records bit 1
 * in the sticky device error word (read it with poetx_device_error) and the
 * kernel returns, leaving the context usable for further calls.  d_out
 * (device, 2 x uint64, 8-byte aligned): [0] = 1 if the wait ended by an
 * arrival (never expected), [1] = nanoseconds waited.  POETX_E_ARG for a
 * limit out of range or a NULL d_out. */
poetx_status poetx_selftest_wait_timeout(uint32_t limit_us, unsigned long long* d_out, void* stream);

/* POET-XQ storage of the frozen weight (write-up section "POET-XQ"): the
 * base weight is kept quantized and dequantized at run time.  The pages fix no
 * format; the reading here is int8, symmetric, one fp32 scale per row of the
 * stored [n][m] weight (per output feature): scale = max|row| / 127, code =
 * round-half-even(w / scale) clamped to [-127, 127] (fp32 arithmetic).
 * quantize: W [n][m] (dtype) -> Wq [n][m] int8 + scale [n] fp32.
 * dequantize: w = code * scale (fp32 product) rounded once to dtype, into W;
 * run it into a scratch weight before poetx_forward / poetx_backward. */
poetx_status poetx_weight_quantize(int32_t n, int32_t m, const void* W, int32_t dtype, int8_t* Wq, float* scale,
                                   void* stream);
poetx_status poetx_weight_dequantize(int32_t n, int32_t m, const int8_t* Wq, const float* scale, int32_t dtype,
                                     void* W, void* stream);

/* Optimizer step on packed triangles (fp32, n entries): AdamW with decoupled
 * weight decay (the write-up names get_poet_optimizer without describing it;
 * AdamW is the reading taken): m1 <- b1 m1 + (1-b1) g; m2 <- b2 m2 + (1-b2) g^2;
 * q <- q (1 - lr wd) - lr (m1 / (1 - b1^step)) / (sqrt(m2 / (1 - b2^step)) + eps).
 * step >= 1 counts the updates so far including this one.  After it, rebuild
 * G (poetx_layers_cnp_build). */
poetx_status poetx_adamw_step(int64_t n, float* q, const float* grad, float* m1, float* m2, float lr, float beta1,
                              float beta2, float eps, float weight_decay, int32_t step, void* stream);

/* Stage profiler (tracing).  Between poetx_profile_begin() and
 * poetx_profile_end(), every kernel the library queues is bracketed by a pair
 * of CUDA events on its stream and tagged with its stage (permute,
 * blockdiag_gemm, w0_gemm, dg_gemm, cnp_gemm, cnp_elementwise, dg_reduce,
 * merge, dequant, optimizer, blockdiag_dg: the backward's block product and
 * dG partials in one kernel).  poetx_profile_end waits for the recorded events, writes the summed
 * device time in ms (HOST array ms_per_stage[nstages]) and the number of
 * launches (HOST array launches_per_stage[nstages]) per stage, and stops
 * recording.  The events are created on first use and reused. */
int32_t poetx_profile_stage_count(void);
const char* poetx_profile_stage_name(int32_t stage);
poetx_status poetx_profile_begin(void);
poetx_status poetx_profile_end(double* ms_per_stage, int64_t* launches_per_stage, int32_t nstages);
/* Per-launch records of the last finished profiling session, in launch
 * order: stage index and device ms (HOST arrays of max_records entries).
 * Returns the number of records (pass NULL / 0 to query it). */
int32_t poetx_profile_records(int32_t* stages, float* ms, int32_t max_records);

#ifdef __cplusplus
}
#endif

#endif /* POETX_H */
