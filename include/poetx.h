/*
 * poetx.h — C ABI of the POET-X layer library (libpoetx.so, CUDA, sm_100a).
 *
 * The layer computes y = R · W0 · P · x for every token x (tokens are rows), where W0 is a
 * frozen base weight and R, P are trainable orthogonal transforms.  R and P are
 * block-diagonal in a randomly permuted basis, and every b×b block is the Cayley–Neumann
 * parameterisation (CNP) of a skew-symmetric block stored as its packed upper triangle.
 * Sources, by page and section:
 *   - agidaily.cc article on POET-X, section on fixing the base weight and training the
 *     two orthogonal transforms: W_RP = R · W0 · P, fast and mem implementations;
 *   - SAI replication review of POET-X (sai.science), "Summary": input-centric matrix-free
 *     chain, compact upper-triangular skew storage, batch-parallel block-diagonal matmul,
 *     two of the four permutations absorbed into W in advance, fused Cayley–Neumann kernel,
 *     POET-Xfast / POET-Xmem; "Reproducibility & code": k = 3, n_elements = b(b-1)/2,
 *     merge_then_reinitialize; "Weaknesses": first-order form I + 2Q of the Cayley map.
 *
 * Conventions (readings of the pages where they are silent; one per line in the design notes):
 *   X [N, d_in], Y [N, d_out], row-major; Y = X · (R · W0 · P)^T.
 *   P acts on the input side (nb_in = d_in / b blocks), R on the output side (nb_out = d_out / b).
 *   Permutations gather: (Π a)_i = a_{π(i)}.  R = Π_L^T · BD_R · Π_L, P = Π_R^T · BD_P · Π_R.
 *   Pre-permuted base weight W0' = Π_L · W0 · Π_R^T, i.e. W0'[i][j] = W0[π_L(i)][π_R(j)].
 *   So y = Π_L^T · BD_R · W0' · BD_P · Π_R · x, evaluated on the activations.
 *   Packed skew block: θ[p] = S[i][j] = -S[j][i] for i < j, p = i·b - i(i+1)/2 + (j - i - 1).
 *   CNP: Q = (I + S)(I + S + S^2 + ... + S^k)  (Neumann truncation of (I+S)(I-S)^-1).
 *
 * Memory and execution model (every entry point):
 *   - All array arguments are DEVICE pointers owned by the caller; the library never
 *     allocates, frees or retains them.  Every pointer must be 16-byte aligned.
 *   - Calls are asynchronous and ordered on `stream` (a cudaStream_t; NULL = legacy default).
 *   - Arguments are validated on the host before anything is launched: an invalid call
 *     returns an error status and launches nothing.
 *   - Activations, W0' and Q use `desc->dtype` (POETX_F32 or POETX_BF16); packed parameters
 *     θ and their gradients are always float32.  Dense arrays are row-major and contiguous.
 *   - Gradients overwrite their outputs (they do not accumulate).
 *   - `workspace` is caller-owned device scratch of at least poetx_workspace_size() bytes;
 *     its contents need not be preserved between calls.  Calls that share a workspace must
 *     not overlap in time (use one stream, or one workspace per stream).
 *   - Device-side waits are bounded; a wait that runs out records POETX_ERR_DEVICE_TIMEOUT,
 *     which poetx_device_status() returns.
 */
#ifndef POETX_H_
#define POETX_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* poetx_stream;   /* same type as cudaStream_t */

typedef enum {
  POETX_OK = 0,
  POETX_ERR_INVALID_ARG = 1,        /* NULL pointer, negative size, bad enum value      */
  POETX_ERR_UNSUPPORTED_SHAPE = 2,  /* d % b != 0, b or k outside the supported set     */
  POETX_ERR_ALIGNMENT = 3,          /* a pointer is not 16-byte aligned                 */
  POETX_ERR_WORKSPACE = 4,          /* workspace NULL or smaller than required          */
  POETX_ERR_CUDA = 5,               /* a CUDA runtime call or kernel launch failed      */
  POETX_ERR_DEVICE_TIMEOUT = 6      /* a bounded device-side wait ran out               */
} poetx_status;

typedef enum { POETX_F32 = 0, POETX_BF16 = 1 } poetx_dtype;

/* POET-Xfast keeps the W0'-GEMM output Z and the permuted input Π_R·x for the backward pass;
 * POET-Xmem keeps only X and recomputes Π_R·x, BD_P·(·) and Z in the backward pass (replication review, "Summary":
 * POET-Xfast and checkpointed POET-Xmem; agidaily.cc article: the mem variant recomputes part
 * of the activations). */
typedef enum { POETX_FAST = 0, POETX_MEM = 1 } poetx_mode;

typedef struct {
  int d_in;          /* input features, multiple of b; at most 32768 (BF16) / 16384 (F32) */
  int d_out;         /* output features, same rules as d_in                               */
  int b;             /* block size: 32, 64, 128, 256 or 512 (BF16: 64..512)              */
  int k;             /* Neumann order, 0 <= k <= 8 (the pages use k = 3)                  */
  poetx_dtype dtype; /* storage type of activations, W0', Q                               */
  poetx_mode mode;   /* POETX_FAST or POETX_MEM                                           */
} poetx_desc;

/* Bytes of device workspace that every entry point below needs for this layer and n_tokens
 * (the maximum over cnp / forward / backward / merge / absorb).  Returns 0 for an invalid
 * descriptor. */
size_t poetx_workspace_size(const poetx_desc* desc, int n_tokens);

/* CNP forward for both sides of one layer (replication review, "Summary": fused
 * Cayley–Neumann series; "Reproducibility & code": k = 3, n_elements = b(b-1)/2).
 *   theta_R  float32 [d_out/b, b(b-1)/2]   packed skew parameters of R's blocks (in)
 *   theta_P  float32 [d_in/b,  b(b-1)/2]   packed skew parameters of P's blocks (in)
 *   Q_R      dtype   [d_out/b, b, b]       Q_i = (I + S_i) Σ_{j<=k} S_i^j, row-major (out)
 *   Q_P      dtype   [d_in/b,  b, b]       (out)
 * For BF16 and b <= 256 the whole computation stays on chip (one launch for both sides, no
 * workspace is touched); F32 and b = 512 go through the library's GEMM kernels and use the
 * workspace.
 * Errors: INVALID_ARG, UNSUPPORTED_SHAPE, ALIGNMENT, WORKSPACE, CUDA. */
poetx_status poetx_cnp(const poetx_desc* desc, const float* theta_R, const float* theta_P,
                       void* Q_R, void* Q_P, void* workspace, size_t ws_bytes, poetx_stream stream);

/* CNP forward over a flat batch of n_blocks blocks that share b and k (e.g. every block of
 * every layer of a model in one launch).  Uses desc->b, desc->k, desc->dtype only.
 *   theta float32 [n_blocks, b(b-1)/2] (in); Q dtype [n_blocks, b, b] (out).
 * Workspace: poetx_cnp_blocks_workspace_size(desc, n_blocks) bytes. */
size_t poetx_cnp_blocks_workspace_size(const poetx_desc* desc, int n_blocks);
poetx_status poetx_cnp_blocks(const poetx_desc* desc, int n_blocks, const float* theta, void* Q,
                              void* workspace, size_t ws_bytes, poetx_stream stream);

/* Allocation-free variant of poetx_cnp_blocks.  The paper has no counterpart: this entry point
 * exists for callers that cannot supply device scratch, such as a plugin inside a host
 * framework that owns all device memory and offers it no allocator, or a latency-critical loop
 * that must not call cudaMalloc.  Its scratch is a fixed array of POETX_NOALLOC_SCRATCH_BYTES
 * (32 MiB) compiled into the library; every GPU that loads the library holds it until the
 * process exits.  The call itself allocates nothing.
 *   theta float32 [n_blocks, b(b-1)/2] (in); Q dtype [n_blocks, b, b] (out), caller-owned.
 * Limit: poetx_cnp_blocks_workspace_size(desc, n_blocks) must not exceed 32 MiB (e.g. bf16,
 * k = 3: at most 85 blocks of b = 256, 341 of b = 128, 9 of b = 512); larger requests return
 * POETX_ERR_WORKSPACE and launch nothing.
 * The first call on a device looks up the array's device address (cudaGetSymbolAddress) with
 * that device current; make that first call before any stream capture.  All calls on a device
 * share the one array: calls that may run at the same time on the GPU (unordered streams)
 * race on it and must be serialised by the caller.  No part of the array needs clearing: each
 * call writes all the scratch it reads. */
#define POETX_NOALLOC_SCRATCH_BYTES ((size_t)32 << 20)
poetx_status poetx_cnp_blocks_noalloc(const poetx_desc* desc, int n_blocks, const float* theta,
                                      void* Q, poetx_stream stream);

/* Absorb two of the four permutations into the base weight in advance (replication review,
 * "Summary": permutation reduction): W0'[i][j] = W0[perm_L[i]][perm_R[j]].
 *   W0 dtype [d_out, d_in] (in); perm_L int32 [d_out], perm_R int32 [d_in] bijections (in);
 *   W0p dtype [d_out, d_in] (out; must not alias W0). */
poetx_status poetx_absorb(const poetx_desc* desc, const void* W0, const int32_t* perm_L,
                          const int32_t* perm_R, void* W0p, poetx_stream stream);

/* Forward pass, input-centric (replication review, "Summary"):
 *   U = X[:, π_R] (gather), V_i = U_i · Q_P,i^T (batched per block), Z = V · W0'^T,
 *   Y'_i = Z_i · Q_R,i^T, Y[:, π_L] = Y' (scatter).
 *   X       dtype [N, d_in]  (in)          W0p dtype [d_out, d_in] (in)
 *   perm_L  int32 [d_out], perm_R int32 [d_in] (in)
 *   Q_R     dtype [d_out/b, b, b], Q_P dtype [d_in/b, b, b] (in, from poetx_cnp)
 *   Y       dtype [N, d_out] (out)
 *   saved   dtype [N*(d_out + d_in)] (out) in POETX_FAST mode: Z = V . W0'^T [N, d_out]
 *           followed by U = X[:, π_R] [N, d_in]; pass it back to poetx_backward.  Must be
 *           NULL in POETX_MEM mode (nothing is kept; the backward pass recomputes both).
 * n_tokens == 0 is valid and launches nothing. */
poetx_status poetx_forward(const poetx_desc* desc, int n_tokens, const void* X, const void* W0p,
                           const int32_t* perm_L, const int32_t* perm_R, const void* Q_R,
                           const void* Q_P, void* Y, void* saved, void* workspace,
                           size_t ws_bytes, poetx_stream stream);

/* poetx_cnp followed by poetx_forward in one call, with the same arguments and results (theta
 * in, Q_R and Q_P out, then the forward pass with those Q).  The CNP of both sides may run on a
 * library-owned side stream of the current device beside the input gather of the forward pass,
 * which does not need Q; everything is complete when `stream` reaches the end of the call (also
 * under stream capture).  Workspace: poetx_workspace_size(desc, n_tokens) bytes.  Errors as for
 * the two calls. */
poetx_status poetx_cnp_forward(const poetx_desc* desc, int n_tokens, const void* X, const void* W0p,
                               const int32_t* perm_L, const int32_t* perm_R, const float* theta_R,
                               const float* theta_P, void* Q_R, void* Q_P, void* Y, void* saved,
                               void* workspace, size_t ws_bytes, poetx_stream stream);

/* Backward pass: dX and the gradients w.r.t. the PACKED skew parameters (only the packed form
 * is written; replication review, "Summary": compact skew storage; W0 is frozen, so there is
 * no dW0).  In POETX_MEM mode `saved` must be NULL and U, V, Z are recomputed from X.
 *   dY dtype [N, d_out], X dtype [N, d_in], W0p, perm_L, perm_R, Q_R, Q_P as in forward (in)
 *   theta_R, theta_P float32 packed (in; the CNP adjoint needs S)
 *   saved   dtype [N*(d_out + d_in)] (in, FAST: as written by poetx_forward) or NULL (MEM)
 *   dX dtype [N, d_in] (out); grad_theta_R float32 [d_out/b, b(b-1)/2] (out);
 *   grad_theta_P float32 [d_in/b, b(b-1)/2] (out).
 * The call may order part of its work on a library-owned side stream of the current device;
 * everything it launches is complete when `stream` reaches the end of the call (also under
 * stream capture).  Concurrent calls from several host threads on one device are serialised
 * while they enqueue.
 * n_tokens == 0 writes zero gradients. */
poetx_status poetx_backward(const poetx_desc* desc, int n_tokens, const void* dY, const void* X,
                            const void* W0p, const int32_t* perm_L, const int32_t* perm_R,
                            const void* Q_R, const void* Q_P, const float* theta_R,
                            const float* theta_P, const void* saved, void* dX, float* grad_theta_R, float* grad_theta_P, void* workspace,
                            size_t ws_bytes, poetx_stream stream);

/* Merge-then-reinitialise (agidaily.cc article: transforms are merged into the weight and
 * re-initialised during training; replication review, "Reproducibility & code":
 * merge_then_reinitialize).  Folds R and P into the weight and absorbs fresh permutations:
 *   M = BD_R · W0' · BD_P;  W0'_new[i][j] = M[π_L^-1(π_L,new(i))][π_R^-1(π_R,new(j))];
 *   theta_R = theta_P = 0.
 *   W0p dtype [d_out, d_in] (in/out); Q_R, Q_P (in, the Q the forward used);
 *   perm_*_old, perm_*_new int32 bijections (in); theta_R, theta_P float32 (out, zeroed). */
poetx_status poetx_merge(const poetx_desc* desc, void* W0p, const void* Q_R, const void* Q_P,
                         const int32_t* perm_L_old, const int32_t* perm_R_old,
                         const int32_t* perm_L_new, const int32_t* perm_R_new, float* theta_R,
                         float* theta_P, void* workspace, size_t ws_bytes, poetx_stream stream);

/* ------------------------------------------------------------------------------- POET-XQ
 * The quantised variant (replication review, "Summary": POET-XQ is possible because POET-Xmem
 * never keeps a high-precision weight resident; "Strengths": it runs through POET-Xmem, whose
 * recompute means the dequantised W is never stored, and it is set against 8-bit baselines;
 * agidaily.cc article, the section on how POET-X differs from existing methods: POET-X has a
 * quantised version).  The pages give no format; this library's reading is 8-bit symmetric
 * with one scale per row of W0':
 *   s_o = max_i |W0'[o, i]| / 127,  q[o, i] = round(W0'[o, i] / s_o) (nearest, ties to even,
 *   clipped to [-127, 127]; a zero row has s_o = 0, q = 0), both in float32 with IEEE division;
 *   the layer uses W0'[o, i] = s_o * q[o, i].
 *   W0q int8 [d_out, d_in], W0s float32 [d_out] (caller-owned device memory, 16-byte aligned).
 * Only POETX_MEM mode and POETX_BF16 (INVALID_ARG otherwise), d_in and d_out multiples of 256
 * (UNSUPPORTED_SHAPE otherwise).  The W0' GEMMs of forward and backward read the codes and
 * dequantise each tile in shared memory; no bf16 W0' exists at any time.  Workspace:
 * poetx_workspace_size(desc, n_tokens) covers every call below.  Other arguments and errors
 * as for the bf16 calls above (poetx_xq_backward: no `saved`).
 *
 * poetx_xq_quantize:   W0p bf16 [d_out, d_in] (in) -> W0q, W0s (out).
 * poetx_xq_dequantize: W0q, W0s (in) -> W0p bf16 (out) = bf16(s_o * q) (for inspection).
 * poetx_xq_merge:      the merge of poetx_merge on W0' = s * q, then the new W0' quantised
 *                      again into W0q, W0s (in/out); the bf16 weight lives only in the workspace
 *                      during the call; theta_R, theta_P zeroed. */
poetx_status poetx_xq_quantize(const poetx_desc* desc, const void* W0p, int8_t* W0q, float* W0s,
                               poetx_stream stream);
poetx_status poetx_xq_dequantize(const poetx_desc* desc, const int8_t* W0q, const float* W0s,
                                 void* W0p, poetx_stream stream);
poetx_status poetx_xq_forward(const poetx_desc* desc, int n_tokens, const void* X,
                              const int8_t* W0q, const float* W0s, const int32_t* perm_L,
                              const int32_t* perm_R, const void* Q_R, const void* Q_P, void* Y,
                              void* workspace, size_t ws_bytes, poetx_stream stream);
poetx_status poetx_xq_backward(const poetx_desc* desc, int n_tokens, const void* dY, const void* X,
                               const int8_t* W0q, const float* W0s, const int32_t* perm_L,
                               const int32_t* perm_R, const void* Q_R, const void* Q_P,
                               const float* theta_R, const float* theta_P, void* dX,
                               float* grad_theta_R, float* grad_theta_P, void* workspace,
                               size_t ws_bytes, poetx_stream stream);
poetx_status poetx_xq_merge(const poetx_desc* desc, int8_t* W0q, float* W0s, const void* Q_R,
                            const void* Q_P, const int32_t* perm_L_old, const int32_t* perm_R_old,
                            const int32_t* perm_L_new, const int32_t* perm_R_new, float* theta_R,
                            float* theta_P, void* workspace, size_t ws_bytes, poetx_stream stream);

/* ------------------------------------------------------ weight-centric comparator (not the path)
 * The original POET order of evaluation, for comparison with the input-centric path above
 * (replication review, "Summary": POET-X's speed-ups are measured against forming the
 * transformed weight; agidaily.cc article: the transformed weight W_RP = R.W0.P).  The same
 * layer arithmetic is done weight-first: T = W0'.BD_P, M = BD_R.T, W = Pi_L^T M Pi_R (the layer
 * weight in the original basis), Y = X.W^T; backward dX = dY.W, dW = dY^T.X, dM = Pi_L dW Pi_R^T,
 * dL/dQ_R,i = dM[blk i,:].T[blk i,:]^T, dL/dQ_P,j = (BD_R.W0')[:,blk j]^T.dM[:,blk j], then the
 * same CNP adjoint as poetx_backward.  Q_R, Q_P come from poetx_cnp.
 *   wc_saved  dtype, poetx_wc_saved_size(desc) bytes: W [d_out, d_in] then T (256-byte aligned)
 *             (out of poetx_wc_forward, in to poetx_wc_backward)
 *   workspace poetx_wc_workspace_size(desc) bytes.
 * poetx_wc_forward with n_tokens == 0 only forms W and T.  Errors as for poetx_forward. */
size_t poetx_wc_saved_size(const poetx_desc* desc);
size_t poetx_wc_workspace_size(const poetx_desc* desc);
poetx_status poetx_wc_forward(const poetx_desc* desc, int n_tokens, const void* X, const void* W0p,
                              const int32_t* perm_L, const int32_t* perm_R, const void* Q_R,
                              const void* Q_P, void* Y, void* wc_saved, void* workspace,
                              size_t ws_bytes, poetx_stream stream);
poetx_status poetx_wc_backward(const poetx_desc* desc, int n_tokens, const void* dY, const void* X,
                               const void* W0p, const int32_t* perm_L, const int32_t* perm_R,
                               const void* Q_R, const float* theta_R, const float* theta_P,
                               const void* wc_saved, void* dX, float* grad_theta_R,
                               float* grad_theta_P, void* workspace, size_t ws_bytes,
                               poetx_stream stream);

/* ----------------------------------------------------- four-permutation comparator (not the path)
 * The same layer with none of the four permutations absorbed (replication review,
 * "Reproducibility & code": the paper's Table 2 compares the 4-permute path with the 2-permute
 * one; "Summary": absorbing two permutations into W is one of POET-X's reductions).  R and P act
 * around the ORIGINAL base weight W0 [d_out, d_in] (not W0'), so each pass permutes the
 * activations four times:
 *   forward:  U = X[:, pi_R], V_i = U_i Q_P,i^T, V scattered back to the original basis by pi_R,
 *             Z = V W0^T, Z' = Z[:, pi_L], Y'_i = Z'_i Q_R,i^T, Y[:, pi_L] = Y'
 *   backward: the adjoints in reverse (four permutations), then the same CNP adjoint.
 * Results equal poetx_forward / poetx_backward on W0' = Pi_L W0 Pi_R^T up to rounding.
 *   saved  dtype [N*(d_out + d_in)]: Z' then U, written by the forward, read by the backward.
 * Workspace: poetx_fourperm_workspace_size(desc, n_tokens) bytes.  Errors as for poetx_forward. */
size_t poetx_fourperm_workspace_size(const poetx_desc* desc, int n_tokens);
poetx_status poetx_fourperm_forward(const poetx_desc* desc, int n_tokens, const void* X, const void* W0,
                                    const int32_t* perm_L, const int32_t* perm_R, const void* Q_R,
                                    const void* Q_P, void* Y, void* saved, void* workspace,
                                    size_t ws_bytes, poetx_stream stream);
poetx_status poetx_fourperm_backward(const poetx_desc* desc, int n_tokens, const void* dY, const void* W0,
                                     const int32_t* perm_L, const int32_t* perm_R, const void* Q_R,
                                     const void* Q_P, const float* theta_R, const float* theta_P,
                                     const void* saved, void* dX, float* grad_theta_R,
                                     float* grad_theta_P, void* workspace, size_t ws_bytes,
                                     poetx_stream stream);

/* ------------------------------------------------------------------ optimiser (packed theta)
 * AdamW on the packed skew parameters, so that the optimiser state stays at the packed size
 * (agidaily.cc article, compact storage: gradients and optimiser state shrink with the
 * parameters; replication review, "Weaknesses": the POET learning-rate scale gamma = 0.5 and
 * the reset gap of 400 steps).  The pages do not give AdamW's own constants; they are
 * arguments.  With step t >= 1 and eta = gamma * lr, elementwise:
 *   m <- beta1 m + (1 - beta1) g;   v <- beta2 v + (1 - beta2) g^2;
 *   theta <- theta - eta * (weight_decay * theta + (m / (1 - beta1^t)) / (sqrt(v / (1 - beta2^t)) + eps)).
 * The paper has no separate routine for it: this is the decoupled-weight-decay Adam of
 * Loshchilov and Hutter applied to theta. */
typedef struct {
  float lr;            /* base learning rate (>= 0)                         */
  float gamma;         /* POET learning-rate scale (the pages use 0.5)       */
  float beta1, beta2;  /* moment decay rates, each in [0, 1)                 */
  float eps;           /* > 0                                                */
  float weight_decay;  /* decoupled decay coefficient (>= 0)                 */
} poetx_adamw_cfg;

/* One AdamW step over n packed parameters (e.g. theta_R and theta_P stored back to back).
 *   theta, m, v float32 [n] (in/out); grad float32 [n] (in); t = step count of the moments (>= 1).
 * All pointers 16-byte aligned, caller-owned device memory.  n == 0 launches nothing.
 * Errors: INVALID_ARG (bad cfg, t < 1, n < 0, NULL pointer), ALIGNMENT, CUDA. */
poetx_status poetx_adamw_step(const poetx_adamw_cfg* cfg, long long n, int t, float* theta,
                              const float* grad, float* m, float* v, poetx_stream stream);

/* Zeroes the moments (m, v float32 [n]) after a merge re-initialises theta: the merge schedule
 * restarts the moments with the parameters (their step count t starts again at 1). */
poetx_status poetx_adamw_reset(long long n, float* m, float* v, poetx_stream stream);

/* Host check of a permutation (HOST memory): POETX_OK if perm holds every value of [0, n)
 * exactly once, else POETX_ERR_INVALID_ARG.  The layer calls assume bijections and do not check
 * them; with the environment variable POETX_DEBUG set (and not "0") when the library first looks
 * at it, poetx_absorb, poetx_forward, poetx_backward and poetx_merge copy their permutations to
 * the host in stream order and return POETX_ERR_INVALID_ARG, launching nothing, when one is not
 * a bijection (skipped while the stream is being captured). */
poetx_status poetx_check_permutation(const int32_t* perm, int n);

/* Human-readable name of a status code (static storage). */
const char* poetx_status_string(poetx_status s);

/* Synchronises the current device, then returns and clears the device-side error word:
 * POETX_OK, or POETX_ERR_DEVICE_TIMEOUT if a kernel gave up on a bounded wait since the last
 * call.  *detail (if not NULL) receives the raw word (kernel id and wait site). */
poetx_status poetx_device_status(int* detail);

/* ---------------------------------------------------------------------------- measurement
 * Launch accounting for benchmarks and profilers (not part of the layer's arithmetic). */

/* Kernel classes of the library's launches. */
typedef enum {
  POETX_KC_W_GEMM = 0,       /* Z = V W0'^T (tensor cores; with BD_R fused for b = 256)     */
  POETX_KC_BD_GEMM = 1,      /* block-diagonal products BD_P, BD_R and their adjoints       */
  POETX_KC_GRAD_GEMM = 2,    /* per-block gradient products G = dY'^T Z, dV^T U (split-K)   */
  POETX_KC_CNP_GEMM = 3,     /* CNP forward (the on-chip kernel, or its products for F32 / b = 512) */
  POETX_KC_MERGE_GEMM = 4,   /* BD_R W0' BD_P of the merge                                  */
  POETX_KC_PERMUTE = 5,      /* feature-dimension gather / scatter                          */
  POETX_KC_ELEMENTWISE = 6,  /* unpack, pack, split-K reduction, permutation inverse        */
  POETX_KC_TEST_GEMM = 7,    /* poetx_test_gemm                                              */
  POETX_KC_OPTIMIZER = 8,    /* poetx_adamw_step                                             */
  POETX_KC_W_GEMM_ADJ = 9,   /* dV = dZ W0' (with the BD_P adjoint fused for b = 256)        */
  POETX_KC_CNP_ADJ = 10,     /* CNP adjoint to the packed gradients (on-chip, or its products) */
  POETX_KC_COUNT = 11
} poetx_kernel_class;

/* Number of kernels this library has launched in the process so far. */
unsigned long long poetx_launch_count(void);

/* on != 0: forget earlier records and bracket every following launch with a CUDA event pair
 * on its stream (host-side bookkeeping only; events are created on first use and reused).
 * on == 0: stop recording. */
poetx_status poetx_profile_enable(int on);

/* Waits for the recorded events and writes, per kernel class, the number of recorded launches
 * (counts[POETX_KC_COUNT]) and their summed device time in ms (total_ms[POETX_KC_COUNT]). */
poetx_status poetx_profile_summary(int* counts, float* total_ms);

#ifdef __cplusplus
}
#endif
#endif /* POETX_H_ */
