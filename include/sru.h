/*
 * sru.h -- C ABI of the B200 (sm_100a) Simple Recurrent Unit layer library (libsru.so).
 *
 * The layer is the SRU cell of "When Attention Meets Fast Recurrence: Training
 * Language Models with Reduced Compute" (T. Lei), background section on SRU:
 *
 *   Eq. (1)      U^T = [W; W'; W''] X^T        one product over all L time steps
 *   Eqs. (2)-(5) f[t] = sigma(U[t,f] + v_f * c[t-1] + b_f)
 *                r[t] = sigma(U[t,r] + v_r * c[t-1] + b_r)
 *                c[t] = f[t] * c[t-1] + (1 - f[t]) * U[t,c]
 *                h[t] = r[t] * c[t] + (1 - r[t]) * alpha * x[t]
 *
 * computed independently for every hidden channel j and batch row b.  The
 * backward pass (not printed on the page) is the reverse-mode derivative of
 * those equations, walked in reverse time.
 *
 * Conventions shared by every call
 * --------------------------------
 * Layouts are time-major and row-major (last index fastest):
 *   X, x     (L, B, d)              layer input; X in the projection's type, x fp32
 *   W_cat    (n_dir * 3 * d, d)     rows [dir][gate][j]; gate 0 = candidate (W),
 *                                    1 = forget (W_f), 2 = reset (W_r)
 *   U        (L, B, n_dir, 3, d)    = (M, N) with M = L*B, N = n_dir*3*d
 *   h, dh    (L, B, n_dir, d)       fp32
 *   v, b     (n_dir, 2, d)          fp32; row 0 = forget gate, row 1 = reset gate
 *   c0, c_T  (B, n_dir, d)          fp32
 *   mask     (L, B) uint8           1 = padded position (nullable = no padding)
 * n_dir = 2 when `bidirectional`: direction 1 walks t = L-1 ... 0 with its own
 * gate block of U, v, b and c0; both directions read the same x.
 * A padded position leaves the state unchanged, writes h = 0, and gets zero
 * gradient (dU = 0, no dx contribution); the state gradient passes through it.
 *
 * Pointers: every data pointer is a DEVICE pointer owned by the caller, at
 * least 16-byte aligned, to densely packed memory of the stated layout (the
 * calls check 16 bytes for the (L, B, ...) tensors and at least 8 bytes for the
 * per-channel vectors v, b, c0, c_T and their gradients; SRU_ERR_INVALID).
 * The library allocates no device memory.  `stream` is a cudaStream_t (NULL =
 * legacy default stream); calls are stream-ordered and asynchronous (none
 * synchronises).  Size limits: d % 8 == 0, 1 <= d, 0 <= L, 0 <= B, L*B < 2^31.
 *
 * Errors: every call returns an sru_status.  Invalid arguments are rejected
 * before anything is launched (SRU_ERR_INVALID / SRU_ERR_UNSUPPORTED).  A
 * failed launch returns SRU_ERR_CUDA (see sru_get_last_cuda_error).  Every
 * wait inside a kernel is bounded (2 s); if one expires the kernel records a
 * code in a device error word and returns early, and the next
 * sru_sync_status() on that device returns SRU_ERR_TIMEOUT.  Nothing aborts,
 * traps or exits.
 */
#ifndef SRU_B200_H
#define SRU_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    SRU_OK = 0,
    SRU_ERR_INVALID = 1,      /* bad pointer, size, alignment or dtype */
    SRU_ERR_CUDA = 2,         /* a CUDA runtime/driver call failed */
    SRU_ERR_TIMEOUT = 3,      /* a bounded device-side wait expired */
    SRU_ERR_UNSUPPORTED = 4   /* valid request outside the library's limits */
} sru_status;

typedef enum { SRU_F32 = 0, SRU_BF16 = 1 } sru_dtype;

/* Caller asserts v == 0 (all entries): the state recurrence is then linear in c
 * and sru_forward may run as a chunked associative scan over t.  (sru_backward
 * may use its chunked scan for any v: the state-gradient recurrence is affine.)
 * The library picks a scan when the sequential kernels would leave SMs idle
 * (fewer than two 64-channel CTAs per SM) and the scan's waves of resident
 * CTAs cost less than the sequence's 16-step chunks (measured on B200: a wave
 * costs about 8 chunks forward, 5 backward). */
#define SRU_FLAG_V_ZERO 0x1u
/* Force the scan paths (the forward scan only with SRU_FLAG_V_ZERO) / force the
 * sequential paths. */
#define SRU_FLAG_FORCE_SCAN 0x2u
#define SRU_FLAG_FORCE_SEQUENTIAL 0x4u
/* Fault injection, for tests of the failure path only: on a chunked-scan
 * launch the first work item publishes no carry, so the bounded waits of the
 * CTAs that look back to it expire (after about 2 s).  They publish an abort
 * that releases their successors, and return; the call's outputs are then
 * undefined and the next sru_sync_status() returns SRU_ERR_TIMEOUT.  No fault,
 * trap or hang is involved, and the context stays usable.  Has no effect on
 * the sequential kernels. */
#define SRU_FLAG_TEST_WITHHOLD_CARRY 0x8u

/* Human-readable name of a status code (static string). */
const char* sru_status_string(int status);

/* The cudaError_t of the most recent SRU_ERR_CUDA on the calling thread (0 if none). */
int sru_get_last_cuda_error(void);

/* Library ABI version (major * 100 + minor). */
int sru_version(void);

/*
 * Bytes of caller-provided device workspace that sru_forward and sru_backward
 * need for a layer of these sizes and flags on the current device (the choice
 * of scan paths depends on its SM count).  The workspace carries state
 * checkpoints from sru_forward to sru_backward (pass the same buffer to both)
 * and holds the backward's partial sums and the scans' flags and carries.
 * Returns 0 on bad sizes.
 */
size_t sru_workspace_bytes(int64_t L, int64_t B, int64_t d, int bidirectional, unsigned flags);

/*
 * Eq. (1): U[M, N] = X[M, K] * W[N, K]^T, fp32 accumulation.
 *   M = L*B tokens, K = d, N = n_dir*3*d.  Supported type triples (x_t, w_t, u_t):
 *   (BF16, BF16, BF16) and (BF16, BF16, F32) on the tcgen05 tensor cores;
 *   (F32, F32, F32) on a CUDA-core kernel.  Requires K % 8 == 0, N % 8 == 0.
 */
sru_status sru_project(const void* X, int x_t, const void* W, int w_t, void* U, int u_t,
                       int64_t M, int64_t N, int64_t K, void* stream);

/*
 * Gradients of Eq. (1), fp32 accumulation, fp32 outputs:
 *   dX[M, K] = dU[M, N] * W[N, K]      (accumulate != 0: dX += ..., e.g. onto the
 *                                       highway part returned by sru_backward)
 *   dW[N, K] = dU[M, N]^T * X[M, K]
 * dU, X and W share one type t (BF16 on the tensor cores, F32 on CUDA cores).
 * Either output may be NULL to skip it.  Requires K % 8 == 0, N % 8 == 0.
 */
sru_status sru_project_backward(const void* dU, const void* X, const void* W, int t,
                                float* dX, int accumulate, float* dW,
                                int64_t M, int64_t N, int64_t K, void* stream);

/*
 * Eqs. (2)-(5) over all t for every (direction, batch row, channel).
 *   U (u_t = F32 or BF16), x, v, b as above; c0 nullable (zero state);
 *   mask nullable.  Outputs h (L, B, n_dir, d) and c_T (B, n_dir, d), fp32.
 *   workspace / workspace_bytes: a device buffer of at least
 *   sru_workspace_bytes(L, B, d, bidirectional, flags) bytes (checked:
 *   SRU_ERR_INVALID if smaller), or NULL for inference only (then no
 *   checkpoints are written, sru_backward cannot follow, and the scan path is
 *   not available).  flags: SRU_FLAG_* above.  With SRU_FLAG_V_ZERO the
 *   library runs the chunked scan where it pays (see SRU_FLAG_V_ZERO), or
 *   when forced.
 */
sru_status sru_forward(const void* U, int u_t, const float* x, const float* v, const float* b,
                       const float* c0, const uint8_t* mask, int64_t L, int64_t B, int64_t d,
                       float alpha, int bidirectional, unsigned flags,
                       float* h, float* c_T, void* workspace, size_t workspace_bytes, void* stream);

/*
 * Backward of sru_forward for Loss = sum(dh * h) + sum(dc_T * c_T).
 * Inputs: the forward's U, x, v, b, c0, mask, sizes, alpha, flags and the
 *   workspace the forward filled (same buffer and size); dh (L, B, n_dir, d);
 *   dc_T nullable (zero).  c0 is not read: the checkpoints carry it.
 * Outputs (overwritten):
 *   dU (L, B, n_dir, 3, d) of type du_t (F32 or BF16),
 *   dx (L, B, d) fp32: the highway part alpha * (1 - r) * dh, summed over directions
 *      (add the projection part with sru_project_backward(..., accumulate = 1)),
 *   dv, db (n_dir, 2, d) fp32 summed over t and b (deterministic order),
 *   dc0 (B, n_dir, d) fp32.
 */
sru_status sru_backward(const void* U, int u_t, const float* x, const float* v, const float* b,
                        const float* c0, const uint8_t* mask, int64_t L, int64_t B, int64_t d,
                        float alpha, int bidirectional, unsigned flags,
                        const float* dh, const float* dc_T, void* workspace, size_t workspace_bytes,
                        void* dU, int du_t, float* dx, float* dv, float* db, float* dc0,
                        void* stream);

/*
 * Allocation-free forward for the linear case v = 0 (the paper has no
 * counterpart to this entry point; it is a deployment variant of sru_forward).
 *
 * Some callers cannot allocate device memory: an inference plugin whose host
 * framework owns every device buffer and hands the op no scratch, or a
 * latency-critical loop that must not call cudaMalloc (which can block and
 * synchronise the device).  This call computes what
 *   sru_forward(U, u_t, x, v = 0, b, c0, mask, L, B, d, alpha, bidirectional,
 *               SRU_FLAG_V_ZERO | SRU_FLAG_FORCE_SCAN, h, c_T, NULL workspace)
 * would (the chunked scan over t, inference only: no checkpoints, so no
 * sru_backward can follow) without any workspace argument: its scan flags,
 * ticket and per-chunk aggregates live in an 8 MiB static device array inside
 * libsru.so, which every GPU that loads the library holds until the process
 * exits.  The caller still passes all inputs and outputs (same layouts and
 * rules as sru_forward; v is not read and is taken as 0).
 *
 * Limit: ceil(L/128) * ceil(d/64) * B * n_dir work items, each needing 772
 * bytes of the scratch (about 10 800 items); a larger request returns
 * SRU_ERR_UNSUPPORTED before anything is launched.
 * The call allocates nothing (no cudaMalloc, cudaFree or allocating library
 * call).  Its first call on a device looks up the array's device address
 * (cudaGetSymbolAddress, once per device, with that device current); make
 * that first call before any stream capture: a first call on a device whose
 * stream is capturing is refused with SRU_ERR_INVALID, before anything is
 * launched.  Every call zeroes the flags it
 * uses before launching and otherwise reuses whatever the previous call left
 * in the array, so calls that overlap on the GPU (concurrent streams, or
 * several host threads on the same device) race on the shared scratch and
 * must be serialised by the caller.
 */
sru_status sru_forward_scan_noalloc(const void* U, int u_t, const float* x, const float* b,
                                    const float* c0, const uint8_t* mask, int64_t L, int64_t B, int64_t d,
                                    float alpha, int bidirectional, float* h, float* c_T, void* stream);

/*
 * Eq. (1) and Eqs. (2)-(5) in one kernel (the page's Figure 2(a): the grouped
 * matrix multiplication and the element-wise recurrence, fused): computes what
 *   sru_project(X, BF16, W, BF16, U, BF16, L*B, n_dir*3*d, d) followed by
 *   sru_forward(U, BF16, x, v, b, c0, mask, L, B, d, alpha, bidirectional, 0,
 *               h, c_T, workspace)
 * computes, without reading U back from memory: each 32-step x 4-row x
 * 64-channel tile of the product is rounded to bf16 (as U is stored on the
 * two-call path) and the recurrence runs on it from shared memory.
 *   X (L*B, d) bf16 time-major, W (n_dir*3*d, d) bf16 (W_cat, gate blocks as
 *   above), x, v, b, c0, mask, h, c_T as for sru_forward.
 *   U nullable: when given ((L, B, n_dir, 3, d) bf16), the projection is also
 *   stored there and the state checkpoints are written to the workspace, so
 *   that sru_backward (flags 0, same workspace) can follow; when NULL, nothing
 *   of U is stored (inference).
 *   workspace: at least sru_workspace_bytes(L, B, d, bidirectional, flags) bytes
 *   for any flags (it also carries the state from one time tile to the next;
 *   that region is cleared on the stream before the launch).
 * The kernel keeps one CTA on every SM of the device and hands the state of a
 * sequence between CTAs: do not run it concurrently with other work on the
 * same GPU (its bounded waits would expire: SRU_ERR_TIMEOUT at the next
 * sru_sync_status).  Limits as for sru_forward (d % 8 == 0).
 */
sru_status sru_forward_fused(const void* X, const void* W, const float* x, const float* v, const float* b,
                             const float* c0, const uint8_t* mask, int64_t L, int64_t B, int64_t d, float alpha,
                             int bidirectional, float* h, float* c_T, void* U, void* workspace,
                             size_t workspace_bytes, void* stream);

/*
 * Factorised projection: the page's variant of Eq. (1) with a low-rank
 * projection (Figure 2, the SRU layer "with projection trick"):
 *   P = X Wq^T        (M, Kp)  Wq (Kp, K): projects d down to d' = Kp
 *   U = P Wo^T        (M, N)   Wo (N, Kp): back up to the n_dir * 3d gate columns
 * X, Wq, Wo bf16; P is a caller-provided bf16 buffer that receives the
 * intermediate (kept for the backward); U of type u_t (BF16 or F32).  Two
 * chained tensor-core products with fp32 accumulation; P is rounded to bf16
 * in between.  K, Kp and N must be multiples of 8 (SRU_ERR_UNSUPPORTED).
 */
sru_status sru_project_factored(const void* X, const void* Wq, const void* Wo, void* P, void* U, int u_t,
                                int64_t M, int64_t N, int64_t K, int64_t Kp, void* stream);

/*
 * Gradients of sru_project_factored for a bf16 dU (M, N):
 *   dWo = dU^T P (N, Kp) fp32;   dP = dU Wo (M, Kp) written to the caller's bf16 buffer dP;
 *   dWq = dP^T X (Kp, K) fp32;   dX = dP Wq (M, K) fp32, added onto dX when accumulate != 0.
 * P is the intermediate the forward wrote.  Any of dX, dWq, dWo may be NULL
 * (not computed); dP is always written.
 * workspace / workspace_bytes (nullable; 16-byte aligned): with at least
 * sru_project_factored_backward_workspace_bytes(M, N, K, Kp) bytes, a weight
 * gradient whose output tiles cannot fill the GPU (dWq and dWo of a narrow d')
 * is cut along its reduction over the M tokens, each part written to its own
 * slab of the workspace and the slabs summed in a fixed order (the same bits
 * every run); without one it runs as a single product.
 */
size_t sru_project_factored_backward_workspace_bytes(int64_t M, int64_t N, int64_t K, int64_t Kp);
sru_status sru_project_factored_backward(const void* dU, const void* X, const void* Wq, const void* Wo,
                                         const void* P, void* dP, float* dX, int accumulate, float* dWq,
                                         float* dWo, int64_t M, int64_t N, int64_t K, int64_t Kp, void* workspace,
                                         size_t workspace_bytes, void* stream);

/*
 * SRU++'s producer of U: single-head attention in place of the linear map of
 * Eq. (1) (the page's SRU++ section).  With d' the attention width:
 *   Q = X Wq^T                  (L*B, d')   Wq  (d', d)
 *   [K | V] = Q Wkv^T           (L*B, 2d')  Wkv (2d', d') = [Wk; Wv]
 *   per batch row b, over its L tokens (rows t*B + b):
 *     A_b = softmax(Q_b K_b^T / sqrt(d')) V_b, token t seeing tokens <= t when causal
 *   R = Q + alpha A, or layernorm(Q + alpha A) * gamma + beta over the d' features
 *       (eps 1e-5) when ln_gamma and ln_beta are given (both or neither)
 *   U = R Wo^T                  (L*B, N)    Wo  (N, d'), U of type u_t (BF16 or F32)
 * X, Wq, Wkv, Wo bf16; X and U time-major as everywhere; ln_gamma and ln_beta
 * (d',) fp32, 16-byte aligned like every other pointer.  Q, [K | V], P and R
 * are rounded to bf16 (they are tensor-core operands), scores and A are fp32.
 * The workspace (>= sru_attention_workspace_bytes(L, B, d')) holds Q, K, V,
 * one batch row's scores and probabilities, A and R.  Limits: d, d', N and L
 * multiples of 8, L <= 65536.  With causal, the score tiles wholly above the
 * diagonal and P V's reduction beyond each row tile's diagonal are skipped
 * (those probabilities are 0).
 */
size_t sru_attention_workspace_bytes(int64_t L, int64_t B, int64_t dp);
sru_status sru_attention_project(const void* X, const void* Wq, const void* Wkv, const void* Wo, float alpha,
                                 const float* ln_gamma, const float* ln_beta, int causal, void* U, int u_t,
                                 int64_t L, int64_t B, int64_t d, int64_t dp, int64_t N, void* workspace,
                                 size_t workspace_bytes, void* stream);

/*
 * Backward of sru_attention_project for Loss = sum(dU * U) (the reverse-mode
 * derivative of the SRU++ producer above; the page trains it end to end):
 *   dWo = dU^T R,  dR = dU Wo
 *   dZ from dR through the layer norm (or dZ = dR), Z = Q + alpha A;
 *   dgamma = sum over tokens of dR * Zhat, dbeta = sum of dR (with the norm)
 *   dQ = dZ;  dA = alpha dZ
 *   per batch row: dP = dA V^T, dS = P * (dP - rowsum(P * dP)) / sqrt(d'),
 *     dV = P^T dA, dK = dS^T Q, dQ += dS K
 *   dQ += [dK | dV] Wkv;  dWkv = [dK | dV]^T Q
 *   dWq = dQ^T X;  dX (+)= dQ Wq
 *   dU (L*B, N) bf16; X, Wq, Wkv, Wo, alpha, ln_gamma, ln_beta, causal and
 *   the sizes exactly as given to the forward call.
 *   fwd_workspace: the workspace of that forward call, unchanged since (its Q,
 *   [K | V], A and R are read; the probabilities are recomputed here one group
 *   of batch rows at a time).
 *   dX (L*B, d) fp32, written, or added onto when accumulate != 0 (so that the
 *   highway part from sru_backward can be summed in place).
 *   dWq (d', d), dWkv (2d', d'), dWo (N, d') fp32, written.
 *   dgamma, dbeta (d',) fp32, written when ln_gamma / ln_beta are given (both
 *   required then; ignored otherwise).  The sums over tokens are taken in a
 *   fixed order: the same bits on every run.
 *   workspace: >= sru_attention_backward_workspace_bytes(L, B, d, d', N) bytes,
 *   16-byte aligned (dQ, dA, the per-group probabilities and their gradients,
 *   [dK | dV], and the k slabs of the weight gradients: a weight gradient with
 *   fewer output tiles than the GPU has CTA pairs is cut along its reduction over
 *   the tokens, each part written to its own slab, and the slabs summed in a
 *   fixed order).  0 for unsupported sizes.
 * dA, dP's softmax gradient dS, [dK | dV] and dQ are rounded to bf16 where they
 * become tensor-core operands.  Limits as for the forward.  Null or misaligned
 * pointers and a short workspace: SRU_ERR_INVALID, before any launch.
 */
size_t sru_attention_backward_workspace_bytes(int64_t L, int64_t B, int64_t d, int64_t dp, int64_t N);
sru_status sru_attention_project_backward(const void* dU, const void* X, const void* Wq, const void* Wkv,
                                          const void* Wo, float alpha, const float* ln_gamma,
                                          const float* ln_beta, int causal, const void* fwd_workspace,
                                          size_t fwd_workspace_bytes, float* dX, int accumulate, float* dWq,
                                          float* dWkv, float* dWo, float* dgamma, float* dbeta, int64_t L,
                                          int64_t B, int64_t d, int64_t dp, int64_t N, void* workspace,
                                          size_t workspace_bytes, void* stream);

/*
 * One time step of a unidirectional layer for inference (token-by-token
 * decoding), with the projection fused in.  The page notes that SRU-based
 * models run as an RNN at inference time (one token per step); there the
 * product of Eq. (1) degenerates to a matrix-vector product per step, and
 * this call does that product and Eqs. (2)-(5) in one kernel:
 *   u[b, g, j] = sum_k X_t[b, k] * W_cat[g*d + j, k]     (fp32, never stored)
 *   c[b, j], h_t[b, j] <- Eqs. (2)-(5) from c[b, j], u, x_t[b, j], v, b, alpha
 * for b < B, j < d.  u is kept in fp32 (sru_project + sru_forward round U to
 * the U dtype in between; here no U exists).
 *   X_t  (B, d) bf16     projection input of this step
 *   W    (3*d, d) bf16   W_cat of one direction (gate blocks as above)
 *   x_t  (B, d) fp32     highway input of this step
 *   v, b (2, d) fp32     forget / reset peepholes and biases
 *   c    (B, d) fp32     state: read as c[t-1], overwritten with c[t]
 *   h_t  (B, d) fp32     output
 * Each W element is read once per call (the step streams 6*d*d bytes of W for
 * any B <= 16; larger B is processed 16 rows at a time).  Same pointer rules as
 * above; X_t, W, x_t, c and h_t must not overlap.  B = 0 is a no-op.
 * workspace / workspace_bytes (nullable): see sru_decode_workspace_bytes; with
 * one, batches of 8, 16, 24, ... rows take the tensor-core path.
 * Limits: d % 8 == 0, d <= 2^24, B <= 2^20, else SRU_ERR_UNSUPPORTED.
 */
sru_status sru_decode_step(const void* X_t, const void* W, const float* x_t, const float* v, const float* b,
                           float* c, float* h_t, int64_t B, int64_t d, float alpha, void* workspace,
                           size_t workspace_bytes, void* stream);
/* Bytes of workspace with which sru_decode_step runs a batched step's product
 * on the tensor cores (u = W_cat X_t^T as 3d x B fp32, then the cell update):
 * nonzero when B is a multiple of 8, at least 8.  With workspace NULL (or any
 * other B) the step runs the fused kernel above. */
size_t sru_decode_workspace_bytes(int64_t B, int64_t d);

/* Synchronise `stream`, then read and clear the device error word of the
 * current device: SRU_ERR_TIMEOUT if a bounded wait expired since the last
 * call, SRU_ERR_CUDA if the stream reported an error, else SRU_OK. */
sru_status sru_sync_status(void* stream);

#ifdef __cplusplus
}
#endif

#endif /* SRU_B200_H */
