/*
 * rope_attn.h - C ABI of librope_attn: exact RoPE softmax attention, its squared-error
 * loss and the closed-form gradient with respect to the three weight matrices, on one
 * NVIDIA B200 (sm_100a).
 *
 * What is computed (per batch b and head h, every (b, h) an independent instance):
 *
 *   Q~ = rot(A1 WQ),  K~ = rot(A2 WK),  V = A3 WV            (row-vector convention)
 *   s  = softmax(Q~ K~^T / sqrt(d))   (row-wise; keys j > i masked when causal)
 *   O  = s V,   l = O - E,   Loss = 1/2 sum_{b,h} ||O - E||_F^2
 *   beta  = l V^T,  gamma = diag(s) beta - s s^T beta
 *         (row-wise gamma_i = s_i o (beta_i - <l_i, O_i>))
 *   dQ~ = gamma K~ / sqrt(d),  dK~ = gamma^T Q~ / sqrt(d),  dV = s^T l
 *   dWQ_h = sum_b A1^T rot^-1(dQ~),  dWK_h = sum_b A2^T rot^-1(dK~),  dWV_h = sum_b A3^T dV
 *
 * rot() turns each adjacent pair (x_2k, x_2k+1) of row i counter-clockwise by the angle
 * pos_i * base^(-2k/d), k = 0 .. d/2-1.
 *
 * Sources: "RoPE Attention kan bijna lineair worden getraind" (summary of arXiv
 * 2412.17316), sections Probleemdefinitie and Methodologie 1 (closed-form gradient
 * dLoss/dx = A~^T vec(gamma(x)) built from s, l, beta, gamma) and Methodologie 2
 * (gamma_1 = diag(s) beta, gamma_2 = s s^T beta); "HyperAttention" article, section
 * 方法の概要 (exact attention D^-1 A V with A = exp(Q K^T) entrywise).
 *
 * Conventions for every entry point:
 *   - The caller owns all memory.  The library never allocates, frees or synchronises
 *     (except rope_attn_last_error, which synchronises the given stream).
 *   - Device pointers must be 16-byte aligned and point to contiguous arrays.
 *   - Arguments are validated before anything is launched; a status other than RA_OK
 *     means nothing was enqueued.  RA_ERR_CUDA means a launch failed.
 *   - Work is enqueued asynchronously on `stream` (a cudaStream_t; NULL = legacy default
 *     stream) on the current CUDA device.
 *   - A kernel that waits on an on-chip barrier gives up after a bounded time, records a
 *     timeout in a device-side status word and returns; rope_attn_last_error reports it.
 */
#ifndef ROPE_ATTN_H
#define ROPE_ATTN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  RA_OK = 0,
  RA_ERR_INVALID_ARG = 1,   /* null pointer, bad size or flag                          */
  RA_ERR_UNSUPPORTED = 2,   /* valid request the library does not implement (d)        */
  RA_ERR_ALIGNMENT = 3,     /* a device pointer is not 16-byte aligned                 */
  RA_ERR_WORKSPACE = 4,     /* workspace missing or smaller than rope_attn_workspace_bytes */
  RA_ERR_CUDA = 5,          /* a CUDA launch or runtime call failed                    */
  RA_ERR_TIMEOUT = 6        /* a kernel gave up waiting on an on-chip barrier          */
} ra_status;

typedef enum {
  RA_F32 = 0,   /* fp32 I/O, fp32 arithmetic on the CUDA cores                          */
  RA_BF16 = 1   /* bf16 I/O, bf16 tensor-core products with fp32 accumulation           */
} ra_dtype;

/* One problem: B x H independent instances of n tokens with head dimension d. */
typedef struct {
  int32_t B, H, n, d;      /* B, H, n >= 1; d in {64, 128}; B*H <= 65535; n <= 2^24, and  */
                           /* n <= 65535*128 with bf16 I/O (else RA_ERR_UNSUPPORTED)       */
  int32_t dtype;           /* ra_dtype: element type of A1, A2, A3, E, WQ, WK, WV and O   */
  int32_t causal;          /* 0 or 1: mask keys j > i (by index)                          */
  double rope_base;        /* RoPE base, > 0 (10000, 500000, ...)                         */
  const int32_t* pos;      /* device [n] positions shared by all (b, h); NULL = 0..n-1    */
  const void* A1;          /* device [B][H][n][d]: input of the query projection          */
  const void* A2;          /* device [B][H][n][d]: input of the key projection            */
  const void* A3;          /* device [B][H][n][d]: input of the value projection          */
  const void* WQ;          /* device [H][d][d]: W[in][out], Q = A1 . WQ                   */
  const void* WK;          /* device [H][d][d]                                            */
  const void* WV;          /* device [H][d][d]                                            */
  const void* E;           /* device [B][H][n][d]: target; may be NULL in rope_attn_fwd   */
  int32_t deterministic;   /* 0 or 1.  1: the backward adds the per-key-tile parts of the  */
                           /* query-side gradient in a fixed order, so dWQ, dWK, dWV and   */
                           /* dA1..dA3 are bitwise the same on every run (a little slower); */
                           /* 0: in whatever order the key tiles finish.  Exact path only;  */
                           /* not part of the workspace tag                                 */
} ra_problem;

/*
 * Bytes of device workspace that rope_attn_fwd and rope_attn_loss_bwd need for `p`
 * (0 if `p` is invalid).  The same workspace may serve both calls.
 */
size_t rope_attn_workspace_bytes(const ra_problem* p);

/*
 * Forward pass and loss.
 *   O    : device [B][H][n][d], element type p->dtype (written)
 *   lse  : device [B][H][n] fp32, natural-log log-sum-exp of each scaled score row (written)
 *   loss : device fp32 scalar, 1/2 ||O - E||_F^2 over all instances (written); must be NULL
 *          when p->E is NULL
 *   ws   : device workspace of at least rope_attn_workspace_bytes(p) bytes
 * When p->E is given, the workspace also keeps Q~, K~, V, l and <l_i, O_i> (and a zeroed
 * accumulator for dQ~) for a following rope_attn_loss_bwd(..., ws_holds_fwd = 1), and its
 * header records the problem's tag (below); without p->E the header is marked as holding
 * nothing a backward could reuse.
 */
ra_status rope_attn_fwd(const ra_problem* p, void* O, float* lse, float* loss,
                        void* ws, size_t ws_bytes, void* stream);

/*
 * Closed-form backward: the weight gradients of Loss = 1/2 ||O - E||_F^2.
 *   O, lse       : device, as written by rope_attn_fwd for the same problem (read)
 *   loss         : device fp32 scalar (written; may be NULL)
 *   dWQ/dWK/dWV  : device [H][d][d] fp32 (overwritten), summed over the batch
 *   ws_holds_fwd : 1 lets the device decide whether the intermediates in `ws` can be reused.
 *                  Every forward (with E) and backward call ends by writing a header at the
 *                  start of the workspace: a tag of the problem (B, H, n, d, dtype, causal,
 *                  rope_base and the pos, A1, A2, A3, WQ, WK, WV, E pointers) and what the
 *                  workspace holds.  With ws_holds_fwd = 1 the backward's recomputation
 *                  kernels (RoPE table, projections, l = O - E and delta from the given O)
 *                  read that header on the device and skip their work only when it carries
 *                  this problem's tag; a workspace of another problem, of a forward without E,
 *                  or never written is recomputed, so the result is right either way.  The
 *                  tag sees pointers, not contents: after changing inputs in place, run
 *                  rope_attn_fwd again (or pass 0) before the backward.
 *                  0 recomputes everything from the inputs unconditionally.
 * p->E must not be NULL.
 */
ra_status rope_attn_loss_bwd(const ra_problem* p, const void* O, const float* lse,
                             float* loss, float* dWQ, float* dWK, float* dWV,
                             void* ws, size_t ws_bytes, int32_t ws_holds_fwd, void* stream);

/*
 * rope_attn_loss_bwd followed by the gradients with respect to the three inputs, by the same
 * chain rule through Q = A1 WQ, K = A2 WK, V = A3 WV (the page's problem stops at the weight
 * gradients; these let layers be stacked):
 *   dA1 = rot^-1(dQ~) WQ^T,  dA2 = rot^-1(dK~) WK^T,  dA3 = dV WV^T
 *   dA1/dA2/dA3 : device [B][H][n][d], element type p->dtype (overwritten); none may be NULL
 * Other arguments, validation and errors as rope_attn_loss_bwd.  With bf16 I/O the products
 * use the bf16-rounded dQ, dK, dV (fp32 accumulation).
 */
ra_status rope_attn_loss_bwd_inputs(const ra_problem* p, const void* O, const float* lse,
                                    float* loss, float* dWQ, float* dWK, float* dWV, void* dA1,
                                    void* dA2, void* dA3, void* ws, size_t ws_bytes,
                                    int32_t ws_holds_fwd, void* stream);

/*
 * One step: rope_attn_fwd with the loss, then rope_attn_loss_bwd on the same workspace, in one
 * call (the page's problem end to end: Loss and its gradient with respect to the weight
 * matrices, "RoPE Attention kan bijna lineair worden getraind", Probleemdefinitie).
 *   O, lse       : device, written as by rope_attn_fwd
 *   loss         : device fp32 scalar (written; may be NULL)
 *   dWQ/dWK/dWV  : device [H][d][d] fp32 (overwritten)
 *   ws           : device workspace of at least rope_attn_workspace_bytes(p) bytes
 * p->E must not be NULL.  The results are those of the two calls (the backward reusing the
 * forward's intermediates); because the backward follows the forward inside the call, the
 * backward's recomputation launches are not made at all and the loss is summed once.  The
 * workspace header ends as after rope_attn_loss_bwd.  Validation and errors as the two calls.
 */
ra_status rope_attn_step(const ra_problem* p, void* O, float* lse, float* loss, float* dWQ,
                         float* dWK, float* dWV, void* ws, size_t ws_bytes, void* stream);

/*
 * One combined weight per head, the parameterisation of the page's problem: the gradient with
 * respect to a single weight x, dLoss/dx = A~^T vec(gamma(x)) ("RoPE Attention kan bijna lineair
 * worden getraind", Probleemdefinitie and Methodologie 1), read as x = vec(X) in the score
 *   z_ij = a1_i^T R_{j-i} X a2_j / sqrt(d)      (R_{j-i}: RoPE rotation by pos_j - pos_i).
 * Since R_{j-i} = R_i^T R_j, this is the general problem with WQ = I and WK = X^T:
 *   rope_attn_combined_weights writes WQ = I and WK = X^T ([H][d][d], element type `dtype`) for
 *   a following rope_attn_fwd / rope_attn_loss_bwd, and rope_attn_combined_grad turns that
 *   call's dWK (fp32 [H][d][d]) into dX = dWK^T (fp32 [H][d][d]).
 * X, WQ, WK, dWK, dX: device, 16-byte aligned; d in {64, 128}; H >= 1.  Errors as above.
 */
ra_status rope_attn_combined_weights(const void* X, int32_t H, int32_t d, int32_t dtype,
                                     void* WQ, void* WK, void* stream);
ra_status rope_attn_combined_grad(const float* dWK, int32_t H, int32_t d, float* dX,
                                  void* stream);

/*
 * The near-linear approximate method of "RoPE Attention kan bijna lineair worden getraind"
 * (Methodologie 2 "Low-Rank Benaderingsstrategie"; Resultaten, Theorem 5.7), with the degree-1
 * polynomial method: on bounded scores exp(z) is replaced by 1 + z = U_i . F_j with the d + 1
 * features U_i = (1, d^-1/4 q~_i), F_j = (1, d^-1/4 k~_j), so s~ = U F^T normalised per row is the
 * low-rank U1 V1^T; gamma_1 = diag(s~) beta is contracted through row-wise Kronecker products
 * of the factors with [l, -delta] and [v, 1], gamma_2 through the precomputed delta = <l, O>.
 * Causal masks use exclusive prefix / suffix sums of the low-rank states over chunks of 256 rows
 * and the pairs inside a chunk directly; work and memory are linear in n.  All arithmetic is
 * fp32 on the CUDA cores (inputs of either dtype).  The result approximates the exact one:
 * its accuracy depends on the bound of the scores (the method's bounded-entry regime).
 *   O           : device [B][H][n][d], element type p->dtype (written): s~ V
 *   loss        : device fp32 scalar 1/2 ||O - E||^2 (written; may be NULL)
 *   dWQ/dWK/dWV : device [H][d][d] fp32 (overwritten): the approximate weight gradients
 *   ws          : device workspace of rope_attn_approx_workspace_bytes(p) bytes (256-byte
 *                 aligned); it grows as n (d + 1)^2 d / 64 floats for the chunk states plus
 *                 ten [B][H][n][d] fp32 arrays
 * p->E must not be NULL.  Validation and errors as the other entry points.
 */
size_t rope_attn_approx_workspace_bytes(const ra_problem* p);
ra_status rope_attn_approx_step(const ra_problem* p, void* O, float* loss, float* dWQ, float* dWK,
                                float* dWV, void* ws, size_t ws_bytes, void* stream);

/*
 * Synchronises `stream`, then reports and clears the device-side status word of the current
 * device: RA_ERR_TIMEOUT if a kernel gave up waiting since the last call, else RA_OK
 * (RA_ERR_CUDA if the synchronisation itself failed).
 */
ra_status rope_attn_last_error(void* stream);

/* Static, human-readable name of a status code. */
const char* rope_attn_status_string(ra_status s);

/*
 * Number of kernel launches the library enqueued on this host thread since the last call
 * (then reset to 0).  Used to count the launches inside a timed region.
 */
int64_t rope_attn_launch_count(void);

/*
 * Per-kernel timing for measurement tools.  While enabled (on != 0), every launch made by
 * this host thread is bracketed by two CUDA events recorded on the launching stream; the
 * events are created on first use and kept for reuse (host-side driver objects, no device
 * memory).  Disabling drops records not yet read.
 */
void rope_attn_profile_enable(int32_t on);

/*
 * Restricts those events to the launches of kernel id `kernel_id` (see rope_attn_kernel_name);
 * a negative or out-of-range id restores events around every launch (the default).  Each
 * event pair adds a few microseconds between two dependent launches, so a timed region that
 * needs one kernel's duration brackets that kernel alone.
 */
void rope_attn_profile_only(int32_t kernel_id);

/*
 * Waits for the recorded events, then writes for each kernel id k < max_kernels the summed
 * device time in milliseconds (ms[k]) and the number of launches (launches[k]) since the
 * last read, and clears the records.  Returns the number of kernel ids (see
 * rope_attn_kernel_name), or -1 if an event query failed.
 */
int32_t rope_attn_profile_read(float* ms, int32_t* launches, int32_t max_kernels);

/* Static name of kernel id `id` (NULL if out of range). */
const char* rope_attn_kernel_name(int32_t id);

/*
 * Size of the scratch array behind rope_attn_step_noalloc: a file-scope device array of the
 * library that every GPU which loads the library holds until the process exits.
 */
#define RA_NOALLOC_SCRATCH_BYTES (16u * 1024u * 1024u)

/*
 * One whole step (rope_attn_fwd with the loss, then rope_attn_loss_bwd reusing the forward's
 * intermediates) for callers that cannot call cudaMalloc, for example code that may not take
 * the device-wide synchronisation an allocation can cause, or that runs inside a component
 * whose device memory is owned by someone else.  There is no counterpart of this entry point
 * in the paper; it exists only for such callers.
 *
 * The caller passes inputs (p, with E) and outputs exactly as for rope_attn_fwd and
 * rope_attn_loss_bwd: O, lse, loss (may be NULL), dWQ, dWK, dWV.  Instead of a caller-owned
 * workspace the step uses the library's static scratch array of RA_NOALLOC_SCRATCH_BYTES on
 * the current device.  Nothing is allocated or freed: no cudaMalloc, cudaFree or allocating
 * library routine is called.
 *
 * Limits and behaviour:
 *   - a problem whose workspace (rope_attn_workspace_bytes) exceeds RA_NOALLOC_SCRATCH_BYTES is
 *     rejected with RA_ERR_WORKSPACE before anything is launched;
 *   - the first call on a device looks up the scratch array's device address
 *     (cudaGetSymbolAddress) with that device current; make that first call before any stream
 *     capture.  Later calls reuse the address while the device's CUDA context stays the same;
 *     after a cudaDeviceReset the next call looks it up again (so make it outside a capture
 *     too);
 *   - every call on a device shares the one scratch array, which keeps the last call's contents;
 *     the step clears what must start at zero itself, but calls whose work overlaps on the GPU
 *     (different streams, or different host threads) race on the scratch: order them.
 */
ra_status rope_attn_step_noalloc(const ra_problem* p, void* O, float* lse, float* loss,
                                 float* dWQ, float* dWK, float* dWV, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* ROPE_ATTN_H */
