/*
 * gradlev.h - C ABI of the GradLev scan library (libgradlev.so, CUDA, sm_100a).
 *
 * The library evaluates the token-parallel scans of one GradLev adaptive
 * linear layer on the GPU: the forward scan that rebuilds the centred
 * fast-weight trajectory from the layer inputs, the gates and the costates,
 * and the reverse scan that backpropagates an upstream gradient through it
 * (gradlev_scan_fwd, gradlev_scan_bwd). Around them:
 *   gradlev_scan_fwd_state / _bwd_state   one part of a split sequence (carried state)
 *   gradlev_decode_step                   deployment: token-by-token forward, costate, update
 *   gradlev_consistency_step              a training step from predicted costates
 *   gradlev_mlp2_recon                    the two-layer reconstruction of the synthetic test
 *   gradlev_scan_bwd_noalloc              the reverse scan without a workspace argument
 *   gradlev_scan_bwd_noalloc_scratch_bytes  its scratch need
 *   gradlev_noalloc_device_status         its device status word
 *
 * Definition (Cognaptus, "Parallelize the Training, Keep the Learning Serial",
 * section "Once the gradient signals are known, the weight trajectory becomes
 * parallelizable"; GradLev abstract, "GradLev: Token-Parallel Test-Time
 * Training Via Costate Prediction"). Per batch row b and head h, with 0-based
 * tokens t and S_t the deviation of the temporary weight from the persistent
 * weight W0 BEFORE token t:
 *
 *     S_0 = 0
 *     y_t     = (W0 + S_t) x_t
 *     S_{t+1} = alpha_t S_t - eta_t g_t x_t^T
 *
 * x_t is the layer input, eta_t the step size, alpha_t the retention gate and
 * g_t the costate (gradient of the token loss with respect to the layer
 * output). In the page's 1-based notation this is D_t = alpha_t D_{t-1} -
 * eta_t g_t x_t^T, y_t = (W0 + D_{t-1}) x_t. The backward returns the exact
 * gradients of L = sum_t <dy_t, y_t> with respect to x, g, eta, alpha and W0
 * (W0 is one matrix per head, shared by all batch rows; dW0 sums over b).
 *
 * Layouts: contiguous, row-major, device memory.
 *     x, dx          [B, H, T, d_in]     dtype
 *     g, y, dy, dg   [B, H, T, d_out]    dtype
 *     eta, alpha, d_eta, d_alpha [B, H, T]   float32 (all dtypes)
 *     W0, dW0        [H, d_out, d_in]    float32 (all dtypes)
 * dtype GRADLEV_F32: float32 I/O, float32 arithmetic (CUDA cores).
 * dtype GRADLEV_BF16: bfloat16 I/O, bf16 tensor-core operands with float32
 *     accumulation and float32 state.
 *
 * Ownership: the caller allocates every buffer (inputs, outputs, optional
 * checkpoint buffer, workspace). The library allocates no device memory per
 * call and keeps no per-call global state. Calls are asynchronous on `stream`
 * (a cudaStream_t passed as void*; NULL = the legacy default stream). Outputs
 * are overwritten, never accumulated.
 *
 * Errors: argument errors (null pointers, non-positive sizes, unsupported
 * shapes, too-small workspace) are detected on the host and returned before
 * any launch; nothing is written. Launch failures return GRADLEV_ERR_CUDA.
 * Preconditions that are not checked (they would need a device read):
 * 0 <= alpha <= 1 and finite inputs.
 */
#ifndef GRADLEV_H_
#define GRADLEV_H_

#include <stddef.h>

#if defined(__GNUC__)
#define GRADLEV_API __attribute__((visibility("default")))
#else
#define GRADLEV_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  GRADLEV_F32 = 0,  /* x, g, y, dy, dx, dg are float32 */
  GRADLEV_BF16 = 1  /* x, g, y, dy, dx, dg are bfloat16 */
} gradlev_dtype;

typedef enum {
  GRADLEV_OK = 0,
  GRADLEV_ERR_INVALID_ARG = 1,  /* null pointer, size <= 0, unknown dtype */
  GRADLEV_ERR_UNSUPPORTED = 2,  /* valid but unsupported shape for this dtype */
  GRADLEV_ERR_WORKSPACE = 3,    /* workspace smaller than gradlev_scan_workspace_bytes() */
  GRADLEV_ERR_CUDA = 4,         /* a CUDA runtime call or kernel launch failed */
  GRADLEV_ERR_TIMEOUT = 5       /* a bounded device-side wait gave up (gradlev_device_status) */
} gradlev_status;

/* Human-readable name of a status code (static string, never NULL). */
GRADLEV_API const char* gradlev_status_string(gradlev_status s);

/* Whether (B, H, T, d_in, d_out, dt) is supported: GRADLEV_OK, or
 * GRADLEV_ERR_INVALID_ARG / GRADLEV_ERR_UNSUPPORTED without touching the GPU.
 * Supported: B, H, T >= 1 with B*H*T < 2^31, and either
 *   - GRADLEV_BF16 with d_in = 128 and d_out in {128, 256} (tensor-core kernels), or
 *   - either dtype with d_in % 4 == 0, d_out % 8 == 0, 8 <= d_in, d_out and
 *     d_in * d_out <= 16384 (CUDA-core kernels). */
GRADLEV_API gradlev_status gradlev_scan_supported(int B, int H, int T, int d_in, int d_out,
                                      gradlev_dtype dt);

/* Bytes of device workspace the forward (is_bwd = 0) or backward (is_bwd = 1)
 * call needs for this shape; 0 if the shape is unsupported. The workspace is
 * scratch: its contents on entry do not matter; on return its first 16 bytes
 * hold the device status word read by gradlev_device_status() and the rest is
 * unspecified. It is never smaller than 256 bytes. It grows with the shape: the
 * backward keeps per-scan dW0 partials there, and calls whose scans are too few
 * to fill the GPU cut each scan into segments whose fp32 summaries live there
 * (a few 64 KB matrices per scan and segment). */
GRADLEV_API size_t gradlev_scan_workspace_bytes(int B, int H, int T, int d_in, int d_out,
                                    gradlev_dtype dt, int is_bwd);

/* Bytes of the optional state-checkpoint buffer that gradlev_scan_fwd can fill
 * and gradlev_scan_bwd can consume for the same shape and dtype; 0 if
 * unsupported. Its contents are implementation-defined (the scan state at fixed
 * token intervals: bfloat16 every 64 tokens for bf16 I/O with d_in = 128 and
 * d_out in {128, 256}, float32 every 32 tokens otherwise) and valid only for the
 * inputs of the forward call that wrote them. */
GRADLEV_API size_t gradlev_scan_ckpt_bytes(int B, int H, int T, int d_in, int d_out, gradlev_dtype dt);

/* Forward scan: y_t = (W0 + S_t) x_t for every (b, h, t).
 *   x [B,H,T,d_in], g [B,H,T,d_out] (dtype); eta, alpha [B,H,T] float32;
 *   W0 [H,d_out,d_in] float32; y [B,H,T,d_out] (dtype) is written.
 *   ckpt: NULL, or gradlev_scan_ckpt_bytes() bytes that receive the state
 *   checkpoints for a later gradlev_scan_bwd on the same inputs.
 *   workspace: at least gradlev_scan_workspace_bytes(..., 0) bytes. */
GRADLEV_API gradlev_status gradlev_scan_fwd(int B, int H, int T, int d_in, int d_out, gradlev_dtype dt,
                                const void* x, const void* g, const float* eta,
                                const float* alpha, const float* W0, void* y, void* ckpt,
                                void* workspace, size_t ws_bytes, void* stream);

/* Reverse scan. With Lam_T = 0 and Lam_t = alpha_t Lam_{t+1} + dy_t x_t^T:
 *   dx_t      = (W0 + S_t)^T dy_t - eta_t Lam_{t+1}^T g_t      [B,H,T,d_in]  (dtype)
 *   dg_t      = -eta_t Lam_{t+1} x_t                            [B,H,T,d_out] (dtype)
 *   d_eta_t   = -g_t . (Lam_{t+1} x_t)                          [B,H,T] float32
 *   d_alpha_t = <Lam_{t+1}, S_t>_F                              [B,H,T] float32
 *   dW0       = sum_{b,t} dy_t x_t^T                            [H,d_out,d_in] float32
 *   ckpt: NULL (the call recomputes the states itself, in the workspace), or the
 *   buffer a gradlev_scan_fwd call on the same inputs filled.
 *   workspace: at least gradlev_scan_workspace_bytes(..., 1) bytes. */
GRADLEV_API gradlev_status gradlev_scan_bwd(int B, int H, int T, int d_in, int d_out, gradlev_dtype dt,
                                const void* x, const void* g, const float* eta,
                                const float* alpha, const float* W0, const void* dy,
                                void* dx, void* dg, float* d_eta, float* d_alpha, float* dW0,
                                const void* ckpt, void* workspace, size_t ws_bytes,
                                void* stream);

/* Split sequences: the carried state.
 *
 * Cognaptus, "Parallelize the Training, Keep the Learning Serial", section "Once
 * the gradient signals are known, the weight trajectory becomes parallelizable":
 * the recurrence is affine, so partial results combine. A sequence cut into
 * consecutive parts can be scanned one call per part, each continuing from the
 * deviation the previous part left.
 *
 * Forward with a carried state: the same as gradlev_scan_fwd, except that the
 * deviation before the first token is S0 instead of 0, and the deviation after
 * the last token is returned:
 *   S_0 = S0,  y_t = (W0 + S_t) x_t,  S_{t+1} = alpha_t S_t - eta_t g_t x_t^T,
 *   ST = S_T.
 *   S0: NULL (zero), or [B,H,d_out,d_in] float32, read only.
 *   ST: NULL (not written), or [B,H,d_out,d_in] float32, written. It may not
 *       alias S0.
 *   Both are 16-byte aligned (else GRADLEV_ERR_INVALID_ARG) and owned by the
 *   caller. Every other argument, the workspace size and the checkpoints are as
 *   in gradlev_scan_fwd; the checkpoints then hold states that include S0. */
GRADLEV_API gradlev_status gradlev_scan_fwd_state(int B, int H, int T, int d_in, int d_out,
                                      gradlev_dtype dt, const void* x, const void* g,
                                      const float* eta, const float* alpha, const float* W0,
                                      const float* S0, void* y, float* ST, void* ckpt,
                                      void* workspace, size_t ws_bytes, void* stream);

/* Reverse scan with a carried state: the derivative of
 *   L = sum_t <dy_t, y_t> + <LamT, S_T>_F
 * for the forward above. The adjoint recurrence starts from Lam_T = LamT instead
 * of 0, every output of gradlev_scan_bwd keeps its formula (with S_t including
 * S0), and the adjoint at the first token is returned:
 *   dS0 = Lam_0 = dL/dS_0.
 *   S0: NULL (zero), or the start deviation the forward began from. It is read
 *       only when ckpt is NULL (the call then recomputes the states from it);
 *       checkpoints from gradlev_scan_fwd_state already include it.
 *   LamT: NULL (zero), or [B,H,d_out,d_in] float32. When this part is followed
 *       by another, LamT is the dS0 the later part's call returned.
 *   dS0: NULL (not written), or [B,H,d_out,d_in] float32.
 *   All three are 16-byte aligned and owned by the caller. dS0 may not alias
 *   another argument. Every other argument, the workspace size and the errors
 *   are as in gradlev_scan_bwd. */
GRADLEV_API gradlev_status gradlev_scan_bwd_state(int B, int H, int T, int d_in, int d_out,
                                      gradlev_dtype dt, const void* x, const void* g,
                                      const float* eta, const float* alpha, const float* W0,
                                      const float* S0, const void* dy, const float* LamT,
                                      void* dx, void* dg, float* d_eta, float* d_alpha,
                                      float* dW0, float* dS0, const void* ckpt,
                                      void* workspace, size_t ws_bytes, void* stream);

/* Deployment decode: T tokens of the token-by-token learner, in order.
 *
 * The GradLev abstract states that the auxiliary predictor is discarded at
 * deployment, and the model then updates itself with token-by-token forward and
 * backward passes. Cognaptus, "Parallelize the Training, Keep the Learning
 * Serial", opening section, says the same: each token costs a forward pass, a
 * backward pass and a weight update. For one adapted linear layer with the inner
 * loss 0.5 ||W x_t - v_t||^2 of the pages' synthetic test, each token is
 *   y_t = (W0 + S) x_t,   g_t = y_t - v_t,   S <- alpha_t S - eta_t g_t x_t^T.
 * S is the deviation from W0, carried between calls. With S = 0 before the
 * first token, this reproduces the serial online learner the scans recover.
 *
 *   x [B,H,T,d_in], v [B,H,T,d_out] (targets), y and g [B,H,T,d_out]: dtype.
 *   eta, alpha [B,H,T]: float32. W0 [H,d_out,d_in]: float32.
 *   S [B,H,d_out,d_in]: float32, read and overwritten with the deviation after
 *     the last token.
 *   g: NULL (costates not written), or the buffer that receives them.
 * Constraints:
 *   - d_in must be a multiple of 4 and at most 256, else
 *     GRADLEV_ERR_UNSUPPORTED. Any d_out >= 1 is accepted.
 *   - Alignment, else GRADLEV_ERR_INVALID_ARG: x to 4 elements; v, y and g to
 *     one element; W0 and S to 16 bytes.
 *   - One launch; no workspace; no device waits; nothing is allocated.
 *   - The buffers are the caller's. y and g may not alias the inputs. */
GRADLEV_API gradlev_status gradlev_decode_step(int B, int H, int T, int d_in, int d_out,
                                   gradlev_dtype dt, const void* x, const void* v,
                                   const float* eta, const float* alpha, const float* W0,
                                   float* S, void* y, void* g, void* stream);

/* One training step of the adapted layer from predicted costates: the forward
 * scan, the reconstructed costates, the token and consistency losses, and every
 * gradient of their sum.
 *
 * Cognaptus, "Parallelize the Training, Keep the Learning Serial", section "The
 * predictor is constrained by the learner it is supposed to reproduce":
 *   - the forward runs on the predicted costates ghat;
 *   - the costates the proposed trajectory implies are reconstructed from it;
 *   - training combines the token loss with a term that pushes ghat toward them.
 * For the synthetic test's inner loss 0.5 ||y - v||^2 the reconstruction is
 * gtil = y - v. The consistency term's formula is missing from the page; this
 * call reads it as lam ||ghat - gtil||^2 with gtil the target (no gradient
 * flows through gtil):
 *   L = sum_t 0.5 ||gtil_t||^2 + lam ||ghat_t - gtil_t||^2.
 *
 * Outputs (all written):
 *   y, gtil [B,H,T,d_out] (dtype)    loss_tok, loss_c [B,H,T] float32 (per token)
 *   dx [B,H,T,d_in] (dtype)          dghat [B,H,T,d_out] (dtype): gradient w.r.t. ghat
 *   d_eta, d_alpha [B,H,T] float32   dW0 [H,d_out,d_in] float32
 *   dv [B,H,T,d_out] (dtype) = -gtil, or NULL (not written).
 * The token loss's output gradient is gtil, so dx, d_eta, d_alpha and dW0 are
 * the reverse scan with dy = gtil. The consistency term adds 2 lam (ghat - gtil)
 * to dghat.
 *
 * Requirements, else the status shown:
 *   - d_out a multiple of 4, and the shapes of gradlev_scan_fwd
 *     (GRADLEV_ERR_UNSUPPORTED);
 *   - workspace at least gradlev_consistency_workspace_bytes() bytes
 *     (GRADLEV_ERR_WORKSPACE);
 *   - alignment (GRADLEV_ERR_INVALID_ARG): workspace 256 bytes; x, ghat, y,
 *     gtil, dx, dghat, W0 and dW0 16 bytes; v and dv 4 elements.
 * Outputs may not alias inputs. gradlev_device_status(workspace) reports the
 * bounded waits of all its launches. */
GRADLEV_API size_t gradlev_consistency_workspace_bytes(int B, int H, int T, int d_in, int d_out,
                                           gradlev_dtype dt);
GRADLEV_API gradlev_status gradlev_consistency_step(int B, int H, int T, int d_in, int d_out,
                                        gradlev_dtype dt, const void* x, const void* ghat,
                                        const float* eta, const float* alpha, const float* W0,
                                        const void* v, float lam, void* y, void* gtil,
                                        float* loss_tok, float* loss_c, void* dx, void* dghat,
                                        float* d_eta, float* d_alpha, float* dW0, void* dv,
                                        void* workspace, size_t ws_bytes, void* stream);

/* Parallel reconstruction of the two-layer adapted MLP of the synthetic test.
 *
 * Cognaptus, "Parallelize the Training, Keep the Learning Serial", section "The
 * synthetic test checks the mechanism, not model quality". Both matrices adapt
 * with the centred rule under the shared gates eta, alpha; the hidden layer is
 * tanh (the pages name no nonlinearity). Given costates g1hat and g2hat for the
 * two layers:
 *   a = scan(x; g1hat, W1)          [B,H,T,d_h]   (the forward scan, d_in = d_x)
 *   h = tanh(a)                      [B,H,T,d_h]
 *   y = scan(h; g2hat, W2)          [B,H,T,d_y]
 *   g2til_t = y_t - v_t              [B,H,T,d_y]
 *   g1til_t = (1 - h_t^2) (.) ((W2 + S2_t)^T g2til_t)   [B,H,T,d_h]
 *   dW1 = sum_t g1til_t x_t^T         [B,H,d_h,d_x] float32
 * S2_t is the second layer's deviation before token t. control = 1 uses the
 * persistent W2 instead of W2 + S2_t: the control of the same section, which
 * leaves y unchanged and breaks g1til and dW1. With the serial learner's costates
 * supplied, the outputs are the serial learner's outputs, hidden costates and
 * first-matrix gradient.
 *
 * Arguments:
 *   W1 [H,d_h,d_x], W2 [H,d_y,d_h], eta and alpha [B,H,T]: float32.
 *   x, g1hat, g2hat, v and every output except dW1: dtype.
 * Requirements, else the status shown:
 *   - (d_x -> d_h) and (d_h -> d_y) must each be a supported scan shape; d_x a
 *     multiple of 4; d_h and d_y multiples of 8; d_h * d_x <= 16384
 *     (GRADLEV_ERR_UNSUPPORTED);
 *   - workspace at least gradlev_mlp2_workspace_bytes() bytes
 *     (GRADLEV_ERR_WORKSPACE);
 *   - alignment (GRADLEV_ERR_INVALID_ARG): workspace 256 bytes; x, g1hat,
 *     g2hat, a, h, y, g2til, g1til, W1, W2 and dW1 16 bytes; v one element.
 * Outputs may not alias inputs.
 * Routes: with a tensor-core second layer (bf16, d_h = 128, d_y in {128, 256})
 * and no control, g1til comes from the reverse-scan kernel in its hidden-costate
 * mode, i.e. dx without the adjoint terms, times (1 - h^2). Every other case uses
 * a CUDA-core reconstruction kernel. */
GRADLEV_API size_t gradlev_mlp2_workspace_bytes(int B, int H, int T, int d_x, int d_h, int d_y,
                                    gradlev_dtype dt);
GRADLEV_API gradlev_status gradlev_mlp2_recon(int B, int H, int T, int d_x, int d_h, int d_y,
                                  gradlev_dtype dt, const void* x, const void* g1hat,
                                  const void* g2hat, const void* v, const float* eta,
                                  const float* alpha, const float* W1, const float* W2,
                                  int control, void* a, void* h, void* y, void* g2til,
                                  void* g1til, float* dW1, void* workspace, size_t ws_bytes,
                                  void* stream);

/* Size of the static scratch array gradlev_scan_bwd_noalloc uses: 64 MiB,
 * held by every GPU that loads the library until the process exits. */
#define GRADLEV_NOALLOC_SCRATCH_BYTES ((size_t)64 << 20)

/* gradlev_scan_bwd without a workspace argument, for callers that cannot
 * allocate device memory: code running where the allocator is unavailable or
 * must not grow (a fixed-pool serving runtime, a plugin that is handed only its
 * tensors, a host binding without a CUDA allocator). The method has no
 * counterpart of this call; it is a deployment convenience of this library.
 *
 * Same arguments, outputs and results as gradlev_scan_bwd minus `workspace`
 * and `ws_bytes`. Scratch comes from one static device array of
 * GRADLEV_NOALLOC_SCRATCH_BYTES on the current device. The call allocates
 * nothing (no cudaMalloc, cudaFree or allocating library routine).
 *   - Limit: the call needs gradlev_scan_bwd_noalloc_scratch_bytes() of
 *     scratch. That is the status word and the per-scan dW0 partials
 *     (B*H*d_out*d_in*4 bytes, times the number of segments per scan when
 *     either kernel family cuts few long scans into segments, plus the segment
 *     summaries), and, when ckpt is NULL, the chunk-start states as well; with
 *     ckpt NULL it equals gradlev_scan_workspace_bytes(.., is_bwd = 1). A
 *     problem that needs more than GRADLEV_NOALLOC_SCRATCH_BYTES returns
 *     GRADLEV_ERR_WORKSPACE before any launch. Shape errors return as in
 *     gradlev_scan_bwd.
 *   - The first call on a device looks up the array's device address
 *     (cudaGetSymbolAddress, with that device current) and caches it; make that
 *     first call before any stream capture.
 *   - Every call on a device shares the one array, and it keeps the last
 *     call's contents (each call clears the part that must start at zero).
 *     Calls whose work overlaps on the GPU (different streams, or other host
 *     threads) race on it and give wrong results: serialise them.
 *   - The device status word of the call lives at the start of the array:
 *     read it with gradlev_noalloc_device_status(), not gradlev_device_status(). */
GRADLEV_API gradlev_status gradlev_scan_bwd_noalloc(
    int B, int H, int T, int d_in, int d_out, gradlev_dtype dt, const void* x, const void* g,
    const float* eta, const float* alpha, const float* W0, const void* dy, void* dx, void* dg,
    float* d_eta, float* d_alpha, float* dW0, const void* ckpt, void* stream);

/* Scratch bytes gradlev_scan_bwd_noalloc needs for this problem (has_ckpt != 0:
 * the caller passes checkpoints), or 0 for an unsupported shape. No GPU call.
 * The method has no counterpart of this call. */
GRADLEV_API size_t gradlev_scan_bwd_noalloc_scratch_bytes(int B, int H, int T, int d_in,
                                                         int d_out, gradlev_dtype dt,
                                                         int has_ckpt);

/* Device status of the last gradlev_scan_bwd_noalloc call on the current
 * device: synchronises `stream` and reads the status word the kernels leave at
 * the start of the static scratch array. GRADLEV_OK, GRADLEV_ERR_TIMEOUT if a
 * bounded device-side wait gave up (that call's outputs are then unspecified),
 * or GRADLEV_ERR_CUDA. Allocates nothing. The method has no counterpart of
 * this call. */
GRADLEV_API gradlev_status gradlev_noalloc_device_status(void* stream);

/* Device status of the last call that used `workspace`: synchronises `stream`
 * and reads the status word the kernels leave at the start of the workspace.
 * GRADLEV_OK, GRADLEV_ERR_TIMEOUT if a bounded device-side wait gave up (the
 * outputs of that call are then unspecified), or GRADLEV_ERR_CUDA. */
GRADLEV_API gradlev_status gradlev_device_status(const void* workspace, void* stream);

/* Number of kernels the last successful fwd / bwd call on this host thread
 * launched (for launch accounting by benchmarks). */
GRADLEV_API int gradlev_last_launch_count(void);

/* Test hook for the failure-detection path (no GPU fault or hang is involved):
 * the next tensor-core launch at `site` withholds one internal completion
 * signal, so one of the kernel's bounded waits runs out after timeout_ms; every
 * CTA then unwinds (in-flight copies and matrix operations are drained, tensor
 * memory is released) and the call's gradlev_device_status() reports
 * GRADLEV_ERR_TIMEOUT. Sites (bf16 tensor-core shapes only):
 *   1  the forward scan's main pass (gradlev_scan_fwd and the calls built on it)
 *   2  the reverse scan's main kernel
 *   3  the forward's segment-summary pass (few long scans, cut into segments)
 *   4  the reverse scan's segment-summary pass
 *   0  off
 * Host-global, one-shot, not thread-safe; for tests only. */
GRADLEV_API void gradlev_debug_inject_timeout(int site, int timeout_ms);

/* Test hook for the segment-summary passes of the bf16 tensor-core path (few
 * long scans, cut into segments). Those passes carry only the state or the
 * adjoint across each segment; they keep the decay accumulated since the last
 * rescale as a scale factor 2^E outside tensor memory (folded into the
 * scaled inputs of each update) and rescale the stored matrix in place once E
 * would fall below -log2_bound. The default bound is 64. A smaller bound in
 * [0, 126] makes the in-place rescale run more often (0: at every chunk that
 * decays), so that tests can reach it on short inputs; a negative or NaN value
 * restores the default, and values above 126 are clamped to 126. Results agree
 * for every bound up to rounding. Host-global, not thread-safe; for tests only. */
GRADLEV_API void gradlev_debug_summary_rescale(float log2_bound);

#ifdef __cplusplus
}
#endif

#endif /* GRADLEV_H_ */
