/*
 * dora.h - C ABI of the B200 (sm_100a) DoRA factored-norm / fused-compose library.
 *
 * Method: "Scaling DoRA: High-Rank Adaptation via Factored Norms and Fused
 * Kernels" (Zelenin & Zhuravlyova, arXiv 2603.22276), Abstract.  DoRA writes
 * the adapted weight as W' = m * (W + s B A) / ||W + s B A||_row.  The row norm
 * is computed from base, cross and Gram terms without forming B A, and the
 * magnitude rescaling is composed with the base and LoRA outputs in one pass.
 *
 * Entry points: the factored norm (one module, many modules at once, or a
 * d_in shard's squared share), the compose forward and its backward with the
 * norm detached (with or without a base-layer bias, with or without a
 * workspace), the compose fused into the GEMMs that produce its inputs, and
 * the norm's own gradients into A and B for training with the norm attached.
 *
 * Conventions shared by every call
 * --------------------------------
 *  - Layout: dense, row-major, contiguous.  W is [d_out, d_in] (frozen base
 *    weight), A is [r, d_in] (lora_A), B is [d_out, r] (lora_B), activations
 *    base_out / lora_out / dy / y / d_base / d_lora are [tokens, d_out].
 *    lora_out is UNSCALED (x A^T B^T); the scaling s is applied here.
 *  - dtype: DORA_BF16 or DORA_F32 applies to W, A, B and the activations.
 *    m, n and d_m are always fp32 [d_out].
 *  - Pointers are device pointers unless stated.  The caller owns and allocates
 *    every buffer, including the workspace; the library never allocates device
 *    memory, so no O(d_out * d_in) temporary ever exists.
 *  - bf16 requires 16-byte aligned pointers and d_in, d_out multiples of 8;
 *    the factored norm also needs r a multiple of 16, the other calls state
 *    their own rules (else DORA_ERR_UNSUPPORTED).  fp32 accepts any shape with
 *    4-byte aligned pointers where a call takes fp32.
 *  - stream is a cudaStream_t passed as void* (NULL = legacy default stream).
 *    Every call is asynchronous on it and returns once the work is enqueued.
 *  - Errors: argument errors are detected on the host before anything is
 *    launched and return DORA_ERR_INVALID_ARG / DORA_ERR_UNSUPPORTED /
 *    DORA_ERR_WORKSPACE.  A failed launch returns DORA_ERR_CUDA.  Kernels that
 *    wait on other threads bound every wait; if one gives up it records
 *    DORA_ERR_TIMEOUT in a device-side word that dora_device_status() reports.
 *    The outputs of that call are undefined.  Nothing in a workspace has to be
 *    cleared by the caller: the compose backward's arrival counters carry a
 *    tag that is new for every call.  A CUDA graph replays its captured tag,
 *    so after a replay of a compose backward that timed out, re-capture the
 *    graph (or zero that workspace) before replaying it.
 *  - Outputs are overwritten, never accumulated into.  Results are
 *    deterministic: every reduction runs in a fixed order.
 */
#ifndef DORA_H_
#define DORA_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define DORA_API __attribute__((visibility("default")))
#else
#define DORA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum { DORA_BF16 = 0, DORA_F32 = 1 } dora_dtype;

typedef enum {
  DORA_OK = 0,
  DORA_ERR_INVALID_ARG = 1, /* null pointer, negative size ... */
  DORA_ERR_UNSUPPORTED = 2, /* alignment / shape / dtype this build does not handle */
  DORA_ERR_WORKSPACE = 3,   /* workspace missing or smaller than the size query */
  DORA_ERR_CUDA = 4,        /* a CUDA runtime call failed (launch, attribute ...) */
  DORA_ERR_TIMEOUT = 5      /* a bounded device-side wait gave up */
} dora_status;

/* Bytes of workspace dora_factored_norm needs for this shape (0 never means
 * "no workspace" for valid shapes; returns 0 for invalid shapes): the
 * O(d_out r + r^2) intermediates of the factored norm (Scaling DoRA, Abstract),
 * here (s/2) A A^T in bf16 and per-row partial sums, never O(d_out d_in). */
DORA_API size_t dora_factored_norm_workspace_size(int64_t d_out, int64_t d_in, int64_t r, dora_dtype dt);

/* Factored row norm of W + s B A (Scaling DoRA, Abstract: the squared norm
 * splits into a base, a cross and a Gram term, which need only
 * O(d_out r + r^2) intermediates):
 *
 *   n_i = sqrt(max(||W_i||^2 + 2 s <B_i, (W A^T)_i> + s^2 B_i (A A^T) B_i^T, 0))
 *
 * n_out: fp32 [d_out], overwritten.  workspace: device buffer of at least
 * dora_factored_norm_workspace_size() bytes, 256-byte aligned, contents
 * ignored on entry and clobbered; it is O(d_out r + r^2 + SMs * 128) and never
 * O(d_out d_in).  r == 0 or s == 0 give the plain row norm of W.  bf16: W is
 * streamed from HBM once by tcgen05 tensor-core GEMM tiles; fp32: CUDA-core
 * fp32 arithmetic (no TF32). */
DORA_API int dora_factored_norm(const void* W, const void* A, const void* B, int64_t d_out, int64_t d_in, int64_t r,
                       float s, dora_dtype dt, float* n_out, void* workspace, size_t workspace_bytes,
                       void* stream);

/* dora_factored_norm without the final square root: n2_out[i] is
 * ||W_i||^2 + 2s <B_i, U_i> + s^2 B_i G B_i^T as summed, not clamped.  Every
 * term is a sum over d_in, so when W and A are split along d_in across ranks
 * (a row-parallel layer), each rank's n2 over its own columns is its share of
 * the full n^2: summing the shares (one all-reduce of d_out fp32) and applying
 * dora_norm_finish gives the norm of the whole layer.  Arguments, workspace
 * and errors as dora_factored_norm. */
DORA_API int dora_factored_norm_sq(const void* W, const void* A, const void* B, int64_t d_out, int64_t d_in,
                                   int64_t r, float s, dora_dtype dt, float* n2_out, void* workspace,
                                   size_t workspace_bytes, void* stream);

/* n[i] = sqrt(max(n[i], 0)) in place for i < d_out (fp32, 4-byte aligned):
 * the last step after summing dora_factored_norm_sq shares.  d_out == 0 does
 * nothing.  Asynchronous on `stream`. */
DORA_API int dora_norm_finish(float* n, int64_t d_out, void* stream);

/* One adapted module for dora_factored_norm_batched: the arguments of
 * dora_factored_norm for that module (device pointers, row-major layouts as
 * above; n_out is overwritten). */
typedef struct {
  const void* W;
  const void* A;
  const void* B;
  int64_t d_out, d_in, r;
  float s;
  float* n_out;
} dora_norm_problem;

/* Bytes of workspace dora_factored_norm_batched needs for these modules
 * (`problems`: host array of `count`); 0 for invalid arguments. */
DORA_API size_t dora_factored_norm_batched_workspace_size(const dora_norm_problem* problems, int count, dora_dtype dt);

/* The factored row norms of `count` adapted modules at once (Scaling DoRA,
 * Abstract: a model carries hundreds of adapted modules), each computing
 * exactly what dora_factored_norm computes for it.  `problems` is a host
 * array, read during the call only.  Modules with bf16 weights and
 * 16 <= r <= 512 share two launches: every 128 x 128 tile of every module's
 * Gram matrix, then one persistent GEMM over a work list of (module, 128-row
 * tile) items, each item finishing its rows' norms; the other modules are
 * computed one by one as by dora_factored_norm, on the same stream.
 * Every module's arguments are checked (as dora_factored_norm checks them)
 * before anything is launched.  workspace: device buffer of at least
 * dora_factored_norm_batched_workspace_size() bytes, 256-byte aligned,
 * contents ignored on entry; it holds the modules' descriptor table (copied
 * from the host with cudaMemcpyAsync), their G' = (s/2) G and the scratch of
 * the one-by-one modules.  Asynchronous on `stream`; count == 0 does nothing. */
DORA_API int dora_factored_norm_batched(const dora_norm_problem* problems, int count, dora_dtype dt, void* workspace,
                                        size_t workspace_bytes, void* stream);

/* Fused DoRA compose, one pass (Scaling DoRA, Abstract: the four-kernel
 * composition collapsed into a single pass, in a numerically stable form for
 * the near-unity regime):
 *
 *   g = m / n,  delta = (m - n) / n            (fp32, per output channel)
 *   y = base + (delta * base + g * s * lora)   (fp32 arithmetic, one rounding)
 *
 * which equals g * (base + s * lora) without rounding g or g - 1 to the
 * activation type.  base_out, lora_out, y: [tokens, d_out] row-major in dt
 * (bf16: d_out a multiple of 8 and 16-byte aligned pointers; fp32: 4-byte
 * aligned); lora_out is the unscaled (x A^T) B^T.  m, n: fp32 [d_out] (n from
 * dora_factored_norm).  tokens may be 0 (nothing is launched).  y must not
 * overlap the inputs. */
DORA_API int dora_compose_fwd(const void* base_out, const void* lora_out, const float* m, const float* n, float s,
                              int64_t tokens, int64_t d_out, dora_dtype dt, void* y, void* stream);

/* dora_compose_fwd for a base layer with a bias b:
 *
 *   y = base + (delta * (base - b) + g * s * lora) = b + g * ((base - b) + s * lora)
 *
 * base_out is the frozen base layer's output x W^T + b.  bias: [d_out] in dt
 * (bf16: 16-byte aligned; fp32: 4-byte aligned), or NULL, which is exactly
 * dora_compose_fwd.  The pages never mention a bias; the rescaling is taken to
 * act on the weight's product only, as the DoRA summary page's Method defines
 * the adapted weight m V / ||V||. */
DORA_API int dora_compose_fwd_bias(const void* base_out, const void* lora_out, const void* bias, const float* m,
                                   const float* n, float s, int64_t tokens, int64_t d_out, dora_dtype dt, void* y,
                                   void* stream);

/* Bytes of workspace dora_compose_bwd needs: per-chunk partial sums of d_m
 * over tokens, O(d_out), independent of tokens beyond a bounded chunk count
 * (the single-pass backward of Scaling DoRA, Abstract, keeps no
 * [tokens, d_out] intermediate). */
DORA_API size_t dora_compose_bwd_workspace_size(int64_t tokens, int64_t d_out);

/* Backward of dora_compose_fwd with n held constant (the norm is detached;
 * Scaling DoRA, Abstract: the fused compose serves the forward pass and the
 * gradients; DoRA summary page, Method: the gradient of the magnitude m and
 * of the direction's low-rank factors):
 *
 *   d_base = g * dy,   d_lora = s * g * dy,
 *   d_m_i  = (sum_t dy[t,i] * (base[t,i] + s * lora[t,i])) / n_i
 *
 * d_base, d_lora: [tokens, d_out] in dt, overwritten.  d_m: fp32 [d_out],
 * overwritten (tokens == 0 gives d_m = 0).  The token reduction accumulates
 * in fp32 and combines per-chunk partials in a fixed order. */
DORA_API int dora_compose_bwd(const void* dy, const void* base_out, const void* lora_out, const float* m,
                              const float* n, float s, int64_t tokens, int64_t d_out, dora_dtype dt, void* d_base,
                              void* d_lora, float* d_m, void* workspace, size_t workspace_bytes, void* stream);

/* Backward of dora_compose_fwd_bias (bias frozen, no gradient returned for it):
 * as dora_compose_bwd with d_m_i = (sum_t dy[t,i] * ((base[t,i] - b_i) +
 * s * lora[t,i])) / n_i.  bias as in dora_compose_fwd_bias; NULL is exactly
 * dora_compose_bwd. */
DORA_API int dora_compose_bwd_bias(const void* dy, const void* base_out, const void* lora_out, const void* bias,
                                   const float* m, const float* n, float s, int64_t tokens, int64_t d_out,
                                   dora_dtype dt, void* d_base, void* d_lora, float* d_m, void* workspace,
                                   size_t workspace_bytes, void* stream);

/* Largest d_out dora_compose_bwd_noalloc accepts, and the size of the
 * library-owned scratch array behind it (16 KiB of counters + 16 row chunks of
 * fp32 column partials). */
#define DORA_NOALLOC_MAX_D_OUT 32768
#define DORA_NOALLOC_SCRATCH_BYTES (16384 + 16 * 4 * DORA_NOALLOC_MAX_D_OUT)

/* dora_compose_bwd for callers that cannot allocate device memory at call
 * time and so cannot provide a workspace: code recorded into a CUDA graph or
 * run under a runtime whose memory is fixed after initialisation, hot loops
 * that must not call cudaMalloc/cudaFree, or foreign-language callers that
 * only hold the tensors themselves.  This entry point has no counterpart on
 * the pages; it computes exactly what dora_compose_bwd computes, with the
 * same arguments minus the workspace.
 *
 * Its scratch lives in one file-scope device array of
 * DORA_NOALLOC_SCRATCH_BYTES inside the library: every GPU that loads the
 * library holds it until the process exits.  Nothing is allocated: no
 * cudaMalloc, cudaFree or allocating library routine is called.  The first
 * call on a device looks the array's device address up (cudaGetSymbolAddress)
 * with that device current; make that first call before any stream capture.
 * The address is kept per device and per CUDA context: after the context is
 * destroyed and created again (cudaDeviceReset), the next call looks it up
 * afresh, so make that call before any capture too.
 * Nothing is cleared before a call either: the arrival counters in the array
 * carry a per-call tag, so whatever they hold is ignored, and the array
 * keeps the last call's contents.  All calls on a device
 * share the one array, so calls whose executions overlap on the GPU (for
 * example on two streams without ordering between them) race and give wrong
 * results; order them on one stream.  d_out > DORA_NOALLOC_MAX_D_OUT returns
 * DORA_ERR_UNSUPPORTED and launches nothing. */
DORA_API int dora_compose_bwd_noalloc(const void* dy, const void* base_out, const void* lora_out, const float* m,
                                      const float* n, float s, int64_t tokens, int64_t d_out, dora_dtype dt,
                                      void* d_base, void* d_lora, float* d_m, void* stream);

/* dora_compose_bwd_bias with the library-owned scratch of
 * dora_compose_bwd_noalloc (same rules); NULL bias is exactly
 * dora_compose_bwd_noalloc. */
DORA_API int dora_compose_bwd_noalloc_bias(const void* dy, const void* base_out, const void* lora_out,
                                           const void* bias, const float* m, const float* n, float s, int64_t tokens,
                                           int64_t d_out, dora_dtype dt, void* d_base, void* d_lora, float* d_m,
                                           void* stream);

/* Bytes of workspace dora_factored_norm_bwd needs: O(r^2 + r d_out), no
 * d_out x d_in term (the Gram partial tiles, s G and s^2 H in bf16, and two
 * [r, d_out] bf16 copies of B), as the factored norm's intermediates are
 * (Scaling DoRA, Abstract). */
DORA_API size_t dora_factored_norm_bwd_workspace_size(int64_t d_out, int64_t d_in, int64_t r);

/* Gradients of the row norms n_i = ||W_i + s B_i A|| into A and B, for
 * training with the norm kept attached (Scaling DoRA, Abstract: gradients
 * through the factored norm; the default DoRA backward, dora_compose_bwd,
 * holds n constant).  With c = d_n / n and never forming B A:
 *
 *   dB = s c * (W A^T + s B G),            G = A A^T
 *   dA = s (c * B)^T W + s^2 H A,          H = (c * B)^T B
 *
 * computed as a Gram product and a CTA-pair tcgen05 GEMM for each (dB:
 * [W | B] [A | s G]^T with a per-row epilogue scale; dA: [(s c B)^T | s^2 H]
 * [W ; A], W read N-contiguous), G, H and (s c B)^T rounded to bf16, fp32
 * accumulation.
 *
 * W: [d_out, d_in]; A: [r, d_in]; B: [d_out, r]; bf16, row-major, 16-byte
 * aligned; d_in, d_out, r multiples of 8.  n: fp32 [d_out], the forward's
 * norms (not recomputed); d_n: fp32 [d_out], the upstream gradient of n (for
 * the DoRA compose y = (m / n) (base + s lora) it is -(m / n) * d_m).  dA:
 * fp32 [r, d_in]; dB: fp32 [d_out, r]; both overwritten with the gradients
 * through the norm alone (the caller adds the LoRA path's own gradients); W
 * gets none.  r = 0 does nothing; d_out = 0 zeroes dA; d_in = 0 zeroes dB.
 * workspace: at least dora_factored_norm_bwd_workspace_size() bytes,
 * 256-byte aligned, contents ignored.  Only DORA_BF16.  Asynchronous on
 * `stream` (five launches: the prep copies, one Gram launch for G and H, its
 * reduction, the dB and the dA GEMMs). */
DORA_API int dora_factored_norm_bwd(const void* W, const void* A, const void* B, float s, const float* n,
                                    const float* d_n, int64_t d_out, int64_t d_in, int64_t r, dora_dtype dt,
                                    float* dA, float* dB, void* workspace, size_t workspace_bytes, void* stream);

/* Bytes of workspace dora_fused_linear_fwd needs: the [tokens, r] bf16
 * intermediate P = s * x A^T (at least 256), the LoRA branch's down
 * projection (DoRA summary page, Method: the low-rank update B A). */
DORA_API size_t dora_fused_linear_fwd_workspace_size(int64_t tokens, int64_t r);

/* The DoRA linear forward with the compose fused into the GEMMs that produce
 * its inputs (Scaling DoRA, Abstract: the composition collapsed into one pass
 * over the activations; here the pass is the GEMM epilogue itself, so the
 * base and LoRA outputs are never written to memory):
 *
 *   y = b + g * (x W^T + s * (x A^T) B^T),   g = m / n   per output channel
 *
 * computed as P = bf16(s * x A^T) (one tcgen05 GEMM into the workspace), then
 * y = bf16(g * [x | P] [W | B]^T + b) (one tcgen05 GEMM whose K runs over d_in
 * and then r; fp32 accumulation, g and b applied in fp32, one rounding).
 * This equals dora_compose_fwd applied to base = x W^T + b and
 * lora = (x A^T) B^T, except that P is rounded to bf16 once, as a framework's
 * LoRA path rounds x A^T.
 *
 * x: [tokens, d_in]; W: [d_out, d_in]; A: [r, d_in]; B: [d_out, r]; y:
 * [tokens, d_out]; all bf16, row-major, 16-byte aligned; d_in, d_out, r
 * multiples of 8; d_in > 0.  bias: bf16 [d_out] or NULL.  m, n: fp32
 * [d_out] (n from dora_factored_norm).  r = 0 gives y = b + g * x W^T (no
 * workspace needed).  workspace: device buffer of at least
 * dora_fused_linear_fwd_workspace_size(tokens, r) bytes, 256-byte aligned,
 * contents ignored on entry.  Only dt = DORA_BF16 is accepted
 * (DORA_ERR_UNSUPPORTED otherwise).  Asynchronous on `stream`; tokens == 0 or
 * d_out == 0 launches nothing.  y must not overlap the inputs. */
DORA_API int dora_fused_linear_fwd(const void* x, const void* W, const void* A, const void* B, const void* bias,
                                   const float* m, const float* n, float s, int64_t tokens, int64_t d_in,
                                   int64_t d_out, int64_t r, dora_dtype dt, void* y, void* workspace,
                                   size_t workspace_bytes, void* stream);

/* Human-readable name of a dora_status value (static storage). */
DORA_API const char* dora_status_string(int status);

/* Reads and clears the device-side status word of the current device
 * (DORA_OK or DORA_ERR_TIMEOUT).  Synchronises `stream` first. */
DORA_API int dora_device_status(void* stream);

/* Self-test of the failure path; no counterpart on the pages.  Launches one
 * warp that waits on an mbarrier phase nothing completes, bounded by
 * limit_cycles SM cycles (1 .. 2e9; about 1 s at 2 GHz), then records
 * DORA_ERR_TIMEOUT in the device-side status word exactly as a real bounded
 * wait that gives up does.  dora_device_status() then returns (and clears)
 * DORA_ERR_TIMEOUT; the context stays usable.  Asynchronous on `stream`.
 * Returns DORA_ERR_INVALID_ARG for a limit outside that range. */
DORA_API int dora_selftest_timeout(int64_t limit_cycles, void* stream);

/* Number of SMs the persistent kernels size their grids to on the current
 * device (the grid is a multiple of this count).  Returns 0 when no device. */
DORA_API int dora_num_sms(void);

/* Kernels this library has launched in this process, on any device and
 * stream (a host-side count, incremented as each launch is enqueued; a
 * launch that fails still counts).  For a caller that counts the library's
 * GPU work over a region: read it before and after. */
DORA_API uint64_t dora_launch_count(void);

#ifdef __cplusplus
}
#endif

#endif /* DORA_H_ */
