/*
 * libcta - certified Top-k attention truncation on NVIDIA B200 (sm_100a).
 *
 * The method: "A Mathematical Theory of Top-k Sparse Attention via Total
 * Variation Distance" (Tzachristas et al., arXiv 2512.07647), abstract.  For
 * one attention distribution P = softmax(s), s_i = q.k_i / sqrt(d), the Top-k
 * truncation P-hat keeps the k largest logits and renormalises them; the
 * total-variation distance TV(P, P-hat) equals the discarded softmax tail mass
 * and equals 1 - exp(-KL(P-hat || P)); certified Top-k uses the minimal k_eps
 * with TV(P, P-hat) <= eps; the output error factorises as
 * ||Attn - Attn_k||_2 = tau ||mu_tail - mu_head||_2 with tau = TV.
 *
 * Conventions shared by every entry point
 *   - Rows.  One row is one (batch b, query head h, query j); rows are numbered
 *     row = (b * n_heads + h) * m + j.
 *   - Layouts (row-major, contiguous, no strides):
 *       q, out : [batch, n_heads, m, d]
 *       K, V   : [batch, n_kv_heads, n, d]
 *     Query head h reads KV head h / (n_heads / n_kv_heads) (grouped-query
 *     attention; n_kv_heads = n_heads is plain multi-head attention).
 *   - Element type of q, K, V and out: cta_opts.dtype (fp32 or bf16).
 *   - Every pointer is device memory owned by the caller.  The library never
 *     allocates device or pinned memory and keeps no state between calls.
 *   - Calls are asynchronous on cta_opts.stream: the return value reports
 *     argument and launch errors only.  Conditions found on the device (a
 *     non-finite logit, a broken internal invariant) are OR-ed as bits into
 *     *cta_opts.status_dev when that pointer is given.  No device code traps.
 *   - For bf16 inputs with d = 128 the four kernels of a call are launched
 *     with programmatic stream serialization (each may become resident while
 *     the one before it finishes).  The first waits for the kernel before it
 *     on the stream to complete (griddepcontrol.wait) before it reads q or K
 *     or writes anything; V is read only after the first has completed.  So a
 *     caller's kernel that writes q, K or V right before the call is ordered
 *     before every read, whether or not it triggers its dependents early.
 *   - Supported: d in {64, 128}; 1 <= n <= 2^28; 0 < eps < 1;
 *     n_heads % n_kv_heads == 0; batch, m >= 1.  There is no mask: every row
 *     sees all n keys.  The logit scale is 1/sqrt(d).
 */
#ifndef CTA_H
#define CTA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum { CTA_F32 = 0, CTA_BF16 = 1 } cta_dtype;

typedef enum {
  CTA_OK = 0,
  CTA_ERR_ARG = -1,         /* NULL pointer, eps outside (0,1), bad count     */
  CTA_ERR_SHAPE = -2,       /* unsupported d, n_heads % n_kv_heads != 0, n    */
  CTA_ERR_WORKSPACE = -3,   /* workspace missing, misaligned or too small     */
  CTA_ERR_CUDA = -4,        /* a CUDA launch or runtime call failed           */
  CTA_ERR_NONFINITE = -5,   /* reserved for host-side reporting of bit 1      */
  CTA_ERR_TIMEOUT = -6,     /* reserved for host-side reporting of bit 4      */
  CTA_ERR_TOO_LARGE = -7    /* needs more scratch than CTA_NOALLOC_SCRATCH_BYTES */
} cta_status;

/* Bits OR-ed into *cta_opts.status_dev by device code. */
#define CTA_DEV_NONFINITE 0x1u  /* a logit was NaN or infinite: outputs of that row are meaningless */
#define CTA_DEV_INTERNAL 0x2u   /* an internal consistency check failed (a library bug)            */
#define CTA_DEV_TIMEOUT 0x4u    /* a pipeline wait in a kernel gave up after ~2 s (results invalid) */

/* Optional arguments.  Initialise with cta_opts_init() and override fields. */
typedef struct {
  int32_t batch;          /* batch size; default 1                                          */
  int32_t m;              /* query rows per head; default 1 (decode)                        */
  int32_t dtype;          /* cta_dtype of q, K, V, out; default CTA_BF16                     */
  int32_t reserved0;
  void* stream;           /* cudaStream_t to launch on; NULL = legacy default stream         */
  void* workspace;        /* device scratch of >= cta_workspace_size() bytes, 256-B aligned  */
  size_t workspace_bytes; /* its size                                                        */
  float* err_out;         /* [batch, n_heads, m] exact head-tail error tau*||mu_t - mu_h||,
                             or NULL (then the value rows of dropped keys are never read)    */
  float* kl_out;          /* [batch, n_heads, m] KL(P-hat || P) = log(sum_all w / sum_head w)
                             from the output pass, or NULL                                   */
  uint32_t* status_dev;   /* device word for CTA_DEV_* bits, or NULL                         */
  void** phase_events;    /* NULL, or 5 cudaEvent_t recorded on the stream (for timing the
                             kernels one by one; an event between two kernels keeps the second
                             from starting early).  bf16 with d = 128 (the tensor-core decode
                             path): before the logits pass, after it, after the row brackets,
                             after the value pass and after the last kernel (cut, indices,
                             outputs).  Other shapes: before the score phase, after it, after
                             selection, after the output pass and after finalisation.          */
  float* gap_out;         /* [batch, n_heads, m] single-gap certificate, or NULL: with
                             u_(k) the last kept and u_(k+1) the largest dropped logit,
                             1 / (1 + k/(n-k) exp((u_(k) - u_(k+1)) / sqrt(d))), an upper
                             bound on TV from the ordering alone (head logits >= u_(k), tail
                             logits <= u_(k+1)); 0 when every key is kept.  The page "A
                             Mathematical Theory of Top-k Sparse Attention via Total Variation
                             Distance" (abstract) names deterministic bounds from ordered
                             logits (single gap first) without printing them; this is the
                             single-gap form derived from that ordering.                      */
} cta_opts;

/* Fill *o with the defaults listed above. */
void cta_opts_init(cta_opts* o);

/*
 * Bytes of device workspace cta_certified_topk_attn needs for this shape
 * (batch, m and dtype are taken from o; NULL = defaults).  Returns 0 for an
 * unsupported shape.  The workspace holds the fp32 logits of every row
 * (4 * rows * n bytes) plus per-row and per-range records; for bf16 with
 * d = 128 also per-range level histograms (6.6 KB per row and key range),
 * a candidate list per row (16 KB) and one bit per key and row.
 */
size_t cta_workspace_size(int64_t n, int d, int n_heads, int n_kv_heads, const cta_opts* o);

/*
 * Certified Top-k attention (paper abstract: minimal k_eps with
 * TV(P, P-hat) <= eps; Attn_k over the kept keys; tau = TV; head-tail error).
 *
 * For every row: logits s_i = q.k_i / sqrt(d) for all n keys; the keys ranked
 * by logit, descending, ties broken by the lower key index; k_eps = the least
 * k whose discarded tail mass TV = sum_{dropped} P_i is <= eps; the output
 * Attn_k = mu_head = sum_{kept} P_i v_i / sum_{kept} P_i.
 *
 *   q, K, V   inputs, layouts above, element type opts->dtype.
 *   n, d      keys per KV head, head dimension.
 *   eps       TV budget, 0 < eps < 1.
 *   out       [batch, n_heads, m, d]  Attn_k, element type opts->dtype.
 *   k_out     [batch, n_heads, m]     k_eps (int32, 1..n).
 *   idx_out   [batch, n_heads, m, n]  int32; entries [0, k_out) of each row are
 *             the kept key indices in ascending order; the rest are not written.
 *   tv_out    [batch, n_heads, m]     TV = discarded tail mass (<= eps).
 *   opts      optional arguments; workspace is required (see above).
 *
 * Numerics: logits are fp32 dot products (bf16 inputs widen exactly); the
 * ranking uses them.  Softmax numerators w_i = exp(s_i - max s) are fp32 and
 * are summed exactly as fixed-point integers (units of 2^-62 in 128-bit sums
 * for bf16 with d = 128; otherwise a 64-bit scale chosen per row from its
 * mass), so the k_eps decision, TV and the kept set do not depend on the
 * reduction order and the rounding of the n numerators moves the total by
 * at most n * 2^-62 of it; the decision is taken in fp64 as
 * (Z - C_k) / Z <= eps.  Output sums accumulate in fp32 over
 * short runs and in fp64 across them.  Results are bit-reproducible.
 * Returns a cta_status.
 */
int cta_certified_topk_attn(const void* q, const void* K, const void* V, int64_t n, int d,
                            int n_heads, int n_kv_heads, double eps, void* out, int32_t* k_out,
                            int32_t* idx_out, float* tv_out, const cta_opts* opts);

/*
 * Dense softmax attention Attn(q, K, V) = sum_i P_i v_i over all keys, the
 * reference output that the head-tail error is measured against.  Same
 * layouts and dtype rules; needs no workspace.  Returns a cta_status.
 */
int cta_dense_attn(const void* q, const void* K, const void* V, int64_t n, int d, int n_heads,
                   int n_kv_heads, void* out, const cta_opts* opts);

/*
 * Certified Top-k attention without any device allocation.  The paper has no
 * counterpart: this is a deployment variant of cta_certified_topk_attn.
 *
 * For callers that cannot call cudaMalloc (for example while a CUDA graph is
 * being captured, inside runtimes that forbid allocation outside their own
 * memory pool, or under a device-memory budget fixed at start-up) and so
 * cannot pass a workspace.  Same arguments, layouts, results and status codes
 * as cta_certified_topk_attn; opts->workspace and opts->workspace_bytes are
 * ignored.  The scratch is a fixed array of CTA_NOALLOC_SCRATCH_BYTES inside
 * the library (32 MiB: enough for the 32K and 128K decode workloads of this
 * library; about 4 * batch * n_heads * m * n bytes plus small records are
 * needed, see cta_workspace_size).  Larger problems return CTA_ERR_TOO_LARGE
 * before anything is launched.
 *
 *   - The array takes 32 MiB of device memory on every GPU where the library's
 *     module is loaded, until the process exits.
 *   - The first call on a device (with that device current) looks up the
 *     array's device address and caches it; make that first call before any
 *     stream capture.
 *   - Every call on a device shares the one array: calls that may overlap on
 *     the GPU (different streams without ordering, or several host threads)
 *     race and corrupt each other's results.  Order them on one stream.
 *   - No cudaMalloc, cudaFree or allocating library routine is called.
 */
#define CTA_NOALLOC_SCRATCH_BYTES ((size_t)32 << 20)
int cta_certified_topk_attn_noalloc(const void* q, const void* K, const void* V, int64_t n, int d,
                                    int n_heads, int n_kv_heads, double eps, void* out,
                                    int32_t* k_out, int32_t* idx_out, float* tv_out,
                                    const cta_opts* opts);

/* Static text for a cta_status value. */
const char* cta_status_string(int status);

/* Library version, major * 10000 + minor * 100 + patch. */
int cta_version(void);

#ifdef __cplusplus
}
#endif

#endif /* CTA_H */
