/*
 * spark.h -- C ABI of libspark.so: the Spark FFN forward pass with statistical
 * top-k, the standalone statistical top-k operator (plain, causally masked and
 * Huber-smoothed with its gradient) and Spark Attention for one decoding
 * position, on NVIDIA B200 (sm_100a).
 *
 * Method source: the paper-notes page "Spark Transformer: Reactivating Sparsity
 * in FFN and Attention" (NeurIPS 2025, arXiv 2506.06644), section 方法详解 /
 * 关键设计, items "Spark FFN", "Statistical Top-k" and "Spark Attention".
 * Notation follows it:
 *
 *   x      = K1^T q[:r]                                   (low-rank predictor)
 *   theta  = mean(x) + std(x) * Q(1 - k/d_ff)             (Q: standard-normal quantile)
 *   s      = max(x - theta, 0)                            (Soft-Threshold)
 *   out    = V . (GELU(s) (.) (K2^T q[r:]))               (only neurons with x > theta)
 *
 * Readings fixed by this library where the page is silent: std is the
 * population standard deviation (as in LayerNorm); GELU is the tanh form; a
 * neuron is active iff x > theta (strict); the number of active neurons is
 * whatever theta selects (no truncation or top-up to exactly k); a row with
 * zero spread selects nothing.
 *
 * Conventions for every entry point:
 *   - All tensor pointers are DEVICE pointers owned by the caller, row-major,
 *     and must stay valid until the work enqueued on `stream` has finished
 *     (spark_ffn_forward_host alone takes q and out in host memory).
 *   - Every call is asynchronous on `stream` (a cudaStream_t; NULL = the legacy
 *     default stream) and returns once the work is enqueued.  Argument errors
 *     are detected on the host before anything is enqueued.
 *   - bf16 means IEEE binary32 truncated to its top 16 bits (__nv_bfloat16).
 *     Scores x and all accumulation are fp32; out is rounded to bf16 (RNE).
 *   - The library keeps a lazily grown scratch workspace per (device, stream),
 *     allocated with cudaMallocAsync on `stream`.  Growing it inside a CUDA
 *     graph capture is refused (SPARK_ENOMEM): make one call of the largest
 *     size first.  spark_release_workspace() frees it.
 *   - Calls made on different streams use different workspaces and may run
 *     concurrently.
 *   - Errors found by a kernel (a bounded wait that ran out) are recorded in a
 *     device status word and reported by spark_query_status(); kernels never
 *     trap.  After such an error, later launches on that stream return without
 *     computing until spark_query_status() has been called.
 */
#ifndef SPARK_H_
#define SPARK_H_

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define SPARK_API __attribute__((visibility("default")))
#else
#define SPARK_API
#endif

/* Same object as cudaStream_t, declared here so that this header needs no CUDA header. */
typedef struct CUstream_st* spark_stream_t;

typedef enum {
  SPARK_OK = 0,
  SPARK_EINVAL = -1,   /* NULL pointer, size out of range, aliasing output, unsupported shape */
  SPARK_EALIGN = -2,   /* pointer not 16-byte aligned, or r / d_model not a multiple of 8 */
  SPARK_ECUDA = -3,    /* a CUDA runtime call or kernel launch failed */
  SPARK_ENOMEM = -4,   /* workspace could not be allocated (or growth requested during capture) */
  SPARK_ETIMEOUT = -5, /* a device-side bounded wait ran out (reported by spark_query_status) */
  SPARK_EDEVICE = -6,  /* current device is not compute capability 10.x (B200 / sm_100a) */
  SPARK_ESCRATCH = -7, /* spark_ffn_forward_noalloc: problem needs more than its fixed scratch */
  SPARK_EBOUNDS = -8   /* bounds-check build only: a kernel index check failed (spark_query_status) */
} spark_status;

/*
 * Spark FFN forward for one token (decode, T = 1).
 *   q   : bf16 [d_model]          (q[:r] feeds the predictor, q[r:] the value path)
 *   K1  : bf16 [d_ff][r]          row i is neuron i's predictor key: x_i = <K1[i,:], q[:r]>
 *   K2  : bf16 [d_ff][d_model-r]  row i is neuron i's compute key
 *   V   : bf16 [d_ff][d_model]    row i is neuron i's value row
 *   out : bf16 [d_model]          must not overlap any input
 *   k   : target number of active neurons, 0 < k < d_ff
 * Requires 0 < r < d_model, r % 8 == 0, d_model % 8 == 0, all pointers 16-byte aligned.
 * Returns SPARK_OK or an error code; see "Spark FFN" in the page's 关键设计.
 */
SPARK_API int spark_ffn_forward(const void* q, const void* K1, const void* K2, const void* V,
                                int d_model, int r, int d_ff, int k, void* out,
                                spark_stream_t stream);

/*
 * Same as spark_ffn_forward over n_tokens independent tokens (batched prefill):
 * q and out are bf16 [n_tokens][d_model]; every token gets its own threshold and
 * active set.  n_tokens == 0 is a no-op returning SPARK_OK; n_tokens < 0 is
 * SPARK_EINVAL.
 *
 * Which weight rows are read: up to 4 tokens, all of K1 and only the rows of K2
 * and V that some token's active set uses.  From 5 tokens on, the tensor-core
 * path reads all of K1, K2 and V in dense tiles (the masked products multiply
 * zero h entries): the union of independent tokens' active sets covers most
 * neurons from a few tokens on (1 - (1 - k/d_ff)^T), and reading only the
 * union's rows -- gathered, or zeroed in shared memory before the product --
 * measured slower than the dense tiles on B200 at every prompt length.  So from
 * 5 tokens on every row of K2 and V must be finite: a NaN or Inf in a row that no
 * token uses still reaches out (0 * NaN is NaN).
 */
SPARK_API int spark_ffn_forward_tokens(const void* q, const void* K1, const void* K2,
                                       const void* V, int n_tokens, int d_model, int r, int d_ff,
                                       int k, void* out, spark_stream_t stream);

/*
 * spark_ffn_forward_tokens with q and out in HOST memory: copies q (bf16
 * [n_tokens][d_model]) to a device buffer, runs the forward, and copies out
 * back, all enqueued on `stream` (one H2D copy, the kernels, one D2H copy).
 * The weights are device pointers as above.  Like any asynchronous copy, q_host
 * must stay unchanged, and out_host unread, until the stream has passed the
 * call: synchronise the stream before reading out_host.  For the call to be
 * asynchronous the host buffers must be pinned (cudaHostAlloc /
 * cudaHostRegister); with pageable memory the CUDA runtime stages them and the
 * call returns only after the output copy has completed.  For one token, with
 * both buffers pinned and mapped for the current device (as unified addressing
 * makes them) and q_host 16-byte aligned, no copy engine is used: the call's
 * first kernel reads q from host memory and its last kernel stores out there.  The device buffers
 * (2 n_tokens d_model bf16) belong to the library, one pair per device and
 * stream, grown like the workspace (so not inside a stream capture) and freed
 * by spark_release_workspace.  Same argument checks and errors as
 * spark_ffn_forward_tokens (q_host and out_host need no alignment but may not
 * overlap), all made before anything is enqueued.
 */
SPARK_API int spark_ffn_forward_host(const void* q_host, const void* K1, const void* K2, const void* V,
                                     int n_tokens, int d_model, int r, int d_ff, int k, void* out_host,
                                     spark_stream_t stream);

/*
 * spark_ffn_forward_tokens that also returns the intermediate values it used,
 * for parity checks.  Each extra output may be NULL:
 *   x_out      : fp32 [n_tokens][d_ff]   predictor scores x (16-byte aligned, else SPARK_EALIGN)
 *   theta_out  : fp32 [n_tokens]         thresholds theta
 *   active_out : uint8 [n_tokens][d_ff]  1 where x > theta (the neuron was used), else 0
 * The kernels and arithmetic are the same as spark_ffn_forward_tokens.
 */
SPARK_API int spark_ffn_forward_debug(const void* q, const void* K1, const void* K2, const void* V,
                                      int n_tokens, int d_model, int r, int d_ff, int k, void* out,
                                      float* x_out, float* theta_out, unsigned char* active_out,
                                      spark_stream_t stream);

/*
 * The low-rank predictor alone ("Spark FFN": x = K1^T q[:r]) for n_tokens
 * tokens: x_out[t][i] = <K1[i,:], q[t][:r]>, fp32 [n_tokens][d_ff], 16-byte
 * aligned, not overlapping q or K1.  The same tensor-core GEMM (bf16 operands,
 * fp32 accumulation) as the predictor stage of batched prefill.  q is bf16
 * [n_tokens][d_model] (only q[:, :r] is read), K1 bf16 [d_ff][r].  Requires
 * 0 < r < d_model, r and d_model multiples of 8, d_ff a multiple of 16
 * (else SPARK_EALIGN).  n_tokens == 0 is a no-op.
 */
SPARK_API int spark_ffn_predictor(const void* q, const void* K1, int n_tokens, int d_model, int r, int d_ff,
                                  float* x_out, spark_stream_t stream);

/*
 * A decoder stack of Spark FFN layers for one token (decode).  Between layers it
 * applies the pre-norm residual of a Gemma-style stack (the notes place Spark FFN
 * inside a Gemma-2 model but do not spell this out; it is how the layers chain):
 *   for l = 0 .. n_layers-1:
 *     q_l     = bf16(h_l / sqrt(mean(h_l^2) + eps))        (RMSNorm, unit gain)
 *     h_{l+1} = h_l + SparkFFN_l(q_l)                       (fp32 residual, bf16 FFN output)
 *   h_in  : fp32 [d_model], h_0;  h_out : fp32 [d_model], h_{n_layers} (may equal h_in);
 *           both 16-byte aligned
 *   K1s, K2s, Vs : HOST arrays of n_layers DEVICE pointers, each as in spark_ffn_forward
 *   q_dbg, out_dbg : optional bf16 [n_layers][d_model]: every q_l and SparkFFN_l(q_l)
 * Each layer runs the single-token kernel chain (score, gather, reduce): the
 * score kernel forms q_l from h_l itself and the reduce kernel writes h_{l+1}.
 * Requires the single-token kernels to support the shape (the Gemma-2-2B shape
 * does), else SPARK_EINVAL.
 */
SPARK_API int spark_ffn_decode_stack(const float* h_in, float* h_out, const void* const* K1s,
                                     const void* const* K2s, const void* const* Vs, int n_layers,
                                     int d_model, int r, int d_ff, int k, float eps, void* q_dbg,
                                     void* out_dbg, spark_stream_t stream);

/*
 * Spark Attention for one decoding position (the page's "Spark Attention": the
 * key vectors split into a predictor part K1 = K[:, :r] and K2 = K[:, r:];
 * statistical top-k over the predictor scores with k_attn keys per query;
 * sigma_1 = softmax, sigma_2 = softplus).  For query head h and its key/value
 * head g = h / (n_heads / n_kv_heads):
 *   s_j    = scale * <K[g][j][:r], q[h][:r]>                      (j < n_ctx)
 *   theta  = mean(s) + std(s) * Q(1 - k_attn/n_ctx)   (population std; when
 *            k_attn >= n_ctx every key is selected)
 *   out[h] = sum_{s_j > theta} softmax_j(s) * softplus(<K[g][j][r:], q[h][r:]>) * V[g][j][:]
 * with the softmax over the selected keys only (readings: the page names the
 * two functions but not where the softmax runs; over all keys it would attend
 * densely).  An empty selection (zero spread) gives out[h] = 0.
 *   q    : bf16 [n_heads][d_head]
 *   K, V : bf16 [n_kv_heads][n_ctx][d_head] (row-major, one row per cached position)
 *   out  : bf16 [n_heads][d_head]; must not overlap q, K or V
 *   scale: the attention temperature (> 0, finite), e.g. 1/sqrt(d_head)
 * Requires n_heads % n_kv_heads == 0, 1 <= n_ctx <= 65536, k_attn >= 1,
 * 0 < r < d_head <= 256 with r and d_head multiples of 8 (else SPARK_EINVAL /
 * SPARK_EALIGN), and 16-byte aligned pointers.  One launch; needs no workspace.
 */
SPARK_API int spark_attention_decode(const void* q, const void* K, const void* V, int n_heads, int n_kv_heads,
                                    int n_ctx, int d_head, int r, int k_attn, float scale, void* out,
                                    spark_stream_t stream);

/* spark_attention_decode, also returning (any may be NULL): s_out fp32
 * [n_heads][n_ctx] (scaled predictor scores), theta_out fp32 [n_heads]
 * (-inf when every key is selected), active_out bytes [n_heads][n_ctx]
 * (1 where s > theta). */
SPARK_API int spark_attention_decode_debug(const void* q, const void* K, const void* V, int n_heads, int n_kv_heads,
                                          int n_ctx, int d_head, int r, int k_attn, float scale, void* out,
                                          float* s_out, float* theta_out, unsigned char* active_out,
                                          spark_stream_t stream);

/*
 * Standalone statistical top-k with soft threshold ("Statistical Top-k"):
 * for every row of x (fp32 [rows][d]), theta = mean + std * Q(1 - k/d) and
 * out = max(x - theta, 0) (fp32 [rows][d]).  out may equal x (in place); any
 * other overlap is SPARK_EINVAL.  Any d >= 2 is accepted (rows need not be
 * 16-byte aligned; aligned rows with d % 4 == 0 take the vectorised path).
 * Requires 0 < k < d.  rows == 0 is a no-op.
 */
SPARK_API int stat_topk_soft_threshold(const float* x, int rows, int d, int k, float* out,
                                       spark_stream_t stream);

/*
 * Huber-smoothed statistical top-k ("Statistical Top-k", Theorem 3.2: with a
 * Huber smoothing the operator is continuously differentiable, for training).
 * Reading of the smoothing: the ramp max{z, 0} of Soft-Threshold becomes
 *   rho(z) = 0 (z <= 0),  z^2 / (2 delta) (0 < z < delta),  z - delta/2 (z >= delta)
 * with z = x - theta(x), theta = mean + std * Q(1 - k/d) per row (population
 * std); delta = 0 is the plain operator (stat_topk_soft_threshold).
 *   stat_topk_huber:          out = rho(x - theta(x)), fp32 [rows][d]; out may equal x.
 *   stat_topk_huber_backward: the gradient for an upstream gradient grad_out
 *     (fp32 [rows][d]) of that output:
 *       grad_x_j = w_j - W (1/d + Q (x_j - mean) / (d std)),
 *       w = grad_out * rho'(x - theta),  W = sum_j w_j
 *     (theta itself depends on every x_j through the row's mean and std; a
 *     row with zero spread gets zero gradient).  grad_x may equal x or
 *     grad_out (in place); other overlaps are SPARK_EINVAL.
 * Require 0 < k < d, d >= 2, finite delta >= 0 and 4-byte aligned pointers.
 * rows == 0 is a no-op.
 */
SPARK_API int stat_topk_huber(const float* x, int rows, int d, int k, float delta, float* out, spark_stream_t stream);
SPARK_API int stat_topk_huber_backward(const float* x, const float* grad_out, int rows, int d, int k, float delta,
                                       float* grad_x, spark_stream_t stream);

/*
 * Statistical top-k with soft threshold on causally masked score rows ("Spark
 * Attention": each token attends to at most k tokens, so a query at position
 * p works on min{k, p + 1} keys).  Row r of x (fp32 [rows][d]) is query
 * r % n_q of its head, at position pos = offset + r % n_q, and sees its first
 * n = min(d, pos + 1) entries:
 *   k <  n: theta = mean + std * Q(1 - k/n) over those n entries (population
 *           std), out = max(x - theta, 0) on them;
 *   k >= n: every visible entry is kept: out = x on them, theta = -inf.
 * Masked entries (index >= n) are written as 0 and do not influence the
 * result (a row's last visible 16-byte group may be read whole).  theta_out
 * (fp32 [rows], may be NULL) receives theta.  For the square causal scores of
 * one prompt, n_q = d and offset = 0; for the last n_q queries of a longer
 * context, offset = d - n_q.  out may equal x (in place); other overlaps are
 * SPARK_EINVAL.  Requires k >= 1, n_q >= 1, offset >= 0, d >= 1, 4-byte
 * aligned pointers.  rows == 0 is a no-op.
 */
SPARK_API int stat_topk_soft_threshold_causal(const float* x, int rows, int d, int k, int n_q, int offset,
                                              float* out, float* theta_out, spark_stream_t stream);

/*
 * Synchronises `stream`, then returns and clears the device status of the
 * workspace used on that stream: SPARK_OK, SPARK_ETIMEOUT, or SPARK_ECUDA if
 * the stream reported a CUDA error.  In the bounds-check build
 * (libspark_debug.so) it returns SPARK_EBOUNDS when no other error is pending
 * and a kernel of the current device has counted a failed index check since
 * the last spark_debug_violations(), which reads and clears that count.
 */
SPARK_API int spark_query_status(spark_stream_t stream);

/* Synchronises the devices involved and frees every workspace.  Not thread-safe
 * with respect to concurrent calls of the other entry points. */
SPARK_API int spark_release_workspace(void);

/* Human-readable name of a status code (static string). */
SPARK_API const char* spark_status_string(int status);

/* Q(1 - k/d) as the library computes it on the host, in double precision
 * (rational first guess, then Newton steps on the C library's erfc).
 * Returns NaN unless 0 < k < d. */
SPARK_API double spark_topk_quantile(int k, int d);

/* Time limit, in nanoseconds, of every device-side wait in later launches
 * (grid barriers, copy completions).  Default 1e9 (one second); 0 restores it. */
SPARK_API int spark_set_wait_limit_ns(unsigned long long ns);

/*
 * Single-token decode (spark_ffn_forward, and _tokens / _debug with one token)
 * runs as three kernels: a score kernel (x, its moments), a gather kernel
 * (theta, the active K2 / V rows, partial outputs) and a reduce kernel (out).
 * With weight overlap enabled (nonzero),
 * the score kernel is launched as a programmatic dependent of whatever kernel
 * precedes the call on the stream: it starts streaming K1 into shared memory
 * while that kernel is still running, and reads q, and writes anything, only
 * after that kernel has completed.  This hides most of K1's transfer behind the
 * previous call (or the previous layer) in a decode loop.  The caller promises
 * that the kernel immediately preceding the call on the stream does not write
 * K1.  Default 0: the score kernel starts after all earlier work.  Process-wide;
 * applies to later calls.  spark_ffn_decode_stack always overlaps its own
 * layers (the kernel ahead of each layer's score kernel is the library's).
 */
SPARK_API int spark_set_weight_overlap(int enable);

/* Self-test of the bounded waits: launches the fused kernel's grid barrier on
 * `stream` with an arrival target that can never be met, so that every CTA runs
 * out its time limit and records SPARK_ETIMEOUT.  Call spark_query_status() on
 * the same stream afterwards; it must return SPARK_ETIMEOUT and clears it. */
SPARK_API int spark_selftest_wait_timeout(spark_stream_t stream);

/* Size in bytes of the fixed scratch buffer used by spark_ffn_forward_noalloc. */
#define SPARK_NOALLOC_SCRATCH_BYTES (2u << 20)

/*
 * spark_ffn_forward_noalloc -- the paper has no counterpart to this entry point;
 * it exists for callers that must not allocate device memory while they run:
 * for example the execute hook of an inference-engine plugin (which must not
 * allocate), or a runtime that plans all device memory ahead of time and
 * treats any later allocation as a failure.
 *
 * It computes what spark_ffn_forward computes for one token (same arguments,
 * same argument checks, same arithmetic up to fp32 summation order; it runs the
 * single-launch fused kernel that also serves 2-4 tokens) but never calls cudaMalloc,
 * cudaMallocAsync, cudaFree or any allocating library routine.  Its scratch
 * (control block, per-CTA moments, per-CTA partial outputs) lives in one
 * buffer of SPARK_NOALLOC_SCRATCH_BYTES (2 MiB) compiled into the library as a
 * static device array; every GPU that loads the library holds those 2 MiB until
 * the process exits.  The caller still provides q, the weights and out.
 *
 * Limit: the problem's scratch must fit the buffer: about
 * 4 * d_model * (number of CTAs, at most the SM count) bytes plus a few KB
 * (1.33 MB for the Gemma-2-2B layer d_model 2304 on 148 SMs).  A larger problem
 * returns SPARK_ESCRATCH and enqueues nothing.
 *
 * Set-up: the first call on a device looks up the buffer's device address
 * (cudaGetSymbolAddress) with that device current and keeps it for the rest of
 * the process.  A cudaDeviceReset (or any reset of the device's primary context) unmaps the
 * buffer and leaves that address stale: do not call this entry point on a
 * device after resetting it.
 *
 * Sharing: all calls on all streams use the same buffer, which keeps the last
 * call's contents.  Each call clears the buffer's arrival counters with a
 * cudaMemsetAsync on `stream` before its kernel.  Calls whose work overlaps on
 * the GPU (on different streams) race on the buffer and give wrong results:
 * order them.
 *
 * Errors: every device-side wait has the time limit of spark_set_wait_limit_ns.
 * A wait that runs out leaves `out` undefined and records SPARK_ETIMEOUT in the
 * buffer; later calls of this entry point then return without computing until
 * spark_query_status() (on any stream of the device, once the failed call has
 * completed) reports the error and clears it.
 */
SPARK_API int spark_ffn_forward_noalloc(const void* q, const void* K1, const void* K2, const void* V,
                                        int d_model, int r, int d_ff, int k, void* out,
                                        spark_stream_t stream);

/*
 * Bounds-check build.  libspark_debug.so is this library compiled with
 * SPARK_DEBUG: its kernels check the indices they compute before using them
 * (gathered neuron rows against d_ff, active counts against the slice,
 * gathered key rows against n_ctx, partial-output slots, GEMM operand blocks)
 * and skip an access whose check fails, counting it; they never trap.  The
 * results of a run without violations are bit-identical to libspark.so's.
 *
 * Returns the number of failed checks since the previous call (summed over the
 * kernels of the current device) and clears the count; synchronises the device
 * first.  While the count is nonzero, spark_query_status reports SPARK_EBOUNDS.
 * Returns -1 in the release library, whose kernels contain no checks, and
 * SPARK_ECUDA (-3) if reading the counts failed.
 */
SPARK_API int spark_debug_violations(void);

/* Library version: major*10000 + minor*100 + patch. */
SPARK_API int spark_version(void);

#ifdef __cplusplus
}
#endif

#endif /* SPARK_H_ */
