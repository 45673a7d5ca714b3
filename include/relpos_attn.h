/*
 * relpos_attn.h -- C ABI of the relative-position attention library (B200, sm_100a).
 *
 * Exact softmax attention with an additive relative-position term,
 *
 *     S_ij = scale * Q_i . K_j + R_ij        (masked to -inf when causal and j > i)
 *     O    = softmax_j(S) V,   LSE_i = ln sum_j exp S_ij,
 *
 * forward and backward, as described by "Fast and Exact Relative-Position
 * Attention via Structure-Aware Kernels" (Abstract: exact FlashAttention-style
 * tiled computation with offset-aware tiling, reuse of the needed key/query
 * relation products, and offset-sharded, atomic-free gradient aggregation) and by
 * the article "结构感知内核让相对位置注意力加速21倍" (section
 * "为什么相对位置注意力难做快": S = Q K^T / sqrt(d) + B, with B never
 * materialised).  The four mechanisms are the ones the paper's Hugging Face page
 * names (Community comment), and ALiBi is the further bias the article lists among
 * the models the method suits (section "工程权衡与适用边界"); their formulas follow
 * their original papers:
 *
 *   RELPOS_T5       R_ij = t[h, bucket(j - i)]                      (added unscaled)
 *   RELPOS_SHAW     R_ij = scale * q_i . a[h, clip(j - i, -c, c) + c]
 *   RELPOS_TXL      R_ij = scale * (u[h] . k_j + (q_i + v[h]) . r[h, row(i - j)])
 *                   row(x) = x when causal (table rows L), x + L - 1 otherwise (2L - 1)
 *   RELPOS_DEBERTA  R_ij = scale * (q_i . Kr[h, clip(i - j + k, 0, 2k - 1)]
 *                                 + k_j . Qr[h, clip(j - i + k, 0, 2k - 1)])
 *   RELPOS_ALIBI   R_ij = -m[h] * |j - i|                           (added unscaled)
 *
 * T5 buckets: bidirectional (upper half for j > i) or unidirectional, exact
 * distances below max_exact = (buckets per side) / 2, then
 * max_exact + floor(log(a / max_exact) / log(max_distance / max_exact) *
 * (per side - max_exact)) capped to the last bucket, evaluated in exact integer
 * arithmetic.
 *
 * Memory and ownership
 *   - Every pointer is a DEVICE pointer allocated by the caller; the library
 *     allocates nothing, never synchronises the host, keeps no global state and
 *     is safe to call from several host threads on different streams.
 *   - Q, K, V, O, dO, dQ, dK, dV: contiguous [B, H, L, d] in the params' dtype
 *     (float32 or bfloat16).  d must be 64.
 *   - Relative parameters rel[0..2] (contiguous, params' dtype unless noted):
 *       T5       rel[0] = t  [H, num_buckets]            float32 always
 *       Shaw     rel[0] = a  [H, 2c + 1, d]  (+ rel[1] = aV [H, 2c + 1, d] with shaw_value)
 *       TXL      rel[0] = r  [H, n_off, d]  (n_off = L causal, 2L - 1 otherwise),
 *                rel[1] = u  [H, d], rel[2] = v [H, d]
 *       DeBERTa  rel[0] = Kr [H, 2k, d], rel[1] = Qr [H, 2k, d]
 *       ALiBi    rel[0] = m  [H]  per-head slopes            float32 always
 *     Unused entries may be NULL.
 *     On the tensor-core path (bfloat16) Q, K, V, dO and the bf16 tables rel[0] (and
 *     rel[1] for DeBERTa and for Shaw's value table) must start on a 16-byte boundary;
 *     RELPOS_ERR_INVALID_ARG otherwise.
 *   - LSE: float32 [B, H, L], natural log.
 *   - drel[0..2]: float32 gradients with the shapes of rel[0..2], summed over the
 *     batch; they are overwritten (not accumulated into).
 *   - workspace: device scratch of at least relpos_attn_workspace_size() bytes,
 *     256-byte aligned; its contents on entry do not matter.
 *   - dev_status: optional device int32; kernels that wait on hardware barriers
 *     write a RELPOS_ERR_* code there when a wait runs out (the caller clears it
 *     to 0 and reads it back after synchronising).  NULL disables it.
 *   - stream: a cudaStream_t (NULL = the legacy default stream).  All work is
 *     enqueued on it asynchronously, on the calling thread's current CUDA device,
 *     which must be the device that holds the pointers and the stream.  A host
 *     thread with no current CUDA context gets the current device's primary context
 *     made current (as the runtime's first call there would do); a current context is
 *     left as it is.
 *
 * Errors: every call returns RELPOS_OK (0) or a negative RELPOS_ERR_* code.  The entry
 * points clear the calling thread's CUDA "last error" before they enqueue anything, so
 * that an error left by an earlier, unrelated runtime call is not reported as theirs.  Argument
 * errors (RELPOS_ERR_INVALID_ARG, _WORKSPACE, _UNSUPPORTED) are found before anything
 * is enqueued; after a launch or runtime failure (RELPOS_ERR_LAUNCH, _CUDA) the work
 * enqueued before it may still run, and the outputs are undefined.
 * Nothing aborts, traps or throws across this boundary.
 *
 * Debug build: the library built with RELPOS_DEBUG (librelpos_attn_debug.so) checks
 * the indices of its kernels' global stores and skew / offset-order shared-memory
 * stores; a failed check skips that access and writes RELPOS_ERR_BOUNDS to the
 * status word (no thread leaves a kernel early: the barriers stay balanced).
 *
 * Determinism: the backward pass uses no atomic operations; the relative-table
 * gradients are reduced from per-shard partials in a fixed order, so repeated
 * calls give bitwise identical results.
 */
#ifndef RELPOS_ATTN_H_
#define RELPOS_ATTN_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define RELPOS_API __attribute__((visibility("default")))
#else
#define RELPOS_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

enum relpos_mech { RELPOS_T5 = 0, RELPOS_SHAW = 1, RELPOS_TXL = 2, RELPOS_DEBERTA = 3, RELPOS_ALIBI = 4 };
enum relpos_dtype { RELPOS_F32 = 0, RELPOS_BF16 = 1 };

/* kernel_path: which kernel family runs the call.  RELPOS_PATH_AUTO picks the
 * tensor-core (tcgen05) kernels for bfloat16 and the fp32 CUDA-core kernels for
 * float32.  RELPOS_PATH_SIMT forces the CUDA-core kernels (fp32 arithmetic on
 * any dtype).  Both are GPU paths; there is no CPU path.
 * bfloat16 cases that the tensor-core kernels do not cover, and that therefore run on the
 * CUDA-core kernels under RELPOS_PATH_AUTO (RELPOS_ERR_UNSUPPORTED under RELPOS_PATH_TC):
 * Shaw with the value-side table and c > 64 (both passes).  (DeBERTa runs on the tensor
 * cores at every span, T5 at every bucket layout.)
 * Shaw without the value-side table and c > 64 runs on the Transformer-XL kernels: its
 * table is expanded to one row per offset (row i - j + off = a[clip(j - i) + c]) with
 * u = v = 0, and the expanded table's gradient is summed back into the 2c + 1 rows; the
 * expanded table and its gradient live in the workspace. */
enum relpos_path { RELPOS_PATH_AUTO = 0, RELPOS_PATH_SIMT = 1, RELPOS_PATH_TC = 2 };

enum relpos_status {
  RELPOS_OK = 0,
  RELPOS_ERR_INVALID_ARG = -1,      /* null pointer, bad enum, d != 64, bad sizes */
  RELPOS_ERR_WORKSPACE = -2,        /* workspace NULL or smaller than required     */
  RELPOS_ERR_UNSUPPORTED = -3,      /* valid but not implemented (e.g. path/dtype)  */
  RELPOS_ERR_LAUNCH = -4,           /* a kernel launch was rejected by the driver  */
  RELPOS_ERR_TIMEOUT = -5,          /* (device status only) a bounded wait ran out  */
  RELPOS_ERR_CUDA = -6,             /* a CUDA runtime call failed                    */
  RELPOS_ERR_BOUNDS = -7            /* (device status only, debug build) an index
                                       check failed; the access was skipped          */
};

typedef struct relpos_params {
  int32_t mech;              /* enum relpos_mech                                  */
  int32_t dtype;             /* enum relpos_dtype                                 */
  int32_t causal;            /* 1: mask keys j > i                                */
  int32_t kernel_path;       /* enum relpos_path                                  */
  int64_t B, H, L, d;        /* batch, heads, sequence length, head dim (64)      */
  float scale;               /* multiplies q.k (and the terms listed above)       */
  int32_t t5_num_buckets;    /* T5: number of buckets (e.g. 32), 2..64            */
  int32_t t5_max_distance;   /* T5: distance of the last bucket (e.g. 128)        */
  int32_t t5_bidirectional;  /* T5: 1 bidirectional, 0 unidirectional             */
  int32_t shaw_clip;         /* Shaw: clip distance c (table rows 2c + 1)         */
  int32_t deberta_span;      /* DeBERTa: relative span k (table rows 2k)          */
  /* Variable-length batches (optional; NULL = every batch has L keys): DEVICE
   * pointer to B int32 key lengths.  Keys j >= seqlens_k[b] of batch b are masked
   * (after causal masking); all L queries are computed and relative positions keep
   * their meaning over the padded length.  Values are clamped to [0, L].  A query
   * with no unmasked key gets O = 0, LSE = -inf and zero gradients; masked keys get
   * dK = dV = 0.  The array is read by the kernels of the call (stream order) and
   * must stay valid until they finish.  Variable-length speech batches: article
   * "结构感知内核让相对位置注意力加速21倍", section "为什么相对位置注意力难做快". */
  const int32_t *seqlens_k;
  /* Shaw only (0 or 1): 1 adds the value-side term of Shaw et al.,
   *     O_i = sum_j P_ij (v_j + aV[h, clip(j - i, -c, c) + c]),
   * with rel[1] = aV [H, 2c + 1, d] (params' dtype) and drel[1] = daV (float32).
   * The paper's Hugging Face page names Shaw among the mechanisms the method covers
   * (Community comment); the value side is the second table of Shaw's own paper.
   * Both passes run on the tensor-core kernels for bf16 and c <= 64. */
  int32_t shaw_value;
  /* Transformer-XL only, causal only (0 = none): length M of the cached memory of the
   * previous segment.  The L queries (q, o, lse, dq, dO: [B, H, L, d]) sit at positions
   * M .. M + L - 1 over M + L keys (k, v, dk, dv: [B, H, M + L, d]: the memory, then the
   * segment); r has M + L rows and seqlens_k counts keys over the M + L.  Computed as the
   * causal attention of the M + L positions read at its last L query rows (the first M
   * rows' work is done and discarded).  Transformer-XL's segment-level recurrence; the
   * mechanism is one of those the paper's Hugging Face page names (Community comment). */
  int64_t mem_len;
} relpos_params_t;

/* Bytes of device workspace a call needs.  pass: 0 forward, 1 backward,
 * 2 backward at its smallest.  relpos_attn_bwd accepts any workspace of at least
 * the pass-2 size.  Between that and the pass-1 size, the Transformer-XL
 * tensor-core backward recomputes S, P and dS in its key-tile and diagonal kernels.
 * With the pass-1 size or more, the query-tile kernel writes every tile's P and dS
 * (64 KB per 128 x 128 tile, e.g. 1.1 GB at B = 1, H = 8, L = 8192 causal) and those
 * kernels stream them back: faster, but the memory grows with L^2.  Past 32 GiB of tiles
 * the pass-1 size leaves them out as well (the recomputing kernels run).  Other calls
 * need the same size for passes 1 and 2.  The split trades memory for time and is
 * no part of the method.
 * Returns RELPOS_OK and sets *bytes, or RELPOS_ERR_INVALID_ARG. */
RELPOS_API int relpos_attn_workspace_size(const relpos_params_t *params, int pass, size_t *bytes);

/* Forward pass: writes O [B,H,L,d] (params dtype) and LSE [B,H,L] (float32).
 * The step of the method: exact tiled attention with the relative term folded
 * into the online softmax ("Fast and Exact Relative-Position Attention via
 * Structure-Aware Kernels", Abstract; article "结构感知内核让相对位置注意力加速21倍",
 * section "结构感知分块如何保持精确性"). */
RELPOS_API int relpos_attn_fwd(const relpos_params_t *params,
                    const void *q, const void *k, const void *v,
                    const void *const rel[3],
                    void *o, float *lse,
                    void *workspace, size_t workspace_bytes,
                    int32_t *dev_status, void *stream);

/* Backward pass: given O and LSE from relpos_attn_fwd and the output gradient
 * dO, writes dQ, dK, dV (params dtype) and drel[0..2] (float32, see above; for
 * ALiBi drel[0] = dm[H] = sum over pairs of dS_ij * -|j - i|, for callers that
 * learn the slopes).
 * Gradients of the relative parameters are sharded by offset into partials and
 * merged by a fixed-order second pass with no atomics (same Abstract, technique
 * (3); article section "3. 基于偏移的梯度分片"). */
RELPOS_API int relpos_attn_bwd(const relpos_params_t *params,
                    const void *q, const void *k, const void *v,
                    const void *const rel[3],
                    const void *o, const float *lse, const void *dout,
                    void *dq, void *dk, void *dv, float *const drel[3],
                    void *workspace, size_t workspace_bytes,
                    int32_t *dev_status, void *stream);

/* Size of the device scratch array built into the library for
 * relpos_attn_fwd_noalloc (per GPU, held until the process exits). */
#define RELPOS_NOALLOC_SCRATCH_BYTES ((size_t)16 << 20)

/* relpos_attn_fwd for callers that cannot allocate device memory -- e.g. a plugin
 * inside a framework that owns the whole device-memory budget, or a latency-critical
 * loop where cudaMalloc / cudaFree would synchronise the device.  It has no
 * counterpart in the paper; it is the same forward pass with its scratch taken from
 * a static device array of RELPOS_NOALLOC_SCRATCH_BYTES instead of a caller
 * workspace.  Arguments, outputs and errors are those of relpos_attn_fwd; a problem
 * whose forward scratch (relpos_attn_workspace_size, pass 0) exceeds the array is
 * rejected with RELPOS_ERR_WORKSPACE before anything is enqueued.  It allocates
 * nothing.  All calls share the array: calls that may overlap on the GPU race and
 * must be ordered by the caller.  The first call on a device looks up the array's
 * device address (with that device current); make it before any stream capture.
 * The address is kept for the life of the process: do not use this entry point after
 * cudaDeviceReset, nor from a context other than the device's primary context. */
RELPOS_API int relpos_attn_fwd_noalloc(const relpos_params_t *params,
                                       const void *q, const void *k, const void *v,
                                       const void *const rel[3],
                                       void *o, float *lse,
                                       int32_t *dev_status, void *stream);

/* Kernel family that pass `pass` (0 forward, 1 backward) of a call with these
 * params runs: RELPOS_PATH_SIMT or RELPOS_PATH_TC (RELPOS_PATH_AUTO resolved),
 * or a negative RELPOS_ERR_* code (RELPOS_ERR_UNSUPPORTED when RELPOS_PATH_TC is
 * forced where it does not apply). */
RELPOS_API int relpos_attn_resolved_path(const relpos_params_t *params, int pass);

/* Self-test of the bounded device waits (failure detection; no counterpart in the
 * paper).  Launches one warp that waits on a device barrier nothing ever completes,
 * through the wait routine of the tensor-core kernels, with a limit of limit_ns
 * (1 ms .. 10 s) instead of their 2 s.  When the kernel has run, *dev_status holds
 * RELPOS_ERR_TIMEOUT and *dev_elapsed_ns the nanoseconds the wait took (the limit plus
 * at most about 1 ms); the context stays usable.  dev_status and dev_elapsed_ns are
 * device pointers.  Returns RELPOS_ERR_INVALID_ARG for a null or host pointer or a
 * limit out of range, RELPOS_ERR_LAUNCH if the launch fails, else RELPOS_OK. */
RELPOS_API int relpos_selftest_wait(uint64_t limit_ns, int32_t *dev_status,
                                    unsigned long long *dev_elapsed_ns, void *stream);

/* Tracing (no counterpart in the paper; a measurement aid).  Every kernel the library
 * launches is wrapped in an NVTX range named after the kernel, which NVTX-aware
 * profilers show and which costs nothing when none is attached.  A caller that wants
 * per-kernel device times without a profiler registers a relpos_trace_t with
 * relpos_trace_begin: until relpos_trace_end, every kernel that this library launches
 * from the SAME host thread is bracketed by two of the caller's CUDA events, recorded on
 * the launch stream: kernel k of the traced calls (in launch order) between
 * events[2k] and events[2k + 1], its static name in names[k].  The caller creates the
 * 2 * capacity events (cudaEvent_t, timing enabled), keeps the struct alive while it is
 * registered, and reads the times with cudaEventElapsedTime after synchronising.
 * Kernels past capacity are not recorded and counted in `dropped`.  With `only` set,
 * kernels of other names are neither recorded nor counted (their NVTX ranges remain), so
 * that one kernel can be timed with two events per launch.  Registration is per host
 * thread: calls from other threads are neither traced nor affected. */
#define RELPOS_TRACE_MAX 64
typedef struct relpos_trace {
  void *const *events;                 /* in: 2 * capacity cudaEvent_t handles        */
  int32_t capacity;                    /* in: kernels to record, 1 .. RELPOS_TRACE_MAX */
  int32_t count;                       /* out: kernels recorded                       */
  int32_t dropped;                     /* out: kernels launched past capacity         */
  const char *only;                    /* in: NULL, or record only kernels of this name */
  const char *names[RELPOS_TRACE_MAX]; /* out: name of kernel k                       */
} relpos_trace_t;

/* Starts recording this thread's launches into *trace (count and dropped reset).
 * Returns RELPOS_ERR_INVALID_ARG for a null struct or event, or a capacity out of range. */
RELPOS_API int relpos_trace_begin(relpos_trace_t *trace);
/* Stops recording for this thread.  Always RELPOS_OK. */
RELPOS_API int relpos_trace_end(void);

/* Static, NUL-terminated description of a status code. */
RELPOS_API const char *relpos_strerror(int status);

/* The cudaError_t value behind the last RELPOS_ERR_LAUNCH that a call made from this
 * host thread returned (0 if none has): a diagnostic for callers. */
RELPOS_API int relpos_last_cuda_error(void);

/* ABI version: major * 10000 + minor * 100 + patch. */
RELPOS_API int relpos_attn_version(void);

#ifdef __cplusplus
}
#endif

#endif /* RELPOS_ATTN_H_ */
