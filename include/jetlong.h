/*
 * jetlong.h -- C ABI of the B200 (sm_100a) bifocal-RoPE attention library.
 *
 * The operation is the attention of "Jet-Long: Efficient Long-Context Extension
 * with Dynamic Bifocal RoPE":
 *
 *   - schedule (§3.1, Eq. (2)):  G = max(1, ceil(L / w_pretrained)),
 *                                f(x) = floor(x / G)   (identity when L <= w_pretrained);
 *   - score rule (§3, display equation of S(q, k)), for query i and key j <= i:
 *         i - j <= w0 :  S = RoPE(x_q, i)    . RoPE(x_k, j)
 *         i - j >  w0 :  S = RoPE(x_q, f(i)) . RoPE(x_k, f(j))
 *     scaled by 1/sqrt(D), softmax over j <= i (causal);
 *   - the two windows are merged as in §3.3 (inclusion-exclusion of three
 *     attention passes); the kernels compute the same sum in one online
 *     softmax that picks the score of each pair by the rule above;
 *   - KV cache (§3.2): keys are stored once, rotated to their true positions,
 *     k_cache[k] = RoPE(x_k, k); decode applies the correction rotation by
 *     Delta k = f(k) - k on the fly and never rewrites the cache.
 *   - The *_interp entry points replace the remote map by the frequency
 *     interpolation of the paper's remote-map ablation (§4.7); see below.
 *
 * RoPE pairs channel i with channel i + D/2 and rotates the pair by the angle
 * p * theta^(-2i/D); angles are formed in double precision and reduced before
 * the sine/cosine, so positions up to 2^31 keep full accuracy.
 *
 * Conventions shared by every entry point
 *   - Positions are 0-based.  The decode query of a cache holding L tokens
 *     (the new one included) sits at position L - 1.
 *   - Tensors are dense, row-major (last index fastest), BF16 unless noted,
 *     in device memory.  Layouts are given as [dim0, dim1, ...].
 *   - GQA: query head h reads KV head h / (Hq / Hkv).
 *   - Supported head dims: D = 64 or 128.  Hq must be a multiple of Hkv.
 *   - Device pointers must be 16-byte aligned.
 *   - Ownership: the caller owns every buffer, and the library performs no
 *     device allocation.  Its only device storage is static in its image:
 *     the error word and the 8 MiB buffer of jetlong_decode_noalloc.
 *     Scratch space is passed in as a caller-owned workspace whose size the
 *     *_workspace_size functions return.
 *   - Execution: asynchronous on `stream` (NULL = the legacy default stream) on
 *     the current CUDA device.  Arguments are validated on the host before
 *     anything is launched; a call that returns an error launched nothing.
 *   - Errors are returned as jl_status codes, never thrown.  JL_ERR_CUDA means
 *     a launch failed (see cudaGetLastError for the CUDA code).  Every wait
 *     inside a kernel is bounded in time; a wait that gives up records
 *     JL_ERR_DEVICE_TIMEOUT, which jetlong_device_status() reports.
 *   - Precision: BF16 inputs; the prefill's tensor-core operands (rotated
 *     Q/K, V, and the probabilities P) are FP16, which holds the rotated
 *     values with three more mantissa bits than BF16; accumulation, softmax
 *     statistics and LSE are FP32.  Inputs must stay inside the FP16 range
 *     (|x| <= 65504 after rotation).  The range is a contract on the
 *     inputs, not a status of the call: a call returns before its kernels
 *     run, so a call that meets a larger value still returns JL_OK, and its
 *     outputs may hold non-finite values.  A prefill (every form) records
 *     the event, and the next jetlong_device_status() returns JL_ERR_RANGE;
 *     read it before trusting outputs of inputs that may be that large.
 *     The decode and chunk calls (whose queries and corrected keys pass
 *     through FP16 too) record nothing: out-of-range values there show up
 *     only as non-finite outputs.
 *   - Calls on different streams may run concurrently as long as they do not
 *     share output or workspace buffers.
 */
#ifndef JETLONG_H
#define JETLONG_H

#include <stddef.h>

#if defined(__GNUC__)
#define JL_API __attribute__((visibility("default")))
#else
#define JL_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* ABI-identical to cudaStream_t; NULL selects the legacy default stream. */
typedef struct CUstream_st *jl_stream_t;

typedef enum {
  JL_OK = 0,
  JL_ERR_NULL = -1,            /* a required pointer is NULL                        */
  JL_ERR_SHAPE = -2,           /* a size is out of range or inconsistent            */
  JL_ERR_UNSUPPORTED = -3,     /* valid but not implemented (e.g. D not 64/128)     */
  JL_ERR_ALIGN = -4,           /* a pointer is not 16-byte aligned                  */
  JL_ERR_WORKSPACE = -5,       /* workspace NULL or smaller than required           */
  JL_ERR_CUDA = -6,            /* a CUDA runtime / launch error                     */
  JL_ERR_DEVICE_TIMEOUT = -7,  /* a bounded in-kernel wait expired (device report)  */
  JL_ERR_NO_DEVICE = -8,       /* no sm_100 device is current                       */
  JL_ERR_RANGE = -9            /* an input exceeds the FP16 range of the MMA operands
                                  (|x| > 65504 after rotation; device report)        */
} jl_status;

typedef enum { JL_BF16 = 0, JL_F32 = 1 } jl_dtype;

/* A prefill chunk of at least this many queries runs on the tensor-core
 * prefill kernel, a shorter one on the decode kernels (jetlong_prefill_chunk). */
#ifndef JL_CHUNK_TENSOR_MIN
#define JL_CHUNK_TENSOR_MIN 6
#endif

/* Human-readable name of a status code (static string, never NULL). */
JL_API const char *jetlong_status_string(int status);

/* Library version as "major.minor.patch" (static string). */
JL_API const char *jetlong_version(void);

/*
 * Forget the per-device state the library keeps on the host (the checked
 * compute capability and the address of each device's error word); the next
 * call on a device looks them up again.  The library holds no device
 * allocation to free: it computes its cos/sin tables inside the kernels and
 * its only device-side storage is static (the error word and the
 * jetlong_decode_noalloc buffer).  Call it when no call of this library is
 * in flight on another thread.
 * It also forgets the device address of the jetlong_decode_noalloc buffer
 * and which kernels already have their shared-memory limit set.  A
 * cudaDeviceReset invalidates both: after one, call jetlong_shutdown before
 * the next call of this library.
 */
JL_API void jetlong_shutdown(void);

/*
 * Dynamic group size of §3.1, Eq. (2): G = max(1, ceil(L / w_pretrained)).
 * Host only, no CUDA call.  Returns G >= 1, or JL_ERR_SHAPE if L < 1 or
 * w_pretrained < 1.
 */
JL_API int jetlong_group_size(int L, int w_pretrained);

/*
 * Bytes of workspace jetlong_prefill needs for these sizes (host only).
 * Returns 0 if a size is invalid.
 */
JL_API size_t jetlong_prefill_workspace_size(int B, int Hq, int Hkv, int L, int D);

/*
 * Bifocal causal attention over a whole prompt (prefill).  One G for the call,
 * from the prompt length L (§3.1).
 *
 *   q   [B, L, Hq,  D] BF16, pre-RoPE queries           (read)
 *   k   [B, L, Hkv, D] BF16, pre-RoPE keys              (read)
 *   v   [B, L, Hkv, D] BF16, values                     (read)
 *   out [B, L, Hq,  D] out_dtype (JL_BF16 or JL_F32)    (written)
 *   lse [B, Hq, L] float32, natural-log log-sum-exp of the scaled scores per
 *       row (written; may be NULL)
 *   w_pretrained >= 1, w0 >= 0, rope_theta > 0.  D is 64 or 128; Hq is a
 *   multiple of Hkv; B * L * Hq <= 2^31; B <= 65535 and
 *   Hkv * ceil(Hq / Hkv / 2) <= 65535 (CUDA grid limits).
 *   k_cache_out: NULL, or [B, k_cache_capacity, Hkv, D] BF16; rows [0, L) are
 *       written with RoPE(x_k, k) at true positions (§3.2), the cache decode
 *       expects.  k_cache_capacity >= L (ignored when k_cache_out is NULL).
 *   workspace: device buffer of at least jetlong_prefill_workspace_size(...)
 *       bytes, 256-byte aligned; contents on entry do not matter.
 *
 * Returns JL_OK or an error code (nothing launched on error).
 */
JL_API int jetlong_prefill(const void *q, const void *k, const void *v, void *out, float *lse,
                    int B, int Hq, int Hkv, int L, int D,
                    int w_pretrained, int w0, float rope_theta, int out_dtype,
                    void *k_cache_out, int k_cache_capacity,
                    void *workspace, size_t workspace_bytes, jl_stream_t stream);

/*
 * The two stages of jetlong_prefill, for callers that schedule them apart
 * (e.g. to time the attention kernel alone, or to rotate once and attend
 * several times).  jetlong_prefill == jetlong_prefill_rotate followed by
 * jetlong_prefill_attend on the same workspace and stream.
 *
 * jetlong_prefill_rotate: the key side of RoPE.  Reads k and v (layouts as
 *   for jetlong_prefill) and writes the key operands into the workspace: keys
 *   rotated to true positions j and, when G > 1, to remote positions f(j),
 *   plus the values, all FP16 head-major [B, Hkv, L, D]; if k_cache_out is
 *   not NULL it also writes the BF16 true-position cache rows [0, L) (§3.2).
 * jetlong_prefill_attend: the attention kernel.  Reads q (pre-RoPE, layout as
 *   for jetlong_prefill: its query side of RoPE runs in the kernel's load
 *   path, rotating each query row to f(i) and to i as the tile is staged)
 *   and the operands a preceding jetlong_prefill_rotate with the same B, Hkv,
 *   L, D, w_pretrained and rope_theta left in `workspace`; writes out and lse
 *   (lse may be NULL).
 */
JL_API int jetlong_prefill_rotate(const void *k, const void *v, int B, int Hkv, int L, int D,
                                  int w_pretrained, float rope_theta, void *k_cache_out,
                                  int k_cache_capacity, void *workspace, size_t workspace_bytes,
                                  jl_stream_t stream);

JL_API int jetlong_prefill_attend(const void *q, void *out, float *lse, int B, int Hq, int Hkv,
                                  int L, int D, int w_pretrained, int w0, float rope_theta,
                                  int out_dtype, const void *workspace, size_t workspace_bytes,
                                  jl_stream_t stream);

/*
 * The unfused three-pass form of the same result (Jet-Long paper, §3.3
 * "Inclusion-exclusion merge"), kept as a cross-check of the fused kernel
 * and to measure what fusion saves.  Three attention passes over the
 * operands of jetlong_prefill_rotate:
 *   A: remote positions f(i), f(j) on every causal pair j <= i;
 *   B: true positions i, j on the band 0 <= i - j <= w0;
 *   C: remote positions on the same band;
 * each writing an fp32 output and lse into the workspace, then
 *   out = (W_A O_A + W_B O_B - W_C O_C) / (W_A + W_B - W_C),  W_X = exp(lse_X),
 *   lse = log(W_A + W_B - W_C).
 * The band passes use w0 even when G = 1 (then B and C coincide and cancel).
 * Arguments and layouts as for jetlong_prefill (no cache output);
 * workspace: at least jetlong_prefill_three_pass_workspace_size(...) bytes,
 * 256-byte aligned (the prefill operands plus 3 fp32 outputs and 3 lse rows).
 * Precision: the subtraction loses accuracy where the band holds most of a
 * row's softmax mass under remote positions; the fused path has no
 * subtraction.  Returns JL_OK or an error code (nothing launched on error).
 */
JL_API size_t jetlong_prefill_three_pass_workspace_size(int B, int Hq, int Hkv, int L, int D);

JL_API int jetlong_prefill_three_pass(const void *q, const void *k, const void *v, void *out,
                                      float *lse, int B, int Hq, int Hkv, int L, int D,
                                      int w_pretrained, int w0, float rope_theta, int out_dtype,
                                      void *workspace, size_t workspace_bytes,
                                      jl_stream_t stream);

/*
 * A prefill chunk: n new tokens at positions P0 .. P0+n-1 appended to a
 * prompt whose cache already holds them (Jet-Long paper, §3.1 and §3.2; the
 * chunk's keys written first, e.g. with jetlong_rope_cache).  One G for the
 * call, from the length after the chunk, L = P0 + n.  Query i sits at
 * p = P0 + i and sees keys [0, p]: local keys (p - j <= w0) as cached,
 * older keys turned by the correction rotation R(f(j) - j) and scored
 * against RoPE(x_q, f(p)).  With P0 = 0 and n = L this equals jetlong_prefill
 * on the same data.  Two execution paths, chosen by n alone
 * (JL_CHUNK_TENSOR_MIN, above):
 *   - n < JL_CHUNK_TENSOR_MIN: the split-KV decode kernels (a chunk is n
 *     decode problems over one cache; cost grows with n * L);
 *   - n >= JL_CHUNK_TENSOR_MIN: the tensor-core prefill kernel.  A pass first writes the
 *     cached keys of [0, P0 + n), as stored and turned by R(f(j) - j), and
 *     the values into the workspace as FP16; 128-row query tiles then run
 *     the same kernel as jetlong_prefill, which rotates the chunk's queries
 *     as it loads them.  When the chunk has too few query tiles to fill the
 *     GPU (fewer than 75 tile x head-pair units), each tile's key tiles are
 *     split into up to 148 / units contiguous ranges, one CTA each, whose
 *     partial results a log-sum-exp merge combines.  The cost is one pass
 *     over the cache plus the tensor-core work of n * L pairs; the FP16
 *     range contract above applies to this path.
 * jetlong_prefill_chunk_workspace_size returns the size the chosen path needs
 * (tensor-core path: 3 x B.Hkv.(P0+n).D FP16 values, plus, when the keys are
 * split into S > 1 ranges, B.n.Hq.S.(D + 2) float32 partial records; each
 * array 256-byte aligned).
 *
 *   q       [B, n, Hq, D] BF16 pre-RoPE queries of the chunk (read)
 *   k_cache [B, Lcap, Hkv, D] BF16, RoPE at true positions, rows [0, P0+n)
 *   v_cache [B, Lcap, Hkv, D] BF16 (read)
 *   out     [B, n, Hq, D] out_dtype (written); lse [B, Hq, n] float32 (may be NULL)
 *   P0 >= 0, n >= 1, P0 + n <= Lcap, B * n <= 65535; Hq / Hkv in {1, 2, 4, 8}.
 *   workspace: at least jetlong_prefill_chunk_workspace_size(...) bytes,
 *       256-byte aligned.
 * Returns JL_OK or an error code (nothing launched on error).
 */
JL_API size_t jetlong_prefill_chunk_workspace_size(int B, int Hq, int Hkv, int P0, int n, int D);

JL_API int jetlong_prefill_chunk(const void *q, const void *k_cache, const void *v_cache,
                                 void *out, float *lse, int B, int Hq, int Hkv, int P0, int n,
                                 int Lcap, int D, int w_pretrained, int w0, float rope_theta,
                                 int out_dtype, void *workspace, size_t workspace_bytes,
                                 jl_stream_t stream);

/*
 * Bytes of workspace jetlong_decode needs for a cache of L tokens (host only).
 * Non-decreasing in L: sizing it for the largest L a generation loop will reach
 * covers every earlier step.  Returns 0 if a size is invalid.
 */
JL_API size_t jetlong_decode_workspace_size(int B, int Hq, int Hkv, int L, int D);

/*
 * One generation step on the true-position cache (§3.2).
 *
 *   q        [B, Hq, D] BF16, pre-RoPE query of the new token, at position L-1
 *   k_cache  [B, Lcap, Hkv, D] BF16, RoPE(x_k, k) at true positions; slots
 *            [0, L) valid (the new token's key included)
 *   v_cache  [B, Lcap, Hkv, D] BF16; slots [0, L) valid
 *   out      [B, Hq, D] out_dtype;   lse [B, Hq] float32 (may be NULL)
 *   L: tokens in the cache including the new one, 1 <= L <= Lcap; G is
 *      recomputed from this L (§3.1).  Keys with (L-1) - j <= w0 are used as
 *      cached; older keys are rotated by Delta j = f(j) - j on the fly and
 *      scored against RoPE(x_q, f(L-1)).
 *   workspace: >= jetlong_decode_workspace_size(B, Hq, Hkv, L, D) bytes,
 *      256-byte aligned; contents on entry do not matter.
 *   Hq / Hkv must be 1, 2, 4 or 8 (JL_ERR_UNSUPPORTED otherwise);
 *   Hkv <= 8 * 65535 (CUDA grid limit).
 */
JL_API int jetlong_decode(const void *q, const void *k_cache, const void *v_cache, void *out,
                   float *lse, int B, int Hq, int Hkv, int L, int Lcap, int D,
                   int w_pretrained, int w0, float rope_theta, int out_dtype,
                   void *workspace, size_t workspace_bytes, jl_stream_t stream);

/*
 * jetlong_decode without a workspace argument, for callers that cannot
 * allocate device memory for one: processes whose device memory belongs to a
 * single arena or caching allocator, or generation loops that must not call
 * cudaMalloc because an allocation would stall the device.  (The paper has no
 * counterpart; this is a property of the library, not of the method.)
 *
 * Same arguments, layouts and results as jetlong_decode.  The split partials
 * live in a fixed 8 MiB buffer inside the library's device image, which every
 * GPU that loads the library holds until the process exits; the call
 * allocates nothing.  Sizes whose workspace
 * (jetlong_decode_workspace_size(B, Hq, Hkv, L, D)) exceeds 8 MiB are
 * rejected with JL_ERR_WORKSPACE before anything is launched.
 *   - The first call on each device looks up the buffer's device address on
 *     the host (once per device, with that device current); make that first
 *     call before any stream capture on that device.
 *   - All calls share the one buffer, and each call fully overwrites the part
 *     it reads, so nothing needs clearing between calls; but calls whose
 *     kernels overlap on the GPU (different streams, or different host
 *     threads) race on the buffer and must be serialised by the caller.
 */
JL_API int jetlong_decode_noalloc(const void *q, const void *k_cache, const void *v_cache,
                                  void *out, float *lse, int B, int Hq, int Hkv, int L, int Lcap,
                                  int D, int w_pretrained, int w0, float rope_theta, int out_dtype,
                                  jl_stream_t stream);

/*
 * Frequency-interpolation remote map: the ablation of §4.7 ("interpolate
 * frequency or alias position", Table 6) of the Jet-Long paper.  The page
 * gives no formula for it; these calls take the following reading.  The local
 * band (i - j <= w0) is unchanged.  A remote pair is scored at TRUE positions
 * with per-frequency interpolated frequencies (YaRN's per-frequency ramp):
 *   r_t      = w_pretrained * theta_t / (2 pi)   (turns within the pretrained window)
 *   gamma_t  = clamp((r_t - ramp_alpha) / (ramp_beta - ramp_alpha), 0, 1)
 *   theta'_t = theta_t * ((1 - gamma_t) / s + gamma_t),  s = max(1, L / w_pretrained)
 * where theta_t = rope_theta^(-2t/D) and s is §3.1's continuous dynamic
 * factor, recomputed from L like G.  There is no attention temperature.
 * YaRN's published bounds are ramp_alpha = 1, ramp_beta = 32.  The cache
 * stays at true positions.  A remote cached key is turned by the angle
 * j (theta'_t - theta_t), and the query is rotated by p theta'_t.  With
 * L <= w_pretrained, s = 1 and the result is plain causal RoPE attention,
 * as in the aliasing calls.
 *
 * Each call takes the arguments, layouts, workspace (the same
 * *_workspace_size function) and error codes of its aliasing counterpart,
 * plus ramp_alpha < ramp_beta, both finite (else JL_ERR_SHAPE, nothing
 * launched).
 */
JL_API int jetlong_prefill_interp(const void *q, const void *k, const void *v, void *out,
                                  float *lse, int B, int Hq, int Hkv, int L, int D,
                                  int w_pretrained, int w0, float rope_theta, float ramp_alpha,
                                  float ramp_beta, int out_dtype, void *k_cache_out,
                                  int k_cache_capacity, void *workspace, size_t workspace_bytes,
                                  jl_stream_t stream);

JL_API int jetlong_decode_interp(const void *q, const void *k_cache, const void *v_cache,
                                 void *out, float *lse, int B, int Hq, int Hkv, int L, int Lcap,
                                 int D, int w_pretrained, int w0, float rope_theta,
                                 float ramp_alpha, float ramp_beta, int out_dtype,
                                 void *workspace, size_t workspace_bytes, jl_stream_t stream);

JL_API int jetlong_prefill_chunk_interp(const void *q, const void *k_cache, const void *v_cache,
                                        void *out, float *lse, int B, int Hq, int Hkv, int P0,
                                        int n, int Lcap, int D, int w_pretrained, int w0,
                                        float rope_theta, float ramp_alpha, float ramp_beta,
                                        int out_dtype, void *workspace, size_t workspace_bytes,
                                        jl_stream_t stream);

/*
 * Two-form key cache for decode (a layout choice of this library; the paper
 * keeps one cache and rotates remote keys on every step, §3.2).  Beside the
 * true-position cache, the caller keeps k_remote [B, Lcap, Hkv, D] FP16:
 *
 *   k_remote[b, j, g, :] = FP16(R(f(j) - j) k_cache[b, j, g, :]),  G = G(L),
 *
 * the remote form of each key for the G of the length L it is read at.
 * jetlong_remote_cache writes rows [j0, j1) of it for the G of L
 * (0 <= j0 <= j1 <= L <= Lcap; j0 == j1 does nothing).  A generation loop
 * writes the new token's row after appending it, and rewrites rows [0, L)
 * whenever G changes (once per w_pretrained tokens).
 *
 * jetlong_decode_two_form is jetlong_decode with remote keys read from
 * k_remote instead of being rotated on the fly.  Rows [0, L - 1 - w0) of
 * k_remote must hold the remote form for G(L).  Same arguments, layouts,
 * workspace and results as jetlong_decode.  The rotation and FP16 rounding
 * are the ones the on-the-fly path applies, so the tensor-core operands are
 * identical.
 */
JL_API int jetlong_remote_cache(const void *k_cache, void *k_remote, int B, int Lcap, int Hkv,
                                int D, int j0, int j1, int L, int w_pretrained, float rope_theta,
                                jl_stream_t stream);

JL_API int jetlong_decode_two_form(const void *q, const void *k_cache, const void *k_remote,
                                   const void *v_cache, void *out, float *lse, int B, int Hq,
                                   int Hkv, int L, int Lcap, int D, int w_pretrained, int w0,
                                   float rope_theta, int out_dtype, void *workspace,
                                   size_t workspace_bytes, jl_stream_t stream);

/*
 * Write keys into the true-position cache (§3.2): for t < n,
 *   k_cache[b, pos0 + t, h, :] = RoPE(k[b, t, h, :], pos0 + t).
 *
 *   k        [B, n, Hkv, D] BF16 pre-RoPE keys (read)
 *   k_cache  [B, Lcap, Hkv, D] BF16 (rows [pos0, pos0 + n) written)
 *   0 <= pos0, n >= 1, pos0 + n <= Lcap, 1 <= B <= 65535.
 */
JL_API int jetlong_rope_cache(const void *k, void *k_cache, int B, int n, int Hkv, int D,
                       int pos0, int Lcap, float rope_theta, jl_stream_t stream);

/*
 * Synchronise `stream` and report kernel-side failures since the last call:
 * JL_ERR_DEVICE_TIMEOUT if a bounded wait expired in any kernel of this
 * library on the current device, JL_ERR_RANGE if a prefill met an input
 * outside the FP16 operand range, JL_ERR_CUDA if the stream reports an error,
 * else JL_OK.  Clears the recorded report.
 */
JL_API int jetlong_device_status(jl_stream_t stream);

/*
 * Diagnostic for the failure path above (no counterpart in the paper).
 * Launches one thread that waits on a shared-memory mbarrier no one ever
 * arrives at, with the same bounded wait the attention kernels use, here
 * limited to limit_ms milliseconds (1 <= limit_ms <= 2000).  The wait gives
 * up and records JL_ERR_DEVICE_TIMEOUT exactly as an expired wait in a real
 * kernel does; the next jetlong_device_status() returns it and clears it.
 * Nothing faults or hangs, and the context stays usable.  Note that a
 * prefill launched while the report is set ends at once without computing
 * (it honours the earlier failure), so read the status first.
 * Returns JL_OK if launched, JL_ERR_SHAPE for a limit out of range.
 */
JL_API int jetlong_check_device_timeout(int limit_ms, jl_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* JETLONG_H */
