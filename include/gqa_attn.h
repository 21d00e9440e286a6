/*
 * gqa_attn.h -- C ABI of libgqa_attn.so: the attention sub-block of a Qwen3-style
 * decoder layer on one NVIDIA B200 (sm_100a):
 *
 *     q-hat = RoPE(RMSNorm(q; w_q, eps); pos)      k-hat = RoPE(RMSNorm(k; w_k, eps); pos)
 *     out   = softmax(q-hat k-hat^T / sqrt(D) + M) V       (M: causal mask, GQA sharing)
 *
 * Sources, by page title and section:
 *   "Qwen3系列1-理论基础&真实结构": D1-4 (softmax(QK^T/sqrt(d_k) + M) V, one softmax per
 *       row), D1-5 (causal mask: row i sees keys j <= i), D2-1 (RMSNorm), D2-2 (QK-Norm
 *       per head, then RoPE; V untouched; one weight vector for all Q heads and one for
 *       all K heads; RoPE as 2x2 rotations of adjacent pairs), D2-3 (GQA; prefill writes
 *       K/V to the cache and is compute-bound; decode feeds one token and is
 *       bandwidth-bound).
 *   "深入剖析Qwen3模型架构": 3.1.2 (GQA via repeat_interleave of K/V over query heads,
 *       so query head hq reads KV head hq / (H/Hkv); RoPE pairs x[2i], x[2i+1]),
 *       3.4.1 (RoPE frequencies base^(-2i/D), base raised to 1e6).
 *   "Qwen3学习日志" section 一 (H query heads in groups of h = H/Hkv sharing a K/V head;
 *       Hkv = H is MHA, Hkv = 1 is MQA).
 *   "Qwen3" (nano-vllm walkthrough), "Attention 的 Forward 流程": q/k norm, then rotary
 *       embedding, then attention that reads and writes the KV cache.
 *
 * Conventions shared by every entry point:
 *   - All tensor pointers are DEVICE pointers (cudaMalloc'd or equivalent) owned by the
 *     caller; the library allocates nothing, keeps no per-call state and never frees.
 *   - bf16 tensors are IEEE bfloat16, row-major, contiguous, 16-byte aligned.
 *   - D (head_dim) must be 128; other values return GQA_ERR_UNSUPPORTED.
 *   - H % Hkv == 0 is required (GQA_ERR_INVALID_ARG otherwise).
 *   - RoPE rotates adjacent pairs (x[2i], x[2i+1]) by pos * theta^(-2i/D), i = 0..D/2-1.
 *   - RMSNorm: w_d * x_d / sqrt(mean(x^2) + eps), over one head vector.
 *   - `stream` is a cudaStream_t passed as void* (NULL = the legacy default stream).
 *     Calls are asynchronous on that stream: they validate host-visible arguments,
 *     enqueue kernels and return.  They never throw and never synchronize.
 *   - Argument errors are reported before anything is launched.  Launch failures
 *     return GQA_ERR_CUDA.  Conditions only the GPU can see (a bounded wait that ran
 *     out, a device-side length outside its bound) set a device error word, read and
 *     cleared by gqa_attn_device_status().
 */
#ifndef GQA_ATTN_H
#define GQA_ATTN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    GQA_OK = 0,
    GQA_ERR_INVALID_ARG = -1,    /* bad pointer, shape, alignment or value */
    GQA_ERR_UNSUPPORTED = -2,    /* valid but not implemented (D != 128) */
    GQA_ERR_WORKSPACE = -3,      /* workspace missing, misaligned or too small */
    GQA_ERR_CUDA = -4,           /* a CUDA runtime/driver call or a launch failed */
    GQA_ERR_DEVICE_TIMEOUT = -5, /* a kernel gave up a bounded wait (device status) */
    GQA_ERR_DEVICE_INPUT = -6    /* a device-side length was out of range (device status) */
} gqa_status;

/* Human-readable name of a status code (static string, never NULL). */
const char *gqa_status_string(gqa_status status);

/* Bytes of the RoPE cos/sin table for n tokens: round_up(n, 128) * D * 4, with D = 128. */
#define GQA_ROPE_TABLE_BYTES(n) ((((size_t)(n) + 127) / 128) * 128 * 128 * 4)

/* Workspace bytes gqa_attn_prefill needs for these sizes: k-hat (bf16 [B,T,Hkv,D],
 * rounded up to 256 bytes) and the RoPE cos/sin table of the B*T tokens
 * (GQA_ROPE_TABLE_BYTES(B*T)).  Returns 0 for an empty problem or invalid sizes. */
size_t gqa_attn_prefill_workspace_size(int B, int T, int H, int Hkv, int D);

/*
 * Prefill: causal grouped-query self-attention over whole sequences, with the q/k
 * RMSNorm and RoPE applied inside ("Qwen3" walkthrough forward steps 4-6;
 * "Qwen3系列1" D1-4, D1-5, D2-1, D2-2; "深入剖析Qwen3模型架构" 3.1.2, 3.4.1).
 *
 *   q        bf16 [B, T, H,   D]   raw (pre-norm, pre-RoPE) queries
 *   k, v     bf16 [B, T, Hkv, D]   raw keys (normed and rotated here) and values
 *   pos      int32 [B, T]          RoPE position of every token (only RoPE reads it;
 *                                  the causal mask is on the token index t)
 *   qnorm_w, knorm_w  fp32 [D]     RMSNorm weights shared by all Q heads / all K heads
 *   theta    RoPE base (> 0), e.g. 1e6;   eps  RMSNorm epsilon (>= 0), e.g. 1e-6
 *   out      fp32 [B, T, H, D]     out[b,t,hq] = sum_{j<=t} p_j v[b,j,hq/(H/Hkv)]
 *   workspace  device buffer of >= gqa_attn_prefill_workspace_size(...) bytes,
 *              256-byte aligned; fully overwritten; may be reused between calls
 *              issued on the same stream.
 *
 * B = 0 or T = 0 is a no-op returning GQA_OK.  Calls that overlap on the GPU must not
 * share a workspace.
 */
gqa_status gqa_attn_prefill(const void *q, const void *k, const void *v, const int32_t *pos,
                            const float *qnorm_w, const float *knorm_w, float theta, float eps,
                            float *out, int B, int T, int H, int Hkv, int D, void *workspace,
                            size_t workspace_bytes, void *stream);

/*
 * The two stages of gqa_attn_prefill, callable on their own (gqa_attn_prefill is
 * exactly gqa_attn_k_norm_rope into its workspace followed by gqa_attn_prefill_khat).
 *
 * gqa_attn_k_norm_rope: k_hat = RoPE(RMSNorm(k; knorm_w, eps); pos), written as bf16
 * in the layout of k.  These are the keys the KV cache holds ("Qwen3系列1" D2-3: K is
 * written to the cache after its norm and rotation, before attention), so the output
 * can be a decode cache directly.
 *   k        bf16 [N, Hkv, D] (N = B*T tokens, any token order); pos int32 [N]
 *   k_hat    bf16 [N, Hkv, D], must not overlap k.   N = 0 is a no-op.
 *   rope_cs  NULL, or GQA_ROPE_TABLE_BYTES(N) bytes (16-byte aligned) that receive the
 *            cos/sin of every token's RoPE angles pos * theta^(-2i/D) in the library's
 *            blocked layout (an opaque intermediate), for gqa_attn_prefill_khat to reuse.
 */
gqa_status gqa_attn_k_norm_rope(const void *k, const int32_t *pos, const float *knorm_w, float theta,
                                float eps, void *k_hat, float *rope_cs, int64_t N, int Hkv, int D,
                                void *stream);

/*
 * gqa_attn_prefill_khat: the attention stage of gqa_attn_prefill on keys that are
 * already normed and rotated (k_hat, e.g. from gqa_attn_k_norm_rope): the raw q tiles
 * are normed (qnorm_w, eps) and rotated (pos, theta) inside the attention kernel.
 * Arguments as for gqa_attn_prefill; k_hat is bf16 [B, T, Hkv, D].  rope_cs is the
 * table gqa_attn_k_norm_rope wrote for the same B*T tokens (flattened b*T + t),
 * positions and theta, or NULL (the kernel then evaluates cos/sin itself, slower).
 * Needs no workspace.
 */
gqa_status gqa_attn_prefill_khat(const void *q, const void *k_hat, const void *v, const int32_t *pos,
                                 const float *rope_cs, const float *qnorm_w, float theta, float eps,
                                 float *out, int B, int T, int H, int Hkv, int D, void *stream);

/* Workspace bytes gqa_attn_decode needs: split-KV partial results for up to max_len
 * cached tokens per sequence.  Returns 0 for an empty problem or invalid sizes. */
size_t gqa_attn_decode_workspace_size(int B, int H, int Hkv, int D, int max_len);

/*
 * Decode: one new query token per sequence attends to that sequence's KV cache
 * ("Qwen3系列1" D2-3: the cache holds K and V per KV head, written before attention;
 * decode feeds a single token and is bound by reading the cache).
 *
 *   q         bf16 [B, H, D]        raw query of the new token; RMSNorm(qnorm_w, eps) and
 *                                   RoPE at position q_pos[b] are applied here
 *   k_cache   bf16 [rows, Hkv, D]   cached keys, already normed and rotated
 *   v_cache   bf16 [rows, Hkv, D]   cached values
 *   cache_offsets int64 [B + 1]     sequence b owns rows cache_offsets[b] ..
 *                                   cache_offsets[b+1]-1 (non-decreasing)
 *   seqlens   int32 [B]             number of valid cached rows of sequence b:
 *                                   1 <= seqlens[b] <= max_len and
 *                                   seqlens[b] <= cache_offsets[b+1] - cache_offsets[b];
 *                                   every one of them is visible to the query
 *   q_pos     int32 [B] or NULL     RoPE position of the query (NULL: seqlens[b])
 *   out       fp32 [B, H, D]
 *   max_len   host-side upper bound on seqlens (sizes the workspace)
 *   workspace >= gqa_attn_decode_workspace_size(B, H, Hkv, D, max_len) bytes,
 *             256-byte aligned; fully overwritten each call.
 *
 * cache_offsets, seqlens and q_pos live on the device, so their values are checked on
 * the device: a sequence that breaks the bounds above gets NaN output, reads nothing
 * outside its rows, and sets GQA_ERR_DEVICE_INPUT in the device status word.
 * B = 0 is a no-op returning GQA_OK.
 */
gqa_status gqa_attn_decode(const void *q, const void *k_cache, const void *v_cache,
                           const int64_t *cache_offsets, const int32_t *seqlens,
                           const int32_t *q_pos, const float *qnorm_w, float theta, float eps,
                           float *out, int B, int H, int Hkv, int D, int max_len,
                           void *workspace, size_t workspace_bytes, void *stream);

/*
 * Decode step that first appends the new token to the cache, then attends
 * ("Qwen3系列1" D2-3: the new token's K and V are written into the per-layer cache
 * before attention; "Qwen3" walkthrough, attention forward: q and k are normed, then
 * rotated).  For sequence b with seqlens[b] = n cached rows:
 *   row n of the sequence (row cache_offsets[b] + n) receives
 *     K: RoPE(RMSNorm(k_new[b, g]; knorm_w, eps), position) rounded to bf16,
 *     V: v_new[b, g] unchanged,
 *   and the query, normed and rotated at the same position, attends to rows 0 .. n
 *   (n + 1 keys).  position = q_pos[b], or n when q_pos is NULL.
 *
 *   q          bf16 [B, H, D]        raw query of the new token
 *   k_new      bf16 [B, Hkv, D]      raw key of the new token (8-byte aligned)
 *   v_new      bf16 [B, Hkv, D]      value of the new token (8-byte aligned)
 *   k_cache, v_cache  bf16 [rows, Hkv, D]  written at row n of each sequence, read at 0 .. n
 *   cache_offsets, q_pos, qnorm_w, theta, eps, out, workspace: as for gqa_attn_decode
 *   seqlens    int32 [B]             rows cached before the step: 0 <= seqlens[b],
 *                                    seqlens[b] + 1 <= max_len and
 *                                    seqlens[b] + 1 <= cache_offsets[b+1] - cache_offsets[b]
 *   knorm_w    fp32 [D]              k RMSNorm weight (16-byte aligned)
 *   max_len    host-side upper bound on seqlens[b] + 1 (sizes the workspace)
 *
 * seqlens is not modified: the caller advances it after the step.  The K/V rows of the
 * new token are in place when the call's work completes on the stream.  A sequence that
 * breaks the bounds above is not written, gets NaN output and sets
 * GQA_ERR_DEVICE_INPUT in the device status word.  Null k_new, v_new or knorm_w is
 * GQA_ERR_INVALID_ARG; every other host-side check is gqa_attn_decode's.
 */
gqa_status gqa_attn_decode_append(const void *q, const void *k_new, const void *v_new, void *k_cache,
                                  void *v_cache, const int64_t *cache_offsets, const int32_t *seqlens,
                                  const int32_t *q_pos, const float *qnorm_w, const float *knorm_w,
                                  float theta, float eps, float *out, int B, int H, int Hkv, int D,
                                  int max_len, void *workspace, size_t workspace_bytes, void *stream);

/* Size of the library's built-in decode scratch used by gqa_attn_decode_noalloc. */
#define GQA_NOALLOC_SCRATCH_BYTES (32u << 20)

/*
 * gqa_attn_decode_noalloc: gqa_attn_decode for callers that cannot hand the library a
 * workspace and cannot allocate one, for example a plugin running inside a host
 * framework that owns every byte of device memory, or a latency-critical serving loop
 * that must not call cudaMalloc (which may synchronize the device).  The pages have no
 * counterpart of this entry point; it exists only for such callers.
 *
 * Same arguments, results and device-side checks as gqa_attn_decode, minus the
 * workspace: the split-KV partial results go to a scratch array that is part of the
 * library itself (GQA_NOALLOC_SCRATCH_BYTES of device memory that every GPU which
 * loads the library holds until the process exits).  No call allocates or frees.
 *   - Every argument check of gqa_attn_decode runs first, with the same status codes.
 *     Then problems whose partials need more than GQA_NOALLOC_SCRATCH_BYTES, i.e.
 *     gqa_attn_decode_workspace_size(B, H, Hkv, D, max_len) > GQA_NOALLOC_SCRATCH_BYTES,
 *     are rejected with GQA_ERR_WORKSPACE before anything is launched.
 *   - The first call on a device looks up the scratch array's device address (once per
 *     device, with that device current); make that first call before any stream capture.
 *   - All calls on a device share the one scratch array, and it keeps the last call's
 *     contents (nothing in it has to start at zero).  Calls that overlap on the GPU
 *     (different streams without ordering between them) race on it and give undefined
 *     results: serialize them.
 */
gqa_status gqa_attn_decode_noalloc(const void *q, const void *k_cache, const void *v_cache,
                                   const int64_t *cache_offsets, const int32_t *seqlens,
                                   const int32_t *q_pos, const float *qnorm_w, float theta,
                                   float eps, float *out, int B, int H, int Hkv, int D,
                                   int max_len, void *stream);

/* ----------------------------------------------------------------- RoPE variants
 *
 * The entry points above rotate adjacent pairs (x[2i], x[2i+1]) by pos * theta_i with
 * theta_i = theta^(-2i/D) ("Qwen3系列1" D2-2; "深入剖析Qwen3模型架构" 3.1.2, 3.4.1).
 * The _ex forms below take a gqa_rope_config instead of theta, for the variants a
 * long-context deployment uses:
 *
 *   pairing  GQA_ROPE_PAIR_ADJACENT: (x[2i], x[2i+1]), as above
 *            GQA_ROPE_PAIR_HALF:     (x[i], x[i + D/2]) (the rotate-half layout)
 *   scaling  GQA_ROPE_SCALE_NONE:    theta_i
 *            GQA_ROPE_SCALE_LINEAR:  theta_i / factor, i.e. the position divided by the
 *                                    extension factor (linear interpolation, 4.2
 *                                    "序列长度扩展的技术方案" of the zizhi168.cn summary of
 *                                    the Qwen3 report)
 *            GQA_ROPE_SCALE_NTK:     (theta * factor^(D/(D-2)))^(-2i/D), the NTK-aware base
 *                                    change (the page's 4.2 formula is garbled; this is the
 *                                    published form)
 *            GQA_ROPE_SCALE_YARN:    YaRN's "NTK-by-parts" (Peng et al. 2023; the page's
 *                                    3.4.2 formula is garbled): with r_i = L theta_i / (2 pi),
 *                                    L = original_max_position, and gamma_i =
 *                                    clamp((r_i - beta_slow) / (beta_fast - beta_slow), 0, 1),
 *                                    theta_i ((1 - gamma_i) / factor + gamma_i); the attention
 *                                    logits are multiplied by (0.1 ln(factor) + 1)^2, YaRN's
 *                                    temperature.  The stored k-hat is not scaled by it.
 *
 * factor must be finite and >= 1 for a scaled variant (1 gives the plain frequencies);
 * YaRN also needs original_max_position >= 1 and finite beta_fast > beta_slow (the YaRN
 * paper uses 32 and 1).  theta must be finite and > 0.  An invalid configuration or a
 * NULL pointer is GQA_ERR_INVALID_ARG.  k-hat written and RoPE tables filled with one
 * configuration must be read with the same one.
 */
typedef enum { GQA_ROPE_PAIR_ADJACENT = 0, GQA_ROPE_PAIR_HALF = 1 } gqa_rope_pairing;
typedef enum {
    GQA_ROPE_SCALE_NONE = 0,
    GQA_ROPE_SCALE_LINEAR = 1,
    GQA_ROPE_SCALE_NTK = 2,
    GQA_ROPE_SCALE_YARN = 3
} gqa_rope_scaling;

typedef struct {
    double theta;               /* frequency base */
    int pairing;                /* gqa_rope_pairing */
    int scaling;                /* gqa_rope_scaling */
    double factor;              /* context extension factor s (scaled variants) */
    int original_max_position;  /* YaRN: training context length L */
    double beta_fast;           /* YaRN: ramp end (pairs with more wavelengths keep theta_i) */
    double beta_slow;           /* YaRN: ramp start (pairs with fewer get theta_i / s) */
} gqa_rope_config;

/* gqa_attn_prefill with a RoPE variant (the same variant for q and k). */
gqa_status gqa_attn_prefill_ex(const void *q, const void *k, const void *v, const int32_t *pos,
                               const float *qnorm_w, const float *knorm_w,
                               const gqa_rope_config *rope, float eps, float *out, int B, int T,
                               int H, int Hkv, int D, void *workspace, size_t workspace_bytes,
                               void *stream);

/* gqa_attn_k_norm_rope with a RoPE variant; the table it fills holds that variant's
 * cos/sin. */
gqa_status gqa_attn_k_norm_rope_ex(const void *k, const int32_t *pos, const float *knorm_w,
                                   const gqa_rope_config *rope, float eps, void *k_hat,
                                   float *rope_cs, int64_t N, int Hkv, int D, void *stream);

/* gqa_attn_prefill_khat with a RoPE variant (the one k_hat and rope_cs were made with). */
gqa_status gqa_attn_prefill_khat_ex(const void *q, const void *k_hat, const void *v,
                                    const int32_t *pos, const float *rope_cs,
                                    const float *qnorm_w, const gqa_rope_config *rope, float eps,
                                    float *out, int B, int T, int H, int Hkv, int D, void *stream);

/* gqa_attn_decode with a RoPE variant (the one the cached keys were rotated with). */
gqa_status gqa_attn_decode_ex(const void *q, const void *k_cache, const void *v_cache,
                              const int64_t *cache_offsets, const int32_t *seqlens,
                              const int32_t *q_pos, const float *qnorm_w,
                              const gqa_rope_config *rope, float eps, float *out, int B, int H,
                              int Hkv, int D, int max_len, void *workspace,
                              size_t workspace_bytes, void *stream);

/* gqa_attn_decode_append with a RoPE variant (for the appended key and the query). */
gqa_status gqa_attn_decode_append_ex(const void *q, const void *k_new, const void *v_new,
                                     void *k_cache, void *v_cache, const int64_t *cache_offsets,
                                     const int32_t *seqlens, const int32_t *q_pos,
                                     const float *qnorm_w, const float *knorm_w,
                                     const gqa_rope_config *rope, float eps, float *out, int B,
                                     int H, int Hkv, int D, int max_len, void *workspace,
                                     size_t workspace_bytes, void *stream);

/* ----------------------------------------------------------------- packed and chunked prefill
 *
 * Variable-length prefill: B sequences of different lengths packed one after another
 * ("Qwen3系列1" D1-5: the causal mask applies within each sequence; "Qwen3" walkthrough,
 * "Attention 的 Forward 流程": the q/k/v of a batch arrive as one [N, heads, D] tensor).
 *
 *   q         bf16 [N, H, D]      raw queries of all N tokens, sequence after sequence
 *   k, v      bf16 [N, Hkv, D]    raw keys (normed and rotated here) and values
 *   pos       int32 [N]           RoPE position of every token
 *   cu_seqlens int64 [B + 1]      device: sequence b is tokens cu_seqlens[b] ..
 *                                 cu_seqlens[b+1] - 1 (0 = cu_seqlens[0] <= ... <=
 *                                 cu_seqlens[B] = N; empty sequences are allowed)
 *   qnorm_w, knorm_w, rope, eps   as for gqa_attn_prefill_ex (rope must not be NULL)
 *   out       fp32 [N, H, D]      row t of sequence b attends to keys 0 .. t of b only
 *   max_seqlen host-side bound on every sequence's length (sizes the launch)
 *   workspace >= gqa_attn_prefill_varlen_workspace_size(N, Hkv, D) bytes, 256-byte
 *             aligned (k-hat of the N tokens, their RoPE cos/sin, and the list of the
 *             (sequence, 128-token query block) pairs that have work, which a small kernel
 *             writes before the attention kernel so that no CTA is dealt empty work).
 * Sequence bounds are read on the device: a sequence that breaks them (or is longer than
 * max_seqlen, whose tail then goes unwritten) is skipped and sets GQA_ERR_DEVICE_INPUT;
 * its output rows are undefined.  B = 0, N = 0 or max_seqlen = 0 is a no-op.
 */
size_t gqa_attn_prefill_varlen_workspace_size(int64_t N, int Hkv, int D);
gqa_status gqa_attn_prefill_varlen(const void *q, const void *k, const void *v, const int32_t *pos,
                                   const int64_t *cu_seqlens, const float *qnorm_w,
                                   const float *knorm_w, const gqa_rope_config *rope, float eps,
                                   float *out, int B, int64_t N, int H, int Hkv, int D,
                                   int max_seqlen, void *workspace, size_t workspace_bytes,
                                   void *stream);

/*
 * Chunked prefill: each sequence already has prefix_len[b] rows in the KV cache (from an
 * earlier prefill or chunk) and a new chunk of tokens arrives ("Qwen3系列1" D2-3: the
 * keys and values of earlier tokens live in the per-layer cache, which grows along the
 * tokens; K/V are written into it before attention).  The call first writes the chunk's
 * k-hat (RMSNorm + RoPE at pos) and v into the cache, right after the cached rows, then
 * chunk row t of sequence b (token prefix_len[b] + t) attends to cache rows
 * 0 .. prefix_len[b] + t of that sequence.
 *
 *   q, k, v, pos, cu_seqlens, out  the N chunk tokens, packed as for gqa_attn_prefill_varlen
 *   k_cache, v_cache  bf16 [cache_rows, Hkv, D]; sequence b owns rows cache_offsets[b] ..
 *                     cache_offsets[b+1] - 1 and must have room for prefix_len[b] +
 *                     chunk length rows; the chunk's rows are written in place
 *   cache_offsets     int64 [B + 1], device, non-decreasing
 *   prefix_len        int32 [B], device, rows already cached (0 = plain prefill of the chunk)
 *   max_chunk_len     host-side bound on every chunk's length
 *   workspace >= gqa_attn_prefill_chunk_workspace_size(N, D) bytes, 256-byte aligned
 *             (the chunk tokens' RoPE cos/sin and the list of the (sequence, query block)
 *             pairs that have work, as for gqa_attn_prefill_varlen).
 * A chunk token whose cache row falls outside its sequence's rows is not written and
 * sets GQA_ERR_DEVICE_INPUT (that sequence's output is then undefined); the same for
 * sequence bounds out of range.  prefix_len is not advanced (the caller does that).
 * Keys are read in 128-row tiles from cache_offsets[b]: up to 127 cache rows after a
 * sequence's last key are read and weighted by zero, so they must hold finite values.
 */
size_t gqa_attn_prefill_chunk_workspace_size(int64_t N, int D);
gqa_status gqa_attn_prefill_chunk(const void *q, const void *k, const void *v, const int32_t *pos,
                                  const int64_t *cu_seqlens, void *k_cache, void *v_cache,
                                  const int64_t *cache_offsets, const int32_t *prefix_len,
                                  int64_t cache_rows, const float *qnorm_w, const float *knorm_w,
                                  const gqa_rope_config *rope, float eps, float *out, int B,
                                  int64_t N, int H, int Hkv, int D, int max_chunk_len,
                                  void *workspace, size_t workspace_bytes, void *stream);

/*
 * Chunked prefill on a paged KV cache: as gqa_attn_prefill_chunk, with cached row r of
 * sequence b kept as row r % page_size of page page_table[b * max_pages + r / page_size]
 * (the decode-side paged layout).  The chunk's k-hat and v are written into the pages at
 * rows prefix_len[b] .. prefix_len[b] + chunk length - 1 of the sequence, then the chunk
 * attends to rows 0 .. prefix_len[b] + t through the page table.
 *
 *   k_pages, v_pages  bf16 [num_pages, page_size, Hkv, D]; the pages the table names for the
 *                     chunk's rows must exist (allocated by the caller)
 *   page_table        int32 [B, max_pages], device; entries past a sequence's rows are unused
 *   page_size         a multiple of 16 (else GQA_ERR_INVALID_ARG) that divides 128 or is a
 *                     multiple of 128 (so that a 128-key tile is whole pages or lies inside
 *                     one page; else GQA_ERR_UNSUPPORTED); num_pages * page_size < 2^31 - 256
 *   workspace >= gqa_attn_prefill_chunk_paged_workspace_size(N, D) bytes (as for
 *             gqa_attn_prefill_chunk).
 * A chunk row behind a page id outside [0, num_pages) (or past max_pages) is not written,
 * and a visible key behind one is read as zero; both set GQA_ERR_DEVICE_INPUT and leave that
 * sequence's output undefined.  Page segments of a 128-key tile past a sequence's last key
 * are not read; the rows after the last key inside its last page are read and weighted by
 * zero, so they must hold finite values (zeros, or finite rows written earlier).
 */
size_t gqa_attn_prefill_chunk_paged_workspace_size(int64_t N, int D);
gqa_status gqa_attn_prefill_chunk_paged(const void *q, const void *k, const void *v, const int32_t *pos,
                                        const int64_t *cu_seqlens, void *k_pages, void *v_pages,
                                        const int32_t *page_table, int num_pages, int page_size,
                                        int max_pages, const int32_t *prefix_len, const float *qnorm_w,
                                        const float *knorm_w, const gqa_rope_config *rope, float eps,
                                        float *out, int B, int64_t N, int H, int Hkv, int D,
                                        int max_chunk_len, void *workspace, size_t workspace_bytes,
                                        void *stream);

/* ----------------------------------------------------------------- paged KV cache
 *
 * The decode cache may also live in fixed-size pages (the layout of paged-attention
 * servers): k_pages and v_pages are bf16 [num_pages, page_size, Hkv, D], and row r of
 * sequence b is row r % page_size of page page_table[b * max_pages_per_seq +
 * r / page_size].  page_table is int32 [B, max_pages_per_seq] on the device; page_size
 * is a multiple of 16 (>= 16).  A sequence may use at most max_pages_per_seq *
 * page_size rows.  The calls otherwise behave as gqa_attn_decode_ex /
 * gqa_attn_decode_append_ex (the append writes the new row into its page).  Page ids are
 * checked on the device: a sequence with an id outside [0, num_pages) among the pages it
 * reads gets NaN output, reads no page memory through that id, and sets
 * GQA_ERR_DEVICE_INPUT.  The workspace is gqa_attn_decode_workspace_size(B, H, Hkv, D,
 * max_len).  rope must not be NULL.  This layout is not on the pages; it follows the
 * paged KV cache that serving engines use, so that a cache managed that way needs no
 * copy into one contiguous block per sequence.
 */
gqa_status gqa_attn_decode_paged(const void *q, const void *k_pages, const void *v_pages,
                                 const int32_t *page_table, int num_pages, int page_size,
                                 int max_pages_per_seq, const int32_t *seqlens,
                                 const int32_t *q_pos, const float *qnorm_w,
                                 const gqa_rope_config *rope, float eps, float *out, int B, int H,
                                 int Hkv, int D, int max_len, void *workspace,
                                 size_t workspace_bytes, void *stream);

gqa_status gqa_attn_decode_append_paged(const void *q, const void *k_new, const void *v_new,
                                        void *k_pages, void *v_pages, const int32_t *page_table,
                                        int num_pages, int page_size, int max_pages_per_seq,
                                        const int32_t *seqlens, const int32_t *q_pos,
                                        const float *qnorm_w, const float *knorm_w,
                                        const gqa_rope_config *rope, float eps, float *out, int B,
                                        int H, int Hkv, int D, int max_len, void *workspace,
                                        size_t workspace_bytes, void *stream);

/* ----------------------------------------------------------------- projections
 *
 * The dense contractions around the attention ("Qwen3" walkthrough, "Attention 的
 * Forward 流程": step 1 qkv = qkv_proj(hidden_states), split and viewed per head in
 * steps 2-3; step 7 output = o_proj(o.flatten(1, -1)); "Qwen3系列1" D1-2: a linear layer
 * is Y = XW + b and Qwen3's projections have no b; D1-4 Q4/Q5: the heads are
 * concatenated, then multiplied by W_O):
 *
 *     y[m][n] = sum_k x[m][k] w[n][k]          (nn.Linear: y = x W^T, no bias)
 *
 *   x   bf16 [M, K] row-major      w  bf16 [N, K] row-major (one output feature per row)
 *   y   [M, N] row-major, bf16 (GQA_DTYPE_BF16, rounded to nearest even) or fp32
 *       (GQA_DTYPE_F32); fp32 accumulation on the tensor cores either way
 *   N must be a multiple of 32 and K of 8; M >= 0 (0 is a no-op).  All pointers 16-byte
 *   aligned device memory.  The fused QKV projection is gqa_linear with w = [W_q; W_k;
 *   W_v] ((H + 2 Hkv) D rows): its output [M, H + 2 Hkv, D] is read in place by
 *   gqa_attn_block_prefill.
 */
typedef enum { GQA_DTYPE_BF16 = 0, GQA_DTYPE_F32 = 1 } gqa_dtype;

gqa_status gqa_linear(const void *x, const void *w, void *y, int y_dtype, int64_t M, int N, int K,
                      void *stream);

/*
 * The whole attention sub-block of a decoder layer for a prefill (the seven steps of the
 * "Qwen3" walkthrough's Qwen3Attention.forward): qkv = x W_qkv^T (bf16), split into
 * q [.., H, D], k [.., Hkv, D], v [.., Hkv, D]; q/k RMSNorm; RoPE; causal GQA attention
 * (bf16 output, the dtype the projection reads); y = o W_o^T over the concatenated heads.
 *
 *   x      bf16 [B*T, hidden]          hidden states of B sequences of T tokens
 *   w_qkv  bf16 [(H + 2 Hkv) D, hidden] = [W_q; W_k; W_v]
 *   w_o    bf16 [hidden, H D]
 *   pos, qnorm_w, knorm_w, rope, eps   as for gqa_attn_prefill_ex (rope not NULL)
 *   y      fp32 [B*T, hidden]
 *   workspace >= gqa_attn_block_prefill_workspace_size(...) bytes, 256-byte aligned:
 *          qkv, k-hat, the RoPE table and the attention output.
 * hidden must be a multiple of 32.  B = 0 or T = 0 is a no-op.
 */
size_t gqa_attn_block_prefill_workspace_size(int B, int T, int hidden, int H, int Hkv, int D);
gqa_status gqa_attn_block_prefill(const void *x, const void *w_qkv, const void *w_o, const int32_t *pos,
                                  const float *qnorm_w, const float *knorm_w,
                                  const gqa_rope_config *rope, float eps, float *y, int B, int T,
                                  int hidden, int H, int Hkv, int D, void *workspace,
                                  size_t workspace_bytes, void *stream);

/*
 * Device status: waits for `stream` (a cudaStream_t as void*, NULL = legacy default
 * stream), then reads and clears the library's device error word on the current
 * device.  Returns GQA_OK, GQA_ERR_DEVICE_TIMEOUT (a kernel gave up a bounded wait and
 * returned early; its outputs are invalid), GQA_ERR_DEVICE_INPUT (a decode sequence
 * broke its length bounds), or GQA_ERR_CUDA.  This is the only synchronizing call.
 */
gqa_status gqa_attn_device_status(void *stream);

/*
 * Test switch for the failure path, not for production use: while enabled (non-zero),
 * every attention launch makes its MMA-issuing thread first wait on a barrier that
 * nothing signals.  That wait gives up after 100 us and records GQA_ERR_DEVICE_TIMEOUT;
 * the thread then issues nothing, and the CTA's other roles give up their own waits
 * after the usual 2 s limit, let their copies in flight land and release tensor memory,
 * so the launch ends (after a few seconds) with garbage output and the device usable.
 * Call with 0 to switch it off.  It affects launches enqueued while it is on.
 */
void gqa_attn_test_stall(int enable);

#ifdef __cplusplus
}
#endif

#endif /* GQA_ATTN_H */
