/*
 * gqa.h -- C ABI of the B200 (sm_100a) library for causal grouped-query attention
 * with rotary position embedding, optional QK-RMSNorm, prompt prefill and
 * single-token decode against a contiguous per-sequence KV cache.
 *
 * The operations follow these passages:
 *   RoPE: page "750美元从零训练3个LLM：一位开发者的实战复盘", section "V1：现代架构基线"
 *     (q and k turn by a position-dependent angle so that q_m . k_n depends on
 *     m - n only); page "从零手训LLaMa：125M模型11小时训练全记录", section
 *     "核心架构：手动实现LLaMa的四个关键组件".
 *   GQA: same first page, section "V2：引入前沿技术" (query heads form groups that
 *     share one K/V head; query head h reads K/V head h / (Hq / Hkv)).
 *   QK-RMSNorm: page "训练3.8B LLM至0.384 CORE，成本998美元 – Hugo Vergnes",
 *     sections "设置" (QK-norm) and "无效的方法" (F.rms_norm: eps inside the root).
 *   Causal attention: same page, section "无效的方法" (causal
 *     scaled_dot_product_attention, default scale 1/sqrt(D)); page "Build a Large
 *     Language Model from Scratch" (nxbn.cn), section 3.1.
 *   KV cache: page "750美元从零训练3个LLM", section "V3：扩容与推理优化" (the new
 *     token computes its own q, k, v, appends k and v to the cache and attends
 *     over the whole cache); page "从零手训LLaMa", section on batched KV-cache
 *     inference.
 *
 * Conventions shared by every entry point
 *   - bf16 tensors are passed as void* and are row-major and contiguous:
 *       q              [B, T, Hq, D]      (prefill / rope)   [B, Hq, D] (decode)
 *       k, v (new)     [B, T, Hkv, D]                        [B, Hkv, D] (decode)
 *       k_cache/v_cache[B, Hkv, Lmax, D]  (one contiguous [Lmax, D] slab per head)
 *       out            [B, T, Hq, D]      (prefill)          [B, Hq, D] (decode)
 *   - D is 64, 96 or 128; Hq % Hkv == 0 (a GQA group is g = Hq / Hkv heads);
 *     Lmax is a multiple of 128.  Every data pointer is 16-byte aligned.
 *   - All pointers except the stream are DEVICE pointers to caller-owned memory.
 *     The library allocates no memory and keeps no per-call state; it caches
 *     one function pointer (the driver's tensor-map encoder) per process.
 *   - stream is a cudaStream_t (NULL = legacy default stream).  All work is
 *     queued asynchronously on it; the host return code covers argument
 *     validation and launch errors only.
 *   - status_dev, where taken, is an optional device int32 that kernels OR
 *     GQA_DEV_* bits into (NULL: device-side errors are not reported).  The
 *     caller zeroes it and reads it after synchronising.
 *   - RoPE pairs coordinate i with i + D/2 and turns pair i at position p by
 *     p * base^(-2i/D) radians; QK-RMSNorm (unit gain) runs before RoPE.
 *   - scale <= 0 selects 1/sqrt(D).
 *   - Every element written is a bf16 rounded to nearest even from fp32 math.
 */
#ifndef GQA_H_
#define GQA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    GQA_OK = 0,
    GQA_ERR_INVALID_ARG = 1,   /* null pointer, bad size, misalignment, Hq % Hkv != 0 */
    GQA_ERR_UNSUPPORTED = 2,   /* D not in {64, 96, 128}, or a device below sm_100 */
    GQA_ERR_CAPACITY = 3,      /* host-known positions or lengths exceed Lmax */
    GQA_ERR_TIMEOUT = 4,       /* reserved for host-side waits */
    GQA_ERR_CUDA = 5,          /* a CUDA runtime / driver call failed */
    GQA_ERR_WORKSPACE = 6      /* workspace missing or smaller than required */
} gqa_status;

/* Bits OR-ed into *status_dev by kernels. */
#define GQA_DEV_CAPACITY 0x1   /* a sequence's writes or reads would pass Lmax: skipped */
#define GQA_DEV_TIMEOUT 0x2    /* a bounded wait inside a kernel gave up: output invalid */
#define GQA_DEV_BAD_LEN 0x4    /* a length or position < 0 (or 0 where >= 1 is needed) */

/*
 * RoPE for contexts longer than the one a model was trained on.  Page "750美元
 * 从零训练3个LLM" (section "V1：现代架构基线") names NTK-aware scaling and YaRN as
 * the length-extension methods RoPE works with; the formulas are those of the
 * published methods (pair i, theta_i = base^(-2i/D), extension factor s):
 *   GQA_ROPE_LINEAR  position interpolation: theta_i / s
 *   GQA_ROPE_NTK     NTK-aware: the base becomes base * s^(D/(D-2)), so the
 *                    fastest pair keeps its angle and the slowest is divided by s
 *   GQA_ROPE_YARN    YaRN: with r_i = L theta_i / (2 pi) (turns of pair i over the
 *                    trained length L) and g_i = clamp((r_i - alpha)/(beta - alpha),
 *                    0, 1), theta_i' = (1 - g_i) theta_i / s + g_i theta_i; both
 *                    rotated q and k are multiplied by 0.1 ln(s) + 1, which
 *                    divides the logits by the temperature t of the method.
 */
#define GQA_ROPE_PLAIN 0
#define GQA_ROPE_LINEAR 1
#define GQA_ROPE_NTK 2
#define GQA_ROPE_YARN 3

typedef struct {
    int qk_norm;          /* nonzero: unit-gain RMSNorm over D before RoPE */
    float eps;            /* RMSNorm epsilon inside the root (1e-6 in the pages' model) */
    float rope_base;      /* RoPE base (10000) */
    int scaling;          /* GQA_ROPE_*; zero-filled = plain RoPE */
    float factor;         /* s >= 1 (used when scaling != GQA_ROPE_PLAIN) */
    int original_max_pos; /* YaRN: L, the trained context length (>= 1) */
    float yarn_alpha;     /* YaRN: 0 <= alpha < beta (the method's defaults: 1, 32) */
    float yarn_beta;
} gqa_rope_params;

/*
 * gqa_rope_apply -- in place on q [B, T, H, D]: q <- RoPE(RMSNorm?(q)) with token
 * t of sequence b at position pos0[b] + t.
 *   pos0: device int32 [B], or NULL for position 0.
 * Errors: GQA_ERR_INVALID_ARG (q null, B/T/H < 1, misaligned), GQA_ERR_UNSUPPORTED.
 */
gqa_status gqa_rope_apply(void *q, const int32_t *pos0, int B, int T, int H, int D,
                          gqa_rope_params p, void *stream);

/*
 * kv_cache_append -- for every new token t of sequence b and KV head h:
 *     k_cache[b, h, pos0[b] + t, :] = RoPE(RMSNorm?(k[b, t, h, :]))   (bf16)
 *     v_cache[b, h, pos0[b] + t, :] = v[b, t, h, :]                  (bit copy)
 * No other cache slot is touched.
 *   pos0: device int32 [B] (current cache lengths), or NULL for 0.
 *   max_pos0_host: a host-known upper bound of pos0, checked against
 *     max_pos0_host + T <= Lmax (pass -1 to skip the host check).  A sequence
 *     whose pos0[b] + T exceeds Lmax on the device is skipped and
 *     GQA_DEV_CAPACITY is raised.
 *   new_len: optional device int32 [B] output, new_len[b] = pos0[b] + T (the
 *     lengths a following gqa_decode reads).  NULL to skip.
 */
gqa_status kv_cache_append(const void *k, const void *v, void *k_cache, void *v_cache,
                           const int32_t *pos0, int max_pos0_host, int32_t *new_len,
                           int B, int T, int Hkv, int D, int Lmax, gqa_rope_params p,
                           int32_t *status_dev, void *stream);

/*
 * gqa_rope_append -- gqa_rope_apply on q [B, T, Hq, D] and kv_cache_append of
 * k, v in ONE launch (the same positions pos0[b] + t for q and k).  Arguments
 * as in the two calls above.
 */
gqa_status gqa_rope_append(void *q, const void *k, const void *v, void *k_cache,
                           void *v_cache, const int32_t *pos0, int max_pos0_host,
                           int32_t *new_len, int B, int T, int Hq, int Hkv, int D,
                           int Lmax, gqa_rope_params p, int32_t *status_dev, void *stream);

/*
 * gqa_prefill -- causal attention of a prompt that starts at position 0:
 *     out[b, t, h, :] = sum_{s <= t} softmax_s(q[b,t,h,:] . K[b, h/g, s, :] * scale)
 *                                   * V[b, h/g, s, :]
 * q must already be rotated (gqa_rope_apply / gqa_rope_append) and the caches
 * must hold the prompt's rotated K and raw V in slots 0 .. T-1 (slots >= T are
 * never read).  Tensor-core kernel (tcgen05 / TMEM, TMA-fed), fp32 softmax.
 *   T <= Lmax.  Alignment: 16 bytes for every pointer.
 * Device errors: GQA_DEV_TIMEOUT (a bounded pipeline wait expired).
 * Scheduling: work items are pairs of 128-row query tiles that share a KV
 * head (two heads of one tile, or two consecutive tiles); with four or more
 * items per SM, the CTAs take items from a counter in device memory (one of 256 slots per device, taken round
 * robin by each call and reset by its last CTA), so up to 256 calls of
 * gqa_prefill, _chunk, _docs or _lse may be in flight on a device at once; a
 * CUDA graph replays the slot it captured, so replays of one graph must not
 * overlap each other.  The same holds for the three other prefill entries.
 */
gqa_status gqa_prefill(const void *q, const void *k_cache, const void *v_cache, void *out,
                       int B, int T, int Hq, int Hkv, int D, int Lmax, float scale,
                       int32_t *status_dev, void *stream);

/*
 * gqa_prefill_chunk -- causal attention of T new tokens per sequence that
 * continue a cached prefix (chunked prefill, multi-turn continuation, a batch of
 * prompts of different cached lengths): query t of sequence b sits at position
 * p = pos0[b] + t and attends to every cache slot s <= p,
 *     out[b, t, h, :] = sum_{s <= pos0[b]+t} softmax_s(q[b,t,h,:] . K[b, h/g, s, :] * scale)
 *                                            * V[b, h/g, s, :]
 * the KV-cache step of page "750美元从零训练3个LLM" (section "V3：扩容与推理优化")
 * taken T tokens at a time.  q must be rotated at those positions and the
 * caches must hold the prefix (slots < pos0[b]) and the chunk's own rotated K
 * and raw V (slots pos0[b] .. pos0[b] + n_tok[b] - 1): gqa_rope_append with the
 * same pos0 does both.  Cache slots from pos0[b] + n_tok[b] on are never used and
 * may hold anything (NaN included).  Same kernel as gqa_prefill.
 *   pos0: device int32 [B] (required); n_tok: device int32 [B], the number of
 *     valid new tokens of sequence b (0 .. T), or NULL for T everywhere.  Rows
 *     t >= n_tok[b] of out are not written.  A sequence with pos0[b] < 0, n_tok
 *     outside 0 .. T or pos0[b] + n_tok[b] > Lmax raises GQA_DEV_BAD_LEN or
 *     GQA_DEV_CAPACITY and none of its rows is written.
 *   max_pos0_host: host-known upper bound of pos0 (max_pos0_host + T <= Lmax,
 *     else GQA_ERR_CAPACITY).  pos0, n_tok 4-byte aligned, the rest 16.
 * pos0 all zero and n_tok NULL give gqa_prefill's result bit for bit.
 */
gqa_status gqa_prefill_chunk(const void *q, const void *k_cache, const void *v_cache,
                             void *out, const int32_t *pos0, const int32_t *n_tok,
                             int max_pos0_host, int B, int T, int Hq, int Hkv, int D,
                             int Lmax, float scale, int32_t *status_dev, void *stream);

/*
 * gqa_prefill_lse -- gqa_prefill that also stores each row's log-sum-exp for
 * the backward: lse[b, h, t] = ln sum_{s <= t} exp(q[b,t,h] . K[b,h/g,s] * scale),
 * lse float32 [B, Hq, round_up(T, 4)] (16-byte aligned; the padding is not
 * written).  Otherwise identical to gqa_prefill.
 */
gqa_status gqa_prefill_lse(const void *q, const void *k_cache, const void *v_cache, void *out,
                           float *lse, int B, int T, int Hq, int Hkv, int D, int Lmax,
                           float scale, int32_t *status_dev, void *stream);

/*
 * gqa_attention_backward -- gradients of causal GQA attention for training (the
 * pages' models train through causal scaled_dot_product_attention: page
 * "训练3.8B LLM…", section "提高吞吐量"; page "Build a Large Language Model from
 * Scratch", section 3.1).  With P = softmax(q K^T * scale) (causal) per query
 * head and the incoming gradient dout of out = P V:
 *     dv = P^T dout,  dP = dout V^T,  dS = P * (dP - rowsum(dout * out)),
 *     dq = scale dS K,  dk = scale dS^T q,
 * dk and dv of a KV head summed over the query heads of its group.
 *   q, out, dout, dq: bf16 [B, T, Hq, D];  k, v, dk, dv: bf16 [B, Hkv, Lmax, D]
 *     (the cache layout; slots 0 .. T-1 are read / written, the rest of dk, dv
 *     is not touched);  lse: the forward's, from gqa_prefill_lse.
 *   ws, ws_bytes: device scratch of gqa_backward_workspace_bytes(B, T, Hq) bytes
 *     (16-byte aligned; contents on entry do not matter).
 * Three launches (rowsum(dout * out); dk and dv per key tile; dq per query
 * tile), each a programmatic dependent of the one before; the dq launch starts
 * on the SMs the dk/dv launch frees and ends after it.  Errors:
 * GQA_ERR_INVALID_ARG also for B > 65535 or T * Hq >= 2^31.  Device errors:
 * GQA_DEV_TIMEOUT.
 */
gqa_status gqa_attention_backward(const void *q, const void *k, const void *v, const void *out,
                                  const void *dout, const float *lse, void *dq, void *dk,
                                  void *dv, int B, int T, int Hq, int Hkv, int D, int Lmax,
                                  float scale, void *ws, size_t ws_bytes, int32_t *status_dev,
                                  void *stream);

/* Bytes of workspace gqa_attention_backward needs (0 on invalid sizes): two
 * float32 arrays [B, Hq, round_up(T, 4)], rowsum(dout * out) and the forward's
 * log-sum-exp scaled to base 2. */
size_t gqa_backward_workspace_bytes(int B, int T, int Hq);

/*
 * gqa_doc_start -- for packed documents: doc_start[b, t] = the first position
 * t' <= t of token t's document, from per-token document ids doc_id [B, T]
 * that do not decrease along a sequence (each document contiguous).  A decrease
 * raises GQA_DEV_BAD_LEN.  Both arrays device int32, 4-byte aligned.
 */
gqa_status gqa_doc_start(const int32_t *doc_id, int32_t *doc_start, int B, int T,
                         int32_t *status_dev, void *stream);

/*
 * gqa_prefill_docs -- causal attention of a prompt of packed documents: query t
 * sees only the keys of its own document,
 *     out[b, t, h, :] = sum_{doc_start[b,t] <= s <= t} softmax_s(q . K[b, h/g, s] * scale)
 *                                                      * V[b, h/g, s]
 * the document-boundary mask of page "训练3.8B LLM…" (section "无效的方法", flex
 * attention with per-token document ids).  doc_start from gqa_doc_start (non-
 * decreasing along each sequence, doc_start[b, t] <= t; a value outside 0 .. t
 * raises GQA_DEV_BAD_LEN and the row attends to itself only).  Key tiles that
 * lie wholly before a query tile's first document are skipped.  Otherwise as
 * gqa_prefill (positions from 0, caches filled by gqa_rope_append).
 */
gqa_status gqa_prefill_docs(const void *q, const void *k_cache, const void *v_cache,
                            void *out, const int32_t *doc_start, int B, int T, int Hq, int Hkv,
                            int D, int Lmax, float scale, int32_t *status_dev, void *stream);

/*
 * gqa_decode -- one query token per sequence against the cache:
 *     out[b, h, :] = sum_{s < lens[b]} softmax_s(q[b,h,:] . K[b, h/g, s, :] * scale)
 *                                      * V[b, h/g, s, :]
 * lens[b] counts the cached tokens INCLUDING the token just appended (the query
 * sits at position lens[b] - 1 and attends to itself).  Split-K over the cache
 * length in 64-slot chunks; each KV head's bytes are read once per group of g
 * query heads; a second kernel merges the chunks.
 *   lens: device int32 [B], 1 <= lens[b] <= Lmax (others: GQA_DEV_BAD_LEN /
 *     GQA_DEV_CAPACITY and that sequence's output is zero).
 *   max_len_host: host-known upper bound of lens (<= Lmax); it sizes the grid
 *     and the workspace.  Lengths above it raise GQA_DEV_CAPACITY.
 *   ws, ws_bytes: device scratch of at least
 *     gqa_decode_workspace_bytes(B, Hq, D, max_len_host) bytes, 16-byte aligned;
 *     contents on entry do not matter.  Calls that may run at the same time on
 *     the GPU must not share one workspace.
 * Both launches are programmatic dependents of the kernel before them on the
 * stream (each waits for its predecessor to complete before reading its data).
 */
gqa_status gqa_decode(const void *q, const void *k_cache, const void *v_cache,
                      const int32_t *lens, int max_len_host, void *out, int B, int Hq,
                      int Hkv, int D, int Lmax, float scale, void *ws, size_t ws_bytes,
                      int32_t *status_dev, void *stream);

/* Bytes of workspace gqa_decode needs for these sizes (0 on invalid sizes). */
size_t gqa_decode_workspace_bytes(int B, int Hq, int D, int max_len);

/* Size of the fixed device array gqa_decode_noalloc keeps its scratch in. */
#define GQA_DECODE_NOALLOC_SCRATCH_BYTES (32u << 20)

/*
 * gqa_decode_noalloc -- gqa_decode for callers that cannot provide device
 * scratch memory (no allocator is available to them, or they must not allocate
 * once running).  The paper has no counterpart of this call; it is a property
 * of this library.  Same arguments and results as gqa_decode minus the
 * workspace: the scratch is a GQA_DECODE_NOALLOC_SCRATCH_BYTES (32 MiB) array
 * inside the library, present on every GPU that loads the library until the
 * process exits; nothing is allocated per call.
 *   - Sizes whose gqa_decode_workspace_bytes(B, Hq, D, max_len_host) exceeds
 *     32 MiB return GQA_ERR_WORKSPACE (the 64 x 24-head x 2049-slot batched
 *     decode needs 26.4 MB).
 *   - The array's device address belongs to the CUDA context the library's
 *     module is loaded into.  The first call from a context (the device's
 *     primary context, or a context the caller created and made current) looks
 *     that address up and keeps it for that context; make that first call
 *     before any stream capture.  A context destroyed and then replaced by a
 *     new one with the same handle would find the old address: load the
 *     library again after destroying a context it has run in.
 *   - Every call on a device uses the same array: calls that may overlap on the
 *     GPU (different streams without ordering) race and corrupt each other.
 *     Calls ordered on one stream are fine; no part of the array has to start
 *     at zero.
 */
gqa_status gqa_decode_noalloc(const void *q, const void *k_cache, const void *v_cache,
                              const int32_t *lens, int max_len_host, void *out, int B, int Hq,
                              int Hkv, int D, int Lmax, float scale, int32_t *status_dev,
                              void *stream);

/*
 * gqa_selftest_bounded_wait -- checks the bounded waits without a fault, through
 * the same wait function every kernel uses (with its limit shortened to
 * limit_ms, 1 .. 10000): one thread first waits on an mbarrier whose phase has
 * completed, which must return at once (GQA_DEV_BAD_LEN is raised if it does
 * not), then waits on an mbarrier that nothing arrives on, gives up after
 * limit_ms and ORs GQA_DEV_TIMEOUT into *status_dev (required).  The context
 * stays usable.  The paper has no counterpart of this call; it is a property of
 * this library.
 */
gqa_status gqa_selftest_bounded_wait(int32_t *status_dev, int limit_ms, void *stream);

/* Static, human-readable text for a status code. */
const char *gqa_status_string(gqa_status s);

/* Library version as MAJOR * 10000 + MINOR * 100 + PATCH. */
int gqa_version(void);

#ifdef __cplusplus
}
#endif

#endif /* GQA_H_ */
