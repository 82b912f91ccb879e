/*
 * rtp.h - C ABI of the head-wise hybrid attention library (librtp.so).
 *
 * The method (RTPurbo / RTPurboV2): most attention heads of a long-context
 * model are "streaming" heads that only need a local window and run causal
 * sliding-window attention (SWA, window 8192 in the deployed recipe); about
 * 15% are "retrieval" heads. For those, a cheap 16-dimensional indexer built
 * from a per-KV-head low-rank projector P (D x 16) scores key blocks (prefill)
 * or tokens (decode); the top-k are selected, and exact softmax attention is
 * computed at the full head dimension over the sink, the local window and the
 * selected keys.
 *   Sources: RTPurboV2 article (th-motor.com), paragraphs on retrieval vs
 *   streaming heads, on the low-rank projector (D -> r = 16) and on the
 *   Qwen3-Coder-30B-A3B recipe (SWA window 8192); RTPurbo digest (Telegram
 *   channel "Data analysis", post 5185): the 16-d indexer is a scout that
 *   picks candidates, then honest attention runs at full dimension on them.
 *
 * Conventions shared by every call
 * --------------------------------
 *  - Every call returns an rtp_status; nothing else crosses the ABI (no C++
 *    exceptions). Arguments are validated on the host before any launch; a
 *    rejected call launches nothing and leaves every output untouched.
 *  - Device pointers: all tensor arguments are caller-owned device memory
 *    (global memory of the current CUDA device). The library keeps no
 *    pointer after a call returns and allocates no device memory itself:
 *    scratch space is the caller's `ws` buffer, whose minimum size the
 *    matching rtp_workspace_size_* call returns. `ws` must be 256-byte
 *    aligned. Arguments documented as "host" are read during the call only.
 *  - Asynchrony: work is enqueued on `stream` (a cudaStream_t; NULL is the
 *    legacy default stream); results are ready when the stream reaches that
 *    point. Launch failures return RTP_ERR_CUDA.
 *  - bf16 tensors are IEEE bfloat16 (uint16 storage); rounding to bf16 is
 *    round-to-nearest-even everywhere.
 *  - Layouts: activations are [B, N, H, D] with element strides given by an
 *    rtp_strides {b, n, h}; the last dimension (D) is contiguous. Every
 *    stride must be a multiple of 8 elements and every base pointer 16-byte
 *    aligned (tensor-memory-access tiles need 16-byte-aligned rows).
 *  - Head mapping: query head h reads KV head h / (Hq / Hkv) (contiguous
 *    grouped-query attention); Hq must be a multiple of Hkv.
 *  - Sizes: D = 128 and block = 64 in this build; N (prefill) must be a
 *    multiple of 64. Other values return RTP_ERR_UNSUPPORTED.
 *  - Thread safety: calls are reentrant; concurrent calls on different
 *    streams must use different workspaces.
 */
#ifndef RTP_H_
#define RTP_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define RTP_VERSION 1

#if defined(__GNUC__)
#define RTP_API __attribute__((visibility("default")))
#else
#define RTP_API
#endif

typedef enum {
  RTP_OK = 0,
  RTP_ERR_INVALID_ARG = 1,   /* null/misaligned pointer, bad size or index */
  RTP_ERR_UNSUPPORTED = 2,   /* shape outside what this build implements, or no sm_100 device */
  RTP_ERR_CUDA = 3,          /* a CUDA launch or runtime call failed */
  RTP_ERR_TIMEOUT = 4,       /* a bounded device-side wait gave up */
  RTP_ERR_WORKSPACE = 5      /* ws too small or misaligned */
} rtp_status;

typedef enum { RTP_BF16 = 0, RTP_F32 = 1 } rtp_dtype;

/* Element strides of a [B, N, H, D] tensor (D contiguous). */
typedef struct { int64_t b, n, h; } rtp_strides;

struct CUstream_st;
typedef struct CUstream_st* rtp_stream_t; /* same type as cudaStream_t */

/* Human-readable name of a status (static storage, never NULL). */
RTP_API const char* rtp_status_string(rtp_status s);
/* RTP_VERSION of the loaded library. */
RTP_API int rtp_version(void);

/*
 * rtp_get_device_status - the device-side status of the last call that used
 * the workspace `ws`.
 *   The tensor-core prefill calls (rtp_select_prefill, rtp_sparse_attn_prefill
 *   and rtp_swa with Nq > 1) keep a status word in the first bytes of their
 *   workspace: cleared on the stream before their launch and set to
 *   RTP_ERR_TIMEOUT by a thread block whose bounded wait ran out (that block
 *   then drains its copies, frees its tensor memory and returns instead of
 *   spinning). The decode calls keep the same word and always leave RTP_OK in
 *   it: their kernels never wait on one another on the device.
 *   This call synchronises `stream` (the word is read after every call queued
 *   on it before), then writes the recorded status to *out (RTP_OK when the
 *   word is zero). Returns RTP_ERR_INVALID_ARG for a NULL `ws` or `out`,
 *   RTP_ERR_CUDA if the synchronisation or the read fails, else RTP_OK.
 */
RTP_API rtp_status rtp_get_device_status(const void* ws, rtp_stream_t stream, rtp_status* out);

/*
 * rtp_index_project - the low-rank indexer projection x~ = x . P.
 *   Source: RTPurboV2 article, paragraph on the low-rank projector (feature
 *   dimension compressed from D to r = 16); the precomputed 16-d key index
 *   of the 128K decode workload.
 *
 *   x        bf16 [B, N, Hx, D] device, strides xs.
 *   P        bf16 [Hp, D, r] device, contiguous; one projector per KV head.
 *   heads    host int32 [n_heads]: which heads of x to project (0 <= . < Hx).
 *   proj_of  host int32 [n_heads]: which projector each listed head uses
 *            (0 <= . < Hp; for a query head h this is h / (Hq/Hkv)).
 *   out      device [B, n_heads, N, r], contiguous; out_dtype RTP_BF16 (the
 *            stored index: fp32 accumulation, one RNE rounding) or RTP_F32
 *            (the decode query index, unrounded fp32 accumulation).
 *   r must be 16. n_heads >= 1. N >= 1 (no multiple-of-64 rule here).
 */
RTP_API rtp_status rtp_index_project(const void* x, rtp_strides xs, int B, int N, int Hx,
                             const void* P, int Hp, int r,
                             const int32_t* heads, const int32_t* proj_of, int n_heads,
                             void* out, rtp_dtype out_dtype, rtp_stream_t stream);

/*
 * rtp_index_append - keeps the decode key index in step with the KV cache:
 * projects the keys of new tokens into their rows of the index.
 *   Source: RTPurboV2 article, paragraph on the low-rank projector (keys
 *   projected from D to r = 16) and the Qwen3-Coder-30B-A3B recipe (the
 *   sparse indexer runs in the decode stage); the 128K decode workload
 *   statement (a 16-d key index of shape [KV heads, context, 16] beside the
 *   cache). The pages give no maintenance scheme; the plain reading is that
 *   the index holds bf16(k . P_g) for every cached token, so every token that
 *   enters the cache enters the index the same way.
 *
 *   k        bf16 [B, n_new, Hkv, D] device (strides ks): the keys of the new
 *            tokens, every KV head (for the prefill -> decode handoff, the
 *            whole prefill K with n_new = N and pos = 0; for a decode step,
 *            the new token's row with n_new = 1 and pos = L - 1).
 *   P        bf16 [Hkv, D, r] device, contiguous: KV head g uses P[g].
 *   kindex   bf16 [B, Hkv, cap, r] device, contiguous, written at rows
 *            pos .. pos + n_new - 1 of every (sequence, KV head) with the
 *            bf16 rounding of the fp32 dot products (as rtp_index_project);
 *            other rows are untouched.
 *   r = 16, pos >= 0, pos + n_new <= cap, Hkv <= 128.
 */
RTP_API rtp_status rtp_index_append(const void* k, rtp_strides ks, int B, int n_new, int Hkv, const void* P, int r,
                                    void* kindex, int64_t cap, int pos, rtp_stream_t stream);

/*
 * rtp_select_prefill - per query block, the top-k key blocks by block score.
 *   Source: block score = max over the (query, key) pairs of a 64 x 64
 *   block pair of q~ . k~, each query block keeping its top-k causal key
 *   blocks (the tiny 2K prefill workload statement); the indexer as a scout
 *   (RTPurbo digest). Only causal pairs (key position <= query position) are
 *   scored; every causal key block j <= i is a candidate; exact ties rank
 *   the smaller block first. The token score matrix is never materialised.
 *
 *   qt       bf16 [B, Hr, N, r] device, contiguous (projected retrieval-head queries).
 *   kt       bf16 [B, Hkv, kt_cap, r] device, contiguous (projected keys; rows
 *            0 .. N-1 are read). kt_cap >= N: a key index kept with headroom
 *            for decode (see rtp_index_append) serves as is.
 *   kv_of    host int32 [Hr]: KV head of each retrieval head.
 *   topk     k >= 1 selected blocks per query block.
 *   blocks   int32 [B, Hr, N/64, topk] device out: ascending block indices,
 *            min(k, i+1) of them, the rest -1.
 *   counts   int32 [B, Hr, N/64] device out: min(k, i+1).
 *   ws       workspace of rtp_workspace_size_select_prefill() bytes (the
 *            status word, see rtp_get_device_status).
 *   N must be a multiple of 64, r = 16; the block scores of a query-block
 *   pair are kept on chip, which bounds N at about 1.4M tokens
 *   (RTP_ERR_UNSUPPORTED beyond).
 */
RTP_API size_t rtp_workspace_size_select_prefill(int B, int N, int Hr, int topk);
RTP_API rtp_status rtp_select_prefill(const void* qt, const void* kt, int64_t kt_cap, int B, int N, int Hr, int Hkv,
                              int r, const int32_t* kv_of, int topk,
                              int32_t* blocks, int32_t* counts,
                              void* ws, size_t ws_bytes, rtp_stream_t stream);

/*
 * rtp_select_decode - token-level top-k over the whole cache.
 *   Source: the 128K decode workload statement (retrieval heads take the
 *   token-level top-2048 by q~ . k~ over the whole cache); RTPurbo digest.
 *   Exact ties rank the smaller token first.
 *
 *   qt       fp32 [B, Hr, r] device (unrounded projected decode queries).
 *   kindex   bf16 [B, Hkv, kindex_cap, r] device, contiguous (the key index;
 *            rows 0 .. L-1 are the cache's tokens). kindex_cap >= L.
 *   kv_of    host int32 [Hr].
 *   idx      int32 [B, Hr, topk] device out: ascending token indices;
 *            min(k, L) of them, the rest -1.
 *   ws       workspace of rtp_workspace_size_select_decode() bytes.
 *   r = 16, 1 <= topk <= 4194304 (topk >= L selects every token: the dense
 *   preset of a full cross-attention decode), L >= 1; Hkv <= 16 and at most 16 retrieval
 *   heads per KV group (RTP_ERR_UNSUPPORTED otherwise).
 */
RTP_API size_t rtp_workspace_size_select_decode(int B, int L, int Hr, int topk);
RTP_API rtp_status rtp_select_decode(const float* qt, const void* kindex, int64_t kindex_cap, int B, int L, int Hr,
                                     int Hkv,
                             int r, const int32_t* kv_of, int topk, int32_t* idx,
                             void* ws, size_t ws_bytes, rtp_stream_t stream);

/*
 * rtp_index_quantize - the 8-bit form of the decode key index.
 *   Source: the Baidu developer article on layered long-context attention
 *   ("深度解析：超长上下文注意力架构的分层优化策略"), section on the
 *   mixed-precision index system: an 8-bit quantised indexer that cuts the
 *   index storage (here the bytes the decode scan reads) with a small loss of
 *   precision. The page fixes no scheme; this is the plain symmetric one.
 *   Per group of 64 consecutive tokens of one (sequence, KV head): amax =
 *   max |x| over its 64 x 16 bf16 values, s = amax / 127 and code =
 *   round-half-even(x / s) clamped to [-127, 127], both divisions IEEE fp32;
 *   an all-zero group gets s = 0 and zero codes.
 *
 *   kindex   bf16 [B, Hkv, cap, 16] device (the bf16 index, rtp_index_append).
 *   kindex8  int8 [B, Hkv, cap, 16] device out: codes of the tokens of groups
 *            g0 .. g1-1 (tokens 64 g0 .. 64 g1 - 1); other rows untouched.
 *   kscale   fp32 [B, Hkv, ceil(cap / 64)] device out: the groups' scales.
 *   0 <= g0 <= g1, 64 g1 <= cap. A decode loop quantises each group once it
 *   is full (after appending token 64 g + 63); the partial last group is
 *   scanned from the bf16 rows.
 */
RTP_API rtp_status rtp_index_quantize(const void* kindex, int64_t cap, int B, int Hkv, int g0, int g1, void* kindex8,
                                      float* kscale, rtp_stream_t stream);

/*
 * rtp_select_decode_q8 - rtp_select_decode over the 8-bit key index.
 *   Source: as rtp_index_quantize and rtp_select_decode. Tokens of the full
 *   64-token groups, 0 .. 64 floor(L/64) - 1, are scored s * sum_c q~_c code_c
 *   (fp32) from kindex8 / kscale, which must hold every full group
 *   (rtp_index_quantize); the rest from the bf16 rows of kindex. Selection,
 *   ties, outputs, limits and workspace as rtp_select_decode (same
 *   rtp_workspace_size_select_decode). The scan reads 16 bytes per token
 *   instead of 32.
 */
RTP_API rtp_status rtp_select_decode_q8(const float* qt, const void* kindex8, const float* kscale, const void* kindex,
                                        int64_t kindex_cap, int B, int L, int Hr, int Hkv, int r,
                                        const int32_t* kv_of, int topk, int32_t* idx, void* ws, size_t ws_bytes,
                                        rtp_stream_t stream);

/*
 * rtp_kcluster_build - clusters the key index of every (sequence, KV head)
 * for the two-level decode selection.
 *   Source: RTPurboV2 article (th-motor.com), the sequence-dimension
 *   compression paragraph (clustering lets decode skip most semantically
 *   unrelated tokens; the low-rank key vectors make the cluster centres
 *   accurate) and the Qwen3-Coder-30B-A3B recipe (the retrieval heads' K
 *   cache is clustered). The pages give no algorithm; this is Lloyd k-means.
 *   Over rows 0 .. L-1 of each (sequence, KV head): C = ceil(L / cluster_size)
 *   centroids start at rows 0, cluster_size, 2 cluster_size, ...; each of
 *   `iters` rounds assigns every row to its nearest centroid (squared
 *   Euclidean distance summed over c = 0..15 with every subtraction, square
 *   and addition rounded to fp32, no fused multiply-add; ties to the smaller
 *   centroid) and moves every centroid to its cluster's mean (exact int64
 *   sums of trunc(x * 2^20), mean = fp32(double(sum) / double(count) *
 *   2^-20); an empty cluster keeps its centroid); a last assignment pairs
 *   every row with its nearest final centroid.
 *
 *   kindex     bf16 [B, Hkv, cap, 16] device (rtp_index_append); cap >= L.
 *   centroids  fp32 [B, Hkv, C, 16] device out.
 *   assign     int32 [B, Hkv, L] device out: each row's cluster.
 *   offsets    int32 [B, Hkv, C + 1] device out, members int32 [B, Hkv, L]
 *              device out: cluster i's rows are members[offsets[i] ..
 *              offsets[i+1]) (in no particular order).
 *   ws         rtp_workspace_size_kcluster_build(B, Hkv, L, cluster_size) bytes.
 *   cluster_size >= 1, 0 <= iters <= 64, B * Hkv <= 65535.
 */
RTP_API size_t rtp_workspace_size_kcluster_build(int B, int Hkv, int L, int cluster_size);
RTP_API rtp_status rtp_kcluster_build(const void* kindex, int64_t cap, int B, int Hkv, int L, int cluster_size,
                                      int iters, float* centroids, int32_t* assign, int32_t* offsets,
                                      int32_t* members, void* ws, size_t ws_bytes, rtp_stream_t stream);

/*
 * rtp_select_decode_clustered - the two-level token selection over a
 * clustered key index.
 *   Source: as rtp_kcluster_build; the 128K decode workload statement for the
 *   token-level top-k, the sink and the window it is unioned with (by the
 *   attention calls, as for rtp_select_decode).
 *   Per (sequence b, retrieval head j): the n_probe clusters of KV head
 *   kv_of[j] whose centroids score highest against q~ (fp32 dot products;
 *   ties to the smaller cluster), then the top-k tokens by q~ . k~ among
 *   those clusters' members and every token appended after the build
 *   (positions L0 .. L-1), ties to the smaller token; all candidates when
 *   there are fewer than k.
 *
 *   qt         fp32 [B, Hr, 16] device; kindex bf16 [B, Hkv, kindex_cap, 16].
 *   centroids, offsets, members  from rtp_kcluster_build over L0 rows (C
 *              clusters).
 *   idx        int32 [B, Hr, topk] device out: ascending tokens, -1 padded.
 *   ws         rtp_workspace_size_select_decode_clustered(B, Hr, C, n_probe, L).
 *   1 <= L0 <= L <= 262144 (RTP_ERR_UNSUPPORTED beyond), n_probe >= 1.
 */
RTP_API size_t rtp_workspace_size_select_decode_clustered(int B, int Hr, int C, int n_probe, int L);
RTP_API rtp_status rtp_select_decode_clustered(const float* qt, const void* kindex, int64_t kindex_cap,
                                               const float* centroids, const int32_t* offsets,
                                               const int32_t* members, int B, int L0, int L, int Hr, int Hkv,
                                               int C, const int32_t* kv_of, int n_probe, int topk, int32_t* idx,
                                               void* ws, size_t ws_bytes, rtp_stream_t stream);

/*
 * rtp_sparse_attn_prefill - exact attention of retrieval heads over their
 * selected key blocks, the sink blocks and the local window blocks.
 *   Source: RTPurbo digest (honest attention at full dimension over the
 *   small selected set); the tiny 2K prefill workload statement (top-k
 *   blocks plus key block 0 plus the window blocks).
 *   For query block i the attended key blocks are the set
 *     blocks[i][0..count) U {0 .. sink_blocks-1} U {i-window_blocks+1 .. i},
 *   each key once, with the causal mask (key position <= query position).
 *
 *   q, o     bf16 [B, N, Hq, D] device (strides qs, os); o is written only for
 *            the listed heads.
 *   k, v     bf16 [B, N, Hkv, D] device (strides ks, vs).
 *   heads    host int32 [Hr]: the retrieval heads; row j of blocks/counts
 *            belongs to heads[j].
 *   blocks   int32 [B, Hr, N/64, topk], counts int32 [B, Hr, N/64] device, as
 *            written by rtp_select_prefill (ascending; entries outside
 *            [0, i] are ignored).
 *   window_blocks >= 1, sink_blocks >= 0, scale > 0 (the softmax scale,
 *   1/sqrt(D) in the method's usual form).
 *   ws       at least rtp_workspace_size_sparse_attn_prefill() bytes (the
 *            status word, see rtp_get_device_status).
 */
RTP_API size_t rtp_workspace_size_sparse_attn_prefill(int B, int N, int Hr, int topk);
RTP_API rtp_status rtp_sparse_attn_prefill(const void* q, rtp_strides qs, const void* k, rtp_strides ks,
                                   const void* v, rtp_strides vs, void* o, rtp_strides os,
                                   int B, int N, int Hq, int Hkv, const int32_t* heads, int Hr,
                                   const int32_t* blocks, const int32_t* counts, int topk,
                                   int window_blocks, int sink_blocks, float scale,
                                   void* ws, size_t ws_bytes, rtp_stream_t stream);

/*
 * rtp_triangle_prefill - prefill attention under the triangle-shaped mask of
 * TriangleMix, a static pattern on the same kernels.
 *   Source: the TriangleMix interview (36kr, "微软研究院杨玉庆：Agent 的注意力系统"),
 *   paragraph on the triangle-shaped mask: deep layers skip the middle Q-K
 *   region and keep only the streaming region (the first keys and the local
 *   band) and the last Q-K region (the last queries against every key). The
 *   page gives no sizes; this call takes them as arguments, with the sink and
 *   the band block-granular as for the retrieval heads of
 *   rtp_sparse_attn_prefill.
 *   Query row t (block i = t / 64) attends the keys u <= t
 *     - in blocks {0 .. sink_blocks-1} U {i-window_blocks+1 .. i}, for
 *       t < N - last_tokens (the streaming region);
 *     - all of them, for t >= N - last_tokens (the last Q-K region).
 *   With last_tokens = N this is dense causal attention.
 *
 *   q, o     bf16 [B, N, Hq, D] device (strides qs, os); o written only for
 *            the listed heads.
 *   k, v     bf16 [B, N, Hkv, D] device (strides ks, vs).
 *   heads    host int32 [n_heads].
 *   N and last_tokens multiples of 64 (RTP_ERR_UNSUPPORTED otherwise),
 *   0 <= last_tokens <= N, window_blocks >= 1, sink_blocks >= 0, scale > 0.
 *   ws       rtp_workspace_size_triangle_prefill() bytes: the status word
 *            (see rtp_get_device_status), shared by the call's two kernels.
 */
RTP_API size_t rtp_workspace_size_triangle_prefill(void);
RTP_API rtp_status rtp_triangle_prefill(const void* q, rtp_strides qs, const void* k, rtp_strides ks,
                                        const void* v, rtp_strides vs, void* o, rtp_strides os,
                                        int B, int N, int Hq, int Hkv, const int32_t* heads, int n_heads,
                                        int sink_blocks, int window_blocks, int last_tokens, float scale,
                                        void* ws, size_t ws_bytes, rtp_stream_t stream);

/*
 * rtp_sparse_attn_decode - one new query token per sequence attends, per
 * retrieval head, the selected tokens, tokens 0..sink-1 and the last
 * `window` tokens of the cache, each key once.
 *   Source: the 128K decode workload statement (top-2048 unioned with the
 *   last 8192 tokens and token 0, then exact softmax attention at D=128);
 *   RTPurbo digest.
 *
 *   q        bf16 [B, Hq, D] device, contiguous; o likewise (written only for
 *            the listed heads).
 *   kc, vc   bf16 [B, L, Hkv, D] device (strides ks, vs): the cache, whose
 *            last row (L-1) is the new token's own key/value.
 *   heads    host int32 [Hr]; idx int32 [B, Hr, topk] device: distinct
 *            token indices first, then -1 padding, as written by
 *            rtp_select_decode (entries in the window or below `sink` are
 *            skipped there, since those keys are attended anyway; with
 *            topk > L only the first L entries of a row are read).
 *   window >= 1, 0 <= sink <= 64, scale > 0; Hq / Hkv <= 16 and Hkv <= 16
 *   (the query heads of a KV group are packed into one 16-row tensor-core
 *   tile).
 */
RTP_API size_t rtp_workspace_size_sparse_attn_decode(int B, int L, int Hq, int Hr, int topk, int window);
RTP_API rtp_status rtp_sparse_attn_decode(const void* q, const void* kc, rtp_strides ks,
                                  const void* vc, rtp_strides vs, void* o,
                                  int B, int L, int Hq, int Hkv, const int32_t* heads, int Hr,
                                  const int32_t* idx, int topk, int window, int sink, float scale,
                                  void* ws, size_t ws_bytes, rtp_stream_t stream);

/*
 * rtp_decode_attn_hybrid - one decode step's attention for retrieval and
 * streaming heads together: rtp_sparse_attn_decode on `ret_heads` (window
 * ret_window) and rtp_swa's decode form on `swa_heads` (window swa_window),
 * in one launch that stages each window K/V row once per KV group, so the
 * heads of a group share it (grouped-query heads read the same keys).
 *   Sources: RTPurboV2 article (streaming heads SWA, retrieval heads sparse);
 *   the 128K decode workload statement.
 *   Arguments as in the two calls it combines; Hr or n_swa may be 0 (not
 *   both); sink <= 64; Hq / Hkv <= 16, Hkv <= 16. ws: rtp_workspace_size_decode_attn_hybrid(
 *   B, L, Hq, topk, max(ret_window, swa_window)) bytes.
 */
RTP_API size_t rtp_workspace_size_decode_attn_hybrid(int B, int L, int Hq, int topk, int window);
RTP_API rtp_status rtp_decode_attn_hybrid(const void* q, const void* kc, rtp_strides ks, const void* vc,
                                          rtp_strides vs, void* o, int B, int L, int Hq, int Hkv,
                                          const int32_t* ret_heads, int Hr, const int32_t* idx, int topk,
                                          int ret_window, int sink, const int32_t* swa_heads, int n_swa,
                                          int swa_window, float scale, void* ws, size_t ws_bytes,
                                          rtp_stream_t stream);

/*
 * rtp_decode_step - one decode step of a layer in one call: the retrieval
 * heads' query index q~ = q . P (fp32, as rtp_index_project), their token
 * top-k over the key index (as rtp_select_decode, written to idx), and the
 * attention of the retrieval and streaming heads (as rtp_decode_attn_hybrid).
 *   Sources: the 128K decode workload statement (selection over the whole
 *   cache unioned with the window and token 0); RTPurboV2 article (streaming
 *   heads SWA). The paper defines the steps, not this grouping: it exists so
 *   that the library knows the order of its own kernels and can start the
 *   attention's window reads while the selection finishes.
 *   q        bf16 [B, Hq, 128] device, contiguous (the new token's queries).
 *   P        bf16 [Hkv, 128, 16] device (projector per KV head).
 *   kindex   bf16 [B, Hkv, kindex_cap, 16] device, contiguous (key index of
 *            the cache; rows 0 .. L-1 are read, the new token's at L - 1 included,
 *            see rtp_index_append). kindex_cap >= L.
 *   kindex8, kscale  NULL, or the 8-bit index of the same cache
 *            (rtp_index_quantize): the selection then runs as
 *            rtp_select_decode_q8 (both NULL or both set).
 *   kc, vc   bf16 [B, L, Hkv, 128] device with element strides ks, vs.
 *   o        bf16 [B, Hq, 128] device out: rows of the listed heads.
 *   ret_heads/swa_heads  host int32 lists (Hr or n_swa may be 0, not both).
 *   idx      int32 [B, Hr, topk] device out (the selected tokens, ascending).
 *   ws       rtp_workspace_size_decode_step(B, L, Hq, Hr, topk,
 *            max(ret_window, swa_window)) bytes, 256-byte aligned; its first
 *            word is the status word read by rtp_get_device_status.
 *   Limits as in the three calls it combines. Asynchronous on `stream`.
 *   idx equals what rtp_select_decode writes; the attention runs on as many
 *   thread blocks as fit beside the selection's last kernel, so its split of
 *   the keys (and hence the fp32 rounding of o) can differ from a separate
 *   rtp_decode_attn_hybrid call's.
 */
RTP_API size_t rtp_workspace_size_decode_step(int B, int L, int Hq, int Hr, int topk, int window);
RTP_API rtp_status rtp_decode_step(const void* q, const void* P, const void* kindex, int64_t kindex_cap,
                                   const void* kindex8, const float* kscale, const void* kc, rtp_strides ks,
                                   const void* vc, rtp_strides vs, void* o, int B, int L, int Hq, int Hkv,
                                   const int32_t* ret_heads, int Hr, int topk, int ret_window, int sink,
                                   const int32_t* swa_heads, int n_swa, int swa_window, float scale, int32_t* idx,
                                   void* ws, size_t ws_bytes, rtp_stream_t stream);

/*
 * rtp_decode_step_clustered - one decode step as rtp_decode_step, with the
 * retrieval heads' tokens chosen by the two-level selection over a clustered
 * key index (as rtp_select_decode_clustered) instead of the scan of the whole
 * index.
 *   Sources: RTPurboV2 article (th-motor.com), the sequence-dimension
 *   compression paragraph and the Qwen3-Coder-30B-A3B recipe (clustered K
 *   cache for the retrieval heads); the 128K decode workload statement for
 *   the union with the window and token 0. As for rtp_decode_step, the
 *   grouping lets the attention stream its window while the selection runs
 *   (the clustered selection occupies one SM per (sequence, retrieval head)).
 *   Arguments as rtp_decode_step, plus:
 *   centroids, offsets, members  from rtp_kcluster_build over the first L0
 *            rows of kindex (C clusters); rows L0 .. L-1 (appended after the
 *            build) are always candidates.
 *   n_probe  clusters probed per (sequence, retrieval head), >= 1.
 *   ws       rtp_workspace_size_decode_step_clustered(B, L, Hq, Hr, C, n_probe,
 *            topk, max(ret_window, swa_window)) bytes, 256-byte aligned; its
 *            first word is the status word read by rtp_get_device_status.
 *   Hr >= 1; 1 <= L0 <= L <= 262144 (RTP_ERR_UNSUPPORTED beyond); other
 *   limits as in the calls it combines. Asynchronous on `stream`.
 */
RTP_API size_t rtp_workspace_size_decode_step_clustered(int B, int L, int Hq, int Hr, int C, int n_probe, int topk,
                                                        int window);
RTP_API rtp_status rtp_decode_step_clustered(const void* q, const void* P, const void* kindex, int64_t kindex_cap,
                                             const float* centroids, const int32_t* offsets,
                                             const int32_t* members, int L0, int C, int n_probe, const void* kc,
                                             rtp_strides ks, const void* vc, rtp_strides vs, void* o, int B, int L,
                                             int Hq, int Hkv, const int32_t* ret_heads, int Hr, int topk,
                                             int ret_window, int sink, const int32_t* swa_heads, int n_swa,
                                             int swa_window, float scale, int32_t* idx, void* ws, size_t ws_bytes,
                                             rtp_stream_t stream);

/*
 * rtp_sparse_attn_decode_noalloc - rtp_sparse_attn_decode without a workspace
 * argument and without allocating anything.
 *   The method's sources have no counterpart of this call: it exists for
 *   callers that cannot provide scratch memory, such as plugins whose host
 *   framework owns every device allocation and gives them no way to call
 *   cudaMalloc, or latency-bound decode loops that must not pay for a
 *   cudaMalloc/cudaFree (both may synchronise the device) on every step.
 *
 *   Arguments, layouts and results are those of rtp_sparse_attn_decode. The
 *   split-K partials go to a fixed array inside the library, 4 MiB per GPU,
 *   held by every GPU that loads the library until the process exits. A call
 *   whose partials would not fit (about 256 + 4 * B * Hr * (ceil(window/64) +
 *   ceil((topk+64)/64)) * 528 bytes > 4 MiB) returns RTP_ERR_WORKSPACE and
 *   launches nothing.
 *   The first call on a device looks up the array's device address (with that
 *   device current) and caches it together with the device's current context;
 *   a later call under a different context (for instance after
 *   cudaDeviceReset) looks it up again. Make the first call on each device
 *   before any stream capture. The call never calls cudaMalloc or cudaFree.
 *   Every call shares the one array, so calls whose work may overlap on the
 *   GPU (different streams, or concurrent host threads) race on it and must
 *   be serialised by the caller. Nothing in the array needs to start at zero:
 *   each call writes every partial it reads. The decode kernels have no
 *   device-side waits, so there is no status word to read for this call:
 *   errors come back in the return value.
 */
RTP_API rtp_status rtp_sparse_attn_decode_noalloc(const void* q, const void* kc, rtp_strides ks,
                                                  const void* vc, rtp_strides vs, void* o,
                                                  int B, int L, int Hq, int Hkv, const int32_t* heads, int Hr,
                                                  const int32_t* idx, int topk, int window, int sink, float scale,
                                                  rtp_stream_t stream);

/*
 * rtp_swa - causal sliding-window attention of streaming heads.
 *   Source: RTPurboV2 article (streaming heads use SWA, local window 8192).
 *   Query row t sits at position q_pos0 + t and attends the keys u with
 *   position - window < u <= position (u < Nk). Prefill: Nq = Nk = N,
 *   q_pos0 = 0. Decode: Nq = 1, Nk = L, q_pos0 = L - 1.
 *
 *   q, o     bf16 [B, Nq, Hq, D] device (strides qs, os); o written only for
 *            the listed heads.
 *   k, v     bf16 [B, Nk, Hkv, D] device (strides ks, vs).
 *   heads    host int32 [n_heads]: the streaming heads to compute.
 *   window >= 1, scale > 0. Prefill (Nq > 1) needs Nq % 64 == 0.
 *   ws       at least rtp_workspace_size_swa() bytes: the split-K partials
 *            for a single query (Nq == 1), the status word otherwise.
 */
RTP_API size_t rtp_workspace_size_swa(int B, int Nq, int Nk, int n_heads, int window);
RTP_API rtp_status rtp_swa(const void* q, rtp_strides qs, const void* k, rtp_strides ks,
                   const void* v, rtp_strides vs, void* o, rtp_strides os,
                   int B, int Nq, int Nk, int q_pos0, int Hq, int Hkv,
                   const int32_t* heads, int n_heads, int window, float scale,
                   void* ws, size_t ws_bytes, rtp_stream_t stream);

#ifdef __cplusplus
}
#endif
#endif /* RTP_H_ */
