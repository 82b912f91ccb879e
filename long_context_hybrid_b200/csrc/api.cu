// C ABI of the head-wise hybrid attention library: argument validation on
// the host, then dispatch to the kernels. See include/rtp.h for the contract.
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/rtp.h"
#include "../../include/rtp_testing.h"
#include "attn_prefill_common.cuh"
#include "rtp_common.cuh"
#include "rtp_internal.h"

using namespace rtp;

namespace {

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned256(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 255u) == 0; }
bool stride_ok(rtp_strides s) { return s.b % 8 == 0 && s.n % 8 == 0 && s.h % 8 == 0 && s.b >= 0 && s.n >= 0 && s.h >= 0; }

rtp_status from_cuda(cudaError_t e) { return e == cudaSuccess ? RTP_OK : RTP_ERR_CUDA; }

// The device must be a Blackwell datacenter part (compute capability 10.x).
rtp_status check_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return RTP_ERR_CUDA;
  int major = 0;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess)
    return RTP_ERR_CUDA;
  return major == 10 ? RTP_OK : RTP_ERR_UNSUPPORTED;
}

rtp_status check_heads(const int32_t* heads, int n, int H) {
  if (!heads || n < 1 || n > kMaxHeads) return RTP_ERR_INVALID_ARG;
  for (int i = 0; i < n; ++i)
    if (heads[i] < 0 || heads[i] >= H) return RTP_ERR_INVALID_ARG;
  for (int i = 0; i < n; ++i)
    for (int k = i + 1; k < n; ++k)
      if (heads[i] == heads[k]) return RTP_ERR_INVALID_ARG;
  return RTP_OK;
}

// Tensor maps for q/k/v and the tcgen05 launch; the status word (first 4 bytes
// of ws) is cleared on the stream first and set by a CTA whose wait ran out.
rtp_status launch_tc(PrefillAttnParams& p, int B, void* ws, cudaStream_t stream, bool clear_status = true) {
  CUtensorMap tq, tk, tv;
  if (!make_tmap_bnhd(&tq, p.q.p, B, p.Nq, p.Hq, p.q.sb, p.q.sn, p.q.sh, 128) ||
      !make_tmap_bnhd(&tk, p.k.p, B, p.Nk, p.Hkv, p.k.sb, p.k.sn, p.k.sh, 64) ||
      !make_tmap_bnhd(&tv, p.v.p, B, p.Nk, p.Hkv, p.v.sb, p.v.sn, p.v.sh, 64))
    return RTP_ERR_CUDA;
  if (prefill_attn_tc_smem_bytes(p) > 227 * 1024) return RTP_ERR_UNSUPPORTED;
  int* status = static_cast<int*>(ws);
  if (clear_status && cudaMemsetAsync(status, 0, sizeof(int), stream) != cudaSuccess) return RTP_ERR_CUDA;
  const int n_tiles = (p.Nq + 127) / 128;
  return from_cuda(launch_prefill_attn_tc(p, tq, tk, tv, n_tiles, B, status, stream));
}

}  // namespace

extern "C" {

rtp_status rtp_get_device_status(const void* ws, rtp_stream_t stream, rtp_status* out) {
  if (!ws || !out) return RTP_ERR_INVALID_ARG;
  int v = 0;
  if (cudaStreamSynchronize((cudaStream_t)stream) != cudaSuccess) return RTP_ERR_CUDA;
  if (cudaMemcpy(&v, ws, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return RTP_ERR_CUDA;
  *out = v == 0 ? RTP_OK : (rtp_status)v;
  return RTP_OK;
}

const char* rtp_status_string(rtp_status s) {
  switch (s) {
    case RTP_OK: return "RTP_OK";
    case RTP_ERR_INVALID_ARG: return "RTP_ERR_INVALID_ARG";
    case RTP_ERR_UNSUPPORTED: return "RTP_ERR_UNSUPPORTED";
    case RTP_ERR_CUDA: return "RTP_ERR_CUDA";
    case RTP_ERR_TIMEOUT: return "RTP_ERR_TIMEOUT";
    case RTP_ERR_WORKSPACE: return "RTP_ERR_WORKSPACE";
  }
  return "RTP_ERR_UNKNOWN";
}

int rtp_version(void) { return RTP_VERSION; }

rtp_status rtp_index_project(const void* x, rtp_strides xs, int B, int N, int Hx,
                             const void* P, int Hp, int r,
                             const int32_t* heads, const int32_t* proj_of, int n_heads,
                             void* out, rtp_dtype out_dtype, rtp_stream_t stream) {
  if (!x || !P || !out || !proj_of) return RTP_ERR_INVALID_ARG;
  if (B < 1 || N < 1 || Hx < 1 || Hp < 1) return RTP_ERR_INVALID_ARG;
  if (r != RTP_R) return RTP_ERR_UNSUPPORTED;
  if (out_dtype != RTP_BF16 && out_dtype != RTP_F32) return RTP_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(out) || !aligned16(P) || !stride_ok(xs)) return RTP_ERR_INVALID_ARG;
  rtp_status st = check_heads(heads, n_heads, Hx);
  if (st != RTP_OK) return st;
  for (int i = 0; i < n_heads; ++i)
    if (proj_of[i] < 0 || proj_of[i] >= Hp) return RTP_ERR_INVALID_ARG;
  if ((st = check_device()) != RTP_OK) return st;
  return from_cuda(launch_project(x, xs.b, xs.n, xs.h, B, N, P, heads, proj_of, n_heads, out,
                                  out_dtype == RTP_F32, (cudaStream_t)stream));
}

rtp_status rtp_index_append(const void* k, rtp_strides ks, int B, int n_new, int Hkv, const void* P, int r,
                            void* kindex, int64_t cap, int pos, rtp_stream_t stream) {
  if (!k || !P || !kindex) return RTP_ERR_INVALID_ARG;
  if (B < 1 || n_new < 1 || Hkv < 1 || Hkv > kMaxHeads || pos < 0 || cap < 1) return RTP_ERR_INVALID_ARG;
  if ((int64_t)pos + n_new > cap) return RTP_ERR_INVALID_ARG;
  if (r != RTP_R) return RTP_ERR_UNSUPPORTED;
  if (!aligned16(k) || !aligned16(P) || !aligned16(kindex) || !stride_ok(ks)) return RTP_ERR_INVALID_ARG;
  rtp_status st = check_device();
  if (st != RTP_OK) return st;
  return from_cuda(launch_index_append(k, ks.b, ks.n, ks.h, B, n_new, Hkv, P, kindex, cap, pos, (cudaStream_t)stream));
}

size_t rtp_workspace_size_select_prefill(int B, int N, int Hr, int topk) {
  return select_prefill_ws_bytes(B, N, Hr, topk);
}

rtp_status rtp_select_prefill(const void* qt, const void* kt, int64_t kt_cap, int B, int N, int Hr, int Hkv,
                              int r, const int32_t* kv_of, int topk,
                              int32_t* blocks, int32_t* counts,
                              void* ws, size_t ws_bytes, rtp_stream_t stream) {
  if (!qt || !kt || !blocks || !counts || !kv_of) return RTP_ERR_INVALID_ARG;
  if (B < 1 || N < RTP_BLOCK || Hr < 1 || Hr > kMaxHeads || Hkv < 1 || topk < 1) return RTP_ERR_INVALID_ARG;
  if (kt_cap < N) return RTP_ERR_INVALID_ARG;
  if (N % RTP_BLOCK != 0 || r != RTP_R) return RTP_ERR_UNSUPPORTED;
  if (select_prefill_tc_smem(N / RTP_BLOCK) > 227 * 1024) return RTP_ERR_UNSUPPORTED;
  if (!aligned16(qt) || !aligned16(kt) || !aligned16(blocks) || !aligned16(counts)) return RTP_ERR_INVALID_ARG;
  for (int j = 0; j < Hr; ++j)
    if (kv_of[j] < 0 || kv_of[j] >= Hkv) return RTP_ERR_INVALID_ARG;
  const size_t need = select_prefill_ws_bytes(B, N, Hr, topk);
  if (!ws || ws_bytes < need || !aligned256(ws)) return RTP_ERR_WORKSPACE;
  rtp_status st = check_device();
  if (st != RTP_OK) return st;
  return from_cuda(launch_select_prefill(qt, kt, kt_cap, B, N, Hr, Hkv, kv_of, topk, blocks, counts, ws,
                                         (cudaStream_t)stream));
}

size_t rtp_workspace_size_select_decode(int B, int L, int Hr, int topk) {
  return select_decode_ws_bytes(B, L, Hr, topk);
}

rtp_status rtp_select_decode(const float* qt, const void* kindex, int64_t kindex_cap, int B, int L, int Hr, int Hkv,
                             int r, const int32_t* kv_of, int topk, int32_t* idx,
                             void* ws, size_t ws_bytes, rtp_stream_t stream) {
  if (!qt || !kindex || !idx || !kv_of) return RTP_ERR_INVALID_ARG;
  if (B < 1 || L < 1 || Hr < 1 || Hr > kMaxHeads || Hkv < 1 || topk < 1) return RTP_ERR_INVALID_ARG;
  if (kindex_cap < L) return RTP_ERR_INVALID_ARG;
  if (r != RTP_R || topk > kMaxDecodeTopk) return RTP_ERR_UNSUPPORTED;
  if (!aligned16(qt) || !aligned16(kindex) || !aligned16(idx)) return RTP_ERR_INVALID_ARG;
  for (int j = 0; j < Hr; ++j)
    if (kv_of[j] < 0 || kv_of[j] >= Hkv) return RTP_ERR_INVALID_ARG;
  if (Hkv > 16) return RTP_ERR_UNSUPPORTED;
  for (int g = 0; g < Hkv; ++g) {
    int c = 0;
    for (int j = 0; j < Hr; ++j) c += kv_of[j] == g;
    if (c > 16) return RTP_ERR_UNSUPPORTED;
  }
  const size_t need = select_decode_ws_bytes(B, L, Hr, topk);
  if (!ws || ws_bytes < need || !aligned256(ws)) return RTP_ERR_WORKSPACE;
  rtp_status st = check_device();
  if (st != RTP_OK) return st;
  return from_cuda(launch_select_decode(qt, nullptr, nullptr, IndexRef{kindex, nullptr, nullptr, kindex_cap}, B, L,
                                        Hr, Hkv, kv_of, topk, idx, ws, (cudaStream_t)stream));
}

rtp_status rtp_index_quantize(const void* kindex, int64_t cap, int B, int Hkv, int g0, int g1, void* kindex8,
                              float* kscale, rtp_stream_t stream) {
  if (!kindex || !kindex8 || !kscale) return RTP_ERR_INVALID_ARG;
  if (B < 1 || Hkv < 1 || cap < 1 || g0 < 0 || g1 < g0 || (int64_t)g1 * QGROUP_TOKENS > cap) return RTP_ERR_INVALID_ARG;
  if (!aligned16(kindex) || !aligned16(kindex8) || (reinterpret_cast<uintptr_t>(kscale) & 3u)) return RTP_ERR_INVALID_ARG;
  rtp_status st = check_device();
  if (st != RTP_OK) return st;
  return from_cuda(launch_index_quantize(kindex, cap, B, Hkv, g0, g1, kindex8, kscale, (cudaStream_t)stream));
}

rtp_status rtp_select_decode_q8(const float* qt, const void* kindex8, const float* kscale, const void* kindex,
                                int64_t kindex_cap, int B, int L, int Hr, int Hkv, int r, const int32_t* kv_of,
                                int topk, int32_t* idx, void* ws, size_t ws_bytes, rtp_stream_t stream) {
  if (!kindex8 || !kscale) return RTP_ERR_INVALID_ARG;
  if (!aligned16(kindex8) || (reinterpret_cast<uintptr_t>(kscale) & 3u)) return RTP_ERR_INVALID_ARG;
  if (!qt || !kindex || !idx || !kv_of) return RTP_ERR_INVALID_ARG;
  if (B < 1 || L < 1 || Hr < 1 || Hr > kMaxHeads || Hkv < 1 || topk < 1) return RTP_ERR_INVALID_ARG;
  if (kindex_cap < L) return RTP_ERR_INVALID_ARG;
  if (r != RTP_R || topk > kMaxDecodeTopk) return RTP_ERR_UNSUPPORTED;
  if (!aligned16(qt) || !aligned16(kindex) || !aligned16(idx)) return RTP_ERR_INVALID_ARG;
  for (int j = 0; j < Hr; ++j)
    if (kv_of[j] < 0 || kv_of[j] >= Hkv) return RTP_ERR_INVALID_ARG;
  if (Hkv > 16) return RTP_ERR_UNSUPPORTED;
  for (int g = 0; g < Hkv; ++g) {
    int c = 0;
    for (int j = 0; j < Hr; ++j) c += kv_of[j] == g;
    if (c > 16) return RTP_ERR_UNSUPPORTED;
  }
  const size_t need = select_decode_ws_bytes(B, L, Hr, topk);
  if (!ws || ws_bytes < need || !aligned256(ws)) return RTP_ERR_WORKSPACE;
  rtp_status st = check_device();
  if (st != RTP_OK) return st;
  return from_cuda(launch_select_decode(qt, nullptr, nullptr, IndexRef{kindex, kindex8, kscale, kindex_cap}, B, L,
                                        Hr, Hkv, kv_of, topk, idx, ws, (cudaStream_t)stream));
}

size_t rtp_workspace_size_kcluster_build(int B, int Hkv, int L, int cluster_size) {
  if (B < 1 || Hkv < 1 || L < 1 || cluster_size < 1) return 0;
  return kcluster_build_ws_bytes(B, Hkv, L, cluster_size);
}

rtp_status rtp_kcluster_build(const void* kindex, int64_t cap, int B, int Hkv, int L, int cluster_size, int iters,
                              float* centroids, int32_t* assign, int32_t* offsets, int32_t* members, void* ws,
                              size_t ws_bytes, rtp_stream_t stream) {
  if (!kindex || !centroids || !assign || !offsets || !members) return RTP_ERR_INVALID_ARG;
  if (B < 1 || Hkv < 1 || L < 1 || cap < L || cluster_size < 1 || iters < 0 || iters > 64) return RTP_ERR_INVALID_ARG;
  if ((int64_t)B * Hkv > 65535) return RTP_ERR_UNSUPPORTED;
  if (!aligned16(kindex) || (reinterpret_cast<uintptr_t>(centroids) & 3u) || (reinterpret_cast<uintptr_t>(assign) & 3u) ||
      (reinterpret_cast<uintptr_t>(offsets) & 3u) || (reinterpret_cast<uintptr_t>(members) & 3u))
    return RTP_ERR_INVALID_ARG;
  const size_t need = kcluster_build_ws_bytes(B, Hkv, L, cluster_size);
  if (!ws || ws_bytes < need || !aligned256(ws)) return RTP_ERR_WORKSPACE;
  rtp_status st = check_device();
  if (st != RTP_OK) return st;
  return from_cuda(launch_kcluster_build(kindex, cap, B, Hkv, L, cluster_size, iters, centroids, assign, offsets,
                                         members, ws, (cudaStream_t)stream));
}

size_t rtp_workspace_size_select_decode_clustered(int B, int Hr, int C, int n_probe, int L) {
  if (B < 1 || Hr < 1 || C < 1 || n_probe < 1 || L < 1) return 0;
  return kcluster_select_ws_bytes(B, Hr, C, n_probe, L);
}

rtp_status rtp_select_decode_clustered(const float* qt, const void* kindex, int64_t kindex_cap, const float* centroids,
                                       const int32_t* offsets, const int32_t* members, int B, int L0, int L, int Hr,
                                       int Hkv, int C, const int32_t* kv_of, int n_probe, int topk, int32_t* idx,
                                       void* ws, size_t ws_bytes, rtp_stream_t stream) {
  if (!qt || !kindex || !centroids || !offsets || !members || !kv_of || !idx) return RTP_ERR_INVALID_ARG;
  if (B < 1 || Hr < 1 || Hr > kMaxHeads || Hkv < 1 || C < 1 || n_probe < 1 || topk < 1) return RTP_ERR_INVALID_ARG;
  if (L0 < 1 || L < L0 || kindex_cap < L) return RTP_ERR_INVALID_ARG;
  if (L > kClusterSelectMaxTokens || topk > kMaxDecodeTopk) return RTP_ERR_UNSUPPORTED;
  if (!aligned16(qt) || !aligned16(kindex) || (reinterpret_cast<uintptr_t>(idx) & 3u)) return RTP_ERR_INVALID_ARG;
  for (int j = 0; j < Hr; ++j)
    if (kv_of[j] < 0 || kv_of[j] >= Hkv) return RTP_ERR_INVALID_ARG;
  const size_t need = kcluster_select_ws_bytes(B, Hr, C, n_probe, L);
  if (!ws || ws_bytes < need || !aligned256(ws)) return RTP_ERR_WORKSPACE;
  rtp_status st = check_device();
  if (st != RTP_OK) return st;
  return from_cuda(launch_kcluster_select(qt, kindex, kindex_cap, centroids, offsets, members, B, L0, L, Hr, Hkv, C,
                                          kv_of, n_probe, topk, idx, ws, (cudaStream_t)stream));
}

size_t rtp_workspace_size_sparse_attn_prefill(int B, int N, int Hr, int topk) {
  (void)B; (void)N; (void)Hr; (void)topk;
  return kStatusBytes;
}

rtp_status rtp_sparse_attn_prefill(const void* q, rtp_strides qs, const void* k, rtp_strides ks,
                                   const void* v, rtp_strides vs, void* o, rtp_strides os,
                                   int B, int N, int Hq, int Hkv, const int32_t* heads, int Hr,
                                   const int32_t* blocks, const int32_t* counts, int topk,
                                   int window_blocks, int sink_blocks, float scale,
                                   void* ws, size_t ws_bytes, rtp_stream_t stream) {
  if (!q || !k || !v || !o || !blocks || !counts) return RTP_ERR_INVALID_ARG;
  if (B < 1 || N < RTP_BLOCK || Hq < 1 || Hkv < 1 || Hq % Hkv != 0 || topk < 1) return RTP_ERR_INVALID_ARG;
  if (window_blocks < 1 || sink_blocks < 0 || !(scale > 0.f)) return RTP_ERR_INVALID_ARG;
  if (N % RTP_BLOCK != 0) return RTP_ERR_UNSUPPORTED;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o)) return RTP_ERR_INVALID_ARG;
  if (!stride_ok(qs) || !stride_ok(ks) || !stride_ok(vs) || !stride_ok(os)) return RTP_ERR_INVALID_ARG;
  rtp_status st = check_heads(heads, Hr, Hq);
  if (st != RTP_OK) return st;
  if (!ws || ws_bytes < kStatusBytes || !aligned256(ws)) return RTP_ERR_WORKSPACE;
  if ((st = check_device()) != RTP_OK) return st;
  PrefillAttnParams p{};
  p.q = {q, qs.b, qs.n, qs.h}; p.k = {k, ks.b, ks.n, ks.h}; p.v = {v, vs.b, vs.n, vs.h};
  p.o = o; p.o_sb = os.b; p.o_sn = os.n; p.o_sh = os.h;
  p.Nq = N; p.Nk = N; p.q_pos0 = 0; p.Hq = Hq; p.Hkv = Hkv; p.G = Hq / Hkv;
  p.sparse = 1; p.blocks = blocks; p.counts = counts; p.topk = topk;
  p.window_tokens = window_blocks * RTP_BLOCK; p.window_blocks = window_blocks;
  p.sink_blocks = sink_blocks;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.n_heads = Hr;
  const int nb = N / RTP_BLOCK;
  p.bitmap_words = (nb + 31) / 32;
  // a CTA serves two query blocks: its list is the union of two attended sets
  const long cap = 2L * ((long)topk + sink_blocks + window_blocks);
  p.list_cap = (int)(cap < nb ? cap : nb);
  for (int j = 0; j < Hr; ++j) p.head[j] = heads[j];
  if (nb > 32 * 4096) return RTP_ERR_UNSUPPORTED;
  return launch_tc(p, B, ws, (cudaStream_t)stream);
}

size_t rtp_workspace_size_triangle_prefill(void) { return kStatusBytes; }

rtp_status rtp_triangle_prefill(const void* q, rtp_strides qs, const void* k, rtp_strides ks,
                                const void* v, rtp_strides vs, void* o, rtp_strides os,
                                int B, int N, int Hq, int Hkv, const int32_t* heads, int n_heads,
                                int sink_blocks, int window_blocks, int last_tokens, float scale,
                                void* ws, size_t ws_bytes, rtp_stream_t stream) {
  if (!q || !k || !v || !o) return RTP_ERR_INVALID_ARG;
  if (B < 1 || N < RTP_BLOCK || Hq < 1 || Hkv < 1 || Hq % Hkv != 0) return RTP_ERR_INVALID_ARG;
  if (window_blocks < 1 || sink_blocks < 0 || last_tokens < 0 || last_tokens > N || !(scale > 0.f))
    return RTP_ERR_INVALID_ARG;
  if (N % RTP_BLOCK != 0 || last_tokens % RTP_BLOCK != 0) return RTP_ERR_UNSUPPORTED;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o)) return RTP_ERR_INVALID_ARG;
  if (!stride_ok(qs) || !stride_ok(ks) || !stride_ok(vs) || !stride_ok(os)) return RTP_ERR_INVALID_ARG;
  rtp_status st = check_heads(heads, n_heads, Hq);
  if (st != RTP_OK) return st;
  if (!ws || ws_bytes < kStatusBytes || !aligned256(ws)) return RTP_ERR_WORKSPACE;
  if ((st = check_device()) != RTP_OK) return st;
  cudaStream_t s = (cudaStream_t)stream;
  if (cudaMemsetAsync(ws, 0, sizeof(int), s) != cudaSuccess) return RTP_ERR_CUDA;
  const int n_stream = N - last_tokens;     // query rows of the streaming region
  const float sl2 = scale * 1.4426950408889634f;
  if (n_stream > 0) {
    // Streaming region: rows 0 .. n_stream-1 attend the sink and window blocks
    // (no selected blocks). Causal, so only the first n_stream keys are read.
    PrefillAttnParams p{};
    p.q = {q, qs.b, qs.n, qs.h}; p.k = {k, ks.b, ks.n, ks.h}; p.v = {v, vs.b, vs.n, vs.h};
    p.o = o; p.o_sb = os.b; p.o_sn = os.n; p.o_sh = os.h;
    p.Nq = n_stream; p.Nk = n_stream; p.q_pos0 = 0; p.Hq = Hq; p.Hkv = Hkv; p.G = Hq / Hkv;
    p.sparse = 1; p.blocks = nullptr; p.counts = nullptr; p.topk = 1;
    p.window_tokens = window_blocks * RTP_BLOCK; p.window_blocks = window_blocks; p.sink_blocks = sink_blocks;
    p.scale_log2 = sl2;
    p.n_heads = n_heads;
    const int nb = n_stream / RTP_BLOCK;
    if (nb > 32 * 4096) return RTP_ERR_UNSUPPORTED;
    p.bitmap_words = (nb + 31) / 32;
    const long cap = 2L * ((long)sink_blocks + window_blocks);
    p.list_cap = (int)(cap < nb ? cap : nb);
    for (int j = 0; j < n_heads; ++j) p.head[j] = heads[j];
    if ((st = launch_tc(p, B, ws, s, false)) != RTP_OK) return st;
  }
  if (last_tokens > 0) {
    // Last Q-K region: rows n_stream .. N-1 attend every earlier key (a
    // window as long as the sequence), by the banded kernel on those rows.
    PrefillAttnParams p{};
    const char* qb = static_cast<const char*>(q) + (int64_t)n_stream * qs.n * 2;
    char* ob = static_cast<char*>(o) + (int64_t)n_stream * os.n * 2;
    p.q = {qb, qs.b, qs.n, qs.h}; p.k = {k, ks.b, ks.n, ks.h}; p.v = {v, vs.b, vs.n, vs.h};
    p.o = ob; p.o_sb = os.b; p.o_sn = os.n; p.o_sh = os.h;
    p.Nq = last_tokens; p.Nk = N; p.q_pos0 = n_stream; p.Hq = Hq; p.Hkv = Hkv; p.G = Hq / Hkv;
    p.sparse = 0; p.window_tokens = N;
    p.scale_log2 = sl2;
    p.n_heads = n_heads;
    p.list_cap = 0;
    for (int j = 0; j < n_heads; ++j) p.head[j] = heads[j];
    if ((st = launch_tc(p, B, ws, s, false)) != RTP_OK) return st;
  }
  return RTP_OK;
}

size_t rtp_workspace_size_sparse_attn_decode(int B, int L, int Hq, int Hr, int topk, int window) {
  (void)Hq;
  return decode_attn_ws_bytes(B, L, Hr, topk, window);
}

rtp_status rtp_sparse_attn_decode(const void* q, const void* kc, rtp_strides ks,
                                  const void* vc, rtp_strides vs, void* o,
                                  int B, int L, int Hq, int Hkv, const int32_t* heads, int Hr,
                                  const int32_t* idx, int topk, int window, int sink, float scale,
                                  void* ws, size_t ws_bytes, rtp_stream_t stream) {
  if (!q || !kc || !vc || !o || !idx) return RTP_ERR_INVALID_ARG;
  if (B < 1 || L < 1 || Hq < 1 || Hkv < 1 || Hq % Hkv != 0 || topk < 1) return RTP_ERR_INVALID_ARG;
  if (window < 1 || sink < 0 || sink > kMaxSink || !(scale > 0.f)) return RTP_ERR_INVALID_ARG;
  if (Hq / Hkv > 16 || Hkv > 16) return RTP_ERR_UNSUPPORTED;
  if (!aligned16(q) || !aligned16(kc) || !aligned16(vc) || !aligned16(o) || !aligned16(idx)) return RTP_ERR_INVALID_ARG;
  if (!stride_ok(ks) || !stride_ok(vs)) return RTP_ERR_INVALID_ARG;
  rtp_status st = check_heads(heads, Hr, Hq);
  if (st != RTP_OK) return st;
  const size_t need = decode_attn_ws_bytes(B, L, Hr, topk, window);
  if (!ws || ws_bytes < need || !aligned256(ws)) return RTP_ERR_WORKSPACE;
  if ((st = check_device()) != RTP_OK) return st;
  return from_cuda(launch_decode_attn(q, (int64_t)Hq * RTP_D, RTP_D, kc, ks.b, ks.n, ks.h,
                                      vc, vs.b, vs.n, vs.h, o, (int64_t)Hq * RTP_D, RTP_D,
                                      B, L, L - 1, Hq, Hkv, heads, Hr, 1, idx, topk, window, sink,
                                      scale, ws, (cudaStream_t)stream));
}

rtp_status rtp_sparse_attn_decode_noalloc(const void* q, const void* kc, rtp_strides ks,
                                          const void* vc, rtp_strides vs, void* o,
                                          int B, int L, int Hq, int Hkv, const int32_t* heads, int Hr,
                                          const int32_t* idx, int topk, int window, int sink, float scale,
                                          rtp_stream_t stream) {
  if (!q || !kc || !vc || !o || !idx) return RTP_ERR_INVALID_ARG;
  if (B < 1 || L < 1 || Hq < 1 || Hkv < 1 || Hq % Hkv != 0 || topk < 1) return RTP_ERR_INVALID_ARG;
  if (window < 1 || sink < 0 || sink > kMaxSink || !(scale > 0.f)) return RTP_ERR_INVALID_ARG;
  if (Hq / Hkv > 16 || Hkv > 16) return RTP_ERR_UNSUPPORTED;
  if (!aligned16(q) || !aligned16(kc) || !aligned16(vc) || !aligned16(o) || !aligned16(idx)) return RTP_ERR_INVALID_ARG;
  if (!stride_ok(ks) || !stride_ok(vs)) return RTP_ERR_INVALID_ARG;
  rtp_status st = check_heads(heads, Hr, Hq);
  if (st != RTP_OK) return st;
  // The partials must fit the library's fixed scratch array.
  if (decode_attn_ws_bytes(B, L, Hr, topk, window) > kNoAllocScratchBytes) return RTP_ERR_WORKSPACE;
  if ((st = check_device()) != RTP_OK) return st;
  return from_cuda(launch_decode_attn_noalloc(q, (int64_t)Hq * RTP_D, RTP_D, kc, ks.b, ks.n, ks.h,
                                              vc, vs.b, vs.n, vs.h, o, (int64_t)Hq * RTP_D, RTP_D,
                                              B, L, L - 1, Hq, Hkv, heads, Hr, idx, topk, window, sink,
                                              scale, (cudaStream_t)stream));
}

size_t rtp_workspace_size_decode_attn_hybrid(int B, int L, int Hq, int topk, int window) {
  return decode_attn_ws_bytes(B, L, Hq, topk, window);
}

// Decode step workspace: [attention][q~ fp32 (256-aligned)][selection], the
// attention part first so that its status word is at the start.
namespace {
size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }
size_t step_qt_bytes(int B, int Hr) { return align256((size_t)B * Hr * RTP_R * sizeof(float)); }
}  // namespace

size_t rtp_workspace_size_decode_step(int B, int L, int Hq, int Hr, int topk, int window) {
  if (B < 1 || L < 1 || Hq < 1 || Hr < 0 || window < 1) return 0;
  size_t n = align256(decode_attn_ws_bytes(B, L, Hq, Hr > 0 ? topk : 0, window));
  if (Hr > 0) n += step_qt_bytes(B, Hr) + align256(select_decode_ws_bytes(B, L, Hr, topk));
  return n;
}

rtp_status rtp_decode_step(const void* q, const void* P, const void* kindex, int64_t kindex_cap,
                           const void* kindex8, const float* kscale, const void* kc, rtp_strides ks,
                           const void* vc, rtp_strides vs, void* o, int B, int L, int Hq, int Hkv,
                           const int32_t* ret_heads, int Hr, int topk, int ret_window, int sink,
                           const int32_t* swa_heads, int n_swa, int swa_window, float scale, int32_t* idx,
                           void* ws, size_t ws_bytes, rtp_stream_t stream) {
  if (!q || !kc || !vc || !o) return RTP_ERR_INVALID_ARG;
  if (B < 1 || L < 1 || Hq < 1 || Hkv < 1 || Hq % Hkv != 0) return RTP_ERR_INVALID_ARG;
  if (Hr < 0 || n_swa < 0 || Hr + n_swa < 1 || Hr + n_swa > kMaxHeads) return RTP_ERR_INVALID_ARG;
  if (Hq / Hkv > 16 || Hkv > 16) return RTP_ERR_UNSUPPORTED;
  if (Hr > 0) {
    if (!P || !kindex || !idx || !ret_heads || topk < 1 || ret_window < 1) return RTP_ERR_INVALID_ARG;
    if (kindex_cap < L) return RTP_ERR_INVALID_ARG;
    if (!kindex8 != !kscale) return RTP_ERR_INVALID_ARG;
    if (kindex8 && (!aligned16(kindex8) || (reinterpret_cast<uintptr_t>(kscale) & 3u))) return RTP_ERR_INVALID_ARG;
    if (topk > kMaxDecodeTopk) return RTP_ERR_UNSUPPORTED;
    if (!aligned16(P) || !aligned16(kindex) || !aligned16(idx)) return RTP_ERR_INVALID_ARG;
  }
  if (n_swa > 0 && swa_window < 1) return RTP_ERR_INVALID_ARG;
  if (sink < 0 || sink > kMaxSink || !(scale > 0.f)) return RTP_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(kc) || !aligned16(vc) || !aligned16(o)) return RTP_ERR_INVALID_ARG;
  if (!stride_ok(ks) || !stride_ok(vs)) return RTP_ERR_INVALID_ARG;
  int32_t all[kMaxHeads];
  for (int i = 0; i < Hr; ++i) all[i] = ret_heads[i];
  for (int i = 0; i < n_swa; ++i) all[Hr + i] = swa_heads ? swa_heads[i] : -1;
  rtp_status st = check_heads(all, Hr + n_swa, Hq);
  if (st != RTP_OK) return st;
  const int G = Hq / Hkv;
  int32_t kv_of[kMaxHeads];
  for (int i = 0; i < Hr; ++i) kv_of[i] = ret_heads[i] / G;
  for (int g = 0; g < Hkv; ++g) {
    int c = 0;
    for (int i = 0; i < Hr; ++i) c += kv_of[i] == g;
    if (c > 16) return RTP_ERR_UNSUPPORTED;
  }
  const int wmax = (Hr > 0 && ret_window > swa_window) || n_swa == 0 ? ret_window : swa_window;
  const size_t need = rtp_workspace_size_decode_step(B, L, Hq, Hr, topk, wmax);
  if (!ws || ws_bytes < need || !aligned256(ws)) return RTP_ERR_WORKSPACE;
  if ((st = check_device()) != RTP_OK) return st;
  cudaStream_t s = (cudaStream_t)stream;
  char* base = static_cast<char*>(ws);
  char* ws_att = base;
  int filter_ctas = 0;
  if (Hr > 0) {
    float* qt = reinterpret_cast<float*>(base + align256(decode_attn_ws_bytes(B, L, Hq, topk, wmax)));
    void* ws_sel = reinterpret_cast<char*>(qt) + step_qt_bytes(B, Hr);
    // q~ = q . P for the retrieval heads (fp32, unrounded, formed by the
    // selection's first kernel), then the top-k
    DecodeQuery dq;
    dq.q = q;
    dq.q_sb = (int64_t)Hq * RTP_D;
    dq.q_sh = RTP_D;
    dq.P = P;
    for (int i = 0; i < Hr; ++i) dq.qhead[i] = ret_heads[i];
    cudaError_t e = launch_select_decode(nullptr, &dq, qt, IndexRef{kindex, kindex8, kscale, kindex_cap}, B, L, Hr,
                                         Hkv, kv_of, topk, idx, ws_sel, s, &filter_ctas);
    if (e != cudaSuccess) return from_cuda(e);
  }
  // The attention CTAs start on the SMs the scan leaves while the filter
  // still runs: where a filter CTA sits, one attention CTA fits beside it.
  // Launching only as many as fit at once keeps any from starting its whole
  // run of window chunks after the filter ends.
  int max_ctas = 0;
  if (filter_ctas > 0) {
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) !=
                                                  cudaSuccess)
      return RTP_ERR_CUDA;
    if (filter_ctas < sms) max_ctas = 2 * sms - filter_ctas;
  }
  // The kernel before the attention is the selection's filter (or nothing of
  // this call): it writes only idx, so the attention may read q, K and V early.
  return from_cuda(launch_decode_hybrid(q, (int64_t)Hq * RTP_D, RTP_D, kc, ks.b, ks.n, ks.h, vc, vs.b, vs.n, vs.h,
                                        o, (int64_t)Hq * RTP_D, RTP_D, B, L, L - 1, Hq, Hkv, ret_heads, Hr, idx, topk,
                                        ret_window, sink, swa_heads, n_swa, swa_window, scale, ws_att, s,
                                        /*early_start=*/Hr > 0, max_ctas));
}

size_t rtp_workspace_size_decode_step_clustered(int B, int L, int Hq, int Hr, int C, int n_probe, int topk,
                                                int window) {
  if (B < 1 || L < 1 || Hq < 1 || Hr < 1 || C < 1 || n_probe < 1 || topk < 1 || window < 1) return 0;
  return align256(decode_attn_ws_bytes(B, L, Hq, topk, window)) + step_qt_bytes(B, Hr) +
         align256(kcluster_select_ws_bytes(B, Hr, C, n_probe, L));
}

rtp_status rtp_decode_step_clustered(const void* q, const void* P, const void* kindex, int64_t kindex_cap,
                                     const float* centroids, const int32_t* offsets, const int32_t* members, int L0,
                                     int C, int n_probe, const void* kc, rtp_strides ks, const void* vc,
                                     rtp_strides vs, void* o, int B, int L, int Hq, int Hkv,
                                     const int32_t* ret_heads, int Hr, int topk, int ret_window, int sink,
                                     const int32_t* swa_heads, int n_swa, int swa_window, float scale, int32_t* idx,
                                     void* ws, size_t ws_bytes, rtp_stream_t stream) {
  if (!q || !P || !kindex || !centroids || !offsets || !members || !kc || !vc || !o || !idx || !ret_heads)
    return RTP_ERR_INVALID_ARG;
  if (B < 1 || L < 1 || Hq < 1 || Hkv < 1 || Hq % Hkv != 0) return RTP_ERR_INVALID_ARG;
  if (Hr < 1 || n_swa < 0 || Hr + n_swa > kMaxHeads) return RTP_ERR_INVALID_ARG;
  if (Hq / Hkv > 16 || Hkv > 16) return RTP_ERR_UNSUPPORTED;
  if (C < 1 || n_probe < 1 || topk < 1 || ret_window < 1) return RTP_ERR_INVALID_ARG;
  if (L0 < 1 || L < L0 || kindex_cap < L) return RTP_ERR_INVALID_ARG;
  if (L > kClusterSelectMaxTokens || topk > kMaxDecodeTopk) return RTP_ERR_UNSUPPORTED;
  if (n_swa > 0 && swa_window < 1) return RTP_ERR_INVALID_ARG;
  if (sink < 0 || sink > kMaxSink || !(scale > 0.f)) return RTP_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(kc) || !aligned16(vc) || !aligned16(o) || !aligned16(P) || !aligned16(kindex) ||
      !aligned16(idx))
    return RTP_ERR_INVALID_ARG;
  if (!stride_ok(ks) || !stride_ok(vs)) return RTP_ERR_INVALID_ARG;
  int32_t all[kMaxHeads];
  for (int i = 0; i < Hr; ++i) all[i] = ret_heads[i];
  for (int i = 0; i < n_swa; ++i) all[Hr + i] = swa_heads ? swa_heads[i] : -1;
  rtp_status st = check_heads(all, Hr + n_swa, Hq);
  if (st != RTP_OK) return st;
  const int G = Hq / Hkv;
  int32_t kv_of[kMaxHeads];
  for (int i = 0; i < Hr; ++i) kv_of[i] = ret_heads[i] / G;
  const int wmax = ret_window > swa_window || n_swa == 0 ? ret_window : swa_window;
  const size_t need = rtp_workspace_size_decode_step_clustered(B, L, Hq, Hr, C, n_probe, topk, wmax);
  if (!ws || ws_bytes < need || !aligned256(ws)) return RTP_ERR_WORKSPACE;
  if ((st = check_device()) != RTP_OK) return st;
  cudaStream_t s = (cudaStream_t)stream;
  char* base = static_cast<char*>(ws);
  float* qt = reinterpret_cast<float*>(base + align256(decode_attn_ws_bytes(B, L, Hq, topk, wmax)));
  void* ws_sel = reinterpret_cast<char*>(qt) + step_qt_bytes(B, Hr);
  // q~ = q . P for the retrieval heads (fp32, unrounded), then the two-level top-k
  cudaError_t e = launch_project(q, (int64_t)Hq * RTP_D, (int64_t)Hq * RTP_D, RTP_D, B, 1, P, ret_heads, kv_of, Hr,
                                 qt, 1, s);
  if (e != cudaSuccess) return from_cuda(e);
  e = launch_kcluster_select(qt, kindex, kindex_cap, centroids, offsets, members, B, L0, L, Hr, Hkv, C, kv_of,
                             n_probe, topk, idx, ws_sel, s);
  if (e != cudaSuccess) return from_cuda(e);
  // The selection holds one SM per (sequence, retrieval head) and no
  // attention CTA fits beside it: launch as many as fit on the others (two
  // per SM), all streaming their window while the selection runs.
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) !=
                                                cudaSuccess)
    return RTP_ERR_CUDA;
  const int n_sel = B * Hr;
  const int max_ctas = n_sel < sms ? 2 * (sms - n_sel) : 0;
  return from_cuda(launch_decode_hybrid(q, (int64_t)Hq * RTP_D, RTP_D, kc, ks.b, ks.n, ks.h, vc, vs.b, vs.n, vs.h,
                                        o, (int64_t)Hq * RTP_D, RTP_D, B, L, L - 1, Hq, Hkv, ret_heads, Hr, idx, topk,
                                        ret_window, sink, swa_heads, n_swa, swa_window, scale, base, s,
                                        /*early_start=*/true, max_ctas));
}

rtp_status rtp_decode_attn_hybrid(const void* q, const void* kc, rtp_strides ks, const void* vc, rtp_strides vs,
                                  void* o, int B, int L, int Hq, int Hkv,
                                  const int32_t* ret_heads, int Hr, const int32_t* idx, int topk, int ret_window,
                                  int sink, const int32_t* swa_heads, int n_swa, int swa_window, float scale,
                                  void* ws, size_t ws_bytes, rtp_stream_t stream) {
  if (!q || !kc || !vc || !o) return RTP_ERR_INVALID_ARG;
  if (B < 1 || L < 1 || Hq < 1 || Hkv < 1 || Hq % Hkv != 0) return RTP_ERR_INVALID_ARG;
  if (Hr < 0 || n_swa < 0 || Hr + n_swa < 1 || Hr + n_swa > kMaxHeads) return RTP_ERR_INVALID_ARG;
  if (Hq / Hkv > 16 || Hkv > 16) return RTP_ERR_UNSUPPORTED;
  if (Hr > 0 && (!idx || topk < 1 || ret_window < 1 || !aligned16(idx))) return RTP_ERR_INVALID_ARG;
  if (n_swa > 0 && swa_window < 1) return RTP_ERR_INVALID_ARG;
  if (sink < 0 || sink > kMaxSink || !(scale > 0.f)) return RTP_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(kc) || !aligned16(vc) || !aligned16(o)) return RTP_ERR_INVALID_ARG;
  if (!stride_ok(ks) || !stride_ok(vs)) return RTP_ERR_INVALID_ARG;
  int32_t all[kMaxHeads];
  for (int i = 0; i < Hr; ++i) all[i] = ret_heads ? ret_heads[i] : -1;
  for (int i = 0; i < n_swa; ++i) all[Hr + i] = swa_heads ? swa_heads[i] : -1;
  rtp_status st = check_heads(all, Hr + n_swa, Hq);
  if (st != RTP_OK) return st;
  const int wmax = (Hr > 0 && ret_window > swa_window) || n_swa == 0 ? ret_window : swa_window;
  const size_t need = decode_attn_ws_bytes(B, L, Hr + n_swa, Hr > 0 ? topk : 0, wmax);
  if (!ws || ws_bytes < need || !aligned256(ws)) return RTP_ERR_WORKSPACE;
  if ((st = check_device()) != RTP_OK) return st;
  return from_cuda(launch_decode_hybrid(q, (int64_t)Hq * RTP_D, RTP_D, kc, ks.b, ks.n, ks.h, vc, vs.b, vs.n, vs.h,
                                        o, (int64_t)Hq * RTP_D, RTP_D, B, L, L - 1, Hq, Hkv, ret_heads, Hr, idx, topk,
                                        ret_window, sink, swa_heads, n_swa, swa_window, scale, ws,
                                        (cudaStream_t)stream));
}

rtp_status rtp_debug_prefill_timeout_probe(const void* q, const void* k, const void* v, void* o, void* ws,
                                           size_t ws_bytes, rtp_stream_t stream) {
  if (!q || !k || !v || !o) return RTP_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o)) return RTP_ERR_INVALID_ARG;
  if (!ws || ws_bytes < kStatusBytes || !aligned256(ws)) return RTP_ERR_WORKSPACE;
  rtp_status st = check_device();
  if (st != RTP_OK) return st;
  // One CTA: a 128-row sliding-window problem, one head, whose Q never arrives.
  PrefillAttnParams p{};
  p.q = {q, 128 * RTP_D, RTP_D, RTP_D}; p.k = {k, 128 * RTP_D, RTP_D, RTP_D}; p.v = {v, 128 * RTP_D, RTP_D, RTP_D};
  p.o = o; p.o_sb = 128 * RTP_D; p.o_sn = RTP_D; p.o_sh = RTP_D;
  p.Nq = 128; p.Nk = 128; p.q_pos0 = 0; p.Hq = 1; p.Hkv = 1; p.G = 1;
  p.sparse = 0; p.window_tokens = 128;
  p.scale_log2 = 0.1f;
  p.n_heads = 1; p.head[0] = 0; p.list_cap = 0;
  p.withhold_q = 1;
  return launch_tc(p, 1, ws, (cudaStream_t)stream);
}

size_t rtp_workspace_size_swa(int B, int Nq, int Nk, int n_heads, int window) {
  if (Nq != 1) return kStatusBytes;
  return decode_attn_ws_bytes(B, Nk, n_heads, 0, window);
}

rtp_status rtp_swa(const void* q, rtp_strides qs, const void* k, rtp_strides ks,
                   const void* v, rtp_strides vs, void* o, rtp_strides os,
                   int B, int Nq, int Nk, int q_pos0, int Hq, int Hkv,
                   const int32_t* heads, int n_heads, int window, float scale,
                   void* ws, size_t ws_bytes, rtp_stream_t stream) {
  if (!q || !k || !v || !o) return RTP_ERR_INVALID_ARG;
  if (B < 1 || Nq < 1 || Nk < 1 || Hq < 1 || Hkv < 1 || Hq % Hkv != 0) return RTP_ERR_INVALID_ARG;
  if (q_pos0 < 0 || (int64_t)q_pos0 + Nq > Nk) return RTP_ERR_INVALID_ARG;
  if (window < 1 || !(scale > 0.f)) return RTP_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o)) return RTP_ERR_INVALID_ARG;
  if (!stride_ok(qs) || !stride_ok(ks) || !stride_ok(vs) || !stride_ok(os)) return RTP_ERR_INVALID_ARG;
  rtp_status st = check_heads(heads, n_heads, Hq);
  if (st != RTP_OK) return st;
  if (Nq == 1) {
    if (Hq / Hkv > 16 || Hkv > 16) return RTP_ERR_UNSUPPORTED;
    const size_t need = decode_attn_ws_bytes(B, Nk, n_heads, 0, window);
    if (!ws || ws_bytes < need || !aligned256(ws)) return RTP_ERR_WORKSPACE;
    if ((st = check_device()) != RTP_OK) return st;
    return from_cuda(launch_decode_attn(q, qs.b, qs.h, k, ks.b, ks.n, ks.h, v, vs.b, vs.n, vs.h,
                                        o, os.b, os.h, B, Nk, q_pos0, Hq, Hkv, heads, n_heads, 0,
                                        nullptr, 0, window, 0, scale, ws, (cudaStream_t)stream));
  }
  if (Nq % RTP_BLOCK != 0) return RTP_ERR_UNSUPPORTED;
  if (!ws || ws_bytes < kStatusBytes || !aligned256(ws)) return RTP_ERR_WORKSPACE;
  if ((st = check_device()) != RTP_OK) return st;
  PrefillAttnParams p{};
  p.q = {q, qs.b, qs.n, qs.h}; p.k = {k, ks.b, ks.n, ks.h}; p.v = {v, vs.b, vs.n, vs.h};
  p.o = o; p.o_sb = os.b; p.o_sn = os.n; p.o_sh = os.h;
  p.Nq = Nq; p.Nk = Nk; p.q_pos0 = q_pos0; p.Hq = Hq; p.Hkv = Hkv; p.G = Hq / Hkv;
  p.sparse = 0; p.window_tokens = window;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.n_heads = n_heads;
  p.list_cap = 0;
  for (int j = 0; j < n_heads; ++j) p.head[j] = heads[j];
  return launch_tc(p, B, ws, (cudaStream_t)stream);
}

}  // extern "C"
