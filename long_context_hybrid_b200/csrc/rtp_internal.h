// Internal launch entry points behind the C ABI (validated arguments only).
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace rtp {

// Launches `kernel` with programmatic stream serialisation: it may begin
// while the previous kernel on the stream is still running, and must call
// pdl_wait() before reading anything that kernel writes.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                       Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<Args&&>(args)...);
}

struct HeadList;

cudaError_t launch_project(const void* x, int64_t sb, int64_t sn, int64_t sh, int B, int N,
                           const void* P, const int32_t* heads, const int32_t* proj, int n_heads,
                           void* out, int out_f32, cudaStream_t stream);

// Projects keys k[b, t, g, :] (t < n_new, every g < Hkv, with P[g]) into
// rows pos .. pos + n_new - 1 of the key index [B, Hkv, cap, 16] (bf16).
cudaError_t launch_index_append(const void* k, int64_t sb, int64_t sn, int64_t sh, int B, int n_new, int Hkv,
                                const void* P, void* kindex, int64_t cap, int pos, cudaStream_t stream);

// The 8-bit key index: int8 codes [B, Hkv, cap, 16] and one fp32 scale per
// group of QGROUP_TOKENS tokens, [B, Hkv, ceil(cap / QGROUP_TOKENS)].
#define QGROUP_TOKENS 64
cudaError_t launch_index_quantize(const void* kindex, int64_t cap, int B, int Hkv, int g0, int g1, void* kindex8,
                                  float* kscale, cudaStream_t stream);

// Where the decode scan reads the key index: bf16 rows [B, Hkv, cap, 16] and,
// when k8 is set, int8 codes for the tokens of the full groups (the first
// QGROUP_TOKENS * floor(L / QGROUP_TOKENS) of each row) with their scales.
struct IndexRef {
  const void* bf16;
  const void* k8;
  const float* scale;
  int64_t cap;
};

// K-cache clustering: k-means over a key index and the two-level selection.
size_t kcluster_build_ws_bytes(int B, int Hkv, int L, int S);
cudaError_t launch_kcluster_build(const void* kindex, int64_t cap, int B, int Hkv, int L, int S, int iters,
                                  float* mu, int32_t* assign, int32_t* offsets, int32_t* members, void* ws,
                                  cudaStream_t stream);
size_t kcluster_select_ws_bytes(int B, int Hr, int C, int n_probe, int L);
cudaError_t launch_kcluster_select(const float* qt, const void* kindex, int64_t cap, const float* mu,
                                   const int32_t* offsets, const int32_t* members, int B, int L0, int L, int Hr,
                                   int Hkv, int C, const int32_t* kv_of, int n_probe, int topk, int32_t* idx,
                                   void* ws, cudaStream_t stream);
constexpr int kClusterSelectMaxTokens = 262144;

// Largest token top-k of a decode selection (any k >= L selects every token).
constexpr int kMaxDecodeTopk = 1 << 22;
size_t select_decode_ws_bytes(int B, int L, int Hr, int topk);
// The step's queries, projected by the selection's first kernel (q~ = q . P
// of the head's KV group, fp32 in the order of the standalone projection).
constexpr int kDecodeQueryHeads = 128;
struct DecodeQuery {
  const void* q;              // bf16 [B, Hq, D] (row strides q_sb, q_sh, elements)
  int64_t q_sb, q_sh;
  const void* P;              // bf16 [Hkv, D, R]
  int qhead[kDecodeQueryHeads];   // query head of each retrieval head
};
// Decode selection: q~ from `qt` ([B, Hr, R] fp32) or, when `dq` is given,
// formed into `qt_out` by the first kernel.
cudaError_t launch_select_decode(const float* qt, const DecodeQuery* dq, float* qt_out, IndexRef index, int B,
                                 int L, int Hr, int Hkv, const int32_t* kv_of, int topk, int32_t* idx, void* ws,
                                 cudaStream_t stream, int* filter_ctas = nullptr);

size_t select_prefill_ws_bytes(int B, int N, int Hr, int topk);
cudaError_t launch_select_prefill(const void* qt, const void* kt, int64_t kt_cap, int B, int N, int Hr, int Hkv,
                                  const int32_t* kv_of, int topk, int32_t* blocks,
                                  int32_t* counts, void* ws, cudaStream_t stream);

// Decode attention (one query per sequence) for a list of heads; retrieval
// heads (is_ret) add their selected tokens and the sink to the window.
size_t decode_attn_ws_bytes(int B, int L, int n_heads, int topk, int window);
cudaError_t launch_decode_attn(const void* q, int64_t q_sb, int64_t q_sh,
                               const void* kc, int64_t k_sb, int64_t k_sn, int64_t k_sh,
                               const void* vc, int64_t v_sb, int64_t v_sn, int64_t v_sh,
                               void* o, int64_t o_sb, int64_t o_sh,
                               int B, int L, int q_pos, int Hq, int Hkv,
                               const int32_t* heads, int n_heads, int is_ret,
                               const int32_t* idx, int topk, int window, int sink, float scale,
                               void* ws, cudaStream_t stream);

// Retrieval heads (selected tokens + sink + window) and streaming heads
// (window) of one decode step in one launch; each window K/V row is staged
// once per KV group.
constexpr int kMaxSink = 64;
cudaError_t launch_decode_hybrid(const void* q, int64_t q_sb, int64_t q_sh,
                                 const void* kc, int64_t k_sb, int64_t k_sn, int64_t k_sh,
                                 const void* vc, int64_t v_sb, int64_t v_sn, int64_t v_sh,
                                 void* o, int64_t o_sb, int64_t o_sh,
                                 int B, int L, int q_pos, int Hq, int Hkv,
                                 const int32_t* ret_heads, int n_ret, const int32_t* idx, int topk,
                                 int ret_window, int sink,
                                 const int32_t* swa_heads, int n_swa, int swa_window,
                                 float scale, void* ws, cudaStream_t stream, bool early_start = false,
                                 int max_ctas = 0);

// Same as launch_decode_attn for retrieval heads, with the partials in a
// library-owned static device array of kNoAllocScratchBytes.
constexpr size_t kNoAllocScratchBytes = (size_t)4 << 20;
cudaError_t launch_decode_attn_noalloc(const void* q, int64_t q_sb, int64_t q_sh,
                                       const void* kc, int64_t k_sb, int64_t k_sn, int64_t k_sh,
                                       const void* vc, int64_t v_sb, int64_t v_sn, int64_t v_sh,
                                       void* o, int64_t o_sb, int64_t o_sh,
                                       int B, int L, int q_pos, int Hq, int Hkv,
                                       const int32_t* heads, int n_heads, const int32_t* idx, int topk,
                                       int window, int sink, float scale, cudaStream_t stream);

// A [B, N, H, D] tensor: base pointer and element strides (D contiguous).
struct Tensor4 {
  const void* p;
  int64_t sb, sn, sh;
};

bool make_tmap_bnhd(CUtensorMap* map, const void* ptr, int B, int N, int H, int64_t sb, int64_t sn,
                    int64_t sh, int box_rows);

bool make_tmap_index(CUtensorMap* map, const void* ptr, int B, int H, int N, int64_t cap, int box_rows);
size_t select_prefill_tc_smem(int nb);
cudaError_t launch_select_prefill_tc(const void* qt, const void* kt, int64_t kt_cap, int B, int N, int Hr, int Hkv,
                                     const int32_t* kv_of, int topk, int32_t* blocks, int32_t* counts,
                                     int* status, cudaStream_t stream);

// Bytes of the status word every prefill attention call keeps in its workspace.
constexpr size_t kStatusBytes = 256;

}  // namespace rtp
