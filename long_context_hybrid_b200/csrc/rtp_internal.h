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

size_t select_decode_ws_bytes(int B, int L, int Hr, int topk);
cudaError_t launch_select_decode(const float* qt, const void* kindex, int B, int L, int Hr,
                                 int Hkv, const int32_t* kv_of, int topk, int32_t* idx,
                                 void* ws, cudaStream_t stream);

size_t select_prefill_ws_bytes(int B, int N, int Hr, int topk);
cudaError_t launch_select_prefill(const void* qt, const void* kt, int B, int N, int Hr, int Hkv,
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
                                 float scale, void* ws, cudaStream_t stream, bool early_start = false);

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

// Prefill attention over per-query-block key-block lists (SWA band or
// selected/sink/window union).
struct Tensor4 {
  const void* p;
  int64_t sb, sn, sh;
};
cudaError_t launch_prefill_attn(Tensor4 q, Tensor4 k, Tensor4 v, void* o, int64_t o_sb,
                                int64_t o_sn, int64_t o_sh, int B, int Nq, int Nk, int q_pos0,
                                int Hq, int Hkv, const int32_t* heads, int n_heads,
                                int sparse, const int32_t* blocks, const int32_t* counts, int topk,
                                int window_tokens, int window_blocks, int sink_blocks, float scale,
                                cudaStream_t stream);

bool make_tmap_bnhd(CUtensorMap* map, const void* ptr, int B, int N, int H, int64_t sb, int64_t sn,
                    int64_t sh, int box_rows);

bool make_tmap_index(CUtensorMap* map, const void* ptr, int B, int H, int N, int box_rows);
size_t select_prefill_tc_smem(int nb);
cudaError_t launch_select_prefill_tc(const void* qt, const void* kt, int B, int N, int Hr, int Hkv,
                                     const int32_t* kv_of, int topk, int32_t* blocks, int32_t* counts,
                                     int* status, cudaStream_t stream);

// Bytes of the status word every prefill attention call keeps in its workspace.
constexpr size_t kStatusBytes = 256;

}  // namespace rtp
