// Decode attention: one new query token per sequence against the KV cache.
//
// Streaming heads attend the last `window` tokens (RTPurboV2 article: SWA on
// streaming heads). Retrieval heads attend, as a set, their selected tokens,
// tokens 0..sink-1 and the last `window` tokens (the 128K decode workload
// statement: top-2048 unioned with the last 8192 tokens and token 0, exact
// softmax at D = 128).
//
// Split-K: every (sequence, head) key set is cut into chunks of kChunk keys
// (window chunks first, then chunks of the selected-token list, the first of
// which also carries the sink). One CTA per chunk produces an unnormalised
// partial (running max m in the log2 domain, sum l, o[128]) in the workspace;
// a merge kernel combines the chunks of each head with the usual rescaling.
#include <mutex>

#include "rtp_common.cuh"
#include "rtp_internal.h"

namespace rtp {

constexpr int kDecThreads = 128;
constexpr int kChunk = 256;
constexpr int kUnroll = 8;
constexpr int kPartStride = 2 + RTP_D;

struct DecodeParams {
  const __nv_bfloat16* q; int64_t q_sb, q_sh;
  const __nv_bfloat16* k; int64_t k_sb, k_sn, k_sh;
  const __nv_bfloat16* v; int64_t v_sb, v_sn, v_sh;
  __nv_bfloat16* o; int64_t o_sb, o_sh;
  int L, q_pos, Hq, Hkv, G;
  int is_ret;
  const int32_t* idx; int topk;
  int window, sink;
  float scale_log2;
  int n_heads, max_splits;
  float* part;
  int head[kMaxHeads];
};

__device__ __forceinline__ void load4(const __nv_bfloat16* p, float* f) {
  uint2 w = __ldg(reinterpret_cast<const uint2*>(p));
  f[0] = bf16_lo(w.x); f[1] = bf16_hi(w.x); f[2] = bf16_lo(w.y); f[3] = bf16_hi(w.y);
}

__global__ void __launch_bounds__(kDecThreads)
decode_attn_partial_kernel(const DecodeParams p) {
  const int split = blockIdx.x, j = blockIdx.y, b = blockIdx.z;
  const int h = p.head[j], g = h / p.G;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int whi = min(p.L, p.q_pos + 1);
  const int wlo = max(0, p.q_pos - p.window + 1);
  const int n_wc = (whi - wlo + kChunk - 1) / kChunk;
  float* part = p.part + (((size_t)b * p.n_heads + j) * p.max_splits + split) * kPartStride;

  // Which keys this chunk covers.
  int kind, c;  // kind 0: window chunk c; 1: selected-list chunk c (+ sink if c == 0)
  if (split < n_wc) { kind = 0; c = split; }
  else if (p.is_ret && split - n_wc < (p.topk + kChunk - 1) / kChunk) { kind = 1; c = split - n_wc; }
  else {
    if (threadIdx.x == 0) { part[0] = -INFINITY; part[1] = 0.f; }
    return;
  }
  const int n_sink = (kind == 1 && c == 0) ? min(p.sink, wlo) : 0;
  const int n_slots = kChunk + n_sink;
  const int32_t* sel = p.idx + ((size_t)b * p.n_heads + j) * p.topk;

  float qv[4];
  load4(p.q + b * p.q_sb + h * p.q_sh + 4 * lane, qv);
#pragma unroll
  for (int e = 0; e < 4; ++e) qv[e] *= p.scale_log2;
  const __nv_bfloat16* kbase = p.k + b * p.k_sb + g * p.k_sh + 4 * lane;
  const __nv_bfloat16* vbase = p.v + b * p.v_sb + g * p.v_sh + 4 * lane;

  float m = -INFINITY, l = 0.f, acc[4] = {0.f, 0.f, 0.f, 0.f};
  for (int s0 = warp * kUnroll; s0 < n_slots; s0 += 4 * kUnroll) {
    int u[kUnroll];
#pragma unroll
    for (int t = 0; t < kUnroll; ++t) {
      const int s = s0 + t;
      int pos = -1;
      if (s < n_slots) {
        if (kind == 0) {
          pos = wlo + c * kChunk + s;
          if (pos >= whi) pos = -1;
        } else if (s < kChunk) {
          const int e = c * kChunk + s;
          if (e < p.topk) {
            pos = __ldg(sel + e);
            if (pos < p.sink || pos >= wlo) pos = -1;   // sink and window keys come from elsewhere
          }
        } else {
          pos = s - kChunk;                             // sink token
        }
      }
      u[t] = pos;
    }
    float kf[kUnroll][4], vf[kUnroll][4];
#pragma unroll
    for (int t = 0; t < kUnroll; ++t) {
      if (u[t] >= 0) {
        load4(kbase + (int64_t)u[t] * p.k_sn, kf[t]);
        load4(vbase + (int64_t)u[t] * p.v_sn, vf[t]);
      }
    }
#pragma unroll
    for (int t = 0; t < kUnroll; ++t) {
      if (u[t] < 0) continue;
      float d = qv[0] * kf[t][0] + qv[1] * kf[t][1] + qv[2] * kf[t][2] + qv[3] * kf[t][3];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) d += __shfl_xor_sync(0xffffffffu, d, o);
      const float mn = fmaxf(m, d);
      const float corr = exp2f(m - mn);
      const float pe = exp2f(d - mn);
      l = l * corr + pe;
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[e] = acc[e] * corr + pe * vf[t][e];
      m = mn;
    }
  }
  // Combine the four warps.
  __shared__ float sm_m[4], sm_l[4];
  __shared__ float sm_o[4][RTP_D];
  if (lane == 0) { sm_m[warp] = m; sm_l[warp] = l; }
#pragma unroll
  for (int e = 0; e < 4; ++e) sm_o[warp][4 * lane + e] = acc[e];
  __syncthreads();
  if (warp == 0) {
    float M = fmaxf(fmaxf(sm_m[0], sm_m[1]), fmaxf(sm_m[2], sm_m[3]));
    float w[4], L = 0.f;
#pragma unroll
    for (int x = 0; x < 4; ++x) {
      w[x] = (sm_m[x] == -INFINITY) ? 0.f : exp2f(sm_m[x] - M);
      L += w[x] * sm_l[x];
    }
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int d = 4 * lane + e;
      part[2 + d] = w[0] * sm_o[0][d] + w[1] * sm_o[1][d] + w[2] * sm_o[2][d] + w[3] * sm_o[3][d];
    }
    if (lane == 0) { part[0] = M; part[1] = L; }
  }
}

__global__ void __launch_bounds__(RTP_D)
decode_attn_merge_kernel(const DecodeParams p) {
  const int j = blockIdx.x, b = blockIdx.y, d = threadIdx.x;
  const float* part = p.part + ((size_t)b * p.n_heads + j) * p.max_splits * kPartStride;
  float M = -INFINITY;
  for (int s = 0; s < p.max_splits; ++s) M = fmaxf(M, part[s * kPartStride]);
  float L = 0.f, acc = 0.f;
  for (int s = 0; s < p.max_splits; ++s) {
    const float ms = part[s * kPartStride];
    if (ms == -INFINITY) continue;
    const float w = exp2f(ms - M);
    L += w * part[s * kPartStride + 1];
    acc += w * part[s * kPartStride + 2 + d];
  }
  const int h = p.head[j];
  p.o[b * p.o_sb + h * p.o_sh + d] = __float2bfloat16_rn(acc / L);
}

static int max_splits_for(int window, int topk, int is_ret) {
  return (window + kChunk - 1) / kChunk + (is_ret ? (topk + kChunk - 1) / kChunk : 0);
}

size_t decode_attn_ws_bytes(int B, int L, int n_heads, int topk, int window) {
  const int w = window < L ? window : L;
  return (size_t)B * n_heads * max_splits_for(w, topk, 1) * kPartStride * sizeof(float);
}

cudaError_t launch_decode_attn(const void* q, int64_t q_sb, int64_t q_sh,
                               const void* kc, int64_t k_sb, int64_t k_sn, int64_t k_sh,
                               const void* vc, int64_t v_sb, int64_t v_sn, int64_t v_sh,
                               void* o, int64_t o_sb, int64_t o_sh,
                               int B, int L, int q_pos, int Hq, int Hkv,
                               const int32_t* heads, int n_heads, int is_ret,
                               const int32_t* idx, int topk, int window, int sink, float scale,
                               void* ws, cudaStream_t stream) {
  DecodeParams p;
  p.q = static_cast<const __nv_bfloat16*>(q); p.q_sb = q_sb; p.q_sh = q_sh;
  p.k = static_cast<const __nv_bfloat16*>(kc); p.k_sb = k_sb; p.k_sn = k_sn; p.k_sh = k_sh;
  p.v = static_cast<const __nv_bfloat16*>(vc); p.v_sb = v_sb; p.v_sn = v_sn; p.v_sh = v_sh;
  p.o = static_cast<__nv_bfloat16*>(o); p.o_sb = o_sb; p.o_sh = o_sh;
  p.L = L; p.q_pos = q_pos; p.Hq = Hq; p.Hkv = Hkv; p.G = Hq / Hkv;
  p.is_ret = is_ret; p.idx = idx; p.topk = is_ret ? topk : 0;
  p.window = window; p.sink = is_ret ? sink : 0;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.n_heads = n_heads;
  const int span = (q_pos + 1 < window ? q_pos + 1 : window);
  p.max_splits = max_splits_for(span, p.topk, is_ret);
  p.part = static_cast<float*>(ws);
  for (int i = 0; i < n_heads; ++i) p.head[i] = heads[i];
  dim3 g1(p.max_splits, n_heads, B);
  decode_attn_partial_kernel<<<g1, kDecThreads, 0, stream>>>(p);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  dim3 g2(n_heads, B);
  decode_attn_merge_kernel<<<g2, RTP_D, 0, stream>>>(p);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// Allocation-free variant: the split-K partials live in a fixed device array.
// ---------------------------------------------------------------------------
// Every GPU that loads the library holds this array until the process exits.
// Host code must not pass `g_decode_scratch` itself to a kernel (on the host
// that name is only a stand-in); it uses the device address fetched below.
static __device__ __align__(256) float g_decode_scratch[kNoAllocScratchBytes / sizeof(float)];

namespace {
constexpr int kMaxDevices = 64;
std::mutex g_scratch_mutex;
void* g_scratch_ptr[kMaxDevices] = {};
}  // namespace

// Device address of g_decode_scratch on the current device, looked up once
// per device (with that device current) and cached.
static cudaError_t decode_scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_scratch_mutex);
  if (!g_scratch_ptr[dev]) {
    void* ptr = nullptr;
    e = cudaGetSymbolAddress(&ptr, g_decode_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_ptr[dev] = ptr;
  }
  *out = g_scratch_ptr[dev];
  return cudaSuccess;
}

cudaError_t launch_decode_attn_noalloc(const void* q, int64_t q_sb, int64_t q_sh,
                                       const void* kc, int64_t k_sb, int64_t k_sn, int64_t k_sh,
                                       const void* vc, int64_t v_sb, int64_t v_sn, int64_t v_sh,
                                       void* o, int64_t o_sb, int64_t o_sh,
                                       int B, int L, int q_pos, int Hq, int Hkv,
                                       const int32_t* heads, int n_heads, const int32_t* idx, int topk,
                                       int window, int sink, float scale, cudaStream_t stream) {
  // Every partial the merge reads is written by the same call's partial
  // kernel, so nothing in the array has to start at zero.
  void* scratch = nullptr;
  cudaError_t e = decode_scratch_address(&scratch);
  if (e != cudaSuccess) return e;
  return launch_decode_attn(q, q_sb, q_sh, kc, k_sb, k_sn, k_sh, vc, v_sb, v_sn, v_sh, o, o_sb, o_sh, B, L,
                            q_pos, Hq, Hkv, heads, n_heads, 1, idx, topk, window, sink, scale, scratch, stream);
}

}  // namespace rtp
