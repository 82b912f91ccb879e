// Indexer selection: decode token top-k and prefill block top-k.
//
// Decode (the 128K decode workload statement): every retrieval head scores
// every cached token by q~ . k~ (r = 16) and keeps the top-k tokens. The key
// index of a KV group is read once for all retrieval heads of that group
// (grouped-query heads share keys); scores go to the caller's workspace, then
// one CTA per (sequence, head) runs an exact radix select over them.
//
// Prefill (the tiny 2K prefill workload statement): the block score of query
// block i against key block j is the max of q~_t . k~_u over causal pairs of
// the two 64-token blocks; each query block keeps its top-k key blocks. The
// block scores of one query block live in shared memory and never reach HBM.
#include "rtp_common.cuh"
#include "rtp_internal.h"

namespace rtp {

// ---------------------------------------------------------------------------
// Decode
// ---------------------------------------------------------------------------
constexpr int kScanThreads = 256;
constexpr int kScanTokensPerThread = 4;

__global__ void __launch_bounds__(kScanThreads)
decode_scan_kernel(const float* __restrict__ qt, const uint4* __restrict__ kindex, int L, int Hr,
                   int Hkv, const HeadList hl, float* __restrict__ scores) {
  const int b = blockIdx.z, g = blockIdx.y;
  __shared__ float qs[kMaxHeads][RTP_R];
  __shared__ int js[kMaxHeads];
  __shared__ int nj;
  if (threadIdx.x == 0) {
    int c = 0;
    for (int j = 0; j < hl.n; ++j)
      if (hl.kv[j] == g) js[c++] = j;
    nj = c;
  }
  __syncthreads();
  const int n = nj;
  if (n == 0) return;
  for (int e = threadIdx.x; e < n * RTP_R; e += blockDim.x)
    qs[e / RTP_R][e % RTP_R] = qt[((size_t)b * Hr + js[e / RTP_R]) * RTP_R + e % RTP_R];
  __syncthreads();
  const uint4* krow = kindex + ((size_t)b * Hkv + g) * (size_t)L * 2;
  const int base = blockIdx.x * kScanThreads * kScanTokensPerThread;
#pragma unroll
  for (int s = 0; s < kScanTokensPerThread; ++s) {
    const int u = base + s * kScanThreads + threadIdx.x;
    if (u >= L) break;
    const uint4 lo = __ldg(krow + (size_t)u * 2), hi = __ldg(krow + (size_t)u * 2 + 1);
    float k[16] = {bf16_lo(lo.x), bf16_hi(lo.x), bf16_lo(lo.y), bf16_hi(lo.y),
                   bf16_lo(lo.z), bf16_hi(lo.z), bf16_lo(lo.w), bf16_hi(lo.w),
                   bf16_lo(hi.x), bf16_hi(hi.x), bf16_lo(hi.y), bf16_hi(hi.y),
                   bf16_lo(hi.z), bf16_hi(hi.z), bf16_lo(hi.w), bf16_hi(hi.w)};
    for (int jj = 0; jj < n; ++jj) {
      float acc = 0.f;
#pragma unroll
      for (int c = 0; c < RTP_R; ++c) acc = fmaf(qs[jj][c], k[c], acc);
      scores[((size_t)b * Hr + js[jj]) * L + u] = acc;
    }
  }
}

constexpr int kSelThreads = 1024;

__global__ void __launch_bounds__(kSelThreads)
decode_topk_kernel(const float* __restrict__ scores, int L, int Hr, int topk, int32_t* __restrict__ idx) {
  __shared__ TopkSmem<kSelThreads> sm;
  const int j = blockIdx.x, b = blockIdx.y;
  const float* s = scores + ((size_t)b * Hr + j) * L;
  auto get_key = [s](int i) { return f2key(__ldg(s + i)); };
  block_topk_ascending<kSelThreads>(get_key, L, topk, idx + ((size_t)b * Hr + j) * topk, sm);
}

size_t select_decode_ws_bytes(int B, int L, int Hr, int topk) {
  (void)topk;
  return (size_t)B * Hr * L * sizeof(float);
}

static void fill_heads(HeadList& hl, const int32_t* kv_of, int Hr) {
  hl.n = Hr;
  for (int j = 0; j < Hr; ++j) { hl.head[j] = j; hl.kv[j] = kv_of[j]; }
}

cudaError_t launch_select_decode(const float* qt, const void* kindex, int B, int L, int Hr,
                                 int Hkv, const int32_t* kv_of, int topk, int32_t* idx,
                                 void* ws, cudaStream_t stream) {
  HeadList hl;
  fill_heads(hl, kv_of, Hr);
  float* scores = static_cast<float*>(ws);
  dim3 g1((L + kScanThreads * kScanTokensPerThread - 1) / (kScanThreads * kScanTokensPerThread), Hkv, B);
  decode_scan_kernel<<<g1, kScanThreads, 0, stream>>>(qt, static_cast<const uint4*>(kindex), L, Hr,
                                                      Hkv, hl, scores);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  dim3 g2(Hr, B);
  decode_topk_kernel<<<g2, kSelThreads, 0, stream>>>(scores, L, Hr, topk, idx);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// Prefill
// ---------------------------------------------------------------------------
constexpr int kPSelThreads = 256;

struct PrefillSelectSmem {
  float q[RTP_BLOCK][RTP_R];
  float part[kPSelThreads / 32];
  TopkSmem<kPSelThreads> topk;
};

__global__ void __launch_bounds__(kPSelThreads)
prefill_select_kernel(const uint4* __restrict__ qt, const uint4* __restrict__ kt, int N, int Hr,
                      int Hkv, const HeadList hl, int topk, int32_t* __restrict__ blocks,
                      int32_t* __restrict__ counts) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  PrefillSelectSmem& sm = *reinterpret_cast<PrefillSelectSmem*>(smem_raw);
  float* s = reinterpret_cast<float*>(smem_raw + sizeof(PrefillSelectSmem));
  const int nb = N / RTP_BLOCK;
  const int i = nb - 1 - blockIdx.x;          // longest lists first
  const int j = blockIdx.y, b = blockIdx.z;
  const int g = hl.kv[j];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

  const uint4* qrow = qt + (((size_t)b * Hr + j) * N + (size_t)i * RTP_BLOCK) * 2;
  for (int e = tid; e < RTP_BLOCK * 2; e += kPSelThreads) {
    uint4 w = __ldg(qrow + e);
    float* d = &sm.q[e >> 1][(e & 1) * 8];
    d[0] = bf16_lo(w.x); d[1] = bf16_hi(w.x); d[2] = bf16_lo(w.y); d[3] = bf16_hi(w.y);
    d[4] = bf16_lo(w.z); d[5] = bf16_hi(w.z); d[6] = bf16_lo(w.w); d[7] = bf16_hi(w.w);
  }
  __syncthreads();
  const uint4* krows = kt + ((size_t)b * Hkv + g) * (size_t)N * 2;
  const int keys_per_iter = kPSelThreads;                 // 4 key blocks per iteration
  const int n_keys = (i + 1) * RTP_BLOCK;
  for (int u0 = 0; u0 < n_keys; u0 += keys_per_iter) {
    const int u = u0 + tid;
    float best = -INFINITY;
    if (u < n_keys) {
      const uint4 lo = __ldg(krows + (size_t)u * 2), hi = __ldg(krows + (size_t)u * 2 + 1);
      const float k[16] = {bf16_lo(lo.x), bf16_hi(lo.x), bf16_lo(lo.y), bf16_hi(lo.y),
                           bf16_lo(lo.z), bf16_hi(lo.z), bf16_lo(lo.w), bf16_hi(lo.w),
                           bf16_lo(hi.x), bf16_hi(hi.x), bf16_lo(hi.y), bf16_hi(hi.y),
                           bf16_lo(hi.z), bf16_hi(hi.z), bf16_lo(hi.w), bf16_hi(hi.w)};
      // Causal pairs only: query t = 64 i + r needs u <= t.
      const int r0 = (u >= i * RTP_BLOCK) ? (u - i * RTP_BLOCK) : 0;
      for (int r = r0; r < RTP_BLOCK; ++r) {
        float acc = 0.f;
#pragma unroll
        for (int c = 0; c < RTP_R; ++c) acc = fmaf(sm.q[r][c], k[c], acc);
        best = fmaxf(best, acc);
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) best = fmaxf(best, __shfl_xor_sync(0xffffffffu, best, o));
    if (lane == 0) sm.part[warp] = best;
    __syncthreads();
    if (tid < kPSelThreads / 64) {
      const int jb = u0 / RTP_BLOCK + tid;
      if (jb <= i) s[jb] = fmaxf(sm.part[2 * tid], sm.part[2 * tid + 1]);
    }
    __syncthreads();
  }
  int32_t* out = blocks + (((size_t)b * Hr + j) * nb + i) * topk;
  auto get_key = [s](int x) { return f2key(s[x]); };
  block_topk_ascending<kPSelThreads>(get_key, i + 1, topk, out, sm.topk);
  if (tid == 0) counts[((size_t)b * Hr + j) * nb + i] = min(topk, i + 1);
}

size_t select_prefill_ws_bytes(int B, int N, int Hr, int topk) {
  (void)B; (void)N; (void)Hr; (void)topk;
  return kStatusBytes;
}

cudaError_t launch_select_prefill(const void* qt, const void* kt, int B, int N, int Hr, int Hkv,
                                  const int32_t* kv_of, int topk, int32_t* blocks,
                                  int32_t* counts, void* ws, cudaStream_t stream) {
  return launch_select_prefill_tc(qt, kt, B, N, Hr, Hkv, kv_of, topk, blocks, counts,
                                  static_cast<int*>(ws), stream);
}

cudaError_t launch_select_prefill_simt(const void* qt, const void* kt, int B, int N, int Hr, int Hkv,
                                       const int32_t* kv_of, int topk, int32_t* blocks,
                                       int32_t* counts, cudaStream_t stream) {
  HeadList hl;
  fill_heads(hl, kv_of, Hr);
  const int nb = N / RTP_BLOCK;
  const size_t smem = sizeof(PrefillSelectSmem) + (size_t)nb * sizeof(float);
  if (smem > 227 * 1024) return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(prefill_select_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid(nb, Hr, B);
  prefill_select_kernel<<<grid, kPSelThreads, smem, stream>>>(
      static_cast<const uint4*>(qt), static_cast<const uint4*>(kt), N, Hr, Hkv, hl, topk, blocks,
      counts);
  return cudaGetLastError();
}

}  // namespace rtp
