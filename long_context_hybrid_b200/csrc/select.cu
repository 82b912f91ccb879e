// Decode token selection: every retrieval head scores every cached token by
// q~ . k~ (r = 16) and keeps its top-k tokens (the 128K decode workload
// statement: token-level top-2048 over the whole cache; RTPurbo digest: the
// 16-d indexer is the scout). Exact ties rank the smaller token first.
//
// Two kernels:
//   scan   one pass over the key index; a KV group's index is read once for all
//          retrieval heads of that group (grouped-query heads share keys). It
//          writes every score (fp32, to the workspace, sized to stay in L2) and
//          a histogram of the top 11 bits of each score's order-preserving key.
//   top-k  one CTA per (sequence, head): from the histogram it knows the bin
//          holding the k-th score (top 11 bits). Pass 1 over the L2-resident
//          scores takes every score above that bin and histograms the next 11
//          bits of the scores inside it; pass 2 takes the scores above the
//          finer bin and gathers that bin's few members as candidates in
//          shared memory, where a radix search over the last 10 bits (and the
//          token index for exact ties) settles the rest; the list is then
//          sorted ascending. If the candidates still overflow shared memory
//          the CTA falls back to a full radix select over the scores.
#include "rtp_common.cuh"
#include "rtp_internal.h"

namespace rtp {

namespace {
constexpr int kScanThreads = 256;
constexpr int kScanTokensPerThread = 32;
constexpr int kScanTokens = kScanThreads * kScanTokensPerThread;   // 8192 per CTA
constexpr int kBins = 2048;                                        // top 11 bits
constexpr int kTopkThreads = 1024;
constexpr int kCandCap = 12288;
constexpr int kMaxTopk = 4096;

struct DecodeTopkSmem {
  TopkSmem<kTopkThreads> tk;
  uint32_t cand_key[kCandCap];
  int cand_idx[kCandCap];
  int sel[kMaxTopk];
  int n_sel, n_cand, n_eq;
};

// Calls f(i, key, valid) over one score list [0, L): each warp takes 512
// consecutive scores per step (16 per lane, four 16-byte loads issued
// together; scalar loads when L is not a multiple of 4). Every lane of a warp
// makes the same calls, so f may use warp votes; `valid` is false past L.
template <int NT, class F>
__device__ __forceinline__ void for_each_key(const float* __restrict__ s, int L, F f) {
  const bool vec = (L & 3) == 0;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  for (int wbase = warp * 512; wbase < L; wbase += NT * 16) {
    const int base = wbase + lane * 16;
    float x[16];
    if (vec && base + 16 <= L) {
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const float4 w = __ldg(reinterpret_cast<const float4*>(s + base) + q);
        x[4 * q] = w.x; x[4 * q + 1] = w.y; x[4 * q + 2] = w.z; x[4 * q + 3] = w.w;
      }
    } else {
#pragma unroll
      for (int e = 0; e < 16; ++e) x[e] = base + e < L ? __ldg(s + base + e) : 0.f;
    }
#pragma unroll
    for (int e = 0; e < 16; ++e) f(base + e, f2key(x[e]), base + e < L);
  }
}

// Appends `i` to list[] (counter *n) for the lanes with `take`, one shared
// atomic per warp.
__device__ __forceinline__ void warp_append(bool take, int i, int* list, int* n) {
  const unsigned m = __ballot_sync(0xffffffffu, take);
  if (m == 0) return;
  const int lane = threadIdx.x & 31, leader = __ffs(m) - 1;
  int base = 0;
  if (lane == leader) base = atomicAdd(n, __popc(m));
  base = __shfl_sync(0xffffffffu, base, leader);
  if (take) list[base + __popc(m & ((1u << lane) - 1u))] = i;
}

size_t hist_offset(int B, int L, int Hr) {
  return (((size_t)B * Hr * L * sizeof(float)) + 255) & ~(size_t)255;
}
}  // namespace

__global__ void __launch_bounds__(kScanThreads)
decode_scan_kernel(const float* __restrict__ qt, const uint4* __restrict__ kindex, int L, int Hr, int Hkv,
                   const HeadList hl, float* __restrict__ scores, uint32_t* __restrict__ ghist) {
  extern __shared__ uint32_t shist[];                  // [n_j][kBins]
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
  for (int e = threadIdx.x; e < n * RTP_R; e += kScanThreads)
    qs[e / RTP_R][e % RTP_R] = qt[((size_t)b * Hr + js[e / RTP_R]) * RTP_R + e % RTP_R];
  for (int e = threadIdx.x; e < n * kBins; e += kScanThreads) shist[e] = 0u;
  __syncthreads();
  const uint4* krow = kindex + ((size_t)b * Hkv + g) * (size_t)L * 2;
  const int base = blockIdx.x * kScanTokens;
#pragma unroll 4
  for (int s = 0; s < kScanTokensPerThread; ++s) {
    const int u = base + s * kScanThreads + threadIdx.x;
    if (u >= L) break;
    const uint4 lo = __ldg(krow + (size_t)u * 2), hi = __ldg(krow + (size_t)u * 2 + 1);
    const float k[16] = {bf16_lo(lo.x), bf16_hi(lo.x), bf16_lo(lo.y), bf16_hi(lo.y),
                         bf16_lo(lo.z), bf16_hi(lo.z), bf16_lo(lo.w), bf16_hi(lo.w),
                         bf16_lo(hi.x), bf16_hi(hi.x), bf16_lo(hi.y), bf16_hi(hi.y),
                         bf16_lo(hi.z), bf16_hi(hi.z), bf16_lo(hi.w), bf16_hi(hi.w)};
    for (int jj = 0; jj < n; ++jj) {
      float acc = 0.f;
#pragma unroll
      for (int c = 0; c < RTP_R; ++c) acc = fmaf(qs[jj][c], k[c], acc);
      scores[((size_t)b * Hr + js[jj]) * L + u] = acc;
      atomicAdd(&shist[jj * kBins + (f2key(acc) >> 21)], 1u);
    }
  }
  __syncthreads();
  for (int e = threadIdx.x; e < n * kBins; e += kScanThreads) {
    const uint32_t c = shist[e];
    if (c) atomicAdd(&ghist[((size_t)b * Hr + js[e / kBins]) * kBins + (e % kBins)], c);
  }
}

__global__ void __launch_bounds__(kTopkThreads)
decode_topk_kernel(const float* __restrict__ scores, const uint32_t* __restrict__ ghist, int L, int Hr, int topk,
                   int32_t* __restrict__ idx) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  DecodeTopkSmem& sm = *reinterpret_cast<DecodeTopkSmem*>(smem_raw);
  const int j = blockIdx.x, b = blockIdx.y, tid = threadIdx.x;
  const float* s = scores + ((size_t)b * Hr + j) * L;
  int32_t* out = idx + ((size_t)b * Hr + j) * topk;
  auto key_of = [s](int i) { return f2key(__ldg(s + i)); };
  if (L <= topk) {
    for (int i = tid; i < topk; i += kTopkThreads) out[i] = (i < L) ? i : -1;
    return;
  }
  // 1. bin of the k-th score from the scan's histogram
  const uint32_t* h = ghist + ((size_t)b * Hr + j) * kBins;
  for (int x = tid; x < kBins; x += kTopkThreads) sm.tk.hist[x] = h[x];
  if (tid == 0) { sm.n_sel = 0; sm.n_cand = 0; sm.n_eq = 0; }
  __syncthreads();
  constexpr int per = kBins / kTopkThreads;
  int local = 0;
  for (int q = 0; q < per; ++q) local += sm.tk.hist[kBins - 1 - (tid * per + q)];
  int tot;
  const int above_t = block_exclusive_scan<kTopkThreads>(local, tot, sm.tk.scan);
  if (above_t < topk && above_t + local >= topk) {
    int run = above_t;
    for (int q = 0; q < per; ++q) {
      const int bin = kBins - 1 - (tid * per + q);
      const int c = sm.tk.hist[bin];
      if (run + c >= topk) { sm.tk.digit = bin; sm.tk.above = run; break; }
      run += c;
    }
  }
  __syncthreads();
  const uint32_t d1 = (uint32_t)sm.tk.digit;
  const int above1 = sm.tk.above;
  __syncthreads();
  // 2a. pass 1: take keys above bin d1, histogram bits [20:10] inside it
  for (int x = tid; x < kBins; x += kTopkThreads) sm.tk.hist[x] = 0u;
  __syncthreads();
  for_each_key<kTopkThreads>(s, L, [&](int i, uint32_t key, bool valid) {
    const uint32_t d = key >> 21;
    warp_append(valid && d > d1, i, sm.sel, &sm.n_sel);
    if (valid && d == d1) atomicAdd(&sm.tk.hist[(key >> 10) & 2047u], 1u);
  });
  __syncthreads();
  const int need1 = topk - above1;
  {
    int loc = 0;
    for (int q = 0; q < per; ++q) loc += sm.tk.hist[kBins - 1 - (tid * per + q)];
    int t2;
    const int ab = block_exclusive_scan<kTopkThreads>(loc, t2, sm.tk.scan);
    if (ab < need1 && ab + loc >= need1) {
      int run = ab;
      for (int q = 0; q < per; ++q) {
        const int bin = kBins - 1 - (tid * per + q);
        const int c = sm.tk.hist[bin];
        if (run + c >= need1) { sm.tk.digit = bin; sm.tk.above = run; break; }
        run += c;
      }
    }
    __syncthreads();
  }
  const uint32_t pre22 = (d1 << 11) | (uint32_t)sm.tk.digit;   // key >> 10 of the k-th key
  const int above = above1 + sm.tk.above;
  __syncthreads();
  // 2b. pass 2: take keys above the 22-bit bin, gather the bin's members
  for_each_key<kTopkThreads>(s, L, [&](int i, uint32_t key, bool valid) {
    const bool in1 = valid && (key >> 21) == d1;
    const uint32_t d = key >> 10;
    warp_append(in1 && d > pre22, i, sm.sel, &sm.n_sel);
    if (in1 && d == pre22) {
      const int pos = atomicAdd(&sm.n_cand, 1);
      if (pos < kCandCap) { sm.cand_key[pos] = key; sm.cand_idx[pos] = i; }
    }
  });
  __syncthreads();
  const int n_cand = sm.n_cand;
  if (n_cand > kCandCap || sm.n_sel != above) {
    // candidates do not fit: exact radix select over all scores instead
    block_topk_ascending<kTopkThreads>(key_of, L, topk, out, sm.tk);
    return;
  }
  // 3. settle the bin: radix search over its remaining bits, then the lowest
  //    token indices among keys equal to the threshold
  int need = topk - above;
  const uint32_t* ck = sm.cand_key;
  auto cand_key = [ck](int x) { return ck[x]; };
  const uint32_t thr = block_radix_threshold<kTopkThreads>(cand_key, n_cand, need, sm.tk, 2, pre22 << 10,
                                                            0x3FFFFFu << 10);
  for (int x = tid; x < n_cand; x += kTopkThreads)
    if (sm.cand_key[x] > thr) sm.sel[atomicAdd(&sm.n_sel, 1)] = sm.cand_idx[x];
  __syncthreads();
  // equal keys: each takes its rank among the equal ones by token index
  for (int x = tid; x < n_cand; x += kTopkThreads) {
    if (sm.cand_key[x] != thr) continue;
    const int me = sm.cand_idx[x];
    int rank = 0;
    for (int y = 0; y < n_cand; ++y)
      if (sm.cand_key[y] == thr && sm.cand_idx[y] < me) ++rank;
    if (rank < need) sm.sel[atomicAdd(&sm.n_sel, 1)] = me;
  }
  __syncthreads();
  // 4. ascending order
  int n_pow2 = 1;
  while (n_pow2 < topk) n_pow2 <<= 1;
  for (int x = topk + tid; x < n_pow2; x += kTopkThreads) sm.sel[x] = 0x7fffffff;
  __syncthreads();
  block_bitonic_sort<kTopkThreads>(sm.sel, n_pow2);
  for (int x = tid; x < topk; x += kTopkThreads) out[x] = sm.sel[x];
}

size_t select_decode_ws_bytes(int B, int L, int Hr, int topk) {
  (void)topk;
  return hist_offset(B, L, Hr) + (size_t)B * Hr * kBins * sizeof(uint32_t);
}

cudaError_t launch_select_decode(const float* qt, const void* kindex, int B, int L, int Hr, int Hkv,
                                 const int32_t* kv_of, int topk, int32_t* idx, void* ws, cudaStream_t stream) {
  if (topk > kMaxTopk) return cudaErrorInvalidValue;
  HeadList hl;
  hl.n = Hr;
  int max_nj = 0;
  for (int g = 0; g < Hkv; ++g) {
    int c = 0;
    for (int j = 0; j < Hr; ++j) c += (kv_of[j] == g);
    max_nj = c > max_nj ? c : max_nj;
  }
  for (int j = 0; j < Hr; ++j) { hl.head[j] = j; hl.kv[j] = kv_of[j]; }
  float* scores = static_cast<float*>(ws);
  uint32_t* ghist = reinterpret_cast<uint32_t*>(static_cast<char*>(ws) + hist_offset(B, L, Hr));
  cudaError_t e = cudaMemsetAsync(ghist, 0, (size_t)B * Hr * kBins * sizeof(uint32_t), stream);
  if (e != cudaSuccess) return e;
  const size_t scan_smem = (size_t)max_nj * kBins * sizeof(uint32_t);
  if (scan_smem > 48 * 1024) {
    e = cudaFuncSetAttribute(decode_scan_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)scan_smem);
    if (e != cudaSuccess) return e;
  }
  dim3 g1((L + kScanTokens - 1) / kScanTokens, Hkv, B);
  decode_scan_kernel<<<g1, kScanThreads, scan_smem, stream>>>(qt, static_cast<const uint4*>(kindex), L, Hr, Hkv,
                                                              hl, scores, ghist);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const size_t topk_smem = sizeof(DecodeTopkSmem);
  e = cudaFuncSetAttribute(decode_topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)topk_smem);
  if (e != cudaSuccess) return e;
  dim3 g2(Hr, B);
  decode_topk_kernel<<<g2, kTopkThreads, topk_smem, stream>>>(scores, ghist, L, Hr, topk, idx);
  return cudaGetLastError();
}

}  // namespace rtp
