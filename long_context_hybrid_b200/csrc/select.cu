// Decode token selection: every retrieval head scores every cached token by
// q~ . k~ (r = 16) and keeps its top-k tokens (the 128K decode workload
// statement: token-level top-2048 over the whole cache; RTPurbo digest: the
// 16-d indexer is the scout). Exact ties rank the smaller token first.
//
// Two kernels:
//   scan    one pass over the key index; a KV group's index is read once for
//           all retrieval heads of that group (grouped-query heads share
//           keys). It writes every score (fp32, to the workspace, sized to stay
//           in L2) and a histogram of the top 11 bits of each score's
//           order-preserving key.
//   filter  several CTAs per (sequence, head), each over a slice of the
//           L2-resident scores. From the histogram every CTA knows the bin
//           holding the k-th score: it marks the scores above that bin in a
//           per-row bitmap (every 32-token word is owned by one CTA, so plain
//           stores) and appends the bin's members to a candidate list. The
//           last CTA of a row to finish settles the bin by a radix search over
//           the candidates' remaining bits (exact ties: smallest token first),
//           sets their bits and compacts the bitmap into the ascending index
//           list. If the candidates overflow their list it runs a full radix
//           select over the row instead.
#include "rtp_common.cuh"
#include "rtp_internal.h"

namespace rtp {

namespace {
constexpr int kScanThreads = 256;
constexpr int kScanTokensPerThread = 16;
constexpr int kScanBatch = 8;
constexpr int kScanTokens = kScanThreads * kScanTokensPerThread;   // 4096 per CTA
constexpr int kBins = 2048;                                        // top 11 bits
constexpr int kFiltThreads = 512;
constexpr int kFiltStep = kFiltThreads * 16;                       // scores per CTA step
constexpr int kMaxTopk = 4096;

// Per-row bookkeeping of the filter kernel (zeroed with the histogram).
struct RowState {
  int n_cand;
  int ticket;
  int pad[2];
};

// Candidate-list capacity per row: an eighth of the row, at least 8192.
__host__ __device__ inline int cand_cap(int L) { return L / 8 > 8192 ? L / 8 : 8192; }

struct DecodeWs {
  float* scores;          // [B, Hr, L]
  uint32_t* hist;         // [B, Hr, kBins]
  RowState* state;        // [B, Hr]      (zeroed together with hist)
  uint32_t* bitmap;       // [B, Hr, ceil(L / 32)]
  uint2* cand;            // [B, Hr, cand_cap(L)] (key, token)
  size_t zero_bytes;      // hist + state
  size_t total;
};

inline size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

DecodeWs decode_ws_layout(void* base, int B, int L, int Hr) {
  const size_t rows = (size_t)B * Hr;
  DecodeWs w;
  char* p = static_cast<char*>(base);
  size_t off = 0;
  w.scores = reinterpret_cast<float*>(p + off);
  off = align256(off + rows * L * sizeof(float));
  w.hist = reinterpret_cast<uint32_t*>(p + off);
  w.state = reinterpret_cast<RowState*>(p + off + rows * kBins * sizeof(uint32_t));
  w.zero_bytes = rows * (kBins * sizeof(uint32_t) + sizeof(RowState));
  off = align256(off + w.zero_bytes);
  w.bitmap = reinterpret_cast<uint32_t*>(p + off);
  off = align256(off + rows * ((L + 31) / 32) * sizeof(uint32_t));
  w.cand = reinterpret_cast<uint2*>(p + off);
  off = align256(off + rows * cand_cap(L) * sizeof(uint2));
  w.total = off;
  return w;
}

// Bin (top 11 key bits) of the k-th largest score of a row from its histogram,
// and how many scores lie in higher bins. All threads get the result.
template <int NT>
__device__ void kth_bin(const uint32_t* __restrict__ h, int k, TopkSmem<NT>& sm, uint32_t& bin, int& above) {
  const int tid = threadIdx.x;
  constexpr int per = kBins / NT;
  int local = 0;
  uint32_t c[per];
#pragma unroll
  for (int q = 0; q < per; ++q) {
    c[q] = __ldcg(h + kBins - 1 - (tid * per + q));
    local += c[q];
  }
  int tot;
  const int ab = block_exclusive_scan<NT>(local, tot, sm.scan);
  if (ab < k && ab + local >= k) {
    int run = ab;
#pragma unroll
    for (int q = 0; q < per; ++q) {
      if (run + (int)c[q] >= k) { sm.digit = kBins - 1 - (tid * per + q); sm.above = run; break; }
      run += c[q];
    }
  }
  __syncthreads();
  bin = (uint32_t)sm.digit;
  above = sm.above;
  __syncthreads();
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
  // batches of kScanBatch tokens per thread: all their loads are issued
  // before any score is computed (32 bytes per token in flight)
#pragma unroll 1
  for (int s0 = 0; s0 < kScanTokensPerThread; s0 += kScanBatch) {
    uint4 lo[kScanBatch], hi[kScanBatch];
#pragma unroll
    for (int t = 0; t < kScanBatch; ++t) {
      const int u = base + (s0 + t) * kScanThreads + threadIdx.x;
      if (u < L) {
        lo[t] = __ldg(krow + (size_t)u * 2);
        hi[t] = __ldg(krow + (size_t)u * 2 + 1);
      }
    }
#pragma unroll
    for (int t = 0; t < kScanBatch; ++t) {
      const int u = base + (s0 + t) * kScanThreads + threadIdx.x;
      if (u >= L) break;
      const float k[16] = {bf16_lo(lo[t].x), bf16_hi(lo[t].x), bf16_lo(lo[t].y), bf16_hi(lo[t].y),
                           bf16_lo(lo[t].z), bf16_hi(lo[t].z), bf16_lo(lo[t].w), bf16_hi(lo[t].w),
                           bf16_lo(hi[t].x), bf16_hi(hi[t].x), bf16_lo(hi[t].y), bf16_hi(hi[t].y),
                           bf16_lo(hi[t].z), bf16_hi(hi[t].z), bf16_lo(hi[t].w), bf16_hi(hi[t].w)};
      for (int jj = 0; jj < n; ++jj) {
        float acc = 0.f;
#pragma unroll
        for (int c = 0; c < RTP_R; ++c) acc = fmaf(qs[jj][c], k[c], acc);
        scores[((size_t)b * Hr + js[jj]) * L + u] = acc;
        atomicAdd(&shist[jj * kBins + (f2key(acc) >> 21)], 1u);
      }
    }
  }
  __syncthreads();
  for (int e = threadIdx.x; e < n * kBins; e += kScanThreads) {
    const uint32_t c = shist[e];
    if (c) atomicAdd(&ghist[((size_t)b * Hr + js[e / kBins]) * kBins + (e % kBins)], c);
  }
}

__global__ void __launch_bounds__(kFiltThreads)
decode_filter_kernel(const DecodeWs w, int L, int Hr, int topk, int slice, int n_split, int32_t* __restrict__ idx) {
  __shared__ TopkSmem<kFiltThreads> sm;
  __shared__ int s_last;
  const int part = blockIdx.x, j = blockIdx.y, b = blockIdx.z, tid = threadIdx.x;
  const int lane = tid & 31, warp = tid >> 5;
  const size_t row = (size_t)b * Hr + j;
  int32_t* out = idx + row * topk;
  if (L <= topk) {
    if (part == 0)
      for (int i = tid; i < topk; i += kFiltThreads) out[i] = i < L ? i : -1;
    return;
  }
  const float* s = w.scores + row * L;
  const int W = (L + 31) >> 5;
  const int cap = cand_cap(L);
  uint32_t* bm = w.bitmap + row * W;
  uint2* cand = w.cand + row * cap;
  uint32_t d1;
  int above1;
  kth_bin<kFiltThreads>(w.hist + row * kBins, topk, sm, d1, above1);

  // 1. this CTA's slice: bits for the scores above bin d1, candidates inside it.
  //    A lane takes 16 consecutive scores; lanes 2m, 2m+1 share one bitmap word.
  const int lo = part * slice, hi = min(L, lo + slice);
  const bool vec = (L & 3) == 0;
  for (int wbase = lo + warp * 512; wbase < hi; wbase += kFiltStep) {
    const int base = wbase + lane * 16;
    float x[16];
    if (vec && base + 16 <= hi) {
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const float4 v = __ldg(reinterpret_cast<const float4*>(s + base) + q);
        x[4 * q] = v.x; x[4 * q + 1] = v.y; x[4 * q + 2] = v.z; x[4 * q + 3] = v.w;
      }
    } else {
#pragma unroll
      for (int e = 0; e < 16; ++e) x[e] = base + e < hi ? __ldg(s + base + e) : 0.f;
    }
    uint32_t bits = 0, cbits = 0;
#pragma unroll
    for (int e = 0; e < 16; ++e) {
      const uint32_t d = f2key(x[e]) >> 21;
      const bool valid = base + e < hi;
      bits |= (valid && d > d1) ? 1u << e : 0u;
      cbits |= (valid && d == d1) ? 1u << e : 0u;
    }
    // candidates: one global atomic per warp, lanes write their own in order
    const int nc = __popc(cbits);
    int incl = nc;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    const int wtot = __shfl_sync(0xffffffffu, incl, 31);
    if (wtot) {
      int cbase = 0;
      if (lane == 31) cbase = atomicAdd(&w.state[row].n_cand, wtot);
      cbase = __shfl_sync(0xffffffffu, cbase, 31);
      int pos = cbase + incl - nc;
#pragma unroll
      for (int e = 0; e < 16; ++e)
        if ((cbits >> e) & 1u) {
          if (pos < cap) cand[pos] = make_uint2(f2key(x[e]), (uint32_t)(base + e));
          ++pos;
        }
    }
    uint32_t word = bits << ((lane & 1) * 16);
    word |= __shfl_xor_sync(0xffffffffu, word, 1);
    if (!(lane & 1) && base < hi) bm[base >> 5] = word;
  }

  // 2. the last CTA of the row settles bin d1 and writes the list
  __threadfence();
  __syncthreads();
  if (tid == 0) s_last = atomicAdd(&w.state[row].ticket, 1) == n_split - 1;
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  const int n_cand = __ldcg(&w.state[row].n_cand);
  if (n_cand > cap) {
    // candidates overflowed: exact radix select over the whole row
    auto key_of = [s](int i) { return f2key(__ldg(s + i)); };
    block_topk_ascending<kFiltThreads>(key_of, L, topk, out, sm);
    return;
  }
  const uint2* cc = cand;
  int need = topk - above1;
  auto ckey = [cc](int x) { return __ldcg(&cc[x].x); };
  const uint32_t thr = block_radix_threshold<kFiltThreads>(ckey, n_cand, need, sm, 1, d1 << 21, 0x7FFu << 21);
  // keys equal to the threshold: the `need` smallest tokens among them
  int n_eq = 0;
  for (int x = tid; x < n_cand; x += kFiltThreads) n_eq += __ldcg(&cc[x].x) == thr;
  int eq_tot;
  block_exclusive_scan<kFiltThreads>(n_eq, eq_tot, sm.scan);
  uint32_t tie_thr = 0;   // on ~token: larger means smaller token
  if (need < eq_tot) {
    int need2 = need;
    auto tkey = [cc, thr](int x) {
      const uint2 e = __ldcg(cc + x);
      return e.x == thr ? ~e.y : 0u;
    };
    tie_thr = block_radix_threshold<kFiltThreads>(tkey, n_cand, need2, sm);
  }
  for (int x = tid; x < n_cand; x += kFiltThreads) {
    const uint2 e = __ldcg(cc + x);
    if (e.x > thr || (e.x == thr && ~e.y >= tie_thr)) atomicOr(bm + (e.y >> 5), 1u << (e.y & 31));
  }
  __syncthreads();
  // 3. ordered compaction of the bitmap: ascending token indices
  const int per = (W + kFiltThreads - 1) / kFiltThreads;
  int cnt = 0;
  for (int q = 0; q < per; ++q) {
    const int wi = tid * per + q;
    if (wi < W) cnt += __popc(__ldcg(bm + wi));
  }
  int tot;
  int pos = block_exclusive_scan<kFiltThreads>(cnt, tot, sm.scan);
  for (int q = 0; q < per; ++q) {
    const int wi = tid * per + q;
    if (wi >= W) break;
    uint32_t v = __ldcg(bm + wi);
    while (v) {
      const int bit = __ffs(v) - 1;
      v &= v - 1;
      if (pos < topk) out[pos] = wi * 32 + bit;
      ++pos;
    }
  }
}

size_t select_decode_ws_bytes(int B, int L, int Hr, int topk) {
  (void)topk;
  return decode_ws_layout(nullptr, B, L, Hr).total;
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
  const DecodeWs w = decode_ws_layout(ws, B, L, Hr);
  cudaError_t e = cudaMemsetAsync(w.hist, 0, w.zero_bytes, stream);
  if (e != cudaSuccess) return e;
  const size_t scan_smem = (size_t)max_nj * kBins * sizeof(uint32_t);
  if (scan_smem > 48 * 1024) {
    e = cudaFuncSetAttribute(decode_scan_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)scan_smem);
    if (e != cudaSuccess) return e;
  }
  dim3 g1((L + kScanTokens - 1) / kScanTokens, Hkv, B);
  decode_scan_kernel<<<g1, kScanThreads, scan_smem, stream>>>(qt, static_cast<const uint4*>(kindex), L, Hr, Hkv,
                                                              hl, w.scores, w.hist);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  // about two CTAs per SM over all rows; slices are whole CTA steps
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int rows = B * Hr;
  int n_split = (2 * sms + rows - 1) / rows;
  int slice = (L + n_split - 1) / n_split;
  slice = (slice + 511) / 512 * 512;
  n_split = (L + slice - 1) / slice;
  dim3 g2(n_split, Hr, B);
  decode_filter_kernel<<<g2, kFiltThreads, 0, stream>>>(w, L, Hr, topk, slice, n_split, idx);
  return cudaGetLastError();
}

}  // namespace rtp
