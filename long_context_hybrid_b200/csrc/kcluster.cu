// K-cache clustering and the two-level decode selection (RTPurboV2 article:
// the sequence-dimension compression paragraph, clustering lets decode skip
// most semantically unrelated tokens, and the low-rank key vectors make the
// cluster centres accurate; the Qwen3-Coder-30B-A3B recipe clusters the
// retrieval heads' K cache). The pages give no algorithm; this is Lloyd
// k-means over each (sequence, KV head)'s key index and a two-level top-k.
//
// Build (once, over the first L tokens of the index):
//   init      C = ceil(L / S) centroids from the rows 0, S, 2 S, ... (fp32);
//   assign    every row to its nearest centroid: sum over c of (x_c - mu_c)^2
//             with each subtraction, square and addition rounded to fp32 in
//             the order c = 0, 1, ... (no fused multiply-add), ties to the
//             smaller centroid; centroids staged through shared memory;
//   accumulate exact int64 sums of trunc(x * 2^20) and counts per cluster
//             (integer atomics: the result does not depend on their order);
//   finalize  mu = fp32(double(sum) / double(count) * 2^-20), an empty
//             cluster keeping its centroid;
//   after `iters` rounds a last assignment, then the members of every
//   cluster as a CSR list (offsets by an exclusive scan of the counts; the
//   order inside a cluster is arbitrary: the selection breaks ties by token).
// Select (per (sequence, retrieval head), one block):
//   the C centroid scores q~ . mu (fp32), an exact top-n_probe of them (ties
//   to the smaller cluster); the probed clusters' members and every token
//   past the clustered prefix (appended after the build) marked in a shared
//   token bitmap and compacted in token order; their scores q~ . k~; an exact
//   top-k by (score, token) and the ascending index list.
#include "rtp_common.cuh"
#include "rtp_internal.h"

namespace rtp {

namespace {
constexpr int kAsgThreads = 256;
constexpr int kAsgChunk = 256;                 // centroids staged per step
constexpr int kSelThreads = 1024;
constexpr int kSelWords = 8192;                // token bitmap words (clustered prefix up to 262144 tokens)
constexpr double kFixScale = 1048576.0;        // 2^20

__device__ __forceinline__ void load_row16(const uint4* p, float* x) {
  const uint4 lo = __ldg(p), hi = __ldg(p + 1);
  const uint32_t v[8] = {lo.x, lo.y, lo.z, lo.w, hi.x, hi.y, hi.z, hi.w};
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    x[2 * i] = bf16_lo(v[i]);
    x[2 * i + 1] = bf16_hi(v[i]);
  }
}
}  // namespace

__global__ void kc_init_kernel(const uint4* __restrict__ kindex, int64_t cap, int S, int C, float* __restrict__ mu) {
  const int bh = blockIdx.y;
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= C) return;
  float x[16];
  load_row16(kindex + ((int64_t)bh * cap + (int64_t)i * S) * 2, x);
#pragma unroll
  for (int c = 0; c < 16; ++c) mu[((int64_t)bh * C + i) * 16 + c] = x[c];
}

// One thread per row; the block walks the centroids in staged chunks.
__global__ void __launch_bounds__(kAsgThreads)
kc_assign_kernel(const uint4* __restrict__ kindex, int64_t cap, int L, int C, const float* __restrict__ mu,
                 int32_t* __restrict__ assign) {
  __shared__ float ms[kAsgChunk][16];
  const int bh = blockIdx.y;
  const int u = blockIdx.x * kAsgThreads + threadIdx.x;
  float x[16];
  if (u < L) load_row16(kindex + ((int64_t)bh * cap + u) * 2, x);
  else
#pragma unroll
    for (int c = 0; c < 16; ++c) x[c] = 0.f;
  float best = INFINITY;
  int besti = 0;
  const float* m = mu + (int64_t)bh * C * 16;
  for (int i0 = 0; i0 < C; i0 += kAsgChunk) {
    const int n = min(kAsgChunk, C - i0);
    __syncthreads();
    for (int e = threadIdx.x; e < n * 16; e += kAsgThreads) ms[e >> 4][e & 15] = m[(int64_t)i0 * 16 + e];
    __syncthreads();
    for (int i = 0; i < n; ++i) {
      float d = 0.f;
#pragma unroll
      for (int c = 0; c < 16; ++c) {
        const float df = __fsub_rn(x[c], ms[i][c]);
        d = __fadd_rn(d, __fmul_rn(df, df));
      }
      if (d < best) { best = d; besti = i0 + i; }       // ascending i: ties keep the smaller
    }
  }
  if (u < L) assign[(int64_t)bh * L + u] = besti;
}

__global__ void kc_accumulate_kernel(const uint4* __restrict__ kindex, int64_t cap, int L, int C,
                                     const int32_t* __restrict__ assign, unsigned long long* __restrict__ sums,
                                     int* __restrict__ counts) {
  const int bh = blockIdx.y;
  const int u = blockIdx.x * blockDim.x + threadIdx.x;
  if (u >= L) return;
  float x[16];
  load_row16(kindex + ((int64_t)bh * cap + u) * 2, x);
  const int a = assign[(int64_t)bh * L + u];
  unsigned long long* s = sums + ((int64_t)bh * C + a) * 16;
#pragma unroll
  for (int c = 0; c < 16; ++c) {
    // x * 2^20 is exact in fp32 here; truncation toward zero to an integer
    const long long f = __float2ll_rz(x[c] * 1048576.0f);
    atomicAdd(s + c, (unsigned long long)f);             // two's complement: exact signed sums
  }
  atomicAdd(counts + (int64_t)bh * C + a, 1);
}

__global__ void kc_finalize_kernel(int C, const unsigned long long* __restrict__ sums, const int* __restrict__ counts,
                                   float* __restrict__ mu) {
  const int bh = blockIdx.y;
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= C) return;
  const int n = counts[(int64_t)bh * C + i];
  if (n == 0) return;
#pragma unroll
  for (int c = 0; c < 16; ++c) {
    const long long sm = (long long)sums[((int64_t)bh * C + i) * 16 + c];
    mu[((int64_t)bh * C + i) * 16 + c] = __double2float_rn(__ddiv_rn(__ll2double_rn(sm), (double)n) / kFixScale);
  }
}

// Exclusive scan of one (sequence, head)'s counts into offsets[0 .. C], and the
// scatter cursors (a copy of the offsets).
__global__ void __launch_bounds__(1024)
kc_offsets_kernel(int C, const int* __restrict__ counts, int32_t* __restrict__ offsets, int* __restrict__ cursor) {
  __shared__ BlockScanSmem<1024> scan;
  const int bh = blockIdx.x;
  const int per = (C + 1023) / 1024;
  const int i0 = threadIdx.x * per;
  int local = 0;
  for (int q = 0; q < per; ++q)
    if (i0 + q < C) local += counts[(int64_t)bh * C + i0 + q];
  int tot;
  int run = block_exclusive_scan<1024>(local, tot, scan);
  for (int q = 0; q < per; ++q) {
    const int i = i0 + q;
    if (i >= C) break;
    offsets[(int64_t)bh * (C + 1) + i] = run;
    cursor[(int64_t)bh * C + i] = run;
    run += counts[(int64_t)bh * C + i];
  }
  if (threadIdx.x == 0) offsets[(int64_t)bh * (C + 1) + C] = tot;
}

__global__ void kc_scatter_kernel(int L, int C, const int32_t* __restrict__ assign, int* __restrict__ cursor,
                                  int32_t* __restrict__ members) {
  const int bh = blockIdx.y;
  const int u = blockIdx.x * blockDim.x + threadIdx.x;
  if (u >= L) return;
  const int a = assign[(int64_t)bh * L + u];
  const int p = atomicAdd(cursor + (int64_t)bh * C + a, 1);
  members[(int64_t)bh * L + p] = u;
}

namespace {
struct BuildWs {
  unsigned long long* sums;   // [B*Hkv, C, 16]
  int* counts;                // [B*Hkv, C]
  int* cursor;                // [B*Hkv, C]
  size_t total;
};
inline size_t al256(size_t x) { return (x + 255) & ~(size_t)255; }
BuildWs build_ws(void* base, int n_bh, int C) {
  BuildWs w;
  char* p = static_cast<char*>(base);
  size_t off = 0;
  w.sums = reinterpret_cast<unsigned long long*>(p + off);
  off = al256(off + (size_t)n_bh * C * 16 * 8);
  w.counts = reinterpret_cast<int*>(p + off);
  off = al256(off + (size_t)n_bh * C * 4);
  w.cursor = reinterpret_cast<int*>(p + off);
  off = al256(off + (size_t)n_bh * C * 4);
  w.total = off;
  return w;
}
}  // namespace

size_t kcluster_build_ws_bytes(int B, int Hkv, int L, int S) {
  const int C = (L + S - 1) / S;
  return build_ws(nullptr, B * Hkv, C).total;
}

cudaError_t launch_kcluster_build(const void* kindex, int64_t cap, int B, int Hkv, int L, int S, int iters,
                                  float* mu, int32_t* assign, int32_t* offsets, int32_t* members, void* ws,
                                  cudaStream_t stream) {
  const int n_bh = B * Hkv;
  const int C = (L + S - 1) / S;
  const BuildWs w = build_ws(ws, n_bh, C);
  const uint4* k = static_cast<const uint4*>(kindex);
  const dim3 gc((C + 255) / 256, n_bh), gl((L + 255) / 256, n_bh), ga((L + kAsgThreads - 1) / kAsgThreads, n_bh);
  kc_init_kernel<<<gc, 256, 0, stream>>>(k, cap, S, C, mu);
  cudaError_t e = cudaGetLastError();
  for (int it = 0; it < iters && e == cudaSuccess; ++it) {
    kc_assign_kernel<<<ga, kAsgThreads, 0, stream>>>(k, cap, L, C, mu, assign);
    e = cudaMemsetAsync(w.sums, 0, (size_t)n_bh * C * 16 * 8, stream);
    if (e != cudaSuccess) break;
    e = cudaMemsetAsync(w.counts, 0, (size_t)n_bh * C * 4, stream);
    if (e != cudaSuccess) break;
    kc_accumulate_kernel<<<gl, 256, 0, stream>>>(k, cap, L, C, assign, w.sums, w.counts);
    kc_finalize_kernel<<<gc, 256, 0, stream>>>(C, w.sums, w.counts, mu);
    e = cudaGetLastError();
  }
  if (e != cudaSuccess) return e;
  kc_assign_kernel<<<ga, kAsgThreads, 0, stream>>>(k, cap, L, C, mu, assign);
  e = cudaMemsetAsync(w.counts, 0, (size_t)n_bh * C * 4, stream);
  if (e != cudaSuccess) return e;
  kc_accumulate_kernel<<<gl, 256, 0, stream>>>(k, cap, L, C, assign, w.sums, w.counts);   // counts (sums unused)
  kc_offsets_kernel<<<n_bh, 1024, 0, stream>>>(C, w.counts, offsets, w.cursor);
  kc_scatter_kernel<<<gl, 256, 0, stream>>>(L, C, assign, w.cursor, members);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// Two-level selection
// ---------------------------------------------------------------------------
namespace {
struct SelWs {
  uint32_t* ckey;    // [rows, C]: centroid score keys
  int32_t* probe;    // [rows, n_probe]: probed clusters
  int32_t* ctok;     // [rows, L]: candidate tokens in token order
  uint32_t* skey;    // [rows, L]: their score keys
  size_t total;
};
SelWs sel_ws(void* base, int rows, int C, int n_probe, int L) {
  SelWs w;
  char* p = static_cast<char*>(base);
  size_t off = 0;
  w.ckey = reinterpret_cast<uint32_t*>(p + off);
  off = al256(off + (size_t)rows * C * 4);
  w.probe = reinterpret_cast<int32_t*>(p + off);
  off = al256(off + (size_t)rows * n_probe * 4);
  w.ctok = reinterpret_cast<int32_t*>(p + off);
  off = al256(off + (size_t)rows * L * 4);
  w.skey = reinterpret_cast<uint32_t*>(p + off);
  off = al256(off + (size_t)rows * L * 4);
  w.total = off;
  return w;
}

constexpr int kSelKeys = 8192;      // centroid or candidate keys (and tokens) kept in shared memory
struct SelSmem {
  TopkSmem<kSelThreads> tk;
  uint32_t bits[kSelWords];
  uint32_t keys[kSelKeys];            // centroid keys, then candidate keys
  int32_t toks[kSelKeys];             // candidate tokens in token order
  float q[16];
  int n_cand;
};
}  // namespace

struct ClusterSelParams {
  const float* qt;            // [B, Hr, 16]
  const uint4* kindex;        // [B, Hkv, cap, 16] bf16 rows
  int64_t cap;
  const float* mu;            // [B, Hkv, C, 16]
  const int32_t* offsets;     // [B, Hkv, C + 1]
  const int32_t* members;     // [B, Hkv, L0]
  int B, L0, L, Hr, Hkv, C, n_probe, topk;
  int32_t* idx;               // [B, Hr, topk]
  int kv[kMaxHeads];
};

__global__ void __launch_bounds__(kSelThreads)
kc_select_kernel(const ClusterSelParams p, const SelWs w) {
  extern __shared__ __align__(16) unsigned char kc_smem[];
  SelSmem& sm = *reinterpret_cast<SelSmem*>(kc_smem);
  pdl_trigger();         // a decode step's attention may launch; it waits for this grid before reading idx
  const int j = blockIdx.x, b = blockIdx.y, tid = threadIdx.x;
  const int row = b * p.Hr + j;
  const int bh = b * p.Hkv + p.kv[j];
  if (tid < 16) sm.q[tid] = p.qt[(int64_t)row * 16 + tid];
  const int W = (p.L + 31) >> 5;
  for (int x = tid; x < W; x += kSelThreads) sm.bits[x] = 0u;
  __syncthreads();
  float q[16];
#pragma unroll
  for (int c = 0; c < 16; ++c) q[c] = sm.q[c];
  // 1. centroid scores, exact top-n_probe of them (ascending cluster ids)
  //    (keys in shared memory when they fit, else in the workspace)
  uint32_t* ck = w.ckey + (int64_t)row * p.C;
  const bool ck_sm = p.C <= kSelKeys;
  const float* mu = p.mu + (int64_t)bh * p.C * 16;
  for (int i = tid; i < p.C; i += kSelThreads) {
    float acc = 0.f;
#pragma unroll
    for (int c = 0; c < 16; ++c) acc = fmaf(q[c], __ldg(mu + (int64_t)i * 16 + c), acc);
    if (ck_sm) sm.keys[i] = f2key(acc);
    else ck[i] = f2key(acc);
  }
  __syncthreads();
  int32_t* probe = w.probe + (int64_t)row * p.n_probe;
  block_topk_ascending<kSelThreads>([&](int i) { return ck_sm ? sm.keys[i] : __ldcg(ck + i); }, p.C, p.n_probe,
                                    probe, sm.tk);
  __syncthreads();
  // 2. candidates: the probed clusters' members and the tokens past the
  //    clustered prefix, marked in the token bitmap
  const int32_t* off = p.offsets + (int64_t)bh * (p.C + 1);
  const int32_t* mem = p.members + (int64_t)bh * p.L0;
  // one warp per probed cluster (every warp's loads in flight together)
  const int n_pr = min(p.n_probe, p.C);
  const int lane = tid & 31, warp = tid >> 5;
  for (int e = warp; e < n_pr; e += kSelThreads / 32) {
    int a0 = 0, a1 = 0;
    if (lane == 0) {
      const int c = __ldcg(probe + e);
      a0 = __ldg(off + c);
      a1 = __ldg(off + c + 1);
    }
    a0 = __shfl_sync(0xffffffffu, a0, 0);
    a1 = __shfl_sync(0xffffffffu, a1, 0);
    for (int x = a0 + lane; x < a1; x += 32) {
      const int u = __ldg(mem + x);
      atomicOr(&sm.bits[u >> 5], 1u << (u & 31));
    }
  }
  for (int u = p.L0 + tid; u < p.L; u += kSelThreads) atomicOr(&sm.bits[u >> 5], 1u << (u & 31));
  __syncthreads();
  // 3. compaction in token order, scores of the candidates
  int32_t* ct = w.ctok + (int64_t)row * p.L;
  uint32_t* sk = w.skey + (int64_t)row * p.L;
  const int per = (W + kSelThreads - 1) / kSelThreads;
  int cnt = 0;
  for (int qq = 0; qq < per; ++qq) {
    const int wi = tid * per + qq;
    if (wi < W) cnt += __popc(sm.bits[wi]);
  }
  int n_cand;
  int pos = block_exclusive_scan<kSelThreads>(cnt, n_cand, sm.tk.scan);
  const bool c_sm = n_cand <= kSelKeys;           // candidates (tokens, keys) in shared memory
  for (int qq = 0; qq < per; ++qq) {
    const int wi = tid * per + qq;
    if (wi >= W) break;
    uint32_t v = sm.bits[wi];
    while (v) {
      const int bit = __ffs(v) - 1;
      v &= v - 1;
      if (c_sm) sm.toks[pos++] = wi * 32 + bit;
      else ct[pos++] = wi * 32 + bit;
    }
  }
  __syncthreads();
  // the candidates' scores, two rows of a thread in flight together
  for (int i0 = 0; i0 < n_cand; i0 += 2 * kSelThreads) {
    int us[2];
#pragma unroll
    for (int t = 0; t < 2; ++t) {
      const int i = i0 + t * kSelThreads + tid;
      us[t] = i < n_cand ? (c_sm ? sm.toks[i] : __ldcg(ct + i)) : -1;
    }
    uint4 lo[2], hi[2];
#pragma unroll
    for (int t = 0; t < 2; ++t)
      if (us[t] >= 0) {
        const uint4* r = p.kindex + ((int64_t)bh * p.cap + us[t]) * 2;
        lo[t] = __ldg(r);
        hi[t] = __ldg(r + 1);
      }
#pragma unroll
    for (int t = 0; t < 2; ++t) {
      if (us[t] < 0) continue;
      const uint32_t v8[8] = {lo[t].x, lo[t].y, lo[t].z, lo[t].w, hi[t].x, hi[t].y, hi[t].z, hi[t].w};
      float acc = 0.f;
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        acc = fmaf(q[2 * c], bf16_lo(v8[c]), acc);
        acc = fmaf(q[2 * c + 1], bf16_hi(v8[c]), acc);
      }
      if (c_sm) sm.keys[i0 + t * kSelThreads + tid] = f2key(acc);
      else sk[i0 + t * kSelThreads + tid] = f2key(acc);
    }
  }
  __syncthreads();
  // 4. top-k by (score, token): candidate positions are in token order
  int32_t* out = p.idx + (int64_t)row * p.topk;
  block_topk_ascending<kSelThreads>([&](int i) { return c_sm ? sm.keys[i] : __ldcg(sk + i); }, n_cand, p.topk, out,
                                    sm.tk);
  __syncthreads();
  for (int i = tid; i < p.topk; i += kSelThreads) {
    const int x = __ldcg(out + i);
    if (x >= 0) out[i] = c_sm ? sm.toks[x] : __ldcg(ct + x);
  }
}

size_t kcluster_select_ws_bytes(int B, int Hr, int C, int n_probe, int L) {
  return sel_ws(nullptr, B * Hr, C, n_probe, L).total;
}

cudaError_t launch_kcluster_select(const float* qt, const void* kindex, int64_t cap, const float* mu,
                                   const int32_t* offsets, const int32_t* members, int B, int L0, int L, int Hr,
                                   int Hkv, int C, const int32_t* kv_of, int n_probe, int topk, int32_t* idx,
                                   void* ws, cudaStream_t stream) {
  ClusterSelParams p;
  p.qt = qt; p.kindex = static_cast<const uint4*>(kindex); p.cap = cap; p.mu = mu; p.offsets = offsets;
  p.members = members; p.B = B; p.L0 = L0; p.L = L; p.Hr = Hr; p.Hkv = Hkv; p.C = C; p.n_probe = n_probe;
  p.topk = topk; p.idx = idx;
  for (int j = 0; j < Hr; ++j) p.kv[j] = kv_of[j];
  const SelWs w = sel_ws(ws, B * Hr, C, n_probe, L);
  cudaError_t e = cudaFuncSetAttribute(kc_select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)sizeof(SelSmem));
  if (e != cudaSuccess) return e;
  kc_select_kernel<<<dim3(Hr, B), kSelThreads, sizeof(SelSmem), stream>>>(p, w);
  return cudaGetLastError();
}

}  // namespace rtp
