// Decode attention: one new query token per sequence against the KV cache.
//
// Streaming heads attend the last `window` tokens (RTPurboV2 article: SWA on
// streaming heads). Retrieval heads attend, as a set, their selected tokens,
// tokens 0..sink-1 and their own last `window` tokens (the 128K decode
// workload statement: top-2048 unioned with the last 8192 tokens and token 0,
// exact softmax at D = 128).
//
// The work is HBM-bound (512 bytes of K and V per attended token), so the
// design goal is to read every K/V row once:
//   * window items: one CTA per (sequence, KV group, 128-token chunk of the
//     window); every listed query head of that group is one row of a
//     16 x 128 query tile (grouped-query heads share the chunk's K/V), and
//     each row masks keys outside its own window;
//   * gathered items: one CTA per (sequence, retrieval head, 128-entry chunk
//     of its selected list, the sink tokens first); entries inside the
//     window or below `sink` are masked (those keys come from elsewhere).
// A CTA stages its 128 K and V rows in shared memory with cp.async (zero-fill
// for masked slots), computes S = Q K^T and O = P V with bf16 mma.sync
// (fp32 accumulate) in four warps of 32 keys, and writes an unnormalised
// partial (running max in the log2 domain, sum, o[128]) per head; a merge
// kernel combines the partials of each head.
#include <mutex>

#include "rtp_common.cuh"
#include "rtp_internal.h"

namespace rtp {

namespace {
constexpr int kThreads = 128;
constexpr int kChunk = 128;                 // keys per CTA (32 per warp)
constexpr int kRowPad = RTP_D + 8;          // shared row stride in elements (272 B: conflict-free ldmatrix)
constexpr int kPartStride = 2 + RTP_D;
constexpr int kMaxGroup = 16;               // query heads per KV group packed in one MMA tile

struct DecodeParams {
  const __nv_bfloat16* q; int64_t q_sb, q_sh;
  const __nv_bfloat16* k; int64_t k_sb, k_sn, k_sh;
  const __nv_bfloat16* v; int64_t v_sb, v_sn, v_sh;
  __nv_bfloat16* o; int64_t o_sb, o_sh;
  int B, L, q_pos, Hq, Hkv, G;
  const int32_t* idx; int topk;
  int sink;
  float scale_log2;
  int n_heads, max_splits;
  int n_wc, wlo_union, whi;          // window chunks over [wlo_union, whi)
  int n_gc;                          // gathered chunks per retrieval head
  int n_window_items;                // B * Hkv * n_wc
  float* part;
  int head[kMaxHeads];
  int ret_row[kMaxHeads];            // row of idx for a retrieval head, -1 for a streaming head
  int wlo[kMaxHeads];                // first position of each head's window
  int ret_list[kMaxHeads];           // call-head index of the r-th retrieval head
  int n_ret;
};

struct Smem {
  __nv_bfloat16 k[kChunk][kRowPad];
  __nv_bfloat16 v[kChunk][kRowPad];
  __nv_bfloat16 q[kMaxGroup][kRowPad];
  int pos[kChunk];
  int rows[kMaxGroup];               // call-head index per tile row, -1 if unused
  float m[4][kMaxGroup], l[4][kMaxGroup];
};

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, bool valid) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(valid ? 16 : 0)
               : "memory");
}
__device__ __forceinline__ void ldsm_x4(uint32_t* r, uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t* r, uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(addr));
}
__device__ __forceinline__ void mma16816(float* c, const uint32_t* a, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
      "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};\n"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ uint32_t pack2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}
__device__ __forceinline__ uint32_t su32(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }
}  // namespace

__global__ void __launch_bounds__(kThreads)
decode_attn_partial_kernel(const DecodeParams p) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  Smem& sm = *reinterpret_cast<Smem*>(smem_raw);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int item = blockIdx.x;
  int b, g, split, n_rows;
  const bool is_window = item < p.n_window_items;
  if (is_window) {
    const int wc = item % p.n_wc;
    const int bg = item / p.n_wc;
    g = bg % p.Hkv; b = bg / p.Hkv; split = wc;
    if (tid == 0) {
      int c = 0;
      for (int j = 0; j < p.n_heads && c < kMaxGroup; ++j)
        if (p.head[j] / p.G == g) sm.rows[c++] = j;
      for (int r = c; r < kMaxGroup; ++r) sm.rows[r] = -1;
    }
  } else {
    const int it = item - p.n_window_items;
    const int gc = it % p.n_gc;
    const int rr = (it / p.n_gc) % p.n_ret;
    b = it / (p.n_gc * p.n_ret);
    const int j = p.ret_list[rr];
    g = p.head[j] / p.G; split = p.n_wc + gc;
    if (tid == 0) {
      sm.rows[0] = j;
      for (int r = 1; r < kMaxGroup; ++r) sm.rows[r] = -1;
    }
  }
  __syncthreads();
  // key positions of the chunk's slots (-1: masked for every row)
  if (is_window) {
    for (int s = tid; s < kChunk; s += kThreads) {
      const int u = p.wlo_union + split * kChunk + s;
      sm.pos[s] = u < p.whi ? u : -1;
    }
  } else {
    const int j = sm.rows[0];
    const int wlo = p.wlo[j];
    const int n_sink = min(p.sink, wlo);
    const int gc = split - p.n_wc;
    const int32_t* sel = p.idx + ((size_t)b * p.n_ret + p.ret_row[j]) * p.topk;
    for (int s = tid; s < kChunk; s += kThreads) {
      const int e = gc * kChunk + s;          // virtual list: sink tokens, then the selected entries
      int pos = -1;
      if (e < n_sink) pos = e;
      else if (e - n_sink < p.topk) {
        const int u = __ldg(sel + (e - n_sink));
        pos = (u >= p.sink && u < wlo) ? u : -1;
      }
      sm.pos[s] = pos;
    }
  }
  __syncthreads();
  n_rows = 0;
  for (int r = 0; r < kMaxGroup; ++r) n_rows += sm.rows[r] >= 0;

  // stage K, V (128 rows x 256 B each) and the query rows
  const __nv_bfloat16* kb = p.k + (int64_t)b * p.k_sb + (int64_t)g * p.k_sh;
  const __nv_bfloat16* vb = p.v + (int64_t)b * p.v_sb + (int64_t)g * p.v_sh;
  // two copy groups: K and the query rows first, V second (S and the softmax
  // run while V is still arriving)
  for (int e = tid; e < kChunk * 16; e += kThreads) {
    const int s = e >> 4, c = (e & 15) * 8;
    const int pos = sm.pos[s];
    const int64_t off = pos >= 0 ? (int64_t)pos : 0;
    cp_async16(su32(&sm.k[s][c]), kb + off * p.k_sn + c, pos >= 0);
  }
  for (int e = tid; e < kMaxGroup * 16; e += kThreads) {
    const int r = e >> 4, c = (e & 15) * 8;
    const int j = sm.rows[r];
    const __nv_bfloat16* src = p.q + (int64_t)b * p.q_sb + (int64_t)(j >= 0 ? p.head[j] : 0) * p.q_sh + c;
    cp_async16(su32(&sm.q[r][c]), src, j >= 0);
  }
  asm volatile("cp.async.commit_group;\n" ::: "memory");
  for (int e = tid; e < kChunk * 16; e += kThreads) {
    const int s = e >> 4, c = (e & 15) * 8;
    const int pos = sm.pos[s];
    const int64_t off = pos >= 0 ? (int64_t)pos : 0;
    cp_async16(su32(&sm.v[s][c]), vb + off * p.v_sn + c, pos >= 0);
  }
  asm volatile("cp.async.commit_group;\n" ::: "memory");
  asm volatile("cp.async.wait_group 1;\n" ::: "memory");
  __syncthreads();

  const int gq = lane >> 2, tq = lane & 3;
  const int key0 = warp * 32;                 // this warp's 32 keys: 4 n-tiles of 8
  // S = Q K^T (16 rows x 32 keys)
  float sacc[4][4];
#pragma unroll
  for (int nt = 0; nt < 4; ++nt)
#pragma unroll
    for (int x = 0; x < 4; ++x) sacc[nt][x] = 0.f;
#pragma unroll
  for (int kk = 0; kk < 8; ++kk) {
    uint32_t a[4];
    {
      const int m = lane >> 3;
      const int row = (lane & 7) + 8 * (m & 1), col = kk * 16 + 8 * (m >> 1);
      ldsm_x4(a, su32(&sm.q[row][col]));
    }
#pragma unroll
    for (int np = 0; np < 2; ++np) {          // two n-tiles per ldmatrix.x4
      uint32_t bf[4];
      const int m = lane >> 3;
      const int key = key0 + 8 * (2 * np + (m >> 1)) + (lane & 7), col = kk * 16 + 8 * (m & 1);
      ldsm_x4(bf, su32(&sm.k[key][col]));
      mma16816(sacc[2 * np], a, bf[0], bf[1]);
      mma16816(sacc[2 * np + 1], a, bf[2], bf[3]);
    }
  }
  // mask + per-row max over this warp's keys (rows gq and gq+8)
  const int ja = sm.rows[gq], jb = sm.rows[gq + 8];
  const int lo_a = ja >= 0 ? (is_window ? p.wlo[ja] : 0) : 0x7fffffff;
  const int lo_b = jb >= 0 ? (is_window ? p.wlo[jb] : 0) : 0x7fffffff;
  float mx_a = -INFINITY, mx_b = -INFINITY;
#pragma unroll
  for (int nt = 0; nt < 4; ++nt)
#pragma unroll
    for (int x = 0; x < 2; ++x) {
      const int pos = sm.pos[key0 + nt * 8 + 2 * tq + x];
      const bool oka = pos >= 0 && pos >= lo_a && ja >= 0;
      const bool okb = pos >= 0 && pos >= lo_b && jb >= 0;
      sacc[nt][x] = oka ? sacc[nt][x] * p.scale_log2 : -INFINITY;
      sacc[nt][2 + x] = okb ? sacc[nt][2 + x] * p.scale_log2 : -INFINITY;
      mx_a = fmaxf(mx_a, sacc[nt][x]);
      mx_b = fmaxf(mx_b, sacc[nt][2 + x]);
    }
  mx_a = fmaxf(mx_a, __shfl_xor_sync(0xffffffffu, mx_a, 1));
  mx_a = fmaxf(mx_a, __shfl_xor_sync(0xffffffffu, mx_a, 2));
  mx_b = fmaxf(mx_b, __shfl_xor_sync(0xffffffffu, mx_b, 1));
  mx_b = fmaxf(mx_b, __shfl_xor_sync(0xffffffffu, mx_b, 2));
  const float base_a = mx_a == -INFINITY ? 0.f : mx_a, base_b = mx_b == -INFINITY ? 0.f : mx_b;
  float l_a = 0.f, l_b = 0.f;
  uint32_t pa[2][4];                          // A fragments of P for the two 16-key steps
#pragma unroll
  for (int nt = 0; nt < 4; ++nt) {
    const float e0 = exp2f(sacc[nt][0] - base_a), e1 = exp2f(sacc[nt][1] - base_a);
    const float e2 = exp2f(sacc[nt][2] - base_b), e3 = exp2f(sacc[nt][3] - base_b);
    l_a += e0 + e1;
    l_b += e2 + e3;
    pa[nt >> 1][(nt & 1) * 2 + 0] = pack2(e0, e1);
    pa[nt >> 1][(nt & 1) * 2 + 1] = pack2(e2, e3);
  }
  l_a += __shfl_xor_sync(0xffffffffu, l_a, 1);
  l_a += __shfl_xor_sync(0xffffffffu, l_a, 2);
  l_b += __shfl_xor_sync(0xffffffffu, l_b, 1);
  l_b += __shfl_xor_sync(0xffffffffu, l_b, 2);
  asm volatile("cp.async.wait_group 0;\n" ::: "memory");
  __syncthreads();
  // O = P V (16 rows x 128 dims)
  float oacc[16][4];
#pragma unroll
  for (int nt = 0; nt < 16; ++nt)
#pragma unroll
    for (int x = 0; x < 4; ++x) oacc[nt][x] = 0.f;
#pragma unroll
  for (int ks = 0; ks < 2; ++ks) {
#pragma unroll
    for (int np = 0; np < 8; ++np) {
      uint32_t bf[4];
      const int m = lane >> 3;
      const int key = key0 + 16 * ks + 8 * (m & 1) + (lane & 7), col = 8 * (2 * np + (m >> 1));
      ldsm_x4_t(bf, su32(&sm.v[key][col]));
      mma16816(oacc[2 * np], pa[ks], bf[0], bf[1]);
      mma16816(oacc[2 * np + 1], pa[ks], bf[2], bf[3]);
    }
  }
  // combine the four warps: stats through shared memory, O rows through the K tile
  if (tq == 0) {
    sm.m[warp][gq] = mx_a; sm.m[warp][gq + 8] = mx_b;
    sm.l[warp][gq] = l_a; sm.l[warp][gq + 8] = l_b;
  }
  __syncthreads();                            // everyone is done with K and V
  float* obuf = reinterpret_cast<float*>(&sm.k[0][0]);   // [4 warps][16 rows][128]
#pragma unroll
  for (int nt = 0; nt < 16; ++nt) {
    const int col = nt * 8 + 2 * tq;
    obuf[(warp * kMaxGroup + gq) * RTP_D + col] = oacc[nt][0];
    obuf[(warp * kMaxGroup + gq) * RTP_D + col + 1] = oacc[nt][1];
    obuf[(warp * kMaxGroup + gq + 8) * RTP_D + col] = oacc[nt][2];
    obuf[(warp * kMaxGroup + gq + 8) * RTP_D + col + 1] = oacc[nt][3];
  }
  __syncthreads();
  const int d = tid;                           // one output column per thread
  for (int r = 0; r < n_rows; ++r) {
    const int j = sm.rows[r];
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < 4; ++w) M = fmaxf(M, sm.m[w][r]);
    float Lsum = 0.f, acc = 0.f;
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      const float mw = sm.m[w][r];
      const float f = mw == -INFINITY ? 0.f : exp2f(mw - M);
      Lsum += f * sm.l[w][r];
      acc += f * obuf[(w * kMaxGroup + r) * RTP_D + d];
    }
    float* part = p.part + (((size_t)b * p.n_heads + j) * p.max_splits + split) * kPartStride;
    part[2 + d] = acc;
    if (d == 0) { part[0] = M; part[1] = Lsum; }
  }
}

__global__ void __launch_bounds__(RTP_D)
decode_attn_merge_kernel(const DecodeParams p) {
  extern __shared__ float wsm[];             // [n_splits] weights
  __shared__ float red[2][4];
  const int j = blockIdx.x, b = blockIdx.y, d = threadIdx.x;
  const int lane = d & 31, warp = d >> 5;
  const float* part = p.part + ((size_t)b * p.n_heads + j) * p.max_splits * kPartStride;
  const bool ret = p.ret_row[j] >= 0;
  const int n_splits = p.n_wc + (ret ? p.n_gc : 0);
  float M = -INFINITY;
  for (int s = d; s < n_splits; s += RTP_D) M = fmaxf(M, part[s * kPartStride]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
  if (lane == 0) red[0][warp] = M;
  __syncthreads();
  M = fmaxf(fmaxf(red[0][0], red[0][1]), fmaxf(red[0][2], red[0][3]));
  float L = 0.f;
  for (int s = d; s < n_splits; s += RTP_D) {
    const float ms = part[s * kPartStride];
    const float w = ms == -INFINITY ? 0.f : exp2f(ms - M);
    wsm[s] = w;
    L += w * part[s * kPartStride + 1];
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) L += __shfl_xor_sync(0xffffffffu, L, o);
  if (lane == 0) red[1][warp] = L;
  __syncthreads();
  L = red[1][0] + red[1][1] + red[1][2] + red[1][3];
  float acc = 0.f;
#pragma unroll 4
  for (int s = 0; s < n_splits; ++s) {
    const float w = wsm[s];
    if (w != 0.f) acc += w * part[s * kPartStride + 2 + d];
  }
  p.o[b * p.o_sb + (int64_t)p.head[j] * p.o_sh + d] = __float2bfloat16_rn(acc / L);
}

namespace {
int n_gathered_chunks(int topk, int sink) { return (topk + sink + kChunk - 1) / kChunk; }
}  // namespace

size_t decode_attn_ws_bytes(int B, int L, int n_heads, int topk, int window) {
  // `window` bounds every head's window; the sink (at most kMaxSink tokens)
  // shares the selected list's chunks.
  const int w = window < L ? window : L;
  const int n_wc = (w + kChunk - 1) / kChunk;
  const int n_gc = topk > 0 ? n_gathered_chunks(topk, kMaxSink) : 0;
  return (size_t)B * n_heads * (n_wc + n_gc) * kPartStride * sizeof(float);
}

cudaError_t launch_decode_hybrid(const void* q, int64_t q_sb, int64_t q_sh,
                                 const void* kc, int64_t k_sb, int64_t k_sn, int64_t k_sh,
                                 const void* vc, int64_t v_sb, int64_t v_sn, int64_t v_sh,
                                 void* o, int64_t o_sb, int64_t o_sh,
                                 int B, int L, int q_pos, int Hq, int Hkv,
                                 const int32_t* ret_heads, int n_ret, const int32_t* idx, int topk,
                                 int ret_window, int sink,
                                 const int32_t* swa_heads, int n_swa, int swa_window,
                                 float scale, void* ws, cudaStream_t stream) {
  DecodeParams p;
  p.q = static_cast<const __nv_bfloat16*>(q); p.q_sb = q_sb; p.q_sh = q_sh;
  p.k = static_cast<const __nv_bfloat16*>(kc); p.k_sb = k_sb; p.k_sn = k_sn; p.k_sh = k_sh;
  p.v = static_cast<const __nv_bfloat16*>(vc); p.v_sb = v_sb; p.v_sn = v_sn; p.v_sh = v_sh;
  p.o = static_cast<__nv_bfloat16*>(o); p.o_sb = o_sb; p.o_sh = o_sh;
  p.B = B; p.L = L; p.q_pos = q_pos; p.Hq = Hq; p.Hkv = Hkv; p.G = Hq / Hkv;
  if (p.G > kMaxGroup) return cudaErrorInvalidValue;
  p.idx = idx; p.topk = n_ret > 0 ? topk : 0; p.sink = sink;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.whi = q_pos + 1 < L ? q_pos + 1 : L;
  p.n_heads = n_ret + n_swa;
  p.n_ret = n_ret;
  int wlo_union = p.whi;
  for (int r = 0; r < n_ret; ++r) {
    p.head[r] = ret_heads[r]; p.ret_row[r] = r; p.ret_list[r] = r;
    p.wlo[r] = q_pos - ret_window + 1 > 0 ? q_pos - ret_window + 1 : 0;
    wlo_union = p.wlo[r] < wlo_union ? p.wlo[r] : wlo_union;
  }
  for (int s = 0; s < n_swa; ++s) {
    const int j = n_ret + s;
    p.head[j] = swa_heads[s]; p.ret_row[j] = -1;
    p.wlo[j] = q_pos - swa_window + 1 > 0 ? q_pos - swa_window + 1 : 0;
    wlo_union = p.wlo[j] < wlo_union ? p.wlo[j] : wlo_union;
  }
  p.wlo_union = wlo_union;
  p.n_wc = (p.whi - wlo_union + kChunk - 1) / kChunk;
  p.n_gc = n_ret > 0 ? n_gathered_chunks(p.topk, sink) : 0;
  p.max_splits = p.n_wc + p.n_gc;
  if (Hkv > kMaxGroup) return cudaErrorInvalidValue;
  p.n_window_items = B * Hkv * p.n_wc;
  p.part = static_cast<float*>(ws);
  const int n_items = p.n_window_items + B * n_ret * p.n_gc;
  const size_t smem = sizeof(Smem);
  cudaError_t e = cudaFuncSetAttribute(decode_attn_partial_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  decode_attn_partial_kernel<<<n_items, kThreads, smem, stream>>>(p);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  dim3 g2(p.n_heads, B);
  const size_t msmem = (size_t)p.max_splits * sizeof(float);
  if (msmem > 48 * 1024) {
    e = cudaFuncSetAttribute(decode_attn_merge_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)msmem);
    if (e != cudaSuccess) return e;
  }
  decode_attn_merge_kernel<<<g2, RTP_D, msmem, stream>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_decode_attn(const void* q, int64_t q_sb, int64_t q_sh,
                               const void* kc, int64_t k_sb, int64_t k_sn, int64_t k_sh,
                               const void* vc, int64_t v_sb, int64_t v_sn, int64_t v_sh,
                               void* o, int64_t o_sb, int64_t o_sh,
                               int B, int L, int q_pos, int Hq, int Hkv,
                               const int32_t* heads, int n_heads, int is_ret,
                               const int32_t* idx, int topk, int window, int sink, float scale,
                               void* ws, cudaStream_t stream) {
  if (is_ret)
    return launch_decode_hybrid(q, q_sb, q_sh, kc, k_sb, k_sn, k_sh, vc, v_sb, v_sn, v_sh, o, o_sb, o_sh, B, L,
                                q_pos, Hq, Hkv, heads, n_heads, idx, topk, window, sink, nullptr, 0, 0, scale, ws,
                                stream);
  return launch_decode_hybrid(q, q_sb, q_sh, kc, k_sb, k_sn, k_sh, vc, v_sb, v_sn, v_sh, o, o_sb, o_sh, B, L,
                              q_pos, Hq, Hkv, nullptr, 0, nullptr, 0, 0, 0, heads, n_heads, window, scale, ws,
                              stream);
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
