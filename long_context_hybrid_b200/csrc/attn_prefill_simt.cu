// Prefill attention over per-query-block key-block lists, fp32 SIMT version.
//
// Streaming heads (RTPurboV2 article: SWA with a local window) walk the
// contiguous band of key blocks that overlaps (pos - W, pos]; retrieval heads
// (RTPurbo digest: exact attention over the small selected set) walk the
// union of their selected key blocks, the sink blocks and the window blocks
// ending at the diagonal block, each block once. Online softmax in the log2
// domain, fp32 accumulation, bf16 output.
//
// This kernel is the portable reference path of the CUDA library: one CTA of
// 256 threads per (sequence, head, 64-query block), tiles in shared memory.
#include "rtp_common.cuh"
#include "rtp_internal.h"
#include "attn_prefill_common.cuh"

namespace rtp {

constexpr int kSimtThreads = 256;
constexpr int kPad = RTP_D + 1;

struct SimtSmem {
  float q[RTP_BLOCK][kPad];
  float k[RTP_BLOCK][kPad];
  float v[RTP_BLOCK][RTP_D];
  float p[RTP_BLOCK][RTP_BLOCK + 1];
  BlockListSmem<kSimtThreads> list;
};

__device__ __forceinline__ void stage_tile(const __nv_bfloat16* base, int64_t sn, int row0, int nrows_valid,
                                           float (*dst)[kPad], float mul) {
  for (int e = threadIdx.x; e < RTP_BLOCK * (RTP_D / 8); e += kSimtThreads) {
    const int r = e / (RTP_D / 8), c8 = (e % (RTP_D / 8)) * 8;
    uint4 w = make_uint4(0, 0, 0, 0);
    if (r < nrows_valid) w = __ldg(reinterpret_cast<const uint4*>(base + (int64_t)(row0 + r) * sn + c8));
    float* d = &dst[r][c8];
    d[0] = bf16_lo(w.x) * mul; d[1] = bf16_hi(w.x) * mul; d[2] = bf16_lo(w.y) * mul; d[3] = bf16_hi(w.y) * mul;
    d[4] = bf16_lo(w.z) * mul; d[5] = bf16_hi(w.z) * mul; d[6] = bf16_lo(w.w) * mul; d[7] = bf16_hi(w.w) * mul;
  }
}

__global__ void __launch_bounds__(kSimtThreads)
prefill_attn_simt_kernel(const PrefillAttnParams p) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  SimtSmem& sm = *reinterpret_cast<SimtSmem*>(smem_raw);
  const int qb = blockIdx.x, j = blockIdx.y, b = blockIdx.z;
  const int h = p.head[j], g = h / p.G;
  const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
  const int pos0 = p.q_pos0 + qb * RTP_BLOCK;

  const int n_list = build_block_list<kSimtThreads>(p, b, j, qb, sm.list, smem_raw + sizeof(SimtSmem));

  const __nv_bfloat16* qbase = static_cast<const __nv_bfloat16*>(p.q.p) + b * p.q.sb + h * p.q.sh;
  const __nv_bfloat16* kbase = static_cast<const __nv_bfloat16*>(p.k.p) + b * p.k.sb + g * p.k.sh;
  const __nv_bfloat16* vbase = static_cast<const __nv_bfloat16*>(p.v.p) + b * p.v.sb + g * p.v.sh;
  stage_tile(qbase, p.q.sn, qb * RTP_BLOCK, RTP_BLOCK, sm.q, p.scale_log2);

  float m[4], l[4], acc[4][8];
#pragma unroll
  for (int ii = 0; ii < 4; ++ii) {
    m[ii] = -INFINITY; l[ii] = 0.f;
#pragma unroll
    for (int cc = 0; cc < 8; ++cc) acc[ii][cc] = 0.f;
  }

  for (int it = 0; it < n_list; ++it) {
    const int kb = list_block(p, sm.list, it, qb);
    const int key0 = kb * RTP_BLOCK;
    const int nvalid = min(RTP_BLOCK, p.Nk - key0);
    __syncthreads();   // previous tiles fully consumed
    stage_tile(kbase, p.k.sn, key0, nvalid, sm.k, 1.f);
    for (int e = tid; e < RTP_BLOCK * (RTP_D / 8); e += kSimtThreads) {
      const int r = e / (RTP_D / 8), c8 = (e % (RTP_D / 8)) * 8;
      uint4 w = make_uint4(0, 0, 0, 0);
      if (r < nvalid) w = __ldg(reinterpret_cast<const uint4*>(vbase + (int64_t)(key0 + r) * p.v.sn + c8));
      float* d = &sm.v[r][c8];
      d[0] = bf16_lo(w.x); d[1] = bf16_hi(w.x); d[2] = bf16_lo(w.y); d[3] = bf16_hi(w.y);
      d[4] = bf16_lo(w.z); d[5] = bf16_hi(w.z); d[6] = bf16_lo(w.w); d[7] = bf16_hi(w.w);
    }
    __syncthreads();
    // S = Q K^T for rows ty+16ii, keys tx+16jj.
    float s[4][4];
#pragma unroll
    for (int ii = 0; ii < 4; ++ii)
#pragma unroll
      for (int jj = 0; jj < 4; ++jj) s[ii][jj] = 0.f;
#pragma unroll 4
    for (int d = 0; d < RTP_D; ++d) {
      float qv[4], kv[4];
#pragma unroll
      for (int ii = 0; ii < 4; ++ii) qv[ii] = sm.q[ty + 16 * ii][d];
#pragma unroll
      for (int jj = 0; jj < 4; ++jj) kv[jj] = sm.k[tx + 16 * jj][d];
#pragma unroll
      for (int ii = 0; ii < 4; ++ii)
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) s[ii][jj] = fmaf(qv[ii], kv[jj], s[ii][jj]);
    }
    // Mask, online softmax.
#pragma unroll
    for (int ii = 0; ii < 4; ++ii) {
      const int pos = pos0 + ty + 16 * ii;
      float rmax = -INFINITY;
#pragma unroll
      for (int jj = 0; jj < 4; ++jj) {
        const int u = key0 + tx + 16 * jj;
        const bool ok = (u < p.Nk) && key_allowed(p, u, pos);
        s[ii][jj] = ok ? s[ii][jj] : -INFINITY;
        rmax = fmaxf(rmax, s[ii][jj]);
      }
#pragma unroll
      for (int o = 8; o > 0; o >>= 1) rmax = fmaxf(rmax, __shfl_xor_sync(0xffffffffu, rmax, o));
      const float mn = fmaxf(m[ii], rmax);
      const float base = (mn == -INFINITY) ? 0.f : mn;
      const float corr = exp2f(m[ii] - base);
      float rsum = 0.f;
#pragma unroll
      for (int jj = 0; jj < 4; ++jj) {
        const float pe = exp2f(s[ii][jj] - base);
        sm.p[ty + 16 * ii][tx + 16 * jj] = pe;
        rsum += pe;
      }
#pragma unroll
      for (int o = 8; o > 0; o >>= 1) rsum += __shfl_xor_sync(0xffffffffu, rsum, o);
      l[ii] = l[ii] * corr + rsum;
      m[ii] = mn;
#pragma unroll
      for (int cc = 0; cc < 8; ++cc) acc[ii][cc] *= corr;
    }
    __syncthreads();
    // O += P V for rows ty+16ii, columns tx+16cc.
#pragma unroll 4
    for (int kk = 0; kk < RTP_BLOCK; ++kk) {
      float pv[4], vv[8];
#pragma unroll
      for (int ii = 0; ii < 4; ++ii) pv[ii] = sm.p[ty + 16 * ii][kk];
#pragma unroll
      for (int cc = 0; cc < 8; ++cc) vv[cc] = sm.v[kk][tx + 16 * cc];
#pragma unroll
      for (int ii = 0; ii < 4; ++ii)
#pragma unroll
        for (int cc = 0; cc < 8; ++cc) acc[ii][cc] = fmaf(pv[ii], vv[cc], acc[ii][cc]);
    }
  }
  __nv_bfloat16* obase = static_cast<__nv_bfloat16*>(p.o) + b * p.o_sb + h * p.o_sh;
#pragma unroll
  for (int ii = 0; ii < 4; ++ii) {
    const int r = qb * RTP_BLOCK + ty + 16 * ii;
    const float inv = 1.f / l[ii];
#pragma unroll
    for (int cc = 0; cc < 8; ++cc)
      obase[(int64_t)r * p.o_sn + tx + 16 * cc] = __float2bfloat16_rn(acc[ii][cc] * inv);
  }
}

cudaError_t launch_prefill_attn_simt(const PrefillAttnParams& p, int n_qblocks, int B,
                                     cudaStream_t stream) {
  const size_t smem = sizeof(SimtSmem) + block_list_bytes(p);
  cudaError_t e = cudaFuncSetAttribute(prefill_attn_simt_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid(n_qblocks, p.n_heads, B);
  prefill_attn_simt_kernel<<<grid, kSimtThreads, smem, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace rtp
