// The 8-bit key index: symmetric int8 codes with one fp32 scale per group of
// 64 consecutive tokens of one KV head (the Baidu article on layered
// long-context attention, section on the mixed-precision index system: an
// 8-bit quantised indexer; the plain symmetric per-group scheme is the reading
// taken where the page fixes none). Per group: amax = max |x| over its
// 64 x 16 bf16 values, s = amax / 127 and code = round-half-even(x / s)
// clamped to [-127, 127], both divisions IEEE fp32 (__fdiv_rn), so that every
// code is the one a plain fp32 implementation of the same definition gives;
// an all-zero group gets s = 0 and zero codes.
//
// One warp per group: lane l holds tokens 2l and 2l+1 (two 32-byte rows, four
// 16-byte loads), the warp reduces amax with shuffles, and each lane stores
// its two 16-byte code rows; lane 0 stores the scale. HBM-bound: 2 KB in and
// 1 KB + 4 B out per group.
#include "rtp_common.cuh"
#include "rtp_internal.h"

namespace rtp {

namespace {
constexpr int kQWarps = 8;

__device__ __forceinline__ uint32_t code_of(float x, float s) {
  int c = __float2int_rn(__fdiv_rn(x, s));
  c = c > 127 ? 127 : (c < -127 ? -127 : c);
  return (uint32_t)(c & 0xff);
}
}  // namespace

__global__ void __launch_bounds__(kQWarps * 32)
index_quantize_kernel(const uint4* __restrict__ kindex, int64_t cap, int n_bh, int g0, int n_groups, int64_t ng,
                      uint4* __restrict__ k8, float* __restrict__ kscale) {
  const int lane = threadIdx.x & 31;
  const int64_t item = (int64_t)blockIdx.x * kQWarps + (threadIdx.x >> 5);
  if (item >= (int64_t)n_bh * n_groups) return;
  const int bh = (int)(item / n_groups);
  const int grp = g0 + (int)(item - (int64_t)bh * n_groups);
  const int64_t tok0 = (int64_t)grp * QGROUP_TOKENS + 2 * lane;
  const uint4* src = kindex + ((int64_t)bh * cap + tok0) * 2;
  uint4 w[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) w[i] = __ldcs(src + i);
  float x[32];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint32_t v[4] = {w[i].x, w[i].y, w[i].z, w[i].w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      x[8 * i + 2 * e] = bf16_lo(v[e]);
      x[8 * i + 2 * e + 1] = bf16_hi(v[e]);
    }
  }
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < 32; ++i) amax = fmaxf(amax, fabsf(x[i]));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  const float s = amax > 0.f ? __fdiv_rn(amax, 127.f) : 0.f;
  uint4 out[2];
#pragma unroll
  for (int t = 0; t < 2; ++t) {
    uint32_t word[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      uint32_t wv = 0;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float xv = x[16 * t + 4 * q + e];
        wv |= (s > 0.f ? code_of(xv, s) : 0u) << (8 * e);
      }
      word[q] = wv;
    }
    out[t] = make_uint4(word[0], word[1], word[2], word[3]);
  }
  uint4* dst = k8 + (int64_t)bh * cap + tok0;
  dst[0] = out[0];
  dst[1] = out[1];
  if (lane == 0) kscale[(int64_t)bh * ng + grp] = s;
}

cudaError_t launch_index_quantize(const void* kindex, int64_t cap, int B, int Hkv, int g0, int g1, void* kindex8,
                                  float* kscale, cudaStream_t stream) {
  const int n_bh = B * Hkv, n_groups = g1 - g0;
  if (n_groups <= 0) return cudaSuccess;
  const int64_t items = (int64_t)n_bh * n_groups;
  const int64_t grid = (items + kQWarps - 1) / kQWarps;
  if (grid > 0x7fffffff) return cudaErrorInvalidValue;
  const int64_t ng = (cap + QGROUP_TOKENS - 1) / QGROUP_TOKENS;
  index_quantize_kernel<<<(int)grid, kQWarps * 32, 0, stream>>>(static_cast<const uint4*>(kindex), cap, n_bh, g0,
                                                                 n_groups, ng, static_cast<uint4*>(kindex8), kscale);
  return cudaGetLastError();
}

}  // namespace rtp
