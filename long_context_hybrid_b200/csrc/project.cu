// Index projection x~ = x . P (D = 128 -> r = 16), the low-rank indexer of
// the RTPurboV2 article (paragraph on the low-rank projector).
//
// Up to 64 rows per (sequence, head) take a small shared-memory kernel (the
// decode step's queries); longer sequences the tensor-core kernel below.
//
// The work is HBM-bound: 256 bytes of x per row in, 32 (bf16) or 64 (fp32)
// bytes out, 2048 multiply-adds per row. One warp computes 16 rows x 16
// outputs with bf16 mma.sync (m16n8k16, fp32 accumulation): the K dimension
// is permuted identically in A and B so that every thread fetches its rows
// with plain 16-byte loads straight into fragment registers, and the
// projector's fragments stay in registers for the whole CTA.
#include "rtp_common.cuh"
#include "rtp_internal.h"

namespace rtp {

// Column of x (0..127) that fragment slot s (0..15) of k-chunk kk holds.
// Thread t of a quad loads 8 consecutive columns 32*(kk/2) + 8t .. +8 with one
// 16-byte load; chunk kk (parity h) uses 4 of them: slots (2t, 2t+1) take
// columns +4h+0/+1 and slots (2t+8, 2t+9) take +4h+2/+3.
__device__ __forceinline__ int slot_col(int kk, int s) {
  int t = (s & 7) >> 1, e = s & 1, hi = s >> 3;
  return 32 * (kk >> 1) + 8 * t + 4 * (kk & 1) + 2 * hi + e;
}

__device__ __forceinline__ uint32_t pack_bf16(__nv_bfloat16 lo, __nv_bfloat16 hi) {
  return (uint32_t)__bfloat16_as_ushort(lo) | ((uint32_t)__bfloat16_as_ushort(hi) << 16);
}

__device__ __forceinline__ void mma_bf16_16816(float* c, const uint32_t* a, const uint32_t* b) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
      "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};\n"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}

struct ProjectParams {
  const __nv_bfloat16* x;
  int64_t sb, sn, sh;
  int B, N;
  const __nv_bfloat16* P;   // [Hp, 128, 16]
  void* out;                // [B, out_nh, out_cap, 16]: row r of listed head j -> [b, out_slot[j], out_pos0 + r]
  int out_f32;
  int n_heads;
  int out_nh;               // heads of the output tensor
  int64_t out_cap;          // rows per (sequence, head) of the output tensor
  int out_pos0;             // first output row
  int head[kMaxHeads];
  int proj[kMaxHeads];
  int out_slot[kMaxHeads];
};

constexpr int kProjWarps = 4;
constexpr int kProjRowsPerWarp = 16;

__global__ void __launch_bounds__(kProjWarps * 32)
project_kernel(const ProjectParams p) {
  const int j = blockIdx.z;               // listed head
  const int b = blockIdx.y;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int g = lane >> 2, t = lane & 3;
  const __nv_bfloat16* P = p.P + (size_t)p.proj[j] * RTP_D * RTP_R;

  // B fragments of the projector: 8 k-chunks x 2 n-tiles x 2 registers.
  uint32_t bfrag[8][2][2];
#pragma unroll
  for (int kk = 0; kk < 8; ++kk)
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
      int n = nt * 8 + g;
      bfrag[kk][nt][0] = pack_bf16(P[slot_col(kk, 2 * t) * RTP_R + n], P[slot_col(kk, 2 * t + 1) * RTP_R + n]);
      bfrag[kk][nt][1] = pack_bf16(P[slot_col(kk, 2 * t + 8) * RTP_R + n], P[slot_col(kk, 2 * t + 9) * RTP_R + n]);
    }

  const __nv_bfloat16* xb = p.x + (size_t)b * p.sb + (size_t)p.head[j] * p.sh;
  const int rows_per_cta = kProjWarps * kProjRowsPerWarp;
  for (int r0 = blockIdx.x * rows_per_cta + warp * kProjRowsPerWarp; r0 < p.N;
       r0 += gridDim.x * rows_per_cta) {
    const int ra = r0 + g, rb = r0 + g + 8;
    uint4 va[4], vb[4];
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      va[c] = ra < p.N ? __ldg(reinterpret_cast<const uint4*>(xb + (size_t)ra * p.sn + 32 * c + 8 * t))
                       : make_uint4(0, 0, 0, 0);
      vb[c] = rb < p.N ? __ldg(reinterpret_cast<const uint4*>(xb + (size_t)rb * p.sn + 32 * c + 8 * t))
                       : make_uint4(0, 0, 0, 0);
    }
    float acc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {
      const uint4 A = va[kk >> 1], Bv = vb[kk >> 1];
      uint32_t a[4];
      // a0: row g, slots 2t/2t+1; a1: row g+8, same slots; a2/a3: slots 2t+8/2t+9.
      a[0] = (kk & 1) ? A.z : A.x;
      a[1] = (kk & 1) ? Bv.z : Bv.x;
      a[2] = (kk & 1) ? A.w : A.y;
      a[3] = (kk & 1) ? Bv.w : Bv.y;
      mma_bf16_16816(acc[0], a, bfrag[kk][0]);
      mma_bf16_16816(acc[1], a, bfrag[kk][1]);
    }
    // D fragment: (row g, cols 2t, 2t+1) and (row g+8, same cols) per n-tile.
    const size_t obase = ((size_t)b * p.out_nh + p.out_slot[j]) * (size_t)p.out_cap + p.out_pos0;
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
      const int col = nt * 8 + 2 * t;
      if (p.out_f32) {
        float* o = reinterpret_cast<float*>(p.out);
        if (ra < p.N) *reinterpret_cast<float2*>(o + (obase + ra) * RTP_R + col) = make_float2(acc[nt][0], acc[nt][1]);
        if (rb < p.N) *reinterpret_cast<float2*>(o + (obase + rb) * RTP_R + col) = make_float2(acc[nt][2], acc[nt][3]);
      } else {
        __nv_bfloat16* o = reinterpret_cast<__nv_bfloat16*>(p.out);
        if (ra < p.N) *reinterpret_cast<__nv_bfloat162*>(o + (obase + ra) * RTP_R + col) = __floats2bfloat162_rn(acc[nt][0], acc[nt][1]);
        if (rb < p.N) *reinterpret_cast<__nv_bfloat162*>(o + (obase + rb) * RTP_R + col) = __floats2bfloat162_rn(acc[nt][2], acc[nt][3]);
      }
    }
  }
}

// Few rows (a decode step's queries): one CTA per (sequence, listed head)
// stages the projector and the rows in shared memory with coalesced loads;
// thread (row, c) forms one output with an fp32 dot product of length 128.
constexpr int kSmallRows = 64;

__global__ void __launch_bounds__(256)
project_small_kernel(const ProjectParams p) {
  __shared__ float Ps[RTP_D][RTP_R];
  __shared__ float xs[kSmallRows][RTP_D + 1];
  const int j = blockIdx.x, b = blockIdx.y;
  const __nv_bfloat16* P = p.P + (size_t)p.proj[j] * RTP_D * RTP_R;
  for (int e = threadIdx.x; e < RTP_D * RTP_R; e += blockDim.x) Ps[e / RTP_R][e % RTP_R] = __bfloat162float(P[e]);
  const __nv_bfloat16* xb = p.x + (size_t)b * p.sb + (size_t)p.head[j] * p.sh;
  for (int e = threadIdx.x; e < p.N * RTP_D; e += blockDim.x)
    xs[e / RTP_D][e % RTP_D] = __bfloat162float(xb[(size_t)(e / RTP_D) * p.sn + e % RTP_D]);
  __syncthreads();
  const size_t obase = ((size_t)b * p.out_nh + p.out_slot[j]) * (size_t)p.out_cap + p.out_pos0;
  for (int e = threadIdx.x; e < p.N * RTP_R; e += blockDim.x) {
    const int row = e / RTP_R, c = e % RTP_R;
    float acc = 0.f;
#pragma unroll 8
    for (int d = 0; d < RTP_D; ++d) acc = fmaf(xs[row][d], Ps[d][c], acc);
    if (p.out_f32) reinterpret_cast<float*>(p.out)[(obase + row) * RTP_R + c] = acc;
    else reinterpret_cast<__nv_bfloat16*>(p.out)[(obase + row) * RTP_R + c] = __float2bfloat16_rn(acc);
  }
}

static cudaError_t launch_project_params(ProjectParams& p, cudaStream_t stream) {
  const int N = p.N, B = p.B, n_heads = p.n_heads;
  if (N <= kSmallRows) {
    dim3 grid(n_heads, B);
    project_small_kernel<<<grid, 256, 0, stream>>>(p);
    return cudaGetLastError();
  }
  const int rows_per_cta = kProjWarps * kProjRowsPerWarp;
  int gx = (N + rows_per_cta - 1) / rows_per_cta;
  // Enough CTAs to fill the GPU a few times; each loops over row tiles.
  const int max_gx = 148 * 16 / (n_heads * B) + 1;
  if (gx > max_gx) gx = max_gx;
  dim3 grid(gx, B, n_heads);
  project_kernel<<<grid, kProjWarps * 32, 0, stream>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_project(const void* x, int64_t sb, int64_t sn, int64_t sh, int B, int N,
                           const void* P, const int32_t* heads, const int32_t* proj, int n_heads,
                           void* out, int out_f32, cudaStream_t stream) {
  ProjectParams p;
  p.x = static_cast<const __nv_bfloat16*>(x);
  p.sb = sb; p.sn = sn; p.sh = sh; p.B = B; p.N = N;
  p.P = static_cast<const __nv_bfloat16*>(P);
  p.out = out; p.out_f32 = out_f32; p.n_heads = n_heads;
  p.out_nh = n_heads; p.out_cap = N; p.out_pos0 = 0;
  for (int i = 0; i < n_heads; ++i) { p.head[i] = heads[i]; p.proj[i] = proj[i]; p.out_slot[i] = i; }
  return launch_project_params(p, stream);
}

cudaError_t launch_index_append(const void* k, int64_t sb, int64_t sn, int64_t sh, int B, int n_new, int Hkv,
                                const void* P, void* kindex, int64_t cap, int pos, cudaStream_t stream) {
  ProjectParams p;
  p.x = static_cast<const __nv_bfloat16*>(k);
  p.sb = sb; p.sn = sn; p.sh = sh; p.B = B; p.N = n_new;
  p.P = static_cast<const __nv_bfloat16*>(P);
  p.out = kindex; p.out_f32 = 0; p.n_heads = Hkv;
  p.out_nh = Hkv; p.out_cap = cap; p.out_pos0 = pos;
  for (int g = 0; g < Hkv; ++g) { p.head[g] = g; p.proj[g] = g; p.out_slot[g] = g; }
  return launch_project_params(p, stream);
}

}  // namespace rtp
