// Prefill block selection on the 5th-generation tensor cores.
//
// Block score (the tiny 2K prefill workload statement): for query block i and
// key block j <= i, the max of q~_t . k~_u over the causal pairs of the two
// 64-token blocks; each query block keeps its top-k key blocks (RTPurbo digest:
// the 16-d indexer picks the candidates). The token score matrix never leaves
// the SM: every 128 x 256 score tile lives in TMEM only until its block maxima
// are taken.
//
// One CTA handles query blocks 2t and 2t+1 (128 query rows) of one retrieval
// head, longest key ranges first. Warp roles (384 threads):
//   warp 0       TMA: the 128 x 16 query-index tile once, then 256 x 16
//                key-index tiles (4 key blocks) into a 4-stage ring (32-byte
//                swizzle);
//   warp 1       TMEM owner and MMA issuer: one tcgen05.mma M=128 N=256 K=16
//                per key tile into one of two TMEM score buffers;
//   warps 4..11  two epilogue warpgroups, one per score buffer: thread r reads
//                row r of the tile, takes the causal max of each 64-column
//                block (3-input max), reduces over the 32 rows of its warp
//                (redux.sync), and folds the result into the block-score array
//                of its query block with a shared-memory atomic max on
//                order-preserving integer keys.
// Finally all threads run the exact radix top-k of each of the two block-score
// arrays (ties to the smaller block) and write ascending lists.
#include "rtp_common.cuh"
#include "rtp_internal.h"
#include "sm100.cuh"

namespace rtp {
using namespace sm100;

namespace {

constexpr int kThreads = 384;
constexpr int kKStages = 4;
constexpr int kChunkKeys = 256;                    // 4 key blocks per MMA
constexpr uint32_t kQOff = 0;                      // 128 rows x 32 B
constexpr uint32_t kKOff = 4096;                   // stage s at +s*8192 (256 rows x 32 B)
constexpr uint32_t kScoreOff = kKOff + kKStages * 8192u;
constexpr int kStatusTimeout = 4;

struct SelBars {
  uint64_t q_full;
  uint64_t k_full[kKStages], k_empty[kKStages];
  uint64_t s_full[2], s_free[2];
  uint64_t fin;
  uint32_t tmem_base;
  int abort;
  TopkSmem<kThreads> topk;
};

__device__ __forceinline__ float max3f(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}
__device__ __forceinline__ float warp_max(float v) {
  float r;
  asm volatile("redux.sync.max.f32 %0, %1, 0xffffffff;" : "=f"(r) : "f"(v));
  return r;
}
__device__ __forceinline__ uint64_t desc_sw32(uint32_t saddr) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
  d |= (uint64_t)1 << 16;             // leading offset (unused for K-major swizzled)
  d |= (uint64_t)(256 >> 4) << 32;    // 8-row groups 256 B apart
  d |= (uint64_t)1 << 46;             // sm_100 descriptor version
  d |= (uint64_t)6 << 61;             // 32-byte swizzle
  return d;
}
__device__ __forceinline__ bool wait_short(uint32_t bar, uint32_t parity) {
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, parity))
    if (clock64() - t0 > 200000000LL) return false;
  return true;
}

}  // namespace

struct SelectTcParams {
  int N, Hr, Hkv, topk, nb;
  int32_t* blocks;
  int32_t* counts;
  int kv[kMaxHeads];
};

__global__ void __launch_bounds__(kThreads, 1)
prefill_select_tc_kernel(const SelectTcParams p, const __grid_constant__ CUtensorMap tmQ,
                         const __grid_constant__ CUtensorMap tmK, int* status) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const uint32_t sb = smem_u32(smem);
  const int n_tiles = (p.nb + 1) / 2;
  const int t = n_tiles - 1 - blockIdx.x;
  const int j = blockIdx.y, b = blockIdx.z, g = p.kv[j];
  const int qa = 2 * t, qb = 2 * t + 1;
  const bool has_b = qb < p.nb;
  const int last_blk = has_b ? qb : qa;
  const int n_chunks = (last_blk + 1 + 3) / 4;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  uint32_t* sA = reinterpret_cast<uint32_t*>(smem + kScoreOff);
  uint32_t* sB = sA + p.nb;
  SelBars& bars = *reinterpret_cast<SelBars*>(smem + kScoreOff + (size_t)p.nb * 8);
  volatile int* abort_flag = &bars.abort;

  for (int x = tid; x <= last_blk; x += kThreads) { sA[x] = 0u; sB[x] = 0u; }
  if (tid == 0) {
    mbar_init(smem_u32(&bars.q_full), 1);
    for (int s = 0; s < kKStages; ++s) {
      mbar_init(smem_u32(&bars.k_full[s]), 1);
      mbar_init(smem_u32(&bars.k_empty[s]), 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(smem_u32(&bars.s_full[s]), 1);
      mbar_init(smem_u32(&bars.s_free[s]), 128);
    }
    mbar_init(smem_u32(&bars.fin), 1);
    bars.abort = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(&bars.tmem_base), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars.tmem_base;

  if (warp == 0) {
    if (lane == 0) {
      tma_prefetch(&tmQ);
      tma_prefetch(&tmK);
      const uint32_t qbar = smem_u32(&bars.q_full);
      mbar_arrive_expect_tx(qbar, 4096);
      tma_load_4d(sb + kQOff, &tmQ, qbar, 0, qa * RTP_BLOCK, j, b);
      int issued = 0;
      for (int c = 0; c < n_chunks; ++c) {
        const int s = c % kKStages;
        if (c >= kKStages && !mbar_wait(smem_u32(&bars.k_empty[s]), ((c / kKStages) - 1) & 1, abort_flag)) break;
        const uint32_t kbar = smem_u32(&bars.k_full[s]);
        mbar_arrive_expect_tx(kbar, 8192);
        tma_load_4d(sb + kKOff + s * 8192u, &tmK, kbar, 0, c * kChunkKeys, g, b);
        issued = c + 1;
      }
      if (*abort_flag) {
        wait_short(qbar, 0);
        for (int c = max(0, issued - kKStages); c < issued; ++c)
          wait_short(smem_u32(&bars.k_full[c % kKStages]), (c / kKStages) & 1);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(128, 256, false, false);
      bool ok = mbar_wait(smem_u32(&bars.q_full), 0, abort_flag);
      const uint64_t qdesc = desc_sw32(sb + kQOff);
      for (int c = 0; ok && c < n_chunks; ++c) {
        const int s = c % kKStages, buf = c & 1;
        if (!mbar_wait(smem_u32(&bars.k_full[s]), (c / kKStages) & 1, abort_flag)) break;
        if (c >= 2 && !mbar_wait(smem_u32(&bars.s_free[buf]), ((c >> 1) - 1) & 1, abort_flag)) break;
        tc_fence_after();
        mma_bf16_ss(tmem + buf * 256u, qdesc, desc_sw32(sb + kKOff + s * 8192u), idesc, 0u);
        mma_commit(smem_u32(&bars.s_full[buf]));
        mma_commit(smem_u32(&bars.k_empty[s]));
      }
      mma_commit(smem_u32(&bars.fin));
      wait_short(smem_u32(&bars.fin), 0);
    }
    __syncwarp();
  } else if (warp >= 4) {
    const int wg = (warp - 4) >> 2;                 // 0 or 1: which score buffer
    const int r = tid - 128 - wg * 128;             // row 0..127 of the tile
    const uint32_t lane_base = tmem + ((uint32_t)((warp & 3) * 32) << 16) + wg * 256u;
    const bool in_a = r < 64;
    const int my_last = in_a ? qa : last_blk;       // key blocks this row's query block may see
    const int rq = in_a ? r : r - 64;               // row within its query block
    const int my_q = in_a ? qa : qb;
    uint32_t* dst = in_a ? sA : sB;
    for (int c = wg; c < n_chunks; c += 2) {
      bool w = mbar_wait(smem_u32(&bars.s_full[wg]), (c >> 1) & 1, abort_flag);
      if (!__all_sync(0xffffffffu, w)) break;
      tc_fence_after();
#pragma unroll
      for (int bi = 0; bi < 4; ++bi) {
        const int kb = c * 4 + bi;
        if (kb > last_blk) break;                   // warp-uniform: same for the whole CTA
        uint32_t v[64];
        tmem_ld32(lane_base + bi * 64u, v);
        tmem_ld32(lane_base + bi * 64u + 32u, v + 32);
        tc_wait_ld();
        float m = -INFINITY;
        if (kb < my_q) {
          // 64 -> 1 in a tree of 3-input maxima (32 instructions, depth 4)
          float a[22], c[8];
#pragma unroll
          for (int x = 0; x < 21; ++x)
            a[x] = max3f(__uint_as_float(v[3 * x]), __uint_as_float(v[3 * x + 1]), __uint_as_float(v[3 * x + 2]));
          a[21] = __uint_as_float(v[63]);
#pragma unroll
          for (int x = 0; x < 7; ++x) c[x] = max3f(a[3 * x], a[3 * x + 1], a[3 * x + 2]);
          c[7] = a[21];
          m = max3f(max3f(c[0], c[1], c[2]), max3f(c[3], c[4], c[5]), fmaxf(c[6], c[7]));
        } else if (kb == my_q) {
          // diagonal block: key column x is causal for this row iff x <= rq
#pragma unroll
          for (int x = 0; x < 64; ++x)
            if (x <= rq) m = fmaxf(m, __uint_as_float(v[x]));
        }
        if (!has_b && !in_a) m = -INFINITY;         // rows of a query block past the end
        const float wm = warp_max(m);
        if (lane == 0 && kb <= my_last && wm != -INFINITY) atomicMax(&dst[kb], f2key(wm));
      }
      tc_fence_before();
      mbar_arrive(smem_u32(&bars.s_free[wg]));
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
  if (bars.abort) {
    if (tid == 0) atomicExch(status, kStatusTimeout);
    return;
  }
  // Top-k per query block (exact, ties to the smaller block), ascending output.
  const size_t rowA = ((size_t)b * p.Hr + j) * p.nb + qa;
  {
    auto keyA = [sA](int x) { return sA[x]; };
    block_topk_ascending<kThreads>(keyA, qa + 1, p.topk, p.blocks + rowA * p.topk, bars.topk);
    if (tid == 0) p.counts[rowA] = min(p.topk, qa + 1);
  }
  __syncthreads();
  if (has_b) {
    auto keyB = [sB](int x) { return sB[x]; };
    block_topk_ascending<kThreads>(keyB, qb + 1, p.topk, p.blocks + (rowA + 1) * p.topk, bars.topk);
    if (tid == 0) p.counts[rowA + 1] = min(p.topk, qb + 1);
  }
}

size_t select_prefill_tc_smem(int nb) {
  return 1024 + kScoreOff + (size_t)nb * 8 + sizeof(SelBars);
}

cudaError_t launch_select_prefill_tc(const void* qt, const void* kt, int B, int N, int Hr, int Hkv,
                                     const int32_t* kv_of, int topk, int32_t* blocks, int32_t* counts,
                                     int* status, cudaStream_t stream) {
  SelectTcParams p;
  p.N = N; p.Hr = Hr; p.Hkv = Hkv; p.topk = topk; p.nb = N / RTP_BLOCK;
  p.blocks = blocks; p.counts = counts;
  for (int j = 0; j < Hr; ++j) p.kv[j] = kv_of[j];
  CUtensorMap tq, tk;
  if (!make_tmap_index(&tq, qt, B, Hr, N, 128) || !make_tmap_index(&tk, kt, B, Hkv, N, kChunkKeys))
    return cudaErrorInvalidValue;
  const size_t smem = select_prefill_tc_smem(p.nb);
  if (smem > 227 * 1024) return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(prefill_select_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  e = cudaMemsetAsync(status, 0, sizeof(int), stream);
  if (e != cudaSuccess) return e;
  dim3 grid((p.nb + 1) / 2, Hr, B);
  prefill_select_tc_kernel<<<grid, kThreads, smem, stream>>>(p, tq, tk, status);
  return cudaGetLastError();
}

size_t select_prefill_ws_bytes(int B, int N, int Hr, int topk) { (void)B; (void)N; (void)Hr; (void)topk; return kStatusBytes; }
cudaError_t launch_select_prefill(const void* qt, const void* kt, int B, int N, int Hr, int Hkv,
                                  const int32_t* kv_of, int topk, int32_t* blocks, int32_t* counts, void* ws,
                                  cudaStream_t stream) {
  return launch_select_prefill_tc(qt, kt, B, N, Hr, Hkv, kv_of, topk, blocks, counts, static_cast<int*>(ws), stream);
}
}  // namespace rtp
