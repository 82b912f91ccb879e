// Prefill attention on the 5th-generation tensor cores (tcgen05 + TMEM + TMA).
//
// One CTA computes 128 query rows of one head against a list of 64-key blocks:
//   * streaming heads (RTPurboV2 article: SWA with a local window): the band of
//     key blocks overlapping (pos - W, pos] for the 128 rows, with a per-element
//     window/causal mask;
//   * retrieval heads (RTPurbo digest: exact attention at full dimension over
//     the indexer-selected set): the rows are query blocks 2t and 2t+1, and the
//     list is the union of their attended sets (selected blocks, sink blocks,
//     window blocks); every entry carries which of the two halves attends it,
//     so a row only ever sees its own block's set, with the causal mask.
//
// Warp roles (256 threads):
//   warp 0      TMA producer: Q once, then K/V tiles of two list blocks per
//               step into a 2-stage ring (128-byte swizzle);
//   warp 1      TMEM owner and single-thread MMA issuer:
//               S_j = Q K_j^T (M=128, N=128, K=128) into one of two TMEM S
//               buffers, then O += P_{j-1} V_{j-1} (V read MN-major);
//   warps 4..7  softmax: thread r owns query row r (TMEM lane r); reads S_j,
//               masks, online softmax in the log2 domain with lazy rescaling
//               (O in TMEM is rescaled only when the running max grows by
//               more than 2^8), writes P_j (bf16) into swizzled shared memory
//               for the next MMA, and finally normalises O and stores it.
// Every wait is bounded; a wait that runs out marks the CTA aborted, all
// roles drain, TMEM is freed and RTP_ERR_TIMEOUT is written to `status`.
#include "attn_prefill_common.cuh"
#include "rtp_common.cuh"
#include "rtp_internal.h"
#include "sm100.cuh"

namespace rtp {
using namespace sm100;

namespace {

constexpr int kThreads = 256;
constexpr int kStages = 2;
constexpr uint32_t kQOff = 0;                                 // [D half][128 rows][128 B] = 32 KB
constexpr uint32_t kKVOff = 32768;                            // stage s: K at s*64K, V at s*64K + 32K
constexpr uint32_t kPOff = kKVOff + kStages * 65536u;         // [key half][128 rows][128 B] = 32 KB
constexpr uint32_t kListOff = kPOff + 32768u;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kOCol = 256;                               // O accumulator columns [256, 384)
constexpr int kStatusTimeout = 4;                             // RTP_ERR_TIMEOUT

struct Bars {
  uint64_t q_full;
  uint64_t k_full[kStages], v_full[kStages], kv_empty[kStages];
  uint64_t s_full[2], s_free[2];
  uint64_t p_full, pv_done, fin;
  uint32_t tmem_base;
  int abort;
  int n_list;
  int kb_lo;
  BlockScanSmem<kThreads> scan;
};

// Marks the attended key blocks of query block q in `bits`.
__device__ void mark_blocks(const PrefillAttnParams& p, int b, int jh, int q, unsigned* bits) {
  const int nb = p.Nq / RTP_BLOCK;
  const size_t row = ((size_t)b * p.n_heads + jh) * nb + q;
  const int cnt = min(p.counts[row], p.topk);
  const int32_t* sel = p.blocks + row * p.topk;
  for (int e = threadIdx.x; e < cnt; e += kThreads) {
    const int x = sel[e];
    if (x >= 0 && x <= q) atomicOr(&bits[x >> 5], 1u << (x & 31));
  }
  for (int x = threadIdx.x; x < min(p.sink_blocks, q + 1); x += kThreads) atomicOr(&bits[x >> 5], 1u << (x & 31));
  for (int x = max(0, q - p.window_blocks + 1) + threadIdx.x; x <= q; x += kThreads)
    atomicOr(&bits[x >> 5], 1u << (x & 31));
}

// Union list of query blocks 2t and 2t+1: entries (block, membership bits).
__device__ int build_pair_list(const PrefillAttnParams& p, int b, int jh, int tile, unsigned* bitsA,
                               unsigned* bitsB, int2* list, BlockScanSmem<kThreads>& scan) {
  const int nb = p.Nq / RTP_BLOCK;
  const int qa = 2 * tile, qb = 2 * tile + 1;
  const bool has_b = qb < nb;
  const int qmax = has_b ? qb : qa;
  const int nw = qmax / 32 + 1;
  for (int w = threadIdx.x; w < nw; w += kThreads) { bitsA[w] = 0u; bitsB[w] = 0u; }
  __syncthreads();
  mark_blocks(p, b, jh, qa, bitsA);
  if (has_b) mark_blocks(p, b, jh, qb, bitsB);
  __syncthreads();
  const int per = (nw + kThreads - 1) / kThreads;
  const int w0 = threadIdx.x * per, w1 = min(nw, w0 + per);
  int c = 0;
  for (int w = w0; w < w1; ++w) c += __popc(bitsA[w] | bitsB[w]);
  int total;
  int off = block_exclusive_scan<kThreads>(c, total, scan);
  for (int w = w0; w < w1; ++w) {
    const unsigned a = bitsA[w], bb = bitsB[w];
    unsigned x = a | bb;
    while (x) {
      const int bit = __ffs(x) - 1;
      x &= x - 1;
      list[off++] = make_int2(w * 32 + bit, (int)(((a >> bit) & 1u) | (((bb >> bit) & 1u) << 1)));
    }
  }
  __syncthreads();
  return total;
}

__device__ __forceinline__ bool wait_short(uint32_t bar, uint32_t parity) {
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, parity))
    if (clock64() - t0 > 200000000LL) return false;
  return true;
}

}  // namespace

__global__ void __launch_bounds__(kThreads, 1)
prefill_attn_tc_kernel(const PrefillAttnParams p, const __grid_constant__ CUtensorMap tmQ,
                       const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                       int* status) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const uint32_t sb = smem_u32(smem);
  const int tile = blockIdx.x, jh = blockIdx.y, b = blockIdx.z;
  const int h = p.head[jh], g = h / p.G;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  int2* list = reinterpret_cast<int2*>(smem + kListOff);
  Bars& bars = *reinterpret_cast<Bars*>(smem + kListOff + (size_t)p.list_cap * sizeof(int2));
  volatile int* abort_flag = &bars.abort;

  // ---- prologue: key-block list, barriers, TMEM
  int n_list;
  if (p.sparse) {
    unsigned* bitsA = reinterpret_cast<unsigned*>(smem + kPOff);
    unsigned* bitsB = bitsA + 4096;
    n_list = build_pair_list(p, b, jh, tile, bitsA, bitsB, list, bars.scan);
  } else {
    const int pos0 = p.q_pos0 + tile * 128;
    const int lo = max(0, pos0 - p.window_tokens + 1) / RTP_BLOCK;
    const int hi = min(p.Nk - 1, pos0 + 127) / RTP_BLOCK;
    n_list = hi - lo + 1;
    if (tid == 0) bars.kb_lo = lo;
  }
  if (tid == 0) {
    mbar_init(smem_u32(&bars.q_full), 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(smem_u32(&bars.k_full[s]), 1);
      mbar_init(smem_u32(&bars.v_full[s]), 1);
      mbar_init(smem_u32(&bars.kv_empty[s]), 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(smem_u32(&bars.s_full[s]), 1);
      mbar_init(smem_u32(&bars.s_free[s]), 128);
    }
    mbar_init(smem_u32(&bars.p_full), 128);
    mbar_init(smem_u32(&bars.pv_done), 1);
    mbar_init(smem_u32(&bars.fin), 1);
    bars.abort = 0;
    bars.n_list = n_list;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(&bars.tmem_base), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars.tmem_base;
  const int kb_lo = bars.kb_lo;
  const int n_tiles = (n_list + 1) / 2;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch(&tmQ);
      tma_prefetch(&tmK);
      tma_prefetch(&tmV);
      const uint32_t qbar = smem_u32(&bars.q_full);
      mbar_arrive_expect_tx(qbar, 32768);
      tma_load_4d(sb + kQOff, &tmQ, qbar, 0, h, tile * 128, b);
      tma_load_4d(sb + kQOff + 16384, &tmQ, qbar, 64, h, tile * 128, b);
      int issued = 0;
      for (int j = 0; j < n_tiles; ++j) {
        const int s = j & 1;
        if (j >= kStages && !mbar_wait(smem_u32(&bars.kv_empty[s]), ((j - kStages) >> 1) & 1, abort_flag)) break;
        int kb0, kb1;
        if (p.sparse) {
          kb0 = list[2 * j].x;
          kb1 = (2 * j + 1 < n_list) ? list[2 * j + 1].x : kb0;
        } else {
          kb0 = kb_lo + 2 * j;
          kb1 = kb0 + 1;
        }
        const uint32_t kdst = sb + kKVOff + s * 65536u, vdst = kdst + 32768u;
        const uint32_t kbar = smem_u32(&bars.k_full[s]), vbar = smem_u32(&bars.v_full[s]);
        mbar_arrive_expect_tx(kbar, 32768);
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          tma_load_4d(kdst + half * 16384u, &tmK, kbar, half * 64, g, kb0 * RTP_BLOCK, b);
          tma_load_4d(kdst + half * 16384u + 8192u, &tmK, kbar, half * 64, g, kb1 * RTP_BLOCK, b);
        }
        mbar_arrive_expect_tx(vbar, 32768);
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          tma_load_4d(vdst + half * 16384u, &tmV, vbar, half * 64, g, kb0 * RTP_BLOCK, b);
          tma_load_4d(vdst + half * 16384u + 8192u, &tmV, vbar, half * 64, g, kb1 * RTP_BLOCK, b);
        }
        issued = j + 1;
      }
      if (*abort_flag) {
        // let copies already in flight land before the CTA exits
        wait_short(qbar, 0);
        for (int j = max(0, issued - kStages); j < issued; ++j) {
          wait_short(smem_u32(&bars.k_full[j & 1]), (j >> 1) & 1);
          wait_short(smem_u32(&bars.v_full[j & 1]), (j >> 1) & 1);
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_qk = idesc_bf16_f32(128, 128, false, false);
      constexpr uint32_t idesc_pv = idesc_bf16_f32(128, 128, false, true);
      bool ok = mbar_wait(smem_u32(&bars.q_full), 0, abort_flag);
      for (int j = 0; ok && j <= n_tiles; ++j) {
        if (j < n_tiles) {
          const int s = j & 1;
          if (!mbar_wait(smem_u32(&bars.k_full[s]), (j >> 1) & 1, abort_flag)) { ok = false; break; }
          if (j >= 2 && !mbar_wait(smem_u32(&bars.s_free[s]), ((j - 2) >> 1) & 1, abort_flag)) { ok = false; break; }
          tc_fence_after();
          const uint32_t kbase = sb + kKVOff + s * 65536u;
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint32_t koff = (kk >> 2) * 16384u + (kk & 3) * 32u;
            mma_bf16_ss(tmem + s * 128u, desc_sw128(sb + kQOff + koff, 16, 1024),
                        desc_sw128(kbase + koff, 16, 1024), idesc_qk, kk > 0 ? 1u : 0u);
          }
          mma_commit(smem_u32(&bars.s_full[s]));
        }
        if (j >= 1) {
          const int jp = j - 1, s = jp & 1;
          if (!mbar_wait(smem_u32(&bars.p_full), jp & 1, abort_flag)) { ok = false; break; }
          if (!mbar_wait(smem_u32(&bars.v_full[s]), (jp >> 1) & 1, abort_flag)) { ok = false; break; }
          tc_fence_after();
          const uint32_t vbase = sb + kKVOff + s * 65536u + 32768u;
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint32_t poff = (kk >> 2) * 16384u + (kk & 3) * 32u;
            mma_bf16_ss(tmem + kOCol, desc_sw128(sb + kPOff + poff, 16, 1024),
                        desc_sw128(vbase + kk * 2048u, 16384, 1024), idesc_pv,
                        (jp > 0 || kk > 0) ? 1u : 0u);
          }
          mma_commit(smem_u32(&bars.pv_done));
          mma_commit(smem_u32(&bars.kv_empty[s]));
        }
      }
      mma_commit(smem_u32(&bars.fin));
      wait_short(smem_u32(&bars.fin), 0);
    }
    __syncwarp();
  } else if (warp >= 4) {
    // ------------------------------------------------------------ softmax
    const int r = tid - 128;
    const uint32_t lane_base = tmem + ((uint32_t)((warp & 3) * 32) << 16);
    const int row = tile * 128 + r;
    const int pos = p.q_pos0 + row;
    const int rowbit = r < 64 ? 1 : 2;
    const float sl2 = p.scale_log2;
    float m_run = -INFINITY, l_run = 0.f;
    bool ok = true;
    for (int j = 0; j < n_tiles; ++j) {
      const int sbuf = j & 1;
      bool w = mbar_wait(smem_u32(&bars.s_full[sbuf]), (j >> 1) & 1, abort_flag);
      if (!__all_sync(0xffffffffu, w)) { ok = false; break; }
      tc_fence_after();
      uint32_t sr[128];
      tmem_ld32(lane_base + sbuf * 128u + 0u, sr);
      tmem_ld32(lane_base + sbuf * 128u + 32u, sr + 32);
      tmem_ld32(lane_base + sbuf * 128u + 64u, sr + 64);
      tmem_ld32(lane_base + sbuf * 128u + 96u, sr + 96);
      tc_wait_ld();
      tc_fence_before();
      mbar_arrive(smem_u32(&bars.s_free[sbuf]));

      // masks: each half of the tile is one 64-key block
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        const int e = 2 * j + half;
        int kb;
        bool att;
        if (p.sparse) {
          att = e < n_list && (list[e].y & rowbit);
          kb = e < n_list ? list[e].x : 0;
        } else {
          att = e < n_list;
          kb = kb_lo + e;
        }
        const int key0 = kb * RTP_BLOCK;
        if (!att) {
#pragma unroll
          for (int c = 0; c < 64; ++c) sr[half * 64 + c] = __float_as_uint(-INFINITY);
        } else {
          const bool full = (key0 + 63 <= pos) && (p.sparse || key0 > pos - p.window_tokens) &&
                            (key0 + 63 < p.Nk);
          if (!full) {
#pragma unroll
            for (int c = 0; c < 64; ++c) {
              const int u = key0 + c;
              const bool okk = u <= pos && (p.sparse || u > pos - p.window_tokens) && u < p.Nk;
              if (!okk) sr[half * 64 + c] = __float_as_uint(-INFINITY);
            }
          }
        }
      }
      float mx = -INFINITY;
#pragma unroll
      for (int c = 0; c < 128; ++c) mx = fmaxf(mx, __uint_as_float(sr[c]));
      const float m_cand = mx * sl2;
      const bool need = m_cand > m_run + 8.f;
      bool pv_waited = false;
      if (__any_sync(0xffffffffu, need && j > 0 && m_run != -INFINITY)) {
        w = mbar_wait(smem_u32(&bars.pv_done), (j - 1) & 1, abort_flag);
        if (!__all_sync(0xffffffffu, w)) { ok = false; break; }
        pv_waited = true;
        tc_fence_after();
        const float f = (need && m_run != -INFINITY) ? ex2(m_run - m_cand) : 1.f;
#pragma unroll
        for (int c4 = 0; c4 < 4; ++c4) {
          uint32_t o[32];
          tmem_ld32(lane_base + kOCol + c4 * 32u, o);
          tc_wait_ld();
#pragma unroll
          for (int c = 0; c < 32; ++c) o[c] = __float_as_uint(__uint_as_float(o[c]) * f);
          tmem_st32(lane_base + kOCol + c4 * 32u, o);
        }
        tc_wait_st();
      }
      if (need) {
        l_run *= ex2(m_run - m_cand);
        m_run = m_cand;
      }
      const float base = (m_run == -INFINITY) ? 0.f : m_run;
      float sum = 0.f;
      uint32_t pk[64];
#pragma unroll
      for (int c = 0; c < 64; ++c) {
        const float p0 = ex2(fmaf(__uint_as_float(sr[2 * c]), sl2, -base));
        const float p1 = ex2(fmaf(__uint_as_float(sr[2 * c + 1]), sl2, -base));
        sum += p0 + p1;
        pk[c] = pack_bf16x2(p0, p1);
      }
      l_run += sum;
      if (j > 0 && !pv_waited) {
        w = mbar_wait(smem_u32(&bars.pv_done), (j - 1) & 1, abort_flag);
        if (!__all_sync(0xffffffffu, w)) { ok = false; break; }
      }
      // P row r into the 128-byte-swizzled K-major tile (two 64-key chunks).
#pragma unroll
      for (int ch = 0; ch < 2; ++ch)
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const uint32_t addr = sb + kPOff + ch * 16384u + (uint32_t)r * 128u + (uint32_t)((u ^ (r & 7)) * 16);
          st_shared_v4(addr, pk[ch * 32 + u * 4], pk[ch * 32 + u * 4 + 1], pk[ch * 32 + u * 4 + 2],
                       pk[ch * 32 + u * 4 + 3]);
        }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(smem_u32(&bars.p_full));
    }
    if (ok) {
      bool w = mbar_wait(smem_u32(&bars.pv_done), (n_tiles - 1) & 1, abort_flag);
      if (__all_sync(0xffffffffu, w)) {
        tc_fence_after();
        const float inv = l_run > 0.f ? 1.f / l_run : 0.f;
        __nv_bfloat16* orow = static_cast<__nv_bfloat16*>(p.o) + (int64_t)b * p.o_sb + (int64_t)row * p.o_sn +
                              (int64_t)h * p.o_sh;
#pragma unroll
        for (int c4 = 0; c4 < 4; ++c4) {
          uint32_t o[32];
          tmem_ld32(lane_base + kOCol + c4 * 32u, o);
          tc_wait_ld();
          if (row < p.Nq) {
            uint4* dst = reinterpret_cast<uint4*>(orow + c4 * 32);
#pragma unroll
            for (int v4 = 0; v4 < 4; ++v4) {
              uint4 w4;
              w4.x = pack_bf16x2(__uint_as_float(o[v4 * 8 + 0]) * inv, __uint_as_float(o[v4 * 8 + 1]) * inv);
              w4.y = pack_bf16x2(__uint_as_float(o[v4 * 8 + 2]) * inv, __uint_as_float(o[v4 * 8 + 3]) * inv);
              w4.z = pack_bf16x2(__uint_as_float(o[v4 * 8 + 4]) * inv, __uint_as_float(o[v4 * 8 + 5]) * inv);
              w4.w = pack_bf16x2(__uint_as_float(o[v4 * 8 + 6]) * inv, __uint_as_float(o[v4 * 8 + 7]) * inv);
              dst[v4] = w4;
            }
          }
        }
      }
    }
  }

  // ---- teardown
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
  if (tid == 0 && bars.abort) atomicExch(status, kStatusTimeout);
}

size_t prefill_attn_tc_smem_bytes(const PrefillAttnParams& p) {
  return 1024 + kListOff + (size_t)p.list_cap * sizeof(int2) + sizeof(Bars);
}

cudaError_t launch_prefill_attn_tc(const PrefillAttnParams& p, const CUtensorMap& tmQ, const CUtensorMap& tmK,
                                   const CUtensorMap& tmV, int n_tiles, int B, int* status, cudaStream_t stream) {
  const size_t smem = prefill_attn_tc_smem_bytes(p);
  cudaError_t e = cudaFuncSetAttribute(prefill_attn_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid(n_tiles, p.n_heads, B);
  prefill_attn_tc_kernel<<<grid, kThreads, smem, stream>>>(p, tmQ, tmK, tmV, status);
  return cudaGetLastError();
}

}  // namespace rtp
