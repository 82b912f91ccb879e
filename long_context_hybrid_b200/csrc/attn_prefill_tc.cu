// Prefill attention on the 5th-generation tensor cores (tcgen05 + TMEM + TMA).
//
// A CTA computes 128 * NQ query rows of one head against a list of 64-key
// blocks:
//   * streaming heads (RTPurboV2 article: SWA with a local window), NQ = 2:
//     two 128-row query tiles share the band of key blocks overlapping
//     (pos - W, pos] of their 256 rows; each row masks its own window;
//   * retrieval heads (RTPurbo digest: exact attention at full dimension over
//     the indexer-selected set), NQ = 1: the 128 rows are query blocks 2t and
//     2t+1 and the list is the union of their attended sets (selected blocks,
//     sink blocks, window blocks); each entry carries which half attends it, so
//     a row only sees its own block's set, with the causal mask.
//
// Warp roles (64 + 128 * NQ threads):
//   warp 0   TMA producer: the Q tiles once (NQ = 2), then K and V of two
//            list blocks (128 keys) per step into an ST-stage ring (128-byte
//            swizzle);
//   warp 1   TMEM owner and single-thread MMA issuer:
//            S_t = Q_t K^T (M=128, N=128, K=128; NQ = 2: Q from shared memory,
//            NQ = 1: Q from TMEM) and O_t += P_t V (P read from TMEM, V read
//            MN-major);
//   softmax  warps 2.. : one warpgroup of 4 warps per query tile; warp w reads
//            TMEM lanes 32 (w % 4) .. +31, so thread r owns row r (TMEM lane r):
//            it reads S, masks, keeps an online softmax in the log2 domain
//            with lazy rescaling (O is rescaled in TMEM only when the running
//            max grows by more than 8), computes P with packed f32x2
//            arithmetic (key halves that are masked for the whole row skip the
//            exponentials), and writes P as bf16 back over the first half of S
//            in TMEM, where the next MMA reads it; each 64-key half is handled
//            on its own so that a thread holds 64 scores at a time.
// With NQ = 2 the MMA order QK0 QK1 | PV0 QK0' PV1 QK1' | ... keeps the tensor
// core busy on one tile while the other tile's softmax runs, and each K/V
// stage feeds both tiles. With NQ = 1 a stage feeds one tile, so the ring is
// three stages deep: the retrieval heads' query tile lives in TMEM (the
// softmax threads store their own rows there), which frees the shared memory
// for the third stage, and the copies of tile j + 2 start one tile earlier
// than with two stages (their key blocks lie anywhere in the sequence, most
// of them in DRAM).
// Every wait is bounded; a wait that runs out marks the CTA aborted, all roles
// drain, TMEM is freed and RTP_ERR_TIMEOUT is written to `status`.
#include "attn_prefill_common.cuh"
#include "rtp_common.cuh"
#include "rtp_internal.h"
#include "sm100.cuh"

namespace rtp {
using namespace sm100;

namespace {

constexpr int kMaxStages = 3;
constexpr uint32_t kQTileBytes = 32768;                       // [D half][128 rows][128 B]
constexpr uint32_t kStageBytes = 65536;                       // K 32 KB + V 32 KB
constexpr uint32_t kTmemCols = 512;
constexpr int kStatusTimeout = 4;

template <int NQ, int ST>
struct Layout {
  static constexpr int kThreads = 64 + 128 * NQ;
  static constexpr uint32_t kQOff = 0;                                   // NQ = 2 only
  static constexpr uint32_t kKVOff = NQ == 2 ? NQ * kQTileBytes : 0;
  static constexpr uint32_t kListOff = kKVOff + ST * kStageBytes;
  // TMEM columns: NQ = 2 -> tile t: S at 256 t, O at 256 t + 128.
  //               NQ = 1 -> S buffers at 0 and 128, O at 256, Q at 384
  //               (64 columns of bf16 pairs).
  static constexpr uint32_t kQTmem = 384;
};

struct Bars {
  uint64_t q_full;
  uint64_t k_full[kMaxStages], v_full[kMaxStages], kv_empty[kMaxStages];
  uint64_t s_full[2], p_full[2], pv_done;
  uint64_t fin;
  uint32_t tmem_base;
  int abort;
  int kb_lo;
  BlockScanSmem<384> scan;
};

__device__ __forceinline__ uint64_t f2(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ void f2_split(uint64_t v, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t f2_fma(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ float max3f(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}
// Marks the attended key blocks of query block q in `bits`.
template <int NT>
__device__ void mark_blocks(const PrefillAttnParams& p, int b, int jh, int q, unsigned* bits) {
  const int nb = p.Nq / RTP_BLOCK;
  const size_t row = ((size_t)b * p.n_heads + jh) * nb + q;
  const int cnt = p.counts ? min(p.counts[row], p.topk) : 0;
  const int32_t* sel = p.blocks + row * p.topk;
  for (int e = threadIdx.x; e < cnt; e += NT) {
    const int x = sel[e];
    if (x >= 0 && x <= q) atomicOr(&bits[x >> 5], 1u << (x & 31));
  }
  for (int x = threadIdx.x; x < min(p.sink_blocks, q + 1); x += NT) atomicOr(&bits[x >> 5], 1u << (x & 31));
  for (int x = max(0, q - p.window_blocks + 1) + threadIdx.x; x <= q; x += NT)
    atomicOr(&bits[x >> 5], 1u << (x & 31));
}

// Union list of query blocks 2t and 2t+1: entries (block, membership bits).
template <int NT>
__device__ int build_pair_list(const PrefillAttnParams& p, int b, int jh, int tile, unsigned* bitsA,
                               unsigned* bitsB, int2* list, BlockScanSmem<NT>& scan) {
  const int nb = p.Nq / RTP_BLOCK;
  const int qa = 2 * tile, qb = 2 * tile + 1;
  const bool has_b = qb < nb;
  const int qmax = has_b ? qb : qa;
  const int nw = qmax / 32 + 1;
  for (int w = threadIdx.x; w < nw; w += NT) { bitsA[w] = 0u; bitsB[w] = 0u; }
  __syncthreads();
  mark_blocks<NT>(p, b, jh, qa, bitsA);
  if (has_b) mark_blocks<NT>(p, b, jh, qb, bitsB);
  __syncthreads();
  const int per = (nw + NT - 1) / NT;
  const int w0 = threadIdx.x * per, w1 = min(nw, w0 + per);
  int c = 0;
  for (int w = w0; w < w1; ++w) c += __popc(bitsA[w] | bitsB[w]);
  int total;
  int off = block_exclusive_scan<NT>(c, total, scan);
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

__device__ __forceinline__ void mma_bf16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                            uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}"
      ::"r"(d_tmem), "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Issue S = Q K^T for one Q tile (8 K-steps of 16 over D = 128).
__device__ __forceinline__ void issue_qk(uint32_t d_tmem, uint32_t q_smem, uint32_t k_smem) {
  constexpr uint32_t idesc = idesc_bf16_f32(128, 128, false, false);
#pragma unroll
  for (int kk = 0; kk < 8; ++kk) {
    const uint32_t off = (kk >> 2) * 16384u + (kk & 3) * 32u;
    mma_bf16_ss(d_tmem, desc_sw128(q_smem + off, 16, 1024), desc_sw128(k_smem + off, 16, 1024), idesc,
                kk > 0 ? 1u : 0u);
  }
}
// Issue S = Q K^T with Q read from TMEM (128 lanes x 64 columns of bf16 pairs).
__device__ __forceinline__ void issue_qk_tq(uint32_t d_tmem, uint32_t q_tmem, uint32_t k_smem) {
  constexpr uint32_t idesc = idesc_bf16_f32(128, 128, false, false);
#pragma unroll
  for (int kk = 0; kk < 8; ++kk) {
    const uint32_t off = (kk >> 2) * 16384u + (kk & 3) * 32u;
    mma_bf16_ts(d_tmem, q_tmem + kk * 8u, desc_sw128(k_smem + off, 16, 1024), idesc, kk > 0 ? 1u : 0u);
  }
}
// Issue O (+)= P V for one Q tile (P in TMEM: 8 K-steps of 16 keys = 8 columns each).
__device__ __forceinline__ void issue_pv(uint32_t o_tmem, uint32_t p_tmem, uint32_t v_smem, bool accumulate) {
  constexpr uint32_t idesc = idesc_bf16_f32(128, 128, false, true);
#pragma unroll
  for (int kk = 0; kk < 8; ++kk)
    mma_bf16_ts(o_tmem, p_tmem + kk * 8u, desc_sw128(v_smem + kk * 2048u, 16384, 1024), idesc,
                (accumulate || kk > 0) ? 1u : 0u);
}

}  // namespace

template <int NQ, int ST>
__global__ void __launch_bounds__(64 + 128 * NQ, 1)
prefill_attn_tc_kernel(const PrefillAttnParams p, const __grid_constant__ CUtensorMap tmQ,
                       const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                       int* status) {
  static_assert(ST >= 2 && ST <= kMaxStages, "ring depth");
  using Lay = Layout<NQ, ST>;
  constexpr int NT = Lay::kThreads;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const uint32_t sb = smem_u32(smem);
  const int tile = blockIdx.x, jh = blockIdx.y, b = blockIdx.z;
  const int h = p.head[jh], g = h / p.G;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  int2* list = reinterpret_cast<int2*>(smem + Lay::kListOff);
  Bars& bars = *reinterpret_cast<Bars*>(smem + Lay::kListOff + (size_t)p.list_cap * sizeof(int2));
  volatile int* abort_flag = &bars.abort;
  const int row0 = tile * 128 * NQ;               // first query row of the CTA

  // ---- prologue: key-block list, barriers, TMEM
  int n_list;
  if constexpr (NQ == 1) {
   if (p.sparse) {
    unsigned* bitsA = reinterpret_cast<unsigned*>(smem + Lay::kKVOff);   // stage 0 is free until the first load
    unsigned* bitsB = bitsA + 8192;
    n_list = build_pair_list<NT>(p, b, jh, tile, bitsA, bitsB, list,
                                 *reinterpret_cast<BlockScanSmem<NT>*>(&bars.scan));
   } else {
    n_list = 0;
   }
  }
  if (NQ == 2 || !p.sparse) {
    const int pos0 = p.q_pos0 + row0;
    const int lo = max(0, pos0 - p.window_tokens + 1) / RTP_BLOCK;
    const int hi = min(p.Nk - 1, pos0 + 128 * NQ - 1) / RTP_BLOCK;
    n_list = hi - lo + 1;
    if (tid == 0) bars.kb_lo = lo;
  }
  if (tid == 0) {
    mbar_init(smem_u32(&bars.q_full), NQ == 1 ? 128 : 1);    // NQ = 1: the softmax threads' Q rows
    for (int s = 0; s < ST; ++s) {
      mbar_init(smem_u32(&bars.k_full[s]), 1);
      mbar_init(smem_u32(&bars.v_full[s]), 1);
      mbar_init(smem_u32(&bars.kv_empty[s]), 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(smem_u32(&bars.s_full[s]), 1);
      mbar_init(smem_u32(&bars.p_full[s]), 128);
    }
    mbar_init(smem_u32(&bars.pv_done), 1);
    mbar_init(smem_u32(&bars.fin), 1);
    bars.abort = 0;
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
      if (NQ == 2 && !p.withhold_q) {
        mbar_arrive_expect_tx(qbar, kQTileBytes * NQ);
#pragma unroll
        for (int t = 0; t < NQ; ++t) {
          tma_load_4d(sb + Lay::kQOff + t * kQTileBytes, &tmQ, qbar, 0, h, row0 + t * 128, b);
          tma_load_4d(sb + Lay::kQOff + t * kQTileBytes + 16384, &tmQ, qbar, 64, h, row0 + t * 128, b);
        }
      }
      int issued = 0;
      for (int j = 0; j < n_tiles; ++j) {
        const int s = j % ST;
        if (j >= ST && !mbar_wait(smem_u32(&bars.kv_empty[s]), (j / ST - 1) & 1, abort_flag)) break;
        int kb0, kb1;
        if (NQ == 1 && p.sparse) {
          kb0 = list[2 * j].x;
          kb1 = (2 * j + 1 < n_list) ? list[2 * j + 1].x : kb0;
        } else {
          kb0 = kb_lo + 2 * j;
          kb1 = kb0 + 1;
        }
        const uint32_t kdst = sb + Lay::kKVOff + s * kStageBytes, vdst = kdst + 32768u;
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
      // The MMA side ends every path by committing `fin`; once it has (or the
      // CTA has aborted), copies this thread issued but nobody consumed are
      // waited for, with a short bound, before the CTA exits.
      {
        const long long t0 = clock64();
        while (!mbar_try_wait(smem_u32(&bars.fin), 0) && !*abort_flag && clock64() - t0 < kWaitLimitCycles) {
        }
      }
      if (*abort_flag) {
        if (NQ == 2 && !p.withhold_q) wait_short(qbar, 0);
        for (int j = max(0, issued - ST); j < issued; ++j) {
          wait_short(smem_u32(&bars.k_full[j % ST]), (j / ST) & 1);
          wait_short(smem_u32(&bars.v_full[j % ST]), (j / ST) & 1);
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t q_s = sb + Lay::kQOff;
      bool ok = mbar_wait(smem_u32(&bars.q_full), 0, abort_flag);
      if (NQ == 2) {
        // QK0(0) QK1(0) | PV0(j) QK0(j+1) PV1(j) QK1(j+1) | ...
        if (ok && n_tiles > 0) {
          ok = mbar_wait(smem_u32(&bars.k_full[0]), 0, abort_flag);
          if (ok) {
            tc_fence_after();
            issue_qk(tmem + 0, q_s, sb + Lay::kKVOff);
            mma_commit(smem_u32(&bars.s_full[0]));
            issue_qk(tmem + 256, q_s + kQTileBytes, sb + Lay::kKVOff);
            mma_commit(smem_u32(&bars.s_full[1]));
          }
        }
        for (int j = 0; ok && j < n_tiles; ++j) {
          const int s = j & 1, s1 = (j + 1) & 1;
          const uint32_t v_s = sb + Lay::kKVOff + s * kStageBytes + 32768u;
          const bool more = j + 1 < n_tiles;
          if (!mbar_wait(smem_u32(&bars.p_full[0]), j & 1, abort_flag)) break;
          if (!mbar_wait(smem_u32(&bars.v_full[s]), (j >> 1) & 1, abort_flag)) break;
          tc_fence_after();
          issue_pv(tmem + 128, tmem + 0, v_s, j > 0);
          if (more) {
            if (!mbar_wait(smem_u32(&bars.k_full[s1]), ((j + 1) >> 1) & 1, abort_flag)) break;
            tc_fence_after();
            issue_qk(tmem + 0, q_s, sb + Lay::kKVOff + s1 * kStageBytes);
            mma_commit(smem_u32(&bars.s_full[0]));
          }
          if (!mbar_wait(smem_u32(&bars.p_full[1]), j & 1, abort_flag)) break;
          tc_fence_after();
          issue_pv(tmem + 384, tmem + 256, v_s, j > 0);
          mma_commit(smem_u32(&bars.kv_empty[s]));
          if (more) {
            issue_qk(tmem + 256, q_s + kQTileBytes, sb + Lay::kKVOff + s1 * kStageBytes);
            mma_commit(smem_u32(&bars.s_full[1]));
          }
        }
      } else {
        // QK(0) | QK(j+1) PV(j) | ... with S double-buffered, Q from TMEM,
        // K/V tile j in ring stage j % ST
        for (int j = 0; ok && j <= n_tiles; ++j) {
          if (j < n_tiles) {
            const int s = j % ST, sb2 = j & 1;
            if (!mbar_wait(smem_u32(&bars.k_full[s]), (j / ST) & 1, abort_flag)) { ok = false; break; }
            tc_fence_after();
            issue_qk_tq(tmem + sb2 * 128u, tmem + Lay::kQTmem, sb + Lay::kKVOff + s * kStageBytes);
            mma_commit(smem_u32(&bars.s_full[sb2]));
          }
          if (j >= 1) {
            const int jp = j - 1, s = jp % ST, sb2 = jp & 1;
            if (!mbar_wait(smem_u32(&bars.p_full[sb2]), (jp >> 1) & 1, abort_flag)) { ok = false; break; }
            if (!mbar_wait(smem_u32(&bars.v_full[s]), (jp / ST) & 1, abort_flag)) { ok = false; break; }
            tc_fence_after();
            issue_pv(tmem + 256, tmem + sb2 * 128u, sb + Lay::kKVOff + s * kStageBytes + 32768u, jp > 0);
            mma_commit(smem_u32(&bars.pv_done));
            mma_commit(smem_u32(&bars.kv_empty[s]));
          }
        }
      }
      mma_commit(smem_u32(&bars.fin));
      wait_short(smem_u32(&bars.fin), 0);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ softmax
    const int t = (warp - 2) >> 2;                  // query tile of this warpgroup
    const int r = (warp & 3) * 32 + lane;           // row within the tile = TMEM lane
    const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
    const int row = row0 + t * 128 + r;
    const int pos = p.q_pos0 + row;
    const int rowbit = r < 64 ? 1 : 2;
    const float sl2 = p.scale_log2;
    const uint32_t o_col = NQ == 2 ? (uint32_t)(t * 256 + 128) : 256u;
    float m_run = -INFINITY, l_run = 0.f;
    bool ok = true;
    if (NQ == 1) {
      // this thread's query row into TMEM lane r, columns kQTmem .. +63 (bf16
      // pairs, in memory order); rows past the sequence are zero
      const __nv_bfloat16* qrow = static_cast<const __nv_bfloat16*>(p.q.p) + (int64_t)b * p.q.sb +
                                  (int64_t)row * p.q.sn + (int64_t)h * p.q.sh;
#pragma unroll
      for (int c2 = 0; c2 < 2; ++c2) {
        uint32_t qv[32];
#pragma unroll
        for (int v4 = 0; v4 < 8; ++v4) {
          const uint4 x = row < p.Nq ? __ldg(reinterpret_cast<const uint4*>(qrow + c2 * 64) + v4)
                                     : make_uint4(0u, 0u, 0u, 0u);
          qv[4 * v4] = x.x; qv[4 * v4 + 1] = x.y; qv[4 * v4 + 2] = x.z; qv[4 * v4 + 3] = x.w;
        }
        tmem_st32(tmem + lane_off + Lay::kQTmem + c2 * 32u, qv);
      }
      tc_wait_st();
      tc_fence_before();
      mbar_arrive(smem_u32(&bars.q_full));
    }
    for (int j = 0; j < n_tiles; ++j) {
      const int sbuf = NQ == 2 ? t : (j & 1);
      const uint32_t s_col = NQ == 2 ? (uint32_t)(t * 256) : (uint32_t)(sbuf * 128);
      const uint32_t par = NQ == 2 ? (uint32_t)(j & 1) : (uint32_t)((j >> 1) & 1);
      bool w = mbar_wait(smem_u32(&bars.s_full[sbuf]), par, abort_flag);
      if (!__all_sync(0xffffffffu, w)) { ok = false; break; }
      tc_fence_after();
      // Each 64-key half of the tile (one key block): mask state (0 none, 1 all,
      // 2 partial), a lazy max update, exponentials, and P written as bf16 pairs
      // over S columns [32 half, 32 half + 32). If the second half raises the
      // running max by more than 8, the first half's P is rescaled in TMEM.
      const uint32_t s_addr = tmem + lane_off + s_col;
      float o_factor = 1.f;
      bool o_scaled = false;
      float sum_a = 0.f, sum_b = 0.f;
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        const int e = 2 * j + half;
        int kb;
        bool att;
        if (NQ == 1 && p.sparse) {
          att = e < n_list && (list[e].y & rowbit);
          kb = e < n_list ? list[e].x : 0;
        } else {
          att = e < n_list;
          kb = kb_lo + e;
        }
        const int key0 = kb * RTP_BLOCK;
        const bool sparse_row = NQ == 1 && p.sparse;
        const bool none = !att || key0 > pos || (!sparse_row && key0 + 63 <= pos - p.window_tokens) ||
                          key0 >= p.Nk;
        const bool full = !none && key0 + 63 <= pos && (sparse_row || key0 > pos - p.window_tokens) &&
                          key0 + 63 < p.Nk;
        uint32_t v[64];
        tmem_ld32(s_addr + half * 64u, v);
        tmem_ld32(s_addr + half * 64u + 32u, v + 32);
        tc_wait_ld();
        if (!none && !full) {
#pragma unroll
          for (int c = 0; c < 64; ++c) {
            const int u = key0 + c;
            const bool okk = u <= pos && (sparse_row || u > pos - p.window_tokens) && u < p.Nk;
            if (!okk) v[c] = __float_as_uint(-INFINITY);
          }
        }
        float mx = -INFINITY;
        if (!none) {
          float a0 = -INFINITY, a1 = -INFINITY;
#pragma unroll
          for (int c = 0; c < 64; c += 4) {
            a0 = max3f(a0, __uint_as_float(v[c]), __uint_as_float(v[c + 1]));
            a1 = max3f(a1, __uint_as_float(v[c + 2]), __uint_as_float(v[c + 3]));
          }
          mx = fmaxf(a0, a1);
        }
        const float m_cand = mx * sl2;
        const bool need = m_cand > m_run + 8.f;
        if (half == 1 && __any_sync(0xffffffffu, need && m_run != -INFINITY)) {
          const float f = (need && m_run != -INFINITY) ? ex2(m_run - m_cand) : 1.f;
          uint32_t w[32];
          tmem_ld32(s_addr, w);
          tc_wait_ld();
#pragma unroll
          for (int c = 0; c < 32; ++c)
            w[c] = pack_bf16x2(__uint_as_float(w[c] << 16) * f, __uint_as_float(w[c] & 0xffff0000u) * f);
          tmem_st32(s_addr, w);
        }
        if (need) {
          const float f = ex2(m_run - m_cand);      // 0 while nothing was attended yet
          if (m_run != -INFINITY) o_scaled = true;
          l_run *= f;
          o_factor *= f;
          sum_a *= f;
          sum_b *= f;
          m_run = m_cand;
        }
        const float base = (m_run == -INFINITY) ? 0.f : m_run;
        uint32_t pk[32];
        if (none) {
#pragma unroll
          for (int c = 0; c < 32; ++c) pk[c] = 0u;
        } else {
          const uint64_t sc2 = f2(sl2, sl2), nb2 = f2(-base, -base);
#pragma unroll
          for (int c = 0; c < 32; ++c) {
            const uint64_t x = f2_fma(f2(__uint_as_float(v[2 * c]), __uint_as_float(v[2 * c + 1])), sc2, nb2);
            float x0, x1;
            f2_split(x, x0, x1);
            const float p0 = ex2(x0), p1 = ex2(x1);
            if (c & 1) sum_b += p0 + p1;
            else sum_a += p0 + p1;
            pk[c] = pack_bf16x2(p0, p1);
          }
        }
        tmem_st32(s_addr + half * 32u, pk);
      }
      l_run += sum_a + sum_b;
      if (__any_sync(0xffffffffu, o_scaled && j > 0)) {
        // the running max grew by more than 8: rescale O in TMEM before PV(j)
        if (NQ == 1) {
          bool w2 = mbar_wait(smem_u32(&bars.pv_done), (j - 1) & 1, abort_flag);   // PV(j-1) must be done
          if (!__all_sync(0xffffffffu, w2)) { ok = false; break; }
          tc_fence_after();
        }
        const float f = o_scaled ? o_factor : 1.f;
#pragma unroll
        for (int c4 = 0; c4 < 4; ++c4) {
          uint32_t o[32];
          tmem_ld32(tmem + lane_off + o_col + c4 * 32u, o);
          tc_wait_ld();
#pragma unroll
          for (int c = 0; c < 32; ++c) o[c] = __float_as_uint(__uint_as_float(o[c]) * f);
          tmem_st32(tmem + lane_off + o_col + c4 * 32u, o);
        }
      }
      tc_wait_st();
      tc_fence_before();
      mbar_arrive(smem_u32(&bars.p_full[sbuf]));
    }
    if (ok) {
      bool w = mbar_wait(smem_u32(&bars.fin), 0, abort_flag);
      if (__all_sync(0xffffffffu, w)) {
        tc_fence_after();
        const float inv = l_run > 0.f ? 1.f / l_run : 0.f;
        __nv_bfloat16* orow = static_cast<__nv_bfloat16*>(p.o) + (int64_t)b * p.o_sb + (int64_t)row * p.o_sn +
                              (int64_t)h * p.o_sh;
#pragma unroll
        for (int c4 = 0; c4 < 4; ++c4) {
          uint32_t o[32];
          tmem_ld32(tmem + lane_off + o_col + c4 * 32u, o);
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

namespace {
size_t smem_bytes(uint32_t list_off, const PrefillAttnParams& p) {
  return 1024 + list_off + (size_t)p.list_cap * sizeof(int2) + sizeof(Bars);
}
}  // namespace

// Retrieval heads take the three-stage ring when their block list leaves room
// for it, else two stages.
size_t prefill_attn_tc_smem_bytes(const PrefillAttnParams& p) {
  if (!p.sparse) return smem_bytes(Layout<2, 2>::kListOff, p);
  const size_t s3 = smem_bytes(Layout<1, 3>::kListOff, p);
  return s3 <= 227 * 1024 ? s3 : smem_bytes(Layout<1, 2>::kListOff, p);
}

cudaError_t launch_prefill_attn_tc(const PrefillAttnParams& p, const CUtensorMap& tmQ, const CUtensorMap& tmK,
                                   const CUtensorMap& tmV, int n_tiles, int B, int* status, cudaStream_t stream) {
  const size_t smem = prefill_attn_tc_smem_bytes(p);
  (void)n_tiles;
  if (p.sparse) {
    const bool three = smem == smem_bytes(Layout<1, 3>::kListOff, p);
    auto kernel = three ? prefill_attn_tc_kernel<1, 3> : prefill_attn_tc_kernel<1, 2>;
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    dim3 grid((p.Nq + 127) / 128, p.n_heads, B);
    kernel<<<grid, Layout<1, 3>::kThreads, smem, stream>>>(p, tmQ, tmK, tmV, status);
  } else {
    cudaError_t e = cudaFuncSetAttribute(prefill_attn_tc_kernel<2, 2>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    dim3 grid((p.Nq + 255) / 256, p.n_heads, B);
    prefill_attn_tc_kernel<2, 2><<<grid, Layout<2, 2>::kThreads, smem, stream>>>(p, tmQ, tmK, tmV, status);
  }
  return cudaGetLastError();
}

}  // namespace rtp
