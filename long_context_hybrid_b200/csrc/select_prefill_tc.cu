// Prefill block selection on the 5th-generation tensor cores.
//
// Block score (the tiny 2K prefill workload statement): for query block i and
// key block j <= i, the max of q~_t . k~_u over the causal pairs of the two
// 64-token blocks; each query block keeps its top-k key blocks (RTPurbo digest:
// the 16-d indexer picks the candidates). The token score matrix never leaves
// the SM: every 128 x 256 score tile lives in TMEM only until the epilogue has
// copied it into registers.
//
// One CTA handles query blocks 2t and 2t+1 (128 query rows) of one retrieval
// head, longest key ranges first. Warp roles (384 threads):
//   warp 0       TMA: the 128 x 16 query-index tile once, then 256 x 16
//                key-index tiles (4 key blocks) into a 4-stage ring (32-byte
//                swizzle);
//   warp 1       TMEM owner; warps 1 and 2 issue the MMAs of the even and the
//                odd key tiles: one tcgen05.mma M=128 N=256 K=16 per tile into
//                TMEM score buffer 0 or 1;
//   warps 4..11  epilogue: every warp takes part in every tile. Warp w reads
//                rows 32*(w%4).. and the 128 columns of key blocks 2*(w/4-1)
//                and the next with one tcgen05.ld, releases the buffer to the
//                MMA warp at once, and reduces each 64-column block of its
//                row to one value with a tree of 3-input maxima. The per-row
//                maxima are staged in shared memory (32 rows x 32 values per
//                warp); every 16 tiles lane l folds column l over the 32 rows
//                and merges it into the block-score array of its query block
//                with a shared-memory atomic max on order-preserving keys.
//                Tiles that reach the diagonal block take a per-block path
//                with the causal mask and a warp reduction.
// Finally all threads run the exact radix top-k of each of the two block-score
// arrays (ties to the smaller block) and write ascending lists.
#include "rtp_common.cuh"
#include "rtp_internal.h"
#include "sm100.cuh"

namespace rtp {
using namespace sm100;

namespace {

constexpr int kThreads = 384;
constexpr int kBpw = 2;                            // 64-key blocks per epilogue warp per tile
constexpr int kKStages = 4;
constexpr int kChunkKeys = 256;                    // 4 key blocks per MMA
constexpr uint32_t kQOff = 0;                      // 128 rows x 32 B
constexpr uint32_t kKOff = 4096;                   // stage s at +s*8192 (256 rows x 32 B)
constexpr int kStageChunks = 32 / kBpw;            // tiles per flush of the staged row maxima
constexpr uint32_t kStgOff = kKOff + kKStages * 8192u;  // per epilogue warp: 32 rows x 33 floats
constexpr uint32_t kScoreOff = kStgOff + 8u * 32u * 33u * 4u;
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
__device__ __forceinline__ void tmem_ld128(uint32_t taddr, uint32_t* r) {
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x128.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32,%33,%34,%35,%36,%37,%38,%39,%40,%41,%42,%43,%44,%45,%46,%47,%48,%49,%50,%51,%52,%53,%54,%55,%56,%57,%58,%59,%60,%61,%62,%63,%64,%65,%66,%67,%68,%69,%70,%71,%72,%73,%74,%75,%76,%77,%78,%79,%80,%81,%82,%83,%84,%85,%86,%87,%88,%89,%90,%91,%92,%93,%94,%95,%96,%97,%98,%99,%100,%101,%102,%103,%104,%105,%106,%107,%108,%109,%110,%111,%112,%113,%114,%115,%116,%117,%118,%119,%120,%121,%122,%123,%124,%125,%126,%127}, [%128];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31]), "=r"(r[32]), "=r"(r[33]), "=r"(r[34]), "=r"(r[35]), "=r"(r[36]), "=r"(r[37]), "=r"(r[38]), "=r"(r[39]), "=r"(r[40]), "=r"(r[41]), "=r"(r[42]), "=r"(r[43]), "=r"(r[44]), "=r"(r[45]), "=r"(r[46]), "=r"(r[47]), "=r"(r[48]), "=r"(r[49]), "=r"(r[50]), "=r"(r[51]), "=r"(r[52]), "=r"(r[53]), "=r"(r[54]), "=r"(r[55]), "=r"(r[56]), "=r"(r[57]), "=r"(r[58]), "=r"(r[59]), "=r"(r[60]), "=r"(r[61]), "=r"(r[62]), "=r"(r[63]), "=r"(r[64]), "=r"(r[65]), "=r"(r[66]), "=r"(r[67]), "=r"(r[68]), "=r"(r[69]), "=r"(r[70]), "=r"(r[71]), "=r"(r[72]), "=r"(r[73]), "=r"(r[74]), "=r"(r[75]), "=r"(r[76]), "=r"(r[77]), "=r"(r[78]), "=r"(r[79]), "=r"(r[80]), "=r"(r[81]), "=r"(r[82]), "=r"(r[83]), "=r"(r[84]), "=r"(r[85]), "=r"(r[86]), "=r"(r[87]), "=r"(r[88]), "=r"(r[89]), "=r"(r[90]), "=r"(r[91]), "=r"(r[92]), "=r"(r[93]), "=r"(r[94]), "=r"(r[95]), "=r"(r[96]), "=r"(r[97]), "=r"(r[98]), "=r"(r[99]), "=r"(r[100]), "=r"(r[101]), "=r"(r[102]), "=r"(r[103]), "=r"(r[104]), "=r"(r[105]), "=r"(r[106]), "=r"(r[107]), "=r"(r[108]), "=r"(r[109]), "=r"(r[110]), "=r"(r[111]), "=r"(r[112]), "=r"(r[113]), "=r"(r[114]), "=r"(r[115]), "=r"(r[116]), "=r"(r[117]), "=r"(r[118]), "=r"(r[119]), "=r"(r[120]), "=r"(r[121]), "=r"(r[122]), "=r"(r[123]), "=r"(r[124]), "=r"(r[125]), "=r"(r[126]), "=r"(r[127])
               : "r"(taddr));
}
__device__ __forceinline__ void sts_f32(uint32_t a, float v) { asm volatile("st.shared.f32 [%0], %1;" ::"r"(a), "f"(v) : "memory"); }
__device__ __forceinline__ float lds_f32(uint32_t a) { float v; asm volatile("ld.shared.f32 %0, [%1];" : "=f"(v) : "r"(a) : "memory"); return v; }
// max of 64 scores: a tree of 3-input maxima (32 instructions, depth 4)
__device__ __forceinline__ float tree_max64(const uint32_t* u) {
  float a[22], c[8];
#pragma unroll
  for (int x = 0; x < 21; ++x)
    a[x] = max3f(__uint_as_float(u[3 * x]), __uint_as_float(u[3 * x + 1]), __uint_as_float(u[3 * x + 2]));
  a[21] = __uint_as_float(u[63]);
#pragma unroll
  for (int x = 0; x < 7; ++x) c[x] = max3f(a[3 * x], a[3 * x + 1], a[3 * x + 2]);
  c[7] = a[21];
  return max3f(max3f(c[0], c[1], c[2]), max3f(c[3], c[4], c[5]), fmaxf(c[6], c[7]));
}
__device__ __forceinline__ bool try_wait_nohint(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile("{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\tselp.u32 %0, 1, 0, p;\n\t}"
               : "=r"(ok) : "r"(bar), "r"(parity) : "memory");
  return ok != 0;
}
// Bounded wait without a suspend hint (the epilogue's per-tile handshake).
__device__ __forceinline__ bool wait_tile(uint32_t bar, uint32_t parity, volatile int* abort_flag) {
  if (try_wait_nohint(bar, parity)) return true;
  const long long t0 = clock64();
  for (uint32_t it = 1;; ++it) {
    if (try_wait_nohint(bar, parity)) return true;
    if ((it & 63u) == 0) {
      if (*abort_flag) return false;
      if (clock64() - t0 > kWaitLimitCycles) { *abort_flag = 1; return false; }
    }
  }
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
      mbar_init(smem_u32(&bars.s_free[s]), 8);     // one arrive per epilogue warp
    }
    mbar_init(smem_u32(&bars.fin), 2);
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
  } else if (warp == 1 || warp == 2) {
    // Two issuers, one per score buffer: a tcgen05.mma and its commits take a
    // few hundred cycles to issue on a scheduler whose epilogue warps keep the
    // ALU busy, so one thread alone cannot keep both buffers full.
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(128, 256, false, false);
      bool ok = mbar_wait(smem_u32(&bars.q_full), 0, abort_flag);
      const uint64_t qdesc = desc_sw32(sb + kQOff);
      const int buf = warp - 1;
      for (int c = buf; ok && c < n_chunks; c += 2) {
        const int s = c % kKStages;
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
    const int wu = __shfl_sync(0xffffffffu, warp, 0);   // warp index, uniform across the warp
    const int quad = wu & 3;                            // TMEM lane quarter = rows 32*quad ..
    const int b_lo = ((wu - 4) >> 2) * kBpw;            // first of this warp's blocks in a tile
    const uint32_t taddr = tmem + ((uint32_t)(quad * 32) << 16) + (uint32_t)(b_lo * 64);
    const bool in_a = quad < 2;
    const int my_q = in_a ? qa : qb;
    const int my_last = in_a ? qa : last_blk;
    const int rq = (quad & 1) * 32 + lane;              // row within its query block
    const bool rows_valid = in_a || has_b;
    uint32_t* dst = in_a ? sA : sB;
    const int n_fast = qa >> 2;                         // tiles whose 4 blocks all precede block qa
    bool live = true;
    int c = 0;
    const uint32_t stg = sb + kStgOff + (uint32_t)((wu - 4) * (32 * 33) * 4);   // shared address
    int n_stg = 0, c_stg = 0;
    // lane l folds staged column l (tile c_stg + l / kBpw, block b_lo + l % kBpw) over the warp's 32 rows
    auto flush = [&](int n_tiles) {
      __syncwarp();
      if (lane < n_tiles * kBpw) {
        const uint32_t col = stg + lane * 4u;
        float x[11];
#pragma unroll
        for (int r = 0; r < 10; ++r)
          x[r] = max3f(lds_f32(col + (3 * r) * 132), lds_f32(col + (3 * r + 1) * 132), lds_f32(col + (3 * r + 2) * 132));
        x[10] = fmaxf(lds_f32(col + 30 * 132), lds_f32(col + 31 * 132));
        const float m = max3f(max3f(x[0], x[1], x[2]), max3f(x[3], x[4], x[5]), max3f(max3f(x[6], x[7], x[8]), x[9], x[10]));
        const int kb = (c_stg + lane / kBpw) * 4 + b_lo + lane % kBpw;
        if (rows_valid) atomicMax(&dst[kb], f2key(m));
      }
      __syncwarp();
    };
    // two tiles (both score buffers) per iteration: constant TMEM offsets, one parity
    for (; c + 1 < n_fast; c += 2) {
      const uint32_t par = (c >> 1) & 1;
#pragma unroll
      for (int buf = 0; buf < 2; ++buf) {
        const bool w = wait_tile(smem_u32(&bars.s_full[buf]), par, abort_flag);
        if (!__all_sync(0xffffffffu, w)) { live = false; break; }
        tc_fence_after();
        uint32_t v[128];
        tmem_ld128(taddr + buf * 256u, v);
        tc_wait_ld();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&bars.s_free[buf]));
        const uint32_t a = stg + (uint32_t)(lane * 33 + (n_stg + buf) * 2) * 4u;
        sts_f32(a, tree_max64(v));
        sts_f32(a + 4, tree_max64(v + 64));
      }
      if (!live) break;
      n_stg += 2;
      if (n_stg == kStageChunks) {
        flush(kStageChunks);
        n_stg = 0;
        c_stg = c + 2;
      }
    }
    for (; live && c < n_fast; ++c) {
      const int buf = c & 1;
      const bool w = wait_tile(smem_u32(&bars.s_full[buf]), (c >> 1) & 1, abort_flag);
      if (!__all_sync(0xffffffffu, w)) { live = false; break; }
      tc_fence_after();
      uint32_t v[128];
      tmem_ld128(taddr + buf * 256u, v);
      tc_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&bars.s_free[buf]));
#pragma unroll
      for (int bb = 0; bb < kBpw; ++bb) sts_f32(stg + (uint32_t)(lane * 33 + n_stg * kBpw + bb) * 4u, tree_max64(v + 64 * bb));
      if (++n_stg == kStageChunks) {
        flush(kStageChunks);
        n_stg = 0;
        c_stg = c + 1;
      }
    }
    if (live && n_stg > 0) flush(n_stg);
    for (; live && c < n_chunks; ++c) {
      const int buf = c & 1;
      const bool w = wait_tile(smem_u32(&bars.s_full[buf]), (c >> 1) & 1, abort_flag);
      if (!__all_sync(0xffffffffu, w)) break;
      tc_fence_after();
      uint32_t v[128];
      tmem_ld128(taddr + buf * 256u, v);
      tc_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&bars.s_free[buf]));
#pragma unroll
      for (int bb = 0; bb < kBpw; ++bb) {
        const int kb = c * 4 + b_lo + bb;
        const uint32_t* u = v + 64 * bb;
        float m = -INFINITY;
        if (kb < my_q) {
          m = tree_max64(u);
        } else if (kb == my_q) {
          // diagonal block: key column x is causal for this row iff x <= rq
#pragma unroll
          for (int x = 0; x < 64; ++x)
            if (x <= rq) m = fmaxf(m, __uint_as_float(u[x]));
        }
        const float wmax = warp_max(m);
        if (lane == 0 && rows_valid && kb <= my_last && wmax != -INFINITY) atomicMax(&dst[kb], f2key(wmax));
      }
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

cudaError_t launch_select_prefill_tc(const void* qt, const void* kt, int64_t kt_cap, int B, int N, int Hr, int Hkv,
                                     const int32_t* kv_of, int topk, int32_t* blocks, int32_t* counts,
                                     int* status, cudaStream_t stream) {
  SelectTcParams p;
  p.N = N; p.Hr = Hr; p.Hkv = Hkv; p.topk = topk; p.nb = N / RTP_BLOCK;
  p.blocks = blocks; p.counts = counts;
  for (int j = 0; j < Hr; ++j) p.kv[j] = kv_of[j];
  CUtensorMap tq, tk;
  if (!make_tmap_index(&tq, qt, B, Hr, N, N, 128) || !make_tmap_index(&tk, kt, B, Hkv, N, kt_cap, kChunkKeys))
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
cudaError_t launch_select_prefill(const void* qt, const void* kt, int64_t kt_cap, int B, int N, int Hr, int Hkv,
                                  const int32_t* kv_of, int topk, int32_t* blocks, int32_t* counts, void* ws,
                                  cudaStream_t stream) {
  return launch_select_prefill_tc(qt, kt, kt_cap, B, N, Hr, Hkv, kv_of, topk, blocks, counts, static_cast<int*>(ws),
                                  stream);
}
}  // namespace rtp
