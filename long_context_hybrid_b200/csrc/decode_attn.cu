// Decode attention: one new query token per sequence against the KV cache.
//
// Streaming heads attend the last `window` tokens (RTPurboV2 article: SWA on
// streaming heads). Retrieval heads attend, as a set, their selected tokens,
// tokens 0..sink-1 and their own last `window` tokens (the 128K decode
// workload statement: top-2048 unioned with the last 8192 tokens and token 0,
// exact softmax at D = 128).
//
// The work is HBM-bound (512 bytes of K and V per attended token), so the
// design goal is to read every K/V row once and keep enough bytes in flight:
//   * the work is two lists of 64-key chunks in segments: a window segment
//     per (sequence, KV group) covers the union of the window, with every
//     listed query head of the group as one row of a 16 x 128 query tile
//     (grouped heads share the chunk's K/V; each row masks keys outside its
//     own window); a gathered segment per (sequence, retrieval head) covers
//     its sink tokens and selected list (entries inside the window or below
//     `sink` are masked: those keys come from elsewhere);
//   * two persistent CTAs per SM each take a contiguous run of each list, so
//     both kinds of chunk are spread evenly. Each of a CTA's four warps owns 16
//     keys of every chunk: it copies its own K and V rows with 16-byte cp.async
//     (zero-filled where masked) two chunks ahead into a private three-stage
//     ring of 256-byte rows whose 16-byte pieces are XOR-swizzled
//     (conflict-free ldmatrix), and computes S = Q K^T and O += P V with bf16
//     mma.sync (fp32 accumulate) and an online softmax carried across the
//     run's chunks of a segment. The warps never wait for one another;
//   * where a run leaves a segment each warp writes its partial of every head
//     of the segment (running max in the log2 domain, sum, o[128]); a second
//     kernel, one CTA per head, merges each head's partials and writes its
//     output.
#include <cuda.h>
#include <mutex>

#include "rtp_common.cuh"
#include "rtp_internal.h"

namespace rtp {

namespace {
constexpr int kWarps = 4;
constexpr int kThreads = kWarps * 32;
constexpr int kCtasPerSm = 2;
constexpr int kChunk = 64;                    // keys per chunk
constexpr int kKeys = kChunk / kWarps;        // keys per warp and chunk (16)
constexpr int kStages = 3;
constexpr int kRowBytes = RTP_D * 2;          // 256
constexpr int kSlab = kKeys * kRowBytes;      // one warp's K (or V) rows of one chunk
constexpr int kPartStride = 4 + RTP_D;        // m, l, 2 pad, o[128] (16-byte aligned rows)
constexpr int kPartO = 4;
constexpr int kMaxGroup = 16;                 // query heads per KV group packed in one MMA tile
constexpr int kMergeBatch = 16;               // partials read at once by a merging warp
constexpr size_t kHeaderBytes = 256;          // status word (cleared by every call)

struct DecodeParams {
  const __nv_bfloat16* q; int64_t q_sb, q_sh;
  const __nv_bfloat16* k; int64_t k_sb, k_sn, k_sh;
  const __nv_bfloat16* v; int64_t v_sb, v_sn, v_sh;
  __nv_bfloat16* o; int64_t o_sb, o_sh;
  int B, G;
  const int32_t* idx; int topk;     // idx rows hold topk entries
  int n_sel;                         // entries read per row: min(topk, L) (valid entries come first)
  int sink;
  float scale_log2;
  int n_heads, n_ret;                // call heads: retrieval heads first (0..n_ret-1)
  int max_slots;                     // partial slots per head
  int n_wc, wlo_union, whi;          // window chunks over [wlo_union, whi)
  int n_gc;                          // gathered chunks per retrieval head
  int n_ag;                          // KV groups with at least one listed head
  int n_win_chunks;                  // B * n_ag * n_wc
  int n_gat_chunks;                  // B * n_ret * n_gc
  float* part;                       // [B, n_heads, max_slots, kPartStride]
  int early_start;                   // window chunks may be read before the previous kernel ends
  int head[kMaxHeads];               // query head of each call head
  int wlo[kMaxHeads];                // first position of each call head's window
  int ag_of[kMaxHeads];              // active-group index of each call head
  int ag_kv[kMaxGroup];              // KV group of each active group
  int ag_n[kMaxGroup];               // rows (call heads) of each active group
  int ag_rows[kMaxGroup][kMaxGroup];
};

struct Smem {
  unsigned char ring[kWarps][kStages][2][kSlab];   // [warp][stage][K, V]
  int pos[kWarps][kStages][kKeys];
};

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
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, bool valid) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(valid ? 16 : 0)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;\n" ::"n"(N) : "memory"); }

// Byte offset of 16-byte piece c (0..15) of row r in a slab of 256-byte rows:
// the piece index is XORed with r mod 8, so the eight rows of an ldmatrix
// read hit distinct banks.
__device__ __forceinline__ uint32_t slab_off(int r, int c) {
  return (uint32_t)(r * kRowBytes + ((c ^ (r & 7)) << 4));
}

// Contiguous runs: CTA c takes chunks [run_start(c), run_start(c + 1)) of a
// list of n chunks (empty runs when there are more CTAs than chunks).
__device__ __forceinline__ int run_start(int c, int n, int n_ctas) { return (int)((int64_t)c * n / n_ctas); }
// CTA whose run holds chunk x.
__device__ __forceinline__ int cta_of(int x, int n, int n_ctas) { return (int)(((int64_t)(x + 1) * n_ctas - 1) / n); }
// Pieces (runs) of a segment [s0, s0 + len) of a list of n chunks, numbered
// 0, 1, ... in chunk order. With n_ctas <= n no run is empty and piece i is
// the i-th CTA from the segment's first; otherwise every run holds at most one
// chunk and piece i is the segment's chunk i.
__device__ __forceinline__ int n_pieces(int s0, int len, int n, int n_ctas) {
  return n_ctas <= n ? cta_of(s0 + len - 1, n, n_ctas) - cta_of(s0, n, n_ctas) + 1 : len;
}
__device__ __forceinline__ int piece_of(int cta, int x_first, int s0, int n, int n_ctas) {
  return n_ctas <= n ? cta - cta_of(s0, n, n_ctas) : x_first - s0;
}

// Walks a CTA's chunks: its window run, then its gathered run. Segments:
// window (sequence-major, then active group), gathered (sequence-major, then
// retrieval head).
struct Cursor {
  int left_w;    // window chunks left after this one (-1: in the gathered run)
  int x;         // chunk index in its list
  int local;     // chunk index in its segment
  int sg;        // segment index in its list
  int b, a;      // sequence; active group (window) or retrieval head (gathered)
  int gathered;
  __device__ int id(const DecodeParams& p) const { return gathered ? p.B * p.n_ag + sg : sg; }
  __device__ int s0() const { return x - local; }
  __device__ void at(const DecodeParams& p, int x_, int gathered_) {
    x = x_;
    gathered = gathered_;
    const int len = gathered ? p.n_gc : p.n_wc, A = gathered ? p.n_ret : p.n_ag;
    sg = x / len; local = x - sg * len;
    b = sg / A; a = sg - b * A;
  }
  __device__ void next(const DecodeParams& p, int g0) {
    if (left_w == 0) {
      left_w = -1;
      if (p.n_gat_chunks > 0) at(p, g0, 1);
      return;
    }
    if (left_w > 0) --left_w;
    ++x;
    const int len = gathered ? p.n_gc : p.n_wc, A = gathered ? p.n_ret : p.n_ag;
    if (++local == len) {
      local = 0; ++sg;
      if (++a == A) { a = 0; ++b; }
    }
  }
};

// Key position of slot `s` (0..kChunk-1) of the cursor's chunk (-1: masked
// for every row), in two steps so that the selected-list read can be issued
// a chunk early: slot_fetch reads what the position depends on, slot_pos
// turns it into the position.
__device__ __forceinline__ int slot_fetch(const DecodeParams& p, const Cursor& c, int s, bool& dep_done) {
  if (!c.gathered) return 0;
  if (!dep_done) {
    pdl_wait();                               // the selected lists come from the previous kernel
    dep_done = true;
  }
  const int j = c.a;                          // retrieval heads are call heads 0..n_ret-1
  const int n_sink = min(p.sink, p.wlo[j]);
  const int e = c.local * kChunk + s;         // virtual list: sink tokens, then the selected entries
  if (e < n_sink || e - n_sink >= p.n_sel) return -1;
  return __ldg(p.idx + ((size_t)c.b * p.n_ret + j) * p.topk + (e - n_sink));
}
__device__ __forceinline__ int slot_pos(const DecodeParams& p, const Cursor& c, int s, int fetched) {
  if (!c.gathered) {
    const int u = p.wlo_union + c.local * kChunk + s;
    return u < p.whi ? u : -1;
  }
  const int wlo = p.wlo[c.a];
  const int n_sink = min(p.sink, wlo);
  const int e = c.local * kChunk + s;
  if (e < n_sink) return e;
  if (e - n_sink >= p.n_sel) return -1;
  return (fetched >= p.sink && fetched < wlo) ? fetched : -1;
}
}  // namespace

__global__ void __launch_bounds__(kThreads, kCtasPerSm)
decode_attn_kernel(const DecodeParams p) {
  extern __shared__ __align__(128) unsigned char smem_raw[];
  Smem& sm = *reinterpret_cast<Smem*>(smem_raw);
  pdl_trigger();                              // the merge may launch; it waits for this grid
  // Unless the caller knows that the previous kernel on the stream writes
  // none of q, K, V (only the selected lists), wait for it before any read.
  if (!p.early_start) pdl_wait();
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int gq = lane >> 2, tq = lane & 3;
  const int n_ctas = gridDim.x;
  const int w0 = run_start(blockIdx.x, p.n_win_chunks, n_ctas);
  const int n_w = run_start(blockIdx.x + 1, p.n_win_chunks, n_ctas) - w0;
  const int g0 = p.n_gat_chunks ? run_start(blockIdx.x, p.n_gat_chunks, n_ctas) : 0;
  const int n_g = p.n_gat_chunks ? run_start(blockIdx.x + 1, p.n_gat_chunks, n_ctas) - g0 : 0;
  const int n_t = n_w + n_g;                  // this CTA's chunks: window run, then gathered run
  if (n_t == 0) return;
  Cursor first;
  first.left_w = n_w > 0 ? n_w - 1 : -1;
  first.at(p, n_w > 0 ? w0 : g0, n_w > 0 ? 0 : 1);

  // this warp's ring and its copies of a chunk into stage st
  const uint32_t ring = su32(sm.ring[warp]);
  Cursor icur = first;                        // next chunk to copy
  const int my_slot = warp * kKeys + (lane & (kKeys - 1));
  bool dep_done = false;
  int fetched = slot_fetch(p, icur, my_slot, dep_done);  // for the next chunk to copy
  auto issue = [&](int t) {
    if (t < n_t) {
      const int st = t % kStages;
      const int g = icur.gathered ? p.head[icur.a] / p.G : p.ag_kv[icur.a];
      // lane r < kKeys owns row r: its position and its K/V row addresses
      const int pos = slot_pos(p, icur, my_slot, fetched);
      if (lane < kKeys) sm.pos[warp][st][lane] = pos;
      const int64_t u = pos >= 0 ? pos : 0;
      const char* krow = reinterpret_cast<const char*>(p.k + (int64_t)icur.b * p.k_sb + (int64_t)g * p.k_sh + u * p.k_sn);
      const char* vrow = reinterpret_cast<const char*>(p.v + (int64_t)icur.b * p.v_sb + (int64_t)g * p.v_sh + u * p.v_sn);
      const uint32_t kdst = ring + (uint32_t)(st * 2) * kSlab, vdst = kdst + kSlab;
      const int c = lane & 15;
#pragma unroll
      for (int i = 0; i < kKeys / 2; ++i) {
        const int r = 2 * i + (lane >> 4);
        const bool ok = __shfl_sync(0xffffffffu, pos, r) >= 0;
        const char* ks = reinterpret_cast<const char*>(__shfl_sync(0xffffffffu, reinterpret_cast<uintptr_t>(krow), r));
        const char* vs = reinterpret_cast<const char*>(__shfl_sync(0xffffffffu, reinterpret_cast<uintptr_t>(vrow), r));
        cp_async16(kdst + slab_off(r, c), ks + c * 16, ok);
        cp_async16(vdst + slab_off(r, c), vs + c * 16, ok);
      }
      icur.next(p, g0);
      if (t + 1 < n_t) fetched = slot_fetch(p, icur, my_slot, dep_done);
    }
    cp_async_commit();                        // one group per chunk, empty past the run
  };

  uint32_t qa[8][4];
  float o[16][4];
  float m_a = -INFINITY, m_b = -INFINITY, l_a = 0.f, l_b = 0.f;
  int ja = -1, jb = -1, lo_a = 0, lo_b = 0;
  Cursor cur = first;                         // chunk being computed
  int cur_id = -1, piece_b = 0, piece_a = 0, piece_x = 0, piece_s0 = 0, piece_gathered = 0, piece_chunks = 0;

  // Writes this warp's partial of every row of the segment (its keys of the
  // run's chunks in the segment).
  auto flush = [&]() {
    l_a += __shfl_xor_sync(0xffffffffu, l_a, 1);
    l_a += __shfl_xor_sync(0xffffffffu, l_a, 2);
    l_b += __shfl_xor_sync(0xffffffffu, l_b, 1);
    l_b += __shfl_xor_sync(0xffffffffu, l_b, 2);
    const int n_list = piece_gathered ? p.n_gat_chunks : p.n_win_chunks;
    int piece = piece_of((int)blockIdx.x, piece_x, piece_s0, n_list, n_ctas);
    if (piece_gathered)
      piece += n_pieces((piece_b * p.n_ag + p.ag_of[piece_a]) * p.n_wc, p.n_wc, p.n_win_chunks, n_ctas);
    const int kslot = piece * kWarps + warp;
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      const int j = half ? jb : ja;
      if (j < 0) continue;
      float* part = p.part + (((size_t)piece_b * p.n_heads + j) * p.max_slots + kslot) * kPartStride;
      if (tq == 0) { part[0] = half ? m_b : m_a; part[1] = half ? l_b : l_a; }
#pragma unroll
      for (int nt = 0; nt < 16; ++nt) {
        const int col = nt * 8 + 2 * tq;
        *reinterpret_cast<float2*>(part + kPartO + col) = make_float2(o[nt][half * 2], o[nt][half * 2 + 1]);
      }
    }
  };

  // prologue: the first kStages - 1 chunks in flight
#pragma unroll
  for (int t = 0; t < kStages - 1; ++t) issue(t);
  for (int t = 0; t < n_t; ++t, cur.next(p, g0)) {
    issue(t + kStages - 1);
    const int id = cur.id(p);
    if (id != cur_id) {
      if (cur_id >= 0) flush();
      cur_id = id;
      piece_b = cur.b; piece_a = cur.a; piece_x = cur.x; piece_s0 = cur.s0(); piece_gathered = cur.gathered;
      piece_chunks = 0;
      // rows of the tile: the group's heads (window) or the one retrieval head
      if (cur.gathered) {
        ja = gq == 0 ? cur.a : -1;
        jb = -1;
      } else {
        ja = gq < p.ag_n[cur.a] ? p.ag_rows[cur.a][gq] : -1;
        jb = gq + 8 < p.ag_n[cur.a] ? p.ag_rows[cur.a][gq + 8] : -1;
      }
      lo_a = ja >= 0 ? (cur.gathered ? 0 : p.wlo[ja]) : 0x7fffffff;
      lo_b = jb >= 0 ? (cur.gathered ? 0 : p.wlo[jb]) : 0x7fffffff;
      // query fragments straight from global memory (A operand, 16 x 128)
      const __nv_bfloat16* qra = p.q + (int64_t)cur.b * p.q_sb + (int64_t)(ja >= 0 ? p.head[ja] : 0) * p.q_sh;
      const __nv_bfloat16* qrb = p.q + (int64_t)cur.b * p.q_sb + (int64_t)(jb >= 0 ? p.head[jb] : 0) * p.q_sh;
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        const int c = kk * 16 + 2 * tq;
        qa[kk][0] = ja >= 0 ? __ldg(reinterpret_cast<const uint32_t*>(qra + c)) : 0u;
        qa[kk][1] = jb >= 0 ? __ldg(reinterpret_cast<const uint32_t*>(qrb + c)) : 0u;
        qa[kk][2] = ja >= 0 ? __ldg(reinterpret_cast<const uint32_t*>(qra + c + 8)) : 0u;
        qa[kk][3] = jb >= 0 ? __ldg(reinterpret_cast<const uint32_t*>(qrb + c + 8)) : 0u;
      }
      m_a = m_b = -INFINITY;
      l_a = l_b = 0.f;
#pragma unroll
      for (int nt = 0; nt < 16; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) o[nt][e] = 0.f;
    }
    cp_async_wait<kStages - 1>();               // chunk t has landed (this lane's copies)
    __syncwarp();                                // ... and every lane's
    const int st = t % kStages;
    const uint32_t kbase = ring + (uint32_t)(st * 2) * kSlab, vbase = kbase + kSlab;
    // S = Q K^T (16 rows x this warp's 16 keys: two n-tiles per ldmatrix.x4)
    float sacc[2][4];
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) sacc[nt][e] = 0.f;
    {
      const int m = lane >> 3;
      const int key = 8 * (m >> 1) + (lane & 7);
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        uint32_t bf[4];
        ldsm_x4(bf, kbase + slab_off(key, kk * 2 + (m & 1)));
        mma16816(sacc[0], qa[kk], bf[0], bf[1]);
        mma16816(sacc[1], qa[kk], bf[2], bf[3]);
      }
    }
    // mask, online softmax (rows gq and gq + 8)
    float mx_a = -INFINITY, mx_b = -INFINITY;
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int pos = sm.pos[warp][st][nt * 8 + 2 * tq + e];
        const bool oka = pos >= 0 && pos >= lo_a;
        const bool okb = pos >= 0 && pos >= lo_b;
        sacc[nt][e] = oka ? sacc[nt][e] * p.scale_log2 : -INFINITY;
        sacc[nt][2 + e] = okb ? sacc[nt][2 + e] * p.scale_log2 : -INFINITY;
        mx_a = fmaxf(mx_a, sacc[nt][e]);
        mx_b = fmaxf(mx_b, sacc[nt][2 + e]);
      }
    mx_a = fmaxf(mx_a, __shfl_xor_sync(0xffffffffu, mx_a, 1));
    mx_a = fmaxf(mx_a, __shfl_xor_sync(0xffffffffu, mx_a, 2));
    mx_b = fmaxf(mx_b, __shfl_xor_sync(0xffffffffu, mx_b, 1));
    mx_b = fmaxf(mx_b, __shfl_xor_sync(0xffffffffu, mx_b, 2));
    // the running max only moves up: rescale O and l when it does
    if (mx_a > m_a || mx_b > m_b) {
      const float na = fmaxf(m_a, mx_a), nb = fmaxf(m_b, mx_b);
      const float ra = m_a == -INFINITY ? 0.f : exp2f(m_a - na);
      const float rb = m_b == -INFINITY ? 0.f : exp2f(m_b - nb);
      m_a = na; m_b = nb;
      l_a *= ra; l_b *= rb;
#pragma unroll
      for (int nt = 0; nt < 16; ++nt) {
        o[nt][0] *= ra; o[nt][1] *= ra;
        o[nt][2] *= rb; o[nt][3] *= rb;
      }
    }
    const float base_a = m_a == -INFINITY ? 0.f : m_a, base_b = m_b == -INFINITY ? 0.f : m_b;
    uint32_t pa[4];                             // A fragment of P (16 rows x 16 keys)
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
      const float e0 = exp2f(sacc[nt][0] - base_a), e1 = exp2f(sacc[nt][1] - base_a);
      const float e2 = exp2f(sacc[nt][2] - base_b), e3 = exp2f(sacc[nt][3] - base_b);
      l_a += e0 + e1;
      l_b += e2 + e3;
      pa[nt * 2 + 0] = pack2(e0, e1);
      pa[nt * 2 + 1] = pack2(e2, e3);
    }
    // O += P V (16 rows x 128 dims)
    {
      const int m = lane >> 3;
      const int key = 8 * (m & 1) + (lane & 7);
#pragma unroll
      for (int np = 0; np < 8; ++np) {
        uint32_t bf[4];
        ldsm_x4_t(bf, vbase + slab_off(key, 2 * np + (m >> 1)));
        mma16816(o[2 * np], pa, bf[0], bf[1]);
        mma16816(o[2 * np + 1], pa, bf[2], bf[3]);
      }
    }
    __syncwarp();                                // stage st is free for chunk t + kStages
    ++piece_chunks;
  }
  cp_async_wait<0>();
  if (cur_id >= 0) flush();
}

// One CTA per (sequence, call head): combines the head's partials (kWarps
// per piece of its window segment, then of its gathered segment) and writes
// o. Warp w takes every kWarps-th partial, reading up to kMergeBatch of them
// with all loads in flight; the four warps then combine through shared memory.
__global__ void __launch_bounds__(128)
decode_merge_kernel(const DecodeParams p, int n_ctas, int* status) {
  __shared__ float wm[4], wl[4];
  __shared__ float4 wo[4][32];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  pdl_wait();                                 // the partials are complete
  if (blockIdx.x == 0 && threadIdx.x == 0) *status = 0;
  const int b = blockIdx.x / p.n_heads, j = blockIdx.x - b * p.n_heads;
  int n = n_pieces((b * p.n_ag + p.ag_of[j]) * p.n_wc, p.n_wc, p.n_win_chunks, n_ctas);
  if (j < p.n_ret) n += n_pieces((b * p.n_ret + j) * p.n_gc, p.n_gc, p.n_gat_chunks, n_ctas);
  n *= kWarps;
  const float* part = p.part + ((size_t)b * p.n_heads + j) * p.max_slots * kPartStride;
  float M = -INFINITY, Lsum = 0.f;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int s0 = warp; s0 < n; s0 += 4 * kMergeBatch) {
    float ms[kMergeBatch], ls[kMergeBatch];
    float4 os[kMergeBatch];
#pragma unroll
    for (int s = 0; s < kMergeBatch; ++s) {
      const int slot = s0 + 4 * s;
      if (slot < n) {
        const float* ps = part + (size_t)slot * kPartStride;
        ms[s] = ps[0];
        ls[s] = ps[1];
        os[s] = reinterpret_cast<const float4*>(ps + kPartO)[lane];
      } else {
        ms[s] = -INFINITY; ls[s] = 0.f; os[s] = make_float4(0.f, 0.f, 0.f, 0.f);
      }
    }
    float Mb = M;
#pragma unroll
    for (int s = 0; s < kMergeBatch; ++s) Mb = fmaxf(Mb, ms[s]);
    if (Mb == -INFINITY) continue;
    const float r = M == -INFINITY ? 0.f : exp2f(M - Mb);
    Lsum *= r; acc.x *= r; acc.y *= r; acc.z *= r; acc.w *= r;
#pragma unroll
    for (int s = 0; s < kMergeBatch; ++s) {
      const float wt = ms[s] == -INFINITY ? 0.f : exp2f(ms[s] - Mb);
      Lsum += wt * ls[s];
      acc.x += wt * os[s].x; acc.y += wt * os[s].y; acc.z += wt * os[s].z; acc.w += wt * os[s].w;
    }
    M = Mb;
  }
  if (lane == 0) { wm[warp] = M; wl[warp] = Lsum; }
  wo[warp][lane] = acc;
  __syncthreads();
  if (warp != 0) return;
  const float Mt = fmaxf(fmaxf(wm[0], wm[1]), fmaxf(wm[2], wm[3]));
  float Lt = 0.f;
  float4 at = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
  for (int w = 0; w < 4; ++w) {
    const float f = wm[w] == -INFINITY ? 0.f : exp2f(wm[w] - Mt);
    Lt += f * wl[w];
    const float4 v = wo[w][lane];
    at.x += f * v.x; at.y += f * v.y; at.z += f * v.z; at.w += f * v.w;
  }
  const float inv = 1.f / Lt;
  __nv_bfloat16* dst = p.o + (int64_t)b * p.o_sb + (int64_t)p.head[j] * p.o_sh + lane * 4;
  uint2 packed;
  packed.x = pack2(at.x * inv, at.y * inv);
  packed.y = pack2(at.z * inv, at.w * inv);
  *reinterpret_cast<uint2*>(dst) = packed;
}

namespace {
int n_gathered_chunks(int topk, int sink) { return (topk + sink + kChunk - 1) / kChunk; }
}  // namespace

size_t decode_attn_ws_bytes(int B, int L, int n_heads, int topk, int window) {
  // `window` bounds every head's window; the sink (at most kMaxSink tokens)
  // shares the selected list's chunks. A segment is split into at most as
  // many pieces as it has chunks.
  const int w = window < L ? window : L;
  const int n_wc = (w + kChunk - 1) / kChunk;
  const int n_gc = topk > 0 ? n_gathered_chunks(topk, kMaxSink) : 0;
  return kHeaderBytes +
         (size_t)B * n_heads * kWarps * (n_wc + n_gc) * kPartStride * sizeof(float);
}

cudaError_t launch_decode_hybrid(const void* q, int64_t q_sb, int64_t q_sh,
                                 const void* kc, int64_t k_sb, int64_t k_sn, int64_t k_sh,
                                 const void* vc, int64_t v_sb, int64_t v_sn, int64_t v_sh,
                                 void* o, int64_t o_sb, int64_t o_sh,
                                 int B, int L, int q_pos, int Hq, int Hkv,
                                 const int32_t* ret_heads, int n_ret, const int32_t* idx, int topk,
                                 int ret_window, int sink,
                                 const int32_t* swa_heads, int n_swa, int swa_window,
                                 float scale, void* ws, cudaStream_t stream, bool early_start, int max_ctas) {
  DecodeParams p;
  p.early_start = early_start ? 1 : 0;
  p.q = static_cast<const __nv_bfloat16*>(q); p.q_sb = q_sb; p.q_sh = q_sh;
  p.k = static_cast<const __nv_bfloat16*>(kc); p.k_sb = k_sb; p.k_sn = k_sn; p.k_sh = k_sh;
  p.v = static_cast<const __nv_bfloat16*>(vc); p.v_sb = v_sb; p.v_sn = v_sn; p.v_sh = v_sh;
  p.o = static_cast<__nv_bfloat16*>(o); p.o_sb = o_sb; p.o_sh = o_sh;
  p.B = B; p.G = Hq / Hkv;
  if (p.G > kMaxGroup || Hkv > kMaxGroup) return cudaErrorInvalidValue;
  p.idx = idx; p.topk = n_ret > 0 ? topk : 0; p.sink = sink;
  p.n_sel = p.topk < L ? p.topk : L;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.whi = q_pos + 1 < L ? q_pos + 1 : L;
  p.n_heads = n_ret + n_swa;
  p.n_ret = n_ret;
  int wlo_union = p.whi;
  for (int r = 0; r < n_ret; ++r) {
    p.head[r] = ret_heads[r];
    p.wlo[r] = q_pos - ret_window + 1 > 0 ? q_pos - ret_window + 1 : 0;
    wlo_union = p.wlo[r] < wlo_union ? p.wlo[r] : wlo_union;
  }
  for (int s = 0; s < n_swa; ++s) {
    const int j = n_ret + s;
    p.head[j] = swa_heads[s];
    p.wlo[j] = q_pos - swa_window + 1 > 0 ? q_pos - swa_window + 1 : 0;
    wlo_union = p.wlo[j] < wlo_union ? p.wlo[j] : wlo_union;
  }
  // active groups and their rows, in call-head order
  int group_to_ag[kMaxGroup];
  for (int g = 0; g < kMaxGroup; ++g) group_to_ag[g] = -1;
  p.n_ag = 0;
  for (int j = 0; j < p.n_heads; ++j) {
    const int g = p.head[j] / p.G;
    if (group_to_ag[g] < 0) {
      group_to_ag[g] = p.n_ag;
      p.ag_kv[p.n_ag] = g;
      p.ag_n[p.n_ag] = 0;
      ++p.n_ag;
    }
    const int a = group_to_ag[g];
    if (p.ag_n[a] >= kMaxGroup) return cudaErrorInvalidValue;
    p.ag_rows[a][p.ag_n[a]++] = j;
    p.ag_of[j] = a;
  }
  p.wlo_union = wlo_union;
  p.n_wc = (p.whi - wlo_union + kChunk - 1) / kChunk;
  p.n_gc = n_ret > 0 ? n_gathered_chunks(p.n_sel, sink) : 0;
  p.max_slots = kWarps * (p.n_wc + p.n_gc);
  p.n_win_chunks = B * p.n_ag * p.n_wc;
  p.n_gat_chunks = B * n_ret * p.n_gc;
  char* base = static_cast<char*>(ws);
  p.part = reinterpret_cast<float*>(base + kHeaderBytes);
  int* status = reinterpret_cast<int*>(base);
  cudaError_t e;
  if (p.n_win_chunks == 0) return cudaSuccess;
  int dev = 0, sms = 148;
  e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return e;
  // every CTA resident at once: two per SM, or the caller's bound (the CTAs
  // that fit beside the kernel still running before this one)
  const int most = p.n_win_chunks > p.n_gat_chunks ? p.n_win_chunks : p.n_gat_chunks;
  const int cap = max_ctas > 0 && max_ctas < kCtasPerSm * sms ? max_ctas : kCtasPerSm * sms;
  const int grid = most < cap ? most : cap;
  const size_t smem = sizeof(Smem);
  e = cudaFuncSetAttribute(decode_attn_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  // both kernels may start while their predecessor runs (with early_start the
  // attention streams its window chunks before it waits for the selected lists)
  e = launch_pdl(decode_attn_kernel, dim3(grid), dim3(kThreads), smem, stream, p);
  if (e != cudaSuccess) return e;
  e = launch_pdl(decode_merge_kernel, dim3(B * p.n_heads), dim3(128), 0, stream, p, grid, status);
  if (e != cudaSuccess) return e;
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
// Allocation-free variant: the workspace is a fixed device array.
// ---------------------------------------------------------------------------
// Every GPU that loads the library holds this array until the process exits.
// Host code must not pass `g_decode_scratch` itself to a kernel (on the host
// that name is only a stand-in); it uses the device address fetched below.
static __device__ __align__(256) float g_decode_scratch[kNoAllocScratchBytes / sizeof(float)];

namespace {
constexpr int kMaxDevices = 64;
struct ScratchSlot {
  void* ctx;     // the context the address belongs to
  void* ptr;     // device address of g_decode_scratch in that context
};
std::mutex g_scratch_mutex;
ScratchSlot g_scratch[kMaxDevices] = {};

// The current context, through the runtime's driver entry-point query (the
// library has no link-time dependency on libcuda). NULL if unavailable.
void* current_context() {
  using Fn = CUresult (*)(CUcontext*);
  static Fn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<Fn>(ptr);
  });
  CUcontext c = nullptr;
  if (!fn || fn(&c) != CUDA_SUCCESS) return nullptr;
  return c;
}
}  // namespace

// Device address of g_decode_scratch on the current device, looked up with
// that device current the first time a call runs on it, and again whenever the
// device's context has changed since (after a cudaDeviceReset the primary
// context, and the array's address with it, is new).
static cudaError_t decode_scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  // No context may be current yet on the first call: the lookup creates the
  // device's primary context, and the slot records the context it found.
  void* ctx = current_context();
  std::lock_guard<std::mutex> lock(g_scratch_mutex);
  ScratchSlot& slot = g_scratch[dev];
  if (!slot.ptr || !ctx || slot.ctx != ctx) {
    void* ptr = nullptr;
    e = cudaGetSymbolAddress(&ptr, g_decode_scratch);
    if (e != cudaSuccess) return e;
    slot.ptr = ptr;
    slot.ctx = current_context();
  }
  *out = slot.ptr;
  return cudaSuccess;
}

cudaError_t launch_decode_attn_noalloc(const void* q, int64_t q_sb, int64_t q_sh,
                                       const void* kc, int64_t k_sb, int64_t k_sn, int64_t k_sh,
                                       const void* vc, int64_t v_sb, int64_t v_sn, int64_t v_sh,
                                       void* o, int64_t o_sb, int64_t o_sh,
                                       int B, int L, int q_pos, int Hq, int Hkv,
                                       const int32_t* heads, int n_heads, const int32_t* idx, int topk,
                                       int window, int sink, float scale, cudaStream_t stream) {
  // Every partial the merge reads is written by the same call, and the merge
  // writes the status word.
  void* scratch = nullptr;
  cudaError_t e = decode_scratch_address(&scratch);
  if (e != cudaSuccess) return e;
  return launch_decode_attn(q, q_sb, q_sh, kc, k_sb, k_sn, k_sh, vc, v_sb, v_sn, v_sh, o, o_sb, o_sh, B, L,
                            q_pos, Hq, Hkv, heads, n_heads, 1, idx, topk, window, sink, scale, scratch, stream);
}

}  // namespace rtp
