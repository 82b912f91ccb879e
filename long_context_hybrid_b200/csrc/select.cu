// Decode token selection: every retrieval head scores every cached token by
// q~ . k~ (r = 16) and keeps its top-k tokens (the 128K decode workload
// statement: token-level top-2048 over the whole cache; RTPurbo digest: the
// 16-d indexer is the scout). Exact ties rank the smaller token first.
//
// Three kernels:
//   zero    clears the histograms and the per-row state; inside a decode step
//           it also forms q~ = q . P. The scan launches behind it at once
//           (programmatic dependent launch) and waits for it before its
//           first read.
//   scan    one pass over the key index by as many CTAs as fit on the GPU, each
//           a contiguous run of the (sequence, KV group) token ranges laid end
//           to end; a group's index is read once for all its retrieval heads
//           (grouped-query heads share keys), with evict-first loads. It
//           writes every score (fp32, to the workspace; they stay in L2) and
//           a histogram of the top 11 bits of each score's order-preserving
//           key.
//   filter  about one CTA per SM, several per (sequence, head), each over a
//           slice of the scores (the SMs keep room for the attention kernel
//           launched behind it, which streams the window meanwhile). From the
//           histogram every CTA knows the bin holding the k-th score (as float
//           bounds): it marks the scores above that bin in a per-row bitmap
//           (every 32-token word is owned by one CTA, so plain stores) and the
//           bin's members in a shared bitmap; the members are then compacted,
//           their keys read back, and appended to the row's candidate list
//           through a shared buffer. The last CTA of a row to
//           finish loads the candidates into shared memory, settles the bin by
//           a radix search over their remaining bits (exact ties: smallest
//           token first), sets their bits and compacts the bitmap into the
//           ascending index list. Larger candidate lists are searched in
//           global memory; if they overflow the list, a full radix select over
//           the row runs instead.
#include "rtp_common.cuh"
#include "rtp_internal.h"

namespace rtp {

namespace {
constexpr int kScanThreads = 256;
constexpr int kScanBatch = 8;
constexpr int kMaxGroups = 16;                                      // KV groups
constexpr int kMaxHeadsPerGroup = 16;                               // retrieval heads of one group
constexpr int kBins = 2048;                                        // top 11 bits
constexpr int kFiltThreads = 512;
constexpr int kFiltStep = kFiltThreads * 16;                       // scores per CTA step
constexpr int kLocCap = 4096;                                      // shared slots for a CTA's candidates
constexpr int kSmemCand = 4096;                                    // shared slots for a row's candidates
constexpr int kSmemWords = 4096;                                   // shared bitmap words (rows up to 128K)

// Per-row bookkeeping of the filter kernel (zeroed with the histogram).
struct RowState {
  int n_cand;      // filter: candidates appended
  int ticket;      // filter: CTAs done
  int pad[2];
};

// Candidate-list capacity per row: an eighth of the row, at least 8192.
__host__ __device__ inline int cand_cap(int L) { return L / 8 > 8192 ? L / 8 : 8192; }

// Smallest float whose order-preserving key (f2key) is >= K: a score x has
// f2key(x) >= K iff x >= key_floor_float(K) (for non-NaN x; -0 and +0 share
// a key and compare equal).
__device__ __forceinline__ float key_floor_float(uint32_t K) {
  return __uint_as_float((K & 0x80000000u) ? (K & 0x7fffffffu) : ~K);
}

struct DecodeWs {
  float* scores;          // [B, Hr, L]
  uint32_t* hist;         // [B, Hr, kBins]: top 11 key bits of every score
  RowState* state;        // [B, Hr]      (zeroed together with hist)
  uint32_t* bitmap;       // [B, Hr, ceil(L / 32)]
  uint2* cand;            // [B, Hr, cand_cap(L)] (key, token)
  size_t zero_bytes;      // hist + state
  size_t total;
};

inline size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

DecodeWs decode_ws_layout(void* base, int B, int L, int Hr) {
  const size_t rows = (size_t)B * Hr;
  DecodeWs w;
  char* p = static_cast<char*>(base);
  size_t off = 0;
  w.scores = reinterpret_cast<float*>(p + off);
  off = align256(off + rows * L * sizeof(float));
  w.hist = reinterpret_cast<uint32_t*>(p + off);
  w.state = reinterpret_cast<RowState*>(p + off + rows * kBins * sizeof(uint32_t));
  w.zero_bytes = rows * (kBins * sizeof(uint32_t) + sizeof(RowState));
  off = align256(off + w.zero_bytes);
  w.bitmap = reinterpret_cast<uint32_t*>(p + off);
  off = align256(off + rows * ((L + 31) / 32) * sizeof(uint32_t));
  w.cand = reinterpret_cast<uint2*>(p + off);
  off = align256(off + rows * cand_cap(L) * sizeof(uint2));
  w.total = off;
  return w;
}

// Bin (top 11 key bits) of the k-th largest score of a row from its histogram,
// and how many scores lie in higher bins. All threads get the result.
template <int NT, class SM>
__device__ void kth_bin(const uint32_t* __restrict__ h, int k, SM& sm, uint32_t& bin, int& above) {
  const int tid = threadIdx.x;
  constexpr int per = kBins / NT;
  int local = 0;
  uint32_t c[per];
#pragma unroll
  for (int q = 0; q < per; ++q) {
    c[q] = __ldcg(h + kBins - 1 - (tid * per + q));
    local += c[q];
  }
  int tot;
  const int ab = block_exclusive_scan<NT>(local, tot, sm.scan);
  if (ab < k && ab + local >= k) {
    int run = ab;
#pragma unroll
    for (int q = 0; q < per; ++q) {
      if (run + (int)c[q] >= k) { sm.digit = kBins - 1 - (tid * per + q); sm.above = run; break; }
      run += c[q];
    }
  }
  __syncthreads();
  bin = (uint32_t)sm.digit;
  above = sm.above;
  __syncthreads();
}
}  // namespace

// Retrieval heads served by each KV group (call-head indices), and the
// groups serving at least one (the active groups) in order.
struct GroupHeads {
  int n[kMaxGroups];
  int j[kMaxGroups][kMaxHeadsPerGroup];
  int n_ag;
  int ag[kMaxGroups];
};


// Persistent scan: the CTAs split the tokens of every (sequence, active
// group) pair, laid end to end, into contiguous equal runs. Over each piece
// of a pair a CTA scores the tokens for the group's retrieval heads and
// histograms the top 11 key bits in shared memory, then adds the histogram to
// the row's. MAXJ > 0: the group's q~ rows sit in
// registers (at most MAXJ heads per group); MAXJ == 0: any number, read from
// shared memory. Each thread keeps the loads of BATCH tokens in flight.
// Q8: tokens of full 64-token groups are scored from the 8-bit index (one
// 16-byte row of codes per token, score = scale * sum q_c code_c), the rest
// (the partial last group) from the bf16 rows.
template <int MAXJ, int BATCH, bool Q8>
__global__ void __launch_bounds__(kScanThreads)
decode_scan_kernel(const float* __restrict__ qt, const IndexRef index, int B, int L,
                   int Hr, int Hkv, const GroupHeads gh, const DecodeWs w) {
  const uint4* __restrict__ kindex = static_cast<const uint4*>(index.bf16);
  const int64_t kcap = index.cap;
  const int ufull = Q8 ? (L / QGROUP_TOKENS) * QGROUP_TOKENS : 0;   // tokens read from the codes
  const int64_t ngroups = (kcap + QGROUP_TOKENS - 1) / QGROUP_TOKENS;
  pdl_trigger();                                       // the filter may launch and wait for this grid
  // q~ and the cleared histograms come from the previous kernel. With a few
  // heads per group (MAXJ > 0) the scan waits for it first, so that its small
  // loads are not queued behind the scan's; with many (MAXJ == 0: long,
  // compute-heavy runs) the first batch of index loads goes out before the
  // wait (128K x 8: 96.3 against 92.2 us; 64K x 32: 483 against 551 us).
  bool waited = false;
  if constexpr (MAXJ > 0) {
    pdl_wait();
    waited = true;
  }
  extern __shared__ uint32_t shist[];                  // [heads of the group][kBins]
  __shared__ float qs[MAXJ > 0 ? 1 : kMaxHeadsPerGroup][RTP_R];
  const int64_t total = (int64_t)B * gh.n_ag * L;
  const int64_t x0 = total * blockIdx.x / gridDim.x, x1 = total * (blockIdx.x + 1) / gridDim.x;
  constexpr int QJ = MAXJ > 0 ? MAXJ : 1;
  for (int64_t x = x0; x < x1;) {
    const int seg = (int)(x / L);
    const int u0 = (int)(x - (int64_t)seg * L);
    const int64_t rem = x1 - x;
    const int u1 = rem < (int64_t)(L - u0) ? u0 + (int)rem : L;
    const int b = seg / gh.n_ag, g = gh.ag[seg - b * gh.n_ag];
    const int n = gh.n[g];
    float q[QJ][RTP_R];
    float* srow[QJ];
    if constexpr (MAXJ > 0) {
#pragma unroll
      for (int jj = 0; jj < MAXJ; ++jj) {
        const int j = jj < n ? gh.j[g][jj] : gh.j[g][0];
#pragma unroll
        for (int c = 0; c < RTP_R; ++c) q[jj][c] = __ldg(qt + ((size_t)b * Hr + j) * RTP_R + c);
        srow[jj] = w.scores + ((size_t)b * Hr + j) * L;
      }
    }
    bool q_loaded = MAXJ > 0;                          // MAXJ == 0: q~ rows after the first loads
    for (int e = threadIdx.x; e < n * kBins; e += kScanThreads) shist[e] = 0u;
    __syncthreads();
    const uint4* krow = kindex + ((size_t)b * Hkv + g) * (size_t)kcap * 2;
    const uint4* k8row = Q8 ? static_cast<const uint4*>(index.k8) + ((size_t)b * Hkv + g) * (size_t)kcap : nullptr;
    const float* srow_scale = Q8 ? index.scale + ((size_t)b * Hkv + g) * (size_t)ngroups : nullptr;
#pragma unroll 1
    for (int base = u0; base < u1; base += kScanThreads * BATCH) {
      uint4 lo[BATCH], hi[BATCH];
#pragma unroll
      for (int t = 0; t < BATCH; ++t) {
        const int u = base + t * kScanThreads + threadIdx.x;
        if (u < u1) {
          // read once: evict-first, so that the scores stay in L2 for the filter
          if (Q8 && u < ufull) {
            lo[t] = __ldcs(k8row + u);
          } else {
            lo[t] = __ldcs(krow + (size_t)u * 2);
            hi[t] = __ldcs(krow + (size_t)u * 2 + 1);
          }
        }
      }
      if (!q_loaded) {
        if (!waited) { pdl_wait(); waited = true; }
        for (int e = threadIdx.x; e < n * RTP_R; e += kScanThreads)
          qs[e / RTP_R][e % RTP_R] = __ldg(qt + ((size_t)b * Hr + gh.j[g][e / RTP_R]) * RTP_R + e % RTP_R);
        __syncthreads();
        q_loaded = true;
      }
#pragma unroll
      for (int t = 0; t < BATCH; ++t) {
        const int u = base + t * kScanThreads + threadIdx.x;
        if (u >= u1) break;
        float k[16];
        float ks = 1.f;
        if (Q8 && u < ufull) {
          const uint32_t v4[4] = {lo[t].x, lo[t].y, lo[t].z, lo[t].w};
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            k[4 * i + 0] = (float)((int32_t)(v4[i] << 24) >> 24);
            k[4 * i + 1] = (float)((int32_t)(v4[i] << 16) >> 24);
            k[4 * i + 2] = (float)((int32_t)(v4[i] << 8) >> 24);
            k[4 * i + 3] = (float)((int32_t)v4[i] >> 24);
          }
          ks = __ldg(srow_scale + (u / QGROUP_TOKENS));
        } else {
          const uint32_t v8[8] = {lo[t].x, lo[t].y, lo[t].z, lo[t].w, hi[t].x, hi[t].y, hi[t].z, hi[t].w};
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            k[2 * i] = bf16_lo(v8[i]);
            k[2 * i + 1] = bf16_hi(v8[i]);
          }
        }
        if constexpr (MAXJ > 0) {
#pragma unroll
          for (int jj = 0; jj < MAXJ; ++jj) {
            if (jj >= n) break;
            float acc = 0.f;
#pragma unroll
            for (int c = 0; c < RTP_R; ++c) acc = fmaf(q[jj][c], k[c], acc);
            if (Q8) acc *= ks;
            srow[jj][u] = acc;
            atomicAdd(&shist[jj * kBins + (f2key(acc) >> 21)], 1u);
          }
        } else {
          for (int jj = 0; jj < n; ++jj) {
            float acc = 0.f;
#pragma unroll
            for (int c = 0; c < RTP_R; ++c) acc = fmaf(qs[jj][c], k[c], acc);
            if (Q8) acc *= ks;
            w.scores[((size_t)b * Hr + gh.j[g][jj]) * L + u] = acc;
            atomicAdd(&shist[jj * kBins + (f2key(acc) >> 21)], 1u);
          }
        }
      }
    }
    __syncthreads();
    for (int e = threadIdx.x; e < n * kBins; e += kScanThreads) {
      const uint32_t c = shist[e];
      if (c) atomicAdd(&w.hist[((size_t)b * Hr + gh.j[g][e / kBins]) * kBins + (e % kBins)], c);
    }
    x += u1 - u0;
  }
}

struct FiltSmem {
  TopkSmem<kFiltThreads> tk;
  union {
    uint2 loc[kLocCap];                         // phase A: this CTA's candidates
    uint2 all[kSmemCand];                       // phase B: the row's candidates
  } cbuf;
  uint32_t bits[kSmemWords];                    // phase B: the row's bitmap
  uint2 fin[32];                                // phase B: the k-th score's 22-bit bin
  int s_last, n_loc, s_base, n_fin;
};

__global__ void __launch_bounds__(kFiltThreads, 2)
decode_filter_kernel(const DecodeWs w, int L, int Hr, int topk, int slice, int n_split, int32_t* __restrict__ idx) {
  extern __shared__ __align__(16) unsigned char filt_smem[];
  FiltSmem& fs = *reinterpret_cast<FiltSmem*>(filt_smem);
  TopkSmem<kFiltThreads>& sm = fs.tk;
  uint2* loc = fs.cbuf.loc;
  int& s_last = fs.s_last;
  int& n_loc = fs.n_loc;
  int& s_base = fs.s_base;
  const int part = blockIdx.x, j = blockIdx.y, b = blockIdx.z, tid = threadIdx.x;
  const int lane = tid & 31, warp = tid >> 5;
  const size_t row = (size_t)b * Hr + j;
  int32_t* out = idx + row * topk;
  pdl_trigger();          // the attention may launch: it waits for this grid before reading idx
  pdl_wait();             // the scan's scores and histogram are complete
  if (L <= topk) {
    if (part == 0)
      for (int i = tid; i < topk; i += kFiltThreads) out[i] = i < L ? i : -1;
    return;
  }
  const float* s = w.scores + row * L;
  const int W = (L + 31) >> 5;
  const int cap = cand_cap(L);
  uint32_t* bm = w.bitmap + row * W;
  uint2* cand = w.cand + row * cap;
  uint32_t d1;
  int above1;
  kth_bin<kFiltThreads>(w.hist + row * kBins, topk, sm, d1, above1);
  if (tid == 0) n_loc = 0;
  __syncthreads();

  // A. this CTA's slice, two steps of 512 scores per warp at a time (all
  //    loads in flight together): the row's bitmap words for the scores above
  //    bin d1, and a shared bitmap of the bin's members. A lane takes 16
  //    consecutive scores; lanes 2m, 2m+1 share one bitmap word. Then the
  //    members' tokens are compacted into a shared buffer (in token order),
  //    their keys read back with all loads in flight, and the buffer goes to
  //    the row's candidate list with one reservation.
  const int lo = part * slice, hi = min(L, lo + slice);
  const bool vec = (L & 3) == 0;
  uint32_t* ibits = fs.bits;                    // phase A: the bin's members of this slice (phase B reuses it)
  // bin d1 as float bounds: a score is in the bin iff lo_f <= x < hi_f
  // (no score lies above the top bin: hi_f is then NaN)
  const float lo_f = key_floor_float(d1 << 21);
  const float hi_f = d1 < 2047u ? key_floor_float((d1 + 1u) << 21) : __int_as_float(0x7fc00000);
  for (int wb0 = lo + warp * 512; wb0 < hi; wb0 += 2 * kFiltStep) {
    float x[2][16];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int base = wb0 + h * kFiltStep + lane * 16;
      if (vec && base + 16 <= hi) {
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const float4 v = __ldg(reinterpret_cast<const float4*>(s + base) + q);
          x[h][4 * q] = v.x; x[h][4 * q + 1] = v.y; x[h][4 * q + 2] = v.z; x[h][4 * q + 3] = v.w;
        }
      } else {
#pragma unroll
        for (int e = 0; e < 16; ++e) x[h][e] = base + e < hi ? __ldg(s + base + e) : 0.f;
      }
    }
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int base = wb0 + h * kFiltStep + lane * 16;
      uint32_t bits = 0, cbits = 0;
#pragma unroll
      for (int e = 0; e < 16; ++e) {
        const bool above = x[h][e] >= hi_f, in_bin = x[h][e] >= lo_f;
        bits |= above ? 1u << e : 0u;
        cbits |= (in_bin && !above) ? 1u << e : 0u;
      }
      if (base + 16 > hi) {
        const uint32_t valid = base >= hi ? 0u : (1u << (hi - base)) - 1u;
        bits &= valid;
        cbits &= valid;
      }
      uint32_t word = bits << ((lane & 1) * 16), cword = cbits << ((lane & 1) * 16);
      word |= __shfl_xor_sync(0xffffffffu, word, 1);
      cword |= __shfl_xor_sync(0xffffffffu, cword, 1);
      if (!(lane & 1) && base < hi) {
        bm[base >> 5] = word;
        ibits[(base - lo) >> 5] = cword;
      }
    }
  }
  __syncthreads();
  {
    // members' tokens, word by word (the loop bound is warp-uniform: the
    // lanes exchange counts)
    const int n_words = (hi - lo + 31) >> 5;
    for (int wbase = warp * 32; wbase < n_words; wbase += kFiltThreads) {
      const int wi = wbase + lane;
      uint32_t cw = wi < n_words ? ibits[wi] : 0u;
      const int nc = __popc(cw);
      int incl = nc;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      const int wtot = __shfl_sync(0xffffffffu, incl, 31);
      int cbase = 0;
      if (lane == 31 && wtot > 0) cbase = atomicAdd(&n_loc, wtot);
      cbase = __shfl_sync(0xffffffffu, cbase, 31);
      int pos = cbase + incl - nc;
      while (cw) {
        const int e = __ffs(cw) - 1;
        cw &= cw - 1;
        const uint32_t tok = (uint32_t)(lo + wi * 32 + e);
        if (pos < kLocCap) loc[pos].y = tok;
        else {
          // the shared buffer is full: straight to the row's list
          const int gp = atomicAdd(&w.state[row].n_cand, 1);
          if (gp < cap) cand[gp] = make_uint2(f2key(__ldcg(s + tok)), tok);
        }
        ++pos;
      }
    }
    __syncthreads();
    // the members' keys, all loads of a thread in flight
    const int n_l = min(n_loc, kLocCap);
    constexpr int kPer = kLocCap / kFiltThreads;
    float v[kPer];
#pragma unroll
    for (int t = 0; t < kPer; ++t) {
      const int xx = tid + t * kFiltThreads;
      v[t] = xx < n_l ? __ldcg(s + loc[xx].y) : 0.f;
    }
#pragma unroll
    for (int t = 0; t < kPer; ++t) {
      const int xx = tid + t * kFiltThreads;
      if (xx < n_l) loc[xx].x = f2key(v[t]);
    }
  }
  __syncthreads();
  {
    const int n_l = min(n_loc, kLocCap);
    if (tid == 0 && n_l > 0) s_base = atomicAdd(&w.state[row].n_cand, n_l);
    __syncthreads();
    const int gb = s_base;
    for (int x = tid; x < n_l; x += kFiltThreads)
      if (gb + x < cap) cand[gb + x] = loc[x];
  }

  // B. the last CTA of the row settles the bin and writes the list
  __threadfence();
  __syncthreads();
  if (tid == 0) s_last = atomicAdd(&w.state[row].ticket, 1) == n_split - 1;
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  const int n_cand = __ldcg(&w.state[row].n_cand);
  if (n_cand > cap) {
    // candidates overflowed: exact radix select over the whole row
    auto key_of = [s](int i) { return f2key(__ldg(s + i)); };
    block_topk_ascending<kFiltThreads>(key_of, L, topk, out, sm);
    return;
  }
  int need = topk - above1;
  const uint2* cc = cand;
  // the row's bitmap (when it fits) and candidates (when they fit) into
  // shared memory, all loads of a thread in flight together
  const bool sbits = W <= kSmemWords, scand = n_cand <= kSmemCand;
  uint2* cs = fs.cbuf.all;
  {
    const int nw = sbits ? W : 0, nc = scand ? n_cand : 0;
    for (int x0 = 0; x0 < max(nw, nc); x0 += kFiltThreads * 8) {
      uint32_t wv[8];
      uint2 e[8];
#pragma unroll
      for (int t = 0; t < 8; ++t) {
        const int x = x0 + t * kFiltThreads + tid;
        wv[t] = x < nw ? __ldcg(bm + x) : 0u;
        e[t] = x < nc ? __ldcg(cc + x) : make_uint2(0u, 0u);
      }
#pragma unroll
      for (int t = 0; t < 8; ++t) {
        const int x = x0 + t * kFiltThreads + tid;
        if (x < nw) fs.bits[x] = wv[t];
        if (x < nc) cs[x] = e[t];
      }
    }
  }
  if (tid == 0) fs.n_fin = 0;
  __syncthreads();
  auto take = [&](uint32_t tok) {
    if (sbits) atomicOr(&fs.bits[tok >> 5], 1u << (tok & 31));
    else atomicOr(bm + (tok >> 5), 1u << (tok & 31));
  };
  // the bin's members, from shared memory when they fit
  auto ckey = [&](int x) { return scand ? cs[x].x : __ldcg(&cc[x].x); };
  auto ctok = [&](int x) { return scand ? cs[x].y : __ldcg(&cc[x].y); };
  // pass 1: key bits 20..10 of the members -> the k-th score's 22-bit bin
  for (int x = tid; x < kBins; x += kFiltThreads) sm.hist[x] = 0u;
  __syncthreads();
  for (int x = tid; x < n_cand; x += kFiltThreads) atomicAdd(&sm.hist[(ckey(x) >> 10) & 2047u], 1u);
  __syncthreads();
  uint32_t d2;
  int above2;
  {
    constexpr int per = kBins / kFiltThreads;
    int local = 0;
    uint32_t c[per];
#pragma unroll
    for (int q = 0; q < per; ++q) {
      c[q] = sm.hist[kBins - 1 - (tid * per + q)];
      local += c[q];
    }
    int tot;
    const int ab = block_exclusive_scan<kFiltThreads>(local, tot, sm.scan);
    if (ab < need && ab + local >= need) {
      int run = ab;
#pragma unroll
      for (int q = 0; q < per; ++q) {
        if (run + (int)c[q] >= need) { sm.digit = kBins - 1 - (tid * per + q); sm.above = run; break; }
        run += c[q];
      }
    }
    __syncthreads();
    d2 = (uint32_t)sm.digit;
    above2 = sm.above;
  }
  const uint32_t pre22 = (d1 << 11) | d2;
  need -= above2;
  // members above the 22-bit bin are taken; the bin's own are gathered
  for (int x = tid; x < n_cand; x += kFiltThreads) {
    const uint32_t k = ckey(x), d = k >> 10;
    if (d > pre22) take(ctok(x));
    else if (d == pre22) {
      const int p = atomicAdd(&fs.n_fin, 1);
      if (p < 32) fs.fin[p] = make_uint2(k, ctok(x));
    }
  }
  __syncthreads();
  const int m = fs.n_fin;
  if (m <= 32) {
    // one warp ranks the bin's members: by key, then smaller token first
    if (warp == 0 && lane < m) {
      const uint2 me = fs.fin[lane];
      int rank = 0;
      for (int y = 0; y < m; ++y) {
        const uint2 o = fs.fin[y];
        rank += (o.x > me.x) || (o.x == me.x && o.y < me.y);
      }
      if (rank < need) take(me.y);
    }
  } else {
    // a crowded bin: radix over the last 10 bits, then the smallest tokens
    // among keys equal to the threshold
    const uint32_t thr = block_radix_threshold<kFiltThreads>(ckey, n_cand, need, sm, 2, pre22 << 10,
                                                              0x3FFFFFu << 10);
    int n_eq = 0;
    for (int x = tid; x < n_cand; x += kFiltThreads) n_eq += ckey(x) == thr;
    int eq_tot;
    block_exclusive_scan<kFiltThreads>(n_eq, eq_tot, sm.scan);
    uint32_t tie_thr = 0;   // on ~token: larger means smaller token
    if (need < eq_tot) {
      int need2 = need;
      auto tkey = [&](int x) { return ckey(x) == thr ? ~ctok(x) : 0u; };
      tie_thr = block_radix_threshold<kFiltThreads>(tkey, n_cand, need2, sm);
    }
    for (int x = tid; x < n_cand; x += kFiltThreads) {
      const uint32_t k = ckey(x);
      if ((k >> 10) != pre22) continue;
      if (k > thr || (k == thr && ~ctok(x) >= tie_thr)) take(ctok(x));
    }
  }
  __syncthreads();
  // 3. ordered compaction of the bitmap: ascending token indices (a thread
  //    holds `per` consecutive words)
  const int per = (W + kFiltThreads - 1) / kFiltThreads;
  auto word = [&](int wi) { return sbits ? fs.bits[wi] : __ldcg(bm + wi); };
  int cnt = 0;
  for (int q = 0; q < per; ++q) {
    const int wi = tid * per + q;
    if (wi < W) cnt += __popc(word(wi));
  }
  int tot;
  int pos = block_exclusive_scan<kFiltThreads>(cnt, tot, sm.scan);
  for (int q = 0; q < per; ++q) {
    const int wi = tid * per + q;
    if (wi >= W) break;
    uint32_t v = word(wi);
    while (v) {
      const int bit = __ffs(v) - 1;
      v &= v - 1;
      if (pos < topk) out[pos] = wi * 32 + bit;
      ++pos;
    }
  }
}

size_t select_decode_ws_bytes(int B, int L, int Hr, int topk) {
  (void)topk;
  return decode_ws_layout(nullptr, B, L, Hr).total;
}

// Clears the selection's histograms and row state and, inside a decode step,
// forms q~ = q . P for the retrieval heads (CTA i < B*Hr forms row i: fp32
// FMAs over d = 0 .. D-1 in order, as the standalone projection does). The
// scan launches behind it at once and waits for it before its first read.
struct ZeroParams {
  uint4* p;
  size_t n16;
  float* qt;                  // [B, Hr, R] out (when q is given)
  int B, Hr;
  DecodeQuery dq;
  int kv[kDecodeQueryHeads];  // KV group of each retrieval head
};

__global__ void __launch_bounds__(256) decode_zero_kernel(const ZeroParams zp) {
  __shared__ __align__(16) __nv_bfloat16 sP[RTP_D * RTP_R];
  __shared__ __align__(16) __nv_bfloat16 sq[RTP_D];
  pdl_trigger();
  const int tid = threadIdx.x;
  if (zp.dq.q && blockIdx.x < (unsigned)(zp.B * zp.Hr)) {
    const int b = blockIdx.x / zp.Hr, j = blockIdx.x - b * zp.Hr;
    const uint4* Pg = static_cast<const uint4*>(zp.dq.P) + (size_t)zp.kv[j] * (RTP_D * RTP_R / 8);
    reinterpret_cast<uint4*>(sP)[tid] = __ldg(Pg + tid);                  // 256 x 16 B = D x R bf16
    if (tid < RTP_D / 8) {
      const __nv_bfloat16* qr = static_cast<const __nv_bfloat16*>(zp.dq.q) + (int64_t)b * zp.dq.q_sb +
                                (int64_t)zp.dq.qhead[j] * zp.dq.q_sh;
      reinterpret_cast<uint4*>(sq)[tid] = __ldg(reinterpret_cast<const uint4*>(qr) + tid);
    }
    __syncthreads();
    if (tid < RTP_R) {
      float acc = 0.f;
#pragma unroll 16
      for (int d = 0; d < RTP_D; ++d) acc = fmaf(__bfloat162float(sq[d]), __bfloat162float(sP[d * RTP_R + tid]), acc);
      zp.qt[(size_t)blockIdx.x * RTP_R + tid] = acc;
    }
  }
  for (size_t e = (size_t)blockIdx.x * 256 + tid; e < zp.n16; e += (size_t)gridDim.x * 256)
    zp.p[e] = make_uint4(0u, 0u, 0u, 0u);
}

cudaError_t launch_select_decode(const float* qt, const DecodeQuery* dq, float* qt_out, IndexRef index, int B,
                                 int L, int Hr, int Hkv, const int32_t* kv_of, int topk, int32_t* idx, void* ws,
                                 cudaStream_t stream, int* filter_ctas) {
  if (topk > kMaxDecodeTopk) return cudaErrorInvalidValue;
  if (Hkv > kMaxGroups) return cudaErrorInvalidValue;
  GroupHeads gh;
  int max_nj = 0;
  gh.n_ag = 0;
  for (int g = 0; g < Hkv; ++g) {
    int c = 0;
    for (int j = 0; j < Hr; ++j)
      if (kv_of[j] == g) {
        if (c >= kMaxHeadsPerGroup) return cudaErrorInvalidValue;
        gh.j[g][c++] = j;
      }
    gh.n[g] = c;
    if (c > 0) gh.ag[gh.n_ag++] = g;
    max_nj = c > max_nj ? c : max_nj;
  }
  const DecodeWs w = decode_ws_layout(ws, B, L, Hr);
  int dev = 0, sms = 148;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return e;
  {
    ZeroParams zp;
    zp.p = reinterpret_cast<uint4*>(w.hist);
    zp.n16 = w.zero_bytes / 16;
    zp.qt = qt_out;
    zp.B = B;
    zp.Hr = Hr;
    if (dq) {
      zp.dq = *dq;
      for (int j = 0; j < Hr; ++j) zp.kv[j] = kv_of[j];
      qt = qt_out;
    } else {
      zp.dq.q = nullptr;
      zp.dq.P = nullptr;
      zp.dq.q_sb = zp.dq.q_sh = 0;
    }
    size_t gz = (zp.n16 + 255) / 256;
    if (gz > (size_t)sms) gz = sms;
    if (dq && gz < (size_t)B * Hr) gz = (size_t)B * Hr;
    if (gz < 1) gz = 1;
    decode_zero_kernel<<<(unsigned)gz, 256, 0, stream>>>(zp);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  // scan: as many CTAs as fit on the GPU at once, each a contiguous run
  const size_t scan_smem = (size_t)max_nj * kBins * sizeof(uint32_t);
  const int64_t total = (int64_t)B * gh.n_ag * L;
  auto scan = [&](auto kernel) -> cudaError_t {
    cudaError_t e2 = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)scan_smem);
    if (e2 != cudaSuccess) return e2;
    int per_sm = 0;
    e2 = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, kScanThreads, scan_smem);
    if (e2 != cudaSuccess) return e2;
    int64_t grid = (int64_t)(per_sm > 0 ? per_sm : 1) * sms;
    const int64_t min_tokens = kScanThreads * kScanBatch;   // at least one batch of tokens per CTA
    if (grid * min_tokens > total) grid = (total + min_tokens - 1) / min_tokens;
    return launch_pdl(kernel, dim3((unsigned)grid), dim3(kScanThreads), scan_smem, stream, qt, index, B, L, Hr, Hkv, gh,
                      w);
  };
  if (index.k8) {
    if (max_nj <= 1) e = scan(decode_scan_kernel<1, kScanBatch, true>);
    else if (max_nj <= 2) e = scan(decode_scan_kernel<2, kScanBatch, true>);
    else if (max_nj <= 4) e = scan(decode_scan_kernel<4, kScanBatch, true>);
    else e = scan(decode_scan_kernel<0, kScanBatch, true>);
  } else {
    if (max_nj <= 1) e = scan(decode_scan_kernel<1, kScanBatch, false>);
    else if (max_nj <= 2) e = scan(decode_scan_kernel<2, kScanBatch, false>);
    else if (max_nj <= 4) e = scan(decode_scan_kernel<4, kScanBatch, false>);
    else e = scan(decode_scan_kernel<0, kScanBatch, false>);
  }
  if (e != cudaSuccess) return e;
  // filter: one wave of CTAs over all rows; slices are whole CTA steps
  e = cudaFuncSetAttribute(decode_filter_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sizeof(FiltSmem));
  if (e != cudaSuccess) return e;
  int per_sm = 0;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, decode_filter_kernel, kFiltThreads, sizeof(FiltSmem));
  if (e != cudaSuccess) return e;
  // about one filter CTA per SM, so that the attention launched behind the
  // filter finds room to start streaming the window while the filter runs;
  // a slice fits the shared bitmap of its bin members
  const int rows = B * Hr;
  (void)per_sm;
  int n_split = sms / rows;
  const int min_split = (L + kSmemWords * 32 - 1) / (kSmemWords * 32);
  if (n_split < min_split) n_split = min_split;
  if (n_split < 1) n_split = 1;
  int slice = (L + n_split - 1) / n_split;
  slice = (slice + 511) / 512 * 512;
  n_split = (L + slice - 1) / slice;
  dim3 g2(n_split, Hr, B);
  if (filter_ctas) *filter_ctas = n_split * rows;
  return launch_pdl(decode_filter_kernel, g2, dim3(kFiltThreads), sizeof(FiltSmem), stream, w, L, Hr, topk, slice,
                    n_split, idx);
}

}  // namespace rtp
