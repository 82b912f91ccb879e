// Key-block lists shared by the prefill attention kernels.
//
// Streaming heads: the band of 64-key blocks overlapping (pos - W, pos] for
// the 64 query positions of the block, with a per-element window mask.
// Retrieval heads: the set {selected blocks} U {0 .. sink-1} U
// {i - window_blocks + 1 .. i} (RTPurbo digest: exact attention over the
// selected set; the tiny 2K prefill workload statement: top-k blocks plus key
// block 0 plus the window blocks), built as a bitmap over the causal blocks
// 0..i so every block appears once whatever the order of the selected list,
// then compacted in ascending order; causal mask u <= pos.
#pragma once
#include "rtp_common.cuh"
#include "rtp_internal.h"

namespace rtp {

struct PrefillAttnParams {
  Tensor4 q, k, v;
  void* o;
  int64_t o_sb, o_sn, o_sh;
  int Nq, Nk, q_pos0, Hq, Hkv, G;
  int sparse;
  const int32_t* blocks;
  const int32_t* counts;
  int topk;
  int window_tokens, window_blocks, sink_blocks;
  float scale_log2;
  int n_heads;
  int bitmap_words;   // words of the block bitmap (sparse)
  int list_cap;       // capacity of the compacted list (sparse)
  int withhold_q;     // test hook: the producer never loads Q, so every wait must run out
  int head[kMaxHeads];
};

template <int NT>
struct BlockListSmem {
  BlockScanSmem<NT> scan;
  int kb_lo;
  unsigned* bits;
  int* list;
};

inline size_t block_list_bytes(const PrefillAttnParams& p) {
  return p.sparse ? (size_t)(p.bitmap_words + p.list_cap) * 4 : 0;
}

__device__ __forceinline__ bool key_allowed(const PrefillAttnParams& p, int u, int pos) {
  return u <= pos && (p.sparse || u > pos - p.window_tokens);
}

// Builds the key-block list of query block qb into smem; returns its length.
// The dynamic shared memory after the kernel's own struct holds the bitmap
// and the list (block_list_bytes). All threads must call it.
template <int NT>
__device__ int build_block_list(const PrefillAttnParams& p, int b, int j, int qb,
                                BlockListSmem<NT>& sm, unsigned char* extra) {
  const int tid = threadIdx.x;
  if (!p.sparse) {
    const int pos0 = p.q_pos0 + qb * RTP_BLOCK;
    const int lo = max(0, pos0 - p.window_tokens + 1) / RTP_BLOCK;
    const int hi = min(p.Nk - 1, pos0 + RTP_BLOCK - 1) / RTP_BLOCK;
    if (tid == 0) sm.kb_lo = lo;
    __syncthreads();
    return hi - lo + 1;
  }
  unsigned* bits = reinterpret_cast<unsigned*>(extra);
  int* list = reinterpret_cast<int*>(extra) + p.bitmap_words;
  const int i = qb;                       // sparse prefill: query block i, positions 64 i ..
  const int nw = (i + 32) / 32;           // words covering blocks 0..i
  for (int w = tid; w < nw; w += NT) bits[w] = 0u;
  __syncthreads();
  const int nb = p.Nq / RTP_BLOCK;
  const size_t row = ((size_t)b * p.n_heads + j) * nb + i;
  const int cnt = min(p.counts[row], p.topk);
  const int32_t* sel = p.blocks + row * p.topk;
  for (int e = tid; e < cnt; e += NT) {
    const int x = sel[e];
    if (x >= 0 && x <= i) atomicOr(&bits[x >> 5], 1u << (x & 31));
  }
  for (int x = tid; x < min(p.sink_blocks, i + 1); x += NT) atomicOr(&bits[x >> 5], 1u << (x & 31));
  for (int x = max(0, i - p.window_blocks + 1) + tid; x <= i; x += NT)
    atomicOr(&bits[x >> 5], 1u << (x & 31));
  __syncthreads();
  // Ordered compaction: thread t owns a contiguous run of words.
  const int per = (nw + NT - 1) / NT;
  const int w0 = tid * per, w1 = min(nw, w0 + per);
  int c = 0;
  for (int w = w0; w < w1; ++w) c += __popc(bits[w]);
  int total;
  int off = block_exclusive_scan<NT>(c, total, sm.scan);
  for (int w = w0; w < w1; ++w) {
    unsigned x = bits[w];
    while (x) {
      const int bit = __ffs(x) - 1;
      x &= x - 1;
      list[off++] = w * 32 + bit;
    }
  }
  sm.list = list;
  __syncthreads();
  return total;
}

template <int NT>
__device__ __forceinline__ int list_block(const PrefillAttnParams& p, const BlockListSmem<NT>& sm,
                                          int it, int qb) {
  (void)qb;
  return p.sparse ? sm.list[it] : sm.kb_lo + it;
}

size_t prefill_attn_tc_smem_bytes(const PrefillAttnParams& p);
cudaError_t launch_prefill_attn_tc(const PrefillAttnParams& p, const CUtensorMap& tmQ, const CUtensorMap& tmK,
                                   const CUtensorMap& tmV, int n_tiles, int B, int* status, cudaStream_t stream);

}  // namespace rtp
