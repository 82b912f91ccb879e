// Parameters of the tensor-core prefill attention kernel.
//
// Streaming heads: the band of 64-key blocks overlapping (pos - W, pos] for
// the query positions of a tile, with a per-element window mask.
// Retrieval heads: the set {selected blocks} U {0 .. sink-1} U
// {i - window_blocks + 1 .. i} (RTPurbo digest: exact attention over the
// selected set; the tiny 2K prefill workload statement: top-k blocks plus key
// block 0 plus the window blocks), each block once; causal mask u <= pos.
// With no selection lists (counts == NULL) only the sink and window blocks
// are attended: the streaming region of the triangle-shaped mask.
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
  const int32_t* blocks;     // NULL with counts: no selected blocks
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

size_t prefill_attn_tc_smem_bytes(const PrefillAttnParams& p);
cudaError_t launch_prefill_attn_tc(const PrefillAttnParams& p, const CUtensorMap& tmQ, const CUtensorMap& tmK,
                                   const CUtensorMap& tmV, int n_tiles, int B, int* status, cudaStream_t stream);

}  // namespace rtp
