// Shared device helpers for the head-wise hybrid attention kernels (sm_100a).
#pragma once
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#define RTP_D 128
#define RTP_R 16
#define RTP_BLOCK 64

namespace rtp {

// Maximum heads one call can name (head lists travel in kernel parameters).
constexpr int kMaxHeads = 128;

struct HeadList {
  int n;
  int head[kMaxHeads];   // query head index
  int kv[kMaxHeads];     // its KV head
};

// Programmatic dependent launch: a kernel launched with programmatic stream
// serialisation may start before the previous kernel of the stream has
// finished; pdl_wait() blocks the calling thread until that kernel has
// completed and its writes are visible (a no-op for a normal launch), and
// pdl_trigger() lets the next such kernel launch before this one ends.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// fp32 -> orderable uint32: a larger key is a larger float. -0 is folded to +0
// so that numerically equal scores tie (and the smaller index wins).
__device__ __forceinline__ uint32_t f2key(float f) {
  f = f + 0.0f;
  uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

template <int NT>
struct BlockScanSmem {
  int warp_tot[NT / 32];
  int total;
};

// Exclusive prefix sum of one int per thread across the block; also returns
// the block total. All threads must call it.
template <int NT>
__device__ __forceinline__ int block_exclusive_scan(int v, int& total, BlockScanSmem<NT>& sm) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) sm.warp_tot[warp] = x;
  __syncthreads();
  if (warp == 0) {
    int w = (lane < NT / 32) ? sm.warp_tot[lane] : 0;
    int incl = w;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    if (lane < NT / 32) sm.warp_tot[lane] = incl - w;
    if (lane == NT / 32 - 1) sm.total = incl;
  }
  __syncthreads();
  int res = sm.warp_tot[warp] + x - v;
  total = sm.total;
  __syncthreads();
  return res;
}

template <int NT>
struct TopkSmem {
  uint32_t hist[2048];
  BlockScanSmem<NT> scan;
  int digit, above;
};

// Block-wide radix search for the k-th largest 32-bit key among n elements
// (keys from get_key(i)), digits of 11, 11 and 10 bits from the top. Starting
// at `first_pass` with the bits of `prefix` under `mask` already fixed (the
// elements considered are those matching it), and `need` the number still to
// take from them. Returns the threshold key; on return `need` is how many
// elements equal to it are taken (the others above it are all taken).
template <int NT, class GetKey>
__device__ uint32_t block_radix_threshold(GetKey get_key, int n, int& need, TopkSmem<NT>& sm,
                                          int first_pass = 0, uint32_t prefix = 0, uint32_t mask = 0) {
  const int tid = threadIdx.x;
#pragma unroll 1
  for (int pass = first_pass; pass < 3; ++pass) {
    const int shift = pass == 0 ? 21 : (pass == 1 ? 10 : 0);
    const int nbins = pass == 2 ? 1024 : 2048;
    for (int b = tid; b < nbins; b += NT) sm.hist[b] = 0;
    __syncthreads();
    for (int i = tid; i < n; i += NT) {
      uint32_t key = get_key(i);
      if ((key & mask) == prefix) atomicAdd(&sm.hist[(key >> shift) & (nbins - 1)], 1u);
    }
    __syncthreads();
    // Thread t owns the bins [nbins-1 - t*per, ...] walking downwards.
    const int per = (nbins + NT - 1) / NT;
    int local = 0;
    for (int q = 0; q < per; ++q) {
      int b = nbins - 1 - (tid * per + q);
      if (b >= 0) local += sm.hist[b];
    }
    int tot;
    int above = block_exclusive_scan<NT>(local, tot, sm.scan);
    if (above < need && above + local >= need) {
      int run = above;
      for (int q = 0; q < per; ++q) {
        int b = nbins - 1 - (tid * per + q);
        if (b < 0) break;
        int c = sm.hist[b];
        if (run + c >= need) { sm.digit = b; sm.above = run; break; }
        run += c;
      }
    }
    __syncthreads();
    need -= sm.above;
    prefix |= (uint32_t)sm.digit << shift;
    mask |= (uint32_t)(nbins - 1) << shift;
    __syncthreads();
  }
  return prefix;
}

// Block-wide exact top-k by (key desc, index asc) over n elements whose keys
// come from get_key(i). Writes the selected indices in ascending order to
// out[0 .. min(k,n)), pads out[min(k,n) .. k) with -1: a radix search for the
// k-th key, then an ordered compaction that takes every key above it and the
// lowest-index keys equal to it.
template <int NT, class GetKey>
__device__ void block_topk_ascending(GetKey get_key, int n, int k, int32_t* __restrict__ out,
                                     TopkSmem<NT>& sm) {
  const int tid = threadIdx.x;
  if (n <= k) {
    for (int i = tid; i < k; i += NT) out[i] = (i < n) ? i : -1;
    return;
  }
  int need = k;
  const uint32_t thr = block_radix_threshold<NT>(get_key, n, need, sm);
  int eq_seen = 0, written = 0;
  for (int base = 0; base < n; base += NT) {
    int i = base + tid;
    uint32_t key = (i < n) ? get_key(i) : 0u;
    int eq = (i < n && key == thr) ? 1 : 0;
    int eq_tot;
    int eq_before = block_exclusive_scan<NT>(eq, eq_tot, sm.scan);
    int take = (i < n) && (key > thr || (eq && eq_seen + eq_before < need));
    int take_tot;
    int pos = block_exclusive_scan<NT>(take, take_tot, sm.scan);
    if (take) out[written + pos] = i;
    written += take_tot;
    eq_seen += eq_tot;
    if (written >= k) break;
  }
}

// Ascending bitonic sort of a[0 .. n) in shared memory, n a power of two.
template <int NT>
__device__ void block_bitonic_sort(int* a, int n) {
  for (int size = 2; size <= n; size <<= 1) {
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      for (int i = threadIdx.x; i < n / 2; i += NT) {
        const int lo = 2 * stride * (i / stride) + (i % stride), hi = lo + stride;
        const bool up = (lo & size) == 0;
        const int x = a[lo], y = a[hi];
        if ((x > y) == up) { a[lo] = y; a[hi] = x; }
      }
      __syncthreads();
    }
  }
}

}  // namespace rtp
