// select_block.cuh -- radix selection of the k-th largest key by one CTA, in
// shared memory, for the kernels that hold a whole row's (or a whole sample's,
// or a whole candidate list's) keys in shared memory at once.
//
// Keys are the order-preserving 32-bit images of fp32 scores (larger float ->
// larger key, +0 and -0 equal, NaN lowest).  Three passes (11 + 11 + 10 bits,
// most significant first) fix the want-th largest key T and how many keys
// equal to T it takes.  Every function here must be called by all
// kBlkThreads threads of the block (they synchronise it).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace fm {

constexpr int kBlkThreads = 512;

__device__ __forceinline__ uint32_t block_order_key(float x) {
  if (x != x) return 0u;
  const uint32_t u = (x == 0.f) ? 0u : __float_as_uint(x);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Shared scratch of the selection: s_warp holds kBlkThreads / 32 + 1 ints.
struct BlockSelScratch {
  uint32_t* hist;  // 2048 bins
  int* warp;       // kBlkThreads / 32 + 1
  uint32_t* pick;  // 2
};

// Block-wide exclusive scan of one int per thread; *total receives the sum.
__device__ __forceinline__ int block_exclusive_scan(int v, int* s_warp, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int u = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += u;
  }
  if (lane == 31) s_warp[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    const int x = lane < kBlkThreads / 32 ? s_warp[lane] : 0;
    int y = x;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int u = __shfl_up_sync(0xffffffffu, y, o);
      if (lane >= o) y += u;
    }
    if (lane < kBlkThreads / 32) s_warp[lane] = y - x;  // exclusive over warps
    if (lane == kBlkThreads / 32 - 1) s_warp[kBlkThreads / 32] = y;
  }
  __syncthreads();
  const int r = s_warp[warp] + incl - v;
  *total = s_warp[kBlkThreads / 32];
  __syncthreads();
  return r;
}

// The want-th largest of the keys key_at(0 .. n-1) (1 <= want <= n): *T
// receives it and *need how many of the keys equal to T are among the want
// largest.  key_at reads a key from shared or global memory.
template <class KeyAt>
__device__ __forceinline__ void block_kth_largest_of(KeyAt key_at, int n, uint32_t want, BlockSelScratch sc,
                                                     uint32_t* T, int* need) {
  const int t = threadIdx.x;
  uint32_t prefix = 0u;
#pragma unroll 1
  for (int pass = 0; pass < 3; ++pass) {
    const int shift = pass == 0 ? 21 : (pass == 1 ? 10 : 0), nbits = pass == 2 ? 10 : 11;
    const int nb = 1 << nbits, hi = shift + nbits;
    for (int i = t; i < nb; i += kBlkThreads) sc.hist[i] = 0u;
    __syncthreads();
    // Keys that reach a selection crowd into a few digits (scores near the
    // cut share their leading bits), so lanes holding the same digit add to
    // the histogram with one atomic.
    const unsigned lane_lt = (1u << (t & 31)) - 1u;
    for (int i0 = 0; i0 < n; i0 += kBlkThreads) {
      const int i = i0 + t;
      const uint32_t key = i < n ? key_at(i) : 0u;
      const bool act = i < n && (hi >= 32 || (key >> hi) == (prefix >> hi));
      const unsigned active = __ballot_sync(0xffffffffu, act);
      if (act) {
        const uint32_t bin = (key >> shift) & (nb - 1);
        const unsigned peers = __match_any_sync(active, bin);
        if ((peers & lane_lt) == 0) atomicAdd(&sc.hist[bin], (uint32_t)__popc(peers));
      }
    }
    __syncthreads();
    // thread t owns bins [t*per, (t+1)*per) in descending digit order
    const int per = nb / kBlkThreads;
    uint32_t mine = 0;
    for (int j = 0; j < per; ++j) mine += sc.hist[nb - 1 - (t * per + j)];
    int tot;
    const uint32_t before = (uint32_t)block_exclusive_scan((int)mine, sc.warp, &tot);
    if (before < want && before + mine >= want) {
      uint32_t acc = before;
      for (int j = 0; j < per; ++j) {
        const int d = nb - 1 - (t * per + j);
        const uint32_t c = sc.hist[d];
        if (acc + c >= want) {
          sc.pick[0] = prefix | ((uint32_t)d << shift);
          sc.pick[1] = want - acc;
          break;
        }
        acc += c;
      }
    }
    __syncthreads();
    prefix = sc.pick[0];
    want = sc.pick[1];
    __syncthreads();
  }
  *T = prefix;
  *need = (int)want;
}

// The same over keys[0:n) in shared memory.
__device__ __forceinline__ void block_kth_largest(const uint32_t* keys, int n, uint32_t want, BlockSelScratch sc,
                                                  uint32_t* T, int* need) {
  block_kth_largest_of([keys](int i) { return keys[i]; }, n, want, sc, T, need);
}

}  // namespace fm
