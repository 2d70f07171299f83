// select_block.cuh -- radix selection of the k-th largest key by one CTA, in
// shared memory, for the kernels that hold a whole row's (or a whole sample's,
// or a whole candidate list's) keys in shared memory at once.
//
// Keys are the order-preserving 32-bit images of fp32 scores (larger float ->
// larger key, +0 and -0 equal, NaN lowest).  Histogram passes over the
// undecided bits (most significant first) fix the want-th largest key T and
// how many keys equal to T it takes.  Every function here must be called by all
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
  uint32_t* hist;  // 2048 words: eight 256-bin histograms, one per pair of warps
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
//
// The keys share every bit above the highest bit in which their maximum and
// minimum differ, so the passes start there: each pass histograms the next
// (up to) 8 undecided bits of the keys that match the bits decided so far
// and picks the digit holding the want-th largest.  Each pair of warps counts
// into its own 256-bin histogram with plain shared-memory atomics, so equal
// digits contend within two warps only (scores near the cut share their
// leading bits); the eight histograms are summed per bin.  Once the picked
// digit holds at most kSelFinish keys, they are gathered and ranked directly.
constexpr int kSelFinish = 256;
constexpr int kSelBits = 8, kSelBins = 1 << kSelBits;
constexpr int kSelCopies = kBlkThreads / 64;  // one histogram per two warps
static_assert(kSelCopies * kSelBins == 2048 && kSelBins <= kBlkThreads, "selection scratch");

template <class KeyAt>
__device__ __forceinline__ void block_kth_largest_of(KeyAt key_at, int n, uint32_t want, BlockSelScratch sc,
                                                     uint32_t* T, int* need) {
  const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
  constexpr int W = kBlkThreads / 32;
  uint32_t kmax = 0u, kmin = 0xffffffffu;
  for (int i = t; i < n; i += kBlkThreads) {
    const uint32_t k = key_at(i);
    kmax = max(kmax, k);
    kmin = min(kmin, k);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    kmax = max(kmax, __shfl_xor_sync(0xffffffffu, kmax, o));
    kmin = min(kmin, __shfl_xor_sync(0xffffffffu, kmin, o));
  }
  if (lane == 0) {
    sc.hist[warp] = kmax;
    sc.hist[W + warp] = kmin;
  }
  __syncthreads();
#pragma unroll
  for (int i = 0; i < W; ++i) {
    kmax = max(kmax, sc.hist[i]);
    kmin = min(kmin, sc.hist[W + i]);
  }
  __syncthreads();
  if (kmax == kmin) {  // every key equal
    *T = kmax;
    *need = (int)want;
    return;
  }
  int lo = 32 - __clz(kmax ^ kmin);  // bits [0, lo) undecided
  uint32_t prefix = lo >= 32 ? 0u : (kmax >> lo) << lo;
  uint32_t* my_hist = sc.hist + (warp >> 1) * kSelBins;
#pragma unroll 1
  while (lo > 0) {
    const int nbits = lo < kSelBits ? lo : kSelBits, shift = lo - nbits, nb = 1 << nbits;
    for (int i = t; i < kSelCopies * kSelBins; i += kBlkThreads) sc.hist[i] = 0u;
    __syncthreads();
    for (int i0 = 0; i0 < n; i0 += kBlkThreads) {
      const int i = i0 + t;
      const uint32_t key = i < n ? key_at(i) : 0u;
      if (i < n && (lo >= 32 || (key >> lo) == (prefix >> lo)))
        atomicAdd(&my_hist[(key >> shift) & (uint32_t)(nb - 1)], 1u);
    }
    __syncthreads();
    // thread t < nb owns digit nb - 1 - t (descending digit order)
    uint32_t mine = 0;
    if (t < nb)
#pragma unroll
      for (int c = 0; c < kSelCopies; ++c) mine += sc.hist[c * kSelBins + (nb - 1 - t)];
    int tot;
    const uint32_t before = (uint32_t)block_exclusive_scan((int)mine, sc.warp, &tot);
    if (t < nb && before < want && before + mine >= want) {
      sc.pick[0] = prefix | ((uint32_t)(nb - 1 - t) << shift);
      sc.pick[1] = want - before;
      sc.warp[W] = (int)mine;  // keys in the picked digit
    }
    __syncthreads();
    prefix = sc.pick[0];
    want = sc.pick[1];
    const int cnt = sc.warp[W];
    lo = shift;
    __syncthreads();
    if (lo > 0 && cnt <= kSelFinish) {
      // gather the picked digit's keys and rank them directly
      uint32_t* list = sc.hist;
      uint32_t* fill = sc.hist + kSelFinish;
      if (t == 0) *fill = 0u;
      __syncthreads();
      for (int i = t; i < n; i += kBlkThreads) {
        const uint32_t key = key_at(i);
        if ((key >> lo) == (prefix >> lo)) list[atomicAdd(fill, 1u)] = key;
      }
      __syncthreads();
      for (int e = t; e < cnt; e += kBlkThreads) {
        const uint32_t k = list[e];
        uint32_t gt = 0, eq = 0;
        for (int f = 0; f < cnt; ++f) {
          gt += list[f] > k ? 1u : 0u;
          eq += list[f] == k ? 1u : 0u;
        }
        if (gt < want && want <= gt + eq) {  // every key equal to k writes the same values
          sc.pick[0] = k;
          sc.pick[1] = want - gt;
        }
      }
      __syncthreads();
      prefix = sc.pick[0];
      want = sc.pick[1];
      __syncthreads();
      break;
    }
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
