// select.cu -- cross-layer ensemble and keep-mask selection.
//
// README "Joint checkpoint + ensemble": per-chunk max (union, default) or mean
// over the layers.  README "Usage" / toy decode loop: keep = top-K of the
// ensembled scores, or sigmoid > thresh.
//
// Top-K is an exact radix select on order-preserving 32-bit keys of the fp32
// scores: three histogram passes (11 + 11 + 10 bits, most significant first)
// fix the K-th largest key T and how many keys equal to T are kept; a mask
// pass then keeps every key > T and the first `need` keys == T in chunk-index
// order (only when the keys equal to T outnumber `need` does it rank them,
// with a per-block count pass and an in-block ordered scan).  Each histogram
// pass ends in its last-arriving block (atomic ticket, no waiting), which
// chooses the digit for the row; no kernel waits on another block.
//
// The sharded form splits one row's chunks over several GPUs (each holds a
// consecutive slice, in shard order).  The same passes run with the digit
// choice taken out of the histogram kernel: each shard histograms its slice
// into a caller buffer, the caller sums the buffers over the shards (one
// all-reduce per pass), and every shard then picks the same digit from the
// same global histogram.  Ties at T are ranked across shards by an exclusive
// sum of the per-shard tie counts in shard order (one all-gather).
#include "fm_internal.cuh"
#include "select_block.cuh"

namespace fm {
namespace {

constexpr int kThreads = 512;  // top-K blocks: 8192 chunks each, so few per-block merges per row
static_assert(kThreads == kBlkThreads, "the block scans assume the selection block size");
constexpr int kPerThread = 16;
constexpr int kChunk = kThreads * kPerThread;  // elements per block slice
constexpr int kBins0 = 2048, kBins1 = 2048, kBins2 = 1024;
constexpr int kHistWords = kBins0 + kBins1 + kBins2;
constexpr int kShardBins = FM_TOPK_SHARD_BINS;  // row stride of the sharded form's histograms
static_assert(kShardBins >= kBins0 && kShardBins >= kBins1 && kShardBins >= kBins2, "histogram row");
constexpr int kShift[3] = {21, 10, 0};
constexpr int kBits[3] = {11, 11, 10};

// kModeFast: the candidate path below; kModeDone: the row's mask is written.
enum : int { kModeEmpty = 0, kModeAll = 1, kModeSelect = 2, kModeFast = 3, kModeDone = 4 };

// Per-row state (in the workspace).
struct RowState {
  int nv;          // valid chunks
  int mode;        // kMode*
  uint32_t prefix; // key digits chosen so far
  int remaining;   // how many of the keys matching `prefix` are still to keep
  int need_eq;     // after the last pass: keys == T to keep
  int cnt_eq;      // after the last pass: keys == T present
  int tickets[3];  // arrival counters of the three histogram passes
  int pad[7];
};
static_assert(sizeof(RowState) == 64, "row state is 64 bytes");

struct Workspace {
  RowState* state;  // [B]
  uint32_t* hist;   // [B, kHistWords]
  int* eqcnt;       // [B, nblk]
};

__host__ __device__ inline size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

__host__ __device__ inline Workspace carve(void* ws, int B, int nblk) {
  uint8_t* p = static_cast<uint8_t*>(ws);
  Workspace w;
  w.state = reinterpret_cast<RowState*>(p);
  p += align256(sizeof(RowState) * (size_t)B);
  w.hist = reinterpret_cast<uint32_t*>(p);
  p += align256(sizeof(uint32_t) * (size_t)B * kHistWords);
  w.eqcnt = reinterpret_cast<int*>(p);
  return w;
}

__host__ __device__ inline size_t ws_bytes(int B, int nblk) {
  return align256(sizeof(RowState) * (size_t)B) + align256(sizeof(uint32_t) * (size_t)B * kHistWords) +
         align256(sizeof(int) * (size_t)B * nblk);
}

// ------------------------------------------------- the candidate fast path
// Exact top-K with one full pass over the scores.  A CTA per row takes a
// sample of up to kSample scores (256 runs of 32 consecutive ones, evenly
// spread over the row) and sets the threshold tau to
// the sample's key of rank 2K * S / n + 16 (about the 2K-th largest score of
// the row).  One pass over the row then writes the mask's zeros and appends
// every valid score >= tau, with its index, to the row's candidate list.  If
// the list holds at least K entries (and fits), the K largest scores of the row
// are all in it -- every other score is below tau, hence below every
// candidate -- and a CTA per row selects them in shared memory and sets their
// mask bytes.  A row whose list is too short or too long, or whose K-th value
// is tied with values it does not keep (the tie order needs the chunk order),
// falls back to the histogram passes, which run after and skip finished rows.
constexpr int kSample = 8192;
constexpr int kCandMax = 16384;  // a candidate list in one CTA's shared memory: 128 KB

__host__ __device__ inline int cand_cap(int N) {
  const int c = (N + 15) / 16;
  return c < 256 ? 256 : (c > kCandMax ? kCandMax : c);
}

struct FastWs {
  uint32_t* tau;   // [B]
  int* cnt;        // [B] candidates found (may exceed the capacity)
  uint32_t* ckey;  // [B, C]
  int* cidx;       // [B, C]
};

__host__ __device__ inline FastWs carve_fast(void* ws, int B, int nblk, int C) {
  uint8_t* p = static_cast<uint8_t*>(ws) + ws_bytes(B, nblk);
  FastWs f;
  f.tau = reinterpret_cast<uint32_t*>(p);
  p += align256(sizeof(uint32_t) * (size_t)B);
  f.cnt = reinterpret_cast<int*>(p);
  p += align256(sizeof(int) * (size_t)B);
  f.ckey = reinterpret_cast<uint32_t*>(p);
  p += align256(sizeof(uint32_t) * (size_t)B * C);
  f.cidx = reinterpret_cast<int*>(p);
  return f;
}

__host__ __device__ inline size_t fast_ws_bytes(int B, int nblk, int C) {
  return ws_bytes(B, nblk) + 2 * align256(sizeof(int) * (size_t)B) + 2 * align256(sizeof(int) * (size_t)B * C);
}

// Order-preserving key: larger float -> larger key; +0 and -0 equal; NaN lowest.
__device__ __forceinline__ uint32_t order_key(float x) {
  if (x != x) return 0u;
  uint32_t u = (x == 0.f) ? 0u : __float_as_uint(x);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ int row_nvalid(const int32_t* n_valid, int b, int N) {
  int v = n_valid ? n_valid[b] : N;
  return max(0, min(v, N));
}

// ------------------------------------------------------------ ensemble
__global__ void ensemble_kernel(const float* __restrict__ scores, int L, int64_t BN, int mode,
                                float* __restrict__ ens) {
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < BN;
       i += (int64_t)gridDim.x * blockDim.x) {
    float e = scores[i];
    if (mode == FM_ENSEMBLE_MAX) {
      for (int l = 1; l < L; ++l) e = fmax_nan(e, scores[(int64_t)l * BN + i]);
    } else {
      for (int l = 1; l < L; ++l) e = e + scores[(int64_t)l * BN + i];
      e = e / (float)L;
    }
    ens[i] = e;
  }
}

// ----------------------------------------------------------- threshold
__global__ void threshold_kernel(const float* __restrict__ ens, const int32_t* __restrict__ n_valid,
                                 int N, float thr, uint8_t* __restrict__ keep) {
  const int b = blockIdx.y;
  const int nv = row_nvalid(n_valid, b, N);
  for (int n = blockIdx.x * blockDim.x + threadIdx.x; n < N; n += gridDim.x * blockDim.x) {
    const float e = ens[(int64_t)b * N + n];
    keep[(int64_t)b * N + n] = (n < nv && e > thr) ? 1 : 0;
  }
}

// --------------------------------------------------------------- top-K
__global__ void topk_init_kernel(Workspace w, const int32_t* __restrict__ n_valid, int N, int k, int fast) {
  const int b = blockIdx.x;
  uint32_t* h = w.hist + (size_t)b * kHistWords;
  for (int i = threadIdx.x; i < kHistWords; i += blockDim.x) h[i] = 0u;
  if (threadIdx.x == 0) {
    RowState s = {};
    s.nv = row_nvalid(n_valid, b, N);
    s.mode = s.nv == 0 ? kModeEmpty : (k >= s.nv ? kModeAll : (fast ? kModeFast : kModeSelect));
    s.prefix = 0u;
    s.remaining = min(k, s.nv);
    w.state[b] = s;
  }
}

// Chooses the digit of pass PASS holding the remaining-th largest key of the
// row from its complete histogram `gh` (bins in digit order), one block of
// kThreads; records the digit in the row state.  Thread t owns bins
// [t*per, (t+1)*per) in descending order of value.  With CLEAR the thread
// also zeroes the bins it read, ready for the next pass; with TOTAL (the first
// pass of the sharded form) the row's mode is settled from the histogram's
// total, which only the summed histogram knows.
// Sharded form: this shard's row states (its own valid count; the mode is
// settled by the first pick, from the summed histogram) and a zeroed histogram.
__global__ void topk_shard_init_kernel(Workspace w, const int32_t* __restrict__ n_valid, int N, int k,
                                       uint32_t* __restrict__ xh) {
  const int b = blockIdx.x;
  uint32_t* h = xh + (size_t)b * kShardBins;
  for (int i = threadIdx.x; i < kShardBins; i += blockDim.x) h[i] = 0u;
  if (threadIdx.x == 0) {
    RowState s = {};
    s.nv = row_nvalid(n_valid, b, N);
    s.mode = kModeSelect;
    s.prefix = 0u;
    s.remaining = k;
    w.state[b] = s;
  }
}

template <int PASS, bool CLEAR, bool TOTAL>
__device__ __forceinline__ void pick_digit(RowState* st, uint32_t* gh, uint32_t* s_suffix) {
  constexpr int bins = PASS == 0 ? kBins0 : (PASS == 1 ? kBins1 : kBins2);
  constexpr int shift = kShift[PASS];
  constexpr int per = bins / kThreads;
  // every thread reads the row state before the first barrier below: the one
  // thread that finds the digit rewrites it after the last barrier
  const uint32_t prefix = st->prefix;
  const uint32_t want0 = (uint32_t)st->remaining;
  uint32_t cnt[per];
  uint32_t mine = 0;
#pragma unroll
  for (int j = 0; j < per; ++j) {
    const int d = bins - 1 - (threadIdx.x * per + j);  // descending digit
    cnt[j] = __ldcg(&gh[d]);
    if (CLEAR) gh[d] = 0u;
    mine += cnt[j];
  }
  s_suffix[threadIdx.x] = mine;
  __syncthreads();
  // inclusive scan over threads (descending digit order)
  for (int off = 1; off < kThreads; off <<= 1) {
    const uint32_t v = threadIdx.x >= off ? s_suffix[threadIdx.x - off] : 0u;
    __syncthreads();
    s_suffix[threadIdx.x] += v;
    __syncthreads();
  }
  uint32_t want = want0;
  if (TOTAL) {
    const uint32_t total = s_suffix[kThreads - 1];
    if (total == 0u || want >= total) {
      if (threadIdx.x == 0) st->mode = total == 0u ? kModeEmpty : kModeAll;
      return;
    }
  }
  const uint32_t before = s_suffix[threadIdx.x] - mine;  // keys with a larger digit
  if (before < want && before + mine >= want) {
    uint32_t acc = before;
#pragma unroll
    for (int j = 0; j < per; ++j) {
      if (acc + cnt[j] >= want) {
        const int d = bins - 1 - (threadIdx.x * per + j);
        st->prefix = prefix | ((uint32_t)d << shift);
        st->remaining = (int)(want - acc);
        if (PASS == 2) {
          st->need_eq = (int)(want - acc);
          st->cnt_eq = (int)cnt[j];
        }
        break;
      }
      acc += cnt[j];
    }
  }
}

// Histogram of digit PASS over the keys of the row that match the digits
// chosen so far.  FUSED: into the workspace, and the last-arriving block of the
// row picks the digit.  Otherwise (sharded form): into the caller's buffer
// `xh` [B, kShardBins], for the caller to sum over the shards.
template <int PASS, bool FUSED>
__global__ void __launch_bounds__(kThreads) topk_hist_kernel(Workspace w, const float* __restrict__ ens,
                                                             int N, uint32_t* __restrict__ xh) {
  constexpr int bins = PASS == 0 ? kBins0 : (PASS == 1 ? kBins1 : kBins2);
  constexpr int shift = kShift[PASS];
  constexpr int hi_shift = shift + kBits[PASS];  // digits above this pass
  __shared__ uint32_t sh[bins];
  __shared__ int s_last;
  __shared__ uint32_t s_suffix[kThreads];
  const int b = blockIdx.y;
  RowState* st = w.state + b;
  if (st->mode != kModeSelect) return;  // uniform across the block
  const int nv = st->nv;
  const uint32_t prefix = st->prefix;
  for (int i = threadIdx.x; i < bins; i += kThreads) sh[i] = 0u;
  __syncthreads();
  const int64_t base = (int64_t)blockIdx.x * kChunk;
  const float* row = ens + (int64_t)b * N;
  // all loads first (16 in flight per thread), then the counting
  float v[kPerThread];
#pragma unroll
  for (int i = 0; i < kPerThread; ++i) {
    const int64_t n = base + (int64_t)i * kThreads + threadIdx.x;
    v[i] = n < nv ? __ldg(row + n) : 0.f;
  }
  // Scores crowd into a few digits (sigmoid outputs share their exponent), so
  // lanes holding the same digit are counted with one shared-memory atomic.
  const unsigned lane_lt = (1u << (threadIdx.x & 31)) - 1u;
#pragma unroll
  for (int i = 0; i < kPerThread; ++i) {
    const int64_t n = base + (int64_t)i * kThreads + threadIdx.x;
    const uint32_t key = order_key(v[i]);
    const bool act = n < nv && ((hi_shift >= 32) || ((key >> (hi_shift & 31)) == (prefix >> (hi_shift & 31))));
    const unsigned active = __ballot_sync(0xffffffffu, act);
    if (act) {
      const uint32_t bin = (key >> shift) & (bins - 1);
      const unsigned peers = __match_any_sync(active, bin);
      if ((peers & lane_lt) == 0) atomicAdd(&sh[bin], (uint32_t)__popc(peers));
    }
  }
  __syncthreads();
  uint32_t* gh = FUSED ? w.hist + (size_t)b * kHistWords + (PASS == 0 ? 0 : (PASS == 1 ? kBins0 : kBins0 + kBins1))
                       : xh + (size_t)b * kShardBins;
  for (int i = threadIdx.x; i < bins; i += kThreads)
    if (sh[i]) atomicAdd(&gh[i], sh[i]);
  if (!FUSED) return;
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) s_last = (atomicAdd(&st->tickets[PASS], 1) == (int)gridDim.x - 1);
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  pick_digit<PASS, false, false>(st, gh, s_suffix);
}

// Sharded form: the digit choice of pass PASS from the histogram summed over
// the shards (one block per row); clears the histogram for the next pass.
template <int PASS>
__global__ void __launch_bounds__(kThreads) topk_shard_pick_kernel(Workspace w, uint32_t* __restrict__ xh) {
  __shared__ uint32_t s_suffix[kThreads];
  RowState* st = w.state + blockIdx.x;
  if (st->mode != kModeSelect) return;
  pick_digit<PASS, true, PASS == 0>(st, xh + (size_t)blockIdx.x * kShardBins, s_suffix);
}

// Per-block count of keys equal to T, only for rows whose tie at T is split;
// with eq_row (zeroed by the caller) also the row's total over the blocks.
__global__ void __launch_bounds__(kThreads) topk_eqcount_kernel(Workspace w, const float* __restrict__ ens,
                                                                int N, int nblk, int32_t* __restrict__ eq_row) {
  const int b = blockIdx.y;
  const RowState* st = w.state + b;
  if (st->mode != kModeSelect || st->need_eq == st->cnt_eq) return;
  const uint32_t T = st->prefix;
  const int nv = st->nv;
  const int64_t base = (int64_t)blockIdx.x * kChunk;
  const float* row = ens + (int64_t)b * N;
  int c = 0;
  for (int i = 0; i < kPerThread; ++i) {
    const int64_t n = base + (int64_t)i * kThreads + threadIdx.x;
    if (n < nv && order_key(row[n]) == T) ++c;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) c += __shfl_xor_sync(0xffffffffu, c, o);
  __shared__ int red[kThreads / 32];
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = c;
  __syncthreads();
  if (threadIdx.x == 0) {
    int t = 0;
    for (int i = 0; i < kThreads / 32; ++i) t += red[i];
    w.eqcnt[(size_t)b * nblk + blockIdx.x] = t;
    if (eq_row && t) atomicAdd(eq_row + b, t);  // sharded form: the slice's total
  }
}

// eq_all [shards, B] (sharded form, else NULL): each shard's count of keys == T
// per row; the ones of the shards before `shard` rank ahead of this slice's.
__global__ void __launch_bounds__(kThreads) topk_mask_kernel(Workspace w, const float* __restrict__ ens,
                                                             int N, int nblk, uint8_t* __restrict__ keep,
                                                             const int32_t* __restrict__ eq_all, int shard,
                                                             int B) {
  const int b = blockIdx.y;
  const RowState* st = w.state + b;
  const int mode = st->mode, nv = st->nv;
  if (mode == kModeDone) return;  // written by the candidate path
  const uint32_t T = st->prefix;
  const bool split_tie = mode == kModeSelect && st->need_eq != st->cnt_eq;
  const int need = st->need_eq;
  const int64_t base = (int64_t)blockIdx.x * kChunk;
  const float* row = ens + (int64_t)b * N;
  uint8_t* out = keep + (int64_t)b * N;
  if (!split_tie) {
    if ((N & 3) == 0 && (reinterpret_cast<uintptr_t>(ens) & 15u) == 0 &&
        (reinterpret_cast<uintptr_t>(keep) & 3u) == 0) {
      // four consecutive chunks per thread: 16-byte loads, one 4-byte mask store
#pragma unroll
      for (int i = 0; i < kPerThread / 4; ++i) {
        const int64_t n = base + ((int64_t)i * kThreads + threadIdx.x) * 4;
        if (n >= N) break;
        const float4 e = __ldg(reinterpret_cast<const float4*>(row + n));
        const float ev[4] = {e.x, e.y, e.z, e.w};
        uint32_t word = 0;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const bool k = n + c < nv && (mode == kModeAll || order_key(ev[c]) >= T);
          word |= (k ? 1u : 0u) << (8 * c);
        }
        *reinterpret_cast<uint32_t*>(out + n) = word;
      }
      return;
    }
    for (int i = 0; i < kPerThread; ++i) {
      const int64_t n = base + (int64_t)i * kThreads + threadIdx.x;
      if (n >= N) break;
      uint8_t k = 0;
      if (n < nv) k = (mode == kModeAll) ? 1 : (order_key(row[n]) >= T ? 1 : 0);
      out[n] = k;
    }
    return;
  }
  // ordered rank among keys == T: blocks before this one, then in-block order
  __shared__ int s_prefix;
  __shared__ int s_warp[kThreads / 32];
  if (threadIdx.x == 0) {
    int p = 0;
    if (eq_all)
      for (int r = 0; r < shard; ++r) p += eq_all[(size_t)r * B + b];
    for (int j = 0; j < (int)blockIdx.x; ++j) p += w.eqcnt[(size_t)b * nblk + j];
    s_prefix = p;
  }
  __syncthreads();
  int running = s_prefix;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  for (int i = 0; i < kPerThread; ++i) {
    const int64_t n = base + (int64_t)i * kThreads + threadIdx.x;
    uint32_t key = 0;
    if (n < nv) key = order_key(row[n]);
    const int eq = (n < nv && key == T) ? 1 : 0;
    // block-wide exclusive scan of eq in index order
    const unsigned ball = __ballot_sync(0xffffffffu, eq);
    const int in_warp = __popc(ball & ((1u << lane) - 1u));
    if (lane == 0) s_warp[warp] = __popc(ball);
    __syncthreads();
    int before_warp = 0, total = 0;
    for (int j = 0; j < kThreads / 32; ++j) {
      if (j < warp) before_warp += s_warp[j];
      total += s_warp[j];
    }
    const int rank = running + before_warp + in_warp;
    if (n < N) {
      uint8_t k = 0;
      if (n < nv) k = (key > T || (eq && rank < need)) ? 1 : 0;
      out[n] = k;
    }
    running += total;
    __syncthreads();
  }
}

// Fast path, per row: the row state (what topk_init_kernel writes for the
// other forms; the fast path uses no histogram), then the sample and the
// threshold tau; zeroes the list.
__global__ void __launch_bounds__(kBlkThreads) topk_sample_kernel(Workspace w, FastWs f,
                                                                  const float* __restrict__ ens, int N,
                                                                  const int32_t* __restrict__ n_valid, int k) {
  extern __shared__ uint32_t s_key[];  // [kSample]
  __shared__ uint32_t s_hist[2048];
  __shared__ int s_warp[kBlkThreads / 32 + 1];
  __shared__ uint32_t s_pick[2];
  const int b = blockIdx.x, t = threadIdx.x;
  grid_dependency_wait();  // the scores (and n_valid) come from the kernels ahead
  const int nv = row_nvalid(n_valid, b, N), K = min(k, nv);
  const int mode = nv == 0 ? kModeEmpty : (k >= nv ? kModeAll : kModeFast);
  if (t == 0) {
    RowState s = {};
    s.nv = nv;
    s.mode = mode;
    s.prefix = 0u;
    s.remaining = K;
    w.state[b] = s;
  }
  if (mode != kModeFast) return;  // uniform across the block
  const int S = nv < kSample ? nv : kSample;
  const float* row = ens + (size_t)b * N;
  {  // all of a thread's loads in flight at once
    // S = kSample: 256 runs of 32 consecutive scores spread evenly over the
    // row (each run one 128-byte line: a warp reads a run per load); else
    // the whole row
    constexpr int kPer = kSample / kBlkThreads;
    static_assert(kSample == 256 * 32 && kBlkThreads % 32 == 0, "sample runs");
    const int64_t run_step = S == kSample ? nv / 256 : 32;
    float v[kPer];
#pragma unroll
    for (int q = 0; q < kPer; ++q) {
      const int j = t + q * kBlkThreads;
      v[q] = j < S ? __ldg(row + (int64_t)(j >> 5) * run_step + (j & 31)) : 0.f;
    }
#pragma unroll
    for (int q = 0; q < kPer; ++q) {
      const int j = t + q * kBlkThreads;
      if (j < S) s_key[j] = order_key(v[q]);
    }
  }
  const int64_t r = (2 * (int64_t)K * S + nv - 1) / nv + 16;
  uint32_t tau = 0u;  // 0: every valid score is a candidate
  if (r < S) {
    __syncthreads();
    int need;
    block_kth_largest(s_key, S, (uint32_t)r, BlockSelScratch{s_hist, s_warp, s_pick}, &tau, &need);
  }
  if (t == 0) {
    f.tau[b] = tau;
    f.cnt[b] = 0;
  }
}

// Fast path, grid-wide: writes the mask of the Fast / All / Empty rows (zeros
// for Fast rows; their kept bytes are set per row afterwards) and appends the
// valid scores >= tau of Fast rows to the row's list.  A CTA takes kThreads *
// PER scores of one row (its own slicing: no workspace is kept per block).
template <int PER>
__global__ void __launch_bounds__(kThreads) topk_collect_kernel(Workspace w, FastWs f, int C,
                                                                const float* __restrict__ ens, int N,
                                                                uint8_t* __restrict__ keep) {
  const int b = blockIdx.y;
  const int64_t base = (int64_t)blockIdx.x * (kThreads * PER);
  const float* row = ens + (int64_t)b * N;
  // the scores are loaded before the row's state and threshold are read, so
  // the two latencies overlap (loads past the row's valid length are masked
  // below; every index here is inside the row).  This grid starts once the
  // sample kernel's CTAs have left, each after its wait on the kernels that
  // wrote the scores, so they may be read before waiting for it.
  uint32_t key[PER];  // the scores' bits, then their order keys
#pragma unroll
  for (int i = 0; i < PER; ++i) {
    const int64_t n = base + (int64_t)i * kThreads + threadIdx.x;
    key[i] = n < N ? __float_as_uint(__ldg(row + n)) : 0u;
  }
  grid_dependency_wait();  // the row state and tau come from the sample kernel
  const RowState* st = w.state + b;
  const int mode = st->mode;
  if (mode != kModeFast && mode != kModeAll && mode != kModeEmpty) return;
  const int nv = st->nv;
  uint8_t* out = keep + (int64_t)b * N;
  if ((N & 3) == 0 && (reinterpret_cast<uintptr_t>(keep) & 3u) == 0) {
#pragma unroll
    for (int i = 0; i < PER / 4; ++i) {
      const int64_t n = base + ((int64_t)i * kThreads + threadIdx.x) * 4;
      if (n >= N) break;
      uint32_t word = 0;
      if (mode == kModeAll)
#pragma unroll
        for (int c = 0; c < 4; ++c) word |= (n + c < nv ? 1u : 0u) << (8 * c);
      *reinterpret_cast<uint32_t*>(out + n) = word;
    }
  } else {
    for (int i = 0; i < PER; ++i) {
      const int64_t n = base + (int64_t)i * kThreads + threadIdx.x;
      if (n >= N) break;
      out[n] = (mode == kModeAll && n < nv) ? 1 : 0;
    }
  }
  if (mode != kModeFast) return;  // uniform across the block
  const uint32_t tau = f.tau[b];
  uint32_t is_cand = 0;  // bit i: element i of this thread is a candidate
#pragma unroll
  for (int i = 0; i < PER; ++i) {
    const int64_t n = base + (int64_t)i * kThreads + threadIdx.x;
    key[i] = order_key(n < nv ? __uint_as_float(key[i]) : 0.f);
    if (n < nv && key[i] >= tau) is_cand |= 1u << i;
  }
  // one atomic per block: the block's candidates go to one range of the list
  __shared__ int s_warp[kThreads / 32 + 1];
  __shared__ int s_base;
  int total;
  const int before = block_exclusive_scan(__popc(is_cand), s_warp, &total);
  if (threadIdx.x == 0) s_base = total ? atomicAdd(f.cnt + b, total) : 0;
  __syncthreads();
  int pos = s_base + before;
#pragma unroll
  for (int i = 0; i < PER; ++i) {
    if (is_cand & (1u << i)) {
      if (pos < C) {
        f.ckey[(size_t)b * C + pos] = key[i];
        f.cidx[(size_t)b * C + pos] = (int)(base + (int64_t)i * kThreads + threadIdx.x);
      }
      ++pos;
    }
  }
}

// The whole row by one CTA from global memory (the candidate path's fallback):
// the K-th largest key T of ens[b, 0:nv), then the mask of [0, N) with the keys
// equal to T taken in chunk order.  Three reads of the row by one SM: slow for
// the row, but only rows the candidate path cannot finish take it.
__device__ void row_select_in_block(const float* __restrict__ row, int nv, int N, int K, uint8_t* __restrict__ out,
                                    BlockSelScratch sc) {
  uint32_t T;
  int need;
  block_kth_largest_of([row](int i) { return order_key(__ldg(row + i)); }, nv, (uint32_t)K, sc, &T, &need);
  // ordered mask: thread t takes kSpan consecutive chunks of each tile
  constexpr int kSpan = 16;
  constexpr int kTileN = kBlkThreads * kSpan;
  int taken = 0;  // keys == T kept in earlier tiles
  for (int c0 = 0; c0 < N; c0 += kTileN) {
    const int lo = c0 + threadIdx.x * kSpan;
    int eq = 0;
    for (int j = 0; j < kSpan; ++j) {
      const int n = lo + j;
      if (n < nv && order_key(__ldg(row + n)) == T) ++eq;
    }
    int tile_eq;
    const int eq_before = taken + block_exclusive_scan(eq, sc.warp, &tile_eq);
    int rank = eq_before;
    for (int j = 0; j < kSpan; ++j) {
      const int n = lo + j;
      if (n >= N) break;
      uint8_t k = 0;
      if (n < nv) {
        const uint32_t key = order_key(__ldg(row + n));
        k = (key > T || (key == T && rank++ < need)) ? 1 : 0;
      }
      out[n] = k;
    }
    taken += tile_eq;
  }
}

// Fast path, per row: the K largest of the candidate list, or the whole row
// by this CTA when the list cannot give them.
__global__ void __launch_bounds__(kBlkThreads) topk_fastsel_kernel(Workspace w, FastWs f, const float* __restrict__ ens,
                                                                   int C, int N, uint8_t* __restrict__ keep) {
  extern __shared__ uint32_t s_dyn[];  // keys [C], then indices [C]
  __shared__ uint32_t s_hist[2048];
  __shared__ int s_warp[kBlkThreads / 32 + 1];
  __shared__ uint32_t s_pick[2];
  const int b = blockIdx.x, t = threadIdx.x;
  grid_dependency_wait();  // the list and the mask's zeros come from the collect pass
  RowState* st = w.state + b;
  // the row's mode, count and K are read together (one latency, not two)
  const int mode = st->mode, cnt = f.cnt[b], K = st->remaining;
  __syncthreads();  // every thread has read the mode before thread 0 may change it
  if (mode == kModeAll || mode == kModeEmpty) {  // the collect pass wrote their masks
    if (t == 0) st->mode = kModeDone;
    return;
  }
  if (mode != kModeFast) return;
  const BlockSelScratch sc{s_hist, s_warp, s_pick};
  uint8_t* out = keep + (int64_t)b * N;
  if (cnt < K || cnt > C) {  // too few candidates (tau too high) or too many to hold
    row_select_in_block(ens + (int64_t)b * N, st->nv, N, K, out, sc);
    if (t == 0) st->mode = kModeDone;
    return;
  }
  uint32_t* keys = s_dyn;
  int* idx = reinterpret_cast<int*>(s_dyn + C);
  {  // eight loads of each list per thread in flight at a time, not one
    const uint32_t* ck = f.ckey + (size_t)b * C;
    const int* ci = f.cidx + (size_t)b * C;
    constexpr int kU = 8;
    for (int i0 = t; i0 < cnt; i0 += kU * kBlkThreads) {
      uint32_t kk[kU];
      int ii[kU];
#pragma unroll
      for (int u = 0; u < kU; ++u) {
        const int i = i0 + u * kBlkThreads;
        kk[u] = i < cnt ? __ldg(ck + i) : 0u;
        ii[u] = i < cnt ? __ldg(ci + i) : 0;
      }
#pragma unroll
      for (int u = 0; u < kU; ++u) {
        const int i = i0 + u * kBlkThreads;
        if (i < cnt) {
          keys[i] = kk[u];
          idx[i] = ii[u];
        }
      }
    }
  }
  __syncthreads();
  uint32_t T;
  int need;
  block_kth_largest(keys, cnt, (uint32_t)K, sc, &T, &need);
  int eq = 0;
  for (int i = t; i < cnt; i += kBlkThreads) eq += keys[i] == T ? 1 : 0;
  int eq_total;
  const int eq_before = block_exclusive_scan(eq, s_warp, &eq_total);
  if (eq_total == need) {  // every candidate equal to the K-th is kept
    for (int i = t; i < cnt; i += kBlkThreads)
      if (keys[i] >= T) out[idx[i]] = 1;
    if (t == 0) st->mode = kModeDone;
    return;
  }
  // The K-th value is tied with candidates it does not keep: the tied
  // candidates are ranked by chunk index among themselves (every chunk with
  // that score is a candidate, since the score is at least tau), in the
  // histogram's shared memory when they fit, else over the whole row.
  constexpr int kTieMax = 2048;
  if (eq_total > kTieMax) {
    row_select_in_block(ens + (int64_t)b * N, st->nv, N, K, out, sc);
    if (t == 0) st->mode = kModeDone;
    return;
  }
  int* tie = reinterpret_cast<int*>(s_hist);  // the selection is done with the histogram
  {
    int pos = eq_before;
    for (int i = t; i < cnt; i += kBlkThreads)
      if (keys[i] == T) tie[pos++] = idx[i];
  }
  __syncthreads();
  for (int i = t; i < cnt; i += kBlkThreads)
    if (keys[i] > T) out[idx[i]] = 1;
  for (int e = t; e < eq_total; e += kBlkThreads) {
    const int me = tie[e];
    int rank = 0;
    for (int f = 0; f < eq_total; ++f) rank += tie[f] < me ? 1 : 0;
    if (rank < need) out[me] = 1;
  }
  if (t == 0) st->mode = kModeDone;
}

}  // namespace

fm_status launch_ensemble(const float* scores, int L, int B, int N, int mode, float* ens,
                          cudaStream_t st) {
  const int64_t BN = (int64_t)B * N;
  int64_t g = (BN + 255) / 256;
  const int grid = (int)(g < 148 * 16 ? g : 148 * 16);
  ensemble_kernel<<<grid, 256, 0, st>>>(scores, L, BN, mode, ens);
  note_launch();
  return check_launch();
}

fm_status launch_threshold(const float* ens, const int32_t* n_valid, int B, int N, float thr,
                           uint8_t* keep, cudaStream_t st) {
  const int64_t gx = ((int64_t)N + 1023) / 1024;
  dim3 grid((unsigned)(gx < 1024 ? gx : 1024), B);
  threshold_kernel<<<grid, 256, 0, st>>>(ens, n_valid, N, thr, keep);
  note_launch();
  return check_launch();
}

size_t topk_workspace_bytes(int B, int N) {
  const int nblk = (int)(((int64_t)N + kChunk - 1) / kChunk);
  return ws_bytes(B, nblk);
}

size_t topk_workspace_bytes_fast(int B, int N) {
  const int nblk = (int)(((int64_t)N + kChunk - 1) / kChunk);
  return fast_ws_bytes(B, nblk, cand_cap(N));
}

fm_status launch_topk(const float* ens, const int32_t* n_valid, int B, int N, int k, uint8_t* keep,
                      void* ws, size_t ws_size, cudaStream_t st) {
  const int nblk = (int)(((int64_t)N + kChunk - 1) / kChunk);
  if (ws_size < ws_bytes(B, nblk)) return FM_ERR_INVALID_ARG;
  if (topk_use_cluster(N)) return launch_topk_cluster(ens, n_valid, B, N, k, keep, st);
  Workspace w = carve(ws, B, nblk);
  const int C = cand_cap(N);
  const bool fast = ws_size >= fast_ws_bytes(B, nblk, C) && 2 * (int64_t)k + 1024 <= C;
  dim3 grid(nblk, B);
  if (fast) {
    static PerDeviceOnce smem_set;
    int dev = 0;
    cudaGetDevice(&dev);
    if (fm_status s = smem_limit_once(smem_set, dev, topk_fastsel_kernel,
                                      (int)(2 * sizeof(uint32_t) * kCandMax)))
      return s;
    const FastWs f = carve_fast(ws, B, nblk, C);
    // three launches that may each start as the one ahead drains (each waits
    // for it where it reads what it wrote).  No kernel lets the next one in
    // earlier: collect CTAs resident during the sample's select, loading
    // their scores, slowed the select (ragged 32-row case: 51 us against 42)
    cudaError_t e = launch_overlapped(topk_sample_kernel, dim3(B), dim3(kBlkThreads), sizeof(uint32_t) * kSample,
                                      st, w, f, ens, N, n_valid, k);
    // 4096 scores per CTA: three CTAs per SM, where 8192 allowed two
    constexpr int kCollectPer = 8;
    const dim3 cgrid((unsigned)(((int64_t)N + kThreads * kCollectPer - 1) / (kThreads * kCollectPer)), (unsigned)B);
    if (e == cudaSuccess)
      e = launch_overlapped(topk_collect_kernel<kCollectPer>, cgrid, dim3(kThreads), 0, st, w, f, C, ens, N, keep);
    if (e == cudaSuccess)
      e = launch_overlapped(topk_fastsel_kernel, dim3(B), dim3(kBlkThreads), 2 * sizeof(uint32_t) * (size_t)C, st,
                            w, f, (const float*)ens, C, N, keep);
    for (int i = 0; i < 3; ++i) note_launch();
    if (e != cudaSuccess) return record_cuda_error(e);
    return check_launch();  // every row is finished by the candidate path or its in-block fallback
  }
  topk_init_kernel<<<B, 256, 0, st>>>(w, n_valid, N, k, 0);
  note_launch();
  topk_hist_kernel<0, true><<<grid, kThreads, 0, st>>>(w, ens, N, nullptr);
  topk_hist_kernel<1, true><<<grid, kThreads, 0, st>>>(w, ens, N, nullptr);
  topk_hist_kernel<2, true><<<grid, kThreads, 0, st>>>(w, ens, N, nullptr);
  topk_eqcount_kernel<<<grid, kThreads, 0, st>>>(w, ens, N, nblk, nullptr);
  topk_mask_kernel<<<grid, kThreads, 0, st>>>(w, ens, N, nblk, keep, nullptr, 0, B);
  for (int i = 0; i < 5; ++i) note_launch();
  return check_launch();
}

// ---------------------------------------------------- sharded top-K phases
static fm_status shard_ws(void* ws, size_t ws_size, int B, int N, Workspace* w, int* nblk) {
  *nblk = (int)(((int64_t)N + kChunk - 1) / kChunk);
  if (ws_size < ws_bytes(B, *nblk)) return FM_ERR_INVALID_ARG;
  *w = carve(ws, B, *nblk);
  return FM_OK;
}

fm_status launch_topk_shard_begin(const int32_t* n_valid, int B, int N, int k, int32_t* hist, void* ws,
                                  size_t ws_size, cudaStream_t st) {
  Workspace w;
  int nblk;
  if (fm_status e = shard_ws(ws, ws_size, B, N, &w, &nblk)) return e;
  topk_shard_init_kernel<<<B, 256, 0, st>>>(w, n_valid, N, k, reinterpret_cast<uint32_t*>(hist));
  note_launch();
  return check_launch();
}

fm_status launch_topk_shard_hist(const float* ens, int B, int N, int pass, int32_t* hist, void* ws,
                                 size_t ws_size, cudaStream_t st) {
  Workspace w;
  int nblk;
  if (fm_status e = shard_ws(ws, ws_size, B, N, &w, &nblk)) return e;
  uint32_t* xh = reinterpret_cast<uint32_t*>(hist);
  dim3 grid(nblk, B);
  if (pass == 0) topk_hist_kernel<0, false><<<grid, kThreads, 0, st>>>(w, ens, N, xh);
  else if (pass == 1) topk_hist_kernel<1, false><<<grid, kThreads, 0, st>>>(w, ens, N, xh);
  else topk_hist_kernel<2, false><<<grid, kThreads, 0, st>>>(w, ens, N, xh);
  note_launch();
  return check_launch();
}

fm_status launch_topk_shard_pick(int B, int N, int pass, int32_t* hist, void* ws, size_t ws_size,
                                 cudaStream_t st) {
  Workspace w;
  int nblk;
  if (fm_status e = shard_ws(ws, ws_size, B, N, &w, &nblk)) return e;
  uint32_t* xh = reinterpret_cast<uint32_t*>(hist);
  if (pass == 0) topk_shard_pick_kernel<0><<<B, kThreads, 0, st>>>(w, xh);
  else if (pass == 1) topk_shard_pick_kernel<1><<<B, kThreads, 0, st>>>(w, xh);
  else topk_shard_pick_kernel<2><<<B, kThreads, 0, st>>>(w, xh);
  note_launch();
  return check_launch();
}

fm_status launch_topk_shard_ties(const float* ens, int B, int N, int32_t* eq_local, void* ws,
                                 size_t ws_size, cudaStream_t st) {
  Workspace w;
  int nblk;
  if (fm_status e = shard_ws(ws, ws_size, B, N, &w, &nblk)) return e;
  if (cudaMemsetAsync(eq_local, 0, sizeof(int32_t) * (size_t)B, st) != cudaSuccess) return check_launch();
  dim3 grid(nblk, B);
  topk_eqcount_kernel<<<grid, kThreads, 0, st>>>(w, ens, N, nblk, eq_local);
  note_launch();
  return check_launch();
}

fm_status launch_topk_shard_mask(const float* ens, int B, int N, const int32_t* eq_all, int shard,
                                 uint8_t* keep, void* ws, size_t ws_size, cudaStream_t st) {
  Workspace w;
  int nblk;
  if (fm_status e = shard_ws(ws, ws_size, B, N, &w, &nblk)) return e;
  dim3 grid(nblk, B);
  topk_mask_kernel<<<grid, kThreads, 0, st>>>(w, ens, N, nblk, keep, eq_all, shard, B);
  note_launch();
  return check_launch();
}

}  // namespace fm
