// topk_cluster.cu -- the top-K keep mask (README "Usage" select_topk(top_k=K);
// toy decode loop "top-K") of rows of up to 262144 chunks in ONE kernel: a
// thread-block cluster per row, the row's keys held in shared memory, the
// histograms merged through distributed shared memory.
//
// The selection is an exact radix select on the order-preserving 32-bit keys
// of select.cu (larger score -> larger key, +0 = -0, NaN lowest).  The passes
// start at the highest bit in which the row's valid keys differ (found first,
// with one OR over the cluster), 8 bits at a time: sigmoid scores share
// their sign and most of their exponent, and a first pass over the top bits
// would pile them into a few bins.  The passes fix the K-th largest key T and
// how many keys equal to T are kept; the mask keeps every key > T and the
// first `need` keys == T in chunk order.
//
// Layout: cluster of C CTAs (a power of two <= 16) per row, CTA r holds the consecutive
// slice [r*S, (r+1)*S) of the row, S = ceil(N / C) <= 16384, as keys in its
// shared memory (thread t handles keys j*512 + t), so the row is read from
// global memory once.  Per pass: every CTA histograms its keys into its own shared
// histogram (a copy per pair of warps, then summed); a cluster barrier; CTA r sums the bins b with b % C == r over the
// cluster (distributed shared memory reads); a cluster barrier; then every
// CTA reads the C owners' sums and finds the digit itself (all CTAs compute
// the same digit from the same sums).  Histograms and sums are double
// buffered across passes, so two cluster barriers per pass suffice.  Ties at
// T are ranked by chunk index: a CTA's offset is the count of keys == T in
// the CTAs before it, then an in-CTA ordered scan.
#include <cooperative_groups.h>

#include "fm_internal.cuh"
#include "select_block.cuh"

namespace cg = cooperative_groups;

namespace fm {
namespace {

constexpr int kCThreads = kBlkThreads;  // 512
constexpr int kKeysPerThread = 32;
constexpr int kSliceMax = kCThreads * kKeysPerThread;  // 16384 keys per CTA
constexpr int kMaxCluster = 16;
constexpr int kBins = 2048;
constexpr int kTargetSlice = 4096;  // keys per CTA the cluster size aims for

struct ClusterSmem {
  uint32_t hist[2][kBins];  // this CTA's histogram of the pass: counted in kSelCopies
                            // 256-bin copies (one per pair of warps), then summed into
                            // its first kSelBins words
  uint32_t sum[2][kBins];   // bins b with b % C == rank: the cluster's total
  int warp[kCThreads / 32 + 1];
  uint32_t pick[3];         // prefix so far, want, count of keys == T (last pass)
  uint32_t diff;            // OR over this CTA's keys of (key ^ reference key)
  int cta_eq;               // this CTA's keys == T
};

__device__ __forceinline__ uint32_t low_mask(int n) { return n >= 32 ? 0xffffffffu : ((1u << n) - 1u); }

__global__ void __launch_bounds__(kCThreads, 2) topk_cluster_kernel(const float* __restrict__ ens,
                                                                    const int32_t* __restrict__ n_valid, int N,
                                                                    int k, int log2C, uint8_t* __restrict__ keep) {
  __shared__ __align__(16) ClusterSmem S;
  // the slice's keys: key[j * 512 + t] for thread t, ceil(slice / 512) rows of 512
  extern __shared__ __align__(16) uint32_t key[];
  cg::cluster_group cl = cg::this_cluster();
  const int C = 1 << log2C;
  const int rank = (int)cl.block_rank();
  const int b = blockIdx.y;
  const int t = threadIdx.x, lane = t & 31;
  int nv = n_valid ? __ldg(n_valid + b) : N;
  nv = max(0, min(nv, N));
  const int slice = (N + C - 1) / C;
  const int rows = (slice + kCThreads - 1) / kCThreads;  // key rows of 512
  const int base = rank * slice;
  const int end = min(base + slice, N);
  const int vend = min(end, nv);  // valid chunks of this CTA: [base, vend)
  const float* row = ens + (size_t)b * N;
  uint8_t* krow = keep + (size_t)b * N;

  if (k >= nv) {  // every valid chunk is kept (none when the row is empty); uniform over the cluster
    for (int i = base + t; i < end; i += kCThreads) krow[i] = i < nv ? 1 : 0;
    return;
  }

  // load the slice (16 loads in flight per thread) and note which key bits
  // differ from the row's first key: the digit passes start at the highest
  // such bit, so the first pass spreads the keys over its bins instead of
  // piling sigmoid outputs (one exponent or two) into a few of them
  const uint32_t ref = block_order_key(__ldg(row));
  uint32_t diff = 0u;
  for (int j0 = 0; j0 < rows; j0 += 16) {
    float v[16];
#pragma unroll
    for (int u = 0; u < 16; ++u) {
      const int i = base + (j0 + u) * kCThreads + t;
      v[u] = (j0 + u < rows && i < vend) ? __ldg(row + i) : 0.f;
    }
#pragma unroll
    for (int u = 0; u < 16; ++u) {
      if (j0 + u >= rows) break;
      const int i = base + (j0 + u) * kCThreads + t;
      const uint32_t kk = block_order_key(v[u]);
      key[(j0 + u) * kCThreads + t] = kk;
      if (i < vend) diff |= kk ^ ref;
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) diff |= __shfl_xor_sync(0xffffffffu, diff, o);
  if (lane == 0) S.warp[t >> 5] = (int)diff;
  __syncthreads();
  if (t == 0) {
    uint32_t d = 0u;
    for (int w = 0; w < kCThreads / 32; ++w) d |= (uint32_t)S.warp[w];
    S.diff = d;
  }
  cl.sync();  // every CTA's diff is set
  if (t == 0) {
    uint32_t d = 0u;
    for (int r = 0; r < C; ++r) d |= *cl.map_shared_rank(&S.diff, r);
    S.pick[0] = d;
  }
  __syncthreads();
  const uint32_t all_diff = S.pick[0];
  __syncthreads();

  // radix passes over the bits below the highest differing bit, 8 at a time:
  // each pair of warps counts into its own 256-bin copy with plain atomics
  // (equal digits contend within two warps only), and the copies are summed
  int top = all_diff ? 32 - __clz(all_diff) : 0;  // bits [top, 32) are the reference's
  uint32_t prefix = ref & ~low_mask(top), want = (uint32_t)k, cnt_eq = (uint32_t)nv;
#pragma unroll 1
  for (int pass = 0; top > 0; ++pass) {
    const int nbits = top < kSelBits ? top : kSelBits, shift = top - nbits, nb = 1 << nbits;
    uint32_t* h = S.hist[pass & 1];
    uint32_t* sm = S.sum[pass & 1];
    for (int i = t; i < kSelCopies * kSelBins; i += kCThreads) h[i] = 0u;
    __syncthreads();
    uint32_t* my_hist = h + (t >> 6) * kSelBins;
#pragma unroll 4
    for (int j = 0; j < kKeysPerThread; ++j) {
      if (j >= rows) break;
      const int i = base + j * kCThreads + t;
      const uint32_t kk = key[j * kCThreads + t];
      if (i < vend && (top >= 32 || (kk >> top) == (prefix >> top)))
        atomicAdd(&my_hist[(kk >> shift) & (uint32_t)(nb - 1)], 1u);
    }
    __syncthreads();
    if (t < nb) {  // bin t of every copy is read and the sum written by thread t alone
      uint32_t x = 0u;
#pragma unroll
      for (int c = 0; c < kSelCopies; ++c) x += h[c * kSelBins + t];
      h[t] = x;
    }
    cl.sync();  // every CTA's histogram of this pass is complete
    // sum the owned bins over the cluster: pair p = (owned bin q, source CTA
    // src), src the fastest index, so the C sources of a bin sit in C
    // consecutive lanes and are added with shuffles
    const int pairs = ((nb + C - 1) >> log2C) << log2C;
    for (int p0 = 0; p0 < pairs; p0 += kCThreads) {
      const int p = p0 + t;
      const int src = p & (C - 1);
      const int bin = ((p >> log2C) << log2C) + rank;
      uint32_t x = (p < pairs && bin < nb) ? cl.map_shared_rank(h, src)[bin] : 0u;
      for (int o = 1; o < C; o <<= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
      if (p < pairs && src == 0 && bin < nb) sm[bin] = x;
    }
    cl.sync();  // the owners' sums are complete
    // thread t takes bins [t*per, (t+1)*per) in descending digit order
    const int per = (nb + kCThreads - 1) / kCThreads;
    uint32_t c[4];
    uint32_t mine = 0u;
#pragma unroll
    for (int jj = 0; jj < 4; ++jj) {
      c[jj] = 0u;
      const int pos = t * per + jj;
      if (jj < per && pos < nb) {
        const int d = nb - 1 - pos;
        c[jj] = cl.map_shared_rank(sm, d & (C - 1))[d];
        mine += c[jj];
      }
    }
    int tot;
    const uint32_t before = (uint32_t)block_exclusive_scan((int)mine, S.warp, &tot);
    if (before < want && before + mine >= want) {
      uint32_t acc = before;
#pragma unroll
      for (int jj = 0; jj < 4; ++jj) {
        if (jj >= per) break;
        const int d = nb - 1 - (t * per + jj);
        if (acc + c[jj] >= want) {
          S.pick[0] = prefix | ((uint32_t)d << shift);
          S.pick[1] = want - acc;
          S.pick[2] = c[jj];
          break;
        }
        acc += c[jj];
      }
    }
    __syncthreads();
    prefix = S.pick[0];
    want = S.pick[1];
    cnt_eq = S.pick[2];
    top = shift;
  }
  const uint32_t T = prefix;
  const uint32_t need = want;  // keys == T to keep (all valid keys equal T when no pass ran)

  if (cnt_eq == need) {  // every key equal to T is kept
#pragma unroll 4
    for (int j = 0; j < kKeysPerThread; ++j) {
      if (j >= rows) break;
      const int i = base + j * kCThreads + t;
      if (i < end) krow[i] = (i < vend && key[j * kCThreads + t] >= T) ? 1 : 0;
    }
  } else {
    // rank the keys equal to T in chunk order: the CTAs before this one first
    int mine = 0;
#pragma unroll 4
    for (int j = 0; j < kKeysPerThread; ++j) {
      if (j >= rows) break;
      const int i = base + j * kCThreads + t;
      mine += (i < vend && key[j * kCThreads + t] == T) ? 1 : 0;
    }
    int tot;
    block_exclusive_scan(mine, S.warp, &tot);
    if (t == 0) S.cta_eq = tot;
    cl.sync();
    uint32_t running = 0u;
    for (int r = 0; r < rank; ++r) running += (uint32_t)*cl.map_shared_rank(&S.cta_eq, r);
#pragma unroll 1
    for (int j = 0; j < kKeysPerThread; ++j) {
      if (j >= rows) break;
      const int i = base + j * kCThreads + t;
      const bool valid = i < vend;
      const uint32_t kk = key[j * kCThreads + t];
      const bool eq = valid && kk == T;
      int all;
      const uint32_t r_in = (uint32_t)block_exclusive_scan(eq ? 1 : 0, S.warp, &all);
      if (i < end) krow[i] = (valid && (kk > T || (eq && running + r_in < need))) ? 1 : 0;
      running += (uint32_t)all;
    }
  }
  cl.sync();  // no CTA leaves while another may still read its shared memory
}

}  // namespace

// The cluster size for rows of N chunks, a power of two (0 when N is beyond
// the one-kernel form).
int topk_cluster_size(int N) {
  const int need = (N + kSliceMax - 1) / kSliceMax;
  if (need > kMaxCluster) return 0;
  if (need == 1) return 1;  // one CTA holds the row
  const int want = (N + kTargetSlice - 1) / kTargetSlice;
  int C = 1;
  while (C < need || (C < want && C < kMaxCluster)) C <<= 1;
  return C;
}

// Rows that fm_select_topk hands to the one-kernel form: up to one CTA's
// slice.  Measured on B200 at 1, 8, 32 and 64 rows of 65536 to 262144 chunks,
// the multi-CTA clusters were slower than the candidate path (for 64 rows of
// 262144, 0.33 ms against 0.09 ms); at 4096 chunks one CTA took half the time
// of the histogram passes' six launches.
bool topk_use_cluster(int N) { return N <= kSliceMax; }

fm_status launch_topk_cluster(const float* ens, const int32_t* n_valid, int B, int N, int k, uint8_t* keep,
                              cudaStream_t st) {
  const int C = topk_cluster_size(N);
  if (C == 0 || B > 65535) return FM_ERR_UNSUPPORTED;
  static PerDeviceOnce attr_set;
  int dev = 0;
  cudaGetDevice(&dev);
  fm_status s = attr_set.run(dev, [] {
    cudaError_t e = cudaFuncSetAttribute(topk_cluster_kernel, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(topk_cluster_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               (int)(sizeof(uint32_t) * kSliceMax));
    return e == cudaSuccess ? FM_OK : record_cuda_error(e);
  });
  if (s != FM_OK) return s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = (unsigned)C;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)C, (unsigned)B);
  cfg.blockDim = dim3(kCThreads);
  // thread t touches key[j * 512 + t] for every j with j * 512 < slice: the
  // slice is held rounded up to whole rows of 512 keys
  const int slice = (N + C - 1) / C;
  cfg.dynamicSmemBytes = sizeof(uint32_t) * (size_t)(((slice + kCThreads - 1) / kCThreads) * kCThreads);
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int log2C = 0;
  while ((1 << log2C) < C) ++log2C;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, topk_cluster_kernel, ens, n_valid, N, k, log2C, keep);
  note_launch();
  return e == cudaSuccess ? FM_OK : record_cuda_error(e);
}

}  // namespace fm
