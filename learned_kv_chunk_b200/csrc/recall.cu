// recall.cu -- from a keep mask to a resident set on the GPU.
//
// The model card's "How it works": every 64 decode steps the Memory Indexer
// selects the query-critical chunks, and that resident set is recalled from
// the CPU-side bulk KV cache to the GPU; only recalled chunks and the
// compressed indexer keys live on the GPU.  Two steps follow the keep mask:
//
//   compaction  keep [B, N] -> idx [B, max_sel] (kept chunk indices in
//               increasing order, -1 past the end) and count [B];
//   gather      for j < min(count[b], max_sel): copy the fixed-size record of
//               chunk idx[b, j] from a bulk store (pinned host memory, read
//               over the bus by the SMs, or device memory) into slot j of a
//               resident buffer on the GPU.
//
// Compaction is one launch with a cluster of up to 4 CTAs per row: each CTA
// counts the kept entries of its part of the mask (landed in shared memory
// by bulk copies when the row starts on 16 bytes), the cluster exchanges the
// counts through distributed shared memory, and each CTA writes its indices
// at the offset the CTAs before it leave.  The gather from device memory
// stages each record's 16-byte granules in shared memory with one bulk copy
// per record and writes tiles of consecutive slots out with 4-byte stores;
// from pinned host memory (or off the 4-byte grid) it is a copy with one
// warp per record and several records in flight per warp.  The selected
// records are scattered, so the copy engines (one call per contiguous run)
// are not used.
#include <cooperative_groups.h>

#include "fm_internal.cuh"

namespace fm {
namespace {

__device__ int g_recall_err;  // kDevErrTimeout once a bulk-copy wait ran out

constexpr int kCThreads = 512;
constexpr int kCBytes = 32;                      // mask bytes per thread
constexpr int kCChunk = kCThreads * kCBytes;     // mask bytes per block

__host__ __device__ inline int compact_blocks(int N) { return (int)(((int64_t)N + kCChunk - 1) / kCChunk); }

// Bit 4i + k set when byte k of word i is nonzero: the kept entries among a
// thread's 32 mask bytes, in byte order.
__device__ __forceinline__ uint32_t kept_bits(const uint32_t (&w)[8]) {
  uint32_t m = 0;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const uint32_t x = __vcmpne4(w[i], 0u) & 0x80808080u;  // the top bit of each nonzero byte
    m |= (((x >> 7) | (x >> 14) | (x >> 21) | (x >> 28)) & 0xfu) << (4 * i);
  }
  return m;
}

// The kept bits of this thread's 32 mask bytes from n0 (bytes past N read as 0).
__device__ __forceinline__ uint32_t load_mask(const uint8_t* __restrict__ row, int64_t n0, int N, bool vec) {
  uint32_t w[8];
  if (vec && n0 + kCBytes <= N) {
    const uint4 a = __ldg(reinterpret_cast<const uint4*>(row + n0));
    const uint4 c = __ldg(reinterpret_cast<const uint4*>(row + n0 + 16));
    w[0] = a.x; w[1] = a.y; w[2] = a.z; w[3] = a.w;
    w[4] = c.x; w[5] = c.y; w[6] = c.z; w[7] = c.w;
  } else {
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      uint32_t x = 0;
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const int64_t n = n0 + 4 * i + k;
        if (n < N) x |= (uint32_t)row[n] << (8 * k);
      }
      w[i] = x;
    }
  }
  return kept_bits(w);
}

// Writes the chunk indices n0 + (bit positions of m) to out[pos ..] in order,
// below max_sel.
__device__ __forceinline__ void write_kept(uint32_t m, int64_t n0, int pos, int max_sel, int32_t* __restrict__ out) {
  for (; m != 0u && pos < max_sel; m &= m - 1u) out[pos++] = (int32_t)(n0 + __ffs(m) - 1);
}

__device__ __forceinline__ bool row_vec_ok(const uint8_t* keep, int N) {
  return (N & 15) == 0 && (reinterpret_cast<uintptr_t>(keep) & 15u) == 0;
}

// Exclusive scan of one int per thread over the block (thread order); also
// returns the block's total.  Two __syncthreads; s_warp has kCThreads/32 ints.
__device__ __forceinline__ int block_exclusive_scan(int v, int* s_warp, int& total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int u = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += u;
  }
  if (lane == 31) s_warp[warp] = incl;
  __syncthreads();
  int before = 0;
  total = 0;
#pragma unroll
  for (int i = 0; i < kCThreads / 32; ++i) {
    const int x = s_warp[i];
    before += i < warp ? x : 0;
    total += x;
  }
  __syncthreads();  // s_warp may be rewritten by the next scan
  return before + incl - v;
}

// One cluster of C <= 4 CTAs per row (blockIdx.y; 4 measured faster than 2
// or 8 on 64 rows of 262144); CTA r of the cluster takes the
// mask chunks [r*nch/C, (r+1)*nch/C) of kCChunk bytes.  Pass 1 counts its
// kept entries; the CTAs exchange their totals through distributed shared
// memory, so every CTA knows how many kept entries of the row come before
// its part; pass 2 writes its indices in order (the first two chunks from
// registers, later ones re-read, from L2).  The cluster's last CTA writes
// the count and the -1 tail.  One read of the mask from DRAM, one launch.
__global__ void __launch_bounds__(kCThreads) compact_cluster_kernel(const uint8_t* __restrict__ keep, int N,
                                                                    int max_sel, int32_t* __restrict__ idx,
                                                                    int32_t* __restrict__ count) {
  namespace cg = cooperative_groups;
  cg::cluster_group cl = cg::this_cluster();
  __shared__ int s_warp[kCThreads / 32];
  __shared__ int s_total;
  const int b = blockIdx.y;
  const int C = (int)cl.num_blocks();
  const int rank = (int)cl.block_rank();
  const int nch = compact_blocks(N);
  const int j0 = (int)((int64_t)nch * rank / C), j1 = (int)((int64_t)nch * (rank + 1) / C);
  const uint8_t* row = keep + (int64_t)b * N;
  const bool vec = row_vec_ok(keep, N);
  const int64_t tb = (int64_t)threadIdx.x * kCBytes;
  // the first two chunks' kept bits stay in registers for pass 2
  const uint32_t m0 = j0 < j1 ? load_mask(row, (int64_t)j0 * kCChunk + tb, N, vec) : 0u;
  const uint32_t m1 = j0 + 1 < j1 ? load_mask(row, (int64_t)(j0 + 1) * kCChunk + tb, N, vec) : 0u;
  int mine = __popc(m0) + __popc(m1);
  for (int j = j0 + 2; j < j1; ++j) mine += __popc(load_mask(row, (int64_t)j * kCChunk + tb, N, vec));
  int cta_total;
  (void)block_exclusive_scan(mine, s_warp, cta_total);
  if (threadIdx.x == 0) s_total = cta_total;
  cl.sync();
  int before = 0, row_total = 0;
  for (int r = 0; r < C; ++r) {
    const int x = *cl.map_shared_rank(&s_total, r);
    before += r < rank ? x : 0;
    row_total += x;
  }
  cl.sync();  // no CTA leaves while another reads its total
  int32_t* out = idx + (size_t)b * max_sel;
  int base = before;
  // writes one chunk's kept indices in order from `base`
  auto write_chunk = [&](int j, uint32_t m) {
    int chunk_total;
    const int pos = base + block_exclusive_scan(__popc(m), s_warp, chunk_total);
    write_kept(m, (int64_t)j * kCChunk + tb, pos, max_sel, out);
    base += chunk_total;
  };
  if (j0 < j1 && base < max_sel) write_chunk(j0, m0);
  if (j0 + 1 < j1 && base < max_sel) write_chunk(j0 + 1, m1);
  for (int j = j0 + 2; j < j1 && base < max_sel; ++j) write_chunk(j, load_mask(row, (int64_t)j * kCChunk + tb, N, vec));
  if (rank == C - 1) {
    if (threadIdx.x == 0) count[b] = row_total;
    for (int j = row_total + (int)threadIdx.x; j < max_sel; j += kCThreads) out[j] = -1;
  }
}

// The same compaction with the CTA's part of the mask landed in shared
// memory by bulk copies (rows that start on 16 bytes and parts of at most
// kCPartChunks chunks): one copy latency for the whole part and no re-read.
// Each thread scans the counts of its 32 bytes of every chunk at once, so
// the CTA's total, every chunk's total and every thread's offsets come from
// one block-wide scan.  Every CTA of the cluster takes both cluster barriers,
// whatever its copies did.
constexpr int kCPartChunks = 4;  // 64 KB of shared memory

// The kept bits of this thread's 32 bytes of chunk c of the part (N is a
// multiple of 16; bytes past it read as 0).
__device__ __forceinline__ uint32_t smem_mask(const uint8_t* part, int c, int64_t n0, int N) {
  const uint8_t* p = part + (size_t)c * kCChunk + threadIdx.x * kCBytes;
  const uint4 a = n0 + 16 <= N ? *reinterpret_cast<const uint4*>(p) : make_uint4(0u, 0u, 0u, 0u);
  const uint4 d = n0 + 32 <= N ? *reinterpret_cast<const uint4*>(p + 16) : make_uint4(0u, 0u, 0u, 0u);
  const uint32_t w[8] = {a.x, a.y, a.z, a.w, d.x, d.y, d.z, d.w};
  return kept_bits(w);
}

__global__ void __launch_bounds__(kCThreads) compact_bulk_kernel(const uint8_t* __restrict__ keep, int N,
                                                                 int max_sel, int32_t* __restrict__ idx,
                                                                 int32_t* __restrict__ count, uint64_t wait_ns) {
  namespace cg = cooperative_groups;
  cg::cluster_group cl = cg::this_cluster();
  extern __shared__ __align__(16) uint8_t s_part[];  // [kCPartChunks][kCChunk]
  __shared__ __align__(8) uint64_t bar;
  __shared__ int s_warp[kCPartChunks][kCThreads / 32];
  __shared__ int s_total;
  __shared__ int s_abort;
  const int b = blockIdx.y, t = threadIdx.x, lane = t & 31, warp = t >> 5;
  const int C = (int)cl.num_blocks();
  const int rank = (int)cl.block_rank();
  const int nch = compact_blocks(N);
  const int j0 = (int)((int64_t)nch * rank / C), j1 = (int)((int64_t)nch * (rank + 1) / C);
  const uint8_t* row = keep + (int64_t)b * N;
  if (t == 0) {
    mbar_init(&bar, 1);
    s_abort = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    uint32_t bytes = 0;
    for (int j = j0; j < j1; ++j) bytes += (uint32_t)min((int64_t)kCChunk, (int64_t)N - (int64_t)j * kCChunk);
    mbar_arrive_expect_tx(&bar, bytes);
    for (int j = j0; j < j1; ++j)
      bulk_g2s(s_part + (size_t)(j - j0) * kCChunk, row + (int64_t)j * kCChunk,
               (uint32_t)min((int64_t)kCChunk, (int64_t)N - (int64_t)j * kCChunk), &bar);
  }
  __syncthreads();  // the barrier is initialised
  const bool ok = mbar_wait_bounded(&bar, 0, &s_abort, &g_recall_err, wait_ns);
  if (!ok) mbar_drain(&bar, 0, &g_recall_err);
  // this thread's kept entries in each chunk of the part, scanned over the
  // block for all chunks at once
  uint32_t m[kCPartChunks];
  int c[kCPartChunks], incl[kCPartChunks];
#pragma unroll
  for (int q = 0; q < kCPartChunks; ++q) {
    m[q] = ok && j0 + q < j1 ? smem_mask(s_part, q, (int64_t)(j0 + q) * kCChunk + t * kCBytes, N) : 0u;
    c[q] = __popc(m[q]);
    incl[q] = c[q];
  }
#pragma unroll
  for (int o = 1; o < 32; o <<= 1)
#pragma unroll
    for (int q = 0; q < kCPartChunks; ++q) {
      const int u = __shfl_up_sync(0xffffffffu, incl[q], o);
      if (lane >= o) incl[q] += u;
    }
  if (lane == 31)
#pragma unroll
    for (int q = 0; q < kCPartChunks; ++q) s_warp[q][warp] = incl[q];
  __syncthreads();
  int before[kCPartChunks], chunk_total[kCPartChunks], cta_total = 0;
#pragma unroll
  for (int q = 0; q < kCPartChunks; ++q) {
    before[q] = 0;
    chunk_total[q] = 0;
#pragma unroll
    for (int i = 0; i < kCThreads / 32; ++i) {
      const int x = s_warp[q][i];
      before[q] += i < warp ? x : 0;
      chunk_total[q] += x;
    }
    cta_total += chunk_total[q];
  }
  if (t == 0) s_total = cta_total;
  cl.sync();
  int base = 0, row_total = 0;
  for (int r = 0; r < C; ++r) {
    const int x = *cl.map_shared_rank(&s_total, r);
    base += r < rank ? x : 0;
    row_total += x;
  }
  cl.sync();  // no CTA leaves while another reads its total
  int32_t* out = idx + (size_t)b * max_sel;
#pragma unroll
  for (int q = 0; q < kCPartChunks; ++q) {
    write_kept(m[q], (int64_t)(j0 + q) * kCChunk + t * kCBytes, base + before[q] + incl[q] - c[q], max_sel, out);
    base += chunk_total[q];
  }
  if (rank == C - 1) {
    if (t == 0) count[b] = row_total;
    for (int j = row_total + t; j < max_sel; j += kCThreads) out[j] = -1;
  }
}

// One warp per record, RU records in flight per warp, each lane moving UPL
// units of VEC bytes per record per round; a record's index and its row's
// count are loaded side by side, so a round waits on one load before the
// record's own.
template <int VEC>
struct Unit;
template <>
struct Unit<16> { using T = uint4; };
template <>
struct Unit<4> { using T = uint32_t; };
template <>
struct Unit<1> { using T = uint8_t; };

template <int VEC>
__global__ void __launch_bounds__(256) gather_kernel(const uint8_t* __restrict__ src, int64_t src_stride,
                                                     int n_src, int64_t rec, const int32_t* __restrict__ idx,
                                                     const int32_t* __restrict__ count, int max_sel,
                                                     int64_t total, uint8_t* __restrict__ dst,
                                                     int64_t dst_stride) {
  using U = typename Unit<VEC>::T;
  constexpr int RU = 8, UPL = 2;
  const int lane = threadIdx.x & 31;
  const int64_t gw = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int64_t nw = ((int64_t)gridDim.x * blockDim.x) >> 5;
  const int64_t units = rec / VEC;
  for (int64_t r0 = gw * RU; r0 < total; r0 += nw * RU) {
    const U* s[RU];
    U* d[RU];
    // (row, slot) of record r0, then stepped: one division per round
    int b = (int)(r0 / max_sel), j = (int)(r0 - (int64_t)b * max_sel);
#pragma unroll
    for (int q = 0; q < RU; ++q, ++j) {
      s[q] = nullptr;
      d[q] = nullptr;
      if (j == max_sel) {
        j = 0;
        ++b;
      }
      const int64_t r = r0 + q;
      if (r < total) {
        const int cnt = min(__ldg(count + b), max_sel);
        const int id = __ldg(idx + r);  // in bounds whatever the count: loaded beside it, not after it
        const int n = j < cnt ? id : -1;
        if (n >= 0 && n < n_src) {
          s[q] = reinterpret_cast<const U*>(src + b * src_stride + (int64_t)n * rec);
          d[q] = reinterpret_cast<U*>(dst + b * dst_stride + (int64_t)j * rec);
        }
      }
    }
    for (int64_t u0 = 0; u0 < units; u0 += 32 * UPL) {
      U v[RU][UPL];
#pragma unroll
      for (int q = 0; q < RU; ++q)
#pragma unroll
        for (int i = 0; i < UPL; ++i) {
          const int64_t u = u0 + i * 32 + lane;
          if (s[q] && u < units) v[q][i] = s[q][u];
        }
#pragma unroll
      for (int q = 0; q < RU; ++q)
#pragma unroll
        for (int i = 0; i < UPL; ++i) {
          const int64_t u = u0 + i * 32 + lane;
          if (d[q] && u < units) d[q][u] = v[q][i];
        }
    }
  }
}

// The bulk gather, for a source in device memory and records, pointers and
// strides that are multiples of 4 bytes.  CTA (b, tile) takes T consecutive
// slots of row b: thread t < T copies the 16-byte granules that record
// idx[b, j0 + t] touches into shared slot t with one bulk copy (the TMA
// engine wants 16-byte aligned addresses and sizes; the granules of a
// record lie in the pages that hold it, so the extra bytes read are
// harmless), all copies completing on one barrier; the warps then write the
// T records out with 4-byte stores, the slots of a row being contiguous in
// dst.  No registers hold data in flight, so the many CTAs an SM holds
// overlap their copies' latencies (64 slots of 132-byte records per CTA, 16
// CTAs per SM, measured faster than 128 slots and 11).  A persistent form
// with two stages per CTA, writing one tile while the next one's copies fly,
// measured slower.
constexpr int kGThreads = 128;        // threads per CTA; T <= kGThreads
constexpr int kGStageBytes = 9216;    // staging shared memory per CTA (T * slot at most)

// Bytes of a record's slot: the 16-byte granules of a record that starts
// 0, 4, 8 or 12 bytes past a granule boundary.
__host__ __device__ inline int gather_slot_bytes(int64_t rec) { return (int)((rec + 12 + 15) & ~(int64_t)15); }

// Records per tile for the bulk gather; 0 when a record is too large for it.
inline int gather_tile(int64_t rec) {
  if (rec > kGStageBytes) return 0;
  const int slot = gather_slot_bytes(rec);
  int T = kGThreads;
  while (T > 8 && T * slot > kGStageBytes) T >>= 1;
  return T * slot <= kGStageBytes ? T : 0;
}

__global__ void __launch_bounds__(kGThreads) gather_bulk_kernel(
    const uint8_t* __restrict__ src, int64_t src_stride, int n_src, int rec,
    const int32_t* __restrict__ idx, const int32_t* __restrict__ count, int max_sel, int tiles_per_row,
    int T, uint8_t* __restrict__ dst, int64_t dst_stride, uint64_t wait_ns) {
  extern __shared__ __align__(16) uint8_t s_stage[];  // [T][slot]
  __shared__ __align__(8) uint64_t bar;
  __shared__ int s_off[kGThreads];  // record t's byte offset in its slot; -1: no record
  __shared__ int s_abort;
  const int t = threadIdx.x;
  const int b = (int)(blockIdx.x / (unsigned)tiles_per_row);
  const int j0 = (int)(blockIdx.x - (unsigned)b * (unsigned)tiles_per_row) * T;
  if (t == 0) {
    mbar_init(&bar, kGThreads);
    s_abort = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  grid_dependency_wait();  // idx and count come from the kernel before this one
  const int cnt = min(__ldg(count + b), max_sel);
  if (j0 >= cnt) return;  // uniform: nothing of this tile is selected
  const int nt = min(T, cnt - j0);
  const int id = t < nt ? __ldg(idx + (int64_t)b * max_sel + j0 + t) : -1;
  const int slot = gather_slot_bytes(rec);
  __syncthreads();  // the barrier is initialised
  if (id >= 0 && id < n_src) {
    const uintptr_t a = reinterpret_cast<uintptr_t>(src + b * src_stride + (int64_t)id * rec);
    const uintptr_t a0 = a & ~(uintptr_t)15, a1 = (a + (uintptr_t)rec + 15) & ~(uintptr_t)15;
    s_off[t] = (int)(a - a0);
    mbar_arrive_expect_tx(&bar, (uint32_t)(a1 - a0));
    bulk_g2s(s_stage + t * slot, reinterpret_cast<const void*>(a0), (uint32_t)(a1 - a0), &bar);
  } else {
    s_off[t] = -1;
    mbar_arrive(&bar);
  }
  const bool ok = mbar_wait_bounded(&bar, 0, &s_abort, &g_recall_err, wait_ns);
  if (__syncthreads_or(!ok)) {  // every thread leaves, after the copies have landed
    mbar_drain(&bar, 0, &g_recall_err);
    return;
  }
  // record r by warp r % 4: its words to dst, 128 contiguous bytes a store
  const int lane = t & 31, words = rec >> 2;
  uint8_t* drow = dst + b * dst_stride + (int64_t)j0 * rec;
  for (int r = t >> 5; r < nt; r += kGThreads / 32) {
    const int o = s_off[r];
    if (o < 0) continue;
    const uint32_t* s = reinterpret_cast<const uint32_t*>(s_stage + r * slot + o);
    uint32_t* d = reinterpret_cast<uint32_t*>(drow + (int64_t)r * rec);
    for (int k = lane; k < words; k += 32) d[k] = s[k];
  }
}

// Device address of `p` for kernels (pinned host memory maps into the GPU's
// address space); null for pageable host memory.  *on_device tells device
// (or managed) memory from pinned host memory.
const void* device_address(const void* p, bool* on_device = nullptr) {
  cudaPointerAttributes a;
  if (cudaPointerGetAttributes(&a, p) != cudaSuccess) {
    cudaGetLastError();
    return nullptr;
  }
  if (on_device) *on_device = a.type == cudaMemoryTypeDevice;
  if (a.type == cudaMemoryTypeDevice || a.type == cudaMemoryTypeManaged) return p;
  if (a.type == cudaMemoryTypeHost) return a.devicePointer;
  return nullptr;
}

}  // namespace
}  // namespace fm

namespace fm {

int take_recall_error() {
  int h = kDevErrNone;
  if (cudaMemcpyFromSymbol(&h, g_recall_err, sizeof(int)) != cudaSuccess) {
    cudaGetLastError();
    return kDevErrNone;
  }
  if (h != kDevErrNone) {
    const int zero = kDevErrNone;
    cudaMemcpyToSymbol(g_recall_err, &zero, sizeof(int));
  }
  return h;
}

// The cluster kernel needs no workspace; the entry point keeps its argument.
size_t compact_workspace_bytes(int B, int N) {
  (void)B;
  (void)N;
  return 256;
}

int compact_cluster_size(int N) { return compact_blocks(N) < 4 ? compact_blocks(N) : 4; }

fm_status launch_compact(const uint8_t* keep, int B, int N, int max_sel, int32_t* idx, int32_t* count,
                         void* ws, cudaStream_t stream) {
  (void)ws;
  if (B > 65535) return FM_ERR_UNSUPPORTED;
  const int C = compact_cluster_size(N);
  const int part = (compact_blocks(N) + C - 1) / C;  // chunks of the largest part
  const bool bulk = (N & 15) == 0 && (reinterpret_cast<uintptr_t>(keep) & 15u) == 0 && part <= kCPartChunks;
  const int smem = bulk ? part * kCChunk : 0;
  if (bulk) {
    static PerDeviceOnce smem_set;
    int dev = 0;
    cudaGetDevice(&dev);
    if (fm_status s = smem_limit_once(smem_set, dev, compact_bulk_kernel, kCPartChunks * kCChunk)) return s;
  }
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = (unsigned)C;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)C, (unsigned)B);
  cfg.blockDim = dim3(kCThreads);
  cfg.dynamicSmemBytes = (size_t)smem;
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const cudaError_t e =
      bulk ? cudaLaunchKernelEx(&cfg, compact_bulk_kernel, keep, N, max_sel, idx, count, kWaitLimitNs)
           : cudaLaunchKernelEx(&cfg, compact_cluster_kernel, keep, N, max_sel, idx, count);
  note_launch();
  return e == cudaSuccess ? check_launch() : record_cuda_error(e);
}

fm_status launch_gather(const void* src, bool src_on_device, int64_t src_row_stride_bytes, int n_src,
                        int64_t rec_bytes, const int32_t* idx, const int32_t* count, int B, int max_sel,
                        void* dst, int64_t dst_row_stride_bytes, cudaStream_t stream) {
  const uint8_t* s = static_cast<const uint8_t*>(src);
  uint8_t* d = static_cast<uint8_t*>(dst);
  auto all_aligned = [&](uintptr_t a) {
    return (reinterpret_cast<uintptr_t>(s) % a) == 0 && (reinterpret_cast<uintptr_t>(d) % a) == 0 &&
           rec_bytes % (int64_t)a == 0 && src_row_stride_bytes % (int64_t)a == 0 &&
           dst_row_stride_bytes % (int64_t)a == 0;
  };
  const int T = gather_tile(rec_bytes);
  const int tiles_per_row = T > 0 ? (max_sel + T - 1) / T : 0;
  // records of under 64 bytes are few bytes per copy: the plain kernel moves them
  if (src_on_device && rec_bytes >= 64 && T > 0 && all_aligned(4) && (int64_t)B * tiles_per_row <= INT32_MAX) {
    const cudaError_t e = launch_overlapped(
        gather_bulk_kernel, dim3((unsigned)(B * tiles_per_row)), dim3(kGThreads),
        (size_t)T * gather_slot_bytes(rec_bytes), stream, s, src_row_stride_bytes, n_src, (int)rec_bytes, idx,
        count, max_sel, tiles_per_row, T, d, dst_row_stride_bytes, kWaitLimitNs);
    note_launch();
    return e == cudaSuccess ? check_launch() : record_cuda_error(e);
  }
  const int64_t total = (int64_t)B * max_sel;
  int sms = 148;
  int dev = 0;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t want = (total + 8 * 8 - 1) / (8 * 8);  // 8 warps of 256 threads, 8 records each
  const int grid = (int)(want < (int64_t)sms * 8 ? (want > 0 ? want : 1) : (int64_t)sms * 8);
  if (all_aligned(16))
    gather_kernel<16><<<grid, 256, 0, stream>>>(s, src_row_stride_bytes, n_src, rec_bytes, idx, count,
                                                max_sel, total, d, dst_row_stride_bytes);
  else if (all_aligned(4))
    gather_kernel<4><<<grid, 256, 0, stream>>>(s, src_row_stride_bytes, n_src, rec_bytes, idx, count,
                                               max_sel, total, d, dst_row_stride_bytes);
  else
    gather_kernel<1><<<grid, 256, 0, stream>>>(s, src_row_stride_bytes, n_src, rec_bytes, idx, count,
                                               max_sel, total, d, dst_row_stride_bytes);
  note_launch();
  return check_launch();
}

}  // namespace fm

using namespace fm;

extern "C" size_t fm_compact_workspace_bytes(int B, int N) {
  if (B < 1 || N < 1) return 0;
  return compact_workspace_bytes(B, N);
}

extern "C" fm_status fm_compact_mask(const uint8_t* keep, int B, int N, int max_sel, int32_t* idx,
                                     int32_t* count, void* ws, size_t ws_bytes, cudaStream_t stream) {
  if (!keep || !idx || !count || !ws || B < 1 || N < 1 || max_sel < 1 || B > 65535)
    return FM_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(idx) & 3u) || (reinterpret_cast<uintptr_t>(count) & 3u) ||
      (reinterpret_cast<uintptr_t>(ws) & 15u))
    return FM_ERR_ALIGNMENT;
  if (ws_bytes < compact_workspace_bytes(B, N)) return FM_ERR_INVALID_ARG;
  return launch_compact(keep, B, N, max_sel, idx, count, ws, stream);
}

extern "C" fm_status fm_gather_records(const void* src, int64_t src_row_stride_bytes, int n_src,
                                       int64_t rec_bytes, const int32_t* idx, const int32_t* count, int B,
                                       int max_sel, void* dst, int64_t dst_row_stride_bytes,
                                       cudaStream_t stream) {
  if (!src || !idx || !count || !dst || B < 1 || max_sel < 1 || n_src < 1 || rec_bytes < 1)
    return FM_ERR_INVALID_ARG;
  if (src_row_stride_bytes < (int64_t)n_src * rec_bytes ||
      dst_row_stride_bytes < (int64_t)max_sel * rec_bytes)
    return FM_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(idx) & 3u) || (reinterpret_cast<uintptr_t>(count) & 3u))
    return FM_ERR_ALIGNMENT;
  bool on_device = false;
  const void* s = device_address(src, &on_device);
  if (!s || !device_address(dst)) return FM_ERR_INVALID_ARG;  // pageable host memory
  return launch_gather(s, on_device, src_row_stride_bytes, n_src, rec_bytes, idx, count, B, max_sel, dst,
                       dst_row_stride_bytes, stream);
}

