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
// counts the kept entries of its part of the mask, the cluster exchanges the
// counts through distributed shared memory, and each CTA writes its indices
// at the offset the CTAs before it leave.  The gather is a copy
// with one warp per record and several records in flight per warp: the
// selected records are scattered, so the copy engines (one call per
// contiguous run) are not used.
#include <cooperative_groups.h>

#include "fm_internal.cuh"

namespace fm {
namespace {

constexpr int kCThreads = 512;
constexpr int kCBytes = 32;                      // mask bytes per thread
constexpr int kCChunk = kCThreads * kCBytes;     // mask bytes per block

__host__ __device__ inline int compact_blocks(int N) { return (int)(((int64_t)N + kCChunk - 1) / kCChunk); }

// The 32 mask bytes of this thread as eight words (bytes past N read as 0),
// and how many of them are nonzero.
__device__ __forceinline__ int load_mask(const uint8_t* __restrict__ row, int64_t n0, int N, bool vec,
                                         uint32_t w[8]) {
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
  int c = 0;
#pragma unroll
  for (int i = 0; i < 8; ++i) c += __popc(__vcmpne4(w[i], 0u)) >> 3;
  return c;
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
  // the first two chunks stay in registers for pass 2
  uint32_t w0[8] = {}, w1[8] = {};
  int c0 = 0, c1 = 0, mine = 0;
  if (j0 < j1) c0 = load_mask(row, (int64_t)j0 * kCChunk + tb, N, vec, w0);
  if (j0 + 1 < j1) c1 = load_mask(row, (int64_t)(j0 + 1) * kCChunk + tb, N, vec, w1);
  mine = c0 + c1;
  for (int j = j0 + 2; j < j1; ++j) {
    uint32_t t[8];
    mine += load_mask(row, (int64_t)j * kCChunk + tb, N, vec, t);
  }
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
  // writes one chunk's kept indices in order from `base`; returns the chunk's total
  auto write_chunk = [&](int j, const uint32_t (&t)[8], int cj) {
    const int64_t n0 = (int64_t)j * kCChunk + tb;
    int chunk_total;
    int pos = base + block_exclusive_scan(cj, s_warp, chunk_total);
    if (cj) {
#pragma unroll
      for (int i = 0; i < 8; ++i) {
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          if ((t[i] >> (8 * k)) & 0xffu) {
            if (pos < max_sel) out[pos] = (int32_t)(n0 + 4 * i + k);
            ++pos;
          }
        }
      }
    }
    base += chunk_total;
  };
  if (j0 < j1 && base < max_sel) write_chunk(j0, w0, c0);
  if (j0 + 1 < j1 && base < max_sel) write_chunk(j0 + 1, w1, c1);
  for (int j = j0 + 2; j < j1 && base < max_sel; ++j) {
    uint32_t t[8];
    const int cj = load_mask(row, (int64_t)j * kCChunk + tb, N, vec, t);
    write_chunk(j, t, cj);
  }
  if (rank == C - 1) {
    if (threadIdx.x == 0) count[b] = row_total;
    for (int j = row_total + (int)threadIdx.x; j < max_sel; j += kCThreads) out[j] = -1;
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

// Device address of `p` for kernels (pinned host memory maps into the GPU's
// address space); null for pageable host memory.
const void* device_address(const void* p) {
  cudaPointerAttributes a;
  if (cudaPointerGetAttributes(&a, p) != cudaSuccess) {
    cudaGetLastError();
    return nullptr;
  }
  if (a.type == cudaMemoryTypeDevice || a.type == cudaMemoryTypeManaged) return p;
  if (a.type == cudaMemoryTypeHost) return a.devicePointer;
  return nullptr;
}

}  // namespace
}  // namespace fm

namespace fm {

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
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = (unsigned)compact_cluster_size(N);
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(attr[0].val.clusterDim.x, (unsigned)B);
  cfg.blockDim = dim3(kCThreads);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, compact_cluster_kernel, keep, N, max_sel, idx, count);
  note_launch();
  return e == cudaSuccess ? check_launch() : record_cuda_error(e);
}

fm_status launch_gather(const void* src, int64_t src_row_stride_bytes, int n_src, int64_t rec_bytes,
                        const int32_t* idx, const int32_t* count, int B, int max_sel, void* dst,
                        int64_t dst_row_stride_bytes, cudaStream_t stream) {
  const uint8_t* s = static_cast<const uint8_t*>(src);
  uint8_t* d = static_cast<uint8_t*>(dst);
  auto all_aligned = [&](uintptr_t a) {
    return (reinterpret_cast<uintptr_t>(s) % a) == 0 && (reinterpret_cast<uintptr_t>(d) % a) == 0 &&
           rec_bytes % (int64_t)a == 0 && src_row_stride_bytes % (int64_t)a == 0 &&
           dst_row_stride_bytes % (int64_t)a == 0;
  };
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
  const void* s = device_address(src);
  if (!s || !device_address(dst)) return FM_ERR_INVALID_ARG;  // pageable host memory
  return launch_gather(s, src_row_stride_bytes, n_src, rec_bytes, idx, count, B, max_sel, dst,
                       dst_row_stride_bytes, stream);
}

