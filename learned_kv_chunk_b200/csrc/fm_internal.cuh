// fm_internal.cuh -- shared declarations and PTX wrappers of libfm (sm_100a).
//
// Everything here is written for Blackwell (sm_100a): mbarrier-tracked bulk
// copies (the TMA engine's 1-D form), tcgen05 tensor-core MMA with TMEM
// accumulators, and bounded waits that record an error instead of hanging.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>

#include "../../include/fm.h"

namespace fm {

// ---------------------------------------------------------------- constants
constexpr int kHeads = 64;        // N_HEADS (the shipped value; checked at create)
constexpr int kHeadDim = 128;     // HEAD_DIM (README "Architecture")
constexpr int kRopeDim = 64;      // ROPE_DIM (README "Architecture")
constexpr int kRecord = 132;      // bytes per compressed chunk (README "compressed_k format")
constexpr int kTile = 128;        // chunks per tensor-core tile (MMA M, one TMEM lane each)
constexpr int kMaxLayers = 4;
constexpr int kMaxBatch = 4096;

// device error codes written into the context's error word
enum : int { kDevErrNone = 0, kDevErrTimeout = 1 };

}  // namespace fm

// The context behind the opaque fm_ctx handle.
struct fm_ctx {
  fm_config cfg;
  int device;
  int num_sms;
  // weights (device)
  float* w_down;    // [L*(R+H), HID]: per layer wq_a rows then weights_proj rows
  float* q_norm;    // [L, R]
  float* w_up;      // [L, H*D, R]
  double* rope_freq;  // [rope_dim/2] YaRN frequencies (fp64)
  // workspace (device), sized for cfg.max_batch rows
  int splitk_max;
  float* a_part;    // [splitk_max, max_batch, L*(R+H)] partial sums of the down projection
  float* r_norm;    // [max_batch, L, R] RMSNorm output
  float* rope_cs;   // [max_batch, rope_dim/2, 2] cos, sin
  uint8_t* qpack;   // [max_batch, L, q_pieces*64*128] e4m3 query pieces (MMA operand image)
  float* wprime;    // [max_batch, L, 64] fused_w * 2^-e per head
  int32_t* qexp;    // [max_batch, L, 64] the exponent e of each head's scaling
  int* d_err;       // device error word
  // tensor-core query path (three-pass TF32): the activations are stored
  // split as hi = tf32(x), lo = x - hi; the weights are split in the GEMM
  int tc_ok;        // the weight tensor maps could be encoded
  float* x_hi; float* x_lo;            // [max_batch, HID] hidden, split
  float* r_hi; float* r_lo;            // [max_batch, L, R] RMSNorm output, split
  float* up_part;                      // [2, max_batch, L*H*D] K-split partial sums of wq_b . r
  alignas(64) unsigned char wmaps[2][128];  // TMA tensor maps (fp32): w_down, w_up
  // test hook (fm_debug_stall_next_score): the next scoring launch withholds
  // its query operand and bounds its waits by debug_wait_ns
  int debug_stall;
  uint64_t debug_wait_ns;
};

namespace fm {

// Device allocations of fm_create and fm_level2_create go through these two,
// so that a test can make the n-th one fail (fm_debug_fail_alloc) and count
// the allocations still held (fm_debug_live_allocations).
cudaError_t dev_alloc(void** p, size_t bytes);
void dev_free(void* p);

// Bound of every wait inside a kernel when no test hook shortens it.
constexpr uint64_t kWaitLimitNs = 2000000000ull;

// launch helpers (fm_api.cu)
void note_launch();
fm_status check_launch();
// Records `e` for fm_last_cuda_error and returns FM_ERR_CUDA.
fm_status record_cuda_error(cudaError_t e);

// A set-up step to run once per device (a kernel's dynamic shared-memory
// limit): run(device, fn) calls fn() until it has returned FM_OK on that
// device and skips it afterwards.  Several host threads may call run() at
// once; two of them may both run fn() the first time, so fn() must be
// idempotent.  Devices past 63 run fn() on every call.
class PerDeviceOnce {
 public:
  template <typename F>
  fm_status run(int device, F&& fn) {
    const bool tracked = device >= 0 && device < 64;
    const uint64_t bit = tracked ? (uint64_t)1 << device : 0;
    if (tracked && (done_.load(std::memory_order_acquire) & bit)) return FM_OK;
    const fm_status s = fn();
    if (s == FM_OK && tracked) done_.fetch_or(bit, std::memory_order_acq_rel);
    return s;
  }

 private:
  std::atomic<uint64_t> done_{0};
};

// Raises `kernel`'s dynamic shared-memory limit to `bytes` once per device.
template <typename K>
fm_status smem_limit_once(PerDeviceOnce& once, int device, K* kernel, int bytes) {
  return once.run(device, [&]() -> fm_status {
    const cudaError_t e =
        cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    return e == cudaSuccess ? FM_OK : record_cuda_error(e);
  });
}

// kernels' host entry points
fm_status launch_query_prep(fm_ctx* ctx, const float* hidden, const int64_t* positions, int B,
                            float* q, float* fused_w, cudaStream_t stream);
fm_status launch_qpack(fm_ctx* ctx, const float* q, const float* fused_w, int B,
                       cudaStream_t stream);
// Encodes the weights' tensor maps for the tensor-core query path (fm_create);
// leaves tc_ok = 0 when they cannot be encoded.
fm_status prepare_tc_weights(fm_ctx* ctx);

struct ScoreArgs {
  const uint8_t* comp_k[kMaxLayers];
  int64_t row_stride;      // bytes between rows of one layer
  const int32_t* n_valid;  // [B] or null
  int B, N, L;
  const uint8_t* qpack;    // [B, L, P*64*128]
  const float* wprime;     // [B, L, 64]
  float* scores;           // [L, B, N] or null
  float* ens;              // [B, N] or null
  uint8_t* keep_thr;       // [B, N] or null
  float thr;
  int mode;                // FM_ENSEMBLE_*
  int* err;
  uint64_t wait_ns = kWaitLimitNs;  // bound of every wait (shortened only by the test hook)
  int withhold_query = 0;  // test hook: the query operand is never loaded, so its wait runs out
  // diagnostic dump of one tile's raw accumulators
  float* dbg_out;          // [128, 192] or null
  int dbg_layer, dbg_b, dbg_t;
};
fm_status launch_score(fm_ctx* ctx, const ScoreArgs& a, cudaStream_t stream);

fm_status launch_ensemble(const float* scores, int L, int B, int N, int mode, float* ens,
                          cudaStream_t stream);
fm_status launch_threshold(const float* ens, const int32_t* n_valid, int B, int N, float thr,
                           uint8_t* keep, cudaStream_t stream);
size_t topk_workspace_bytes(int B, int N);
// With the candidate fast path's buffers (launch_topk takes that path when
// the workspace is this large).
size_t topk_workspace_bytes_fast(int B, int N);
fm_status launch_topk(const float* ens, const int32_t* n_valid, int B, int N, int k, uint8_t* keep,
                      void* ws, size_t ws_bytes, cudaStream_t stream);
// The one-kernel form for rows of up to 16 * 16384 chunks (a thread-block
// cluster per row, no workspace): its cluster size for N, 0 past that bound;
// whether fm_select_topk takes it for N.
int topk_cluster_size(int N);
bool topk_use_cluster(int N);
fm_status launch_topk_cluster(const float* ens, const int32_t* n_valid, int B, int N, int k, uint8_t* keep,
                              cudaStream_t stream);
size_t compact_workspace_bytes(int B, int N);
fm_status launch_compact(const uint8_t* keep, int B, int N, int max_sel, int32_t* idx, int32_t* count,
                         void* ws, cudaStream_t stream);
// src and dst: addresses a kernel can dereference (device memory, or the
// device address of pinned host memory); src_on_device: src is device memory.
fm_status launch_gather(const void* src, bool src_on_device, int64_t src_row_stride_bytes, int n_src,
                        int64_t rec_bytes, const int32_t* idx, const int32_t* count, int B, int max_sel,
                        void* dst, int64_t dst_row_stride_bytes, cudaStream_t stream);
fm_status launch_topk_shard_begin(const int32_t* n_valid, int B, int N, int k, int32_t* hist, void* ws,
                                  size_t ws_bytes, cudaStream_t stream);
fm_status launch_topk_shard_hist(const float* ens, int B, int N, int pass, int32_t* hist, void* ws,
                                 size_t ws_bytes, cudaStream_t stream);
fm_status launch_topk_shard_pick(int B, int N, int pass, int32_t* hist, void* ws, size_t ws_bytes,
                                 cudaStream_t stream);
fm_status launch_topk_shard_ties(const float* ens, int B, int N, int32_t* eq_local, void* ws,
                                 size_t ws_bytes, cudaStream_t stream);
fm_status launch_topk_shard_mask(const float* ens, int B, int N, const int32_t* eq_all, int shard,
                                 uint8_t* keep, void* ws, size_t ws_bytes, cudaStream_t stream);

// ------------------------------------------------------------ PTX wrappers
// Reads and clears the error word of the decode attention's segment kernel
// on the current device (kDevErrNone when no wait ran out).
int take_attention_error();
// The same for the recall kernels' bulk-copy waits (compaction and gather).
int take_recall_error();

#if defined(__CUDACC__)

// Launches `kernel` so that it may start while the kernel ahead of it in
// `stream` is still running (programmatic dependent launch): the kernel must
// pass grid_dependency_wait() before it touches memory that kernel writes.
// Inside a stream capture the launch is a plain one.
template <typename... KArgs, typename... Args>
cudaError_t launch_overlapped(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                              cudaStream_t stream, Args... args) {
  cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(stream, &cap) != cudaSuccess) return cudaGetLastError();
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = cap == cudaStreamCaptureStatusNone ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kernel, args...);
}

// Waits until the kernels this one was launched after (launch_overlapped)
// have finished and their writes are visible; returns at once otherwise.
__device__ __forceinline__ void grid_dependency_wait() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
}

// Lets a kernel launched after this one with launch_overlapped start now.
__device__ __forceinline__ void grid_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t global_timer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count)
               : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Waits until the phase with the given parity of `bar` has completed.  Gives
// up after `limit_ns` of wall time or as soon as *abort becomes non-zero; on
// a timeout it records kDevErrTimeout in *err and sets *abort.  Returns true
// when the phase completed.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity,
                                                  volatile int* abort, int* err,
                                                  uint64_t limit_ns = 2000000000ull) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  for (uint32_t i = 1;; ++i) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((i & 63u) == 0) {
      if (*abort) return false;
      if (global_timer_ns() - t0 > limit_ns) {
        atomicExch(err, kDevErrTimeout);
        *abort = 1;
        return false;
      }
    }
  }
}

// Waits for a phase that an asynchronous operation this CTA issued will
// complete (a bulk copy landing, an MMA commit arriving) before the CTA may
// exit.  Ignores the abort flag -- the operation is in flight whatever else
// failed -- and gives up only after `limit_ns`, recording kDevErrTimeout.
__device__ __forceinline__ bool mbar_drain(uint64_t* bar, uint32_t parity, int* err,
                                           uint64_t limit_ns = 200000000ull) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  for (uint32_t i = 1;; ++i) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((i & 63u) == 0 && global_timer_ns() - t0 > limit_ns) {
      atomicExch(err, kDevErrTimeout);
      return false;
    }
  }
}

// 1-D bulk copy global -> shared through the TMA engine, completing on `bar`
// (transaction bytes).  dst, src and bytes must be multiples of 16.
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes,
                                         uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
          "r"(smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}




// Makes this thread's generic-proxy shared-memory writes visible to the async
// proxy (tensor-core operand reads).
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}


// ---------------------------------------------------------------- tcgen05
__device__ __forceinline__ void tmem_alloc(uint32_t* dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                   smem_u32(dst_smem)),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// D[tmem] (+)= A[smem desc] * B[smem desc]^T, fp8 (kind::f8f6f4) inputs, fp32 accumulate.
__device__ __forceinline__ void umma_f8f6f4(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                            uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// D[tmem] (+)= A[tmem] * B[smem desc]^T, fp8 (kind::f8f6f4) inputs, fp32
// accumulate.  A (M = 128 rows, K = 32 bytes) sits in TMEM: row r in lane r,
// its 32 bytes in 8 consecutive 32-bit columns starting at a_tmem.
__device__ __forceinline__ void umma_f8f6f4_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                               uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}


// As tmem_st32_wait, plus one more 32-bit column per lane at taddr1 (the same
// wait covers both stores).
__device__ __forceinline__ void tmem_st32_st1_wait(uint32_t taddr, const uint32_t* v, uint32_t taddr1,
                                                   uint32_t v1) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x1.b32 [%33], {%34};\n\t"
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, "
      "%17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};\n\t"
      "tcgen05.wait::st.sync.aligned;" ::"r"(taddr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]),
      "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]),
      "r"(v[15]), "r"(v[16]), "r"(v[17]), "r"(v[18]), "r"(v[19]), "r"(v[20]), "r"(v[21]),
      "r"(v[22]), "r"(v[23]), "r"(v[24]), "r"(v[25]), "r"(v[26]), "r"(v[27]), "r"(v[28]),
      "r"(v[29]), "r"(v[30]), "r"(v[31]), "r"(taddr1), "r"(v1)
      : "memory");
}


// Tiled TMA loads (no multicast) of a box at the given element coordinates,
// completing on `bar`.  The innermost coordinate times the element size is a
// multiple of 16 bytes at every call site.
__device__ __forceinline__ void tma_load_2d(void* dst, const void* tmap, int x, int y, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], "
      "[%4];" ::"r"(smem_u32(dst)),
      "l"(tmap), "r"(x), "r"(y), "r"(smem_u32(bar))
      : "memory");
}
__device__ __forceinline__ void tma_load_3d(void* dst, const void* tmap, int x, int y, int z, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, "
      "%4}], [%5];" ::"r"(smem_u32(dst)),
      "l"(tmap), "r"(x), "r"(y), "r"(z), "r"(smem_u32(bar))
      : "memory");
}

// Arrives on `bar` once every tcgen05.mma this thread issued before has completed.
__device__ __forceinline__ void umma_commit(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
          smem_u32(bar))
      : "memory");
}

// tcgen05.ld writes its destination registers asynchronously: they hold the
// data only after tcgen05.wait::ld.  The loads and the wait are therefore
// issued in ONE asm statement, so the compiler never sees the registers as
// defined (and never copies or reuses them) before the data has landed.
#define FM_TMEM_REGS32(p)                                                                   \
  "=r"(p[0]), "=r"(p[1]), "=r"(p[2]), "=r"(p[3]), "=r"(p[4]), "=r"(p[5]), "=r"(p[6]),     \
      "=r"(p[7]), "=r"(p[8]), "=r"(p[9]), "=r"(p[10]), "=r"(p[11]), "=r"(p[12]),          \
      "=r"(p[13]), "=r"(p[14]), "=r"(p[15]), "=r"(p[16]), "=r"(p[17]), "=r"(p[18]),       \
      "=r"(p[19]), "=r"(p[20]), "=r"(p[21]), "=r"(p[22]), "=r"(p[23]), "=r"(p[24]),       \
      "=r"(p[25]), "=r"(p[26]), "=r"(p[27]), "=r"(p[28]), "=r"(p[29]), "=r"(p[30]),       \
      "=r"(p[31])

// 32 lanes x 32 consecutive fp32 columns at taddr (thread i gets lane base+i), waited.
__device__ __forceinline__ void tmem_ld32_wait(uint32_t taddr, uint32_t* a) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
      "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : FM_TMEM_REGS32(a)
      : "r"(taddr)
      : "memory");
}

// Two 32-column loads (taddr0, taddr1) and one wait.
__device__ __forceinline__ void tmem_ld32x2_wait(uint32_t t0, uint32_t t1, uint32_t* a,
                                                 uint32_t* b) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
      "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%64];\n\t"
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%32, %33, %34, %35, %36, %37, %38, %39, %40, %41, %42, %43, %44, %45, %46, %47, "
      "%48, %49, %50, %51, %52, %53, %54, %55, %56, %57, %58, %59, %60, %61, %62, %63}, [%65];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : FM_TMEM_REGS32(a), FM_TMEM_REGS32(b)
      : "r"(t0), "r"(t1)
      : "memory");
}


// One 32-column load plus one single column (ts, result in *s), one wait.
__device__ __forceinline__ void tmem_ld32_x1_wait(uint32_t t0, uint32_t ts, uint32_t* a, uint32_t* s) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x1.b32 {%32}, [%34];\n\t"
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
      "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%33];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : FM_TMEM_REGS32(a), "=r"(*s)
      : "r"(t0), "r"(ts)
      : "memory");
}

// Three 32-column loads and one wait.
// Two 32-column loads plus one single column (ts, result in *s), one wait.
__device__ __forceinline__ void tmem_ld32x2_x1_wait(uint32_t t0, uint32_t t1, uint32_t ts, uint32_t* a,
                                                    uint32_t* b, uint32_t* s) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x1.b32 {%64}, [%67];\n\t"
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
      "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%65];\n\t"
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%32, %33, %34, %35, %36, %37, %38, %39, %40, %41, %42, %43, %44, %45, %46, %47, "
      "%48, %49, %50, %51, %52, %53, %54, %55, %56, %57, %58, %59, %60, %61, %62, %63}, [%66];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : FM_TMEM_REGS32(a), FM_TMEM_REGS32(b), "=r"(*s)
      : "r"(t0), "r"(t1), "r"(ts)
      : "memory");
}
// Three 32-column loads plus one single column (ts, result in *s), one wait.
__device__ __forceinline__ void tmem_ld32x3_x1_wait(uint32_t t0, uint32_t t1, uint32_t t2, uint32_t ts,
                                                    uint32_t* a, uint32_t* b, uint32_t* c, uint32_t* s) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x1.b32 {%96}, [%100];\n\t"
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
      "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%97];\n\t"
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%32, %33, %34, %35, %36, %37, %38, %39, %40, %41, %42, %43, %44, %45, %46, %47, "
      "%48, %49, %50, %51, %52, %53, %54, %55, %56, %57, %58, %59, %60, %61, %62, %63}, [%98];\n\t"
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%64, %65, %66, %67, %68, %69, %70, %71, %72, %73, %74, %75, %76, %77, %78, %79, "
      "%80, %81, %82, %83, %84, %85, %86, %87, %88, %89, %90, %91, %92, %93, %94, %95}, [%99];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : FM_TMEM_REGS32(a), FM_TMEM_REGS32(b), FM_TMEM_REGS32(c), "=r"(*s)
      : "r"(t0), "r"(t1), "r"(t2), "r"(ts)
      : "memory");
}
__device__ __forceinline__ void tmem_ld32x3_wait(uint32_t t0, uint32_t t1, uint32_t t2,
                                                 uint32_t* a, uint32_t* b, uint32_t* c) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
      "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%96];\n\t"
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%32, %33, %34, %35, %36, %37, %38, %39, %40, %41, %42, %43, %44, %45, %46, %47, "
      "%48, %49, %50, %51, %52, %53, %54, %55, %56, %57, %58, %59, %60, %61, %62, %63}, [%97];\n\t"
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%64, %65, %66, %67, %68, %69, %70, %71, %72, %73, %74, %75, %76, %77, %78, %79, "
      "%80, %81, %82, %83, %84, %85, %86, %87, %88, %89, %90, %91, %92, %93, %94, %95}, [%98];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : FM_TMEM_REGS32(a), FM_TMEM_REGS32(b), FM_TMEM_REGS32(c)
      : "r"(t0), "r"(t1), "r"(t2)
      : "memory");
}

// max(a, b) that is NaN when either operand is NaN (fmaxf returns the other
// operand instead).  relu(x) = fmax_nan(x, 0) and the max ensemble use it, so
// a NaN key element or scale carries through to the chunk's score, as it does
// through the README's torch operations.
__device__ __forceinline__ float fmax_nan(float a, float b) {
  float r;
  asm("max.NaN.f32 %0, %1, %2;" : "=f"(r) : "f"(a), "f"(b));
  return r;
}

// Packed fp32x2 arithmetic (sm_100): one instruction for two lanes of data.
__device__ __forceinline__ uint64_t f2_pack(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ void f2_unpack(uint64_t v, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t f2_fma(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t r;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
  return r;
}

// Shared-memory matrix descriptor for a K-major operand stored in the
// canonical 128-byte-swizzled layout: rows of 128 bytes, groups of 8 rows
// 1024 bytes apart, the 16-byte chunk c of row r stored at chunk c ^ (r % 8).
// `addr` is the shared address of the first element used (1024-aligned tile
// base plus a k offset of a multiple of 32 bytes inside the row).
__device__ __forceinline__ uint64_t sdesc_kmajor_sw128(uint32_t addr) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((addr & 0x3FFFFu) >> 4);  // start address, 16-byte units
  d |= static_cast<uint64_t>(1) << 16;                 // leading byte offset (unused here)
  d |= static_cast<uint64_t>(1024 >> 4) << 32;         // stride byte offset: 8-row groups
  d |= static_cast<uint64_t>(1) << 46;                 // descriptor version (sm_100)
  d |= static_cast<uint64_t>(2) << 61;                 // layout: 128-byte swizzle
  return d;
}

// Instruction descriptor: kind::f8f6f4, A = B = E4M3, D = F32, both K-major.
__host__ __device__ constexpr uint32_t idesc_e4m3_f32(int M, int N) {
  return (1u << 4)                                    // D format F32
         | (0u << 7) | (0u << 10)                     // A, B format E4M3
         | (0u << 15) | (0u << 16)                    // A, B K-major
         | (static_cast<uint32_t>(N >> 3) << 17)      // N / 8
         | (static_cast<uint32_t>(M >> 4) << 24);     // M / 16
}

// Byte offset of element (row, k) inside a K-major 128B-swizzled tile of
// 128-byte rows (one fp8 element per byte).
__host__ __device__ __forceinline__ uint32_t sw128_offset(uint32_t row, uint32_t kbyte) {
  return (row >> 3) * 1024u + (row & 7u) * 128u + ((((kbyte >> 4) ^ (row & 7u)) & 7u) << 4) +
         (kbyte & 15u);
}

#endif  // __CUDACC__

}  // namespace fm
