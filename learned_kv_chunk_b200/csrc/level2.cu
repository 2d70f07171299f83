// level2.cu -- the per-step selection over the resident set, as one CUDA graph.
//
// The model card's "How it works": Level 1 (the Memory Indexer, every 64
// decode steps) recalls a resident set; Level 2 runs at every decode step, a
// top-512 confined to the resident set, inside a CUDA graph.  DS-V4's own
// Level-2 indexer is not part of the pages; here the step runs this library's
// own stages on the resident chunks:
//
//   query prep (hidden, positions -> q, fused_w)
//   -> fused scoring of the R resident records of every layer + ensemble
//   -> top-k of the ensembled scores (k = 512 in the card)
//   -> compaction of the keep mask into resident slots
//   -> slot -> chunk id through the resident set's index list
// (the last three in one kernel, one CTA per row, for up to 8192 slots).
//
// fm_level2_create runs the step once eagerly (which also sets the kernels'
// shared-memory attributes) and then records the same launches on a private
// stream into a graph; fm_level2_launch replays it.  The graph holds the
// pointers of the descriptor, so the caller rewrites the inputs in place
// between launches.
#include <new>

#include "fm_internal.cuh"
#include "select_block.cuh"

struct fm_level2 {
  fm_ctx* ctx;
  fm_level2_desc d;
  float* q;            // [B, L, 64, 128]
  float* fused_w;      // [B, L, 64]
  float* ens;          // [B, R]
  uint8_t* keep;       // [B, R]
  int32_t* slots;      // [B, k]
  int32_t* slot_count; // [B]
  void* topk_ws;
  size_t topk_ws_bytes;
  void* compact_ws;
  cudaGraph_t graph;
  cudaGraphExec_t exec;
};

namespace fm {
namespace {

// ------------------------------------------------ small-row top-k -> chunk ids
// For resident sets of up to kSelMaxR slots the selection, the compaction and
// the slot -> chunk id mapping run in one CTA per row, entirely in shared
// memory: the row's order-preserving keys, three radix passes (11 + 11 + 10
// bits) that fix the k-th largest key T and how many keys equal to T are kept,
// then an ordered scan that writes the kept slots' chunk ids in slot order
// (equal keys taken in increasing slot).  The general top-K (grid-wide passes
// with a block per 8192 scores) pays six launches of one block per row here.
constexpr int kSelThreads = kBlkThreads;
constexpr int kSelMaxR = 8192;

__global__ void __launch_bounds__(kSelThreads) level2_select_kernel(const float* __restrict__ ens,
                                                                    const int32_t* __restrict__ resident_count,
                                                                    const int32_t* __restrict__ resident_ids,
                                                                    int R, int k, int32_t* __restrict__ out_ids,
                                                                    int32_t* __restrict__ out_count) {
  extern __shared__ uint32_t s_key[];  // [R]
  __shared__ uint32_t s_hist[2048];
  __shared__ int s_warp[kSelThreads / 32 + 1];
  __shared__ uint32_t s_pick[2];
  const BlockSelScratch sc{s_hist, s_warp, s_pick};
  const int b = blockIdx.x, t = threadIdx.x;
  const int nv = max(0, min(resident_count[b], R));
  const float* row = ens + (size_t)b * R;
  for (int i = t; i < nv; i += kSelThreads) s_key[i] = block_order_key(row[i]);
  const bool all = k >= nv;
  uint32_t T = 0u;
  int need = 0;  // keys equal to T to keep
  if (!all) {
    __syncthreads();
    block_kth_largest(s_key, nv, (uint32_t)k, sc, &T, &need);
  }
  __syncthreads();
  // ordered compaction: thread t scans the contiguous slots [lo, hi)
  const int span = (nv + kSelThreads - 1) / kSelThreads;
  const int lo = min(nv, t * span), hi = min(nv, lo + span);
  int eq = 0, gt = 0;
  if (!all)
    for (int i = lo; i < hi; ++i) {
      eq += s_key[i] == T ? 1 : 0;
      gt += s_key[i] > T ? 1 : 0;
    }
  int tot;
  const int eq_before = all ? 0 : block_exclusive_scan(eq, s_warp, &tot);
  const int keep_eq = all ? 0 : max(0, min(eq, need - eq_before));
  const int kept = all ? hi - lo : gt + keep_eq;
  int pos = block_exclusive_scan(kept, s_warp, &tot);
  int32_t* out = out_ids + (size_t)b * k;
  const int32_t* ids = resident_ids + (size_t)b * R;
  int eq_seen = 0;
  for (int i = lo; i < hi; ++i) {
    bool kp = all;
    if (!all) {
      const uint32_t key = s_key[i];
      kp = key > T || (key == T && eq_seen++ < keep_eq);
    }
    if (kp) out[pos++] = ids[i];
  }
  for (int j = tot + t; j < k; j += kSelThreads) out[j] = -1;
  if (t == 0 && out_count) out_count[b] = tot;
}

// The step's launches on `st`, in order.
fm_status record_step(fm_level2* s, cudaStream_t st) {
  const fm_level2_desc& d = s->d;
  fm_ctx* c = s->ctx;
  const int L = c->cfg.n_layers;
  fm_status e = launch_query_prep(c, d.hidden, d.positions, d.B, s->q, s->fused_w, st);
  if (e != FM_OK) return e;
  e = launch_qpack(c, s->q, s->fused_w, d.B, st);
  if (e != FM_OK) return e;
  ScoreArgs a = {};
  for (int l = 0; l < L; ++l) a.comp_k[l] = d.resident_keys[l];
  a.row_stride = (int64_t)d.R * kRecord;
  a.n_valid = d.resident_count;
  a.B = d.B;
  a.N = d.R;
  a.L = L;
  a.qpack = c->qpack;
  a.wprime = c->wprime;
  a.ens = s->ens;
  a.mode = d.mode;
  a.err = c->d_err;
  a.wait_ns = kWaitLimitNs;
  e = launch_score(c, a, st);
  if (e != FM_OK) return e;
  if (d.R <= kSelMaxR) {  // one CTA per row does selection, compaction and id mapping
    level2_select_kernel<<<d.B, kSelThreads, (size_t)d.R * sizeof(uint32_t), st>>>(
        s->ens, d.resident_count, d.resident_ids, d.R, d.k, d.out_ids, d.out_count);
    note_launch();
    return check_launch();
  }
  e = launch_topk(s->ens, d.resident_count, d.B, d.R, d.k, s->keep, s->topk_ws, s->topk_ws_bytes, st);
  if (e != FM_OK) return e;
  e = launch_compact(s->keep, d.B, d.R, d.k, s->slots, s->slot_count, s->compact_ws, st);
  if (e != FM_OK) return e;
  if (cudaMemsetAsync(d.out_ids, 0xff, sizeof(int32_t) * (size_t)d.B * d.k, st) != cudaSuccess)
    return check_launch();
  e = launch_gather(d.resident_ids, true, (int64_t)d.R * 4, d.R, 4, s->slots, s->slot_count, d.B, d.k, d.out_ids,
                    (int64_t)d.k * 4, st);
  if (e != FM_OK) return e;
  if (d.out_count &&
      cudaMemcpyAsync(d.out_count, s->slot_count, sizeof(int32_t) * (size_t)d.B, cudaMemcpyDeviceToDevice,
                      st) != cudaSuccess)
    return check_launch();
  return FM_OK;
}

void release(fm_level2* s) {
  if (s->exec) cudaGraphExecDestroy(s->exec);
  if (s->graph) cudaGraphDestroy(s->graph);
  void* ptrs[] = {s->q, s->fused_w, s->ens, s->keep, s->slots, s->slot_count, s->topk_ws, s->compact_ws};
  for (void* p : ptrs) dev_free(p);
  delete s;
}

}  // namespace
}  // namespace fm

using namespace fm;

extern "C" fm_status fm_level2_create(fm_ctx* ctx, const fm_level2_desc* d, cudaStream_t stream,
                                      fm_level2** out) {
  if (!out) return FM_ERR_INVALID_ARG;
  *out = nullptr;
  if (!ctx || !d || !d->hidden || !d->positions || !d->resident_ids || !d->resident_count || !d->out_ids)
    return FM_ERR_INVALID_ARG;
  const int L = ctx->cfg.n_layers;
  for (int l = 0; l < L; ++l)
    if (!d->resident_keys[l]) return FM_ERR_INVALID_ARG;
  if (d->B < 1 || d->B > ctx->cfg.max_batch || d->R < 1 || d->k < 1 || d->k > d->R)
    return FM_ERR_INVALID_ARG;
  if (d->mode != FM_ENSEMBLE_MAX && d->mode != FM_ENSEMBLE_MEAN) return FM_ERR_INVALID_ARG;
  if (d->R % 4 != 0) return FM_ERR_UNSUPPORTED;  // resident key rows on 16-byte boundaries
  for (int l = 0; l < L; ++l)
    if (reinterpret_cast<uintptr_t>(d->resident_keys[l]) & 15u) return FM_ERR_ALIGNMENT;
  if ((reinterpret_cast<uintptr_t>(d->hidden) & 15u) || (reinterpret_cast<uintptr_t>(d->positions) & 7u) ||
      (reinterpret_cast<uintptr_t>(d->resident_ids) & 3u) ||
      (reinterpret_cast<uintptr_t>(d->resident_count) & 3u) || (reinterpret_cast<uintptr_t>(d->out_ids) & 3u) ||
      (reinterpret_cast<uintptr_t>(d->out_count) & 3u))
    return FM_ERR_ALIGNMENT;

  fm_level2* s = new (std::nothrow) fm_level2();
  if (!s) return FM_ERR_OOM;
  s->ctx = ctx;
  s->d = *d;
  int prev = 0;
  cudaGetDevice(&prev);
  cudaSetDevice(ctx->device);
  const int B = d->B, R = d->R, k = d->k;
  s->topk_ws_bytes = topk_workspace_bytes(B, R);
  struct Alloc { void** p; size_t bytes; } allocs[] = {
      {(void**)&s->q, (size_t)B * L * kHeads * kHeadDim * sizeof(float)},
      {(void**)&s->fused_w, (size_t)B * L * kHeads * sizeof(float)},
      {(void**)&s->ens, (size_t)B * R * sizeof(float)},
      {(void**)&s->keep, (size_t)B * R},
      {(void**)&s->slots, (size_t)B * k * sizeof(int32_t)},
      {(void**)&s->slot_count, (size_t)B * sizeof(int32_t)},
      {&s->topk_ws, s->topk_ws_bytes},
      {&s->compact_ws, compact_workspace_bytes(B, R)},
  };
  for (auto& a : allocs) {
    if (dev_alloc(a.p, a.bytes) != cudaSuccess) {
      cudaGetLastError();
      release(s);
      cudaSetDevice(prev);
      return FM_ERR_OOM;
    }
  }
  // one eager step: sets the kernels' attributes, and checks every launch
  fm_status st = record_step(s, stream);
  cudaError_t e = cudaSuccess;
  if (st == FM_OK && (e = cudaStreamSynchronize(stream)) != cudaSuccess) st = FM_ERR_CUDA;
  cudaStream_t cap = nullptr;
  if (st == FM_OK && (e = cudaStreamCreateWithFlags(&cap, cudaStreamNonBlocking)) != cudaSuccess)
    st = FM_ERR_CUDA;
  if (st == FM_OK && (e = cudaStreamBeginCapture(cap, cudaStreamCaptureModeThreadLocal)) != cudaSuccess)
    st = FM_ERR_CUDA;
  if (st == FM_OK) {
    const fm_status rs = record_step(s, cap);
    e = cudaStreamEndCapture(cap, &s->graph);
    if (rs != FM_OK) st = rs;
    else if (e != cudaSuccess) st = FM_ERR_CUDA;
  }
  if (st == FM_OK && (e = cudaGraphInstantiate(&s->exec, s->graph, 0)) != cudaSuccess) st = FM_ERR_CUDA;
  if (cap) cudaStreamDestroy(cap);
  if (st != FM_OK) {
    if (st == FM_ERR_CUDA && e != cudaSuccess) record_cuda_error(e);
    release(s);
    cudaSetDevice(prev);
    return st;
  }
  cudaSetDevice(prev);
  *out = s;
  return FM_OK;
}

extern "C" fm_status fm_level2_launch(fm_level2* s, cudaStream_t stream) {
  if (!s || !s->exec) return FM_ERR_INVALID_ARG;
  const cudaError_t e = cudaGraphLaunch(s->exec, stream);
  return e == cudaSuccess ? FM_OK : record_cuda_error(e);
}

extern "C" fm_status fm_level2_copy_scores(const fm_level2* s, float* dst, cudaStream_t stream) {
  if (!s || !dst) return FM_ERR_INVALID_ARG;
  const cudaError_t e = cudaMemcpyAsync(dst, s->ens, sizeof(float) * (size_t)s->d.B * s->d.R,
                                        cudaMemcpyDeviceToDevice, stream);
  return e == cudaSuccess ? FM_OK : record_cuda_error(e);
}

extern "C" fm_status fm_level2_destroy(fm_level2* s) {
  if (!s) return FM_ERR_INVALID_ARG;
  int prev = 0;
  cudaGetDevice(&prev);
  cudaSetDevice(s->ctx->device);
  cudaDeviceSynchronize();
  release(s);
  cudaSetDevice(prev);
  return FM_OK;
}
