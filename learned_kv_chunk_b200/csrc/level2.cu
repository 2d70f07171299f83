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
//   -> slot -> chunk id through the resident set's index list.
//
// fm_level2_create runs the step once eagerly (which also sets the kernels'
// shared-memory attributes) and then records the same launches on a private
// stream into a graph; fm_level2_launch replays it.  The graph holds the
// pointers of the descriptor, so the caller rewrites the inputs in place
// between launches.
#include <new>

#include "fm_internal.cuh"

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
  e = launch_score(c, a, st);
  if (e != FM_OK) return e;
  e = launch_topk(s->ens, d.resident_count, d.B, d.R, d.k, s->keep, s->topk_ws, s->topk_ws_bytes, st);
  if (e != FM_OK) return e;
  e = launch_compact(s->keep, d.B, d.R, d.k, s->slots, s->slot_count, s->compact_ws, st);
  if (e != FM_OK) return e;
  if (cudaMemsetAsync(d.out_ids, 0xff, sizeof(int32_t) * (size_t)d.B * d.k, st) != cudaSuccess)
    return check_launch();
  e = launch_gather(d.resident_ids, (int64_t)d.R * 4, d.R, 4, s->slots, s->slot_count, d.B, d.k, d.out_ids,
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
  for (void* p : ptrs)
    if (p) cudaFree(p);
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
    if (cudaMalloc(a.p, a.bytes) != cudaSuccess) {
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
