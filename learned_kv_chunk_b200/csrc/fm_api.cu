// fm_api.cu -- the C ABI of libfm: argument checks, context lifetime, and the
// launches behind each call (see include/fm.h for the contract of each call).
#include <atomic>
#include <cmath>
#include <cstdlib>
#include <cstring>
#include <vector>

#include "fm_internal.cuh"

namespace fm {
namespace {

thread_local int g_last_cuda_error = 0;
std::atomic<uint64_t> g_launches{0};
std::atomic<int64_t> g_fail_alloc_in{0};  // > 0: allocations until the one that is made to fail
std::atomic<int64_t> g_live_allocs{0};

fm_status cuda_fail(cudaError_t e) {
  g_last_cuda_error = (int)e;
  return FM_ERR_CUDA;
}

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// YaRN rotary frequencies f_j (fp64), README "Architecture": RoPE (YaRN, last
// ROPE_DIM = 64 dims, base 160000).  Frequencies between the two correction
// dims of beta_fast / beta_slow are interpolated linearly between base^(-2j/d)
// and base^(-2j/d) / factor.
void yarn_frequencies(const fm_config& c, std::vector<double>& f) {
  const int half = c.rope_dim / 2;
  const double pi = 3.14159265358979323846;
  auto corr_dim = [&](double n_rot) {
    return c.rope_dim * std::log(c.rope_orig_max_pos / (n_rot * 2.0 * pi)) /
           (2.0 * std::log(c.rope_base));
  };
  double low = std::floor(corr_dim(c.rope_beta_fast));
  double high = std::ceil(corr_dim(c.rope_beta_slow));
  if (low < 0) low = 0;
  if (high > c.rope_dim - 1) high = c.rope_dim - 1;
  const double span = (high == low) ? 0.001 : (high - low);
  f.resize(half);
  for (int j = 0; j < half; ++j) {
    const double inv = std::pow(c.rope_base, -2.0 * j / c.rope_dim);
    double ramp = (j - low) / span;
    ramp = ramp < 0 ? 0 : (ramp > 1 ? 1 : ramp);
    f[j] = inv * (1.0 - ramp) + (inv / c.rope_factor) * ramp;
  }
}

fm_status check_config(const fm_config* c) {
  if (!c) return FM_ERR_INVALID_ARG;
  if (c->hidden <= 0 || c->q_lora_rank <= 0 || c->n_layers < 1 || c->max_batch < 1)
    return FM_ERR_INVALID_ARG;
  if (c->n_layers > kMaxLayers || c->max_batch > kMaxBatch) return FM_ERR_UNSUPPORTED;
  if (c->hidden % 128 || c->q_lora_rank % 128) return FM_ERR_UNSUPPORTED;
  if (c->n_heads != kHeads || c->head_dim != kHeadDim || c->rope_dim != kRopeDim)
    return FM_ERR_UNSUPPORTED;
  if (c->q_pieces != 2 && c->q_pieces != 3) return FM_ERR_INVALID_ARG;
  if (c->cta_pairs != 0 && c->cta_pairs != 1) return FM_ERR_INVALID_ARG;
  if (!(c->rope_base > 1.0) || !(c->rope_factor >= 1.0) || !(c->rope_orig_max_pos > 0) ||
      !(c->rope_beta_fast > 0) || !(c->rope_beta_slow > 0) || !(c->rms_eps >= 0.f))
    return FM_ERR_INVALID_ARG;
  return FM_OK;
}

fm_status check_keys(const fm_ctx* ctx, const uint8_t* const* comp_k, int64_t row_stride,
                     int B, int N) {
  if (!comp_k || B < 1 || N < 1 || B > ctx->cfg.max_batch) return FM_ERR_INVALID_ARG;
  for (int l = 0; l < ctx->cfg.n_layers; ++l) {
    if (!comp_k[l]) return FM_ERR_INVALID_ARG;
    if (!aligned(comp_k[l], 16)) return FM_ERR_ALIGNMENT;
  }
  const int64_t need = (((int64_t)N + 3) / 4) * 4 * kRecord;
  if (row_stride % 16 != 0) return FM_ERR_ALIGNMENT;
  if (row_stride < need) return FM_ERR_INVALID_ARG;
  return FM_OK;
}

}  // namespace

cudaError_t dev_alloc(void** p, size_t bytes) {
  *p = nullptr;
  int64_t n = g_fail_alloc_in.load();
  while (n > 0 && !g_fail_alloc_in.compare_exchange_weak(n, n - 1)) {
  }
  if (n == 1) return cudaErrorMemoryAllocation;  // this is the allocation the test asked to fail
  const cudaError_t e = cudaMalloc(p, bytes);
  if (e == cudaSuccess) g_live_allocs.fetch_add(1);
  return e;
}

void dev_free(void* p) {
  if (p && cudaFree(p) == cudaSuccess) g_live_allocs.fetch_sub(1);
}

void note_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }

fm_status check_launch() {
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? FM_OK : cuda_fail(e);
}

fm_status record_cuda_error(cudaError_t e) {
  cudaGetLastError();  // clear the sticky copy of a non-fatal error
  return cuda_fail(e);
}

}  // namespace fm

using namespace fm;

extern "C" {

void fm_config_default(fm_config* c) {
  if (!c) return;
  std::memset(c, 0, sizeof(*c));
  c->hidden = 4096;
  c->q_lora_rank = 1024;
  c->n_heads = 64;
  c->head_dim = 128;
  c->n_layers = 3;
  c->rope_dim = 64;
  c->rope_base = 160000.0;
  c->rope_factor = 16.0;
  c->rope_orig_max_pos = 65536.0;
  c->rope_beta_fast = 32.0;
  c->rope_beta_slow = 1.0;
  c->rms_eps = 1e-6f;
  c->max_batch = 64;
  c->q_pieces = 2;
  c->cta_pairs = 0;
}

fm_status fm_create(const fm_config* cfg, const fm_layer_weights* w, int device, fm_ctx** out) {
  if (!out) return FM_ERR_INVALID_ARG;
  *out = nullptr;
  fm_status s = check_config(cfg);
  if (s != FM_OK) return s;
  if (!w) return FM_ERR_INVALID_ARG;
  for (int l = 0; l < cfg->n_layers; ++l)
    if (!w[l].wq_a || !w[l].q_norm || !w[l].wq_b || !w[l].weights_proj) return FM_ERR_INVALID_ARG;
  int ndev = 0;
  cudaError_t e = cudaGetDeviceCount(&ndev);
  if (e != cudaSuccess) return cuda_fail(e);
  if (device < 0 || device >= ndev) return FM_ERR_INVALID_ARG;
  int prev = 0;
  cudaGetDevice(&prev);
  if ((e = cudaSetDevice(device)) != cudaSuccess) return cuda_fail(e);

  fm_ctx* c = new fm_ctx();
  std::memset(c, 0, sizeof(*c));
  c->cfg = *cfg;
  c->device = device;
  cudaDeviceGetAttribute(&c->num_sms, cudaDevAttrMultiProcessorCount, device);
  const int L = cfg->n_layers, R = cfg->q_lora_rank, HID = cfg->hidden, H = kHeads, D = kHeadDim;
  const int Bm = cfg->max_batch;
  c->splitk_max = 16;
  const size_t M = (size_t)L * (R + H);
  struct Alloc { void** p; size_t bytes; };
  Alloc allocs[] = {
      {(void**)&c->w_down, M * HID * sizeof(float)},
      {(void**)&c->q_norm, (size_t)L * R * sizeof(float)},
      {(void**)&c->w_up, (size_t)L * H * D * R * sizeof(float)},
      {(void**)&c->rope_freq, (size_t)(kRopeDim / 2) * sizeof(double)},
      {(void**)&c->a_part, (size_t)c->splitk_max * Bm * M * sizeof(float)},
      {(void**)&c->r_norm, (size_t)Bm * L * R * sizeof(float)},
      {(void**)&c->rope_cs, (size_t)Bm * (kRopeDim / 2) * 2 * sizeof(float)},
      {(void**)&c->qpack, (size_t)Bm * L * cfg->q_pieces * H * D},
      {(void**)&c->wprime, (size_t)Bm * L * H * sizeof(float)},
      {(void**)&c->qexp, (size_t)Bm * L * H * sizeof(int32_t)},
      {(void**)&c->d_err, sizeof(int)},
      {(void**)&c->x_hi, (size_t)Bm * HID * sizeof(float)},
      {(void**)&c->x_lo, (size_t)Bm * HID * sizeof(float)},
      {(void**)&c->r_hi, (size_t)Bm * L * R * sizeof(float)},
      {(void**)&c->r_lo, (size_t)Bm * L * R * sizeof(float)},
      {(void**)&c->up_part, (size_t)2 * Bm * L * H * D * sizeof(float)},
  };
  fm_status st = FM_OK;
  for (auto& a : allocs) {
    if (dev_alloc(a.p, a.bytes) != cudaSuccess) {
      cudaGetLastError();
      st = FM_ERR_OOM;
      break;
    }
  }
  if (st == FM_OK) {
    for (int l = 0; l < L && st == FM_OK; ++l) {
      float* dn = c->w_down + (size_t)l * (R + H) * HID;
      if ((e = cudaMemcpy(dn, w[l].wq_a, (size_t)R * HID * sizeof(float), cudaMemcpyDefault)) ||
          (e = cudaMemcpy(dn + (size_t)R * HID, w[l].weights_proj, (size_t)H * HID * sizeof(float),
                          cudaMemcpyDefault)) ||
          (e = cudaMemcpy(c->q_norm + (size_t)l * R, w[l].q_norm, (size_t)R * sizeof(float),
                          cudaMemcpyDefault)) ||
          (e = cudaMemcpy(c->w_up + (size_t)l * H * D * R, w[l].wq_b,
                          (size_t)H * D * R * sizeof(float), cudaMemcpyDefault)))
        st = cuda_fail(e);
    }
  }
  if (st == FM_OK) {
    std::vector<double> f;
    yarn_frequencies(*cfg, f);
    if ((e = cudaMemcpy(c->rope_freq, f.data(), f.size() * sizeof(double), cudaMemcpyHostToDevice)) ||
        (e = cudaMemset(c->d_err, 0, sizeof(int))) || (e = cudaDeviceSynchronize()))
      st = cuda_fail(e);
  }
  if (st == FM_OK) st = prepare_tc_weights(c);
  if (st == FM_OK && (e = cudaDeviceSynchronize())) st = cuda_fail(e);
  if (st != FM_OK) {
    fm_destroy(c);
    cudaSetDevice(prev);
    return st;
  }
  cudaSetDevice(prev);
  *out = c;
  return FM_OK;
}

fm_status fm_destroy(fm_ctx* c) {
  if (!c) return FM_ERR_INVALID_ARG;
  int prev = 0;
  cudaGetDevice(&prev);
  cudaSetDevice(c->device);
  cudaDeviceSynchronize();
  void* ptrs[] = {c->w_down, c->q_norm, c->w_up,   c->rope_freq, c->a_part, c->r_norm, c->rope_cs,
                  c->qpack,  c->wprime, c->qexp,   c->d_err,     c->x_hi,   c->x_lo,   c->r_hi,
                  c->r_lo,   c->up_part};
  for (void* p : ptrs) dev_free(p);
  cudaSetDevice(prev);
  delete c;
  return FM_OK;
}

fm_status fm_query_prep(fm_ctx* c, const float* hidden, const int64_t* positions, int B, float* q,
                        float* fused_w, cudaStream_t stream) {
  if (!c || !hidden || !positions || !q || !fused_w) return FM_ERR_INVALID_ARG;
  if (B < 1 || B > c->cfg.max_batch) return FM_ERR_INVALID_ARG;
  if (!aligned(hidden, 16) || !aligned(q, 16) || !aligned(fused_w, 4) || !aligned(positions, 8))
    return FM_ERR_ALIGNMENT;
  return launch_query_prep(c, hidden, positions, B, q, fused_w, stream);
}

static fm_status score_common(fm_ctx* c, const uint8_t* const* comp_k, int64_t row_stride,
                              const int32_t* n_valid, int B, int N, const float* q,
                              const float* fused_w, int mode, float thr, float* scores, float* ens,
                              uint8_t* keep_thr, cudaStream_t stream, float* dbg_out = nullptr,
                              int dbg_layer = -1, int dbg_b = -1, int dbg_t = -1) {
  if (!c || !q || !fused_w) return FM_ERR_INVALID_ARG;
  fm_status s = check_keys(c, comp_k, row_stride, B, N);
  if (s != FM_OK) return s;
  if (mode != FM_ENSEMBLE_MAX && mode != FM_ENSEMBLE_MEAN) return FM_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(fused_w, 4)) return FM_ERR_ALIGNMENT;
  if ((int64_t)B * N > ((int64_t)1 << 40)) return FM_ERR_INVALID_ARG;
  s = launch_qpack(c, q, fused_w, B, stream);
  if (s != FM_OK) return s;
  ScoreArgs a = {};
  for (int l = 0; l < c->cfg.n_layers; ++l) a.comp_k[l] = comp_k[l];
  a.row_stride = row_stride;
  a.n_valid = n_valid;
  a.B = B;
  a.N = N;
  a.L = c->cfg.n_layers;
  a.qpack = c->qpack;
  a.wprime = c->wprime;
  a.scores = scores;
  a.ens = ens;
  a.keep_thr = keep_thr;
  a.thr = thr;
  a.mode = mode;
  a.err = c->d_err;
  a.wait_ns = kWaitLimitNs;
  if (c->debug_stall) {  // one launch only
    a.wait_ns = c->debug_wait_ns;
    a.withhold_query = 1;
    c->debug_stall = 0;
  }
  a.dbg_out = dbg_out;
  a.dbg_layer = dbg_layer;
  a.dbg_b = dbg_b;
  a.dbg_t = dbg_t;
  return launch_score(c, a, stream);
}

fm_status fm_score(fm_ctx* c, const uint8_t* const* comp_k, int64_t row_stride,
                   const int32_t* n_valid, int B, int N, const float* q, const float* fused_w,
                   float* scores, cudaStream_t stream) {
  if (!scores) return FM_ERR_INVALID_ARG;
  return score_common(c, comp_k, row_stride, n_valid, B, N, q, fused_w, FM_ENSEMBLE_MAX, 0.f,
                      scores, nullptr, nullptr, stream);
}

fm_status fm_score_fused(fm_ctx* c, const uint8_t* const* comp_k, int64_t row_stride,
                         const int32_t* n_valid, int B, int N, const float* q,
                         const float* fused_w, int mode, float thr, float* scores, float* ens,
                         uint8_t* keep_thr, cudaStream_t stream) {
  if (!ens) return FM_ERR_INVALID_ARG;
  return score_common(c, comp_k, row_stride, n_valid, B, N, q, fused_w, mode, thr, scores, ens,
                      keep_thr, stream);
}

fm_status fm_ensemble(const float* scores, int L, int B, int N, int mode, float* ens,
                      cudaStream_t stream) {
  if (!scores || !ens || L < 1 || L > kMaxLayers || B < 1 || N < 1) return FM_ERR_INVALID_ARG;
  if (mode != FM_ENSEMBLE_MAX && mode != FM_ENSEMBLE_MEAN) return FM_ERR_INVALID_ARG;
  return launch_ensemble(scores, L, B, N, mode, ens, stream);
}

size_t fm_topk_workspace_bytes(int B, int N) {
  if (B < 1 || N < 1) return 0;
  return topk_workspace_bytes(B, N);
}

size_t fm_topk_workspace_bytes_fast(int B, int N) {
  if (B < 1 || N < 1) return 0;
  return topk_workspace_bytes_fast(B, N);
}

fm_status fm_select_topk(const float* ens, const int32_t* n_valid, int B, int N, int k,
                         uint8_t* keep, void* ws, size_t ws_bytes, cudaStream_t stream) {
  if (!ens || !keep || !ws || B < 1 || N < 1 || k < 1 || B > 65535) return FM_ERR_INVALID_ARG;
  if (!aligned(ws, 16) || !aligned(ens, 4)) return FM_ERR_ALIGNMENT;
  if (ws_bytes < topk_workspace_bytes(B, N)) return FM_ERR_INVALID_ARG;
  return launch_topk(ens, n_valid, B, N, k, keep, ws, ws_bytes, stream);
}

fm_status fm_select_threshold(const float* ens, const int32_t* n_valid, int B, int N, float thr,
                              uint8_t* keep, cudaStream_t stream) {
  if (!ens || !keep || B < 1 || N < 1 || B > 65535) return FM_ERR_INVALID_ARG;
  return launch_threshold(ens, n_valid, B, N, thr, keep, stream);
}

// Checks shared by the sharded top-K phases.
static fm_status shard_args(int B, int N, const void* hist, const void* ws, size_t ws_bytes) {
  if (!ws || B < 1 || N < 1 || B > 65535) return FM_ERR_INVALID_ARG;
  if (!aligned(ws, 16) || (hist && !aligned(hist, 16))) return FM_ERR_ALIGNMENT;
  if (ws_bytes < topk_workspace_bytes(B, N)) return FM_ERR_INVALID_ARG;
  return FM_OK;
}

fm_status fm_topk_shard_begin(const int32_t* n_valid_local, int B, int N, int k, int32_t* hist,
                              void* ws, size_t ws_bytes, cudaStream_t stream) {
  if (!hist || k < 1) return FM_ERR_INVALID_ARG;
  if (fm_status s = shard_args(B, N, hist, ws, ws_bytes)) return s;
  return launch_topk_shard_begin(n_valid_local, B, N, k, hist, ws, ws_bytes, stream);
}

fm_status fm_topk_shard_hist(const float* ens_local, int B, int N, int pass, int32_t* hist, void* ws,
                             size_t ws_bytes, cudaStream_t stream) {
  if (!ens_local || !hist || pass < 0 || pass > 2) return FM_ERR_INVALID_ARG;
  if (fm_status s = shard_args(B, N, hist, ws, ws_bytes)) return s;
  if (!aligned(ens_local, 4)) return FM_ERR_ALIGNMENT;
  return launch_topk_shard_hist(ens_local, B, N, pass, hist, ws, ws_bytes, stream);
}

fm_status fm_topk_shard_pick(int B, int N, int pass, int32_t* hist, void* ws, size_t ws_bytes,
                             cudaStream_t stream) {
  if (!hist || pass < 0 || pass > 2) return FM_ERR_INVALID_ARG;
  if (fm_status s = shard_args(B, N, hist, ws, ws_bytes)) return s;
  return launch_topk_shard_pick(B, N, pass, hist, ws, ws_bytes, stream);
}

fm_status fm_topk_shard_ties(const float* ens_local, int B, int N, int32_t* eq_local, void* ws,
                             size_t ws_bytes, cudaStream_t stream) {
  if (!ens_local || !eq_local) return FM_ERR_INVALID_ARG;
  if (fm_status s = shard_args(B, N, nullptr, ws, ws_bytes)) return s;
  if (!aligned(ens_local, 4) || !aligned(eq_local, 4)) return FM_ERR_ALIGNMENT;
  return launch_topk_shard_ties(ens_local, B, N, eq_local, ws, ws_bytes, stream);
}

fm_status fm_topk_shard_mask(const float* ens_local, int B, int N, const int32_t* eq_all, int shard,
                             uint8_t* keep_local, void* ws, size_t ws_bytes, cudaStream_t stream) {
  if (!ens_local || !eq_all || !keep_local || shard < 0) return FM_ERR_INVALID_ARG;
  if (fm_status s = shard_args(B, N, nullptr, ws, ws_bytes)) return s;
  if (!aligned(ens_local, 4) || !aligned(eq_all, 4)) return FM_ERR_ALIGNMENT;
  return launch_topk_shard_mask(ens_local, B, N, eq_all, shard, keep_local, ws, ws_bytes, stream);
}

fm_status fm_retrieve_host(fm_ctx* c, const fm_host_batch* in, const fm_device_staging* d,
                           cudaStream_t stream) {
  if (!c || !in || !d) return FM_ERR_INVALID_ARG;
  const int B = in->B, N = in->N, L = c->cfg.n_layers;
  if (B < 1 || B > c->cfg.max_batch || N < 1 || !in->hidden || !in->positions) return FM_ERR_INVALID_ARG;
  if (!in->keep_topk && !in->keep_thr) return FM_ERR_INVALID_ARG;
  if (in->keep_topk && (in->top_k < 1 || !d->keep_topk || !d->topk_ws)) return FM_ERR_INVALID_ARG;
  if (in->keep_thr && !d->keep_thr) return FM_ERR_INVALID_ARG;
  if (in->mode != FM_ENSEMBLE_MAX && in->mode != FM_ENSEMBLE_MEAN) return FM_ERR_INVALID_ARG;
  if (!d->hidden || !d->positions || !d->q || !d->fused_w || !d->ens || (in->n_valid && !d->n_valid))
    return FM_ERR_INVALID_ARG;
  for (int l = 0; l < L; ++l)
    if (!in->comp_k[l]) return FM_ERR_INVALID_ARG;
  if (fm_status s = check_keys(c, d->comp_k, in->row_stride_bytes, B, N)) return s;
  if (!aligned(d->hidden, 16) || !aligned(d->q, 16) || !aligned(d->positions, 8) || !aligned(d->fused_w, 4) ||
      !aligned(d->ens, 4) || (d->n_valid && !aligned(d->n_valid, 4)) || (d->topk_ws && !aligned(d->topk_ws, 16)))
    return FM_ERR_ALIGNMENT;
  if (in->keep_topk && d->topk_ws_bytes < topk_workspace_bytes(B, N)) return FM_ERR_INVALID_ARG;
  const size_t mask = (size_t)B * N;
  cudaError_t e = cudaSuccess;
  auto copy = [&](void* dst, const void* src, size_t bytes, cudaMemcpyKind kind) {
    if (e == cudaSuccess) e = cudaMemcpyAsync(dst, src, bytes, kind, stream);
  };
  copy(d->hidden, in->hidden, sizeof(float) * (size_t)B * c->cfg.hidden, cudaMemcpyHostToDevice);
  copy(d->positions, in->positions, sizeof(int64_t) * (size_t)B, cudaMemcpyHostToDevice);
  if (in->n_valid) copy(d->n_valid, in->n_valid, sizeof(int32_t) * (size_t)B, cudaMemcpyHostToDevice);
  for (int l = 0; l < L; ++l)
    copy(d->comp_k[l], in->comp_k[l], (size_t)B * (size_t)in->row_stride_bytes, cudaMemcpyHostToDevice);
  if (e != cudaSuccess) return record_cuda_error(e);
  const int32_t* nv = in->n_valid ? d->n_valid : nullptr;
  fm_status s = fm_query_prep(c, d->hidden, d->positions, B, d->q, d->fused_w, stream);
  if (s == FM_OK)
    s = fm_score_fused(c, d->comp_k, in->row_stride_bytes, nv, B, N, d->q, d->fused_w, in->mode, in->thr,
                       nullptr, d->ens, in->keep_thr ? d->keep_thr : nullptr, stream);
  if (s == FM_OK && in->keep_topk)
    s = fm_select_topk(d->ens, nv, B, N, in->top_k, d->keep_topk, d->topk_ws, d->topk_ws_bytes, stream);
  if (s != FM_OK) return s;
  if (in->keep_topk) copy(in->keep_topk, d->keep_topk, mask, cudaMemcpyDeviceToHost);
  if (in->keep_thr) copy(in->keep_thr, d->keep_thr, mask, cudaMemcpyDeviceToHost);
  return e == cudaSuccess ? FM_OK : record_cuda_error(e);
}

fm_status fm_sync_status(fm_ctx* c, cudaStream_t stream) {
  if (!c) return FM_ERR_INVALID_ARG;
  cudaError_t e = cudaStreamSynchronize(stream);
  if (e != cudaSuccess) return cuda_fail(e);
  int h = 0;
  if ((e = cudaMemcpy(&h, c->d_err, sizeof(int), cudaMemcpyDeviceToHost)) != cudaSuccess)
    return cuda_fail(e);
  if (h != kDevErrNone) {
    cudaMemset(c->d_err, 0, sizeof(int));
    return FM_ERR_DEVICE;
  }
  const bool attn = take_attention_error() != kDevErrNone;
  const bool recall = take_recall_error() != kDevErrNone;
  if (attn || recall) return FM_ERR_DEVICE;
  return FM_OK;
}

const char* fm_strerror(fm_status s) {
  switch (s) {
    case FM_OK: return "ok";
    case FM_ERR_INVALID_ARG: return "invalid argument";
    case FM_ERR_ALIGNMENT: return "pointer or stride breaks the alignment rule";
    case FM_ERR_UNSUPPORTED: return "unsupported shape or configuration";
    case FM_ERR_CUDA: return "CUDA runtime error";
    case FM_ERR_OOM: return "device allocation failed";
    case FM_ERR_DEVICE: return "a kernel recorded an error (bounded wait ran out)";
    default: return "unknown status";
  }
}

int fm_last_cuda_error(void) { return g_last_cuda_error; }

uint64_t fm_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

void fm_debug_fail_alloc(int n) { g_fail_alloc_in.store(n > 0 ? n : 0); }

int64_t fm_debug_live_allocations(void) { return g_live_allocs.load(); }

fm_status fm_debug_stall_next_score(fm_ctx* c, uint64_t wait_limit_ns) {
  if (!c || wait_limit_ns == 0 || wait_limit_ns > kWaitLimitNs) return FM_ERR_INVALID_ARG;
  c->debug_wait_ns = wait_limit_ns;
  c->debug_stall = 1;
  return FM_OK;
}

fm_status fm_debug_tile_dots(fm_ctx* c, const uint8_t* const* comp_k, int64_t row_stride, int B,
                             int N, const float* q, const float* fused_w, int layer, int b, int t,
                             float* out, int32_t* pow2_exp, cudaStream_t stream) {
  if (!c || !out || !pow2_exp) return FM_ERR_INVALID_ARG;
  if (layer < 0 || layer >= c->cfg.n_layers || b < 0 || b >= B || t < 0 ||
      (int64_t)t * kTile >= N)
    return FM_ERR_INVALID_ARG;
  fm_status s = score_common(c, comp_k, row_stride, nullptr, B, N, q, fused_w, FM_ENSEMBLE_MAX,
                             0.f, nullptr, nullptr, nullptr, stream, out, layer, b, t);
  if (s != FM_OK) return s;
  cudaError_t e = cudaMemcpyAsync(pow2_exp, c->qexp + ((size_t)b * c->cfg.n_layers + layer) * kHeads,
                                  kHeads * sizeof(int32_t), cudaMemcpyDeviceToDevice, stream);
  return e == cudaSuccess ? FM_OK : cuda_fail(e);
}

}  // extern "C"
