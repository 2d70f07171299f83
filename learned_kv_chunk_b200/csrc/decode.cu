// decode.cu -- the toy sparse decode step of the README's decode loop.
//
// README "Toy inference reference": at every decode step the toy decoder runs
// a sparse memory attention over the N compressed chunks, in which the chunks
// the last retrieval did not keep have their attention logits set to -inf
// (they contribute nothing, as if their KV had not been loaded); every 64
// steps the retriever scores all chunks again and refreshes the keep mask.
// The pages do not define the toy decoder; this file takes the plainest
// weight-free reading:
//
//   query      the step's hidden state [4096] as 32 heads of 128
//   memory     chunk i's vector x_i = e4m3(bytes[0:128]) * f32le(bytes[128:132])
//              (the compressed record is the only per-chunk data the toy has),
//              used as key and value
//   attention  o_h = sum_i p_hi x_i,  p_h = softmax_i(q_h . x_i / sqrt(128)),
//              over the kept chunks only (-inf elsewhere); no kept chunk: o = 0
//   update     hidden' = RMSNorm(hidden + o), eps 1e-6, no gain
//
// The attention reads only the kept chunks (the index list of the keep mask,
// fm_compact_mask), which is what -inf masking computes.  Each CTA takes one
// row and a segment of 128 kept chunks: it gathers and dequantizes their
// records into shared memory, computes the 32 x 128 logits, the segment's
// per-head max and exp-sum, and the unnormalised output; a second kernel
// merges the segments (the split-softmax identity).  fp32 on the CUDA cores.
#include <cuda_fp8.h>

#include <cmath>

#include "fm_internal.cuh"

namespace fm {
namespace {

constexpr int kAH = 32;        // attention heads (4096 / 128)
constexpr int kAD = 128;       // head dim = chunk vector dim
constexpr int kSeg = 128;      // kept chunks per CTA
constexpr int kAThreads = 256;
constexpr int kXStride = 132;  // shared row stride (floats): 16-byte rows, conflict-free strided reads
constexpr int kPStride = kAH + 1;

struct AttnSmem {
  float x[kSeg][kXStride];  // dequantized chunk vectors
  float q[kAH][kXStride];   // the row's query heads
  float p[kSeg][kPStride];  // logits, then exp(logit - max)
  float m[kAH], l[kAH];
  uint8_t valid[kSeg];      // slot c holds an index inside the memory
};

__device__ __forceinline__ void dequant4(uint32_t w, float s, float* out) {
  const __half2_raw lo = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)(w & 0xffffu), __NV_E4M3);
  const __half2_raw hi = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)(w >> 16), __NV_E4M3);
  const float2 a = __half22float2(*reinterpret_cast<const __half2*>(&lo));
  const float2 b = __half22float2(*reinterpret_cast<const __half2*>(&hi));
  out[0] = a.x * s;
  out[1] = a.y * s;
  out[2] = b.x * s;
  out[3] = b.y * s;
}

// Partial attention of (segment blockIdx.x, row blockIdx.y): per head the
// segment's max logit m, sum of exp(logit - m) l, and sum of exp(logit - m) x.
__global__ void __launch_bounds__(kAThreads) sparse_attn_partial_kernel(
    const float* __restrict__ q, const uint8_t* __restrict__ mem, int64_t row_stride, int n_mem,
    const int32_t* __restrict__ idx, const int32_t* __restrict__ count, int max_sel, int nseg,
    float* __restrict__ part_o, float* __restrict__ part_ml) {
  extern __shared__ uint8_t smem_raw[];
  AttnSmem& S = *reinterpret_cast<AttnSmem*>(smem_raw);
  const int b = blockIdx.y, seg = blockIdx.x;
  const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
  const int cnt = min(count[b], max_sel);
  const int c0 = seg * kSeg;
  const int nc = max(0, min(kSeg, cnt - c0));
  float* po = part_o + ((size_t)b * nseg + seg) * kAH * kAD;
  float* pml = part_ml + ((size_t)b * nseg + seg) * kAH * 2;
  if (nc == 0) {  // an empty segment: nothing to merge
    for (int i = t; i < kAH; i += kAThreads) {
      pml[2 * i] = -INFINITY;
      pml[2 * i + 1] = 0.f;
    }
    return;
  }
  // the row's query (32 x 128 fp32), 16-byte loads
  const float4* qr = reinterpret_cast<const float4*>(q + (size_t)b * kAH * kAD);
  for (int i = t; i < kAH * kAD / 4; i += kAThreads) {
    const int h = i / (kAD / 4), d4 = i % (kAD / 4);
    *reinterpret_cast<float4*>(&S.q[h][4 * d4]) = __ldg(qr + i);
  }
  // gather + dequantize: warp w takes records w + 8k (k < 16), lane l the 4
  // codes l of each; all 16 records' loads are issued before any is used
  const uint8_t* row = mem + (size_t)b * row_stride;
  const int32_t* ids = idx + (size_t)b * max_sel + c0;
  {
    constexpr int kPer = kSeg / (kAThreads / 32);
    int id[kPer];
#pragma unroll
    for (int k = 0; k < kPer; ++k) {
      const int c = warp + 8 * k;
      id[k] = c < nc ? __ldg(ids + c) : -1;
    }
    uint32_t w[kPer], sc[kPer];
#pragma unroll
    for (int k = 0; k < kPer; ++k) {
      w[k] = 0u;
      sc[k] = 0u;
      if (id[k] >= 0 && id[k] < n_mem) {  // an index outside the memory counts as masked
        const uint8_t* rec = row + (int64_t)id[k] * kRecord;
        w[k] = __ldg(reinterpret_cast<const uint32_t*>(rec + 4 * lane));
        sc[k] = __ldg(reinterpret_cast<const uint32_t*>(rec + 128));
      }
    }
#pragma unroll
    for (int k = 0; k < kPer; ++k) {
      const int c = warp + 8 * k;
      const bool ok = id[k] >= 0 && id[k] < n_mem;
      float v[4] = {0.f, 0.f, 0.f, 0.f};
      if (ok) dequant4(w[k], __uint_as_float(sc[k]), v);
      if (lane == 0) S.valid[c] = ok ? 1 : 0;
      *reinterpret_cast<float4*>(&S.x[c][4 * lane]) = make_float4(v[0], v[1], v[2], v[3]);
    }
  }
  __syncthreads();
  // logits: thread t -> heads hg + 8i, chunks cg + 32j (i, j < 4)
  {
    const int hg = t & 7, cg = t >> 3;
    float acc[4][4] = {};
#pragma unroll 4
    for (int d = 0; d < kAD; d += 4) {
      float4 qv[4], xv[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) qv[i] = *reinterpret_cast<const float4*>(&S.q[hg + 8 * i][d]);
#pragma unroll
      for (int j = 0; j < 4; ++j) xv[j] = *reinterpret_cast<const float4*>(&S.x[cg + 32 * j][d]);
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          acc[i][j] = fmaf(qv[i].x, xv[j].x, acc[i][j]);
          acc[i][j] = fmaf(qv[i].y, xv[j].y, acc[i][j]);
          acc[i][j] = fmaf(qv[i].z, xv[j].z, acc[i][j]);
          acc[i][j] = fmaf(qv[i].w, xv[j].w, acc[i][j]);
        }
    }
    const float scale = 0.088388347648318447f;  // 128^-1/2
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int c = cg + 32 * j;
        S.p[c][hg + 8 * i] = S.valid[c] ? acc[i][j] * scale : -INFINITY;
      }
  }
  __syncthreads();
  // per head: max and exp-sum over the segment (warp w: heads 4w .. 4w+3)
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const int h = 4 * warp + k;
    float mx = -INFINITY;
    for (int c = lane; c < kSeg; c += 32) mx = fmaxf(mx, S.p[c][h]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    float sum = 0.f;
    for (int c = lane; c < kSeg; c += 32) {
      const float e = (S.valid[c] && mx != -INFINITY) ? expf(S.p[c][h] - mx) : 0.f;
      S.p[c][h] = e;
      sum += e;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
    if (lane == 0) {
      S.m[h] = mx;
      S.l[h] = sum;
    }
  }
  __syncthreads();
  // unnormalised output: thread t -> heads hg + 8i, dims 4dg .. 4dg+3
  {
    const int hg = t & 7, dg = t >> 3;
    float4 acc[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) acc[i] = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 4
    for (int c = 0; c < nc; ++c) {
      const float4 xv = *reinterpret_cast<const float4*>(&S.x[c][4 * dg]);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float p = S.p[c][hg + 8 * i];
        acc[i].x = fmaf(p, xv.x, acc[i].x);
        acc[i].y = fmaf(p, xv.y, acc[i].y);
        acc[i].z = fmaf(p, xv.z, acc[i].z);
        acc[i].w = fmaf(p, xv.w, acc[i].w);
      }
    }
#pragma unroll
    for (int i = 0; i < 4; ++i)
      *reinterpret_cast<float4*>(po + (size_t)(hg + 8 * i) * kAD + 4 * dg) = acc[i];
  }
  for (int h = t; h < kAH; h += kAThreads) {
    pml[2 * h] = S.m[h];
    pml[2 * h + 1] = S.l[h];
  }
}

// Merges the segments of (head blockIdx.x, row blockIdx.y), thread d one
// output dim: o = sum_s e^(m_s - M) o_s / sum_s e^(m_s - M) l_s.
__global__ void __launch_bounds__(kAD) sparse_attn_combine_kernel(const float* __restrict__ part_o,
                                                                  const float* __restrict__ part_ml, int nseg,
                                                                  float* __restrict__ out) {
  const int h = blockIdx.x, b = blockIdx.y, d = threadIdx.x;
  const float* pml = part_ml + (size_t)b * nseg * kAH * 2;
  const float* po = part_o + (size_t)b * nseg * kAH * kAD;
  float M = -INFINITY;
  for (int s = 0; s < nseg; ++s) M = fmaxf(M, __ldg(pml + ((size_t)s * kAH + h) * 2));
  float num = 0.f, den = 0.f;
  if (M != -INFINITY) {
    for (int s = 0; s < nseg; ++s) {
      const float ms = __ldg(pml + ((size_t)s * kAH + h) * 2);
      if (ms == -INFINITY) continue;
      const float w = expf(ms - M);
      num = fmaf(w, __ldg(po + ((size_t)s * kAH + h) * kAD + d), num);
      den = fmaf(w, __ldg(pml + ((size_t)s * kAH + h) * 2 + 1), den);
    }
  }
  out[((size_t)b * kAH + h) * kAD + d] = den > 0.f ? num / den : 0.f;
}

// hidden'[b] = RMSNorm(hidden[b] + o[b]) (eps, no gain); one CTA per row.
__global__ void __launch_bounds__(kAThreads) toy_update_kernel(const float* __restrict__ hidden,
                                                               const float* __restrict__ o, int H, float eps,
                                                               float* __restrict__ out) {
  const int b = blockIdx.x;
  __shared__ float red[kAThreads / 32];
  float ss = 0.f;
  for (int i = threadIdx.x; i < H; i += kAThreads) {
    const float v = hidden[(size_t)b * H + i] + o[(size_t)b * H + i];
    ss = fmaf(v, v, ss);
  }
#pragma unroll
  for (int k = 16; k > 0; k >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, k);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = ss;
  __syncthreads();
  float tot = 0.f;
#pragma unroll
  for (int i = 0; i < kAThreads / 32; ++i) tot += red[i];
  const float r = rsqrtf(tot / (float)H + eps);
  for (int i = threadIdx.x; i < H; i += kAThreads)
    out[(size_t)b * H + i] = (hidden[(size_t)b * H + i] + o[(size_t)b * H + i]) * r;
}

int attn_segments(int max_sel) { return (max_sel + kSeg - 1) / kSeg; }

}  // namespace
}  // namespace fm

using namespace fm;

extern "C" size_t fm_decode_attention_workspace_bytes(int B, int max_sel) {
  if (B < 1 || max_sel < 1) return 0;
  const size_t nseg = (size_t)attn_segments(max_sel);
  return (size_t)B * nseg * kAH * (kAD + 2) * sizeof(float);
}

extern "C" fm_status fm_decode_attention(const float* q, const uint8_t* mem, int64_t row_stride_bytes, int n_mem,
                                         const int32_t* idx, const int32_t* count, int B, int max_sel,
                                         float* out, void* ws, size_t ws_bytes, cudaStream_t stream) {
  if (!q || !mem || !idx || !count || !out || !ws || B < 1 || B > 65535 || max_sel < 1 || n_mem < 1)
    return FM_ERR_INVALID_ARG;
  if (row_stride_bytes < (int64_t)n_mem * kRecord) return FM_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(q) & 15u) || (reinterpret_cast<uintptr_t>(mem) & 3u) ||
      (row_stride_bytes & 3) || (reinterpret_cast<uintptr_t>(ws) & 15u) ||
      (reinterpret_cast<uintptr_t>(idx) & 3u) || (reinterpret_cast<uintptr_t>(count) & 3u) ||
      (reinterpret_cast<uintptr_t>(out) & 3u))
    return FM_ERR_ALIGNMENT;
  if (ws_bytes < fm_decode_attention_workspace_bytes(B, max_sel)) return FM_ERR_INVALID_ARG;
  const int nseg = attn_segments(max_sel);
  float* part_o = static_cast<float*>(ws);
  float* part_ml = part_o + (size_t)B * nseg * kAH * kAD;
  static PerDeviceOnce smem_set;
  int dev = 0;
  cudaGetDevice(&dev);
  if (fm_status s = smem_limit_once(smem_set, dev, sparse_attn_partial_kernel, (int)sizeof(AttnSmem)))
    return s;
  sparse_attn_partial_kernel<<<dim3(nseg, B), kAThreads, sizeof(AttnSmem), stream>>>(
      q, mem, row_stride_bytes, n_mem, idx, count, max_sel, nseg, part_o, part_ml);
  sparse_attn_combine_kernel<<<dim3(kAH, B), kAD, 0, stream>>>(part_o, part_ml, nseg, out);
  note_launch();
  note_launch();
  return check_launch();
}

extern "C" fm_status fm_toy_decoder_update(const float* hidden, const float* attn_out, int B, int H, float eps,
                                           float* hidden_out, cudaStream_t stream) {
  if (!hidden || !attn_out || !hidden_out || B < 1 || B > 65535 || H != kAH * kAD || !(eps >= 0.f))
    return FM_ERR_INVALID_ARG;
  toy_update_kernel<<<B, kAThreads, 0, stream>>>(hidden, attn_out, H, eps, hidden_out);
  note_launch();
  return check_launch();
}
