// qprep.cu -- the indexer query side (README "Architecture", upper two chains):
//
//   hidden -> wq_a -> RMSNorm -> wq_b -> [H, D] -> YaRN RoPE (last 64 dims)
//          -> normalised Walsh-Hadamard                       = q
//   hidden -> weights_proj -> * HEAD_DIM^-1/2 N_HEADS^-1/2     = fused_w
//
// and the packing of q into the e4m3 operand image the scoring kernel's tensor
// cores read.  Three kernels do the chain:
//   qdown_kernel  C[b, m] = sum_k Wdown[m, k] hidden[b, k] for the stacked
//                 [wq_a; weights_proj] rows of every layer, split over K
//                 (weight-bandwidth bound for small B, fp32 FMA bound at B=64);
//   qnorm_kernel  sums the K splits, RMSNorm, fused_w, and the per-row RoPE
//                 cos/sin table (angles and cos/sin in fp64, rounded once);
//   qup_kernel    one CTA per (layer, head, row block): the 128 rows of one
//                 head of wq_b, then RoPE and the 128-point Hadamard butterfly
//                 in registers (warp shuffles), writing q in fp32.
#include <cuda_fp8.h>

#include "fm_internal.cuh"

namespace fm {
namespace {

constexpr int BM = 128;       // output rows per CTA (one head for the up projection)
constexpr int BK = 32;        // K slice staged in shared memory
constexpr int BM_PAD = 132;   // row pitch of the transposed weight tile (16-byte rows)
constexpr int kThreads = 256;

// Skinny GEMM tile: C[b0 + 0..BN, m0 + 0..BM] = sum_{k in [k0, k1)} W[m, k] X[b, k].
// Thread (tx, ty) owns rows m0 + 4tx .. 4tx+3 and columns b0 + ty*TN .. +TN.
template <int TN>
struct SkinnyTile {
  static constexpr int BN = 8 * TN;
  float acc[4][TN];

  __device__ void run(const float* __restrict__ W, int ldw, int M, const float* __restrict__ X,
                      int ldx, int nb, int m0, int k0, int k1, float (*Ws)[BM_PAD],
                      float (*Xs)[BN]) {
    const int tid = threadIdx.x;
    const int tx = tid & 31, ty = tid >> 5;
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < TN; ++j) acc[i][j] = 0.f;

    // global -> register staging (one K slice ahead)
    float4 wreg[4];
    float4 xreg[(BN * 8 + kThreads - 1) / kThreads];
    auto load = [&](int kb) {
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int r = (tid >> 3) + 32 * i;
        const int m = m0 + r;
        wreg[i] = (m < M) ? __ldg(reinterpret_cast<const float4*>(W + (size_t)m * ldw + kb) +
                                  (tid & 7))
                          : make_float4(0.f, 0.f, 0.f, 0.f);
      }
#pragma unroll
      for (int i = 0; i < (BN * 8 + kThreads - 1) / kThreads; ++i) {
        const int idx = tid + kThreads * i;
        if (idx < BN * 8) {
          const int b = idx >> 3;
          xreg[i] = (b < nb) ? __ldg(reinterpret_cast<const float4*>(X + (size_t)b * ldx + kb) +
                                     (idx & 7))
                             : make_float4(0.f, 0.f, 0.f, 0.f);
        }
      }
    };
    auto store = [&]() {
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int r = (tid >> 3) + 32 * i;
        const int c = (tid & 7) * 4;
        Ws[c + 0][r] = wreg[i].x;
        Ws[c + 1][r] = wreg[i].y;
        Ws[c + 2][r] = wreg[i].z;
        Ws[c + 3][r] = wreg[i].w;
      }
#pragma unroll
      for (int i = 0; i < (BN * 8 + kThreads - 1) / kThreads; ++i) {
        const int idx = tid + kThreads * i;
        if (idx < BN * 8) {
          const int b = idx >> 3;
          const int c = (idx & 7) * 4;
          Xs[c + 0][b] = xreg[i].x;
          Xs[c + 1][b] = xreg[i].y;
          Xs[c + 2][b] = xreg[i].z;
          Xs[c + 3][b] = xreg[i].w;
        }
      }
    };

    load(k0);
    for (int kb = k0; kb < k1; kb += BK) {
      __syncthreads();  // previous slice fully consumed
      store();
      __syncthreads();
      if (kb + BK < k1) load(kb + BK);
#pragma unroll 8
      for (int kk = 0; kk < BK; ++kk) {
        const float4 w = *reinterpret_cast<const float4*>(&Ws[kk][tx * 4]);
        float x[TN];
        if constexpr (TN % 4 == 0) {
#pragma unroll
          for (int j = 0; j < TN; j += 4) {
            const float4 v = *reinterpret_cast<const float4*>(&Xs[kk][ty * TN + j]);
            x[j] = v.x; x[j + 1] = v.y; x[j + 2] = v.z; x[j + 3] = v.w;
          }
        } else if constexpr (TN == 2) {
          const float2 v = *reinterpret_cast<const float2*>(&Xs[kk][ty * TN]);
          x[0] = v.x; x[1] = v.y;
        } else {
          x[0] = Xs[kk][ty];
        }
#pragma unroll
        for (int j = 0; j < TN; ++j) {
          acc[0][j] = fmaf(w.x, x[j], acc[0][j]);
          acc[1][j] = fmaf(w.y, x[j], acc[1][j]);
          acc[2][j] = fmaf(w.z, x[j], acc[2][j]);
          acc[3][j] = fmaf(w.w, x[j], acc[3][j]);
        }
      }
    }
  }
};

// a_part[s, b, m] = sum over split s of K of Wdown[m, k] * hidden[b, k].
template <int TN>
__global__ void __launch_bounds__(kThreads) qdown_kernel(const float* __restrict__ Wdown, int M,
                                                         int K, const float* __restrict__ hidden,
                                                         int B, int ksplit,
                                                         float* __restrict__ a_part) {
  using Tile = SkinnyTile<TN>;
  __shared__ __align__(16) float Ws[BK][BM_PAD];
  __shared__ __align__(16) float Xs[BK][Tile::BN];
  const int m0 = blockIdx.x * BM;
  const int s = blockIdx.y;
  const int b0 = blockIdx.z * Tile::BN;
  const int kper = K / ksplit;
  Tile t;
  t.run(Wdown, K, M, hidden + (size_t)b0 * K, K, min(Tile::BN, B - b0), m0, s * kper,
        (s + 1) * kper, Ws, Xs);
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;
  const int m = m0 + tx * 4;
#pragma unroll
  for (int j = 0; j < TN; ++j) {
    const int b = b0 + ty * TN + j;
    if (b < B && m < M) {
      float* dst = a_part + ((size_t)s * B + b) * M + m;
      *reinterpret_cast<float4*>(dst) = make_float4(t.acc[0][j], t.acc[1][j], t.acc[2][j],
                                                    t.acc[3][j]);
    }
  }
}

// One CTA per (row b, layer l): reduce the K splits, RMSNorm the wq_a part,
// scale the weights_proj part into fused_w, and (layer 0) the RoPE table.
__global__ void __launch_bounds__(kThreads) qnorm_kernel(
    const float* __restrict__ a_part, int ksplit, int B, int L, int R, int H,
    const float* __restrict__ q_norm, float eps, float w_scale, const int64_t* __restrict__ positions,
    const double* __restrict__ rope_freq, int rope_half, float* __restrict__ r_norm,
    float* __restrict__ fused_w, float* __restrict__ rope_cs) {
  const int b = blockIdx.x, l = blockIdx.y;
  const int M = L * (R + H);
  const float* base = a_part + (size_t)b * M + (size_t)l * (R + H);
  __shared__ float red[kThreads / 32];
  float ss = 0.f;
  for (int i = threadIdx.x; i < R; i += kThreads) {
    float a = 0.f;
    for (int s = 0; s < ksplit; ++s) a += base[(size_t)s * B * M + i];
    ss = fmaf(a, a, ss);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = ss;
  __syncthreads();
  float tot = 0.f;
#pragma unroll
  for (int w = 0; w < kThreads / 32; ++w) tot += red[w];
  const float inv_rms = 1.0f / sqrtf(tot / (float)R + eps);
  for (int i = threadIdx.x; i < R; i += kThreads) {
    float a = 0.f;
    for (int s = 0; s < ksplit; ++s) a += base[(size_t)s * B * M + i];
    r_norm[((size_t)b * L + l) * R + i] = a * inv_rms * q_norm[(size_t)l * R + i];
  }
  for (int h = threadIdx.x; h < H; h += kThreads) {
    float a = 0.f;
    for (int s = 0; s < ksplit; ++s) a += base[(size_t)s * B * M + R + h];
    fused_w[((size_t)b * L + l) * H + h] = a * w_scale;
  }
  if (l == 0 && threadIdx.x < rope_half) {
    const int j = threadIdx.x;
    const double theta = (double)positions[b] * rope_freq[j];
    double sn, cs;
    sincos(theta, &sn, &cs);
    rope_cs[((size_t)b * rope_half + j) * 2 + 0] = (float)cs;
    rope_cs[((size_t)b * rope_half + j) * 2 + 1] = (float)sn;
  }
}

// One CTA per (layer, head, row block): qf = wq_b[head rows] . r, then RoPE on
// dims 64..127 (pairs (64+j, 96+j)) and the normalised 128-point Hadamard.
template <int TN>
__global__ void __launch_bounds__(kThreads) qup_kernel(const float* __restrict__ w_up, int R,
                                                       const float* __restrict__ r_norm, int B,
                                                       int L, const float* __restrict__ rope_cs,
                                                       float* __restrict__ q) {
  using Tile = SkinnyTile<TN>;
  __shared__ __align__(16) float Ws[BK][BM_PAD];
  __shared__ __align__(16) float Xs[BK][Tile::BN];
  const int lh = blockIdx.x;  // l * 64 + h
  const int l = lh / kHeads, h = lh % kHeads;
  const int b0 = blockIdx.y * Tile::BN;
  const int nb = min(Tile::BN, B - b0);
  const float* W = w_up + ((size_t)l * kHeads + h) * kHeadDim * R;
  Tile t;
  t.run(W, R, kHeadDim, r_norm + ((size_t)b0 * L + l) * R, L * R, nb, 0, 0, R, Ws, Xs);

  // stage the [BN, 128] head block through shared memory (reuse Ws)
  __syncthreads();
  float* Cs = &Ws[0][0];  // BN * 128 floats <= BK * BM_PAD for BN <= 32
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;
#pragma unroll
  for (int j = 0; j < TN; ++j) {
    const int bl = ty * TN + j;
    *reinterpret_cast<float4*>(&Cs[bl * kHeadDim + tx * 4]) =
        make_float4(t.acc[0][j], t.acc[1][j], t.acc[2][j], t.acc[3][j]);
  }
  __syncthreads();

  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  for (int bl = warp; bl < nb; bl += kThreads / 32) {
    const int b = b0 + bl;
    float4 v4 = *reinterpret_cast<const float4*>(&Cs[bl * kHeadDim + lane * 4]);
    float x[4] = {v4.x, v4.y, v4.z, v4.w};
    // RoPE: lanes 16..23 hold dims 64..95 (x1), lanes 24..31 dims 96..127 (x2)
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float other = __shfl_xor_sync(0xffffffffu, x[i], 8);
      if (lane >= 16) {
        const int j = (lane * 4 + i - 64) & 31;
        const float c = rope_cs[((size_t)b * 32 + j) * 2 + 0];
        const float s = rope_cs[((size_t)b * 32 + j) * 2 + 1];
        x[i] = (lane < 24) ? (x[i] * c - other * s) : (x[i] * c + other * s);
      }
    }
    // Walsh-Hadamard butterflies, Sylvester order: bits 0,1 inside the thread,
    // bits 2..6 across lanes.
    {
      float a0 = x[0] + x[1], a1 = x[0] - x[1], a2 = x[2] + x[3], a3 = x[2] - x[3];
      x[0] = a0 + a2; x[2] = a0 - a2; x[1] = a1 + a3; x[3] = a1 - a3;
    }
#pragma unroll
    for (int sbit = 0; sbit < 5; ++sbit) {
      const int mask = 1 << sbit;
      const bool upper = (lane & mask) != 0;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float o = __shfl_xor_sync(0xffffffffu, x[i], mask);
        x[i] = upper ? (o - x[i]) : (x[i] + o);
      }
    }
    const float inv_sqrt_d = 0.088388347648318440f;  // 128^-1/2
    float* dst = q + (((size_t)b * L + l) * kHeads + h) * kHeadDim + lane * 4;
    *reinterpret_cast<float4*>(dst) =
        make_float4(x[0] * inv_sqrt_d, x[1] * inv_sqrt_d, x[2] * inv_sqrt_d, x[3] * inv_sqrt_d);
  }
}

// Exact decode of one OCP E4M3 byte (finite codes only).
__device__ __forceinline__ float e4m3_value(uint32_t c) {
  const int e = (c >> 3) & 15;
  const int m = c & 7;
  const float mag = e ? ldexpf(1.0f + 0.125f * (float)m, e - 7) : ldexpf(0.125f * (float)m, -6);
  return (c & 0x80u) ? -mag : mag;
}

__device__ __forceinline__ uint32_t to_e4m3(float x) {
  return (uint32_t)__nv_cvt_float_to_fp8(x, __NV_SATFINITE, __NV_E4M3);
}

// One warp per (b, l, h): choose the head's power-of-two scale 2^e so that
// max|q| 2^e lies in [128, 256), split x = q 2^e into P e4m3 pieces
// x ~= p0 + p1/16 + p2/256 and write them into the 128B-swizzled K-major
// operand image (row p*64 + h, 128 bytes per row); wprime = fused_w 2^-e.
template <int P>
__global__ void __launch_bounds__(kThreads) qpack_kernel(const float* __restrict__ q,
                                                         const float* __restrict__ fused_w, int n,
                                                         uint8_t* __restrict__ qpack,
                                                         float* __restrict__ wprime,
                                                         int32_t* __restrict__ qexp) {
  const int idx = blockIdx.x * (kThreads / 32) + (threadIdx.x >> 5);  // (b*L + l)*64 + h
  if (idx >= n) return;
  const int lane = threadIdx.x & 31;
  const int h = idx % kHeads;
  const int bl = idx / kHeads;
  const float4 v = __ldg(reinterpret_cast<const float4*>(q + (size_t)idx * kHeadDim) + lane);
  float m = fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w)));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  int e = 0;
  if (m > 0.f && isfinite(m)) e = 7 - ilogbf(m);
  e = max(-120, min(120, e));
  const float up = ldexpf(1.0f, e);
  float x[4] = {v.x * up, v.y * up, v.z * up, v.w * up};
  uint8_t* img = qpack + (size_t)bl * (P * kHeads * kHeadDim);
#pragma unroll
  for (int p = 0; p < P; ++p) {
    uint32_t word = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint32_t c = to_e4m3(x[i]);
      word |= c << (8 * i);
      x[i] = (x[i] - e4m3_value(c)) * 16.0f;  // exact: the residual of a 4-bit rounding
    }
    const int row = p * kHeads + h;
    *reinterpret_cast<uint32_t*>(img + sw128_offset(row, lane * 4)) = word;
  }
  if (lane == 0) {
    wprime[idx] = fused_w[idx] * ldexpf(1.0f, -e);
    qexp[idx] = e;
  }
}

template <int TN>
void launch_qdown(fm_ctx* ctx, const float* hidden, int B, int ksplit, cudaStream_t st) {
  const int M = ctx->cfg.n_layers * (ctx->cfg.q_lora_rank + ctx->cfg.n_heads);
  constexpr int BN = 8 * TN;
  dim3 grid((M + BM - 1) / BM, ksplit, (B + BN - 1) / BN);
  qdown_kernel<TN><<<grid, kThreads, 0, st>>>(ctx->w_down, M, ctx->cfg.hidden, hidden, B, ksplit,
                                              ctx->a_part);
  note_launch();
}

template <int TN>
void launch_qup(fm_ctx* ctx, int B, float* q, cudaStream_t st) {
  constexpr int BN = 8 * TN;
  dim3 grid(ctx->cfg.n_layers * kHeads, (B + BN - 1) / BN);
  qup_kernel<TN><<<grid, kThreads, 0, st>>>(ctx->w_up, ctx->cfg.q_lora_rank, ctx->r_norm, B,
                                            ctx->cfg.n_layers, ctx->rope_cs, q);
  note_launch();
}

}  // namespace

fm_status launch_query_prep(fm_ctx* ctx, const float* hidden, const int64_t* positions, int B,
                            float* q, float* fused_w, cudaStream_t st) {
  const fm_config& c = ctx->cfg;
  const int M = c.n_layers * (c.q_lora_rank + c.n_heads);
  const int mtiles = (M + BM - 1) / BM;
  // K splits: enough CTAs to cover the SMs a few times, K slices of >= 256.
  const int btiles = (B + 63) / 64;
  int ksplit = 1;
  while (ksplit * 2 <= ctx->splitk_max && c.hidden % (ksplit * 2 * BK) == 0 &&
         c.hidden / (ksplit * 2) >= 256 && mtiles * btiles * ksplit < 4 * ctx->num_sms)
    ksplit *= 2;
  if (B <= 8)
    launch_qdown<1>(ctx, hidden, B, ksplit, st);
  else if (B <= 16)
    launch_qdown<2>(ctx, hidden, B, ksplit, st);
  else if (B <= 32)
    launch_qdown<4>(ctx, hidden, B, ksplit, st);
  else
    launch_qdown<8>(ctx, hidden, B, ksplit, st);

  const float w_scale = (float)(1.0 / sqrt((double)c.head_dim * (double)c.n_heads));
  qnorm_kernel<<<dim3(B, c.n_layers), kThreads, 0, st>>>(
      ctx->a_part, ksplit, B, c.n_layers, c.q_lora_rank, c.n_heads, ctx->q_norm, c.rms_eps,
      w_scale, positions, ctx->rope_freq, c.rope_dim / 2, ctx->r_norm, fused_w, ctx->rope_cs);
  note_launch();

  if (B <= 8)
    launch_qup<1>(ctx, B, q, st);
  else
    launch_qup<2>(ctx, B, q, st);
  return check_launch();
}

fm_status launch_qpack(fm_ctx* ctx, const float* q, const float* fused_w, int B,
                       cudaStream_t st) {
  const int n = B * ctx->cfg.n_layers * kHeads;
  const int grid = (n + kThreads / 32 - 1) / (kThreads / 32);
  if (ctx->cfg.q_pieces == 3)
    qpack_kernel<3><<<grid, kThreads, 0, st>>>(q, fused_w, n, ctx->qpack, ctx->wprime, ctx->qexp);
  else
    qpack_kernel<2><<<grid, kThreads, 0, st>>>(q, fused_w, n, ctx->qpack, ctx->wprime, ctx->qexp);
  note_launch();
  return check_launch();
}

}  // namespace fm
