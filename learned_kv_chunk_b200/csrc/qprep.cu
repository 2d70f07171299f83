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
#include <cuda.h>
#include <cudaTypedefs.h>
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

// fp32 -> tf32 (round to nearest, ties away; low 13 mantissa bits zero).
__device__ __forceinline__ float tf32_round(float x) {
  uint32_t r;
  asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
  return __uint_as_float(r);
}

// x = hi + lo with hi = tf32(x): the operand split of three-pass TF32.
__global__ void split_tf32_kernel(const float* __restrict__ x, float* __restrict__ hi,
                                  float* __restrict__ lo, int64_t n) {
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += (int64_t)gridDim.x * blockDim.x) {
    const float v = x[i];
    const float h = tf32_round(v);
    hi[i] = h;
    lo[i] = v - h;
  }
}

// ------------------------------------------------ tensor-core skinny GEMM
// part[s][n][m] = W[m][:] . X[n][:] over one stretch of K, at fp32-level
// accuracy on the tensor cores: each operand is split as hi = tf32(v),
// lo = v - hi and the product is taken as hi*hi + hi*lo + lo*hi (TF32 MMAs,
// fp32 accumulation in TMEM).  X (a few hundred KB) arrives already split; W,
// the bulk of the bytes, streams in as fp32 once and is split in the CTA.
//
// Stream-K: the (tile, 32-wide K block) units of the whole product, tiles
// being 128 rows of W x BN rows of X, are dealt out in equal contiguous
// ranges to one persistent CTA per SM, so no CTA waits on a wave tail and the
// pipeline runs across tile boundaries.  A CTA's run of units inside one tile
// is a segment; its partial goes to slot (CTA - first CTA of the tile), and
// the consumer sums the tile's StreamK::slots partials (a fixed order:
// deterministic).
//
//   warp 0 lane 0   TMA producer: per unit the fp32 W tile (128 x 32) and the
//                   X hi / lo tiles (BN x 32 each, adjacent), 128B-swizzled
//   warps 4..7      split: thread t reads row t of the W tile and writes its
//                   hi and lo parts into the stage's TMEM columns (A operand)
//   warp 1 lane 0   MMA issuer: A from TMEM, B from shared memory:
//                   hi x [Xhi; Xlo] (N = 2 BN) + lo x Xhi (N = BN)
//   warps 8..11     epilogue: per segment, accumulator halves summed
//                   (hi.Xhi + lo.Xhi | hi.Xlo) and stored to the slot
//
// TMEM: the accumulator buffer(s) of 2 BN columns, then 64 columns (hi, lo) per
// stage.  A stage's TMEM columns are rewritten only after its shared-memory
// stage was refilled, which waits for the MMAs of the previous use to retire.
constexpr int kTcThreads = 384;
constexpr int kTcBM = 128;                              // rows of W per tile (MMA M)
constexpr int kTcBK = 32;                               // K per unit: 32 fp32 = one 128-byte row
constexpr uint32_t kTcWTile = kTcBM * kTcBK * 4;        // 16 KB
constexpr int kTcSplitWarp0 = 4;                        // warps 4..7: TMEM lane quarters 0..3
constexpr int kTcEpiWarp0 = 8;                          // warps 8..11

struct StreamK {
  int KB;       // K blocks per tile
  int mtiles;   // tiles along M; tile t = ntile * mtiles + mtile
  int bn;       // X rows per tile
  int G;        // CTAs
  int64_t U;    // units = tiles * KB
  __host__ __device__ int64_t start(int c) const { return U * c / G; }
  __host__ __device__ int cta_of(int64_t u) const { return (int)(((int64_t)G * (u + 1) - 1) / U); }
  __host__ __device__ int first_cta(int t) const { return cta_of((int64_t)t * KB); }
  __host__ __device__ int slots(int t) const { return cta_of((int64_t)t * KB + KB - 1) - first_cta(t) + 1; }
};

struct TcGemmArgs {
  int M, N, K;          // W [M, K]; X [N, K] (one layer of it); part [slot][N][M]
  int rows_per_layer;   // W rows per X layer (the up projection); 0: X has one layer
  float* part;
  int64_t split_stride;
  int* err;
  StreamK sk;
};

__host__ __device__ constexpr uint32_t idesc_tf32_f32(int M, int N) {
  return (1u << 4)                                // D format F32
         | (2u << 7) | (2u << 10)                 // A, B format TF32
         | (static_cast<uint32_t>(N >> 3) << 17)  // N / 8
         | (static_cast<uint32_t>(M >> 4) << 24); // M / 16
}

// D[tmem] (+)= A[tmem] * B[smem desc]^T, TF32 inputs, fp32 accumulate.  A's
// rows are the TMEM lanes, one TF32 value per 32-bit column.
__device__ __forceinline__ void umma_tf32_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                             uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::tf32 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Two 32-lane x 32-column TMEM stores (thread i writes lane base+i of each),
// then one wait that covers both.
__device__ __forceinline__ void tmem_st32x2_wait(uint32_t taddr0, const uint32_t* v, uint32_t taddr1,
                                                 const uint32_t* w) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, "
      "%17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};\n\t"
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%33], "
      "{%34, %35, %36, %37, %38, %39, %40, %41, %42, %43, %44, %45, %46, %47, %48, %49, "
      "%50, %51, %52, %53, %54, %55, %56, %57, %58, %59, %60, %61, %62, %63, %64, %65};\n\t"
      "tcgen05.wait::st.sync.aligned;" ::"r"(taddr0),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]),
      "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15]),
      "r"(v[16]), "r"(v[17]), "r"(v[18]), "r"(v[19]), "r"(v[20]), "r"(v[21]), "r"(v[22]), "r"(v[23]),
      "r"(v[24]), "r"(v[25]), "r"(v[26]), "r"(v[27]), "r"(v[28]), "r"(v[29]), "r"(v[30]), "r"(v[31]),
      "r"(taddr1),
      "r"(w[0]), "r"(w[1]), "r"(w[2]), "r"(w[3]), "r"(w[4]), "r"(w[5]), "r"(w[6]), "r"(w[7]),
      "r"(w[8]), "r"(w[9]), "r"(w[10]), "r"(w[11]), "r"(w[12]), "r"(w[13]), "r"(w[14]), "r"(w[15]),
      "r"(w[16]), "r"(w[17]), "r"(w[18]), "r"(w[19]), "r"(w[20]), "r"(w[21]), "r"(w[22]), "r"(w[23]),
      "r"(w[24]), "r"(w[25]), "r"(w[26]), "r"(w[27]), "r"(w[28]), "r"(w[29]), "r"(w[30]), "r"(w[31])
      : "memory");
}

template <int BN>
struct TcCfg {
  static constexpr int kAccBufs = BN <= 64 ? 2 : 1;
  static constexpr int kAccCols = 2 * BN;
  static constexpr int kStages = (512 - kAccBufs * kAccCols) / 64;  // TMEM A stages = smem stages
  static constexpr uint32_t kStageBytes = kTcWTile + 2u * BN * kTcBK * 4;
  static constexpr uint32_t kSmem = kStages * kStageBytes + (3 * kStages + 4) * 8 + 16 + 1024;
};

template <int BN>
__global__ void __launch_bounds__(kTcThreads, 1)
    tc_gemm_kernel(const __grid_constant__ CUtensorMap w_map, const __grid_constant__ CUtensorMap x_hi,
                   const __grid_constant__ CUtensorMap x_lo, TcGemmArgs a) {
  using C = TcCfg<BN>;
  constexpr int S = C::kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  constexpr uint32_t kXTile = BN * kTcBK * 4;
  constexpr uint32_t kStage = C::kStageBytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + (size_t)S * kStage);
  uint64_t* split = full + S;
  uint64_t* empty = split + S;
  uint64_t* acc_full = empty + S;    // [2]
  uint64_t* acc_empty = acc_full + 2;  // [2]
  uint32_t* sTmem = reinterpret_cast<uint32_t*>(acc_empty + 2);
  volatile int* sAbort = reinterpret_cast<volatile int*>(sTmem + 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const StreamK& sk = a.sk;
  const int64_t u0 = sk.start(blockIdx.x), u1 = sk.start(blockIdx.x + 1);

  if (threadIdx.x == 0) {
    for (int i = 0; i < S; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&split[i], 4);  // one arrival per split warp
      mbar_init(&empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&acc_full[i], 1);
      mbar_init(&acc_empty[i], 4);  // one arrival per epilogue warp
    }
    *sAbort = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 2) {
    tmem_alloc(sTmem, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *sTmem;
  const uint32_t a_col0 = (uint32_t)(C::kAccBufs * C::kAccCols);

  if (warp == 0 && lane == 0) {
    // ------------------------------------------------------------ producer
    // The unit's tile coordinates advance incrementally: divisions run once
    // per tile, not per unit (a dependent chain of integer divisions cost
    // this single thread ~0.6 us per unit, longer than the copies took).
    uint32_t stage = 0, phase = 0, issued = 0;
    int t = (int)(u0 / sk.KB), kb = (int)(u0 - (int64_t)t * sk.KB);
    int m0 = 0, n0 = 0, layer = 0;
    const auto tile_coords = [&]() {
      m0 = (t % sk.mtiles) * kTcBM;
      n0 = (t / sk.mtiles) * BN;
      layer = a.rows_per_layer ? m0 / a.rows_per_layer : 0;
    };
    tile_coords();
    for (int64_t u = u0; u < u1; ++u) {
      if (!mbar_wait_bounded(&empty[stage], phase ^ 1, sAbort, a.err)) break;
      const int k = kb * kTcBK;
      uint8_t* st = smem + (size_t)stage * kStage;
      mbar_arrive_expect_tx(&full[stage], kStage);
      tma_load_2d(st, &w_map, k, m0, &full[stage]);
      tma_load_3d(st + kTcWTile, &x_hi, k, layer, n0, &full[stage]);
      tma_load_3d(st + kTcWTile + kXTile, &x_lo, k, layer, n0, &full[stage]);
      ++issued;
      if (++stage == (uint32_t)S) { stage = 0; phase ^= 1u; }
      if (++kb == sk.KB) {
        kb = 0;
        ++t;
        tile_coords();
      }
    }
    // every copy issued lands before the CTA can exit
    const uint32_t inflight = issued < (uint32_t)S ? issued : (uint32_t)S;
    for (uint32_t j = 0; j < inflight; ++j) {
      const uint32_t it = issued - 1 - j;
      mbar_drain(&full[it % S], (it / S) & 1, a.err);
    }
  } else if (warp == 1 && lane == 0) {
    // ---------------------------------------------------------- MMA issuer
    constexpr uint32_t idesc2 = idesc_tf32_f32(kTcBM, 2 * BN), idesc1 = idesc_tf32_f32(kTcBM, BN);
    uint32_t stage = 0, phase = 0, buf = 0;
    uint32_t par = 0;  // bit b: parity of accumulator buffer b's uses
    bool ok = true;
    for (int64_t u = u0; u < u1 && ok;) {
      const int t = (int)(u / sk.KB);
      const int64_t seg_end = min(u1, (int64_t)(t + 1) * sk.KB);
      if (!mbar_wait_bounded(&acc_empty[buf], ((par >> buf) & 1u) ^ 1u, sAbort, a.err)) break;
      tc_fence_after();
      const uint32_t d = tmem + buf * (uint32_t)C::kAccCols;
      for (bool first = true; u < seg_end; ++u, first = false) {
        if (!mbar_wait_bounded(&split[stage], phase, sAbort, a.err)) { ok = false; break; }
        tc_fence_after();
        const uint32_t base = smem_u32(smem + (size_t)stage * kStage);
        const uint64_t dx = sdesc_kmajor_sw128(base + kTcWTile);  // [Xhi; Xlo]: 2 BN rows
        const uint32_t a_hi = tmem + a_col0 + stage * 64u, a_lo = a_hi + 32u;
#pragma unroll
        for (int k = 0; k < kTcBK / 8; ++k) {  // K = 8 tf32 per MMA: 8 TMEM columns, 32 smem bytes
          const uint64_t o = 2u * (uint32_t)k;  // +32 bytes in the 16-byte address field
          const uint32_t c = 8u * (uint32_t)k;
          umma_tf32_ts(d, a_hi + c, dx + o, idesc2, (first && k == 0) ? 0u : 1u);
          umma_tf32_ts(d, a_lo + c, dx + o, idesc1, 1u);
        }
        umma_commit(&empty[stage]);  // the stage may be refilled once these MMAs retire
        if (++stage == (uint32_t)S) { stage = 0; phase ^= 1u; }
      }
      if (!ok) break;
      umma_commit(&acc_full[buf]);
      par ^= 1u << buf;
      if (C::kAccBufs == 2) buf ^= 1u;
    }
  } else if (warp >= kTcSplitWarp0 && warp < kTcEpiWarp0) {
    // --------------------------------------------------------------- split
    const int q = warp - kTcSplitWarp0;  // TMEM lane quarter
    const int r = q * 32 + lane;         // row of the W tile
    const uint32_t lane_base = tmem + ((uint32_t)(q * 32) << 16);
    uint32_t stage = 0, phase = 0;
    for (int64_t u = u0; u < u1; ++u) {
      // every lane waits (each needs the TMA data visible); the warp leaves
      // together if any lane's wait ran out, before the .aligned TMEM stores
      const bool ok = mbar_wait_bounded(&full[stage], phase, sAbort, a.err);
      if (!__all_sync(0xffffffffu, ok)) break;
      tc_fence_after();
      // row r: 128 bytes, its 16-byte chunk c stored at chunk c ^ (r % 8)
      const uint8_t* row = smem + (size_t)stage * kStage + (size_t)r * 128;
      uint32_t hi[32], lo[32];
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        const float4 v = *reinterpret_cast<const float4*>(row + ((c ^ (r & 7)) << 4));
        const float e[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float h = tf32_round(e[i]);
          hi[4 * c + i] = __float_as_uint(h);
          lo[4 * c + i] = __float_as_uint(e[i] - h);
        }
      }
      const uint32_t col = a_col0 + stage * 64u;
      tmem_st32x2_wait(lane_base + col, hi, lane_base + col + 32u, lo);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&split[stage]);
      if (++stage == (uint32_t)S) { stage = 0; phase ^= 1u; }
    }
  } else if (warp >= kTcEpiWarp0) {
    // ------------------------------------------------------------ epilogue
    const int q = warp - kTcEpiWarp0;
    const uint32_t lane_base = tmem + ((uint32_t)(q * 32) << 16);
    uint32_t buf = 0;
    uint32_t par = 0;  // bit b: parity of accumulator buffer b's uses
    for (int64_t u = u0; u < u1;) {
      const int t = (int)(u / sk.KB);
      u = min(u1, (int64_t)(t + 1) * sk.KB);
      int good = 1;
      if (lane == 0) good = mbar_wait_bounded(&acc_full[buf], (par >> buf) & 1u, sAbort, a.err);
      good = __shfl_sync(0xffffffffu, good, 0);
      if (!good) break;
      tc_fence_after();
      const int m = (t % sk.mtiles) * kTcBM + q * 32 + lane, n0 = (t / sk.mtiles) * BN;
      float* out = a.part + (int64_t)((int)blockIdx.x - sk.first_cta(t)) * a.split_stride;
      const uint32_t dcol = buf * (uint32_t)C::kAccCols;
#pragma unroll 1
      for (int c0 = 0; c0 < BN; c0 += 32) {
        uint32_t v[32], w[32];
        tmem_ld32_wait(lane_base + dcol + (uint32_t)c0, v);        // hi.Xhi + lo.Xhi
        tmem_ld32_wait(lane_base + dcol + (uint32_t)(BN + c0), w);  // hi.Xlo
        if (m < a.M) {
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const int n = n0 + c0 + j;
            if (n < a.N) out[(int64_t)n * a.M + m] = __uint_as_float(v[j]) + __uint_as_float(w[j]);
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[buf]);
      par ^= 1u << buf;
      if (C::kAccBufs == 2) buf ^= 1u;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// The up projection's K-split partials summed, then RoPE and the Hadamard:
// one warp per (row, layer, head).
__global__ void __launch_bounds__(kThreads) qup_finish_kernel(const float* __restrict__ part, StreamK sk,
                                                              int nsplit, int64_t split_stride, int B, int L,
                                                              const float* __restrict__ rope_cs,
                                                              float* __restrict__ q);

// One CTA per (row b, layer l): reduce the K splits, RMSNorm the wq_a part,
// scale the weights_proj part into fused_w, and (layer 0) the RoPE table.
// ------------------------------------------------ GEMV for up to 8 rows
// part[s, b, m] = sum over the s-th K slice of W[m, k] X[b, layer(m), k], for
// B <= TB <= 8 rows of X: bound by the bytes of W, each read once.  A warp owns
// 4 consecutive rows of W and one K slice; lane j streams the float4 columns
// k = 4j + 128i of its 4 rows with gemv_unroll(TB) slices of loads in flight, the
// CTA's X slice sits in shared memory, and the 4 x TB sums are reduced across
// the warp by a butterfly in which every exchange halves the values a lane
// holds (4 TB - 1 shuffles in all) and lane j ends with sum number j.
constexpr int kGemvWarps = 8;
constexpr int kGemvRows = 4;  // rows of W per warp
constexpr int kGemvUnroll = 4;
// One row: three slices per warp in flight and three CTAs per SM (registers
// for 3 x 256 threads), so a down projection of 408 CTAs runs in one wave;
// more rows: four slices, two CTAs per SM.
__host__ __device__ constexpr int gemv_unroll(int TB) { return TB == 1 ? 3 : kGemvUnroll; }
__host__ __device__ constexpr int gemv_min_blocks(int TB) { return TB == 1 ? 3 : 1; }
__host__ __device__ constexpr int gemv_ctas_per_sm(int TB) { return TB == 1 ? 3 : 2; }

template <int TB>
__global__ void __launch_bounds__(kGemvWarps * 32, gemv_min_blocks(TB)) gemv_kernel(
    const float* __restrict__ W, int M, int K, int kslice, const float* __restrict__ X,
    int64_t x_row_stride, int64_t x_layer_stride, int rows_per_layer, int B, float* __restrict__ part) {
  extern __shared__ __align__(16) float Xs[];  // [TB][kslice]
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m_cta = blockIdx.x * kGemvWarps * kGemvRows;
  const int m0 = m_cta + warp * kGemvRows;
  const int s = blockIdx.y;
  const int k0 = s * kslice;
  const int layer = rows_per_layer > 0 ? m_cta / rows_per_layer : 0;
  const bool rows_ok = m0 + kGemvRows <= M;
  constexpr int kU = gemv_unroll(TB);
  // W does not depend on the kernel ahead: start its first slices now.  The
  // register ring w holds kU slices (slice i in w[i % kU]);
  // a slot is reloaded with slice i + kU as soon as slice i is used.
  float4 w[kU][kGemvRows];
  const float* wrow = W + (size_t)m0 * K + k0 + 4 * lane;
  auto load_slice = [&](float4* dst, int i) {
#pragma unroll
    for (int r = 0; r < kGemvRows; ++r)
      dst[r] = (rows_ok && i * 128 < kslice)
                   ? __ldg(reinterpret_cast<const float4*>(wrow + (size_t)r * K + i * 128))
                   : make_float4(0.f, 0.f, 0.f, 0.f);
  };
#pragma unroll
  for (int u = 0; u < kU; ++u) load_slice(w[u], u);
  grid_dependency_wait();  // X is written by the kernel ahead
  const float* xsrc = X + (size_t)layer * x_layer_stride + k0;
  for (int i = threadIdx.x; i < TB * kslice / 4; i += kGemvWarps * 32) {
    const int b = (i * 4) / kslice, k = (i * 4) % kslice;
    reinterpret_cast<float4*>(Xs)[i] =
        b < B ? __ldg(reinterpret_cast<const float4*>(xsrc + (size_t)b * x_row_stride + k))
              : make_float4(0.f, 0.f, 0.f, 0.f);
  }
  __syncthreads();
  float acc[kGemvRows * TB];
#pragma unroll
  for (int v = 0; v < kGemvRows * TB; ++v) acc[v] = 0.f;
  const int nslices = kslice / 128;
  for (int i0 = 0; i0 < nslices; i0 += kU) {
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      const int i = i0 + u;
      if (i >= nslices) break;
#pragma unroll
      for (int b = 0; b < TB; ++b) {
        const float4 x = *reinterpret_cast<const float4*>(Xs + (size_t)b * kslice + i * 128 + 4 * lane);
#pragma unroll
        for (int r = 0; r < kGemvRows; ++r) {
          float a = acc[r * TB + b];
          a = fmaf(w[u][r].x, x.x, a);
          a = fmaf(w[u][r].y, x.y, a);
          a = fmaf(w[u][r].z, x.z, a);
          a = fmaf(w[u][r].w, x.w, a);
          acc[r * TB + b] = a;
        }
      }
      load_slice(w[u], i + kU);
    }
  }
  // butterfly: at stride h, the lanes with bit h set keep the upper half of
  // their values and the others the lower half, each adding its partner's copy
  constexpr int V = kGemvRows * TB;
#pragma unroll
  for (int h = V / 2; h >= 1; h >>= 1) {
    const bool upper = (lane & h) != 0;
#pragma unroll
    for (int i = 0; i < h; ++i) {
      const float send = upper ? acc[i] : acc[i + h];
      const float keep = upper ? acc[i + h] : acc[i];
      acc[i] = keep + __shfl_xor_sync(0xffffffffu, send, h);
    }
  }
#pragma unroll
  for (int h = V; h < 32; h <<= 1) acc[0] += __shfl_xor_sync(0xffffffffu, acc[0], h);
  if (lane < V && rows_ok) {
    const int r = lane / TB, b = lane % TB;
    if (b < B) part[((size_t)s * B + b) * M + m0 + r] = acc[0];
  }
}

constexpr int kNormThreads = 1024;  // one thread per element of a (row, layer) block, two past 1024

__global__ void __launch_bounds__(kNormThreads) qnorm_kernel(
    const float* __restrict__ a_part, int ksplit, StreamK sk, int B, int L, int R, int H,
    const float* __restrict__ q_norm, float eps, float w_scale, const int64_t* __restrict__ positions,
    const double* __restrict__ rope_freq, int rope_half, float* __restrict__ r_norm,
    float* __restrict__ fused_w, float* __restrict__ rope_cs, float* __restrict__ r_hi,
    float* __restrict__ r_lo) {
  grid_dependency_wait();  // the partial sums come from the kernel ahead
  const int b = blockIdx.x, l = blockIdx.y;
  const int t = threadIdx.x;
  const int M = L * (R + H);
  const float* base = a_part + (size_t)b * M + (size_t)l * (R + H);
  // partials of element i: ksplit (K splits), or its tile's stream-K slots,
  // looked up per tile from a table built once
  constexpr int kMaxTiles = 64;  // tiles in the table; a (row, layer) block spans (R + H) / 128 + 2
  __shared__ int s_slots[kMaxTiles];
  __shared__ float red[kNormThreads / 32];
  const int t0 = (l * (R + H)) / kTcBM;
  if (ksplit <= 0)
    for (int j = t; j < kMaxTiles; j += kNormThreads) s_slots[j] = sk.slots((b / sk.bn) * sk.mtiles + t0 + j);
  // the row's RoPE table (layer 0's block): angles and cos/sin in fp64,
  // rounded once; computed while the partial sums below are in flight
  const int last_warp = kNormThreads - 32;
  if (l == 0 && t >= last_warp && t - last_warp < rope_half) {
    const int j = t - last_warp;
    const double theta = (double)positions[b] * rope_freq[j];
    double sn, cs;
    sincos(theta, &sn, &cs);
    rope_cs[((size_t)b * rope_half + j) * 2 + 0] = (float)cs;
    rope_cs[((size_t)b * rope_half + j) * 2 + 1] = (float)sn;
  }
  __syncthreads();
  auto nparts = [&](int i) {
    if (ksplit > 0) return ksplit;
    const int j = (l * (R + H) + i) / kTcBM - t0;
    return j < kMaxTiles ? s_slots[j] : sk.slots((b / sk.bn) * sk.mtiles + t0 + j);
  };
  // elements t and t + 1024 of the block: every partial of both is loaded
  // before any is summed
  const int n = R + H;
  constexpr int kMaxParts = 16;
  float v0[kMaxParts], v1[kMaxParts];
  const int i0 = t, i1 = t + kNormThreads;
  const int np0 = i0 < n ? nparts(i0) : 0, np1 = i1 < n ? nparts(i1) : 0;
#pragma unroll
  for (int s = 0; s < kMaxParts; ++s) {
    v0[s] = s < np0 ? __ldg(base + (size_t)s * B * M + i0) : 0.f;
    v1[s] = s < np1 ? __ldg(base + (size_t)s * B * M + i1) : 0.f;
  }
  float a0 = 0.f, a1 = 0.f;
#pragma unroll
  for (int s = 0; s < kMaxParts; ++s) { a0 += v0[s]; a1 += v1[s]; }
  for (int s = kMaxParts; s < np0; ++s) a0 += base[(size_t)s * B * M + i0];
  for (int s = kMaxParts; s < np1; ++s) a1 += base[(size_t)s * B * M + i1];
  auto sum_of = [&](int i) {  // elements past the first 2048 (ranks above 1984 only)
    float a = 0.f;
    for (int s = 0, np = nparts(i); s < np; ++s) a += base[(size_t)s * B * M + i];
    return a;
  };
  float ss = (i0 < R ? a0 * a0 : 0.f) + (i1 < R ? a1 * a1 : 0.f);
  for (int i = t + 2 * kNormThreads; i < R; i += kNormThreads) {
    const float a = sum_of(i);
    ss = fmaf(a, a, ss);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  if ((t & 31) == 0) red[t >> 5] = ss;
  __syncthreads();
  float tot = 0.f;
#pragma unroll
  for (int w = 0; w < kNormThreads / 32; ++w) tot += red[w];
  const float inv_rms = 1.0f / sqrtf(tot / (float)R + eps);
  auto emit = [&](int i, float a) {
    if (i >= n) return;
    if (i >= R) {
      fused_w[((size_t)b * L + l) * H + (i - R)] = a * w_scale;
      return;
    }
    const float r = a * inv_rms * q_norm[(size_t)l * R + i];
    r_norm[((size_t)b * L + l) * R + i] = r;
    if (r_hi) {  // the split operand of the tensor-core up projection
      const float hi = tf32_round(r);
      r_hi[((size_t)b * L + l) * R + i] = hi;
      r_lo[((size_t)b * L + l) * R + i] = r - hi;
    }
  };
  emit(i0, a0);
  emit(i1, a1);
  for (int i = t + 2 * kNormThreads; i < n; i += kNormThreads) emit(i, sum_of(i));
}

// RoPE on dims 64..127 (pairs (64+j, 96+j)) and the normalised Hadamard of
// one head vector held by a warp, four dims per lane (lane holds dims
// 4*lane .. 4*lane+3), written to q[b, l, h, :].
__device__ __forceinline__ void rope_wht_store(float x[4], int b, int l, int h, int L, int lane,
                                               const float* __restrict__ rope_cs,
                                               float* __restrict__ q) {
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

// Sums the partials of wq_b . r (nsplit slices, or when nsplit is 0 the
// stream-K slots of the head's tile), then RoPE and the Hadamard: one warp per
// (b, l, h).
__global__ void __launch_bounds__(kThreads) qup_finish_kernel(const float* __restrict__ part, StreamK sk,
                                                              int nsplit, int64_t split_stride, int B, int L,
                                                              const float* __restrict__ rope_cs,
                                                              float* __restrict__ q) {
  grid_dependency_wait();  // the partials come from the kernel ahead
  const int idx = blockIdx.x * (kThreads / 32) + (threadIdx.x >> 5);  // (b*L + l)*64 + h
  if (idx >= B * L * kHeads) return;
  const int lane = threadIdx.x & 31;
  const int h = idx % kHeads, bl = idx / kHeads, l = bl % L, b = bl / L;
  const float* src = part + (size_t)b * L * kHeads * kHeadDim + ((size_t)l * kHeads + h) * kHeadDim + lane * 4;
  // one head's 128 rows of wq_b are one tile: its partials are the tile's slots
  const int nslots = nsplit > 0 ? nsplit : sk.slots((b / sk.bn) * sk.mtiles + l * kHeads + h);
  float4 acc = __ldg(reinterpret_cast<const float4*>(src));
  for (int s = 1; s < nslots; ++s) {
    const float4 v = __ldg(reinterpret_cast<const float4*>(src + (int64_t)s * split_stride));
    acc.x += v.x; acc.y += v.y; acc.z += v.z; acc.w += v.w;
  }
  float x[4] = {acc.x, acc.y, acc.z, acc.w};
  rope_wht_store(x, b, l, h, L, lane, rope_cs, q);
}

// The same for rows [b0, b0 + nb) of one head staged in Cs ([rows, 128]
// floats); one warp per row.
__device__ __forceinline__ void qup_epilogue(const float* Cs, int rows, int b0, int nb, int L, int l,
                                             int h, int lane, int warp, const float* __restrict__ rope_cs,
                                             float* __restrict__ q) {
  for (int bl = warp; bl < nb && bl < rows; bl += kThreads / 32) {
    const float4 v4 = *reinterpret_cast<const float4*>(&Cs[bl * kHeadDim + lane * 4]);
    float x[4] = {v4.x, v4.y, v4.z, v4.w};
    rope_wht_store(x, b0 + bl, l, h, L, lane, rope_cs, q);
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

  // stage the [BN, 128] head block through shared memory (reuse Ws), at most
  // 32 rows at a time (32 * 128 floats <= BK * BM_PAD)
  constexpr int kStageRows = Tile::BN < 32 ? Tile::BN : 32;
  float* Cs = &Ws[0][0];
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int half = 0; half < Tile::BN / kStageRows; ++half) {
    __syncthreads();
#pragma unroll
    for (int j = 0; j < TN; ++j) {
      const int bl = ty * TN + j - half * kStageRows;
      if (bl >= 0 && bl < kStageRows)
        *reinterpret_cast<float4*>(&Cs[bl * kHeadDim + tx * 4]) =
            make_float4(t.acc[0][j], t.acc[1][j], t.acc[2][j], t.acc[3][j]);
    }
    __syncthreads();
    qup_epilogue(Cs, kStageRows, b0 + half * kStageRows, min(kStageRows, nb - half * kStageRows), L, l,
                 h, lane, warp, rope_cs, q);
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
  grid_launch_dependents();  // the scoring pass may start its key stream now
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
      // exact: the residual of a 4-bit rounding; two pieces are summed as they
      // are by the tensor core, three carry the residuals scaled by 16
      x[i] = P == 2 ? (x[i] - e4m3_value(c)) : (x[i] - e4m3_value(c)) * 16.0f;
    }
    const int row = p * kHeads + h;
    *reinterpret_cast<uint32_t*>(img + sw128_offset(row, lane * 4)) = word;
  }
  if (lane == 0) {
    wprime[idx] = fused_w[idx] * ldexpf(1.0f, -e);
    qexp[idx] = e;
  }
}

template <int TB>
fm_status launch_gemv(const float* W, int M, int K, int ksplit, const float* X, int64_t x_row_stride,
                      int64_t x_layer_stride, int rows_per_layer, int B, float* part, cudaStream_t st) {
  const int kslice = K / ksplit;
  const size_t smem = sizeof(float) * TB * (size_t)kslice;
  static PerDeviceOnce smem_set;
  int dev = 0;
  cudaGetDevice(&dev);
  if (fm_status e = smem_limit_once(smem_set, dev, gemv_kernel<TB>, 64 * 1024)) return e;
  const dim3 grid((M + kGemvWarps * kGemvRows - 1) / (kGemvWarps * kGemvRows), ksplit);
  const cudaError_t e = launch_overlapped(gemv_kernel<TB>, grid, dim3(kGemvWarps * 32), smem, st, W, M, K,
                                          kslice, X, x_row_stride, x_layer_stride, rows_per_layer, B, part);
  note_launch();
  return e == cudaSuccess ? FM_OK : record_cuda_error(e);
}

// The query chain for up to 8 rows: both projections as GEMVs bound by the
// weights' bytes, the RMSNorm between them, then RoPE and the Hadamard.
template <int TB>
fm_status launch_query_prep_gemv(fm_ctx* ctx, const float* hidden, const int64_t* positions, int B,
                                 float* q, float* fused_w, cudaStream_t st) {
  const fm_config& c = ctx->cfg;
  const int L = c.n_layers, R = c.q_lora_rank, HID = c.hidden;
  const int Md = L * (R + kHeads), Mu = L * kHeads * kHeadDim;
  // K slices of the down projection: enough CTAs for two per SM, slices of
  // at least 1024 columns (a multiple of 128) that fit the shared X slice
  int ks = 1;
  const int row_blocks = (Md + kGemvWarps * kGemvRows - 1) / (kGemvWarps * kGemvRows);
  while (ks * 2 <= ctx->splitk_max && HID % (ks * 2 * 128) == 0 && HID / (ks * 2) >= 1024 &&
         row_blocks * ks < gemv_ctas_per_sm(TB) * ctx->num_sms)
    ks *= 2;
  while (sizeof(float) * TB * (size_t)(HID / ks) > 64 * 1024 && ks * 2 <= ctx->splitk_max &&
         HID % (ks * 2 * 128) == 0)
    ks *= 2;
  if (sizeof(float) * TB * (size_t)(HID / ks) > 64 * 1024 || sizeof(float) * TB * (size_t)R > 64 * 1024)
    return FM_ERR_UNSUPPORTED;
  fm_status s = launch_gemv<TB>(ctx->w_down, Md, HID, ks, hidden, HID, 0, 0, B, ctx->a_part, st);
  if (s != FM_OK) return s;
  const float w_scale = (float)(1.0 / sqrt((double)c.head_dim * (double)c.n_heads));
  cudaError_t e = launch_overlapped(qnorm_kernel, dim3(B, L), dim3(kNormThreads), 0, st, (const float*)ctx->a_part,
                                    ks, StreamK{}, B, L, R, (int)c.n_heads, (const float*)ctx->q_norm,
                                    c.rms_eps, w_scale, positions, (const double*)ctx->rope_freq,
                                    c.rope_dim / 2, ctx->r_norm, fused_w, ctx->rope_cs, (float*)nullptr,
                                    (float*)nullptr);
  note_launch();
  if (e != cudaSuccess) return record_cuda_error(e);
  s = launch_gemv<TB>(ctx->w_up, Mu, R, 1, ctx->r_norm, (int64_t)L * R, R, kHeads * kHeadDim, B, ctx->up_part,
                      st);
  if (s != FM_OK) return s;
  const int warps = B * L * kHeads;
  e = launch_overlapped(qup_finish_kernel, dim3((warps + kThreads / 32 - 1) / (kThreads / 32)), dim3(kThreads), 0,
                        st, (const float*)ctx->up_part, StreamK{}, 1, (int64_t)B * Mu, B, L,
                        (const float*)ctx->rope_cs, q);
  note_launch();
  return e == cudaSuccess ? check_launch() : record_cuda_error(e);
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

// ------------------------------------------------ tensor maps (host)
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static bool tried = false;
  if (!tried) {
    tried = true;
    void* p = nullptr;
    cudaDriverEntryPointQueryResult qr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &qr) == cudaSuccess &&
        qr == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    else
      cudaGetLastError();
  }
  return fn;
}

// fp32 tensor of `rank` dims (innermost first), 128-byte swizzled boxes of
// 32 elements along dim 0; out-of-range elements of a box read as zero.
bool encode_f32_map(void* map, const float* base, int rank, const cuuint64_t* dims,
                    const cuuint64_t* strides_bytes, const cuuint32_t* box) {
  PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
  if (!enc) return false;
  const cuuint32_t elem[3] = {1, 1, 1};
  return enc(reinterpret_cast<CUtensorMap*>(map), CU_TENSOR_MAP_DATA_TYPE_FLOAT32, (cuuint32_t)rank,
             const_cast<float*>(base), dims, strides_bytes, box, elem, CU_TENSOR_MAP_INTERLEAVE_NONE,
             CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// W [rows, K] row-major, boxes of 32 x 128 rows.
bool encode_weight_map(void* map, const float* w, int rows, int K) {
  const cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)K * 4};
  const cuuint32_t box[2] = {(cuuint32_t)kTcBK, (cuuint32_t)kTcBM};
  return encode_f32_map(map, w, 2, dims, strides, box);
}

// X [n, layers, K] row-major (K innermost), boxes of 32 x 1 x bn.
bool encode_act_map(void* map, const float* x, int n, int layers, int K, int bn) {
  const cuuint64_t dims[3] = {(cuuint64_t)K, (cuuint64_t)layers, (cuuint64_t)n};
  const cuuint64_t strides[2] = {(cuuint64_t)K * 4, (cuuint64_t)K * layers * 4};
  const cuuint32_t box[3] = {(cuuint32_t)kTcBK, 1u, (cuuint32_t)bn};
  return encode_f32_map(map, x, 3, dims, strides, box);
}

void launch_split(const float* x, float* hi, float* lo, int64_t n, cudaStream_t st) {
  const int64_t g = (n + 255) / 256;
  split_tf32_kernel<<<(unsigned)(g < 4096 ? g : 4096), 256, 0, st>>>(x, hi, lo, n);
  note_launch();
}

template <int BN>
fm_status launch_tc_gemm_bn(fm_ctx* ctx, const void* wmap, const void* xh, const void* xl, const TcGemmArgs& a,
                            cudaStream_t st) {
  static PerDeviceOnce smem_set;
  constexpr uint32_t smem = TcCfg<BN>::kSmem;
  static_assert(smem <= 227u * 1024u, "shared memory");
  if (fm_status s = smem_limit_once(smem_set, ctx->device, tc_gemm_kernel<BN>, (int)smem)) return s;
  tc_gemm_kernel<BN><<<a.sk.G, kTcThreads, smem, st>>>(*reinterpret_cast<const CUtensorMap*>(wmap),
                                                       *reinterpret_cast<const CUtensorMap*>(xh),
                                                       *reinterpret_cast<const CUtensorMap*>(xl), a);
  note_launch();
  return check_launch();
}

// The stream-K partition of an M x N product over K for at most `G` CTAs,
// with no tile split over more than `max_slots` CTAs.
StreamK make_stream_k(int M, int N, int K, int bn, int G, int max_slots) {
  StreamK sk;
  sk.KB = K / kTcBK;
  sk.mtiles = (M + kTcBM - 1) / kTcBM;
  sk.bn = bn;
  const int tiles = sk.mtiles * ((N + bn - 1) / bn);
  sk.U = (int64_t)tiles * sk.KB;
  sk.G = (int)(sk.U < G ? sk.U : G);
  for (;;) {
    int worst = 0;
    for (int t = 0; t < tiles; ++t) worst = worst > sk.slots(t) ? worst : sk.slots(t);
    if (worst <= max_slots || sk.G == 1) break;
    --sk.G;
  }
  return sk;
}

// part[slot][n][m] for W (fp32 map: [M, K]) against X (split maps), stream-K.
fm_status launch_tc_gemm(fm_ctx* ctx, const void* wmap, const float* x_hi, const float* x_lo, int x_layers,
                         int M, int N, int K, int max_slots, int rows_per_layer, float* part, StreamK* sk_out,
                         cudaStream_t st) {
  const int bn = N <= 32 ? 32 : N <= 64 ? 64 : 128;
  alignas(64) unsigned char xh[128], xl[128];
  if (!encode_act_map(xh, x_hi, N, x_layers, K, bn) || !encode_act_map(xl, x_lo, N, x_layers, K, bn))
    return FM_ERR_CUDA;
  TcGemmArgs a;
  a.M = M; a.N = N; a.K = K;
  a.rows_per_layer = rows_per_layer;
  a.part = part;
  a.split_stride = (int64_t)N * M;
  a.err = ctx->d_err;
  a.sk = make_stream_k(M, N, K, bn, ctx->num_sms, max_slots);
  *sk_out = a.sk;
  switch (bn) {
    case 32: return launch_tc_gemm_bn<32>(ctx, wmap, xh, xl, a, st);
    case 64: return launch_tc_gemm_bn<64>(ctx, wmap, xh, xl, a, st);
    default: return launch_tc_gemm_bn<128>(ctx, wmap, xh, xl, a, st);
  }
}

// The query chain with both projections on the tensor cores (three-pass TF32).
fm_status launch_query_prep_tc(fm_ctx* ctx, const float* hidden, const int64_t* positions, int B,
                               float* q, float* fused_w, cudaStream_t st) {
  const fm_config& c = ctx->cfg;
  const int L = c.n_layers, R = c.q_lora_rank, HID = c.hidden;
  const int Md = L * (R + kHeads), Mu = L * kHeads * kHeadDim;
  // down projection (stream-K; its partials buffer holds splitk_max slots)
  launch_split(hidden, ctx->x_hi, ctx->x_lo, (int64_t)B * HID, st);
  StreamK sk_d, sk_u;
  fm_status s = launch_tc_gemm(ctx, ctx->wmaps[0], ctx->x_hi, ctx->x_lo, 1, Md, B, HID, ctx->splitk_max, 0,
                               ctx->a_part, &sk_d, st);
  if (s != FM_OK) return s;
  const float w_scale = (float)(1.0 / sqrt((double)c.head_dim * (double)c.n_heads));
  qnorm_kernel<<<dim3(B, L), kNormThreads, 0, st>>>(ctx->a_part, 0, sk_d, B, L, R, c.n_heads, ctx->q_norm,
                                                 c.rms_eps, w_scale, positions, ctx->rope_freq, c.rope_dim / 2,
                                                 ctx->r_norm, fused_w, ctx->rope_cs, ctx->r_hi, ctx->r_lo);
  note_launch();
  // up projection (stream-K; its partials buffer holds two slots)
  s = launch_tc_gemm(ctx, ctx->wmaps[1], ctx->r_hi, ctx->r_lo, L, Mu, B, R, 2, kHeads * kHeadDim, ctx->up_part,
                     &sk_u, st);
  if (s != FM_OK) return s;
  const int warps = B * L * kHeads;
  qup_finish_kernel<<<(warps + kThreads / 32 - 1) / (kThreads / 32), kThreads, 0, st>>>(
      ctx->up_part, sk_u, 0, (int64_t)B * Mu, B, L, ctx->rope_cs, q);
  note_launch();
  return check_launch();
}

}  // namespace

fm_status prepare_tc_weights(fm_ctx* ctx) {
  const fm_config& c = ctx->cfg;
  const int L = c.n_layers, R = c.q_lora_rank, HID = c.hidden;
  const int Md = L * (R + kHeads), Mu = L * kHeads * kHeadDim;
  ctx->tc_ok = encode_weight_map(ctx->wmaps[0], ctx->w_down, Md, HID) &&
               encode_weight_map(ctx->wmaps[1], ctx->w_up, Mu, R);
  return FM_OK;
}

fm_status launch_query_prep(fm_ctx* ctx, const float* hidden, const int64_t* positions, int B,
                            float* q, float* fused_w, cudaStream_t st) {
  // Past 8 rows the projections are bound by fp32 FMA on the CUDA cores and
  // the tensor-core path (three-pass TF32) takes over; up to 8 rows the
  // CUDA-core GEMVs are bound by the weight bytes, which both paths read once.
  if (ctx->tc_ok && B > 8) return launch_query_prep_tc(ctx, hidden, positions, B, q, fused_w, st);
  if (B == 1) return launch_query_prep_gemv<1>(ctx, hidden, positions, B, q, fused_w, st);
  if (B == 2) return launch_query_prep_gemv<2>(ctx, hidden, positions, B, q, fused_w, st);
  if (B <= 4) return launch_query_prep_gemv<4>(ctx, hidden, positions, B, q, fused_w, st);
  if (B <= 8) return launch_query_prep_gemv<8>(ctx, hidden, positions, B, q, fused_w, st);
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
  qnorm_kernel<<<dim3(B, c.n_layers), kNormThreads, 0, st>>>(
      ctx->a_part, ksplit, StreamK{}, B, c.n_layers, c.q_lora_rank, c.n_heads, ctx->q_norm, c.rms_eps,
      w_scale, positions, ctx->rope_freq, c.rope_dim / 2, ctx->r_norm, fused_w, ctx->rope_cs, nullptr,
      nullptr);
  note_launch();

  // one row block covers the batch up to 64 rows, so each head's wq_b rows
  // are read once per 64 rows
  if (B <= 8)
    launch_qup<1>(ctx, B, q, st);
  else if (B <= 16)
    launch_qup<2>(ctx, B, q, st);
  else if (B <= 32)
    launch_qup<4>(ctx, B, q, st);
  else
    launch_qup<8>(ctx, B, q, st);
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
