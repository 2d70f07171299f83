// score_tc.cu -- the chunk-scoring pass (README "Architecture", score line):
//
//   score[l,b,n] = sigmoid( sum_h relu(k[l,b,n] . q[b,l,h]) * fused_w[b,l,h] )
//   k = e4m3(record[0:128]) * f32le(record[128:132])      ("compressed_k format")
//
// fused with the cross-layer ensemble ("Joint checkpoint + ensemble") and the
// threshold keep rule (toy decode loop, "sigmoid > thresh").
//
// Design (sm_100a):
//  * one persistent CTA per SM walks a contiguous range of (row, 128-chunk
//    tile) units; each unit is scored for all L layers back to back so the
//    ensemble stays in registers and one fp32 per chunk is written;
//  * the keys go to the tensor cores as stored: kind::f8f6f4 MMA with A = the
//    128 e4m3 bytes of 128 records (M = 128 chunks, K = 128 dims) and B = the
//    query split into P e4m3 pieces per head (N = P*64), fp32 accumulators in
//    TMEM.  The per-chunk fp32 scale, the per-head power-of-two scale of the
//    pieces, relu, the head-weighted sum and the sigmoid run in the epilogue;
//  * the 132-byte records are not 16-byte aligned, so a tile is fetched with
//    one 1-D bulk copy (TMA engine) of 128 * 132 bytes and re-laid into the
//    128B-swizzled K-major operand layout by four transform warps;
//  * warp roles: 0 key loader, 1 MMA issuer, 2 TMEM owner + query loader,
//    4-7 transform, 8-11 epilogue (one TMEM lane quarter each).
#include "fm_internal.cuh"

namespace fm {
namespace {

constexpr int kWarps = 12;
constexpr int kThreads = kWarps * 32;
constexpr int kRawBytes = kTile * kRecord;    // 16896
constexpr int kABytes = kTile * kHeadDim;     // 16384
constexpr int kWarpLoader = 0, kWarpMma = 1, kWarpQ = 2;
constexpr int kWarpXform0 = 4, kWarpEpi0 = 8;
constexpr uint32_t kTmemCols = 512;

struct Layout {
  int L, P, NA, NR, NACC, NSC;
  uint32_t q_off, a_off, raw_off, sc_off, wp_off, bar_off, misc_off, total;
};

__host__ __device__ inline Layout make_layout(int L, int P, int NA, int NR) {
  Layout s;
  s.L = L; s.P = P; s.NA = NA; s.NR = NR;
  s.NACC = (P == 3) ? 2 : 4;
  s.NSC = NA + s.NACC;
  uint32_t o = 0;
  s.q_off = o;   o += (uint32_t)L * P * kHeads * kHeadDim;           // multiple of 1024
  s.a_off = o;   o += (uint32_t)NA * kABytes;                         // 1024-aligned tiles
  s.raw_off = o; o += (uint32_t)NR * kRawBytes;                       // 16-aligned
  s.sc_off = o;  o += (uint32_t)s.NSC * kTile * 4;
  s.wp_off = o;  o += 4u * (uint32_t)L * kHeads * 4;  // one copy per epilogue warp
  o = (o + 7u) & ~7u;
  s.bar_off = o; o += (uint32_t)(2 * NR + 2 * NA + 2 * s.NACC + 2 * s.NSC + 2) * 8;
  s.misc_off = o; o += 64;
  s.total = o + 1024;  // slack to align the base to 1024
  return s;
}

struct Bars {
  uint64_t *raw_full, *raw_empty, *a_full, *a_empty, *acc_full, *acc_empty, *sc_full, *sc_empty,
      *q_full, *q_empty;
};

// Walks this CTA's contiguous range of valid (row, tile) units.
struct UnitWalk {
  const int32_t* n_valid;
  int N, B;
  int b, t, nv, tiles;
  int64_t left;
  __device__ int nvalid_of(int row) const {
    int v = n_valid ? __ldg(n_valid + row) : N;
    return max(0, min(v, N));
  }
  __device__ void start(int b0, int t0, int64_t count) {
    b = b0; t = t0; left = count;
    if (left > 0) { nv = nvalid_of(b); tiles = (nv + kTile - 1) / kTile; }
  }
  __device__ bool valid() const { return left > 0; }
  __device__ void next() {
    --left;
    if (left <= 0) return;
    if (++t >= tiles) {
      t = 0;
      do { ++b; nv = nvalid_of(b); tiles = (nv + kTile - 1) / kTile; } while (tiles == 0);
    }
  }
};

template <int P>
__global__ void __launch_bounds__(kThreads, 1) score_kernel(ScoreArgs args, int NA, int NR) {
  extern __shared__ uint8_t smem_raw[];
  const Layout lay = make_layout(args.L, P, NA, NR);
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  const int L = args.L;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  constexpr int NQ = P * kHeads;
  constexpr uint32_t kQLayerBytes = (uint32_t)P * kHeads * kHeadDim;

  uint8_t* sQ = smem + lay.q_off;
  uint8_t* sA = smem + lay.a_off;
  uint8_t* sRaw = smem + lay.raw_off;
  float* sSc = reinterpret_cast<float*>(smem + lay.sc_off);
  float* sWp = reinterpret_cast<float*>(smem + lay.wp_off);
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + lay.bar_off);
  Bars B_;
  B_.raw_full = bar;                B_.raw_empty = B_.raw_full + NR;
  B_.a_full = B_.raw_empty + NR;    B_.a_empty = B_.a_full + NA;
  B_.acc_full = B_.a_empty + NA;    B_.acc_empty = B_.acc_full + lay.NACC;
  B_.sc_full = B_.acc_empty + lay.NACC; B_.sc_empty = B_.sc_full + lay.NSC;
  B_.q_full = B_.sc_empty + lay.NSC;   B_.q_empty = B_.q_full + 1;
  uint32_t* sTmem = reinterpret_cast<uint32_t*>(smem + lay.misc_off);
  volatile int* sAbort = reinterpret_cast<volatile int*>(smem + lay.misc_off + 4);
  int* sRange = reinterpret_cast<int*>(smem + lay.misc_off + 8);  // b0, t0, count lo, count hi

  // ---------------------------------------------------------------- setup
  if (threadIdx.x == 0) {
    for (int i = 0; i < NR; ++i) { mbar_init(&B_.raw_full[i], 1); mbar_init(&B_.raw_empty[i], 4); }
    for (int i = 0; i < NA; ++i) { mbar_init(&B_.a_full[i], 4); mbar_init(&B_.a_empty[i], 1); }
    for (int i = 0; i < lay.NACC; ++i) { mbar_init(&B_.acc_full[i], 1); mbar_init(&B_.acc_empty[i], 4); }
    for (int i = 0; i < lay.NSC; ++i) { mbar_init(&B_.sc_full[i], 4); mbar_init(&B_.sc_empty[i], 4); }
    mbar_init(B_.q_full, 1);
    mbar_init(B_.q_empty, 1);
    *sAbort = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == kWarpMma) {
    // this CTA's share of the valid units: rows contribute ceil(n_b / 128) tiles
    if (lane == 0) {
      int64_t total = 0;
      for (int b = 0; b < args.B; ++b) {
        int v = args.n_valid ? __ldg(args.n_valid + b) : args.N;
        v = max(0, min(v, args.N));
        total += (v + kTile - 1) / kTile;
      }
      const int64_t u0 = total * blockIdx.x / gridDim.x;
      const int64_t u1 = total * (blockIdx.x + 1) / gridDim.x;
      int64_t acc = 0;
      int b0 = 0, t0 = 0;
      for (int b = 0; b < args.B; ++b) {
        int v = args.n_valid ? __ldg(args.n_valid + b) : args.N;
        v = max(0, min(v, args.N));
        const int tiles = (v + kTile - 1) / kTile;
        if (acc + tiles > u0) { b0 = b; t0 = (int)(u0 - acc); break; }
        acc += tiles;
      }
      sRange[0] = b0; sRange[1] = t0;
      sRange[2] = (int)((u1 - u0) & 0xffffffff); sRange[3] = (int)((u1 - u0) >> 32);
    }
  }
  if (warp == kWarpQ) {
    tmem_alloc(sTmem, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *sTmem;
  const int b_start = sRange[0], t_start = sRange[1];
  const int64_t count = (int64_t)(uint32_t)sRange[2] | ((int64_t)sRange[3] << 32);

  UnitWalk walk;
  walk.n_valid = args.n_valid; walk.N = args.N; walk.B = args.B;

  if (warp == kWarpLoader) {
    // ------------------------------------------------------- key tile loader
    if (lane == 0) {
      const uint64_t policy = policy_evict_first();
      uint32_t item = 0;
      for (walk.start(b_start, t_start, count); walk.valid() && !*sAbort; walk.next()) {
        const int nrem = min(kTile, walk.nv - walk.t * kTile);
        const uint32_t bytes = (uint32_t)((nrem + 3) & ~3) * kRecord;
        for (int l = 0; l < L; ++l, ++item) {
          const int rs = item % NR;
          if (!mbar_wait_bounded(&B_.raw_empty[rs], ((item / NR) & 1) ^ 1, sAbort, args.err)) break;
          mbar_arrive_expect_tx(&B_.raw_full[rs], bytes);
          const uint8_t* src = args.comp_k[l] + (int64_t)walk.b * args.row_stride +
                               (int64_t)walk.t * kRawBytes;
          bulk_g2s_hint(sRaw + (size_t)rs * kRawBytes, src, bytes, &B_.raw_full[rs], policy);
        }
      }
      // let copies still in flight land before the CTA can exit
      const uint32_t inflight = item < (uint32_t)NR ? item : (uint32_t)NR;
      for (uint32_t k = 0; k < inflight; ++k) {
        const uint32_t it = item - 1 - k;
        mbar_wait_bounded(&B_.raw_full[it % NR], (it / NR) & 1, sAbort, args.err, 100000000ull);
      }
    }
  } else if (warp == kWarpQ) {
    // ------------------------------------------------ query operand loader
    if (lane == 0) {
      int cur = -1;
      uint32_t loads = 0;
      for (walk.start(b_start, t_start, count); walk.valid() && !*sAbort; walk.next()) {
        if (walk.b == cur) continue;
        if (loads > 0 && !mbar_wait_bounded(B_.q_empty, (loads - 1) & 1, sAbort, args.err)) break;
        mbar_arrive_expect_tx(B_.q_full, (uint32_t)L * kQLayerBytes);
        for (int l = 0; l < L; ++l)
          bulk_g2s(sQ + (size_t)l * kQLayerBytes,
                   args.qpack + ((size_t)walk.b * L + l) * kQLayerBytes, kQLayerBytes, B_.q_full);
        cur = walk.b;
        ++loads;
      }
      if (loads > 0)
        mbar_wait_bounded(B_.q_full, (loads - 1) & 1, sAbort, args.err, 100000000ull);
    }
  } else if (warp == kWarpMma) {
    // ---------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_e4m3_f32(kTile, NQ);
      uint32_t item = 0, rows = 0;
      int cur = -1;
      bool ok = true;
      walk.start(b_start, t_start, count);
      while (ok && walk.valid() && !*sAbort) {
        const int b = walk.b;
        if (b != cur) {
          if (!mbar_wait_bounded(B_.q_full, rows & 1, sAbort, args.err)) break;
          ++rows;
          cur = b;
        }
        for (int l = 0; l < L && ok; ++l, ++item) {
          const int as = item % NA, ac = item % lay.NACC;
          ok = mbar_wait_bounded(&B_.a_full[as], (item / NA) & 1, sAbort, args.err) &&
               mbar_wait_bounded(&B_.acc_empty[ac], ((item / lay.NACC) & 1) ^ 1, sAbort, args.err);
          if (!ok) break;
          tc_fence_after();
          const uint32_t d = tmem_base + (uint32_t)(ac * NQ);
          const uint32_t a0 = smem_u32(sA + (size_t)as * kABytes);
          const uint32_t b0 = smem_u32(sQ + (size_t)l * kQLayerBytes);
#pragma unroll
          for (int k = 0; k < kHeadDim / 32; ++k)
            umma_f8f6f4(d, sdesc_kmajor_sw128(a0 + 32u * k), sdesc_kmajor_sw128(b0 + 32u * k), idesc,
                        k > 0 ? 1u : 0u);
          umma_commit(&B_.a_empty[as]);
          umma_commit(&B_.acc_full[ac]);
        }
        if (!ok) break;
        walk.next();
        if (!walk.valid() || walk.b != b) umma_commit(B_.q_empty);
      }
      if (item > 0) {  // all issued MMAs retired before TMEM is released
        const uint32_t it = item - 1;
        mbar_wait_bounded(&B_.acc_full[it % lay.NACC], (it / lay.NACC) & 1, sAbort, args.err,
                          100000000ull);
      }
    }
  } else if (warp >= kWarpXform0 && warp < kWarpXform0 + 4) {
    // ------------------------------- transform: raw records -> MMA operand
    const int tw = warp - kWarpXform0;
    uint32_t item = 0;
    for (walk.start(b_start, t_start, count); walk.valid(); walk.next()) {
      bool ok = true;
      for (int l = 0; l < L; ++l, ++item) {
        const int rs = item % NR, as = item % NA, sc = item % lay.NSC;
        ok = mbar_wait_bounded(&B_.raw_full[rs], (item / NR) & 1, sAbort, args.err) &&
             mbar_wait_bounded(&B_.a_empty[as], ((item / NA) & 1) ^ 1, sAbort, args.err) &&
             mbar_wait_bounded(&B_.sc_empty[sc], ((item / lay.NSC) & 1) ^ 1, sAbort, args.err);
        if (!ok) break;
        const uint8_t* raw = sRaw + (size_t)rs * kRawBytes;
        uint8_t* A = sA + (size_t)as * kABytes;
        uint32_t v[32];
#pragma unroll
        for (int rr = 0; rr < 32; ++rr) {
          const int r = tw * 32 + rr;
          v[rr] = *reinterpret_cast<const uint32_t*>(raw + r * kRecord + lane * 4);
        }
#pragma unroll
        for (int rr = 0; rr < 32; ++rr) {
          const int r = tw * 32 + rr;
          *reinterpret_cast<uint32_t*>(A + sw128_offset(r, lane * 4)) = v[rr];
        }
        const int rme = tw * 32 + lane;
        sSc[sc * kTile + rme] = *reinterpret_cast<const float*>(raw + rme * kRecord + kHeadDim);
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&B_.raw_empty[rs]);
          mbar_arrive(&B_.a_full[as]);
          mbar_arrive(&B_.sc_full[sc]);
        }
      }
      if (!ok) break;
    }
  } else if (warp >= kWarpEpi0) {
    // ------------------------------------------------------------ epilogue
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;
    float* sWpw = sWp + (warp - kWarpEpi0) * L * kHeads;
    const uint32_t lane_base = tmem_base + ((uint32_t)(quarter * 32) << 16);
    uint32_t item = 0;
    int cur = -1;
    const float inv16 = 0.0625f, inv256 = 0.00390625f;
    for (walk.start(b_start, t_start, count); walk.valid(); walk.next()) {
      const int b = walk.b;
      if (b != cur) {  // this warp's private copy of the row's head weights
        __syncwarp();
        for (int i = lane; i < L * kHeads; i += 32)
          sWpw[i] = __ldg(args.wprime + (size_t)b * L * kHeads + i);
        __syncwarp();
        cur = b;
      }
      const int n = walk.t * kTile + r;
      const bool valid = n < walk.nv;
      const bool in_row = n < args.N;
      float ens = 0.f;
      bool ok = true;
      for (int l = 0; l < L; ++l, ++item) {
        const int ac = item % lay.NACC, sc = item % lay.NSC;
        ok = mbar_wait_bounded(&B_.sc_full[sc], (item / lay.NSC) & 1, sAbort, args.err);
        if (!ok) break;
        const float s = sSc[sc * kTile + r];
        __syncwarp();
        if (lane == 0) mbar_arrive(&B_.sc_empty[sc]);
        ok = mbar_wait_bounded(&B_.acc_full[ac], (item / lay.NACC) & 1, sAbort, args.err);
        if (!ok) break;
        tc_fence_after();
        const bool nonneg = __all_sync(0xffffffffu, !(s < 0.f));
        const bool dump = args.dbg_out && b == args.dbg_b && walk.t == args.dbg_t &&
                          l == args.dbg_layer;
        const float* wp = sWpw + l * kHeads;
        float acc0 = 0.f, acc1 = 0.f, acc2 = 0.f, acc3 = 0.f;
#pragma unroll
        for (int hc = 0; hc < 2; ++hc) {
          float v0[32], v1[32], v2[32];
          const uint32_t col = lane_base + (uint32_t)(ac * NQ + hc * 32);
          tmem_ld_32cols(col, v0);
          tmem_ld_32cols(col + kHeads, v1);
          if constexpr (P == 3) tmem_ld_32cols(col + 2 * kHeads, v2);
          tmem_ld_wait();
          if (dump) {
            for (int i = 0; i < 32; ++i) {
              args.dbg_out[r * NQ + hc * 32 + i] = v0[i];
              args.dbg_out[r * NQ + kHeads + hc * 32 + i] = v1[i];
              if constexpr (P == 3) args.dbg_out[r * NQ + 2 * kHeads + hc * 32 + i] = v2[i];
            }
          }
          if (nonneg) {
#pragma unroll
            for (int i = 0; i < 32; i += 4) {
              float d0 = fmaf(v1[i + 0], inv16, v0[i + 0]);
              float d1 = fmaf(v1[i + 1], inv16, v0[i + 1]);
              float d2 = fmaf(v1[i + 2], inv16, v0[i + 2]);
              float d3 = fmaf(v1[i + 3], inv16, v0[i + 3]);
              if constexpr (P == 3) {
                d0 = fmaf(v2[i + 0], inv256, d0);
                d1 = fmaf(v2[i + 1], inv256, d1);
                d2 = fmaf(v2[i + 2], inv256, d2);
                d3 = fmaf(v2[i + 3], inv256, d3);
              }
              acc0 = fmaf(fmaxf(d0, 0.f), wp[hc * 32 + i + 0], acc0);
              acc1 = fmaf(fmaxf(d1, 0.f), wp[hc * 32 + i + 1], acc1);
              acc2 = fmaf(fmaxf(d2, 0.f), wp[hc * 32 + i + 2], acc2);
              acc3 = fmaf(fmaxf(d3, 0.f), wp[hc * 32 + i + 3], acc3);
            }
          } else {
#pragma unroll
            for (int i = 0; i < 32; ++i) {
              float d = fmaf(v1[i], inv16, v0[i]);
              if constexpr (P == 3) d = fmaf(v2[i], inv256, d);
              acc0 = fmaf(fmaxf(d * s, 0.f), wp[hc * 32 + i], acc0);
            }
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&B_.acc_empty[ac]);
        float logit = (acc0 + acc1) + (acc2 + acc3);
        if (nonneg) logit *= s;
        float score = 1.0f / (1.0f + __expf(-logit));
        if (!valid) score = 0.f;
        if (args.scores && in_row) args.scores[((size_t)l * args.B + b) * args.N + n] = score;
        ens = (args.mode == FM_ENSEMBLE_MAX) ? (l == 0 ? score : fmaxf(ens, score)) : ens + score;
      }
      if (!ok) break;
      if (args.mode != FM_ENSEMBLE_MAX) ens = ens / (float)L;
      if (!valid) ens = 0.f;
      if (in_row) {
        if (args.ens) args.ens[(size_t)b * args.N + n] = ens;
        if (args.keep_thr) args.keep_thr[(size_t)b * args.N + n] = (valid && ens > args.thr) ? 1 : 0;
      }
    }
    // zero the tail of every row that no tile covers: [128 * ceil(n_b / 128), N)
    const int et = threadIdx.x - kWarpEpi0 * 32;
    const int64_t gt = (int64_t)blockIdx.x * 128 + et, gs = (int64_t)gridDim.x * 128;
    for (int b = 0; b < args.B; ++b) {
      const int v = walk.nvalid_of(b);
      const int from = min(args.N, ((v + kTile - 1) / kTile) * kTile);
      for (int64_t n = from + gt; n < args.N; n += gs) {
        if (args.scores)
          for (int l = 0; l < L; ++l) args.scores[((size_t)l * args.B + b) * args.N + n] = 0.f;
        if (args.ens) args.ens[(size_t)b * args.N + n] = 0.f;
        if (args.keep_thr) args.keep_thr[(size_t)b * args.N + n] = 0;
      }
    }
  }

  // ------------------------------------------------------------- teardown
  tc_fence_before();
  __syncthreads();
  if (warp == kWarpQ) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

template <int P>
fm_status launch_score_p(fm_ctx* ctx, const ScoreArgs& a, cudaStream_t st) {
  static int configured_dev = -1;
  int max_smem = 0;
  if (cudaDeviceGetAttribute(&max_smem, cudaDevAttrMaxSharedMemoryPerBlockOptin, ctx->device) !=
      cudaSuccess)
    return check_launch();
  int NA = 4, NR = 4;
  Layout lay = make_layout(a.L, P, NA, NR);
  while (lay.total > (uint32_t)max_smem && NA > 2) {
    --NA; --NR;
    lay = make_layout(a.L, P, NA, NR);
  }
  if (lay.total > (uint32_t)max_smem) return FM_ERR_UNSUPPORTED;
  if (configured_dev != ctx->device) {
    if (cudaFuncSetAttribute(score_kernel<P>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             max_smem) != cudaSuccess)
      return check_launch();
    configured_dev = ctx->device;
  }
  int64_t units = 0;  // upper bound (exact count needs n_valid on the host)
  units = (int64_t)a.B * ((a.N + kTile - 1) / kTile);
  int grid = ctx->num_sms;
  if (units < grid) grid = (int)(units > 0 ? units : 1);
  score_kernel<P><<<grid, kThreads, lay.total, st>>>(a, NA, NR);
  note_launch();
  return check_launch();
}

}  // namespace

fm_status launch_score(fm_ctx* ctx, const ScoreArgs& a, cudaStream_t st) {
  return ctx->cfg.q_pieces == 3 ? launch_score_p<3>(ctx, a, st) : launch_score_p<2>(ctx, a, st);
}

}  // namespace fm
