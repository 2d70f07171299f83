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
//    tile) units; each unit is scored for all L layers back to back (one
//    "item" per layer) so the ensemble stays in registers and one fp32 per
//    chunk is written;
//  * the keys go to the tensor cores as stored: kind::f8f6f4 MMA with A = the
//    128 e4m3 bytes of 128 records (M = 128 chunks, K = 128 dims) and B = the
//    query split into P e4m3 pieces per head (N = P*64), fp32 accumulators in
//    TMEM.  The per-chunk fp32 scale, the per-head power-of-two scale of the
//    pieces, relu, the head-weighted sum and the sigmoid run in the epilogue;
//  * the 132-byte records are not 16-byte aligned, so a tile is fetched with
//    one 1-D bulk copy (TMA engine) of 128 * 132 bytes and re-laid in place,
//    inside the same shared-memory stage, into the 128B-swizzled K-major
//    operand layout by four transform warps (every warp reads all its rows
//    before any warp writes: row r's destination [128r, 128r+128) overlaps
//    only rows <= r of the source).  The stage goes back to the key loader
//    when the MMA that read it retires, so the whole ring holds keys in
//    flight -- about 170 KB per SM;
//  * warp roles (16 warps): 0 key loader, 1 MMA issuer, 2 TMEM owner + query
//    loader, 4-7 transform, 8-11 and 12-15 two epilogue groups (one TMEM lane
//    quarter per warp, all 64 heads of a chunk row) that take alternate
//    units.  Each group owns half of the accumulator stages, so every stage's
//    phases are consumed in order by one group (a parity wait cannot tell
//    phases two apart).  Each item crosses four mbarrier hand-offs (copy
//    landed, operand ready, accumulator ready, accumulator free); every ring
//    index is advanced incrementally, and the epilogue reads each chunk's
//    scale from global memory (an L2 hit: the tile was fetched moments
//    earlier) instead of through another ring.
#include <cstdlib>

#include "fm_internal.cuh"

namespace fm {
namespace {

constexpr int kWarps = 16;
constexpr int kThreads = kWarps * 32;
constexpr int kRawBytes = kTile * kRecord;    // 16896
constexpr int kStageBytes = 17408;           // one key stage: 16896 B rounded to 1 KB
constexpr int kBarXform = 1;                 // named barrier id of the transform warps
constexpr int kWarpLoader = 0, kWarpMma = 1, kWarpQ = 2;
constexpr int kWarpXform0 = 4, kWarpEpi0 = 8;
constexpr uint32_t kTmemCols = 512;

struct Layout {
  int L, P, NR, NACC;
  uint32_t q_off, raw_off, wp_off, bar_off, misc_off, total;
};

__host__ __device__ inline Layout make_layout(int L, int P, int NR) {
  Layout s;
  s.L = L; s.P = P; s.NR = NR;
  s.NACC = (P == 3) ? 2 : 4;  // accumulator stages of P*64 TMEM columns (<= 512)
  uint32_t o = 0;
  s.q_off = o;    o += (uint32_t)L * P * kHeads * kHeadDim;           // multiple of 1024
  s.raw_off = o;  o += (uint32_t)NR * kStageBytes;                     // 1024-aligned stages
  s.wp_off = o;   o += 8u * (uint32_t)L * kHeads * 4;                 // per epilogue warp
  o = (o + 7u) & ~7u;
  s.bar_off = o;  o += (uint32_t)(3 * NR + 2 * s.NACC + 3) * 8;
  s.misc_off = o; o += 64;
  s.total = o + 1024;  // slack to align the base to 1024
  return s;
}

struct Bars {
  uint64_t *raw_full, *raw_empty, *a_full, *acc_full, *acc_empty, *q_full, *q_empty, *done;
};

// Position in a ring of n stages: the stage index and the parity of the
// stage's mbarrier phase for the current pass.  Advanced once per item, so no
// role ever divides by a runtime ring size (an integer division is a long
// dependent instruction sequence on the GPU, and it sat in every role's loop).
struct Ring {
  uint32_t stage, phase, n;
  __device__ explicit Ring(uint32_t n_) : stage(0), phase(0), n(n_) {}
  __device__ __forceinline__ void advance() {
    if (++stage == n) { stage = 0; phase ^= 1u; }
  }
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

// 32 lanes x 32 heads x P pieces of one accumulator stage, read in one load+wait.
template <int P>
struct HeadCols {
  uint32_t u[P][32];
  __device__ __forceinline__ void load(uint32_t col0) {
    if constexpr (P == 3)
      tmem_ld32x3_wait(col0, col0 + kHeads, col0 + 2 * kHeads, u[0], u[1], u[2]);
    else
      tmem_ld32x2_wait(col0, col0 + kHeads, u[0], u[1]);
  }
  __device__ __forceinline__ float at(int p, int i) const { return __uint_as_float(u[p][i]); }
};

// Head sum over 32 heads for one chunk row:
//   sum_h relu(d_h) * w'_h  with d_h = D0 + D1/16 (+ D2/256),  when s >= 0
//   sum_h relu(s d_h) * w'_h                                  otherwise
// where D_p are the accumulator columns of piece p and w' the head weights
// with the pieces' power-of-two scale folded in.
template <int P>
__device__ __forceinline__ float head_sum32(const HeadCols<P>& c, const float* __restrict__ w,
                                            float s, bool nonneg) {
  constexpr float kInv16 = 0.0625f, kInv256 = 0.00390625f;
  if (nonneg) {
    const uint64_t c16 = f2_pack(kInv16, kInv16), c256 = f2_pack(kInv256, kInv256);
    uint64_t acc_a = f2_pack(0.f, 0.f), acc_b = f2_pack(0.f, 0.f);
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      const uint64_t p0 = f2_pack(c.at(0, 2 * j), c.at(0, 2 * j + 1));
      const uint64_t p1 = f2_pack(c.at(1, 2 * j), c.at(1, 2 * j + 1));
      uint64_t d = f2_fma(p1, c16, p0);
      if constexpr (P == 3) d = f2_fma(f2_pack(c.at(2, 2 * j), c.at(2, 2 * j + 1)), c256, d);
      float dx, dy;
      f2_unpack(d, dx, dy);
      const float2 ww = *reinterpret_cast<const float2*>(w + 2 * j);
      const uint64_t rr = f2_pack(fmaxf(dx, 0.f), fmaxf(dy, 0.f));
      if (j & 1)
        acc_b = f2_fma(rr, f2_pack(ww.x, ww.y), acc_b);
      else
        acc_a = f2_fma(rr, f2_pack(ww.x, ww.y), acc_a);
    }
    float a0, a1, b0, b1;
    f2_unpack(acc_a, a0, a1);
    f2_unpack(acc_b, b0, b1);
    return (a0 + a1) + (b0 + b1);
  }
  float acc = 0.f;
  for (int i = 0; i < 32; ++i) {
    float d = fmaf(c.at(1, i), kInv16, c.at(0, i));
    if constexpr (P == 3) d = fmaf(c.at(2, i), kInv256, d);
    acc = fmaf(fmaxf(d * s, 0.f), w[i], acc);
  }
  return acc;
}

template <int P, bool DUMP>
__global__ void __launch_bounds__(kThreads, 1) score_kernel(ScoreArgs args, int NR) {
  extern __shared__ uint8_t smem_raw[];
  const Layout lay = make_layout(args.L, P, NR);
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  const int L = args.L;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  constexpr int NQ = P * kHeads;
  constexpr uint32_t kQLayerBytes = (uint32_t)P * kHeads * kHeadDim;

  uint8_t* sQ = smem + lay.q_off;
  uint8_t* sRaw = smem + lay.raw_off;
  float* sWp = reinterpret_cast<float*>(smem + lay.wp_off);
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + lay.bar_off);
  Bars B_;
  B_.raw_full = bar;                      B_.raw_empty = B_.raw_full + NR;
  B_.a_full = B_.raw_empty + NR;
  B_.acc_full = B_.a_full + NR;           B_.acc_empty = B_.acc_full + lay.NACC;
  B_.q_full = B_.acc_empty + lay.NACC;
  B_.q_empty = B_.q_full + 1;             B_.done = B_.q_empty + 1;
  uint32_t* sTmem = reinterpret_cast<uint32_t*>(smem + lay.misc_off);
  volatile int* sAbort = reinterpret_cast<volatile int*>(smem + lay.misc_off + 4);
  int* sRange = reinterpret_cast<int*>(smem + lay.misc_off + 8);  // b0, t0, count lo, count hi
  volatile int* sXStatus = reinterpret_cast<volatile int*>(smem + lay.misc_off + 24);

  // ---------------------------------------------------------------- setup
  if (threadIdx.x == 0) {
    for (int i = 0; i < NR; ++i) {
      mbar_init(&B_.raw_full[i], 1);   // bulk copy landed
      mbar_init(&B_.a_full[i], 4);     // re-laid in place (one arrival per transform warp)
      mbar_init(&B_.raw_empty[i], 1);  // the MMA that read the stage retired
    }
    for (int i = 0; i < lay.NACC; ++i) { mbar_init(&B_.acc_full[i], 1); mbar_init(&B_.acc_empty[i], 4); }
    mbar_init(B_.q_full, 1);
    mbar_init(B_.q_empty, 1);
    mbar_init(B_.done, 1);
    *sAbort = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == kWarpMma && lane == 0) {
    // this CTA's share of the valid units: rows contribute ceil(n_b / 128) tiles
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
      // a second walker runs `prefetch_units` units ahead and pulls their
      // records into L2, so far more bytes are in flight from HBM than the
      // shared-memory ring holds; the ring's bulk copies then hit L2
      UnitWalk pf = walk;
      pf.start(b_start, t_start, count);
      auto prefetch_unit = [&]() {
        const int nrem = min(kTile, pf.nv - pf.t * kTile);
        const uint32_t bytes = (uint32_t)((nrem + 3) & ~3) * kRecord;
        for (int l = 0; l < L; ++l)
          bulk_prefetch_l2(args.comp_k[l] + (int64_t)pf.b * args.row_stride +
                               (int64_t)pf.t * kRawBytes, bytes);
        pf.next();
      };
      for (int u = 0; u < args.prefetch_units && pf.valid(); ++u) prefetch_unit();
      uint32_t item = 0;
      Ring raw(NR);
      for (walk.start(b_start, t_start, count); walk.valid() && !*sAbort; walk.next()) {
        if (args.prefetch_units > 0 && pf.valid()) prefetch_unit();
        const int nrem = min(kTile, walk.nv - walk.t * kTile);
        const uint32_t bytes = (uint32_t)((nrem + 3) & ~3) * kRecord;
        bool ok = true;
        for (int l = 0; l < L; ++l) {
          ok = mbar_wait_bounded(&B_.raw_empty[raw.stage], raw.phase ^ 1, sAbort, args.err);
          if (!ok) break;
          mbar_arrive_expect_tx(&B_.raw_full[raw.stage], bytes);
          const uint8_t* src = args.comp_k[l] + (int64_t)walk.b * args.row_stride +
                               (int64_t)walk.t * kRawBytes;
          bulk_g2s(sRaw + (size_t)raw.stage * kStageBytes, src, bytes, &B_.raw_full[raw.stage]);
          ++item;
          raw.advance();
        }
        if (!ok) break;
      }
      // every copy issued must land before the CTA can exit (runs once: the
      // divisions here are off the hot loop)
      const uint32_t inflight = item < (uint32_t)NR ? item : (uint32_t)NR;
      for (uint32_t k = 0; k < inflight; ++k) {
        const uint32_t it = item - 1 - k;
        mbar_drain(&B_.raw_full[it % NR], (it / NR) & 1, args.err);
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
      if (loads > 0) mbar_drain(B_.q_full, (loads - 1) & 1, args.err);
    }
  } else if (warp == kWarpMma) {
    // ---------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_e4m3_f32(kTile, NQ);
      uint32_t item = 0, rows = 0;
      const uint32_t nacc_g = (uint32_t)lay.NACC / 2;
      Ring ast(NR), acc0(nacc_g), acc1(nacc_g);  // key stages; accumulator stages of group 0 / 1
      uint32_t unit = 0;                         // CTA-local unit index: unit & 1 = group
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
        const bool g1 = (unit & 1u) != 0;
        Ring acc = g1 ? acc1 : acc0;  // register copy, written back after the unit
        for (int l = 0; l < L; ++l) {
          const int as = ast.stage;
          const uint32_t ac = (g1 ? nacc_g : 0u) + acc.stage;
          ok = mbar_wait_bounded(&B_.a_full[as], ast.phase, sAbort, args.err) &&
               mbar_wait_bounded(&B_.acc_empty[ac], acc.phase ^ 1, sAbort, args.err);
          if (!ok) break;
          tc_fence_after();
          const uint32_t d = tmem_base + ac * (uint32_t)NQ;
          const uint32_t a0 = smem_u32(sRaw + (size_t)as * kStageBytes);
          const uint32_t b0 = smem_u32(sQ + (size_t)l * kQLayerBytes);
#pragma unroll
          for (int k = 0; k < kHeadDim / 32; ++k)
            umma_f8f6f4(d, sdesc_kmajor_sw128(a0 + 32u * k), sdesc_kmajor_sw128(b0 + 32u * k), idesc,
                        k > 0 ? 1u : 0u);
          umma_commit(&B_.raw_empty[as]);  // the key stage may be refilled
          umma_commit(&B_.acc_full[ac]);
          ++item;
          ast.advance();
          acc.advance();
        }
        if (g1) acc1 = acc; else acc0 = acc;
        ++unit;
        if (!ok) break;
        walk.next();
        if (!walk.valid() || walk.b != b) umma_commit(B_.q_empty);
      }
      if (item > 0) {  // every issued MMA and commit retired before TMEM and smem go away
        umma_commit(B_.done);
        mbar_drain(B_.done, 0, args.err);
      }
    }
  } else if (warp >= kWarpXform0 && warp < kWarpXform0 + 4) {
    // --------------------- transform: raw records -> MMA operand, in place
    // One leader thread waits on the copy barrier and the four warps follow it
    // through a named barrier, so the group always stops together.
    const int tw = warp - kWarpXform0;
    const bool leader = tw == 0 && lane == 0;
    Ring raw(NR);
    bool alive = true, stop = false;
    for (walk.start(b_start, t_start, count); walk.valid() && !stop; walk.next()) {
      for (int l = 0; l < L; ++l, raw.advance()) {
        if (leader) {
          alive = alive && mbar_wait_bounded(&B_.raw_full[raw.stage], raw.phase, sAbort, args.err);
          *sXStatus = alive ? 1 : 0;
        }
        __syncwarp();
        named_bar_sync(kBarXform, 128);
        if (*sXStatus == 0) { stop = true; break; }
        uint8_t* st = sRaw + (size_t)raw.stage * kStageBytes;
        uint32_t v[32];
#pragma unroll
        for (int rr = 0; rr < 32; ++rr)
          v[rr] = *reinterpret_cast<const uint32_t*>(st + (tw * 32 + rr) * kRecord + lane * 4);
        named_bar_sync(kBarXform, 128);  // every row read before any row is overwritten
#pragma unroll
        for (int rr = 0; rr < 32; ++rr)
          *reinterpret_cast<uint32_t*>(st + sw128_offset(tw * 32 + rr, lane * 4)) = v[rr];
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&B_.a_full[raw.stage]);
      }
    }
    if (leader && !alive) *sAbort = 1;
  } else if (warp >= kWarpEpi0) {
    // ------------------------------------------------------------ epilogue
    const int ew = warp - kWarpEpi0;  // 0..7
    const uint32_t group = (uint32_t)ew >> 2;
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;
    float* sWpw = sWp + ew * L * kHeads;
    const uint32_t lane_base = tmem_base + ((uint32_t)(quarter * 32) << 16);
    const uint32_t nacc_g = (uint32_t)lay.NACC / 2;
    Ring acc(nacc_g);  // this group's own accumulator stages
    int cur = -1;
    uint32_t unit = 0;
    for (walk.start(b_start, t_start, count); walk.valid(); walk.next(), ++unit) {
      if ((unit & 1u) != group) continue;  // the other group's unit
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
      // the chunk's scales, read from L2 while the accumulators are computed
      float sc[kMaxLayers];
#pragma unroll
      for (int l = 0; l < kMaxLayers; ++l) {
        sc[l] = 0.f;
        if (l < L && valid)
          sc[l] = __ldg(reinterpret_cast<const float*>(args.comp_k[l] + (int64_t)b * args.row_stride +
                                                       (int64_t)n * kRecord + kHeadDim));
      }
      float ens = 0.f;
      bool ok = true;
      for (int l = 0; l < L; ++l, acc.advance()) {
        const float s = l == 0 ? sc[0] : l == 1 ? sc[1] : l == 2 ? sc[2] : sc[3];
        const uint32_t slot = group * nacc_g + acc.stage;
        ok = mbar_wait_bounded(&B_.acc_full[slot], acc.phase, sAbort, args.err);
        if (!ok) break;
        tc_fence_after();
        const bool nonneg = __all_sync(0xffffffffu, !(s < 0.f));
        const uint32_t col = lane_base + slot * (uint32_t)NQ;
        const float* w = sWpw + l * kHeads;
        HeadCols<P> c;
        c.load(col);
        if constexpr (DUMP) {
          if (b == args.dbg_b && walk.t == args.dbg_t && l == args.dbg_layer)
            for (int p = 0; p < P; ++p)
              for (int i = 0; i < 32; ++i) args.dbg_out[(size_t)r * NQ + p * kHeads + i] = c.at(p, i);
        }
        float part = head_sum32<P>(c, w, s, nonneg);
        c.load(col + 32);
        // the accumulator stage is free once this warp holds all its columns
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&B_.acc_empty[slot]);
        if constexpr (DUMP) {
          if (b == args.dbg_b && walk.t == args.dbg_t && l == args.dbg_layer)
            for (int p = 0; p < P; ++p)
              for (int i = 0; i < 32; ++i)
                args.dbg_out[(size_t)r * NQ + p * kHeads + 32 + i] = c.at(p, i);
        }
        part += head_sum32<P>(c, w + 32, s, nonneg);
        const float logit = nonneg ? part * s : part;
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
    const int64_t gt = (int64_t)blockIdx.x * 256 + et, gs = (int64_t)gridDim.x * 256;
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

template <int P, bool DUMP>
fm_status launch_score_p(fm_ctx* ctx, const ScoreArgs& a, cudaStream_t st) {
  static int configured_dev = -1;
  int max_smem = 0;
  if (cudaDeviceGetAttribute(&max_smem, cudaDevAttrMaxSharedMemoryPerBlockOptin, ctx->device) !=
      cudaSuccess)
    return check_launch();
  // deepest key ring that fits: every stage is keys in flight
  int NR = 16;
  if (const char* e = getenv("FM_RAW_STAGES")) NR = atoi(e) < 2 ? 2 : atoi(e);
  Layout lay = make_layout(a.L, P, NR);
  while (lay.total > (uint32_t)max_smem && NR > 2) {
    --NR;
    lay = make_layout(a.L, P, NR);
  }
  if (lay.total > (uint32_t)max_smem) return FM_ERR_UNSUPPORTED;
  if (configured_dev != ctx->device) {
    if (cudaFuncSetAttribute(score_kernel<P, DUMP>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             max_smem) != cudaSuccess)
      return check_launch();
    configured_dev = ctx->device;
  }
  const int64_t units = (int64_t)a.B * ((a.N + kTile - 1) / kTile);  // upper bound
  int grid = ctx->num_sms;
  if (units < grid) grid = (int)(units > 0 ? units : 1);
  score_kernel<P, DUMP><<<grid, kThreads, lay.total, st>>>(a, NR);
  note_launch();
  return check_launch();
}

}  // namespace

fm_status launch_score(fm_ctx* ctx, const ScoreArgs& a, cudaStream_t st) {
  if (a.dbg_out)
    return ctx->cfg.q_pieces == 3 ? launch_score_p<3, true>(ctx, a, st)
                                  : launch_score_p<2, true>(ctx, a, st);
  return ctx->cfg.q_pieces == 3 ? launch_score_p<3, false>(ctx, a, st)
                                : launch_score_p<2, false>(ctx, a, st);
}

}  // namespace fm
