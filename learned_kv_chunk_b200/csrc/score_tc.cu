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
//  * warp roles (16 warps): 0 key loader, 1 MMA issuer, 2 TMEM owner + query
//    loader, 4-7 transform, 8-11 epilogue group A (heads 0-31), 12-15 epilogue
//    group B (heads 32-63).  Warps w and w+4 of the epilogue read the same TMEM
//    lane quarter; group B hands its partial head sum to group A through
//    shared memory, and group A finishes the chunk (sigmoid, ensemble, stores).
#include <cstdlib>

#include "fm_internal.cuh"

namespace fm {
namespace {

constexpr int kWarps = 16;
constexpr int kThreads = kWarps * 32;
constexpr int kRawBytes = kTile * kRecord;    // 16896
constexpr int kABytes = kTile * kHeadDim;     // 16384
constexpr int kWarpLoader = 0, kWarpMma = 1, kWarpQ = 2;
constexpr int kWarpXform0 = 4, kWarpEpi0 = 8;
constexpr int kHalfHeads = kHeads / 2;
constexpr uint32_t kTmemCols = 512;

struct Layout {
  int L, P, NA, NR, NACC, NSC, NPART;
  uint32_t q_off, a_off, raw_off, sc_off, part_off, wp_off, bar_off, misc_off, total;
};

__host__ __device__ inline Layout make_layout(int L, int P, int NA, int NR) {
  Layout s;
  s.L = L; s.P = P; s.NA = NA; s.NR = NR;
  s.NACC = (P == 3) ? 2 : 4;  // accumulator stages of P*64 TMEM columns (<= 512)
  s.NSC = NA + s.NACC;
  s.NPART = 4;                // group B -> group A partial-sum slots
  uint32_t o = 0;
  s.q_off = o;    o += (uint32_t)L * P * kHeads * kHeadDim;           // multiple of 1024
  s.a_off = o;    o += (uint32_t)NA * kABytes;                         // 1024-aligned tiles
  s.raw_off = o;  o += (uint32_t)NR * kRawBytes;                       // 16-aligned
  s.sc_off = o;   o += (uint32_t)s.NSC * kTile * 4;
  s.part_off = o; o += (uint32_t)s.NPART * kTile * 4;
  s.wp_off = o;   o += 8u * (uint32_t)L * kHalfHeads * 4;             // per epilogue warp
  o = (o + 7u) & ~7u;
  s.bar_off = o;  o += (uint32_t)(2 * NR + 2 * NA + 2 * s.NACC + 2 * s.NPART + 2 * s.NSC + 3) * 8;
  s.misc_off = o; o += 64;
  s.total = o + 1024;  // slack to align the base to 1024
  return s;
}

struct Bars {
  uint64_t *raw_full, *raw_empty, *a_full, *a_empty, *acc_full, *acc_empty, *part_full, *part_empty,
      *sc_full, *sc_empty, *q_full, *q_empty, *done;
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

// One epilogue warp's accumulator columns for its 32 heads: P pieces x 32
// fp32 per chunk row, read from TMEM in one load+wait.
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

// Partial head sum of one epilogue warp over its 32 heads for one chunk row:
//   sum_h relu(d_h) * w'_h  with d_h = D0 + D1/16 (+ D2/256),  when s >= 0
//   sum_h relu(s d_h) * w'_h                                  otherwise
// where D_p are the accumulator columns of piece p and w' the head weights
// with the pieces' power-of-two scale folded in.
template <int P>
__device__ __forceinline__ float head_partial(const HeadCols<P>& c, const float* __restrict__ w,
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
  float* sPart = reinterpret_cast<float*>(smem + lay.part_off);
  float* sWp = reinterpret_cast<float*>(smem + lay.wp_off);
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + lay.bar_off);
  Bars B_;
  B_.raw_full = bar;                      B_.raw_empty = B_.raw_full + NR;
  B_.a_full = B_.raw_empty + NR;          B_.a_empty = B_.a_full + NA;
  B_.acc_full = B_.a_empty + NA;          B_.acc_empty = B_.acc_full + lay.NACC;
  B_.part_full = B_.acc_empty + lay.NACC; B_.part_empty = B_.part_full + lay.NPART;
  B_.sc_full = B_.part_empty + lay.NPART;
  B_.sc_empty = B_.sc_full + lay.NSC;     B_.q_full = B_.sc_empty + lay.NSC;
  B_.q_empty = B_.q_full + 1;             B_.done = B_.q_empty + 1;
  uint32_t* sTmem = reinterpret_cast<uint32_t*>(smem + lay.misc_off);
  volatile int* sAbort = reinterpret_cast<volatile int*>(smem + lay.misc_off + 4);
  int* sRange = reinterpret_cast<int*>(smem + lay.misc_off + 8);  // b0, t0, count lo, count hi

  // ---------------------------------------------------------------- setup
  if (threadIdx.x == 0) {
    for (int i = 0; i < NR; ++i) { mbar_init(&B_.raw_full[i], 1); mbar_init(&B_.raw_empty[i], 4); }
    for (int i = 0; i < NA; ++i) { mbar_init(&B_.a_full[i], 4); mbar_init(&B_.a_empty[i], 1); }
    for (int i = 0; i < lay.NACC; ++i) { mbar_init(&B_.acc_full[i], 1); mbar_init(&B_.acc_empty[i], 8); }
    for (int i = 0; i < lay.NPART; ++i) { mbar_init(&B_.part_full[i], 4); mbar_init(&B_.part_empty[i], 4); }
    for (int i = 0; i < lay.NSC; ++i) { mbar_init(&B_.sc_full[i], 4); mbar_init(&B_.sc_empty[i], 8); }
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
      const uint64_t policy = policy_evict_first();
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
        if (pf.valid()) prefetch_unit();
        const int nrem = min(kTile, walk.nv - walk.t * kTile);
        const uint32_t bytes = (uint32_t)((nrem + 3) & ~3) * kRecord;
        bool ok = true;
        for (int l = 0; l < L; ++l) {
          ok = mbar_wait_bounded(&B_.raw_empty[raw.stage], raw.phase ^ 1, sAbort, args.err);
          if (!ok) break;
          mbar_arrive_expect_tx(&B_.raw_full[raw.stage], bytes);
          const uint8_t* src = args.comp_k[l] + (int64_t)walk.b * args.row_stride +
                               (int64_t)walk.t * kRawBytes;
          bulk_g2s_hint(sRaw + (size_t)raw.stage * kRawBytes, src, bytes, &B_.raw_full[raw.stage],
                        policy);
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
      Ring ast(NA), acc(lay.NACC);
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
        for (int l = 0; l < L; ++l) {
          const int as = ast.stage, ac = acc.stage;
          ok = mbar_wait_bounded(&B_.a_full[as], ast.phase, sAbort, args.err) &&
               mbar_wait_bounded(&B_.acc_empty[ac], acc.phase ^ 1, sAbort, args.err);
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
          ++item;
          ast.advance();
          acc.advance();
        }
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
    // ------------------------------- transform: raw records -> MMA operand
    const int tw = warp - kWarpXform0;
    Ring raw(NR), ast(NA), scr(lay.NSC);
    for (walk.start(b_start, t_start, count); walk.valid(); walk.next()) {
      bool ok = true;
      for (int l = 0; l < L; ++l, raw.advance(), ast.advance(), scr.advance()) {
        const int rs = raw.stage, as = ast.stage, sc = scr.stage;
        ok = mbar_wait_bounded(&B_.raw_full[rs], raw.phase, sAbort, args.err) &&
             mbar_wait_bounded(&B_.a_empty[as], ast.phase ^ 1, sAbort, args.err) &&
             mbar_wait_bounded(&B_.sc_empty[sc], scr.phase ^ 1, sAbort, args.err);
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
    const int ew = warp - kWarpEpi0;
    const bool group_a = ew < 4;  // heads 0-31 (finishes the chunk) vs 32-63
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;
    const int head0 = group_a ? 0 : kHalfHeads;
    float* sWpw = sWp + ew * L * kHalfHeads;
    const uint32_t lane_base = tmem_base + ((uint32_t)(quarter * 32) << 16) + (uint32_t)head0;
    Ring acc(lay.NACC), scr(lay.NSC), prt(lay.NPART);
    int cur = -1;
    for (walk.start(b_start, t_start, count); walk.valid(); walk.next()) {
      const int b = walk.b;
      if (b != cur) {  // this warp's private copy of its heads' weights for the row
        __syncwarp();
        for (int i = lane; i < L * kHalfHeads; i += 32)
          sWpw[i] = __ldg(args.wprime + ((size_t)b * L + i / kHalfHeads) * kHeads + head0 +
                          i % kHalfHeads);
        __syncwarp();
        cur = b;
      }
      const int n = walk.t * kTile + r;
      const bool valid = n < walk.nv;
      const bool in_row = n < args.N;
      float ens = 0.f;
      bool ok = true;
      for (int l = 0; l < L; ++l, acc.advance(), scr.advance(), prt.advance()) {
        const int ac = acc.stage, sc = scr.stage;
        const uint32_t ph_acc = acc.phase;
        ok = mbar_wait_bounded(&B_.sc_full[sc], scr.phase, sAbort, args.err);
        if (!ok) break;
        const float s = sSc[sc * kTile + r];
        __syncwarp();
        if (lane == 0) mbar_arrive(&B_.sc_empty[sc]);
        ok = mbar_wait_bounded(&B_.acc_full[ac], ph_acc, sAbort, args.err);
        if (!ok) break;
        tc_fence_after();
        const bool nonneg = __all_sync(0xffffffffu, !(s < 0.f));
        HeadCols<P> cols;
        cols.load(lane_base + (uint32_t)(ac * NQ));
        // the accumulator stage is free as soon as every warp holds its columns
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&B_.acc_empty[ac]);
        if constexpr (DUMP) {
          if (b == args.dbg_b && walk.t == args.dbg_t && l == args.dbg_layer)
            for (int p = 0; p < P; ++p)
              for (int i = 0; i < kHalfHeads; ++i)
                args.dbg_out[(size_t)r * NQ + p * kHeads + head0 + i] = cols.at(p, i);
        }
        const float part = head_partial<P>(cols, sWpw + l * kHalfHeads, s, nonneg);
        const int ps = prt.stage;
        const uint32_t ph_part = prt.phase;
        if (!group_a) {
          ok = mbar_wait_bounded(&B_.part_empty[ps], ph_part ^ 1, sAbort, args.err);
          if (!ok) break;
          sPart[ps * kTile + r] = part;
          __syncwarp();
          if (lane == 0) mbar_arrive(&B_.part_full[ps]);
          continue;
        }
        ok = mbar_wait_bounded(&B_.part_full[ps], ph_part, sAbort, args.err);
        if (!ok) break;
        const float other = sPart[ps * kTile + r];
        __syncwarp();
        if (lane == 0) mbar_arrive(&B_.part_empty[ps]);
        float logit = part + other;
        if (nonneg) logit *= s;
        float score = 1.0f / (1.0f + __expf(-logit));
        if (!valid) score = 0.f;
        if (args.scores && in_row) args.scores[((size_t)l * args.B + b) * args.N + n] = score;
        ens = (args.mode == FM_ENSEMBLE_MAX) ? (l == 0 ? score : fmaxf(ens, score)) : ens + score;
      }
      if (!ok) break;
      if (group_a) {
        if (args.mode != FM_ENSEMBLE_MAX) ens = ens / (float)L;
        if (!valid) ens = 0.f;
        if (in_row) {
          if (args.ens) args.ens[(size_t)b * args.N + n] = ens;
          if (args.keep_thr) args.keep_thr[(size_t)b * args.N + n] = (valid && ens > args.thr) ? 1 : 0;
        }
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
  // deepest key ring that fits: more raw stages keep more bytes in flight
  int NA = 4, NR = 8;
  if (const char* e = getenv("FM_A_STAGES")) NA = atoi(e) < 2 ? 2 : atoi(e);
  if (const char* e = getenv("FM_RAW_STAGES")) NR = atoi(e) < 2 ? 2 : atoi(e);
  Layout lay = make_layout(a.L, P, NA, NR);
  while (lay.total > (uint32_t)max_smem && NR > 3) {
    --NR;
    lay = make_layout(a.L, P, NA, NR);
  }
  while (lay.total > (uint32_t)max_smem && NA > 2) {
    --NA;
    lay = make_layout(a.L, P, NA, NR);
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
  score_kernel<P, DUMP><<<grid, kThreads, lay.total, st>>>(a, NA, NR);
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
