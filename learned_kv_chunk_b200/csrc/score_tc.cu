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
//    tile) units; each unit is scored for all L layers (one "item" per layer)
//    so the ensemble stays in registers and one fp32 per chunk is written;
//  * the keys go to the tensor cores as stored: kind::f8f6f4 MMA with A = the
//    128 e4m3 bytes of each record (K = 128 dims) and B = the query split into
//    P e4m3 pieces, fp32 accumulators in TMEM, M = 128 chunks in the 128 TMEM
//    lanes.  With two pieces the residual piece is stored unscaled and the
//    tensor core adds both into one 64-column accumulator (eight MMAs of
//    N = 64 per item: four K steps per piece), and each epilogue group has two
//    accumulator stages; with three pieces each piece keeps its own 64
//    columns (four MMAs of N = 192) and one stage per group.  The per-chunk
//    fp32 scale, the per-head power-of-two scale of the pieces, relu, the
//    head-weighted sum and the sigmoid run in the epilogue;
//  * the 132-byte records are not 16-byte aligned, so a tile is fetched with
//    one 1-D bulk copy (TMA engine) of 128 * 132 bytes into a shared-memory
//    stage; four transform warps (one TMEM lane quarter each, one chunk row
//    per thread) read each row with conflict-free 4-byte loads (row stride 33
//    words) and store it into TMEM, where the MMA takes A from; each thread
//    also moves its record's fp32 scale into a TMEM column that the epilogue
//    reads with the accumulators, so no scale is read from global memory.  A
//    stage goes back to the key loader as soon as it has been read, so the
//    ring holds little besides keys in flight from HBM;
//  * single threads pace the pass: the key loader (its copies in flight set
//    the HBM rate) and the MMA issuers (each tcgen05.mma, commit or mbarrier
//    probe costs its thread tens of cycles, so an item is four MMAs with
//    descriptors advanced by constant adds, two issuing threads on two
//    schedulers share the items, and per-item work is kept off every role:
//    scales travel through TMEM instead of as scattered global loads, which
//    doubled the L2 request count).  Warp w runs on scheduler w % 4 and may
//    only touch TMEM lanes 32*(w % 4) .. +31, so every scheduler hosts one
//    transform warp and two epilogue warps;
//  * warp roles (16 warps): 0 key loader, 1 and 3 MMA issuers (one per
//    epilogue group), 2 TMEM owner + query loader, 4-7 transform, 8-11 and
//    12-15 two epilogue groups (one lane
//    quarter per warp, all 64 heads of a chunk row), each with its
//    accumulator stages.  Units are taken in pairs from the same row,
//    the first for group 0 and the second for group 1, and their items are
//    issued layer by layer alternately, (u0,l0) (u1,l0) (u0,l1) (u1,l1) ...,
//    so each group has a whole MMA to drain its stage before it is needed
//    again.  Every ring index is advanced incrementally (no runtime division
//    in any loop);
//  * the pass is launched to overlap the query-packing kernel ahead of it:
//    set-up and the key stream start at once, and only the query loader and
//    the epilogue (the head weights) wait for the packing kernel's writes.
#include "fm_internal.cuh"

namespace fm {
namespace {

constexpr int kWarps = 16;
constexpr int kThreads = kWarps * 32;
constexpr int kRawBytes = kTile * kRecord;  // 16896, a multiple of 128
constexpr int kMmaM = kTile;                // MMA rows = TMEM lanes = chunks of a tile
constexpr int kQuarters = 4;                // TMEM lane quarters (32 lanes, one warp each)
constexpr int kWarpLoader = 0, kWarpMma = 1, kWarpQ = 2, kWarpMma2 = 3;
constexpr int kWarpXform0 = 4, kWarpEpi0 = 8;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kACols = 32;  // 128 e4m3 bytes per row = 32 columns per key tile
constexpr uint32_t kPieceBytes = kHeads * kHeadDim;  // one query piece of one layer

// TMEM columns: accumulator of group g at [g * P*64, (g+1) * P*64), key tiles
// after them, and the last 32 columns two rings of per-chunk scales, 16
// columns per epilogue group: the scale of the g-th group's n-th key tile
// (item, or unit with shared keys) in column kScaleCol + 16 g + n mod 16.
constexpr uint32_t kScaleSlots = 32;
constexpr uint32_t kScaleCol = kTmemCols - kScaleSlots;
constexpr uint32_t kGroupSlots = kScaleSlots / 2;
// P = 2: the two query pieces go to one accumulator (piece 1 is stored
// unscaled, so the tensor core sums p0 + p1), two stages per epilogue group;
// P = 3: one accumulator block per piece, one stage per group.
template <int P>
constexpr bool fold() { return P == 2; }
template <int P>
constexpr int acc_pieces() { return fold<P>() ? 1 : P; }
template <int P>
constexpr uint32_t acc_stages() { return fold<P>() ? 2u : 1u; }
template <int P>
constexpr uint32_t acc_cols() { return (uint32_t)acc_pieces<P>() * kHeads; }
template <int P>
constexpr uint32_t a_col_base() { return 2u * acc_stages<P>() * acc_cols<P>(); }
template <int P>
constexpr uint32_t a_stages() { return (kScaleCol - a_col_base<P>()) / kACols; }  // 7 (P=2), 3 (P=3)
// A group's scale slot is rewritten 16 of that group's key tiles later.  The
// transform stores tile x only after the key stage of the tile NA before it
// (in the CTA's order) was released, so after every tile up to x - NA had all
// its MMAs issued.  With 16 > NA + 1, at least one tile of the same group lies
// between the slot's previous tile y and x - NA, and that group's issuer
// issued it only after the group's epilogue had released y -- scale included.
// Each group's ring depends on its own epilogue only, whatever the other group
// does (a row's lone last tile leaves the second group idle for that pair).
static_assert(a_stages<2>() + 1 < kGroupSlots && a_stages<3>() + 1 < kGroupSlots, "scale ring too short");


struct Layout {
  uint32_t q_off, raw_off, wp_off, bar_off, misc_off, total;
};

// qheads: query rows per piece held by this CTA (64, or 32 for a CTA pair)
__host__ __device__ inline Layout make_layout(int L, int P, int NR, int NA, int qheads = kHeads) {
  Layout s;
  uint32_t o = 0;
  s.q_off = o;    o += (uint32_t)L * P * (uint32_t)qheads * kHeadDim;  // multiple of 1024
  s.raw_off = o;  o += (uint32_t)NR * kRawBytes;                       // 128-aligned stages
  s.wp_off = o;   o += 2u * kQuarters * (uint32_t)L * kHeads * 4;     // per epilogue warp
  o = (o + 7u) & ~7u;
  s.bar_off = o;  o += (uint32_t)(2 * NR + 2 * NA + 8 + 4) * 8;
  s.misc_off = o; o += 64;
  s.total = o + 1024;  // slack to align the base to 1024
  return s;
}

struct Bars {
  uint64_t *raw_full, *raw_empty, *a_full, *a_empty, *acc_full, *acc_empty, *q_full, *q_empty,
      *done, *q_peer;
};

// ------------------------------------------------------------ CTA pairs
// The pair form (cta_group::2): two CTAs of a cluster share each MMA, M = 256
// chunks (128 in each CTA's TMEM), so one instruction does the work of two.
// The leader (cluster rank 0) issues every MMA and commit; each CTA copies
// and stores its own key tile and holds half of the query (32 heads per
// piece); the MMA reads both halves.  The peer's transform and epilogue
// warps signal the leader's barriers across the cluster; the commits arrive
// on the barrier of the same offset in both CTAs.
__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
// Shared-memory address of `p` in the CTA of cluster rank `rank`.
__device__ __forceinline__ uint32_t cluster_smem(const void* p, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_u32(p)), "r"(rank));
  return r;
}
// Arrive on a barrier of either CTA of the pair.  Default (CTA-scope release)
// semantics: a cluster-scope release waits for every earlier write of the
// thread (the epilogue's score stores) to become visible to the cluster,
// which cost each transform and epilogue step over a thousand cycles; what
// the arrival publishes is ordered by the tcgen05 fences around it (the
// TMEM stores before it, the MMA after the leader's wait).
__device__ __forceinline__ void mbar_arrive_remote(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}
__device__ __forceinline__ void umma_f8f6f4_ts_pair(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                                    uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f8f6f4 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// Arrives on `bar` (same offset) in both CTAs of the pair once every MMA this
// thread issued before has completed.
__device__ __forceinline__ void umma_commit_pair(uint64_t* bar) {
  const uint16_t mask = 3;
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(
          smem_u32(bar)),
      "h"(mask)
      : "memory");
}
__device__ __forceinline__ void tmem_alloc_pair(uint32_t* dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst_smem)),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish_pair() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// mbarrier wait with cluster-scope acquire (for barriers the peer arrives on)
__device__ __forceinline__ bool mbar_try_wait_cluster(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
__device__ __forceinline__ bool mbar_wait_cluster_bounded(uint64_t* bar, uint32_t parity, volatile int* abort,
                                                          int* err, uint64_t limit_ns) {
  if (mbar_try_wait_cluster(bar, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  for (uint32_t i = 1;; ++i) {
    if (mbar_try_wait_cluster(bar, parity)) return true;
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

// Position in a ring of n stages: the stage index and the parity of the
// stage's mbarrier phase for the current pass.  Advanced once per item, so no
// role ever divides by a runtime ring size.
struct Ring {
  uint32_t stage, phase, n;
  __device__ explicit Ring(uint32_t n_) : stage(0), phase(0), n(n_) {}
  __device__ __forceinline__ void advance() {
    if (++stage == n) { stage = 0; phase ^= 1u; }
  }
};

// Walks this CTA's contiguous range of valid (row, unit) units; a unit is
// one 128-chunk tile, or for a CTA pair two (the tile of each CTA).
struct UnitWalk {
  const int32_t* n_valid;
  int N, B, span;  // span: chunks per unit
  int b, t, nv, tiles;
  int64_t left;
  __device__ int nvalid_of(int row) const {
    int v = n_valid ? __ldg(n_valid + row) : N;
    return max(0, min(v, N));
  }
  __device__ void start(int b0, int t0, int64_t count) {
    b = b0; t = t0; left = count;
    if (left > 0) { nv = nvalid_of(b); tiles = (nv + span - 1) / span; }
  }
  __device__ bool valid() const { return left > 0; }
  __device__ void next() {
    --left;
    if (left <= 0) return;
    if (++t >= tiles) {
      t = 0;
      do { ++b; nv = nvalid_of(b); tiles = (nv + span - 1) / span; } while (tiles == 0);
    }
  }
};

struct Unit {
  int b, t, nv;
};

// The walk in pairs of units of the same row: u[0] for epilogue group 0 and,
// when the row has a next unit in this CTA's range, u[1] for group 1.  Every
// role derives the same pairs from the same range.
struct PairWalk {
  UnitWalk w;
  Unit u[2];
  bool has0, has1;
  __device__ void fill() {
    has0 = w.valid();
    has1 = false;
    if (!has0) return;
    u[0] = Unit{w.b, w.t, w.nv};
    w.next();
    if (w.valid() && w.b == u[0].b) {
      u[1] = Unit{w.b, w.t, w.nv};
      has1 = true;
      w.next();
    }
  }
  __device__ void start(const int32_t* n_valid, int N, int B, int b0, int t0, int64_t count, int span) {
    w.n_valid = n_valid; w.N = N; w.B = B; w.span = span;
    w.start(b0, t0, count);
    fill();
  }
  __device__ bool valid() const { return has0; }
  __device__ void next() { fill(); }
};

// 32 lanes x 32 heads x P pieces of one accumulator stage, read in one load+wait
// (optionally with one more column, the chunk's scale).
template <int P>
struct HeadCols {
  uint32_t u[P][32];
  __device__ __forceinline__ void load(uint32_t col0) {
    if constexpr (P == 1)
      tmem_ld32_wait(col0, u[0]);
    else if constexpr (P == 3)
      tmem_ld32x3_wait(col0, col0 + kHeads, col0 + 2 * kHeads, u[0], u[1], u[2]);
    else
      tmem_ld32x2_wait(col0, col0 + kHeads, u[0], u[1]);
  }
  __device__ __forceinline__ void load_with(uint32_t col0, uint32_t scol, uint32_t* sv) {
    if constexpr (P == 1)
      tmem_ld32_x1_wait(col0, scol, u[0], sv);
    else if constexpr (P == 3)
      tmem_ld32x3_x1_wait(col0, col0 + kHeads, col0 + 2 * kHeads, scol, u[0], u[1], u[2], sv);
    else
      tmem_ld32x2_x1_wait(col0, col0 + kHeads, scol, u[0], u[1], sv);
  }
  __device__ __forceinline__ float at(int p, int i) const { return __uint_as_float(u[p][i]); }
};

// Head sum over 32 heads for one chunk row:
//   sum_h relu(d_h) * w'_h  with d_h = D0 (one accumulator for two pieces)
//                           or D0 + D1/16 + D2/256 (three),   when s >= 0
//   sum_h relu(s d_h) * w'_h                                  otherwise
// where D_p are the accumulator columns of piece p and w' the head weights
// with the pieces' power-of-two scale folded in.
template <int P>
__device__ __forceinline__ float head_sum32(const HeadCols<P>& c, const float* __restrict__ w,
                                            float s, bool nonneg) {
  constexpr float kInv16 = 0.0625f, kInv256 = 0.00390625f;
  if (nonneg) {
    const uint64_t c16 = f2_pack(kInv16, kInv16), c256 = f2_pack(kInv256, kInv256);
    uint64_t acc = f2_pack(0.f, 0.f);
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      float dx, dy;
      if constexpr (P == 1) {
        dx = c.at(0, 2 * j);
        dy = c.at(0, 2 * j + 1);
      } else {
        const uint64_t p0 = f2_pack(c.at(0, 2 * j), c.at(0, 2 * j + 1));
        const uint64_t p1 = f2_pack(c.at(1, 2 * j), c.at(1, 2 * j + 1));
        uint64_t d = f2_fma(p1, c16, p0);
        if constexpr (P == 3) d = f2_fma(f2_pack(c.at(2, 2 * j), c.at(2, 2 * j + 1)), c256, d);
        f2_unpack(d, dx, dy);
      }
      const float2 ww = *reinterpret_cast<const float2*>(w + 2 * j);
      const uint64_t rr = f2_pack(fmax_nan(dx, 0.f), fmax_nan(dy, 0.f));
      acc = f2_fma(rr, f2_pack(ww.x, ww.y), acc);  // one chain: fewer registers, same issue count
    }
    float a0, a1;
    f2_unpack(acc, a0, a1);
    return a0 + a1;
  }
  float acc = 0.f;
  for (int i = 0; i < 32; ++i) {
    float d = c.at(0, i);
    if constexpr (P >= 2) d = fmaf(c.at(1, i), kInv16, d);
    if constexpr (P == 3) d = fmaf(c.at(2, i), kInv256, d);
    acc = fmaf(fmax_nan(d * s, 0.f), w[i], acc);
  }
  return acc;
}

// SK (shared keys): every layer's pointer is the same key tensor, so each
// unit's tile is copied and stored into TMEM once and every layer's MMAs read
// it; the key ring, the TMEM key stages and the scale slots then go per unit
// instead of per (unit, layer).
template <int P, bool DUMP, bool SK, bool PAIR>
__global__ void __launch_bounds__(kThreads, 1) score_kernel(ScoreArgs args, int NR) {
  extern __shared__ uint8_t smem_raw[];
  constexpr uint32_t ACCW = acc_cols<P>();
  constexpr uint32_t ABASE = a_col_base<P>();
  constexpr uint32_t NA = a_stages<P>();
  constexpr int kSpan = PAIR ? 2 * kTile : kTile;             // chunks per unit
  constexpr uint32_t kQHeads = PAIR ? kHeads / 2 : kHeads;     // query rows per piece in this CTA
  constexpr uint32_t kQPiece = kQHeads * kHeadDim;             // bytes of one piece in shared memory
  constexpr uint32_t kArrivals = PAIR ? 2 * kQuarters : kQuarters;  // warps arriving on a_full, acc_empty
  const uint32_t rank = PAIR ? cluster_rank() : 0u;
  const Layout lay = make_layout(args.L, P, NR, NA, (int)kQHeads);
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  const int L = args.L;
  const int LK = SK ? 1 : L;  // key tiles copied per unit
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  constexpr uint32_t kQLayerBytes = (uint32_t)P * kQPiece;  // one layer's query in shared memory

  uint8_t* sQ = smem + lay.q_off;
  uint8_t* sRaw = smem + lay.raw_off;
  float* sWp = reinterpret_cast<float*>(smem + lay.wp_off);
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + lay.bar_off);
  Bars B_;
  B_.raw_full = bar;                B_.raw_empty = B_.raw_full + NR;
  B_.a_full = B_.raw_empty + NR;    B_.a_empty = B_.a_full + NA;
  B_.acc_full = B_.a_empty + NA;    B_.acc_empty = B_.acc_full + 4;
  B_.q_full = B_.acc_empty + 4;
  B_.q_empty = B_.q_full + 1;       B_.done = B_.q_empty + 1;
  B_.q_peer = B_.done + 1;
  uint32_t* sTmem = reinterpret_cast<uint32_t*>(smem + lay.misc_off);
  volatile int* sAbort = reinterpret_cast<volatile int*>(smem + lay.misc_off + 4);
  int* sRange = reinterpret_cast<int*>(smem + lay.misc_off + 8);  // b0, t0, count lo, count hi

  // ---------------------------------------------------------------- setup
  if (threadIdx.x == 0) {
    for (int i = 0; i < NR; ++i) {
      mbar_init(&B_.raw_full[i], 1);           // bulk copy landed
      mbar_init(&B_.raw_empty[i], kQuarters);  // read by all transform warps
    }
    for (uint32_t i = 0; i < NA; ++i) {
      mbar_init(&B_.a_full[i], kArrivals);     // key tile stored in TMEM (one arrival per warp)
      mbar_init(&B_.a_empty[i], 1);            // the MMA that read it retired
    }
    for (int g = 0; g < 4; ++g) { mbar_init(&B_.acc_full[g], 1); mbar_init(&B_.acc_empty[g], kArrivals); }
    mbar_init(B_.q_full, 1);
    mbar_init(B_.q_empty, 2);                // both MMA issuers' commits
    mbar_init(B_.done, 2);
    mbar_init(B_.q_peer, 1);                 // pair: the peer's query half landed
    *sAbort = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == kWarpMma && lane == 0) {
    // this CTA's (or pair's) share of the valid units: rows contribute
    // ceil(n_b / span) units
    int64_t total = 0;
    for (int b = 0; b < args.B; ++b) {
      int v = args.n_valid ? __ldg(args.n_valid + b) : args.N;
      v = max(0, min(v, args.N));
      total += (v + kSpan - 1) / kSpan;
    }
    const int64_t slot = PAIR ? blockIdx.x >> 1 : blockIdx.x, slots = PAIR ? gridDim.x >> 1 : gridDim.x;
    const int64_t u0 = total * slot / slots;
    const int64_t u1 = total * (slot + 1) / slots;
    int64_t acc = 0;
    int b0 = 0, t0 = 0;
    for (int b = 0; b < args.B; ++b) {
      int v = args.n_valid ? __ldg(args.n_valid + b) : args.N;
      v = max(0, min(v, args.N));
      const int tiles = (v + kSpan - 1) / kSpan;
      if (acc + tiles > u0) { b0 = b; t0 = (int)(u0 - acc); break; }
      acc += tiles;
    }
    sRange[0] = b0; sRange[1] = t0;
    sRange[2] = (int)((u1 - u0) & 0xffffffff); sRange[3] = (int)((u1 - u0) >> 32);
  }
  if (warp == kWarpQ) {
    if constexpr (PAIR) {
      tmem_alloc_pair(sTmem, kTmemCols);
      tmem_relinquish_pair();
    } else {
      tmem_alloc(sTmem, kTmemCols);
      tmem_relinquish();
    }
  }
  tc_fence_before();
  __syncthreads();
  if constexpr (PAIR) cluster_sync_all();  // both CTAs' barriers exist before any cross-CTA arrival
  tc_fence_after();
  const uint32_t tmem_base = *sTmem;
  const int b_start = sRange[0], t_start = sRange[1];
  const int64_t count = (int64_t)(uint32_t)sRange[2] | ((int64_t)sRange[3] << 32);
  PairWalk pw;

  if (warp == kWarpLoader) {
    // ------------------------------------------------------- key tile loader
    if (lane == 0) {
      uint32_t item = 0;
      Ring raw(NR);
      bool ok = true;
      for (pw.start(args.n_valid, args.N, args.B, b_start, t_start, count, kSpan); ok && pw.valid() && !*sAbort;
           pw.next()) {
        for (int l = 0; l < LK && ok; ++l) {
#pragma unroll
          for (int j = 0; j < 2; ++j) {
            if (j == 1 && !pw.has1) break;
            const Unit U = j == 0 ? pw.u[0] : pw.u[1];
            const int tt = PAIR ? 2 * U.t + (int)rank : U.t;  // this CTA's tile of the unit
            const int nrem = min(kTile, U.nv - tt * kTile);
            ok = mbar_wait_bounded(&B_.raw_empty[raw.stage], raw.phase ^ 1, sAbort, args.err, args.wait_ns);
            if (!ok) break;
            if (PAIR && nrem <= 0) {
              // the pair's odd last tile: this CTA has none, its stage passes through unread
              mbar_arrive(&B_.raw_full[raw.stage]);
            } else {
              const uint32_t bytes = (uint32_t)((nrem + 3) & ~3) * kRecord;
              mbar_arrive_expect_tx(&B_.raw_full[raw.stage], bytes);
              const uint8_t* src = args.comp_k[l] + (int64_t)U.b * args.row_stride + (int64_t)tt * kRawBytes;
              bulk_g2s(sRaw + (size_t)raw.stage * kRawBytes, src, bytes, &B_.raw_full[raw.stage]);
            }
            ++item;
            raw.advance();
          }
        }
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
    if (lane == 0 && !args.withhold_query) {
      grid_dependency_wait();  // the query image is written by the packing kernel ahead
      int cur = -1;
      uint32_t loads = 0;
      for (pw.start(args.n_valid, args.N, args.B, b_start, t_start, count, kSpan); pw.valid() && !*sAbort; pw.next()) {
        const int b = pw.u[0].b;
        if (b == cur) continue;
        if (loads > 0 && !mbar_wait_bounded(B_.q_empty, (loads - 1) & 1, sAbort, args.err, args.wait_ns)) break;
        mbar_arrive_expect_tx(B_.q_full, (uint32_t)L * kQLayerBytes);
        // piece p of layer l: this CTA's heads (all 64, or 32 rank .. of a pair)
        for (int l = 0; l < L; ++l)
          for (int pc = 0; pc < P; ++pc)
            bulk_g2s(sQ + (size_t)l * kQLayerBytes + (size_t)pc * kQPiece,
                     args.qpack + (((size_t)b * L + l) * P + pc) * kPieceBytes + (size_t)rank * kQPiece, kQPiece,
                     B_.q_full);
        if (PAIR && rank == 1) {  // tell the leader, which issues the MMAs, that this half landed
          if (!mbar_wait_bounded(B_.q_full, loads & 1, sAbort, args.err, args.wait_ns)) break;
          mbar_arrive_remote(cluster_smem(B_.q_peer, 0));
        }
        cur = b;
        ++loads;
      }
      if (loads > 0) mbar_drain(B_.q_full, (loads - 1) & 1, args.err);
    }
  } else if ((warp == kWarpMma || warp == kWarpMma2) && PAIR && rank != 0) {
    // pair peer: the leader issues; wait for every MMA that uses this CTA's
    // TMEM and shared memory to retire before they go away
    if (lane == 0) mbar_drain(B_.done, 0, args.err);
  } else if (warp == kWarpMma || warp == kWarpMma2) {
    // --------------------------------------------------------- MMA issuers
    // Two issuing threads on two schedulers, one per epilogue group: thread
    // `me` issues the items of group `me` (the pair's unit u[me]) into that
    // group's accumulator.  A tcgen05.mma costs its issuing thread tens of
    // cycles, so two issuers double the issue rate; each commit tracks only
    // its own thread's MMAs, and both walk every item to keep the key ring's
    // stage and phase.
    if (lane == 0) {
      const int me = warp == kWarpMma ? 0 : 1;
      constexpr uint32_t idesc = idesc_e4m3_f32(PAIR ? 2 * kMmaM : kMmaM, (int)ACCW);  // N = 64 with the pieces folded
      // B descriptors: the start-address field counts 16-byte units, so the
      // layer and K-step offsets are plain adds (the field cannot carry: the
      // query image lies in the first 256 KB of shared memory)
      const uint64_t bdesc0 = sdesc_kmajor_sw128(smem_u32(sQ));
      constexpr uint64_t kLayerStep = kQLayerBytes >> 4, kKStep = 32 >> 4;
      uint32_t item = 0, rows = 0, phs = 0, gcnt = 0;  // phs: phase bit per accumulator stage
      Ring ast(NA);
      int cur = -1;
      bool ok = true;
      for (pw.start(args.n_valid, args.N, args.B, b_start, t_start, count, kSpan); ok && pw.valid() && !*sAbort;) {
        const int b = pw.u[0].b;
        if (b != cur) {
          if (!mbar_wait_bounded(B_.q_full, rows & 1, sAbort, args.err, args.wait_ns)) break;
          if (PAIR && !mbar_wait_cluster_bounded(B_.q_peer, rows & 1, sAbort, args.err, args.wait_ns)) break;
          ++rows;
          cur = b;
        }
        uint64_t bd = bdesc0;
        Ring su = ast;  // shared keys: the key stage of unit u[me]
        if (SK && me == 1) su.advance();
        for (int l = 0; l < L && ok; ++l, bd += kLayerStep) {
#pragma unroll
          for (int j = 0; j < 2; ++j) {
            if (j == 1 && !pw.has1) break;
            if (j != me) {
              if (!SK) ast.advance();
              continue;
            }
            const Ring& as = SK ? su : ast;
            const uint32_t st = acc_stages<P>() == 2 ? (gcnt & 1u) : 0u;
            const uint32_t slot_i = (uint32_t)j * acc_stages<P>() + st;
            const uint32_t ph = (phs >> st) & 1u;
            if constexpr (PAIR)
              ok = mbar_wait_cluster_bounded(&B_.a_full[as.stage], as.phase, sAbort, args.err, args.wait_ns) &&
                   mbar_wait_cluster_bounded(&B_.acc_empty[slot_i], ph ^ 1, sAbort, args.err, args.wait_ns);
            else
              ok = ((SK && l > 0) ||
                    mbar_wait_bounded(&B_.a_full[as.stage], as.phase, sAbort, args.err, args.wait_ns)) &&
                   mbar_wait_bounded(&B_.acc_empty[slot_i], ph ^ 1, sAbort, args.err, args.wait_ns);
            if (!ok) break;
            tc_fence_after();
            const uint32_t d = tmem_base + slot_i * ACCW;
            const uint32_t a = tmem_base + ABASE + as.stage * kACols;
            const auto mma = [&](uint32_t aa, uint64_t bb, uint32_t acc) {
              if constexpr (PAIR) umma_f8f6f4_ts_pair(d, aa, bb, idesc, acc);
              else umma_f8f6f4_ts(d, aa, bb, idesc, acc);
            };
            const auto commit = [&](uint64_t* bar) {
              if constexpr (PAIR) umma_commit_pair(bar);
              else umma_commit(bar);
            };
            mma(a, bd, 0u);
            mma(a + 8u, bd + kKStep, 1u);
            mma(a + 16u, bd + 2 * kKStep, 1u);
            mma(a + 24u, bd + 3 * kKStep, 1u);
            if constexpr (fold<P>()) {  // piece 1 of the layer's image into the same accumulator
              const uint64_t bd1 = bd + (kQPiece >> 4);
              mma(a, bd1, 1u);
              mma(a + 8u, bd1 + kKStep, 1u);
              mma(a + 16u, bd1 + 2 * kKStep, 1u);
              mma(a + 24u, bd1 + 3 * kKStep, 1u);
            }
            if (!SK || l == L - 1) commit(&B_.a_empty[as.stage]);  // the TMEM key tile may be overwritten
            commit(&B_.acc_full[slot_i]);
            ++item;
            if (!SK) ast.advance();
            phs ^= 1u << st;
            ++gcnt;
          }
        }
        if (!ok) break;
        if (SK) {  // the pair's units each held one key stage
          ast.advance();
          if (pw.has1) ast.advance();
        }
        pw.next();
        if (!pw.valid() || pw.u[0].b != b) {
          if constexpr (PAIR) umma_commit_pair(B_.q_empty);
          else umma_commit(B_.q_empty);
        }
      }
      {  // every issued MMA and commit retired before TMEM and smem go away (both issuers arrive)
        if constexpr (PAIR) umma_commit_pair(B_.done);
        else umma_commit(B_.done);
        mbar_drain(B_.done, 0, args.err);
      }
    }
  } else if (warp >= kWarpXform0 && warp < kWarpXform0 + 4) {
    // ------------------------- transform: raw records -> TMEM key tile (A)
    // Thread `lane` of this warp owns one chunk row of the tile: it reads the
    // row's 128 key bytes (the 33-word row stride puts the 32 lanes of a load
    // in 32 different banks) and stores them to its TMEM lane.  The four
    // warps run independently; each arrives once per key tile on both
    // barriers.  Tiles arrive in the loader's order (pairs, then the layers
    // copied per unit, then the pair's units), which also gives each tile's
    // epilogue group and so its scale slot.
    const uint32_t quarter = (uint32_t)warp & 3u;
    const uint32_t row = quarter * 32u + (uint32_t)lane;
    const uint32_t lane_base = tmem_base + ((quarter * 32u) << 16);
    Ring raw(NR), ast(NA);
    uint32_t gtiles[2] = {0u, 0u};  // key tiles of each group so far
    bool go = true;
    for (pw.start(args.n_valid, args.N, args.B, b_start, t_start, count, kSpan); go && pw.valid(); pw.next())
    for (int l = 0; l < LK && go; ++l)
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      if (j == 1 && !pw.has1) break;
      int good = 1;
      if (lane == 0)
        good = mbar_wait_bounded(&B_.raw_full[raw.stage], raw.phase, sAbort, args.err, args.wait_ns) &&
               mbar_wait_bounded(&B_.a_empty[ast.stage], ast.phase ^ 1, sAbort, args.err, args.wait_ns);
      good = __shfl_sync(0xffffffffu, good, 0);
      if (!good) {
        go = false;
        break;
      }
      const uint32_t* src =
          reinterpret_cast<const uint32_t*>(sRaw + (size_t)raw.stage * kRawBytes + row * kRecord);
      uint32_t v[32];
#pragma unroll
      for (int w = 0; w < 32; ++w) v[w] = src[w];
      const uint32_t scale_bits = src[32];  // the record's little-endian fp32 scale
      tc_fence_after();  // the MMA that last read this TMEM stage has retired (a_empty)
      tmem_st32_st1_wait(lane_base + ABASE + ast.stage * kACols, v,
                         lane_base + kScaleCol + (uint32_t)j * kGroupSlots + (gtiles[j] & (kGroupSlots - 1)),
                         scale_bits);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&B_.raw_empty[raw.stage]);
        if constexpr (PAIR) mbar_arrive_remote(cluster_smem(&B_.a_full[ast.stage], 0));
        else mbar_arrive(&B_.a_full[ast.stage]);
      }
      ++gtiles[j];
      raw.advance();
      ast.advance();
    }
  } else if (warp >= kWarpEpi0) {
    // ------------------------------------------------------------ epilogue
    grid_dependency_wait();  // the head weights are written by the packing kernel ahead
    const int group = (warp - kWarpEpi0) >> 2;
    const int quarter = warp & 3;
    const int ew = group * kQuarters + quarter;  // 0..7
    const int r = quarter * 32 + lane;           // row of the tile
    float* sWpw = sWp + ew * L * kHeads;
    const uint32_t col_base0 = tmem_base + ((uint32_t)(quarter * 32) << 16) + (uint32_t)group * acc_stages<P>() * ACCW;
    const uint32_t scale_base =
        tmem_base + ((uint32_t)(quarter * 32) << 16) + kScaleCol + (uint32_t)group * kGroupSlots;
    uint32_t phs = 0, gtiles = 0, gitems = 0;  // gtiles: this group's key tiles so far (its scale slots)
    int cur = -1;
    for (pw.start(args.n_valid, args.N, args.B, b_start, t_start, count, kSpan); pw.valid(); pw.next()) {
      if (group == 1 && !pw.has1) continue;
      const Unit U = group == 0 ? pw.u[0] : pw.u[1];
      if (U.b != cur) {  // this warp's private copy of the row's head weights
        __syncwarp();
        for (int i = lane; i < L * kHeads; i += 32)
          sWpw[i] = __ldg(args.wprime + (size_t)U.b * L * kHeads + i);
        __syncwarp();
        cur = U.b;
      }
      const int n = (PAIR ? 2 * U.t + (int)rank : U.t) * kTile + r;
      const bool valid = n < U.nv;
      const bool in_row = n < args.N;
      float ens = 0.f;
      bool ok = true;
      for (int l = 0; l < L; ++l, ++gitems) {
        const uint32_t st = acc_stages<P>() == 2 ? (gitems & 1u) : 0u;
        const uint32_t slot_i = (uint32_t)group * acc_stages<P>() + st;
        const uint32_t col_base = col_base0 + st * ACCW;
        ok = mbar_wait_bounded(&B_.acc_full[slot_i], (phs >> st) & 1u, sAbort, args.err, args.wait_ns);
        phs ^= 1u << st;
        if (!ok) break;
        tc_fence_after();
        // the scale slot of the key tile this item read (one tile per unit with shared keys)
        const uint32_t slot = (gtiles + (SK ? 0u : (uint32_t)l)) & (kGroupSlots - 1);
        const float* w = sWpw + l * kHeads;
        HeadCols<acc_pieces<P>()> c;
        uint32_t s_bits;
        c.load_with(col_base, scale_base + slot, &s_bits);
        const float s = valid ? __uint_as_float(s_bits) : 0.f;  // rows past the tail hold stale bytes
        const bool nonneg = __all_sync(0xffffffffu, !(s < 0.f));
        if constexpr (DUMP) {
          if (U.b == args.dbg_b && U.t == args.dbg_t && l == args.dbg_layer)
            for (int p = 0; p < acc_pieces<P>(); ++p)
              for (int i = 0; i < 32; ++i) args.dbg_out[(size_t)r * 192 + p * kHeads + i] = c.at(p, i);
        }
        float part = head_sum32<acc_pieces<P>()>(c, w, s, nonneg);
        c.load(col_base + 32);
        // the accumulator stage is free once this warp holds all its columns
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          if constexpr (PAIR) mbar_arrive_remote(cluster_smem(&B_.acc_empty[slot_i], 0));
          else mbar_arrive(&B_.acc_empty[slot_i]);
        }
        if constexpr (DUMP) {
          if (U.b == args.dbg_b && U.t == args.dbg_t && l == args.dbg_layer)
            for (int p = 0; p < acc_pieces<P>(); ++p)
              for (int i = 0; i < 32; ++i)
                args.dbg_out[(size_t)r * 192 + p * kHeads + 32 + i] = c.at(p, i);
        }
        part += head_sum32<acc_pieces<P>()>(c, w + 32, s, nonneg);
        const float logit = nonneg ? part * s : part;
        float score = 1.0f / (1.0f + __expf(-logit));
        if (!valid) score = 0.f;
        if (args.scores && in_row) args.scores[((size_t)l * args.B + U.b) * args.N + n] = score;
        ens = (args.mode == FM_ENSEMBLE_MAX) ? (l == 0 ? score : fmax_nan(ens, score)) : ens + score;
      }
      if (!ok) break;
      gtiles += SK ? 1u : (uint32_t)L;
      if (args.mode != FM_ENSEMBLE_MAX) ens = ens / (float)L;
      if (!valid) ens = 0.f;
      if (in_row) {
        if (args.ens) args.ens[(size_t)U.b * args.N + n] = ens;
        if (args.keep_thr) args.keep_thr[(size_t)U.b * args.N + n] = (valid && ens > args.thr) ? 1 : 0;
      }
    }
    // zero the tail of every row that no tile covers: [128 * ceil(n_b / 128), N)
    const int et = ew * 32 + lane;  // 0..255
    const int64_t gt = (int64_t)blockIdx.x * 256 + et, gs = (int64_t)gridDim.x * 256;
    for (int b = 0; b < args.B; ++b) {
      const int v = pw.w.nvalid_of(b);
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
  if constexpr (PAIR) cluster_sync_all();  // neither CTA leaves while the other may still signal it
  if (warp == kWarpQ) {
    tc_fence_after();
    if constexpr (PAIR) tmem_dealloc_pair(tmem_base, kTmemCols);
    else tmem_dealloc(tmem_base, kTmemCols);
  }
}

template <int P, bool DUMP, bool SK, bool PAIR>
fm_status launch_score_p(fm_ctx* ctx, const ScoreArgs& a, cudaStream_t st) {
  if (a.wait_ns == 0) return FM_ERR_INVALID_ARG;  // every wait needs a bound that lets work finish
  static PerDeviceOnce smem_set;
  int max_smem = 0;
  if (cudaDeviceGetAttribute(&max_smem, cudaDevAttrMaxSharedMemoryPerBlockOptin, ctx->device) !=
      cudaSuccess)
    return check_launch();
  // deepest key ring that fits: every stage is keys in flight
  int NR = 16;
  constexpr int NA = (int)a_stages<P>();
  constexpr int kQHeads = PAIR ? kHeads / 2 : kHeads;
  Layout lay = make_layout(a.L, P, NR, NA, kQHeads);
  while (lay.total > (uint32_t)max_smem && NR > 2) {
    --NR;
    lay = make_layout(a.L, P, NR, NA, kQHeads);
  }
  if (lay.total > (uint32_t)max_smem) return FM_ERR_UNSUPPORTED;
  if (fm_status s = smem_limit_once(smem_set, ctx->device, score_kernel<P, DUMP, SK, PAIR>, max_smem)) return s;
  const int span = PAIR ? 2 * kTile : kTile;
  const int64_t units = (int64_t)a.B * ((a.N + span - 1) / span);  // upper bound
  int grid = ctx->num_sms;
  if constexpr (PAIR) {
    // the CTAs are persistent, so every pair must be resident at once: as
    // many pairs as the device holds together (a GPC with an odd number of
    // SMs leaves one SM out), found once per device
    static PerDeviceOnce pairs_set;
    static std::atomic<int> max_pairs[64];
    const int dev = ctx->device;
    if (fm_status s = pairs_set.run(dev, [&]() -> fm_status {
          cudaLaunchAttribute ca[1];
          ca[0].id = cudaLaunchAttributeClusterDimension;
          ca[0].val.clusterDim.x = 2;
          ca[0].val.clusterDim.y = 1;
          ca[0].val.clusterDim.z = 1;
          cudaLaunchConfig_t qc = {};
          qc.gridDim = dim3(grid & ~1);
          qc.blockDim = dim3(kThreads);
          qc.dynamicSmemBytes = lay.total;
          qc.attrs = ca;
          qc.numAttrs = 1;
          int n = 0;
          const cudaError_t e = cudaOccupancyMaxActiveClusters(&n, score_kernel<P, DUMP, SK, PAIR>, &qc);
          if (e != cudaSuccess) return record_cuda_error(e);
          if (dev >= 0 && dev < 64) max_pairs[dev].store(n);
          return FM_OK;
        }))
      return s;
    const int pairs = dev >= 0 && dev < 64 ? max_pairs[dev].load() : 0;
    if (pairs < 1) return FM_ERR_UNSUPPORTED;
    grid = 2 * (pairs < ctx->num_sms / 2 ? pairs : ctx->num_sms / 2);
    if (units * 2 < grid) grid = (int)(units > 0 ? units * 2 : 2);
  } else if (units < grid) {
    grid = (int)(units > 0 ? units : 1);
  }
  // the packing kernel ahead of this one writes only the query image and the
  // head weights, which the query loader and the epilogue wait for; the key
  // stream starts while it runs
  cudaError_t e;
  if constexpr (PAIR) {
    cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(st, &cap) != cudaSuccess) return record_cuda_error(cudaGetLastError());
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = lay.total;
    cfg.stream = st;
    cfg.attrs = attr;
    cfg.numAttrs = cap == cudaStreamCaptureStatusNone ? 2 : 1;
    e = cudaLaunchKernelEx(&cfg, score_kernel<P, DUMP, SK, PAIR>, a, NR);
  } else {
    e = launch_overlapped(score_kernel<P, DUMP, SK, PAIR>, dim3(grid), dim3(kThreads), lay.total, st, a, NR);
  }
  note_launch();
  return e == cudaSuccess ? check_launch() : record_cuda_error(e);
}

}  // namespace

fm_status launch_score(fm_ctx* ctx, const ScoreArgs& a, cudaStream_t st) {
  if (a.dbg_out)
    return ctx->cfg.q_pieces == 3 ? launch_score_p<3, true, false, false>(ctx, a, st)
                                  : launch_score_p<2, true, false, false>(ctx, a, st);
  bool shared = a.L > 1;
  for (int l = 1; l < a.L; ++l) shared = shared && a.comp_k[l] == a.comp_k[0];
  if (shared)
    return ctx->cfg.q_pieces == 3 ? launch_score_p<3, false, true, false>(ctx, a, st)
                                  : launch_score_p<2, false, true, false>(ctx, a, st);
  if (ctx->cfg.q_pieces == 3) return launch_score_p<3, false, false, false>(ctx, a, st);
  return ctx->cfg.cta_pairs ? launch_score_p<2, false, false, true>(ctx, a, st)
                            : launch_score_p<2, false, false, false>(ctx, a, st);
}

}  // namespace fm
