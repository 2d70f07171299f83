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
// The attention reads only the kept chunks, which is what -inf masking
// computes: through the index list of the keep mask (fm_compact_mask), or,
// with no list, from a resident buffer that holds the kept records in order
// (fm_gather_records after each retrieval), which a decode loop reads at
// every step without the scattered accesses.  Each CTA takes one
// row and a segment of 128 kept chunks; a second kernel merges the segments
// (the split-softmax identity).
//
// The two contractions of a segment run on the tensor cores (tcgen05, bf16
// operands, fp32 accumulators in TMEM) at fp32 accuracy:
//  * the e4m3 codes convert to bf16 exactly, so the chunk vectors enter the
//    MMAs as codes and their fp32 scale is applied outside: a logit is
//    scale_i * (q_h . code_i) / sqrt(128), and the output weights are
//    p_hi * scale_i;
//  * q is split into three bf16 pieces (q = q0 + q1 + q2 up to 2^-27
//    relative, each residual exact in fp32), and p * scale into two (2^-18
//    relative); the pieces run as extra K steps into the same accumulator;
//  * one copy of the segment's codes in shared memory (128-byte swizzled,
//    [dim block][chunk][64 dims]) is the K-major A operand of QK^T
//    (M = chunks) and the MN-major A operand of PV (M = dims);
//  * eight warps: warp w reads TMEM lanes 32 (w % 4) .. +31 (its chunk rows,
//    then its dim rows) and heads 16 (w / 4) .. +15; the per-head max and
//    exp-sum over the segment's chunks are warp reduce-scatters merged
//    across the four warps of each half; the softmax runs in log2 units
//    (exp2), and the merge kernel keeps them.
#include <cuda_bf16.h>
#include <cuda_fp8.h>

#include <cmath>
#include <type_traits>

#include "fm_internal.cuh"

namespace fm {
namespace {

constexpr int kAH = 32;          // attention heads (4096 / 128)
constexpr int kAD = 128;         // head dim = chunk vector dim
constexpr int kSeg = 128;        // kept chunks per CTA
constexpr int kPThreads = 256;   // segment kernel: 8 warps, warp w on TMEM lanes 32 (w % 4) and heads 16 (w / 4)
constexpr int kAThreads = 256;   // state update
constexpr int kQPieces = 3, kPPieces = 2;
constexpr uint32_t kXBytes = kSeg * kAD * 2;            // bf16 codes, 2 blocks of 64 dims
constexpr uint32_t kXBlock = kSeg * 128;                // one 64-dim block: 128 rows of 128 bytes
constexpr uint32_t kPieceBytes = kAH * kAD * 2;          // a [32 x 128] bf16 piece, 2 blocks of 64
constexpr uint32_t kPieceBlock = kAH * 128;
constexpr uint32_t kTileBytes = kXBytes + (kQPieces + kPPieces) * kPieceBytes;  // 73728
constexpr uint32_t kTmemCols = 64;                      // logits D1 [0, 32), output D2 [32, 64)

// shared memory ahead of the 1024-aligned operand tiles
struct AttnMisc {
  float scale[kSeg];
  float red[2][2][4][16];  // [max, sum][head half][lane quarter][head]
  float m[kAH], l[kAH];    // m in log2 units: max of logit * log2(e)
  uint32_t valid[8];  // bit k of word w: record w + 8k holds an index inside the memory
  uint64_t bar;
  uint32_t tmem;
  int abort;
};
constexpr uint32_t kAttnSmem = ((sizeof(AttnMisc) + 15) & ~15u) + 1024 + kTileBytes;

__device__ int g_attn_err;  // kDevErrTimeout once an MMA completion wait ran out

__device__ __forceinline__ void umma_bf16_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                             uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Instruction descriptor: kind::f16 with A = B = BF16, D = F32; a_mn / b_mn
// select the MN-major form of the operand.
__host__ __device__ constexpr uint32_t idesc_bf16_f32(int M, int N, bool a_mn, bool b_mn) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((a_mn ? 1u : 0u) << 15) | ((b_mn ? 1u : 0u) << 16) |
         (static_cast<uint32_t>(N >> 3) << 17) | (static_cast<uint32_t>(M >> 4) << 24);
}

// Shared-memory descriptor of an MN-major operand in the 128-byte-swizzled
// canonical layout: 64 MN elements (128 bytes) per row, one row per K index,
// groups of 8 K rows `sbo` bytes apart, blocks of 64 MN elements `lbo` bytes
// apart.
__device__ __forceinline__ uint64_t sdesc_mn_sw128(uint32_t addr, uint32_t lbo, uint32_t sbo) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((addr & 0x3FFFFu) >> 4);
  d |= static_cast<uint64_t>((lbo >> 4) & 0x3FFFu) << 16;
  d |= static_cast<uint64_t>((sbo >> 4) & 0x3FFFu) << 32;
  d |= static_cast<uint64_t>(1) << 46;
  d |= static_cast<uint64_t>(2) << 61;
  return d;
}

// Byte offset of bf16 element (row, k) in a 128-byte-swizzled tile whose
// rows hold 64 elements: rows 128 bytes apart, the 16-byte unit u of row r
// at unit u ^ (r % 8).
__device__ __forceinline__ uint32_t sw_bf16(uint32_t row, uint32_t k) {
  return row * 128u + ((((k >> 3) ^ row) & 7u) << 4) + ((k & 7u) << 1);
}

// Reduce-scatter over the warp of 16 values per lane (v[h] of every lane
// combined with `op`): each step trades half of the remaining values with the
// partner lane and keeps the half picked by the lane's bit, and a last
// exchange combines the two lanes that hold the same index.
// Lane l returns the result for index l / 2.
template <class Op>
__device__ __forceinline__ float reduce_scatter16(float (&v)[16], int lane, Op op) {
  const auto step = [&](auto n_c) {
    constexpr int N = decltype(n_c)::value;
    const bool up = (lane & (2 * N)) != 0;
#pragma unroll
    for (int i = 0; i < N; ++i) {
      const float send = up ? v[i] : v[i + N];
      const float keep = up ? v[i + N] : v[i];
      v[i] = op(keep, __shfl_xor_sync(0xffffffffu, send, 2 * N));
    }
  };
  step(std::integral_constant<int, 8>{});
  step(std::integral_constant<int, 4>{});
  step(std::integral_constant<int, 2>{});
  step(std::integral_constant<int, 1>{});
  return op(v[0], __shfl_xor_sync(0xffffffffu, v[0], 1));
}

// 32 lanes x 16 consecutive fp32 columns at taddr, waited.
__device__ __forceinline__ void tmem_ld16_wait(uint32_t taddr, uint32_t* a) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(a[0]), "=r"(a[1]), "=r"(a[2]), "=r"(a[3]), "=r"(a[4]), "=r"(a[5]), "=r"(a[6]), "=r"(a[7]),
        "=r"(a[8]), "=r"(a[9]), "=r"(a[10]), "=r"(a[11]), "=r"(a[12]), "=r"(a[13]), "=r"(a[14]), "=r"(a[15])
      : "r"(taddr)
      : "memory");
}

struct MaxOp {
  __device__ float operator()(float a, float b) const { return fmaxf(a, b); }
};
struct AddOp {
  __device__ float operator()(float a, float b) const { return a + b; }
};

// Four e4m3 codes (little-endian in w) as four bf16 values, exactly.
__device__ __forceinline__ uint2 e4m3x4_to_bf16x4(uint32_t w) {
  const __half2_raw lo = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)(w & 0xffffu), __NV_E4M3);
  const __half2_raw hi = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)(w >> 16), __NV_E4M3);
  const float2 a = __half22float2(*reinterpret_cast<const __half2*>(&lo));
  const float2 b = __half22float2(*reinterpret_cast<const __half2*>(&hi));
  const __nv_bfloat162 x = __floats2bfloat162_rn(a.x, a.y);
  const __nv_bfloat162 y = __floats2bfloat162_rn(b.x, b.y);
  return make_uint2(*reinterpret_cast<const uint32_t*>(&x), *reinterpret_cast<const uint32_t*>(&y));
}

__device__ __forceinline__ uint32_t bf162_bits(__nv_bfloat162 v) { return *reinterpret_cast<uint32_t*>(&v); }

// Partial attention of (segment blockIdx.x, row blockIdx.y): per head the
// segment's max logit m, sum of exp(logit - m) l, and sum of exp(logit - m) x.
__global__ void __launch_bounds__(kPThreads) sparse_attn_partial_kernel(
    const float* __restrict__ q, const uint8_t* __restrict__ mem, int64_t row_stride, int n_mem,
    const int32_t* __restrict__ idx, const int32_t* __restrict__ count, int max_sel, int nseg,
    float* __restrict__ part_o, float* __restrict__ part_ml, uint64_t wait_ns) {
  extern __shared__ uint8_t smem_raw[];
  AttnMisc& S = *reinterpret_cast<AttnMisc*>(smem_raw);
  uint8_t* tiles = smem_raw + ((sizeof(AttnMisc) + 15) & ~15u);
  tiles += (1024u - (smem_u32(tiles) & 1023u)) & 1023u;
  uint8_t* sX = tiles;                                // [2][128 chunks][128 B]
  uint8_t* sQ = sX + kXBytes;                         // [3 pieces][2][32 heads][128 B]
  uint8_t* sP = sQ + kQPieces * kPieceBytes;          // [2 pieces][2][32 heads][128 B] (K = chunks)
  const int b = blockIdx.y, seg = blockIdx.x;
  const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
  const int cnt = max(0, min(__ldg(count + b), max_sel));
  const int c0 = seg * kSeg;
  const int nc = max(0, min(kSeg, cnt - c0));
  float* po = part_o + ((size_t)b * nseg + seg) * kAH * kAD;
  float* pml = part_ml + ((size_t)b * nseg + seg) * kAH * 2;
  if (nc == 0) {  // an empty segment: nothing to merge
    if (t < kAH) {
      pml[2 * t] = -INFINITY;
      pml[2 * t + 1] = 0.f;
    }
    return;
  }
  if (t == 0) {
    mbar_init(&S.bar, 1);
    S.abort = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 0) {
    tmem_alloc(&S.tmem, kTmemCols);
    tmem_relinquish();
  }
  // loads first, so the query's and the records' latencies overlap.
  // gather: warp w takes records w + 8k (k < 16); lane k < 16 holds record
  // k's index and scale, lane l moves the 4 codes l of every record
  uint32_t w[16];
  {
    const int ck = warp + 8 * (lane & 15);
    int id = -1;
    if (lane < 16 && ck < nc) {
      id = idx ? __ldg(idx + (size_t)b * max_sel + c0 + ck) : c0 + ck;  // no list: resident records in order
      if (id < 0 || id >= n_mem) id = -1;  // an index outside the memory counts as masked
    }
    const uint8_t* row = mem + (size_t)b * row_stride;
    if (lane < 16)
      S.scale[ck] = id >= 0 ? __ldg(reinterpret_cast<const float*>(row + (int64_t)id * kRecord + 128)) : 0.f;
    const uint32_t vmask = __ballot_sync(0xffffffffu, id >= 0);
    if (lane == 0) S.valid[warp] = vmask;
#pragma unroll
    for (int k = 0; k < 16; ++k) {
      const int idk = __shfl_sync(0xffffffffu, id, k);
      w[k] = idk >= 0 ? __ldg(reinterpret_cast<const uint32_t*>(row + (int64_t)idk * kRecord) + lane) : 0u;
    }
  }
  // the row's query split into three bf16 pieces: thread t takes head t / 8,
  // dims 16 (t % 8) .. +15 (32 bytes of one swizzled row per piece)
  {
    const int h = t >> 3, part = t & 7;
    const float4* src = reinterpret_cast<const float4*>(q + ((size_t)b * kAH + h) * kAD + 16 * part);
    float v[16];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float4 f = __ldg(src + i);
      v[4 * i] = f.x; v[4 * i + 1] = f.y; v[4 * i + 2] = f.z; v[4 * i + 3] = f.w;
    }
    uint32_t pc[kQPieces][8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float a = v[2 * i], c = v[2 * i + 1];
      const __nv_bfloat162 p0 = __floats2bfloat162_rn(a, c);
      const float2 f0 = __bfloat1622float2(p0);
      const float ra = a - f0.x, rc = c - f0.y;  // exact
      const __nv_bfloat162 p1 = __floats2bfloat162_rn(ra, rc);
      const float2 f1 = __bfloat1622float2(p1);
      const __nv_bfloat162 p2 = __floats2bfloat162_rn(ra - f1.x, rc - f1.y);
      pc[0][i] = bf162_bits(p0);
      pc[1][i] = bf162_bits(p1);
      pc[2][i] = bf162_bits(p2);
    }
    const uint32_t blk = (uint32_t)(part >> 2) * kPieceBlock;
    const uint32_t k0 = (uint32_t)(part & 3) * 16;
#pragma unroll
    for (int p = 0; p < kQPieces; ++p)
#pragma unroll
      for (int u = 0; u < 2; ++u)
        *reinterpret_cast<uint4*>(sQ + p * kPieceBytes + blk + sw_bf16(h, k0 + 8 * u)) =
            make_uint4(pc[p][4 * u], pc[p][4 * u + 1], pc[p][4 * u + 2], pc[p][4 * u + 3]);
  }
  {  // the records' codes as bf16, rows of the swizzled tile
    const uint32_t blk = (uint32_t)(lane >> 4) * kXBlock;
    const uint32_t k0 = (uint32_t)(lane & 15) * 4;
#pragma unroll
    for (int k = 0; k < 16; ++k) {
      const uint32_t c = (uint32_t)(warp + 8 * k);
      *reinterpret_cast<uint2*>(sX + blk + sw_bf16(c, k0)) = e4m3x4_to_bf16x4(w[k]);
    }
  }
  fence_proxy_async_smem();  // the tiles are read by the tensor core
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = S.tmem;
  const int quarter = warp & 3, hh = warp >> 2;  // TMEM lanes 32 quarter .., heads 16 hh ..
  const uint32_t lane_base = tmem + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(16 * hh);
  // QK^T: D1[c, h] = sum over pieces and dims of code[c, d] q_p[h, d]
  if (t == 0) {
    constexpr uint32_t idesc = idesc_bf16_f32(kSeg, kAH, false, false);
    const uint32_t x0 = smem_u32(sX), q0 = smem_u32(sQ);
    uint32_t acc = 0;
#pragma unroll
    for (int p = 0; p < kQPieces; ++p)
#pragma unroll
      for (int ks = 0; ks < kAD / 16; ++ks) {
        const uint32_t ko = (uint32_t)(ks & 3) * 32;
        umma_bf16_ss(tmem, sdesc_kmajor_sw128(x0 + (ks >> 2) * kXBlock + ko),
                     sdesc_kmajor_sw128(q0 + p * kPieceBytes + (ks >> 2) * kPieceBlock + ko), idesc, acc);
        acc = 1;
      }
    umma_commit(&S.bar);
  }
  bool ok = mbar_wait_bounded(&S.bar, 0, &S.abort, &g_attn_err, wait_ns);
  if (__syncthreads_and(ok)) {
    tc_fence_after();
    // logits (log2 units), per-head max and exp-sum over the segment: this
    // thread has chunk 32 quarter + lane, heads 16 hh .. +15
    const int c = quarter * 32 + lane;
    const bool valid = (S.valid[c & 7] >> (c >> 3)) & 1u;
    const float f = S.scale[c] * 0.12751743082459868f;  // scale * log2(e) / sqrt(128)
    float lg[16];
    {
      uint32_t r[16];
      tmem_ld16_wait(lane_base, r);
#pragma unroll
      for (int h = 0; h < 16; ++h) lg[h] = valid ? __uint_as_float(r[h]) * f : -INFINITY;
    }
    {
      float v[16];
#pragma unroll
      for (int h = 0; h < 16; ++h) v[h] = lg[h];
      const float x = reduce_scatter16(v, lane, MaxOp());
      if ((lane & 1) == 0) S.red[0][hh][quarter][lane >> 1] = x;
    }
    __syncthreads();
    if (t < kAH) {
      const float* r = S.red[0][t >> 4][0] + (t & 15);
      S.m[t] = fmaxf(fmaxf(r[0], r[16]), fmaxf(r[32], r[48]));
    }
    __syncthreads();
    float pr[16];
#pragma unroll
    for (int h = 0; h < 16; ++h) pr[h] = valid ? exp2f(lg[h] - S.m[16 * hh + h]) : 0.f;
    {
      float v[16];
#pragma unroll
      for (int h = 0; h < 16; ++h) v[h] = pr[h];
      const float x = reduce_scatter16(v, lane, AddOp());
      if ((lane & 1) == 0) S.red[1][hh][quarter][lane >> 1] = x;
    }
    // the output weights p * scale in two bf16 pieces, stored as [head][chunk]
    const float sc = valid ? S.scale[c] : 0.f;
    const uint32_t blk = (uint32_t)(c >> 6) * kPieceBlock;
#pragma unroll
    for (int h = 0; h < 16; ++h) {
      const float w = pr[h] * sc;
      const __nv_bfloat16 w0 = __float2bfloat16_rn(w);
      const __nv_bfloat16 w1 = __float2bfloat16_rn(w - __bfloat162float(w0));
      const uint32_t o = blk + sw_bf16((uint32_t)(16 * hh + h), (uint32_t)(c & 63));
      *reinterpret_cast<__nv_bfloat16*>(sP + o) = w0;
      *reinterpret_cast<__nv_bfloat16*>(sP + kPieceBytes + o) = w1;
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (t < kAH) {
      const float* r = S.red[1][t >> 4][0] + (t & 15);
      S.l[t] = (r[0] + r[16]) + (r[32] + r[48]);
    }
    // PV: D2[d, h] = sum over pieces and chunks of code[c, d] (p s)_p[h, c]
    if (t == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(kAD, kAH, true, false);
      const uint32_t x0 = smem_u32(sX), p0 = smem_u32(sP);
      uint32_t acc = 0;
#pragma unroll
      for (int p = 0; p < kPPieces; ++p)
#pragma unroll
        for (int ks = 0; ks < kSeg / 16; ++ks) {
          umma_bf16_ss(tmem + kAH, sdesc_mn_sw128(x0 + ks * 16 * 128, kXBlock, 1024),
                       sdesc_kmajor_sw128(p0 + p * kPieceBytes + (ks >> 2) * kPieceBlock + (ks & 3) * 32), idesc,
                       acc);
          acc = 1;
        }
      umma_commit(&S.bar);
    }
    ok = mbar_wait_bounded(&S.bar, 1, &S.abort, &g_attn_err, wait_ns);
    if (__syncthreads_and(ok)) {
      tc_fence_after();
      uint32_t r[16];
      tmem_ld16_wait(lane_base + kAH, r);  // dim 32 quarter + lane, heads 16 hh ..
      const int d = quarter * 32 + lane;
#pragma unroll
      for (int h = 0; h < 16; ++h) po[(size_t)(16 * hh + h) * kAD + d] = __uint_as_float(r[h]);
      if (t < kAH) {
        pml[2 * t] = S.m[t];
        pml[2 * t + 1] = S.l[t];
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// Merges the segments of (head blockIdx.x, row blockIdx.y), thread d one
// output dim: o = sum_s 2^(m_s - M) o_s / sum_s 2^(m_s - M) l_s (m in log2
// units).  Lane s of every warp takes segment s of each group of 32, so the
// group's 32 partial outputs are loaded at once.
__global__ void __launch_bounds__(kAD) sparse_attn_combine_kernel(const float* __restrict__ part_o,
                                                                  const float* __restrict__ part_ml, int nseg,
                                                                  float* __restrict__ out) {
  const int h = blockIdx.x, b = blockIdx.y, d = threadIdx.x, lane = d & 31;
  const float* pml = part_ml + (size_t)b * nseg * kAH * 2;
  const float* po = part_o + (size_t)b * nseg * kAH * kAD;
  const auto ml_at = [&](int s) {
    return s < nseg ? __ldg(reinterpret_cast<const float2*>(pml + ((size_t)s * kAH + h) * 2))
                    : make_float2(-INFINITY, 0.f);
  };
  const float2 ml0 = ml_at(lane);  // the first group's (m, l), kept for its merge
  float M = ml0.x;
  for (int s = lane + 32; s < nseg; s += 32) M = fmaxf(M, ml_at(s).x);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
  float num = 0.f, den = 0.f;
  if (M != -INFINITY) {
    for (int s0 = 0; s0 < nseg; s0 += 32) {
      const int s = s0 + lane;
      float w = 0.f;
      if (s < nseg) {
        const float2 ml = s0 == 0 ? ml0 : ml_at(s);
        if (ml.x != -INFINITY) {
          w = exp2f(ml.x - M);
          den = fmaf(w, ml.y, den);
        }
      }
      // an empty segment (weight 0) wrote no partial output: its slot is not read
      float wj[32], v[32];
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        wj[j] = __shfl_sync(0xffffffffu, w, j);
        v[j] = wj[j] != 0.f ? __ldg(po + ((size_t)(s0 + j) * kAH + h) * kAD + d) : 0.f;
      }
#pragma unroll
      for (int j = 0; j < 32; ++j) num = fmaf(wj[j], v[j], num);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) den += __shfl_xor_sync(0xffffffffu, den, o);
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

int take_attention_error() {
  int h = kDevErrNone;
  if (cudaMemcpyFromSymbol(&h, g_attn_err, sizeof(int)) != cudaSuccess) {
    cudaGetLastError();
    return kDevErrNone;
  }
  if (h != kDevErrNone) {
    const int zero = kDevErrNone;
    cudaMemcpyToSymbol(g_attn_err, &zero, sizeof(int));
  }
  return h;
}

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
  if (!q || !mem || !count || !out || !ws || B < 1 || B > 65535 || max_sel < 1 || n_mem < 1)
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
  if (fm_status s = smem_limit_once(smem_set, dev, sparse_attn_partial_kernel, (int)kAttnSmem)) return s;
  sparse_attn_partial_kernel<<<dim3(nseg, B), kPThreads, kAttnSmem, stream>>>(
      q, mem, row_stride_bytes, n_mem, idx, count, max_sel, nseg, part_o, part_ml, kWaitLimitNs);
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
