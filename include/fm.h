/*
 * fm.h -- C ABI of libfm, a B200 (sm_100a) implementation of the FlashMemory
 * DS-V4 retriever's hot path: the Memory Indexer that scores every
 * fp8-compressed CSA KV chunk against a decode token's indexer query for three
 * CSA layers (l10, l12, l20), ensembles the layers and selects a keep-mask.
 *
 * Source of the operations: the FlashMemory DS-V4 Retriever README
 * (libertywing/FlashMemory-Deepseek-V4, translated copy on
 * bittide.aicompass.dev): "Usage" (the calls and their shapes),
 * "compressed_k format" (the 132-byte record), "Architecture" (the query
 * chain and the score formula), "Joint checkpoint + ensemble" (max / mean),
 * and the decode-loop figure of "Toy inference reference" (top-K or
 * sigmoid > thresh keep-mask).
 *
 * Conventions shared by every call
 *   - Pointers marked "device" are CUDA device pointers owned by the caller;
 *     the library never frees them.  Pointers marked "host or device" may be
 *     either (copied with cudaMemcpyDefault).
 *   - Every call is asynchronous on `stream` (a cudaStream_t; NULL = the
 *     legacy default stream) and returns an fm_status.  Argument errors are
 *     detected on the host before anything is launched, and nothing is
 *     written in that case.  Errors raised inside a kernel (a bounded wait
 *     that ran out) are recorded in the context and reported by
 *     fm_sync_status.
 *   - No call allocates device memory except fm_create and fm_level2_create
 *     (and their destroy calls free).
 *     Calls on one context must not run concurrently on different streams:
 *     they share the context's packed-query workspace.
 *   - Shapes: L = n_layers (1..4), H = n_heads = 64, D = head_dim = 128,
 *     HID = hidden, R = q_lora_rank.  B rows (decode tokens), N chunks per row.
 *   - A keep mask is one byte per chunk, 0 or 1 (the layout of torch.bool).
 *     Entries past a row's valid length n_valid[b] score 0.0f and are never
 *     kept.
 */
#ifndef FM_H_
#define FM_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* cudaStream_t;

typedef int fm_status;
enum {
  FM_OK = 0,
  FM_ERR_INVALID_ARG = 1,  /* a size, pointer or option is out of range          */
  FM_ERR_ALIGNMENT = 2,    /* a pointer or stride breaks the alignment rule      */
  FM_ERR_UNSUPPORTED = 3,  /* shape the kernels are not built for                */
  FM_ERR_CUDA = 4,         /* a CUDA runtime call failed (see fm_last_cuda_error) */
  FM_ERR_OOM = 5,          /* cudaMalloc failed in fm_create                     */
  FM_ERR_DEVICE = 6        /* a kernel recorded an error (bounded wait ran out)  */
};

enum { FM_ENSEMBLE_MAX = 0, FM_ENSEMBLE_MEAN = 1 };

/* Model constants.  README "Architecture" fixes HEAD_DIM = 128, ROPE_DIM = 64,
 * base 160000, eps 1e-6 and hidden 4096; the hyper-parameter table that would
 * give Q_LORA_RANK and N_HEADS is missing from the pages, so they are inputs
 * (1024 and 64 in every shipped workload).  Supported: hidden % 128 == 0,
 * q_lora_rank % 128 == 0, n_heads == 64, head_dim == 128, rope_dim == 64,
 * 1 <= n_layers <= 4, 1 <= max_batch <= 4096, q_pieces in {2, 3}, cta_pairs in {0, 1}. */
typedef struct fm_config {
  int hidden;             /* 4096 */
  int q_lora_rank;        /* 1024 */
  int n_heads;            /* 64 */
  int head_dim;           /* 128 */
  int n_layers;           /* 3: l10, l12, l20 */
  int rope_dim;           /* 64: the last 64 dims of each head */
  double rope_base;       /* 160000 */
  double rope_factor;     /* YaRN scaling factor, 16 */
  double rope_orig_max_pos; /* YaRN original context, 65536 */
  double rope_beta_fast;  /* 32 */
  double rope_beta_slow;  /* 1 */
  float rms_eps;          /* 1e-6 */
  int max_batch;          /* largest B any call on this context will pass */
  int q_pieces;           /* e4m3 pieces per query element in the tensor-core
                             product: 2 (default; the residual piece stored
                             unscaled so the tensor core sums both into one
                             accumulator; query split error ~2^-8 relative,
                             scores within ~5e-4 on the shipped workloads) or
                             3 (~2^-12, ~1e-5; one accumulator per piece,
                             slower) */
  int cta_pairs;          /* scoring pass with q_pieces 2 and one key tensor
                             per layer: 0 (default) one CTA per SM issues its
                             own MMAs; 1 pairs of CTAs share each MMA
                             (tcgen05 cta_group::2, M = 256 chunks), which
                             halves the MMA instructions per SM but couples
                             the two SMs' key streams; same results.  Other
                             forms ignore it. */
} fm_config;

/* One layer's weights, fp32, row-major [out, in], no biases (README
 * "Architecture": wq_a 4096 -> Q_LORA_RANK, RMSNorm weight, wq_b
 * Q_LORA_RANK -> N_HEADS*HEAD_DIM, weights_proj 4096 -> N_HEADS).
 * Host or device pointers; fm_create copies them. */
typedef struct fm_layer_weights {
  const float* wq_a;         /* [R, HID]   */
  const float* q_norm;       /* [R]        */
  const float* wq_b;         /* [H*D, R]   */
  const float* weights_proj; /* [H, HID]   */
} fm_layer_weights;

typedef struct fm_ctx fm_ctx;

/* Fills *cfg with the shipped constants (hidden 4096, rank 1024, 64 heads,
 * head_dim 128, 3 layers, YaRN 160000/16/65536/32/1, eps 1e-6, max_batch 64,
 * q_pieces 2, cta_pairs 0). */
void fm_config_default(fm_config* cfg);

/* Creates a context on `device`: uploads the weights (cfg->n_layers entries of
 * `weights`) and allocates the packed-query workspace for cfg->max_batch rows.
 * Synchronous.  FM_ERR_INVALID_ARG / FM_ERR_UNSUPPORTED for a bad config,
 * FM_ERR_OOM, FM_ERR_CUDA.  *out is NULL on failure. */
fm_status fm_create(const fm_config* cfg, const fm_layer_weights* weights, int device,
                    fm_ctx** out);

/* Frees everything fm_create allocated (synchronises the device first). */
fm_status fm_destroy(fm_ctx* ctx);

/* Query side of every layer (README "Architecture", upper two chains):
 *   q[b,l]       = Hadamard(RoPE_YaRN(reshape(wq_b . RMSNorm(wq_a . hidden[b]))))
 *   fused_w[b,l] = (weights_proj . hidden[b]) * HEAD_DIM^-1/2 * N_HEADS^-1/2
 * hidden    [B, HID] fp32 device, row-major.
 * positions [B] int64 device (token position of each row, >= 0).
 * q         [B, L, H, D] fp32 device (written).
 * fused_w   [B, L, H] fp32 device (written).
 * 1 <= B <= max_batch.  All fp32 arithmetic; the RoPE angles pos * f_j and
 * their cos/sin are taken in fp64 and rounded once. */
fm_status fm_query_prep(fm_ctx* ctx, const float* hidden, const int64_t* positions, int B,
                        float* q, float* fused_w, cudaStream_t stream);

/* Per-layer chunk scores (README "Architecture", score line):
 *   scores[l,b,n] = sigmoid( sum_h relu(k[l,b,n] . q[b,l,h]) * fused_w[b,l,h] )
 *   k[l,b,n]      = e4m3(comp_k[l][b,n,0:128]) * f32le(comp_k[l][b,n,128:132])
 * comp_k    array of L device pointers (host array); layer l's keys are
 *           [B, N_pad, 132] uint8 with row b starting at
 *           comp_k[l] + b * row_stride_bytes.  Each pointer 16-byte aligned,
 *           row_stride_bytes a multiple of 16 and >= N * 132 rounded up to a
 *           multiple of 528 (i.e. N_pad >= N rounded up to 4) -- the tile
 *           copy reads whole 4-record groups.  Otherwise FM_ERR_ALIGNMENT.
 * n_valid   [B] int32 device, 0 <= n_valid[b] <= N, or NULL (= N for all).
 * q, fused_w as written by fm_query_prep (any producer is fine).
 * scores    [L, B, N] fp32 device (written; 0.0f past n_valid).
 * The product k.q runs on the tensor cores with q split into q_pieces e4m3
 * terms (per-head power-of-two scaling) and the keys used as stored.
 * The comp_k pointers may alias.  All layers reading one key tensor is the
 * README "Usage" signature taken literally (one compressed_k scored by the
 * three layers' queries): when every layer's pointer is the same, the pass
 * copies each 128-chunk key tile once and runs every layer's product from it. */
fm_status fm_score(fm_ctx* ctx, const uint8_t* const* comp_k, int64_t row_stride_bytes,
                   const int32_t* n_valid, int B, int N, const float* q, const float* fused_w,
                   float* scores, cudaStream_t stream);

/* Cross-layer ensemble (README "Joint checkpoint + ensemble"):
 *   mode FM_ENSEMBLE_MAX:  ens[b,n] = max_l scores[l,b,n]   (union, default)
 *   mode FM_ENSEMBLE_MEAN: ens[b,n] = (((s0 + s1) + s2) ...) / L   in fp32
 * scores [L, B, N] fp32 device; ens [B, N] fp32 device (written). */
fm_status fm_ensemble(const float* scores, int L, int B, int N, int mode, float* ens,
                      cudaStream_t stream);

/* One pass that scores all L layers, ensembles them and (optionally) applies
 * the threshold rule, writing one fp32 per chunk instead of L.
 * Inputs as fm_score.  mode as fm_ensemble.
 * scores_or_null [L, B, N] fp32 device or NULL (per-layer scores not written).
 * ens            [B, N] fp32 device (written).
 * keep_thr_or_null [B, N] uint8 device or NULL: keep = (ens > thr) for valid
 *                chunks (strict, README toy loop "sigmoid > thresh"); thr is
 *                ignored when this pointer is NULL. */
fm_status fm_score_fused(fm_ctx* ctx, const uint8_t* const* comp_k, int64_t row_stride_bytes,
                         const int32_t* n_valid, int B, int N, const float* q,
                         const float* fused_w, int mode, float thr, float* scores_or_null,
                         float* ens, uint8_t* keep_thr_or_null, cudaStream_t stream);

/* Bytes of device workspace fm_select_topk needs for B rows of N chunks. */
size_t fm_topk_workspace_bytes(int B, int N);

/* Bytes of workspace with which fm_select_topk can take its candidate path
 * on rows of more than 16384 chunks (shorter rows take the one-kernel form
 * described at fm_select_topk):
 * a threshold from a sample of each row, one pass that lists the scores above
 * it, and the selection among those in shared memory, instead of three
 * histogram passes and a mask pass over all scores.  The mask is the same
 * (exact) either way; a row the candidate list cannot finish (too few or too
 * many candidates, or the K-th value tied with values not kept) is selected
 * by one CTA over the whole row, ties in chunk order.  Taken when the
 * workspace given is at least this large and
 * 2k + 1024 <= min(16384, max(256, N / 16)). */
size_t fm_topk_workspace_bytes_fast(int B, int N);

/* Top-K keep mask (README "Usage" select_topk(top_k=K); toy loop "top-K"):
 * keep[b,n] = 1 for the min(k, n_b) largest ens[b, 0:n_b], equal scores taken
 * in increasing chunk index; 0 elsewhere.  Scores must be >= 0 (sigmoid
 * outputs); NaN ranks below every number.
 * ens [B, N] fp32 device; n_valid [B] int32 device or NULL; k >= 1;
 * keep [B, N] uint8 device (written);
 * ws device workspace of at least fm_topk_workspace_bytes(B, N) bytes (the
 * faster candidate path needs fm_topk_workspace_bytes_fast(B, N)), 16-byte
 * aligned, owned by the caller; its contents on entry do not matter.
 * Rows of up to 16384 chunks are selected by one kernel, one CTA per row
 * holding the row's keys in shared memory; it leaves the workspace
 * untouched.  Longer rows take the candidate path or the histogram passes. */
fm_status fm_select_topk(const float* ens, const int32_t* n_valid, int B, int N, int k,
                         uint8_t* keep, void* ws, size_t ws_bytes, cudaStream_t stream);

/* Size of the scratch array fm_select_topk_static uses: 4 MiB, compiled into
 * the library, one per GPU that loads it, held until the process exits.  It
 * covers fm_topk_workspace_bytes(B, N) up to about 200 rows of 262144 chunks. */
#define FM_TOPK_STATIC_SCRATCH_BYTES (4u << 20)

/* fm_select_topk for callers that cannot allocate device memory: the same
 * keep mask, with the scratch taken from a fixed array inside the library
 * instead of a caller workspace.  The README's interface has no counterpart;
 * this is an integration entry point.  Callers that need it: a serving process whose
 * device memory is all handed to its KV-cache pool at start-up, a plugin that
 * must leave device memory to its host framework's allocator, a decode loop
 * that cannot afford the device synchronisation cudaMalloc/cudaFree may cause.
 * Allocates nothing; the caller passes inputs and outputs as for
 * fm_select_topk (ens, n_valid, keep: device; same shapes and rules).
 * Runs on the calling thread's current device, which must own `stream`; the
 * first call on each device looks up the array's device address (with
 * cudaGetSymbolAddress) and caches it, so make that first call before any
 * stream capture.  Every call on a device shares the one array and the call's
 * first kernel re-initialises what it uses: calls whose kernels overlap on the
 * GPU (different streams or threads) race and give wrong masks; order them.
 * Rows of up to 16384 chunks take fm_select_topk's one-kernel form, which
 * uses none of the array; longer rows take its candidate path when the array
 * also holds the candidate lists (fm_topk_workspace_bytes_fast(B, N) <=
 * FM_TOPK_STATIC_SCRATCH_BYTES, and the rule on k given there), otherwise the
 * histogram form; the mask is the same either way.
 * Returns FM_ERR_UNSUPPORTED, launching nothing, when
 * fm_topk_workspace_bytes(B, N) > FM_TOPK_STATIC_SCRATCH_BYTES. */
fm_status fm_select_topk_static(const float* ens, const int32_t* n_valid, int B, int N, int k,
                                uint8_t* keep, cudaStream_t stream);

/* ------------------------------------------------- whole path from host memory
 * README "Usage" composed for a caller whose inputs live in host memory: the
 * inputs are copied to device staging buffers, the path runs (fm_query_prep,
 * fm_score_fused, fm_select_topk), and the masks are copied back. */
typedef struct fm_host_batch {
  int B;                      /* rows, 1..max_batch */
  int N;                      /* chunks per row */
  const float* hidden;        /* [B, HID] fp32 host */
  const int64_t* positions;   /* [B] int64 host */
  const uint8_t* comp_k[4];   /* per layer (n_layers used): [B, N_pad, 132] host, row b at
                                 comp_k[l] + b * row_stride_bytes */
  int64_t row_stride_bytes;   /* as fm_score (a multiple of 16, >= ceil4(N) * 132) */
  const int32_t* n_valid;     /* [B] int32 host, or NULL (= N for all) */
  int mode;                   /* FM_ENSEMBLE_MAX or FM_ENSEMBLE_MEAN */
  int top_k;                  /* >= 1 with keep_topk, else ignored */
  float thr;                  /* threshold, used with keep_thr */
  uint8_t* keep_topk;         /* [B, N] host (written) or NULL: the top-K mask */
  uint8_t* keep_thr;          /* [B, N] host (written) or NULL: the threshold mask */
} fm_host_batch;

/* Device buffers the call stages through, owned by the caller (the call
 * allocates nothing).  Sizes for the batch's B and N: */
typedef struct fm_device_staging {
  uint8_t* comp_k[4];         /* per layer, B * row_stride_bytes bytes, 16-byte aligned */
  float* hidden;              /* [B, HID], 16-byte aligned */
  int64_t* positions;         /* [B] */
  int32_t* n_valid;           /* [B] (used when the batch has n_valid) */
  float* q;                   /* [B, L, H, D], 16-byte aligned */
  float* fused_w;             /* [B, L, H] */
  float* ens;                 /* [B, N] */
  uint8_t* keep_topk;         /* [B, N] (used with keep_topk) */
  uint8_t* keep_thr;          /* [B, N] (used with keep_thr) */
  void* topk_ws;              /* fm_topk_workspace_bytes(B, N) bytes or more (the candidate path
                                 takes fm_topk_workspace_bytes_fast), 16-byte aligned */
  size_t topk_ws_bytes;
} fm_device_staging;

/* The whole path for one batch in host memory, asynchronous on `stream`: one
 * cudaMemcpyAsync per input buffer (host to the staging buffers), query prep,
 * the fused scoring pass with the ensemble and the threshold mask, top-K,
 * then one cudaMemcpyAsync per requested mask back to the host.  The host
 * masks hold their values once `stream` has reached the end of the call
 * (fm_sync_status waits for it); the host inputs must stay unchanged until
 * then.  Pinned host memory (cudaHostAlloc) keeps the copies asynchronous;
 * pageable memory works, with the runtime staging the copies.  Argument and
 * alignment errors are reported before anything is copied. */
fm_status fm_retrieve_host(fm_ctx* ctx, const fm_host_batch* batch, const fm_device_staging* dev,
                           cudaStream_t stream);

/* Threshold keep mask (README "Usage" select_topk(threshold=t)):
 * keep[b,n] = (n < n_b) && (ens[b,n] > thr).  Shapes as fm_select_topk. */
fm_status fm_select_threshold(const float* ens, const int32_t* n_valid, int B, int N, float thr,
                              uint8_t* keep, cudaStream_t stream);

/* Sharded top-K: the keep mask of fm_select_topk (README "Usage"
 * select_topk(top_k=K)) for rows whose chunks are split over G shards (GPUs),
 * shard g holding a consecutive slice of each row, slices in shard order.  The
 * pages describe no multi-GPU form of the retriever; this is the same mask,
 * computed without moving scores between shards: the caller runs the phases
 * below on every shard in the same order and does the two exchanges between
 * them (with NCCL or any other collective library):
 *
 *   fm_topk_shard_begin(n_valid_local, B, N, k, hist, ws, ...)
 *   for pass in 0, 1, 2:
 *     fm_topk_shard_hist(ens_local, B, N, pass, hist, ws, ...)
 *     all-reduce (sum) `hist` over the shards            -- exchange 1
 *     fm_topk_shard_pick(B, N, pass, hist, ws, ...)
 *   fm_topk_shard_ties(ens_local, B, N, eq_local, ws, ...)
 *   all-gather `eq_local` into eq_all [G, B], shard order -- exchange 2
 *   fm_topk_shard_mask(ens_local, B, N, eq_all, g, keep_local, ws, ...)
 *
 * After it, the union of the shards' masks keeps, per row, the min(k, total
 * valid) largest scores of the whole row, equal scores in increasing global
 * chunk index, exactly as fm_select_topk on the concatenated row would.
 * Every shard passes the same B and k; N (its slice length) may differ.
 * ens_local [B, N] fp32 device: this shard's slice; n_valid_local [B] int32
 * device or NULL (= N): valid chunks in this slice (a row's valid prefix
 * split over the slices: clamp(n_b - slice_start, 0, N));
 * hist [B, FM_TOPK_SHARD_BINS] int32 device, 16-byte aligned, owned by the
 * caller, written by begin and pick, summed in place by the caller;
 * eq_local [B] int32 device; eq_all [G, B] int32 device; keep_local [B, N]
 * uint8 device; ws: this shard's workspace of fm_topk_workspace_bytes(B, N)
 * bytes, 16-byte aligned, kept between the phases.  Exchange sizes: 8 KiB
 * per row per pass, 4 bytes per row for the ties. */
#define FM_TOPK_SHARD_BINS 2048
fm_status fm_topk_shard_begin(const int32_t* n_valid_local, int B, int N, int k, int32_t* hist,
                              void* ws, size_t ws_bytes, cudaStream_t stream);
fm_status fm_topk_shard_hist(const float* ens_local, int B, int N, int pass, int32_t* hist, void* ws,
                             size_t ws_bytes, cudaStream_t stream);
fm_status fm_topk_shard_pick(int B, int N, int pass, int32_t* hist, void* ws, size_t ws_bytes,
                             cudaStream_t stream);
fm_status fm_topk_shard_ties(const float* ens_local, int B, int N, int32_t* eq_local, void* ws,
                             size_t ws_bytes, cudaStream_t stream);
fm_status fm_topk_shard_mask(const float* ens_local, int B, int N, const int32_t* eq_all, int shard,
                             uint8_t* keep_local, void* ws, size_t ws_bytes, cudaStream_t stream);

/* ----------------------------------------------------------------- recall
 * The model card's "How it works" (Level 1): the chunks the Memory Indexer
 * selects form a resident set recalled from the CPU-side bulk KV cache to the
 * GPU.  These two calls turn a keep mask into that set. */

/* Bytes of device workspace fm_compact_mask needs for B rows of N chunks. */
size_t fm_compact_workspace_bytes(int B, int N);

/* Keep mask -> index list.  keep [B, N] uint8 device (nonzero = kept);
 * idx [B, max_sel] int32 device (written): the kept chunk indices of row b in
 * increasing order in idx[b, 0:min(count[b], max_sel)], -1 after them;
 * count [B] int32 device (written): the number of kept chunks of row b (it
 * may exceed max_sel; then only the first max_sel indices are listed);
 * ws: fm_compact_workspace_bytes(B, N) bytes, 16-byte aligned, caller-owned,
 * contents on entry irrelevant.  idx and count 4-byte aligned. */
fm_status fm_compact_mask(const uint8_t* keep, int B, int N, int max_sel, int32_t* idx, int32_t* count,
                          void* ws, size_t ws_bytes, cudaStream_t stream);

/* Gathers the selected chunks' records into a resident buffer (the model
 * card's "How it works": the resident set recalled to the GPU):
 * for every row b and j < min(count[b], max_sel) with 0 <= idx[b, j] < n_src,
 *   dst[b*dst_row_stride + j*rec_bytes, +rec_bytes) =
 *   src[b*src_row_stride + idx[b, j]*rec_bytes, +rec_bytes).
 * Other slots of dst are not written.  src: the bulk store of fixed-size
 * records (n_src per row), in device memory or in pinned host memory
 * (cudaHostAlloc / torch pin_memory; read over the bus by the kernel);
 * pageable host memory is rejected with FM_ERR_INVALID_ARG.  dst: device
 * memory.  idx, count as written by fm_compact_mask (device).  Any record
 * size.  From device memory, records of 64 B or more whose pointers, strides
 * and size are multiples of 4 move by bulk copies staged in shared memory
 * (each copy covers the 16-byte granules of its record); otherwise 16-byte
 * loads and stores when both pointers, the strides and rec_bytes are
 * multiples of 16, 4-byte ones when of 4, else byte copies. */
fm_status fm_gather_records(const void* src, int64_t src_row_stride_bytes, int n_src, int64_t rec_bytes,
                            const int32_t* idx, const int32_t* count, int B, int max_sel, void* dst,
                            int64_t dst_row_stride_bytes, cudaStream_t stream);

/* ---------------------------------------------------------------- Level 2
 * The model card's "How it works", Level 2: at every decode step a top-512
 * confined to the resident set, run inside a CUDA graph.  DS-V4's own Level-2
 * indexer is not described by the pages; this step runs this library's stages
 * on the resident chunks: query prep for the step's hidden states, fused
 * scoring of the R resident records of every layer with the ensemble, top-k
 * of the ensembled scores (ties to the lower resident slot, which is the
 * lower chunk id), and the mapping of the kept slots to chunk ids. */
typedef struct fm_level2 fm_level2;

typedef struct fm_level2_desc {
  const float* hidden;             /* [B, HID] fp32 device, 16-byte aligned: read at every launch */
  const int64_t* positions;        /* [B] int64 device: read at every launch */
  const uint8_t* resident_keys[4]; /* per layer (n_layers used): [B, R, 132] device, 16-byte aligned;
                                      the resident chunks' compressed_k records (fm_gather_records) */
  const int32_t* resident_ids;     /* [B, R] int32 device: chunk id of each resident slot, ascending
                                      (fm_compact_mask's idx) */
  const int32_t* resident_count;   /* [B] int32 device: resident chunks per row (clamped to R) */
  int B;                           /* rows, 1..max_batch of the context */
  int R;                           /* resident slots per row, a multiple of 4 */
  int k;                           /* chunks selected per row, 1..R (512 in the model card) */
  int mode;                        /* FM_ENSEMBLE_MAX or FM_ENSEMBLE_MEAN */
  int32_t* out_ids;                /* [B, k] int32 device, written at every launch: the selected chunk
                                      ids, ascending, -1 past the row's count */
  int32_t* out_count;              /* [B] int32 device or NULL: min(k, resident_count[b]) */
} fm_level2_desc;

/* Builds the step for the buffers of `d` (the pointers are kept; the contents
 * are read at every launch): allocates its intermediates (q, fused_w, scores,
 * mask, index lists and workspaces; one of the two calls besides fm_create
 * that allocate device memory), runs the step once on `stream` (synchronous),
 * then captures the same launches into a CUDA graph.  The step uses the
 * context's packed-query workspace: no other call on `ctx` may run while a
 * launch is in flight.  *out is NULL on failure. */
fm_status fm_level2_create(fm_ctx* ctx, const fm_level2_desc* d, cudaStream_t stream, fm_level2** out);

/* Runs one step (one graph launch) on `stream`. */
fm_status fm_level2_launch(fm_level2* step, cudaStream_t stream);

/* Copies the ensembled scores [B, R] of the last step (fp32) into dst (device),
 * on `stream`. */
fm_status fm_level2_copy_scores(const fm_level2* step, float* dst, cudaStream_t stream);

/* Waits for the device and frees the step. */
fm_status fm_level2_destroy(fm_level2* step);

/* ------------------------------------------------------- toy sparse decode
 * README "Toy inference reference": every decode step runs a sparse memory
 * attention over the N compressed chunks in which the chunks the last
 * retrieval did not keep get -inf logits; every 64 steps the retriever
 * refreshes the keep mask.  The toy decoder is not defined by the pages; these
 * calls take the plainest weight-free reading:
 *   query   the step's hidden state [4096] as 32 heads of 128 (q [B, 32, 128]);
 *   memory  chunk i's vector x_i = e4m3(bytes[0:128]) * f32le(bytes[128:132]),
 *           used as key and value;
 *   o_h     = sum_i softmax_i(q_h . x_i / sqrt(128)) x_i over the kept chunks
 *           (the others' logits are -inf); a row with no kept chunk gives 0;
 *   update  hidden' = RMSNorm(hidden + o), no gain. */

/* Bytes of device workspace fm_decode_attention needs. */
size_t fm_decode_attention_workspace_bytes(int B, int max_sel);

/* The sparse attention, reading only the kept chunks: idx/count as written by
 * fm_compact_mask for the keep mask (the first min(count[b], max_sel) entries
 * of idx[b] are the kept chunk indices; an index outside [0, n_mem) counts as
 * masked).  idx NULL: the resident form, in which row b of mem holds the kept
 * records themselves in increasing chunk order (fm_gather_records with the
 * same idx/count), and record j < min(count[b], max_sel, n_mem) is used.  q [B, 32, 128] fp32 device, 16-byte aligned; mem: the chunk
 * records [B, n_mem, 132] uint8 device, row b at mem + b*row_stride_bytes
 * (4-byte aligned, row_stride_bytes >= n_mem*132, a multiple of 4);
 * out [B, 32, 128] fp32 device (written); ws: the workspace, 16-byte aligned. */
fm_status fm_decode_attention(const float* q, const uint8_t* mem, int64_t row_stride_bytes, int n_mem,
                              const int32_t* idx, const int32_t* count, int B, int max_sel, float* out,
                              void* ws, size_t ws_bytes, cudaStream_t stream);

/* The toy decoder's state update: hidden_out[b] = RMSNorm(hidden[b] + attn_out[b])
 * with eps and no gain; H = 4096 (the attention output flattened head-major).
 * All [B, H] fp32 device; hidden_out may alias hidden. */
fm_status fm_toy_decoder_update(const float* hidden, const float* attn_out, int B, int H, float eps,
                                float* hidden_out, cudaStream_t stream);

/* Synchronises `stream` and returns FM_ERR_DEVICE if a kernel launched on this
 * context recorded an error since the last call (the record is cleared), or
 * if one of the context-free kernels of the current device did (decode
 * attention, compaction, gather: a bounded wait that ran out), FM_ERR_CUDA
 * if the stream reports a CUDA error, FM_OK otherwise. */
fm_status fm_sync_status(fm_ctx* ctx, cudaStream_t stream);

/* Static text for a status code. */
const char* fm_strerror(fm_status status);

/* The last CUDA runtime error code seen by any call of this thread (0 = none). */
int fm_last_cuda_error(void);

/* Number of kernel launches issued by this process since load (all calls). */
uint64_t fm_launch_count(void);

/* ---------------------------------------------------- failure-path test hooks
 * The pages have no counterpart; these exist so that tests can drive the
 * library's error paths without faulting or hanging a GPU. */

/* Makes the n-th device allocation from now (n >= 1, counted over all threads)
 * made by fm_create or fm_level2_create fail as an out-of-memory cudaMalloc
 * would; those calls then free what they had allocated and return
 * FM_ERR_OOM.  n <= 0 turns the hook off. */
void fm_debug_fail_alloc(int n);

/* Number of device allocations currently held by live contexts and Level-2
 * steps (what fm_destroy / fm_level2_destroy will free). */
int64_t fm_debug_live_allocations(void);

/* The next scoring launch on `ctx` (fm_score, fm_score_fused) never loads its
 * query operand and bounds each of its waits by wait_limit_ns (1 ..
 * 2e9 ns) instead of the usual 2 s: the wait for the query runs out, the
 * kernel's roles stop at their next wait, copies already in flight land, and
 * the launch ends with the context's error word set.  fm_sync_status then
 * returns FM_ERR_DEVICE and clears it; the context stays usable.  No result
 * of that launch is valid.  Call it only on a context no other thread uses. */
fm_status fm_debug_stall_next_score(fm_ctx* ctx, uint64_t wait_limit_ns);

/* Diagnostic: the raw tensor-core dot products of one 128-chunk tile of layer
 * `layer`, row b, tile t (chunks t*128 .. t*128+127), before the per-chunk
 * scale, the per-head power-of-two scale and the epilogue.  With q_pieces = 3:
 *   out[r, p*64 + h] = sum_d e4m3(comp_k[layer][b, t*128 + r, d]) * piece_p(q[b,layer,h])[d]
 * for p < 3, the pieces satisfying q[b,layer,h,d] ~= 2^-pow2_exp[h] * sum_p 16^-p * piece_p[d].
 * With q_pieces = 2 the tensor core adds the two pieces in one accumulator:
 *   out[r, h] = sum_d e4m3(comp_k[layer][b, t*128 + r, d]) * (piece_0 + piece_1)(q[b,layer,h])[d]
 * with q[b,layer,h,d] ~= 2^-pow2_exp[h] * (piece_0[d] + piece_1[d]) (piece 1 the
 * unscaled e4m3 residual); out[r, 64:] is left untouched.
 * out [128, 192] fp32 device (the entries above written, the rest untouched),
 * pow2_exp [64] int32 device (written).  Rows of the tile past N
 * hold unspecified values.  Used by the
 * tests to check the tensor-core operand layouts in isolation. */
fm_status fm_debug_tile_dots(fm_ctx* ctx, const uint8_t* const* comp_k, int64_t row_stride_bytes,
                             int B, int N, const float* q, const float* fused_w, int layer, int b,
                             int t, float* out, int32_t* pow2_exp, cudaStream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* FM_H_ */
