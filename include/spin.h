/*
 * spin.h -- C ABI of libspin.so, the SPIN (Shadow Predictive Indexer) decode
 * step on NVIDIA B200 (sm_100a).
 *
 * SPIN predicts which paged-KV blocks the indexer of a DSA-style sparse
 * attention layer will find important, scores only those blocks, takes the
 * token top-k for core attention and keeps the predictor's history fresh.
 * Sources, cited by page and section:
 *   SPIN digest   -- ai4snews digest "SPIN用历史索引分数预测KV块重要性..." (核心概要,
 *                    arXiv深度剖析, 启示与展望)
 *   SPIN listing  -- thelatestinai listing "SaveSPIN: Shadow Predictive Indexer
 *                    for Sparse Attention" (Abstract, Figures 1-4, Tables 1-7)
 *   SPIN v3 record-- paperdot record of arXiv:2610.09025 v3 (摘要)
 *   AI Radio      -- AI Radio episode "SPIN: Shadow Predictive Indexer for
 *                    Sparse Attention" ("Title and authors", "The paper's summary")
 * The indexer formula is the DSA lightning indexer
 *   I_{r,s} = sigma_s * sum_h w_{r,h} * ReLU(q_{r,h} . k8_s).
 *
 * Conventions (every call):
 *  - Device pointers are owned by the caller (allocate them with any CUDA
 *    allocator, e.g. PyTorch).  Pointers documented as *_host are host memory.
 *  - Every call is asynchronous on the given stream and never synchronises,
 *    except spin_get_error and the export / import calls.  No call allocates
 *    device memory: all scratch lives in the block handed to spin_state_create.
 *  - Argument errors are reported synchronously through the return value and
 *    launch nothing.  Errors only visible on the device (a ctx_len past the
 *    capacity, a page id outside the cache, an accepted length outside 1..rows,
 *    a bounded wait that gave up, a ctx_len other than a prepared selection's)
 *    set a device error word and skip the affected work; they never trap.
 *    spin_get_error reads and clears it.
 *  - Results are deterministic for a given (seed, step, inputs).
 *  - A state is not thread-safe; use it from one stream at a time.
 *
 * Positions: ctx_len[q] is the number of slots visible to query row 0 of
 * request q, including that row's own key (already in the cache).  Row r
 * (MTP verification rows, r < rows) sits at position p_r = ctx_len - 1 + r
 * and sees slots 0..p_r.  Logical block j holds slots j*b .. j*b + b - 1.
 */
#ifndef SPIN_H_
#define SPIN_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define SPIN_API __attribute__((visibility("default")))
#else
#define SPIN_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t; NULL is the legacy default stream. */
typedef struct CUstream_st* spin_stream_t;

typedef enum {
  SPIN_OK = 0,
  SPIN_EINVAL = 1,       /* bad argument; nothing was launched */
  SPIN_ENOMEM = 2,       /* the caller's state block is smaller than spin_state_bytes() */
  SPIN_ECUDA = 3,        /* a CUDA runtime call failed */
  SPIN_ESTATE = 4,       /* NULL or destroyed state handle */
  SPIN_ETIMEOUT = 5,     /* a device-side bounded wait gave up (device error word) */
  SPIN_EDEVICE = 6,      /* a device-side argument check failed (device error word) */
  SPIN_EUNSUPPORTED = 7  /* shape not supported by the requested kernel */
} spin_status;

typedef enum { SPIN_F32 = 0, SPIN_BF16 = 1, SPIN_FP8_E4M3 = 2 } spin_dtype;

/* Score kernel choice (spin_set_score_kernel). */
typedef enum {
  SPIN_SCORE_AUTO = 0,   /* tcgen05 when the shape allows it, else SIMT */
  SPIN_SCORE_SIMT = 1,   /* CUDA-core kernel: any supported shape, fp32 or FP8 keys */
  SPIN_SCORE_TCGEN05 = 2 /* TMA + tcgen05 FP8 MMA with TMEM accumulators:
                            FP8 keys, head_dim 128, block_size 64,
                            rows * num_heads a multiple of 16 and <= 256 */
} spin_score_kernel;

typedef struct {
  int32_t num_layers;      /* EMA states kept per layer */
  int32_t num_requests;    /* Q: request slots */
  int32_t max_slots;       /* KV capacity per request (slots) */
  int32_t block_size;      /* b: paged-KV block size (AI Radio, "Title and authors") */
  int32_t num_heads;       /* H: indexer heads */
  int32_t head_dim;        /* d: indexer key / query width */
  int32_t topk;            /* k: tokens handed to core attention */
  int32_t max_rows;        /* 1..4 query rows per step (1 verify + drafts) */
  int32_t key_dtype;       /* SPIN_F32 or SPIN_FP8_E4M3 (+ per-token fp32 scale) */
  int32_t q_dtype;         /* SPIN_F32 or SPIN_BF16 (SPIN_F32 keys need SPIN_F32 queries) */
  float alpha;             /* EMA decay: x <- alpha*x + (1-alpha)*score */
  float gamma;             /* exploration share of the block budget (SPIN listing, Figure 4) */
  float target_sparsity;   /* default per-layer target block sparsity, [0, 1) */
  uint64_t seed;           /* exploration RNG seed (Philox4x32-10 key) */
  int32_t pooling;         /* block reduction of the predicted slot scores: spin_pooling */
  int32_t mtp_policy;      /* mask and EMA policy for several query rows: spin_mtp_policy */
} spin_config;

/* Block reduction of the predicted slot scores z into a block score (SPIN
 * listing, Figure 3 compares Max, the method's, with Mean and Top-4 pooling;
 * the pages do not define the latter two).  Over a block's visible slots:
 *   SPIN_POOL_MAX   the largest z;
 *   SPIN_POOL_MEAN  the mean of z;
 *   SPIN_POOL_TOP4  the mean of the min(4, count) largest z.
 * Mean and Top-4 are computed in double and rounded once to float, in a
 * fixed order (runs of 8 consecutive slots summed in slot order, then the
 * runs added pairwise; the Top-4 values from the largest down), so the
 * result does not depend on the launch. */
typedef enum { SPIN_POOL_MAX = 0, SPIN_POOL_MEAN = 1, SPIN_POOL_TOP4 = 2 } spin_pooling;

/* Policy for steps with several query rows (MTP verification; SPIN listing,
 * Table 7 and Figure 2 compare the two).
 *   SPIN_MTP_UNION_PREFIX  the method's: each row predicts with its own
 *     budget, the kept mask is the union, and the EMA update replays the
 *     accepted prefix rows 0..a-1 in order.
 *   SPIN_MTP_ROW0  the baseline: row 0 alone predicts (its budget, and the
 *     exploration share of it drawn among row 0's unkept blocks) and every
 *     row uses that mask; blocks past row 0's range, which hold only the new
 *     keys of this step's drafts, are kept (label 1).  The EMA update uses
 *     row 0's scores alone, whatever the accepted length.
 * With one row the two are the same. */
typedef enum { SPIN_MTP_UNION_PREFIX = 0, SPIN_MTP_ROW0 = 1 } spin_mtp_policy;

typedef struct spin_state_s* spin_state;

/* Bytes of device memory a state needs: EMA states V and D for every layer
 * and request (with max pooling and block_size >= 32 also V's maximum over
 * each aligned 32-slot group, which the prediction reads in place of V for
 * the blocks below the newest one), block-score / work-list / quantised-query / score scratch, the
 * per-layer selection a pipelined step prepares (spin_set_lookahead), a
 * block-score scratch (as large as the one above) for each of
 * min(num_layers, 8) streams of spin_prepare_selections, and the device
 * error word.  Returns 0 for an
 * invalid config. */
SPIN_API size_t spin_state_bytes(const spin_config* cfg);

/* Creates a state in the caller's device block dev_mem (>= spin_state_bytes,
 * 256-byte aligned; the caller keeps ownership and must keep it alive until
 * spin_state_destroy).  V is set to +inf and D to -inf (never observed) on
 * `stream`.  The handle itself is host memory owned by the library. */
SPIN_API spin_status spin_state_create(const spin_config* cfg, void* dev_mem, size_t bytes,
                              spin_stream_t stream, spin_state* out);

/* Frees the host handle only; dev_mem stays the caller's. */
SPIN_API spin_status spin_state_destroy(spin_state st);

/* Per-layer target block sparsity s_l in [0, 1), from host memory
 * [num_layers].  s_l = 0 is the all-keep control (no prediction, no
 * exploration).  Used by the per-layer budget of the SPIN v3 record (摘要). */
SPIN_API spin_status spin_set_layer_sparsity(spin_state st, const float* s_host);

/* Selects the score kernel used by spin_indexer_score / spin_decode_step. */
SPIN_API spin_status spin_set_score_kernel(spin_state st, int kind);

/* Sets V = +inf, D = -inf for requests req_host[0..n) of one layer (layer <
 * 0: every layer), e.g. when a slot starts a new sequence. */
SPIN_API spin_status spin_reset_requests(spin_state st, int layer, const int32_t* req_host, int n,
                                spin_stream_t stream);

/* Decode step numbers.  Every call that takes `step` accepts either an
 * explicit step >= 0 or SPIN_STEP_DEVICE, which reads the state's device step
 * counter when the kernels run.  spin_set_step / spin_advance_step change the
 * counter in stream order and launch nothing else, so a decode step (all its
 * layers) followed by spin_advance_step can be captured once in a CUDA graph
 * and replayed every step with the right exploration draw. */
#define SPIN_STEP_DEVICE (-1)
SPIN_API spin_status spin_set_step(spin_state st, int64_t step, spin_stream_t stream);
SPIN_API spin_status spin_advance_step(spin_state st, spin_stream_t stream);

/* a1 + a2: predicted slot score z = max(V_i, D_{p_r - i}) (AI Radio, "Title
 * and authors"; SPIN digest, arXiv深度剖析), block max-pool S_{r,j}, block
 * budget B_r = n_r - floor(s * n_r), exploration share n_exp = floor(gamma *
 * B_0) of uniformly random unkept blocks (SPIN digest, arXiv深度剖析; SPIN
 * listing, Figure 4), and for rows > 1 the union of the rows' predicted sets
 * (SPIN listing, Table 7), or row 0's set under SPIN_MTP_ROW0 (whose block
 * scores then hold row 0 only).  Ties go to the lower block index.
 *   ctx_len_dev [Q] int32, mask_dev [Q][max_blocks] uint8 out:
 *   0 skipped, 1 predicted, 2 explored (blocks past the last row's range: 0).
 *   step: decode step (>= 0, or SPIN_STEP_DEVICE), part of the exploration
 *   RNG counter. */
SPIN_API spin_status spin_predict_select(spin_state st, int layer, int rows, int64_t step,
                                const int32_t* ctx_len_dev, uint8_t* mask_dev,
                                spin_stream_t stream);

/* a0 + a3: indexer scores on the kept blocks only (SPIN listing, Abstract;
 * SPIN digest, arXiv深度剖析).
 *   keys [num_pages][b][d]: uint8 E4M3 codes (key_dtype FP8) or fp32;
 *   key_scale [num_pages][b] fp32 per-token scale (FP8 keys; NULL for fp32);
 *   block_table [Q][bt_stride] int32 logical block -> page;
 *   q [Q][rows][H][d] in q_dtype; w [Q][rows][H] fp32 head weights;
 *   mask_dev as written by spin_predict_select;
 *   scores_dev [Q][max_rows][max_slots_padded] fp32 out, with
 *   max_slots_padded = ceil(max_slots / b) * b (spin_score_stride); only
 *   entries of kept blocks with s <= p_r are written.
 * FP8 keys: each (row, head) query is quantised to E4M3 with a power-of-two
 * scale folded into its head weight; accumulation is fp32. */
SPIN_API spin_status spin_indexer_score(spin_state st, int layer, int rows, const void* keys,
                               const float* key_scale, int32_t num_pages,
                               const int32_t* block_table, int32_t bt_stride, const void* q,
                               const float* w, const int32_t* ctx_len_dev,
                               const uint8_t* mask_dev, float* scores_dev, spin_stream_t stream);

/* a4: token top-k per (request, row) over the scored slots (SPIN digest,
 * arXiv深度剖析: the fixed top-k budget of core attention is unchanged).
 * Higher score first, ties to the lower slot; emitted in ascending slot
 * order; padded with -1.  topk_dev [Q][rows][k] int32 out. */
SPIN_API spin_status spin_topk(spin_state st, int rows, const float* scores_dev, const uint8_t* mask_dev,
                      const int32_t* ctx_len_dev, int32_t* topk_dev, spin_stream_t stream);

/* Token top-k for callers that cannot allocate device memory (no SPIN page
 * has a counterpart to this call; it is a deployment convenience).  Code that
 * runs during CUDA graph capture cannot call cudaMalloc, and some host
 * applications or plug-in hosts own all device memory and give a library
 * none, so they cannot hand spin_state_create a block.  This call needs no
 * state: it computes exactly what spin_topk computes for the same scores,
 * mask and context lengths, with its scratch (kept-block lists, counts and an
 * error word) in a fixed 4 MiB array that the library reserves on every GPU
 * that loads it, for the life of the process.  It allocates nothing.
 *   scores_dev [num_requests][max_rows][ceil(max_slots/b)*b] fp32,
 *   mask_dev [num_requests][ceil(max_slots/b)] uint8, ctx_len_dev [Q] int32,
 *   topk_dev [num_requests][rows][topk] int32 out (same order and -1 padding
 *   as spin_topk; rows whose ctx_len is out of range come back all -1).
 * Limit: 4 + ceil(Q/64)*64 + Q * ceil(ceil(max_slots/b)/16)*16 must not
 * exceed 2^20 (e.g. 96 requests at 512K slots with b = 64); larger problems
 * return SPIN_EINVAL.  The first call on a device looks up the array's device
 * address (cudaGetSymbolAddress), so make that first call before any stream
 * capture; a new context on the device (after cudaDeviceReset) is detected
 * by its context id and the address is looked up again on the next call,
 * which should then also come before any capture.  All calls share the one
 * array: calls that overlap on the GPU (on different streams, or from several
 * host threads) race and must be serialised by the caller.  Device-side
 * errors (a ctx_len outside 1..max_slots-rows+1 sets bit 0, value 1, of the
 * error word) leave the rows of that request at -1 and are read with
 * spin_topk_noalloc_error. */
SPIN_API spin_status spin_topk_noalloc(int num_requests, int rows, int max_rows, int32_t max_slots,
                                       int block_size, int topk, const float* scores_dev,
                                       const uint8_t* mask_dev, const int32_t* ctx_len_dev,
                                       int32_t* topk_dev, spin_stream_t stream);

/* Error word of the last spin_topk_noalloc call on the current device (the
 * call clears it when it starts): synchronises the stream, copies the word to
 * *word_out (may be NULL) and returns SPIN_EDEVICE when a bit is set, else
 * SPIN_OK.  Not for use during stream capture. */
SPIN_API spin_status spin_topk_noalloc_error(spin_stream_t stream, uint32_t* word_out);

/* a5: EMA update of V (per slot) and D (per offset p_r - s) from the scores
 * of scored slots only (SPIN digest, 核心概要 / arXiv深度剖析; AI Radio, "The
 * paper's summary").  x <- score if x is the never-observed sentinel, else
 * fmaf(alpha, x, (1 - alpha) * score).  Rows 0..accepted[q]-1 are replayed in
 * order (prefix-valid update of MTP rows, SPIN digest, arXiv深度剖析); under
 * SPIN_MTP_ROW0 row 0 alone is applied (accepted_dev is still checked).
 * accepted_dev [Q] int32 in 1..rows, or NULL for all rows. */
SPIN_API spin_status spin_ema_update(spin_state st, int layer, int rows, const float* scores_dev,
                            const uint8_t* mask_dev, const int32_t* ctx_len_dev,
                            const int32_t* accepted_dev, spin_stream_t stream);

/* a0..a5 fused on one stream: quantise q, predict + select (skipped at
 * sparsity 0), score, top-k and -- unless defer_update -- the EMA update of
 * all rows.  With defer_update the caller calls spin_ema_update once the
 * accepted lengths are known.  scores_dev may be NULL (internal scratch) when
 * defer_update is 0. */
SPIN_API spin_status spin_decode_step(spin_state st, int layer, int rows, int64_t step, const void* keys,
                             const float* key_scale, int32_t num_pages, const int32_t* block_table,
                             int32_t bt_stride, const void* q, const float* w,
                             const int32_t* ctx_len_dev, int defer_update, uint8_t* mask_dev,
                             int32_t* topk_dev, float* scores_dev, spin_stream_t stream);

/* Pipelined one-row decode steps (enable = 1; 0 turns it off).  A step's
 * selection (a1 + a2) depends only on the EMA state, the positions and the
 * step number, all known once the previous step's score kernel has updated
 * the state (SPIN digest, arXiv深度剖析: the history comes from earlier
 * steps' indexer scores).  With lookahead on, spin_decode_step with rows = 1,
 * no deferred update and FP8 keys on the tensor-core kernel also prepares
 * the next step's selection of the same layer, for ctx_len + 1 and step + 1
 * (SPIN_STEP_DEVICE: the counter + 1).  The next step's predict kernel runs
 * right after the score kernel, and this step's top-k then runs on a second
 * stream of the state beside the next step's select; the call joins that
 * stream back into `stream` before it returns, so its outputs are ready in
 * stream order as before.  Results are bit-identical to the sequential
 * step's.  The next call of the layer must then pass ctx_len + 1 for every
 * request, the next step number and the same target: a different target or
 * step number (host steps), or an intervening spin_ema_update,
 * spin_reset_requests or spin_state_import, makes the call select afresh; a
 * request whose ctx_len is not the prepared one sets ERR_LOOKAHEAD (bit 5,
 * value 32) in the device error word and comes back unscored with all -1
 * top-k.  The first call on a state creates the second stream and two events
 * (no device memory); make it outside stream capture. */
SPIN_API spin_status spin_set_lookahead(spin_state st, int enable);

/* Every layer's one-row selection of one step, made at once (SPIN digest,
 * arXiv深度剖析: a layer's selection comes from its own EMA history, the
 * positions and the step, not from the step's queries, so the selections of
 * all layers are known before the first layer's indexer runs).  Needs
 * lookahead on (spin_set_lookahead; else SPIN_EINVAL).  For each layer, with
 * its current target, the predict and select kernels of rows = 1 run for
 * `step` (>= 0, or SPIN_STEP_DEVICE: the counter's current value) at
 * ctx_len_dev [Q] (device, slots visible to row 0), into the per-layer slots
 * the pipelined step uses.  With max pooling (and block_size >= 32) one
 * predict and one select launch on `stream` cover up to eight layers at a
 * time; with the other poolings the layers' kernels are spread over up to
 * eight streams of the state, forked from and joined back into `stream` (the
 * first such call creates the streams and nine events, no device memory;
 * make it outside stream capture).  A layer's next spin_decode_step with rows = 1, no
 * deferred update, that step, the same ctx_len and the same target then
 * scores this selection, runs its top-k on `stream` and prepares no next
 * selection; results are bit-identical to the sequential step's.  A request
 * whose ctx_len differs at the step sets ERR_LOOKAHEAD as for the pipelined
 * step; a different step or target, spin_ema_update, spin_reset_requests or
 * spin_state_import makes the step select afresh.  Argument errors return
 * SPIN_EINVAL and launch nothing; device-side errors go to the error word as
 * for spin_predict_select. */
SPIN_API spin_status spin_prepare_selections(spin_state st, int64_t step, const int32_t* ctx_len_dev,
                                             spin_stream_t stream);

/* Predictor-quality profile (SPIN listing, Table 1 compares predictors of the
 * indexer's scores by Pearson correlation and top-k recall).
 *
 * spin_slot_prediction writes one predictor's value for every visible slot
 * s <= p_r of every request and row: pred_dev [Q][max_rows][slot_stride] fp32
 * (the scores layout; slots past p_r are not written).
 *   SPIN_PRED_EMA     the SPIN predictor before block pooling, z = max(V_s,
 *                     D_{p_r - s}) from the layer's state; -inf where z is not
 *                     finite (a slot no step has scored has no prediction).
 *   SPIN_PRED_RANDOM  the random baseline: the top 24 bits of word 0 of
 *                     Philox4x32-10 at counter (s, request, layer, step mod
 *                     2^32), key (seed lo, seed hi), times 2^-24 (uniform in
 *                     [0, 1)), the same for every row; step >= 0 or
 *                     SPIN_STEP_DEVICE.
 * The previous iteration's or the previous layer's scores (a scores buffer of
 * an earlier spin_decode_step) are predictors as they stand.
 *
 * spin_pearson: pearson_dev [Q][rows] double, the Pearson correlation of x_dev
 * and y_dev (both [Q][max_rows][slot_stride] fp32) over the visible slots of
 * each (request, row) where both are finite, computed in double in two passes
 * (means, then centred sums) in a fixed order; 0 when fewer than two such
 * slots remain or either side is constant on them.
 *
 * spin_topk_overlap: overlap_dev [Q][rows] int32, the number of slots that two
 * top-k lists a_dev, b_dev ([Q][rows][k] int32, ascending, -1 padded, as
 * spin_topk writes them) share.  The top-k recall of a predictor is the
 * overlap of its top-k (spin_topk of pred_dev with every block kept) with the
 * indexer's, divided by k.
 * A ctx_len out of range sets ERR_CTX_LEN in the device error word and leaves
 * that request's outputs unwritten (prediction) or 0 (correlation). */
typedef enum { SPIN_PRED_EMA = 0, SPIN_PRED_RANDOM = 1 } spin_predictor;
SPIN_API spin_status spin_slot_prediction(spin_state st, int layer, int rows, int kind, int64_t step,
                                 const int32_t* ctx_len_dev, float* pred_dev, spin_stream_t stream);
SPIN_API spin_status spin_pearson(spin_state st, int rows, const float* x_dev, const float* y_dev,
                         const int32_t* ctx_len_dev, double* pearson_dev, spin_stream_t stream);
SPIN_API spin_status spin_topk_overlap(spin_state st, int rows, const int32_t* a_dev, const int32_t* b_dev,
                              int32_t* overlap_dev, spin_stream_t stream);

/* Miss count of the fidelity metric (SPIN listing, Table 5 caption): for each
 * (request, row), the number of entries of full_topk_dev [Q][rows][k] (a
 * full-indexer top-k, -1 padded) whose block is skipped in mask_dev.
 *   missed_dev [Q][rows] int32 out; total_dev [Q][rows] int32 out (entries >= 0). */
SPIN_API spin_status spin_miss_count(spin_state st, int rows, const int32_t* full_topk_dev,
                            const uint8_t* mask_dev, int32_t* missed_dev, int32_t* total_dev,
                            spin_stream_t stream);

/* Host-side per-layer budget (SPIN v3 record, 摘要: the block budget is spread
 * over layers by their measured miss rates).  Kept fraction
 * f_l = clamp(c * (miss_l + 1e-3), lo_l, 1) with c such that
 * sum f_l * blocks_l = (1 - s_glob) * sum blocks_l; if the floors alone
 * exceed the budget, f_l = lo_l.  s_out_host[l] = 1 - f_l.  No state, no GPU. */
SPIN_API spin_status spin_allocate_layer_sparsity(int num_layers, const double* miss_host,
                                         const double* blocks_host, const double* lo_host,
                                         double s_glob, float* s_out_host);

/* Per-stage timing and launch counts of the library's own kernels.
 * Stages: 0 predict + pool, 1 select, 2 query quantisation, 3 indexer score,
 * 4 top-k, 5 EMA update (standalone), 6 mask compaction, 7 miss count.
 * With timing enabled, every launch is bracketed by two CUDA events recorded
 * on the launch's stream.  spin_kernel_times synchronises on the recorded
 * events, writes the summed milliseconds and the launch counts since the last
 * call into ms_out[n] / launches_out[n] (either may be NULL; n <= 8) and
 * resets both.  Launches are counted whether or not timing is enabled. */
SPIN_API spin_status spin_set_kernel_timing(spin_state st, int enable);
/* Times only the stages in stage_mask (bit n = stage n, as listed above);
 * the other launches get no events, so they keep running back to back.
 * 0 turns timing off.  SPIN_EINVAL for bits past the last stage. */
SPIN_API spin_status spin_set_kernel_timing_mask(spin_state st, uint32_t stage_mask);
SPIN_API spin_status spin_kernel_times(spin_state st, double* ms_out, int64_t* launches_out, int n);

/* Test hook for the device error path.  mode 1: on its next launch, CTA 0
 * of the tensor-core score kernel withholds the copy of its first key stage,
 * so the matrix-issue thread's bounded wait (2 s) runs out; the kernel then
 * raises ERR_TIMEOUT in the device error word, drains its copies, frees its
 * tensor memory and returns, and the call's outputs are incomplete.  The
 * mode resets to 0 after one launch.  mode 0: off. */
SPIN_API spin_status spin_set_fault_injection(spin_state st, int mode);

/* Synchronises `stream`, then reads and clears the device error word:
 * SPIN_OK, SPIN_EDEVICE or SPIN_ETIMEOUT.  Optionally returns the raw word. */
SPIN_API spin_status spin_get_error(spin_state st, spin_stream_t stream, uint32_t* word_out);

SPIN_API const char* spin_status_string(spin_status s);

/* Checkpoint of the EMA state (V and D of every layer): export_bytes() bytes,
 * copied synchronously through host memory on `stream`. */
SPIN_API size_t spin_state_export_bytes(spin_state st);
SPIN_API spin_status spin_state_export(spin_state st, void* host, size_t bytes, spin_stream_t stream);
SPIN_API spin_status spin_state_import(spin_state st, const void* host, size_t bytes, spin_stream_t stream);

/* After writing V (or D) of the EMA state through the pointers spin_state_ema
 * returns, the caller calls this before the next library call that reads the
 * state: it recomputes V's 32-slot group maxima of `layer` (layer -1: every
 * layer) on `stream`, and drops any selection a pipelined step prepared.
 * Every library call that writes V keeps them current by itself. */
SPIN_API spin_status spin_state_refresh(spin_state st, int layer, spin_stream_t stream);

/* Inspection: device pointers into the state block.
 *   spin_state_ema: V, D of `layer`, each [Q][*stride] fp32.  Writing through
 *     them is allowed, followed by spin_state_refresh.
 *   spin_state_vmax: V's group maxima of `layer`, [Q][*stride] fp32 with
 *     (*vmax)[q][g] = max(V[q][32 g .. 32 g + 31]); NULL and stride 0 when the
 *     state keeps none (block_size 16, or a pooling other than max).
 *   spin_state_block_scores: S [Q][max_rows][*stride] fp32 of the last predict.
 *   spin_state_qquant: quantised queries [Q][max_rows][H][d] E4M3 and their
 *   folded head weights [Q][max_rows][H] fp32 of the last FP8 score call.
 *   spin_score_stride: slot stride of a score row (ceil(max_slots/b)*b);
 *   spin_mask_stride: block stride of a mask row (ceil(max_slots/b)). */
SPIN_API spin_status spin_state_ema(spin_state st, int layer, float** V, float** D, int64_t* stride);
SPIN_API spin_status spin_state_vmax(spin_state st, int layer, const float** vmax, int64_t* stride);
SPIN_API spin_status spin_state_block_scores(spin_state st, const float** S, int64_t* stride);
SPIN_API spin_status spin_state_qquant(spin_state st, const uint8_t** q8, const float** wq);
SPIN_API int64_t spin_score_stride(spin_state st);
SPIN_API int64_t spin_mask_stride(spin_state st);

#ifdef __cplusplus
}
#endif
#endif /* SPIN_H_ */
