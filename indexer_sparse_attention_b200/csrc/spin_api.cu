// spin_api.cu -- host side of the libspin.so C ABI (include/spin.h):
// argument validation, carving of the caller's state block, kernel launches
// and the fused decode step.  No call allocates device memory.
#include <algorithm>
#include <cmath>
#include <cstdio>
#include <cstring>
#include <new>
#include <vector>

#include "spin_internal.cuh"

using namespace spin;

// Streams spin_prepare_selections spreads the layers over (created on first use).
constexpr int kPrepStreams = 8;

struct spin_state_s {
  spin_config cfg;
  Layout lay;
  char* base;
  size_t bytes;
  ErrWord* err;
  float* V;       // [L][Q][slot_stride]
  float* D;
  float* vmax;    // [L][Q][vg_stride] max of V over each aligned 32-slot group, or null
  float* S;       // [Q][R][blk_stride]
  int32_t* work;  // [Q][blk_stride]
  int32_t* kept;  // [Q]
  uint8_t* q8;    // [Q][R][H][d]
  float* wq;      // [Q][R][H]
  float* scores;  // [Q][R][slot_stride]
  float* gmax;    // [Q][R][gstride] group maxima of the last tensor-core score
  int64_t gstride;
  int64_t* step_dev;  // device step counter (SPIN_STEP_DEVICE)
  std::vector<float> sparsity;
  int score_kernel;
  int inject;
  void* encode_fn;  // cuTensorMapEncodeTiled, resolved at create
  // per-stage timing (spin_set_kernel_timing / spin_kernel_times)
  uint32_t timing;  // stages whose launches are bracketed by events (bit n = stage n)
  struct Rec { int stage; cudaEvent_t a, b; };
  std::vector<Rec> recs;
  std::vector<cudaEvent_t> pool;
  int64_t launches[8];
  // Lookahead (spin_set_lookahead): each one-row decode step also prepares
  // the next step's selection of its layer, so that the step's top-k runs on
  // a second stream beside the next step's predict kernel.
  int lookahead;
  cudaStream_t side;                 // this step's top-k runs here (created on first use)
  cudaEvent_t ev_scored, ev_copied, ev_topk;  // see decode_step_lookahead
  struct Prepared {
    bool ready;
    int64_t step;                    // the step the selection is for (SPIN_STEP_DEVICE: the counter's)
    float sparsity;                  // the layer's target it was made with
    bool batch;                      // made by spin_prepare_selections: the step prepares no next one
  };
  std::vector<Prepared> prep;        // per layer
  int32_t* la_work;                  // [L][Q][blk_stride] kept block ids of the prepared selection
  int32_t* la_kept;                  // [L][Q]
  uint8_t* la_mask;                  // [L][Q][max_blocks]
  int32_t* la_ctx;                   // [L][Q] ctx_len each request's selection was made for (-1: none)
  int32_t* ctx_next;                 // [Q] ctx_len + 1, written by the score kernel
  int32_t* tk_work;                  // [Q][blk_stride] the top-k's copy of the selection it reads, so that
  int32_t* tk_kept;                  // [Q]   the next selection can be written while it runs
  int32_t* tk_ctx;                   // [Q]
  // spin_prepare_selections: every layer's predict + select on prep_k
  // streams at once, each stream with its own block-score scratch
  int prep_k;
  float* prep_S;                     // [prep_k][Q][max_rows][blk_stride] (the block-score layout)
  cudaStream_t pstream[kPrepStreams];
  cudaEvent_t pev[kPrepStreams + 1]; // [0]: the fork; [1 + i]: stream i done
  uint32_t magic;
};

namespace {

constexpr uint32_t kMagic = 0x5350494eu;  // "SPIN"
constexpr int64_t kMaxBlocksSelect = 40960;  // K2 keeps S and the mask of a request on chip

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

bool valid_config(const spin_config* c) {
  if (!c) return false;
  if (c->num_layers < 1 || c->num_requests < 1 || c->max_slots < 1) return false;
  const int b = c->block_size;
  if (b < 16 || b > 256 || (b & (b - 1))) return false;
  if (c->num_heads < 1 || c->num_heads > 256 || c->head_dim < 1 || c->head_dim > 512) return false;
  if (c->topk < 1 || c->topk > 65536) return false;
  if (c->max_rows < 1 || c->max_rows > 4) return false;
  if (c->key_dtype != SPIN_F32 && c->key_dtype != SPIN_FP8_E4M3) return false;
  if (c->q_dtype != SPIN_F32 && c->q_dtype != SPIN_BF16) return false;
  if (c->key_dtype == SPIN_F32 && c->q_dtype != SPIN_F32) return false;
  if (c->key_dtype == SPIN_FP8_E4M3 && (c->head_dim % 16)) return false;
  if (!(c->alpha >= 0.0f && c->alpha <= 1.0f)) return false;
  if (!(c->gamma >= 0.0f && c->gamma <= 1.0f)) return false;
  if (!(c->target_sparsity >= 0.0f && c->target_sparsity < 1.0f)) return false;
  if (c->pooling < SPIN_POOL_MAX || c->pooling > SPIN_POOL_TOP4) return false;
  if (c->mtp_policy < SPIN_MTP_UNION_PREFIX || c->mtp_policy > SPIN_MTP_ROW0) return false;
  const int64_t max_blocks = (c->max_slots + (int64_t)b - 1) / b;
  if (max_blocks > kMaxBlocksSelect) return false;
  // top-k: bitmap of one (request, row) plus the candidate area on chip
  if ((max_blocks * b + 31) / 32 * 4 > 160 * 1024) return false;
  // SIMT score kernel keeps the queries of a request and one page on chip
  const size_t simt = sizeof(float) * ((size_t)c->max_rows * c->num_heads * c->head_dim +
                                       (size_t)c->max_rows * c->num_heads + (size_t)b * (c->head_dim + 1));
  if (simt > 220 * 1024) return false;
  return true;
}

Layout make_layout(const spin_config* c) {
  Layout L;
  L.L = c->num_layers;
  L.Q = c->num_requests;
  L.R = c->max_rows;
  L.H = c->num_heads;
  L.d = c->head_dim;
  L.b = c->block_size;
  L.k = c->topk;
  L.max_slots = c->max_slots;
  L.max_blocks = (c->max_slots + (int64_t)c->block_size - 1) / c->block_size;
  L.slot_stride = L.max_blocks * c->block_size;
  L.blk_stride = (L.max_blocks + 15) / 16 * 16;
  // V's 32-slot group maxima: read by the max-pooled prediction in place of V
  L.vg_stride = (c->block_size >= 32 && c->pooling == SPIN_POOL_MAX) ? L.slot_stride / 32 : 0;
  return L;
}

// Group maxima: one per 32 slots of the kept-slot order.
int64_t gmax_stride(const Layout& L) { return L.blk_stride * std::max(1, L.b / 32); }

struct Carve {
  size_t err, V, D, vmax, S, work, kept, q8, wq, scores, gmax, step, la_work, la_kept, la_mask, la_ctx, ctx_next, tk_work,
      tk_kept, tk_ctx, prep_S, total;
};

int prep_streams(const Layout& L) { return (int)std::min<int64_t>(L.L, kPrepStreams); }

Carve carve(const Layout& L) {
  Carve k;
  size_t off = 0;
  auto take = [&](size_t bytes) { size_t at = off; off = align256(off + bytes); return at; };
  k.err = take(sizeof(ErrWord));
  k.V = take((size_t)L.L * L.Q * L.slot_stride * 4);
  k.D = take((size_t)L.L * L.Q * L.slot_stride * 4);
  k.vmax = take((size_t)L.L * L.Q * L.vg_stride * 4);
  k.S = take((size_t)L.Q * L.R * L.blk_stride * 4);
  k.work = take((size_t)L.Q * L.blk_stride * 4);
  k.kept = take((size_t)L.Q * 4);
  k.q8 = take((size_t)L.Q * L.R * L.H * L.d);
  k.wq = take((size_t)L.Q * L.R * L.H * 4);
  k.scores = take((size_t)L.Q * L.R * L.slot_stride * 4);
  k.gmax = take((size_t)L.Q * L.R * gmax_stride(L) * 4);
  k.step = take(sizeof(int64_t));
  k.la_work = take((size_t)L.L * L.Q * L.blk_stride * 4);
  k.la_kept = take((size_t)L.L * L.Q * 4);
  k.la_mask = take((size_t)L.L * L.Q * L.max_blocks);
  k.la_ctx = take((size_t)L.L * L.Q * 4);
  k.ctx_next = take((size_t)L.Q * 4);
  k.tk_work = take((size_t)L.Q * L.blk_stride * 4);
  k.tk_kept = take((size_t)L.Q * 4);
  k.tk_ctx = take((size_t)L.Q * 4);
  k.prep_S = take((size_t)prep_streams(L) * L.Q * L.R * L.blk_stride * 4);
  k.total = off;
  return k;
}

bool alive(spin_state st) { return st && st->magic == kMagic; }

spin_status cuda_status(cudaError_t e) {
  if (e == cudaSuccess) return SPIN_OK;
  fprintf(stderr, "libspin: CUDA error %s\n", cudaGetErrorString(e));
  return SPIN_ECUDA;
}

float beta_of(float alpha) { return (float)(1.0 - (double)alpha); }

float* vmax_of(spin_state st, int layer) {
  return st->vmax ? st->vmax + (size_t)st->lay.Q * st->lay.vg_stride * layer : nullptr;
}

StepArgs step_args(spin_state st, int layer, int rows, int64_t step, const int32_t* ctx_len, uint8_t* mask) {
  StepArgs a;
  a.lay = st->lay;
  a.layer = layer;
  a.rows = rows;
  a.pooling = st->cfg.pooling;
  a.mtp_row0 = st->cfg.mtp_policy == SPIN_MTP_ROW0 && rows > 1;
  a.step = step < 0 ? 0 : step;
  a.step_dev = step == SPIN_STEP_DEVICE ? st->step_dev : nullptr;
  a.step_add = 0;
  a.ctx_sel = nullptr;
  a.quiet = 0;
  a.no_pdl = 0;
  a.sparsity = st->sparsity[layer];
  a.gamma = st->cfg.gamma;
  a.alpha = st->cfg.alpha;
  a.seed = st->cfg.seed;
  a.ctx_len = ctx_len;
  a.mask = mask;
  a.S = st->S;
  a.work = st->work;
  a.kept = st->kept;
  const size_t per_layer = (size_t)st->lay.Q * st->lay.slot_stride;
  a.V = st->V + per_layer * layer;
  a.D = st->D + per_layer * layer;
  a.vmax = vmax_of(st, layer);
  a.err = st->err;
  a.q = nullptr;
  a.w = nullptr;
  a.q_bf16 = st->cfg.q_dtype == SPIN_BF16;
  a.q8 = nullptr;
  a.nl = 1;
  a.state_stride = a.vg_layer_stride = a.s_stride = a.mask_stride = a.work_stride = a.req_stride = 0;
  for (int i = 0; i < kMaxLayerBatch; ++i) a.sp[i] = 0.0f;
  a.wq = nullptr;
  return a;
}

bool use_tc(spin_state st, int rows) {
  const bool ok = tc_supported(st->lay, rows, st->cfg.key_dtype == SPIN_FP8_E4M3) && st->encode_fn;
  if (st->score_kernel == SPIN_SCORE_SIMT) return false;
  return ok;
}

enum Stage { kPredict = 0, kSelect, kQuant, kScore, kTopk, kEma, kCompact, kMiss, kNumStages };

cudaEvent_t take_event(spin_state st) {
  if (!st->pool.empty()) {
    cudaEvent_t e = st->pool.back();
    st->pool.pop_back();
    return e;
  }
  cudaEvent_t e = nullptr;
  cudaEventCreate(&e);
  return e;
}

// Launches one kernel, counting it and -- with timing on -- bracketing it by
// two events on its stream.
template <class F>
cudaError_t staged(spin_state st, int stage, cudaStream_t s, F launch) {
  st->launches[stage] += 1;
  if (!((st->timing >> stage) & 1u)) return launch();
  cudaEvent_t a = take_event(st), b = take_event(st);
  if (!a || !b) return cudaErrorMemoryAllocation;
  cudaEventRecord(a, s);
  cudaError_t e = launch();
  cudaEventRecord(b, s);
  st->recs.push_back({stage, a, b});
  return e;
}

// Quantise (FP8 keys) and score the kept blocks listed in st->work / st->kept.
// The kept-block list a score reads, and the checks of a prepared selection.
struct Selection {
  const int32_t* work;
  const int32_t* kept;
  const int32_t* ctx_sel;  // or null
  int32_t* ctx_next;       // or null
};

spin_status run_score(spin_state st, int layer, int rows, const void* keys, const float* key_scale,
                      int32_t num_pages, const int32_t* block_table, int32_t bt_stride, const void* q,
                      const float* w, const int32_t* ctx_len, const uint8_t* mask, float* scores,
                      bool fuse_ema, cudaStream_t stream, bool* wrote_gmax = nullptr, bool quantized = false,
                      const Selection* sel = nullptr) {
  ScoreArgs a;
  a.lay = st->lay;
  a.rows = rows;
  a.key_fp8 = st->cfg.key_dtype == SPIN_FP8_E4M3;
  a.q_bf16 = st->cfg.q_dtype == SPIN_BF16;
  a.keys = keys;
  a.kscale = key_scale;
  a.num_pages = num_pages;
  a.block_table = block_table;
  a.bt_stride = bt_stride;
  a.q = q;
  a.w = w;
  a.ctx_len = ctx_len;
  a.mask = mask;
  a.work = sel ? sel->work : st->work;
  a.kept = sel ? sel->kept : st->kept;
  a.ctx_sel = sel ? sel->ctx_sel : nullptr;
  a.ctx_next = sel ? sel->ctx_next : nullptr;
  a.q8 = st->q8;
  a.wq = st->wq;
  a.scores = scores;
  a.err = st->err;
  const size_t per_layer = (size_t)st->lay.Q * st->lay.slot_stride;
  a.V = fuse_ema ? st->V + per_layer * layer : nullptr;
  a.D = fuse_ema ? st->D + per_layer * layer : nullptr;
  a.vmax = fuse_ema ? vmax_of(st, layer) : nullptr;
  a.alpha = st->cfg.alpha;
  a.beta = beta_of(st->cfg.alpha);
  a.inject = 0;
  a.gmax = nullptr;
  a.gstride = st->gstride;
  if (wrote_gmax) *wrote_gmax = false;
  if (a.key_fp8 && !quantized) {
    spin_status s = cuda_status(staged(st, kQuant, stream, [&] { return launch_quantize_q(a, stream); }));
    if (s != SPIN_OK) return s;
  }
  if (st->score_kernel == SPIN_SCORE_TCGEN05 && !use_tc(st, rows)) return SPIN_EUNSUPPORTED;
  if (use_tc(st, rows)) {
    a.inject = st->inject;
    st->inject = 0;
    if (wrote_gmax) {
      a.gmax = st->gmax;
      *wrote_gmax = true;
    }
    return cuda_status(staged(st, kScore, stream, [&] { return launch_score_tc(a, st->encode_fn, stream); }));
  }
  return cuda_status(staged(st, kScore, stream, [&] { return launch_score_simt(a, stream); }));
}

spin_status check_rows(spin_state st, int rows) {
  return (rows >= 1 && rows <= st->cfg.max_rows) ? SPIN_OK : SPIN_EINVAL;
}

// The pipelined one-row decode step (spin_set_lookahead).  The step's
// selection was prepared by the previous step of this layer (or is made here
// when there is none, or it was made for another step or target):
//   stream:  a0 -> score + fused EMA (writes ctx_len + 1) -> predict(next) -------> select(next) -> [join]
//   side:                                  [fork] -> copy selection, mask -> top-k ---^ ------------^
// The next step's predict reads only V and D, which the score kernel has
// finished; its many short blocks take the SMs the top-k (one CTA per
// request) leaves idle, and the next select follows once the kept lists are
// copied.  The top-k reads that copy, because the next select overwrites
// them.  Results are those of the sequential step: the next selection is
// computed from the same state, positions (ctx_len + 1) and step number as
// the next call would compute it.  The step's query quantisation (a0) cannot
// ride in the predict here, which runs a step ahead: it is a launch of its own.
spin_status decode_step_lookahead(spin_state st, int layer, int64_t step, const void* keys, const float* key_scale,
                                  int32_t num_pages, const int32_t* block_table, int32_t bt_stride, const void* q,
                                  const float* w, const int32_t* ctx_len, uint8_t* mask_dev, int32_t* topk_dev,
                                  float* scores, cudaStream_t s) {
  const Layout& L = st->lay;
  spin_state_s::Prepared& P = st->prep[layer];
  const float sp = st->sparsity[layer];
  int32_t* work = st->la_work + (size_t)layer * L.Q * L.blk_stride;
  int32_t* kept = st->la_kept + (size_t)layer * L.Q;
  uint8_t* lmask = st->la_mask + (size_t)layer * L.Q * L.max_blocks;
  int32_t* lctx = st->la_ctx + (size_t)layer * L.Q;
  const int64_t next = step == SPIN_STEP_DEVICE ? SPIN_STEP_DEVICE : step + 1;
  auto select_args = [&](const int32_t* ctx, int64_t stp, bool ahead) {
    StepArgs a = step_args(st, layer, 1, stp, ctx, lmask);
    a.step_add = (ahead && stp == SPIN_STEP_DEVICE) ? 1 : 0;
    a.work = work;
    a.kept = kept;
    a.ctx_sel = lctx;
    a.quiet = ahead ? 1 : 0;
    return a;
  };
  spin_status r;
  P.ready = P.ready && P.sparsity == sp && P.step == step;
  const bool batch = P.ready && P.batch;  // made by spin_prepare_selections for this step alone
  if (!P.ready) {  // no selection prepared for this step: make it now
    StepArgs a = select_args(ctx_len, step, false);
    if (sp > 0.0f) {
      r = cuda_status(staged(st, kPredict, s, [&] { return launch_predict_pool(a, s); }));
      if (r != SPIN_OK) return r;
    }
    r = cuda_status(staged(st, kSelect, s, [&] { return launch_select(a, s); }));
    if (r != SPIN_OK) return r;
  }
  P.ready = false;  // consumed below; set again once the next one is issued
  const Selection sel{work, kept, lctx, st->ctx_next};
  bool gm = false;
  r = run_score(st, layer, 1, keys, key_scale, num_pages, block_table, bt_stride, q, w, ctx_len, lmask, scores,
                true, s, &gm, false, &sel);
  if (r != SPIN_OK) return r;
  if (batch) {
    // the next selection of this layer comes from the next spin_prepare_selections:
    // the top-k reads this one in place, on this stream
    P.batch = false;
    cudaError_t e = cudaMemcpyAsync(mask_dev, lmask, (size_t)L.Q * L.max_blocks, cudaMemcpyDeviceToDevice, s);
    if (e != cudaSuccess) return cuda_status(e);
    TopkArgs t{L, 1, scores, mask_dev, ctx_len, work, kept, topk_dev, st->err, gm ? st->gmax : nullptr,
               st->gstride, lctx};
    return cuda_status(staged(st, kTopk, s, [&] { return launch_topk(t, s); }));
  }
  // fork: the side stream copies the selection the top-k reads, and the mask
  cudaError_t e = cudaEventRecord(st->ev_scored, s);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(st->side, st->ev_scored, 0);
  if (e == cudaSuccess)
    e = cudaMemcpyAsync(st->tk_work, work, (size_t)L.Q * L.blk_stride * 4, cudaMemcpyDeviceToDevice, st->side);
  if (e == cudaSuccess) e = cudaMemcpyAsync(st->tk_kept, kept, (size_t)L.Q * 4, cudaMemcpyDeviceToDevice, st->side);
  if (e == cudaSuccess) e = cudaMemcpyAsync(st->tk_ctx, lctx, (size_t)L.Q * 4, cudaMemcpyDeviceToDevice, st->side);
  if (e == cudaSuccess)
    e = cudaMemcpyAsync(mask_dev, lmask, (size_t)L.Q * L.max_blocks, cudaMemcpyDeviceToDevice, st->side);
  if (e == cudaSuccess) e = cudaEventRecord(st->ev_copied, st->side);
  if (e != cudaSuccess) return cuda_status(e);
  // this step's top-k on the side stream; the next step's predict fills the
  // SMs the top-k leaves idle, then the next select runs
  TopkArgs t{L, 1, scores, mask_dev, ctx_len, st->tk_work, st->tk_kept, topk_dev, st->err, gm ? st->gmax : nullptr,
             st->gstride, st->tk_ctx};
  r = cuda_status(staged(st, kTopk, st->side, [&] { return launch_topk(t, st->side); }));
  if (r != SPIN_OK) return r;
  StepArgs a = select_args(st->ctx_next, next, true);
  if (sp > 0.0f) {
    r = cuda_status(staged(st, kPredict, s, [&] { return launch_predict_pool(a, s); }));
    if (r != SPIN_OK) return r;
  }
  e = cudaEventRecord(st->ev_topk, st->side);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(s, st->ev_copied, 0);  // the kept lists are copied
  if (e != cudaSuccess) return cuda_status(e);
  a.no_pdl = 1;  // follows a wait on the other stream's event
  r = cuda_status(staged(st, kSelect, s, [&] { return launch_select(a, s); }));
  if (r != SPIN_OK) return r;
  e = cudaStreamWaitEvent(s, st->ev_topk, 0);  // join
  if (e != cudaSuccess) return cuda_status(e);
  P.ready = true;
  P.step = next;
  P.sparsity = sp;
  P.batch = false;
  return SPIN_OK;
}

}  // namespace

extern "C" {

size_t spin_state_bytes(const spin_config* cfg) {
  if (!valid_config(cfg)) return 0;
  return carve(make_layout(cfg)).total;
}

spin_status spin_state_create(const spin_config* cfg, void* dev_mem, size_t bytes, spin_stream_t stream,
                              spin_state* out) {
  if (!out) return SPIN_EINVAL;
  *out = nullptr;
  if (!valid_config(cfg) || !dev_mem || ((uintptr_t)dev_mem & 255)) return SPIN_EINVAL;
  const Layout L = make_layout(cfg);
  const Carve k = carve(L);
  if (bytes < k.total) return SPIN_ENOMEM;
  spin_state st = new (std::nothrow) spin_state_s();
  if (!st) return SPIN_EINVAL;
  st->cfg = *cfg;
  st->lay = L;
  st->base = (char*)dev_mem;
  st->bytes = bytes;
  st->err = (ErrWord*)(st->base + k.err);
  st->V = (float*)(st->base + k.V);
  st->D = (float*)(st->base + k.D);
  st->vmax = L.vg_stride ? (float*)(st->base + k.vmax) : nullptr;
  st->S = (float*)(st->base + k.S);
  st->work = (int32_t*)(st->base + k.work);
  st->kept = (int32_t*)(st->base + k.kept);
  st->q8 = (uint8_t*)(st->base + k.q8);
  st->wq = (float*)(st->base + k.wq);
  st->scores = (float*)(st->base + k.scores);
  st->gmax = (float*)(st->base + k.gmax);
  st->gstride = gmax_stride(L);
  st->step_dev = (int64_t*)(st->base + k.step);
  st->la_work = (int32_t*)(st->base + k.la_work);
  st->la_kept = (int32_t*)(st->base + k.la_kept);
  st->la_mask = (uint8_t*)(st->base + k.la_mask);
  st->la_ctx = (int32_t*)(st->base + k.la_ctx);
  st->ctx_next = (int32_t*)(st->base + k.ctx_next);
  st->tk_work = (int32_t*)(st->base + k.tk_work);
  st->tk_kept = (int32_t*)(st->base + k.tk_kept);
  st->tk_ctx = (int32_t*)(st->base + k.tk_ctx);
  st->prep_k = prep_streams(L);
  st->prep_S = (float*)(st->base + k.prep_S);
  for (int i = 0; i < kPrepStreams; ++i) st->pstream[i] = nullptr;
  for (int i = 0; i <= kPrepStreams; ++i) st->pev[i] = nullptr;
  st->lookahead = 0;
  st->side = nullptr;
  st->ev_scored = st->ev_copied = st->ev_topk = nullptr;
  st->prep.assign(cfg->num_layers, spin_state_s::Prepared{false, 0, 0.0f, false});
  st->sparsity.assign(cfg->num_layers, cfg->target_sparsity);
  st->score_kernel = SPIN_SCORE_AUTO;
  st->inject = 0;
  st->timing = 0;
  for (int i = 0; i < 8; ++i) st->launches[i] = 0;
  st->encode_fn = nullptr;
  cudaDriverEntryPointQueryResult qres;
  void* fn = nullptr;
  if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &qres) == cudaSuccess &&
      qres == cudaDriverEntryPointSuccess)
    st->encode_fn = fn;
  cudaGetLastError();
  cudaStream_t s = (cudaStream_t)stream;
  cudaError_t e = cudaMemsetAsync(st->err, 0, sizeof(ErrWord), s);
  if (e == cudaSuccess)
    e = launch_init_state(st->V, st->D, (int64_t)L.L * L.Q * L.slot_stride, st->vmax,
                          (int64_t)L.L * L.Q * L.vg_stride, s);
  if (e == cudaSuccess) e = cudaMemsetAsync(st->step_dev, 0, sizeof(int64_t), s);
  if (e != cudaSuccess) {
    delete st;
    return cuda_status(e);
  }
  st->magic = kMagic;
  *out = st;
  return SPIN_OK;
}

spin_status spin_state_destroy(spin_state st) {
  if (!alive(st)) return SPIN_ESTATE;
  for (auto& r : st->recs) {
    cudaEventDestroy(r.a);
    cudaEventDestroy(r.b);
  }
  for (auto e : st->pool) cudaEventDestroy(e);
  for (cudaEvent_t e : {st->ev_scored, st->ev_copied, st->ev_topk})
    if (e) cudaEventDestroy(e);
  if (st->side) cudaStreamDestroy(st->side);
  for (int i = 0; i <= kPrepStreams; ++i)
    if (st->pev[i]) cudaEventDestroy(st->pev[i]);
  for (int i = 0; i < kPrepStreams; ++i)
    if (st->pstream[i]) cudaStreamDestroy(st->pstream[i]);
  st->magic = 0;
  delete st;
  return SPIN_OK;
}

spin_status spin_set_layer_sparsity(spin_state st, const float* s_host) {
  if (!alive(st)) return SPIN_ESTATE;
  if (!s_host) return SPIN_EINVAL;
  for (int l = 0; l < st->cfg.num_layers; ++l)
    if (!(s_host[l] >= 0.0f && s_host[l] < 1.0f)) return SPIN_EINVAL;
  st->sparsity.assign(s_host, s_host + st->cfg.num_layers);
  return SPIN_OK;  // a prepared selection made with another target is dropped at its next use
}

spin_status spin_set_score_kernel(spin_state st, int kind) {
  if (!alive(st)) return SPIN_ESTATE;
  if (kind < SPIN_SCORE_AUTO || kind > SPIN_SCORE_TCGEN05) return SPIN_EINVAL;
  if (kind == SPIN_SCORE_TCGEN05 && !(tc_supported(st->lay, 1, st->cfg.key_dtype == SPIN_FP8_E4M3) &&
                                      st->encode_fn))
    return SPIN_EUNSUPPORTED;
  st->score_kernel = kind;
  return SPIN_OK;
}

spin_status spin_set_lookahead(spin_state st, int enable) {
  if (!alive(st)) return SPIN_ESTATE;
  if (enable != 0 && enable != 1) return SPIN_EINVAL;
  if (enable && !st->side) {
    cudaError_t e = cudaStreamCreateWithFlags(&st->side, cudaStreamNonBlocking);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&st->ev_scored, cudaEventDisableTiming);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&st->ev_copied, cudaEventDisableTiming);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&st->ev_topk, cudaEventDisableTiming);
    if (e != cudaSuccess) return cuda_status(e);
  }
  st->lookahead = enable;
  for (auto& p : st->prep) p.ready = false;
  return SPIN_OK;
}

spin_status spin_prepare_selections(spin_state st, int64_t step, const int32_t* ctx_len_dev, spin_stream_t stream) {
  if (!alive(st)) return SPIN_ESTATE;
  if (!st->lookahead || !ctx_len_dev || (step < 0 && step != SPIN_STEP_DEVICE)) return SPIN_EINVAL;
  const Layout& L = st->lay;
  cudaStream_t s = (cudaStream_t)stream;
  auto mark = [&](int layer) {
    spin_state_s::Prepared& P = st->prep[layer];
    P.ready = true;
    P.batch = true;
    P.step = step;
    P.sparsity = st->sparsity[layer];
  };
  if (st->cfg.pooling == SPIN_POOL_MAX && vmax_of(st, 0)) {
    // one predict and one select launch over up to eight layers at a time, on
    // `stream` (a layer's place in the launch picks its state, scratch and target)
    for (int l0 = 0; l0 < L.L; l0 += kMaxLayerBatch) {
      const int nl = std::min(kMaxLayerBatch, L.L - l0);
      StepArgs a = step_args(st, l0, 1, step, ctx_len_dev, st->la_mask + (size_t)l0 * L.Q * L.max_blocks);
      a.nl = nl;
      a.S = st->prep_S;
      a.work = st->la_work + (size_t)l0 * L.Q * L.blk_stride;
      a.kept = st->la_kept + (size_t)l0 * L.Q;
      a.ctx_sel = st->la_ctx + (size_t)l0 * L.Q;
      a.state_stride = (int64_t)L.Q * L.slot_stride;
      a.vg_layer_stride = (int64_t)L.Q * L.vg_stride;
      a.s_stride = (int64_t)L.Q * L.R * L.blk_stride;
      a.mask_stride = (int64_t)L.Q * L.max_blocks;
      a.work_stride = (int64_t)L.Q * L.blk_stride;
      a.req_stride = L.Q;
      bool any = false;
      for (int i = 0; i < nl; ++i) {
        a.sp[i] = st->sparsity[l0 + i];
        any = any || a.sp[i] > 0.0f;
        st->prep[l0 + i].ready = false;
      }
      spin_status r = SPIN_OK;
      if (any) r = cuda_status(staged(st, kPredict, s, [&] { return launch_predict_pool(a, s); }));
      if (r == SPIN_OK) r = cuda_status(staged(st, kSelect, s, [&] { return launch_select(a, s); }));
      if (r != SPIN_OK) return r;
      for (int i = 0; i < nl; ++i) mark(l0 + i);
    }
    return SPIN_OK;
  }
  // other poolings: the per-layer kernels, layer l on stream l mod prep_k of
  // the state, whose block-score scratch only its own layers use
  cudaError_t e = cudaSuccess;
  for (int i = 0; i <= st->prep_k && e == cudaSuccess; ++i)
    if (!st->pev[i]) e = cudaEventCreateWithFlags(&st->pev[i], cudaEventDisableTiming);
  for (int i = 0; i < st->prep_k && e == cudaSuccess; ++i)
    if (!st->pstream[i]) e = cudaStreamCreateWithFlags(&st->pstream[i], cudaStreamNonBlocking);
  if (e == cudaSuccess) e = cudaEventRecord(st->pev[0], s);  // fork: after everything before on `stream`
  for (int i = 0; i < st->prep_k && e == cudaSuccess; ++i) e = cudaStreamWaitEvent(st->pstream[i], st->pev[0], 0);
  if (e != cudaSuccess) return cuda_status(e);
  for (int layer = 0; layer < L.L; ++layer) {
    const int i = layer % st->prep_k;
    cudaStream_t ps = st->pstream[i];
    st->prep[layer].ready = false;
    StepArgs a = step_args(st, layer, 1, step, ctx_len_dev, st->la_mask + (size_t)layer * L.Q * L.max_blocks);
    a.S = st->prep_S + (size_t)i * L.Q * L.R * L.blk_stride;
    a.work = st->la_work + (size_t)layer * L.Q * L.blk_stride;
    a.kept = st->la_kept + (size_t)layer * L.Q;
    a.ctx_sel = st->la_ctx + (size_t)layer * L.Q;
    a.no_pdl = layer < st->prep_k ? 1 : 0;  // a stream's first launch follows the fork's wait
    spin_status r = SPIN_OK;
    if (a.sparsity > 0.0f) {
      r = cuda_status(staged(st, kPredict, ps, [&] { return launch_predict_pool(a, ps); }));
      a.no_pdl = 0;
    }
    if (r == SPIN_OK) r = cuda_status(staged(st, kSelect, ps, [&] { return launch_select(a, ps); }));
    if (r != SPIN_OK) return r;
    mark(layer);
  }
  for (int i = 0; i < st->prep_k && e == cudaSuccess; ++i) {  // join
    e = cudaEventRecord(st->pev[1 + i], st->pstream[i]);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(s, st->pev[1 + i], 0);
  }
  return cuda_status(e);
}

spin_status spin_set_step(spin_state st, int64_t step, spin_stream_t stream) {
  if (!alive(st)) return SPIN_ESTATE;
  if (step < 0) return SPIN_EINVAL;
  return cuda_status(launch_step_op(st->step_dev, true, step, (cudaStream_t)stream));
}

spin_status spin_advance_step(spin_state st, spin_stream_t stream) {
  if (!alive(st)) return SPIN_ESTATE;
  return cuda_status(launch_step_op(st->step_dev, false, 0, (cudaStream_t)stream));
}

spin_status spin_set_kernel_timing(spin_state st, int enable) {
  if (!alive(st)) return SPIN_ESTATE;
  st->timing = enable != 0 ? 0xFFu : 0u;
  return SPIN_OK;
}

spin_status spin_set_kernel_timing_mask(spin_state st, uint32_t stage_mask) {
  if (!alive(st)) return SPIN_ESTATE;
  if (stage_mask >> kNumStages) return SPIN_EINVAL;
  st->timing = stage_mask;
  return SPIN_OK;
}

spin_status spin_kernel_times(spin_state st, double* ms_out, int64_t* launches_out, int n) {
  if (!alive(st)) return SPIN_ESTATE;
  if (n < 0 || n > kNumStages) return SPIN_EINVAL;
  double ms[kNumStages] = {0};
  cudaError_t err = cudaSuccess;
  for (auto& r : st->recs) {
    float t = 0.f;
    cudaError_t e = cudaEventSynchronize(r.b);
    if (e == cudaSuccess) e = cudaEventElapsedTime(&t, r.a, r.b);
    if (e != cudaSuccess && err == cudaSuccess) err = e;
    ms[r.stage] += t;
    st->pool.push_back(r.a);
    st->pool.push_back(r.b);
  }
  st->recs.clear();
  for (int i = 0; i < n; ++i) {
    if (ms_out) ms_out[i] = ms[i];
    if (launches_out) launches_out[i] = st->launches[i];
  }
  for (int i = 0; i < kNumStages; ++i) st->launches[i] = 0;
  return cuda_status(err);
}

spin_status spin_set_fault_injection(spin_state st, int mode) {
  if (!alive(st)) return SPIN_ESTATE;
  if (mode < 0 || mode > 1) return SPIN_EINVAL;
  st->inject = mode;
  return SPIN_OK;
}

spin_status spin_reset_requests(spin_state st, int layer, const int32_t* req_host, int n,
                                spin_stream_t stream) {
  if (!alive(st)) return SPIN_ESTATE;
  if (n < 0 || (n > 0 && !req_host) || layer >= st->cfg.num_layers) return SPIN_EINVAL;
  if (n == 0) return SPIN_OK;
  for (int i = 0; i < n; ++i)
    if (req_host[i] < 0 || req_host[i] >= st->cfg.num_requests) return SPIN_EINVAL;
  cudaStream_t s = (cudaStream_t)stream;
  const size_t per_layer = (size_t)st->lay.Q * st->lay.slot_stride;
  for (int l = 0; l < st->cfg.num_layers; ++l)
    if (layer < 0 || l == layer) st->prep[l].ready = false;   // the state changes under the prepared selection
  for (int i0 = 0; i0 < n; i0 += ReqList::kMax) {
    ReqList list;
    list.n = std::min(n - i0, ReqList::kMax);
    for (int i = 0; i < list.n; ++i) list.ids[i] = req_host[i0 + i];
    for (int l = 0; l < st->cfg.num_layers; ++l) {
      if (layer >= 0 && l != layer) continue;
      cudaError_t e = launch_reset_rows(st->V + per_layer * l, st->D + per_layer * l, vmax_of(st, l), list,
                                        st->lay.slot_stride, st->lay.vg_stride, s);
      if (e != cudaSuccess) return cuda_status(e);
    }
  }
  return SPIN_OK;
}

spin_status spin_predict_select(spin_state st, int layer, int rows, int64_t step,
                                const int32_t* ctx_len_dev, uint8_t* mask_dev, spin_stream_t stream) {
  if (!alive(st)) return SPIN_ESTATE;
  if (layer < 0 || layer >= st->cfg.num_layers || check_rows(st, rows) || !ctx_len_dev || !mask_dev ||
      step < SPIN_STEP_DEVICE)
    return SPIN_EINVAL;
  StepArgs a = step_args(st, layer, rows, step, ctx_len_dev, mask_dev);
  cudaStream_t s = (cudaStream_t)stream;
  if (a.sparsity > 0.0f) {
    spin_status r = cuda_status(staged(st, kPredict, s, [&] { return launch_predict_pool(a, s); }));
    if (r != SPIN_OK) return r;
  }
  return cuda_status(staged(st, kSelect, s, [&] { return launch_select(a, s); }));
}

spin_status spin_indexer_score(spin_state st, int layer, int rows, const void* keys, const float* key_scale,
                               int32_t num_pages, const int32_t* block_table, int32_t bt_stride,
                               const void* q, const float* w, const int32_t* ctx_len_dev,
                               const uint8_t* mask_dev, float* scores_dev, spin_stream_t stream) {
  if (!alive(st)) return SPIN_ESTATE;
  if (layer < 0 || layer >= st->cfg.num_layers || check_rows(st, rows)) return SPIN_EINVAL;
  if (!keys || !block_table || !q || !w || !ctx_len_dev || !mask_dev || !scores_dev || num_pages < 1 ||
      bt_stride < st->lay.max_blocks)
    return SPIN_EINVAL;
  if (st->cfg.key_dtype == SPIN_FP8_E4M3 && !key_scale) return SPIN_EINVAL;
  cudaStream_t s = (cudaStream_t)stream;
  spin_status r = cuda_status(staged(st, kCompact, s, [&] {
    return launch_compact(st->lay, rows, ctx_len_dev, mask_dev, st->work, st->kept, st->err, s);
  }));
  if (r != SPIN_OK) return r;
  return run_score(st, layer, rows, keys, key_scale, num_pages, block_table, bt_stride, q, w, ctx_len_dev,
                   mask_dev, scores_dev, false, s);
}

spin_status spin_topk(spin_state st, int rows, const float* scores_dev, const uint8_t* mask_dev,
                      const int32_t* ctx_len_dev, int32_t* topk_dev, spin_stream_t stream) {
  if (!alive(st)) return SPIN_ESTATE;
  if (check_rows(st, rows) || !scores_dev || !mask_dev || !ctx_len_dev || !topk_dev) return SPIN_EINVAL;
  cudaStream_t s = (cudaStream_t)stream;
  spin_status r = cuda_status(staged(st, kCompact, s, [&] {
    return launch_compact(st->lay, rows, ctx_len_dev, mask_dev, st->work, st->kept, st->err, s);
  }));
  if (r != SPIN_OK) return r;
  TopkArgs a{st->lay, rows, scores_dev, mask_dev, ctx_len_dev, st->work, st->kept, topk_dev, st->err, nullptr, 0};
  return cuda_status(staged(st, kTopk, s, [&] { return launch_topk(a, s); }));
}

spin_status spin_ema_update(spin_state st, int layer, int rows, const float* scores_dev, const uint8_t* mask_dev,
                            const int32_t* ctx_len_dev, const int32_t* accepted_dev, spin_stream_t stream) {
  if (!alive(st)) return SPIN_ESTATE;
  if (layer < 0 || layer >= st->cfg.num_layers || check_rows(st, rows) || !scores_dev || !mask_dev || !ctx_len_dev)
    return SPIN_EINVAL;
  EmaArgs a;
  a.lay = st->lay;
  a.rows = rows;
  a.row0 = st->cfg.mtp_policy == SPIN_MTP_ROW0 && rows > 1;
  a.scores = scores_dev;
  a.mask = mask_dev;
  a.ctx_len = ctx_len_dev;
  a.accepted = accepted_dev;
  const size_t per_layer = (size_t)st->lay.Q * st->lay.slot_stride;
  a.V = st->V + per_layer * layer;
  a.D = st->D + per_layer * layer;
  a.vmax = vmax_of(st, layer);
  a.alpha = st->cfg.alpha;
  a.beta = beta_of(st->cfg.alpha);
  a.err = st->err;
  cudaStream_t s = (cudaStream_t)stream;
  st->prep[layer].ready = false;
  return cuda_status(staged(st, kEma, s, [&] { return launch_ema_update(a, s); }));
}

spin_status spin_decode_step(spin_state st, int layer, int rows, int64_t step, const void* keys,
                             const float* key_scale, int32_t num_pages, const int32_t* block_table,
                             int32_t bt_stride, const void* q, const float* w, const int32_t* ctx_len_dev,
                             int defer_update, uint8_t* mask_dev, int32_t* topk_dev, float* scores_dev,
                             spin_stream_t stream) {
  if (!alive(st)) return SPIN_ESTATE;
  if (layer < 0 || layer >= st->cfg.num_layers || check_rows(st, rows) || step < SPIN_STEP_DEVICE)
    return SPIN_EINVAL;
  if (!keys || !block_table || !q || !w || !ctx_len_dev || !mask_dev || !topk_dev || num_pages < 1 ||
      bt_stride < st->lay.max_blocks)
    return SPIN_EINVAL;
  if (st->cfg.key_dtype == SPIN_FP8_E4M3 && !key_scale) return SPIN_EINVAL;
  if (defer_update && !scores_dev) return SPIN_EINVAL;
  float* scores = scores_dev ? scores_dev : st->scores;
  cudaStream_t s = (cudaStream_t)stream;
  const bool fp8 = st->cfg.key_dtype == SPIN_FP8_E4M3;
  if (st->lookahead && rows == 1 && !defer_update && fp8 && use_tc(st, 1))
    return decode_step_lookahead(st, layer, step, keys, key_scale, num_pages, block_table, bt_stride, q, w,
                                 ctx_len_dev, mask_dev, topk_dev, scores, s);
  st->prep[layer].ready = false;  // this step's EMA update moves the state under any prepared selection
  StepArgs a = step_args(st, layer, rows, step, ctx_len_dev, mask_dev);
  if (fp8) {  // a0 rides in the predict kernel, or in select when there is no prediction
    a.q = q;
    a.w = w;
    a.q8 = st->q8;
    a.wq = st->wq;
  }
  spin_status r;
  if (a.sparsity > 0.0f) {
    r = cuda_status(staged(st, kPredict, s, [&] { return launch_predict_pool(a, s); }));
    if (r != SPIN_OK) return r;
    a.q8 = nullptr;  // done
  }
  r = cuda_status(staged(st, kSelect, s, [&] { return launch_select(a, s); }));
  if (r != SPIN_OK) return r;
  const bool fuse = !defer_update && rows == 1;
  bool gm = false;
  r = run_score(st, layer, rows, keys, key_scale, num_pages, block_table, bt_stride, q, w, ctx_len_dev, mask_dev,
                scores, fuse, s, &gm, fp8);
  if (r != SPIN_OK) return r;
  TopkArgs t{st->lay, rows, scores, mask_dev, ctx_len_dev, st->work, st->kept, topk_dev, st->err,
             gm ? st->gmax : nullptr, st->gstride};
  r = cuda_status(staged(st, kTopk, s, [&] { return launch_topk(t, s); }));
  if (r != SPIN_OK) return r;
  if (!defer_update && rows > 1) return spin_ema_update(st, layer, rows, scores, mask_dev, ctx_len_dev, nullptr, stream);
  return SPIN_OK;
}

spin_status spin_slot_prediction(spin_state st, int layer, int rows, int kind, int64_t step,
                                 const int32_t* ctx_len_dev, float* pred_dev, spin_stream_t stream) {
  if (!alive(st)) return SPIN_ESTATE;
  if (layer < 0 || layer >= st->cfg.num_layers || check_rows(st, rows) || step < SPIN_STEP_DEVICE ||
      (kind != SPIN_PRED_EMA && kind != SPIN_PRED_RANDOM) || !ctx_len_dev || !pred_dev)
    return SPIN_EINVAL;
  const size_t per_layer = (size_t)st->lay.Q * st->lay.slot_stride;
  cudaStream_t s = (cudaStream_t)stream;
  return cuda_status(launch_slot_prediction(st->lay, rows, kind, step < 0 ? 0 : step,
                                            step == SPIN_STEP_DEVICE ? st->step_dev : nullptr, st->cfg.seed, layer,
                                            ctx_len_dev, st->V + per_layer * layer, st->D + per_layer * layer,
                                            pred_dev, st->err, s));
}

spin_status spin_pearson(spin_state st, int rows, const float* x_dev, const float* y_dev,
                         const int32_t* ctx_len_dev, double* pearson_dev, spin_stream_t stream) {
  if (!alive(st)) return SPIN_ESTATE;
  if (check_rows(st, rows) || !x_dev || !y_dev || !ctx_len_dev || !pearson_dev) return SPIN_EINVAL;
  cudaStream_t s = (cudaStream_t)stream;
  return cuda_status(launch_pearson(st->lay, rows, x_dev, y_dev, ctx_len_dev, pearson_dev, st->err, s));
}

spin_status spin_topk_overlap(spin_state st, int rows, const int32_t* a_dev, const int32_t* b_dev,
                              int32_t* overlap_dev, spin_stream_t stream) {
  if (!alive(st)) return SPIN_ESTATE;
  if (check_rows(st, rows) || !a_dev || !b_dev || !overlap_dev) return SPIN_EINVAL;
  cudaStream_t s = (cudaStream_t)stream;
  return cuda_status(launch_topk_overlap(st->lay.Q * rows, st->lay.k, a_dev, b_dev, overlap_dev, s));
}

spin_status spin_miss_count(spin_state st, int rows, const int32_t* full_topk_dev, const uint8_t* mask_dev,
                            int32_t* missed_dev, int32_t* total_dev, spin_stream_t stream) {
  if (!alive(st)) return SPIN_ESTATE;
  if (check_rows(st, rows) || !full_topk_dev || !mask_dev || !missed_dev || !total_dev) return SPIN_EINVAL;
  cudaStream_t s = (cudaStream_t)stream;
  return cuda_status(staged(st, kMiss, s, [&] {
    return launch_miss_count(st->lay, rows, full_topk_dev, mask_dev, missed_dev, total_dev, s);
  }));
}

// Exact water-filling: g(c) = sum_l clamp(c a_l, lo_l, 1) N_l is piecewise
// linear and non-decreasing in c with breakpoints lo_l / a_l and 1 / a_l;
// walk the sorted breakpoints to the segment that reaches the target and
// solve the linear piece.
spin_status spin_allocate_layer_sparsity(int n, const double* miss, const double* blocks, const double* lo,
                                         double s_glob, float* s_out) {
  if (n < 1 || !miss || !blocks || !lo || !s_out || !(s_glob >= 0.0 && s_glob < 1.0)) return SPIN_EINVAL;
  std::vector<double> a(n);
  double total = 0.0, floor_kept = 0.0;
  for (int l = 0; l < n; ++l) {
    if (!(miss[l] >= 0.0) || !(blocks[l] > 0.0) || !(lo[l] > 0.0 && lo[l] <= 1.0)) return SPIN_EINVAL;
    a[l] = miss[l] + 1e-3;
    total += blocks[l];
    floor_kept += lo[l] * blocks[l];
  }
  const double target = (1.0 - s_glob) * total;
  if (floor_kept >= target) {
    for (int l = 0; l < n; ++l) s_out[l] = (float)(1.0 - lo[l]);
    return SPIN_OK;
  }
  auto g = [&](double c) {
    double t = 0.0;
    for (int l = 0; l < n; ++l) t += std::min(1.0, std::max(lo[l], c * a[l])) * blocks[l];
    return t;
  };
  std::vector<double> bp;
  for (int l = 0; l < n; ++l) {
    bp.push_back(lo[l] / a[l]);
    bp.push_back(1.0 / a[l]);
  }
  std::sort(bp.begin(), bp.end());
  double c = bp.back();
  double prev = 0.0, g_prev = g(0.0);
  for (double x : bp) {
    const double gx = g(x);
    if (gx >= target) {
      // linear between prev and x
      c = (gx == g_prev) ? x : prev + (target - g_prev) * (x - prev) / (gx - g_prev);
      break;
    }
    prev = x;
    g_prev = gx;
  }
  for (int l = 0; l < n; ++l) s_out[l] = (float)(1.0 - std::min(1.0, std::max(lo[l], c * a[l])));
  return SPIN_OK;
}

spin_status spin_get_error(spin_state st, spin_stream_t stream, uint32_t* word_out) {
  if (!alive(st)) return SPIN_ESTATE;
  cudaStream_t s = (cudaStream_t)stream;
  ErrWord h{};
  cudaError_t e = cudaStreamSynchronize(s);
  if (e == cudaSuccess) e = cudaMemcpyAsync(&h, st->err, sizeof(ErrWord), cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaMemsetAsync(st->err, 0, sizeof(ErrWord), s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_status(e);
  if (word_out) *word_out = h.flags;
  if (h.flags & ERR_TIMEOUT) return SPIN_ETIMEOUT;
  if (h.flags) return SPIN_EDEVICE;
  return SPIN_OK;
}

const char* spin_status_string(spin_status s) {
  switch (s) {
    case SPIN_OK: return "ok";
    case SPIN_EINVAL: return "invalid argument";
    case SPIN_ENOMEM: return "state block too small";
    case SPIN_ECUDA: return "CUDA runtime error";
    case SPIN_ESTATE: return "invalid state handle";
    case SPIN_ETIMEOUT: return "device wait timed out";
    case SPIN_EDEVICE: return "device-side argument check failed";
    case SPIN_EUNSUPPORTED: return "shape not supported by the requested kernel";
  }
  return "unknown status";
}

size_t spin_state_export_bytes(spin_state st) {
  if (!alive(st)) return 0;
  return (size_t)2 * st->lay.L * st->lay.Q * st->lay.slot_stride * sizeof(float);
}

spin_status spin_state_export(spin_state st, void* host, size_t bytes, spin_stream_t stream) {
  if (!alive(st)) return SPIN_ESTATE;
  const size_t half = spin_state_export_bytes(st) / 2;
  if (!host || bytes < 2 * half) return SPIN_EINVAL;
  cudaStream_t s = (cudaStream_t)stream;
  cudaError_t e = cudaMemcpyAsync(host, st->V, half, cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaMemcpyAsync((char*)host + half, st->D, half, cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  return cuda_status(e);
}

spin_status spin_state_import(spin_state st, const void* host, size_t bytes, spin_stream_t stream) {
  if (!alive(st)) return SPIN_ESTATE;
  const size_t half = spin_state_export_bytes(st) / 2;
  if (!host || bytes < 2 * half) return SPIN_EINVAL;
  cudaStream_t s = (cudaStream_t)stream;
  for (auto& p : st->prep) p.ready = false;
  cudaError_t e = cudaMemcpyAsync(st->V, host, half, cudaMemcpyHostToDevice, s);
  if (e == cudaSuccess) e = cudaMemcpyAsync(st->D, (const char*)host + half, half, cudaMemcpyHostToDevice, s);
  if (e == cudaSuccess)
    e = launch_vmax_refresh(st->V, st->vmax, (int64_t)st->lay.L * st->lay.Q, st->lay.slot_stride, st->lay.vg_stride, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  return cuda_status(e);
}

spin_status spin_state_refresh(spin_state st, int layer, spin_stream_t stream) {
  if (!alive(st)) return SPIN_ESTATE;
  if (layer < -1 || layer >= st->cfg.num_layers) return SPIN_EINVAL;
  for (int l = 0; l < st->cfg.num_layers; ++l)
    if (layer < 0 || l == layer) st->prep[l].ready = false;  // the state changed under the prepared selection
  if (!st->vmax) return SPIN_OK;
  const int64_t layers = layer < 0 ? st->lay.L : 1;
  const size_t per_layer = (size_t)st->lay.Q * st->lay.slot_stride;
  const float* V = st->V + per_layer * (layer < 0 ? 0 : layer);
  return cuda_status(launch_vmax_refresh(V, vmax_of(st, layer < 0 ? 0 : layer), layers * st->lay.Q,
                                         st->lay.slot_stride, st->lay.vg_stride, (cudaStream_t)stream));
}

spin_status spin_state_ema(spin_state st, int layer, float** V, float** D, int64_t* stride) {
  if (!alive(st)) return SPIN_ESTATE;
  if (layer < 0 || layer >= st->cfg.num_layers) return SPIN_EINVAL;
  const size_t per_layer = (size_t)st->lay.Q * st->lay.slot_stride;
  if (V) *V = st->V + per_layer * layer;
  if (D) *D = st->D + per_layer * layer;
  if (stride) *stride = st->lay.slot_stride;
  return SPIN_OK;
}

spin_status spin_state_vmax(spin_state st, int layer, const float** vmax, int64_t* stride) {
  if (!alive(st)) return SPIN_ESTATE;
  if (layer < 0 || layer >= st->cfg.num_layers) return SPIN_EINVAL;
  if (vmax) *vmax = vmax_of(st, layer);
  if (stride) *stride = st->lay.vg_stride;
  return SPIN_OK;
}

spin_status spin_state_block_scores(spin_state st, const float** S, int64_t* stride) {
  if (!alive(st)) return SPIN_ESTATE;
  if (S) *S = st->S;
  if (stride) *stride = st->lay.blk_stride;
  return SPIN_OK;
}

spin_status spin_state_qquant(spin_state st, const uint8_t** q8, const float** wq) {
  if (!alive(st)) return SPIN_ESTATE;
  if (q8) *q8 = st->q8;
  if (wq) *wq = st->wq;
  return SPIN_OK;
}

int64_t spin_score_stride(spin_state st) { return alive(st) ? st->lay.slot_stride : -1; }
int64_t spin_mask_stride(spin_state st) { return alive(st) ? st->lay.max_blocks : -1; }

}  // extern "C"
