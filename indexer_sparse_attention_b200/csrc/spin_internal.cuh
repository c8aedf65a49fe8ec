// spin_internal.cuh -- state layout, error word and device helpers shared by
// the SPIN kernels (sm_100a).  Nothing here is part of the C ABI.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <stdint.h>

#include "../../include/spin.h"

namespace spin {

// ---------------------------------------------------------------------------
// Device error word: bits OR-ed by kernels, read by spin_get_error.
// ---------------------------------------------------------------------------
enum : uint32_t {
  ERR_CTX_LEN = 1u << 0,      // ctx_len < 1 or ctx_len + rows - 1 > max_slots
  ERR_PAGE = 1u << 1,         // block-table entry outside [0, num_pages)
  ERR_ACCEPTED = 1u << 2,     // accepted length outside 1..rows
  ERR_TIMEOUT = 1u << 3,      // a bounded mbarrier wait gave up
  ERR_CAPACITY = 1u << 4,     // a shape exceeded a kernel's on-chip capacity
  ERR_LOOKAHEAD = 1u << 5,    // ctx_len differs from the one a prepared selection was made for
};

// Error word block: [0] flags, [1] first offending request, [2] first value.
struct ErrWord {
  uint32_t flags;
  uint32_t request;
  uint32_t value;
  uint32_t pad;
};

__device__ __forceinline__ void raise_error(ErrWord* e, uint32_t bit, uint32_t req, uint32_t val) {
  uint32_t old = atomicOr(&e->flags, bit);
  if (old == 0) {
    e->request = req;
    e->value = val;
  }
}

// Host-side view of a state; the device block is carved as documented in
// spin_state_bytes (spin_api.cu).
struct Layout {
  int32_t L, Q, R, H, d, b, k;
  int64_t max_slots;
  int64_t max_blocks;    // ceil(max_slots / b)
  int64_t slot_stride;   // max_blocks * b  (a score / V / D row)
  int64_t blk_stride;    // max_blocks rounded up to 16 (mask, S, work-list rows)
  int64_t vg_stride;     // slot_stride / 32 (a row of V's 32-slot group maxima), or 0 when
                         // they are not kept (block size 16, or a pooling other than max)
};

// ---------------------------------------------------------------------------
// Positions (see spin.h): row r sits at p_r = ctx_len - 1 + r.
// ---------------------------------------------------------------------------
__host__ __device__ __forceinline__ int64_t row_pos(int64_t ctx_len, int r) { return ctx_len - 1 + r; }
__host__ __device__ __forceinline__ int64_t row_blocks(int64_t ctx_len, int r, int b) {
  return (ctx_len + r + b - 1) / b;
}

// Budget of a row and the exploration count (computed in double from the
// fp32 parameters, the same definition the host code uses).
__device__ __forceinline__ int64_t block_budget(int64_t n, float s) {
  return n - (int64_t)floor((double)s * (double)n);
}
__device__ __forceinline__ int64_t explore_count(int64_t budget0, float g) {
  return (int64_t)floor((double)g * (double)budget0);
}

// ---------------------------------------------------------------------------
// Order-preserving map float -> uint32: larger float <=> larger key.  -0 is
// folded onto +0 so that the two compare equal, as floats do.
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t fkey(float x) {
  uint32_t u = __float_as_uint(x == 0.0f ? 0.0f : x);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// ---------------------------------------------------------------------------
// Philox4x32-10 (Salmon et al., "Parallel Random Numbers: As Easy as 1, 2, 3",
// SC'11).  Per round: two 32x32->64 products of counter words 0 and 2 with the
// Philox-4x32 multipliers, outputs (hi(c2*M1)^c1^k0, lo(c2*M1),
// hi(c0*M0)^c3^k1, lo(c0*M0)); the key advances by the Weyl increments.
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint4 philox4x32_10(uint4 c, uint2 k) {
  constexpr uint32_t kMulA = 0xD2511F53u, kMulB = 0xCD9E8D57u;
  constexpr uint32_t kWeylA = 0x9E3779B9u, kWeylB = 0xBB67AE85u;
#pragma unroll
  for (int i = 0; i < 10; ++i) {
    const uint32_t loA = kMulA * c.x, hiA = __umulhi(kMulA, c.x);
    const uint32_t loB = kMulB * c.z, hiB = __umulhi(kMulB, c.z);
    c = make_uint4(hiB ^ c.y ^ k.x, loB, hiA ^ c.w ^ k.y, loA);
    k.x += kWeylA;
    k.y += kWeylB;
  }
  return c;
}

// Exploration keys of blocks 4i .. 4i+3: words 0..3 of Philox at counter
// (i, request, layer, step mod 2^32) under key (seed lo, seed hi); block j
// takes word j mod 4 of counter j div 4.
__device__ __forceinline__ uint4 explore_keys4(uint64_t seed, uint32_t i, uint32_t req, uint32_t layer,
                                               uint64_t step) {
  return philox4x32_10(make_uint4(i, req, layer, (uint32_t)step), make_uint2((uint32_t)seed, (uint32_t)(seed >> 32)));
}
__device__ __forceinline__ uint32_t word_of(uint4 w, int k) {
  return k == 0 ? w.x : k == 1 ? w.y : k == 2 ? w.z : w.w;
}
__device__ __forceinline__ uint32_t explore_key(uint64_t seed, uint32_t j, uint32_t req,
                                                uint32_t layer, uint64_t step) {
  return word_of(explore_keys4(seed, j >> 2, req, layer, step), (int)(j & 3));
}

// Maximum of x over the 32 lanes of a warp, all of them active: one
// redux.sync on sm_100a.  The callers' values are never NaN.
__device__ __forceinline__ float warp_max(float x) {
  float r;
  asm volatile("redux.sync.max.f32 %0, %1, 0xffffffff;" : "=f"(r) : "f"(x));
  return r;
}

// EMA update with never-observed sentinels (+inf for V, -inf for D).
__device__ __forceinline__ float ema_v(float x, float y, float alpha, float beta) {
  return (x == __int_as_float(0x7f800000)) ? y : __fmaf_rn(alpha, x, __fmul_rn(beta, y));
}
__device__ __forceinline__ float ema_d(float x, float y, float alpha, float beta) {
  return (x == __int_as_float(0xff800000)) ? y : __fmaf_rn(alpha, x, __fmul_rn(beta, y));
}

// E4M3 pair -> float2 (exact).
__device__ __forceinline__ float2 e4m3x2_to_float2(uint16_t v) {
  __half2_raw h = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)v, __NV_E4M3);
  __half2 hh;
  memcpy(&hh, &h, sizeof(hh));
  return __half22float2(hh);
}

// ---------------------------------------------------------------------------
// a0: query quantisation of one (request, row, head) vector by one warp.  The
// vector is scaled by 2^-e, e = smallest integer with amax <= 448 * 2^e, and
// rounded to E4M3 (nearest, saturating); the head weight absorbs 2^e, since
// ReLU(c x) = c ReLU(x) for c > 0.  The pages give no precision; this is the
// reading used throughout.
// ---------------------------------------------------------------------------
// 2^k as a float for k in [-126, 127].
__device__ __forceinline__ float pow2f(int k) { return __uint_as_float((uint32_t)(k + 127) << 23); }

// Smallest e with amax <= 448 * 2^e from the exponent and mantissa bits:
// amax = (1 + f) 2^E -> e = E - 8 if 1 + f <= 1.75 else E - 7.
__device__ __forceinline__ int q_exponent(float amax) {
  if (!(amax > 0.0f)) return 0;
  uint32_t u = __float_as_uint(amax);
  int E = (int)((u >> 23) & 0xFF);
  uint32_t frac = u & 0x7FFFFFu;
  if (E == 0) {  // subnormal: normalise the fraction
    int msb = 31 - __clz(frac);
    E = msb - 149 + 127;
    frac = (frac << (23 - msb)) & 0x7FFFFFu;
  }
  return (E - 127) - 8 + (frac > 0x600000u ? 1 : 0);
}

__device__ __forceinline__ float load_q(const void* q, int64_t i, int bf16) {
  if (bf16) return __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(q)[i]);
  return reinterpret_cast<const float*>(q)[i];
}

// Vector v (elements v*d .. v*d + d - 1 of q, weight w[v]) -> q8, wq[v].
// Called by all 32 lanes of a warp.
__device__ __forceinline__ void quantize_vec(const void* q, const float* w, int q_bf16, int d, int64_t v,
                                             uint8_t* q8, float* wq) {
  const int lane = threadIdx.x & 31;
  const int64_t base = v * d;
  float amax = 0.0f;
  for (int i = lane; i < d; i += 32) amax = fmaxf(amax, fabsf(load_q(q, base + i, q_bf16)));
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  const int e = q_exponent(amax);
  // x * 2^-e, split in two exact steps when 2^-e is not a normal float.
  const int ne = -e;
  const int s1 = ne > 127 ? 127 : ne;
  const int s2 = ne - s1;
  const float f1 = pow2f(s1), f2 = pow2f(s2);
  for (int i = 2 * lane; i < d; i += 64) {
    float x0 = load_q(q, base + i, q_bf16) * f1 * f2;
    float x1 = (i + 1 < d) ? load_q(q, base + i + 1, q_bf16) * f1 * f2 : 0.0f;
    __nv_fp8x2_storage_t p = __nv_cvt_float2_to_fp8x2(make_float2(x0, x1), __NV_SATFINITE, __NV_E4M3);
    q8[base + i] = (uint8_t)(p & 0xFF);
    if (i + 1 < d) q8[base + i + 1] = (uint8_t)(p >> 8);
  }
  if (lane == 0) wq[v] = __double2float_rn((double)w[v] * ldexp(1.0, e));  // w * 2^e rounded once
}

// ---------------------------------------------------------------------------
// Programmatic dependent launch.  The decode step's kernels are launched so
// that each may be scheduled while its predecessor in the stream finishes,
// which hides the launch gap.  Each of them starts by waiting until every
// earlier grid has completed and its memory is visible (a no-op for an
// ordinary launch), and only then lets its own successor be scheduled, so
// the stream's ordering is kept for every byte either kernel touches.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void pdl_enter() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// Launch configuration with programmatic stream serialization; use in place.
struct PdlLaunch {
  cudaLaunchConfig_t cfg;
  cudaLaunchAttribute attr[2];
  PdlLaunch(dim3 grid, dim3 block, size_t smem, cudaStream_t s) : cfg(), attr() {
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
  }
  PdlLaunch(const PdlLaunch&) = delete;
  PdlLaunch& operator=(const PdlLaunch&) = delete;
};

// ---------------------------------------------------------------------------
// Kernel launchers (one per .cu file).  All return cudaGetLastError().
// ---------------------------------------------------------------------------
constexpr int kMaxLayerBatch = 8;  // layers in one launch of the prepared selections

// Candidates the top-k keeps on chip (k_topk.cu).
constexpr int kTopkCandCap = 8192;

// Whether the top-k can take its group-maxima path for a row whose request
// kept `kept_blocks` blocks of b slots: the path is tried only when the scored
// slots overflow the on-chip candidates (so it wants min(k, kTopkCandCap + 1)
// scores at the least) and needs at least two 32-slot groups per wanted
// score.  Where it cannot, the score kernel need not write the group maxima.
__host__ __device__ inline bool topk_group_path_possible(int64_t kept_blocks, int b, int k) {
  const int64_t want_min = k < kTopkCandCap + 1 ? k : kTopkCandCap + 1;
  return kept_blocks * b + 31 >= 64 * want_min;
}

struct StepArgs {
  Layout lay;
  int layer, rows;
  int64_t step;
  const int64_t* step_dev;  // non-null: the step is read from the state's counter
  int64_t step_add;         // added to the counter's step (a selection prepared one step ahead)
  int pooling;              // spin_pooling: block reduction of the predicted scores
  int mtp_row0;             // SPIN_MTP_ROW0 with rows > 1: row 0 alone predicts
  float sparsity, gamma, alpha;
  uint64_t seed;
  const int32_t* ctx_len;
  uint8_t* mask;
  float* S;
  int32_t* work;      // [Q][blk_stride] kept block ids, ascending
  int32_t* kept;      // [Q] kept counts
  int32_t* ctx_sel;   // [Q] out, or null: the ctx_len each request's selection was made for (-1: none)
  int quiet;          // a selection prepared one step ahead: an out-of-range ctx_len is no error
                      // (the request gets no selection, ctx_sel -1)
  int no_pdl;         // launch as an ordinary dependent (after a wait on another stream's event)

  float* V;           // layer base [Q][slot_stride]
  float* D;
  const float* vmax;  // layer base [Q][vg_stride]: max of V over each aligned 32-slot group, or null
  ErrWord* err;
  // a0 folded into the select kernel (decode step with FP8 keys), or q8 null
  const void* q;      // [Q][rows][H][d]
  const float* w;     // [Q][rows][H]
  int q_bf16;
  uint8_t* q8;
  float* wq;
  // Several layers in one launch (prepared selections; one-row max-pooled
  // predict and the one-CTA select): blockIdx.z is the layer's place in the
  // batch, every per-layer pointer above advances by its stride per place,
  // and the layer's target is sp[place].  nl = 1: the fields above are the
  // one layer's.
  int nl;
  int64_t state_stride, vg_layer_stride, s_stride, mask_stride, work_stride, req_stride;
  float sp[kMaxLayerBatch];
};

// The layer of this block in a launch over several layers (StepArgs::nl).
__device__ __forceinline__ void layer_of_block(StepArgs& a) {
  const int l = (int)blockIdx.z;
  a.layer += l;
  a.sparsity = a.sp[l];
  a.V += l * a.state_stride;
  a.D += l * a.state_stride;
  if (a.vmax) a.vmax += l * a.vg_layer_stride;
  a.S += l * a.s_stride;
  a.mask += l * a.mask_stride;
  a.work += l * a.work_stride;
  a.kept += l * a.req_stride;
  if (a.ctx_sel) a.ctx_sel += l * a.req_stride;
}

// V = +inf, D = -inf over n slots, and vmax (nv groups, or null) = +inf.
cudaError_t launch_init_state(float* V, float* D, int64_t n, float* vmax, int64_t nv, cudaStream_t s);
// vmax[g] = max(V[32 g .. 32 g + 31]) for rows rows of V (stride slot_stride) and vmax (stride vg_stride).
cudaError_t launch_vmax_refresh(const float* V, float* vmax, int64_t rows, int64_t slot_stride, int64_t vg_stride,
                                cudaStream_t s);
// Sets (*p = value) or advances (*p += 1) the device step counter.
cudaError_t launch_step_op(int64_t* p, bool set, int64_t value, cudaStream_t s);
struct ReqList {
  static constexpr int kMax = 32;
  int32_t ids[kMax];
  int n;
};
cudaError_t launch_reset_rows(float* V, float* D, float* vmax, const ReqList& list, int64_t stride,
                              int64_t vg_stride, cudaStream_t s);
cudaError_t launch_predict_pool(const StepArgs& a, cudaStream_t s);
cudaError_t launch_select(const StepArgs& a, cudaStream_t s);
cudaError_t launch_compact(const Layout& L, int rows, const int32_t* ctx_len, const uint8_t* mask,
                           int32_t* work, int32_t* kept, ErrWord* err, cudaStream_t s);

struct ScoreArgs {
  Layout lay;
  int rows;
  int key_fp8;        // 1: E4M3 keys + scale; 0: fp32 keys
  int q_bf16;         // 1: bf16 queries; 0: fp32
  const void* keys;
  const float* kscale;
  int32_t num_pages;
  const int32_t* block_table;
  int32_t bt_stride;
  const void* q;
  const float* w;
  const int32_t* ctx_len;
  const uint8_t* mask;
  const int32_t* work;
  const int32_t* kept;
  uint8_t* q8;        // [Q][R][H][d] quantised queries (FP8 keys)
  float* wq;          // [Q][R][H] folded weights
  float* scores;      // [Q][R][slot_stride]
  ErrWord* err;
  // fused EMA (rows == 1 only): V, D of the layer, or null
  float* V;
  float* D;
  float* vmax;         // with V: V's 32-slot group maxima of the layer, kept current, or null
  float alpha, beta;   // beta = fl32(1 - alpha), computed once on the host
  int inject;          // test hook: withhold the first key stage of CTA 0
  const int32_t* ctx_sel;  // [Q] or null: the ctx_len the selection was made for; a request whose
                           // ctx_len differs raises ERR_LOOKAHEAD and is not scored
  int32_t* ctx_next;       // [Q] or null: written with ctx_len + 1 (the next step's, one row a step)
  float* gmax;         // [Q][R][gstride] max score of each 32-slot group of the
  int64_t gstride;     // kept-slot order (tensor-core kernel only), or null
};

cudaError_t launch_quantize_q(const ScoreArgs& a, cudaStream_t s);
cudaError_t launch_score_simt(const ScoreArgs& a, cudaStream_t s);
bool tc_supported(const Layout& lay, int rows, int key_fp8);
cudaError_t launch_score_tc(const ScoreArgs& a, void* encode_fn, cudaStream_t s);

struct TopkArgs {
  Layout lay;
  int rows;
  const float* scores;
  const uint8_t* mask;
  const int32_t* ctx_len;
  const int32_t* work;
  const int32_t* kept;
  int32_t* topk;
  ErrWord* err;
  const float* gmax;  // group maxima written by the score kernel, or null
  int64_t gstride;
  const int32_t* ctx_sel;  // [Q] or null: a request whose ctx_len differs comes back all -1
};
cudaError_t launch_topk(const TopkArgs& a, cudaStream_t s);

struct EmaArgs {
  Layout lay;
  int rows;
  int row0;           // SPIN_MTP_ROW0: row 0's scores alone update the state
  const float* scores;
  const uint8_t* mask;
  const int32_t* ctx_len;
  const int32_t* accepted;
  float* V;
  float* D;
  float* vmax;        // V's 32-slot group maxima of the layer, kept current, or null
  float alpha, beta;
  ErrWord* err;
};
cudaError_t launch_ema_update(const EmaArgs& a, cudaStream_t s);

// Predictor-quality profile (k_quality.cu).
cudaError_t launch_slot_prediction(const Layout& L, int rows, int kind, int64_t step, const int64_t* step_dev,
                                   uint64_t seed, int layer, const int32_t* ctx_len, const float* V, const float* D,
                                   float* pred, ErrWord* err, cudaStream_t s);
cudaError_t launch_pearson(const Layout& L, int rows, const float* x, const float* y, const int32_t* ctx_len,
                           double* out, ErrWord* err, cudaStream_t s);
cudaError_t launch_topk_overlap(int pairs, int k, const int32_t* a, const int32_t* b, int32_t* out, cudaStream_t s);

cudaError_t launch_miss_count(const Layout& lay, int rows, const int32_t* full_topk,
                              const uint8_t* mask, int32_t* missed, int32_t* total,
                              cudaStream_t s);

}  // namespace spin
