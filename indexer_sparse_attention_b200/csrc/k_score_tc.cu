// k_score_tc.cu -- a3 paged FP8 indexer score on the 5th-generation tensor
// cores (sm_100a): TMA gathers key pages through the block table into
// shared memory, tcgen05.mma (kind::f8f6f4) accumulates in TMEM, and four
// epilogue warps finish the DSA lightning-indexer score
//   I_{r,s} = sigma_s * sum_h w'_{r,h} * ReLU(q8_{r,h} . k8_s)
// for the kept blocks only (SPIN listing, Abstract; SPIN digest, arXiv深度剖析:
// the indexer input is pruned to the kept blocks), plus -- for a single query
// row -- the EMA update of the scored slots (SPIN digest, 核心概要).
//
// Tile: M = 128 key tokens (two 64-token pages of one request, in kept-list
// order) x N = rows * H query heads x K = d = 128.  Both operands are
// K-major, 128-byte swizzled.  The contraction is dense and small per tile;
// the kernel is HBM-bound on the key stream (132 bytes per kept slot).
//
// Warp roles (320 threads, persistent, two CTAs per SM when N <= 128):
//   warp 0      producer: lanes gather the tile metadata one and two batches
//               of 32 tiles ahead; lane 0 handles the query tile (per request),
//               the stage barriers and the tile-info ring; two lanes issue the
//               tile's two key-page TMA loads.  The copy engine's cost is per
//               request, so it moves only key pages; a second CTA per SM adds
//               a second issuer.
//   warp 1      TMEM allocation; lane 0 issues the MMAs and one commit per
//               tile, which frees the key stage for the producer and marks
//               the accumulator full for the epilogue
//   warps 2..9  two epilogue groups of four warps, taking alternate tiles; a
//               thread owns one token: it loads the token's scale and EMA
//               values two tiles ahead, reads its accumulator row from the TMEM
//               quarter its warp may access (lanes 32*(warp%4) ..), hands
//               the accumulator back as soon as its last columns are in
//               registers, applies ReLU, head weights and the scale, and
//               stores the score and the fused EMA update (a warp's 32
//               tokens are one aligned group of V, whose maximum it also
//               stores for the next prediction).  With one CTA
//               per SM (N > 128) there are four groups; for several query
//               rows two groups share each tile, one taking the even rows and
//               the other the odd ones, so an accumulator is read out in half
//               the time
// Pipelines: key stages freed as soon as the MMAs have read them (6 per CTA
// at N = 64, 8 with one CTA per SM); a 16-slot ring of tile info freed by the
// epilogue; 1 query buffer with two CTAs per SM (2 with one); 4 TMEM
// accumulators (2 when N > 64), so that all CTAs of an SM fit the 512 TMEM
// columns.  Every wait is bounded (2 s of
// %globaltimer); on expiry the CTA raises ERR_TIMEOUT, stops issuing, drains
// what it issued and frees TMEM.
#include <cuda.h>

#include <algorithm>
#include <type_traits>

#include "block_scan.cuh"
#include "spin_internal.cuh"

namespace spin {
namespace {

constexpr int kTileM = 128;
constexpr int kPage = 64;          // tokens per page (block size)
constexpr int kRowBytes = 128;     // d = 128 FP8 values
constexpr int kPageBytes = kPage * kRowBytes;
constexpr int kStageBytes = kTileM * kRowBytes;
// Epilogue groups of 4 warps take tiles round robin: 2 groups with two CTAs
// per SM (N <= 128), 4 groups with one CTA per SM (the MTP rows' N = 256, whose
// epilogue reduces four rows of heads per token).
__host__ __device__ constexpr int threads_for(int groups) { return 64 + groups * 128; }
constexpr uint64_t kTimeoutNs = 2000000000ull;

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// ---------------------------------------------------------------------------
// PTX wrappers
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}
__device__ __forceinline__ uint64_t gtimer() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

struct Ctl {
  volatile int* abort_flag;
  ErrWord* err;
};

// Bounded wait on a phase parity: false on timeout (raises ERR_TIMEOUT and
// the CTA abort flag) or when another role already aborted.  The first test
// is inline; only a phase that is not yet complete calls the out-of-line
// loop, so a wait that succeeds at once is no function call (a call would
// make the caller's loads still in flight, such as the next tile's
// prefetch, complete first).
__device__ __noinline__ bool wait_parity_slow(uint32_t bar, uint32_t parity, Ctl c) {
  const uint64_t t0 = gtimer();
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 31u) == 0) {
      if (*c.abort_flag) return false;
      if (gtimer() - t0 > kTimeoutNs) {
        *c.abort_flag = 1;
        raise_error(c.err, ERR_TIMEOUT, blockIdx.x, bar);
        return false;
      }
    }
  }
}
__device__ __forceinline__ bool wait_parity(uint32_t bar, uint32_t parity, Ctl c) {
  return mbar_try_wait(bar, parity) || wait_parity_slow(bar, parity, c);
}

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, uint32_t bar, int x, int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], [%2];" ::"r"(
          dst),
      "l"((uint64_t)map), "r"(bar), "r"(x), "r"(y)
      : "memory");
}

// Shared-memory matrix descriptor, K-major, 128-byte swizzle: 8-row atoms of
// 128 B, stride between atoms (SBO) 1024 B, LBO unused (1), sm_100 version 1,
// base offset 0 (atoms 1024-byte aligned), layout type 2 = SWIZZLE_128B.
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr) {
  return (uint64_t)((saddr & 0x3FFFFu) >> 4) | ((uint64_t)1 << 16) | ((uint64_t)(1024 >> 4) << 32) |
         ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}

// Instruction descriptor of kind::f8f6f4: D fp32 (bit 4), A and B E4M3
// (format 0), both K-major, N >> 3 at bit 17, M >> 4 at bit 24.
__host__ __device__ constexpr uint32_t idesc_e4m3(int M, int N) {
  return (1u << 4) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

__device__ __forceinline__ void umma_e4m3(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a), "l"(b), "r"(idesc), "r"(acc)
      : "memory");
}
__device__ __forceinline__ void umma_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}
// Two independent fp32 fused multiply-adds (round to nearest) in one packed
// instruction: (a0, a1) += (w0 * x0, w1 * x1), each rounded once as fmaf.
__device__ __forceinline__ void fma2_rn(float& a0, float& a1, float w0, float w1, float x0, float x1) {
  asm("{\n\t.reg .b64 acc, w, x;\n\tmov.b64 acc, {%0, %1};\n\tmov.b64 w, {%2, %3};\n\t"
      "mov.b64 x, {%4, %5};\n\tfma.rn.f32x2 acc, w, x, acc;\n\tmov.b64 {%0, %1}, acc;\n\t}"
      : "+f"(a0), "+f"(a1)
      : "f"(w0), "f"(w1), "f"(x0), "f"(x1));
}
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// ---------------------------------------------------------------------------
// Tile schedule: tiles of a request are consecutive pairs of its kept-block
// list; the global tile order is (request, pair); CTA c takes a contiguous
// share, so a CTA mostly stays on one request and its query tile.
// ---------------------------------------------------------------------------
struct Sched {
  const int* prefix;  // [Q+1] tile prefix in shared memory
  int Q;
  __device__ int locate(int g) const {  // request holding global tile g
    int lo = 0, hi = Q - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (prefix[mid] <= g) lo = mid; else hi = mid - 1;
    }
    return lo;
  }
};

// Tile metadata the producer hands to the epilogue through a small ring in
// shared memory (the copy engine moves only key pages: its cost is per request,
// so the per-token scales and EMA values are read by the epilogue threads).
struct TileInfo {
  int q, ctx, np, t;  // t: pair index of the tile within its request
  int j[2], pg[2];    // block ids and pages; pg < 0 marks a page outside the cache
};

struct SmemLayout {
  uint32_t keys;     // stages * kStageBytes
  uint32_t aux;      // kAuxSlots * sizeof(TileInfo)
  uint32_t qbuf;     // 2 * N * 128
  uint32_t wq;       // 4 * groups * N floats: one copy per epilogue warp
  uint32_t prefix;   // (Q + 1) ints
  uint32_t bars;     // barriers
  uint32_t total;
};

constexpr int kMaxStages = 8;
constexpr int kMaxAcc = 4;
constexpr int kAuxSlots = 16;  // tile-info ring: freed by the epilogue, not by the MMA

__host__ __device__ inline SmemLayout smem_layout(int N, int Q, int stages, int nq, int groups) {
  SmemLayout s;
  uint32_t off = 0;
  s.keys = off;
  off += stages * kStageBytes;
  s.aux = off;
  off += kAuxSlots * (uint32_t)sizeof(TileInfo);
  off = (off + 1023) / 1024 * 1024;
  s.qbuf = off;
  off += nq * N * kRowBytes;
  s.wq = off;
  off += 4 * groups * N * 4;
  s.prefix = off;
  off += ((Q + 1) * 4 + 15) / 16 * 16;
  s.bars = off;
  off += (2 * kMaxStages + 2 * kAuxSlots + 4 + 2 * kMaxAcc + 1) * 8 + 16;
  s.total = off + 1024;  // slack for 1024-byte alignment of the base
  return s;
}

// Launch plan: two CTAs per SM when shared memory and TMEM allow (each CTA
// has one copy-issuing warp, and one issuer per CTA caps the copy rate), with
// accumulators sized so that CTAs * accumulators * N <= 512 TMEM columns.
struct TcPlan {
  int stages, nacc, ctas, nq;  // key stages, TMEM accumulators, CTAs per SM, query buffers
  int groups;                  // epilogue groups of four warps
};

__host__ __device__ inline TcPlan tc_plan(int N, int Q) {
  // two CTAs share an SM's 228 KB when each takes <= 113 KB (1 KB per CTA is
  // reserved); one query buffer (a request change drains the MMAs first, a
  // CTA meets one or two) leaves room for more key stages
  constexpr uint32_t kTwoPerSm = 115712;
  if (N <= 128)
    for (int st = kMaxStages; st >= 3; --st)
      if (smem_layout(N, Q, st, 1, 2).total <= kTwoPerSm) return {st, N <= 64 ? 4 : 2, 2, 1, 2};
  return {kMaxStages, 2, 1, 2, 4};
}

// Epilogue groups that share one tile: with four groups and several rows two
// groups split a tile's rows, so an accumulator is read out in half the time.
__host__ __device__ constexpr int groups_per_tile(int groups, int rows) { return (groups == 4 && rows >= 2) ? 2 : 1; }

// How many tiles (of its own group) ahead an epilogue group issues the side
// loads (scale, V, D).  The wait for the tile-info of tile i + dist*T
// (T = tiles in the epilogue at once) must not need this group's hand-back of
// tile i: the MMAs run up to tile i + nacc - 1 without it, and the producer
// writes the info of tile k once the MMAs of tile k - stages are done and, at
// a request change, once the MMA issuer has reached the first tile of the
// request nq requests back (one tile before k at the least).  So
// dist*T < nq + nacc and dist*T < stages + nacc; the largest of 2, 1, 0 that
// satisfies both.  It is a template parameter of the kernel, so that the side
// data of the tiles ahead stay in fixed registers.
__host__ __device__ constexpr int prefetch_dist(int tiles_at_once, int nq, int nacc, int stages) {
  return (2 * tiles_at_once < nq + nacc && 2 * tiles_at_once < stages + nacc)   ? 2
         : (1 * tiles_at_once < nq + nacc && 1 * tiles_at_once < stages + nacc) ? 1
                                                                                 : 0;
}

struct Bars {
  uint32_t full, empty, afull, aempty, qfull, qempty, accempty, done;
  __device__ uint32_t f(int s) const { return full + 8 * s; }
  __device__ uint32_t e(int s) const { return empty + 8 * s; }
  __device__ uint32_t xf(int s) const { return afull + 8 * s; }
  __device__ uint32_t xe(int s) const { return aempty + 8 * s; }
  __device__ uint32_t qf(int i) const { return qfull + 8 * i; }
  __device__ uint32_t qe(int i) const { return qempty + 8 * i; }
  __device__ uint32_t ae(int i) const { return accempty + 8 * i; }
};


// Tile metadata, gathered by one producer lane per tile in two phases one
// batch apart, so no load result is needed before a batch later:
//   phase A: request, pair index, context length, kept count, block ids
//   phase B: page ids from the block table (needs the block ids)
struct TileMeta {
  int q, t, ctx, kept, j0, j1, pg0, pg1;
};

__device__ __forceinline__ void meta_phase_a(TileMeta& m, const ScoreArgs& a, const Sched& sched, const int* prefix,
                                             int g, int g1) {
  m.q = -1;
  if (g >= g1) return;
  const Layout& L = a.lay;
  const int q = sched.locate(g);
  const int t = g - prefix[q];
  m.q = q;
  m.t = t;
  m.ctx = a.ctx_len[q];
  m.kept = a.kept[q];
  const int32_t* work = a.work + (int64_t)q * L.blk_stride;
  m.j0 = work[2 * t];
  m.j1 = (2 * t + 1 < L.blk_stride) ? work[2 * t + 1] : -1;
}

__device__ __forceinline__ void meta_phase_b(TileMeta& m, const ScoreArgs& a) {
  if (m.q < 0) return;
  const int32_t* bt = a.block_table + (int64_t)m.q * a.bt_stride;
  m.pg0 = bt[m.j0];
  m.pg1 = (2 * m.t + 1 < m.kept) ? bt[m.j1] : 0;
}

__device__ __forceinline__ TileMeta shfl_meta(const TileMeta& m, int src) {
  TileMeta r;
  r.q = __shfl_sync(0xffffffffu, m.q, src);
  r.t = __shfl_sync(0xffffffffu, m.t, src);
  r.ctx = __shfl_sync(0xffffffffu, m.ctx, src);
  r.kept = __shfl_sync(0xffffffffu, m.kept, src);
  r.j0 = __shfl_sync(0xffffffffu, m.j0, src);
  r.j1 = __shfl_sync(0xffffffffu, m.j1, src);
  r.pg0 = __shfl_sync(0xffffffffu, m.pg0, src);
  r.pg1 = __shfl_sync(0xffffffffu, m.pg1, src);
  return r;
}

// KH: the head count when it is fixed at compile time (64, the DSA indexer's),
// so that the epilogue's column loops unroll; 0 reads it from the layout.
// DIST: the side-load prefetch distance, prefetch_dist() of the plan.
// RC: the number of query rows when fixed at compile time (0: a.rows), so
// that the epilogue's row loop and its per-row conditions fold.  FU: the
// fused EMA update known at compile time (1 on, 0 off, -1: a.V decides).
template <int G, int KH, int DIST, int RC = 0, int FU = -1>
__global__ void __launch_bounds__(threads_for(G), G == 2 ? 2 : 1)
    k_score_tc(ScoreArgs a, TcPlan plan, const __grid_constant__ CUtensorMap tmap_k,
               const __grid_constant__ CUtensorMap tmap_q) {
  pdl_enter();
  constexpr int kThreads = threads_for(G);
  constexpr int kEpiGroups = G;
  const Layout L = a.lay;
  const int H = KH ? KH : L.H;
  const int rows = RC ? RC : a.rows;
  const int N = rows * H;
  // the four-group plan is always 8 stages, 2 accumulators, 2 query buffers
  const int stages = G == 4 ? kMaxStages : plan.stages, nacc = G == 4 ? 2 : plan.nacc;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const SmemLayout lay = smem_layout(N, L.Q, stages, plan.nq, G);
  const int nq = G == 4 ? 2 : plan.nq;
  const uint32_t sbase = smem_u32(smem);
  TileInfo* aux = reinterpret_cast<TileInfo*>(smem + lay.aux);
  int* prefix = reinterpret_cast<int*>(smem + lay.prefix);
  float* wqs = reinterpret_cast<float*>(smem + lay.wq);
  uint64_t* bar_mem = reinterpret_cast<uint64_t*>(smem + lay.bars);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar_mem + 2 * kMaxStages + 2 * kAuxSlots + 4 + 2 * kMaxAcc + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  Bars B;
  B.full = smem_u32(bar_mem);
  B.empty = B.full + 8 * kMaxStages;
  B.afull = B.empty + 8 * kMaxStages;
  B.aempty = B.afull + 8 * kAuxSlots;
  B.qfull = B.aempty + 8 * kAuxSlots;
  B.qempty = B.qfull + 16;
  B.accempty = B.qempty + 16;
  B.done = B.accempty + 8 * kMaxAcc;
  const Ctl ctl{abort_flag, a.err};
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const bool fused = FU >= 0 ? FU == 1 : a.V != nullptr;
  // With four groups and several rows, two groups share a tile, each taking
  // every other row: the accumulator (two fit TMEM at N > 128) is read in half
  // the time, so the MMA waits half as long for it.
  const int share = groups_per_tile(kEpiGroups, rows);  // groups per tile

  // ---- tile prefix over requests (all threads: one load pair each, block
  // scan), barriers ------------------------------------------------------
  {
    int* scan_tmp = reinterpret_cast<int*>(wqs);  // 33 ints; the epilogue fills wqs later
    int carry = 0;
    for (int base = 0; base < L.Q; base += kThreads) {
      const int q = base + (int)threadIdx.x;
      int v = 0;
      if (q < L.Q) {
        const int64_t ctx = a.ctx_len[q];
        bool ok = ctx >= 1 && ctx + rows - 1 <= L.max_slots;
        if (ok && a.ctx_sel && a.ctx_sel[q] != ctx) {  // the prepared selection is for another ctx_len
          ok = false;
          if (blockIdx.x == 0) raise_error(a.err, ERR_LOOKAHEAD, q, (uint32_t)ctx);
        }
        if (a.ctx_next && blockIdx.x == 0) a.ctx_next[q] = (int32_t)(ctx + 1);
        v = ok ? (a.kept[q] + 1) / 2 : 0;
      }
      int tot;
      const int ex = block_exclusive_scan(v, scan_tmp, &tot);
      if (q < L.Q) prefix[q] = carry + ex;
      carry += tot;
    }
    if (threadIdx.x == 0) prefix[L.Q] = carry;
  }
  if (threadIdx.x == 0) {
    *abort_flag = 0;
    for (int s = 0; s < stages; ++s) {
      mbar_init(B.f(s), 1);
      mbar_init(B.e(s), 1);  // the MMA commit: keys are free once the MMAs read them
    }
    for (int s = 0; s < kAuxSlots; ++s) {
      mbar_init(B.xf(s), 1);  // the producer's arrive after writing the tile info
      mbar_init(B.xe(s), 4 * share);  // the epilogue warps of the groups that own the tile
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(B.qf(i), 1);
      mbar_init(B.qe(i), 1);
    }
    for (int i = 0; i < nacc; ++i) mbar_init(B.ae(i), 4 * share);  // the warps of the groups that own the tile
    mbar_init(B.done, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  const int acc_cols = nacc * N;
  const uint32_t ncols = acc_cols <= 32 ? 32 : acc_cols <= 64 ? 64 : acc_cols <= 128 ? 128 : acc_cols <= 256 ? 256 : 512;
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                 "r"(ncols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  const int total = prefix[L.Q];
  const int g0 = (int)(((int64_t)total * blockIdx.x) / gridDim.x);
  const int g1 = (int)(((int64_t)total * (blockIdx.x + 1)) / gridDim.x);
  const Sched sched{prefix, L.Q};

  if (warp == 0) {
    // ======================= producer (whole warp) =======================
    int stage = 0;
    uint32_t phase = 0;
    int cur_q = -1, qiter = 0;
    int xslot = 0;
    uint32_t xphase = 0;
    int inflight[kMaxStages];
    for (int i = 0; i < kMaxStages; ++i) inflight[i] = -1;
    bool withhold = a.inject && blockIdx.x == 0;
    bool stop = false;
    TileMeta cur, nxt, nxt2;
    meta_phase_a(cur, a, sched, prefix, g0 + lane, g1);
    meta_phase_b(cur, a);
    meta_phase_a(nxt, a, sched, prefix, g0 + 32 + lane, g1);
    for (int gb = g0; gb < g1 && !stop; gb += 32) {
      meta_phase_b(nxt, a);                                        // block ids arrived a batch ago
      meta_phase_a(nxt2, a, sched, prefix, gb + 64 + lane, g1);    // used two batches later
      const int nb_tiles = min(32, g1 - gb);
      for (int i = 0; i < nb_tiles; ++i) {
        const TileMeta m = shfl_meta(cur, i);
        const int np = (2 * m.t + 1 < m.kept) ? 2 : 1;
        const int pg0 = (m.pg0 >= 0 && m.pg0 < a.num_pages) ? m.pg0 : -1;
        const int pg1 = (np == 2 && m.pg1 >= 0 && m.pg1 < a.num_pages) ? m.pg1 : -1;
        int ok = 1;
        if (lane == 0) {
          if (m.q != cur_q) {
            const int nb = qiter % nq;
            ok = wait_parity(B.qe(nb), ((qiter / nq) & 1) ^ 1, ctl);
            if (ok) {
              mbar_expect_tx(B.qf(nb), (uint32_t)(N * kRowBytes));
              tma_load_2d(sbase + lay.qbuf + nb * N * kRowBytes, &tmap_q, B.qf(nb), 0, m.q * N);
            }
          }
          if (ok) ok = wait_parity(B.e(stage), phase ^ 1, ctl);
          if (ok) ok = wait_parity(B.xe(xslot), xphase ^ 1, ctl);
          if (ok) {
            if (pg0 < 0) raise_error(a.err, ERR_PAGE, m.q, (uint32_t)m.pg0);
            if (np == 2 && pg1 < 0) raise_error(a.err, ERR_PAGE, m.q, (uint32_t)m.pg1);
            TileInfo* x = aux + xslot;
            x->q = m.q;
            x->ctx = m.ctx;
            x->np = np;
            x->t = m.t;
            x->j[0] = m.j0;
            x->j[1] = m.j1;
            x->pg[0] = pg0;
            x->pg[1] = pg1;
            mbar_arrive(B.xf(xslot));  // release: the epilogue's wait sees the info
            if (!withhold) {
              mbar_expect_tx(B.f(stage), (uint32_t)(np * kPageBytes));
              inflight[stage] = (int)phase;
            }
          }
        }
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) { stop = true; break; }
        if (m.q != cur_q) { cur_q = m.q; ++qiter; }
        const bool issue = !__shfl_sync(0xffffffffu, withhold ? 1 : 0, 0);
        withhold = false;  // test hook: at most the first stage is withheld
        if (issue && lane < np) {
          const int pg = lane ? (pg1 < 0 ? 0 : pg1) : (pg0 < 0 ? 0 : pg0);  // bad pages load page 0; skipped later
          tma_load_2d(sbase + lay.keys + stage * kStageBytes + lane * kPageBytes, &tmap_k, B.f(stage), 0, pg * kPage);
        }
        if (++stage == stages) { stage = 0; phase ^= 1; }
        if (++xslot == kAuxSlots) { xslot = 0; xphase ^= 1; }
      }
      cur = nxt;
      nxt = nxt2;
    }
    // On abort, wait (bounded) until every copy this warp issued has landed.
    if (lane == 0 && *abort_flag) {
      for (int s = 0; s < stages; ++s) {
        if (inflight[s] < 0) continue;
        const uint64_t t0 = gtimer();
        while (!mbar_try_wait(B.f(s), (uint32_t)inflight[s]) && gtimer() - t0 < kTimeoutNs) {}
      }
    }
  } else if (warp == 1) {
    // ======================= MMA issuer =======================
    if (lane == 0 && g0 < g1) {
      // The loop is the serial path of the CTA: counters advance without
      // divisions, the request is re-resolved only at its last tile, and one
      // commit per tile signals both the producer (stage free) and the
      // epilogue (accumulator full).
      const uint32_t idesc = idesc_e4m3(kTileM, N);
      int q = sched.locate(g0);
      int q_end = prefix[q + 1];  // first global tile of the next request
      int qiter = 0, qbuf = 0;
      uint32_t qphase = 0;
      int stage = 0, acc = 0;
      uint32_t phase = 0, acc_phase = 0;
      bool ok = wait_parity(B.qf(0), 0, ctl);
      for (int g = g0; ok && g < g1; ++g) {
        if (g >= q_end) {
          do { ++q; } while (prefix[q + 1] <= g);
          q_end = prefix[q + 1];
          umma_commit(B.qe(qbuf));  // the previous query tile is free once its MMAs complete
          ++qiter;
          qbuf = qiter % nq;
          qphase = (uint32_t)(qiter / nq) & 1u;
          if (!wait_parity(B.qf(qbuf), qphase, ctl)) break;
        }
        if (!wait_parity(B.ae(acc), acc_phase ^ 1, ctl)) break;
        if (!wait_parity(B.f(stage), phase, ctl)) break;
        tc_fence_after();
        const uint64_t a_desc = sw128_desc(sbase + lay.keys + stage * kStageBytes);
        const uint64_t b_desc = sw128_desc(sbase + lay.qbuf + qbuf * N * kRowBytes);
        const uint32_t d_tmem = tmem_base + (uint32_t)(acc * N);
        // K = 128 bytes as four K = 32 steps; a 32-byte step inside the
        // swizzled atom advances the descriptor's start address by 2 (16-byte units)
#pragma unroll
        for (int kk = 0; kk < kRowBytes / 32; ++kk)
          umma_e4m3(d_tmem, a_desc + 2 * kk, b_desc + 2 * kk, idesc, kk > 0 ? 1u : 0u);
        umma_commit(B.e(stage));
        if (++stage == stages) { stage = 0; phase ^= 1u; }
        if (++acc == nacc) { acc = 0; acc_phase ^= 1u; }
      }
      // all MMAs issued by this thread complete before TMEM is released
      umma_commit(B.done);
      const uint64_t t0 = gtimer();
      while (!mbar_try_wait(B.done, 0) && gtimer() - t0 < kTimeoutNs) {}
    }
  } else {
    // ======================= epilogue (warps 2..9) =======================
    const int ew = warp - 2;              // 0 .. 4*kEpiGroups-1
    const int tgroups = kEpiGroups / share;  // tiles in the epilogue at once
    const int group = ew / (4 * share);      // tile group: tiles group, group + tgroups, ...
    const int sub = (ew >> 2) % share;       // rows sub, sub + share, ... of the tile
    const int quarter = warp & 3;         // TMEM lanes this warp may access
    const int m = quarter * 32 + lane;    // accumulator row = tile token
    const int pg_idx = m >> 6, tok = m & 63;
    int cur_q = -1;
    float* wcur = wqs + ew * N;           // this warp's copy of the head weights
    const int n_local = g1 - g0;
    // Per-token operands of a tile.  The tile's metadata comes from the
    // tile-info ring when the tile is processed (the slot is held until the
    // hand-back); the three global loads (scale, V, D) are issued DIST tiles
    // of this group ahead (T = tile groups apart), because under full load a
    // global load takes longer than one tile of the epilogue.  DIST follows
    // the rule of prefetch_dist(), which the host checked for this plan.
    struct Pre {
      int q, s, pres, valid, upd, t;
      int p0;  // ctx_len - 1 < 2^31 (max_slots is an int32)
      float sigma, v, d;
      int kq;  // four rows: the request's kept blocks (whether the top-k can use the group maxima)
    };
    struct SideData {
      float sigma, v, d;
    };
    // With four groups (one CTA per SM, several rows) a tile's metadata is
    // carried from its side loads to its processing, so the tile-info slot is
    // read once; with two groups the registers are scarcer (two CTAs per SM,
    // two tiles of prefetch) and it is read again.
    constexpr bool kCarry = G == 4;
    using Side = std::conditional_t<kCarry, Pre, SideData>;
    auto info_ready = [&](int i) -> bool {
      return __all_sync(0xffffffffu, wait_parity(B.xf(i & (kAuxSlots - 1)), (uint32_t)(i / kAuxSlots) & 1u, ctl));
    };
    auto meta_of = [&](int i, int& pg) -> Pre {  // after info_ready(i)
      const TileInfo* x = aux + (i & (kAuxSlots - 1));
      Pre r;
      r.q = x->q;
      r.t = x->t;
      r.p0 = x->ctx - 1;
      pg = x->pg[pg_idx];
      const bool present = pg_idx < x->np && pg >= 0;
      r.s = present ? x->j[pg_idx] * kPage + tok : 0;
      r.pres = present;
      r.valid = present && r.s <= r.p0 + (rows - 1);
      r.upd = fused && r.valid && r.s <= r.p0;
      return r;
    };
    auto load_side = [&](int i) -> Side {
      int pg;
      const Pre m = meta_of(i, pg);
      Side r;
      if constexpr (kCarry) {
        r = m;
        // safe addresses instead of predicates, so that nothing waits for
        // the loads before the tile that uses them: a value that is not
        // needed (the scale of an invalid slot, V or D of a slot that is not
        // updated) is read from a valid place and never used
        r.sigma = __ldg(a.kscale + (int64_t)(m.valid ? pg : 0) * kPage + tok);
        r.v = fused ? a.V[(int64_t)m.q * L.slot_stride + m.s] : 0.f;
        r.d = fused ? a.D[(int64_t)m.q * L.slot_stride + (m.upd ? m.p0 - m.s : 0)] : 0.f;
        if constexpr (RC == 4) r.kq = __ldg(a.kept + m.q);
      } else {
        r.sigma = m.valid ? __ldg(a.kscale + (int64_t)pg * kPage + tok) : 0.f;
        // V of the page's slots past the context too, for its group maxima
        r.v = (m.upd || (fused && a.vmax && m.pres)) ? a.V[(int64_t)m.q * L.slot_stride + m.s] : 0.f;
        r.d = m.upd ? a.D[(int64_t)m.q * L.slot_stride + (m.p0 - m.s)] : 0.f;
      }
      return r;
    };
    Side nx1{}, nx2{};  // side data of tiles i and i + T
    bool alive_ = group < n_local;
    if constexpr (DIST >= 1) {
      if (alive_) {
        alive_ = info_ready(group);
        if (alive_) nx1 = load_side(group);
      }
    }
    if constexpr (DIST == 2) {
      if (alive_ && group + tgroups < n_local) {
        alive_ = info_ready(group + tgroups);
        if (alive_) nx2 = load_side(group + tgroups);
      }
    }
    // ring positions of tile i, advanced by T per tile without divisions
    int acc = group % nacc, stage = group % stages;
    uint32_t phase = (uint32_t)(group / stages) & 1u;
    for (int i = group; alive_ && i < n_local; i += tgroups) {
      Side side;
      if constexpr (DIST == 0) {
        if (!info_ready(i)) break;
        side = load_side(i);
      } else if constexpr (DIST == 1) {
        side = nx1;
        if (i + tgroups < n_local) {
          if (!info_ready(i + tgroups)) break;
          nx1 = load_side(i + tgroups);
        }
      } else {
        side = nx1;
        nx1 = nx2;
        if (i + 2 * tgroups < n_local) {
          if (!info_ready(i + 2 * tgroups)) break;
          nx2 = load_side(i + 2 * tgroups);
        }
      }
      Pre cur;
      if constexpr (kCarry) {
        cur = side;
      } else {
        int pg_unused;
        cur = meta_of(i, pg_unused);
        cur.sigma = side.sigma;
        cur.v = side.v;
        cur.d = side.d;
      }
      const int xs = i & (kAuxSlots - 1);
      if (cur.q != cur_q) {
        __syncwarp();
        for (int k = lane; k < N; k += 32) wcur[k] = a.wq[(int64_t)cur.q * N + k];
        __syncwarp();
        cur_q = cur.q;
      }
      // The MMA's commit on the key stage also marks the accumulator full.
      // Every lane waits; the warp leaves together if any lane gave up, so
      // the .sync.aligned TMEM loads below never run on a partial warp.
      if (!__all_sync(0xffffffffu, wait_parity(B.e(stage), phase, ctl))) break;
      tc_fence_after();
      const uint32_t trow = tmem_base + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(acc * N);
      // this warp's rows sub, sub + share, ...; with the row count fixed at
      // compile time the loop unrolls, and one row's reduction and stores
      // overlap the next row's accumulator loads
      constexpr int kRowsPerWarp = RC ? (RC + groups_per_tile(G, RC) - 1) / groups_per_tile(G, RC) : 0;
      const int nrw = kRowsPerWarp ? kRowsPerWarp : (rows - sub + share - 1) / share;
#pragma unroll
      for (int k = 0; k < nrw; ++k) {
        const int r = sub + k * share;
        if (kRowsPerWarp && r >= rows) break;
        float part[4] = {0.f, 0.f, 0.f, 0.f};
        for (int c = 0; c < H; c += 32) {
          uint32_t v[32];
          if (c + 32 <= H)  // 32 columns in one load
            tmem_ld32(trow + (uint32_t)(r * H + c), v);
          else
            tmem_ld16(trow + (uint32_t)(r * H + c), *reinterpret_cast<uint32_t(*)[16]>(&v[0]));
          tmem_wait_ld();
          if (r + share >= rows && c + 32 >= H) {
            // last accumulator columns are in registers: hand the accumulator
            // (and the tile-info slot, read a tile ago) back before the math
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
              mbar_arrive(B.ae(acc));
              mbar_arrive(B.xe(xs));
            }
          }
          const float4* wr = reinterpret_cast<const float4*>(wcur + r * H + c);
          const int nu = min(32, H - c);  // 16 or 32: H is a multiple of 16
#pragma unroll
          for (int u = 0; u < 32; u += 4) {
            if (u < nu) {
              const float4 w4 = wr[u >> 2];
              fma2_rn(part[0], part[1], w4.x, w4.y, fmaxf(__uint_as_float(v[u + 0]), 0.0f),
                      fmaxf(__uint_as_float(v[u + 1]), 0.0f));
              fma2_rn(part[2], part[3], w4.z, w4.w, fmaxf(__uint_as_float(v[u + 2]), 0.0f),
                      fmaxf(__uint_as_float(v[u + 3]), 0.0f));
            }
          }
        }
        const float sum = (part[0] + part[1]) + (part[2] + part[3]);
        const bool scored = cur.valid && cur.s <= cur.p0 + r;
        // (four MTP rows of a request whose kept blocks are too few for the
        // top-k's group path skip the maxima: nothing would read them)
        if (a.gmax && (RC != 4 || topk_group_path_possible(cur.kq, L.b, L.k))) {
          // max over this warp's 32 slots = group 4t + quarter of the kept-slot order
          const float g = warp_max(scored ? sum * cur.sigma : __int_as_float(0xff800000));
          if (lane == 0) a.gmax[((int64_t)cur.q * L.R + r) * a.gstride + 4 * cur.t + quarter] = g;
        }
        float vnew = cur.v;
        if (scored) {
          const float score = sum * cur.sigma;
          a.scores[((int64_t)cur.q * L.R + r) * L.slot_stride + cur.s] = score;
          if (cur.upd && r == 0) {
            vnew = ema_v(cur.v, score, a.alpha, a.beta);
            a.V[(int64_t)cur.q * L.slot_stride + cur.s] = vnew;
            a.D[(int64_t)cur.q * L.slot_stride + (cur.p0 - cur.s)] = ema_d(cur.d, score, a.alpha, a.beta);
          }
        }
        if (fused && a.vmax && r == 0 && cur.pres) {
          // this warp's 32 slots are one aligned group of V (present is warp-uniform)
          const float g = warp_max(vnew);
          if (lane == 0) a.vmax[(int64_t)cur.q * L.vg_stride + (cur.s >> 5)] = g;
        }
      }
      acc += tgroups;
      while (acc >= nacc) acc -= nacc;
      stage += tgroups;
      while (stage >= stages) {
        stage -= stages;
        phase ^= 1u;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(ncols) : "memory");
  }
}

bool encode_2d(EncodeTiledFn fn, CUtensorMap* map, const void* base, uint64_t rows, uint32_t box_rows) {
  const cuuint64_t dims[2] = {(cuuint64_t)kRowBytes, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)kRowBytes};
  const cuuint32_t box[2] = {(cuuint32_t)kRowBytes, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

}  // namespace

bool tc_supported(const Layout& lay, int rows, int key_fp8) {
  const int N = rows * lay.H;
  if (!(key_fp8 && lay.d == 128 && lay.b == kPage && lay.H % 16 == 0 && N >= 16 && N <= 256 && N % 16 == 0))
    return false;
  const TcPlan plan = tc_plan(N, lay.Q);
  return smem_layout(N, lay.Q, plan.stages, plan.nq, plan.groups).total <= 227 * 1024;
}

cudaError_t launch_score_tc(const ScoreArgs& a, void* encode_fn, cudaStream_t s) {
  const Layout& L = a.lay;
  const int N = a.rows * L.H;
  if (!tc_supported(L, a.rows, a.key_fp8) || !encode_fn) return cudaErrorInvalidValue;
  if (((uintptr_t)a.keys & 15) || ((uintptr_t)a.q8 & 15)) return cudaErrorInvalidValue;
  CUtensorMap tk, tq;
  EncodeTiledFn fn = reinterpret_cast<EncodeTiledFn>(encode_fn);
  if (!encode_2d(fn, &tk, a.keys, (uint64_t)a.num_pages * kPage, kPage)) return cudaErrorInvalidValue;
  if (!encode_2d(fn, &tq, a.q8, (uint64_t)L.Q * N, (uint32_t)N)) return cudaErrorInvalidValue;
  const TcPlan plan = tc_plan(N, L.Q);
  if (plan.groups == 4 && (plan.stages != kMaxStages || plan.nacc != 2 || plan.nq != 2))
    return cudaErrorInvalidValue;  // the four-group kernels take this plan as constants
  const uint32_t smem = smem_layout(N, L.Q, plan.stages, plan.nq, plan.groups).total;
  const int dist = prefetch_dist(plan.groups / groups_per_tile(plan.groups, a.rows), plan.nq, plan.nacc,
                                 plan.stages);
  // the instances the plans reach: two groups with 4 accumulators (N <= 64)
  // or 2 (N <= 128); four groups sharing tiles (several rows) or not (one row)
  void (*kernel)(ScoreArgs, TcPlan, const CUtensorMap, const CUtensorMap) = nullptr;
  if (plan.groups == 2 && dist == 2)
    kernel = L.H != 64 ? k_score_tc<2, 0, 2>
             : a.rows != 1 ? k_score_tc<2, 64, 2>
             : a.V        ? k_score_tc<2, 64, 2, 1, 1>
                          : k_score_tc<2, 64, 2, 1, 0>;
  if (plan.groups == 2 && dist == 1) kernel = L.H == 64 ? k_score_tc<2, 64, 1> : k_score_tc<2, 0, 1>;
  if (plan.groups == 4 && dist == 1)
    // (the EMA is fused for one row only, so four rows come without V)
    kernel = L.H != 64 ? k_score_tc<4, 0, 1> : (a.rows == 4 && !a.V) ? k_score_tc<4, 64, 1, 4, 0> : k_score_tc<4, 64, 1>;
  if (plan.groups == 4 && dist == 0) kernel = k_score_tc<4, 0, 0>;
  if (!kernel) return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  PdlLaunch l(dim3(sms * plan.ctas), dim3(threads_for(plan.groups)), smem, s);
  return cudaLaunchKernelEx(&l.cfg, kernel, a, plan, tk, tq);
}

}  // namespace spin
