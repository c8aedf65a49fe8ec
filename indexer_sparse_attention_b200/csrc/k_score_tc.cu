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
// Warp roles (192 threads, persistent, one CTA per SM):
//   warp 0      TMA producer: query tile per request, key pages per tile
//   warp 1      TMEM allocation; lane 0 issues the MMAs and the commits
//   warps 2..5  epilogue: tcgen05.ld of the accumulator quarter this warp may
//               access (lanes 32*(warp%4) ..), ReLU, head weights, scale,
//               store, fused EMA
// Pipelines: kStages key stages (full/empty), 2 query buffers, 2 TMEM
// accumulators.  Every wait is bounded (2 s of %globaltimer); on expiry the
// CTA raises ERR_TIMEOUT, stops issuing, drains what it issued and frees TMEM.
#include <cuda.h>

#include <algorithm>

#include "spin_internal.cuh"

namespace spin {
namespace {

constexpr int kStages = 6;
constexpr int kTileM = 128;
constexpr int kPage = 64;          // tokens per page (block size)
constexpr int kRowBytes = 128;     // d = 128 FP8 values
constexpr int kPageBytes = kPage * kRowBytes;
constexpr int kStageBytes = kTileM * kRowBytes;
constexpr int kThreads = 192;
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
// the CTA abort flag) or when another role already aborted.
__device__ __noinline__ bool wait_parity(uint32_t bar, uint32_t parity, Ctl c) {
  if (mbar_try_wait(bar, parity)) return true;
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

struct SmemLayout {
  uint32_t keys;     // kStages * kStageBytes
  uint32_t qbuf;     // 2 * N * 128
  uint32_t wq;       // 4 * N floats: one copy per epilogue warp
  uint32_t prefix;   // (Q + 1) ints
  uint32_t bars;     // barriers
  uint32_t total;
};

__host__ __device__ inline SmemLayout smem_layout(int N, int Q) {
  SmemLayout s;
  uint32_t off = 0;
  s.keys = off;
  off += kStages * kStageBytes;
  s.qbuf = off;
  off += 2 * N * kRowBytes;
  s.wq = off;
  off += 4 * N * 4;
  s.prefix = off;
  off += ((Q + 1) * 4 + 15) / 16 * 16;
  s.bars = off;
  off += (2 * kStages + 8) * 8 + 16;
  s.total = off + 1024;  // slack for 1024-byte alignment of the base
  return s;
}

struct Bars {
  uint32_t full, empty, qfull, qempty, accfull, accempty, done;
  __device__ uint32_t f(int s) const { return full + 8 * s; }
  __device__ uint32_t e(int s) const { return empty + 8 * s; }
  __device__ uint32_t qf(int i) const { return qfull + 8 * i; }
  __device__ uint32_t qe(int i) const { return qempty + 8 * i; }
  __device__ uint32_t af(int i) const { return accfull + 8 * i; }
  __device__ uint32_t ae(int i) const { return accempty + 8 * i; }
};

__global__ void __launch_bounds__(kThreads, 1)
    k_score_tc(ScoreArgs a, const __grid_constant__ CUtensorMap tmap_k, const __grid_constant__ CUtensorMap tmap_q) {
  const Layout L = a.lay;
  const int N = a.rows * L.H;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const SmemLayout lay = smem_layout(N, L.Q);
  const uint32_t sbase = smem_u32(smem);
  int* prefix = reinterpret_cast<int*>(smem + lay.prefix);
  float* wqs = reinterpret_cast<float*>(smem + lay.wq);
  uint64_t* bar_mem = reinterpret_cast<uint64_t*>(smem + lay.bars);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar_mem + 2 * kStages + 7);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  Bars B;
  B.full = smem_u32(bar_mem);
  B.empty = B.full + 8 * kStages;
  B.qfull = B.empty + 8 * kStages;
  B.qempty = B.qfull + 16;
  B.accfull = B.qempty + 16;
  B.accempty = B.accfull + 16;
  B.done = B.accempty + 16;
  const Ctl ctl{abort_flag, a.err};
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // ---- tile prefix over requests ------------------------------------------
  if (threadIdx.x == 0) {
    int acc = 0;
    for (int q = 0; q < L.Q; ++q) {
      prefix[q] = acc;
      const int64_t ctx = a.ctx_len[q];
      const bool ok = ctx >= 1 && ctx + a.rows - 1 <= L.max_slots;
      acc += ok ? (a.kept[q] + 1) / 2 : 0;
    }
    prefix[L.Q] = acc;
    *abort_flag = 0;
    for (int s = 0; s < kStages; ++s) {
      mbar_init(B.f(s), 1);
      mbar_init(B.e(s), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(B.qf(i), 1);
      mbar_init(B.qe(i), 1);
      mbar_init(B.af(i), 1);
      mbar_init(B.ae(i), 4);
    }
    mbar_init(B.done, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  const uint32_t ncols = (2 * N <= 32) ? 32 : (2 * N <= 64) ? 64 : (2 * N <= 128) ? 128 : (2 * N <= 256) ? 256 : 512;
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
    // ======================= TMA producer =======================
    if (lane == 0 && g0 < g1) {
      int q = sched.locate(g0), t = g0 - prefix[q];
      int stage = 0;
      uint32_t phase = 0;
      int cur_q = -1, qiter = 0;
      int inflight[kStages];  // parity of the last load issued into each stage, -1: none
      for (int i = 0; i < kStages; ++i) inflight[i] = -1;
      bool withhold = a.inject && blockIdx.x == 0;
      for (int g = g0; g < g1; ++g, ++t) {
        while (t >= prefix[q + 1] - prefix[q]) { ++q; t = 0; }
        if (q != cur_q) {
          const int nb = qiter & 1;
          if (!wait_parity(B.qe(nb), ((qiter >> 1) & 1) ^ 1, ctl)) break;
          mbar_expect_tx(B.qf(nb), (uint32_t)(N * kRowBytes));
          tma_load_2d(sbase + lay.qbuf + nb * N * kRowBytes, &tmap_q, B.qf(nb), 0, q * N);
          cur_q = q;
          ++qiter;
        }
        if (!wait_parity(B.e(stage), phase ^ 1, ctl)) break;
        const int32_t* work = a.work + (int64_t)q * L.blk_stride;
        const int nk = a.kept[q];
        const int i0 = 2 * t, i1 = 2 * t + 1;
        int pages[2];
        int np = (i1 < nk) ? 2 : 1;
        for (int i = 0; i < np; ++i) {
          const int j = work[i0 + i];
          int pg = a.block_table[(int64_t)q * a.bt_stride + j];
          if (pg < 0 || pg >= a.num_pages) {
            raise_error(a.err, ERR_PAGE, q, (uint32_t)pg);
            pg = 0;  // keep the pipeline in step; the epilogue skips this page
          }
          pages[i] = pg;
        }
        if (withhold) {
          withhold = false;  // test hook: this stage never fills
        } else {
          mbar_expect_tx(B.f(stage), (uint32_t)(np * kPageBytes));
          for (int i = 0; i < np; ++i)
            tma_load_2d(sbase + lay.keys + stage * kStageBytes + i * kPageBytes, &tmap_k, B.f(stage), 0,
                        pages[i] * kPage);
          inflight[stage] = (int)phase;
        }
        if (++stage == kStages) { stage = 0; phase ^= 1; }
      }
      // On abort, wait (bounded) until every copy this thread issued has landed.
      if (*abort_flag) {
        for (int s = 0; s < kStages; ++s) {
          if (inflight[s] < 0) continue;
          const uint64_t t0 = gtimer();
          while (!mbar_try_wait(B.f(s), (uint32_t)inflight[s]) && gtimer() - t0 < kTimeoutNs) {}
        }
      }
    }
  } else if (warp == 1) {
    // ======================= MMA issuer =======================
    if (lane == 0 && g0 < g1) {
      const uint32_t idesc = idesc_e4m3(kTileM, N);
      int q = sched.locate(g0), t = g0 - prefix[q];
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      int cur_q = -1, qiter = 0;
      for (int g = g0; g < g1; ++g, ++t) {
        while (t >= prefix[q + 1] - prefix[q]) { ++q; t = 0; }
        if (q != cur_q) {
          if (cur_q >= 0) umma_commit(B.qe((qiter - 1) & 1));
          const int nb = qiter & 1;
          if (!wait_parity(B.qf(nb), (qiter >> 1) & 1, ctl)) break;
          cur_q = q;
          ++qiter;
        }
        if (!wait_parity(B.ae(acc), acc_phase ^ 1, ctl)) break;
        if (!wait_parity(B.f(stage), phase, ctl)) break;
        tc_fence_after();
        const uint32_t a_addr = sbase + lay.keys + stage * kStageBytes;
        const uint32_t b_addr = sbase + lay.qbuf + ((qiter - 1) & 1) * N * kRowBytes;
        const uint32_t d_tmem = tmem_base + (uint32_t)(acc * N);
#pragma unroll
        for (int kk = 0; kk < kRowBytes / 32; ++kk)
          umma_e4m3(d_tmem, sw128_desc(a_addr + kk * 32), sw128_desc(b_addr + kk * 32), idesc, kk > 0 ? 1u : 0u);
        umma_commit(B.e(stage));
        umma_commit(B.af(acc));
        if (++stage == kStages) { stage = 0; phase ^= 1; }
        if (++acc == 2) { acc = 0; acc_phase ^= 1; }
      }
      // all MMAs issued by this thread complete before TMEM is released
      umma_commit(B.done);
      const uint64_t t0 = gtimer();
      while (!mbar_try_wait(B.done, 0) && gtimer() - t0 < kTimeoutNs) {}
    }
  } else {
    // ======================= epilogue (warps 2..5) =======================
    const int quarter = warp & 3;
    const int m = quarter * 32 + lane;  // accumulator row = tile token
    const int pg_idx = m >> 6, tok = m & 63;
    if (g0 < g1) {
      int q = sched.locate(g0), t = g0 - prefix[q];
      int acc = 0;
      uint32_t acc_phase = 0;
      int cur_q = -1;
      int64_t ctx = 0;
      float* wcur = wqs + (warp - 2) * N;  // this warp's copy of the head weights
      for (int g = g0; g < g1; ++g, ++t) {
        while (t >= prefix[q + 1] - prefix[q]) { ++q; t = 0; }
        if (q != cur_q) {
          __syncwarp();
          for (int i = lane; i < N; i += 32) wcur[i] = a.wq[(int64_t)q * N + i];
          __syncwarp();
          cur_q = q;
          ctx = a.ctx_len[q];
        }
        // slot, page and per-slot operands (independent of the MMA: issue first)
        const int32_t* work = a.work + (int64_t)q * L.blk_stride;
        const int nk = a.kept[q];
        const int li = 2 * t + pg_idx;
        bool valid = li < nk;
        int64_t s = 0;
        int page = 0;
        float sigma = 0.f, v_old = 0.f, d_old = 0.f;
        if (valid) {
          const int j = work[li];
          page = a.block_table[(int64_t)q * a.bt_stride + j];
          valid = page >= 0 && page < a.num_pages;
          s = (int64_t)j * kPage + tok;
          valid = valid && s <= ctx - 1 + (a.rows - 1);
          if (valid) {
            sigma = a.kscale[(int64_t)page * kPage + tok];
            if (a.V && s <= ctx - 1) {
              v_old = a.V[(int64_t)q * L.slot_stride + s];
              d_old = a.D[(int64_t)q * L.slot_stride + (ctx - 1 - s)];
            }
          }
        }
        // every lane waits; the warp leaves together if any lane gave up, so
        // the .sync.aligned TMEM loads below never run on a partial warp
        if (!__all_sync(0xffffffffu, wait_parity(B.af(acc), acc_phase, ctl))) break;
        tc_fence_after();
        const uint32_t trow = tmem_base + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(acc * N);
        for (int r = 0; r < a.rows; ++r) {
          float sum = 0.f;
          for (int c = 0; c < L.H; c += 16) {
            uint32_t v[16];
            tmem_ld16(trow + (uint32_t)(r * L.H + c), v);
            tmem_wait_ld();
#pragma unroll
            for (int u = 0; u < 16; ++u)
              sum = __fmaf_rn(wcur[r * L.H + c + u], fmaxf(__uint_as_float(v[u]), 0.0f), sum);
          }
          if (valid && s <= ctx - 1 + r) {
            const float score = sum * sigma;
            a.scores[((int64_t)q * L.R + r) * L.slot_stride + s] = score;
            if (a.V && r == 0) {
              a.V[(int64_t)q * L.slot_stride + s] = ema_v(v_old, score, a.alpha, a.beta);
              a.D[(int64_t)q * L.slot_stride + (ctx - 1 - s)] = ema_d(d_old, score, a.alpha, a.beta);
            }
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(B.ae(acc));
        if (++acc == 2) { acc = 0; acc_phase ^= 1; }
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
  return key_fp8 && lay.d == 128 && lay.b == kPage && lay.H % 16 == 0 && N >= 16 && N <= 256 && N % 16 == 0 &&
         smem_layout(N, lay.Q).total <= 227 * 1024;
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
  const uint32_t smem = smem_layout(N, L.Q).total;
  cudaError_t e = cudaFuncSetAttribute(k_score_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  k_score_tc<<<sms, kThreads, smem, s>>>(a, tk, tq);
  return cudaGetLastError();
}

}  // namespace spin
