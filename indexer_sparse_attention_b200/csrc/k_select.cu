// k_select.cu -- a1 predict + block max-pool, a2 budget / predicted top /
// exploration / row union, and mask compaction.
//
// a1: z_{r,i} = max(V_i, D_{p_r - i}) and S_{r,j} = max over the valid slots
//     of block j (AI Radio episode, "Title and authors"; SPIN digest,
//     arXiv深度剖析: per-slot and per-offset EMA states).  HBM-bound: 8 bytes
//     per slot of context (V and D read once for all rows); with max pooling,
//     4 bytes of D plus 4 bytes of V's maximum per 32 slots.
// a2: block budget B_r = n_r - floor(s n_r); a share n_exp = floor(gamma B_0)
//     of it goes to uniformly random unkept blocks (SPIN digest, arXiv深度剖析;
//     SPIN listing, Figure 4); each row's top (B_r - n_exp) blocks are unioned
//     (SPIN listing, Table 7, "Row-local union").  Ties: lower block index.
//     The row-0 MTP policy (same table) predicts with row 0 alone, keeps the
//     blocks past row 0's range (the drafts' new keys) and draws the
//     exploration among row 0's unkept blocks.
#include <cooperative_groups.h>

#include <algorithm>

#include "spin_internal.cuh"
#include "block_scan.cuh"

namespace spin {

// ---------------------------------------------------------------------------
// a1 for Mean and Top-4 pooling, and for max pooling at block size 16 (no
// group maxima): grid column x = request; its blocks' warps take 256-slot
// chunks of that request in turn (no division per chunk).  A lane takes
// SPL = 8 consecutive slots: two float4 loads of V and the D window its rows
// need (offsets p0-i0-7 .. p0-i0+R-1) as aligned float4 loads, all issued
// before any use; the b/8 lanes of a block reduce with shuffles.  When a0
// rides along, the row's first warps quantise that request's (row, head)
// query vectors first: the kernel is bound by memory, so they cost next to
// nothing and the select kernel that follows is spared them.  Block sizes
// 16..256 (powers of two).
// ---------------------------------------------------------------------------
template <int R, int P>
__global__ void __launch_bounds__(256, 4) k_predict_pool(StepArgs a) {
  pdl_enter();
  constexpr int SPL = 8, CH = 32 * SPL;
  const Layout L = a.lay;
  const int lane = threadIdx.x & 31;
  const int lb = __ffs(L.b) - 1;
  const int lpb = L.b >= SPL ? L.b / SPL : 1;  // lanes per block
  const int q = blockIdx.x;
  const int wpr = (int)gridDim.y * (blockDim.x >> 5);                   // warps of this request
  const int wr = (int)blockIdx.y * (blockDim.x >> 5) + (threadIdx.x >> 5);  // this warp among them
  if (a.q8) {
    const int nv = a.rows * L.H;
    for (int v = wr; v < nv; v += wpr) quantize_vec(a.q, a.w, a.q_bf16, L.d, (int64_t)q * nv + v, a.q8, a.wq);
  }
  const int64_t ctx = a.ctx_len[q];
  if (ctx < 1 || ctx + R - 1 > L.max_slots) return;  // block-uniform; select reports it
  const int64_t n_last = row_blocks(ctx, R - 1, L.b);
  const int nchunks = (int)((n_last * L.b + CH - 1) / CH);
  const int64_t p0 = ctx - 1;
  const float* V = a.V + (int64_t)q * L.slot_stride;
  const float* D = a.D + (int64_t)q * L.slot_stride;
  // the D window of every lane starts at p0 - i0 - (SPL-1) with i0 = 0 mod
  // SPL: its offset from a 16-byte boundary is the same for all lanes
  const int sh = (int)((p0 + 1) & 3);
  constexpr int kW = R + SPL - 1;            // D values a lane's rows need
  constexpr int kNV = (kW + 3 + 3) / 4;      // float4 loads covering them at any offset
  for (int c = wr; c < nchunks; c += wpr) {
    const int64_t i0 = (int64_t)c * CH + lane * SPL;
    const int64_t j = i0 >> lb;
    const bool active = j < n_last && i0 <= p0 + R - 1;
    float vv[SPL];
    float dw[kW];  // D at offsets p0 - i0 - (SPL-1) .. p0 - i0 + R - 1
#pragma unroll
    for (int k = 0; k < SPL; ++k) vv[k] = __int_as_float(0xff800000);
#pragma unroll
    for (int t = 0; t < kW; ++t) dw[t] = __int_as_float(0xff800000);
    if (active) {
#pragma unroll
      for (int u = 0; u < SPL / 4; ++u) {
        const float4 v4 = __ldg(reinterpret_cast<const float4*>(V + i0) + u);
        vv[4 * u] = v4.x; vv[4 * u + 1] = v4.y; vv[4 * u + 2] = v4.z; vv[4 * u + 3] = v4.w;
      }
      const int64_t ob = p0 - i0 - (SPL - 1) - sh;  // 16-byte aligned start of the window
      if (ob >= 0 && ob + 4 * kNV <= L.slot_stride) {
        float buf[4 * kNV];
#pragma unroll
        for (int u = 0; u < kNV; ++u) {
          const float4 d4 = __ldg(reinterpret_cast<const float4*>(D + ob) + u);
          buf[4 * u] = d4.x; buf[4 * u + 1] = d4.y; buf[4 * u + 2] = d4.z; buf[4 * u + 3] = d4.w;
        }
#define SPIN_DW_FROM(S)                                       \
  _Pragma("unroll") for (int t = 0; t < kW; ++t) dw[t] = buf[t + (S)];
        switch (sh) {  // warp-uniform
          case 0: SPIN_DW_FROM(0) break;
          case 1: SPIN_DW_FROM(1) break;
          case 2: SPIN_DW_FROM(2) break;
          default: SPIN_DW_FROM(3) break;
        }
#undef SPIN_DW_FROM
      } else {  // the window reaches below offset 0 (the newest slots) or past the row
#pragma unroll
        for (int t = 0; t < kW; ++t) {
          const int64_t di = p0 - i0 - (SPL - 1) + t;
          if (di >= 0) dw[t] = __ldg(D + di);
        }
      }
    }
#pragma unroll
    for (int r = 0; r < R; ++r) {
      // this lane's slots i0 .. i0+SPL-1 visible to row r: z = max(V_i, D_{p_r - i}),
      // slot i0+k at offset p_r - (i0+k) = p0 - i0 + r - k  -> dw[r - k + SPL - 1]
      float x;
      if (P == SPIN_POOL_MAX) {
        x = __int_as_float(0xff800000);
#pragma unroll
        for (int k = 0; k < SPL; ++k)
          if (active && i0 + k <= p0 + r) x = fmaxf(x, fmaxf(vv[k], dw[r - k + SPL - 1]));
        for (int o = lpb >> 1; o >= 1; o >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, o));
      } else if (P == SPIN_POOL_MEAN) {
        // the run of SPL slots in slot order, then runs added pairwise (lanes
        // l and l^1, then pairs of pairs, ...): the order the reduction fixes
        double sum = 0.0;
        int cnt = 0;
#pragma unroll
        for (int k = 0; k < SPL; ++k)
          if (active && i0 + k <= p0 + r) {
            sum += (double)fmaxf(vv[k], dw[r - k + SPL - 1]);
            ++cnt;
          }
        for (int o = 1; o < lpb; o <<= 1) {
          sum += __shfl_xor_sync(0xffffffffu, sum, o);
          cnt += __shfl_xor_sync(0xffffffffu, cnt, o);
        }
        x = cnt ? (float)(sum / (double)cnt) : 0.f;
      } else {
        // the block's four largest z (a multiset: any merge order gives it),
        // summed from the largest down
        float t[4] = {__int_as_float(0xff800000), __int_as_float(0xff800000), __int_as_float(0xff800000),
                      __int_as_float(0xff800000)};
        int cnt = 0;
#pragma unroll
        for (int k = 0; k < SPL; ++k)
          if (active && i0 + k <= p0 + r) {
            float z = fmaxf(vv[k], dw[r - k + SPL - 1]);
            ++cnt;
#pragma unroll
            for (int u = 0; u < 4; ++u) {  // insert, keeping t descending
              const float hi = fmaxf(t[u], z), lo = fminf(t[u], z);
              t[u] = hi;
              z = lo;
            }
          }
        for (int o = 1; o < lpb; o <<= 1) {
          float u4[4];
#pragma unroll
          for (int u = 0; u < 4; ++u) u4[u] = __shfl_xor_sync(0xffffffffu, t[u], o);
          cnt += __shfl_xor_sync(0xffffffffu, cnt, o);
#pragma unroll
          for (int u = 0; u < 4; ++u) {  // insert the partner's values
            float z = u4[u];
#pragma unroll
            for (int w = 0; w < 4; ++w) {
              const float hi = fmaxf(t[w], z), lo = fminf(t[w], z);
              t[w] = hi;
              z = lo;
            }
          }
        }
        const int mtop = cnt < 4 ? cnt : 4;
        double sum = 0.0;
#pragma unroll
        for (int u = 0; u < 4; ++u)
          if (u < mtop) sum += (double)t[u];
        x = mtop ? (float)(sum / (double)mtop) : 0.f;
      }
      if (active && (lane & (lpb - 1)) == 0 && j < row_blocks(ctx, r, L.b))
        a.S[((int64_t)q * L.R + r) * L.blk_stride + j] = x;
    }
  }
}

// ---------------------------------------------------------------------------
// a1 for one row (R = 1), max pooling, V's group maxima kept, block size
// B in {32, 64, 128, 256}: every load is coalesced.  A warp takes 1,024
// slots, NB = 1024 / B blocks J0 .. J0+NB-1.  In offset space (delta = p0 - i)
// those blocks are one run of 1,024 offsets, and block J0+NB-1-s is its s-th
// run of B offsets.  The warp loads the run as eight float4 per lane from a
// 16-byte boundary (the run starts sh = (p0 + 1) mod 4 past it) plus one
// float4 past its end: every load instruction reads 512 contiguous bytes.
// A lane's float4 f holds run positions 4f - sh .. 4f + 3 - sh; its last
// 4 - sh values and the first sh values of float4 f + 1 (one shuffle down)
// are run positions 4f .. 4f + 3, all in run block floor(4f / B), so the B/4
// lanes of a block reduce with xor shuffles and no value crosses a block
// edge.  V's part: one group maximum per lane (32 groups per chunk, one
// coalesced load), the group of the newest slot read from V itself; a
// block's groups reduce with shuffles.  Lanes 0 .. NB-1 store the chunk's
// block scores, one coalesced store.
// ---------------------------------------------------------------------------
template <int B, bool ML = false>
__global__ void __launch_bounds__(256, 4) k_predict_max_r1(StepArgs a_in) {
  pdl_enter();
  StepArgs a = a_in;
  if constexpr (ML) layer_of_block(a);  // ML: one launch over several layers
  constexpr int NB = 1024 / B;                 // blocks per chunk
  constexpr int LPS = B / 4 < 32 ? B / 4 : 32;  // lanes of a block's run in one load instruction
  constexpr int IPB = B / 4 > 32 ? B / 128 : 1;  // load instructions per block (B = 256: 2)
  constexpr int SPI = 32 / LPS;                // blocks per load instruction
  constexpr int GPB = B / 32;                  // V groups per block
  const Layout L = a.lay;
  const int lane = threadIdx.x & 31;
  const int q = blockIdx.x;
  const int wpr = (int)gridDim.y * (blockDim.x >> 5);
  const int wr = (int)blockIdx.y * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (a.q8) {
    const int nv = a.rows * L.H;
    for (int v = wr; v < nv; v += wpr) quantize_vec(a.q, a.w, a.q_bf16, L.d, (int64_t)q * nv + v, a.q8, a.wq);
  }
  const int64_t ctx = a.ctx_len[q];
  if (ctx < 1 || ctx > L.max_slots) return;  // block-uniform; select reports it
  const int64_t n_last = (ctx + B - 1) / B;
  const int nchunks = (int)((n_last + NB - 1) / NB);
  const int64_t p0 = ctx - 1;
  const float* V = a.V + (int64_t)q * L.slot_stride;
  const float* D = a.D + (int64_t)q * L.slot_stride;
  const float* VG = a.vmax + (int64_t)q * L.vg_stride;
  const int sh = (int)((p0 + 1) & 3);
  const float kNeg = __int_as_float(0xff800000);
  for (int c = wr; c < nchunks; c += wpr) {
    const int64_t J0 = (int64_t)c * NB;
    const int64_t A = p0 + 1 - (J0 + NB) * B - sh;  // 16-byte boundary at or below the run's start
    float4 x[9];
#pragma unroll
    for (int u = 0; u < 9; ++u) {
      const int64_t o = A + 128 * u + 4 * lane;  // a float4 lies wholly inside or outside [0, stride)
      x[u] = make_float4(kNeg, kNeg, kNeg, kNeg);
      if ((u < 8 || lane == 0) && o >= 0 && o < L.slot_stride) x[u] = __ldg(reinterpret_cast<const float4*>(D + o));
    }
    // V's part: lane = group g0 + lane of the chunk; groups past the newest
    // slot see nothing, and the newest slot's group gp is read from V itself
    // (the whole warp: one coalesced load of its visible values)
    const int64_t g0 = (J0 * B) >> 5, g = g0 + lane, gp = p0 >> 5;
    float vg = kNeg;
    if (g < gp) vg = __ldg(VG + g);
    if (gp >= g0 && gp < g0 + 32) {  // warp-uniform
      const int64_t i = 32 * gp + lane;
      const float m = warp_max(i <= p0 ? __ldg(V + i) : kNeg);
      if (g == gp) vg = m;
    }
    // run-aligned float4 maxima: hi = values e >= sh of x[u], lo = values e < sh
    float hi[9], lo[9];
#pragma unroll
    for (int u = 0; u < 9; ++u) {
      const float e[4] = {x[u].x, x[u].y, x[u].z, x[u].w};
      float h = kNeg, l = kNeg;
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        if (k >= sh) h = fmaxf(h, e[k]);
        else l = fmaxf(l, e[k]);
      }
      hi[u] = h;
      lo[u] = l;
    }
    float seg[8];  // block maxima of D per load instruction (each lane of a block's lanes)
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      float nxt = __shfl_down_sync(0xffffffffu, lo[u], 1);
      const float wrap = __shfl_sync(0xffffffffu, lo[u + 1], 0);  // lane 31: the next instruction's lane 0
      if (lane == 31) nxt = wrap;
      float m = fmaxf(hi[u], nxt);
#pragma unroll
      for (int o = LPS >> 1; o >= 1; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
      seg[u] = m;
    }
    // lane k < NB gathers block J0 + k, run block s = NB - 1 - k
    const int k = lane;
    const int s = NB - 1 - k;
    float res = kNeg;
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int src = IPB == 1 ? ((s & (SPI - 1)) * LPS) & 31 : 0;
      const float v = __shfl_sync(0xffffffffu, seg[u], src);
      const bool mine = IPB == 1 ? (u == s / SPI) : (u / IPB == s);
      if (k < NB && mine) res = fmaxf(res, v);
    }
#pragma unroll
    for (int o = GPB >> 1; o >= 1; o >>= 1) vg = fmaxf(vg, __shfl_xor_sync(0xffffffffu, vg, o));
    const float vb = __shfl_sync(0xffffffffu, vg, (k * GPB) & 31);
    if (k < NB && J0 + k < n_last) a.S[(int64_t)q * L.R * L.blk_stride + J0 + k] = fmaxf(res, vb);
  }
}

// ---------------------------------------------------------------------------
// a1 for max pooling with V's 32-slot group maxima kept (block size >= 32).
// The max over a block of max(V_i, D_{p_r-i}) is the larger of V's maximum
// and D's, so a lane takes one aligned group of 32 slots i0 .. i0+31:
//   V's part: the group's maximum when the whole group is visible (i0 + 31
//     <= p0), else -- only in the group of the newest slots -- the max of
//     its visible V values, read directly;
//   D's part: row r needs offsets p_r - i0 - 31 .. p_r - i0, so the rows
//     share one window of 31 + R values of D, loaded as aligned float4 (its
//     offset from a 16-byte boundary is the same for every lane) and reduced
//     once over the part all rows share.
// A warp's chunk is 1,024 slots: 4.1 B of memory per slot (D and one group
// maximum) in 10 loads per lane, one round trip.  The b/32 lanes of a block
// reduce with shuffles.  a0 rides along as in k_predict_pool.
// ---------------------------------------------------------------------------
// Row maxima of D from the window buf[S .. S + 30 + R]: row r takes
// buf[S + r .. S + r + 31].
template <int S, int R>
__device__ __forceinline__ void d_row_max(const float* buf, float* dmax) {
  float common = buf[S + R - 1];
#pragma unroll
  for (int t = S + R; t <= S + 31; ++t) common = fmaxf(common, buf[t]);
#pragma unroll
  for (int r = 0; r < R; ++r) {
    float x = common;
#pragma unroll
    for (int t = S + r; t < S + R - 1; ++t) x = fmaxf(x, buf[t]);    // head only row r sees
#pragma unroll
    for (int t = S + 32; t <= S + 31 + r; ++t) x = fmaxf(x, buf[t]);  // tail only row r sees
    dmax[r] = x;
  }
}

template <int R>
__global__ void __launch_bounds__(256, 4) k_predict_max(StepArgs a) {
  pdl_enter();
  const Layout L = a.lay;
  const int lane = threadIdx.x & 31;
  const int lb = __ffs(L.b) - 1;
  const int lpb = L.b >> 5;  // lanes per block
  const int q = blockIdx.x;
  const int wpr = (int)gridDim.y * (blockDim.x >> 5);
  const int wr = (int)blockIdx.y * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (a.q8) {
    const int nv = a.rows * L.H;
    for (int v = wr; v < nv; v += wpr) quantize_vec(a.q, a.w, a.q_bf16, L.d, (int64_t)q * nv + v, a.q8, a.wq);
  }
  const int64_t ctx = a.ctx_len[q];
  if (ctx < 1 || ctx + R - 1 > L.max_slots) return;  // block-uniform; select reports it
  const int64_t n_last = row_blocks(ctx, R - 1, L.b);
  const int nchunks = (int)((n_last * L.b + 1023) / 1024);
  const int64_t p0 = ctx - 1;
  const float* V = a.V + (int64_t)q * L.slot_stride;
  const float* D = a.D + (int64_t)q * L.slot_stride;
  const float* VG = a.vmax + (int64_t)q * L.vg_stride;
  const int sh = (int)((p0 + 1) & 3);       // (p0 - i0 - 31) mod 4, the same for every lane
  constexpr int kNV = (31 + R + 3 + 3) / 4;  // float4 loads covering 31 + R values at any offset
  for (int c = wr; c < nchunks; c += wpr) {
    const int64_t i0 = (int64_t)c * 1024 + lane * 32;
    const int64_t j = i0 >> lb;
    const bool active = j < n_last && i0 <= p0 + R - 1;
    float x[R];
#pragma unroll
    for (int r = 0; r < R; ++r) x[r] = __int_as_float(0xff800000);
    if (active) {
      const bool whole = i0 + 31 <= p0;
      const float g = whole ? __ldg(VG + (i0 >> 5)) : __int_as_float(0xff800000);
      float buf[4 * kNV];  // D at offsets ob .. ob + 4 kNV - 1
      const int64_t ob = p0 - i0 - 31 - sh;
      if (ob >= 0 && ob + 4 * kNV <= L.slot_stride) {
#pragma unroll
        for (int u = 0; u < kNV; ++u) {
          const float4 d4 = __ldg(reinterpret_cast<const float4*>(D + ob) + u);
          buf[4 * u] = d4.x; buf[4 * u + 1] = d4.y; buf[4 * u + 2] = d4.z; buf[4 * u + 3] = d4.w;
        }
      } else {  // the newest slots (offsets below 0 are past the row) or the end of the row
#pragma unroll
        for (int t = 0; t < 4 * kNV; ++t) {
          const int64_t di = ob + t;
          buf[t] = (di >= 0 && di < L.slot_stride) ? __ldg(D + di) : __int_as_float(0xff800000);
        }
      }
      float dmax[R];
      switch (sh) {  // warp-uniform
        case 0: d_row_max<0, R>(buf, dmax); break;
        case 1: d_row_max<1, R>(buf, dmax); break;
        case 2: d_row_max<2, R>(buf, dmax); break;
        default: d_row_max<3, R>(buf, dmax); break;
      }
#pragma unroll
      for (int r = 0; r < R; ++r) x[r] = fmaxf(g, dmax[r]);
      if (!whole) {  // the group of the newest slots: V's visible values
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const float4 v4 = __ldg(reinterpret_cast<const float4*>(V + i0) + u);
          const float vals[4] = {v4.x, v4.y, v4.z, v4.w};
#pragma unroll
          for (int e = 0; e < 4; ++e)
#pragma unroll
            for (int r = 0; r < R; ++r)
              if (i0 + 4 * u + e <= p0 + r) x[r] = fmaxf(x[r], vals[e]);
        }
      }
    }
#pragma unroll
    for (int r = 0; r < R; ++r) {
      float y = x[r];
      for (int o = lpb >> 1; o >= 1; o >>= 1) y = fmaxf(y, __shfl_xor_sync(0xffffffffu, y, o));
      if (active && (lane & (lpb - 1)) == 0 && j < row_blocks(ctx, r, L.b))
        a.S[((int64_t)q * L.R + r) * L.blk_stride + j] = y;
    }
  }
}

cudaError_t launch_predict_pool(const StepArgs& a, cudaStream_t s) {
  // one wave (4 blocks of 256 threads per SM at <= 64 registers) over all
  // requests, each request's chunks shared by the gx blocks of its column
  const int64_t chunks = (a.lay.slot_stride + 255) / 256;
  int64_t gx = (148 * 4) / a.lay.Q;
  gx = std::min<int64_t>(gx, (chunks + 7) / 8);
  gx = std::max<int64_t>(std::min<int64_t>(gx, 65535), 1);
  PdlLaunch l(dim3((unsigned)a.lay.Q, (unsigned)gx), dim3(256), 0, s);
  l.attr[0].val.programmaticStreamSerializationAllowed = a.no_pdl ? 0 : 1;
  void (*k)(StepArgs) = nullptr;
  if (a.nl > 1) {  // several layers: one row, max pooling with V's group maxima only
    if (a.nl > kMaxLayerBatch || a.rows != 1 || a.mtp_row0 || a.pooling != SPIN_POOL_MAX || !a.vmax)
      return cudaErrorInvalidValue;
    // a few blocks per (layer, request) and SM, each warp looping over its chunks: a grid
    // sized by the longest context would be mostly blocks with nothing to do
    int64_t cy = (a.lay.slot_stride + 8 * 1024 - 1) / (8 * 1024);
    cy = std::max<int64_t>(1, std::min<int64_t>(cy, (148 * 8 + a.lay.Q * a.nl - 1) / (a.lay.Q * a.nl)));
    PdlLaunch m(dim3((unsigned)a.lay.Q, (unsigned)std::min<int64_t>(cy, 65535), (unsigned)a.nl), dim3(256), 0, s);
    m.attr[0].val.programmaticStreamSerializationAllowed = a.no_pdl ? 0 : 1;
    k = a.lay.b == 32 ? k_predict_max_r1<32, true> : a.lay.b == 64 ? k_predict_max_r1<64, true>
      : a.lay.b == 128 ? k_predict_max_r1<128, true> : k_predict_max_r1<256, true>;
    return cudaLaunchKernelEx(&m.cfg, k, a);
  }
  if (a.pooling == SPIN_POOL_MAX && a.vmax && (a.mtp_row0 || a.rows == 1)) {
    // one 1,024-slot chunk per warp, many short blocks: the hardware hands
    // them to SMs as they free up, so the kernel also fills the SMs another
    // stream's kernel leaves idle
    const int64_t cy = (a.lay.slot_stride + 8 * 1024 - 1) / (8 * 1024);
    PdlLaunch m(dim3((unsigned)a.lay.Q, (unsigned)std::min<int64_t>(cy, 65535)), dim3(256), 0, s);
    m.attr[0].val.programmaticStreamSerializationAllowed = a.no_pdl ? 0 : 1;
    k = a.lay.b == 32 ? k_predict_max_r1<32> : a.lay.b == 64 ? k_predict_max_r1<64>
      : a.lay.b == 128 ? k_predict_max_r1<128> : k_predict_max_r1<256>;
    return cudaLaunchKernelEx(&m.cfg, k, a);
  }
  if (a.pooling == SPIN_POOL_MAX && a.vmax) {  // V's group maxima kept (block size >= 32)
    switch (a.rows) {
      case 2: k = k_predict_max<2>; break;
      case 3: k = k_predict_max<3>; break;
      default: k = k_predict_max<4>;
    }
    return cudaLaunchKernelEx(&l.cfg, k, a);
  }
#define SPIN_PREDICT_CASE(R)                                            \
  case R:                                                               \
    k = a.pooling == SPIN_POOL_MEAN   ? k_predict_pool<R, SPIN_POOL_MEAN> \
        : a.pooling == SPIN_POOL_TOP4 ? k_predict_pool<R, SPIN_POOL_TOP4> \
                                      : k_predict_pool<R, SPIN_POOL_MAX>; \
    break;
  switch (a.mtp_row0 ? 1 : a.rows) {  // R: the rows whose block scores are needed
    SPIN_PREDICT_CASE(1)
    SPIN_PREDICT_CASE(2)
    SPIN_PREDICT_CASE(3)
    default:
      k = a.pooling == SPIN_POOL_MEAN   ? k_predict_pool<4, SPIN_POOL_MEAN>
          : a.pooling == SPIN_POOL_TOP4 ? k_predict_pool<4, SPIN_POOL_TOP4>
                                        : k_predict_pool<4, SPIN_POOL_MAX>;
  }
#undef SPIN_PREDICT_CASE
  return cudaLaunchKernelEx(&l.cfg, k, a);
}

// ---------------------------------------------------------------------------
// a2: one CTA (1024 threads) per request.  Keys of the candidates live in
// shared memory; an MSB-first radix select (4 x 8-bit digits) finds the
// threshold key T of the wanted rank and how many elements equal to T to
// take; an ordered pass then takes every key > T and the lowest-index keys
// == T.  Exploration reuses the same routine on ~Philox keys of the unkept
// blocks (largest ~key = smallest key).  Finally the mask row and the
// ascending kept-block list are written.
// ---------------------------------------------------------------------------
constexpr int kSelThreads = 1024;

struct SelShared {
  uint32_t hist[256];
  uint32_t digit[2];
  uint32_t digit_r[4][2];  // per-row digits of the batched radix passes
  int scan[33];
};

// Shared memory of the one-CTA select: block keys, labels and the
// exploration list; with several predicting rows whose keys fit next to
// them, every row's keys too, so the rows' radix passes run together.
constexpr size_t kSelBatchCap = 160 * 1024;
__host__ __device__ inline size_t select_smem(int64_t blk_stride, int rows) {
  const size_t base = (size_t)blk_stride * 5 + (size_t)2048 * 8;  // keys, labels, kExpCap (key, block) pairs
  const size_t extra = (size_t)rows * 4 * (size_t)blk_stride;
  return (rows > 1 && base + extra <= kSelBatchCap) ? base + extra : base;
}
__host__ __device__ inline bool select_batched(int64_t blk_stride, int rows) {
  return rows > 1 && (size_t)blk_stride * 5 + (size_t)2048 * 8 + (size_t)rows * 4 * blk_stride <= kSelBatchCap;
}

// Radix select over keys[0..n) restricted to elements with valid(j).  `want`
// must be in [1, #valid].  Returns T and the number of elements equal to T
// that belong to the top `want`.
template <class Valid>
__device__ void radix_select_desc(const uint32_t* keys, int n, Valid valid, uint32_t want,
                                  SelShared& sh, uint32_t* T_out, uint32_t* eq_out) {
  uint32_t prefix = 0, pmask = 0, remaining = want;
  for (int shift = 24; shift >= 0; shift -= 8) {
    for (int i = threadIdx.x; i < 256; i += blockDim.x) sh.hist[i] = 0;
    __syncthreads();
    for (int j = threadIdx.x; j < n; j += blockDim.x) {
      if (!valid(j)) continue;
      const uint32_t k = keys[j];
      if ((k & pmask) == prefix) atomicAdd(&sh.hist[(k >> shift) & 255u], 1u);
    }
    __syncthreads();
    if (threadIdx.x < 32) warp_find_digit_desc<256>(sh.hist, remaining, sh.digit);
    __syncthreads();
    prefix |= sh.digit[0] << shift;
    pmask |= 255u << shift;
    remaining = sh.digit[1];
    __syncthreads();
  }
  *T_out = prefix;
  *eq_out = remaining;
}

// Marks m[j] = label for the top `want` valid elements (keys > T, then the
// lowest-index keys == T).  Each thread walks a contiguous chunk so that the
// "lowest index" order is a block scan.
// The radix passes of several rows at once.  Row r's keys are kb[r stride
// + j], j < n_r; rows with want_r = 0 take no select.  One sweep over every
// row's keys per 8-bit digit fills a histogram per row, and one warp per row
// finds its digit.  Each row gets the T and eq of radix_select_desc.  The
// per-row values live in scalars (a row index selects among them), so
// nothing goes to local memory.
__device__ void radix_select_rows(const uint32_t* kb, int stride, int pr, const int (&n)[4], const uint32_t (&want)[4],
                                  uint32_t (*hist)[256], SelShared& sh, uint32_t (&T)[4], uint32_t (&eq)[4]) {
  uint32_t p0 = 0, p1 = 0, p2 = 0, p3 = 0;
  uint32_t m0 = want[0], m1 = want[1], m2 = want[2], m3 = want[3];
  uint32_t pmask = 0;
  for (int shift = 24; shift >= 0; shift -= 8) {
    for (int i = threadIdx.x; i < pr * 256; i += blockDim.x) hist[i >> 8][i & 255] = 0;
    __syncthreads();
    for (int i = threadIdx.x; i < pr * stride; i += blockDim.x) {
      const int r = (i >= stride) + (i >= 2 * stride) + (i >= 3 * stride);
      const int j = i - r * stride;
      const int nr = r == 0 ? n[0] : r == 1 ? n[1] : r == 2 ? n[2] : n[3];
      const uint32_t rem = r == 0 ? m0 : r == 1 ? m1 : r == 2 ? m2 : m3;
      const uint32_t pre = r == 0 ? p0 : r == 1 ? p1 : r == 2 ? p2 : p3;
      if (j >= nr || rem == 0) continue;
      const uint32_t k = kb[i];
      if ((k & pmask) == pre) atomicAdd(&hist[r][(k >> shift) & 255u], 1u);
    }
    __syncthreads();
    const int w = threadIdx.x >> 5;
    if (w < pr) {
      const uint32_t rem = w == 0 ? m0 : w == 1 ? m1 : w == 2 ? m2 : m3;
      if (rem != 0) warp_find_digit_desc<256>(hist[w], rem, sh.digit_r[w]);
    }
    __syncthreads();
    if (m0) { p0 |= sh.digit_r[0][0] << shift; m0 = sh.digit_r[0][1]; }
    if (pr > 1 && m1) { p1 |= sh.digit_r[1][0] << shift; m1 = sh.digit_r[1][1]; }
    if (pr > 2 && m2) { p2 |= sh.digit_r[2][0] << shift; m2 = sh.digit_r[2][1]; }
    if (pr > 3 && m3) { p3 |= sh.digit_r[3][0] << shift; m3 = sh.digit_r[3][1]; }
    pmask |= 255u << shift;
    __syncthreads();
  }
  T[0] = p0; T[1] = p1; T[2] = p2; T[3] = p3;
  eq[0] = m0; eq[1] = m1; eq[2] = m2; eq[3] = m3;
}

template <class Valid>
__device__ void mark_selected(const uint32_t* keys, int n, Valid valid, uint32_t T, uint32_t eq_take,
                              uint8_t* m, uint8_t label, SelShared& sh) {
  const int chunk = (n + blockDim.x - 1) / blockDim.x;
  const int lo = threadIdx.x * chunk, hi = min(n, lo + chunk);
  int eq = 0;
  for (int j = lo; j < hi; ++j)
    if (valid(j) && keys[j] == T) ++eq;
  int total;
  int base = block_exclusive_scan(eq, sh.scan, &total);
  for (int j = lo; j < hi; ++j) {
    if (!valid(j)) continue;
    const uint32_t k = keys[j];
    if (k > T) {
      m[j] = label;
    } else if (k == T) {
      if ((uint32_t)base < eq_take) m[j] = label;
      ++base;
    }
  }
  __syncthreads();
}

constexpr int kExpCap = 2048;

// The `take` entries of list[0 .. cnt) first by (key, block index) go to
// mark(block): a radix select of the largest ~key (the smallest key) over
// the list, then the entries past the threshold, and the lowest blocks among
// those equal to it.  `scratch` holds cnt words.  All threads of the CTA call
// it; 1 <= take <= cnt.
template <class Mark>
__device__ void draw_from_list(const uint2* list, int cnt, int take, int* scratch, Mark mark, SelShared& sh) {
  uint32_t* nk = reinterpret_cast<uint32_t*>(scratch);
  for (int i = threadIdx.x; i < cnt; i += blockDim.x) nk[i] = ~list[i].x;
  __syncthreads();
  uint32_t T, eq_take;
  radix_select_desc(nk, cnt, [](int) { return true; }, (uint32_t)take, sh, &T, &eq_take);
  if (threadIdx.x == 0) sh.digit[0] = 0;
  __syncthreads();
  for (int i = threadIdx.x; i < cnt; i += blockDim.x) {
    if (nk[i] > T) mark((int)list[i].y);
    else if (nk[i] == T) atomicAdd(&sh.digit[0], 1u);
  }
  __syncthreads();
  const uint32_t n_eq = sh.digit[0];
  if (n_eq == eq_take) {
    for (int i = threadIdx.x; i < cnt; i += blockDim.x)
      if (nk[i] == T) mark((int)list[i].y);
  } else if (threadIdx.x == 0) {
    // equal 32-bit keys: the eq_take lowest blocks among them, one at a time
    uint32_t last = 0;
    for (uint32_t t = 0; t < eq_take; ++t) {
      uint32_t best = 0xFFFFFFFFu;
      for (int i = 0; i < cnt; ++i)
        if (nk[i] == T && list[i].y < best && (t == 0 || list[i].y > last)) best = list[i].y;
      mark((int)best);
      last = best;
    }
  }
  __syncthreads();
}

// Exploration draw by a short list: the Philox keys are uniform, so the
// `take` smallest of n_cand lie below t = (1.25 take + 64) / n_cand * 2^32
// with overwhelming probability.  Candidates under t are appended to a
// shared list (one atomic per warp), and a radix select over the list takes
// its `take` smallest (key, block index) pairs.  Returns false -- nothing marked -- when the list holds fewer
// than `take` entries or overflows, and the caller runs the radix select.

__device__ bool explore_by_list(const StepArgs& a, int q, uint8_t* m, int n_last, int take, int n_cand,
                                uint2* list, int* rank, SelShared& sh) {
  const double frac = (1.25 * take + 64.0) / (double)n_cand;
  const uint64_t t = frac >= 1.0 ? (1ull << 32) : (uint64_t)(frac * 4294967296.0);
  if (threadIdx.x == 0) sh.digit[0] = 0;
  __syncthreads();
  const int lane = threadIdx.x & 31;
  // a thread takes blocks 4i .. 4i+3: one Philox gives their four keys
  for (int i0 = 0; 4 * i0 < n_last; i0 += blockDim.x) {  // warp-uniform trip count
    const int i = i0 + (int)threadIdx.x;
    bool c4[4];
    bool any = false;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int j = 4 * i + k;
      c4[k] = j < n_last && m[j] == 0;
      any |= c4[k];
    }
    const uint4 w = any ? explore_keys4(a.seed, (uint32_t)i, (uint32_t)q, (uint32_t)a.layer, (uint64_t)a.step)
                        : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const uint32_t u = word_of(w, k);
      const bool in = c4[k] && (uint64_t)u < t;
      const uint32_t bal = __ballot_sync(0xffffffffu, in);
      if (!bal) continue;
      uint32_t at = 0;
      if (lane == 0) at = atomicAdd(&sh.digit[0], (uint32_t)__popc(bal));
      at = __shfl_sync(0xffffffffu, at, 0) + __popc(bal & ((1u << lane) - 1u));
      if (in && at < (uint32_t)kExpCap) list[at] = make_uint2(u, (uint32_t)(4 * i + k));
    }
  }
  __syncthreads();
  const int cnt = (int)sh.digit[0];
  if (cnt < take || cnt > kExpCap) return false;  // uniform: every thread reads the same count
  draw_from_list(list, cnt, take, rank, [m](int j) { m[j] = 2; }, sh);
  return true;
}

// Ordered compaction of the kept blocks of one request into its work list;
// with mask_out, the labels of blocks 0 .. n_last-1 are written there too.
// With stage (shared memory, n_last ints), the list is built there and both
// outputs go out with coalesced stores.
__device__ void compact_row(const uint8_t* m, int n_last, int32_t* work, int32_t* kept, int* scan,
                            uint8_t* mask_out = nullptr, int32_t* stage = nullptr) {
  const int chunk = (n_last + blockDim.x - 1) / blockDim.x;
  const int lo = threadIdx.x * chunk, hi = min(n_last, lo + chunk);
  int c = 0;
  for (int j = lo; j < hi; ++j) c += m[j] != 0;
  int total;
  int pos = block_exclusive_scan(c, scan, &total);
  if (stage) {
    for (int j = lo; j < hi; ++j)
      if (m[j]) stage[pos++] = j;
    if (mask_out)
      for (int j = threadIdx.x; j < n_last; j += blockDim.x) mask_out[j] = m[j];
    __syncthreads();
    for (int i = threadIdx.x; i < total; i += blockDim.x) work[i] = stage[i];
  } else {
    for (int j = lo; j < hi; ++j) {
      const uint8_t v = m[j];
      if (mask_out) mask_out[j] = v;
      if (v) work[pos++] = j;
    }
  }
  if (threadIdx.x == 0) *kept = total;
}

// RC: the number of query rows when fixed at compile time (0: a.rows); the
// decode step's one row and the MTP step's four have their own instances.
template <int RC, bool ML = false>
__global__ void __launch_bounds__(kSelThreads) k_select(StepArgs a_in) {
  pdl_enter();
  StepArgs a = a_in;
  if constexpr (ML) layer_of_block(a);  // ML: one launch over several layers
  if (a.step_dev) a.step = *a.step_dev + a.step_add;  // the state's counter (read after the predecessors finished)
  const Layout L = a.lay;
  const int rows = RC ? RC : a.rows;
  const int q = blockIdx.x;
  extern __shared__ __align__(16) uint8_t dyn[];
  uint32_t* keys = reinterpret_cast<uint32_t*>(dyn);
  uint8_t* m = dyn + 4 * L.blk_stride;
  uint2* list = reinterpret_cast<uint2*>(dyn + 5 * L.blk_stride);  // kExpCap (key, block) pairs
  __shared__ SelShared sh;
  __shared__ uint32_t hist_r[4][256];

  if (a.q8) {
    // a0 for this request's (row, head) vectors, one warp each; the score
    // kernel reads them after this kernel
    const int nv = rows * L.H, warp = threadIdx.x >> 5;
    for (int i = warp; i < nv; i += kSelThreads / 32)
      quantize_vec(a.q, a.w, a.q_bf16, L.d, (int64_t)q * nv + i, a.q8, a.wq);
  }
  const int64_t ctx = a.ctx_len[q];
  uint8_t* mask_row = a.mask + (int64_t)q * L.max_blocks;
  if (ctx < 1 || ctx + rows - 1 > L.max_slots) {
    if (threadIdx.x == 0) {
      if (!a.quiet) raise_error(a.err, ERR_CTX_LEN, q, (uint32_t)ctx);
      a.kept[q] = 0;
      if (a.ctx_sel) a.ctx_sel[q] = -1;
    }
    for (int64_t j = threadIdx.x; j < L.max_blocks; j += blockDim.x) mask_row[j] = 0;
    return;
  }
  if (a.ctx_sel && threadIdx.x == 0) a.ctx_sel[q] = (int32_t)ctx;
  const int n_last = (int)row_blocks(ctx, rows - 1, L.b);
  for (int j = threadIdx.x; j < n_last; j += blockDim.x) m[j] = 0;
  __syncthreads();

  if (a.sparsity == 0.0f) {
    for (int j = threadIdx.x; j < n_last; j += blockDim.x) m[j] = 1;
    __syncthreads();
  } else {
    const int64_t n0 = row_blocks(ctx, 0, L.b);
    const int64_t n_exp = explore_count(block_budget(n0, a.sparsity), a.gamma);
    const int pr = (RC == 1 || a.mtp_row0) ? 1 : rows;  // rows whose predicted sets are unioned
    if (pr > 1 && select_batched(L.blk_stride, rows)) {
      // every row's keys on chip (row r at kb + r blk_stride), the rows'
      // radix passes together
      uint32_t* kb = reinterpret_cast<uint32_t*>(dyn + select_smem(L.blk_stride, 1));
      const int stride = (int)L.blk_stride;
      int nrow[4] = {0, 0, 0, 0};
      uint32_t want[4] = {0u, 0u, 0u, 0u};
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        if (r >= pr) break;
        nrow[r] = (int)row_blocks(ctx, r, L.b);
        const int64_t n_pred = block_budget(nrow[r], a.sparsity) - n_exp;
        want[r] = (n_pred > 0 && n_pred < nrow[r]) ? (uint32_t)n_pred : 0u;
        const float* S = a.S + ((int64_t)q * L.R + r) * L.blk_stride;
        for (int j = threadIdx.x; j < nrow[r]; j += blockDim.x) {
          kb[r * stride + j] = fkey(S[j]);
          if (n_pred >= nrow[r]) m[j] = 1;  // this row keeps all its blocks
        }
      }
      __syncthreads();
      uint32_t T[4], eq[4];
      radix_select_rows(kb, stride, pr, nrow, want, hist_r, sh, T, eq);
      auto all = [](int) { return true; };
#pragma unroll
      for (int r = 0; r < 4; ++r)
        if (r < pr && want[r]) mark_selected(kb + r * stride, nrow[r], all, T[r], eq[r], m, 1, sh);
    }
    for (int r = 0; r < pr && !(pr > 1 && select_batched(L.blk_stride, rows)); ++r) {
      const int n = (int)row_blocks(ctx, r, L.b);
      const int64_t n_pred = block_budget(n, a.sparsity) - n_exp;
      const float* S = a.S + ((int64_t)q * L.R + r) * L.blk_stride;
      for (int j0 = 0; j0 < n; j0 += 4 * kSelThreads) {  // four loads in flight per thread
        float v[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int j = j0 + u * kSelThreads + (int)threadIdx.x;
          v[u] = j < n ? S[j] : 0.f;
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int j = j0 + u * kSelThreads + (int)threadIdx.x;
          if (j < n) keys[j] = fkey(v[u]);
        }
      }
      __syncthreads();
      auto all = [](int) { return true; };
      if (n_pred >= n) {
        for (int j = threadIdx.x; j < n; j += blockDim.x) m[j] = 1;
        __syncthreads();
      } else if (n_pred > 0) {
        uint32_t T, eq;
        radix_select_desc(keys, n, all, (uint32_t)n_pred, sh, &T, &eq);
        mark_selected(keys, n, all, T, eq, m, 1, sh);
      }
    }
    if (a.mtp_row0) {  // the drafts' new blocks
      for (int j = (int)n0 + threadIdx.x; j < n_last; j += blockDim.x) m[j] = 1;
      __syncthreads();
    }
    // exploration among the unkept blocks of the last row's range
    auto cand = [m](int j) { return m[j] == 0; };
    int n_cand;
    if (rows == 1) {  // one row: exactly min(max(n_pred, 0), n) blocks are predicted
      const int64_t n_pred = block_budget(n_last, a.sparsity) - n_exp;
      n_cand = n_last - (int)(n_pred < 0 ? 0 : n_pred > n_last ? n_last : n_pred);
    } else {
      int c = 0;
      for (int j = threadIdx.x; j < n_last; j += blockDim.x) c += (m[j] == 0);
      block_exclusive_scan(c, sh.scan, &n_cand);
    }
    const int64_t take = n_exp < n_cand ? n_exp : n_cand;
    if (take == n_cand) {
      for (int j = threadIdx.x; j < n_last; j += blockDim.x)
        if (m[j] == 0) m[j] = 2;
      __syncthreads();
    } else if (take > 0 && explore_by_list(a, q, m, n_last, (int)take, n_cand, list,
                                           reinterpret_cast<int*>(keys), sh)) {  // block keys are spent
      // done: the `take` smallest keys came from the short list
    } else if (take > 0) {
      for (int i = threadIdx.x; 4 * i < n_last; i += blockDim.x) {
        const uint4 w = explore_keys4(a.seed, (uint32_t)i, (uint32_t)q, (uint32_t)a.layer, (uint64_t)a.step);
#pragma unroll
        for (int k = 0; k < 4; ++k)
          if (4 * i + k < n_last) keys[4 * i + k] = ~word_of(w, k);
      }
      __syncthreads();
      {
        uint32_t T, eq;
        radix_select_desc(keys, n_last, cand, (uint32_t)take, sh, &T, &eq);
        // mark into a separate pass: `cand` reads m, so label after the scan
        const int chunk = (n_last + blockDim.x - 1) / blockDim.x;
        const int lo = threadIdx.x * chunk, hi = min(n_last, lo + chunk);
        int e = 0;
        for (int j = lo; j < hi; ++j)
          if (m[j] == 0 && keys[j] == T) ++e;
        int tot;
        int base = block_exclusive_scan(e, sh.scan, &tot);
        for (int j = lo; j < hi; ++j) {
          if (m[j] != 0) continue;
          if (keys[j] > T) {
            m[j] = 2;
          } else if (keys[j] == T) {
            if ((uint32_t)base < eq) m[j] = 2;
            ++base;
          }
        }
        __syncthreads();
      }
    }
  }
  for (int64_t j = n_last + threadIdx.x; j < L.max_blocks; j += blockDim.x) mask_row[j] = 0;
  compact_row(m, n_last, a.work + (int64_t)q * L.blk_stride, a.kept + q, sh.scan, mask_row,
              reinterpret_cast<int32_t*>(keys));  // the block keys are spent
}

// ---------------------------------------------------------------------------
// a2 spread over a cluster of C CTAs per request (few requests, many idle
// SMs).  Rank c owns the contiguous block range [j0_c, j1_c) of the request:
// its block keys, its part of the mask and of the kept list.  The radix
// passes merge the ranks' 256-bin histograms through distributed shared
// memory (every rank finds the same digit); keys equal to the threshold are
// taken in block order across ranks through a prefix of the ranks' counts;
// the exploration list gathers in rank 0, which marks the drawn blocks in
// their owners' masks.  Results equal the one-CTA kernel's.
// ---------------------------------------------------------------------------
struct SelCluster {
  uint32_t hist[2][256];  // this rank's histogram, double-buffered by pass
  int cnt[4];             // per-phase counts read by the other ranks
  uint32_t list_n;        // rank 0: entries of the exploration list
};

__device__ __forceinline__ int range_lo(int n, int c, int C) { return (int)((int64_t)n * c / C); }

// Radix select over the cluster's keys: this rank's keys[0 .. hi) (block
// j0 + i) with valid(i); want in [1, #valid cluster-wide].  Every rank
// returns the same T and eq.
template <class Valid>
__device__ void cl_radix_select_desc(const uint32_t* keys, int hi, Valid valid, uint32_t want, SelShared& sh,
                                     SelCluster& sc, uint32_t* T_out, uint32_t* eq_out) {
  namespace cg = cooperative_groups;
  cg::cluster_group cl = cg::this_cluster();
  const int C = (int)cl.num_blocks();
  uint32_t prefix = 0, pmask = 0, remaining = want;
  int pass = 0;
  for (int shift = 24; shift >= 0; shift -= 8, ++pass) {
    uint32_t* h = sc.hist[pass & 1];
    for (int i = threadIdx.x; i < 256; i += blockDim.x) h[i] = 0;
    __syncthreads();
    for (int i = threadIdx.x; i < hi; i += blockDim.x) {
      if (!valid(i)) continue;
      const uint32_t k = keys[i];
      if ((k & pmask) == prefix) atomicAdd(&h[(k >> shift) & 255u], 1u);
    }
    cl.sync();  // every rank's histogram of this pass is complete
    for (int b = threadIdx.x; b < 256; b += blockDim.x) {
      uint32_t t = 0;
      for (int r = 0; r < C; ++r) t += cl.map_shared_rank(h, r)[b];
      sh.hist[b] = t;
    }
    __syncthreads();
    if (threadIdx.x < 32) warp_find_digit_desc<256>(sh.hist, remaining, sh.digit);
    __syncthreads();
    prefix |= sh.digit[0] << shift;
    pmask |= 255u << shift;
    remaining = sh.digit[1];
    __syncthreads();
  }
  *T_out = prefix;
  *eq_out = remaining;
}

// Sum of `v` over the ranks below this one, and over all ranks, through
// counter slot `slot` (each slot is used once per kernel).
__device__ __forceinline__ int cl_rank_prefix(int v, int slot, SelCluster& sc, int* total) {
  namespace cg = cooperative_groups;
  cg::cluster_group cl = cg::this_cluster();
  const int C = (int)cl.num_blocks(), cr = (int)cl.block_rank();
  if (threadIdx.x == 0) sc.cnt[slot] = v;
  cl.sync();
  int below = 0, all = 0;
  for (int r = 0; r < C; ++r) {
    const int x = cl.map_shared_rank(sc.cnt, r)[slot];
    all += x;
    if (r < cr) below += x;
  }
  *total = all;
  return below;
}

// Marks m[i] = label for this rank's share of the cluster's top `want`:
// keys > T, then keys == T in block order across ranks (eq_take of them).
template <class Valid>
__device__ void cl_mark_selected(const uint32_t* keys, int hi, Valid valid, uint32_t T, uint32_t eq_take,
                                 uint8_t* m, uint8_t label, SelShared& sh, SelCluster& sc, int slot) {
  const int chunk = (hi + blockDim.x - 1) / blockDim.x;
  const int lo = threadIdx.x * chunk, up = min(hi, lo + chunk);
  int eq = 0;
  for (int i = lo; i < up; ++i)
    if (valid(i) && keys[i] == T) ++eq;
  int local_total, all;
  int base = block_exclusive_scan(eq, sh.scan, &local_total);
  base += cl_rank_prefix(local_total, slot, sc, &all);
  for (int i = lo; i < up; ++i) {
    if (!valid(i)) continue;
    const uint32_t k = keys[i];
    if (k > T) {
      m[i] = label;
    } else if (k == T) {
      if ((uint32_t)base < eq_take) m[i] = label;
      ++base;
    }
  }
  __syncthreads();
}

__global__ void __launch_bounds__(kSelThreads) k_select_cluster(StepArgs a_in) {
  pdl_enter();
  StepArgs a = a_in;
  if (a.step_dev) a.step = *a.step_dev + a.step_add;  // the state's counter (read after the predecessors finished)
  namespace cg = cooperative_groups;
  cg::cluster_group cl = cg::this_cluster();
  const int C = (int)cl.num_blocks(), cr = (int)cl.block_rank();
  const Layout L = a.lay;
  const int q = (int)(blockIdx.x / (unsigned)C);
  extern __shared__ __align__(16) uint8_t dyn[];
  uint32_t* keys = reinterpret_cast<uint32_t*>(dyn);  // this rank's range
  uint8_t* m = dyn + 4 * L.blk_stride;
  uint2* list = reinterpret_cast<uint2*>(dyn + 5 * L.blk_stride);  // rank 0: kExpCap entries
  __shared__ SelShared sh;
  __shared__ SelCluster sc;

  if (a.q8) {  // a0 on all-keep steps, the request's vectors split over the ranks
    const int nv = a.rows * L.H, warp = threadIdx.x >> 5;
    for (int i = cr * (kSelThreads / 32) + warp; i < nv; i += C * (kSelThreads / 32))
      quantize_vec(a.q, a.w, a.q_bf16, L.d, (int64_t)q * nv + i, a.q8, a.wq);
  }
  const int64_t ctx = a.ctx_len[q];
  uint8_t* mask_row = a.mask + (int64_t)q * L.max_blocks;
  if (ctx < 1 || ctx + a.rows - 1 > L.max_slots) {  // alike in every rank
    if (cr == 0 && threadIdx.x == 0) {
      if (!a.quiet) raise_error(a.err, ERR_CTX_LEN, q, (uint32_t)ctx);
      a.kept[q] = 0;
      if (a.ctx_sel) a.ctx_sel[q] = -1;
    }
    const int z0 = range_lo((int)L.max_blocks, cr, C), z1 = range_lo((int)L.max_blocks, cr + 1, C);
    for (int j = z0 + threadIdx.x; j < z1; j += blockDim.x) mask_row[j] = 0;
    return;
  }
  if (a.ctx_sel && cr == 0 && threadIdx.x == 0) a.ctx_sel[q] = (int32_t)ctx;
  const int n_last = (int)row_blocks(ctx, a.rows - 1, L.b);
  const int j0 = range_lo(n_last, cr, C), j1 = range_lo(n_last, cr + 1, C);
  const int nl = j1 - j0;  // this rank's blocks: j = j0 + i
  for (int i = threadIdx.x; i < nl; i += blockDim.x) m[i] = 0;
  if (threadIdx.x == 0) sc.list_n = 0;
  __syncthreads();

  if (a.sparsity == 0.0f) {
    for (int i = threadIdx.x; i < nl; i += blockDim.x) m[i] = 1;
    __syncthreads();
  } else {
    const int64_t n0 = row_blocks(ctx, 0, L.b);
    const int64_t n_exp = explore_count(block_budget(n0, a.sparsity), a.gamma);
    auto all = [](int) { return true; };
    for (int r = 0; r < (a.mtp_row0 ? 1 : a.rows); ++r) {
      const int n = (int)row_blocks(ctx, r, L.b);
      const int64_t n_pred = block_budget(n, a.sparsity) - n_exp;
      const int hi = max(0, min(j1, n) - j0);  // this rank's blocks visible to row r
      const float* S = a.S + ((int64_t)q * L.R + r) * L.blk_stride + j0;
      for (int i0 = 0; i0 < hi; i0 += 4 * kSelThreads) {
        float v[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int i = i0 + u * kSelThreads + (int)threadIdx.x;
          v[u] = i < hi ? S[i] : 0.f;
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int i = i0 + u * kSelThreads + (int)threadIdx.x;
          if (i < hi) keys[i] = fkey(v[u]);
        }
      }
      __syncthreads();
      if (n_pred >= n) {
        for (int i = threadIdx.x; i < hi; i += blockDim.x) m[i] = 1;
        __syncthreads();
      } else if (n_pred > 0) {
        uint32_t T, eq;
        cl_radix_select_desc(keys, hi, all, (uint32_t)n_pred, sh, sc, &T, &eq);
        cl_mark_selected(keys, hi, all, T, eq, m, 1, sh, sc, r);  // slots 0..3: one per row
      }
    }
    if (a.mtp_row0) {  // the drafts' new blocks in this rank's range
      for (int i = max(0, (int)n0 - j0) + threadIdx.x; i < nl; i += blockDim.x) m[i] = 1;
      __syncthreads();
    }
    // exploration among the unkept blocks of the last row's range
    int c = 0;
    for (int i = threadIdx.x; i < nl; i += blockDim.x) c += (m[i] == 0);
    int local_cand, n_cand;
    block_exclusive_scan(c, sh.scan, &local_cand);
    cl.sync();  // every rank's row marks are final before the counts are shared
    if (threadIdx.x == 0) sc.cnt[0] = local_cand;  // slot 0 is free again: its last reader passed the barrier
    cl.sync();
    n_cand = 0;
    for (int rr = 0; rr < C; ++rr) n_cand += cl.map_shared_rank(sc.cnt, rr)[0];
    const int64_t take = n_exp < n_cand ? n_exp : n_cand;
    if (take == n_cand) {
      for (int i = threadIdx.x; i < nl; i += blockDim.x)
        if (m[i] == 0) m[i] = 2;
      __syncthreads();
    } else if (take > 0) {
      // candidates under the Philox-key threshold go to rank 0's list
      const double frac = (1.25 * take + 64.0) / (double)n_cand;
      const uint64_t t = frac >= 1.0 ? (1ull << 32) : (uint64_t)(frac * 4294967296.0);
      uint32_t* list_n0 = &cl.map_shared_rank(&sc, 0)->list_n;
      uint2* list0 = cl.map_shared_rank(list, 0);
      const int lane = threadIdx.x & 31;
      // a thread takes the blocks 4c .. 4c+3 of one Philox call that lie in
      // this rank's range
      const int c0 = j0 >> 2, nq = ((j0 + nl + 3) >> 2) - c0;
      for (int i0 = 0; i0 < nq; i0 += blockDim.x) {  // warp-uniform trip count
        const int cq = c0 + i0 + (int)threadIdx.x;
        bool c4[4];
        bool any = false;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const int i = 4 * cq + k - j0;
          c4[k] = i0 + (int)threadIdx.x < nq && i >= 0 && i < nl && m[i] == 0;
          any |= c4[k];
        }
        const uint4 w = any ? explore_keys4(a.seed, (uint32_t)cq, (uint32_t)q, (uint32_t)a.layer, (uint64_t)a.step)
                            : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const uint32_t u = word_of(w, k);
          const bool in = c4[k] && (uint64_t)u < t;
          const uint32_t bal = __ballot_sync(0xffffffffu, in);
          if (!bal) continue;
          uint32_t at = 0;
          if (lane == 0) at = atomicAdd(list_n0, (uint32_t)__popc(bal));
          at = __shfl_sync(0xffffffffu, at, 0) + __popc(bal & ((1u << lane) - 1u));
          if (in && at < (uint32_t)kExpCap) list0[at] = make_uint2(u, (uint32_t)(4 * cq + k));
        }
      }
      cl.sync();
      const int cnt = (int)*list_n0;  // alike in every rank
      if (cnt >= take && cnt <= kExpCap) {
        if (cr == 0) {
          // the first `take` entries by (key, block), marked in their owners' masks
          draw_from_list(list, cnt, (int)take, reinterpret_cast<int*>(keys), [&](int j) {
            int owner = C - 1;
            while (owner > 0 && range_lo(n_last, owner, C) > j) --owner;
            cl.map_shared_rank(m, owner)[j - range_lo(n_last, owner, C)] = 2;
          }, sh);
        }
        cl.sync();  // the drawn blocks are marked in every owner's mask
      } else {
        // radix select over all candidates' ~keys (largest ~key = smallest key)
        for (int i = threadIdx.x; i < nl; i += blockDim.x)
          keys[i] = ~explore_key(a.seed, (uint32_t)(j0 + i), (uint32_t)q, (uint32_t)a.layer, (uint64_t)a.step);
        __syncthreads();
        auto cand = [m](int i) { return m[i] == 0; };
        uint32_t T, eq;
        cl_radix_select_desc(keys, nl, cand, (uint32_t)take, sh, sc, &T, &eq);
        // count ties first (cand reads m), then label
        const int chunk = (nl + blockDim.x - 1) / blockDim.x;
        const int lo = threadIdx.x * chunk, up = min(nl, lo + chunk);
        int e = 0;
        for (int i = lo; i < up; ++i)
          if (m[i] == 0 && keys[i] == T) ++e;
        int local_e, all_e;
        int base = block_exclusive_scan(e, sh.scan, &local_e);
        base += cl_rank_prefix(local_e, 1, sc, &all_e);  // slot 1: its row-1 use is behind two barriers
        for (int i = lo; i < up; ++i) {
          if (m[i] != 0) continue;
          if (keys[i] > T) {
            m[i] = 2;
          } else if (keys[i] == T) {
            if ((uint32_t)base < eq) m[i] = 2;
            ++base;
          }
        }
        __syncthreads();
      }
    }
  }
  // mask row and the ascending kept list, each rank its own range
  for (int i = threadIdx.x; i < nl; i += blockDim.x) mask_row[j0 + i] = m[i];
  if (cr == C - 1)
    for (int64_t j = n_last + threadIdx.x; j < L.max_blocks; j += blockDim.x) mask_row[j] = 0;
  const int chunk = (nl + blockDim.x - 1) / blockDim.x;
  const int lo = threadIdx.x * chunk, up = min(nl, lo + chunk);
  int kc = 0;
  for (int i = lo; i < up; ++i) kc += m[i] != 0;
  int local_kept, total_kept;
  int pos = block_exclusive_scan(kc, sh.scan, &local_kept);
  cl.sync();  // slot 2 / 3 readers of earlier phases are done
  const int base = cl_rank_prefix(local_kept, 2, sc, &total_kept);
  // this rank's part of the list staged in shared memory (the block keys are
  // spent), then stored coalesced
  int32_t* stage = reinterpret_cast<int32_t*>(keys);
  for (int i = lo; i < up; ++i)
    if (m[i]) stage[pos++] = j0 + i;
  __syncthreads();
  int32_t* work = a.work + (int64_t)q * L.blk_stride + base;
  for (int i = threadIdx.x; i < local_kept; i += blockDim.x) work[i] = stage[i];
  if (cr == 0 && threadIdx.x == 0) a.kept[q] = total_kept;
  cl.sync();  // no rank leaves while another may still read its counters
}

cudaError_t launch_select(const StepArgs& a, cudaStream_t s) {
  static_assert(kExpCap * sizeof(uint2) == 2048 * 8, "select_smem counts kExpCap entries");
  const size_t smem = select_smem(a.lay.blk_stride, a.mtp_row0 ? 1 : a.rows);
  cudaError_t e = cudaFuncSetAttribute(k_select<0>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e == cudaSuccess) e = cudaFuncSetAttribute(k_select<1>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e == cudaSuccess) e = cudaFuncSetAttribute(k_select<4>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(k_select<1, true>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e == cudaSuccess) e = cudaFuncSetAttribute(k_select_cluster, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  if (a.nl > 1) {  // several layers of one-row steps: one CTA per (layer, request)
    if (a.nl > kMaxLayerBatch || a.rows != 1 || a.mtp_row0) return cudaErrorInvalidValue;
    PdlLaunch l(dim3(a.lay.Q, 1, a.nl), dim3(kSelThreads), smem, s);
    l.attr[0].val.programmaticStreamSerializationAllowed = a.no_pdl ? 0 : 1;
    return cudaLaunchKernelEx(&l.cfg, k_select<1, true>, a);
  }
  // Few requests with long contexts leave most SMs idle: a cluster of up to 8
  // CTAs per request, each keeping >= 2048 blocks (below that the cluster
  // barriers cost more than the split saves).  A cluster shape the device
  // cannot place falls back to one CTA each.
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  int C = 1;
  while (C < 8 && a.lay.Q * C * 2 <= sms && a.lay.max_blocks >= (int64_t)C * 2 * 2048) C *= 2;
  if (C > 1) {
    PdlLaunch l(dim3(a.lay.Q * C), dim3(kSelThreads), smem, s);
    l.attr[0].val.programmaticStreamSerializationAllowed = a.no_pdl ? 0 : 1;
    l.attr[1].id = cudaLaunchAttributeClusterDimension;
    l.attr[1].val.clusterDim.x = (unsigned)C;
    l.attr[1].val.clusterDim.y = 1;
    l.attr[1].val.clusterDim.z = 1;
    l.cfg.numAttrs = 2;
    int clusters = 0;
    e = cudaOccupancyMaxActiveClusters(&clusters, k_select_cluster, &l.cfg);
    if (e == cudaSuccess && clusters >= 1) return cudaLaunchKernelEx(&l.cfg, k_select_cluster, a);
    cudaGetLastError();  // this shape cannot be placed
  }
  PdlLaunch l(dim3(a.lay.Q), dim3(kSelThreads), smem, s);
  l.attr[0].val.programmaticStreamSerializationAllowed = a.no_pdl ? 0 : 1;
  return cudaLaunchKernelEx(&l.cfg, a.rows == 1 ? k_select<1> : a.rows == 4 ? k_select<4> : k_select<0>, a);
}

// ---------------------------------------------------------------------------
// Compaction of a caller-given mask into the work list (standalone score /
// top-k calls).  One CTA per request.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(1024) k_compact(Layout L, int rows, const int32_t* ctx_len,
                                                  const uint8_t* mask, int32_t* work, int32_t* kept,
                                                  ErrWord* err) {
  __shared__ int scan[33];
  const int q = blockIdx.x;
  const int64_t ctx = ctx_len[q];
  if (ctx < 1 || ctx + rows - 1 > L.max_slots) {
    if (threadIdx.x == 0) {
      raise_error(err, ERR_CTX_LEN, q, (uint32_t)ctx);
      kept[q] = 0;
    }
    return;
  }
  const int n_last = (int)row_blocks(ctx, rows - 1, L.b);
  compact_row(mask + (int64_t)q * L.max_blocks, n_last, work + (int64_t)q * L.blk_stride, kept + q, scan);
}

cudaError_t launch_compact(const Layout& L, int rows, const int32_t* ctx_len, const uint8_t* mask,
                           int32_t* work, int32_t* kept, ErrWord* err, cudaStream_t s) {
  k_compact<<<L.Q, 1024, 0, s>>>(L, rows, ctx_len, mask, work, kept, err);
  return cudaGetLastError();
}

}  // namespace spin
