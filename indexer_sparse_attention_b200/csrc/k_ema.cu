// k_ema.cu -- a5 EMA update, state initialisation and the miss counter.
//
// a5: only slots that were scored update the state (SPIN digest, 核心概要 and
//     arXiv深度剖析; AI Radio episode, "The paper's summary": skipped blocks get
//     no update).  V_s and D_{p_r - s} move toward the observed score I_{r,s}:
//     x <- I if x is the never-observed sentinel (V: +inf, D: -inf), else
//     fmaf(alpha, x, beta * I), beta = fl32(1 - alpha).  For speculative rows
//     the update waits for the accepted length a and replays rows 0..a-1 in
//     order (SPIN digest, arXiv深度剖析: prefix-valid replay); under the
//     row-0 MTP policy row 0 alone is applied (SPIN listing, Table 7).
//
// Parallel layout: one warp per block j of a request at a time.  The vertical state of
// a slot is owned by the slot (its rows run in order inside one thread); the
// diagonal state D_delta is owned by the block of row 0's slot
// s_0 = p_0 - delta, and its rows r = 0..a-1 (slot s_0 + r) run in order
// inside one thread.  Offsets delta > p_0 (only later rows see them) belong to
// block 0.  Every (row, slot) pair is applied exactly once, in row order.
//
// Group maxima of V: where the state keeps vmax[g] = max(V[32 g .. 32 g + 31])
// (the max-pooled prediction reads them in place of V: max over a block of
// max(V_i, D_{p-i}) is the max of V's maximum and D's), every writer of V
// brings the groups it wrote up to date: the replay kernel from the values in
// its registers, the fills with +inf, k_vmax_refresh after a bulk write.
#include <algorithm>

#include "spin_internal.cuh"

namespace spin {

__global__ void k_fill(float* V, float* D, int64_t n, float* vmax, int64_t nv) {
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
    V[i] = __int_as_float(0x7f800000);
    D[i] = __int_as_float(0xff800000);
  }
  if (vmax)
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < nv; i += (int64_t)gridDim.x * blockDim.x)
      vmax[i] = __int_as_float(0x7f800000);
}

cudaError_t launch_init_state(float* V, float* D, int64_t n, float* vmax, int64_t nv, cudaStream_t s) {
  int64_t blocks = (n + 255) / 256;
  if (blocks > 148 * 32) blocks = 148 * 32;
  if (blocks < 1) blocks = 1;
  k_fill<<<(int)blocks, 256, 0, s>>>(V, D, n, vmax, nv);
  return cudaGetLastError();
}

// One warp per 32-slot group: a coalesced 128-byte row of V and a warp max.
__global__ void __launch_bounds__(256) k_vmax_refresh(const float* V, float* vmax, int64_t rows, int64_t slot_stride,
                                                      int64_t vg_stride) {
  const int lane = threadIdx.x & 31;
  const int64_t groups = rows * vg_stride;
  const int64_t warps = (int64_t)gridDim.x * (blockDim.x >> 5);
  for (int64_t g = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); g < groups; g += warps) {
    const int64_t row = g / vg_stride, c = g - row * vg_stride;
    const float x = warp_max(V[row * slot_stride + c * 32 + lane]);
    if (lane == 0) vmax[g] = x;
  }
}

cudaError_t launch_vmax_refresh(const float* V, float* vmax, int64_t rows, int64_t slot_stride, int64_t vg_stride,
                                cudaStream_t s) {
  if (!vmax || rows < 1 || vg_stride < 1) return cudaSuccess;
  int64_t blocks = (rows * vg_stride + 7) / 8;
  if (blocks > 148 * 16) blocks = 148 * 16;
  k_vmax_refresh<<<(int)blocks, 256, 0, s>>>(V, vmax, rows, slot_stride, vg_stride);
  return cudaGetLastError();
}

__global__ void k_step_op(int64_t* p, int set, int64_t value) { *p = set ? value : *p + 1; }

cudaError_t launch_step_op(int64_t* p, bool set, int64_t value, cudaStream_t s) {
  k_step_op<<<1, 1, 0, s>>>(p, set ? 1 : 0, value);
  return cudaGetLastError();
}

__global__ void k_reset_rows(float* V, float* D, float* vmax, ReqList list, int64_t stride, int64_t vg_stride) {
  for (int k = blockIdx.y; k < list.n; k += gridDim.y) {
    const int64_t base = (int64_t)list.ids[k] * stride;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < stride; i += (int64_t)gridDim.x * blockDim.x) {
      V[base + i] = __int_as_float(0x7f800000);
      D[base + i] = __int_as_float(0xff800000);
    }
    if (vmax) {
      const int64_t vb = (int64_t)list.ids[k] * vg_stride;
      for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < vg_stride;
           i += (int64_t)gridDim.x * blockDim.x)
        vmax[vb + i] = __int_as_float(0x7f800000);
    }
  }
}

cudaError_t launch_reset_rows(float* V, float* D, float* vmax, const ReqList& list, int64_t stride,
                              int64_t vg_stride, cudaStream_t s) {
  dim3 grid((unsigned)std::min<int64_t>((stride + 255) / 256, 1024), (unsigned)list.n);
  k_reset_rows<<<grid, 256, 0, s>>>(V, D, vmax, list, stride, vg_stride);
  return cudaGetLastError();
}

// R: the most rows one update applies (the call's rows, or 1 under the row-0
// policy); a.rows, the call's rows, bounds the context and accepted lengths.
// Grid: column x = request, its gridDim.y blocks' warps take the request's
// blocks j in turn (no division per block).
template <int R>
__global__ void __launch_bounds__(256, 4) k_ema_update(EmaArgs a) {
  pdl_enter();
  const Layout L = a.lay;
  const int lane = threadIdx.x & 31;
  const int q = blockIdx.x;
  const int64_t ctx = a.ctx_len[q];
  if (ctx < 1 || ctx + a.rows - 1 > L.max_slots) return;  // block-uniform
  int acc = R;
  if (a.accepted) {
    acc = a.accepted[q];
    if (acc < 1 || acc > a.rows) {
      if (blockIdx.y == 0 && threadIdx.x == 0) raise_error(a.err, ERR_ACCEPTED, q, (uint32_t)acc);
      return;
    }
    acc = min(acc, R);
  }
  const int64_t p0 = ctx - 1;
  const int64_t n_last = row_blocks(ctx, acc - 1, L.b);
  const int lb = __ffs(L.b) - 1;  // the block size is a power of two
  const int wpr = (int)gridDim.y * (blockDim.x >> 5);
  const int64_t j_first = (int64_t)blockIdx.y * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const uint8_t* mask = a.mask + (int64_t)q * L.max_blocks;
  // The warp's blocks j_first + t wpr, 32 at a time: lane t reads the mask of
  // block t (and of the next block), so the blocks to update are known
  // before the first one is loaded.
  for (int64_t jb = j_first; jb < n_last; jb += 32 * (int64_t)wpr) {
    const int64_t jl = jb + (int64_t)lane * wpr;
    const bool ml = jl < n_last && mask[jl] != 0;
    const bool ml1 = (R > 1) && jl + 1 < n_last && mask[jl + 1] != 0;
    const uint32_t bk = __ballot_sync(0xffffffffu, ml), bk1 = __ballot_sync(0xffffffffu, ml1);
    uint32_t todo = bk | bk1 | ((R > 1 && jb == 0) ? 1u : 0u);  // block 0 holds the offsets past p0
    while (todo) {
      const int t = __ffs(todo) - 1;
      todo &= todo - 1;
      const int64_t j = jb + (int64_t)t * wpr;
      const bool kj = (bk >> t) & 1u;
      const bool kj1 = (bk1 >> t) & 1u;
      float* V = a.V + (int64_t)q * L.slot_stride;
      float* D = a.D + (int64_t)q * L.slot_stride;
      const float* sc = a.scores + (int64_t)q * L.R * L.slot_stride;
      if (R > 1 && L.b == 64 && j > 0 && kj && kj1 && (j + 1) * 64 - 1 <= p0) {
        // A kept block (not block 0) below p0 whose successor is kept too:
        // every accepted row updates V and D of every slot, so only r < acc
        // (uniform) is tested.  Two slots per lane; offsets in 32 bits.
        const int s0 = (int)(j * 64) + lane, p = (int)p0;
        float v[2], dv[2], sv[2][R], sd[2][R];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          v[h] = V[s0 + 32 * h];
          dv[h] = D[p - (s0 + 32 * h)];
#pragma unroll
          for (int r = 0; r < R; ++r) {
            const float* sr = sc + (int64_t)r * L.slot_stride;
            sv[h][r] = r < acc ? sr[s0 + 32 * h] : 0.f;
            sd[h][r] = r < acc ? sr[s0 + 32 * h + r] : 0.f;
          }
        }
#pragma unroll
        for (int h = 0; h < 2; ++h) {
#pragma unroll
          for (int r = 0; r < R; ++r) {  // rows in order
            if (r < acc) {
              v[h] = ema_v(v[h], sv[h][r], a.alpha, a.beta);
              dv[h] = ema_d(dv[h], sd[h][r], a.alpha, a.beta);
            }
          }
          V[s0 + 32 * h] = v[h];
          D[p - (s0 + 32 * h)] = dv[h];
        }
        if (a.vmax) {
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const float g = warp_max(v[h]);
            if (lane == 0) a.vmax[(int64_t)q * L.vg_stride + ((s0 - lane + 32 * h) >> 5)] = g;
          }
        }
        continue;  // (block 0, which also holds the offsets past p0, takes the general path)
      }
      // Two slots per lane per pass (i, i + 32): every load of the pass is
      // issued before the first store, so the pass costs one memory latency.
      for (int i0 = lane; i0 < L.b; i0 += 64) {
        float v[2], dv[2], sv[2][R], sd[2][R];
        bool do_v[2], do_d[2], use_v[2][R], use_d[2][R];
        int64_t sl[2];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int i = i0 + 32 * h;
          sl[h] = j * L.b + i;
          const int64_t s = sl[h];
          do_v[h] = i < L.b && kj;                         // vertical state of slot s
          do_d[h] = i < L.b && s <= p0 && (kj || kj1);     // diagonal state delta = p0 - s
          v[h] = do_v[h] ? V[s] : 0.f;
          dv[h] = do_d[h] ? D[p0 - s] : 0.f;
#pragma unroll
          for (int r = 0; r < R; ++r) {
            use_v[h][r] = do_v[h] && r < acc && s <= p0 + r;
            const int64_t sr = s + r;  // row r's slot for delta: in block j, or past its end in block j + 1
            use_d[h][r] = do_d[h] && r < acc && (((sr >> lb) == j) ? kj : kj1);
            sv[h][r] = use_v[h][r] ? sc[(int64_t)r * L.slot_stride + s] : 0.f;
            sd[h][r] = use_d[h][r] ? sc[(int64_t)r * L.slot_stride + sr] : 0.f;
          }
        }
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          bool tv = false, td = false;
#pragma unroll
          for (int r = 0; r < R; ++r) {  // rows in order
            if (use_v[h][r]) {
              v[h] = ema_v(v[h], sv[h][r], a.alpha, a.beta);
              tv = true;
            }
            if (use_d[h][r]) {
              dv[h] = ema_d(dv[h], sd[h][r], a.alpha, a.beta);
              td = true;
            }
          }
          if (tv) V[sl[h]] = v[h];
          if (td) D[p0 - sl[h]] = dv[h];
        }
        // a kept block's 32-slot groups: every lane holds its slot's V, new or
        // not (vmax is kept only for b >= 32, so the whole warp is here)
        if (a.vmax && kj) {
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            if (i0 - lane + 32 * h < L.b) {  // warp-uniform
              const float g = warp_max(v[h]);
              if (lane == 0) a.vmax[(int64_t)q * L.vg_stride + (sl[h] >> 5)] = g;
            }
          }
        }
      }
      // offsets delta = p0 + m (m >= 1): seen only by rows r >= m at slot r - m
      if (R > 1 && j == 0 && lane < R - 1) {
        const int m = lane + 1;
        const int64_t dlt = p0 + m;
        float dv = D[dlt];
        bool touched = false;
#pragma unroll
        for (int r = 0; r < R; ++r) {
          if (r >= m && r < acc) {
            const int64_t sr = r - m;  // in block 0 (r < R <= 4 < b)
            if (kj) {
              dv = ema_d(dv, sc[(int64_t)r * L.slot_stride + sr], a.alpha, a.beta);
              touched = true;
            }
          }
        }
        if (touched) D[dlt] = dv;
      }
    }
  }
}

cudaError_t launch_ema_update(const EmaArgs& a, cudaStream_t s) {
  // about 8 blocks of 256 threads per SM over all requests
  int64_t gy = (148 * 8 + a.lay.Q - 1) / a.lay.Q;
  gy = std::min<int64_t>(gy, (a.lay.max_blocks + 7) / 8);
  gy = std::max<int64_t>(std::min<int64_t>(gy, 65535), 1);
  PdlLaunch l(dim3((unsigned)a.lay.Q, (unsigned)gy), dim3(256), 0, s);
  switch (a.row0 ? 1 : a.rows) {
    case 1: return cudaLaunchKernelEx(&l.cfg, k_ema_update<1>, a);
    case 2: return cudaLaunchKernelEx(&l.cfg, k_ema_update<2>, a);
    case 3: return cudaLaunchKernelEx(&l.cfg, k_ema_update<3>, a);
    default: return cudaLaunchKernelEx(&l.cfg, k_ema_update<4>, a);
  }
}

// Miss counter of the fidelity metric: per (request, row), the entries of a
// full-indexer top-k whose block is skipped (SPIN listing, Table 5 caption).
__global__ void k_miss_count(Layout L, int rows, const int32_t* topk, const uint8_t* mask,
                             int32_t* missed, int32_t* total) {
  const int q = blockIdx.x / rows;
  const int32_t* t = topk + (int64_t)blockIdx.x * L.k;
  const uint8_t* m = mask + (int64_t)q * L.max_blocks;
  int mc = 0, tc = 0;
  for (int i = threadIdx.x; i < L.k; i += blockDim.x) {
    const int32_t s = t[i];
    if (s < 0) continue;
    ++tc;
    const int64_t j = s / L.b;
    if (j >= L.max_blocks || m[j] == 0) ++mc;
  }
  __shared__ int red[2][32];
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) {
    mc += __shfl_xor_sync(0xffffffffu, mc, o);
    tc += __shfl_xor_sync(0xffffffffu, tc, o);
  }
  if ((threadIdx.x & 31) == 0) {
    red[0][threadIdx.x >> 5] = mc;
    red[1][threadIdx.x >> 5] = tc;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    int a = 0, b = 0;
    for (int w = 0; w < (int)(blockDim.x >> 5); ++w) { a += red[0][w]; b += red[1][w]; }
    missed[blockIdx.x] = a;
    total[blockIdx.x] = b;
  }
}

cudaError_t launch_miss_count(const Layout& L, int rows, const int32_t* full_topk,
                              const uint8_t* mask, int32_t* missed, int32_t* total, cudaStream_t s) {
  k_miss_count<<<L.Q * rows, 256, 0, s>>>(L, rows, full_topk, mask, missed, total);
  return cudaGetLastError();
}

}  // namespace spin
