// k_quality.cu -- predictor-quality profile: how well a slot-level prediction
// of the indexer's scores matches the scores themselves, by Pearson
// correlation and by top-k recall (SPIN listing, Table 1, which profiles a
// random baseline, the previous layer's and the previous iteration's scores).
//
//   k_slot_prediction  one predictor's value per visible slot: the SPIN
//                      predictor before block pooling, z = max(V_s, D_{p_r-s})
//                      (-inf where z is not finite: a slot never scored), or
//                      the random baseline (uniform [0, 1) from Philox).
//   k_pearson          per (request, row), in double, two passes over the
//                      slots where both values are finite: means, then the
//                      centred sums.  One CTA per (request, row); the sums run
//                      in a fixed order, so the result does not depend on the
//                      launch.
//   k_topk_overlap     per (request, row), the slots two ascending top-k lists
//                      share (the recall's numerator).
//
// These kernels serve measurement, not the decode step: each streams its
// inputs once (k_pearson twice) with coalesced loads.
#include <algorithm>

#include "spin_internal.cuh"

namespace spin {

__global__ void __launch_bounds__(256) k_slot_prediction(Layout L, int rows, int kind, int64_t step,
                                                         const int64_t* step_dev, uint64_t seed, int layer,
                                                         const int32_t* ctx_len, const float* V, const float* D,
                                                         float* pred, ErrWord* err) {
  pdl_enter();
  if (step_dev) step = *step_dev;
  const int64_t chunks = (L.slot_stride + 255) / 256;
  const int64_t n = (int64_t)L.Q * rows * chunks;
  for (int64_t t = blockIdx.x; t < n; t += gridDim.x) {
    const int64_t c = t % chunks;
    const int r = (int)((t / chunks) % rows);
    const int q = (int)(t / (chunks * rows));
    const int64_t ctx = ctx_len[q];
    if (ctx < 1 || ctx + rows - 1 > L.max_slots) {
      if (c == 0 && r == 0 && threadIdx.x == 0) raise_error(err, ERR_CTX_LEN, q, (uint32_t)ctx);
      continue;
    }
    const int64_t p = row_pos(ctx, r);
    const int64_t s = c * 256 + threadIdx.x;
    if (s > p) continue;
    float v;
    if (kind == SPIN_PRED_EMA) {
      const float z = fmaxf(V[(int64_t)q * L.slot_stride + s], D[(int64_t)q * L.slot_stride + (p - s)]);
      v = isfinite(z) ? z : __int_as_float(0xff800000);
    } else {
      const uint32_t w = explore_key(seed, (uint32_t)s, (uint32_t)q, (uint32_t)layer, (uint64_t)step);
      v = (float)(w >> 8) * 5.9604644775390625e-08f;  // 2^-24: exact
    }
    pred[((int64_t)q * L.R + r) * L.slot_stride + s] = v;
  }
}

// Block-wide sums of up to three doubles in a fixed order (warp tree, then
// the warps in order by thread 0); every thread gets the totals.
template <int N>
__device__ void block_sum(double (&v)[N], double (*red)[32]) {
#pragma unroll
  for (int i = 0; i < N; ++i)
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) v[i] += __shfl_xor_sync(0xffffffffu, v[i], o);
  const int w = threadIdx.x >> 5, nw = blockDim.x >> 5;
  if ((threadIdx.x & 31) == 0)
#pragma unroll
    for (int i = 0; i < N; ++i) red[i][w] = v[i];
  __syncthreads();
  if (threadIdx.x == 0)
#pragma unroll
    for (int i = 0; i < N; ++i) {
      double t = 0.0;
      for (int k = 0; k < nw; ++k) t += red[i][k];
      red[i][0] = t;
    }
  __syncthreads();
#pragma unroll
  for (int i = 0; i < N; ++i) v[i] = red[i][0];
  __syncthreads();
}

constexpr int kPearsonThreads = 1024;

__global__ void __launch_bounds__(kPearsonThreads) k_pearson(Layout L, int rows, const float* x, const float* y,
                                                             const int32_t* ctx_len, double* out, ErrWord* err) {
  pdl_enter();
  const int q = blockIdx.x / rows, r = blockIdx.x % rows;
  __shared__ double red[3][32];
  const int64_t ctx = ctx_len[q];
  if (ctx < 1 || ctx + rows - 1 > L.max_slots) {
    if (threadIdx.x == 0) {
      if (r == 0) raise_error(err, ERR_CTX_LEN, q, (uint32_t)ctx);
      out[blockIdx.x] = 0.0;
    }
    return;
  }
  const int64_t n = row_pos(ctx, r) + 1;
  const float* xr = x + ((int64_t)q * L.R + r) * L.slot_stride;
  const float* yr = y + ((int64_t)q * L.R + r) * L.slot_stride;
  double a[3] = {0.0, 0.0, 0.0};  // count, sum x, sum y
  for (int64_t i0 = 0; i0 < n; i0 += 4 * kPearsonThreads) {
    float xv[4], yv[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {  // four loads of each in flight
      const int64_t i = i0 + u * kPearsonThreads + threadIdx.x;
      xv[u] = i < n ? xr[i] : 0.f;
      yv[u] = i < n ? yr[i] : 0.f;
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int64_t i = i0 + u * kPearsonThreads + threadIdx.x;
      if (i < n && isfinite(xv[u]) && isfinite(yv[u])) {
        a[0] += 1.0;
        a[1] += (double)xv[u];
        a[2] += (double)yv[u];
      }
    }
  }
  block_sum(a, red);
  if (a[0] < 2.0) {
    if (threadIdx.x == 0) out[blockIdx.x] = 0.0;
    return;
  }
  const double mx = a[1] / a[0], my = a[2] / a[0];
  double c[3] = {0.0, 0.0, 0.0};  // sxy, sxx, syy
  for (int64_t i0 = 0; i0 < n; i0 += 4 * kPearsonThreads) {
    float xv[4], yv[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int64_t i = i0 + u * kPearsonThreads + threadIdx.x;
      xv[u] = i < n ? xr[i] : 0.f;
      yv[u] = i < n ? yr[i] : 0.f;
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int64_t i = i0 + u * kPearsonThreads + threadIdx.x;
      if (i < n && isfinite(xv[u]) && isfinite(yv[u])) {
        const double dx = (double)xv[u] - mx, dy = (double)yv[u] - my;
        c[0] = fma(dx, dy, c[0]);
        c[1] = fma(dx, dx, c[1]);
        c[2] = fma(dy, dy, c[2]);
      }
    }
  }
  block_sum(c, red);
  if (threadIdx.x == 0) out[blockIdx.x] = (c[1] == 0.0 || c[2] == 0.0) ? 0.0 : c[0] / sqrt(c[1] * c[2]);
}

// One warp per (request, row): each lane looks its entries of list a up in
// list b by binary search over b's valid prefix (ascending, -1 padded).
__global__ void __launch_bounds__(256) k_topk_overlap(int pairs, int k, const int32_t* a, const int32_t* b,
                                                      int32_t* out) {
  pdl_enter();
  const int lane = threadIdx.x & 31;
  const int pair = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (pair >= pairs) return;  // warp-uniform
  const int32_t* ar = a + (int64_t)pair * k;
  const int32_t* br = b + (int64_t)pair * k;
  int nb = 0;
  for (int i = lane; i < k; i += 32) nb += br[i] >= 0;
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) nb += __shfl_xor_sync(0xffffffffu, nb, o);
  int hits = 0;
  for (int i = lane; i < k; i += 32) {
    const int32_t s = ar[i];
    if (s < 0) continue;
    int lo = 0, hi = nb;  // first index with br[idx] >= s
    while (lo < hi) {
      const int mid = (lo + hi) >> 1;
      if (br[mid] < s) lo = mid + 1; else hi = mid;
    }
    hits += lo < nb && br[lo] == s;
  }
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) hits += __shfl_xor_sync(0xffffffffu, hits, o);
  if (lane == 0) out[pair] = hits;
}

cudaError_t launch_slot_prediction(const Layout& L, int rows, int kind, int64_t step, const int64_t* step_dev,
                                   uint64_t seed, int layer, const int32_t* ctx_len, const float* V, const float* D,
                                   float* pred, ErrWord* err, cudaStream_t s) {
  const int64_t n = (int64_t)L.Q * rows * ((L.slot_stride + 255) / 256);
  PdlLaunch l(dim3((unsigned)std::min<int64_t>(n, 148 * 16)), dim3(256), 0, s);
  return cudaLaunchKernelEx(&l.cfg, k_slot_prediction, L, rows, kind, step, step_dev, seed, layer, ctx_len, V, D,
                            pred, err);
}

cudaError_t launch_pearson(const Layout& L, int rows, const float* x, const float* y, const int32_t* ctx_len,
                           double* out, ErrWord* err, cudaStream_t s) {
  PdlLaunch l(dim3((unsigned)(L.Q * rows)), dim3(kPearsonThreads), 0, s);
  return cudaLaunchKernelEx(&l.cfg, k_pearson, L, rows, x, y, ctx_len, out, err);
}

cudaError_t launch_topk_overlap(int pairs, int k, const int32_t* a, const int32_t* b, int32_t* out, cudaStream_t s) {
  PdlLaunch l(dim3((unsigned)((pairs + 7) / 8)), dim3(256), 0, s);
  return cudaLaunchKernelEx(&l.cfg, k_topk_overlap, pairs, k, a, b, out);
}

}  // namespace spin
