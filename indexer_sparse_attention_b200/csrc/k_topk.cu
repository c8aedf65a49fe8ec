// k_topk.cu -- a4 token top-k over the scored slots (SPIN digest,
// arXiv深度剖析: SPIN leaves the fixed top-k budget of core attention as it
// is).  Order: higher score first, ties to the lower slot; the chosen slots
// are emitted in ascending slot order, padded with -1.
//
// One CTA (1024 threads) per (request, row).  Three MSB-first radix passes
// (11 + 11 + 10 bits of the order-preserving key) over the scored slots find
// the exact threshold key T and how many slots equal to T belong to the top
// k.  A fourth pass marks every slot with key >= T in a shared-memory bitmap
// indexed by position in the ascending kept-slot order; two block scans over
// the bitmap then take the lowest-index ties and give each chosen slot its
// output position, so the output is ascending without a sort.
#include "spin_internal.cuh"
#include "block_scan.cuh"

namespace spin {

constexpr int kTopkThreads = 1024;

struct TopkShared {
  uint32_t hist[2048];
  uint32_t digit[2];
  int scan[33];
  int total;
};

template <class F>
__device__ __forceinline__ void for_each_scored(const float* sc, const int32_t* work, int nk, int b,
                                                int64_t p, F f) {
  const int64_t n_elem = (int64_t)nk * b;
  for (int64_t e = (int64_t)threadIdx.x * 4; e < n_elem; e += (int64_t)blockDim.x * 4) {
    const int64_t j = work[e / b];
    const int64_t s = j * b + (e % b);
    if (s > p) continue;
    const float4 v = *reinterpret_cast<const float4*>(sc + s);
    f(e, s, fkey(v.x));
    if (s + 1 <= p) f(e + 1, s + 1, fkey(v.y));
    if (s + 2 <= p) f(e + 2, s + 2, fkey(v.z));
    if (s + 3 <= p) f(e + 3, s + 3, fkey(v.w));
  }
}

__global__ void __launch_bounds__(kTopkThreads) k_topk(TopkArgs a) {
  const Layout L = a.lay;
  const int q = blockIdx.x / a.rows, r = blockIdx.x % a.rows;
  int32_t* out = a.topk + ((int64_t)q * a.rows + r) * L.k;
  __shared__ TopkShared sh;
  extern __shared__ uint32_t bits[];
  const int64_t ctx = a.ctx_len[q];
  if (ctx < 1 || ctx + a.rows - 1 > L.max_slots) {
    for (int t = threadIdx.x; t < L.k; t += blockDim.x) out[t] = -1;
    return;
  }
  const int64_t p = ctx - 1 + r;
  const int nk = a.kept[q];
  const int32_t* work = a.work + (int64_t)q * L.blk_stride;
  const float* sc = a.scores + ((int64_t)q * L.R + r) * L.slot_stride;

  // ---- radix passes -------------------------------------------------------
  uint32_t prefix = 0, remaining = 0;
  int shift_hi = 32;
  const int shifts[3] = {21, 10, 0};
  for (int pass = 0; pass < 3; ++pass) {
    const int sh_lo = shifts[pass];
    const int width = shift_hi - sh_lo;
    const uint32_t dmask = (1u << width) - 1u;
    for (int i = threadIdx.x; i < 2048; i += blockDim.x) sh.hist[i] = 0;
    __syncthreads();
    for_each_scored(sc, work, nk, L.b, p, [&](int64_t, int64_t, uint32_t key) {
      const bool match = (shift_hi == 32) || ((key >> shift_hi) == prefix);
      if (match) atomicAdd(&sh.hist[(key >> sh_lo) & dmask], 1u);
    });
    __syncthreads();
    if (pass == 0) {
      // total scored and the rank wanted
      int c = 0;
      for (int i = threadIdx.x; i < 2048; i += blockDim.x) c += sh.hist[i];
      int tot;
      block_exclusive_scan(c, sh.scan, &tot);
      if (threadIdx.x == 0) sh.total = tot;
      __syncthreads();
      remaining = (uint32_t)min(sh.total, L.k);
      if (remaining == 0) break;
    }
    if (threadIdx.x < 32) {
      if (width == 11) warp_find_digit_desc<2048>(sh.hist, remaining, sh.digit);
      else warp_find_digit_desc<1024>(sh.hist, remaining, sh.digit);
    }
    __syncthreads();
    prefix = (prefix << width) | sh.digit[0];
    remaining = sh.digit[1];
    shift_hi = sh_lo;
    __syncthreads();
  }
  const int want = min(sh.total, L.k);
  if (want == 0) {
    for (int t = threadIdx.x; t < L.k; t += blockDim.x) out[t] = -1;
    return;
  }
  const uint32_t T = prefix;
  const uint32_t eq_take = remaining;

  // ---- bitmap of keys >= T in kept-slot order -----------------------------
  const int64_t n_elem = (int64_t)nk * L.b;
  const int nwords = (int)((n_elem + 31) / 32);
  for (int i = threadIdx.x; i < nwords; i += blockDim.x) bits[i] = 0;
  __syncthreads();
  for_each_scored(sc, work, nk, L.b, p, [&](int64_t e, int64_t, uint32_t key) {
    if (key >= T) atomicOr(&bits[e >> 5], 1u << (e & 31));
  });
  __syncthreads();

  // ---- ordered tie handling and emission -----------------------------------
  const int chunk = (nwords + blockDim.x - 1) / blockDim.x;
  const int w0 = threadIdx.x * chunk, w1 = min(nwords, w0 + chunk);
  int n_gt = 0, n_eq = 0;
  for (int w = w0; w < w1; ++w) {
    uint32_t m = bits[w];
    while (m) {
      const int bit = __ffs(m) - 1;
      m &= m - 1;
      const int64_t e = (int64_t)w * 32 + bit;
      const int64_t s = (int64_t)work[e / L.b] * L.b + (e % L.b);
      if (fkey(sc[s]) > T) ++n_gt; else ++n_eq;
    }
  }
  int tot;
  const int eq_base = block_exclusive_scan(n_eq, sh.scan, &tot);
  const int take = max(0, min(n_eq, (int)eq_take - eq_base));
  int pos = block_exclusive_scan(n_gt + take, sh.scan, &tot);
  int eq_rank = eq_base;
  for (int w = w0; w < w1; ++w) {
    uint32_t m = bits[w];
    while (m) {
      const int bit = __ffs(m) - 1;
      m &= m - 1;
      const int64_t e = (int64_t)w * 32 + bit;
      const int64_t s = (int64_t)work[e / L.b] * L.b + (e % L.b);
      if (fkey(sc[s]) > T) {
        out[pos++] = (int32_t)s;
      } else {
        if ((uint32_t)eq_rank < eq_take) out[pos++] = (int32_t)s;
        ++eq_rank;
      }
    }
  }
  for (int t = want + threadIdx.x; t < L.k; t += blockDim.x) out[t] = -1;
}

cudaError_t launch_topk(const TopkArgs& a, cudaStream_t s) {
  const size_t smem = (size_t)((a.lay.slot_stride + 31) / 32) * 4;
  cudaError_t e = cudaFuncSetAttribute(k_topk, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  k_topk<<<a.lay.Q * a.rows, kTopkThreads, smem, s>>>(a);
  return cudaGetLastError();
}

}  // namespace spin
