// k_topk.cu -- a4 token top-k over the scored slots (SPIN digest,
// arXiv深度剖析: SPIN leaves the fixed top-k budget of core attention as it
// is).  Order: higher score first, ties to the lower slot; the chosen slots
// are emitted in ascending slot order, padded with -1.
//
// One CTA (1024 threads) per (request, row).
//  1. A 13-bit histogram of the order-preserving score keys (sign, exponent
//     and 4 mantissa bits) over a fixed 1/16 sample of the scored slots gives
//     a lower threshold whose expected count is about 1.3 k.
//  2. One pass over all scored slots appends every key at or above it to a
//     shared-memory candidate list (key, position in the ascending kept-slot
//     order), one atomic per warp.  If the list holds at least k keys it holds
//     the whole top k, so the rest is exact:
//  3. a radix select over the candidates (4 x 8-bit digits) gives the
//     threshold key T and how many keys equal to T belong to the top k;
//  4. chosen positions are set in a shared-memory bitmap; two block scans
//     over it take the lowest-position ties and give each chosen slot its
//     output index, so the output is ascending without a sort.
// When the estimate misses (fewer than k candidates, or more than fit), the
// kernel falls back to an exact histogram of all keys, then a collection of
// the keys in its threshold bin, then -- if even those do not fit -- three
// more full radix passes.
#include <algorithm>

#include "spin_internal.cuh"
#include "block_scan.cuh"

namespace spin {

constexpr int kTopkThreads = 1024;
constexpr int kBins = 8192;           // 13-bit first digit
constexpr int kFirstShift = 19;
constexpr int kCandCap = 8192;        // candidates kept on chip

struct TopkShared {
  uint32_t digit[2];
  int scan[33];
  int total;
  int n_cand;
  int overflow;
};

// Visits every scored slot (kept blocks, s <= p) as f(position, slot, key),
// four float4 loads in flight per thread.
template <class F>
__device__ __forceinline__ void for_each_scored(const float* sc, const int32_t* work, int nk, int lb, int p, F f) {
  const int n_elem = nk << lb;
  const int step = blockDim.x * 4;
  for (int base = threadIdx.x * 4; base < n_elem; base += 4 * step) {
    float4 v[4];
    int s0[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int e = base + u * step;
      s0[u] = -1;
      if (e < n_elem) {
        const int s = (work[e >> lb] << lb) + (e & ((1 << lb) - 1));
        if (s <= p) {
          s0[u] = s;
          v[u] = *reinterpret_cast<const float4*>(sc + s);
        }
      }
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int s = s0[u];
      if (s < 0) continue;
      const int e = base + u * step;
      f(e, s, fkey(v[u].x));
      if (s + 1 <= p) f(e + 1, s + 1, fkey(v[u].y));
      if (s + 2 <= p) f(e + 2, s + 2, fkey(v[u].z));
      if (s + 3 <= p) f(e + 3, s + 3, fkey(v[u].w));
    }
  }
}

// Histogram add with the lanes of a warp that hit the same bin combined.
__device__ __forceinline__ void hist_add(uint32_t* hist, uint32_t bin, bool active) {
  const uint32_t mask = __ballot_sync(0xffffffffu, active);
  if (!active) return;
  const uint32_t peers = __match_any_sync(mask, bin);
  const int leader = __ffs(peers) - 1;
  if ((int)(threadIdx.x & 31) == leader) atomicAdd(&hist[bin], (uint32_t)__popc(peers));
}

// Block-wide search of the bin holding the `want`-th largest element of a
// histogram with nb bins (nb a positive multiple of blockDim.x): writes the
// bin and the rank left inside it to digit[0..1].
__device__ void block_find_bin_desc(const uint32_t* hist, int nb, uint32_t want, TopkShared& sh) {
  const int per = nb / blockDim.x;
  // thread t covers bins nb-1-t*per .. nb-per-t*per (from the top)
  const int hi = nb - 1 - threadIdx.x * per;
  uint32_t s = 0;
  for (int i = 0; i < per; ++i) s += hist[hi - i];
  int tot;
  const uint32_t exc = (uint32_t)block_exclusive_scan((int)s, sh.scan, &tot);
  if (exc < want && want <= exc + s) {
    uint32_t cum = exc;
    for (int i = 0; i < per; ++i) {
      const uint32_t c = hist[hi - i];
      if (cum + c >= want) {
        sh.digit[0] = (uint32_t)(hi - i);
        sh.digit[1] = want - cum;
        break;
      }
      cum += c;
    }
  }
  __syncthreads();
}

__global__ void __launch_bounds__(kTopkThreads) k_topk(TopkArgs a) {
  const Layout L = a.lay;
  const int q = blockIdx.x / a.rows, r = blockIdx.x % a.rows;
  int32_t* out = a.topk + ((int64_t)q * a.rows + r) * L.k;
  __shared__ TopkShared sh;
  extern __shared__ __align__(16) uint8_t dyn[];
  const int64_t ctx = a.ctx_len[q];
  if (ctx < 1 || ctx + a.rows - 1 > L.max_slots) {
    for (int t = threadIdx.x; t < L.k; t += blockDim.x) out[t] = -1;
    return;
  }
  const int p = (int)(ctx - 1 + r);
  const int nk = a.kept[q];
  const int32_t* work = a.work + (int64_t)q * L.blk_stride;
  const float* sc = a.scores + ((int64_t)q * L.R + r) * L.slot_stride;
  const int lb = __ffs(L.b) - 1;  // block size is a power of two
  const int bmask = L.b - 1;
  const int n_elem = nk << lb;
  const int nwords = (n_elem + 31) / 32;
  uint32_t* bits = reinterpret_cast<uint32_t*>(dyn);
  uint8_t* work_area = dyn + (((size_t)(L.slot_stride + 31) / 32) * 4 + 15) / 16 * 16;
  uint32_t* hist = reinterpret_cast<uint32_t*>(work_area);          // kBins (pass 1)
  uint32_t* ckey = reinterpret_cast<uint32_t*>(work_area);          // kCandCap (after pass 1)
  uint32_t* cpos = ckey + kCandCap;
  uint32_t* hist2 = cpos + kCandCap;                                // 256 bins (candidate passes)

  // ---- number of scored slots -------------------------------------------
  {
    int c = 0;
    for (int t = threadIdx.x; t < nk; t += blockDim.x) c += min(max(p - (work[t] << lb) + 1, 0), L.b);
    int tot;
    block_exclusive_scan(c, sh.scan, &tot);
    if (threadIdx.x == 0) {
      sh.total = tot;
      sh.n_cand = 0;
    }
    __syncthreads();
  }
  const int total = sh.total;
  const int want = min(total, L.k);
  if (want == 0) {
    for (int t = threadIdx.x; t < L.k; t += blockDim.x) out[t] = -1;
    return;
  }
  uint32_t T = 0, remaining = 0;
  bool done = false;

  // ---- sampled threshold, one collecting pass, exact select on chip ---------
  {
    uint32_t t_lo = 0;  // keep everything when all scored slots fit
    bool est_ok = true;
    if (total > kCandCap) {
      for (int i = threadIdx.x; i < kBins; i += blockDim.x) hist[i] = 0;
      __syncthreads();
      const int n_smp = n_elem >> 6;  // one float4 out of every 64 scored positions
      for (int it = 0; it < n_smp; it += blockDim.x) {
        const int i = it + threadIdx.x;
        float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
        int s = -1;
        if (i < n_smp) {
          const int e = i << 6;
          s = (work[e >> lb] << lb) + (e & bmask);
          if (s <= p) v = *reinterpret_cast<const float4*>(sc + s);
        }
        const float vals[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const bool act = s >= 0 && s + c <= p;
          hist_add(hist, act ? fkey(vals[c]) >> kFirstShift : 0u, act);
        }
      }
      __syncthreads();
      int c = 0;
      for (int i = threadIdx.x; i < kBins; i += blockDim.x) c += hist[i];
      int n_s;
      block_exclusive_scan(c, sh.scan, &n_s);
      const int ks = min(n_s, (int)ceilf(1.3f * (float)want * (float)n_s / (float)total) + 16);
      if (ks >= 1) {
        block_find_bin_desc(hist, kBins, (uint32_t)ks, sh);
        t_lo = sh.digit[0] << kFirstShift;
      } else {
        est_ok = false;
      }
      __syncthreads();
    }
    if (est_ok) {
      // warp-uniform pass: a warp appends its takers with one atomic
      const int step = blockDim.x * 4;
      const int lane = threadIdx.x & 31;
      for (int it = 0; it < n_elem; it += 4 * step) {
        const int base = it + threadIdx.x * 4;
        float4 v[4];
        int s0[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int e = base + u * step;
          s0[u] = -1;
          v[u] = make_float4(0.f, 0.f, 0.f, 0.f);
          if (e < n_elem) {
            const int s = (work[e >> lb] << lb) + (e & bmask);
            if (s <= p) {
              s0[u] = s;
              v[u] = *reinterpret_cast<const float4*>(sc + s);
            }
          }
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const float vals[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            const uint32_t key = fkey(vals[c]);
            const bool take = s0[u] >= 0 && s0[u] + c <= p && key >= t_lo;
            const uint32_t bal = __ballot_sync(0xffffffffu, take);
            if (bal) {
              const int leader = __ffs(bal) - 1;
              int at = 0;
              if (lane == leader) at = atomicAdd(&sh.n_cand, __popc(bal));
              at = __shfl_sync(0xffffffffu, at, leader) + __popc(bal & ((1u << lane) - 1u));
              if (take && at < kCandCap) {
                ckey[at] = key;
                cpos[at] = (uint32_t)(base + u * step + c);
              }
            }
          }
        }
      }
      __syncthreads();
      const int n_cand = sh.n_cand;
      if (n_cand >= want && n_cand <= kCandCap) {
        uint32_t prefix = 0, rem = (uint32_t)want;
        for (int shift = 24; shift >= 0; shift -= 8) {
          for (int i = threadIdx.x; i < 256; i += blockDim.x) hist2[i] = 0;
          __syncthreads();
          const uint32_t pmask = shift == 24 ? 0u : (0xFFFFFFFFu << (shift + 8));
          for (int i = threadIdx.x; i < n_cand; i += blockDim.x) {
            const uint32_t k = ckey[i];
            if ((k & pmask) == prefix) atomicAdd(&hist2[(k >> shift) & 255u], 1u);
          }
          __syncthreads();
          if (threadIdx.x < 32) warp_find_digit_desc<256>(hist2, rem, sh.digit);
          __syncthreads();
          prefix |= sh.digit[0] << shift;
          rem = sh.digit[1];
          __syncthreads();
        }
        T = prefix;
        remaining = rem;
        for (int i = threadIdx.x; i < nwords; i += blockDim.x) bits[i] = 0;
        __syncthreads();
        for (int i = threadIdx.x; i < n_cand; i += blockDim.x)
          if (ckey[i] >= T) atomicOr(&bits[cpos[i] >> 5], 1u << (cpos[i] & 31));
        __syncthreads();
        done = true;
      }
    }
    __syncthreads();
    if (threadIdx.x == 0) sh.n_cand = 0;
    __syncthreads();
  }

  if (!done) {
    // ---- pass 1: 13-bit histogram ------------------------------------------
    for (int i = threadIdx.x; i < kBins; i += blockDim.x) hist[i] = 0;
    __syncthreads();
    {
      const int step = blockDim.x * 4;
      for (int it = 0; it < n_elem; it += 4 * step) {
        const int base = it + threadIdx.x * 4;
        float4 v[4];
        int s0[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int e = base + u * step;
          s0[u] = -1;
          if (e < n_elem) {
            const int s = (work[e >> lb] << lb) + (e & bmask);
            if (s <= p) {
              s0[u] = s;
              v[u] = *reinterpret_cast<const float4*>(sc + s);
            }
          }
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int s = s0[u];
          const float vals[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            const bool act = s >= 0 && s + c <= p;
            hist_add(hist, act ? fkey(vals[c]) >> kFirstShift : 0u, act);
          }
        }
      }
    }
    __syncthreads();
    block_find_bin_desc(hist, kBins, (uint32_t)want, sh);
    const uint32_t d1 = sh.digit[0];
    remaining = sh.digit[1];
    __syncthreads();

    // ---- pass 2: collect keys in bin d1 and above ------------------------------
    // (the histogram area becomes the candidate list)
    for_each_scored(sc, work, nk, lb, p, [&](int e, int, uint32_t key) {
      if ((key >> kFirstShift) >= d1) {
        const int slot = atomicAdd(&sh.n_cand, 1);
        if (slot < kCandCap) {
          ckey[slot] = key;
          cpos[slot] = (uint32_t)e;
        }
      }
    });
    __syncthreads();
    const int n_cand = sh.n_cand;
    if (n_cand <= kCandCap) {
      // ---- exact select among the candidates (rank counted from the top) -------
      // elements above bin d1 are all chosen; `remaining` is the rank inside d1
      uint32_t prefix = d1, pbits = 32 - kFirstShift;
      const int shifts[3] = {11, 3, 0};
      const int widths[3] = {8, 8, 3};
      for (int ps = 0; ps < 3; ++ps) {
        const int shf = shifts[ps], w = widths[ps];
        for (int i = threadIdx.x; i < 256; i += blockDim.x) hist2[i] = 0;
        __syncthreads();
        for (int i = threadIdx.x; i < n_cand; i += blockDim.x) {
          const uint32_t k = ckey[i];
          if ((k >> (32 - pbits)) == prefix) atomicAdd(&hist2[(k >> shf) & ((1u << w) - 1u)], 1u);
        }
        __syncthreads();
        if (threadIdx.x < 32) warp_find_digit_desc<256>(hist2, remaining, sh.digit);  // bins >= 2^w are empty
        __syncthreads();
        prefix = (prefix << w) | sh.digit[0];
        pbits += w;
        remaining = sh.digit[1];
        __syncthreads();
      }
      T = prefix;
      for (int i = threadIdx.x; i < nwords; i += blockDim.x) bits[i] = 0;
      __syncthreads();
      for (int i = threadIdx.x; i < n_cand; i += blockDim.x)
        if (ckey[i] >= T) atomicOr(&bits[cpos[i] >> 5], 1u << (cpos[i] & 31));
      __syncthreads();
    } else {
      // ---- fallback: three more full passes over HBM --------------------------
      uint32_t prefix = d1;
      int shift_hi = kFirstShift;
      const int shifts[3] = {11, 3, 0};
      for (int ps = 0; ps < 3; ++ps) {
        const int sh_lo = shifts[ps];
        const int width = shift_hi - sh_lo;
        const uint32_t dmask = (1u << width) - 1u;
        for (int i = threadIdx.x; i < 256; i += blockDim.x) hist2[i] = 0;
        __syncthreads();
        for_each_scored(sc, work, nk, lb, p, [&](int, int, uint32_t key) {
          if ((key >> shift_hi) == prefix) atomicAdd(&hist2[(key >> sh_lo) & dmask], 1u);
        });
        __syncthreads();
        if (threadIdx.x < 32) warp_find_digit_desc<256>(hist2, remaining, sh.digit);
        __syncthreads();
        prefix = (prefix << width) | sh.digit[0];
        remaining = sh.digit[1];
        shift_hi = sh_lo;
        __syncthreads();
      }
      T = prefix;
      for (int i = threadIdx.x; i < nwords; i += blockDim.x) bits[i] = 0;
      __syncthreads();
      for_each_scored(sc, work, nk, lb, p, [&](int e, int, uint32_t key) {
        if (key >= T) atomicOr(&bits[e >> 5], 1u << (e & 31));
      });
      __syncthreads();
    }
  }
  const uint32_t eq_take = remaining;

  // ---- ordered tie handling and emission -----------------------------------
  const int chunk = (nwords + blockDim.x - 1) / blockDim.x;
  const int w0 = threadIdx.x * chunk, w1 = min(nwords, w0 + chunk);
  int n_gt = 0, n_eq = 0;
  for (int w = w0; w < w1; ++w) {
    uint32_t m = bits[w];
    while (m) {
      const int bit = __ffs(m) - 1;
      m &= m - 1;
      const int e = w * 32 + bit;
      const int s = (work[e >> lb] << lb) + (e & bmask);
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
      const int e = w * 32 + bit;
      const int s = (work[e >> lb] << lb) + (e & bmask);
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

size_t topk_smem_bytes(const Layout& L) {
  const size_t bitmap = ((size_t)(L.slot_stride + 31) / 32) * 4;
  const size_t area = std::max<size_t>((size_t)kBins * 4, (size_t)kCandCap * 8 + 256 * 4);
  return (bitmap + 15) / 16 * 16 + area;
}

cudaError_t launch_topk(const TopkArgs& a, cudaStream_t s) {
  const size_t smem = topk_smem_bytes(a.lay);
  cudaError_t e = cudaFuncSetAttribute(k_topk, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  k_topk<<<a.lay.Q * a.rows, kTopkThreads, smem, s>>>(a);
  return cudaGetLastError();
}

}  // namespace spin
