// k_topk.cu -- a4 token top-k over the scored slots (SPIN digest,
// arXiv深度剖析: SPIN leaves the fixed top-k budget of core attention as it
// is).  Order: higher score first, ties to the lower slot; the chosen slots
// are emitted in ascending slot order, padded with -1.
//
// One CTA (1024 threads) per (request, row).  Scores are compared through
// their order-preserving 32-bit keys.
//  1. Candidates.  When the score kernel left the maximum of every 32 slots
//     (the fused decode step) and there are at least two groups per wanted
//     score, M = the k-th largest group maximum bounds the k-th score from
//     below; only the groups whose maximum is >= M are read and their scores
//     >= M kept (compared with the float whose key is M).  With fewer groups
//     nearly all of them qualify and the list would overflow, so, as without
//     group maxima, a lower threshold comes from the
//     13-bit histogram of a fixed 1/16 sample (about 1.3 k keys expected
//     above it) and one pass over all scored slots keeps the keys above it.
//     Candidates are (key, position in the ascending kept-slot order) in
//     shared memory, appended with one shared atomic per warp.  If the list
//     holds at least k keys it holds the whole top k, so the rest is exact:
//  3. a radix select over the candidates (4 x 8-bit digits) gives the
//     threshold key T and how many keys equal to T belong to the top k; the
//     keys equal to T are ranked by position (lowest first) with a second
//     radix select;
//  4. the chosen positions are set in a shared-memory bitmap, and one block
//     scan over it gives every chosen slot its output index, so the output is
//     ascending without a sort.
// A sample that misses (too few or too many candidates) falls back to an
// exact histogram of all keys, a collection of the keys in its threshold bin
// and -- if even those do not fit -- three more full radix passes, after
// which ties are resolved by re-reading the scores.  Every path gives the
// same result; the sample only decides the speed.
#include <cooperative_groups.h>

#include <algorithm>

#include "spin_internal.cuh"
#include "block_scan.cuh"

namespace spin {

constexpr int kTopkThreads = 1024;
constexpr int kBins = 8192;           // 13-bit first digit
constexpr int kFirstShift = 19;
constexpr int kCandCap = kTopkCandCap;  // candidates kept on chip
constexpr uint32_t kEmptyGroup = 0x007FFFFFu;  // key of -inf: a group with no scored slot

// Dynamic shared memory: the slot bitmap, the histogram / candidate area and,
// when it fits, a copy of the request's kept-block list.
__host__ __device__ inline size_t topk_bitmap_bytes(const Layout& L) {
  return (((size_t)(L.slot_stride + 31) / 32) * 4 + 15) / 16 * 16;
}
__host__ __device__ constexpr size_t topk_area_bytes() {
  return (size_t)kBins * 4 > (size_t)kCandCap * 8 + 256 * 4 ? (size_t)kBins * 4 : (size_t)kCandCap * 8 + 256 * 4;
}
__host__ __device__ inline bool topk_stages_work(const Layout& L) {
  return topk_bitmap_bytes(L) + topk_area_bytes() + (size_t)L.blk_stride * 4 <= 220 * 1024;
}

struct TopkShared {
  uint32_t k_and, k_or, M;
  uint32_t digit[2];
  int scan[33];
  int total;
  int n_cand;
  int n_eq;
};

struct TopkCtx {
  const float* sc;
  const int32_t* work;
  int nk, lb, bmask, p, n_elem, nwords;
  int bits_cap;     // words of the bitmap area
  uint32_t* bits;
  uint32_t* hist;   // kBins
  uint32_t* ckey;   // kCandCap (aliases hist)
  uint32_t* cpos;   // kCandCap
  uint32_t* hist2;  // 256
};


// Visits every scored slot (kept blocks, s <= p) as f(position, key), with
// the work-list loads of eight float4s issued before their score loads.
template <class F>
__device__ __forceinline__ void for_each_scored(const TopkCtx& c, F f) {
  const int step = blockDim.x * 4;
  for (int it = 0; it < c.n_elem; it += 8 * step) {
    int blk[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int e = it + threadIdx.x * 4 + u * step;
      blk[u] = e < c.n_elem ? c.work[e >> c.lb] : -1;
    }
    float4 v[8];
    int s0[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int e = it + threadIdx.x * 4 + u * step;
      s0[u] = -1;
      if (blk[u] >= 0) {
        const int s = (blk[u] << c.lb) + (e & c.bmask);
        if (s <= c.p) {
          s0[u] = s;
          v[u] = *reinterpret_cast<const float4*>(c.sc + s);
        }
      }
    }
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      if (s0[u] < 0) continue;
      const int e = it + threadIdx.x * 4 + u * step;
      const float vals[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
#pragma unroll
      for (int k = 0; k < 4; ++k)
        if (s0[u] + k <= c.p) f(e + k, fkey(vals[k]));
    }
  }
}

// Histogram add: one shared atomic per lane.  Combining the lanes of a warp
// that hit the same bin (__match_any_sync) cost more than the contention it
// saves (the sampled top-k of 78K-slot rows: 0.050 -> 0.047 ms without it).
__device__ __forceinline__ void hist_add(uint32_t* hist, uint32_t bin, bool active) {
  if (active) atomicAdd(&hist[bin], 1u);
}

// Block-wide search of the bin holding the `want`-th largest element of a
// histogram with nb bins (nb a positive multiple of blockDim.x): writes the
// bin and the rank left inside it to digit[0..1].
__device__ void block_find_bin_desc(const uint32_t* hist, int nb, uint32_t want, TopkShared& sh) {
  const int per = nb / blockDim.x;
  const int hi = nb - 1 - threadIdx.x * per;  // this thread's bins, from the top
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

// Lower threshold from the 13-bit histogram of a fixed 1/16 sample (one
// float4 out of every 64 scored positions) where about 1.3 `want` keys of
// the `total` are expected above it.
__device__ uint32_t sample_threshold(const TopkCtx& c, int want, int total, TopkShared& sh) {
  for (int i = threadIdx.x; i < kBins; i += blockDim.x) c.hist[i] = 0;
  __syncthreads();
  const int n_smp = c.n_elem >> 6;
  for (int it = 0; it < n_smp; it += 4 * blockDim.x) {
    float4 v[4];
    int s0[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int i = it + u * blockDim.x + threadIdx.x;
      s0[u] = -1;
      v[u] = make_float4(0.f, 0.f, 0.f, 0.f);
      if (i < n_smp) {
        const int e = i << 6;
        const int s = (c.work[e >> c.lb] << c.lb) + (e & c.bmask);
        if (s <= c.p) {
          s0[u] = s;
          v[u] = *reinterpret_cast<const float4*>(c.sc + s);
        }
      }
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const float vals[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const bool act = s0[u] >= 0 && s0[u] + k <= c.p;
        hist_add(c.hist, act ? fkey(vals[k]) >> kFirstShift : 0u, act);
      }
    }
  }
  __syncthreads();
  int cnt = 0;
  for (int i = threadIdx.x; i < kBins; i += blockDim.x) cnt += c.hist[i];
  int n_s;
  block_exclusive_scan(cnt, sh.scan, &n_s);
  const int ks = min(n_s, (int)ceilf(1.3f * (float)want * (float)n_s / (float)total) + 16);
  uint32_t t_lo = 0;
  if (ks >= 1) {
    block_find_bin_desc(c.hist, kBins, (uint32_t)ks, sh);
    t_lo = sh.digit[0] << kFirstShift;
  }
  __syncthreads();
  return t_lo;
}

// Appends every scored key >= t_lo; returns how many there are (the list
// keeps the first kCandCap).  The loop is uniform across a warp, so takers
// are counted with a ballot and reserved with one atomic per warp.
__device__ int collect_ge(const TopkCtx& c, uint32_t t_lo, TopkShared& sh) {
  if (threadIdx.x == 0) sh.n_cand = 0;
  __syncthreads();
  const int lane = threadIdx.x & 31;
  const int step = blockDim.x * 4;
  for (int it = 0; it < c.n_elem; it += 8 * step) {
    int blk[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int e = it + threadIdx.x * 4 + u * step;
      blk[u] = e < c.n_elem ? c.work[e >> c.lb] : -1;
    }
    float4 v[8];
    int s0[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int e = it + threadIdx.x * 4 + u * step;
      s0[u] = -1;
      v[u] = make_float4(0.f, 0.f, 0.f, 0.f);
      if (blk[u] >= 0) {
        const int s = (blk[u] << c.lb) + (e & c.bmask);
        if (s <= c.p) {
          s0[u] = s;
          v[u] = *reinterpret_cast<const float4*>(c.sc + s);
        }
      }
    }
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const float vals[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
      uint32_t takes = 0;
#pragma unroll
      for (int k = 0; k < 4; ++k)
        if (s0[u] >= 0 && s0[u] + k <= c.p && fkey(vals[k]) >= t_lo) takes |= 1u << k;
      const int n_my = __popc(takes);
      if (!__any_sync(0xffffffffu, n_my != 0)) continue;  // the common case
      int incl = n_my;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int t = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += t;
      }
      int base = 0;
      if (lane == 31) base = atomicAdd(&sh.n_cand, incl);
      base = __shfl_sync(0xffffffffu, base, 31) + incl - n_my;
      const int e0 = it + threadIdx.x * 4 + u * step;
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        if (takes & (1u << k)) {
          if (base < kCandCap) {
            c.ckey[base] = fkey(vals[k]);
            c.cpos[base] = (uint32_t)(e0 + k);
          }
          ++base;
        }
      }
    }
  }
  __syncthreads();
  return sh.n_cand;
}

// Radix select over the first n entries of `keys` (largest first when desc,
// else smallest first): the key of rank `want` and how many keys equal to it
// are taken.
__device__ void radix_select_list(const uint32_t* keys, int n, uint32_t want, bool desc, uint32_t* hist2,
                                  TopkShared& sh, uint32_t* key_out, uint32_t* eq_out) {
  uint32_t prefix = 0, rem = want;
  for (int shift = 24; shift >= 0; shift -= 8) {
    for (int i = threadIdx.x; i < 256; i += blockDim.x) hist2[i] = 0;
    __syncthreads();
    const uint32_t pmask = shift == 24 ? 0u : (0xFFFFFFFFu << (shift + 8));
    for (int i = threadIdx.x; i < n; i += blockDim.x) {
      const uint32_t k = desc ? keys[i] : ~keys[i];
      if ((k & pmask) == prefix) atomicAdd(&hist2[(k >> shift) & 255u], 1u);
    }
    __syncthreads();
    if (threadIdx.x < 32) warp_find_digit_desc<256>(hist2, rem, sh.digit);
    __syncthreads();
    prefix |= sh.digit[0] << shift;
    rem = sh.digit[1];
    __syncthreads();
  }
  *key_out = desc ? prefix : ~prefix;
  *eq_out = rem;
}

// Exact top `want` among n_cand (>= want) candidates: sets exactly the chosen
// positions in the bitmap.  Returns the threshold key T.
__device__ uint32_t select_candidates(const TopkCtx& c, int n_cand, int want, TopkShared& sh) {
  uint32_t T, eq_take;
  radix_select_list(c.ckey, n_cand, (uint32_t)want, true, c.hist2, sh, &T, &eq_take);
  for (int i = threadIdx.x; i < c.nwords; i += blockDim.x) c.bits[i] = 0;
  if (threadIdx.x == 0) sh.n_eq = 0;
  __syncthreads();
  for (int i = threadIdx.x; i < n_cand; i += blockDim.x)
    if (c.ckey[i] > T) atomicOr(&c.bits[c.cpos[i] >> 5], 1u << (c.cpos[i] & 31));
  // Keys equal to T: their positions are compacted to the front of the key
  // array (the keys are no longer needed; a round reads before it writes,
  // and writes only reach indices already read), then the eq_take lowest
  // positions are chosen.
  uint32_t* epos = c.ckey;
  for (int base = 0; base < n_cand; base += blockDim.x) {
    const int i = base + threadIdx.x;
    const bool eq = i < n_cand && c.ckey[i] == T;
    const uint32_t pos = i < n_cand ? c.cpos[i] : 0u;
    __syncthreads();
    if (eq) epos[atomicAdd(&sh.n_eq, 1)] = pos;
    __syncthreads();
  }
  const int n_eq = sh.n_eq;
  if ((uint32_t)n_eq <= eq_take) {
    for (int i = threadIdx.x; i < n_eq; i += blockDim.x) atomicOr(&c.bits[epos[i] >> 5], 1u << (epos[i] & 31));
  } else {
    uint32_t P, unused;
    radix_select_list(epos, n_eq, eq_take, false, c.hist2, sh, &P, &unused);
    for (int i = threadIdx.x; i < n_eq; i += blockDim.x)
      if (epos[i] <= P) atomicOr(&c.bits[epos[i] >> 5], 1u << (epos[i] & 31));
  }
  __syncthreads();
  return T;
}

// Candidates from group maxima (the score kernel's max of every 32 slots of
// the kept-slot order), for n_groups > want.  Any M no larger than the
// want-th largest group maximum works: at least `want` scores are >= M (each
// of the want best groups holds one), and every score >= M lies in a group
// whose maximum is >= M, so gathering those groups' scores >= M yields a
// candidate list that holds the whole top `want`.  M is the lower edge of the
// 13-bit histogram bin that holds the want-th largest group key, with the bin
// window placed just below the leading bits all group keys share.  The group
// keys and then the compacted group list live in the bitmap area.
// The float whose key is M (the inverse of fkey, M never a NaN pattern): for
// every score x, fkey(x) >= M exactly when x >= key_float(M), -0 and +0 alike.
__device__ __forceinline__ float key_float(uint32_t M) {
  return __uint_as_float((M & 0x80000000u) ? (M & 0x7FFFFFFFu) : ~M);
}

// Bit 4u + k: the k-th score of float4 v[u] (slot s0[u] + k, s0[u] < 0 for
// none) is visible (slot <= p) and at least Mf.
__device__ __forceinline__ uint32_t takes_at_least(const float4 (&v)[8], const int (&s0)[8], int p, float Mf) {
  uint32_t takes = 0;
#pragma unroll
  for (int u = 0; u < 8; ++u) {
    const int nv = s0[u] < 0 ? 0 : min(4, p - s0[u] + 1);  // visible values of this float4
    const uint32_t ge = (v[u].x >= Mf ? 1u : 0u) | (v[u].y >= Mf ? 2u : 0u) | (v[u].z >= Mf ? 4u : 0u) |
                        (v[u].w >= Mf ? 8u : 0u);
    takes |= (ge & ((1u << nv) - 1u)) << (4 * u);
  }
  return takes;
}

__device__ int collect_from_groups(const TopkCtx& c, const float* gmax, int want, TopkShared& sh) {
  const int n_groups = (c.n_elem + 31) / 32;  // == c.nwords
  uint32_t* gk = c.bits;
  if (threadIdx.x == 0) {
    sh.k_and = 0xFFFFFFFFu;
    sh.k_or = 0u;
  }
  __syncthreads();
  uint32_t k_and = 0xFFFFFFFFu, k_or = 0u;
  for (int g0 = 0; g0 < n_groups; g0 += 4 * blockDim.x) {
    float v[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int g = g0 + u * blockDim.x + threadIdx.x;
      v[u] = g < n_groups ? gmax[g] : 0.f;
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int g = g0 + u * blockDim.x + threadIdx.x;
      if (g < n_groups) {
        const uint32_t k = fkey(v[u]);
        gk[g] = k;
        if (k != kEmptyGroup) {  // a group with no scored slot never qualifies
          k_and &= k;
          k_or |= k;
        }
      }
    }
  }
  k_and = __reduce_and_sync(0xffffffffu, k_and);
  k_or = __reduce_or_sync(0xffffffffu, k_or);
  for (int i = threadIdx.x; i < kBins; i += blockDim.x) c.hist[i] = 0;
  if ((threadIdx.x & 31) == 0) {
    atomicAnd(&sh.k_and, k_and);
    atomicOr(&sh.k_or, k_or);
  }
  __syncthreads();
  const uint32_t diff = sh.k_and ^ sh.k_or;
  uint32_t M = sh.k_and;  // every scored group's key is equal (or none is scored)
  if (sh.k_or == 0u) M = kEmptyGroup;
  if (diff) {
    const int hb = 31 - __clz(diff);                 // highest bit where keys differ
    const int shift = hb >= 12 ? hb - 12 : 0;        // 13-bit window [shift, shift + 12]
    for (int g0 = 0; g0 < n_groups; g0 += blockDim.x) {  // warp-uniform trip count
      const int g = g0 + threadIdx.x;
      const bool act = g < n_groups && gk[g] != kEmptyGroup;
      if (act) atomicAdd(&c.hist[(gk[g] >> shift) & (kBins - 1)], 1u);  // spread keys: little contention
    }
    __syncthreads();
    int cnt = 0;
    for (int i = threadIdx.x; i < kBins; i += blockDim.x) cnt += c.hist[i];
    int n_scored_groups;
    block_exclusive_scan(cnt, sh.scan, &n_scored_groups);
    if (n_scored_groups >= want) {
      block_find_bin_desc(c.hist, kBins, (uint32_t)want, sh);
      const uint32_t high = shift + 13 >= 32 ? 0u : (sh.k_and & ~((1u << (shift + 13)) - 1u));
      M = high | (sh.digit[0] << shift);
    } else {
      M = sh.k_and;  // fewer scored groups than wanted: every scored group qualifies
    }
  }
  // compact the qualifying group ids to the front, in place (a round reads
  // before it writes, and writes only reach indices already read); one
  // shared atomic per warp and round
  if (threadIdx.x == 0) sh.n_eq = 0;
  __syncthreads();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  for (int base = 0; base < n_groups; base += blockDim.x) {  // block-uniform trip count
    const int g = base + threadIdx.x;
    const bool take = g < n_groups && gk[g] >= M;
    const uint32_t bal = __ballot_sync(0xffffffffu, take);
    __syncthreads();
    if (bal) {
      uint32_t at = 0;
      if (lane == 0) at = atomicAdd((uint32_t*)&sh.n_eq, (uint32_t)__popc(bal));
      at = __shfl_sync(0xffffffffu, at, 0) + __popc(bal & ((1u << lane) - 1u));
      if (take) gk[at] = (uint32_t)g;
    }
    __syncthreads();
  }
  const int n_q = sh.n_eq;
  const float Mf = key_float(M);
  if (threadIdx.x == 0) sh.n_cand = 0;
  __syncthreads();
  // gather: a warp takes 32 groups at a time, 8 lanes x float4 per group.
  // Pass 1 keeps no score: each lane records which of its 32 values reach M
  // (4 bits per float4) in the free part of the bitmap area, so every pass
  // issues its eight loads with nothing held from the pass before.  Pass 2
  // reads the taken values again (from L2) and appends them.
  const int q_al = (n_q + 31) & ~31;
  uint32_t* tmask = gk + q_al;  // one word per lane per warp pass: entry base + lane
  const bool two_pass = 2 * q_al <= c.bits_cap;
  int my_cnt = 0;
  for (int base = warp * 32; base < n_q; base += nw * 32) {
    int e0[8];
    float4 v[8];
    int s0[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int gi = base + u * 4 + (lane >> 3);
      e0[u] = gi < n_q ? (int)gk[gi] * 32 + (lane & 7) * 4 : -1;
    }
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      s0[u] = -1;
      v[u] = make_float4(0.f, 0.f, 0.f, 0.f);
      if (e0[u] >= 0 && e0[u] < c.n_elem) {
        const int s = (c.work[e0[u] >> c.lb] << c.lb) + (e0[u] & c.bmask);
        if (s <= c.p) {
          s0[u] = s;
          v[u] = *reinterpret_cast<const float4*>(c.sc + s);
        }
      }
    }
    const uint32_t takes = takes_at_least(v, s0, c.p, Mf);
    if (two_pass) {
      tmask[base + lane] = takes;
      my_cnt += __popc(takes);
      continue;
    }
    // one pass (no room for the masks): append now
    const int n_my = __popc(takes);
    if (!__any_sync(0xffffffffu, n_my != 0)) continue;
    int incl = n_my;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int t = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += t;
    }
    int at = 0;
    if (lane == 31) at = atomicAdd(&sh.n_cand, incl);
    at = __shfl_sync(0xffffffffu, at, 31) + incl - n_my;
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const float vals[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        if (takes & (1u << (4 * u + k))) {
          if (at < kCandCap) {
            c.ckey[at] = fkey(vals[k]);
            c.cpos[at] = (uint32_t)(e0[u] + k);
          }
          ++at;
        }
      }
    }
  }
  if (two_pass) {
    // this lane's places in the candidate list: one atomic per warp
    int incl = my_cnt;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int t = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += t;
    }
    int at = 0;
    if (lane == 31 && incl) at = atomicAdd(&sh.n_cand, incl);
    at = __shfl_sync(0xffffffffu, at, 31) + incl - my_cnt;
    for (int base = warp * 32; base < n_q; base += nw * 32) {
      uint32_t takes = tmask[base + lane];
      while (takes) {
        const int bit = __ffs(takes) - 1;
        takes &= takes - 1;
        const int u = bit >> 2, k = bit & 3;
        const int e = (int)gk[base + u * 4 + (lane >> 3)] * 32 + (lane & 7) * 4 + k;
        const int s = (c.work[e >> c.lb] << c.lb) + (e & c.bmask);
        if (at < kCandCap) {
          c.ckey[at] = fkey(c.sc[s]);
          c.cpos[at] = (uint32_t)e;
        }
        ++at;
      }
    }
  }
  __syncthreads();
  return sh.n_cand;
}

// The group path spread over a cluster of CTAs (few requests, many idle SMs):
// rank c takes the c-th share of the groups, the ranks' key bits and
// histograms meet in rank 0 through distributed shared memory, rank 0 finds
// M and sends it back, and every rank gathers its share's candidates
// straight into rank 0's list.  Returns the candidate count in rank 0 and -2
// in the other ranks, which are done.
__device__ __forceinline__ int collect_from_groups_cluster(const TopkCtx& c, const float* gmax, int want, TopkShared& sh) {
  namespace cg = cooperative_groups;
  cg::cluster_group cl = cg::this_cluster();
  const int C = (int)cl.num_blocks(), cr = (int)cl.block_rank();
  const int n_groups = (c.n_elem + 31) / 32;
  const int gs0 = (int)((int64_t)n_groups * cr / C), gs1 = (int)((int64_t)n_groups * (cr + 1) / C);
  const int n_my = gs1 - gs0;
  uint32_t* gk = c.bits;  // this share's group keys, then its qualifying group ids
  TopkShared* sh0 = cl.map_shared_rank(&sh, 0);
  if (threadIdx.x == 0) {
    sh.k_and = 0xFFFFFFFFu;
    sh.k_or = 0u;
    sh.n_cand = 0;
    sh.n_eq = 0;
  }
  for (int i = threadIdx.x; i < kBins; i += blockDim.x) c.hist[i] = 0;
  cl.sync();
  uint32_t k_and = 0xFFFFFFFFu, k_or = 0u;
  for (int g0 = 0; g0 < n_my; g0 += 4 * blockDim.x) {
    float v[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int g = g0 + u * blockDim.x + threadIdx.x;
      v[u] = g < n_my ? gmax[gs0 + g] : 0.f;
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int g = g0 + u * blockDim.x + threadIdx.x;
      if (g < n_my) {
        const uint32_t k = fkey(v[u]);
        gk[g] = k;
        if (k != kEmptyGroup) {
          k_and &= k;
          k_or |= k;
        }
      }
    }
  }
  k_and = __reduce_and_sync(0xffffffffu, k_and);
  k_or = __reduce_or_sync(0xffffffffu, k_or);
  if ((threadIdx.x & 31) == 0) {
    atomicAnd(&sh0->k_and, k_and);
    atomicOr(&sh0->k_or, k_or);
  }
  cl.sync();
  const uint32_t all_and = sh0->k_and, all_or = sh0->k_or;
  const uint32_t diff = all_and ^ all_or;
  const int hb = diff ? 31 - __clz(diff) : 0;
  const int shift = hb >= 12 ? hb - 12 : 0;
  if (diff) {
    for (int g0 = 0; g0 < n_my; g0 += blockDim.x) {
      const int g = g0 + threadIdx.x;
      if (g < n_my && gk[g] != kEmptyGroup) atomicAdd(&c.hist[(gk[g] >> shift) & (kBins - 1)], 1u);
    }
  }
  cl.sync();
  // The cluster's histogram: rank k sums slice k of the bins over the ranks
  // into its own copy of that slice (no rank reads another's slice of its
  // own bins), with the slice's total beside it; rank 0 then finds the slice
  // that holds the wanted rank, and the bin inside it.
  const int per = kBins / C, b0 = cr * per;  // C is 2, 4 or 8
  if (diff) {
    int cnt = 0;
    for (int b = b0 + threadIdx.x; b < b0 + per; b += blockDim.x) {
      uint32_t t = 0;
      for (int k = 0; k < C; ++k) t += cl.map_shared_rank(c.hist, k)[b];
      c.hist[b] = t;
      cnt += (int)t;
    }
    int slice_total;
    block_exclusive_scan(cnt, sh.scan, &slice_total);
    if (threadIdx.x == 0) sh.total = slice_total;  // the kernel keeps its own copy of the scored total
  }
  cl.sync();
  if (cr == 0) {
    uint32_t M = all_or == 0u ? kEmptyGroup : all_and;
    if (diff) {
      if (threadIdx.x == 0) {
        uint32_t above = 0;
        int hit = -1;
        for (int k = C - 1; k >= 0; --k) {  // the largest keys sit in the last slice
          const uint32_t t = (uint32_t)cl.map_shared_rank(&sh, k)->total;
          if (above + t >= (uint32_t)want) {
            hit = k;
            break;
          }
          above += t;
        }
        sh.digit[0] = (uint32_t)hit;
        sh.digit[1] = above;
      }
      __syncthreads();
      const int hit = (int)sh.digit[0];
      const uint32_t above = sh.digit[1];
      __syncthreads();
      if (hit >= 0) {
        if (hit != 0)  // that slice's merged bins, from their owner
          for (int b = threadIdx.x; b < per; b += blockDim.x) c.hist[b] = cl.map_shared_rank(c.hist, hit)[hit * per + b];
        __syncthreads();
        block_find_bin_desc(c.hist, per, (uint32_t)want - above, sh);
        const uint32_t high = shift + 13 >= 32 ? 0u : (all_and & ~((1u << (shift + 13)) - 1u));
        M = high | ((uint32_t)(hit * per + (int)sh.digit[0]) << shift);
      } else {
        M = all_and;  // fewer scored groups than wanted: every scored group qualifies
      }
    }
    if ((int)threadIdx.x < C) cl.map_shared_rank(&sh, (int)threadIdx.x)->M = M;
  }
  cl.sync();
  const uint32_t M = sh.M;
  const float Mf = key_float(M);
  // this share's qualifying groups to the front of gk, in place (a round
  // reads before it writes, and writes only reach indices already read)
  for (int base = 0; base < n_my; base += blockDim.x) {
    const int g = base + threadIdx.x;
    const bool take = g < n_my && gk[g] >= M;
    __syncthreads();
    if (take) gk[atomicAdd(&sh.n_eq, 1)] = (uint32_t)(gs0 + g);
    __syncthreads();
  }
  const int n_q = sh.n_eq;
  uint32_t* ckey0 = cl.map_shared_rank(c.ckey, 0);
  uint32_t* cpos0 = cl.map_shared_rank(c.cpos, 0);
  // gather: a warp takes 32 groups at a time, 8 lanes x float4 per group
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  for (int base = warp * 32; base < n_q; base += nw * 32) {
    int e0[8];
    float4 v[8];
    int s0[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int gi = base + u * 4 + (lane >> 3);
      e0[u] = gi < n_q ? (int)gk[gi] * 32 + (lane & 7) * 4 : -1;
    }
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      s0[u] = -1;
      v[u] = make_float4(0.f, 0.f, 0.f, 0.f);
      if (e0[u] >= 0 && e0[u] < c.n_elem) {
        const int s = (c.work[e0[u] >> c.lb] << c.lb) + (e0[u] & c.bmask);
        if (s <= c.p) {
          s0[u] = s;
          v[u] = *reinterpret_cast<const float4*>(c.sc + s);
        }
      }
    }
    const uint32_t takes = takes_at_least(v, s0, c.p, Mf);
    const int n_t = __popc(takes);
    if (!__any_sync(0xffffffffu, n_t != 0)) continue;
    int incl = n_t;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int t = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += t;
    }
    int at = 0;
    if (lane == 31) at = atomicAdd(&sh0->n_cand, incl);
    at = __shfl_sync(0xffffffffu, at, 31) + incl - n_t;
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const float vals[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        if (takes & (1u << (4 * u + k))) {
          if (at < kCandCap) {
            ckey0[at] = fkey(vals[k]);
            cpos0[at] = (uint32_t)(e0[u] + k);
          }
          ++at;
        }
      }
    }
  }
  cl.sync();  // every rank's candidates are in rank 0 before it goes on
  return cr == 0 ? sh.n_cand : -2;
}

// The sampled-threshold path spread over a cluster (contexts with fewer
// 32-slot groups than k): rank 0 takes the threshold from its sample and
// sends it to every rank; each rank then collects its share of the kept
// slots (whole blocks) straight into rank 0's candidate list.  Returns the
// candidate count in rank 0 and -2 in the other ranks, which are done.
__device__ __forceinline__ int collect_sampled_cluster(const TopkCtx& c, int want, int total, TopkShared& sh) {
  namespace cg = cooperative_groups;
  cg::cluster_group cl = cg::this_cluster();
  const int C = (int)cl.num_blocks(), cr = (int)cl.block_rank();
  if (cr == 0) {
    const uint32_t t_lo = sample_threshold(c, want, total, sh);
    if (threadIdx.x == 0) sh.n_cand = 0;
    if ((int)threadIdx.x < C) cl.map_shared_rank(&sh, (int)threadIdx.x)->M = t_lo;
  }
  cl.sync();
  const uint32_t t_lo = sh.M;
  TopkShared* sh0 = cl.map_shared_rank(&sh, 0);
  uint32_t* ckey0 = cl.map_shared_rank(c.ckey, 0);
  uint32_t* cpos0 = cl.map_shared_rank(c.cpos, 0);
  const int b0 = (int)((int64_t)c.nk * cr / C), b1 = (int)((int64_t)c.nk * (cr + 1) / C);
  const int E0 = b0 << c.lb, E1 = b1 << c.lb;  // this rank's kept-slot positions
  const int lane = threadIdx.x & 31;
  const int step = blockDim.x * 4;
  for (int it = E0; it < E1; it += 4 * step) {
    float4 v[4];
    int s0[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int e = it + threadIdx.x * 4 + u * step;
      s0[u] = -1;
      v[u] = make_float4(0.f, 0.f, 0.f, 0.f);
      if (e < E1) {
        const int s = (c.work[e >> c.lb] << c.lb) + (e & c.bmask);
        if (s <= c.p) {
          s0[u] = s;
          v[u] = *reinterpret_cast<const float4*>(c.sc + s);
        }
      }
    }
    uint32_t takes = 0;
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const float vals[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
#pragma unroll
      for (int k = 0; k < 4; ++k)
        if (s0[u] >= 0 && s0[u] + k <= c.p && fkey(vals[k]) >= t_lo) takes |= 1u << (4 * u + k);
    }
    const int n_t = __popc(takes);
    if (!__any_sync(0xffffffffu, n_t != 0)) continue;
    int incl = n_t;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int t = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += t;
    }
    int at = 0;
    if (lane == 31) at = atomicAdd(&sh0->n_cand, incl);
    at = __shfl_sync(0xffffffffu, at, 31) + incl - n_t;
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const float vals[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
      const int e0 = it + threadIdx.x * 4 + u * step;
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        if (takes & (1u << (4 * u + k))) {
          if (at < kCandCap) {
            ckey0[at] = fkey(vals[k]);
            cpos0[at] = (uint32_t)(e0 + k);
          }
          ++at;
        }
      }
    }
  }
  cl.sync();  // every rank's candidates are in rank 0 before it goes on
  return cr == 0 ? sh.n_cand : -2;
}

// kCluster: launched with a cluster of C CTAs per (request, row), which share
// the group path; otherwise one CTA per pair.
// R1B64: one row and 64-slot blocks known at compile time (the decode
// step's common case), so the position arithmetic of every pass folds.
template <bool kCluster, int R1B64 = 0>
__global__ void __launch_bounds__(kTopkThreads) k_topk(TopkArgs a) {
  pdl_enter();
  const Layout L = a.lay;
  namespace cg = cooperative_groups;
  const int C = kCluster ? (int)cg::this_cluster().num_blocks() : 1;
  const int cr = kCluster ? (int)cg::this_cluster().block_rank() : 0;
  const unsigned rid = blockIdx.x / (unsigned)C;
  const int rows = R1B64 ? 1 : a.rows;
  const int q = rid / rows, r = rid % rows;
  int32_t* out = a.topk + ((int64_t)q * rows + r) * L.k;
  __shared__ TopkShared sh;
  extern __shared__ __align__(16) uint8_t dyn[];
  const int64_t ctx = a.ctx_len[q];
  if (ctx < 1 || ctx + rows - 1 > L.max_slots || (a.ctx_sel && a.ctx_sel[q] != ctx)) {
    if (cr == 0)
      for (int t = threadIdx.x; t < L.k; t += blockDim.x) out[t] = -1;
    return;
  }
  TopkCtx c;
  c.p = (int)(ctx - 1 + r);
  c.nk = a.kept[q];
  c.work = a.work + (int64_t)q * L.blk_stride;
  c.sc = a.scores + ((int64_t)q * L.R + r) * L.slot_stride;
  c.lb = R1B64 ? 6 : __ffs(L.b) - 1;  // block size is a power of two
  c.bmask = R1B64 ? 63 : L.b - 1;
  c.n_elem = c.nk << c.lb;
  c.nwords = (c.n_elem + 31) / 32;
  c.bits = reinterpret_cast<uint32_t*>(dyn);
  c.bits_cap = (int)(topk_bitmap_bytes(L) / 4);
  uint8_t* area = dyn + topk_bitmap_bytes(L);
  c.hist = reinterpret_cast<uint32_t*>(area);
  c.ckey = reinterpret_cast<uint32_t*>(area);
  c.cpos = c.ckey + kCandCap;
  c.hist2 = c.cpos + kCandCap;

  // ---- number of scored slots; the kept-block list is staged on chip when
  // the launch reserved room for it (every later pass reads it) ------------
  {
    int32_t* staged = topk_stages_work(L) ? reinterpret_cast<int32_t*>(area + topk_area_bytes()) : nullptr;
    int cnt = 0;
    for (int t0 = 0; t0 < c.nk; t0 += 4 * blockDim.x) {  // four loads in flight per thread
      int w[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int t = t0 + u * blockDim.x + threadIdx.x;
        w[u] = t < c.nk ? c.work[t] : 0;
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int t = t0 + u * blockDim.x + threadIdx.x;
        if (t < c.nk) {
          cnt += min(max(c.p - (w[u] << c.lb) + 1, 0), L.b);
          if (staged) staged[t] = w[u];
        }
      }
    }
    if (staged) c.work = staged;  // visible to every thread after the scan's barriers
    int tot;
    block_exclusive_scan(cnt, sh.scan, &tot);
    if (threadIdx.x == 0) sh.total = tot;
    __syncthreads();
  }
  const int total = sh.total;
  const int want = min(total, L.k);
  // every rank computed the same count; the cluster shares the candidate
  // search when not everything fits on chip
  if (kCluster && cr != 0 && total <= kCandCap) return;
  if (want == 0) {
    for (int t = threadIdx.x; t < L.k; t += blockDim.x) out[t] = -1;
    return;
  }

  // ---- fast path: threshold, one collecting pass, exact select on chip ----
  bool exact_bits = false;
  uint32_t T = 0, eq_take = 0;
  {
    int n_cand = -1;
    if (total <= kCandCap) {
      n_cand = collect_ge(c, 0u, sh);  // everything fits
    } else {
      // The group path pays when the wanted scores lie in a small share of
      // the groups.  With fewer than two groups per wanted score nearly every
      // group qualifies, the candidates overflow the on-chip list, and the
      // sampled threshold below is taken anyway.
      if (a.gmax && c.nwords >= 2 * want) {
        const float* gm = a.gmax + ((int64_t)q * L.R + r) * a.gstride;
        if constexpr (kCluster) {
          n_cand = collect_from_groups_cluster(c, gm, want, sh);
          if (n_cand == -2) return;  // a helper rank of the cluster: its part is done
        } else {
          n_cand = collect_from_groups(c, gm, want, sh);
        }
      }
      if constexpr (kCluster) {
        if (!(a.gmax && c.nwords >= 2 * want)) {  // every rank takes this branch alike
          n_cand = collect_sampled_cluster(c, want, total, sh);
          if (n_cand == -2) return;
        }
      }
      if (n_cand < want || n_cand > kCandCap) n_cand = collect_ge(c, sample_threshold(c, want, total, sh), sh);
    }
    if (n_cand >= want && n_cand <= kCandCap) {
      T = select_candidates(c, n_cand, want, sh);
      exact_bits = true;
    }
  }

  if (!exact_bits) {
    // ---- exact fallback: 13-bit histogram of all keys ---------------------
    for (int i = threadIdx.x; i < kBins; i += blockDim.x) c.hist[i] = 0;
    __syncthreads();
    {
      const int step = blockDim.x * 4;
      for (int it = 0; it < c.n_elem; it += 4 * step) {
        float4 v[4];
        int s0[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int e = it + threadIdx.x * 4 + u * step;
          s0[u] = -1;
          v[u] = make_float4(0.f, 0.f, 0.f, 0.f);
          if (e < c.n_elem) {
            const int s = (c.work[e >> c.lb] << c.lb) + (e & c.bmask);
            if (s <= c.p) {
              s0[u] = s;
              v[u] = *reinterpret_cast<const float4*>(c.sc + s);
            }
          }
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const float vals[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const bool act = s0[u] >= 0 && s0[u] + k <= c.p;
            hist_add(c.hist, act ? fkey(vals[k]) >> kFirstShift : 0u, act);
          }
        }
      }
    }
    __syncthreads();
    block_find_bin_desc(c.hist, kBins, (uint32_t)want, sh);
    const uint32_t d1 = sh.digit[0];
    uint32_t remaining = sh.digit[1];
    __syncthreads();
    const int n_cand = collect_ge(c, d1 << kFirstShift, sh);
    if (n_cand <= kCandCap) {
      // exact select among the keys of bin d1 (rank `remaining` inside it)
      uint32_t prefix = d1, pbits = 32 - kFirstShift;
      const int shifts[3] = {11, 3, 0};
      const int widths[3] = {8, 8, 3};
      for (int ps = 0; ps < 3; ++ps) {
        const int shf = shifts[ps], w = widths[ps];
        for (int i = threadIdx.x; i < 256; i += blockDim.x) c.hist2[i] = 0;
        __syncthreads();
        for (int i = threadIdx.x; i < n_cand; i += blockDim.x) {
          const uint32_t k = c.ckey[i];
          if ((k >> (32 - pbits)) == prefix) atomicAdd(&c.hist2[(k >> shf) & ((1u << w) - 1u)], 1u);
        }
        __syncthreads();
        if (threadIdx.x < 32) warp_find_digit_desc<256>(c.hist2, remaining, sh.digit);  // bins >= 2^w are empty
        __syncthreads();
        prefix = (prefix << w) | sh.digit[0];
        pbits += w;
        remaining = sh.digit[1];
        __syncthreads();
      }
      T = prefix;
      for (int i = threadIdx.x; i < c.nwords; i += blockDim.x) c.bits[i] = 0;
      __syncthreads();
      for (int i = threadIdx.x; i < n_cand; i += blockDim.x)
        if (c.ckey[i] >= T) atomicOr(&c.bits[c.cpos[i] >> 5], 1u << (c.cpos[i] & 31));
      __syncthreads();
    } else {
      // three more full passes over the scores
      uint32_t prefix = d1;
      int shift_hi = kFirstShift;
      const int shifts[3] = {11, 3, 0};
      for (int ps = 0; ps < 3; ++ps) {
        const int sh_lo = shifts[ps];
        const int width = shift_hi - sh_lo;
        const uint32_t dmask = (1u << width) - 1u;
        for (int i = threadIdx.x; i < 256; i += blockDim.x) c.hist2[i] = 0;
        __syncthreads();
        for_each_scored(c, [&](int, uint32_t key) {
          if ((key >> shift_hi) == prefix) atomicAdd(&c.hist2[(key >> sh_lo) & dmask], 1u);
        });
        __syncthreads();
        if (threadIdx.x < 32) warp_find_digit_desc<256>(c.hist2, remaining, sh.digit);
        __syncthreads();
        prefix = (prefix << width) | sh.digit[0];
        remaining = sh.digit[1];
        shift_hi = sh_lo;
        __syncthreads();
      }
      T = prefix;
      for (int i = threadIdx.x; i < c.nwords; i += blockDim.x) c.bits[i] = 0;
      __syncthreads();
      for_each_scored(c, [&](int e, uint32_t key) {
        if (key >= T) atomicOr(&c.bits[e >> 5], 1u << (e & 31));
      });
      __syncthreads();
    }
    eq_take = remaining;
  }

  // ---- emission in ascending slot order --------------------------------------
  // Exact bitmaps need no score; the fallback's bitmap holds every key >= T
  // and takes the lowest-position eq_take of the keys equal to T.
  const int chunk = (c.nwords + blockDim.x - 1) / blockDim.x;
  const int w0 = threadIdx.x * chunk, w1 = min(c.nwords, w0 + chunk);
  int n_gt = 0, n_eq = 0;
  for (int w = w0; w < w1; ++w) {
    uint32_t m = c.bits[w];
    if (exact_bits) {
      n_gt += __popc(m);
      continue;
    }
    while (m) {
      const int bit = __ffs(m) - 1;
      m &= m - 1;
      const int e = w * 32 + bit;
      const int s = (c.work[e >> c.lb] << c.lb) + (e & c.bmask);
      if (fkey(c.sc[s]) > T) ++n_gt; else ++n_eq;
    }
  }
  int tot;
  const int eq_base = exact_bits ? 0 : block_exclusive_scan(n_eq, sh.scan, &tot);  // exact: no ties left
  const int take = max(0, min(n_eq, (int)eq_take - eq_base));
  int pos = block_exclusive_scan(n_gt + take, sh.scan, &tot);
  int eq_rank = eq_base;
  for (int w = w0; w < w1; ++w) {
    uint32_t m = c.bits[w];
    while (m) {
      const int bit = __ffs(m) - 1;
      m &= m - 1;
      const int e = w * 32 + bit;
      const int s = (c.work[e >> c.lb] << c.lb) + (e & c.bmask);
      if (exact_bits || fkey(c.sc[s]) > T) {
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
  return topk_bitmap_bytes(L) + topk_area_bytes() + (topk_stages_work(L) ? (size_t)L.blk_stride * 4 : 0);
}

cudaError_t launch_topk(const TopkArgs& a, cudaStream_t s) {
  const size_t smem = topk_smem_bytes(a.lay);
  cudaError_t e = cudaFuncSetAttribute(k_topk<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e == cudaSuccess) e = cudaFuncSetAttribute(k_topk<false, 1>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e == cudaSuccess) e = cudaFuncSetAttribute(k_topk<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  // Few (request, row) pairs leave most SMs idle: give each a cluster of up to
  // 8 CTAs for the candidate search.  A cluster shape the device cannot place falls
  // back to one CTA per pair.
  const int pairs = a.lay.Q * a.rows;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  int C = 1;
  while (C < 8 && pairs * C * 2 <= sms) C *= 2;
  if (C > 1) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(pairs * C));
    cfg.blockDim = dim3(kTopkThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)C;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    int clusters = 0;
    e = cudaOccupancyMaxActiveClusters(&clusters, k_topk<true>, &cfg);
    if (e == cudaSuccess && clusters >= 1) return cudaLaunchKernelEx(&cfg, k_topk<true>, a);
    cudaGetLastError();  // this shape cannot be placed: one CTA per pair
  }
  PdlLaunch l(dim3(pairs), dim3(kTopkThreads), smem, s);
  return cudaLaunchKernelEx(&l.cfg, (a.rows == 1 && a.lay.b == 64) ? k_topk<false, 1> : k_topk<false>, a);
}

}  // namespace spin
