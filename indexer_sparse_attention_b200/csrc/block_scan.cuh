// block_scan.cuh -- small block-wide primitives (scan, radix digit search).
#pragma once
#include <cuda_runtime.h>
#include <stdint.h>

namespace spin {

__device__ __forceinline__ int warp_inclusive_scan(int v) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    int t = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += t;
  }
  return v;
}

// Exclusive scan over the block; `tmp` holds >= 33 ints of shared memory.
// Returns this thread's exclusive prefix; *total gets the block sum.  All
// threads of the block must call it.
__device__ __forceinline__ int block_exclusive_scan(int v, int* tmp, int* total) {
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  const int nw = (blockDim.x + 31) >> 5;
  int inc = warp_inclusive_scan(v);
  if (lane == 31) tmp[wid] = inc;
  __syncthreads();
  if (wid == 0) {
    int x = lane < nw ? tmp[lane] : 0;
    int xi = warp_inclusive_scan(x);
    if (lane < nw) tmp[lane] = xi - x;
    if (lane == 31) tmp[32] = xi;
  }
  __syncthreads();
  int r = tmp[wid] + inc - v;
  *total = tmp[32];
  __syncthreads();
  return r;
}

// Given a histogram `hist` of NB bins (NB = 32 * BPL) and a 1-based rank
// `want` counted from the top bin down, one warp finds the bin holding that
// rank and the rank left inside it.  Only warp 0 calls it; results go to
// out[0] (bin) and out[1] (remaining rank).
template <int NB>
__device__ __forceinline__ void warp_find_digit_desc(const uint32_t* hist, uint32_t want,
                                                     uint32_t* out) {
  constexpr int BPL = NB / 32;
  const int lane = threadIdx.x & 31;
  const int hi = NB - 1 - lane * BPL;  // this lane covers bins hi .. hi-BPL+1
  uint32_t s = 0;
#pragma unroll 4
  for (int i = 0; i < BPL; ++i) s += hist[hi - i];
  uint32_t inc = s;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    uint32_t t = __shfl_up_sync(0xffffffffu, inc, o);
    if (lane >= o) inc += t;
  }
  uint32_t exc = inc - s;
  if (exc < want && want <= inc) {
    uint32_t cum = exc;
    for (int i = 0; i < BPL; ++i) {
      uint32_t c = hist[hi - i];
      if (cum + c >= want) {
        out[0] = (uint32_t)(hi - i);
        out[1] = want - cum;
        break;
      }
      cum += c;
    }
  }
}

}  // namespace spin
