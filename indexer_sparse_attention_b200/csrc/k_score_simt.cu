// k_score_simt.cu -- a0 query quantisation and the CUDA-core indexer score.
//
// a0: each (row, head) query vector is quantised to E4M3 with a power-of-two
//     scale 2^e, e = smallest integer with amax <= 448 * 2^e, and the scale is
//     folded into the head weight (ReLU(c x) = c ReLU(x) for c > 0), so the
//     FP8 indexer computes the same score.  The pages give no precision; this
//     is the reading used throughout.
// a3: I_{r,s} = sigma_s * sum_h w'_{r,h} * ReLU(q8_{r,h} . k8_s) over the slots
//     of kept blocks with s <= p_r (SPIN listing, Abstract; SPIN digest,
//     arXiv深度剖析: the indexer input is pruned to the kept blocks).  fp32 keys:
//     I = sum_h w_{r,h} ReLU(q_{r,h} . k_s).  This kernel serves the fp32-key
//     workloads and any shape the tensor-core kernel does not take, and is the
//     cross-check of the tensor-core kernel.
#include <algorithm>

#include "spin_internal.cuh"

namespace spin {

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

// One warp per (request, row, head).
__global__ void __launch_bounds__(256) k_quantize_q(ScoreArgs a) {
  const Layout L = a.lay;
  const int64_t nvec = (int64_t)L.Q * a.rows * L.H;
  const int lane = threadIdx.x & 31;
  const int64_t v = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (v >= nvec) return;
  const int64_t base = v * L.d;
  float amax = 0.0f;
  for (int i = lane; i < L.d; i += 32) amax = fmaxf(amax, fabsf(load_q(a.q, base + i, a.q_bf16)));
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  const int e = q_exponent(amax);
  // x * 2^-e, split in two exact steps when 2^-e is not a normal float.
  const int ne = -e;
  const int s1 = ne > 127 ? 127 : ne;
  const int s2 = ne - s1;
  const float f1 = pow2f(s1), f2 = pow2f(s2);
  for (int i = 2 * lane; i < L.d; i += 64) {
    float x0 = load_q(a.q, base + i, a.q_bf16) * f1 * f2;
    float x1 = (i + 1 < L.d) ? load_q(a.q, base + i + 1, a.q_bf16) * f1 * f2 : 0.0f;
    __nv_fp8x2_storage_t p = __nv_cvt_float2_to_fp8x2(make_float2(x0, x1), __NV_SATFINITE, __NV_E4M3);
    a.q8[base + i] = (uint8_t)(p & 0xFF);
    if (i + 1 < L.d) a.q8[base + i + 1] = (uint8_t)(p >> 8);
  }
  if (lane == 0) {
    // w * 2^e rounded once (double holds the exact product).
    a.wq[v] = __double2float_rn((double)a.w[v] * ldexp(1.0, e));
  }
}

cudaError_t launch_quantize_q(const ScoreArgs& a, cudaStream_t s) {
  const int64_t nvec = (int64_t)a.lay.Q * a.rows * a.lay.H;
  k_quantize_q<<<(unsigned)((nvec + 7) / 8), 256, 0, s>>>(a);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// SIMT score: grid (request, G); a CTA walks kept blocks t = blockIdx.y,
// +gridDim.y, ... of its request.  Queries (decoded to fp32) and one key page
// sit in shared memory; 4 threads per slot split the heads, then reduce.
// ---------------------------------------------------------------------------
constexpr int kSimtThreads = 256;
constexpr int kSimtTPS = 4;  // threads per slot

__global__ void __launch_bounds__(kSimtThreads) k_score_simt(ScoreArgs a) {
  const Layout L = a.lay;
  const int q = blockIdx.x;
  const int64_t ctx = a.ctx_len[q];
  if (ctx < 1 || ctx + a.rows - 1 > L.max_slots) return;  // reported by compaction / select
  const int nk = a.kept[q];
  if ((int)blockIdx.y >= nk) return;
  extern __shared__ __align__(16) float sm[];
  const int Hd = L.H * L.d;
  const int kpad = L.d + 1;
  float* qs = sm;                         // [rows][H][d]
  float* ws = qs + a.rows * Hd;           // [rows][H]
  float* ks = ws + a.rows * L.H;          // [b][d+1]
  for (int i = threadIdx.x; i < a.rows * Hd; i += blockDim.x) {
    const int64_t g = (int64_t)q * a.rows * Hd + i;
    qs[i] = a.key_fp8 ? e4m3x2_to_float2((uint16_t)a.q8[g]).x : reinterpret_cast<const float*>(a.q)[g];
  }
  for (int i = threadIdx.x; i < a.rows * L.H; i += blockDim.x) {
    const int64_t g = (int64_t)q * a.rows * L.H + i;
    ws[i] = a.key_fp8 ? a.wq[g] : a.w[g];
  }
  const int tps_lane = threadIdx.x % kSimtTPS;
  const int slot_lane = threadIdx.x / kSimtTPS;
  const int slots_per_pass = kSimtThreads / kSimtTPS;
  const int32_t* work = a.work + (int64_t)q * L.blk_stride;
  for (int t = blockIdx.y; t < nk; t += gridDim.y) {
    const int j = work[t];
    const int page = a.block_table[(int64_t)q * a.bt_stride + j];
    if (page < 0 || page >= a.num_pages) {
      if (threadIdx.x == 0) raise_error(a.err, ERR_PAGE, q, (uint32_t)page);
      continue;
    }
    __syncthreads();  // previous page fully consumed
    for (int i = threadIdx.x; i < L.b * L.d; i += blockDim.x) {
      const int sl = i / L.d, c = i % L.d;
      const int64_t g = ((int64_t)page * L.b + sl) * L.d + c;
      float v;
      if (a.key_fp8) v = e4m3x2_to_float2((uint16_t)reinterpret_cast<const uint8_t*>(a.keys)[g]).x;
      else v = reinterpret_cast<const float*>(a.keys)[g];
      ks[sl * kpad + c] = v;
    }
    __syncthreads();
    for (int sl0 = 0; sl0 < L.b; sl0 += slots_per_pass) {
      const int sl = sl0 + slot_lane;
      const int64_t s = (int64_t)j * L.b + sl;
      float acc[4] = {0.f, 0.f, 0.f, 0.f};
      if (sl < L.b) {
        const float* kr = ks + sl * kpad;
        for (int h = tps_lane; h < L.H; h += kSimtTPS) {
          for (int r = 0; r < a.rows; ++r) {
            const float* qr = qs + (r * L.H + h) * L.d;
            float dot = 0.f;
            for (int c = 0; c < L.d; ++c) dot = __fmaf_rn(qr[c], kr[c], dot);
            acc[r] = __fmaf_rn(ws[r * L.H + h], fmaxf(dot, 0.0f), acc[r]);
          }
        }
      }
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        acc[r] += __shfl_xor_sync(0xffffffffu, acc[r], 1);
        acc[r] += __shfl_xor_sync(0xffffffffu, acc[r], 2);
      }
      if (sl < L.b && tps_lane == 0) {
        const float sigma = a.key_fp8 ? a.kscale[(int64_t)page * L.b + sl] : 1.0f;
        for (int r = 0; r < a.rows; ++r) {
          if (s > ctx - 1 + r) continue;
          const float score = a.key_fp8 ? acc[r] * sigma : acc[r];
          a.scores[((int64_t)q * L.R + r) * L.slot_stride + s] = score;
          if (a.V && r == 0) {  // fused EMA (single row)
            float* V = a.V + (int64_t)q * L.slot_stride;
            float* D = a.D + (int64_t)q * L.slot_stride;
            V[s] = ema_v(V[s], score, a.alpha, a.beta);
            const int64_t dlt = ctx - 1 - s;
            D[dlt] = ema_d(D[dlt], score, a.alpha, a.beta);
          }
        }
      }
    }
  }
}

cudaError_t launch_score_simt(const ScoreArgs& a, cudaStream_t s) {
  const Layout& L = a.lay;
  const size_t smem = sizeof(float) * ((size_t)a.rows * L.H * L.d + (size_t)a.rows * L.H +
                                       (size_t)L.b * (L.d + 1));
  cudaError_t e = cudaFuncSetAttribute(k_score_simt, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  int64_t gy = (4 * 148 + L.Q - 1) / L.Q;
  gy = std::max<int64_t>(1, std::min<int64_t>(gy, L.max_blocks));
  dim3 grid(L.Q, (unsigned)gy);
  k_score_simt<<<grid, kSimtThreads, smem, s>>>(a);
  return cudaGetLastError();
}

}  // namespace spin
