// k_score_simt.cu -- a0 query quantisation and the CUDA-core indexer score.
//
// a0: each (row, head) query vector is quantised to E4M3 with a power-of-two
//     scale folded into the head weight (quantize_vec); the decode step does
//     this inside its predict or select kernel, the standalone score call and
//     the pipelined decode step (spin_set_lookahead) here.
// a3: I_{r,s} = sigma_s * sum_h w'_{r,h} * ReLU(q8_{r,h} . k8_s) over the slots
//     of kept blocks with s <= p_r (SPIN listing, Abstract; SPIN digest,
//     arXiv深度剖析: the indexer input is pruned to the kept blocks).  fp32 keys:
//     I = sum_h w_{r,h} ReLU(q_{r,h} . k_s).  This kernel serves the fp32-key
//     workloads and any shape the tensor-core kernel does not take, and is the
//     cross-check of the tensor-core kernel.
#include <algorithm>

#include "spin_internal.cuh"

namespace spin {

// One warp per (request, row, head).
__global__ void __launch_bounds__(256) k_quantize_q(ScoreArgs a) {
  pdl_enter();  // q8 and wq may still be read by the previous score launch
  const Layout L = a.lay;
  const int64_t nvec = (int64_t)L.Q * a.rows * L.H;
  const int64_t v = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (v >= nvec) return;
  quantize_vec(a.q, a.w, a.q_bf16, L.d, v, a.q8, a.wq);
}

cudaError_t launch_quantize_q(const ScoreArgs& a, cudaStream_t s) {
  const int64_t nvec = (int64_t)a.lay.Q * a.rows * a.lay.H;
  PdlLaunch l(dim3((unsigned)((nvec + 7) / 8)), dim3(256), 0, s);
  return cudaLaunchKernelEx(&l.cfg, k_quantize_q, a);
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
    if (a.vmax) {  // kernel-uniform: the block's 32-slot groups of V, after its update
      __syncthreads();
      const int lane = threadIdx.x & 31;
      const float* V = a.V + (int64_t)q * L.slot_stride + (int64_t)j * L.b;
      for (int g = threadIdx.x >> 5; g < L.b / 32; g += kSimtThreads / 32) {
        const float x = warp_max(V[g * 32 + lane]);
        if (lane == 0) a.vmax[(int64_t)q * L.vg_stride + (((int64_t)j * L.b) >> 5) + g] = x;
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
