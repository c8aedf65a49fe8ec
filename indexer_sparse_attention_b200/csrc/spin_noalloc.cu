// spin_noalloc.cu -- token top-k for callers that cannot allocate device
// memory at all.
//
// spin_topk needs a state, and a state needs a device block from the caller.
// Some callers have no way to provide one: code that runs while a CUDA graph
// is being captured (cudaMalloc is not allowed then), plug-ins whose host
// application owns every byte of device memory through its own pool, or
// embedded runtimes that forbid device allocation after start-up.  For them
// spin_topk_noalloc runs the same compaction and top-k kernels with their
// scratch (the kept-block work lists, the kept counts and an error word) in
// the fixed array below, which the library image reserves on every GPU that
// loads it.  The caller still passes scores, mask, context lengths and the
// output buffer.
#include <cstdio>
#include <mutex>

#include "spin_internal.cuh"

namespace spin {
namespace {

// 4 MiB of scratch, reserved on each device that loads the library and held
// until the process exits.  Layout (int32 units): [0, 4) error word,
// [4, 4 + Qpad) kept counts (Qpad = Q rounded up to 64), then Q work lists of
// blk_stride entries each.
constexpr int64_t kNoAllocInts = 1 << 20;
static __device__ __align__(256) int32_t g_noalloc_scratch[kNoAllocInts];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
struct Cached {
  unsigned long long ctx_id;  // unique id of the context the address belongs to
  int32_t* ptr;
};
Cached g_cache[kMaxDevices] = {};

typedef int (*CtxGetCurrentFn)(void**);
typedef int (*CtxGetIdFn)(void*, unsigned long long*);

// Unique id of the current context (cuCtxGetCurrent + cuCtxGetId through the
// runtime's driver entry points), or 0 when it cannot be read.
unsigned long long current_ctx_id() {
  static CtxGetCurrentFn get_cur = nullptr;
  static CtxGetIdFn get_id = nullptr;
  static bool tried = false;
  if (!tried) {
    tried = true;
    cudaDriverEntryPointQueryResult q1, q2;
    void* f1 = nullptr;
    void* f2 = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f1, cudaEnableDefault, &q1) == cudaSuccess &&
        q1 == cudaDriverEntryPointSuccess &&
        cudaGetDriverEntryPoint("cuCtxGetId", &f2, cudaEnableDefault, &q2) == cudaSuccess &&
        q2 == cudaDriverEntryPointSuccess) {
      get_cur = reinterpret_cast<CtxGetCurrentFn>(f1);
      get_id = reinterpret_cast<CtxGetIdFn>(f2);
    }
    cudaGetLastError();
  }
  if (!get_cur || !get_id) return 0;
  void* ctx = nullptr;
  unsigned long long id = 0;
  if (get_cur(&ctx) != 0 || !ctx || get_id(ctx, &id) != 0) return 0;
  return id;
}

// Device address of the array on the current device, resolved with that
// device current (in host code the symbol itself is only a stand-in, not a
// device address).  The address is cached per device together with the id of
// the context it was resolved in; a new context on the device (after
// cudaDeviceReset, for example) loads the module again, so the address is
// resolved again.  If the context id cannot be read, it is resolved on every
// call.
cudaError_t scratch_on_current_device(int32_t** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_mu);
  Cached& c = g_cache[dev];
  unsigned long long id = current_ctx_id();
  if (!c.ptr || id == 0 || id != c.ctx_id) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);  // makes the primary context current if needed
    if (e != cudaSuccess) return e;
    c.ptr = static_cast<int32_t*>(p);
    c.ctx_id = id ? id : current_ctx_id();
  }
  *out = c.ptr;
  return cudaSuccess;
}

}  // namespace
}  // namespace spin

using namespace spin;

extern "C" SPIN_API spin_status spin_topk_noalloc(int num_requests, int rows, int max_rows, int32_t max_slots,
                                                  int block_size, int topk, const float* scores_dev,
                                                  const uint8_t* mask_dev, const int32_t* ctx_len_dev,
                                                  int32_t* topk_dev, spin_stream_t stream) {
  if (num_requests < 1 || max_rows < 1 || max_rows > 4 || rows < 1 || rows > max_rows || max_slots < 1 || topk < 1 ||
      topk > 65536 || block_size < 16 || block_size > 256 || (block_size & (block_size - 1)))
    return SPIN_EINVAL;
  if (!scores_dev || !mask_dev || !ctx_len_dev || !topk_dev) return SPIN_EINVAL;
  Layout L{};
  L.L = 1;
  L.Q = num_requests;
  L.R = max_rows;
  L.H = 1;
  L.d = 1;
  L.b = block_size;
  L.k = topk;
  L.max_slots = max_slots;
  L.max_blocks = (max_slots + (int64_t)block_size - 1) / block_size;
  L.slot_stride = L.max_blocks * block_size;
  L.blk_stride = (L.max_blocks + 15) / 16 * 16;
  // the top-k kernel keeps one (request, row) bitmap on chip
  if ((L.slot_stride + 31) / 32 * 4 > 160 * 1024) return SPIN_EINVAL;
  const int64_t qpad = ((int64_t)num_requests + 63) / 64 * 64;
  if (4 + qpad + (int64_t)num_requests * L.blk_stride > kNoAllocInts) return SPIN_EINVAL;  // beyond the fixed scratch
  int32_t* base = nullptr;
  cudaError_t e = scratch_on_current_device(&base);
  if (e != cudaSuccess) {
    fprintf(stderr, "libspin: cudaGetSymbolAddress failed: %s\n", cudaGetErrorString(e));
    return SPIN_ECUDA;
  }
  ErrWord* err = reinterpret_cast<ErrWord*>(base);
  int32_t* kept = base + 4;
  int32_t* work = base + 4 + qpad;
  cudaStream_t s = (cudaStream_t)stream;
  // only the error word must start at zero; the work lists and counts are
  // fully rewritten by the compaction before the top-k reads them
  e = cudaMemsetAsync(err, 0, sizeof(ErrWord), s);
  if (e == cudaSuccess) e = launch_compact(L, rows, ctx_len_dev, mask_dev, work, kept, err, s);
  if (e == cudaSuccess) {
    TopkArgs a{L, rows, scores_dev, mask_dev, ctx_len_dev, work, kept, topk_dev, err, nullptr, 0};
    e = launch_topk(a, s);
  }
  if (e != cudaSuccess) {
    fprintf(stderr, "libspin: CUDA error %s\n", cudaGetErrorString(e));
    return SPIN_ECUDA;
  }
  return SPIN_OK;
}

// Reads the error word the last spin_topk_noalloc call on this device left in
// the fixed array.  Synchronises the stream first.
extern "C" SPIN_API spin_status spin_topk_noalloc_error(spin_stream_t stream, uint32_t* word_out) {
  int32_t* base = nullptr;
  cudaError_t e = scratch_on_current_device(&base);
  cudaStream_t s = (cudaStream_t)stream;
  ErrWord h{};
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e == cudaSuccess) e = cudaMemcpyAsync(&h, base, sizeof(ErrWord), cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) {
    fprintf(stderr, "libspin: CUDA error %s\n", cudaGetErrorString(e));
    return SPIN_ECUDA;
  }
  if (word_out) *word_out = h.flags;
  return h.flags ? SPIN_EDEVICE : SPIN_OK;
}
