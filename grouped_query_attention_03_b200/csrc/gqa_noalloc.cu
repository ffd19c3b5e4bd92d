// gqa_noalloc.cu -- single-token decode for callers that cannot allocate.
//
// gqa_decode needs a device workspace for its split-K partials, and normally
// the caller allocates it.  Some callers cannot call cudaMalloc at all: a
// host application that hands this library pointers from its own fixed
// memory pool and forbids any other allocation, a latency-critical serving
// loop where cudaMalloc's implicit device synchronisation is not acceptable,
// or a foreign-language caller that only receives device pointers from
// another component and has no allocator of its own.  gqa_decode_noalloc
// serves them: it runs exactly the gqa_decode path, with the workspace taken
// from a fixed array in device memory that this library defines.
//
// Costs and rules of the fixed array:
//   - It is GQA_NOALLOC_SCRATCH_BYTES (8 MiB).  Every GPU that loads the
//     library holds it until the process exits.
//   - Sizes whose workspace would not fit are rejected with
//     GQA_ERR_WORKSPACE before anything is enqueued.
//   - Every call on a device shares the one array, and it keeps whatever the
//     last call wrote.  The decode kernels overwrite every partial they read
//     within the same call; only the arrival counters at the start of the
//     workspace must be zero when a kernel starts.  A call that completes
//     leaves them zero, but one that gave up on a bounded wait may not, and
//     a caller of this entry point cannot reach the array to clear it, so
//     each call clears the counter region itself (a cudaMemsetAsync of a few
//     KB on the caller's stream; no allocation).  Two calls whose kernels
//     overlap on the GPU (different streams, no ordering between them) race
//     on the array and give wrong results.  Order them.
//   - The first call on each device looks up the array's device address
//     (cudaGetSymbolAddress with that device current) and caches it, keyed
//     by the device's current context; make that first call before any
//     stream capture begins.  After a cudaDeviceReset the device has a new
//     context and the module is loaded again, so the next call looks the
//     address up again (again: not inside a capture).
//   - Nothing here calls cudaMalloc, cudaFree or an allocating library.
#include <cuda.h>

#include <mutex>

#include "../../include/gqa.h"
#include "common.cuh"

namespace gqa {
namespace detail {
// gqa_decode, clearing the workspace's counter region on the stream right
// before the kernel (defined with the other entry points).
gqa_status decode_clearing_counters(gqa_dtype dtype, const void *q,
                                    const void *k_cache, const void *v_cache,
                                    void *o, const int32_t *seq_lens, int B,
                                    int Hq, int Hkv, int C, int d, int window,
                                    float scale, void *workspace,
                                    size_t workspace_bytes, int32_t *dev_status,
                                    gqa_stream_t stream);
}  // namespace detail
}  // namespace gqa

namespace {

constexpr size_t kScratchBytes = GQA_NOALLOC_SCRATCH_BYTES;

// The workspace.  In host code `g_noalloc_scratch` names a host-side shadow,
// not device memory: only the address returned by cudaGetSymbolAddress may
// be handed to a kernel.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kScratchBytes];

// Unique id of the calling thread's current context (driver entry points
// looked up through the runtime, so the library needs no libcuda link);
// false if it cannot be read.
bool current_context_id(unsigned long long *id) {
  typedef CUresult (*GetCurrentFn)(CUcontext *);
  typedef CUresult (*GetIdFn)(CUcontext, unsigned long long *);
  static GetCurrentFn get_current = nullptr;
  static GetIdFn get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *p = nullptr, *q = nullptr;
    cudaDriverEntryPointQueryResult r1, r2;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &r1) ==
            cudaSuccess &&
        r1 == cudaDriverEntryPointSuccess &&
        cudaGetDriverEntryPoint("cuCtxGetId", &q, cudaEnableDefault, &r2) ==
            cudaSuccess &&
        r2 == cudaDriverEntryPointSuccess) {
      get_current = reinterpret_cast<GetCurrentFn>(p);
      get_id = reinterpret_cast<GetIdFn>(q);
    } else {
      cudaGetLastError();
    }
  });
  CUcontext ctx = nullptr;
  return get_current && get_id && get_current(&ctx) == CUDA_SUCCESS && ctx &&
         get_id(ctx, id) == CUDA_SUCCESS;
}

// Device address of the array on the current device, looked up once per
// device and context (and on every call if the context id cannot be read).
// Returns NULL (and leaves no CUDA error pending) on failure.
void *scratch_on_current_device() {
  static std::mutex mu;
  static void *addr[64] = {};
  static unsigned long long ctx_of[64] = {};
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
    cudaGetLastError();
    return nullptr;
  }
  // With no current context yet (the caller has made no CUDA call on this
  // thread) the id is unknown and the address is looked up, which makes the
  // device's primary context current.
  unsigned long long ctx = 0;
  const bool have_ctx = current_context_id(&ctx);
  std::lock_guard<std::mutex> lock(mu);
  if (!addr[dev] || !have_ctx || ctx_of[dev] != ctx) {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) {
      cudaGetLastError();
      addr[dev] = nullptr;
      return nullptr;
    }
    addr[dev] = p;
    ctx_of[dev] = have_ctx ? ctx : 0;
  }
  return addr[dev];
}

}  // namespace

extern "C" gqa_status gqa_decode_noalloc(gqa_dtype dtype, const void *q,
                                         const void *k_cache,
                                         const void *v_cache, void *o,
                                         const int32_t *seq_lens, int B,
                                         int Hq, int Hkv, int C, int d,
                                         int window, float scale,
                                         int32_t *dev_status,
                                         gqa_stream_t stream) {
  const size_t need = gqa_decode_workspace_bytes(dtype, B, Hq, Hkv, C, d);
  if (need > kScratchBytes) return GQA_ERR_WORKSPACE;
  void *ws = scratch_on_current_device();
  if (!ws) return GQA_ERR_CUDA;
  // gqa_decode's path, with the counter region cleared on the stream after
  // every host-side check has passed and just before the kernel.
  return gqa::detail::decode_clearing_counters(
      dtype, q, k_cache, v_cache, o, seq_lens, B, Hq, Hkv, C, d, window, scale,
      ws, kScratchBytes, dev_status, stream);
}
