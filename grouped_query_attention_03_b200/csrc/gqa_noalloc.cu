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
//     last call wrote.  The decode kernels overwrite every workspace byte they
//     read within the same call, so nothing has to start at zero; but two
//     calls whose kernels overlap on the GPU (different streams, no ordering
//     between them) race on the array and give wrong results.  Order them.
//   - The first call on each device looks up the array's device address
//     (cudaGetSymbolAddress with that device current) and caches it; make
//     that first call before any stream capture begins.
//   - Nothing here calls cudaMalloc, cudaFree or an allocating library.
#include <mutex>

#include "../../include/gqa.h"
#include "common.cuh"

namespace {

constexpr size_t kScratchBytes = GQA_NOALLOC_SCRATCH_BYTES;

// The workspace.  In host code `g_noalloc_scratch` names a host-side shadow,
// not device memory: only the address returned by cudaGetSymbolAddress may
// be handed to a kernel.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kScratchBytes];

// Device address of the array on the current device, looked up once per
// device.  Returns NULL (and leaves no CUDA error pending) on failure.
void *scratch_on_current_device() {
  static std::mutex mu;
  static void *addr[64] = {};
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
    cudaGetLastError();
    return nullptr;
  }
  std::lock_guard<std::mutex> lock(mu);
  if (!addr[dev]) {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) {
      cudaGetLastError();
      return nullptr;
    }
    addr[dev] = p;
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
  return gqa_decode(dtype, q, k_cache, v_cache, o, seq_lens, B, Hq, Hkv, C, d,
                    window, scale, ws, kScratchBytes, dev_status, stream);
}
