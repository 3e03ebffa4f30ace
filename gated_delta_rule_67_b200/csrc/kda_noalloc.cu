// kda_noalloc.cu -- kda_chunk_fwd for callers that cannot allocate device memory.
//
// The bf16 chunked prefill needs a scratch workspace (the per-chunk operand
// records handed from the preparation kernel to the state pass).  Normally
// the caller allocates it.  Some callers cannot: a host program that links
// only this library and has no allocator of its own, or a plugin running
// inside a framework that owns all device memory and forbids further
// cudaMalloc calls once it has started.  For them this file keeps the
// scratch in a fixed, statically sized device array that the CUDA runtime
// creates when the library's module is loaded, so no call here allocates.
//
// Facts a caller must know:
//  * Size: kNoAllocScratchBytes (64 MiB) on every GPU that loads the library,
//    held until the process exits.  Problems whose workspace
//    (kda_chunk_fwd_workspace_size) is larger -- for bf16 at d = 128 about
//    900 chunk-heads, B * H * ceil(T / 64) -- are rejected with
//    KDA_ERR_UNSUPPORTED before anything is launched.
//  * The array's host-side name is only a stand-in for the device symbol, so
//    its device address is looked up once per device, with that device
//    current, on the first call made on that device (cudaGetSymbolAddress).
//    Make that first call before any stream capture.
//  * All calls share the one array, and it keeps the contents of the last
//    call.  Calls whose work overlaps on the GPU (two streams at once) race
//    on it and must be serialised by the caller.  The parts that must start
//    at zero (the error word) are cleared on every call; everything else is
//    fully rewritten before it is read.
//  * A bounded wait that gave up inside a kernel is recorded in the error
//    word at the start of the scratch; kda_chunk_fwd_noalloc_check reads it
//    (the caller has no other way to reach the array).
#include <mutex>

#include "kda_common.cuh"

namespace {

constexpr size_t kNoAllocScratchBytes = size_t(64) << 20;
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_kda_scratch[kNoAllocScratchBytes];

std::mutex g_setup_mutex;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of g_kda_scratch on the current device (set up once per device).
cudaError_t scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_setup_mutex);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_kda_scratch);
    if (e != cudaSuccess) return e;
    if (!p) return cudaErrorInvalidSymbol;
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return cudaSuccess;
}

}  // namespace

extern "C" KDA_API kda_status kda_chunk_fwd_noalloc(const void* q, const void* k, const void* v, const void* g,
                                                    const void* beta, float scale, const float* initial_state,
                                                    void* o, float* final_state, int B, int T, int H, int dk,
                                                    int dv, int chunk, int dtype, void* stream) {
  const size_t need = kda_chunk_fwd_workspace_size(B, T, H, dk, dv, chunk, dtype);
  if (need > kNoAllocScratchBytes) return KDA_ERR_UNSUPPORTED;
  void* scratch = nullptr;
  if (scratch_address(&scratch) != cudaSuccess) return KDA_ERR_CUDA;
  return kda_chunk_fwd(q, k, v, g, beta, scale, initial_state, o, final_state, B, T, H, dk, dv, chunk, dtype,
                       scratch, kNoAllocScratchBytes, stream);
}

extern "C" KDA_API kda_status kda_chunk_fwd_noalloc_check(void* stream) {
  void* scratch = nullptr;
  if (scratch_address(&scratch) != cudaSuccess) return KDA_ERR_CUDA;
  return kda_chunk_fwd_check(scratch, kNoAllocScratchBytes, stream);
}
