// noalloc.cu -- gdn_chunk_fwd for callers that cannot allocate device memory.
//
// Some callers hold only device pointers that another runtime handed them and have no allocator
// they may use during a call: a kernel plugin inside an inference engine that plans all device
// memory ahead and forbids allocation while a forward pass runs (cudaMalloc can synchronise the
// device and stall the engine's other streams), or a host that keeps a fixed device-memory budget
// and owns every buffer.  Those callers cannot provide gdn_chunk_fwd's workspace, so this entry
// point takes the scratch from a fixed array that lives in the library itself instead.
//
// The array is a file-scope __device__ variable: every GPU that loads the library holds it until
// the process exits.  In host code its name is only a host-side stand-in, not a device address,
// so the device address is looked up with cudaGetSymbolAddress once per device (with that device
// current) and cached; that lookup happens on the first call on each device.
#include <mutex>

#include "gdn_internal.cuh"

namespace {

constexpr size_t kNoAllocScratchBytes = 64 * 1024;  // GDN_NOALLOC_SCRATCH_BYTES in gdn.h
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

std::mutex g_scratch_mutex;
void* g_scratch_addr[kMaxDevices] = {};

// Device address of g_noalloc_scratch on the current device, looked up once per device.
cudaError_t scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_scratch_mutex);
  if (!g_scratch_addr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return cudaSuccess;
}

}  // namespace

extern "C" gdn_status gdn_chunk_fwd_noalloc(const void* q, const void* k, const void* v,
                                            const float* g, const float* beta, gdn_dtype dtype,
                                            float scale, const float* initial_state,
                                            const int32_t* cu_seqlens, int N, int B, int64_t T,
                                            int Hk, int Hv, int dk, int dv, int chunk, void* out,
                                            float* final_state, void* stream) {
  const size_t need = gdn_chunk_fwd_workspace_size(N, B, T, Hk, Hv, dk, dv, chunk);
  if (need > kNoAllocScratchBytes) return GDN_ERR_UNSUPPORTED;
  void* scratch = nullptr;
  if (scratch_address(&scratch) != cudaSuccess) return GDN_ERR_CUDA;
  // gdn_chunk_fwd clears the status word at the front of the scratch before its kernel runs,
  // so what an earlier call left in the array does not matter.
  return gdn_chunk_fwd(q, k, v, g, beta, dtype, scale, initial_state, cu_seqlens, N, B, T, Hk, Hv,
                       dk, dv, chunk, out, final_state, scratch, kNoAllocScratchBytes, stream);
}
