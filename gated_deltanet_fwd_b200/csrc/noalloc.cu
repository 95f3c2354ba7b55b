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
// so every call looks up the array's device address on the current device with
// cudaGetSymbolAddress (a lookup that allocates nothing).  Looking it up on every call rather
// than caching it keeps the address right after a cudaDeviceReset, which reloads the module.
#include "gdn_internal.cuh"

namespace {

constexpr size_t kNoAllocScratchBytes = GDN_NOALLOC_SCRATCH_BYTES;
static_assert(kNoAllocScratchBytes % 256 == 0, "scratch keeps the workspace alignment");

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

// Device address of g_noalloc_scratch on the current device.
cudaError_t scratch_address(void** out) {
  void* p = nullptr;
  cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
  if (e != cudaSuccess) return e;
  *out = p;
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
