// kda_noalloc.cu -- kda_chunk_fwd for callers that cannot allocate device memory.
//
// Some callers of libkda have no way to hand it a workspace: an inference
// engine plugin that may only use the memory its host engine planned before
// serving starts, a service whose allocator is locked after warm-up so that
// latency never depends on cudaMalloc or on fragmentation, or a caller with a
// fixed device-memory budget fixed at start-up.  kda_chunk_fwd_noalloc gives
// them the chunkwise forward without any allocation: its scratch (device
// status word, varlen processing order, long-sequence segment states) is a
// file-scope __device__ array compiled into the library, and it otherwise
// runs exactly the kda_chunk_fwd path.
//
// Costs and rules of that choice:
//  - every GPU on which the library's module is loaded holds the array
//    (KDA_NOALLOC_SCRATCH_BYTES) until the process exits;
//  - all calls share the one array: calls whose GPU work overlaps (other
//    streams, other host threads) race on it and must be serialised by the
//    caller; each call clears the status word it needs to start at zero;
//  - problems whose scratch would exceed the array are rejected on the host
//    with KDA_ERR_WORKSPACE before anything is enqueued;
//  - the device address of the array is looked up (cudaGetSymbolAddress) on
//    the first call made on each device, with that device current; make that
//    first call before any stream capture begins.  cudaDeviceReset destroys
//    the context that held the array; the next call on that device sees a new
//    context (its driver-assigned ID differs) and looks the address up again;
//  - device-side status (a timeout, malformed cu_seqlens) lands in the
//    array's first 256 bytes, which kda_noalloc_get_device_status reads.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <mutex>

#include "kda_internal.cuh"

namespace {

static __device__ __align__(256) unsigned char g_noalloc_scratch[KDA_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
struct ScratchSlot {
  unsigned long long ctx_id;  // driver ID of the context the address belongs to
  void* addr;
};
ScratchSlot g_slots[kMaxDevices] = {};
std::mutex g_scratch_mu;

// The driver-assigned ID of the calling thread's current context (IDs are
// never reused within a process).  False when there is none or the driver
// predates cuCtxGetId; the address is then looked up on every call.
bool current_context_id(unsigned long long* id) {
  static const auto get_current = []() {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    return (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
               ? reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(p)
               : nullptr;
  }();
  static const auto get_id = []() {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    return (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
               ? reinterpret_cast<PFN_cuCtxGetId_v12000>(p)
               : nullptr;
  }();
  if (!get_current || !get_id) return false;
  CUcontext ctx = nullptr;
  if (get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr) return false;
  return get_id(ctx, id) == CUDA_SUCCESS;
}

// In host code g_noalloc_scratch names a host-side stand-in, not device
// memory.  Set-up, once per device and context, with that device current:
// look the device address up and keep it for later calls.
cudaError_t scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  unsigned long long id = 0;
  bool have_id = current_context_id(&id);
  ScratchSlot& s = g_slots[dev];
  if (s.addr == nullptr || !have_id || s.ctx_id != id) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);  // also makes the context current
    if (e != cudaSuccess) return e;
    if (!have_id) have_id = current_context_id(&id);
    s.addr = p;
    s.ctx_id = have_id ? id : 0;
    if (!have_id) {  // no context ID to key on: do not keep the address
      *out = p;
      s.addr = nullptr;
      return cudaSuccess;
    }
  }
  *out = s.addr;
  return cudaSuccess;
}

}  // namespace

extern "C" kda_status kda_chunk_fwd_noalloc(const void* q, const void* k, const void* v,
                                            const float* g, const float* beta,
                                            kda_dtype in_dtype, const float* init_state,
                                            const int32_t* cu_seqlens, int num_seqs, int B,
                                            int T, int H, int dk, int dv, float scale,
                                            int chunk_size, void* out, float* final_state,
                                            void* stream) {
  void* scratch = nullptr;
  if (cudaError_t e = scratch_address(&scratch)) return kda::cuda_failure(e);
  // kda_chunk_fwd checks every argument and returns KDA_ERR_WORKSPACE, with
  // nothing enqueued, when the problem needs more scratch than the array holds.
  return kda_chunk_fwd(q, k, v, g, beta, in_dtype, init_state, cu_seqlens, num_seqs, B, T, H,
                       dk, dv, scale, chunk_size, out, final_state, scratch,
                       (size_t)KDA_NOALLOC_SCRATCH_BYTES, stream);
}

extern "C" kda_status kda_noalloc_get_device_status(int32_t* detail, void* stream) {
  void* scratch = nullptr;
  if (cudaError_t e = scratch_address(&scratch)) return kda::cuda_failure(e);
  // the status block is the first 256 bytes of the scratch, as of a workspace
  return kda_get_device_status(scratch, stream, detail);
}
