// kda_chunk_tc.cu -- placeholder until the tcgen05 kernel lands: routes the
// tensor-core configuration to the CUDA-core kernel.
#include "kda_internal.cuh"

namespace kda {

size_t tc_workspace_bytes(int, int, int, int, int) { return 0; }

cudaError_t launch_chunk_tc(const ChunkArgs& a, void*, size_t, cudaStream_t stream) {
  ChunkArgs b = a;
  b.chunk = 32;
  return launch_chunk_simt(b, stream);
}

}  // namespace kda
