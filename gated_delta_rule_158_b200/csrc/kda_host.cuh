// kda_host.cuh -- host-side pieces shared by the C entry points: the
// chunked-prefill body and the gate backward's launcher.
#pragma once

#include "kda_internal.cuh"

namespace kda {

kda_status chunk_fwd_impl(const void* q, const void* k, const void* v, const float* g,
                          const float* A_log, float g_min, const float* beta,
                          kda_dtype in_dtype, const float* init_state,
                          const int32_t* cu_seqlens, int num_seqs, int B, int T, int H, int dk,
                          int dv, float scale, int chunk_size, void* out, float* final_state,
                          void* workspace, size_t workspace_bytes, void* stream,
                          bool reset_status = true);

// Gate backward (kda_gate.cu): dz, and dA_log through per-(head, part)
// partial sums (kGateBwdMaxParts per head at most) added in a fixed order.
constexpr int kGateBwdMaxParts = 256;
int gate_bwd_parts(int64_t rows);
cudaError_t launch_gate_bwd(const float* z, const float* A_log, float g_min, const float* dg,
                            float* dz, float* dA_log, int64_t rows, int H, int dk,
                            float* partial, cudaStream_t stream);

}  // namespace kda
