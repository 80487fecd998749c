// kda_host.cuh -- the chunked-prefill body shared by the C entry points.
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

}  // namespace kda
