// kda_bwd.cuh -- declarations of the backward kernel's launcher.
#pragma once

#include "kda_internal.cuh"

namespace kda {

// Backward through the recurrence (fp32): per (sequence, head) the gradients
// of q, k, v, g, beta and the initial state.
struct BwdArgs {
  const void* q;
  const void* k;
  const void* v;
  const float* g;
  const float* beta;
  const float* init;    // nullable: zero initial state
  const void* dout;     // same element type as q
  const float* dfinal;  // nullable: no gradient on the final state
  const int32_t* cu_seqlens;  // nullable: dense batch
  int num_seqs;               // sequences of a packed batch
  kda_dtype dt;
  int B, T, H, dk_dim, dv_dim;
  float scale;
  float* dq;
  float* dk;
  float* dv;
  float* dg;
  float* dbeta;
  float* dinit;  // nullable
  void* ws;      // bwd_chunk_workspace_bytes(B, T, H, dk, dv, num_seqs), 16-byte aligned
};

// In chunk form (kda_bwd_chunk.cu): a forward pass saving chunk-start states,
// a reverse pass of the state gradient, then every chunk's token gradients in
// parallel.
size_t bwd_chunk_workspace_bytes(int B, int T, int H, int dk, int dv, int num_seqs);
cudaError_t launch_bwd_chunk(const BwdArgs& a, cudaStream_t stream);

}  // namespace kda
