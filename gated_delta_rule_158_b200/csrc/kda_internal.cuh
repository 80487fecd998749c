// kda_internal.cuh -- shared declarations of libkda's kernels and launchers.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/kda.h"

namespace kda {

// ---------------------------------------------------------------- workspace
// The first 256 bytes of every workspace: the device status block.
struct StatusBlock {
  int32_t status;     // first kda_status recorded on the device (0 = OK)
  int32_t detail;     // block index (or other code-specific value)
  int32_t never_set;  // a flag nothing writes (bounded-wait self test)
  int32_t seqlens_ok; // varlen plan verdict: 1 valid, 0 invalid
  int32_t pad[60];
};
static_assert(sizeof(StatusBlock) == 256, "status block is 256 bytes");

constexpr size_t kStatusBytes = 256;

__device__ __forceinline__ void record_status(StatusBlock* sb, int32_t code,
                                              int32_t detail) {
  if (sb == nullptr) return;
  if (atomicCAS(&sb->status, 0, code) == 0) atomicExch(&sb->detail, detail);
}

// Device bounds checks of the KDA_DEBUG_CHECKS build: an index outside
// [0, limit) records KDA_ERR_BOUNDS with the check site as detail and the
// caller skips the access.  Release builds compile the check away (true).
__device__ __forceinline__ bool in_bounds(StatusBlock* sb, int64_t idx, int64_t limit,
                                          int32_t site) {
#ifdef KDA_DEBUG_CHECKS
  if (idx >= 0 && idx < limit) return true;
  record_status(sb, KDA_ERR_BOUNDS, site);
  return false;
#else
  (void)sb; (void)idx; (void)limit; (void)site;
  return true;
#endif
}

// check sites (the detail recorded with KDA_ERR_BOUNDS)
enum BoundsSite : int32_t {
  kSiteSelftest = 0x5E1F,
  kSiteTcUnitRows = 0xB101,    // chunk_tc_kernel: a unit's rows within the batch
  kSiteTcStateSlot = 0xB102,   // chunk_tc_kernel: init / final / segment state slot
  kSiteTcOutRows = 0xB103,     // chunk_tc_kernel: rows of o a chunk stores
  kSiteSimtUnitRows = 0xB201,  // chunk_simt_kernel: a unit's rows
  kSiteSimtStateSlot = 0xB202, // chunk_simt_kernel: state slot
  kSiteBwdUnitRows = 0xB401,   // backward: a unit's rows within the batch
  kSiteBwdChunks = 0xB402,     // backward: a unit's chunk slice of the workspace
};

// --------------------------------------------------------------- element io
template <typename T> struct Elem;
template <> struct Elem<float> {
  static __device__ __forceinline__ float load(const float* p) { return *p; }
  static __device__ __forceinline__ void store(float* p, float x) { *p = x; }
};
template <> struct Elem<__nv_bfloat16> {
  static __device__ __forceinline__ float load(const __nv_bfloat16* p) {
    return __bfloat162float(*p);
  }
  static __device__ __forceinline__ void store(__nv_bfloat16* p, float x) {
    *p = __float2bfloat16_rn(x);
  }
};

// ---------------------------------------------------------- unit addressing
// A "unit" is one (sequence, head) pair processed start to end by one CTA.
// Dense batches: sequence b spans rows [b*T, b*T + T) of the [B*T, H, *]
// view.  Varlen: sequence n spans [cu[n], cu[n+1]).
struct UnitMap {
  const int32_t* cu_seqlens;  // nullptr = dense
  const int32_t* order;       // varlen processing order (longest first) or nullptr
  const StatusBlock* status;  // varlen validity verdict lives here
  int B, T, H;
};

// Launchers (host side).  All return cudaSuccess or the launch error.
cudaError_t launch_gate(const float* z, const float* A_log, float g_min,
                        float* g, int64_t rows, int H, int dk,
                        cudaStream_t stream);

// g_or_z is g, or z when A_log != nullptr (gate fused into the kernel)
cudaError_t launch_decode(const void* q, const void* k, const void* v,
                          const float* g_or_z, const float* A_log, float g_min,
                          const float* beta, kda_dtype dt, float* state, int N,
                          int H, int dk, int dv, float scale, void* out,
                          cudaStream_t stream);

struct DecodeMultiArgs {
  const void* q;
  const void* k;
  const void* v;
  const float* g;      // log-decay g, or z when A_log is set
  const float* A_log;  // nullable
  float g_min;
  const float* beta;
  kda_dtype dt;
  float* state;
  const int32_t* accept_len;  // replay only
  void* out;                  // verify only
  int N, H, K, dk, dv;
  float scale;
};

int decode_multi_max_tokens();
cudaError_t launch_decode_multi(const DecodeMultiArgs& a, bool verify, cudaStream_t stream);

__device__ __forceinline__ float gate_value(float z, float a, float g_min) {
  return g_min / (1.0f + expf(-a * z));
}

cudaError_t launch_varlen_plan(const int32_t* cu_seqlens, int num_seqs, int T,
                               int32_t* order, StatusBlock* sb,
                               cudaStream_t stream);

struct ChunkArgs {
  const void* q;
  const void* k;
  const void* v;
  const float* g;       // log-decay g, or z when `gated`
  const float* A_log;   // gated only: per-head gate parameter
  float g_min;          // gated only
  bool gated;           // g = g_min * sigmoid(exp(A_log[h]) * z) formed in-kernel
  const float* beta;
  kda_dtype dt;
  const float* init_state;
  float* final_state;
  void* out;
  UnitMap map;
  int num_units;  // sequences * H
  int dk, dv;
  float scale;
  int chunk;
  StatusBlock* sb;
};

cudaError_t launch_chunk_simt(const ChunkArgs& a, cudaStream_t stream);

// fp32-accurate chunkwise forward on warp-level tensor-core products with
// split tf32 operands (fp32 inputs, or dk / dv other than 128; chunk 32):
// the workspace tail it needs after the status word and the varlen order,
// and its launcher (two kernels: every chunk's key-side matrices, then the
// state scan with the outputs).
size_t chunk_f32_tail_bytes(int B, int T, int H, int num_seqs);
cudaError_t launch_chunk_f32(const ChunkArgs& a, void* ws_tail, cudaStream_t stream);

// tcgen05 tensor-core path (bf16, dk = dv = 128, chunk 32).
size_t tc_workspace_bytes(int B, int T, int H, int num_seqs, int num_sms);
cudaError_t launch_chunk_tc(const ChunkArgs& a, void* ws_tail,
                            size_t ws_tail_bytes, cudaStream_t stream);

// Cross-device context parallelism: per (sequence, head) unit of the whole
// [B, T] range, S~ (from a zero state) and M (the segment's transition) into
// pairs[unit] = {S~, M}; and the incoming state of segment `index` of `count`.
cudaError_t launch_chunk_tc_transition(const ChunkArgs& a, float* pairs, cudaStream_t stream);
cudaError_t launch_state_prefix(const float* pairs, int count, int index, const float* init,
                                int units, float* state_out, cudaStream_t stream);

// Bound of every mbarrier wait in the tensor-core chunk kernel (diagnostics).
void set_wait_limit_ns(long long ns);

cudaError_t launch_selftest_bounds(StatusBlock* sb, cudaStream_t stream);
cudaError_t launch_selftest_wait(StatusBlock* sb, long long limit_ns,
                                 cudaStream_t stream);

int device_sm_count();

// Remembers the CUDA error behind a KDA_ERR_CUDA return (per host thread).
kda_status cuda_failure(cudaError_t e);
const char* last_cuda_error_text();

}  // namespace kda
