// kda_api.cu -- the C ABI of libkda: host-side argument checks, workspace
// layout, path selection and launches.  The contract of every entry point is
// in include/kda.h.
#include <math.h>
#include <stdio.h>
#include <string.h>

#include "kda_internal.cuh"
#include "kda_bwd.cuh"
#include "kda_host.cuh"
#include "kda_sync.cuh"

namespace kda {

namespace {
thread_local cudaError_t t_last_cuda_error = cudaSuccess;
}

kda_status cuda_failure(cudaError_t e) {
  t_last_cuda_error = e;
  return KDA_ERR_CUDA;
}

const char* last_cuda_error_text() {
  thread_local char buf[256];
  snprintf(buf, sizeof(buf), "%s: %s", cudaGetErrorName(t_last_cuda_error),
           cudaGetErrorString(t_last_cuda_error));
  return buf;
}

int device_sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
    return 148;
  return n;
}

namespace {

// ---------------------------------------------------------------- varlen plan
// Validates cu_seqlens on the device and orders sequences longest first, so
// the longest (sequence, head) units start in the first wave.  One CTA; the
// order is a rank count, O(N^2), done only for N <= kMaxSortSeqs (larger
// batches keep their given order).
constexpr int kMaxSortSeqs = 8192;

__global__ void varlen_plan_kernel(const int32_t* __restrict__ cu, int N, int T,
                                   int32_t* __restrict__ order, StatusBlock* sb) {
  __shared__ int bad;
  if (threadIdx.x == 0) bad = (cu[0] != 0 || cu[N] != T) ? 1 : 0;
  __syncthreads();
  for (int n = threadIdx.x; n < N; n += blockDim.x)
    if (cu[n + 1] < cu[n]) atomicOr(&bad, 1);
  __syncthreads();
  if (bad) {
    if (threadIdx.x == 0) {
      sb->seqlens_ok = 0;
      record_status(sb, KDA_ERR_BAD_SEQLENS, 0);
    }
    return;
  }
  for (int n = threadIdx.x; n < N; n += blockDim.x) {
    if (N > kMaxSortSeqs) {
      order[n] = n;
      continue;
    }
    const int Ln = cu[n + 1] - cu[n];
    int rank = 0;
    for (int m = 0; m < N; ++m) {
      const int Lm = cu[m + 1] - cu[m];
      rank += (Lm > Ln) || (Lm == Ln && m < n);
    }
    order[rank] = n;
  }
  if (threadIdx.x == 0) sb->seqlens_ok = 1;
}

// ------------------------------------------------------ bounded-wait selftest
__global__ void selftest_wait_kernel(StatusBlock* sb, long long limit_ns) {
  if (threadIdx.x != 0) return;
  bounded_flag_wait(&sb->never_set, limit_ns, sb, (int32_t)blockIdx.x);
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool dim_ok(int d) { return d == 32 || d == 64 || d == 128; }

size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

bool use_tc_path(kda_dtype dt, int dk, int dv, int chunk) {
  return dt == KDA_BF16 && dk == 128 && dv == 128 && (chunk == 0 || chunk == 32);
}

// Everything else with the default chunk takes the fp32-accurate chunk form
// on warp-level tensor-core products; an explicit chunk of 16 or 64 takes
// the CUDA-core kernel (the only one built for those chunk sizes).
bool use_f32_path(int chunk) { return chunk == 0 || chunk == 32; }

}  // namespace

cudaError_t launch_varlen_plan(const int32_t* cu_seqlens, int num_seqs, int T, int32_t* order,
                               StatusBlock* sb, cudaStream_t stream) {
  varlen_plan_kernel<<<1, 1024, 0, stream>>>(cu_seqlens, num_seqs, T, order, sb);
  return cudaGetLastError();
}

// ------------------------------------------------------- bounds-check selftest
__global__ void selftest_bounds_kernel(StatusBlock* sb) {
  // index 1 in a buffer of one element: the debug check records the failure;
  // nothing is read or written either way
  (void)in_bounds(sb, 1, 1, kSiteSelftest);
}

cudaError_t launch_selftest_bounds(StatusBlock* sb, cudaStream_t stream) {
  selftest_bounds_kernel<<<1, 1, 0, stream>>>(sb);
  return cudaGetLastError();
}

cudaError_t launch_selftest_wait(StatusBlock* sb, long long limit_ns, cudaStream_t stream) {
  selftest_wait_kernel<<<1, 32, 0, stream>>>(sb, limit_ns);
  return cudaGetLastError();
}

}  // namespace kda

using namespace kda;

extern "C" {

const char* kda_status_string(kda_status s) {
  switch (s) {
    case KDA_OK: return "KDA_OK";
    case KDA_ERR_INVALID_ARG: return "KDA_ERR_INVALID_ARG";
    case KDA_ERR_UNSUPPORTED: return "KDA_ERR_UNSUPPORTED";
    case KDA_ERR_MISALIGNED: return "KDA_ERR_MISALIGNED";
    case KDA_ERR_WORKSPACE: return "KDA_ERR_WORKSPACE";
    case KDA_ERR_CUDA: return "KDA_ERR_CUDA";
    case KDA_ERR_TIMEOUT: return "KDA_ERR_TIMEOUT";
    case KDA_ERR_BAD_SEQLENS: return "KDA_ERR_BAD_SEQLENS";
    case KDA_ERR_BOUNDS: return "KDA_ERR_BOUNDS";
  }
  return "KDA_ERR_UNKNOWN";
}

kda_status kda_gate_fwd(const float* z, const float* A_log, float g_min, float* g, int64_t rows,
                        int H, int dk, void* stream) {
  if (!z || !A_log || !g) return KDA_ERR_INVALID_ARG;
  if (rows < 0 || H <= 0 || dk <= 0 || dk % 4 != 0) return KDA_ERR_INVALID_ARG;
  if (!(g_min < 0.f) || !isfinite(g_min)) return KDA_ERR_INVALID_ARG;
  if (z == g) return KDA_ERR_INVALID_ARG;
  if (!aligned16(z) || !aligned16(g) || !aligned16(A_log)) return KDA_ERR_MISALIGNED;
  if (rows == 0) return KDA_OK;
  cudaError_t e = launch_gate(z, A_log, g_min, g, rows, H, dk, (cudaStream_t)stream);
  return e == cudaSuccess ? KDA_OK : cuda_failure(e);
}

size_t kda_gate_bwd_workspace_size(int H) {
  return H > 0 ? sizeof(float) * (size_t)H * kGateBwdMaxParts : 0;
}

kda_status kda_gate_bwd(const float* z, const float* A_log, float g_min, const float* dg,
                        float* dz, float* dA_log, int64_t rows, int H, int dk, void* workspace,
                        size_t workspace_bytes, void* stream) {
  if (!z || !A_log || !dg || !dz || !dA_log) return KDA_ERR_INVALID_ARG;
  if (rows < 0 || H <= 0 || dk <= 0) return KDA_ERR_INVALID_ARG;
  if (!(g_min < 0.f) || !isfinite(g_min)) return KDA_ERR_INVALID_ARG;
  if (dk < 4 || dk > 1024 || (dk & (dk - 1)) != 0) return KDA_ERR_UNSUPPORTED;
  if (rows * (int64_t)H > ((int64_t)1 << 40)) return KDA_ERR_UNSUPPORTED;
  if (!workspace || workspace_bytes < kda_gate_bwd_workspace_size(H)) return KDA_ERR_WORKSPACE;
  const void* ptrs[] = {z, A_log, dg, dz, dA_log, workspace};
  for (const void* p : ptrs)
    if (!aligned16(p)) return KDA_ERR_MISALIGNED;
  // dz may overwrite dg; nothing else may alias
  if (dz == z || dz == A_log || (const void*)dA_log == z || (const void*)dA_log == dg ||
      dA_log == dz || workspace == z || workspace == dg || workspace == dz ||
      workspace == dA_log)
    return KDA_ERR_INVALID_ARG;
  cudaStream_t st = (cudaStream_t)stream;
  if (rows == 0) {
    cudaError_t em = cudaMemsetAsync(dA_log, 0, sizeof(float) * (size_t)H, st);
    return em == cudaSuccess ? KDA_OK : cuda_failure(em);
  }
  cudaError_t e = launch_gate_bwd(z, A_log, g_min, dg, dz, dA_log, rows, H, dk,
                                  static_cast<float*>(workspace), st);
  return e == cudaSuccess ? KDA_OK : cuda_failure(e);
}

size_t kda_chunk_fwd_workspace_size(int B, int T, int H, int dk, int dv, int num_seqs,
                                    int chunk_size, kda_dtype in_dtype) {
  size_t bytes = kStatusBytes;
  if (num_seqs > 0) bytes += round_up(sizeof(int32_t) * (size_t)num_seqs, 256);
  if (B > 0 && T > 0 && H > 0) {
    if (use_tc_path(in_dtype, dk, dv, chunk_size))
      bytes += tc_workspace_bytes(B, T, H, num_seqs, device_sm_count());
    else if (use_f32_path(chunk_size))
      bytes += chunk_f32_tail_bytes(B, T, H, num_seqs);
  }
  return bytes;
}

}  // extern "C"

namespace kda {

// Shared body of kda_chunk_fwd and kda_chunk_fwd_gated: g is the log-decay,
// or z when A_log is not null.  reset_status = false keeps the device status
// word as it is (a caller running several slices on one workspace).
kda_status chunk_fwd_impl(const void* q, const void* k, const void* v, const float* g,
                          const float* A_log, float g_min, const float* beta,
                          kda_dtype in_dtype, const float* init_state,
                          const int32_t* cu_seqlens, int num_seqs, int B, int T, int H, int dk,
                          int dv, float scale, int chunk_size, void* out, float* final_state,
                          void* workspace, size_t workspace_bytes, void* stream,
                          bool reset_status) {
  if (!q || !k || !v || !g || !beta || !out || !workspace) return KDA_ERR_INVALID_ARG;
  if (A_log && (!(g_min < 0.f) || !isfinite(g_min))) return KDA_ERR_INVALID_ARG;
  if (in_dtype != KDA_F32 && in_dtype != KDA_BF16) return KDA_ERR_INVALID_ARG;
  if (B <= 0 || T <= 0 || H <= 0) return KDA_ERR_INVALID_ARG;
  if (!isfinite(scale)) return KDA_ERR_INVALID_ARG;
  if (!dim_ok(dk) || !dim_ok(dv)) return KDA_ERR_UNSUPPORTED;
  if (chunk_size != 0 && chunk_size != 16 && chunk_size != 32 && chunk_size != 64)
    return KDA_ERR_UNSUPPORTED;
  if (cu_seqlens) {
    if (B != 1 || num_seqs <= 0) return KDA_ERR_INVALID_ARG;
  } else if (num_seqs != 0 && num_seqs != B) {
    return KDA_ERR_INVALID_ARG;
  }
  const void* ptrs[] = {q, k, v, g, beta, out, workspace, init_state, final_state, cu_seqlens, A_log};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return KDA_ERR_MISALIGNED;
  const void* outs[] = {out};
  const void* ins[] = {q, k, v, g, beta, init_state, cu_seqlens, A_log};
  for (const void* o : outs)
    for (const void* i : ins)
      if (i && o == i) return KDA_ERR_INVALID_ARG;
  const int nseq = cu_seqlens ? num_seqs : B;
  const size_t need =
      kda_chunk_fwd_workspace_size(B, T, H, dk, dv, cu_seqlens ? num_seqs : 0, chunk_size, in_dtype);
  if (workspace_bytes < need) return KDA_ERR_WORKSPACE;
  if ((int64_t)nseq * H > (int64_t)1 << 30) return KDA_ERR_UNSUPPORTED;

  cudaStream_t st = (cudaStream_t)stream;
  StatusBlock* sb = static_cast<StatusBlock*>(workspace);
  char* tail = static_cast<char*>(workspace) + kStatusBytes;
  if (reset_status)
    if (cudaError_t em = cudaMemsetAsync(sb, 0, kStatusBytes, st)) return cuda_failure(em);

  ChunkArgs a{};
  a.q = q;
  a.k = k;
  a.v = v;
  a.g = g;
  a.A_log = A_log;
  a.g_min = g_min;
  a.gated = A_log != nullptr;
  a.beta = beta;
  a.dt = in_dtype;
  a.init_state = init_state;
  a.final_state = final_state;
  a.out = out;
  a.map.cu_seqlens = cu_seqlens;
  a.map.order = nullptr;
  a.map.status = sb;
  a.map.B = B;
  a.map.T = T;
  a.map.H = H;
  a.num_units = nseq * H;
  a.dk = dk;
  a.dv = dv;
  a.scale = scale;
  a.chunk = chunk_size;
  a.sb = sb;
  if (cu_seqlens) {
    int32_t* order = reinterpret_cast<int32_t*>(tail);
    tail += round_up(sizeof(int32_t) * (size_t)num_seqs, 256);
    if (cudaError_t ep = launch_varlen_plan(cu_seqlens, num_seqs, T, order, sb, st))
      return cuda_failure(ep);
    a.map.order = order;
  }
  cudaError_t e;
  if (use_tc_path(in_dtype, dk, dv, chunk_size)) {
    a.chunk = 32;
    const size_t tail_bytes = workspace_bytes - (size_t)(tail - static_cast<char*>(workspace));
    e = launch_chunk_tc(a, tail, tail_bytes, st);
  } else if (use_f32_path(chunk_size)) {
    a.chunk = 32;
    e = launch_chunk_f32(a, tail, st);
  } else {
    e = launch_chunk_simt(a, st);
  }
  return e == cudaSuccess ? KDA_OK : cuda_failure(e);
}

}  // namespace kda

extern "C" {

kda_status kda_chunk_fwd(const void* q, const void* k, const void* v, const float* g,
                         const float* beta, kda_dtype in_dtype, const float* init_state,
                         const int32_t* cu_seqlens, int num_seqs, int B, int T, int H, int dk,
                         int dv, float scale, int chunk_size, void* out, float* final_state,
                         void* workspace, size_t workspace_bytes, void* stream) {
  return chunk_fwd_impl(q, k, v, g, nullptr, 0.f, beta, in_dtype, init_state, cu_seqlens,
                        num_seqs, B, T, H, dk, dv, scale, chunk_size, out, final_state,
                        workspace, workspace_bytes, stream);
}

kda_status kda_chunk_segment_transition(const void* q, const void* k, const void* v,
                                        const float* z, const float* A_log, float g_min,
                                        const float* beta, kda_dtype in_dtype, int B, int T,
                                        int H, int dk, int dv, float* pairs, void* workspace,
                                        size_t workspace_bytes, void* stream) {
  if (!q || !k || !v || !z || !A_log || !beta || !pairs || !workspace)
    return KDA_ERR_INVALID_ARG;
  if (!(g_min < 0.f) || !isfinite(g_min)) return KDA_ERR_INVALID_ARG;
  if (in_dtype != KDA_F32 && in_dtype != KDA_BF16) return KDA_ERR_INVALID_ARG;
  if (B <= 0 || T <= 0 || H <= 0) return KDA_ERR_INVALID_ARG;
  if (!dim_ok(dk) || !dim_ok(dv)) return KDA_ERR_UNSUPPORTED;
  if (!use_tc_path(in_dtype, dk, dv, 0)) return KDA_ERR_UNSUPPORTED;  // bf16, 128 x 128 only
  if ((int64_t)B * H > (int64_t)1 << 30) return KDA_ERR_UNSUPPORTED;
  const void* ptrs[] = {q, k, v, z, A_log, beta, pairs, workspace};
  for (const void* p : ptrs)
    if (!aligned16(p)) return KDA_ERR_MISALIGNED;
  const void* ins[] = {q, k, v, z, A_log, beta};
  for (const void* i : ins)
    if (i == pairs) return KDA_ERR_INVALID_ARG;
  if (workspace_bytes < kStatusBytes) return KDA_ERR_WORKSPACE;
  cudaStream_t st = (cudaStream_t)stream;
  StatusBlock* sb = static_cast<StatusBlock*>(workspace);
  if (cudaError_t em = cudaMemsetAsync(sb, 0, kStatusBytes, st)) return cuda_failure(em);
  ChunkArgs a{};
  a.q = q;
  a.k = k;
  a.v = v;
  a.g = z;
  a.A_log = A_log;
  a.g_min = g_min;
  a.gated = true;
  a.beta = beta;
  a.dt = in_dtype;
  a.map.status = sb;
  a.map.B = B;
  a.map.T = T;
  a.map.H = H;
  a.num_units = B * H;
  a.dk = dk;
  a.dv = dv;
  a.scale = 1.f;
  a.chunk = 32;
  a.sb = sb;
  const cudaError_t e = launch_chunk_tc_transition(a, pairs, st);
  return e == cudaSuccess ? KDA_OK : cuda_failure(e);
}

kda_status kda_chunk_state_prefix(const float* pairs, int count, int index,
                                  const float* init_state, int B, int H, int dk, int dv,
                                  float* state_out, void* stream) {
  if (!pairs || !state_out) return KDA_ERR_INVALID_ARG;
  if (count <= 0 || index < 0 || index >= count || B <= 0 || H <= 0)
    return KDA_ERR_INVALID_ARG;
  if (dk != 128 || dv != 128) return KDA_ERR_UNSUPPORTED;
  if ((int64_t)B * H > (int64_t)1 << 30) return KDA_ERR_UNSUPPORTED;
  const void* ptrs[] = {pairs, init_state, state_out};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return KDA_ERR_MISALIGNED;
  if (state_out == pairs || (init_state && state_out == init_state)) return KDA_ERR_INVALID_ARG;
  const cudaError_t e = launch_state_prefix(pairs, count, index, init_state, B * H, state_out,
                                            (cudaStream_t)stream);
  return e == cudaSuccess ? KDA_OK : cuda_failure(e);
}

kda_status kda_chunk_fwd_gated(const void* q, const void* k, const void* v, const float* z,
                               const float* A_log, float g_min, const float* beta,
                               kda_dtype in_dtype, const float* init_state,
                               const int32_t* cu_seqlens, int num_seqs, int B, int T, int H,
                               int dk, int dv, float scale, int chunk_size, void* out,
                               float* final_state, void* workspace, size_t workspace_bytes,
                               void* stream) {
  if (!A_log) return KDA_ERR_INVALID_ARG;
  return chunk_fwd_impl(q, k, v, z, A_log, g_min, beta, in_dtype, init_state, cu_seqlens,
                        num_seqs, B, T, H, dk, dv, scale, chunk_size, out, final_state,
                        workspace, workspace_bytes, stream);
}

}  // extern "C"

namespace {

kda_status decode_impl(const void* q, const void* k, const void* v, const float* g,
                       const float* A_log, float g_min, const float* beta, kda_dtype in_dtype,
                       float* state, int N, int H, int dk, int dv, float scale, void* out,
                       void* stream) {
  if (!q || !k || !v || !g || !beta || !state || !out) return KDA_ERR_INVALID_ARG;
  if (in_dtype != KDA_F32 && in_dtype != KDA_BF16) return KDA_ERR_INVALID_ARG;
  if (N <= 0 || H <= 0 || !isfinite(scale)) return KDA_ERR_INVALID_ARG;
  if (A_log && (!(g_min < 0.f) || !isfinite(g_min))) return KDA_ERR_INVALID_ARG;
  if ((int64_t)N * H > 0x7fffffffLL) return KDA_ERR_UNSUPPORTED;
  if (!dim_ok(dk) || !dim_ok(dv)) return KDA_ERR_UNSUPPORTED;
  const void* ptrs[] = {q, k, v, g, beta, state, out, A_log};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return KDA_ERR_MISALIGNED;
  const void* ins[] = {q, k, v, g, beta, state, A_log};
  for (const void* i : ins)
    if (i == out) return KDA_ERR_INVALID_ARG;
  cudaError_t e = launch_decode(q, k, v, g, A_log, g_min, beta, in_dtype, state, N, H, dk, dv,
                                scale, out, (cudaStream_t)stream);
  return e == cudaSuccess ? KDA_OK : cuda_failure(e);
}

}  // namespace

extern "C" {

kda_status kda_decode_step(const void* q, const void* k, const void* v, const float* g,
                           const float* beta, kda_dtype in_dtype, float* state, int N, int H,
                           int dk, int dv, float scale, void* out, void* stream) {
  return decode_impl(q, k, v, g, nullptr, 0.f, beta, in_dtype, state, N, H, dk, dv, scale, out,
                     stream);
}

kda_status kda_decode_step_gated(const void* q, const void* k, const void* v, const float* z,
                                 const float* A_log, float g_min, const float* beta,
                                 kda_dtype in_dtype, float* state, int N, int H, int dk, int dv,
                                 float scale, void* out, void* stream) {
  if (!A_log) return KDA_ERR_INVALID_ARG;
  return decode_impl(q, k, v, z, A_log, g_min, beta, in_dtype, state, N, H, dk, dv, scale, out,
                     stream);
}

kda_status kda_decode_verify(const void* q, const void* k, const void* v, const float* g,
                             const float* A_log, float g_min, const float* beta,
                             kda_dtype in_dtype, const float* state, int N, int H, int K, int dk,
                             int dv, float scale, void* out, void* stream) {
  if (!q || !k || !v || !g || !beta || !state || !out) return KDA_ERR_INVALID_ARG;
  if (in_dtype != KDA_F32 && in_dtype != KDA_BF16) return KDA_ERR_INVALID_ARG;
  if (N <= 0 || H <= 0 || !isfinite(scale)) return KDA_ERR_INVALID_ARG;
  if (K < 1 || K > decode_multi_max_tokens()) return KDA_ERR_UNSUPPORTED;
  if (A_log && (!(g_min < 0.f) || !isfinite(g_min))) return KDA_ERR_INVALID_ARG;
  if ((int64_t)N * H > 0x7fffffffLL) return KDA_ERR_UNSUPPORTED;
  if (!dim_ok(dk) || !dim_ok(dv)) return KDA_ERR_UNSUPPORTED;
  const void* ptrs[] = {q, k, v, g, beta, state, out, A_log};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return KDA_ERR_MISALIGNED;
  const void* ins[] = {q, k, v, g, beta, state, A_log};
  for (const void* i : ins)
    if (i == out) return KDA_ERR_INVALID_ARG;
  DecodeMultiArgs a{q, k, v, g, A_log, g_min, beta, in_dtype, const_cast<float*>(state), nullptr,
                    out, N, H, K, dk, dv, scale};
  const cudaError_t e = launch_decode_multi(a, true, (cudaStream_t)stream);
  return e == cudaSuccess ? KDA_OK : cuda_failure(e);
}

kda_status kda_decode_replay(const void* k, const void* v, const float* g, const float* A_log,
                             float g_min, const float* beta, kda_dtype in_dtype, float* state,
                             const int32_t* accept_len, int N, int H, int K, int dk, int dv,
                             void* stream) {
  if (!k || !v || !g || !beta || !state || !accept_len) return KDA_ERR_INVALID_ARG;
  if (in_dtype != KDA_F32 && in_dtype != KDA_BF16) return KDA_ERR_INVALID_ARG;
  if (N <= 0 || H <= 0) return KDA_ERR_INVALID_ARG;
  if (K < 1 || K > decode_multi_max_tokens()) return KDA_ERR_UNSUPPORTED;
  if (A_log && (!(g_min < 0.f) || !isfinite(g_min))) return KDA_ERR_INVALID_ARG;
  if ((int64_t)N * H > 0x7fffffffLL) return KDA_ERR_UNSUPPORTED;
  if (!dim_ok(dk) || !dim_ok(dv)) return KDA_ERR_UNSUPPORTED;
  const void* ptrs[] = {k, v, g, beta, state, accept_len, A_log};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return KDA_ERR_MISALIGNED;
  const void* ins[] = {k, v, g, beta, accept_len, A_log};
  for (const void* i : ins)
    if (i == state) return KDA_ERR_INVALID_ARG;
  DecodeMultiArgs a{nullptr, k, v, g, A_log, g_min, beta, in_dtype, state, accept_len, nullptr,
                    N, H, K, dk, dv, 1.f};
  const cudaError_t e = launch_decode_multi(a, false, (cudaStream_t)stream);
  return e == cudaSuccess ? KDA_OK : cuda_failure(e);
}

size_t kda_recurrent_bwd_workspace_size(int B, int T, int H, int dk, int dv, int num_seqs) {
  if (B <= 0 || T < 0 || H <= 0 || num_seqs < 0 || !dim_ok(dk) || !dim_ok(dv)) return 0;
  if (num_seqs > 0 && B != 1) return 0;
  return bwd_chunk_workspace_bytes(B, T, H, dk, dv, num_seqs);
}

kda_status kda_recurrent_bwd(const void* q, const void* k, const void* v, const float* g,
                             const float* beta, kda_dtype in_dtype, const float* init_state,
                             const void* dout, const float* d_final, const int32_t* cu_seqlens,
                             int num_seqs, int B, int T, int H, int dk, int dv, float scale,
                             float* dq, float* dk_out, float* dv_out, float* dg, float* dbeta,
                             float* d_init, void* workspace, size_t workspace_bytes,
                             void* stream) {
  if (in_dtype != KDA_F32 && in_dtype != KDA_BF16) return KDA_ERR_INVALID_ARG;
  if (B <= 0 || T < 0 || H <= 0 || !isfinite(scale)) return KDA_ERR_INVALID_ARG;
  if (cu_seqlens) {
    if (B != 1 || num_seqs <= 0) return KDA_ERR_INVALID_ARG;
  } else if (num_seqs != 0) {
    return KDA_ERR_INVALID_ARG;
  }
  if (T > 0 && (!q || !k || !v || !g || !beta || !dout || !dq || !dk_out || !dv_out || !dg ||
                !dbeta))
    return KDA_ERR_INVALID_ARG;
  const int64_t nseq = cu_seqlens ? num_seqs : B;
  if (nseq * H > 0x7fffffffLL || (int64_t)B * T * H > 0x7fffffffLL) return KDA_ERR_UNSUPPORTED;
  if (!dim_ok(dk) || !dim_ok(dv)) return KDA_ERR_UNSUPPORTED;
  const size_t need = bwd_chunk_workspace_bytes(B, T, H, dk, dv, cu_seqlens ? num_seqs : 0);
  if (!workspace || workspace_bytes < need) return KDA_ERR_WORKSPACE;
  const void* ptrs[] = {q, k, v, g, beta, init_state, dout, d_final, cu_seqlens, dq, dk_out,
                        dv_out, dg, dbeta, d_init, workspace};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return KDA_ERR_MISALIGNED;
  const void* ins[] = {q, k, v, g, beta, init_state, dout, d_final, cu_seqlens, workspace};
  const void* outs[] = {dq, dk_out, dv_out, dg, dbeta, d_init};
  for (const void* o : outs) {
    if (!o) continue;
    for (const void* i : ins)
      if (i == o) return KDA_ERR_INVALID_ARG;
  }
  if (T == 0 && !d_init) return KDA_OK;
  BwdArgs a{};
  a.q = q;
  a.k = k;
  a.v = v;
  a.g = g;
  a.beta = beta;
  a.init = init_state;
  a.dout = dout;
  a.dfinal = d_final;
  a.cu_seqlens = cu_seqlens;
  a.num_seqs = num_seqs;
  a.dt = in_dtype;
  a.B = B;
  a.T = T;
  a.H = H;
  a.dk_dim = dk;
  a.dv_dim = dv;
  a.scale = scale;
  a.dq = dq;
  a.dk = dk_out;
  a.dv = dv_out;
  a.dg = dg;
  a.dbeta = dbeta;
  a.dinit = d_init;
  a.ws = workspace;
  const cudaError_t e = launch_bwd_chunk(a, (cudaStream_t)stream);
  return e == cudaSuccess ? KDA_OK : cuda_failure(e);
}

const char* kda_last_cuda_error_string(void) { return last_cuda_error_text(); }

kda_status kda_get_device_status(const void* workspace, void* stream, int32_t* detail) {
  if (!workspace) return KDA_ERR_INVALID_ARG;
  cudaStream_t st = (cudaStream_t)stream;
  if (cudaError_t es = cudaStreamSynchronize(st)) return cuda_failure(es);
  int32_t host[2] = {0, 0};
  if (cudaError_t ec = cudaMemcpy(host, workspace, sizeof(host), cudaMemcpyDeviceToHost))
    return cuda_failure(ec);
  if (detail) *detail = host[1];
  return (kda_status)host[0];
}

kda_status kda_set_wait_limit_ns(int64_t limit_ns) {
  long long lim = limit_ns;
  if (lim < 0) lim = 0;
  if (lim > 5000000000LL) lim = 5000000000LL;
  set_wait_limit_ns(lim);
  return KDA_OK;
}

int kda_debug_checks_enabled(void) {
#ifdef KDA_DEBUG_CHECKS
  return 1;
#else
  return 0;
#endif
}

kda_status kda_selftest_bounds_check(void* workspace, void* stream) {
  if (!workspace) return KDA_ERR_INVALID_ARG;
  if (!aligned16(workspace)) return KDA_ERR_MISALIGNED;
  if (!kda_debug_checks_enabled()) return KDA_ERR_UNSUPPORTED;
  cudaStream_t st = (cudaStream_t)stream;
  if (cudaError_t em = cudaMemsetAsync(workspace, 0, kStatusBytes, st)) return cuda_failure(em);
  const cudaError_t e = launch_selftest_bounds(static_cast<StatusBlock*>(workspace), st);
  return e == cudaSuccess ? KDA_OK : cuda_failure(e);
}

kda_status kda_selftest_bounded_wait(void* workspace, int64_t spin_limit_ns, void* stream) {
  if (!workspace) return KDA_ERR_INVALID_ARG;
  if (!aligned16(workspace)) return KDA_ERR_MISALIGNED;
  long long lim = spin_limit_ns;
  if (lim < 1000) lim = 1000;
  if (lim > 5000000000LL) lim = 5000000000LL;
  cudaStream_t st = (cudaStream_t)stream;
  if (cudaError_t em = cudaMemsetAsync(workspace, 0, kStatusBytes, st)) return cuda_failure(em);
  cudaError_t e = launch_selftest_wait(static_cast<StatusBlock*>(workspace), lim, st);
  return e == cudaSuccess ? KDA_OK : cuda_failure(e);
}

}  // extern "C"
