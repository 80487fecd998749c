// kda_host_stream.cu -- gated chunked prefill of a dense batch that lives in
// host memory, streamed through the device in time slices.
//
// The batch [B, T, H, *] is cut along T into slices of Ts tokens (all B
// sequences at once).  Slice s is copied in on the copy stream while slice
// s - 1 is computed and slice s - 2's outputs are copied out on the compute
// stream, so the two copy directions and the kernels overlap.  The state
// crosses from one slice to the next on the device (slice s starts from the
// state slice s - 1 left), so the result is the recurrence over the whole
// sequence.  Two device slots for inputs and two for outputs, ping-pong
// states, one chunk workspace reused by every slice.
#include <limits.h>
#include <math.h>

#include "kda_host.cuh"

namespace kda {
namespace {

size_t align256(size_t x) { return (x + 255) / 256 * 256; }

// slice length: about an eighth of T in multiples of 64 tokens, at least 512
int slice_tokens(int T) {
  if (T <= 1024) return T;
  int ts = (T + 7) / 8;
  ts = (ts + 63) / 64 * 64;
  return ts < 512 ? 512 : ts;
}

struct HostLayout {
  int Ts, nslices, last;
  size_t es;                              // bytes of a q/k/v/o element
  size_t chunk_ws;                        // chunk workspace (status word first)
  size_t off_alog, off_state[2];
  size_t off_q[2], off_k[2], off_v[2], off_z[2], off_beta[2], off_out[2];
  size_t total;
};

HostLayout host_layout(int B, int T, int H, int dk, int dv, kda_dtype dt) {
  HostLayout L{};
  L.Ts = slice_tokens(T);
  L.nslices = (T + L.Ts - 1) / L.Ts;
  L.last = T - (L.nslices - 1) * L.Ts;
  L.es = dt == KDA_BF16 ? 2 : 4;
  const size_t a = kda_chunk_fwd_workspace_size(B, L.Ts, H, dk, dv, 0, 0, dt);
  const size_t b = kda_chunk_fwd_workspace_size(B, L.last, H, dk, dv, 0, 0, dt);
  L.chunk_ws = align256(a > b ? a : b);
  const size_t tok = (size_t)B * L.Ts * H;  // token-heads of a full slice
  size_t off = L.chunk_ws;
  L.off_alog = off;
  off += align256((size_t)H * 4);
  for (int i = 0; i < 2; ++i) {
    L.off_state[i] = off;
    off += align256((size_t)B * H * dk * dv * 4);
  }
  for (int i = 0; i < 2; ++i) {
    L.off_q[i] = off; off += align256(tok * dk * L.es);
    L.off_k[i] = off; off += align256(tok * dk * L.es);
    L.off_v[i] = off; off += align256(tok * dv * L.es);
    L.off_z[i] = off; off += align256(tok * dk * 4);
    L.off_beta[i] = off; off += align256(tok * 4);
    L.off_out[i] = off; off += align256(tok * dv * L.es);
  }
  L.total = off;
  return L;
}

// Tokens [t0, t0 + n) of every sequence b of a [B, T, row-bytes] tensor,
// between the full host tensor and a dense [B, n, row] device slice: one 2D
// copy, or one copy per sequence when B = 1 or the host pitch is beyond
// what a 2D copy takes.
cudaError_t copy_rows(void* dst, const void* src, size_t row, int B, int T, int t0, int n,
                      bool to_device, cudaStream_t st) {
  const size_t width = (size_t)n * row, full = (size_t)T * row;
  const cudaMemcpyKind kind = to_device ? cudaMemcpyHostToDevice : cudaMemcpyDeviceToHost;
  const char* s = static_cast<const char*>(src);
  char* d = static_cast<char*>(dst);
  if (B == 1 || full > (size_t)INT_MAX) {
    for (int b = 0; b < B; ++b) {
      const cudaError_t e =
          to_device ? cudaMemcpyAsync(d + b * width, s + b * full + (size_t)t0 * row, width, kind, st)
                    : cudaMemcpyAsync(d + b * full + (size_t)t0 * row, s + b * width, width, kind, st);
      if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
  }
  if (to_device) return cudaMemcpy2DAsync(d, width, s + (size_t)t0 * row, full, width, B, kind, st);
  return cudaMemcpy2DAsync(d + (size_t)t0 * row, full, s, width, width, B, kind, st);
}

struct Events {
  cudaEvent_t e[5] = {};
  ~Events() {
    for (cudaEvent_t x : e)
      if (x) cudaEventDestroy(x);  // released once pending work completes
  }
  cudaError_t create() {
    for (cudaEvent_t& x : e)
      if (cudaError_t r = cudaEventCreateWithFlags(&x, cudaEventDisableTiming)) return r;
    return cudaSuccess;
  }
};

}  // namespace
}  // namespace kda

using namespace kda;

extern "C" {

size_t kda_chunk_fwd_gated_host_workspace_size(int B, int T, int H, int dk, int dv,
                                               kda_dtype in_dtype) {
  if (B <= 0 || T <= 0 || H <= 0) return 0;
  if ((dk != 32 && dk != 64 && dk != 128) || (dv != 32 && dv != 64 && dv != 128)) return 0;
  if (in_dtype != KDA_F32 && in_dtype != KDA_BF16) return 0;
  return host_layout(B, T, H, dk, dv, in_dtype).total;
}

kda_status kda_chunk_fwd_gated_host(const void* q, const void* k, const void* v, const float* z,
                                    const float* A_log, float g_min, const float* beta,
                                    kda_dtype in_dtype, const float* init_state, int B, int T,
                                    int H, int dk, int dv, float scale, void* out,
                                    float* final_state, void* workspace, size_t workspace_bytes,
                                    void* stream, void* copy_stream) {
  if (!q || !k || !v || !z || !A_log || !beta || !out || !workspace) return KDA_ERR_INVALID_ARG;
  if (in_dtype != KDA_F32 && in_dtype != KDA_BF16) return KDA_ERR_INVALID_ARG;
  if (B <= 0 || T <= 0 || H <= 0 || !isfinite(scale)) return KDA_ERR_INVALID_ARG;
  if (!(g_min < 0.f) || !isfinite(g_min)) return KDA_ERR_INVALID_ARG;
  if ((dk != 32 && dk != 64 && dk != 128) || (dv != 32 && dv != 64 && dv != 128))
    return KDA_ERR_UNSUPPORTED;
  if ((int64_t)B * H > (int64_t)1 << 30) return KDA_ERR_UNSUPPORTED;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return KDA_ERR_MISALIGNED;
  const HostLayout L = host_layout(B, T, H, dk, dv, in_dtype);
  if (workspace_bytes < L.total) return KDA_ERR_WORKSPACE;
  const void* ins[] = {q, k, v, z, A_log, beta, init_state};
  for (const void* i : ins)
    if (i == out || (final_state && i == final_state)) return KDA_ERR_INVALID_ARG;

  cudaStream_t cs = (cudaStream_t)stream;
  cudaStream_t xs = copy_stream ? (cudaStream_t)copy_stream : cs;
  char* ws = static_cast<char*>(workspace);
  Events ev;  // 0: entry; 1, 2: slot s filled; 3, 4: slot s free again
  if (cudaError_t e = ev.create()) return cuda_failure(e);
  // the slots may still be read by an earlier call's kernels on `stream`
  if (cudaError_t e = cudaEventRecord(ev.e[0], cs)) return cuda_failure(e);
  if (cudaError_t e = cudaStreamWaitEvent(xs, ev.e[0], 0)) return cuda_failure(e);
  if (cudaError_t e = cudaMemsetAsync(ws, 0, kStatusBytes, cs)) return cuda_failure(e);
  float* alog_d = reinterpret_cast<float*>(ws + L.off_alog);
  if (cudaError_t e = cudaMemcpyAsync(alog_d, A_log, (size_t)H * 4, cudaMemcpyHostToDevice, xs))
    return cuda_failure(e);
  float* state[2] = {reinterpret_cast<float*>(ws + L.off_state[0]),
                     reinterpret_cast<float*>(ws + L.off_state[1])};
  const size_t sbytes = (size_t)B * H * dk * dv * 4;
  if (init_state)  // slice 0 starts from state[1]
    if (cudaError_t e = cudaMemcpyAsync(state[1], init_state, sbytes, cudaMemcpyHostToDevice, xs))
      return cuda_failure(e);

  const size_t rq = (size_t)H * dk * L.es, rv = (size_t)H * dv * L.es;
  const size_t rz = (size_t)H * dk * 4, rb = (size_t)H * 4;
  for (int s = 0; s < L.nslices; ++s) {
    const int p = s & 1, t0 = s * L.Ts;
    const int n = s == L.nslices - 1 ? L.last : L.Ts;
    if (s >= 2)
      if (cudaError_t e = cudaStreamWaitEvent(xs, ev.e[3 + p], 0)) return cuda_failure(e);
    const struct { size_t off; const void* src; size_t row; } cp[] = {
        {L.off_q[p], q, rq}, {L.off_k[p], k, rq}, {L.off_v[p], v, rv},
        {L.off_z[p], z, rz}, {L.off_beta[p], beta, rb}};
    for (const auto& c : cp)
      if (cudaError_t e = copy_rows(ws + c.off, c.src, c.row, B, T, t0, n, true, xs))
        return cuda_failure(e);
    if (cudaError_t e = cudaEventRecord(ev.e[1 + p], xs)) return cuda_failure(e);
    if (cudaError_t e = cudaStreamWaitEvent(cs, ev.e[1 + p], 0)) return cuda_failure(e);
    const float* init = (s == 0 && !init_state) ? nullptr : state[(s + 1) & 1];
    const kda_status r = chunk_fwd_impl(
        ws + L.off_q[p], ws + L.off_k[p], ws + L.off_v[p],
        reinterpret_cast<const float*>(ws + L.off_z[p]), alog_d, g_min,
        reinterpret_cast<const float*>(ws + L.off_beta[p]), in_dtype, init, nullptr, 0, B, n, H,
        dk, dv, scale, 0, ws + L.off_out[p], state[s & 1], ws, L.chunk_ws, stream, false);
    if (r != KDA_OK) return r;
    if (cudaError_t e = cudaEventRecord(ev.e[3 + p], cs)) return cuda_failure(e);
    if (cudaError_t e = copy_rows(out, ws + L.off_out[p], rv, B, T, t0, n, false, cs))
      return cuda_failure(e);
  }
  if (final_state)
    if (cudaError_t e = cudaMemcpyAsync(final_state, state[(L.nslices - 1) & 1], sbytes,
                                        cudaMemcpyDeviceToHost, cs))
      return cuda_failure(e);
  return KDA_OK;
}

}  // extern "C"
