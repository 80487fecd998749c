// kda_decode.cu -- single-token KDA decode step, state updated in place.
//
// KDA decoding ("NLP--技术报告解读-Kimi-K3", joezjh.github.io, Online serving >
// high-performance kernels; "Kimi K3 技术报告 · 大白话版", 5.4): every new
// token rewrites the recurrent state in place.  For one (sequence, head):
//   S' = Diag(exp(g)) S,   p = S'^T k,   r = S'^T q,
//   e  = beta (v - p),     S = S' + k e^T,
//   o  = scale (r + (k.q) e)          (= scale * S^T q after the update).
// This is the recurrence of the Model Architecture > KDA section applied to
// one token.
//
// The step is bound by HBM: the fp32 state (dk*dv*4 bytes) is read once and
// written once; q, k, v, g, beta and o add ~1.5 KB per head at dk = dv = 128.
// One CTA of 256 threads owns one (sequence, head).  Thread t holds a float4
// column group of RPT rows in registers: every warp-wide load or store moves
// 512 contiguous bytes.  The two column reductions (S'^T k, S'^T q) go through
// shared memory, after which the rank-one update is applied to the registers
// and written back.
#include "kda_internal.cuh"

namespace kda {
namespace {

constexpr int kThreads = 256;

__device__ __forceinline__ float4 f4_scale(float4 a, float s) {
  return make_float4(a.x * s, a.y * s, a.z * s, a.w * s);
}
__device__ __forceinline__ float4 f4_fma(float4 a, float s, float4 c) {
  return make_float4(fmaf(a.x, s, c.x), fmaf(a.y, s, c.y), fmaf(a.z, s, c.z),
                     fmaf(a.w, s, c.w));
}

template <typename Tin, int DK, int DV>
__global__ void __launch_bounds__(kThreads, 2)
    decode_kernel(const Tin* __restrict__ q, const Tin* __restrict__ k,
                  const Tin* __restrict__ v, const float* __restrict__ g,
                  const float* __restrict__ A_log, float g_min, int H,
                  const float* __restrict__ beta, float* __restrict__ state, float scale,
                  Tin* __restrict__ out) {
  constexpr int CG = DV / 4;         // threads per state row (float4 each)
  constexpr int RG = kThreads / CG;  // row groups
  constexpr int RPT = DK / RG;       // rows per thread
  static_assert(RPT >= 1 && DK % RG == 0, "tile shape");

  __shared__ float sk[DK], sq[DK], sa[DK];
  __shared__ float4 red_p[RG][CG], red_r[RG][CG];
  __shared__ __align__(16) float se[DV];  // read back as float4
  __shared__ float s_kq;

  const int unit = blockIdx.x;  // n * H + h
  const int tid = threadIdx.x;
  const int cg = tid % CG, rg = tid / CG;

  float4* S4 = reinterpret_cast<float4*>(state + (size_t)unit * DK * DV);
  float4 s[RPT];
#pragma unroll
  for (int r = 0; r < RPT; ++r) s[r] = __ldcs(S4 + (rg + r * RG) * CG + cg);

  // g is the log-decay, or z when A_log is given (gate fused in)
  const float a_h = A_log ? expf(A_log[unit % H]) : 0.f;
  for (int i = tid; i < DK; i += kThreads) {
    sk[i] = Elem<Tin>::load(k + (size_t)unit * DK + i);
    sq[i] = Elem<Tin>::load(q + (size_t)unit * DK + i);
    const float gi = g[(size_t)unit * DK + i];
    sa[i] = expf(A_log ? gate_value(gi, a_h, g_min) : gi);
  }
  __syncthreads();

  float4 p = make_float4(0.f, 0.f, 0.f, 0.f), rr = p;
#pragma unroll
  for (int r = 0; r < RPT; ++r) {
    const int i = rg + r * RG;
    s[r] = f4_scale(s[r], sa[i]);
    p = f4_fma(s[r], sk[i], p);
    rr = f4_fma(s[r], sq[i], rr);
  }
  red_p[rg][cg] = p;
  red_r[rg][cg] = rr;
  if (tid < 32) {
    float acc = 0.f;
    for (int i = tid; i < DK; i += 32) acc = fmaf(sk[i], sq[i], acc);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (tid == 0) s_kq = acc;
  }
  __syncthreads();

  if (tid < DV) {
    const float* rp = reinterpret_cast<const float*>(red_p);
    const float* rq = reinterpret_cast<const float*>(red_r);
    float pj = 0.f, rj = 0.f;
#pragma unroll 8
    for (int w = 0; w < RG; ++w) {
      pj += rp[w * DV + tid];
      rj += rq[w * DV + tid];
    }
    const float e = beta[unit] * (Elem<Tin>::load(v + (size_t)unit * DV + tid) - pj);
    se[tid] = e;
    Elem<Tin>::store(out + (size_t)unit * DV + tid, scale * fmaf(s_kq, e, rj));
  }
  __syncthreads();

  const float4 e4 = reinterpret_cast<const float4*>(se)[cg];
#pragma unroll
  for (int r = 0; r < RPT; ++r) {
    const float ki = sk[rg + r * RG];
    float4 x = s[r];
    x.x = fmaf(ki, e4.x, x.x);
    x.y = fmaf(ki, e4.y, x.y);
    x.z = fmaf(ki, e4.z, x.z);
    x.w = fmaf(ki, e4.w, x.w);
    __stcs(S4 + (rg + r * RG) * CG + cg, x);
  }
}

template <typename Tin, int DK>
cudaError_t dispatch_dv(const ChunkArgs& a, int N, int H, int dv, cudaStream_t st) {
  const unsigned grid = (unsigned)(N * H);
  const Tin* q = static_cast<const Tin*>(a.q);
  const Tin* k = static_cast<const Tin*>(a.k);
  const Tin* v = static_cast<const Tin*>(a.v);
  Tin* o = static_cast<Tin*>(a.out);
  float* S = const_cast<float*>(a.init_state);
  switch (dv) {
    case 32: decode_kernel<Tin, DK, 32><<<grid, kThreads, 0, st>>>(q, k, v, a.g, a.A_log, a.g_min, H, a.beta, S, a.scale, o); break;
    case 64: decode_kernel<Tin, DK, 64><<<grid, kThreads, 0, st>>>(q, k, v, a.g, a.A_log, a.g_min, H, a.beta, S, a.scale, o); break;
    case 128: decode_kernel<Tin, DK, 128><<<grid, kThreads, 0, st>>>(q, k, v, a.g, a.A_log, a.g_min, H, a.beta, S, a.scale, o); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

template <typename Tin>
cudaError_t dispatch_dk(const ChunkArgs& a, int N, int H, cudaStream_t st) {
  switch (a.dk) {
    case 32: return dispatch_dv<Tin, 32>(a, N, H, a.dv, st);
    case 64: return dispatch_dv<Tin, 64>(a, N, H, a.dv, st);
    case 128: return dispatch_dv<Tin, 128>(a, N, H, a.dv, st);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace

cudaError_t launch_decode(const void* q, const void* k, const void* v, const float* g_or_z,
                          const float* A_log, float g_min, const float* beta, kda_dtype dt,
                          float* state, int N, int H, int dk, int dv, float scale, void* out,
                          cudaStream_t stream) {
  ChunkArgs a{};
  a.q = q;
  a.k = k;
  a.v = v;
  a.g = g_or_z;
  a.A_log = A_log;
  a.g_min = g_min;
  a.beta = beta;
  a.dt = dt;
  a.init_state = state;
  a.out = out;
  a.dk = dk;
  a.dv = dv;
  a.scale = scale;
  if (dt == KDA_BF16) return dispatch_dk<__nv_bfloat16>(a, N, H, stream);
  return dispatch_dk<float>(a, N, H, stream);
}

}  // namespace kda
