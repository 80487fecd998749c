// kda_decode_multi.cu -- multi-token decode for speculative decoding:
// verify K draft tokens without touching the state, then replay the accepted
// prefix into the state.
//
// "NLP--技术报告解读-Kimi-K3" (joezjh.github.io), Online serving > high-
// performance kernels > KDA Decoding: with multi-token-prediction drafts, the
// recurrent state is not snapshotted for rollback; the projected inputs of the
// draft tokens are kept and the state is rebuilt on demand by replaying the
// accepted tokens (also "Kimi K3 技术报告 · 大白话版" 5.4, and the latetalk
// digest's description of storing ~1 KB per step and replaying from the last
// checkpoint).
//
//  verify : for each (sequence, head), run the recurrence of the Model
//           Architecture > KDA section over the K draft tokens starting from
//           the committed state, emitting o_t for every token; the state in
//           HBM is only read.
//  replay : apply the first m_n = accept_len[n] tokens of the same inputs to
//           the committed state in place (m_n = 0 leaves it untouched).
//
// Both keep one (sequence, head) state in registers for all K tokens, so the
// fp32 state (dk*dv*4 bytes) crosses HBM once per launch instead of once per
// token.  The value columns of the recurrence are independent given k, q, g
// and beta, so for dv >= 64 each state is split over two CTAs by column halves:
// half the registers per thread, four CTAs per SM, twice the loads in flight.
// Thread layout and reductions follow kda_decode.cu.
#include "kda_internal.cuh"

namespace kda {
namespace {

constexpr int kThreads = 256;
constexpr int kMaxK = 16;  // draft tokens per launch

template <int DV>
constexpr int cols_per_cta() { return DV >= 64 ? DV / 2 : DV; }

template <typename Tin, int DK, int DV, bool VERIFY>
__global__ void __launch_bounds__(kThreads, (cols_per_cta<DV>() * DK <= 64 * 128) ? 4 : 2)
    decode_multi_kernel(const Tin* __restrict__ q, const Tin* __restrict__ k,
                        const Tin* __restrict__ v, const float* __restrict__ g,
                        const float* __restrict__ A_log, float g_min,
                        const float* __restrict__ beta, float* __restrict__ state,
                        const int32_t* __restrict__ accept_len, int H, int K, float scale,
                        Tin* __restrict__ out) {
  constexpr int DVC = cols_per_cta<DV>();  // value columns of this CTA
  constexpr int NSPLIT = DV / DVC;
  constexpr int CG = DVC / 4;
  constexpr int RG = kThreads / CG;
  constexpr int RPT = DK / RG;
  static_assert(RPT >= 1 && DK % RG == 0, "tile shape");

  __shared__ float sk[kMaxK][DK], sq[kMaxK][DK], sa[kMaxK][DK];
  __shared__ float sv[kMaxK][DVC], sb[kMaxK], skq[kMaxK];
  __shared__ float4 red_p[RG][CG], red_r[RG][CG];
  __shared__ __align__(16) float se[DVC];  // read back as float4

  const int unit = blockIdx.x / NSPLIT;  // n * H + h
  const int j0 = (blockIdx.x % NSPLIT) * DVC;
  const int n = unit / H, h = unit % H;
  const int tid = threadIdx.x;
  const int cg = tid % CG, rg = tid / CG;

  int steps = K;
  if (!VERIFY) {
    steps = accept_len[n];
    steps = steps < 0 ? 0 : (steps > K ? K : steps);
    if (steps == 0) return;  // nothing accepted: the committed state stands
  }

  float4* S4 = reinterpret_cast<float4*>(state + (size_t)unit * DK * DV + j0);
  float4 s[RPT];
#pragma unroll
  for (int r = 0; r < RPT; ++r) s[r] = S4[(rg + r * RG) * (DV / 4) + cg];

  // inputs of the tokens, [N, K, H, *] layouts; g is the log-decay, or z
  // when A_log is given (gate fused in)
  const float a_h = A_log ? expf(A_log[h]) : 0.f;
  for (int idx = tid; idx < steps * DK; idx += kThreads) {
    const int t = idx / DK, i = idx % DK;
    const size_t off = (((size_t)n * K + t) * H + h) * DK + i;
    sk[t][i] = Elem<Tin>::load(k + off);
    if (VERIFY) sq[t][i] = Elem<Tin>::load(q + off);
    const float gi = g[off];
    sa[t][i] = expf(A_log ? gate_value(gi, a_h, g_min) : gi);
  }
  for (int idx = tid; idx < steps * DVC; idx += kThreads) {
    const int t = idx / DVC, j = idx % DVC;
    sv[t][j] = Elem<Tin>::load(v + (((size_t)n * K + t) * H + h) * DV + j0 + j);
  }
  for (int t = tid; t < steps; t += kThreads) sb[t] = beta[((size_t)n * K + t) * H + h];
  __syncthreads();
  if (VERIFY) {  // k_t . q_t for every token, one warp per token
    for (int t = tid >> 5; t < steps; t += kThreads / 32) {
      float acc = 0.f;
      for (int i = tid & 31; i < DK; i += 32) acc = fmaf(sk[t][i], sq[t][i], acc);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
      if ((tid & 31) == 0) skq[t] = acc;
    }
  }

  for (int t = 0; t < steps; ++t) {
    float4 p = make_float4(0.f, 0.f, 0.f, 0.f), rr = p;
#pragma unroll
    for (int r = 0; r < RPT; ++r) {
      const int i = rg + r * RG;
      const float a = sa[t][i], ki = sk[t][i];
      s[r].x *= a; s[r].y *= a; s[r].z *= a; s[r].w *= a;
      p.x = fmaf(s[r].x, ki, p.x); p.y = fmaf(s[r].y, ki, p.y);
      p.z = fmaf(s[r].z, ki, p.z); p.w = fmaf(s[r].w, ki, p.w);
      if (VERIFY) {
        const float qi = sq[t][i];
        rr.x = fmaf(s[r].x, qi, rr.x); rr.y = fmaf(s[r].y, qi, rr.y);
        rr.z = fmaf(s[r].z, qi, rr.z); rr.w = fmaf(s[r].w, qi, rr.w);
      }
    }
    red_p[rg][cg] = p;
    if (VERIFY) red_r[rg][cg] = rr;
    __syncthreads();
    if (tid < DVC) {
      const float* rp = reinterpret_cast<const float*>(red_p);
      float pj = 0.f;
#pragma unroll 8
      for (int w = 0; w < RG; ++w) pj += rp[w * DVC + tid];
      const float e = sb[t] * (sv[t][tid] - pj);
      se[tid] = e;
      if (VERIFY) {
        const float* rq = reinterpret_cast<const float*>(red_r);
        float rj = 0.f;
#pragma unroll 8
        for (int w = 0; w < RG; ++w) rj += rq[w * DVC + tid];
        Elem<Tin>::store(out + (((size_t)n * K + t) * H + h) * DV + j0 + tid,
                         scale * fmaf(skq[t], e, rj));
      }
    }
    __syncthreads();
    const float4 e4 = reinterpret_cast<const float4*>(se)[cg];
#pragma unroll
    for (int r = 0; r < RPT; ++r) {
      const float ki = sk[t][rg + r * RG];
      s[r].x = fmaf(ki, e4.x, s[r].x); s[r].y = fmaf(ki, e4.y, s[r].y);
      s[r].z = fmaf(ki, e4.z, s[r].z); s[r].w = fmaf(ki, e4.w, s[r].w);
    }
    __syncthreads();  // se / red_* are rewritten by the next token
  }
  if (!VERIFY) {
#pragma unroll
    for (int r = 0; r < RPT; ++r) S4[(rg + r * RG) * (DV / 4) + cg] = s[r];
  }
}

template <typename Tin, int DK, int DV, bool VERIFY>
cudaError_t launch3(const DecodeMultiArgs& a, cudaStream_t st) {
  decode_multi_kernel<Tin, DK, DV, VERIFY>
      <<<(unsigned)(a.N * a.H * (DV / cols_per_cta<DV>())), kThreads, 0, st>>>(
      static_cast<const Tin*>(a.q), static_cast<const Tin*>(a.k), static_cast<const Tin*>(a.v),
      a.g, a.A_log, a.g_min, a.beta, a.state, a.accept_len, a.H, a.K, a.scale,
      static_cast<Tin*>(a.out));
  return cudaGetLastError();
}

template <typename Tin, int DK, bool VERIFY>
cudaError_t by_dv(const DecodeMultiArgs& a, cudaStream_t st) {
  switch (a.dv) {
    case 32: return launch3<Tin, DK, 32, VERIFY>(a, st);
    case 64: return launch3<Tin, DK, 64, VERIFY>(a, st);
    case 128: return launch3<Tin, DK, 128, VERIFY>(a, st);
    default: return cudaErrorInvalidValue;
  }
}

template <typename Tin, bool VERIFY>
cudaError_t by_dk(const DecodeMultiArgs& a, cudaStream_t st) {
  switch (a.dk) {
    case 32: return by_dv<Tin, 32, VERIFY>(a, st);
    case 64: return by_dv<Tin, 64, VERIFY>(a, st);
    case 128: return by_dv<Tin, 128, VERIFY>(a, st);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace

int decode_multi_max_tokens() { return kMaxK; }

cudaError_t launch_decode_multi(const DecodeMultiArgs& a, bool verify, cudaStream_t stream) {
  if (a.dt == KDA_BF16)
    return verify ? by_dk<__nv_bfloat16, true>(a, stream) : by_dk<__nv_bfloat16, false>(a, stream);
  return verify ? by_dk<float, true>(a, stream) : by_dk<float, false>(a, stream);
}

}  // namespace kda
