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
// and beta, so a CTA takes at most 64 of them (a state of dv = 128 is split
// over two CTAs) and each warp owns 16 whole columns: lane (rl, cl) holds
// the dk/8 consecutive rows from rl*dk/8 of the warp's columns 4cl .. 4cl + 3
// (one float4 per row, 64-byte row segments per warp), and reads its rows of
// k, q and the decay as float4 from shared memory.  Every dot product over
// the key rows is then a sum over the 8 row lanes of a warp -- three
// butterfly shuffles -- and the token loop runs without a CTA barrier; the
// only barrier publishes the token inputs staged in shared memory, one warp
// per token (k.q is reduced there once).  The first token's loads go out
// before the state's, so the state streams while the inputs are staged.
#include "kda_internal.cuh"

namespace kda {
namespace {

constexpr int kMaxK = 16;        // draft tokens per launch
constexpr int kRowLanes = 8;     // lanes splitting the key rows of a column quad
constexpr int kWarpCols = 16;    // value columns per warp (4 lanes x float4)

template <int DV>
constexpr int cols_per_cta() { return DV >= 64 ? 64 : DV; }

template <int DV>
constexpr int threads_per_cta() { return 32 * (cols_per_cta<DV>() / kWarpCols); }

__device__ __forceinline__ float4 f4_mul(float4 a, float s) {
  const float2 s2 = make_float2(s, s);
  const float2 lo = __fmul2_rn(make_float2(a.x, a.y), s2);
  const float2 hi = __fmul2_rn(make_float2(a.z, a.w), s2);
  return make_float4(lo.x, lo.y, hi.x, hi.y);
}

// acc + a * s, elementwise
__device__ __forceinline__ float4 f4_fma(float4 a, float s, float4 acc) {
  const float2 s2 = make_float2(s, s);
  const float2 lo = __ffma2_rn(make_float2(a.x, a.y), s2, make_float2(acc.x, acc.y));
  const float2 hi = __ffma2_rn(make_float2(a.z, a.w), s2, make_float2(acc.z, acc.w));
  return make_float4(lo.x, lo.y, hi.x, hi.y);
}

// sum over the row lanes (lane bits 2..4); every lane ends with the total
__device__ __forceinline__ float row_sum(float x) {
#pragma unroll
  for (int o = 4; o < 32; o <<= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

// E consecutive elements (E = 1, 2, 4; the address is E-element aligned) as
// floats
template <int E>
__device__ __forceinline__ void load_vec(const float* p, float* x) {
  if constexpr (E == 4) {
    const float4 v = *reinterpret_cast<const float4*>(p);
    x[0] = v.x; x[1] = v.y; x[2] = v.z; x[3] = v.w;
  } else if constexpr (E == 2) {
    const float2 v = *reinterpret_cast<const float2*>(p);
    x[0] = v.x; x[1] = v.y;
  } else {
    x[0] = *p;
  }
}
template <int E>
__device__ __forceinline__ void load_vec(const __nv_bfloat16* p, float* x) {
  if constexpr (E == 4) {
    const uint2 u = *reinterpret_cast<const uint2*>(p);
    const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.x));
    const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.y));
    x[0] = a.x; x[1] = a.y; x[2] = b.x; x[3] = b.y;
  } else if constexpr (E == 2) {
    const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(p));
    x[0] = a.x; x[1] = a.y;
  } else {
    x[0] = __bfloat162float(*p);
  }
}
template <int E>
__device__ __forceinline__ void store_vec(float* p, const float* x) {
  if constexpr (E == 4) {
    *reinterpret_cast<float4*>(p) = make_float4(x[0], x[1], x[2], x[3]);
  } else if constexpr (E == 2) {
    *reinterpret_cast<float2*>(p) = make_float2(x[0], x[1]);
  } else {
    p[0] = x[0];
  }
}

// four consecutive outputs (16-byte aligned for fp32, 8-byte for bf16)
__device__ __forceinline__ void store4(float* p, float4 x) { *reinterpret_cast<float4*>(p) = x; }
__device__ __forceinline__ void store4(__nv_bfloat16* p, float4 x) {
  const __nv_bfloat162 a = __floats2bfloat162_rn(x.x, x.y), b = __floats2bfloat162_rn(x.z, x.w);
  uint2 u;
  u.x = *reinterpret_cast<const uint32_t*>(&a);
  u.y = *reinterpret_cast<const uint32_t*>(&b);
  *reinterpret_cast<uint2*>(p) = u;
}

template <typename Tin, int DK, int DV, bool VERIFY>
__global__ void __launch_bounds__(threads_per_cta<DV>())
    decode_multi_kernel(const Tin* __restrict__ q, const Tin* __restrict__ k,
                        const Tin* __restrict__ v, const float* __restrict__ g,
                        const float* __restrict__ A_log, float g_min,
                        const float* __restrict__ beta, float* __restrict__ state,
                        const int32_t* __restrict__ accept_len, int H, int K, float scale,
                        Tin* __restrict__ out) {
  constexpr int DVC = cols_per_cta<DV>();  // value columns of this CTA
  constexpr int NSPLIT = DV / DVC;
  constexpr int NT = threads_per_cta<DV>();
  constexpr int NW = NT / 32;
  constexpr int RPL = DK / kRowLanes;      // key rows per lane
  constexpr int EPL = DK / 32;             // key elements per lane when staging a token
  // token rows in shared memory: each row lane's RPL keys padded by 4 floats,
  // so the 8 row lanes' float4 reads fall in distinct bank groups
  constexpr int RPS = RPL + 4, KS = kRowLanes * RPS;
  static_assert(DVC % kWarpCols == 0 && RPL % 4 == 0 && RPL % EPL == 0, "tile shape");
  auto kpos = [](int i) { return (i / RPL) * RPS + i % RPL; };

  // read as float4
  __shared__ __align__(16) float sk[kMaxK][KS], sq[VERIFY ? kMaxK : 1][KS], sa[kMaxK][KS];
  __shared__ __align__(16) float sv[kMaxK][DVC];
  __shared__ float sb[kMaxK], skq[kMaxK];

  const int unit = blockIdx.x / NSPLIT;  // n * H + h
  const int j0 = (blockIdx.x % NSPLIT) * DVC;
  const int n = unit / H, h = unit % H;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int rl = lane >> 2;                             // row lane
  const int jc = warp * kWarpCols + (lane & 3) * 4;     // first column, within the slice

  int steps = K;
  if (!VERIFY) {
    steps = accept_len[n];
    steps = steps < 0 ? 0 : (steps > K ? K : steps);
    if (steps == 0) return;  // nothing accepted: the committed state stands
  }

  // Token inputs, [N, K, H, *] layouts, one warp per token; g is the
  // log-decay, or z when A_log is given (gate fused in).  The first token's
  // loads go out before the state's, the rest after.
  const float a_h = A_log ? expf(A_log[h]) : 0.f;
  float kv[EPL], qv[EPL], gv[EPL];
  auto load_token = [&](int t) {
    const size_t off = (((size_t)n * K + t) * H + h) * DK + lane * EPL;
    load_vec<EPL>(k + off, kv);
    if (VERIFY) load_vec<EPL>(q + off, qv);
    load_vec<EPL>(g + off, gv);
  };
  if (warp < steps) load_token(warp);

  float4* S4 = reinterpret_cast<float4*>(state + (size_t)unit * DK * DV + j0 + jc);
  float4 s[RPL];
#pragma unroll
  for (int r = 0; r < RPL; ++r) s[r] = S4[(size_t)(rl * RPL + r) * (DV / 4)];

  for (int t = warp; t < steps; t += NW) {
    if (t != warp) load_token(t);
    float av[EPL];
    float kq = 0.f;
#pragma unroll
    for (int e = 0; e < EPL; ++e) {
      av[e] = expf(A_log ? gate_value(gv[e], a_h, g_min) : gv[e]);
      if (VERIFY) kq = fmaf(kv[e], qv[e], kq);
    }
    store_vec<EPL>(&sk[t][kpos(lane * EPL)], kv);
    store_vec<EPL>(&sa[t][kpos(lane * EPL)], av);
    if (VERIFY) {
      store_vec<EPL>(&sq[t][kpos(lane * EPL)], qv);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) kq += __shfl_xor_sync(0xffffffffu, kq, o);
      if (lane == 0) skq[t] = kq;
    }
  }
  for (int idx = tid; idx < steps * (DVC / 4); idx += NT) {
    const int t = idx / (DVC / 4), j = 4 * (idx % (DVC / 4));
    float x[4];
    load_vec<4>(v + (((size_t)n * K + t) * H + h) * DV + j0 + j, x);
    store_vec<4>(&sv[t][j], x);
  }
  for (int t = tid; t < steps; t += NT) sb[t] = beta[((size_t)n * K + t) * H + h];
  __syncthreads();

  for (int t = 0; t < steps; ++t) {
    // decay, then p = S^T k and (verify) r = S^T q over this lane's rows
    float4 p = make_float4(0.f, 0.f, 0.f, 0.f), rq = p;
    const float4* k4 = reinterpret_cast<const float4*>(&sk[t][rl * RPS]);
    const float4* q4 = reinterpret_cast<const float4*>(&sq[VERIFY ? t : 0][rl * RPS]);
    const float4* a4 = reinterpret_cast<const float4*>(&sa[t][rl * RPS]);
#pragma unroll
    for (int r4 = 0; r4 < RPL / 4; ++r4) {
      const float4 kk = k4[r4], aa = a4[r4];
      const float kx[4] = {kk.x, kk.y, kk.z, kk.w}, ax[4] = {aa.x, aa.y, aa.z, aa.w};
      float qx[4] = {0.f, 0.f, 0.f, 0.f};
      if (VERIFY) {
        const float4 qq = q4[r4];
        qx[0] = qq.x; qx[1] = qq.y; qx[2] = qq.z; qx[3] = qq.w;
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        float4& x = s[4 * r4 + u];
        x = f4_mul(x, ax[u]);
        p = f4_fma(x, kx[u], p);
        if (VERIFY) rq = f4_fma(x, qx[u], rq);
      }
    }
    p.x = row_sum(p.x); p.y = row_sum(p.y); p.z = row_sum(p.z); p.w = row_sum(p.w);
    const float bt = sb[t];
    const float4 vj = *reinterpret_cast<const float4*>(&sv[t][jc]);
    const float4 e = make_float4(bt * (vj.x - p.x), bt * (vj.y - p.y),
                                 bt * (vj.z - p.z), bt * (vj.w - p.w));
    if (VERIFY) {
      // o_t = scale * q_t^T S_t = scale * (r + (q.k) e), S_t after the update
      rq.x = row_sum(rq.x); rq.y = row_sum(rq.y); rq.z = row_sum(rq.z); rq.w = row_sum(rq.w);
      if (rl == (t & (kRowLanes - 1))) {
        const float kq = skq[t];
        store4(out + (((size_t)n * K + t) * H + h) * DV + j0 + jc,
               make_float4(scale * fmaf(kq, e.x, rq.x), scale * fmaf(kq, e.y, rq.y),
                           scale * fmaf(kq, e.z, rq.z), scale * fmaf(kq, e.w, rq.w)));
      }
    }
    // S_t = S' + k_t e^T
    const float2 e01 = make_float2(e.x, e.y), e23 = make_float2(e.z, e.w);
#pragma unroll
    for (int r4 = 0; r4 < RPL / 4; ++r4) {
      const float4 kk = k4[r4];
      const float kx[4] = {kk.x, kk.y, kk.z, kk.w};
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        float4& x = s[4 * r4 + u];
        const float2 k2 = make_float2(kx[u], kx[u]);
        const float2 lo = __ffma2_rn(k2, e01, make_float2(x.x, x.y));
        const float2 hi = __ffma2_rn(k2, e23, make_float2(x.z, x.w));
        x = make_float4(lo.x, lo.y, hi.x, hi.y);
      }
    }
  }
  if (!VERIFY) {
#pragma unroll
    for (int r = 0; r < RPL; ++r) S4[(size_t)(rl * RPL + r) * (DV / 4)] = s[r];
  }
}

template <typename Tin, int DK, int DV, bool VERIFY>
cudaError_t launch3(const DecodeMultiArgs& a, cudaStream_t st) {
  decode_multi_kernel<Tin, DK, DV, VERIFY>
      <<<(unsigned)(a.N * a.H * (DV / cols_per_cta<DV>())), threads_per_cta<DV>(), 0, st>>>(
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
