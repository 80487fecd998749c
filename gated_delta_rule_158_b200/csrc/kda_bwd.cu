// kda_bwd.cu -- gradients through the KDA recurrence (the training backward).
//
// Forward ("NLP--技术报告解读-Kimi-K3", joezjh.github.io, Model Architecture >
// Kimi Delta Attention (KDA)), per (sequence, head) and token t:
//   S'_t = Diag(a_t) S_{t-1},  a_t = exp(g_t);   p_t = S'_t^T k_t;
//   e_t = beta_t (v_t - p_t);  S_t = S'_t + k_t e_t^T;  o_t = scale S_t^T q_t.
// The pages give no backward; this is the chain rule on those steps, in
// reverse token order, with G = dL/dS_t:
//   G += scale q_t do_t^T;                 dq_t = scale (a_t . (S_{t-1} do_t) + k_t (e_t . do_t))
//   de = G^T k_t;  dv_t = beta_t de;       dbeta_t = de . (v_t - p_t)
//   dk_t = G e_t - beta_t a_t . (S_{t-1} de)
//   G' = G - beta_t k_t de^T;              dg_t = a_t . rowsum(G' . S_{t-1})
//   G = Diag(a_t) G'   (= dL/dS_{t-1}),    dS_0 = G at the end.
//
// Layout and roles as in kda_decode.cu: one CTA of 256 threads per
// (sequence, head); thread t keeps a float4 column group of RPT rows of the
// state and of G in registers.  The states the reverse sweep needs are
// recomputed: pass 1 runs the recurrence forward and saves the state every
// kCB tokens; pass 2 takes the blocks last to first, recomputes a block's
// pre-token states into the workspace (p_t and e_t into shared memory) and
// then sweeps it backward.  Column sums go through shared memory, row sums
// through warp shuffles; every output element has one writer.
//
// Cost: about two state reads and one state write per token (128 KB of
// traffic per token-head at dk = dv = 128) on top of the forward's
// arithmetic -- a correctness-first kernel, bound by that traffic.
#include "kda_bwd.cuh"

namespace kda {
namespace {

constexpr int kThreads = 256;
constexpr int kCB = 64;  // tokens per recompute block

template <int CG>
__device__ __forceinline__ float row_sum(float x) {  // over the CG lanes of a row group
#pragma unroll
  for (int o = CG / 2; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

__device__ __forceinline__ float dot4(float4 a, float4 b) {
  return fmaf(a.x, b.x, fmaf(a.y, b.y, fmaf(a.z, b.z, a.w * b.w)));
}

template <typename Tin, int DK, int DV>
__global__ void __launch_bounds__(kThreads, 1)
    bwd_kernel(const Tin* __restrict__ q, const Tin* __restrict__ k, const Tin* __restrict__ v,
               const float* __restrict__ g, const float* __restrict__ beta,
               const float* __restrict__ init, const Tin* __restrict__ dout,
               const float* __restrict__ dfinal, int T, int H, float scale,
               float* __restrict__ dq, float* __restrict__ dk, float* __restrict__ dv,
               float* __restrict__ dg, float* __restrict__ dbeta, float* __restrict__ dinit,
               float* __restrict__ ws) {
  constexpr int CG = DV / 4;         // threads per state row (float4 each)
  constexpr int RG = kThreads / CG;  // row groups
  constexpr int RPT = DK / RG;       // rows per thread
  static_assert(RPT >= 1 && DK % RG == 0 && CG <= 32, "tile shape");

  extern __shared__ __align__(16) float dsm[];
  float* sp = dsm;              // p_t of the block's tokens [kCB][DV]
  float* se = dsm + kCB * DV;   // e_t                       [kCB][DV]
  __shared__ float4 red[RG][CG];
  __shared__ float sk[DK], sa[DK], sq[DK];
  // read back as float4
  __shared__ __align__(16) float sv[DV];
  __shared__ __align__(16) float sdo[DV];
  __shared__ __align__(16) float sde[DV];
  __shared__ __align__(16) float secur[DV];
  __shared__ float sred[2][kThreads / 32];
  __shared__ float s_bt, s_edo;

  const int unit = blockIdx.x;  // b * H + h
  const int b = unit / H, h = unit % H;
  const int tid = threadIdx.x, cg = tid % CG, rg = tid / CG;
  const int lane = tid & 31, wid = tid >> 5;
  const int nblk = (T + kCB - 1) / kCB;
  const size_t SZ = (size_t)DK * DV;
  float4* ckpt = reinterpret_cast<float4*>(ws + (size_t)unit * (nblk + kCB) * SZ);
  float4* pre = ckpt + (size_t)nblk * (SZ / 4);
  auto row = [&](int r) { return rg + r * RG; };
  auto tok = [&](int t) { return ((size_t)b * T + t) * H + h; };

  float4 S[RPT];
#pragma unroll
  for (int r = 0; r < RPT; ++r)
    S[r] = init ? reinterpret_cast<const float4*>(init + unit * SZ)[row(r) * CG + cg]
                : make_float4(0.f, 0.f, 0.f, 0.f);

  // one token of the recurrence on S (registers); p_t, e_t into row u of
  // sp / se when u >= 0
  auto fwd_step = [&](int t, int u) {
    const size_t o = tok(t);
    for (int i = tid; i < DK; i += kThreads) {
      sk[i] = Elem<Tin>::load(k + o * DK + i);
      sa[i] = expf(g[o * DK + i]);
    }
    for (int j = tid; j < DV; j += kThreads) sv[j] = Elem<Tin>::load(v + o * DV + j);
    if (tid == 0) s_bt = beta[o];
    __syncthreads();
    float4 p = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int r = 0; r < RPT; ++r) {
      const int i = row(r);
      const float a = sa[i], ki = sk[i];
      S[r].x *= a; S[r].y *= a; S[r].z *= a; S[r].w *= a;
      p.x = fmaf(S[r].x, ki, p.x); p.y = fmaf(S[r].y, ki, p.y);
      p.z = fmaf(S[r].z, ki, p.z); p.w = fmaf(S[r].w, ki, p.w);
    }
    red[rg][cg] = p;
    __syncthreads();
    if (tid < DV) {
      const float* rp = reinterpret_cast<const float*>(red);
      float pj = 0.f;
#pragma unroll 8
      for (int w = 0; w < RG; ++w) pj += rp[w * DV + tid];
      const float ej = s_bt * (sv[tid] - pj);
      secur[tid] = ej;
      if (u >= 0) {
        sp[u * DV + tid] = pj;
        se[u * DV + tid] = ej;
      }
    }
    __syncthreads();
    const float4 e4 = reinterpret_cast<const float4*>(secur)[cg];
#pragma unroll
    for (int r = 0; r < RPT; ++r) {
      const float ki = sk[row(r)];
      S[r].x = fmaf(ki, e4.x, S[r].x); S[r].y = fmaf(ki, e4.y, S[r].y);
      S[r].z = fmaf(ki, e4.z, S[r].z); S[r].w = fmaf(ki, e4.w, S[r].w);
    }
    __syncthreads();  // sk, sa, sv, red, secur are rewritten by the next token
  };

  // ---- pass 1: forward, saving the state at every block start
  for (int t = 0; t < T; ++t) {
    if (t % kCB == 0) {
#pragma unroll
      for (int r = 0; r < RPT; ++r) ckpt[(size_t)(t / kCB) * (SZ / 4) + row(r) * CG + cg] = S[r];
    }
    fwd_step(t, -1);
  }

  // ---- pass 2: blocks last to first
  float4 G[RPT];
#pragma unroll
  for (int r = 0; r < RPT; ++r)
    G[r] = dfinal ? reinterpret_cast<const float4*>(dfinal + unit * SZ)[row(r) * CG + cg]
                  : make_float4(0.f, 0.f, 0.f, 0.f);
  for (int blk = nblk - 1; blk >= 0; --blk) {
    const int t0 = blk * kCB;
    const int n = (T - t0) < kCB ? (T - t0) : kCB;
#pragma unroll
    for (int r = 0; r < RPT; ++r) S[r] = ckpt[(size_t)blk * (SZ / 4) + row(r) * CG + cg];
    for (int u = 0; u < n; ++u) {  // the block's pre-token states
#pragma unroll
      for (int r = 0; r < RPT; ++r) pre[(size_t)u * (SZ / 4) + row(r) * CG + cg] = S[r];
      fwd_step(t0 + u, u);
    }
    for (int u = n - 1; u >= 0; --u) {
      const int t = t0 + u;
      const size_t o = tok(t);
#pragma unroll
      for (int r = 0; r < RPT; ++r) S[r] = pre[(size_t)u * (SZ / 4) + row(r) * CG + cg];  // S_{t-1}
      for (int i = tid; i < DK; i += kThreads) {
        sk[i] = Elem<Tin>::load(k + o * DK + i);
        sq[i] = Elem<Tin>::load(q + o * DK + i);
        sa[i] = expf(g[o * DK + i]);
      }
      for (int j = tid; j < DV; j += kThreads) {
        sv[j] = Elem<Tin>::load(v + o * DV + j);
        sdo[j] = Elem<Tin>::load(dout + o * DV + j);
      }
      if (tid == 0) s_bt = beta[o];
      __syncthreads();
      // G += scale q do^T;  de = G^T k
      const float4 do4 = reinterpret_cast<const float4*>(sdo)[cg];
      float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int r = 0; r < RPT; ++r) {
        const int i = row(r);
        G[r] = make_float4(fmaf(scale * sq[i], do4.x, G[r].x), fmaf(scale * sq[i], do4.y, G[r].y),
                           fmaf(scale * sq[i], do4.z, G[r].z), fmaf(scale * sq[i], do4.w, G[r].w));
        const float ki = sk[i];
        acc.x = fmaf(G[r].x, ki, acc.x); acc.y = fmaf(G[r].y, ki, acc.y);
        acc.z = fmaf(G[r].z, ki, acc.z); acc.w = fmaf(G[r].w, ki, acc.w);
      }
      red[rg][cg] = acc;
      __syncthreads();
      float pb = 0.f, pe = 0.f;  // partials of dbeta and of e . do
      if (tid < DV) {
        const float* rp = reinterpret_cast<const float*>(red);
        float dej = 0.f;
#pragma unroll 8
        for (int w = 0; w < RG; ++w) dej += rp[w * DV + tid];
        sde[tid] = dej;
        dv[o * DV + tid] = s_bt * dej;
        pb = dej * (sv[tid] - sp[u * DV + tid]);
        pe = se[u * DV + tid] * sdo[tid];
      }
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) {
        pb += __shfl_xor_sync(0xffffffffu, pb, off);
        pe += __shfl_xor_sync(0xffffffffu, pe, off);
      }
      if (lane == 0) {
        sred[0][wid] = pb;
        sred[1][wid] = pe;
      }
      __syncthreads();
      if (tid == 0) {
        float tb = 0.f, te = 0.f;
        for (int w = 0; w < kThreads / 32; ++w) {
          tb += sred[0][w];
          te += sred[1][w];
        }
        dbeta[o] = tb;
        s_edo = te;
      }
      __syncthreads();
      // per row i: dq, dk, then G' = G - beta k de^T, dg, G = Diag(a) G'
      const float4 e4 = reinterpret_cast<const float4*>(se + u * DV)[cg];
      const float4 de4 = reinterpret_cast<const float4*>(sde)[cg];
      const float bt = s_bt, edo = s_edo;
#pragma unroll
      for (int r = 0; r < RPT; ++r) {
        const int i = row(r);
        const float a = sa[i], ki = sk[i];
        const float s_do = row_sum<CG>(dot4(S[r], do4));
        const float g_e = row_sum<CG>(dot4(G[r], e4));
        const float s_de = row_sum<CG>(dot4(S[r], de4));
        const float nb = -bt * ki;
        G[r] = make_float4(fmaf(de4.x, nb, G[r].x), fmaf(de4.y, nb, G[r].y),
                           fmaf(de4.z, nb, G[r].z), fmaf(de4.w, nb, G[r].w));
        const float gs = row_sum<CG>(dot4(G[r], S[r]));
        if (cg == 0) {
          dq[o * DK + i] = scale * fmaf(a, s_do, ki * edo);
          dk[o * DK + i] = g_e - bt * a * s_de;
          dg[o * DK + i] = gs * a;
        }
        G[r].x *= a; G[r].y *= a; G[r].z *= a; G[r].w *= a;
      }
      __syncthreads();  // the token's shared inputs are rewritten by the next
    }
  }
  if (dinit) {
#pragma unroll
    for (int r = 0; r < RPT; ++r)
      reinterpret_cast<float4*>(dinit + unit * SZ)[row(r) * CG + cg] = G[r];
  }
}

template <typename Tin, int DK, int DV>
cudaError_t launch3(const BwdArgs& a, cudaStream_t st) {
  const size_t smem = (size_t)2 * kCB * DV * sizeof(float);
  static bool attr_done = false;
  if (!attr_done) {
    cudaError_t e = cudaFuncSetAttribute(bwd_kernel<Tin, DK, DV>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    attr_done = true;
  }
  bwd_kernel<Tin, DK, DV><<<(unsigned)(a.B * a.H), kThreads, smem, st>>>(
      static_cast<const Tin*>(a.q), static_cast<const Tin*>(a.k), static_cast<const Tin*>(a.v),
      a.g, a.beta, a.init, static_cast<const Tin*>(a.dout), a.dfinal, a.T, a.H, a.scale, a.dq,
      a.dk, a.dv, a.dg, a.dbeta, a.dinit, a.ws);
  return cudaGetLastError();
}

template <typename Tin, int DK>
cudaError_t by_dv(const BwdArgs& a, cudaStream_t st) {
  switch (a.dv_dim) {
    case 32: return launch3<Tin, DK, 32>(a, st);
    case 64: return launch3<Tin, DK, 64>(a, st);
    case 128: return launch3<Tin, DK, 128>(a, st);
    default: return cudaErrorInvalidValue;
  }
}

template <typename Tin>
cudaError_t by_dk(const BwdArgs& a, cudaStream_t st) {
  switch (a.dk_dim) {
    case 32: return by_dv<Tin, 32>(a, st);
    case 64: return by_dv<Tin, 64>(a, st);
    case 128: return by_dv<Tin, 128>(a, st);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace

size_t bwd_workspace_bytes(int B, int T, int H, int dk, int dv) {
  const size_t nblk = ((size_t)T + kCB - 1) / kCB;
  return (size_t)B * H * (nblk + kCB) * dk * dv * sizeof(float);
}

cudaError_t launch_bwd(const BwdArgs& a, cudaStream_t stream) {
  if (a.B * a.H == 0) return cudaSuccess;
  return a.dt == KDA_BF16 ? by_dk<__nv_bfloat16>(a, stream) : by_dk<float>(a, stream);
}

}  // namespace kda
