// kda_chunk_simt.cu -- chunkwise KDA forward on CUDA cores, fp32 throughout.
//
// This kernel serves fp32 inputs (where single-pass tensor-core operands
// would not meet fp32 accuracy) and every (dk, dv, chunk) combination the
// tcgen05 kernel does not cover.  It evaluates the same chunk form as the
// tensor-core kernel (the WY/UT representation of the product of
// (I - beta k k^T) Diag(alpha) factors, "NLP--技术报告解读-Kimi-K3",
// Model Architecture > KDA update equation; chunkwise evaluation per
// Infrastructure > KDA kernels), with every exponent taken as a difference
// Gamma_r - Gamma_s <= 0 so nothing can overflow:
//
//   Gamma = cumsum(g) within the chunk;  L[r,s] = sum_i k_ri k_si e^{Gamma_ri - Gamma_si}
//   A = Diag(beta) strict_lower(L);  T = (I + A)^-1 Diag(beta)
//   U = T (V - (k e^Gamma) S);  O = scale((q e^Gamma) S + lower(Lq) U)
//   S <- Diag(e^{Gamma_C}) S + (k e^{Gamma_C - Gamma})^T U
//
// One CTA owns one (sequence, head) and a 32-wide slice of the dv columns
// (the key-side work is recomputed per slice).  The state slice stays in
// shared memory for the whole sequence.
#include "kda_internal.cuh"

namespace kda {
namespace {

constexpr int kThreads = 256;
constexpr int kDVS = 32;  // dv columns per CTA

template <int DK, int C>
struct SimtSmem {
  static constexpr int LDK = DK + 1, LDC = C + 1, LDV = kDVS + 1;
  static constexpr int floats = 3 * C * LDK      // k/Kc, q/Qg, Gamma/Ka
                                + 3 * C * LDC    // A (then T), Aq, X
                                + 3 * C * LDV    // V-P, P, U
                                + DK * LDV       // state slice
                                + C + DK;        // beta, gamma_C
  static constexpr size_t bytes = sizeof(float) * floats;
};

template <typename Tin, int DK, int C>
__global__ void __launch_bounds__(kThreads, 1)
    chunk_simt_kernel(const Tin* __restrict__ q, const Tin* __restrict__ k,
                      const Tin* __restrict__ v, const float* __restrict__ g,
                      const float* __restrict__ A_log, float g_min,
                      const float* __restrict__ beta, const float* __restrict__ init_state,
                      float* __restrict__ final_state, Tin* __restrict__ out, UnitMap map,
                      int dv, float scale) {
  using SM = SimtSmem<DK, C>;
  constexpr int LDK = SM::LDK, LDC = SM::LDC, LDV = SM::LDV;
  extern __shared__ float smem[];
  float* kS = smem;                 // [C][LDK]  k, later Kc
  float* qS = kS + C * LDK;         // [C][LDK]  q, later Q_gamma
  float* GS = qS + C * LDK;         // [C][LDK]  Gamma, later Ka
  float* AS = GS + C * LDK;         // [C][LDC]  A_kk, later T
  float* AqS = AS + C * LDC;        // [C][LDC]  A_qk
  float* XS = AqS + C * LDC;        // [C][LDC]  (I + A)^-1
  float* VS = XS + C * LDC;         // [C][LDV]  V, later V - P
  float* PS = VS + C * LDV;         // [C][LDV]  Ka S
  float* US = PS + C * LDV;         // [C][LDV]  U
  float* SS = US + C * LDV;         // [DK][LDV] state slice
  float* bS = SS + DK * LDV;        // [C]
  float* gC = bS + C;               // [DK]

  const int tid = threadIdx.x;
  const int H = map.H;
  const int nslices = dv / kDVS;
  const int unit = blockIdx.x / nslices;
  const int j0 = (blockIdx.x % nslices) * kDVS;
  const int h = unit % H;
  int64_t row0, L, sidx;
  if (map.cu_seqlens == nullptr) {
    const int b = unit / H;
    row0 = (int64_t)b * map.T;
    L = map.T;
    sidx = unit;
  } else {
    if (map.status->seqlens_ok != 1) return;
    const int n = map.order ? map.order[unit / H] : unit / H;
    row0 = map.cu_seqlens[n];
    L = (int64_t)map.cu_seqlens[n + 1] - row0;
    sidx = (int64_t)n * H + h;
  }
  {  // KDA_DEBUG_CHECKS builds: the unit's rows and state slot
    StatusBlock* sb = const_cast<StatusBlock*>(map.status);
    const int64_t rows = (int64_t)map.B * map.T;
    if (!in_bounds(sb, L, rows + 1, kSiteSimtUnitRows) ||
        (L > 0 && !(in_bounds(sb, row0, rows, kSiteSimtUnitRows) &&
                    in_bounds(sb, row0 + L - 1, rows, kSiteSimtUnitRows))) ||
        !in_bounds(sb, sidx, gridDim.x / nslices, kSiteSimtStateSlot))
      return;
  }

  // g is the log-decay, or z when A_log is given (gate fused in)
  const float a_h = A_log ? expf(A_log[h]) : 0.f;

  // state slice
  for (int idx = tid; idx < DK * kDVS; idx += kThreads) {
    const int i = idx / kDVS, j = idx % kDVS;
    SS[i * LDV + j] = init_state ? init_state[(sidx * DK + i) * dv + j0 + j] : 0.f;
  }

  for (int64_t t0 = 0; t0 < L; t0 += C) {
    const int n = (int)((L - t0) < C ? (L - t0) : C);
    __syncthreads();
    for (int idx = tid; idx < C * DK; idx += kThreads) {
      const int r = idx / DK, i = idx % DK;
      float kv = 0.f, qv = 0.f, gv = 0.f;
      if (r < n) {
        const size_t off = ((size_t)(row0 + t0 + r) * H + h) * DK + i;
        kv = Elem<Tin>::load(k + off);
        qv = Elem<Tin>::load(q + off);
        gv = g[off];
        if (A_log) gv = gate_value(gv, a_h, g_min);
      }
      kS[r * LDK + i] = kv;
      qS[r * LDK + i] = qv;
      GS[r * LDK + i] = gv;
    }
    for (int idx = tid; idx < C * kDVS; idx += kThreads) {
      const int r = idx / kDVS, j = idx % kDVS;
      VS[r * LDV + j] = r < n ? Elem<Tin>::load(v + ((size_t)(row0 + t0 + r) * H + h) * dv + j0 + j) : 0.f;
    }
    for (int r = tid; r < C; r += kThreads)
      bS[r] = r < n ? beta[(size_t)(row0 + t0 + r) * H + h] : 0.f;
    __syncthreads();

    // Gamma = inclusive cumsum of g along the chunk
    for (int i = tid; i < DK; i += kThreads) {
      float acc = 0.f;
      for (int r = 0; r < C; ++r) {
        acc += GS[r * LDK + i];
        GS[r * LDK + i] = acc;
      }
    }
    __syncthreads();

    // Gram matrices with exact exponent differences (s <= r)
    constexpr int npairs = C * (C + 1) / 2;
    for (int p = tid; p < npairs; p += kThreads) {
      int r = (int)((sqrtf(8.f * p + 1.f) - 1.f) * 0.5f);
      while ((r + 1) * (r + 2) / 2 <= p) ++r;
      while (r * (r + 1) / 2 > p) --r;
      const int s = p - r * (r + 1) / 2;
      float lk = 0.f, lq = 0.f;
      for (int i = 0; i < DK; ++i) {
        const float d = expf(GS[r * LDK + i] - GS[s * LDK + i]);
        const float ks = kS[s * LDK + i] * d;
        lk = fmaf(kS[r * LDK + i], ks, lk);
        lq = fmaf(qS[r * LDK + i], ks, lq);
      }
      AS[r * LDC + s] = s < r ? bS[r] * lk : 0.f;
      AqS[r * LDC + s] = lq;
    }
    for (int idx = tid; idx < C * C; idx += kThreads) {
      const int r = idx / C, s = idx % C;
      if (s > r) {
        AS[r * LDC + s] = 0.f;
        AqS[r * LDC + s] = 0.f;
      }
    }
    __syncthreads();

    // X = (I + A)^-1, one column per thread (forward substitution)
    for (int c = tid; c < C; c += kThreads) {
      for (int r = 0; r < C; ++r) XS[r * LDC + c] = r == c ? 1.f : 0.f;
      for (int r = c + 1; r < C; ++r) {
        float acc = 0.f;
        for (int s = c; s < r; ++s) acc = fmaf(AS[r * LDC + s], XS[s * LDC + c], acc);
        XS[r * LDC + c] = -acc;
      }
    }
    // decayed operands; Gamma_C saved first
    for (int i = tid; i < DK; i += kThreads) gC[i] = GS[(C - 1) * LDK + i];
    __syncthreads();
    for (int idx = tid; idx < C * C; idx += kThreads) {
      const int r = idx / C, s = idx % C;
      AS[r * LDC + s] = XS[r * LDC + s] * bS[s];  // T = X Diag(beta)
    }
    for (int idx = tid; idx < C * DK; idx += kThreads) {
      const int r = idx / DK, i = idx % DK;
      const float G = GS[r * LDK + i];
      const float e = expf(G);
      qS[r * LDK + i] *= e;                               // Q_gamma
      const float kv = kS[r * LDK + i];
      GS[r * LDK + i] = kv * e;                           // Ka
      kS[r * LDK + i] = kv * expf(gC[i] - G);             // Kc
    }
    __syncthreads();
    for (int i = tid; i < DK; i += kThreads) gC[i] = expf(gC[i]);

    // P = Ka S;  V <- V - P
    for (int idx = tid; idx < C * kDVS; idx += kThreads) {
      const int r = idx / kDVS, j = idx % kDVS;
      float acc = 0.f;
      for (int i = 0; i < DK; ++i) acc = fmaf(GS[r * LDK + i], SS[i * LDV + j], acc);
      PS[r * LDV + j] = acc;
      VS[r * LDV + j] -= acc;
    }
    __syncthreads();
    // U = T (V - P)
    for (int idx = tid; idx < C * kDVS; idx += kThreads) {
      const int r = idx / kDVS, j = idx % kDVS;
      float acc = 0.f;
      for (int s = 0; s <= r; ++s) acc = fmaf(AS[r * LDC + s], VS[s * LDV + j], acc);
      US[r * LDV + j] = acc;
    }
    __syncthreads();
    // O = scale (Q_gamma S + A_qk U)
    for (int idx = tid; idx < C * kDVS; idx += kThreads) {
      const int r = idx / kDVS, j = idx % kDVS;
      if (r >= n) continue;
      float acc = 0.f;
      for (int i = 0; i < DK; ++i) acc = fmaf(qS[r * LDK + i], SS[i * LDV + j], acc);
      for (int s = 0; s <= r; ++s) acc = fmaf(AqS[r * LDC + s], US[s * LDV + j], acc);
      Elem<Tin>::store(out + ((size_t)(row0 + t0 + r) * H + h) * dv + j0 + j, scale * acc);
    }
    __syncthreads();
    // S <- Diag(gamma_C) S + Kc^T U
    for (int idx = tid; idx < DK * kDVS; idx += kThreads) {
      const int i = idx / kDVS, j = idx % kDVS;
      float acc = gC[i] * SS[i * LDV + j];
      for (int s = 0; s < C; ++s) acc = fmaf(kS[s * LDK + i], US[s * LDV + j], acc);
      SS[i * LDV + j] = acc;
    }
  }
  __syncthreads();
  if (final_state) {
    for (int idx = tid; idx < DK * kDVS; idx += kThreads) {
      const int i = idx / kDVS, j = idx % kDVS;
      final_state[(sidx * DK + i) * dv + j0 + j] = SS[i * LDV + j];
    }
  }
}

template <typename Tin, int DK, int C>
cudaError_t launch_one(const ChunkArgs& a, cudaStream_t st) {
  auto kern = chunk_simt_kernel<Tin, DK, C>;
  const size_t smem = SimtSmem<DK, C>::bytes;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const unsigned grid = (unsigned)(a.num_units * (a.dv / kDVS));
  kern<<<grid, kThreads, smem, st>>>(static_cast<const Tin*>(a.q), static_cast<const Tin*>(a.k),
                                     static_cast<const Tin*>(a.v), a.g,
                                     a.gated ? a.A_log : nullptr, a.g_min, a.beta, a.init_state,
                                     a.final_state, static_cast<Tin*>(a.out), a.map, a.dv,
                                     a.scale);
  return cudaGetLastError();
}

template <typename Tin, int DK>
cudaError_t by_chunk(const ChunkArgs& a, cudaStream_t st) {
  switch (a.chunk) {
    case 16: return launch_one<Tin, DK, 16>(a, st);
    case 32: return launch_one<Tin, DK, 32>(a, st);
    case 64: return launch_one<Tin, DK, 64>(a, st);
    default: return cudaErrorInvalidValue;
  }
}

template <typename Tin>
cudaError_t by_dk(const ChunkArgs& a, cudaStream_t st) {
  switch (a.dk) {
    case 32: return by_chunk<Tin, 32>(a, st);
    case 64: return by_chunk<Tin, 64>(a, st);
    case 128: return by_chunk<Tin, 128>(a, st);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace

cudaError_t launch_chunk_simt(const ChunkArgs& a, cudaStream_t stream) {
  if (a.num_units == 0) return cudaSuccess;
  if (a.dt == KDA_BF16) return by_dk<__nv_bfloat16>(a, stream);
  return by_dk<float>(a, stream);
}

}  // namespace kda
