// kda_chunk_tc.cu -- chunkwise KDA forward on the sm_100a tensor cores
// (tcgen05 + TMEM + TMA), bf16 q/k/v, fp32 g/beta/state, dk = dv = 128.
//
// What it computes: the KDA recurrence of "NLP--技术报告解读-Kimi-K3"
// (joezjh.github.io), Model Architecture > Kimi Delta Attention (KDA),
//   S_t = (I - b_t k_t k_t^T) Diag(e^{g_t}) S_{t-1} + b_t k_t v_t^T,  o_t = S_t^T q_t,
// evaluated chunk by chunk (FlashKDA: Infrastructure > KDA kernels, "training
// and prefill") in the WY/UT form.  For a chunk of C = 32 tokens starting
// from state S, with Gamma_r the in-chunk cumulative sum of g:
//   L[r,s] = sum_i k_ri k_si e^{Gamma_ri - Gamma_si}          (Gram, s <= r)
//   T      = (I + Diag(b) strict_lower(L))^-1 Diag(b)
//   P      = (k e^Gamma) S,   U = T V - T P,
//   O      = (q e^Gamma) S + lower(Lq) U,
//   S     <- Diag(e^{Gamma_C}) S + (k e^{Gamma_C - Gamma})^T U.
// (T P is the W S of the WY form with W = T (k e^Gamma), associated the other
// way so that no W has to be formed.)
//
// Why C = 32 and one rebasing point.  The lower bound g >= -5 of the gate
// (same section, Lower-bounded decay) is what lets every Gram tile,
// diagonal included, be a plain tensor-core GEMM: with the rebasing point at
// row 15, the left factors x_r e^{Gamma_r - Gamma_15} and the right factor
// k_s e^{Gamma_15 - Gamma_s} both stay inside [e^-80, e^80] (16 steps of at
// most -5 on either side), far from fp32's e^88.7 limit; a longer chunk
// would need more than one rebasing point per tile.
//
// B200 mapping.  One CTA (256 threads) owns one (sequence, head) for its
// whole length; two CTAs share an SM (110 KB shared memory, 256 TMEM columns
// each), so one CTA's SIMT phases overlap the other's GEMMs.  The fp32 state
// never leaves the SM: it lives in TMEM as S^T (lane = value channel, column =
// key channel) and is read directly as the tf32 A operand of the state-side
// GEMMs.  tcgen05.mma costs a roughly fixed number of cycles per instruction
// up to N = 128-256 (measured: ~90 with A in TMEM, ~190 with A in shared
// memory), so products that share an A operand are fused into one wide MMA:
//   [O^T | P^T]  = S^T [q e^G ; k e^G]^T            (N = 64, 16 k-steps)
//   U^T         -= P^T T^T   onto  U^T = V^T T^T     (N = 32)
//   [S^T | O^T] += U^T [Kc ; A_qk]^T  after the decay (N = 160, 4 k-steps)
// The Gram and U~ = T V are bf16 (A in shared memory).  TMA brings q/k/g for
// the next chunk while the current one computes, and v into the Gram operand
// region once the Gram is done.  All MMAs are issued by one thread and
// tracked by mbarriers; every wait is bounded (kda_sync.cuh).
//
// TMEM columns: S^T [0,128) | O^T [128,160) | P^T [160,192) | U^T [192,224)
//               | Gram (M = 64 layout, lanes 0-15 of each quarter) [224,256)
#include <cuda.h>
#include <cudaTypedefs.h>

#include "kda_internal.cuh"
#include "kda_sync.cuh"
#include "kda_tc_ptx.cuh"

namespace kda {
namespace {

using namespace tc;

constexpr int C = 32;     // tokens per chunk
constexpr int D = 128;    // dk = dv
constexpr int NT = 256;   // threads per CTA

constexpr uint32_t S_COL = 0, O_COL = 128, P_COL = 160, U_COL = 192, G_COL = 224;
constexpr uint32_t TMEM_COLS = 256;

// shared memory map (byte offsets from a 1024-aligned base)
constexpr uint32_t SM_Q = 0;         // q tile  bf16 [32][128] row-major (TMA, no swizzle)
constexpr uint32_t SM_K = 8192;      // k tile  bf16 [32][128]
constexpr uint32_t SM_G = 16384;     // g (or z) tile fp32 [32][128]; 4-row cumsum totals in prep
constexpr uint32_t SM_R1 = 32768;    // 24 KB, two lives:
constexpr uint32_t SM_KQL = SM_R1;            //  [k;q] e^{G-G15}  bf16 64 x 128 (Gram A)
constexpr uint32_t SM_KB = SM_R1 + 16384;     //  k e^{G15-G}      bf16 32 x 128 (Gram B)
                                              // and once the Gram GEMM is done:
constexpr uint32_t SM_TT = SM_R1;             //  T      bf16 [r][s] (B of U~)
constexpr uint32_t SM_TF = SM_R1 + 4096;      //  T      fp32 [r][s] (tf32 B of U -= P^T T^T)
constexpr uint32_t SM_V = SM_R1 + 8192;       //  v tile bf16, 2 x [32 rows x 128 B] swizzled (TMA)
constexpr uint32_t SM_AKKT = SM_R1 + 16384;   //  A_kk^T fp32 [s][r] 32 x 32 (inverse input)
constexpr uint32_t SM_XS = SM_R1 + 20480;     //  inverse blocks X00, X11 and A10 X00, fp32 32 x 32
constexpr uint32_t SM_QK = 57344;    // [q e^G ; k e^G] fp32, per 32-channel block 64 rows x 128 B
                                     // (tf32 B of [O | P])
constexpr uint32_t SM_KC = 90112;    // k e^{GC-G}   fp32 [i][s] (K-major tf32 B of S), rows 0-127,
constexpr uint32_t SM_AQK = 106496;  // A_qk         fp32 [r][s], rows 128-159 of the same B tile
constexpr uint32_t SM_MISC = 110592;
constexpr uint32_t SM_GAMC = SM_MISC;          // e^{Gamma_C}  fp32 [128]
constexpr uint32_t SM_BETA = SM_MISC + 512;    // beta         fp32 [32]
constexpr uint32_t SM_BAR = SM_MISC + 640;     // 5 mbarriers
constexpr uint32_t SM_TMEM = SM_MISC + 680;    // TMEM base address
constexpr uint32_t SM_ABORT = SM_MISC + 684;   // abort flag
constexpr uint32_t SMEM_BYTES = SM_MISC + 1024;
constexpr uint32_t SMEM_ALLOC = SMEM_BYTES + 1024;  // room to align the base to 1024
static_assert(SM_AQK == SM_KC + 16384, "A_qk rows must follow the Kc^T rows");
static_assert(2 * (SMEM_ALLOC + 1024) <= 228 * 1024, "two CTAs per SM");

constexpr uint32_t TX_QKG = 8192 + 8192 + 16384;
constexpr uint32_t TX_V = 8192;

struct TcParams {
  CUtensorMap tm_q, tm_k, tm_v, tm_g;  // tm_g maps g, or z when A_log is set
  const float* A_log;                  // gate fused in when not null
  float g_min;
  const float* beta;
  __nv_bfloat16* out;
  const float* init_state;
  float* final_state;
  const int32_t* cu_seqlens;
  const int32_t* order;
  StatusBlock* sb;
  float* seg_ws;  // segment states (split modes)
  int B, T, H;
  int mode;       // 0 whole units, 1 segment transitions, 2 segment outputs
  int G;          // segments per unit (modes 1, 2)
  int seg_len;    // tokens per segment (multiple of C)
  float scale;
};

struct Unit {
  int64_t row0, len;
  int h;
  const float* init;
  bool init_identity, vzero, out_on;
  float* final_state;
};

__device__ __forceinline__ bool resolve_unit(const TcParams& P, Unit& u) {
  const int H = P.H;
  const size_t DD = (size_t)D * D;
  u.init_identity = false;
  u.vzero = false;
  u.out_on = true;
  if (P.mode == 0) {
    const int idx = blockIdx.x;
    int64_t sidx;
    u.h = idx % H;
    if (P.cu_seqlens == nullptr) {
      const int b = idx / H;
      u.row0 = (int64_t)b * P.T;
      u.len = P.T;
      sidx = idx;
    } else {
      if (P.sb->seqlens_ok != 1) return false;
      const int n = P.order ? P.order[idx / H] : idx / H;
      u.row0 = P.cu_seqlens[n];
      u.len = (int64_t)P.cu_seqlens[n + 1] - u.row0;
      sidx = (int64_t)n * H + u.h;
    }
    u.init = P.init_state ? P.init_state + sidx * DD : nullptr;
    u.final_state = P.final_state ? P.final_state + sidx * DD : nullptr;
    return true;
  }
  const int U = P.B * H;
  if (P.mode == 1) {  // pairs (S~ from zero with v, M from I with v = 0)
    const int pair = blockIdx.x >> 1, kind = blockIdx.x & 1;
    const int un = pair / (P.G - 1), g = pair % (P.G - 1);
    u.h = un % H;
    u.row0 = (int64_t)(un / H) * P.T + (int64_t)g * P.seg_len;
    u.len = P.seg_len;
    u.init = nullptr;
    u.init_identity = kind == 1;
    u.vzero = kind == 1;
    u.out_on = false;
    u.final_state = P.seg_ws + ((size_t)(un * (P.G - 1) + g) * 2 + kind) * DD;
    return true;
  }
  // mode 2: outputs of every segment from its true incoming state
  const int un = blockIdx.x / P.G, g = blockIdx.x % P.G;
  u.h = un % H;
  u.row0 = (int64_t)(un / H) * P.T + (int64_t)g * P.seg_len;
  const int64_t rem = (int64_t)P.T - (int64_t)g * P.seg_len;
  u.len = rem < P.seg_len ? rem : P.seg_len;
  if (g == 0)
    u.init = P.init_state ? P.init_state + (size_t)un * DD : nullptr;
  else
    u.init = P.seg_ws + ((size_t)U * (P.G - 1) * 2 + (size_t)un * (P.G - 1) + (g - 1)) * DD;
  u.final_state = (g == P.G - 1 && P.final_state) ? P.final_state + (size_t)un * DD : nullptr;
  return true;
}

__global__ void __launch_bounds__(NT, 2) chunk_tc_kernel(const __grid_constant__ TcParams P) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_s = smem_u32(smem_raw);
  uint8_t* sm = smem_raw + ((1024u - (raw_s & 1023u)) & 1023u);
  const uint32_t sb = smem_u32(sm);

  Unit U;
  if (!resolve_unit(P, U)) return;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  uint64_t* bar_in = reinterpret_cast<uint64_t*>(sm + SM_BAR);
  uint64_t* bar_v = bar_in + 1;
  uint64_t* bar_mma = bar_in + 2;
  uint64_t* bar_u = bar_in + 3;      // U -= P^T T^T done
  uint64_t* bar_drain = bar_in + 4;  // abort path: every MMA issued so far done
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + SM_TMEM);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + SM_ABORT);
  float* gamc = reinterpret_cast<float*>(sm + SM_GAMC);
  float* betas = reinterpret_cast<float*>(sm + SM_BETA);
  const int H = P.H, h = U.h;

  if (tid == 0) {
    mbar_init(bar_in, 1);
    mbar_init(bar_v, 1);
    mbar_init(bar_mma, 1);
    mbar_init(bar_u, 1);
    mbar_init(bar_drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, TMEM_COLS);
    tmem_relinquish();
  }
  fence_before_sync();
  __syncthreads();
  fence_after_sync();
  const uint32_t tbase = *tmem_slot;
  const uint32_t lane_base = (uint32_t)(32 * (warp & 3)) << 16;  // this warp's TMEM lanes
  const int half = warp >> 2;                                   // column half (8-warp passes)

  const int nchunks = (int)((U.len + C - 1) / C);
  const float a2 = P.A_log ? expf(P.A_log[h]) * 1.4426950408889634f : 0.f;
  bool pend_in = false, pend_v = false;  // thread 0: TMA loads issued, not yet waited
  auto issue_qkg = [&](int c) {
    const int row = (int)(U.row0 + (int64_t)c * C);
    mbar_arrive_expect_tx(bar_in, TX_QKG);
    tma_load_3d(sm + SM_Q, &P.tm_q, bar_in, 0, h, row);
    tma_load_3d(sm + SM_K, &P.tm_k, bar_in, 0, h, row);
    tma_load_3d(sm + SM_G, &P.tm_g, bar_in, 0, h, row);
    pend_in = true;
  };
  auto issue_v = [&](int c) {  // into the Gram operand region: only once the Gram is done
    const int row = (int)(U.row0 + (int64_t)c * C);
    mbar_arrive_expect_tx(bar_v, TX_V);
    tma_load_3d(sm + SM_V, &P.tm_v, bar_v, 0, h, row);
    tma_load_3d(sm + SM_V + 4096, &P.tm_v, bar_v, 64, h, row);
    pend_v = true;
  };
  auto prefetch_v = [&](int c) {
    const int row = (int)(U.row0 + (int64_t)c * C);
    tma_prefetch_3d(&P.tm_v, 0, h, row);
    tma_prefetch_3d(&P.tm_v, 64, h, row);
  };
  if (tid == 0 && nchunks > 0) {
    issue_qkg(0);
    if (!U.vzero) prefetch_v(0);
  }

  // ---- initial state -> TMEM (S^T: lane j, column i)
  {
    const int j = 32 * (warp & 3) + lane;
    float v[32];
#pragma unroll
    for (int cc = 0; cc < 2; ++cc) {
      const int i0 = 64 * half + 32 * cc;
#pragma unroll
      for (int k = 0; k < 32; ++k) {
        const int i = i0 + k;
        v[k] = U.init ? U.init[(size_t)i * D + j] : ((U.init_identity && i == j) ? 1.f : 0.f);
      }
      tmem_st32(tbase + lane_base + S_COL + i0, v);
    }
    wait_st();
  }
  fence_before_sync();
  __syncthreads();

  uint32_t ph_in = 0, ph_v = 0, ph_mma = 0, ph_u = 0;
  const uint32_t id_gram = idesc(kFmtBF16, 64, C, false, false, false);
  const uint32_t id_tv = idesc(kFmtBF16, 128, C, true, false, false);        // U~^T = V^T T^T
  const uint32_t id_op = idesc(kFmtTF32, 128, 2 * C, false, false, false);   // [O^T | P^T]
  const uint32_t id_u = idesc(kFmtTF32, 128, C, false, false, true);         // U^T -= P^T T^T
  const uint32_t id_so = idesc(kFmtTF32, 128, D + C, false, false, false);   // [S^T | O^T]

  // prep thread mapping: channels c0 .. c0+3 and rows 4ro .. 4ro+3 (warp ro)
  const int cq = tid & 31, ro = tid >> 5, c0 = 4 * cq;
  // byte offsets of (row 4ro, channel c0) in each swizzled operand; a row
  // 4ro + rr adds rr*128 and xors the 16-byte chunk index with (4ro + rr) & 7
  const uint32_t ck16 = ((c0 & 63) * 2) >> 4, lo16 = ((c0 & 63) * 2) & 15;   // bf16 tiles
  const uint32_t ck32 = ((c0 & 31) * 4) >> 4;                                 // fp32 tiles
  const uint32_t o_kql = (c0 >> 6) * 8192 + ro * 512 + lo16;
  const uint32_t o_kb = (c0 >> 6) * 4096 + ro * 512 + lo16;
  const uint32_t o_qk = (c0 >> 5) * 8192 + ro * 512;
  constexpr float kLog2e = 1.4426950408889634f;
  const float gmin2 = P.g_min * kLog2e;
  auto chunk_rows = [&](int cc) -> int {
    const int64_t rem = U.len - (int64_t)cc * C;
    return (int)(rem < C ? rem : C);
  };

  float beta_next = 0.f;  // beta of the chunk after the one being prepared
  float4 G4[4];           // in-chunk cumulative log2-decay of the chunk being prepared
  float kc[4][4];         // its Kc values [channel][row], stored after the state update

  // ---- prep, part 1: wait for the chunk's tiles, beta, cumulative sums of g

  // ---- prep, part 2 (after a barrier): rescaled operands of the chunk

  // ---- Kc^T rows c0, c0+1: this thread's 8 rows are two 16-byte chunks of each

  // ---- O^T of chunk cc (lane j, column r) -> o rows; lanes j, j^1 swap values so
  //      each writes a bf16 pair (even lane rows 2m, odd lane rows 2m+1).  Warps 4-7.
  auto export_o = [&](int cc) {
    const int n = chunk_rows(cc);
    const int j = 32 * (warp & 3) + lane;
    const bool odd = lane & 1;
    float v[32];
    tmem_ld32(tbase + lane_base + O_COL, v);
    wait_ld();
    const int jp = j & ~1;
    __nv_bfloat16* obase = P.out + ((size_t)(U.row0 + (int64_t)cc * C) * H + h) * D + jp;
#pragma unroll
    for (int m = 0; m < 16; ++m) {
      const float send = odd ? v[2 * m] : v[2 * m + 1];
      const float recv = __shfl_xor_sync(0xffffffffu, send, 1);
      const int r = 2 * m + (odd ? 1 : 0);
      const float lo = odd ? recv : v[2 * m];      // column jp
      const float hi = odd ? v[2 * m + 1] : recv;  // column jp + 1
      if (r < n)
        *reinterpret_cast<__nv_bfloat162*>(obase + (size_t)r * H * D) =
            __floats2bfloat162_rn(P.scale * lo, P.scale * hi);
    }
  };

  // the loop starts at c = -1: that pass only prepares chunk 0's operands
  if (nchunks > 0 && tid < C && tid < U.len) beta_next = P.beta[(size_t)(U.row0 + tid) * H + h];
  for (int c = -1; c < nchunks && !*abort_flag; ++c) {
    const bool has_next = c + 1 < nchunks;
    if (c >= 0) {

    // ===== A: Gram GEMM (M64 N32 K128) of chunk c; warps 4-7 export O of chunk c-1
    if (tid == 0) {
      fence_after_sync();
#pragma unroll
      for (int ks = 0; ks < 8; ++ks) {
        const uint32_t kb = ks >> 2, kk = ks & 3;
        const uint64_t a = sw128_desc(sb + SM_KQL + kb * (64 * 128) + kk * 32, 16, 1024);
        const uint64_t b = sw128_desc(sb + SM_KB + kb * (32 * 128) + kk * 32, 16, 1024);
        mma_ss(tbase + G_COL, a, b, id_gram, 0, ks > 0);
      }
      mma_commit(bar_mma);
    }
    if (c > 0 && U.out_on && warp >= 4) export_o(c - 1);
    mbar_wait_bounded(bar_mma, ph_mma, abort_flag, P.sb, 2);
    ph_mma ^= 1;
    fence_after_sync();
    if (tid == 0 && !U.vzero && !*abort_flag) issue_v(c);  // the Gram operands are dead now

    // ===== B: A_kk (transposed, x beta) and A_qk from the Gram accumulator
    if (warp < 4) {
      float v[32];
      tmem_ld32(tbase + lane_base + G_COL, v);
      wait_ld();
      if (lane < 16) {
        const int r = 16 * (warp & 1) + lane;
        if (warp < 2) {
          const float br = betas[r];
          float* akkt = reinterpret_cast<float*>(sm + SM_AKKT);
#pragma unroll
          for (int s2 = 0; s2 < 32; ++s2) akkt[s2 * 32 + r] = s2 < r ? br * v[s2] : 0.f;
        } else {
#pragma unroll
          for (int s4 = 0; s4 < 8; ++s4) {
            float4 w4;
            w4.x = (4 * s4 + 0 <= r) ? v[4 * s4 + 0] : 0.f;
            w4.y = (4 * s4 + 1 <= r) ? v[4 * s4 + 1] : 0.f;
            w4.z = (4 * s4 + 2 <= r) ? v[4 * s4 + 2] : 0.f;
            w4.w = (4 * s4 + 3 <= r) ? v[4 * s4 + 3] : 0.f;
            *reinterpret_cast<float4*>(sm + SM_AQK + r * 128 + ((s4 ^ (r & 7)) << 4)) = w4;
          }
        }
      }
    }
    fence_proxy_async();
    fence_before_sync();
    __syncthreads();
    if (*abort_flag) break;

    // ===== C: T = (I + A_kk)^-1 Diag(beta), blocked 2 x 2 over 16-row blocks
    if (warp < 4) {
      const float* akkt = reinterpret_cast<const float*>(sm + SM_AKKT);
      float* xs = reinterpret_cast<float*>(sm + SM_XS);
      auto tt_store = [&](int r, int col, float val) {  // bf16 and fp32 copies of T[r][col]
        *reinterpret_cast<__nv_bfloat16*>(
            sm + SM_TT + r * 128 + ((((uint32_t)(col * 2) >> 4) ^ (uint32_t)(r & 7)) << 4) +
            ((col * 2) & 15)) = __float2bfloat16_rn(val);
        *reinterpret_cast<float*>(
            sm + SM_TF + r * 128 + ((((uint32_t)(col * 4) >> 4) ^ (uint32_t)(r & 7)) << 4) +
            ((col * 4) & 15)) = val;
      };
      if (warp == 0) {  // diagonal blocks: lane = (block b, column cb)
        const int b = lane >> 4, cb = lane & 15, o = 16 * b;
        float x[16];
#pragma unroll
        for (int r = 0; r < 16; ++r) x[r] = (r == cb) ? 1.f : 0.f;
#pragma unroll
        for (int s2 = 0; s2 < 15; ++s2) {
          const float xv = x[s2];
          const float* col = akkt + (o + s2) * 32 + o;  // A[o + r][o + s2], r = 0..15
#pragma unroll
          for (int r4 = (s2 + 1) / 4; r4 < 4; ++r4) {
            const float4 a4 = reinterpret_cast<const float4*>(col)[r4];
            if (4 * r4 + 0 > s2) x[4 * r4 + 0] = fmaf(-a4.x, xv, x[4 * r4 + 0]);
            if (4 * r4 + 1 > s2) x[4 * r4 + 1] = fmaf(-a4.y, xv, x[4 * r4 + 1]);
            if (4 * r4 + 2 > s2) x[4 * r4 + 2] = fmaf(-a4.z, xv, x[4 * r4 + 2]);
            if (4 * r4 + 3 > s2) x[4 * r4 + 3] = fmaf(-a4.w, xv, x[4 * r4 + 3]);
          }
        }
        const float bc = betas[o + cb];
#pragma unroll
        for (int r = 0; r < 16; ++r) {
          xs[(o + r) * 32 + o + cb] = x[r];
          tt_store(o + r, o + cb, x[r] * bc);
          if (b == 0) tt_store(r, 16 + cb, 0.f);  // upper-right block of T is zero
        }
      }
      asm volatile("bar.sync 1, 128;" ::: "memory");
      // Y = A10 X00 (rows 16..31 x columns 0..15), into the lower-left block of xs
      const int cl = tid & 15, rp = tid >> 4;  // tid < 128 here
#pragma unroll
      for (int h2 = 0; h2 < 2; ++h2) {
        const int r = 2 * rp + h2;
        float y = 0.f;
#pragma unroll
        for (int s2 = 0; s2 < 16; ++s2) y = fmaf(akkt[s2 * 32 + 16 + r], xs[s2 * 32 + cl], y);
        xs[(16 + r) * 32 + cl] = y;
      }
      asm volatile("bar.sync 1, 128;" ::: "memory");
      // X10 = -X11 Y;  T[16 + r][c] = X10[r][c] beta_c
      const float bcl = betas[cl];
#pragma unroll
      for (int h2 = 0; h2 < 2; ++h2) {
        const int r = 2 * rp + h2;
        float x10 = 0.f;
#pragma unroll
        for (int t2 = 0; t2 < 16; ++t2)
          x10 = fmaf(xs[(16 + r) * 32 + 16 + t2], xs[(16 + t2) * 32 + cl], x10);
        tt_store(16 + r, cl, -x10 * bcl);
      }
    }
    fence_proxy_async();
    __syncthreads();
    if (*abort_flag) break;

    // ===== D: U~^T = V^T T^T (bf16) and [O^T | P^T] = S^T [Qg ; Ka]^T (tf32, A = S^T
    //          in TMEM); meanwhile part 1 of the next chunk's prep
    if (tid == 0) {
      if (!U.vzero) {
        mbar_wait_bounded(bar_v, ph_v, abort_flag, P.sb, 3);
        ph_v ^= 1;
        pend_v = false;
      }
      fence_after_sync();
      if (!U.vzero) {
#pragma unroll
        for (int ks = 0; ks < 2; ++ks)
          mma_ss(tbase + U_COL, sw128_desc(sb + SM_V + ks * 2048, 4096, 1024),
                 sw128_desc(sb + SM_TT + ks * 32, 16, 1024), id_tv, 0, ks > 0);
      }
#pragma unroll
      for (int ks = 0; ks < 16; ++ks)
        mma_ts_tf32(tbase + O_COL, tbase + S_COL + 8 * ks,
                    sw128_desc(sb + SM_QK + (ks >> 2) * 8192 + (ks & 3) * 32, 16, 1024), id_op,
                    ks > 0);
      mma_commit(bar_mma);
    }
    }  // c >= 0

    if (has_next) {  // prep, part 1: tiles, beta, cumulative sums of g (log2 units)
      const int cc = c + 1;
      const int n = chunk_rows(cc);
      if (tid < C) {
        betas[tid] = beta_next;
        const int64_t t1 = (int64_t)(cc + 1) * C + tid;
        beta_next = (t1 < U.len) ? P.beta[(size_t)(U.row0 + t1) * H + h] : 0.f;
      }
      mbar_wait_bounded(bar_in, ph_in, abort_flag, P.sb, 1);
      ph_in ^= 1;
      if (tid == 0) pend_in = false;
      float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int rr = 0; rr < 4; ++rr) {
        const int r = 4 * ro + rr;
        float4 gv = *reinterpret_cast<const float4*>(sm + SM_G + (r * D + c0) * 4);
        if (P.A_log) {  // fused gate: tile holds z; g log2e = g_min log2e sigmoid(e^A z)
          gv.x = gmin2 * rcp_approx(1.f + ex2_approx(-a2 * gv.x));
          gv.y = gmin2 * rcp_approx(1.f + ex2_approx(-a2 * gv.y));
          gv.z = gmin2 * rcp_approx(1.f + ex2_approx(-a2 * gv.z));
          gv.w = gmin2 * rcp_approx(1.f + ex2_approx(-a2 * gv.w));
        } else {
          gv.x *= kLog2e;
          gv.y *= kLog2e;
          gv.z *= kLog2e;
          gv.w *= kLog2e;
        }
        if (r >= n) {  // tail rows act as g = 0, k = q = 0
          gv = make_float4(0.f, 0.f, 0.f, 0.f);
          *reinterpret_cast<uint2*>(sm + SM_K + (r * D + c0) * 2) = make_uint2(0u, 0u);
          *reinterpret_cast<uint2*>(sm + SM_Q + (r * D + c0) * 2) = make_uint2(0u, 0u);
        }
        acc.x += gv.x;
        acc.y += gv.y;
        acc.z += gv.z;
        acc.w += gv.w;
        G4[rr] = acc;
      }
      // 4-row group total, over the g values of (row 4ro, channels c0..c0+3) that
      // only this thread reads
      *reinterpret_cast<float4*>(sm + SM_G + (4 * ro * D + c0) * 4) = acc;
    }
    __syncthreads();
    if (c >= 0) {
    mbar_wait_bounded(bar_mma, ph_mma, abort_flag, P.sb, 5);
    ph_mma ^= 1;
    fence_after_sync();

    // ===== G: U^T -= P^T T^T (tf32, A = P^T in TMEM, onto U~^T), issued once P is
    //          complete; meanwhile decay the state, S^T[j][i] *= e^{Gamma_C, i}
    if (tid == 0) {
#pragma unroll
      for (int ks = 0; ks < 4; ++ks)
        mma_ts_tf32(tbase + U_COL, tbase + P_COL + 8 * ks,
                    sw128_desc(sb + SM_TF + ks * 32, 16, 1024), id_u, (ks > 0) || !U.vzero);
      mma_commit(bar_u);
    }
    {
#pragma unroll
      for (int cc = 0; cc < 2; ++cc) {
        const uint32_t col = S_COL + 64 * half + 32 * cc;
        const float4* g4 = reinterpret_cast<const float4*>(gamc + 64 * half + 32 * cc);
        float v[32];
        tmem_ld32(tbase + lane_base + col, v);
        wait_ld();
#pragma unroll
        for (int k4 = 0; k4 < 8; ++k4) {
          const float4 gg = g4[k4];
          v[4 * k4 + 0] *= gg.x;
          v[4 * k4 + 1] *= gg.y;
          v[4 * k4 + 2] *= gg.z;
          v[4 * k4 + 3] *= gg.w;
        }
        tmem_st32(tbase + lane_base + col, v);
      }
      wait_st();
    }
    fence_before_sync();
    __syncthreads();
    if (*abort_flag) break;

    // ===== H: [S^T | O^T] += U^T [Kc ; A_qk^T] (tf32, U^T from TMEM, one N = 160 MMA
    //          per k-step); meanwhile part 2 of the next chunk's prep
    // U is also the last reader of T in the Gram operand region, which part 2
    // of the prep overwrites: everyone waits for it
    mbar_wait_bounded(bar_u, ph_u, abort_flag, P.sb, 9);
    ph_u ^= 1;
    if (tid == 0) {
      fence_after_sync();
#pragma unroll
      for (int ks = 0; ks < 4; ++ks)
        mma_ts_tf32(tbase + S_COL, tbase + U_COL + 8 * ks,
                    sw128_desc(sb + SM_KC + ks * 32, 16, 1024), id_so, 1);
      mma_commit(bar_mma);
    }
    }  // c >= 0
    if (has_next) {  // prep, part 2: rescaled operands (Kc kept in registers)
      float4 off = make_float4(0.f, 0.f, 0.f, 0.f), g15 = off, g31 = off;
#pragma unroll
      for (int o8 = 0; o8 < 8; ++o8) {
        const float4 t = *reinterpret_cast<const float4*>(sm + SM_G + (4 * o8 * D + c0) * 4);
        if (o8 < ro) { off.x += t.x; off.y += t.y; off.z += t.z; off.w += t.w; }
        if (o8 < 4) { g15.x += t.x; g15.y += t.y; g15.z += t.z; g15.w += t.w; }
        g31.x += t.x; g31.y += t.y; g31.z += t.z; g31.w += t.w;
      }
      const float4 e15 = make_float4(ex2_approx(g15.x), ex2_approx(g15.y), ex2_approx(g15.z),
                                     ex2_approx(g15.w));
      const float4 e3115 = make_float4(ex2_approx(g31.x - g15.x), ex2_approx(g31.y - g15.y),
                                       ex2_approx(g31.z - g15.z), ex2_approx(g31.w - g15.w));
      if (ro == 7) {
        *reinterpret_cast<float4*>(gamc + c0) = make_float4(
            ex2_approx(g31.x), ex2_approx(g31.y), ex2_approx(g31.z), ex2_approx(g31.w));
      }
      // G4[rr] - g15 + off: exponent of e^{Gamma_r - Gamma_15} in log2 units
      const float4 sh = make_float4(off.x - g15.x, off.y - g15.y, off.z - g15.z, off.w - g15.w);
#pragma unroll
      for (int rr = 0; rr < 4; ++rr) {
        const int r = 4 * ro + rr;
        float ex[4], ix[4];
        ex[0] = ex2_approx(G4[rr].x + sh.x);
        ex[1] = ex2_approx(G4[rr].y + sh.y);
        ex[2] = ex2_approx(G4[rr].z + sh.z);
        ex[3] = ex2_approx(G4[rr].w + sh.w);
#pragma unroll
        for (int k4 = 0; k4 < 4; ++k4) ix[k4] = rcp_approx(ex[k4]);
        const uint2 kw = *reinterpret_cast<const uint2*>(sm + SM_K + (r * D + c0) * 2);
        const uint2 qw = *reinterpret_cast<const uint2*>(sm + SM_Q + (r * D + c0) * 2);
        const float kv[4] = {__uint_as_float(kw.x << 16), __uint_as_float(kw.x & 0xffff0000u),
                             __uint_as_float(kw.y << 16), __uint_as_float(kw.y & 0xffff0000u)};
        const float qv[4] = {__uint_as_float(qw.x << 16), __uint_as_float(qw.x & 0xffff0000u),
                             __uint_as_float(qw.y << 16), __uint_as_float(qw.y & 0xffff0000u)};
        float kl[4], ql[4], kb[4];
#pragma unroll
        for (int k4 = 0; k4 < 4; ++k4) {
          kl[k4] = kv[k4] * ex[k4];
          ql[k4] = qv[k4] * ex[k4];
          kb[k4] = kv[k4] * ix[k4];
        }
        const uint32_t rb = rr * 128;
        const uint32_t sw = (uint32_t)((4 * ro + rr) & 7);
        const uint32_t s16 = (ck16 ^ sw) << 4, s32 = (ck32 ^ sw) << 4;
        auto pack = [](float lo, float hi) {
          const __nv_bfloat162 b2 = __floats2bfloat162_rn(lo, hi);
          return *reinterpret_cast<const uint32_t*>(&b2);
        };
        *reinterpret_cast<uint2*>(sm + SM_KQL + o_kql + rb + s16) =
            make_uint2(pack(kl[0], kl[1]), pack(kl[2], kl[3]));
        *reinterpret_cast<uint2*>(sm + SM_KQL + o_kql + 4096 + rb + s16) =
            make_uint2(pack(ql[0], ql[1]), pack(ql[2], ql[3]));
        *reinterpret_cast<uint2*>(sm + SM_KB + o_kb + rb + s16) =
            make_uint2(pack(kb[0], kb[1]), pack(kb[2], kb[3]));
        *reinterpret_cast<float4*>(sm + SM_QK + o_qk + rb + s32) =
            make_float4(ql[0] * e15.x, ql[1] * e15.y, ql[2] * e15.z, ql[3] * e15.w);
        *reinterpret_cast<float4*>(sm + SM_QK + o_qk + 4096 + rb + s32) =
            make_float4(kl[0] * e15.x, kl[1] * e15.y, kl[2] * e15.z, kl[3] * e15.w);
        kc[0][rr] = kb[0] * e3115.x;
        kc[1][rr] = kb[1] * e3115.y;
        kc[2][rr] = kb[2] * e3115.z;
        kc[3][rr] = kb[3] * e3115.w;
      }
    }
    if (c >= 0) {
      mbar_wait_bounded(bar_mma, ph_mma, abort_flag, P.sb, 6);
      ph_mma ^= 1;
      fence_after_sync();
    }
    if (has_next) {  // Kc^T rows c0..c0+3: this thread's 4 rows are one 16-byte chunk of each
#pragma unroll
      for (int k4 = 0; k4 < 4; ++k4) {
        const int row = c0 + k4;
        *reinterpret_cast<float4*>(sm + SM_KC + row * 128 + ((ro ^ (row & 7)) << 4)) =
            make_float4(kc[k4][0], kc[k4][1], kc[k4][2], kc[k4][3]);
      }
    }
    fence_proxy_async();
    fence_before_sync();
    __syncthreads();
    if (tid == 0 && c + 2 < nchunks) {
      fence_proxy_async();
      issue_qkg(c + 2);
    }
    if (tid == 0 && c + 1 < nchunks && !U.vzero) prefetch_v(c + 1);
  }
  __syncthreads();
  if (nchunks > 0 && U.out_on && warp >= 4 && !*abort_flag) export_o(nchunks - 1);
  fence_before_sync();
  __syncthreads();

  // ---- final state (S^T lane j, column i -> final[i][j])
  if (U.final_state && !*abort_flag) {
    const int j = 32 * (warp & 3) + lane;
#pragma unroll
    for (int cc = 0; cc < 2; ++cc) {
      const int i0 = 64 * half + 32 * cc;
      float v[32];
      tmem_ld32(tbase + lane_base + S_COL + i0, v);
      wait_ld();
#pragma unroll
      for (int k = 0; k < 32; ++k) U.final_state[(size_t)(i0 + k) * D + j] = v[k];
    }
  }
  fence_before_sync();
  __syncthreads();
  if (tid == 0 && *abort_flag) {
    // let every MMA and TMA load still in flight land before the CTA's shared
    // memory and TMEM are released
    mma_commit(bar_drain);
    mbar_wait_drain(bar_drain, 0);
    if (pend_in) mbar_wait_drain(bar_in, ph_in);
    if (pend_v) mbar_wait_drain(bar_v, ph_v);
  }
  __syncthreads();
  if (warp == 0) tmem_dealloc(tbase, TMEM_COLS);
}

// S_in[g+1] = S~_g + M_g S_in[g] for every unit, one 32-column slice per CTA.
__global__ void __launch_bounds__(256) segment_combine_kernel(const float* __restrict__ init,
                                                              float* __restrict__ ws, int U,
                                                              int G) {
  __shared__ float X[D][33];
  const size_t DD = (size_t)D * D;
  const int un = blockIdx.x >> 2, j0 = (blockIdx.x & 3) * 32;
  const int tid = threadIdx.x, jj = tid & 31, i0 = tid >> 5;
  for (int k = 0; k < 16; ++k) {
    const int i = i0 + 8 * k;
    X[i][jj] = init ? init[un * DD + (size_t)i * D + j0 + jj] : 0.f;
  }
  __syncthreads();
  const float* pairs = ws + (size_t)un * (G - 1) * 2 * DD;
  float* s_in = ws + ((size_t)U * (G - 1) * 2 + (size_t)un * (G - 1)) * DD;
  for (int g = 0; g < G - 1; ++g) {
    const float* St = pairs + (size_t)(2 * g) * DD;
    const float* M = pairs + (size_t)(2 * g + 1) * DD;
    float acc[16];
#pragma unroll
    for (int k = 0; k < 16; ++k) acc[k] = St[(size_t)(i0 + 8 * k) * D + j0 + jj];
    for (int ip = 0; ip < D; ++ip) {
      const float x = X[ip][jj];
#pragma unroll
      for (int k = 0; k < 16; ++k) acc[k] = fmaf(__ldg(M + (size_t)(i0 + 8 * k) * D + ip), x, acc[k]);
    }
    __syncthreads();
#pragma unroll
    for (int k = 0; k < 16; ++k) {
      X[i0 + 8 * k][jj] = acc[k];
      s_in[(size_t)g * DD + (size_t)(i0 + 8 * k) * D + j0 + jj] = acc[k];
    }
    __syncthreads();
  }
}

// ------------------------------------------------------------------- host
PFN_cuTensorMapEncodeTiled_v12000 get_encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

bool encode_3d(CUtensorMap* m, CUtensorMapDataType dt, int esz, const void* base, int H,
               int64_t R, uint32_t box0, CUtensorMapSwizzle sw) {
  auto fn = get_encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)H, (cuuint64_t)R};
  cuuint64_t strides[2] = {(cuuint64_t)D * esz, (cuuint64_t)H * D * esz};
  cuuint32_t box[3] = {box0, 1, (cuuint32_t)C};
  cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, dt, 3, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Segment split for long dense sequences with too few (sequence, head)
// units to occupy the GPU: returns G >= 2 and the segment length, or G = 1.
void plan_split(int B, int T, int H, int num_sms, int* G_out, int* seg_out) {
  const int U = B * H;
  *G_out = 1;
  *seg_out = T;
  if (2 * U >= num_sms || T < 4 * 1024) return;
  int G = (2 * num_sms + U - 1) / U;
  const int max_g = T / 1024;
  if (G > max_g) G = max_g;
  if (G < 2) return;
  int seg = (T + G - 1) / G;
  seg = (seg + C - 1) / C * C;
  G = (T + seg - 1) / seg;
  if (G < 2) return;
  *G_out = G;
  *seg_out = seg;
}

}  // namespace

size_t tc_workspace_bytes(int B, int T, int H, int num_seqs, int num_sms) {
  if (num_seqs > 0) return 0;
  int G, seg;
  plan_split(B, T, H, num_sms, &G, &seg);
  if (G < 2) return 0;
  return (size_t)B * H * (G - 1) * 3 * D * D * sizeof(float);
}

cudaError_t launch_chunk_tc(const ChunkArgs& a, void* ws_tail, size_t ws_tail_bytes,
                            cudaStream_t stream) {
  if (a.num_units == 0) return cudaSuccess;
  static bool attr_done = false;
  if (!attr_done) {
    cudaError_t e = cudaFuncSetAttribute(chunk_tc_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_ALLOC);
    if (e != cudaSuccess) return e;
    attr_done = true;
  }
  TcParams P;
  memset(&P, 0, sizeof(P));
  const int64_t R = (int64_t)a.map.B * a.map.T;
  const int H = a.map.H;
  if (!encode_3d(&P.tm_q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, a.q, H, R, 128,
                 CU_TENSOR_MAP_SWIZZLE_NONE) ||
      !encode_3d(&P.tm_k, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, a.k, H, R, 128,
                 CU_TENSOR_MAP_SWIZZLE_NONE) ||
      !encode_3d(&P.tm_v, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, a.v, H, R, 64,
                 CU_TENSOR_MAP_SWIZZLE_128B) ||
      !encode_3d(&P.tm_g, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, a.g, H, R, 128,
                 CU_TENSOR_MAP_SWIZZLE_NONE))
    return cudaErrorInvalidValue;
  P.A_log = a.gated ? a.A_log : nullptr;
  P.g_min = a.g_min;
  P.beta = a.beta;
  P.out = static_cast<__nv_bfloat16*>(a.out);
  P.init_state = a.init_state;
  P.final_state = a.final_state;
  P.cu_seqlens = a.map.cu_seqlens;
  P.order = a.map.order;
  P.sb = a.sb;
  P.B = a.map.B;
  P.T = a.map.T;
  P.H = H;
  P.scale = a.scale;
  P.mode = 0;
  P.G = 1;
  P.seg_len = a.map.T;

  int G = 1, seg = a.map.T;
  if (a.map.cu_seqlens == nullptr) plan_split(a.map.B, a.map.T, H, device_sm_count(), &G, &seg);
  if (G < 2) {
    chunk_tc_kernel<<<a.num_units, NT, SMEM_ALLOC, stream>>>(P);
    return cudaGetLastError();
  }
  const int U = a.map.B * H;
  const size_t need = (size_t)U * (G - 1) * 3 * D * D * sizeof(float);
  if (ws_tail_bytes < need) return cudaErrorInvalidValue;
  P.seg_ws = static_cast<float*>(ws_tail);
  P.G = G;
  P.seg_len = seg;
  P.mode = 1;
  chunk_tc_kernel<<<U * (G - 1) * 2, NT, SMEM_ALLOC, stream>>>(P);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  segment_combine_kernel<<<U * 4, 256, 0, stream>>>(a.init_state, P.seg_ws, U, G);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  P.mode = 2;
  chunk_tc_kernel<<<U * G, NT, SMEM_ALLOC, stream>>>(P);
  return cudaGetLastError();
}

}  // namespace kda
