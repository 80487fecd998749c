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
// B200 mapping.  One CTA (14 warps) owns one (sequence, head) for its whole
// length, one CTA per SM.  The fp32 state never leaves the SM: it lives in
// TMEM as S^T (lane = value channel, column = key channel), next to a bf16
// copy of it that is the A operand of the [O | P] GEMM (the state is cast to
// bf16 for that product, as is usual for chunked delta-rule kernels; it is
// accumulated in fp32 throughout).  tcgen05.mma costs
// a roughly fixed number of cycles per instruction up to N = 128-256
// (measured: ~90-125 with A in TMEM, ~190-210 with A in shared memory), so products
// that share an A operand are fused into one wide MMA:
//   [O^T | P^T] += S^T [q e^G ; k e^G]^T  onto [0 | -V^T]  (bf16, N = 64, 8 k-steps)
//   U^T          = -P^T T^T,  i.e. U = T (V - k e^G S)       (tf32, N = 32)
//   [S^T | O^T] += U^T [Kc ; A_qk]^T  after the decay        (tf32, N = 160, 4 k-steps)
// The Gram ([k;q] e^{G-G15} against k e^{G15-G}, 64 x 32 x 128) is small and
// off the state chain: the solve warps compute it with warp-level bf16 MMAs
// (mma.sync, fp32 accumulation) straight from the swizzled operand tiles, so
// it costs the tcgen05 pipe nothing and its result is already in registers.
//
// The warps are specialised and hand work over through mbarriers, so the
// key-side work of later chunks (which does not depend on the state)
// overlaps the state-side chain of the current one:
//   warps 0-3   prep: gate, in-chunk cumulative decay, rescaled operands
//   warps 4-7   solve: Gram (warp MMA), T = (I + A_kk)^-1 Diag(beta)
//   warps 8-11  state: once [S | O] of a chunk is done, the bf16 copy of S and
//               the seed [0 | -V^T] of the next chunk's [O | P] (the critical
//               path), then export of O and the next chunk's decay of S
//   warp  12    one lane issues the state-side MMAs ([O | P], U, [S | O]) in
//               chunk order, each after a blocking wait on what it needs
//   warp  13    one lane issues the TMA loads
// Per-chunk operands are double-buffered by chunk parity (v four-deep); the
// Gram operand region of a chunk is reused for T and the inverse's scratch
// once the Gram is done.  Every wait is bounded (kda_sync.cuh).
//
// TMEM columns: S^T [0,128) | O^T [128,160) | P^T [160,192) | U^T [192,224)
//               | bf16 S^T [384,448)
#include <cuda.h>
#include <cudaTypedefs.h>

#include <atomic>

#include "kda_internal.cuh"
#include "kda_sync.cuh"
#include "kda_tc_ptx.cuh"

namespace kda {
namespace {

using namespace tc;

constexpr int C = 32;    // tokens per chunk
constexpr int D = 128;   // dk = dv
constexpr int PREP_W0 = 0, SOLVE_W0 = 4, STATE_W0 = 8, ISSUE_W = 12;  // warp 13: TMA issue
constexpr int NT = 32 * 14;

// [O | P] and its O are double-buffered by chunk parity b, each buffer next to
// S on the side the fused GEMMs need: b = 0 as [P | O] left of S and [O | S];
// b = 1 as [S | O] and [O | P] right of S.  A chunk's O is then read out, and
// the next-but-one chunk's [O | P] seeded, while the chain goes on.
constexpr uint32_t S_COL = 64, U_COL = 256;
constexpr uint32_t SB_COL = 288;  // bf16 S^T: column c holds key channels 2c, 2c + 1
__device__ __forceinline__ uint32_t o_col(int b) { return b ? 192u : 32u; }
__device__ __forceinline__ uint32_t p_col(int b) { return b ? 224u : 0u; }
__device__ __forceinline__ uint32_t op_col(int b) { return b ? 192u : 0u; }   // [O|P] / [P|O]
__device__ __forceinline__ uint32_t so_col(int b) { return b ? 64u : 32u; }   // [S|O] / [O|S]
// operand rows of those GEMMs: q e^G / k e^G rows of [O | P], Kc^T / A_qk rows of [S | O]
__device__ __forceinline__ uint32_t q_row(int b) { return b ? 0u : 32u; }
__device__ __forceinline__ uint32_t k_row(int b) { return b ? 32u : 0u; }
__device__ __forceinline__ uint32_t kc_row(int b) { return b ? 0u : 32u; }
__device__ __forceinline__ uint32_t aqk_row(int b) { return b ? 128u : 0u; }
constexpr uint32_t TMEM_COLS = 512;

// shared memory map (byte offsets from a 1024-aligned base)
constexpr uint32_t STAGE = 32768;   // input stage s at s * STAGE, two stages
constexpr uint32_t OFF_Q = 0;       //   q bf16 [32][128] (TMA, no swizzle)
constexpr uint32_t OFF_K = 8192;    //   k bf16 [32][128]
constexpr uint32_t OFF_G = 16384;   //   g or z fp32 [32][128]; in-chunk cumsum (log2) in prep
constexpr uint32_t SM_KEY = 65536;  // key buffer b at SM_KEY + b * KEYB
constexpr uint32_t KEYB = 24576;
constexpr uint32_t K_KQL = 0;       //   Gram A [k;q] e^{G-G15} bf16 64 x 128, per 64-channel
                                    //   block 64 rows x 128 B (rows 0-31 k, 32-63 q)
constexpr uint32_t K_KB = 16384;    //   Gram B k e^{G15-G} bf16 32 x 128, per block 32 x 128 B
                                    //   and once the Gram is done:
constexpr uint32_t K_TF = 4096;     //   T fp32 [r][s] (tf32 B of U = -P^T T^T)
constexpr uint32_t K_AKKT = 16384;  //   A_kk^T fp32 [s][r] (inverse input)
constexpr uint32_t K_XS = 20480;    //   inverse blocks, fp32 32 x 32
constexpr uint32_t SM_HB = SM_KEY + 2 * KEYB;  // hand-off buffer b at SM_HB + b * HBB
constexpr uint32_t HBB = 39936;
constexpr uint32_t H_QK = 0;        //   [q e^G ; k e^G] bf16, per 64-channel block 64 rows x 128 B
constexpr uint32_t H_KC = 16384;    //   B of [S | O], tf32 K-major without swizzle: rows n < 128
                                    //   key channel i of k e^{GC-G}, n >= 128 row r = n - 128 of
                                    //   A_qk; K = token s.  Core matrices of 8 rows x 16 bytes;
                                    //   8-row groups KC_SBO apart (16 bytes of padding, so the
                                    //   prep warps' 16-byte stores of 8 consecutive row groups
                                    //   fall in distinct banks), 4-token groups KC_LBO apart.
constexpr uint32_t KC_SBO = 144, KC_LBO = 20 * KC_SBO;
static_assert(H_KC + 8 * KC_LBO <= HBB, "[S | O] operand tile fits the hand-off buffer");
__device__ __forceinline__ uint32_t kc_off(uint32_t n, uint32_t s) {
  return (s >> 2) * KC_LBO + (n >> 3) * KC_SBO + (n & 7) * 16 + (s & 3) * 4;
}
constexpr uint32_t SM_V = SM_HB + 2 * HBB;  // v tile of chunk c at SM_V + (c % 4) * 8192:
constexpr int NVBUF = 4;                    //   bf16, 2 x [32 rows x 128 B] swizzled (TMA)
constexpr uint32_t SM_MISC = SM_V + NVBUF * 8192;
constexpr uint32_t SM_GAMC = SM_MISC;          // e^{Gamma_C} fp32 [2][128]
constexpr uint32_t SM_BETA = SM_MISC + 1024;   // beta        fp32 [2][32]
constexpr uint32_t SM_BAR = SM_MISC + 1280;    // mbarriers
constexpr uint32_t SM_TMEM = SM_MISC + 1536;   // TMEM base address
constexpr uint32_t SM_ABORT = SM_MISC + 1540;  // abort flag
constexpr uint32_t SMEM_BYTES = SM_MISC + 2048;
constexpr uint32_t SMEM_ALLOC = SMEM_BYTES + 1024;  // room to align the base to 1024
static_assert(SMEM_ALLOC <= 227 * 1024, "one CTA per SM");

// mbarriers ([2] = one per chunk parity, [4] = one per v buffer)
enum : int {
  B_IN_FULL = 0,    // [2] TMA q, k, g landed                      (tx)
  B_IN_EMPTY = 2,   // [2] prep done with the input stage          (4 prep warps)
  B_OPER = 4,       // [2] chunk operands written                  (4 prep warps)
  B_T = 6,          // [2] T and A_qk written                      (4 solve warps)
  B_UO = 8,         //     [O | P] GEMM done                       (commit)
  B_U = 9,          //     U GEMM done                             (commit)
  B_DECAY = 10,     //     state decayed for the chunk (with B_OREADY) (4 state warps)
  B_SO = 11,        // [2] [S | O] GEMM done                       (commit)
  B_OREADY = 13,    //     O read out, [O | P] seeded, bf16 S written (4 state warps)
  B_DRAIN = 14,     //     abort path: every MMA the state issuer issued done (commit)
  B_V = 15,         // [4] TMA v landed                            (tx)
  B_VEMPTY = 19,    // [4] v buffer read                           (4 state warps)
  NBARS = 23
};
static_assert(NBARS * 8 <= SM_TMEM - SM_BAR, "mbarrier space");

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
  long long wait_limit_ns;  // bound of every mbarrier wait (lowered only by diagnostics)
};

struct Unit {
  int64_t row0, len;
  int h;
  const float* init;
  bool init_identity, vzero, out_on;
  float* final_state;
};

// KDA_DEBUG_CHECKS builds: the rows [row0, row0 + len) lie in the batch
__device__ __forceinline__ bool unit_rows_ok(const TcParams& P, int64_t row0, int64_t len) {
  const int64_t rows = (int64_t)P.B * P.T;
  return in_bounds(P.sb, len, rows + 1, kSiteTcUnitRows) &&
         (len == 0 || (in_bounds(P.sb, row0, rows, kSiteTcUnitRows) &&
                       in_bounds(P.sb, row0 + len - 1, rows, kSiteTcUnitRows)));
}

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
    // one unit per CTA: the state slots are the grid's units
    if (!unit_rows_ok(P, u.row0, u.len) ||
        !in_bounds(P.sb, sidx, gridDim.x, kSiteTcStateSlot))
      return false;
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
    const int64_t slot = (int64_t)(un * (P.G - 1) + g) * 2 + kind;
    if (!unit_rows_ok(P, u.row0, u.len) ||
        !in_bounds(P.sb, slot, (int64_t)U * (P.G - 1) * 2, kSiteTcStateSlot))
      return false;
    u.final_state = P.seg_ws + (size_t)slot * DD;
    return true;
  }
  // mode 2: outputs of every segment from its true incoming state
  const int un = blockIdx.x / P.G, g = blockIdx.x % P.G;
  u.h = un % H;
  u.row0 = (int64_t)(un / H) * P.T + (int64_t)g * P.seg_len;
  const int64_t rem = (int64_t)P.T - (int64_t)g * P.seg_len;
  u.len = rem < P.seg_len ? rem : P.seg_len;
  if (!unit_rows_ok(P, u.row0, u.len)) return false;
  if (g == 0) {
    u.init = P.init_state ? P.init_state + (size_t)un * DD : nullptr;
  } else {
    const int64_t slot = (int64_t)U * (P.G - 1) * 2 + (int64_t)un * (P.G - 1) + (g - 1);
    if (!in_bounds(P.sb, slot, (int64_t)U * (P.G - 1) * 3, kSiteTcStateSlot)) return false;
    u.init = P.seg_ws + (size_t)slot * DD;
  }
  u.final_state = (g == P.G - 1 && P.final_state) ? P.final_state + (size_t)un * DD : nullptr;
  return true;
}

// The register file is split across the SM's four sub-partitions and a CTA's
// warps are dealt to them in turn, so with 14 warps two quarters hold four of
// them: 16384 / (4 * 32) = 128 registers per thread is the most that launches.
__global__ void __maxnreg__(128) chunk_tc_kernel(const __grid_constant__ TcParams P) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_s = smem_u32(smem_raw);
  uint8_t* sm = smem_raw + ((1024u - (raw_s & 1023u)) & 1023u);
  const uint32_t sb = smem_u32(sm);

  Unit U;
  if (!resolve_unit(P, U)) return;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + SM_BAR);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + SM_TMEM);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + SM_ABORT);
  const int H = P.H, h = U.h;
  const int nchunks = (int)((U.len + C - 1) / C);
  // every mbarrier wait of the pipeline: bounded, abort-aware, `where` names it
  auto wait = [&](uint64_t* bar, uint32_t parity, int32_t where) {
    return mbar_wait_bounded(bar, parity, abort_flag, P.sb, where, P.wait_limit_ns);
  };
  auto chunk_rows = [&](int cc) -> int {
    const int64_t rem = U.len - (int64_t)cc * C;
    return (int)(rem < C ? rem : C);
  };

  if (tid == 0) {
#pragma unroll
    for (int i = 0; i < NBARS; ++i) {
      const bool four = i == B_IN_EMPTY || i == B_IN_EMPTY + 1 || i == B_OPER ||
                        i == B_OPER + 1 || i == B_T || i == B_T + 1 || i == B_DECAY ||
                        i == B_OREADY || (i >= B_VEMPTY && i < B_VEMPTY + NVBUF);
      mbar_init(&bars[i], four ? 4u : 1u);
    }
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

  // ---- initial state -> TMEM (S^T: lane j, column i), by the state warps
  if (warp >= STATE_W0 && warp < ISSUE_W) {
    const int j = 32 * (warp & 3) + lane;
    float v[32];
#pragma unroll 1
    for (int cc = 0; cc < 4; ++cc) {
#pragma unroll
      for (int k = 0; k < 32; ++k) {
        const int i = 32 * cc + k;
        v[k] = U.init ? U.init[(size_t)i * D + j] : ((U.init_identity && i == j) ? 1.f : 0.f);
      }
      tmem_st32(tbase + lane_base + S_COL + 32 * cc, v);
    }
    wait_st();
  }
  fence_before_sync();
  __syncthreads();
  fence_after_sync();

  if (warp < SOLVE_W0) {
    // =============================================================== prep warps
    // thread: channels c0 .. c0+3, rows 8pw .. 8pw+7; fp32 pairs in packed
    // f32x2 arithmetic (two lanes of work per instruction)
    const int pw = warp - PREP_W0, c0 = 4 * lane;
    const uint32_t ck16 = ((c0 & 63) * 2) >> 4, lo16 = ((c0 & 63) * 2) & 15;  // bf16 tiles
    const uint32_t o_kql = (c0 >> 6) * 8192 + lo16;
    const uint32_t o_kb = (c0 >> 6) * 4096 + lo16;
    constexpr float kLog2e = 1.4426950408889634f;
    const float gmin2 = P.g_min * kLog2e;
    const float a2 = P.A_log ? expf(P.A_log[h]) * kLog2e : 0.f;
    const float2 na2 = make_float2(-a2, -a2), one2 = make_float2(1.f, 1.f);
    float beta_next = 0.f;
    if (pw == 0 && lane < U.len) beta_next = P.beta[(size_t)(U.row0 + lane) * H + h];
    auto pack = [](float lo_, float hi_) {
      const __nv_bfloat162 b2 = __floats2bfloat162_rn(lo_, hi_);
      return *reinterpret_cast<const uint32_t*>(&b2);
    };
    auto bf_lo = [](uint32_t w) { return __uint_as_float(w << 16); };
    auto bf_hi = [](uint32_t w) { return __uint_as_float(w & 0xffff0000u); };

    for (int c = 0; c < nchunks; ++c) {
      const int st = c & 1, b = c & 1;
      const int n = chunk_rows(c);
      uint8_t* in = sm + st * STAGE;
      uint8_t* kb_buf = sm + SM_KEY + b * KEYB;
      uint8_t* hb = sm + SM_HB + b * HBB;
      const float beta_cur = beta_next;
      wait(&bars[B_IN_FULL + st], (c >> 1) & 1, 1);
      __syncwarp();
      if (n < C) {  // tail rows act as k = q = 0 (and g = 0 below)
#pragma unroll 1
        for (int rr = 0; rr < 8; ++rr) {
          const int r = 8 * pw + rr;
          if (r >= n) {
            *reinterpret_cast<uint2*>(in + OFF_K + (r * D + c0) * 2) = make_uint2(0u, 0u);
            *reinterpret_cast<uint2*>(in + OFF_Q + (r * D + c0) * 2) = make_uint2(0u, 0u);
          }
        }
      }

      // ---- part 1: gate and cumulative log2-decay over rows 8pw .. 8pw+7, written
      //      back in place (only this thread touches these elements)
      {
        float2 acc01 = make_float2(0.f, 0.f), acc23 = acc01;
#pragma unroll
        for (int rr = 0; rr < 8; ++rr) {
          const int r = 8 * pw + rr;
          float4* gp = reinterpret_cast<float4*>(in + OFF_G + (r * D + c0) * 4);
          const float4 gv = *gp;
          const float2 g01 = make_float2(gv.x, gv.y), g23 = make_float2(gv.z, gv.w);
          if (P.A_log) {  // fused gate: tile holds z; g log2e = g_min log2e sigmoid(e^A z)
            const float gm = r < n ? gmin2 : 0.f;
            const float2 gm2 = make_float2(gm, gm);
            const float2 x01 = __fmul2_rn(g01, na2), x23 = __fmul2_rn(g23, na2);
            const float2 d01 = __fadd2_rn(make_float2(ex2_approx(x01.x), ex2_approx(x01.y)), one2);
            const float2 d23 = __fadd2_rn(make_float2(ex2_approx(x23.x), ex2_approx(x23.y)), one2);
            acc01 = __ffma2_rn(make_float2(rcp_approx(d01.x), rcp_approx(d01.y)), gm2, acc01);
            acc23 = __ffma2_rn(make_float2(rcp_approx(d23.x), rcp_approx(d23.y)), gm2, acc23);
          } else {
            const float lm = r < n ? kLog2e : 0.f;
            const float2 lm2 = make_float2(lm, lm);
            acc01 = __ffma2_rn(g01, lm2, acc01);
            acc23 = __ffma2_rn(g23, lm2, acc23);
          }
          *gp = make_float4(acc01.x, acc01.y, acc23.x, acc23.y);
        }
      }
      // every prep warp's partial sums are in; the same barrier agrees on an abort
      if (bar_red_or(1, 128, *abort_flag != 0)) break;

      // ---- part 2: rescaled operands; buffer b is free once chunk c - 2 is
      //      completely done (its [S | O] GEMM is the last reader)
      if (c >= 2) wait(&bars[B_SO + b], ((c - 2) >> 1) & 1, 2);
      __syncwarp();
      // beta of the next chunk: issued here, after this chunk's waits, so that no
      // out-of-line wait call has to hold the pending load
      if (pw == 0) {
        const int64_t t1 = (int64_t)(c + 1) * C + lane;
        beta_next = (t1 < U.len) ? __ldg(P.beta + (size_t)(U.row0 + t1) * H + h) : 0.f;
      }
      {
        float2 off01 = make_float2(0.f, 0.f), off23 = off01, g15_01 = off01, g15_23 = off01;
        float2 g31_01 = off01, g31_23 = off01;
#pragma unroll
        for (int o4 = 0; o4 < 4; ++o4) {  // group totals: the partial sums at rows 8 o4 + 7
          const float4 t =
              *reinterpret_cast<const float4*>(in + OFF_G + ((8 * o4 + 7) * D + c0) * 4);
          const float2 t01 = make_float2(t.x, t.y), t23 = make_float2(t.z, t.w);
          if (o4 < pw) { off01 = __fadd2_rn(off01, t01); off23 = __fadd2_rn(off23, t23); }
          if (o4 < 2) { g15_01 = __fadd2_rn(g15_01, t01); g15_23 = __fadd2_rn(g15_23, t23); }
          g31_01 = __fadd2_rn(g31_01, t01);
          g31_23 = __fadd2_rn(g31_23, t23);
        }
        const float2 e15_01 = make_float2(ex2_approx(g15_01.x), ex2_approx(g15_01.y));
        const float2 e15_23 = make_float2(ex2_approx(g15_23.x), ex2_approx(g15_23.y));
        const float2 d31_01 = __fadd2_rn(g31_01, make_float2(-g15_01.x, -g15_01.y));
        const float2 d31_23 = __fadd2_rn(g31_23, make_float2(-g15_23.x, -g15_23.y));
        const float2 e3115_01 = make_float2(ex2_approx(d31_01.x), ex2_approx(d31_01.y));
        const float2 e3115_23 = make_float2(ex2_approx(d31_23.x), ex2_approx(d31_23.y));
        if (pw == 0) {
          *reinterpret_cast<float4*>(sm + SM_GAMC + b * 512 + c0 * 4) = make_float4(
              ex2_approx(g31_01.x), ex2_approx(g31_01.y), ex2_approx(g31_23.x),
              ex2_approx(g31_23.y));
          reinterpret_cast<float*>(sm + SM_BETA + b * 128)[lane] = beta_cur;
        }
        // shift of this warp's rows: the earlier groups' totals, re-based at row 15
        const float2 sh01 = __fadd2_rn(off01, make_float2(-g15_01.x, -g15_01.y));
        const float2 sh23 = __fadd2_rn(off23, make_float2(-g15_23.x, -g15_23.y));
#pragma unroll 1
        for (int hf = 0; hf < 2; ++hf) {
          float kc[4][4];  // [channel][row] of rows 8pw + 4hf .. +3
#pragma unroll
          for (int r4 = 0; r4 < 4; ++r4) {
            const int r = 8 * pw + 4 * hf + r4;
            const float4 G = *reinterpret_cast<const float4*>(in + OFF_G + (r * D + c0) * 4);
            const float2 t01 = __fadd2_rn(make_float2(G.x, G.y), sh01);
            const float2 t23 = __fadd2_rn(make_float2(G.z, G.w), sh23);
            // e^{G_r - G_15} and its inverse (two independent exponentials)
            const float2 ex01 = make_float2(ex2_approx(t01.x), ex2_approx(t01.y));
            const float2 ex23 = make_float2(ex2_approx(t23.x), ex2_approx(t23.y));
            const float2 ix01 = make_float2(ex2_approx(-t01.x), ex2_approx(-t01.y));
            const float2 ix23 = make_float2(ex2_approx(-t23.x), ex2_approx(-t23.y));
            const uint2 kw = *reinterpret_cast<const uint2*>(in + OFF_K + (r * D + c0) * 2);
            const uint2 qw = *reinterpret_cast<const uint2*>(in + OFF_Q + (r * D + c0) * 2);
            const float2 k01 = make_float2(bf_lo(kw.x), bf_hi(kw.x));
            const float2 k23 = make_float2(bf_lo(kw.y), bf_hi(kw.y));
            const float2 q01 = make_float2(bf_lo(qw.x), bf_hi(qw.x));
            const float2 q23 = make_float2(bf_lo(qw.y), bf_hi(qw.y));
            const float2 kl01 = __fmul2_rn(k01, ex01), kl23 = __fmul2_rn(k23, ex23);
            const float2 ql01 = __fmul2_rn(q01, ex01), ql23 = __fmul2_rn(q23, ex23);
            const float2 kb01 = __fmul2_rn(k01, ix01), kb23 = __fmul2_rn(k23, ix23);
            const float2 qg01 = __fmul2_rn(ql01, e15_01), qg23 = __fmul2_rn(ql23, e15_23);
            const float2 kg01 = __fmul2_rn(kl01, e15_01), kg23 = __fmul2_rn(kl23, e15_23);
            const float2 kc01 = __fmul2_rn(kb01, e3115_01), kc23 = __fmul2_rn(kb23, e3115_23);
            kc[0][r4] = kc01.x;
            kc[1][r4] = kc01.y;
            kc[2][r4] = kc23.x;
            kc[3][r4] = kc23.y;
            const uint32_t sw = (uint32_t)(r & 7);
            const uint32_t s16 = (ck16 ^ sw) << 4;
            // Gram operands (rows 64 hh + r, 64 hh + 32 + r of A and 32 hh + r of B
            // for channel half hh = c0 / 64)
            *reinterpret_cast<uint2*>(kb_buf + K_KQL + o_kql + r * 128 + s16) =
                make_uint2(pack(kl01.x, kl01.y), pack(kl23.x, kl23.y));
            *reinterpret_cast<uint2*>(kb_buf + K_KQL + o_kql + (32 + r) * 128 + s16) =
                make_uint2(pack(ql01.x, ql01.y), pack(ql23.x, ql23.y));
            *reinterpret_cast<uint2*>(kb_buf + K_KB + o_kb + r * 128 + s16) =
                make_uint2(pack(kb01.x, kb01.y), pack(kb23.x, kb23.y));
            // B of [O | P] (bf16, same layout as the Gram A): q e^G and k e^G rows
            // of each 64-channel block in the order of buffer b's columns
            *reinterpret_cast<uint2*>(hb + H_QK + o_kql + (q_row(b) + r) * 128 + s16) =
                make_uint2(pack(qg01.x, qg01.y), pack(qg23.x, qg23.y));
            *reinterpret_cast<uint2*>(hb + H_QK + o_kql + (k_row(b) + r) * 128 + s16) =
                make_uint2(pack(kg01.x, kg01.y), pack(kg23.x, kg23.y));
          }
          // Kc^T rows c0..c0+3 (K-major: row = channel), tokens 8pw + 4hf .. +3 of each
#pragma unroll
          for (int k4 = 0; k4 < 4; ++k4)
            *reinterpret_cast<float4*>(hb + H_KC + kc_off(kc_row(b) + c0 + k4, 8 * pw + 4 * hf)) =
                make_float4(kc[k4][0], kc[k4][1], kc[k4][2], kc[k4][3]);
        }
      }
      fence_proxy_async();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&bars[B_OPER + b]);
        mbar_arrive(&bars[B_IN_EMPTY + st]);
      }
    }
  } else if (warp < STATE_W0) {
    // ============================================================== solve warps
    const int sw = warp - SOLVE_W0;  // TMEM lane quarter
    const int stid = tid - 32 * SOLVE_W0;
    for (int c = 0; c < nchunks; ++c) {
      if (bar_red_or(2, 128, *abort_flag != 0)) break;
      const int b = c & 1;
      uint8_t* kb_buf = sm + SM_KEY + b * KEYB;
      uint8_t* hb = sm + SM_HB + b * HBB;
      const float* betas = reinterpret_cast<const float*>(sm + SM_BETA + b * 128);
      wait(&bars[B_OPER + b], (c >> 1) & 1, 3);
      __syncwarp();
      {  // Gram: warp sw computes rows 16 sw .. +15 of [K_L ; Q_L] K_B^T (64 x 32,
         // K = 128 channels) with m16n8k16 MMAs from the swizzled tiles, then
         // A_kk^T (x beta, strictly lower; sw 0, 1) or A_qk (lower; sw 2, 3)
        const uint32_t kbase = sb + SM_KEY + b * KEYB;
        const int jm = lane >> 3, rr = lane & 7;
        float acc[4][4];
#pragma unroll
        for (int nt = 0; nt < 4; ++nt)
#pragma unroll
          for (int e = 0; e < 4; ++e) acc[nt][e] = 0.f;
#pragma unroll 2
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t kb = (uint32_t)(kk >> 2), c16 = (uint32_t)((kk & 3) * 2);
          const int arow = 16 * sw + rr + 8 * (jm & 1);  // matrices: rows x channel halves
          const uint32_t ac = c16 + (uint32_t)(jm >> 1);
          uint32_t a0, a1, a2, a3;
          ldsm_x4(kbase + K_KQL + kb * 8192 + arow * 128 + ((ac ^ (uint32_t)(arow & 7)) << 4), a0,
                  a1, a2, a3);
#pragma unroll
          for (int np = 0; np < 2; ++np) {  // n-tiles 2np, 2np + 1
            const int brow = 8 * (2 * np + (jm >> 1)) + rr;
            const uint32_t bc = c16 + (uint32_t)(jm & 1);
            uint32_t b0, b1, b2, b3;
            ldsm_x4(kbase + K_KB + kb * 4096 + brow * 128 + ((bc ^ (uint32_t)(brow & 7)) << 4), b0,
                    b1, b2, b3);
            mma_m16n8k16_bf16(acc[2 * np], a0, a1, a2, a3, b0, b1);
            mma_m16n8k16_bf16(acc[2 * np + 1], a0, a1, a2, a3, b2, b3);
          }
        }
        // A_kk^T goes where K_B was: every warp's Gram must be done first
        named_bar(2, 128);
        // fragment: rows lane / 4 (+ 8), columns 8 nt + 2 (lane % 4) + {0, 1}
        const int rl = lane >> 2, cq = 2 * (lane & 3);
        if (sw < 2) {
          float* akkt = reinterpret_cast<float*>(kb_buf + K_AKKT);
#pragma unroll
          for (int hh = 0; hh < 2; ++hh) {
            const int r = 16 * sw + rl + 8 * hh;
            const float br = betas[r];
#pragma unroll
            for (int nt = 0; nt < 4; ++nt)
#pragma unroll
              for (int e = 0; e < 2; ++e) {
                const int s2 = 8 * nt + cq + e;
                akkt[s2 * 32 + r] = s2 < r ? br * acc[nt][2 * hh + e] : 0.f;
              }
          }
        } else {
#pragma unroll
          for (int hh = 0; hh < 2; ++hh) {
            const int r = 16 * (sw - 2) + rl + 8 * hh;
#pragma unroll
            for (int nt = 0; nt < 4; ++nt) {
              const int s2 = 8 * nt + cq;
              const float2 w2 = make_float2(s2 <= r ? acc[nt][2 * hh] : 0.f,
                                            s2 + 1 <= r ? acc[nt][2 * hh + 1] : 0.f);
              *reinterpret_cast<float2*>(hb + H_KC + kc_off(aqk_row(b) + r, (uint32_t)s2)) = w2;
            }
          }
        }
      }
      named_bar(2, 128);

      // ---- T = (I + A_kk)^-1 Diag(beta), blocked 2 x 2 over 16-row blocks
      const float* akkt = reinterpret_cast<const float*>(kb_buf + K_AKKT);
      float* xs = reinterpret_cast<float*>(kb_buf + K_XS);
      auto tt_store = [&](int r, int col, float val) {  // T[r][col], tf32 B operand layout
        *reinterpret_cast<float*>(
            kb_buf + K_TF + r * 128 + ((((uint32_t)(col * 4) >> 4) ^ (uint32_t)(r & 7)) << 4) +
            ((col * 4) & 15)) = val;
      };
      if (sw == 0) {  // diagonal blocks: lane = (block bb, column cb)
        const int bb = lane >> 4, cb = lane & 15, o = 16 * bb;
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
          if (bb == 0) tt_store(r, 16 + cb, 0.f);  // upper-right block of T is zero
        }
      }
      named_bar(2, 128);
      const int cl = stid & 15, rp = stid >> 4;
#pragma unroll
      for (int h2 = 0; h2 < 2; ++h2) {  // Y = A10 X00 into the lower-left block of xs
        const int r = 2 * rp + h2;
        float y = 0.f;
#pragma unroll
        for (int s2 = 0; s2 < 16; ++s2) y = fmaf(akkt[s2 * 32 + 16 + r], xs[s2 * 32 + cl], y);
        xs[(16 + r) * 32 + cl] = y;
      }
      named_bar(2, 128);
      const float bcl = betas[cl];
#pragma unroll
      for (int h2 = 0; h2 < 2; ++h2) {  // X10 = -X11 Y
        const int r = 2 * rp + h2;
        float x10 = 0.f;
#pragma unroll
        for (int t2 = 0; t2 < 16; ++t2)
          x10 = fmaf(xs[(16 + r) * 32 + 16 + t2], xs[(16 + t2) * 32 + cl], x10);
        tt_store(16 + r, cl, -x10 * bcl);
      }
      fence_proxy_async();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars[B_T + b]);
    }
  } else if (warp < ISSUE_W) {
    // ============================================================== state warps
    const int j = 32 * (warp & 3) + lane;
    float vn[32];  // -v of the next chunk, column j
    // -V^T (lane j, column r) of chunk cc from its v tile; rows past the end
    // read as 0 (T has zero columns there, so any finite value would do)
    const uint32_t v_off = (uint32_t)(j >> 6) * 4096 + (uint32_t)(((j & 63) * 2) & 15);
    const uint32_t v_ck = (uint32_t)((j & 63) * 2) >> 4;
    auto load_v = [&](int cc) {
      const int n = chunk_rows(cc);
      const int vb = cc % NVBUF;
      if (!U.vzero) {
        wait(&bars[B_V + vb], (cc / NVBUF) & 1, 9);
        __syncwarp();
      }
      const uint8_t* vt = sm + SM_V + vb * 8192 + v_off;
#pragma unroll
      for (int r = 0; r < C; ++r) {
        const uint32_t bits = *reinterpret_cast<const unsigned short*>(
            vt + r * 128 + ((v_ck ^ (uint32_t)(r & 7)) << 4));
        vn[r] = (!U.vzero && r < n) ? -__uint_as_float(bits << 16) : 0.f;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars[B_VEMPTY + vb]);
    };
    // chunk cc's [O^T | P^T] starts as [0 | -V^T], in buffer cc & 1 (free once
    // chunk cc - 2's O is read out and its U GEMM has read its P)
    auto seed = [&](int cc) {
      load_v(cc);
      tmem_st32(tbase + lane_base + p_col(cc & 1), vn);
      const uint32_t z[16] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
      tmem_st16(tbase + lane_base + o_col(cc & 1), z);
      tmem_st16(tbase + lane_base + o_col(cc & 1) + 16, z);
    };
    // One pass over the state once the previous [S | O] GEMM is done: the bf16
    // copy of S^T (the A operand of chunk cc's [O | P]) and, from the same load,
    // S^T *= e^{Gamma_C, i} of chunk cc (what chunk cc's [S | O] accumulates onto).
    // Doing both here keeps tensor-memory traffic off the time the GEMMs run.
    auto copy_and_decay = [&](int cc) {
      wait(&bars[B_OPER + (cc & 1)], (cc >> 1) & 1, 5);  // e^{Gamma_C} of chunk cc
      __syncwarp();
      const float4* g4 = reinterpret_cast<const float4*>(sm + SM_GAMC + (cc & 1) * 512);
#pragma unroll 1
      for (int q = 0; q < 4; ++q) {
        float v[32];
        tmem_ld32(tbase + lane_base + S_COL + 32 * q, v);
        wait_ld();
        uint32_t pk[16];
#pragma unroll
        for (int k = 0; k < 16; ++k) {
          const __nv_bfloat162 b2 = __floats2bfloat162_rn(v[2 * k], v[2 * k + 1]);
          pk[k] = *reinterpret_cast<const uint32_t*>(&b2);
        }
        tmem_st16(tbase + lane_base + SB_COL + 16 * q, pk);
#pragma unroll
        for (int k4 = 0; k4 < 8; ++k4) {
          const float4 gg = g4[8 * q + k4];
          const float2 a = __fmul2_rn(make_float2(v[4 * k4], v[4 * k4 + 1]), make_float2(gg.x, gg.y));
          const float2 b2 =
              __fmul2_rn(make_float2(v[4 * k4 + 2], v[4 * k4 + 3]), make_float2(gg.z, gg.w));
          v[4 * k4 + 0] = a.x;
          v[4 * k4 + 1] = a.y;
          v[4 * k4 + 2] = b2.x;
          v[4 * k4 + 3] = b2.y;
        }
        tmem_st32(tbase + lane_base + S_COL + 32 * q, v);
      }
    };
    // hand-off to the issuer: [O | P] seeded, the bf16 state written, the state decayed
    auto publish = [&]() {
      wait_st();
      fence_before_sync();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&bars[B_OREADY]);
        mbar_arrive(&bars[B_DECAY]);
      }
    };
    if (nchunks > 0) {  // chunks 0 and 1
      seed(0);
      if (nchunks > 1) seed(1);
      copy_and_decay(0);
      publish();
    }
    for (int c = 0; c < nchunks; ++c) {
      if (bar_red_or(3, 128, *abort_flag != 0)) break;
      const int b = c & 1;
      const bool more = c + 1 < nchunks;
      wait(&bars[B_SO + b], (c >> 1) & 1, 7);
      __syncwarp();
      fence_after_sync();
      // critical path: bf16 S and decay for the next chunk
      if (more) {
        copy_and_decay(c + 1);
        publish();
      }
      float vo[32];  // O^T (lane j, column r)
      tmem_ld32(tbase + lane_base + o_col(b), vo);
      wait_ld();
      if (U.out_on && in_bounds(P.sb, U.row0 + (int64_t)c * C + chunk_rows(c) - 1,
                                (int64_t)P.B * P.T, kSiteTcOutRows)) {
        // lanes j, j^1 swap values so each writes a bf16 pair
        const int n = chunk_rows(c);
        const bool odd = lane & 1;
        const int jp = j & ~1;
        __nv_bfloat16* obase = P.out + ((size_t)(U.row0 + (int64_t)c * C) * H + h) * D + jp;
#pragma unroll
        for (int m = 0; m < 16; ++m) {
          const float send = odd ? vo[2 * m] : vo[2 * m + 1];
          const float recv = __shfl_xor_sync(0xffffffffu, send, 1);
          const int r = 2 * m + (odd ? 1 : 0);
          const float lo = odd ? recv : vo[2 * m];      // column jp
          const float hi = odd ? vo[2 * m + 1] : recv;  // column jp + 1
          if (r < n)
            *reinterpret_cast<__nv_bfloat162*>(obase + (size_t)r * H * D) =
                __floats2bfloat162_rn(P.scale * lo, P.scale * hi);
        }
      }
      if (c + 2 < nchunks) seed(c + 2);  // buffer b is free again: O read, P used
    }
    // final state (S^T lane j, column i -> final[i][j]); every S GEMM is done
    if (U.final_state && !*abort_flag) {
#pragma unroll 1
      for (int cc = 0; cc < 4; ++cc) {
        float v[32];
        tmem_ld32(tbase + lane_base + S_COL + 32 * cc, v);
        wait_ld();
#pragma unroll
        for (int k = 0; k < 32; ++k) U.final_state[(size_t)(32 * cc + k) * D + j] = v[k];
      }
    }
  } else if (warp == ISSUE_W) {
    // ============================================ state-side MMA issue (lane 0)
    if (lane == 0) {
      const uint32_t id_op = idesc(kFmtBF16, 128, 2 * C, false, false, false);    // [O^T | P^T]
      const uint32_t id_u = idesc(kFmtTF32, 128, C, false, false, true);          // U^T = -P^T T^T
      const uint32_t id_so = idesc(kFmtTF32, 128, D + C, false, false, false);    // [S^T | O^T]
      for (int c = 0; c < nchunks; ++c) {
        if (*abort_flag) break;
        const int b = c & 1;
        // [O^T | P^T] += S^T [Qg ; Ka]^T (bf16, A = the bf16 copy of S^T) once the
        // operands are written and O / P are seeded (which the state warps do
        // after the previous [S | O] completed)
        wait(&bars[B_OPER + b], (c >> 1) & 1, 10);
        wait(&bars[B_OREADY], c & 1, 11);
        if (*abort_flag) break;
        fence_after_sync();
        const uint32_t hb = sb + SM_HB + b * HBB;
#pragma unroll 1
        for (int ks = 0; ks < 8; ++ks)
          mma_ts_bf16(tbase + op_col(b), tbase + SB_COL + 8 * ks,
                      sw128_desc(hb + H_QK + (ks >> 2) * 8192 + (ks & 3) * 32, 16, 1024), id_op,
                      1);
        mma_commit(&bars[B_UO]);
        // U^T = -P^T T^T once P is complete and T is in
        wait(&bars[B_T + b], (c >> 1) & 1, 12);
        wait(&bars[B_UO], c & 1, 13);
        if (*abort_flag) break;
        fence_after_sync();
        const uint32_t kbb = sb + SM_KEY + b * KEYB;
#pragma unroll 1
        for (int ks = 0; ks < 4; ++ks)
          mma_ts_tf32(tbase + U_COL, tbase + p_col(b) + 8 * ks,
                      sw128_desc(kbb + K_TF + ks * 32, 16, 1024), id_u, ks > 0);
        mma_commit(&bars[B_U]);
        // [S^T | O^T] += U^T [Kc ; A_qk]^T once U is done and the state is decayed
        wait(&bars[B_U], c & 1, 14);
        wait(&bars[B_DECAY], c & 1, 15);
        if (*abort_flag) break;
        fence_after_sync();
#pragma unroll 1
        for (int ks = 0; ks < 4; ++ks)
          mma_ts_tf32(tbase + so_col(b), tbase + U_COL + 8 * ks,
                      plain_desc(hb + H_KC + 2 * ks * KC_LBO, KC_LBO, KC_SBO), id_so, 1);
        mma_commit(&bars[B_SO + b]);
      }
      if (*abort_flag) {  // every MMA this thread issued lands before TMEM is released
        mma_commit(&bars[B_DRAIN]);
        mbar_wait_drain(&bars[B_DRAIN], 0);
      }
    }
    __syncwarp();
  } else {
    // ========================================= TMA issue (lane 0 of the last warp)
    if (lane == 0) {
      int nv = 0;  // v loads issued
      auto issue_qkg = [&](int cc) {  // into stage cc & 1
        const int row = (int)(U.row0 + (int64_t)cc * C);
        uint8_t* in = sm + (cc & 1) * STAGE;
        uint64_t* bf = &bars[B_IN_FULL + (cc & 1)];
        fence_proxy_async();
        mbar_arrive_expect_tx(bf, TX_QKG);
        tma_load_3d(in + OFF_Q, &P.tm_q, bf, 0, h, row);
        tma_load_3d(in + OFF_K, &P.tm_k, bf, 0, h, row);
        tma_load_3d(in + OFF_G, &P.tm_g, bf, 0, h, row);
        if (!U.vzero) {  // v into its ring slot, once the chunk 4 back has been read
          const int vb = cc % NVBUF;
          if (cc >= NVBUF && !wait(&bars[B_VEMPTY + vb], ((cc - NVBUF) / NVBUF) & 1, 18))
            return;
          uint8_t* dst = sm + SM_V + vb * 8192;
          uint64_t* bv = &bars[B_V + vb];
          mbar_arrive_expect_tx(bv, TX_V);
          tma_load_3d(dst, &P.tm_v, bv, 0, h, row);
          tma_load_3d(dst + 4096, &P.tm_v, bv, 64, h, row);
          nv = cc + 1;
        }
      };
      int nq = 0;
      for (; nq < 2 && nq < nchunks; ++nq) issue_qkg(nq);
      for (int c = 0; c + 2 < nchunks; ++c) {
        if (*abort_flag) break;
        // q, k, g of chunk c + 2 into the stage chunk c's prep has released
        wait(&bars[B_IN_EMPTY + (c & 1)], (c >> 1) & 1, 17);
        if (*abort_flag) break;
        issue_qkg(nq++);
      }
      if (*abort_flag) {
        // every TMA load this thread issued lands before shared memory is released
        for (int k = (nq > 2 ? nq - 2 : 0); k < nq; ++k)
          mbar_wait_drain(&bars[B_IN_FULL + (k & 1)], (k >> 1) & 1);
        for (int k = (nv > NVBUF ? nv - NVBUF : 0); k < nv; ++k)
          mbar_wait_drain(&bars[B_V + k % NVBUF], (k / NVBUF) & 1);
      }
    }
    __syncwarp();
  }
  fence_before_sync();
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

// S_in of segment `index`: fold S_in <- S~_r + M_r S_in over r < index, from
// pairs laid out [count][units]{S~, M}; one 32-column slice per CTA.
__global__ void __launch_bounds__(256) state_prefix_kernel(const float* __restrict__ pairs,
                                                           int count, int index,
                                                           const float* __restrict__ init,
                                                           int units, float* __restrict__ out) {
  __shared__ float X[D][33];
  const size_t DD = (size_t)D * D;
  const int un = blockIdx.x >> 2, j0 = (blockIdx.x & 3) * 32;
  const int tid = threadIdx.x, jj = tid & 31, i0 = tid >> 5;
  for (int k = 0; k < 16; ++k) {
    const int i = i0 + 8 * k;
    X[i][jj] = init ? init[un * DD + (size_t)i * D + j0 + jj] : 0.f;
  }
  __syncthreads();
  for (int r = 0; r < index && r < count; ++r) {
    const float* St = pairs + ((size_t)r * units + un) * 2 * DD;
    const float* M = St + DD;
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
    for (int k = 0; k < 16; ++k) X[i0 + 8 * k][jj] = acc[k];
    __syncthreads();
  }
  for (int k = 0; k < 16; ++k) {
    const int i = i0 + 8 * k;
    out[un * DD + (size_t)i * D + j0 + jj] = X[i][jj];
  }
}

// ------------------------------------------------------------------- host
// The driver's entry point is the same for every device; the function-local
// static is initialised once, thread-safely.
PFN_cuTensorMapEncodeTiled_v12000 get_encode_fn() {
  static const PFN_cuTensorMapEncodeTiled_v12000 fn = []() {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    return static_cast<PFN_cuTensorMapEncodeTiled_v12000>(nullptr);
  }();
  return fn;
}

// Bound of the kernel's mbarrier waits: kWaitLimitNs unless a diagnostic
// lowered it (kda_set_wait_limit_ns), process-wide.
std::atomic<long long> g_wait_limit_ns{kWaitLimitNs};
long long wait_limit_ns() { return g_wait_limit_ns.load(std::memory_order_relaxed); }

// The shared-memory limit is a per-device attribute of the kernel: set it on
// every launch (a cheap host call) so that any device the caller makes
// current gets it, from any host thread.
cudaError_t allow_chunk_smem() {
  return cudaFuncSetAttribute(chunk_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              SMEM_ALLOC);
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
  // one CTA per SM: split when the units fill less than half the SMs.  A split
  // into G segments runs 2 (G - 1) U transition CTAs, then G U output CTAs,
  // each over T / G tokens; take the G with the fewest waves per token, and
  // a larger G only when it saves more than 5 % (each segment adds
  // 3 x 64 KB of workspace per unit and a step of the serial combine).
  const int U = B * H;
  *G_out = 1;
  *seg_out = T;
  if (2 * U >= num_sms || T < 4 * 1024) return;
  const int max_g = T / 1024;
  int best_g = 1;
  double best_cost = 1.0;  // no split: one wave over T tokens
  for (int G = 2; G <= max_g && G <= 64; ++G) {
    const int w1 = (2 * (G - 1) * U + num_sms - 1) / num_sms;
    const int w2 = (G * U + num_sms - 1) / num_sms;
    const double cost = (double)(w1 + w2) / G;
    if (cost < 0.95 * best_cost) {
      best_cost = cost;
      best_g = G;
    }
  }
  if (best_g < 2) return;
  int seg = (T + best_g - 1) / best_g;
  seg = (seg + C - 1) / C * C;
  const int G = (T + seg - 1) / seg;
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
  {
    const cudaError_t e = allow_chunk_smem();
    if (e != cudaSuccess) return e;
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
  P.wait_limit_ns = wait_limit_ns();
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

cudaError_t launch_chunk_tc_transition(const ChunkArgs& a, float* pairs, cudaStream_t stream) {
  if (a.num_units == 0) return cudaSuccess;
  {
    const cudaError_t e = allow_chunk_smem();
    if (e != cudaSuccess) return e;
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
  P.sb = a.sb;
  P.B = a.map.B;
  P.T = a.map.T;
  P.H = H;
  P.scale = 1.f;
  P.wait_limit_ns = wait_limit_ns();
  // transition mode over the whole range as the one segment before a second:
  // CTA pair u = (S~ from zero with v, M from the identity with v = 0)
  P.mode = 1;
  P.G = 2;
  P.seg_len = a.map.T;
  P.seg_ws = pairs;
  chunk_tc_kernel<<<a.num_units * 2, NT, SMEM_ALLOC, stream>>>(P);
  return cudaGetLastError();
}

void set_wait_limit_ns(long long ns) { g_wait_limit_ns.store(ns, std::memory_order_relaxed); }

cudaError_t launch_state_prefix(const float* pairs, int count, int index, const float* init,
                                int units, float* state_out, cudaStream_t stream) {
  if (units == 0) return cudaSuccess;
  state_prefix_kernel<<<units * 4, 256, 0, stream>>>(pairs, count, index, init, units,
                                                     state_out);
  return cudaGetLastError();
}

}  // namespace kda
