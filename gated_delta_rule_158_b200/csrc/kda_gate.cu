// kda_gate.cu -- the lower-bounded log-decay gate.
//
// "NLP--技术报告解读-Kimi-K3" (joezjh.github.io), Model Architecture > Kimi
// Delta Attention (KDA) > Lower-bounded decay:
//   g_t^h = g_min * Sigmoid(exp(A_h) * z_t^h),  g_min = -5,
// which keeps the retention alpha = exp(g) above e^-5.
//
// Forward: purely elementwise and HBM-bound: 4 bytes read and 4 written per
// element.
// Each thread handles float4 groups with a grid-stride loop; the grid is a
// multiple of the SM count.
#include "kda_host.cuh"

namespace kda {
namespace {

__global__ void __launch_bounds__(256) gate_kernel(const float4* __restrict__ z,
                                                   const float* __restrict__ A_log,
                                                   float g_min, float4* __restrict__ g,
                                                   int64_t n4, int H, int dk4) {
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < n4; e += stride) {
    const int h = (int)((e / dk4) % H);
    const float a = expf(__ldg(A_log + h));
    const float4 x = __ldcs(z + e);  // streamed once: evict-first
    float4 y;
    y.x = g_min / (1.0f + expf(-a * x.x));
    y.y = g_min / (1.0f + expf(-a * x.y));
    y.z = g_min / (1.0f + expf(-a * x.z));
    y.w = g_min / (1.0f + expf(-a * x.w));
    g[e] = y;
  }
}

// Gradients of the gate (its chain rule): with x = e^{A_h} z, s = sigmoid(x),
//   dz = dg g_min s (1 - s) e^{A_h},   dA_log[h] = sum dg g_min s (1 - s) x.
// Block (h, part) takes rows part, part + nparts, ... of head h, writes dz and
// one partial sum of dA_log[h]; a second kernel adds the partials of each head
// in a fixed order, so the result does not depend on scheduling.
constexpr int kGateBwdThreads = 256;

__global__ void __launch_bounds__(kGateBwdThreads)
    gate_bwd_kernel(const float* __restrict__ z, const float* __restrict__ A_log, float g_min,
                    const float* dg, float* dz, int64_t rows, int H, int dk, int nparts,
                    float* __restrict__ partial) {
  const int h = blockIdx.x / nparts, part = blockIdx.x % nparts;
  const float a = expf(A_log[h]);
  const int dk4 = dk / 4;
  const int per = kGateBwdThreads / dk4;  // rows per step (dk4 divides 256)
  const int tid = threadIdx.x, c4 = tid % dk4, rsub = tid / dk4;
  float acc = 0.f;
  for (int64_t r = (int64_t)part * per + rsub; r < rows; r += (int64_t)nparts * per) {
    const int64_t e = (r * H + h) * dk4 + c4;
    const float4 x4 = reinterpret_cast<const float4*>(z)[e];
    const float4 d4 = reinterpret_cast<const float4*>(dg)[e];
    float xs[4] = {a * x4.x, a * x4.y, a * x4.z, a * x4.w};
    float ds[4] = {d4.x, d4.y, d4.z, d4.w};
    float out[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float sg = 1.0f / (1.0f + expf(-xs[j]));
      const float d = ds[j] * g_min * sg * (1.0f - sg);
      out[j] = d * a;
      acc = fmaf(d, xs[j], acc);
    }
    reinterpret_cast<float4*>(dz)[e] = make_float4(out[0], out[1], out[2], out[3]);
  }
  __shared__ float red[kGateBwdThreads / 32];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  if ((tid & 31) == 0) red[tid >> 5] = acc;
  __syncthreads();
  if (tid == 0) {
    float t = 0.f;
    for (int w = 0; w < kGateBwdThreads / 32; ++w) t += red[w];
    partial[blockIdx.x] = t;
  }
}

__global__ void gate_bwd_sum_kernel(const float* __restrict__ partial, int H, int nparts,
                                    float* __restrict__ dA_log) {
  for (int h = threadIdx.x; h < H; h += blockDim.x) {
    float t = 0.f;
    for (int p = 0; p < nparts; ++p) t += partial[h * nparts + p];
    dA_log[h] = t;
  }
}

}  // namespace

int gate_bwd_parts(int64_t rows) {
  return (int)(rows < kGateBwdMaxParts ? (rows > 0 ? rows : 1) : kGateBwdMaxParts);
}

cudaError_t launch_gate_bwd(const float* z, const float* A_log, float g_min, const float* dg,
                            float* dz, float* dA_log, int64_t rows, int H, int dk,
                            float* partial, cudaStream_t stream) {
  const int nparts = gate_bwd_parts(rows);
  gate_bwd_kernel<<<(unsigned)(H * nparts), kGateBwdThreads, 0, stream>>>(
      z, A_log, g_min, dg, dz, rows, H, dk, nparts, partial);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  gate_bwd_sum_kernel<<<1, 256, 0, stream>>>(partial, H, nparts, dA_log);
  return cudaGetLastError();
}

cudaError_t launch_gate(const float* z, const float* A_log, float g_min, float* g,
                        int64_t rows, int H, int dk, cudaStream_t stream) {
  const int64_t n4 = rows * (int64_t)H * dk / 4;
  const int sms = device_sm_count();
  int64_t blocks = (n4 + 255) / 256;
  const int64_t cap = (int64_t)sms * 16;
  if (blocks > cap) blocks = cap;
  if (blocks < 1) blocks = 1;
  gate_kernel<<<(unsigned)blocks, 256, 0, stream>>>(
      reinterpret_cast<const float4*>(z), A_log, g_min, reinterpret_cast<float4*>(g), n4, H,
      dk / 4);
  return cudaGetLastError();
}

}  // namespace kda
