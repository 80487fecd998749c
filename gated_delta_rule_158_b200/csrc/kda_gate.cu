// kda_gate.cu -- the lower-bounded log-decay gate.
//
// "NLP--技术报告解读-Kimi-K3" (joezjh.github.io), Model Architecture > Kimi
// Delta Attention (KDA) > Lower-bounded decay:
//   g_t^h = g_min * Sigmoid(exp(A_h) * z_t^h),  g_min = -5,
// which keeps the retention alpha = exp(g) above e^-5.
//
// Purely elementwise and HBM-bound: 4 bytes read and 4 written per element.
// Each thread handles float4 groups with a grid-stride loop; the grid is a
// multiple of the SM count.
#include "kda_internal.cuh"

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

}  // namespace

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
