// Kernels of the I-sharded layer (see partial.cuh).
#include "partial.cuh"

namespace moe {
namespace {

__global__ void combine_f32_kernel(const float* __restrict__ ypair, const int32_t* __restrict__ inv, int T, int K,
                                   int H, float* __restrict__ y) {
  const int H4 = H / 4;
  const int64_t n = (int64_t)T * H4;
  for (int64_t g = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; g < n; g += (int64_t)gridDim.x * blockDim.x) {
    const int t = (int)(g / H4), h = (int)(g % H4) * 4;
    float4 s = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int slot = 0; slot < K; ++slot) {
      const int pos = __ldg(inv + t * K + slot);
      const float4 v = __ldcg(reinterpret_cast<const float4*>(ypair + (int64_t)pos * H + h));
      s.x += v.x; s.y += v.y; s.z += v.z; s.w += v.w;
    }
    *reinterpret_cast<float4*>(y + (int64_t)t * H + h) = s;
  }
}

__global__ void round_bf16_kernel(const float* __restrict__ in, __nv_bfloat16* __restrict__ out, int64_t n) {
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x)
    out[i] = __float2bfloat16_rn(in[i]);
}

unsigned blocks_for(int64_t n) {
  const int64_t b = (n + 255) / 256;
  return (unsigned)(b < 4096 ? (b > 0 ? b : 1) : 4096);
}

}  // namespace

cudaError_t combine_f32_launch(const float* ypair, const int32_t* inv, int T, int K, int H, float* y,
                               cudaStream_t s) {
  combine_f32_kernel<<<blocks_for((int64_t)T * H / 4), 256, 0, s>>>(ypair, inv, T, K, H, y);
  return cudaGetLastError();
}

cudaError_t round_bf16_launch(const float* in, __nv_bfloat16* out, int64_t n, cudaStream_t s) {
  round_bf16_kernel<<<blocks_for(n), 256, 0, s>>>(in, out, n);
  return cudaGetLastError();
}

}  // namespace moe
