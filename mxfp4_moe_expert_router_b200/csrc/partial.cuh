// The I-sharded layer's two small kernels: a rank's fp32 partial output (the
// engine's pair outputs summed over the k slots, without rounding), and the
// bf16 rounding of the sum over ranks.
#pragma once
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace moe {

// y[t][h] = sum over slots s = 0 .. K-1, in slot order, of ypair[inv[t*K + s]][h]
// (fp32, the order of the engine's own combine).  H % 4 == 0.
cudaError_t combine_f32_launch(const float* ypair, const int32_t* inv, int T, int K, int H, float* y,
                               cudaStream_t s);
// out[i] = bf16(in[i]), round to nearest even.
cudaError_t round_bf16_launch(const float* in, __nv_bfloat16* out, int64_t n, cudaStream_t s);

}  // namespace moe
