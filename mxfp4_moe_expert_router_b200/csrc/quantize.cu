// MXFP4 quantiser (bf16 -> E2M1 codes + E8M0 scales) and the repack of
// canonical MXFP4 tensors into the tensor-core streaming stages of engine.cu.
//
// Format: OCP Microscaling v1.0 MXFP4, the expert-weight format the MiMo /
// TileRT pages name (bjdmk.com.cn news, section "极致协同，通向千速之路": 4 bits
// per expert parameter).  Per 32-element block along K:
//   s = max(floor(log2 amax) - 2, -127), scale byte = s + 127;
//   code = sign bit | nearest E2M1 magnitude of |w| / 2^s (ties to even,
//   saturating at 6); a block holding Inf/NaN gets scale 255 and zero codes.
// floor(log2 amax) is the biased exponent field of the bf16 amax minus 127
// (amax below 2^-126 clamps s to -127), so the scale byte is max(e - 2, 0).
#include "engine.cuh"
#include "ptx.cuh"

namespace moe {

namespace {

// Nearest E2M1 magnitude (0..7) of a non-negative fp32 value, ties to even,
// saturating at 6.  Both nibbles of the conversion hold the same code, so the
// result does not depend on which operand lands in which nibble.
__device__ __forceinline__ uint32_t e2m1_magnitude(float a) {
  return f32x2_to_e2m1x2(a, a) & 0x7u;
}

__global__ void __launch_bounds__(256) quantize_kernel(const uint16_t* __restrict__ w,
                                                       int64_t nblocks,
                                                       uint8_t* __restrict__ codes,
                                                       uint8_t* __restrict__ scales) {
  const int64_t b = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
  if (b >= nblocks) return;
  const uint4* src = reinterpret_cast<const uint4*>(w + b * 32);
  uint32_t v[16];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    uint4 q = __ldg(src + i);
    v[4 * i + 0] = q.x; v[4 * i + 1] = q.y; v[4 * i + 2] = q.z; v[4 * i + 3] = q.w;
  }
  uint32_t amax = 0, special = 0;
#pragma unroll
  for (int m = 0; m < 16; ++m) {
    uint32_t lo = v[m] & 0x7FFFu, hi = (v[m] >> 16) & 0x7FFFu;
    special |= (lo >= 0x7F80u) | (hi >= 0x7F80u);
    amax = max(amax, max(lo, hi));
  }
  uint4* dst = reinterpret_cast<uint4*>(codes + b * 16);
  if (special) {
    *dst = make_uint4(0, 0, 0, 0);
    scales[b] = 255;
    return;
  }
  const uint32_t e = amax >> 7;                       // biased exponent of amax
  const uint32_t sbyte = e > 2 ? e - 2 : 0;           // s + 127
  const float inv = __uint_as_float((254u - sbyte) << 23);  // 2^-s, exact
  uint32_t out[4] = {0, 0, 0, 0};
#pragma unroll
  for (int m = 0; m < 16; ++m) {
    const uint32_t lo = v[m] & 0xFFFFu, hi = v[m] >> 16;
    const float flo = __uint_as_float((lo & 0x7FFFu) << 16) * inv;
    const float fhi = __uint_as_float((hi & 0x7FFFu) << 16) * inv;
    const uint32_t clo = e2m1_magnitude(flo) | ((lo >> 15) << 3);
    const uint32_t chi = e2m1_magnitude(fhi) | ((hi >> 15) << 3);
    out[m >> 2] |= (clo | (chi << 4)) << (8 * (m & 3));
  }
  *dst = make_uint4(out[0], out[1], out[2], out[3]);
  scales[b] = static_cast<uint8_t>(sbyte);
}

// Streaming stages for the tensor-core weight stream.  A stage is JOB_ROWS =
// 128 weight rows x KS = 128 K elements (four MX blocks), stored as the
// block-scaled MMA reads it from shared memory:
//   codes: byte kk * 4096 + (m / 8) * 256 + kc * 128 + (m % 8) * 16 + j holds
//          elements 64 kk + 32 kc + 2 j (low nibble) and + 1 (high nibble) of
//          row m -- a straight copy of 16-byte pieces of the canonical rows,
//          whose nibble order is the MMA's;
//   scales: byte 8192 + (m % 32) * 16 + (m / 32) * 4 + b = scale of block b.
// Row m of a gate/up job (q = m / 32, l = m % 32) is gate (l < 16) or up
// (l >= 16) row i0 + 16 q + (l % 16), i0 = 64 * job row block; row m of a
// down job is hidden row h0 + m, h0 = 128 * job row block.
__device__ __forceinline__ int64_t stage_src_row(int is_down, int e, int nrows, int rb, int m,
                                                 int* which) {
  if (is_down) { *which = 0; return (int64_t)e * nrows + (int64_t)rb * JOB_ROWS + m; }
  const int q = m >> 5, l = m & 31;
  *which = l >= 16;  // 0 gate, 1 up
  return (int64_t)e * nrows + (int64_t)rb * GU_I_ROWS + 16 * q + (l & 15);
}

// One thread per (stage, row m, 16-byte chunk): a 128-element row is 64 bytes,
// four chunks (kk = chunk / 2, kc = chunk % 2).
__global__ void repack_codes_kernel(const uint8_t* __restrict__ c0, const uint8_t* __restrict__ c1,
                                    int is_down, int E, int nrows, int K, uint8_t* __restrict__ out) {
  const int nc = K / KS, nrb = is_down ? nrows / JOB_ROWS : nrows / GU_I_ROWS;
  const int64_t total = (int64_t)E * nrb * nc * JOB_ROWS * 4;
  const int64_t gidx = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
  if (gidx >= total) return;
  const int ch = (int)(gidx % 4);
  const int m = (int)((gidx / 4) % JOB_ROWS);
  const int64_t st = gidx / (4 * JOB_ROWS);
  const int c = (int)(st % nc);
  const int rb = (int)((st / nc) % nrb);
  const int e = (int)(st / ((int64_t)nc * nrb));
  int which = 0;
  const int64_t row = stage_src_row(is_down, e, nrows, rb, m, &which);
  const uint8_t* src = (which ? c1 : c0) + row * (K / 2) + (int64_t)c * (KS / 2) + ch * 16;
  const int kk = ch >> 1, kc = ch & 1;
  uint8_t* dst = out + st * STAGE_A_BYTES + kk * 4096 + (m >> 3) * 256 + kc * 128 + (m & 7) * 16;
  *reinterpret_cast<uint4*>(dst) = *reinterpret_cast<const uint4*>(src);
}

// One thread per (stage, row m): the row's four block scales.
__global__ void repack_scales_kernel(const uint8_t* __restrict__ s0, const uint8_t* __restrict__ s1,
                                     int is_down, int E, int nrows, int K, uint8_t* __restrict__ out) {
  const int nc = K / KS, nrb = is_down ? nrows / JOB_ROWS : nrows / GU_I_ROWS;
  const int64_t total = (int64_t)E * nrb * nc * JOB_ROWS;
  const int64_t gidx = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
  if (gidx >= total) return;
  const int m = (int)(gidx % JOB_ROWS);
  const int64_t st = gidx / JOB_ROWS;
  const int c = (int)(st % nc);
  const int rb = (int)((st / nc) % nrb);
  const int e = (int)(st / ((int64_t)nc * nrb));
  int which = 0;
  const int64_t row = stage_src_row(is_down, e, nrows, rb, m, &which);
  const uint8_t* src = (which ? s1 : s0) + row * (K / 32) + (int64_t)c * KB;
  uint8_t* dst = out + st * STAGE_A_BYTES + STAGE_CODE_BYTES + (m & 31) * 16 + (m >> 5) * 4;
  *reinterpret_cast<uint32_t*>(dst) =
      (uint32_t)src[0] | ((uint32_t)src[1] << 8) | ((uint32_t)src[2] << 16) | ((uint32_t)src[3] << 24);
}

}  // namespace

cudaError_t quantize_launch(const void* w, int64_t rows, int64_t K, uint8_t* codes,
                            uint8_t* scales, cudaStream_t s) {
  const int64_t nblocks = rows * (K / 32);
  if (nblocks == 0) return cudaSuccess;
  const int64_t grid = (nblocks + 255) / 256;
  quantize_kernel<<<(unsigned)grid, 256, 0, s>>>(static_cast<const uint16_t*>(w), nblocks, codes,
                                                 scales);
  return cudaGetLastError();
}

cudaError_t repack_gu_launch(const uint8_t* gc, const uint8_t* gs, const uint8_t* uc,
                             const uint8_t* us, int E, int I, int H, uint8_t* out, cudaStream_t s) {
  const int64_t stages = (int64_t)E * (I / GU_I_ROWS) * (H / KS);
  const int64_t n1 = stages * JOB_ROWS * 4, n2 = stages * JOB_ROWS;
  repack_codes_kernel<<<(unsigned)((n1 + 255) / 256), 256, 0, s>>>(gc, uc, 0, E, I, H, out);
  repack_scales_kernel<<<(unsigned)((n2 + 255) / 256), 256, 0, s>>>(gs, us, 0, E, I, H, out);
  return cudaGetLastError();
}

cudaError_t repack_d_launch(const uint8_t* dc, const uint8_t* ds, int E, int H, int I,
                            uint8_t* out, cudaStream_t s) {
  const int64_t stages = (int64_t)E * (H / JOB_ROWS) * (I / KS);
  const int64_t n1 = stages * JOB_ROWS * 4, n2 = stages * JOB_ROWS;
  repack_codes_kernel<<<(unsigned)((n1 + 255) / 256), 256, 0, s>>>(dc, dc, 1, E, H, I, out);
  repack_scales_kernel<<<(unsigned)((n2 + 255) / 256), 256, 0, s>>>(ds, ds, 1, E, H, I, out);
  return cudaGetLastError();
}

}  // namespace moe
