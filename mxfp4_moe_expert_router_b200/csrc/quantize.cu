// MXFP4 quantiser (bf16 -> E2M1 codes + E8M0 scales) and the repack of
// canonical MXFP4 tensors into the streaming stage layout of engine.cu.
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

// Gate/up stages: stage (e, rb, c) holds rows r<16: gate row rb*16+r, r>=16: up
// row rb*16+r-16, K blocks c*KB .. c*KB+KB-1.  One thread per (stage, row, block).
__global__ void repack_gu_kernel(const uint8_t* __restrict__ gc, const uint8_t* __restrict__ gs,
                                 const uint8_t* __restrict__ uc, const uint8_t* __restrict__ us,
                                 int E, int I, int H, uint8_t* __restrict__ out) {
  const int nc = H / KC, nrb = I / GU_ROWS;
  const int64_t total = (int64_t)E * nrb * nc * ROWS * KB;
  const int64_t g = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
  if (g >= total) return;
  const int kb = (int)(g % KB);
  const int r = (int)((g / KB) % ROWS);
  const int64_t st = g / (KB * ROWS);
  const int c = (int)(st % nc);
  const int rb = (int)((st / nc) % nrb);
  const int e = (int)(st / ((int64_t)nc * nrb));
  const int i = rb * GU_ROWS + (r & 15);
  const uint8_t* sc = r < 16 ? gc : uc;
  const uint8_t* ss = r < 16 ? gs : us;
  const int kbg = c * KB + kb;
  const int64_t row = (int64_t)e * I + i;
  const uint4 q = *reinterpret_cast<const uint4*>(sc + row * (H / 2) + kbg * 16);
  uint8_t* so = out + st * STAGE_W_BYTES;
  *reinterpret_cast<uint4*>(so + kb * (ROWS * 16) + r * 16) = q;
  so[STAGE_CODE_BYTES + r * KB + kb] = ss[row * (H / 32) + kbg];
}

// Down stages: stage (e, rb, c) holds rows rb*32 .. rb*32+31 of Wd [H][I].
__global__ void repack_d_kernel(const uint8_t* __restrict__ dc, const uint8_t* __restrict__ ds,
                                int E, int H, int I, uint8_t* __restrict__ out) {
  const int nc = I / KC, nrb = H / ROWS;
  const int64_t total = (int64_t)E * nrb * nc * ROWS * KB;
  const int64_t g = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
  if (g >= total) return;
  const int kb = (int)(g % KB);
  const int r = (int)((g / KB) % ROWS);
  const int64_t st = g / (KB * ROWS);
  const int c = (int)(st % nc);
  const int rb = (int)((st / nc) % nrb);
  const int e = (int)(st / ((int64_t)nc * nrb));
  const int kbg = c * KB + kb;
  const int64_t row = (int64_t)e * H + rb * ROWS + r;
  const uint4 q = *reinterpret_cast<const uint4*>(dc + row * (I / 2) + kbg * 16);
  uint8_t* so = out + st * STAGE_W_BYTES;
  *reinterpret_cast<uint4*>(so + kb * (ROWS * 16) + r * 16) = q;
  so[STAGE_CODE_BYTES + r * KB + kb] = ds[row * (I / 32) + kbg];
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
  const int64_t total = (int64_t)E * (I / GU_ROWS) * (H / KC) * ROWS * KB;
  repack_gu_kernel<<<(unsigned)((total + 255) / 256), 256, 0, s>>>(gc, gs, uc, us, E, I, H, out);
  return cudaGetLastError();
}

cudaError_t repack_d_launch(const uint8_t* dc, const uint8_t* ds, int E, int H, int I,
                            uint8_t* out, cudaStream_t s) {
  const int64_t total = (int64_t)E * (H / ROWS) * (I / KC) * ROWS * KB;
  repack_d_kernel<<<(unsigned)((total + 255) / 256), 256, 0, s>>>(dc, ds, E, H, I, out);
  return cudaGetLastError();
}

}  // namespace moe
