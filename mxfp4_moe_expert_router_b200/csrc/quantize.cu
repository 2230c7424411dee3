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

// Streaming stages for the tensor-core weight stream.  A stage is 64 weight
// rows (four 16-row MMA tiles t) x KC = 128 K elements (four MX blocks b).
// Codes: [b][half][lane][16 B]; for lane (g = lane/4, c = lane%4) the 16 bytes
// of half h hold tiles 2h and 2h+1, each as two k16 steps s of four bytes
//   R[g][c + 8s], R[g+8][c + 8s], R[g][c + 4 + 8s], R[g+8][c + 4 + 8s]
// where R[r][j] is byte j (elements 2j, 2j+1) of row r's 16-byte block chunk:
// exactly the A-fragment registers a0..a3 of mma.m16n8k16 after E2M1 -> f16x2.
// Scales: [row 64][b 4].  Gate/up stage rows: tile 0/1 = gate rows i0..i0+31,
// tile 2/3 = up rows i0..i0+31 (i0 = 32 * row block); down stage rows:
// h0 + 16 t + r (h0 = 64 * row block).
__device__ __forceinline__ int64_t stage_src_row(int is_down, int e, int nrows, int rb, int t, int rr,
                                                 int* which) {
  if (is_down) { *which = 0; return (int64_t)e * nrows + rb * STAGE_ROWS + t * 16 + rr; }
  *which = t >= 2;  // 0 gate, 1 up
  return (int64_t)e * nrows + rb * (STAGE_ROWS / 2) + (t & 1) * 16 + rr;
}

__global__ void repack_codes_kernel(const uint8_t* __restrict__ c0, const uint8_t* __restrict__ c1,
                                    int is_down, int E, int nrows, int K, uint8_t* __restrict__ out) {
  const int nc = K / KC, nrb = is_down ? nrows / STAGE_ROWS : nrows / (STAGE_ROWS / 2);
  const int64_t total = (int64_t)E * nrb * nc * KB * 2 * 32;
  const int64_t gidx = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
  if (gidx >= total) return;
  const int lane = (int)(gidx % 32);
  const int half = (int)((gidx / 32) % 2);
  const int b = (int)((gidx / 64) % KB);
  const int64_t st = gidx / (64 * KB);
  const int c = (int)(st % nc);
  const int rb = (int)((st / nc) % nrb);
  const int e = (int)(st / ((int64_t)nc * nrb));
  const int g = lane >> 2, cc = lane & 3;
  const int kbg = c * KB + b;
  uint32_t w[4];
#pragma unroll
  for (int tt = 0; tt < 2; ++tt) {
    const int t = half * 2 + tt;
    int which = 0;
    const int64_t r0 = stage_src_row(is_down, e, nrows, rb, t, g, &which);
    const int64_t r1 = stage_src_row(is_down, e, nrows, rb, t, g + 8, &which);
    const uint8_t* src = which ? c1 : c0;
    const uint8_t* p0 = src + r0 * (K / 2) + kbg * 16;
    const uint8_t* p1 = src + r1 * (K / 2) + kbg * 16;
#pragma unroll
    for (int s = 0; s < 2; ++s) {
      const uint32_t b0 = p0[cc + 8 * s], b1 = p1[cc + 8 * s];
      const uint32_t b2 = p0[cc + 4 + 8 * s], b3 = p1[cc + 4 + 8 * s];
      w[tt * 2 + s] = b0 | (b1 << 8) | (b2 << 16) | (b3 << 24);
    }
  }
  uint8_t* so = out + st * STAGE_W_BYTES + ((b * 2 + half) * 32 + lane) * 16;
  *reinterpret_cast<uint4*>(so) = make_uint4(w[0], w[1], w[2], w[3]);
}

__global__ void repack_scales_kernel(const uint8_t* __restrict__ s0, const uint8_t* __restrict__ s1,
                                     int is_down, int E, int nrows, int K, uint8_t* __restrict__ out) {
  const int nc = K / KC, nrb = is_down ? nrows / STAGE_ROWS : nrows / (STAGE_ROWS / 2);
  const int64_t total = (int64_t)E * nrb * nc * STAGE_ROWS * KB;
  const int64_t gidx = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
  if (gidx >= total) return;
  const int b = (int)(gidx % KB);
  const int r = (int)((gidx / KB) % STAGE_ROWS);
  const int64_t st = gidx / (KB * STAGE_ROWS);
  const int c = (int)(st % nc);
  const int rb = (int)((st / nc) % nrb);
  const int e = (int)(st / ((int64_t)nc * nrb));
  int which = 0;
  const int64_t row = stage_src_row(is_down, e, nrows, rb, r >> 4, r & 15, &which);
  const uint8_t* src = which ? s1 : s0;
  out[st * STAGE_W_BYTES + STAGE_CODE_BYTES + r * KB + b] = src[row * (K / 32) + c * KB + b];
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
  const int64_t stages = (int64_t)E * (I / (STAGE_ROWS / 2)) * (H / KC);
  const int64_t n1 = stages * KB * 64, n2 = stages * STAGE_ROWS * KB;
  repack_codes_kernel<<<(unsigned)((n1 + 255) / 256), 256, 0, s>>>(gc, uc, 0, E, I, H, out);
  repack_scales_kernel<<<(unsigned)((n2 + 255) / 256), 256, 0, s>>>(gs, us, 0, E, I, H, out);
  return cudaGetLastError();
}

cudaError_t repack_d_launch(const uint8_t* dc, const uint8_t* ds, int E, int H, int I,
                            uint8_t* out, cudaStream_t s) {
  const int64_t stages = (int64_t)E * (H / STAGE_ROWS) * (I / KC);
  const int64_t n1 = stages * KB * 64, n2 = stages * STAGE_ROWS * KB;
  repack_codes_kernel<<<(unsigned)((n1 + 255) / 256), 256, 0, s>>>(dc, dc, 1, E, H, I, out);
  repack_scales_kernel<<<(unsigned)((n2 + 255) / 256), 256, 0, s>>>(ds, ds, 1, E, H, I, out);
  return cudaGetLastError();
}

}  // namespace moe
