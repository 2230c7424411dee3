// Persistent MXFP4 MoE engine: one cooperative launch runs, per layer,
//   A  router partial logits (fp64 accumulation), per-token f16 activations
//   B  top-k + renormalised weights, stable per-expert permutation, unit table
//   C  the MXFP4 weight stream on tensor cores: gate/up projection + SwiGLU,
//      then down projection x routing weight
//   D  weighted combine to bf16 (+ RMSNorm into the next layer's input)
// separated by bounded grid barriers.  The design follows the TileRT pages'
// execution model -- a resident engine kernel that keeps prefetching through
// shared memory while the current tile computes, a tile-level pipeline, and
// warp-specialised roles (TileRT blog "Breaking 1000 TPS", section
// "第一次跃迁：Execution Model Revolution"; bjdmk.com.cn news, section
// "极致协同，通向千速之路", on the persistent engine kernel) -- applied to the
// MoE expert layer whose routing is the runtime dynamism (HyperAI salon
// transcript, section "Achieving maximum speed improvement ...").
//
// Weight stream (phase C).  Work is cut into CTA jobs of 64 weight rows x the
// whole contraction dimension.  Warp NCW is the producer: it takes jobs from a
// global counter, publishes them in a shared-memory job queue and streams each
// job's K chunks (one 4352-byte MXFP4 stage + the matching activation slices)
// into a ring of NSLOT slots with 1-D bulk copies (full/empty mbarriers).
// Warps 0..NCW-1 consume chunk c of every job in warp c % NCW: E2M1 bytes are
// turned into f16 A fragments in registers, the tokens form the N side of
// mma.m16n8k16 (fp32 accumulate), and each MX block's E8M0 scale multiplies its
// block partial in fp32.  The per-warp partial sums meet in shared memory
// behind a named barrier and are reduced in warp order (deterministic), then
// one warp per token (gate/up) or per pair (down) runs the epilogue.
//
// Every wait (grid barrier, mbarrier, job queue, per-unit readiness) is bounded
// by p.timeout_ns of %globaltimer; on expiry the kernel records a status code
// in sync[SY_ERROR], stops issuing work, lets every copy in flight land and
// returns.
#include <math.h>
#include <cuda_fp16.h>

#include "engine.cuh"
#include "ptx.cuh"

namespace moe {
namespace {

constexpr uint32_t FULL = 0xFFFFFFFFu;
constexpr int SMALL_UNITS = 256 + SMALL_PAIRS / NT_MAX;
constexpr int SMALL_DUNITS = 256 + SMALL_PAIRS / ND_MAX;

struct JobEntry {
  int32_t flag;  // queue index + 1 once the entry is written
  int32_t job;   // -1: no more jobs in this phase
  int32_t s0;    // stage sequence number of chunk 0
  int32_t nc;    // chunks (stages)
  int32_t unit, rb, isD, e, pos0, nt, pad0, pad1;
};

struct alignas(16) CtaTables {
  int32_t units[SMALL_UNITS * 4];  // first: read as int4
  int32_t dunits[SMALL_DUNITS * 4];
  int32_t idx[SMALL_PAIRS];
  float w[SMALL_PAIRS];
  int32_t perm[SMALL_PAIRS];
  int32_t inv[SMALL_PAIRS];
  int32_t tokpos[SMALL_PAIRS];
  float wpos[SMALL_PAIRS];
  float pxf[SMALL_PAIRS];
  int32_t counts[MAX_EXPERTS];
  int32_t offsets[MAX_EXPERTS + 1];
  float red[WARPS];
  int32_t n_units, n_dunits;
};

constexpr size_t align16(size_t v) { return (v + 15) & ~size_t(15); }
constexpr size_t OFF_RING = 0;
constexpr size_t OFF_FULL = OFF_RING + (size_t)NSLOT * SLOT_BYTES;
constexpr size_t OFF_EMPTY = OFF_FULL + NSLOT * 8;
constexpr size_t OFF_JQ = align16(OFF_EMPTY + NSLOT * 8);
constexpr size_t OFF_PART = align16(OFF_JQ + JQ * sizeof(JobEntry));
constexpr size_t PART_BUF = (size_t)NCW * PART_COLS * PART_LD;  // floats per buffer
constexpr size_t OFF_TABLES = align16(OFF_PART + 2 * PART_BUF * 4);
constexpr size_t SMEM_BYTES = OFF_TABLES + sizeof(CtaTables);
static_assert(SMEM_BYTES <= 232448, "shared memory budget");
static_assert((size_t)WARPS * MAX_EXPERTS * 4 <= (size_t)NSLOT * SLOT_BYTES, "routing scratch in ring");

__device__ __forceinline__ uint8_t* ring_slot(uint8_t* smem, int s) { return smem + OFF_RING + (size_t)s * SLOT_BYTES; }
__device__ __forceinline__ uint64_t* full_bar(uint8_t* smem, int s) { return reinterpret_cast<uint64_t*>(smem + OFF_FULL) + s; }
__device__ __forceinline__ uint64_t* empty_bar(uint8_t* smem, int s) { return reinterpret_cast<uint64_t*>(smem + OFF_EMPTY) + s; }
__device__ __forceinline__ JobEntry* job_queue(uint8_t* smem) { return reinterpret_cast<JobEntry*>(smem + OFF_JQ); }
__device__ __forceinline__ float* part_buf(uint8_t* smem, int b) { return reinterpret_cast<float*>(smem + OFF_PART) + b * PART_BUF; }
__device__ __forceinline__ CtaTables& tables(uint8_t* smem) { return *reinterpret_cast<CtaTables*>(smem + OFF_TABLES); }

__device__ __forceinline__ void set_error(uint32_t* sync, uint32_t code, uint32_t info) {
  if (atomicCAS(sync + SY_ERROR, 0u, code) == 0u) atomicExch(sync + SY_ERRINFO, info);
}
__device__ __forceinline__ bool error_set(const uint32_t* sync) {
  return ld_volatile_u32(sync + SY_ERROR) != 0u;
}

// Grid-wide barrier over co-resident CTAs (cooperative launch), bounded.
__device__ bool grid_barrier(uint32_t* sync, uint64_t timeout_ns, uint32_t where) {
  __syncthreads();
  int ok = 1;
  if (threadIdx.x == 0) {
    const uint32_t gen = ld_volatile_u32(sync + SY_BAR_GEN);
    __threadfence();
    const uint32_t prev = atomicAdd(sync + SY_BAR_COUNT, 1u);
    if (prev == gridDim.x - 1) {
      atomicExch(sync + SY_BAR_COUNT, 0u);
      __threadfence();
      st_release_u32(sync + SY_BAR_GEN, gen + 1);
    } else {
      const uint64_t t0 = globaltimer_ns();
      uint32_t spins = 0;
      while (ld_acquire_u32(sync + SY_BAR_GEN) == gen) {
        if ((++spins & 15u) == 0u) {
          if (error_set(sync)) { ok = 0; break; }
          if (globaltimer_ns() - t0 > timeout_ns) { set_error(sync, DEV_TIMEOUT_BARRIER, where); ok = 0; break; }
        }
        __nanosleep(64);
      }
    }
    __threadfence();
    if (ok && error_set(sync)) ok = 0;
  }
  return __syncthreads_and(ok) != 0;
}

// Bounded wait on an mbarrier phase; false on timeout or a recorded error.
__device__ bool wait_mbar(uint64_t* bar, uint32_t parity, uint32_t* sync, uint64_t timeout_ns,
                          uint32_t code, uint32_t info) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  uint32_t spins = 0;
  while (!mbar_try_wait(bar, parity)) {
    if ((++spins & 63u) == 0u) {
      if (error_set(sync)) return false;
      if (globaltimer_ns() - t0 > timeout_ns) { set_error(sync, code, info); return false; }
    }
  }
  return true;
}

__device__ __forceinline__ unsigned long long pclock(bool on) { return on ? clock64() : 0ull; }

__device__ __forceinline__ float pow2f(int e) {  // 2^e for e in [-126, 127]
  return __uint_as_float((uint32_t)(e + 127) << 23);
}

// ---- phase A: activations in f16 fragments, router partial logits -----------------------
// Each token's x is scaled by 2^-px so that max|x| lies in [2^14, 2^15); then
// every bf16 value is exact in f16 unless it is below max|x| * 2^-28.  The
// 32-element blocks are stored in the mma B-fragment order (see chunk_mma).
__device__ void phase_prepare(const EngineParams& p, const LayerPtrs& lp, const __nv_bfloat16* x,
                              int layer, uint8_t* smem, uint64_t* stamp) {
  const int T = p.T, H = p.H, E = p.E;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int64_t gt = (int64_t)blockIdx.x * THREADS + threadIdx.x;
  const int64_t gs = (int64_t)gridDim.x * THREADS;
  const int64_t wg = (int64_t)blockIdx.x * WARPS + warp, ws = (int64_t)gridDim.x * WARPS;
  // one CTA per token: CTA-wide max, then every thread converts whole blocks
  float* red = tables(smem).red;
  for (int64_t t = blockIdx.x; t < T; t += gridDim.x) {
    const __nv_bfloat16* xr = x + t * H;
    float m = 0.f;
    for (int h = threadIdx.x * 8; h < H; h += THREADS * 8) {
      const uint4 v = *reinterpret_cast<const uint4*>(xr + h);
      const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        m = fmaxf(m, fabsf(__uint_as_float(u[i] << 16)));
        m = fmaxf(m, fabsf(__uint_as_float(u[i] & 0xFFFF0000u)));
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(FULL, m, o));
    __syncthreads();
    if (lane == 0) red[warp] = m;
    __syncthreads();
#pragma unroll
    for (int w2 = 0; w2 < WARPS; ++w2) m = fmaxf(m, red[w2]);
    const int eb = (int)((__float_as_uint(m) >> 23) & 0xFF);
    int px = m > 0.f ? eb - 127 - 14 : 0;
    px = max(px, -126);
    const float inv = pow2f(-px);
    if (threadIdx.x == 0) p.pxf[t] = pow2f(px);
    for (int b = threadIdx.x; b < H / 32; b += THREADS) {
      const uint4* src = reinterpret_cast<const uint4*>(xr + b * 32);
      float v[32];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const uint4 q = src[i];
        const uint32_t u[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          v[i * 8 + 2 * k] = __uint_as_float(u[k] << 16) * inv;
          v[i * 8 + 2 * k + 1] = __uint_as_float(u[k] & 0xFFFF0000u) * inv;
        }
      }
      uint4* dst = reinterpret_cast<uint4*>(p.xh + (t * H + b * 32) * 2);
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        __half2 h0 = __floats2half2_rn(v[2 * c], v[2 * c + 1]);
        __half2 h1 = __floats2half2_rn(v[2 * c + 8], v[2 * c + 9]);
        __half2 h2 = __floats2half2_rn(v[16 + 2 * c], v[17 + 2 * c]);
        __half2 h3 = __floats2half2_rn(v[24 + 2 * c], v[25 + 2 * c]);
        dst[c] = make_uint4(*reinterpret_cast<uint32_t*>(&h0), *reinterpret_cast<uint32_t*>(&h1),
                            *reinterpret_cast<uint32_t*>(&h2), *reinterpret_cast<uint32_t*>(&h3));
      }
    }
  }
  if (stamp) stamp[0] = globaltimer_ns();
  if (p.layer_io) {
    const int64_t n8 = (int64_t)T * H / 8;
    const uint4* s8 = reinterpret_cast<const uint4*>(x);
    uint4* d8 = reinterpret_cast<uint4*>(p.layer_io + (int64_t)layer * T * H);
    for (int64_t i = gt; i < n8; i += gs) d8[i] = s8[i];
  }
  // per-layer resets of the stream's counters (used only after the next barrier)
  const int umax = max_units(E, p.TK);
  if (gt == 0) p.sync[SY_JOBS] = 0u;
  for (int64_t u = gt; u < umax; u += gs) p.sync[SY_READY + u] = 0u;

  // partial logits[hs][t][e] = sum over the hs-th H part of x[t][h] * Wr[e][h];
  // bf16 * fp32 products are exact in fp64 and the sums are fp64.  A token
  // block that fits in the (idle) stage ring is staged there first, so that
  // only the router weights come from L2.
  const __nv_bfloat16* xr = x;
  if ((int64_t)T * H * 2 <= (int64_t)NSLOT * SLOT_BYTES) {
    uint4* d = reinterpret_cast<uint4*>(ring_slot(smem, 0));
    const uint4* s8 = reinterpret_cast<const uint4*>(x);
    for (int64_t i = threadIdx.x; i < (int64_t)T * H / 8; i += THREADS) d[i] = s8[i];
    __syncthreads();
    xr = reinterpret_cast<const __nv_bfloat16*>(ring_slot(smem, 0));
  }
  const int HS = p.HS, hpart = H / HS;
  const int nchunk = (T + 7) / 8;
  const int64_t njobs = (int64_t)E * HS * nchunk;
  for (int64_t job = wg; job < njobs; job += ws) {
    const int e = (int)(job % E);
    const int hs = (int)((job / E) % HS);
    const int t0 = (int)(job / ((int64_t)E * HS)) * 8;
    const int nt = min(8, T - t0);
    double acc[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[j] = 0.0;
    const float4* wr = reinterpret_cast<const float4*>(lp.router_w + (int64_t)e * H + hs * hpart);
#pragma unroll 8
    for (int h4 = lane; h4 < hpart / 4; h4 += 32) {
      const float4 w4 = __ldg(wr + h4);
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        if (j < nt) {
          const uint2 xb = *reinterpret_cast<const uint2*>(xr + (int64_t)(t0 + j) * H + hs * hpart + h4 * 4);
          acc[j] = fma((double)__uint_as_float(xb.x << 16), (double)w4.x, acc[j]);
          acc[j] = fma((double)__uint_as_float(xb.x & 0xFFFF0000u), (double)w4.y, acc[j]);
          acc[j] = fma((double)__uint_as_float(xb.y << 16), (double)w4.z, acc[j]);
          acc[j] = fma((double)__uint_as_float(xb.y & 0xFFFF0000u), (double)w4.w, acc[j]);
        }
      }
    }
#pragma unroll
    for (int j = 0; j < 8; ++j) {
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) acc[j] += __shfl_xor_sync(FULL, acc[j], o);
    }
    if (lane == 0) {
#pragma unroll
      for (int j = 0; j < 8; ++j)
        if (j < nt) p.logits[((int64_t)hs * T + t0 + j) * E + e] = acc[j];
    }
  }
  if (stamp) stamp[1] = globaltimer_ns();
}

// ---- phase B: top-k, weights, permutation ------------------------------------------------
__device__ __forceinline__ uint64_t order_key(double v) {
  const uint64_t b = (uint64_t)__double_as_longlong(v);
  return (b >> 63) ? ~b : (b | 0x8000000000000000ull);
}
__device__ __forceinline__ double key_value(uint64_t k) {
  const uint64_t b = (k >> 63) ? (k & 0x7FFFFFFFFFFFFFFFull) : ~k;
  return __longlong_as_double((long long)b);
}

// One warp: logits of token t (partials summed in order, plus bias), the K
// largest (descending, ties to the lower expert), weights exp(l - lmax) / sum
// over the K.  Lane r < K writes slot r.  Each lane holds experts lane + 32 i
// (i < PER) as order-preserving 64-bit keys, sorts them once (descending, the
// lower expert first on equal keys), and each of the K rounds takes the
// warp-wide maximum of the lanes' heads; the winning lane drops its head.
template <int PER>
__device__ void topk_row_n(const EngineParams& p, const float* bias, int t, int32_t* out_idx,
                           float* out_w) {
  const int lane = threadIdx.x & 31;
  const int E = p.E, K = p.K;
  uint64_t key[PER];
  int ix[PER];
#pragma unroll
  for (int i = 0; i < PER; ++i) {
    const int e = lane + 32 * i;
    ix[i] = i;
    if (e < E) {
      double part[MAX_HSPLIT];
#pragma unroll
      for (int hs = 0; hs < MAX_HSPLIT; ++hs)
        part[hs] = hs < p.HS ? p.logits[((int64_t)hs * p.T + t) * E + e] : 0.0;
      double l = 0.0;
#pragma unroll
      for (int hs = 0; hs < MAX_HSPLIT; ++hs) l += part[hs];
      if (bias) l += (double)bias[e];
      key[i] = order_key(l);
    } else {
      key[i] = 0ull;
    }
  }
  // odd-even transposition sort, descending; on equal keys the lower index first
#pragma unroll
  for (int r = 0; r < PER; ++r) {
#pragma unroll
    for (int i = r & 1; i + 1 < PER; i += 2) {
      const bool sw = key[i + 1] > key[i] || (key[i + 1] == key[i] && ix[i + 1] < ix[i]);
      const uint64_t k0 = key[i], k1 = key[i + 1];
      const int i0 = ix[i], i1 = ix[i + 1];
      key[i] = sw ? k1 : k0; key[i + 1] = sw ? k0 : k1;
      ix[i] = sw ? i1 : i0; ix[i + 1] = sw ? i0 : i1;
    }
  }
  int my_e = -1;
  double my_l = 0.0, lmax = 0.0;
  for (int r = 0; r < K; ++r) {
    const uint64_t best = key[0];
    const uint32_t hi = __reduce_max_sync(FULL, (uint32_t)(best >> 32));
    const uint32_t lo = __reduce_max_sync(FULL, (uint32_t)(best >> 32) == hi ? (uint32_t)best : 0u);
    const uint64_t top = ((uint64_t)hi << 32) | lo;
    const int ehead = lane + 32 * ix[0];
    const uint32_t m = __reduce_max_sync(FULL, best == top ? (65536u - (uint32_t)ehead) : 0u);
    const int esel = (int)(65536u - m);
    if (esel == ehead) {  // the winning lane drops its head
#pragma unroll
      for (int i = 0; i + 1 < PER; ++i) { key[i] = key[i + 1]; ix[i] = ix[i + 1]; }
      key[PER - 1] = 0ull;
    }
    const double v = key_value(top);
    if (r == 0) lmax = v;
    if (lane == r) { my_e = esel; my_l = v; }
  }
  const double ex = lane < K ? exp(my_l - lmax) : 0.0;
  double sum = ex;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(FULL, sum, o);
  if (lane < K) { out_idx[lane] = my_e; out_w[lane] = (float)(ex / sum); }
}

__device__ __forceinline__ void topk_row(const EngineParams& p, const float* bias, int t,
                                         int32_t* out_idx, float* out_w) {
  if (p.E <= 128) topk_row_n<4>(p, bias, t, out_idx, out_w);
  else if (p.E <= 256) topk_row_n<8>(p, bias, t, out_idx, out_w);
  else topk_row_n<16>(p, bias, t, out_idx, out_w);
}

// Exclusive scan of n <= 512 ints in shared memory by one warp (in place);
// the total goes to *total.
__device__ void warp_exclusive_scan(int32_t* a, int n, int32_t* total) {
  const int lane = threadIdx.x & 31;
  constexpr int PER = 16;
  int32_t v[PER];
  int32_t s = 0;
#pragma unroll
  for (int i = 0; i < PER; ++i) {
    const int k = lane * PER + i;
    v[i] = k < n ? a[k] : 0;
    s += v[i];
  }
  int32_t incl = s;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int32_t t = __shfl_up_sync(FULL, incl, o);
    if (lane >= o) incl += t;
  }
  int32_t run = incl - s;
#pragma unroll
  for (int i = 0; i < PER; ++i) {
    const int k = lane * PER + i;
    if (k < n) a[k] = run;
    run += v[i];
  }
  if (lane == 31) *total = incl;
}

// Unit tables from per-expert counts/offsets: gate/up units of <= NT_MAX
// consecutive positions of one expert's segment, down units of <= ND_MAX
// (each inside one gate/up unit).  scratch: 2*E ints.
__device__ void build_units(const int32_t* counts, const int32_t* offsets, int E, int32_t* scratch,
                            int32_t* units, int32_t* dunits, int32_t* n_units, int32_t* n_dunits) {
  const int warp = threadIdx.x >> 5;
  int32_t* ubase = scratch;
  int32_t* dbase = scratch + E;
  for (int x = threadIdx.x; x < E; x += THREADS) {
    ubase[x] = (counts[x] + NT_MAX - 1) / NT_MAX;
    dbase[x] = (counts[x] + ND_MAX - 1) / ND_MAX;
  }
  __syncthreads();
  if (warp == 0) warp_exclusive_scan(ubase, E, n_units);
  if (warp == 1) warp_exclusive_scan(dbase, E, n_dunits);
  __syncthreads();
  for (int x = threadIdx.x; x < E; x += THREADS) {
    const int c = counts[x];
    for (int s = 0; s * NT_MAX < c; ++s) {
      int32_t* u = units + (int64_t)(ubase[x] + s) * 4;
      u[0] = x; u[1] = offsets[x] + s * NT_MAX; u[2] = min(NT_MAX, c - s * NT_MAX); u[3] = 0;
    }
    for (int s = 0; s * ND_MAX < c; ++s) {
      int32_t* u = dunits + (int64_t)(dbase[x] + s) * 4;
      u[0] = x; u[1] = offsets[x] + s * ND_MAX; u[2] = min(ND_MAX, c - s * ND_MAX);
      u[3] = ubase[x] + (s * ND_MAX) / NT_MAX;
    }
  }
}

// Small T*K: every CTA routes all tokens itself (no barrier); CTA 0 also writes
// the maps to global memory.
__device__ void phase_route_small(const EngineParams& p, const LayerPtrs& lp, uint8_t* smem,
                                  uint64_t* stamp) {
  CtaTables& tb = tables(smem);
  const int T = p.T, E = p.E, K = p.K, TK = p.TK;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  for (int t = warp; t < T; t += WARPS) topk_row(p, lp.router_b, t, tb.idx + t * K, tb.w + t * K);
  for (int t = threadIdx.x; t < T; t += THREADS) tb.pxf[t] = p.pxf[t];
  if (stamp) *stamp = globaltimer_ns();
  int32_t* hist = reinterpret_cast<int32_t*>(ring_slot(smem, 0));  // [WARPS][E] scratch
  for (int i = threadIdx.x; i < WARPS * E; i += THREADS) hist[i] = 0;
  __syncthreads();
  const int pr = threadIdx.x;  // TK <= SMALL_PAIRS <= THREADS: one pair per thread
  const bool valid = pr < TK;
  const int e = valid ? tb.idx[pr] : -1 - lane;
  const uint32_t peers = __match_any_sync(FULL, e);
  const int rank_w = __popc(peers & ((1u << lane) - 1u));
  if (valid && lane == __ffs(peers) - 1) hist[warp * E + e] = __popc(peers);
  __syncthreads();
  for (int x = threadIdx.x; x < E; x += THREADS) {
    int32_t c = 0;
    for (int w = 0; w < WARPS; ++w) c += hist[w * E + x];
    tb.counts[x] = c;
    tb.offsets[x] = c;
  }
  __syncthreads();
  if (warp == 0) warp_exclusive_scan(tb.offsets, E, tb.offsets + E);
  __syncthreads();
  if (valid) {
    int32_t before = 0;
    for (int w = 0; w < warp; ++w) before += hist[w * E + e];
    const int pos = tb.offsets[e] + before + rank_w;
    tb.perm[pos] = pr;
    tb.inv[pr] = pos;
    tb.tokpos[pos] = pr / K;
    tb.wpos[pos] = tb.w[pr];
  }
  __syncthreads();
  build_units(tb.counts, tb.offsets, E, hist, tb.units, tb.dunits, &tb.n_units, &tb.n_dunits);
  __syncthreads();
  if (blockIdx.x == 0) {
    for (int i = threadIdx.x; i < TK; i += THREADS) {
      p.idx[i] = tb.idx[i]; p.wts[i] = tb.w[i]; p.perm[i] = tb.perm[i]; p.inv[i] = tb.inv[i];
    }
    for (int i = threadIdx.x; i < E; i += THREADS) p.counts[i] = tb.counts[i];
    for (int i = threadIdx.x; i <= E; i += THREADS) p.offsets[i] = tb.offsets[i];
  }
}

// Large T*K, step 1: top-k of every token, distributed over all warps.
__device__ void phase_topk_large(const EngineParams& p, const LayerPtrs& lp) {
  const int warp = threadIdx.x >> 5;
  const int64_t wg = (int64_t)blockIdx.x * WARPS + warp, ws = (int64_t)gridDim.x * WARPS;
  for (int64_t t = wg; t < p.T; t += ws)
    topk_row(p, lp.router_b, (int)t, p.idx + t * p.K, p.wts + t * p.K);
}

// Large T*K, step 2: counts/offsets in every CTA (shared-memory histogram),
// unit table by CTA 0, stable positions by one warp per expert (ballot scan).
__device__ void phase_permute_large(const EngineParams& p, uint8_t* smem) {
  CtaTables& tb = tables(smem);
  const int E = p.E, K = p.K, TK = p.TK;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  for (int i = threadIdx.x; i < E; i += THREADS) tb.counts[i] = 0;
  __syncthreads();
  for (int i = threadIdx.x; i < TK; i += THREADS) atomicAdd(&tb.counts[p.idx[i]], 1);
  __syncthreads();
  for (int i = threadIdx.x; i < E; i += THREADS) tb.offsets[i] = tb.counts[i];
  __syncthreads();
  if (warp == 0) warp_exclusive_scan(tb.offsets, E, tb.offsets + E);
  __syncthreads();
  if (blockIdx.x == 0) {
    int32_t* scratch = reinterpret_cast<int32_t*>(ring_slot(smem, 0));
    build_units(tb.counts, tb.offsets, E, scratch, p.units, p.dunits, &tb.n_units, &tb.n_dunits);
    for (int i = threadIdx.x; i < E; i += THREADS) p.counts[i] = tb.counts[i];
    for (int i = threadIdx.x; i <= E; i += THREADS) p.offsets[i] = tb.offsets[i];
    if (threadIdx.x == 0) { p.n_units[0] = tb.n_units; p.n_units[1] = tb.n_dunits; }
  }
  const int64_t wg = (int64_t)blockIdx.x * WARPS + warp, ws = (int64_t)gridDim.x * WARPS;
  for (int64_t x = wg; x < E; x += ws) {
    int run = tb.offsets[x];
    for (int base = 0; base < TK; base += 32) {
      const int pr = base + lane;
      const bool hit = pr < TK && p.idx[pr] == (int)x;
      const uint32_t b = __ballot_sync(FULL, hit);
      if (hit) {
        const int pos = run + __popc(b & ((1u << lane) - 1u));
        p.perm[pos] = pr; p.inv[pr] = pos; p.tokpos[pos] = pr / K; p.wpos[pos] = p.wts[pr];
      }
      run += __popc(b);
    }
  }
}

// ---- phase C: the MXFP4 weight stream on tensor cores --------------------------------------
// E8M0 byte B of a word -> 2^(byte-127) as fp32; byte 0 gives 2^-127 exactly,
// byte 255 gives +inf (its blocks hold zero codes, so the product is NaN).
template <int B>
__device__ __forceinline__ float e8m0_byte(uint32_t w) {
  uint32_t bits;
  if constexpr (B == 3) bits = (w >> 1) & 0x7F800000u;
  else bits = (w << (23 - 8 * B)) & 0x7F800000u;
  return __uint_as_float(max(bits, 0x00400000u));
}

// One K chunk (4 MX blocks) of a 64-row job for this warp:
//   acc[t][i] += sum over blocks b of 2^s(row, b) [* 2^q(col, b)] * (A_b B_b)
// A = the chunk's E2M1 codes of tile t as f16 fragments (from the ring slot
// st), B = the lane's activation fragments bfr[b] (loaded by the caller).
// Gate/up: the 8 columns are tokens (x in f16, scaled per token).  Down:
// columns 2j, 2j+1 are the hi and lo f16 halves of pair j's SwiGLU output,
// scaled per (pair, block) by 2^q, q4 holding this lane's pair's 4 exponents.
template <bool ISD>
__device__ __forceinline__ void chunk_mma(const uint8_t* st, int lane, const uint4 (&bfr)[KB],
                                          uint32_t q4, float (&acc)[4][4]) {
  const int g = lane >> 2;
  uint32_t sw0[4], sw1[4];
#pragma unroll
  for (int t = 0; t < 4; ++t) {
    sw0[t] = *reinterpret_cast<const uint32_t*>(st + STAGE_CODE_BYTES + (t * 16 + g) * KB);
    sw1[t] = *reinterpret_cast<const uint32_t*>(st + STAGE_CODE_BYTES + (t * 16 + g + 8) * KB);
  }
#pragma unroll
  for (int b = 0; b < KB; ++b) {
    const uint4 qa = *reinterpret_cast<const uint4*>(st + ((b * 2 + 0) * 32 + lane) * 16);
    const uint4 qb = *reinterpret_cast<const uint4*>(st + ((b * 2 + 1) * 32 + lane) * 16);
    const uint4 bf = bfr[b];
    const float qf = ISD ? pow2f((int)(int8_t)((q4 >> (8 * b)) & 0xFFu)) : 1.f;
    const uint32_t wd[8] = {qa.x, qa.y, qa.z, qa.w, qb.x, qb.y, qb.z, qb.w};
#pragma unroll
    for (int t = 0; t < 4; ++t) {
      uint32_t a0[4], a1[4];
      e2m1x8_to_f16x2x4(wd[2 * t], a0);
      e2m1x8_to_f16x2x4(wd[2 * t + 1], a1);
      float ct[4] = {0.f, 0.f, 0.f, 0.f};
      mma_f16_16816(ct, a0, bf.x, bf.y);
      mma_f16_16816(ct, a1, bf.z, bf.w);
      float f0, f1;
      if (b == 0) { f0 = e8m0_byte<0>(sw0[t]); f1 = e8m0_byte<0>(sw1[t]); }
      else if (b == 1) { f0 = e8m0_byte<1>(sw0[t]); f1 = e8m0_byte<1>(sw1[t]); }
      else if (b == 2) { f0 = e8m0_byte<2>(sw0[t]); f1 = e8m0_byte<2>(sw1[t]); }
      else { f0 = e8m0_byte<3>(sw0[t]); f1 = e8m0_byte<3>(sw1[t]); }
      if (ISD) { f0 *= qf; f1 *= qf; }
      acc[t][0] = fmaf(ct[0], f0, acc[t][0]);
      acc[t][1] = fmaf(ct[1], f0, acc[t][1]);
      acc[t][2] = fmaf(ct[2], f1, acc[t][2]);
      acc[t][3] = fmaf(ct[3], f1, acc[t][3]);
    }
  }
}

struct StreamCtx {
  const int32_t* units;   // gate/up units
  const int32_t* dunits;  // down units
  const int32_t* tokpos;
  const float* wpos;
  const float* pxf;       // per-token activation scale 2^px
  int n_units, n_dunits;
};

// Producer warp: jobs -> queue entries -> stages into the ring.  Gate/up jobs
// (unit, 32-row block of I) come first in unit order, then down jobs (down
// unit, 64-row block of H); a down job waits until its gate/up unit's
// SwiGLU output is complete.
__device__ void stream_producer(const EngineParams& p, const LayerPtrs& lp, uint8_t* smem,
                                const StreamCtx& cx, uint32_t& seq, int32_t& qk) {
  const int lane = threadIdx.x & 31;
  JobEntry* jq = job_queue(smem);
  uint32_t* ready = p.sync + SY_READY;
  const int gub = p.I / (STAGE_ROWS / 2), db = p.H / STAGE_ROWS;
  const int64_t n_gu = (int64_t)cx.n_units * gub, n_all = n_gu + (int64_t)cx.n_dunits * db;
  const int nc_gu = p.H / KC, nc_d = p.I / KC;
  const uint32_t seq_start = seq;
  bool ok = true;
  unsigned long long t_empty = 0, t_ready = 0;
  const unsigned long long t_begin = clock64();
  fence_proxy_async_global();
  long long next = 0;
  if (lane == 0) next = atomicAdd(p.sync + SY_JOBS, 1u);
  for (;;) {
    const int64_t j = __shfl_sync(FULL, next, 0);
    if (j >= n_all || !ok) {
      if (lane == 0) {
        JobEntry* en = jq + (qk % JQ);
        en->job = -1; en->s0 = (int32_t)seq; en->nc = 0;
        __threadfence_block();
        *reinterpret_cast<volatile int32_t*>(&en->flag) = qk + 1;
      }
      ++qk;
      break;
    }
    if (lane == 0) next = atomicAdd(p.sync + SY_JOBS, 1u);  // prefetch the following job
    const bool isD = j >= n_gu;
    const int64_t jj = isD ? j - n_gu : j;
    const int per = isD ? db : gub;
    const int u = (int)(jj / per), rb = (int)(jj % per);
    const int4 ur = *reinterpret_cast<const int4*>((isD ? cx.dunits : cx.units) + (int64_t)u * 4);
    const int e = ur.x, pos0 = ur.y, nt = ur.z;
    const int nc = isD ? nc_d : nc_gu;
    if (isD) {  // the down stages read the SwiGLU output: wait for the gate/up unit
      const int gu = ur.w;
      const uint32_t need = (uint32_t)gub * (uint32_t)cx.units[(int64_t)gu * 4 + 2];
      const unsigned long long tr0 = clock64();
      if (ld_acquire_u32(ready + gu) < need) {
        const uint64_t t0 = globaltimer_ns();
        uint32_t spins = 0;
        while (ld_acquire_u32(ready + gu) < need) {
          if ((++spins & 15u) == 0u) {
            if (error_set(p.sync)) { ok = false; break; }
            if (globaltimer_ns() - t0 > p.timeout_ns) { set_error(p.sync, DEV_TIMEOUT_READY, gu); ok = false; break; }
          }
          __nanosleep(100);
        }
      }
      t_ready += clock64() - tr0;
      if (!ok) continue;  // publishes the end entry
    }
    // publish the job (after the readiness acquire, so the consumers' reads of
    // the SwiGLU output are ordered after it)
    if (lane == 0) {
      JobEntry* en = jq + (qk % JQ);
      en->job = (int32_t)j; en->s0 = (int32_t)seq; en->nc = nc; en->unit = u; en->rb = rb;
      en->isD = isD; en->e = e; en->pos0 = pos0; en->nt = nt;
      __threadfence_block();
      *reinterpret_cast<volatile int32_t*>(&en->flag) = qk + 1;
    }
    ++qk;
    const uint8_t* wbase = isD ? lp.w_d + ((int64_t)e * db + rb) * nc * STAGE_W_BYTES
                               : lp.w_gu + ((int64_t)e * gub + rb) * nc * STAGE_W_BYTES;
    // Stages are issued in batches: successive 1-D bulk copies issued by one
    // warp instruction each are serialised, while the copies of one
    // instruction (one per lane) proceed in parallel.
    for (int c0 = 0; c0 < nc && ok; c0 += PRODUCER_BATCH) {
      const int nb = min(PRODUCER_BATCH, nc - c0);
      const unsigned long long te0 = clock64();
      bool bad = false;
      const uint32_t s = seq + lane;
      const int slot = (int)(s % NSLOT);
      if (lane < nb && s >= (uint32_t)NSLOT)  // wait until the slot is free
        bad = !wait_mbar(empty_bar(smem, slot), ((s / NSLOT) + 1) & 1u, p.sync, p.timeout_ns,
                         DEV_TIMEOUT_PIPE, s);
      if (__any_sync(FULL, bad)) { ok = false; break; }
      t_empty += clock64() - te0;
      if (lane < nb) {
        mbar_arrive_expect_tx(full_bar(smem, slot), STAGE_W_BYTES);
        bulk_g2s(ring_slot(smem, slot), wbase + (int64_t)(c0 + lane) * STAGE_W_BYTES, STAGE_W_BYTES,
                 full_bar(smem, slot));
      }
      seq += nb;
    }
  }
  if (p.prof && lane == 0) {
    atomicAdd(p.prof + PF_PROD_EMPTY, t_empty);
    atomicAdd(p.prof + PF_PROD_READY, t_ready);
    atomicAdd(p.prof + PF_PROD_TOTAL, clock64() - t_begin);
    atomicAdd(p.prof + PF_STAGES, (unsigned long long)(seq - seq_start));
  }
  // let every issued copy land before the ring is reused or the CTA exits
  const uint32_t issued = seq - seq_start;
  const uint32_t n = issued < (uint32_t)NSLOT ? issued : (uint32_t)NSLOT;
  for (uint32_t s = seq - n; s != seq; ++s) {
    const uint64_t t0 = globaltimer_ns();
    while (!mbar_try_wait(full_bar(smem, (int)(s % NSLOT)), (s / NSLOT) & 1u)) {
      if (globaltimer_ns() - t0 > p.timeout_ns) break;
    }
  }
}

// Consumer warps: chunks of every job, partial sums, reduction, epilogues.
__device__ void stream_consumer(const EngineParams& p, uint8_t* smem, const StreamCtx& cx,
                                int32_t& qk) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  const int g = lane >> 2, c = lane & 3;
  JobEntry* jq = job_queue(smem);
  uint32_t* ready = p.sync + SY_READY;
  bool poison = false;
  const bool prof = p.prof != nullptr;
  unsigned long long t_full = 0, t_mma = 0, t_bar = 0, t_epi = 0, t_queue = 0, n_jobs = 0;
  const unsigned long long t_begin = pclock(prof);
  // A gate/up epilogue's readiness signal (release fence + counter add) is
  // deferred until after this warp's next chunk, when its stores have landed
  // and the fence is cheap; it is flushed at once whenever the warp would wait
  // for the producer (which may itself wait for that signal).
  int pend_u = -1;
  auto flush_ready = [&]() {
    if (pend_u >= 0) {
      if (lane == 0) {
        __threadfence();
        red_release_add_u32(ready + pend_u, 1u);
      }
      pend_u = -1;
    }
  };
  for (;;) {
    JobEntry* en = jq + (qk % JQ);
    const unsigned long long tq0 = pclock(prof);
    // the producer publishes the entry (bounded wait; the producer's own waits
    // are bounded by the same timeout, after which it publishes an end entry)
    if (*reinterpret_cast<volatile int32_t*>(&en->flag) != qk + 1) {
      flush_ready();
      const uint64_t t0 = globaltimer_ns();
      while (*reinterpret_cast<volatile int32_t*>(&en->flag) != qk + 1) {
        if (globaltimer_ns() - t0 > 2 * p.timeout_ns) { set_error(p.sync, DEV_TIMEOUT_QUEUE, qk); return; }
        __nanosleep(32);
      }
    }
    const int job = *reinterpret_cast<volatile int32_t*>(&en->job);
    t_queue += pclock(prof) - tq0;
    if (job < 0) { ++qk; break; }
    ++n_jobs;
    const int s0 = en->s0, nc = en->nc, u = en->unit, rb = en->rb, isD = en->isD;
    const int pos0 = en->pos0, nt = en->nt;
    const int buf = qk & 1;
    // order the reads of activations (written by other CTAs, seen through the
    // producer's acquire) after the queue entry
    __threadfence_block();
    // this lane's activation fragments: base address of chunk 0 and the step
    // between K chunks.  Gate/up: column g is token g (columns >= nt repeat
    // token 0 and are ignored).  Down: column g is the hi (g even) or lo half
    // of pair g/2, and the lane's output pair c supplies the block exponents.
    const uint8_t* fbase;
    const uint8_t* qbase = nullptr;
    int64_t cstep;
    int bstep;
    if (!isD) {
      const int tok = cx.tokpos[pos0 + (g < nt ? g : 0)];
      fbase = p.xh + (int64_t)tok * p.H * 2 + c * 16;
      cstep = (int64_t)KC * 2;
      bstep = 64;
    } else {
      const int pj = (g >> 1) < nt ? (g >> 1) : 0;
      fbase = p.a16 + (int64_t)(pos0 + pj) * A16_CHUNK_BYTES + A16_HDR + (g & 1) * 64 + c * 16;
      qbase = p.a16 + (int64_t)(pos0 + (c < nt ? c : 0)) * A16_CHUNK_BYTES;
      cstep = (int64_t)p.TK * A16_CHUNK_BYTES;
      bstep = 128;
    }
    float acc[4][4];
#pragma unroll
    for (int t = 0; t < 4; ++t)
#pragma unroll
      for (int i = 0; i < 4; ++i) acc[t][i] = 0.f;
    uint4 fcur[KB];
    uint32_t qcur = 0;
    if (w < nc) {
#pragma unroll
      for (int b = 0; b < KB; ++b) fcur[b] = ld_cg_v4(fbase + w * cstep + b * bstep);
      if (isD) qcur = ld_cg_u32(qbase + w * cstep);
    }
    for (int cc = w; cc < nc; cc += NCW) {
      // fetch the next chunk's fragments while this one computes
      uint4 fnext[KB];
      uint32_t qnext = 0;
      const int cn = cc + NCW < nc ? cc + NCW : cc;
#pragma unroll
      for (int b = 0; b < KB; ++b) fnext[b] = ld_cg_v4(fbase + cn * cstep + b * bstep);
      if (isD) qnext = ld_cg_u32(qbase + cn * cstep);
      const uint32_t s = (uint32_t)s0 + cc;
      const int slot = (int)(s % NSLOT);
      const unsigned long long tf0 = pclock(prof);
      if (!poison &&
          !wait_mbar(full_bar(smem, slot), (s / NSLOT) & 1u, p.sync, p.timeout_ns, DEV_TIMEOUT_PIPE, s))
        poison = true;
      const unsigned long long tm0 = pclock(prof);
      t_full += tm0 - tf0;
      if (!poison) {
        const uint8_t* st = ring_slot(smem, slot);
        if (!isD) chunk_mma<false>(st, lane, fcur, 0u, acc);
        else chunk_mma<true>(st, lane, fcur, qcur, acc);
      }
      t_mma += pclock(prof) - tm0;
      __syncwarp();
      if (lane == 0) mbar_arrive(empty_bar(smem, slot));
      flush_ready();
#pragma unroll
      for (int b = 0; b < KB; ++b) fcur[b] = fnext[b];
      qcur = qnext;
    }
    // deposit this warp's partial sums: part[w][col][row]
    float* pb = part_buf(smem, buf) + (size_t)w * PART_COLS * PART_LD;
    if (w < nc) {
#pragma unroll
      for (int t = 0; t < 4; ++t)
#pragma unroll
        for (int i = 0; i < 4; ++i) pb[(2 * c + (i & 1)) * PART_LD + t * 16 + g + (i >> 1) * 8] = acc[t][i];
    }
    const unsigned long long tb0 = pclock(prof);
    named_barrier(1 + buf, NCW * 32);
    const unsigned long long te0 = pclock(prof);
    t_bar += te0 - tb0;
    const int nw = nc < NCW ? nc : NCW;
    const float* pall = part_buf(smem, buf);
    // the epilogue of column j runs on warp (j + qk) % NCW: the duty rotates
    const int j = (w + NCW - (qk % NCW)) % NCW;
    if (!poison && j < nt) {
      if (!isD) {  // gate/up epilogue: token column j, lane = intermediate row i0 + lane
        const float px = cx.pxf[cx.tokpos[pos0 + j]];
        float gs = 0.f, us = 0.f;
        for (int ww = 0; ww < nw; ++ww) {
          gs += pall[((size_t)ww * PART_COLS + j) * PART_LD + lane];
          us += pall[((size_t)ww * PART_COLS + j) * PART_LD + 32 + lane];
        }
        const float gv = gs * px, uv = us * px;
        const float a = gv / (1.0f + expf(-gv)) * uv;
        float am = fabsf(a);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) am = fmaxf(am, __shfl_xor_sync(FULL, am, o));
        const int eb = (int)((__float_as_uint(am) >> 23) & 0xFF);
        int q = am > 0.f ? eb - 127 - 14 : 0;
        q = max(q, -126);
        const float v = a * pow2f(-q);
        const __half hi = __float2half_rn(v);
        const __half lo = __float2half_rn(v - __half2float(hi));
        const int i0 = rb * (STAGE_ROWS / 2);
        uint8_t* base = p.a16 + ((int64_t)(i0 / KC) * p.TK + pos0 + j) * A16_CHUNK_BYTES;
        const int bi = (i0 % KC) / 32;
        const int kk = lane & 15;
        const int off = A16_HDR + bi * 128 + ((kk & 7) >> 1) * 16 +
                        ((lane >> 4) * 4 + ((kk >> 3) << 1) + (kk & 1)) * 2;
        *reinterpret_cast<__half*>(base + off) = hi;
        *reinterpret_cast<__half*>(base + off + 64) = lo;
        if (lane == 0) base[bi] = (uint8_t)(int8_t)q;
        __syncwarp();
        flush_ready();  // a previous job's signal, if still pending
        pend_u = u;
      } else {  // down epilogue: pair j, lane = rows h0 + lane and h0 + 32 + lane
        const float wp = cx.wpos[pos0 + j];
        const int h0 = rb * STAGE_ROWS;
#pragma unroll
        for (int r2 = 0; r2 < 2; ++r2) {
          const int r = lane + 32 * r2;
          float y = 0.f;
          for (int ww = 0; ww < nw; ++ww) {
            const float* pw = pall + (size_t)ww * PART_COLS * PART_LD;
            y += pw[(2 * j) * PART_LD + r] + pw[(2 * j + 1) * PART_LD + r];
          }
          p.ypair[(int64_t)(pos0 + j) * p.H + h0 + r] = y * wp;
        }
      }
    }
    t_epi += pclock(prof) - te0;
    ++qk;
  }
  flush_ready();
  if (p.prof && lane == 0) {
    atomicAdd(p.prof + PF_CONS_FULL, t_full);
    atomicAdd(p.prof + PF_CONS_MMA, t_mma);
    atomicAdd(p.prof + PF_CONS_BAR, t_bar);
    atomicAdd(p.prof + PF_CONS_EPI, t_epi);
    atomicAdd(p.prof + PF_CONS_QUEUE, t_queue);
    atomicAdd(p.prof + PF_CONS_TOTAL, pclock(prof) - t_begin);
    atomicAdd(p.prof + PF_JOBS, n_jobs);
  }
}

// ---- phase D: combine (+ RMSNorm) ------------------------------------------------------------
__device__ __forceinline__ void store_bf16x4(__nv_bfloat16* dst, float4 v) {
  __nv_bfloat162 a = __floats2bfloat162_rn(v.x, v.y), b = __floats2bfloat162_rn(v.z, v.w);
  uint2 u;
  u.x = *reinterpret_cast<uint32_t*>(&a);
  u.y = *reinterpret_cast<uint32_t*>(&b);
  *reinterpret_cast<uint2*>(dst) = u;
}

__device__ __forceinline__ float4 combine4(const EngineParams& p, const int32_t* inv, int t, int h) {
  float4 s = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int slot = 0; slot < p.K; ++slot) {
    const int pos = inv[t * p.K + slot];
    const float4 v = *reinterpret_cast<const float4*>(p.ypair + (int64_t)pos * p.H + h);
    s.x += v.x; s.y += v.y; s.z += v.z; s.w += v.w;
  }
  return s;
}

__device__ void phase_combine_out(const EngineParams& p, const int32_t* inv) {
  const int64_t gt = (int64_t)blockIdx.x * THREADS + threadIdx.x;
  const int64_t gs = (int64_t)gridDim.x * THREADS;
  const int H4 = p.H / 4;
  __nv_bfloat16* dump = p.layer_io ? p.layer_io + (int64_t)p.L * p.T * p.H : nullptr;
  for (int64_t g = gt; g < (int64_t)p.T * H4; g += gs) {
    const int t = (int)(g / H4), h = (int)(g % H4) * 4;
    const float4 s = combine4(p, inv, t, h);
    store_bf16x4(p.y_out + (int64_t)t * p.H + h, s);
    if (dump) store_bf16x4(dump + (int64_t)t * p.H + h, s);
  }
}

// Per token (one CTA each): y = bf16(combine); x_next = bf16(y / sqrt(mean(y^2) + eps)).
__device__ void phase_combine_rmsnorm(const EngineParams& p, const int32_t* inv, uint8_t* smem) {
  CtaTables& tb = tables(smem);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  constexpr int MAXV = (8192 / 4 + THREADS - 1) / THREADS;
  for (int t = blockIdx.x; t < p.T; t += gridDim.x) {
    float4 yv[MAXV];
    float ss = 0.f;
#pragma unroll
    for (int i = 0; i < MAXV; ++i) {
      const int h = (threadIdx.x + i * THREADS) * 4;
      if (h < p.H) {
        float4 s = combine4(p, inv, t, h);
        s.x = __bfloat162float(__float2bfloat16_rn(s.x));
        s.y = __bfloat162float(__float2bfloat16_rn(s.y));
        s.z = __bfloat162float(__float2bfloat16_rn(s.z));
        s.w = __bfloat162float(__float2bfloat16_rn(s.w));
        yv[i] = s;
        ss += s.x * s.x + s.y * s.y + s.z * s.z + s.w * s.w;
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(FULL, ss, o);
    if (lane == 0) tb.red[warp] = ss;
    __syncthreads();
    float tot = 0.f;
#pragma unroll
    for (int w = 0; w < WARPS; ++w) tot += tb.red[w];
    const float r = 1.0f / sqrtf(tot / (float)p.H + p.rms_eps);
#pragma unroll
    for (int i = 0; i < MAXV; ++i) {
      const int h = (threadIdx.x + i * THREADS) * 4;
      if (h < p.H) {
        const float4 s = yv[i];
        store_bf16x4(p.xnext + (int64_t)t * p.H + h, make_float4(s.x * r, s.y * r, s.z * r, s.w * r));
      }
    }
    __syncthreads();
  }
}

__global__ void __launch_bounds__(THREADS, 1) engine_kernel(const EngineParams p) {
  extern __shared__ __align__(128) uint8_t smem[];
  const int warp = threadIdx.x >> 5;
  if (threadIdx.x == 0) {
    for (int i = 0; i < NSLOT; ++i) {
      mbar_init(full_bar(smem, i), 1);
      mbar_init(empty_bar(smem, i), 1);
    }
    fence_mbar_init();
  }
  for (int i = threadIdx.x; i < JQ; i += THREADS) job_queue(smem)[i].flag = 0;
  __syncthreads();
  const bool stamp = p.stamps != nullptr && blockIdx.x == 0 && threadIdx.x == 0;
  if (stamp) p.stamps[0] = globaltimer_ns();
  uint32_t seq = 0;   // stage sequence (producer), continues across layers
  int32_t qk = 0;     // job queue position, continues across layers
  const bool small = p.TK <= SMALL_PAIRS;
  CtaTables& tb = tables(smem);
  for (int layer = 0; layer < p.L; ++layer) {
    const LayerPtrs& lp = p.layers[layer];
    const __nv_bfloat16* x = layer == 0 ? p.x_in : p.xnext;
    uint64_t* st = stamp ? p.stamps + 1 + layer * STAMPS_PER_LAYER : nullptr;
    phase_prepare(p, lp, x, layer, smem, st);
    if (!grid_barrier(p.sync, p.timeout_ns, 10 * layer + 1)) return;
    if (st) st[2] = globaltimer_ns();
    StreamCtx cx;
    const int32_t* inv;
    if (small) {
      phase_route_small(p, lp, smem, st ? st + 3 : nullptr);
      cx = StreamCtx{tb.units, tb.dunits, tb.tokpos, tb.wpos, tb.pxf, tb.n_units, tb.n_dunits};
      inv = tb.inv;
      if (p.route_only) return;
    } else {
      phase_topk_large(p, lp);
      if (!grid_barrier(p.sync, p.timeout_ns, 10 * layer + 2)) return;
      if (st) st[3] = globaltimer_ns();
      phase_permute_large(p, smem);
      if (!grid_barrier(p.sync, p.timeout_ns, 10 * layer + 3)) return;
      if (p.route_only) return;
      cx = StreamCtx{p.units, p.dunits, p.tokpos, p.wpos, p.pxf, p.n_units[0], p.n_units[1]};
      inv = p.inv;
    }
    if (st) st[4] = globaltimer_ns();
    fence_proxy_async_smem();  // the ring held routing scratch written by generic stores
    __syncthreads();
    if (warp == NCW) stream_producer(p, lp, smem, cx, seq, qk);
    else stream_consumer(p, smem, cx, qk);
    if (!grid_barrier(p.sync, p.timeout_ns, 10 * layer + 4)) return;
    if (st) st[5] = globaltimer_ns();
    if (layer + 1 < p.L) {
      phase_combine_rmsnorm(p, inv, smem);
      if (!grid_barrier(p.sync, p.timeout_ns, 10 * layer + 5)) return;
    } else {
      phase_combine_out(p, inv);
    }
    if (st) st[6] = globaltimer_ns();
  }
}

}  // namespace

size_t engine_smem_bytes() { return SMEM_BYTES; }

int engine_max_grid(int device, int* err) {
  cudaError_t e = cudaFuncSetAttribute(engine_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)SMEM_BYTES);
  if (e != cudaSuccess) { *err = (int)e; return 0; }
  int per_sm = 0, sms = 0;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, engine_kernel, THREADS, SMEM_BYTES);
  if (e != cudaSuccess) { *err = (int)e; return 0; }
  e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, device);
  if (e != cudaSuccess) { *err = (int)e; return 0; }
  *err = 0;
  return per_sm * sms;
}

cudaError_t engine_launch(const EngineParams& p, int grid, cudaStream_t s) {
  void* args[] = {const_cast<EngineParams*>(&p)};
  return cudaLaunchCooperativeKernel((const void*)engine_kernel, dim3(grid), dim3(THREADS), args,
                                     SMEM_BYTES, s);
}

}  // namespace moe
