// Persistent MXFP4 MoE engine: one cooperative launch runs, per layer,
//   A  router logits (fp64 accumulation) and fp32 copy of the activations
//   B  top-k + renormalised weights, stable per-expert permutation, unit table
//   C  the MXFP4 weight stream: gate/up projection + SwiGLU, then down
//      projection x routing weight, as warp jobs fed by bulk copies
//   D  weighted combine to bf16 (+ RMSNorm into the next layer's input)
// separated by bounded grid barriers.  The design follows the TileRT pages'
// execution model: a resident engine kernel with continuous prefetch through
// shared memory while the current tile computes, a tile-level pipeline and
// warp-specialised roles (TileRT blog "Breaking 1000 TPS", section
// "第一次跃迁：Execution Model Revolution"; bjdmk.com.cn news, section
// "极致协同，通向千速之路", on the persistent engine kernel), applied to the
// MoE expert layer whose routing is the runtime dynamism (HyperAI salon
// transcript, section "Achieving maximum speed improvement ...").
//
// Every wait (grid barrier, mbarrier, per-unit readiness) is bounded by
// p.timeout_ns of %globaltimer; on expiry the kernel records a status code in
// sync[SY_ERROR], drains its own copies in flight and returns.
#include <math.h>
#include <cuda_fp16.h>

#include "engine.cuh"
#include "ptx.cuh"

namespace moe {
namespace {

constexpr uint32_t FULL = 0xFFFFFFFFu;
constexpr int WARP_BYTES = RING_BYTES + NBAR * 8 + JQ * 4;
constexpr int SMALL_UNITS = 256 + SMALL_PAIRS / NT_MAX;

struct alignas(16) CtaTables {
  int32_t units[SMALL_UNITS * 4];  // first: read as int4
  int32_t idx[SMALL_PAIRS];
  float w[SMALL_PAIRS];
  int32_t perm[SMALL_PAIRS];
  int32_t inv[SMALL_PAIRS];
  int32_t tokpos[SMALL_PAIRS];
  float wpos[SMALL_PAIRS];
  int32_t counts[MAX_EXPERTS];
  int32_t offsets[MAX_EXPERTS + 1];
  float red[WARPS];
  int32_t n_units;
};
constexpr size_t SMEM_BYTES = (size_t)WARPS * WARP_BYTES + sizeof(CtaTables);

__device__ __forceinline__ uint8_t* warp_ring(uint8_t* smem, int w) { return smem + (size_t)w * WARP_BYTES; }
__device__ __forceinline__ uint64_t* warp_bars(uint8_t* smem, int w) {
  return reinterpret_cast<uint64_t*>(smem + (size_t)w * WARP_BYTES + RING_BYTES);
}
__device__ __forceinline__ int32_t* warp_jq(uint8_t* smem, int w) {
  return reinterpret_cast<int32_t*>(smem + (size_t)w * WARP_BYTES + RING_BYTES + NBAR * 8);
}
__device__ __forceinline__ CtaTables& tables(uint8_t* smem) {
  return *reinterpret_cast<CtaTables*>(smem + (size_t)WARPS * WARP_BYTES);
}

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

// ---- phase A: router logits (fp64) ---------------------------------------------------
// logits[t][e] = sum_h x[t][h] * Wr[e][h] + b[e]; bf16*fp32 products are exact
// in fp64 and the sums are fp64, so top-k decisions match an fp64 reference
// except on gaps below ~1e-10.
__device__ void phase_logits(const EngineParams& p, const LayerPtrs& lp, const __nv_bfloat16* x,
                             int layer) {
  const int T = p.T, H = p.H, E = p.E;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int64_t gt = (int64_t)blockIdx.x * THREADS + threadIdx.x;
  const int64_t gs = (int64_t)gridDim.x * THREADS;
  // fp32 activations for the weight stream; optional dump of the layer input
  const int64_t n2 = (int64_t)T * H / 2;
  const __nv_bfloat162* x2 = reinterpret_cast<const __nv_bfloat162*>(x);
  float2* xf2 = reinterpret_cast<float2*>(p.xf);
  __nv_bfloat162* dump = p.layer_io ? reinterpret_cast<__nv_bfloat162*>(p.layer_io + (int64_t)layer * T * H) : nullptr;
  for (int64_t i = gt; i < n2; i += gs) {
    const __nv_bfloat162 v = x2[i];
    xf2[i] = __bfloat1622float2(v);
    if (dump) dump[i] = v;
  }
  // per-layer resets of the stream's counters (used only after the next barrier)
  const int umax = min(E, p.TK) + p.TK / NT_MAX + 1;
  if (gt == 0) p.sync[SY_JOBS] = 0u;
  for (int64_t u = gt; u < umax; u += gs) p.sync[SY_READY + u] = 0u;

  const int nchunk = (T + 7) / 8;
  const int64_t njobs = (int64_t)E * nchunk;
  const int64_t wg = (int64_t)blockIdx.x * WARPS + warp, ws = (int64_t)gridDim.x * WARPS;
  for (int64_t job = wg; job < njobs; job += ws) {
    const int e = (int)(job % E), t0 = (int)(job / E) * 8;
    const int nt = min(8, T - t0);
    double acc[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[j] = 0.0;
    const float4* wr = reinterpret_cast<const float4*>(lp.router_w + (int64_t)e * H);
    for (int h4 = lane; h4 < H / 4; h4 += 32) {
      const float4 w4 = __ldg(wr + h4);
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        if (j < nt) {
          const uint2 xb = *reinterpret_cast<const uint2*>(x + (int64_t)(t0 + j) * H + h4 * 4);
          const float x0 = __uint_as_float(xb.x << 16), x1 = __uint_as_float(xb.x & 0xFFFF0000u);
          const float x2v = __uint_as_float(xb.y << 16), x3 = __uint_as_float(xb.y & 0xFFFF0000u);
          acc[j] = fma((double)x0, (double)w4.x, acc[j]);
          acc[j] = fma((double)x1, (double)w4.y, acc[j]);
          acc[j] = fma((double)x2v, (double)w4.z, acc[j]);
          acc[j] = fma((double)x3, (double)w4.w, acc[j]);
        }
      }
    }
#pragma unroll
    for (int j = 0; j < 8; ++j) {
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) acc[j] += __shfl_xor_sync(FULL, acc[j], o);
    }
    if (lane == 0) {
      const double b = lp.router_b ? (double)lp.router_b[e] : 0.0;
#pragma unroll
      for (int j = 0; j < 8; ++j)
        if (j < nt) p.logits[(int64_t)(t0 + j) * E + e] = acc[j] + b;
    }
  }
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

// One warp: the K largest logits of a row (descending, ties to the lower
// expert), weights exp(l - lmax) / sum over the K.  Lane r < K writes slot r.
__device__ void topk_row(const double* lg, int E, int K, int32_t* out_idx, float* out_w) {
  const int lane = threadIdx.x & 31;
  constexpr int PER = MAX_EXPERTS / 32;
  uint64_t key[PER];
#pragma unroll
  for (int i = 0; i < PER; ++i) {
    const int e = lane + 32 * i;
    key[i] = e < E ? order_key(lg[e]) : 0ull;
  }
  uint32_t taken = 0;
  int my_e = -1;
  double my_l = 0.0, lmax = 0.0;
  for (int r = 0; r < K; ++r) {
    uint64_t best = 0;
    int bi = -1;
#pragma unroll
    for (int i = 0; i < PER; ++i) {
      const int e = lane + 32 * i;
      if (e < E && !((taken >> i) & 1u) && (bi < 0 || key[i] > best)) { best = key[i]; bi = i; }
    }
    const uint32_t hi = __reduce_max_sync(FULL, bi >= 0 ? (uint32_t)(best >> 32) : 0u);
    const uint32_t lo = __reduce_max_sync(FULL, (bi >= 0 && (uint32_t)(best >> 32) == hi) ? (uint32_t)best : 0u);
    const uint64_t top = ((uint64_t)hi << 32) | lo;
    const uint32_t m = __reduce_max_sync(FULL, (bi >= 0 && best == top) ? (65536u - (uint32_t)(lane + 32 * bi)) : 0u);
    const int esel = (int)(65536u - m);
    if ((esel & 31) == lane) taken |= 1u << (esel >> 5);
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

// Exclusive scan of n <= 512 ints in shared memory by warp 0 (in place);
// returns the total through *total.
__device__ void warp0_exclusive_scan(int32_t* a, int n, int32_t* total) {
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

// Small T*K: every CTA routes all tokens itself (no barrier); CTA 0 also writes
// the maps to global memory.
__device__ void phase_route_small(const EngineParams& p, uint8_t* smem) {
  CtaTables& tb = tables(smem);
  const int T = p.T, E = p.E, K = p.K, TK = p.TK;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  for (int t = warp; t < T; t += WARPS) topk_row(p.logits + (int64_t)t * E, E, K, tb.idx + t * K, tb.w + t * K);
  // per-warp histograms (scratch in warp 0's ring, unused until phase C)
  int32_t* hist = reinterpret_cast<int32_t*>(warp_ring(smem, 0));  // [WARPS][E]
  for (int i = threadIdx.x; i < WARPS * E; i += THREADS) hist[i] = 0;
  __syncthreads();
  const int pr = threadIdx.x;  // TK <= SMALL_PAIRS == THREADS: one pair per thread
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
  if (warp == 0) warp0_exclusive_scan(tb.offsets, E, tb.offsets + E);
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
  // units: ceil(count/NT_MAX) per hit expert, in expert order
  int32_t* ubase = hist;  // reuse scratch after the pass above
  __syncthreads();
  for (int x = threadIdx.x; x < E; x += THREADS) ubase[x] = (tb.counts[x] + NT_MAX - 1) / NT_MAX;
  __syncthreads();
  if (warp == 0) warp0_exclusive_scan(ubase, E, &tb.n_units);
  __syncthreads();
  for (int x = threadIdx.x; x < E; x += THREADS) {
    const int c = tb.counts[x];
    for (int s = 0; s * NT_MAX < c; ++s) {
      int32_t* u = tb.units + (ubase[x] + s) * 4;
      u[0] = x; u[1] = tb.offsets[x] + s * NT_MAX; u[2] = min(NT_MAX, c - s * NT_MAX); u[3] = 0;
    }
  }
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
__device__ void phase_topk_large(const EngineParams& p) {
  const int warp = threadIdx.x >> 5;
  const int64_t wg = (int64_t)blockIdx.x * WARPS + warp, ws = (int64_t)gridDim.x * WARPS;
  for (int64_t t = wg; t < p.T; t += ws)
    topk_row(p.logits + t * p.E, p.E, p.K, p.idx + t * p.K, p.wts + t * p.K);
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
  if (warp == 0) warp0_exclusive_scan(tb.offsets, E, tb.offsets + E);
  __syncthreads();
  if (blockIdx.x == 0) {
    int32_t* ubase = reinterpret_cast<int32_t*>(warp_ring(smem, 0));
    for (int x = threadIdx.x; x < E; x += THREADS) ubase[x] = (tb.counts[x] + NT_MAX - 1) / NT_MAX;
    __syncthreads();
    if (warp == 0) warp0_exclusive_scan(ubase, E, &tb.n_units);
    __syncthreads();
    for (int x = threadIdx.x; x < E; x += THREADS) {
      const int c = tb.counts[x];
      for (int s = 0; s * NT_MAX < c; ++s) {
        int32_t* u = p.units + (int64_t)(ubase[x] + s) * 4;
        u[0] = x; u[1] = tb.offsets[x] + s * NT_MAX; u[2] = min(NT_MAX, c - s * NT_MAX); u[3] = 0;
      }
    }
    for (int i = threadIdx.x; i < E; i += THREADS) p.counts[i] = tb.counts[i];
    for (int i = threadIdx.x; i <= E; i += THREADS) p.offsets[i] = tb.offsets[i];
    if (threadIdx.x == 0) *p.n_units = tb.n_units;
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

// ---- phase C: the MXFP4 weight stream ------------------------------------------------------
__device__ __forceinline__ float e8m0_to_f32(uint32_t b) {
  if (b == 0u) return __uint_as_float(0x00400000u);  // 2^-127
  if (b == 255u) return __uint_as_float(0x7FC00000u);
  return __uint_as_float(b << 23);
}

// acc[j] += sum over this stage's KC elements of W[row][k] * x_j[k] for the
// lane's row; weights decoded E2M1 -> f16x2 -> fp32 pairs, packed fp32 FMA,
// one MX block at a time, scaled by its E8M0 factor.
template <int NT>
__device__ __forceinline__ void stage_dot(const uint8_t* st, int lane, float (&acc)[NT_MAX]) {
  const uint32_t sc4 = *reinterpret_cast<const uint32_t*>(st + STAGE_CODE_BYTES + lane * KB);
  const float* xs = reinterpret_cast<const float*>(st + STAGE_W_BYTES);
#pragma unroll
  for (int b = 0; b < KB; ++b) {
    const uint4 q = *reinterpret_cast<const uint4*>(st + b * (ROWS * 16) + lane * 16);
    const uint32_t qw[4] = {q.x, q.y, q.z, q.w};
    f32x2 part[NT];
#pragma unroll
    for (int j = 0; j < NT; ++j) part[j] = {0.f, 0.f};
#pragma unroll
    for (int m = 0; m < 4; ++m) {
#pragma unroll
      for (int hb = 0; hb < 2; ++hb) {  // two bytes (four codes) per step
        const uint32_t h0 = e2m1x2_to_f16x2(qw[m] >> (16 * hb));
        const uint32_t h1 = e2m1x2_to_f16x2(qw[m] >> (16 * hb + 8));
        const float2 w0 = __half22float2(*reinterpret_cast<const __half2*>(&h0));
        const float2 w1 = __half22float2(*reinterpret_cast<const __half2*>(&h1));
        const int k = b * 32 + m * 8 + hb * 4;
#pragma unroll
        for (int j = 0; j < NT; ++j) {
          const float4 xv = *reinterpret_cast<const float4*>(xs + j * KC + k);
          ffma2(part[j], {w0.x, w0.y}, {xv.x, xv.y});
          ffma2(part[j], {w1.x, w1.y}, {xv.z, xv.w});
        }
      }
    }
    const float sc = e8m0_to_f32((sc4 >> (8 * b)) & 0xFFu);
#pragma unroll
    for (int j = 0; j < NT; ++j) acc[j] = fmaf(part[j].x + part[j].y, sc, acc[j]);
  }
}

__device__ __forceinline__ void stage_dot_nt(int nt, const uint8_t* st, int lane, float (&acc)[NT_MAX]) {
  switch (nt) {
    case 1: stage_dot<1>(st, lane, acc); break;
    case 2: stage_dot<2>(st, lane, acc); break;
    case 3: stage_dot<3>(st, lane, acc); break;
    case 4: stage_dot<4>(st, lane, acc); break;
    case 5: stage_dot<5>(st, lane, acc); break;
    case 6: stage_dot<6>(st, lane, acc); break;
    case 7: stage_dot<7>(st, lane, acc); break;
    default: stage_dot<8>(st, lane, acc); break;
  }
}

struct Job {
  int unit, rb, isD, e, pos0, nt, nc;
};

__device__ __forceinline__ Job decode_job(const EngineParams& p, const int32_t* units, int64_t j,
                                          int64_t n_gu, int gub, int db) {
  Job jb;
  int64_t u;
  if (j < n_gu) { u = j / gub; jb.rb = (int)(j % gub); jb.isD = 0; jb.nc = p.H / KC; }
  else { const int64_t jj = j - n_gu; u = jj / db; jb.rb = (int)(jj % db); jb.isD = 1; jb.nc = p.I / KC; }
  jb.unit = (int)u;
  const int4 ur = *reinterpret_cast<const int4*>(units + u * 4);
  jb.e = ur.x; jb.pos0 = ur.y; jb.nt = ur.z;
  return jb;
}

__device__ __forceinline__ uint32_t ring_place(uint32_t v, uint32_t size) {
  const uint32_t off = v % RING_BYTES;
  return off + size > (uint32_t)RING_BYTES ? v + (RING_BYTES - off) : v;
}

// Runs this warp's share of the gate/up and down jobs.  Returns false on timeout.
__device__ bool phase_stream(const EngineParams& p, const LayerPtrs& lp, uint8_t* smem,
                             const int32_t* units, int n_units, const int32_t* tokpos,
                             const float* wpos, uint32_t& seq_base) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint8_t* ring = warp_ring(smem, warp);
  uint64_t* bars = warp_bars(smem, warp);
  int32_t* jq = warp_jq(smem, warp);
  const int gub = p.I / GU_ROWS, db = p.H / ROWS;
  const int64_t n_gu = (int64_t)n_units * gub, n_all = n_gu + (int64_t)n_units * db;
  uint32_t* ready = p.sync + SY_READY;

  // producer state (warp-uniform except tok)
  bool fetch_done = false, have_pjob = false, p_ready = true;
  Job pj{};
  int p_c = 0, tok = 0;
  uint32_t p_v = 0, p_seq = seq_base, p_nj = 0;
  // consumer state
  Job cj{};
  int c_c = 0;
  uint32_t c_v = 0, c_seq = seq_base, c_nj = 0;
  float acc[NT_MAX];
  bool ok = true;
  fence_proxy_async_global();
  fence_proxy_async_smem();  // the ring held routing scratch written by generic stores

  for (;;) {
    // ---- issue as many stages as the ring allows
    for (;;) {
      if (!have_pjob) {
        if (fetch_done) break;
        int64_t j = 0;
        if (lane == 0) j = atomicAdd(p.sync + SY_JOBS, 1u);
        j = __shfl_sync(FULL, (long long)j, 0);
        if (j >= n_all) { fetch_done = true; break; }
        pj = decode_job(p, units, j, n_gu, gub, db);
        if (lane == 0) jq[p_nj % JQ] = (int32_t)j;
        ++p_nj;
        p_c = 0;
        have_pjob = true;
        p_ready = !pj.isD;
        if (!pj.isD && lane < pj.nt) tok = tokpos[pj.pos0 + lane];
      }
      if (!p_ready) {
        if (ld_acquire_u32(ready + pj.unit) < (uint32_t)gub) break;
        p_ready = true;
        fence_proxy_async_global();
      }
      const uint32_t size = STAGE_W_BYTES + pj.nt * X_SLICE_BYTES;
      const uint32_t start = ring_place(p_v, size);
      if (p_seq - c_seq >= (uint32_t)NBAR || start + size - c_v > (uint32_t)RING_BYTES) break;
      uint8_t* dst = ring + (start % RING_BYTES);
      uint64_t* bar = bars + (p_seq % NBAR);
      if (lane == 0) {
        mbar_arrive_expect_tx(bar, size);
        const uint8_t* wsrc = pj.isD
            ? lp.w_d + (((int64_t)pj.e * db + pj.rb) * pj.nc + p_c) * STAGE_W_BYTES
            : lp.w_gu + (((int64_t)pj.e * gub + pj.rb) * pj.nc + p_c) * STAGE_W_BYTES;
        bulk_g2s(dst, wsrc, STAGE_W_BYTES, bar);
        if (pj.isD)
          bulk_g2s(dst + STAGE_W_BYTES, p.abuf + ((int64_t)p_c * p.TK + pj.pos0) * KC,
                   pj.nt * X_SLICE_BYTES, bar);
      }
      __syncwarp();
      if (!pj.isD && lane < pj.nt)
        bulk_g2s(dst + STAGE_W_BYTES + lane * X_SLICE_BYTES, p.xf + (int64_t)tok * p.H + p_c * KC,
                 X_SLICE_BYTES, bar);
      p_v = start + size;
      ++p_seq;
      if (++p_c == pj.nc) have_pjob = false;
    }

    if (c_seq == p_seq) {  // nothing in flight
      if (!have_pjob && fetch_done) break;
      if (have_pjob && !p_ready) {  // wait for this unit's gate/up jobs (bounded)
        const uint64_t t0 = globaltimer_ns();
        uint32_t spins = 0;
        while (ld_acquire_u32(ready + pj.unit) < (uint32_t)gub) {
          if ((++spins & 15u) == 0u) {
            if (error_set(p.sync)) { ok = false; break; }
            if (globaltimer_ns() - t0 > p.timeout_ns) { set_error(p.sync, DEV_TIMEOUT_READY, pj.unit); ok = false; break; }
          }
          __nanosleep(128);
        }
        if (!ok) break;
      }
      continue;
    }

    // ---- consume the oldest stage
    if (c_c == 0) {
      const int64_t j = jq[c_nj % JQ];
      cj = decode_job(p, units, j, n_gu, gub, db);
#pragma unroll
      for (int i = 0; i < NT_MAX; ++i) acc[i] = 0.f;
    }
    const uint32_t size = STAGE_W_BYTES + cj.nt * X_SLICE_BYTES;
    const uint32_t start = ring_place(c_v, size);
    uint64_t* bar = bars + (c_seq % NBAR);
    const uint32_t parity = (c_seq / NBAR) & 1u;
    if (!mbar_try_wait(bar, parity)) {
      const uint64_t t0 = globaltimer_ns();
      uint32_t spins = 0;
      while (!mbar_try_wait(bar, parity)) {
        if ((++spins & 63u) == 0u) {
          if (error_set(p.sync)) { ok = false; break; }
          if (globaltimer_ns() - t0 > p.timeout_ns) { set_error(p.sync, DEV_TIMEOUT_PIPE, c_seq); ok = false; break; }
        }
      }
      if (!ok) break;
    }
    stage_dot_nt(cj.nt, ring + (start % RING_BYTES), lane, acc);
    __syncwarp();
    c_v = start + size;
    ++c_seq;
    if (++c_c == cj.nc) {
      c_c = 0;
      ++c_nj;
      if (!cj.isD) {  // SwiGLU epilogue: lanes 0-15 gate rows, 16-31 the same up rows
        float u[NT_MAX];
#pragma unroll
        for (int j = 0; j < NT_MAX; ++j) u[j] = __shfl_down_sync(FULL, acc[j], 16);
        if (lane < 16) {
          const int i = cj.rb * GU_ROWS + lane;
          float* dst = p.abuf + ((int64_t)(i / KC) * p.TK + cj.pos0) * KC + (i % KC);
#pragma unroll
          for (int j = 0; j < NT_MAX; ++j) {
            if (j < cj.nt) {
              const float g = acc[j];
              dst[(int64_t)j * KC] = g / (1.0f + expf(-g)) * u[j];
            }
          }
        }
        __threadfence();
        __syncwarp();
        if (lane == 0) red_release_add_u32(ready + cj.unit, 1u);
      } else {  // down epilogue: weighted pair output rows
        const int h = cj.rb * ROWS + lane;
#pragma unroll
        for (int j = 0; j < NT_MAX; ++j)
          if (j < cj.nt) p.ypair[(int64_t)(cj.pos0 + j) * p.H + h] = wpos[cj.pos0 + j] * acc[j];
      }
    }
  }
  if (!ok) {  // drain this warp's copies still in flight (bounded) before leaving
    const uint64_t t0 = globaltimer_ns();
    while (c_seq != p_seq && globaltimer_ns() - t0 < p.timeout_ns) {
      if (mbar_try_wait(bars + (c_seq % NBAR), (c_seq / NBAR) & 1u)) ++c_seq;
    }
  }
  seq_base = p_seq;  // keep barrier phases consistent across layers
  return ok;
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
  constexpr int MAXV = 8;  // float4 per thread: H <= 8 * 4 * THREADS = 8192
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
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (lane == 0) {
    uint64_t* bars = warp_bars(smem, warp);
    for (int i = 0; i < NBAR; ++i) mbar_init(bars + i, 1);
    fence_mbar_init();
  }
  __syncthreads();
  uint32_t seq = 0;
  const bool small = p.TK <= SMALL_PAIRS;
  CtaTables& tb = tables(smem);
  for (int layer = 0; layer < p.L; ++layer) {
    const LayerPtrs& lp = p.layers[layer];
    const __nv_bfloat16* x = layer == 0 ? p.x_in : p.xnext;
    phase_logits(p, lp, x, layer);
    if (!grid_barrier(p.sync, p.timeout_ns, 10 * layer + 1)) return;
    const int32_t *units, *tokpos, *inv;
    const float* wpos;
    int n_units;
    if (small) {
      phase_route_small(p, smem);
      units = tb.units; tokpos = tb.tokpos; wpos = tb.wpos; inv = tb.inv; n_units = tb.n_units;
      if (p.route_only) return;
    } else {
      phase_topk_large(p);
      if (!grid_barrier(p.sync, p.timeout_ns, 10 * layer + 2)) return;
      phase_permute_large(p, smem);
      if (!grid_barrier(p.sync, p.timeout_ns, 10 * layer + 3)) return;
      if (p.route_only) return;
      units = p.units; tokpos = p.tokpos; wpos = p.wpos; inv = p.inv; n_units = *p.n_units;
    }
    __syncthreads();
    const bool ok = phase_stream(p, lp, smem, units, n_units, tokpos, wpos, seq);
    if (!ok) set_error(p.sync, DEV_TIMEOUT_PIPE, 0xFFFFFFFFu);  // no-op if already set
    if (!grid_barrier(p.sync, p.timeout_ns, 10 * layer + 4)) return;
    if (layer + 1 < p.L) {
      phase_combine_rmsnorm(p, inv, smem);
      if (!grid_barrier(p.sync, p.timeout_ns, 10 * layer + 5)) return;
    } else {
      phase_combine_out(p, inv);
    }
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
