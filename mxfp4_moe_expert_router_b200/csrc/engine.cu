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
// Weight stream (phase C).  Work is cut into CTA jobs of 128 weight rows x the
// whole contraction dimension (see engine.cuh).  Warp 0 is the producer: it
// takes jobs from a global counter, publishes them in a shared-memory job
// queue and streams each job's K stages -- an 8704-byte MXFP4 weight stage
// plus the E2M1 term images of the unit's activations -- into a ring of NSLOT
// slots with 1-D bulk copies (full/empty mbarriers).  One thread of warp 1
// issues the fifth-generation tensor-core MMAs: per stage it copies the
// weight and activation E8M0 scales into tensor memory and runs two
// block-scaled kind::mxf4 MMAs (M = 128, K = 64, N = 8 columns per token or
// pair) accumulating in tensor memory; a commit frees the ring slot when they
// complete, and a commit at the job's end hands the accumulator buffer to the
// epilogue.  Warps 4..11 (two groups of four, one warp per 32-lane
// sub-partition of tensor memory) run the epilogues of alternate jobs: sum the
// 8 term columns, SwiGLU and the term expansion of its output (gate/up), or
// scale by the routing weight (down).  No CUDA core touches a weight.
//
// Activations as E2M1 terms.  The MMA multiplies E2M1 by E2M1, so a value v of
// a 32-element block with amax A is written as v = sum_k c_k 2^s_k, c_k E2M1,
// s_0 = ceil(log2(A / 6)), s_k = s_0 + 1 - 3k (k >= 1): each term rounds the
// remaining residual to nearest, exactly, and the residual after NTERM = 8
// terms is below 2^(s_0 - 21) <= A * 2^-21 -- beneath the fp32 accumulation.
//
// Every wait (grid barrier, mbarrier, job queue, per-unit readiness) is bounded
// by p.timeout_ns of %globaltimer; on expiry the kernel records a status code
// in sync[SY_ERROR], stops issuing work, lets every copy and MMA in flight
// complete, frees its tensor memory and returns.
#include <math.h>
#include <cuda_fp16.h>

#include "engine.cuh"
#include "ptx.cuh"

namespace moe {
namespace {

constexpr uint32_t FULL = 0xFFFFFFFFu;
// Bound of the drains before a CTA reuses or releases memory that bulk copies
// or MMAs it already issued still target (the ring, tensor memory).  Issued
// work completes on its own within microseconds, so this bound is fixed and
// independent of the caller's wait bound: a short p.timeout_ns stops new work
// early but never frees shared or tensor memory under work in flight.
constexpr uint64_t DRAIN_NS = 2000000000ull;
constexpr int SMALL_UNITS = 256 + SMALL_PAIRS / NT_MAX;
constexpr int SMALL_DUNITS = 256 + SMALL_PAIRS / ND_MAX;

struct JobEntry {
  int32_t flag;  // queue index + 1 once the entry is written
  int32_t job;   // -1: no more jobs in this phase
  int32_t s0;    // stage sequence number of stage 0
  int32_t nc;    // stages
  int32_t unit, rb, isD, e, pos0, nt;
  int32_t wj;    // work index (per CTA): accumulator buffer wj % NACC, epilogue group wj % 2
  int32_t pad;
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
  int32_t counts[MAX_EXPERTS];
  int32_t offsets[MAX_EXPERTS + 1];
  float red[WARPS];
  int32_t n_units, n_dunits;
  int32_t last, gen;  // route barrier: this CTA arrived last; barrier generation
  int32_t claim;      // x image tasks claimed by this CTA (small T*K)
};

constexpr size_t align16(size_t v) { return (v + 15) & ~size_t(15); }
constexpr size_t RING_BYTES = (size_t)NPIPE * NSLOT * SLOT_BYTES;   // all pipelines' rings
constexpr size_t OFF_RING = 0;
constexpr size_t OFF_FULL = OFF_RING + RING_BYTES;                  // [NPIPE][NSLOT]
constexpr size_t OFF_EMPTY = OFF_FULL + NPIPE * NSLOT * 8;          // [NPIPE][NSLOT]
constexpr size_t OFF_ACCF = OFF_EMPTY + NPIPE * NSLOT * 8;          // [NPIPE][NACC]
constexpr size_t OFF_ACCE = OFF_ACCF + NPIPE * NACC * 8;            // [NPIPE][NACC]
constexpr size_t OFF_XBAR = OFF_ACCE + NPIPE * NACC * 8;            // [NPIPE][2] amax exchange
constexpr size_t OFF_DRAIN = OFF_XBAR + NPIPE * 2 * 8;              // [NPIPE]
constexpr size_t OFF_TMEMBASE = OFF_DRAIN + NPIPE * 8;
constexpr size_t OFF_JQ = align16(OFF_TMEMBASE + 8);                // [NPIPE][JQ]
constexpr size_t OFF_XCH = align16(OFF_JQ + NPIPE * JQ * sizeof(JobEntry));  // [NPIPE][2][NT_MAX][4] floats
constexpr size_t XCH_FLOATS = (NPIPE * 2 * NT_BIG > 4 * ET_MAX ? NPIPE * 2 * NT_BIG : 4 * ET_MAX) * 4;
static_assert(ET_MAX >= LT_MAX, "amax exchange sized by the largest tile");
constexpr size_t OFF_TABLES = align16(OFF_XCH + XCH_FLOATS * 4);
constexpr size_t SMEM_BYTES = OFF_TABLES + sizeof(CtaTables);
static_assert(SMEM_BYTES <= 232448, "shared memory budget");
static_assert((size_t)WARPS * MAX_EXPERTS * 8 <= RING_BYTES, "routing scratch in ring");
static_assert((size_t)16 * (8192 / MAX_HSPLIT) * 8 <= RING_BYTES, "router x slice in ring");
static_assert((size_t)LT_NSLOT * LT_SLOT_BYTES <= RING_BYTES && LT_SLOT_BYTES % 16 == 0, "tile ring");
static_assert(SLOT_BYTES % 16 == 0 && STAGE_A_BYTES % 16 == 0 && IMG_BYTES % 16 == 0, "bulk-copy alignment");

__device__ __forceinline__ uint8_t* ring_slot(uint8_t* smem, int pipe, int s) {
  return smem + OFF_RING + ((size_t)pipe * NSLOT + s) * SLOT_BYTES;
}
// The pipeline stream for units of at most U positions (NT_MAX, or NT_BIG
// for big units): ring slots and, in tensor memory, pipeline p's
// accumulators, then its scale-factor buffers.
template <int U> struct PipeCfg;
template <> struct PipeCfg<NT_MAX> {
  static constexpr int NS = NSLOT, SLOTB = SLOT_BYTES, ACCW = ACC_COLS;
};
template <> struct PipeCfg<NT_BIG> {
  static constexpr int NS = NSLOT_BIG, SLOTB = SLOT_BYTES_BIG, ACCW = ACC_COLS_BIG;
};
static_assert((size_t)NPIPE * NSLOT_BIG * SLOT_BYTES_BIG <= RING_BYTES && SLOT_BYTES_BIG % 16 == 0, "big-unit ring");
template <int U>
__device__ __forceinline__ uint32_t pipe_ring(uint8_t* smem, int pipe) {
  return smem_u32(smem + OFF_RING + (size_t)pipe * PipeCfg<U>::NS * PipeCfg<U>::SLOTB);
}
template <int U>
__device__ __forceinline__ uint32_t pipe_acc(int pipe, int b) { return (uint32_t)(pipe * NACC + b) * PipeCfg<U>::ACCW; }
template <int U>
__device__ __forceinline__ uint32_t pipe_sf(int pipe, int i) {
  return (uint32_t)(NPIPE * NACC * PipeCfg<U>::ACCW + (pipe * NSF + i) * SF_COLS);
}
__device__ __forceinline__ uint64_t* full_bar(uint8_t* smem, int pipe, int s) { return reinterpret_cast<uint64_t*>(smem + OFF_FULL) + pipe * NSLOT + s; }
__device__ __forceinline__ uint64_t* empty_bar(uint8_t* smem, int pipe, int s) { return reinterpret_cast<uint64_t*>(smem + OFF_EMPTY) + pipe * NSLOT + s; }
__device__ __forceinline__ uint64_t* accf_bar(uint8_t* smem, int pipe, int b) { return reinterpret_cast<uint64_t*>(smem + OFF_ACCF) + pipe * NACC + b; }
__device__ __forceinline__ uint64_t* acce_bar(uint8_t* smem, int pipe, int b) { return reinterpret_cast<uint64_t*>(smem + OFF_ACCE) + pipe * NACC + b; }
__device__ __forceinline__ uint64_t* xch_bar(uint8_t* smem, int pipe, int i) { return reinterpret_cast<uint64_t*>(smem + OFF_XBAR) + pipe * 2 + i; }
__device__ __forceinline__ uint64_t* drain_bar(uint8_t* smem, int pipe) { return reinterpret_cast<uint64_t*>(smem + OFF_DRAIN) + pipe; }
__device__ __forceinline__ uint32_t* tmem_base_word(uint8_t* smem) { return reinterpret_cast<uint32_t*>(smem + OFF_TMEMBASE); }
__device__ __forceinline__ JobEntry* job_queue(uint8_t* smem, int pipe) { return reinterpret_cast<JobEntry*>(smem + OFF_JQ) + pipe * JQ; }
__device__ __forceinline__ float* xch_buf(uint8_t* smem, int pipe, int i, int u = NT_MAX) {
  return reinterpret_cast<float*>(smem + OFF_XCH) + (pipe * 2 + i) * u * 4;
}
__device__ __forceinline__ CtaTables& tables(uint8_t* smem) { return *reinterpret_cast<CtaTables*>(smem + OFF_TABLES); }

// Stream modes: 0 = pipeline stream (units of <= NT_MAX positions, or of
// <= NT_BIG for big units; two pipelines per CTA), 1 = tiles (<= LT_MAX
// positions, one row block per job),
// 4 = tile pairs (<= LTA_MAX positions, LTA_R row blocks per job sharing each
// B stage).  The tile modes run one pipeline per CTA.
template <int TM> struct TileCfg;
template <> struct TileCfg<1> {
  static constexpr int R = 1, ACCW = LT_ACC_COLS, NACCV = LT_NACC, NS = LT_NSLOT,
                       SLOTB = LT_SLOT_BYTES;
};
template <> struct TileCfg<4> {
  static constexpr int R = LTA_R, ACCW = LTA_ACC_COLS, NACCV = LTA_NACC, NS = LTA_NSLOT,
                       SLOTB = LTA_SLOT_BYTES;
};
static_assert((size_t)LTA_NSLOT * LTA_SLOT_BYTES <= RING_BYTES && LTA_SLOT_BYTES % 16 == 0, "tile pair ring");
static_assert(PRODUCER_BATCH <= LT_NSLOT, "producer batch (tiles)");

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
    // the arrival releases this CTA's writes; the last arrival acquires them
    // all, resets the count (every CTA touches it again only after it sees
    // the new generation) and releases the new generation
    const uint32_t gen = ld_volatile_u32(sync + SY_BAR_GEN);
    const uint32_t prev = atom_add_acq_rel_u32(sync + SY_BAR_COUNT, 1u);
    if (prev == gridDim.x - 1) {
      *reinterpret_cast<volatile uint32_t*>(sync + SY_BAR_COUNT) = 0u;
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
      __threadfence();
    }
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

// ---- E2M1 term expansion of activations ----------------------------------------------------
// Exponent of term 0 for a block with amax A > 0: the least s with A <= 6 * 2^s
// (A = m 2^E, m in [1, 2): s = E - 2 if m <= 1.5, else E - 1), kept in
// [-126, 126] so that every term exponent has an E8M0 byte in [1, 253].
__device__ __forceinline__ int term0_exp(float amax) {
  const uint32_t u = __float_as_uint(amax);
  const int E = (int)((u >> 23) & 0xFF) - 127;
  if (E < -126) return -126;  // zero or subnormal amax
  const int s = (u & 0x7FFFFFu) <= 0x400000u ? E - 2 : E - 1;
  return min(max(s, -126), 126);
}
__device__ __forceinline__ int term_exp(int s0, int k) { return max(k == 0 ? s0 : s0 + 1 - 3 * k, -126); }

// E2M1 value of a code (low nibble), exact.
__device__ __forceinline__ float e2m1_value(uint32_t code) {
  return __half2float(__ushort_as_half((uint16_t)(e2m1x2_to_f16x2(code) & 0xFFFFu)));
}

// The NTERM E2M1 codes c_k of v = sum_k c_k 2^s_k (+ a residual below
// 2^(s_0 - 21)); code k in bits 4k..4k+3.  Each step rounds the current
// residual r to the nearest E2M1 multiple of 2^s_k and subtracts it exactly.
template <int NT = NTERM>
__device__ __forceinline__ uint32_t e2m1_terms(float v, int s0) {
  uint32_t w = 0;
  float r = v;
#pragma unroll
  for (int k = 0; k < NT; ++k) {
    const int sk = term_exp(s0, k);
    const uint32_t c = f32x2_to_e2m1x2(0.f, r * pow2f(-sk)) & 0xFu;
    r = fmaf(-e2m1_value(c), pow2f(sk), r);
    w |= c << (4 * k);
  }
  return w;
}

// Warp transpose of term codes: lane i holds the NTERM codes of element i of
// `n` consecutive elements (n = 16 or 32); lane o receives the 32-bit word of
// term o / (n / 8) covering elements 8 (o % (n / 8)) .. +7 (element 8q + j at
// bits 4j, so the word is little-endian bytes of packed E2M1 pairs).
template <int NEL>
__device__ __forceinline__ uint32_t term_word(uint32_t codes, int lane) {
  constexpr int WPT = NEL / 8;  // words per term
  const int k = (lane / WPT) % NTERM, q = lane % WPT;
  uint32_t out = 0;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const uint32_t v = __shfl_sync(FULL, codes, 8 * q + j);
    out |= ((v >> (4 * k)) & 0xFu) << (4 * j);
  }
  return out;
}

// ---- phase A: activation term images, router partial logits --------------------------------
constexpr int RTC = 16;  // tokens per router chunk

// Router work of this CTA: the H parts hs = hs0, hs0 + hstep, ... and, for
// each, the experts e = e0, e0 + estep, ...  With at least HS CTAs every CTA
// owns one part (the CTAs of part hs share its experts), so each converts a
// single slice of x; with fewer CTAs a CTA owns whole parts.
struct RouterWork { int hs0, hstep, e0, estep; };
__device__ __forceinline__ RouterWork router_work(const EngineParams& p) {
  const int g = (int)gridDim.x, c = (int)blockIdx.x;
  if (g >= p.HS) {
    const int hs = c % p.HS;
    return RouterWork{hs, p.HS, c / p.HS, (g - hs + p.HS - 1) / p.HS};
  }
  return RouterWork{c, g, 0, 1};
}

// Sum over the warp of P values per lane (P a power of two <= 32),
// reduce-scatter order: afterwards lane l holds the total of value l % P
// (P - 1 + 5 - log2 P double shuffles instead of 5 P).
template <int P>
__device__ __forceinline__ double warp_sum_rs(double (&v)[P], int lane) {
#pragma unroll
  for (int st = 0; (1 << st) < P; ++st) {
    const int n = P >> (st + 1);  // values kept after this step
    const bool hi = (lane >> st) & 1;
#pragma unroll
    for (int k = 0; k < n; ++k) {
      const double send = hi ? v[2 * k] : v[2 * k + 1];
      const double keep = hi ? v[2 * k + 1] : v[2 * k];
      v[k] = keep + __shfl_xor_sync(FULL, send, 1 << st);
    }
  }
  double r = v[0];
#pragma unroll
  for (int o = P; o < 32; o <<= 1) r += __shfl_xor_sync(FULL, r, o);
  return r;
}

// Router dot products of one token chunk of nt <= NT tokens: warp per expert
// k of this CTA, lanes along this H part, fp64 accumulation (bf16 x as fp64
// in xd[RTC][hpart]; rows nt..NT-1 are ignored), fp32 weights, then one
// reduce-scatter over the lanes.
// (Scalar arguments: a reference to the kernel's parameter block would move
// that block to local memory for the whole kernel.)
__host__ __device__ constexpr int pow2_at_least(int n) { return n <= 1 ? 1 : 2 * pow2_at_least((n + 1) / 2); }
template <int NT>
__device__ __forceinline__ void router_dots(const double* xd, const float* wsm, const float* router_w,
                                         int nexp, int e0, int estep, int H, int hpart, int hs,
                                         double* logits, int T, int t0, int nt, int E) {
  constexpr int P = pow2_at_least(NT);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  for (int k = warp; k < nexp; k += WARPS) {
    const int e = e0 + k * estep;
    const float* wr = wsm ? wsm + (size_t)k * hpart : router_w + (int64_t)e * H + hs * hpart;
    double acc[P];
#pragma unroll
    for (int j = 0; j < P; ++j) acc[j] = 0.0;
#pragma unroll 4
    for (int h = lane; h < hpart; h += 32) {
      const double w = (double)wr[h];
#pragma unroll
      for (int j = 0; j < NT; ++j) acc[j] = fma(xd[j * hpart + h], w, acc[j]);
    }
    const double v = warp_sum_rs<P>(acc, lane);  // lane l (< nt <= NT) holds token t0 + l
    if (lane < nt) logits[((int64_t)hs * T + t0 + lane) * E + e] = v;
  }
}

// The same dot products, two experts per warp pass.
template <int NT>
__device__ __forceinline__ void router_dots2(const double* xd, const float* wsm, const float* router_w,
                                         int nexp, int e0, int estep, int H, int hpart, int hs,
                                         double* logits, int T, int t0, int nt, int E) {
  constexpr int P = pow2_at_least(NT);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  // experts 2 k2 and 2 k2 + 1 per pass: each x value read from shared memory
  // serves both (the reads of x, not the FMAs, bound this loop); each
  // expert's sums keep the order of a single-expert pass
  for (int k2 = warp; 2 * k2 < nexp; k2 += WARPS) {
    const int ka = 2 * k2, kb = min(ka + 1, nexp - 1);
    const int ea = e0 + ka * estep, eb = e0 + kb * estep;
    const float* wa = wsm ? wsm + (size_t)ka * hpart : router_w + (int64_t)ea * H + hs * hpart;
    const float* wb = wsm ? wsm + (size_t)kb * hpart : router_w + (int64_t)eb * H + hs * hpart;
    double acc[P], bcc[P];
#pragma unroll
    for (int j = 0; j < P; ++j) acc[j] = bcc[j] = 0.0;
#pragma unroll 2
    for (int h = lane; h < hpart; h += 32) {
      const double w = (double)wa[h], u = (double)wb[h];
#pragma unroll
      for (int j = 0; j < NT; ++j) {
        const double xv = xd[j * hpart + h];
        acc[j] = fma(xv, w, acc[j]);
        bcc[j] = fma(xv, u, bcc[j]);
      }
    }
    const double va = warp_sum_rs<P>(acc, lane);  // lane l (< nt <= NT) holds token t0 + l
    const double vb = warp_sum_rs<P>(bcc, lane);
    if (lane < nt) {
      logits[((int64_t)hs * T + t0 + lane) * E + ea] = va;
      if (kb != ka) logits[((int64_t)hs * T + t0 + lane) * E + eb] = vb;
    }
  }
}

// One token chunk: nt rounded up to 1, 2, 4, 8, 9, 12 or 16; PAIR: two
// experts per warp pass (the chained instance; the decode instance keeps the
// single-expert pass and its code generation).
template <bool PAIR>
__device__ __noinline__ void router_chunk(const double* xd, const float* wsm, const float* router_w,
                                          int nexp, int e0, int estep, int H, int hpart, int hs,
                                          double* logits, int T, int t0, int nt, int E) {
#define MOE_ROUTER_DOTS(NT)                                                                                 \
  if constexpr (PAIR) router_dots2<NT>(xd, wsm, router_w, nexp, e0, estep, H, hpart, hs, logits, T, t0, nt, E); \
  else router_dots<NT>(xd, wsm, router_w, nexp, e0, estep, H, hpart, hs, logits, T, t0, nt, E)
  if (nt == 1) MOE_ROUTER_DOTS(1);
  else if (nt == 2) MOE_ROUTER_DOTS(2);
  else if (nt <= 4) MOE_ROUTER_DOTS(4);
  else if (nt <= 8) MOE_ROUTER_DOTS(8);
  else if (nt == 9) MOE_ROUTER_DOTS(9);
  else if (nt <= 12) MOE_ROUTER_DOTS(12);
  else MOE_ROUTER_DOTS(16);
#undef MOE_ROUTER_DOTS
}

// One warp: the image of 32-element block gb of token t in xt[stage][t], its
// values expanded into E2M1 terms (codes at the MMA's B-operand rows, scales
// at the scale-factor rows of the image): all NTERM, or the first NT (the
// tile streams read only LT_NTERM; term rows past NT get zero codes).
template <int NT>
__device__ __forceinline__ void image_task(const EngineParams& p, const __nv_bfloat16* x, int t, int gb) {
  const int lane = threadIdx.x & 31;
  const float v = __bfloat162float(__ldcg(x + (int64_t)t * p.H + gb * 32 + lane));
  float am = fabsf(v);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) am = fmaxf(am, __shfl_xor_sync(FULL, am, o));
  const int s0 = term0_exp(am);
  const uint32_t word = term_word<32>(e2m1_terms<NT>(v, s0), lane);
  const int b = gb % KB, kk = b >> 1, kc = b & 1;
  uint8_t* img = p.xt + ((int64_t)(gb / KB) * p.T + t) * IMG_BYTES;
  *reinterpret_cast<uint32_t*>(img + kk * 256 + kc * 128 + (lane >> 2) * 16 + (lane & 3) * 4) = word;
  if (lane < NTERM) img[IMG_CODE_BYTES + lane * 16 + b] = (uint8_t)(term_exp(s0, lane) + 127);
}

// The layer-input copy of the optional per-layer output (grid-stride).
__device__ __forceinline__ void layer_input_copy(const EngineParams& p, const __nv_bfloat16* x, int layer) {
  if (!p.layer_io) return;
  const int64_t gt = (int64_t)blockIdx.x * THREADS + threadIdx.x;
  const int64_t gs = (int64_t)gridDim.x * THREADS;
  const int64_t n8 = (int64_t)p.T * p.H / 8;
  const uint4* s8 = reinterpret_cast<const uint4*>(x);
  uint4* d8 = reinterpret_cast<uint4*>(p.layer_io + (int64_t)layer * p.T * p.H);
  for (int64_t i = gt; i < n8; i += gs) d8[i] = __ldcg(s8 + i);
}

// x[t] (bf16) -> xt[stage][t], one warp per 32-element block (grid-stride
// over the warps), then the layer-input copy of the optional per-layer output.
template <int NT = NTERM>
__device__ void phase_images(const EngineParams& p, const __nv_bfloat16* x, int layer) {
  const int warp = threadIdx.x >> 5;
  const int64_t wg = (int64_t)blockIdx.x * WARPS + warp, ws = (int64_t)gridDim.x * WARPS;
  const int nblk = p.H / 32;
  const int64_t ntask = p.route_only ? 0 : (int64_t)p.T * nblk;  // routing alone needs no images
  for (int64_t task = wg; task < ntask; task += ws) image_task<NT>(p, x, (int)(task / nblk), (int)(task % nblk));
  layer_input_copy(p, x, layer);
}

// The same images for the per-CTA routing, where one CTA (the last to arrive)
// computes the routing while the others write the images: tasks are claimed
// from sync[SY_IMGQ], one per warp of the claiming CTA, so that the CTA busy
// with the routing takes none of them late (the stream's producers wait for
// every image before their first gate/up stage).
__device__ void phase_images_claimed(const EngineParams& p, const __nv_bfloat16* x, int layer, uint8_t* smem) {
  CtaTables& tb = tables(smem);
  const int warp = threadIdx.x >> 5;
  const int nblk = p.H / 32, ntask = p.T * nblk;  // T*K <= SMALL_PAIRS: far below 2^31
  for (;;) {
    if (threadIdx.x == 0) tb.claim = (int32_t)atomicAdd(p.sync + SY_IMGQ, (uint32_t)WARPS);
    __syncthreads();
    const int base = tb.claim;
    __syncthreads();  // every warp has read the claim before the next one replaces it
    if (base >= ntask) break;
    const int task = base + warp;
    if (task < ntask) image_task<NTERM>(p, x, task / nblk, task % nblk);
  }
  layer_input_copy(p, x, layer);
}

// ---- E4M3 term expansion (kind::mxf8f6f4 tiles) -------------------------------------------
// Exponent of term 0 for a block with amax A: the least s with A <= 448 * 2^s
// (A = m 2^E, m in [1, 2): s = E - 8 if m <= 1.75, else E - 7), kept in
// [-118, 127] so that every term exponent s - ET_STEP k (k < 3) has an E8M0
// byte in [1, 254].
__device__ __forceinline__ int et_term0_exp(float amax) {
  const uint32_t u = __float_as_uint(amax);
  const int E = (int)((u >> 23) & 0xFF) - 127;
  if (E < -126) return -118;  // zero or subnormal amax
  const int s = (u & 0x7FFFFFu) <= 0x600000u ? E - 8 : E - 7;
  return min(max(s, -118), 127);
}
// Term k's E4M3 code of v (residual after the previous terms in r, updated).
__device__ __forceinline__ uint32_t et_term(float& r, int s0, int k) {
  const int sk = s0 - ET_STEP * k;
  const uint32_t c = f32_to_e4m3(r * pow2f(-sk));
  r = fmaf(-e4m3_to_f32(c), pow2f(sk), r);
  return c;
}

// x[t] (bf16) -> xe[stage][t]: per 32-element block one warp expands the
// values into ET_XTERMS E4M3 terms (lane = element); term k's codes at
// k * 128 + 32 b + lane, its scale byte at 256 + 4 k + b (b = the block in
// the stage).  Also the layer-input copy of the optional per-layer output.
__device__ void phase_images_e4m3(const EngineParams& p, const __nv_bfloat16* x, int layer) {
  const int T = p.T, H = p.H;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int64_t gt = (int64_t)blockIdx.x * THREADS + threadIdx.x;
  const int64_t gs = (int64_t)gridDim.x * THREADS;
  const int64_t wg = (int64_t)blockIdx.x * WARPS + warp, ws = (int64_t)gridDim.x * WARPS;
  const int nblk = H / 32;
  for (int64_t task = wg; task < (int64_t)T * nblk; task += ws) {
    const int t = (int)(task / nblk), gb = (int)(task % nblk);
    float r = __bfloat162float(__ldcg(x + (int64_t)t * H + gb * 32 + lane));
    float am = fabsf(r);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) am = fmaxf(am, __shfl_xor_sync(FULL, am, o));
    const int s0 = et_term0_exp(am), b = gb % KB;
    uint8_t* img = p.xe + ((int64_t)(gb / KB) * T + t) * ET_XIMG;
#pragma unroll
    for (int k = 0; k < ET_XTERMS; ++k) img[k * 128 + b * 32 + lane] = (uint8_t)et_term(r, s0, k);
    if (lane < ET_XTERMS) img[256 + 4 * lane + b] = (uint8_t)(s0 - ET_STEP * lane + 127);
  }
  if (p.layer_io) {
    const int64_t n8 = (int64_t)T * H / 8;
    const uint4* s8 = reinterpret_cast<const uint4*>(x);
    uint4* d8 = reinterpret_cast<uint4*>(p.layer_io + (int64_t)layer * T * H);
    for (int64_t i = gt; i < n8; i += gs) d8[i] = __ldcg(s8 + i);
  }
}

// Router partial logits (and the per-layer resets of the stream's counters).
// RB: 16-byte loads in flight per thread while staging (the chained-layer
// instance stages a few thousand per CTA in one or two round trips; the
// single-layer decode instance keeps its register budget with 2).  PAIR: two
// experts per warp pass in the dot products (the chained-layer instance).
template <int RB = 2, bool PAIR = false>
__device__ void phase_router(const EngineParams& p, const LayerPtrs& lp, const __nv_bfloat16* x,
                             uint8_t* smem) {
  const int T = p.T, H = p.H, E = p.E;
  const int64_t gt = (int64_t)blockIdx.x * THREADS + threadIdx.x;
  const int64_t gs = (int64_t)gridDim.x * THREADS;
  // per-layer resets of the stream's counters (used only after the next barrier)
  const int umax = max_units(E, p.TK);
  if (gt == 0) p.sync[SY_JOBS] = 0u;
  for (int64_t u = gt; u < umax; u += gs) p.sync[SY_READY + u] = 0u;

  // partial logits[hs][t][e] = sum over the hs-th H part of x[t][h] * Wr[e][h];
  // bf16 * fp32 products are exact in fp64 and the sums are fp64.  The (hs, e)
  // dot products are cut into one contiguous range per CTA (mostly a single
  // hs), so that a CTA converts its slice of x to fp64 once, in shared
  // memory, and every warp then runs one expert over all tokens of a chunk.
  const RouterWork rw = router_work(p);
  const int HS = p.HS, hpart = H / HS;
  double* xd = reinterpret_cast<double*>(ring_slot(smem, 0, 0));  // [RTC][hpart], idle ring
  // this CTA's router weight slices (one per expert it owns) are staged in
  // shared memory once and reused by every token chunk, when they fit
  float* wsm = reinterpret_cast<float*>(xd + (size_t)RTC * hpart);
  const int nexp = rw.e0 < E ? (E - rw.e0 + rw.estep - 1) / rw.estep : 0;
  const bool wstaged = ((size_t)RTC * hpart * 8 + (size_t)nexp * hpart * 4) <= RING_BYTES;
  const int hp8 = hpart / 8, hp4 = hpart / 4;  // 16-byte loads (H / HS is a multiple of 8)
  for (int hs = rw.hs0; hs < HS; hs += rw.hstep) {
    for (int t0 = 0; t0 < T; t0 += RTC) {
      const int nt = min(RTC, T - t0);
      __syncthreads();  // the previous chunk's readers are done
      // stage the chunk's x slice as fp64 and, with a part's first chunk, the
      // part's weight slices; a thread's loads are all in flight before its
      // stores (one memory round trip for both)
      const int nx = nt * hp8, nw = (t0 == 0 && wstaged) ? nexp * hp4 : 0;
#pragma unroll 1
      for (int i0 = threadIdx.x; i0 < nx + nw; i0 += RB * THREADS) {
        uint4 v[RB];
#pragma unroll
        for (int r = 0; r < RB; ++r) {
          const int i = i0 + r * THREADS;
          if (i < nx) {
            const int t = i / hp8, h8 = i - t * hp8;
            v[r] = __ldcg(reinterpret_cast<const uint4*>(x + (int64_t)(t0 + t) * H + hs * hpart) + h8);
          } else if (i < nx + nw) {
            const int k = (i - nx) / hp4, h4 = (i - nx) - k * hp4;
            v[r] = __ldg(reinterpret_cast<const uint4*>(lp.router_w + (int64_t)(rw.e0 + k * rw.estep) * H + hs * hpart) + h4);
          }
        }
#pragma unroll
        for (int r = 0; r < RB; ++r) {
          const int i = i0 + r * THREADS;
          if (i < nx) {
            const int t = i / hp8, h8 = i - t * hp8;
            double* d = xd + (size_t)t * hpart + h8 * 8;
            const uint32_t u[4] = {v[r].x, v[r].y, v[r].z, v[r].w};
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              d[2 * q] = (double)__uint_as_float(u[q] << 16);
              d[2 * q + 1] = (double)__uint_as_float(u[q] & 0xFFFF0000u);
            }
          } else if (i < nx + nw) {
            reinterpret_cast<uint4*>(wsm)[i - nx] = v[r];
          }
        }
      }
      __syncthreads();
      router_chunk<PAIR>(xd, wstaged ? wsm : nullptr, lp.router_w, nexp, rw.e0, rw.estep, H, hpart, hs, p.logits,
                   T, t0, nt, E);
    }
  }
}

// Router for large T (tile-stream launches), on the fp64 MMA path
// (mma.sync m8n8k4 f64: 256 exact fp64 FMAs from two register operands).
// Each CTA takes the same (H part, experts) share as phase_router.  Token
// chunks of RTB = 16 (two 8-row tiles) are staged as fp32 (exact for bf16) in
// two buffers, the next chunk's loads in flight while this one computes.
// Experts go in groups of 16 (two 8-column tiles).  The 12 warps split the H
// part; their partial tiles meet in shared memory and are summed in warp
// order (deterministic), then stored.
constexpr int RTB = 16, REB = 16, RXL = 6;  // RXL: 16-byte x loads per thread and chunk
static_assert(RTB * (8192 / MAX_HSPLIT / 8) <= RXL * THREADS, "chunk loads per thread");
__device__ __forceinline__ void dmma_m8n8k4(double (&c)[2], double a, double b) {
  asm("mma.sync.aligned.m8n8k4.row.col.f64.f64.f64.f64 {%0, %1}, {%2}, {%3}, {%0, %1};"
      : "+d"(c[0]), "+d"(c[1]) : "d"(a), "d"(b));
}
// (Out of line, with scalar arguments: the tile stream's code generation then
// does not depend on this phase, and the kernel's parameter block stays out of
// local memory.)
__device__ __noinline__ void phase_router_tiles(const __nv_bfloat16* x, const float* router_w,
                                                double* logits, uint32_t* sync, int T, int H, int E,
                                                int TK, int HS, uint8_t* smem) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int64_t gt = (int64_t)blockIdx.x * THREADS + threadIdx.x;
  const int64_t gs = (int64_t)gridDim.x * THREADS;
  // per-layer resets of the stream's counters (used only after the next barrier)
  const int umax = max_units(E, TK);
  if (gt == 0) sync[SY_JOBS] = 0u;
  for (int64_t u = gt; u < umax; u += gs) sync[SY_READY + u] = 0u;

  RouterWork rw;
  {
    const int g = (int)gridDim.x, c = (int)blockIdx.x;
    rw = g >= HS ? RouterWork{c % HS, HS, c / HS, (g - c % HS + HS - 1) / HS} : RouterWork{c, g, 0, 1};
  }
  const int hpart = H / HS, hp8 = hpart / 8, hp4 = hpart / 4;
  const int xstride = hpart + 4;  // the 8 rows of a tile fall in 8 different bank groups
  const int nexp = rw.e0 < E ? (E - rw.e0 + rw.estep - 1) / rw.estep : 0;
  const int ng = (nexp + REB - 1) / REB;
  // shared memory: red [WARPS][4 tiles][64] doubles, x [2][RTB][xstride], then
  // (when they fit) the part's weight rows [ng * REB][xstride]
  double* red = reinterpret_cast<double*>(ring_slot(smem, 0, 0));
  float* xs = reinterpret_cast<float*>(red + WARPS * 4 * 64);
  float* wsm = xs + 2 * RTB * xstride;
  const bool wstaged =
      (size_t)WARPS * 4 * 64 * 8 + ((size_t)2 * RTB + (size_t)ng * REB) * xstride * 4 <= RING_BYTES;
  const int nchunk = (T + RTB - 1) / RTB;
  const int g8 = lane >> 2, q4 = lane & 3;  // fragment row/column group, k within the step
  for (int hs = rw.hs0; hs < HS; hs += rw.hstep) {
    __syncthreads();  // the previous part's readers are done
    if (wstaged)
      for (int i = threadIdx.x; i < nexp * hp4; i += THREADS) {
        const int k = i / hp4, h4 = i - k * hp4;
        *reinterpret_cast<uint4*>(wsm + (size_t)k * xstride + 4 * h4) =
            __ldg(reinterpret_cast<const uint4*>(router_w + (int64_t)(rw.e0 + k * rw.estep) * H + hs * hpart) + h4);
      }
    uint4 xr[RXL];
    auto load_chunk = [&](int c) {
      const int t0 = c * RTB, nt = min(RTB, T - t0);
#pragma unroll
      for (int r = 0; r < RXL; ++r) {
        const int i = threadIdx.x + r * THREADS;
        if (i < nt * hp8) {
          const int t = i / hp8, h8 = i - t * hp8;
          xr[r] = __ldcg(reinterpret_cast<const uint4*>(x + (int64_t)(t0 + t) * H + hs * hpart) + h8);
        }
      }
    };
    auto store_chunk = [&](int c) {
      const int t0 = c * RTB, nt = min(RTB, T - t0);
      float* b = xs + (c & 1) * RTB * xstride;
#pragma unroll
      for (int r = 0; r < RXL; ++r) {
        const int i = threadIdx.x + r * THREADS;
        if (i < nt * hp8) {
          const int t = i / hp8, h8 = i - t * hp8;
          const uint32_t u[4] = {xr[r].x, xr[r].y, xr[r].z, xr[r].w};
          float4* d = reinterpret_cast<float4*>(b + (size_t)t * xstride + h8 * 8);
          d[0] = make_float4(__uint_as_float(u[0] << 16), __uint_as_float(u[0] & 0xFFFF0000u),
                             __uint_as_float(u[1] << 16), __uint_as_float(u[1] & 0xFFFF0000u));
          d[1] = make_float4(__uint_as_float(u[2] << 16), __uint_as_float(u[2] & 0xFFFF0000u),
                             __uint_as_float(u[3] << 16), __uint_as_float(u[3] & 0xFFFF0000u));
        }
      }
    };
    load_chunk(0);
    store_chunk(0);
    __syncthreads();
#pragma unroll 1
    for (int c = 0; c < nchunk; ++c) {
      const int t0 = c * RTB, nt = min(RTB, T - t0);
      const bool next = c + 1 < nchunk;
      if (next) load_chunk(c + 1);
      const float* xb = xs + (c & 1) * RTB * xstride;
#pragma unroll 1
      for (int g = 0; g < ng; ++g) {
        // operand rows of this lane: tokens g8 and 8 + g8, experts g * 16 + g8 and + 8
        const float* xa0 = xb + (size_t)g8 * xstride + q4;
        const float* xa1 = xa0 + (size_t)8 * xstride;
        const float* wb[2];
#pragma unroll
        for (int n = 0; n < 2; ++n) {
          const int k = g * REB + 8 * n + g8;
          wb[n] = wstaged ? wsm + (size_t)k * xstride + q4
                          : router_w + (int64_t)(rw.e0 + min(k, nexp - 1) * rw.estep) * H + hs * hpart + q4;
        }
        double acc[4][2] = {};
#pragma unroll 2
        for (int ks = warp; ks < hp4; ks += WARPS) {
          const int h = 4 * ks;
          const double a0 = (double)xa0[h], a1 = (double)xa1[h];
          const double b0 = (double)wb[0][h], b1 = (double)wb[1][h];
          dmma_m8n8k4(acc[0], a0, b0);
          dmma_m8n8k4(acc[1], a0, b1);
          dmma_m8n8k4(acc[2], a1, b0);
          dmma_m8n8k4(acc[3], a1, b1);
        }
        // lane l holds tile elements (row l / 4, columns 2 (l % 4) and + 1): index 2 l (+ 1) row-major
#pragma unroll
        for (int tile = 0; tile < 4; ++tile)
          *reinterpret_cast<double2*>(red + ((size_t)warp * 4 + tile) * 64 + 2 * lane) =
              make_double2(acc[tile][0], acc[tile][1]);
        __syncthreads();
        for (int o = threadIdx.x; o < 4 * 64; o += THREADS) {
          const int tile = o >> 6, r = o & 63;
          double v = 0.0;
          for (int w = 0; w < WARPS; ++w) v += red[((size_t)w * 4 + tile) * 64 + r];
          const int tl = 8 * (tile >> 1) + (r >> 3), k = g * REB + 8 * (tile & 1) + (r & 7);
          if (tl < nt && k < nexp) logits[((int64_t)hs * T + t0 + tl) * E + rw.e0 + k * rw.estep] = v;
        }
        __syncthreads();
      }
      if (next) store_chunk(c + 1);
      __syncthreads();
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

// Key order: descending key, ascending expert on equal keys.
__device__ __forceinline__ bool key_before(uint64_t ka, int ea, uint64_t kb, int eb) {
  return ka > kb || (ka == kb && ea < eb);
}
__device__ __forceinline__ void key_exchange(uint64_t& ka, int& ea, uint64_t& kb, int& eb) {
  if (key_before(kb, eb, ka, ea)) {
    const uint64_t tk = ka; ka = kb; kb = tk;
    const int te = ea; ea = eb; eb = te;
  }
}
// The best of a lane's NK keys (a pairwise tournament; on equal keys the
// lower index, which is the lower expert, wins).
template <int NK>
__device__ __forceinline__ void lane_best(const uint64_t (&key)[NK], uint64_t& best, int& bj) {
  uint64_t k[NK];
  int j[NK];
#pragma unroll
  for (int i = 0; i < NK; ++i) { k[i] = key[i]; j[i] = i; }
#pragma unroll
  for (int w = 1; w < NK; w <<= 1)
#pragma unroll
    for (int i = 0; i + w < NK; i += 2 * w)
      if (k[i + w] > k[i]) { k[i] = k[i + w]; j[i] = j[i + w]; }
  best = k[0];
  bj = j[0];
}

// One warp: logits of token t (the H-part partials summed pairwise, plus
// bias), the K largest (descending, ties to the lower expert), weights
// exp(l - lmax) / sum over the K (fp32).  Lane r < K writes slot r and, when
// `sel` is given, sets bit t of the winner's token mask sel[e * tw + t / 32].
// Expert e = lane + 32 j is key j of its lane (an order-preserving 64-bit
// image of the fp64 logit, in registers, NK >= E / 32 per lane).  Each of
// the K rounds finds the warp-wide maximum of the lanes' best keys (the lower
// expert on equal keys): one reduction of the keys' upper words, and only
// when several lanes share that word, two more.  The winning lane then moves
// to its next key: with four keys a lane keeps them sorted (five exchanges)
// and shifts; with more it rescans them (a tournament).
// (Scalar arguments: a reference to the kernel's parameter block would move
// that block to local memory for the whole kernel.)
template <int NK>
__device__ __noinline__ void topk_nk(const double* logits, int T, int E, int K, int HS,
                                     const float* bias, int t, int32_t* out_idx, float* out_w,
                                     uint32_t* sel, int tw) {
  const int lane = threadIdx.x & 31;
  uint64_t key[NK];
  // four experts per lane at a time, all their partial loads in flight at once
#pragma unroll
  for (int c = 0; c < NK / 4; ++c) {
    double part[4][MAX_HSPLIT];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int hs = 0; hs < MAX_HSPLIT; ++hs) {
        const int e = 32 * (4 * c + i) + lane;
        part[i][hs] = (hs < HS && e < E) ? __ldcg(logits + ((int64_t)hs * T + t) * E + e) : 0.0;
      }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int e = 32 * (4 * c + i) + lane;
      static_assert(MAX_HSPLIT == 8, "pairwise sum written for 8 parts");
      const double l = ((part[i][0] + part[i][1]) + (part[i][2] + part[i][3])) +
                       ((part[i][4] + part[i][5]) + (part[i][6] + part[i][7]));
      key[4 * c + i] = e < E ? order_key(bias ? l + (double)bias[e] : l) : 0ull;
    }
  }
  uint64_t best;
  int be;  // expert of `best`
  int ex[4];
  if constexpr (NK == 4) {
#pragma unroll
    for (int j = 0; j < 4; ++j) ex[j] = 32 * j + lane;
    key_exchange(key[0], ex[0], key[1], ex[1]);
    key_exchange(key[2], ex[2], key[3], ex[3]);
    key_exchange(key[0], ex[0], key[2], ex[2]);
    key_exchange(key[1], ex[1], key[3], ex[3]);
    key_exchange(key[1], ex[1], key[2], ex[2]);
    best = key[0];
    be = ex[0];
  } else {
    int bj;
    lane_best<NK>(key, best, bj);
    be = 32 * bj + lane;
  }
  int my_e = -1;
  double my_l = 0.0, lmax = 0.0;
#pragma unroll 1
  for (int r = 0; r < K; ++r) {
    const uint32_t hi = __reduce_max_sync(FULL, (uint32_t)(best >> 32));
    const uint32_t tied = __ballot_sync(FULL, (uint32_t)(best >> 32) == hi);
    uint32_t lo, esel;
    if ((tied & (tied - 1u)) == 0u) {  // one lane holds the maximum
      const int wl = __ffs(tied) - 1;
      lo = __shfl_sync(FULL, (uint32_t)best, wl);
      esel = (uint32_t)__shfl_sync(FULL, be, wl);
    } else {
      lo = __reduce_max_sync(FULL, (uint32_t)(best >> 32) == hi ? (uint32_t)best : 0u);
      const uint64_t top = ((uint64_t)hi << 32) | lo;
      esel = __reduce_min_sync(FULL, best == top ? (uint32_t)be : 0xFFFFFFFFu);
    }
    if ((uint32_t)be == esel) {  // the winner's lane moves to its next key
      if constexpr (NK == 4) {
        key[0] = key[1]; key[1] = key[2]; key[2] = key[3]; key[3] = 0ull;
        ex[0] = ex[1]; ex[1] = ex[2]; ex[2] = ex[3]; ex[3] = 0x7FFFFFFF;
        best = key[0];
        be = ex[0];
      } else {
#pragma unroll
        for (int j = 0; j < NK; ++j)
          if (32 * j + lane == be) key[j] = 0ull;
        int bj;
        lane_best<NK>(key, best, bj);
        be = 32 * bj + lane;
      }
    }
    const double v = key_value(((uint64_t)hi << 32) | lo);
    if (r == 0) lmax = v;
    if (lane == r) { my_e = (int)esel; my_l = v; }
  }
  const float w = lane < K ? expf((float)(my_l - lmax)) : 0.f;
  float sum = w;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(FULL, sum, o);
  if (lane < K) {
    out_idx[lane] = my_e;
    out_w[lane] = w / sum;
    if (sel) atomicOr(sel + my_e * tw + (t >> 5), 1u << (t & 31));
  }
}

// Top-k of token t with the smallest key list that holds E experts.
__device__ __noinline__ void topk_row(const double* logits, int T, int E, int K, int HS,
                                         const float* bias, int t, int32_t* out_idx, float* out_w,
                                         uint32_t* sel, int tw) {
  static_assert(MAX_EXPERTS == 512, "key lists of 4, 8 and 16 per lane");
  if (E <= 128) topk_nk<4>(logits, T, E, K, HS, bias, t, out_idx, out_w, sel, tw);
  else if (E <= 256) topk_nk<8>(logits, T, E, K, HS, bias, t, out_idx, out_w, sel, tw);
  else topk_nk<16>(logits, T, E, K, HS, bias, t, out_idx, out_w, sel, tw);
}

// Exclusive scan of n <= 512 ints in shared memory by one warp (in place);
// the total goes to *total.
__device__ __noinline__ void warp_exclusive_scan(int32_t* a, int n, int32_t* total) {
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

// Unit tables from per-expert counts/offsets: gate/up units of <= us
// consecutive positions of one expert's segment; the down units are the same
// ranges, each naming its gate/up unit.  scratch: 2*E ints.
__device__ __noinline__ void build_units(const int32_t* counts, const int32_t* offsets, int E, int32_t* scratch,
                            int32_t* units, int32_t* dunits, int32_t* n_units, int32_t* n_dunits, int us) {
  const int warp = threadIdx.x >> 5;
  int32_t* ubase = scratch;
  int32_t* dbase = scratch + E;
  for (int x = threadIdx.x; x < E; x += THREADS) {
    ubase[x] = (counts[x] + us - 1) / us;
    dbase[x] = (counts[x] + us - 1) / us;
  }
  __syncthreads();
  if (warp == 0) warp_exclusive_scan(ubase, E, n_units);
  if (warp == 1) warp_exclusive_scan(dbase, E, n_dunits);
  __syncthreads();
  for (int x = threadIdx.x; x < E; x += THREADS) {
    const int c = counts[x];
    for (int s = 0; s * us < c; ++s) {
      int32_t* u = units + (int64_t)(ubase[x] + s) * 4;
      u[0] = x; u[1] = offsets[x] + s * us; u[2] = min(us, c - s * us); u[3] = 0;
    }
    for (int s = 0; s * us < c; ++s) {  // down units are the gate/up units
      int32_t* u = dunits + (int64_t)(dbase[x] + s) * 4;
      u[0] = x; u[1] = offsets[x] + s * us; u[2] = min(us, c - s * us);
      u[3] = ubase[x] + s;
    }
  }
}

// Small T*K: the routing of all tokens by one CTA, into its shared-memory
// tables and the global maps at once.  Every expert keeps a mask of the
// tokens that chose it (a token chooses an expert at most once), so its count
// is the mask's population, and the stable position of pair (t, r) is the
// expert's offset plus the number of earlier tokens in its mask.  Counts and
// unit counts (ceil(count / NT_MAX)) are scanned together as one packed word.
__device__ void phase_route_small(const EngineParams& p, const LayerPtrs& lp, uint8_t* smem) {
  CtaTables& tb = tables(smem);
  const int T = p.T, E = p.E, K = p.K, TK = p.TK;
  const int warp = threadIdx.x >> 5;
  const int tw = (T + 31) >> 5;  // mask words per expert
  uint32_t* sel = reinterpret_cast<uint32_t*>(ring_slot(smem, 0, 0));  // [E][tw], idle ring
  int32_t* pk = reinterpret_cast<int32_t*>(sel + E * tw);             // [E + 1] packed counts
  for (int i = threadIdx.x; i < E * tw; i += THREADS) sel[i] = 0u;
  __syncthreads();
  for (int t = warp; t < T; t += WARPS)
    topk_row(p.logits, T, E, K, p.HS, lp.router_b, t, tb.idx + t * K, tb.w + t * K, sel, tw);
  __syncthreads();
  // per expert x (one thread each): count and unit count, packed; scanned
  // within each 32-expert chunk by its warp, then offset by the chunk totals
  int32_t* ctot = pk + MAX_EXPERTS + 1;  // [MAX_EXPERTS / 32] chunk totals
  const int lane = threadIdx.x & 31;
  int32_t vx[MAX_EXPERTS / THREADS + 1];
#pragma unroll
  for (int r = 0; r * THREADS < MAX_EXPERTS; ++r) {
    const int x = r * THREADS + threadIdx.x;
    int c = 0;
    if (x < E)
      for (int w = 0; w < tw; ++w) c += __popc(sel[x * tw + w]);
    const int32_t v = (((c + NT_MAX - 1) / NT_MAX) << 16) | c;  // c <= 256, units <= 320
    int32_t incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int32_t y = __shfl_up_sync(FULL, incl, o);
      if (lane >= o) incl += y;
    }
    vx[r] = v;
    if (x < E) pk[x] = incl - v;
    if (lane == 31 && x - 31 < E) ctot[x >> 5] = incl;
  }
  __syncthreads();
#pragma unroll
  for (int r = 0; r * THREADS < MAX_EXPERTS; ++r) {
    const int x = r * THREADS + threadIdx.x;
    if (x < E) {
      int32_t base = 0;
      for (int q = 0; q < (x >> 5); ++q) base += ctot[q];
      const int32_t ex = base + pk[x];
      pk[x] = ex;
      const int c = vx[r] & 0xFFFF, o = ex & 0xFFFF;
      tb.counts[x] = c; p.counts[x] = c;
      tb.offsets[x] = o; p.offsets[x] = o;
      if (x == E - 1) {
        const int32_t tot = ex + vx[r];
        pk[E] = tot;
        tb.offsets[E] = tot & 0xFFFF;
        p.offsets[E] = tot & 0xFFFF;
      }
    }
  }
  __syncthreads();
  for (int pr = threadIdx.x; pr < TK; pr += THREADS) {
    const int e = tb.idx[pr], t = pr / K;
    const uint32_t* m = sel + e * tw;
    int before = __popc(m[t >> 5] & ((1u << (t & 31)) - 1u));
    for (int w = 0; w < (t >> 5); ++w) before += __popc(m[w]);
    const int pos = (pk[e] & 0xFFFF) + before;
    const float wt = tb.w[pr];
    tb.perm[pos] = pr; tb.inv[pr] = pos; tb.tokpos[pos] = t; tb.wpos[pos] = wt;
    p.idx[pr] = e; p.wts[pr] = wt; p.perm[pos] = pr; p.inv[pr] = pos; p.tokpos[pos] = t; p.wpos[pos] = wt;
  }
  // gate/up units of <= NT_MAX consecutive positions of one expert's segment;
  // the down units are the same ranges, each naming its gate/up unit
  for (int x = threadIdx.x; x < E; x += THREADS) {
    const int c = pk[x + 1] - pk[x];  // packed difference: units << 16 | count
    const int n = c & 0xFFFF, off = pk[x] & 0xFFFF, ub = pk[x] >> 16;
    for (int s = 0; s * NT_MAX < n; ++s) {
      const int4 gu = make_int4(x, off + s * NT_MAX, min(NT_MAX, n - s * NT_MAX), 0);
      const int4 dn = make_int4(gu.x, gu.y, gu.z, ub + s);
      reinterpret_cast<int4*>(tb.units)[ub + s] = gu;
      reinterpret_cast<int4*>(tb.dunits)[ub + s] = dn;
      reinterpret_cast<int4*>(p.units)[ub + s] = gu;
      reinterpret_cast<int4*>(p.dunits)[ub + s] = dn;
    }
  }
  if (threadIdx.x == 0) {
    const int nu = pk[E] >> 16;
    tb.n_units = nu; tb.n_dunits = nu;
    p.n_units[0] = nu; p.n_units[1] = nu;
  }
}

// Small T*K: the grid barrier after the router phase.  The CTA that arrives
// last computes the routing once (top-k, permutation, unit tables) and
// publishes it before releasing the barrier; every other CTA then copies the
// stream's tables (a few KB) into shared memory.  One CTA reading all partial
// logits is much faster than every CTA reading them at once.  While the
// routing runs, the other CTAs write the x term images (tasks claimed from a
// counter, so that the routing CTA, which claims after it, finds them taken)
// and every CTA counts itself in sync[SY_XDONE]; the stream's producers wait
// for the full count before their first gate/up stage.  Bounded like
// grid_barrier; false on timeout or a recorded error.
__device__ bool route_barrier(const EngineParams& p, const LayerPtrs& lp, const __nv_bfloat16* x,
                              int layer, uint8_t* smem, uint32_t where, uint64_t* stamp) {
  CtaTables& tb = tables(smem);
  __syncthreads();
  if (threadIdx.x == 0) {
    // the arrival releases this CTA's partial logits and, for the last CTA,
    // acquires everyone else's
    const uint32_t gen = ld_volatile_u32(p.sync + SY_BAR_GEN);
    const uint32_t prev = atom_add_acq_rel_u32(p.sync + SY_BAR_COUNT, 1u);
    tb.last = prev == gridDim.x - 1;
    tb.gen = (int32_t)gen;
  }
  __syncthreads();
  const bool last = tb.last != 0;
  if (last) {
    phase_route_small(p, lp, smem);
    __syncthreads();
    if (threadIdx.x == 0) {
      // every CTA has arrived and touches the count again only after it sees
      // the new generation: a plain store resets it, and the release orders
      // it and all tables before that generation
      __threadfence();
      *reinterpret_cast<volatile uint32_t*>(p.sync + SY_BAR_COUNT) = 0u;
      st_release_u32(p.sync + SY_BAR_GEN, (uint32_t)tb.gen + 1u);
    }
  }
  if (!p.route_only) {
    phase_images_claimed(p, x, layer, smem);
    __syncthreads();
    if (threadIdx.x == 0) {
      __threadfence();
      atomicAdd(p.sync + SY_XDONE, 1u);
    }
  }
  if (stamp) stamp[0] = globaltimer_ns();
  int ok = 1;
  if (last) {
    if (threadIdx.x == 0 && error_set(p.sync)) ok = 0;
    if (stamp) stamp[1] = stamp[0];
    return __syncthreads_and(ok) != 0;
  }
  if (threadIdx.x == 0) {
    const uint32_t gen = (uint32_t)tb.gen;
    const uint64_t t0 = globaltimer_ns();
    uint32_t spins = 0;
    while (ld_acquire_u32(p.sync + SY_BAR_GEN) == gen) {
      if ((++spins & 15u) == 0u) {
        if (error_set(p.sync)) { ok = 0; break; }
        if (globaltimer_ns() - t0 > p.timeout_ns) { set_error(p.sync, DEV_TIMEOUT_BARRIER, where); ok = 0; break; }
      }
      __nanosleep(32);
    }
    __threadfence();
    if (ok && error_set(p.sync)) ok = 0;
  }
  if (!__syncthreads_and(ok)) return false;
  if (stamp) stamp[1] = globaltimer_ns();
  if (p.route_only) return true;
  // one round trip: every entry the tables can hold for this T*K is loaded
  // at once, the counts alongside (entries past them are never read)
  static_assert(THREADS >= SMALL_UNITS && THREADS >= SMALL_PAIRS, "one table entry per thread");
  const int i = threadIdx.x;
  const int ucap = min(max_units(p.E, p.TK), SMALL_UNITS);
  uint4 gu = {}, dn = {};
  uint32_t tp = 0, wp = 0, iv = 0;
  if (i < ucap) {
    gu = ld_cg_v4(reinterpret_cast<const uint4*>(p.units) + i);
    dn = ld_cg_v4(reinterpret_cast<const uint4*>(p.dunits) + i);
  }
  if (i < p.TK) {
    tp = ld_cg_u32(p.tokpos + i);
    wp = ld_cg_u32(p.wpos + i);
    iv = ld_cg_u32(p.inv + i);
  }
  if (i == 0) { tb.n_units = (int32_t)ld_cg_u32(p.n_units); tb.n_dunits = (int32_t)ld_cg_u32(p.n_units + 1); }
  if (i < ucap) {
    reinterpret_cast<uint4*>(tb.units)[i] = gu;
    reinterpret_cast<uint4*>(tb.dunits)[i] = dn;
  }
  if (i < p.TK) {
    tb.tokpos[i] = (int32_t)tp;
    tb.wpos[i] = __uint_as_float(wp);
    tb.inv[i] = (int32_t)iv;
  }
  __syncthreads();
  return true;
}

// Large T*K, step 1: top-k of every token, distributed over all warps.
__device__ void phase_topk_large(const EngineParams& p, const LayerPtrs& lp) {
  const int warp = threadIdx.x >> 5;
  const int64_t wg = (int64_t)blockIdx.x * WARPS + warp, ws = (int64_t)gridDim.x * WARPS;
  for (int64_t t = wg; t < p.T; t += ws)
    topk_row(p.logits, p.T, p.E, p.K, p.HS, lp.router_b, (int)t, p.idx + t * p.K, p.wts + t * p.K, nullptr, 0);
}

// Large T*K, step 2: counts/offsets in every CTA (shared-memory histogram),
// unit table by CTA 0 (units of at most `us` positions), stable positions by
// one warp per expert (ballot scan).
__device__ void phase_permute_large(const EngineParams& p, uint8_t* smem, int us) {
  CtaTables& tb = tables(smem);
  const int E = p.E, K = p.K, TK = p.TK;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  for (int i = threadIdx.x; i < E; i += THREADS) tb.counts[i] = 0;
  __syncthreads();
  for (int i = threadIdx.x; i < TK; i += THREADS) atomicAdd(&tb.counts[__ldcg(p.idx + i)], 1);
  __syncthreads();
  for (int i = threadIdx.x; i < E; i += THREADS) tb.offsets[i] = tb.counts[i];
  __syncthreads();
  if (warp == 0) warp_exclusive_scan(tb.offsets, E, tb.offsets + E);
  __syncthreads();
  if (blockIdx.x == 0) {
    int32_t* scratch = reinterpret_cast<int32_t*>(ring_slot(smem, 0, 0));
    build_units(tb.counts, tb.offsets, E, scratch, p.units, p.dunits, &tb.n_units, &tb.n_dunits, us);
    for (int i = threadIdx.x; i < E; i += THREADS) p.counts[i] = tb.counts[i];
    for (int i = threadIdx.x; i <= E; i += THREADS) p.offsets[i] = tb.offsets[i];
    if (threadIdx.x == 0) { p.n_units[0] = tb.n_units; p.n_units[1] = tb.n_dunits; }
  }
  const int64_t wg = (int64_t)blockIdx.x * WARPS + warp, ws = (int64_t)gridDim.x * WARPS;
  for (int64_t x = wg; x < E; x += ws) {
    int run = tb.offsets[x];
    for (int base = 0; base < TK; base += 32) {
      const int pr = base + lane;
      const bool hit = pr < TK && __ldcg(p.idx + pr) == (int)x;
      const uint32_t b = __ballot_sync(FULL, hit);
      if (hit) {
        const int pos = run + __popc(b & ((1u << lane) - 1u));
        p.perm[pos] = pr; p.inv[pr] = pos; p.tokpos[pos] = pr / K; p.wpos[pos] = __ldcg(p.wts + pr);
      }
      run += __popc(b);
    }
  }
}

// Big units: the x image of every (stage, permuted position), copied from
// its token's image, so that a unit's B operand is one contiguous run of
// positions (one bulk copy per stage).  In the scale row r of position j < 4
// of a unit, bytes 4..7 take the scale bytes of row r of position j + 4 when
// the unit has it (B row 32 + 8 j + r's scales, for tensor-memory column 5).
// A warp moves one (unit, stage): 40 16-byte chunks per position (32 of
// codes, then the 8 scale rows), eight chunks per lane in flight.
__device__ void phase_pos_gather(const EngineParams& p) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  constexpr int CPP = IMG_BYTES / 16, CCODE = IMG_CODE_BYTES / 16;
  const int ns = p.H / KS, nu = ld_cg_u32(p.n_units);
  const int64_t ntask = (int64_t)nu * ns;
  for (int64_t us = (int64_t)blockIdx.x * WARPS + warp; us < ntask; us += (int64_t)gridDim.x * WARPS) {
    const int u = (int)(us / ns), st = (int)(us % ns);
    const int4 ur = __ldcg(reinterpret_cast<const int4*>(p.units) + u);
    const int pos0 = ur.y, n = ur.z;  // n <= NT_BIG
    const int tok = lane < n ? __ldcg(p.tokpos + pos0 + lane) : 0;
    const uint8_t* xs = p.xt + (int64_t)st * p.T * IMG_BYTES;
    uint4* dst = reinterpret_cast<uint4*>(p.xp + ((int64_t)st * p.TK + pos0) * IMG_BYTES);
    constexpr int B8 = 8;
    for (int f0 = 0; f0 < n * CPP; f0 += 32 * B8) {
      uint4 v[B8];
#pragma unroll
      for (int i = 0; i < B8; ++i) {
        const int f = f0 + 32 * i + lane, j = f / CPP, ch = f - j * CPP;
        const int tj = __shfl_sync(FULL, tok, j & 7), tp = __shfl_sync(FULL, tok, (j + NT_MAX) & 7);
        if (f < n * CPP) {
          v[i] = __ldcg(reinterpret_cast<const uint4*>(xs + (int64_t)tj * IMG_BYTES) + ch);
          if (ch >= CCODE && j < NT_MAX && j + NT_MAX < n)  // the partner's scale bytes of this row
            v[i].y = __ldcg(reinterpret_cast<const uint32_t*>(xs + (int64_t)tp * IMG_BYTES + 16 * ch));
        }
      }
#pragma unroll
      for (int i = 0; i < B8; ++i) {
        const int f = f0 + 32 * i + lane;
        if (f < n * CPP) dst[f] = v[i];
      }
    }
  }
}

// Large T*K: the x term images of every tile, gathered from the per-token
// images: the first LT_NTERM term rows of each position (row k of a token's
// image becomes B row LT_NTERM * tl + k) and their scale words.  A warp moves
// one (tile, stage): its 16-byte chunks (position, term, K chunk) and scale
// words spread over the lanes, eight chunk loads of a lane in flight at once.
__device__ void phase_tile_gather(const EngineParams& p) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int ns = p.H / KS, nu = ld_cg_u32(p.n_units);
  constexpr int CPP = LT_NTERM * 4;  // 16-byte chunks per position
  const int64_t ntask = (int64_t)nu * ns;
  for (int64_t us = (int64_t)blockIdx.x * WARPS + warp; us < ntask; us += (int64_t)gridDim.x * WARPS) {
    const int u = (int)(us / ns), st = (int)(us % ns);
    const int4 ur = __ldcg(reinterpret_cast<const int4*>(p.units) + u);
    const int n = ur.z;
    static_assert(LT_MAX <= 64, "two token words per lane");
    const int tok0 = lane < n ? __ldcg(p.tokpos + ur.y + lane) : 0;
    const int tok1 = lane + 32 < n ? __ldcg(p.tokpos + ur.y + lane + 32) : 0;
    const uint8_t* xs = p.xt + (int64_t)st * p.T * IMG_BYTES;
    uint8_t* dst = p.xtl + us * LT_IMG_BYTES;
    constexpr int B8 = 8;
    for (int f0 = 0; f0 < n * CPP; f0 += 32 * B8) {
      uint4 v[B8];
#pragma unroll
      for (int i = 0; i < B8; ++i) {
        const int f = f0 + 32 * i + lane, tl = f / CPP, r = f - tl * CPP, k = r >> 2, kch = r & 3;
        const int ta = __shfl_sync(FULL, tok0, tl & 31), tb = __shfl_sync(FULL, tok1, tl & 31);
        if (f < n * CPP)
          v[i] = __ldcg(reinterpret_cast<const uint4*>(xs + (int64_t)(tl < 32 ? ta : tb) * IMG_BYTES + kch * 128 + k * 16));
      }
#pragma unroll
      for (int i = 0; i < B8; ++i) {
        const int f = f0 + 32 * i + lane, tl = f / CPP, r = f - tl * CPP, k = r >> 2, kch = r & 3;
        if (f < n * CPP) *reinterpret_cast<uint4*>(dst + lt_row_offset(LT_NTERM * tl + k) + kch * 128) = v[i];
      }
    }
    for (int f0 = 0; f0 < n * LT_NTERM; f0 += 32) {  // scale words: (position, term)
      const int f = f0 + lane, tl = f / LT_NTERM, k = f - tl * LT_NTERM;
      const int ta = __shfl_sync(FULL, tok0, tl & 31), tb = __shfl_sync(FULL, tok1, tl & 31);
      if (f < n * LT_NTERM) {
        const uint32_t w = __ldcg(reinterpret_cast<const uint32_t*>(xs + (int64_t)(tl < 32 ? ta : tb) * IMG_BYTES +
                                                                   IMG_CODE_BYTES + k * 16));
        *reinterpret_cast<uint32_t*>(dst + lt_sf_offset(f, 0)) = w;
      }
    }
  }
}

// Large T*K, E4M3 tiles: the x image of every (tile, stage), gathered from the
// per-token images: term k of position tl is B row n = ET_XTERMS tl + k (its
// 128 codes as eight 16-byte chunks at et_code_offset(n, 16 c, N)), its scale
// word at lt_sf_offset(n, 0).  A warp moves one (tile, stage).
__device__ void phase_tile_gather_e4m3(const EngineParams& p) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int ns = p.H / KS, nu = ld_cg_u32(p.n_units);
  constexpr int CPP = ET_XTERMS * 8;  // 16-byte chunks per position
  const int64_t ntask = (int64_t)nu * ns;
  for (int64_t us = (int64_t)blockIdx.x * WARPS + warp; us < ntask; us += (int64_t)gridDim.x * WARPS) {
    const int u = (int)(us / ns), st = (int)(us % ns);
    const int4 ur = __ldcg(reinterpret_cast<const int4*>(p.units) + u);
    const int n = ur.z, N = et_cols(n, ET_XTERMS);
    static_assert(ET_MAX <= 64, "two token words per lane");
    const int tok0 = lane < n ? __ldcg(p.tokpos + ur.y + lane) : 0;
    const int tok1 = lane + 32 < n ? __ldcg(p.tokpos + ur.y + lane + 32) : 0;
    const uint8_t* xs = p.xe + (int64_t)st * p.T * ET_XIMG;
    uint8_t* dst = p.xte + us * ET_XB_BYTES;
    constexpr int B8 = 8;
    for (int f0 = 0; f0 < n * CPP; f0 += 32 * B8) {
      uint4 v[B8];
#pragma unroll
      for (int i = 0; i < B8; ++i) {
        const int f = f0 + 32 * i + lane, tl = f / CPP, r = f - tl * CPP, k = r >> 3, c = r & 7;
        const int ta = __shfl_sync(FULL, tok0, tl & 31), tb = __shfl_sync(FULL, tok1, tl & 31);
        if (f < n * CPP)
          v[i] = __ldcg(reinterpret_cast<const uint4*>(xs + (int64_t)(tl < 32 ? ta : tb) * ET_XIMG + k * 128 + c * 16));
      }
#pragma unroll
      for (int i = 0; i < B8; ++i) {
        const int f = f0 + 32 * i + lane, tl = f / CPP, r = f - tl * CPP, k = r >> 3, c = r & 7;
        if (f < n * CPP) *reinterpret_cast<uint4*>(dst + et_code_offset(ET_XTERMS * tl + k, 16 * c, N)) = v[i];
      }
    }
    for (int f0 = 0; f0 < n * ET_XTERMS; f0 += 32) {  // scale words: (position, term)
      const int f = f0 + lane, tl = f / ET_XTERMS, k = f - tl * ET_XTERMS;
      const int ta = __shfl_sync(FULL, tok0, tl & 31), tb = __shfl_sync(FULL, tok1, tl & 31);
      if (f < n * ET_XTERMS) {
        const uint32_t w =
            __ldcg(reinterpret_cast<const uint32_t*>(xs + (int64_t)(tl < 32 ? ta : tb) * ET_XIMG + 256 + 4 * k));
        *reinterpret_cast<uint32_t*>(dst + lt_sf_offset(f, 0)) = w;
      }
    }
  }
}

// ---- bf16 tile stream: permutation into balanced tiles, gather of x ------------------------
// Unit tables of the bf16 tile stream: an expert's segment of c positions
// becomes nb = ceil(c / FT_MAX) tiles of c / nb or c / nb + 1 consecutive
// positions (the larger ones first); the down units are the same tiles, each
// naming itself.  scratch: E ints.
__device__ __noinline__ void build_ftiles(const int32_t* counts, const int32_t* offsets, int E, int32_t* scratch,
                                          int32_t* units, int32_t* dunits, int32_t* n_units, int32_t* n_dunits) {
  const int warp = threadIdx.x >> 5;
  for (int x = threadIdx.x; x < E; x += THREADS) scratch[x] = (counts[x] + FT_MAX - 1) / FT_MAX;
  __syncthreads();
  if (warp == 0) warp_exclusive_scan(scratch, E, n_units);
  __syncthreads();
  if (threadIdx.x == 0) *n_dunits = *n_units;
  for (int x = threadIdx.x; x < E; x += THREADS) {
    const int c = counts[x];
    const int nb = (c + FT_MAX - 1) / FT_MAX;
    if (nb == 0) continue;
    const int base = c / nb, rem = c % nb;
    int pos = offsets[x];
    for (int s = 0; s < nb; ++s) {
      const int n = base + (s < rem ? 1 : 0);
      const int u = scratch[x] + s;
      int32_t* g = units + (int64_t)u * 4;
      g[0] = x; g[1] = pos; g[2] = n; g[3] = 0;
      int32_t* d = dunits + (int64_t)u * 4;
      d[0] = x; d[1] = pos; d[2] = n; d[3] = u;
      pos += n;
    }
  }
}

// Large T*K, bf16 tiles, step 2: as phase_permute_large, with balanced tiles.
__device__ void phase_permute_f16(const EngineParams& p, uint8_t* smem) {
  CtaTables& tb = tables(smem);
  const int E = p.E, K = p.K, TK = p.TK;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  for (int i = threadIdx.x; i < E; i += THREADS) tb.counts[i] = 0;
  __syncthreads();
  for (int i = threadIdx.x; i < TK; i += THREADS) atomicAdd(&tb.counts[__ldcg(p.idx + i)], 1);
  __syncthreads();
  for (int i = threadIdx.x; i < E; i += THREADS) tb.offsets[i] = tb.counts[i];
  __syncthreads();
  if (warp == 0) warp_exclusive_scan(tb.offsets, E, tb.offsets + E);
  __syncthreads();
  if (blockIdx.x == 0) {
    int32_t* scratch = reinterpret_cast<int32_t*>(ring_slot(smem, 0, 0));
    build_ftiles(tb.counts, tb.offsets, E, scratch, p.units, p.dunits, &tb.n_units, &tb.n_dunits);
    __syncthreads();
    for (int i = threadIdx.x; i < E; i += THREADS) p.counts[i] = tb.counts[i];
    for (int i = threadIdx.x; i <= E; i += THREADS) p.offsets[i] = tb.offsets[i];
    if (threadIdx.x == 0) { p.n_units[0] = tb.n_units; p.n_units[1] = tb.n_dunits; }
  }
  const int64_t wg = (int64_t)blockIdx.x * WARPS + warp, ws = (int64_t)gridDim.x * WARPS;
  for (int64_t x = wg; x < E; x += ws) {
    int run = tb.offsets[x];
    for (int base = 0; base < TK; base += 32) {
      const int pr = base + lane;
      const bool hit = pr < TK && __ldcg(p.idx + pr) == (int)x;
      const uint32_t b = __ballot_sync(FULL, hit);
      if (hit) {
        const int pos = run + __popc(b & ((1u << lane) - 1u));
        p.perm[pos] = pr; p.inv[pr] = pos; p.tokpos[pos] = pr / K; p.wpos[pos] = __ldcg(p.wts + pr);
      }
      run += __popc(b);
    }
  }
}

// Large T*K, bf16 tiles: the B block of every (tile, 64-K half-stage) of the
// gate/up projection, gathered from the bf16 rows of x.  A warp moves one
// (tile, half-stage): 8 lanes per position (16 bytes = 8 elements along K
// each), four positions per step and eight steps of loads in flight.
__device__ void phase_tile_gather_f16(const EngineParams& p, const __nv_bfloat16* x) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int ns = p.H / FT_HK, nu = ld_cg_u32(p.n_units);
  const int sub = lane >> 3, ch = lane & 7;  // position within a step of 4, chunk along K
  const int64_t ntask = (int64_t)nu * ns;
  for (int64_t us = (int64_t)blockIdx.x * WARPS + warp; us < ntask; us += (int64_t)gridDim.x * WARPS) {
    const int u = (int)(us / ns), st = (int)(us % ns);
    const int4 ur = __ldcg(reinterpret_cast<const int4*>(p.units) + u);
    const int n = ur.z, rows = (n + 15) & ~15;
    int tok[FT_MAX / 32];
#pragma unroll
    for (int i = 0; i < FT_MAX / 32; ++i) tok[i] = lane + 32 * i < n ? __ldcg(p.tokpos + ur.y + lane + 32 * i) : 0;
    uint8_t* dst = p.xtf + us * FT_TERM_BYTES;
    constexpr int STEPS = 8;
    for (int tl0 = 0; tl0 < n; tl0 += 4 * STEPS) {
      uint4 v[STEPS];
#pragma unroll
      for (int i = 0; i < STEPS; ++i) {
        const int tl = tl0 + 4 * i + sub;
        int t = 0;
#pragma unroll
        for (int q = 0; q < FT_MAX / 32; ++q) {
          const int tq = __shfl_sync(FULL, tok[q], tl & 31);
          if ((tl >> 5) == q) t = tq;
        }
        if (tl < n) v[i] = __ldcg(reinterpret_cast<const uint4*>(x + (int64_t)t * p.H + st * FT_HK) + ch);
      }
#pragma unroll
      for (int i = 0; i < STEPS; ++i) {
        const int tl = tl0 + 4 * i + sub;
        if (tl < n) *reinterpret_cast<uint4*>(dst + ft_b_offset(tl, 8 * ch, rows)) = v[i];
      }
    }
  }
}

// ---- phase C: the MXFP4 weight stream on tensor cores --------------------------------------
struct StreamCtx {
  const int32_t* units;   // gate/up units
  const int32_t* dunits;  // down units
  const int32_t* tokpos;
  const float* wpos;
  int n_units, n_dunits;
  bool global;            // tables in global memory (written in this launch: read through L2)
};

// Table read: shared memory, or global memory bypassing the (non-coherent) L1.
template <class V>
__device__ __forceinline__ V ld_tab(const V* ptr, bool global) { return global ? __ldcg(ptr) : *ptr; }

// Per-thread pipeline positions, continued across layers.
struct RoleState {
  uint32_t seq = 0;  // producer: stage sequence number
  int32_t qk = 0;    // job queue position (every role reads every entry)
  int32_t wj = 0;    // producer: next work index
  uint32_t sfc = 0;  // MMA issuer: scale-factor buffer counter
  uint32_t gcount = 0;  // epilogue warp: gate/up jobs done (amax exchange buffer and phase)
};

// Bounded wait for queue entry qk; false on timeout or a recorded error.
__device__ bool wait_entry(const EngineParams& p, JobEntry* en, int32_t qk) {
  if (*reinterpret_cast<volatile int32_t*>(&en->flag) == qk + 1) return true;
  const uint64_t t0 = globaltimer_ns();
  uint32_t spins = 0;
  while (*reinterpret_cast<volatile int32_t*>(&en->flag) != qk + 1) {
    if ((++spins & 15u) == 0u) {
      if (error_set(p.sync)) return false;
      if (globaltimer_ns() - t0 > 2 * p.timeout_ns) { set_error(p.sync, DEV_TIMEOUT_QUEUE, qk); return false; }
    }
    __nanosleep(32);
  }
  return true;
}

// Producer warp: jobs -> queue entries -> stages into the ring.  Gate/up jobs
// (unit, 64-row block of I) come first in unit order, then down jobs (down
// unit, 128-row block of H); a down job waits until its gate/up unit's SwiGLU
// term images are complete.  A stage is the job's weight stage plus one term
// image per token (gate/up, from xt), the unit's gathered position images
// (gate/up of big units, from xp) or the unit's consecutive pair images
// (down, from aimg).
// SPLIT (operator-by-operator launches only): 1 runs the gate/up jobs alone, 2
// the down jobs alone (their gate/up units are then complete).
template <int TM, int SPLIT = 0>
__device__ void stream_producer(const EngineParams& p, const LayerPtrs& lp, uint8_t* smem,
                                const StreamCtx& cx, int pipe, RoleState& rs) {
  constexpr bool LT = TM == 1 || TM == 4 || TM == 6;  // tile modes (TM 0, 7: the pipeline stream)
  constexpr int NS = TM == 1 ? LT_NSLOT : TM == 4 ? LTA_NSLOT : TM == 6 ? ET_NSLOT : TM == 7 ? NSLOT_BIG : NSLOT;
  constexpr int SLOTB = TM == 1   ? LT_SLOT_BYTES
                        : TM == 4 ? LTA_SLOT_BYTES
                        : TM == 6 ? ET_SLOT_BYTES
                        : TM == 7 ? SLOT_BYTES_BIG
                                  : SLOT_BYTES;
  constexpr int R = TM == 4 ? LTA_R : 1;      // row blocks per job
  constexpr int NP = LT ? 1 : NPIPE;         // pipelines per CTA
  constexpr int PB = PRODUCER_BATCH < NS ? PRODUCER_BATCH : NS;
  const int lane = threadIdx.x & 31;
  JobEntry* jq = job_queue(smem, pipe);
  uint32_t* ready = p.sync + SY_READY;
  const int gub = p.I / GU_I_ROWS, db = p.H / JOB_ROWS;
  const int gpu_ = gub / R, dpu = db / R;    // jobs per unit
  const int64_t n_gu = (int64_t)cx.n_units * gpu_;
  const int64_t n_all = SPLIT == 1 ? n_gu : n_gu + (int64_t)cx.n_dunits * dpu;
  const int64_t j0 = SPLIT == 2 ? n_gu : 0;  // first job of this launch
  const int nc_gu = p.H / KS, nc_d = p.I / KS;
  const uint32_t need = (uint32_t)gpu_ * (LT ? 8u : 4u);  // readiness signals per gate/up unit: epilogue warps per job
  bool xwait = !LT && !cx.global;  // x term images written during the routing (small T*K)
  // Units of at most NT_MAX positions read most expert weights once: the
  // weight stages go to L2 as evict-first, so that the routing's working set
  // (code, router weights, activations, tables) stays in L2 across launches.
  // Tiles re-read each expert's weights once per tile and keep the default.
  const uint64_t wpolicy = LT ? 0ull : l2_evict_first();
  const uint32_t seq_start = rs.seq;
  bool ok = true;
  unsigned long long t_empty = 0, t_ready = 0;
  const unsigned long long t_begin = clock64();
  fence_proxy_async_global();
  // the first job of every pipeline is static (no atomic round trip at the
  // start of the stream); later jobs come from the global counter
  const int64_t jbase = j0 + (int64_t)NP * gridDim.x;
  long long next = j0 + (int64_t)blockIdx.x + (int64_t)pipe * gridDim.x;
  for (;;) {
    const int64_t j = __shfl_sync(FULL, next, 0);
    if (j >= n_all || !ok) {
      if (lane == 0) {
        JobEntry* en = jq + (rs.qk % JQ);
        en->job = -1; en->s0 = (int32_t)rs.seq; en->nc = 0;
        __threadfence_block();
        *reinterpret_cast<volatile int32_t*>(&en->flag) = rs.qk + 1;
      }
      ++rs.qk;
      break;
    }
    if (lane == 0) next = jbase + atomicAdd(p.sync + (SPLIT == 2 ? SY_JOBS2 : SY_JOBS), 1u);  // prefetch the following job
    const bool isD = j >= n_gu;
    const int64_t jj = isD ? j - n_gu : j;
    const int per = isD ? dpu : gpu_;
    const int u = (int)(jj / per), rb = (int)(jj % per) * R;  // first row block of the job
    const int4 ur = ld_tab(reinterpret_cast<const int4*>((isD ? cx.dunits : cx.units) + (int64_t)u * 4), cx.global);
    const int e = ur.x, pos0 = ur.y, nt = ur.z;
    const int nc = isD ? nc_d : nc_gu;
    if (isD) {  // the down stages read the SwiGLU term images: wait for the gate/up unit
      const int gu = ur.w;
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
      fence_proxy_async_global();  // the images were written by generic stores of other CTAs
    }
    if (!isD && xwait) {  // every CTA's x images, before the first gate/up stage
      xwait = false;
      const unsigned long long tr0 = clock64();
      if (lane == 0 && ld_acquire_u32(p.sync + SY_XDONE) < gridDim.x) {
        const uint64_t t0 = globaltimer_ns();
        uint32_t spins = 0;
        while (ld_acquire_u32(p.sync + SY_XDONE) < gridDim.x) {
          if ((++spins & 15u) == 0u) {
            if (error_set(p.sync)) { ok = false; break; }
            if (globaltimer_ns() - t0 > p.timeout_ns) { set_error(p.sync, DEV_TIMEOUT_IMAGES, (uint32_t)j); ok = false; break; }
          }
          __nanosleep(32);
        }
      }
      ok = __shfl_sync(FULL, ok, 0);
      __syncwarp();  // orders lane 0's acquire before every lane's copies
      t_ready += clock64() - tr0;
      if (!ok) continue;  // publishes the end entry
      fence_proxy_async_global();  // the images were written by generic stores of other CTAs
    }
    if (lane == 0) {
      JobEntry* en = jq + (rs.qk % JQ);
      en->job = (int32_t)j; en->s0 = (int32_t)rs.seq; en->nc = nc; en->unit = u; en->rb = rb;
      en->isD = isD; en->e = e; en->pos0 = pos0; en->nt = nt; en->wj = rs.wj;
      __threadfence_block();
      *reinterpret_cast<volatile int32_t*>(&en->flag) = rs.qk + 1;
    }
    ++rs.qk;
    ++rs.wj;
    const uint8_t* wbase = isD ? lp.w_d + ((int64_t)e * db + rb) * nc * STAGE_A_BYTES
                               : lp.w_gu + ((int64_t)e * gub + rb) * nc * STAGE_A_BYTES;
    const int tok = (!LT && TM != 7 && !isD && lane < nt) ? ld_tab(cx.tokpos + pos0 + lane, cx.global) : 0;
    const uint32_t bbytes = TM == 6 ? (uint32_t)et_img_bytes(et_cols(nt, isD ? ET_ATERMS : ET_XTERMS))
                            : LT    ? (uint32_t)(LT_SF_BYTES + lt_cols(nt) * (IMG_CODE_BYTES / 8))
                                    : (uint32_t)nt * IMG_BYTES;
    const uint32_t stage_bytes = R * STAGE_A_BYTES + bbytes;
    const int64_t rstep = (int64_t)nc * STAGE_A_BYTES;  // between the stages of consecutive row blocks
    // Stages are issued in batches, one stage per lane: successive 1-D bulk
    // copies issued by one warp instruction each are serialised, while the
    // copies of one instruction proceed in parallel.  A batch is the run of
    // consecutive stages whose slots are already free (non-blocking test), so
    // the ring refills as soon as the MMAs release slots and the batch grows
    // whenever the producer falls behind.
    int c0 = 0;
    while (c0 < nc && ok) {
      const int nb = min(PB, nc - c0);
      const uint32_t s = rs.seq + lane;
      const int slot = (int)(s % NS);
      const uint32_t par = ((s / NS) + 1) & 1u;  // completion of the slot's previous use
      const bool fr = lane < nb && (s < (uint32_t)NS || mbar_test_wait(empty_bar(smem, pipe, slot), par));
      const int k = __ffs(~__ballot_sync(FULL, fr)) - 1;  // leading run of free slots
      if (k == 0) {
        const unsigned long long te0 = clock64();
        bool bad = false;
        if (lane == 0) bad = !wait_mbar(empty_bar(smem, pipe, slot), par, p.sync, p.timeout_ns, DEV_TIMEOUT_PIPE, s);
        t_empty += clock64() - te0;
        if (__any_sync(FULL, bad)) ok = false;
        continue;
      }
      uint8_t* dst = smem + OFF_RING + ((size_t)(LT ? 0 : pipe) * NS + slot) * SLOTB;
      uint64_t* fb = full_bar(smem, pipe, slot);
      const int c = c0 + lane;
      if (lane < k) {
        mbar_arrive_expect_tx(fb, stage_bytes);
        if constexpr (LT) {
#pragma unroll
          for (int r = 0; r < R; ++r)
            bulk_g2s(dst + r * STAGE_A_BYTES, wbase + r * rstep + (int64_t)c * STAGE_A_BYTES, STAGE_A_BYTES, fb);
        } else {
          bulk_g2s_hint(dst, wbase + (int64_t)c * STAGE_A_BYTES, STAGE_A_BYTES, fb, wpolicy);
        }
        if (LT)  // the tile's B operand of this stage, one image
          bulk_g2s(dst + R * STAGE_A_BYTES,
                   TM == 6 ? (isD ? p.ate + ((int64_t)u * nc + c) * ET_AB_BYTES : p.xte + ((int64_t)u * nc + c) * ET_XB_BYTES)
                           : (isD ? p.atl : p.xtl) + ((int64_t)u * nc + c) * LT_IMG_BYTES,
                   bbytes, fb);
        else if (isD)
          bulk_g2s(dst + STAGE_A_BYTES, p.aimg + ((int64_t)c * p.TK + pos0) * IMG_BYTES,
                   (uint32_t)nt * IMG_BYTES, fb);
      }
      if (TM == 7 && !isD) {  // big units: the unit's gathered positions, one copy
        if (lane < k)
          bulk_g2s(dst + STAGE_A_BYTES, p.xp + ((int64_t)c * p.TK + pos0) * IMG_BYTES, (uint32_t)nt * IMG_BYTES, fb);
      } else if (!LT && !isD) {
        for (int tl = 0; tl < nt; ++tl) {
          const int tk = __shfl_sync(FULL, tok, tl);
          if (lane < k)
            bulk_g2s(dst + STAGE_A_BYTES + tl * IMG_BYTES, p.xt + ((int64_t)c * p.T + tk) * IMG_BYTES,
                     IMG_BYTES, fb);
        }
      }
      rs.seq += k;
      c0 += k;
    }
  }
  if (p.prof && lane == 0) {
    atomicAdd(p.prof + PF_PROD_EMPTY, t_empty);
    atomicAdd(p.prof + PF_PROD_READY, t_ready);
    atomicAdd(p.prof + PF_PROD_TOTAL, clock64() - t_begin);
    atomicAdd(p.prof + PF_STAGES, (unsigned long long)(rs.seq - seq_start));
  }
  // let every issued copy land before the ring is reused or the CTA exits
  const uint32_t issued = rs.seq - seq_start;
  const uint32_t n = issued < (uint32_t)NS ? issued : (uint32_t)NS;
  for (uint32_t s = rs.seq - n; s != rs.seq; ++s) {
    const uint64_t t0 = globaltimer_ns();
    while (!mbar_try_wait(full_bar(smem, pipe, (int)(s % NS)), (s / NS) & 1u)) {
      if (globaltimer_ns() - t0 > DRAIN_NS) break;
    }
  }
}

// MMA issuer (one thread): per stage, the weight and activation scale factors
// go to tensor memory and two block-scaled MMAs (K = 64 each, N = 8 columns
// per token or pair) accumulate into the job's tensor-memory buffer; the slot
// is released by a commit when they complete.
template <int U = NT_MAX>
__device__ void stream_mma(const EngineParams& p, uint8_t* smem, uint32_t tmem, int pipe, RoleState& rs) {
  using C = PipeCfg<U>;
  JobEntry* jq = job_queue(smem, pipe);
  const uint32_t ring0 = pipe_ring<U>(smem, pipe);
  const bool prof = p.prof != nullptr;
  unsigned long long t_full = 0, t_issue = 0, t_acc = 0;
  bool ok = true;
  for (;;) {
    JobEntry* en = jq + (rs.qk % JQ);
    if (!wait_entry(p, en, rs.qk)) return;
    const int job = *reinterpret_cast<volatile int32_t*>(&en->job);
    if (job < 0) { ++rs.qk; break; }
    const int s0 = en->s0, nc = en->nc, nt = en->nt, wj = en->wj;
    ++rs.qk;
    if (!ok) continue;
    const int b = wj % NACC;
    const uint32_t use = (uint32_t)(wj / NACC);
    const unsigned long long ta0 = pclock(prof);
    if (use > 0 &&
        !wait_mbar(acce_bar(smem, pipe, b), (use - 1) & 1u, p.sync, p.timeout_ns, DEV_TIMEOUT_PIPE, wj)) {
      ok = false;
      continue;
    }
    t_acc += pclock(prof) - ta0;
    tc_fence_after();
    const uint32_t tacc = tmem + pipe_acc<U>(pipe, b);
    const uint32_t idesc0 = mxf4_idesc(nt * NTERM, 0u), idesc1 = mxf4_idesc(nt * NTERM, 2u);
    for (int c = 0; c < nc; ++c) {
      const uint32_t s = (uint32_t)s0 + c;
      const int slot = (int)(s % C::NS);
      const unsigned long long tf0 = pclock(prof);
      if (!wait_mbar(full_bar(smem, pipe, slot), (s / C::NS) & 1u, p.sync, p.timeout_ns, DEV_TIMEOUT_PIPE, s)) {
        ok = false;
        break;
      }
      const unsigned long long tm0 = pclock(prof);
      t_full += tm0 - tf0;
      const uint32_t sa = ring0 + (uint32_t)slot * C::SLOTB, sb = sa + STAGE_A_BYTES;
      const uint32_t tsf = tmem + pipe_sf<U>(pipe, (int)(rs.sfc++ % NSF));
      tmem_cp_sf(tsf, smem_desc(sa + STAGE_CODE_BYTES, 0, 128));
      tmem_cp_sf(tsf + 4, smem_desc(sb + IMG_CODE_BYTES, 0, IMG_BYTES));
      mma_mxf4(tacc, smem_desc(sa, 128, 256), smem_desc(sb, 128, IMG_BYTES), idesc0, tsf, tsf + 4,
               c > 0 ? 1u : 0u);
      mma_mxf4(tacc, smem_desc(sa + 4096, 128, 256), smem_desc(sb + 256, 128, IMG_BYTES), idesc1,
               tsf | (2u << 30), (tsf + 4) | (2u << 30), 1u);
      tc_commit(empty_bar(smem, pipe, slot));
      t_issue += pclock(prof) - tm0;
    }
    if (ok) tc_commit(accf_bar(smem, pipe, b));
  }
  if (prof) {
    atomicAdd(p.prof + PF_MMA_FULL, t_full);
    atomicAdd(p.prof + PF_MMA_ISSUE, t_issue);
    atomicAdd(p.prof + PF_MMA_ACC, t_acc);
  }
}

// Epilogue of pipeline `pipe` (four warps, warp q = warp % 4 reading
// tensor-memory lanes 32q..32q+31).
//   gate/up: lane l of warp q holds gate (l < 16) or up (l >= 16) of
//     intermediate row i0 + 16 q + l % 16 for every token column group;
//     a = silu(g) u, then its E2M1 term image (block amax shared by warps q,
//     q ^ 1 through shared memory) goes to aimg and the unit's readiness
//     counter is incremented once per warp.
//   down: row h0 + 32 q + l of every pair, times the routing weight -> ypair.
template <int U = NT_MAX>
__device__ void stream_epilogue(const EngineParams& p, uint8_t* smem, const StreamCtx& cx,
                                uint32_t tmem, int pipe, RoleState& rs) {
  const int lane = threadIdx.x & 31, q = (threadIdx.x >> 5) & 3;
  JobEntry* jq = job_queue(smem, pipe);
  uint32_t* ready = p.sync + SY_READY;
  const bool prof = p.prof != nullptr;
  unsigned long long t_wait = 0, t_work = 0, n_jobs = 0;
  const unsigned long long t_begin = pclock(prof);
  bool ok = true;
  for (;;) {
    JobEntry* en = jq + (rs.qk % JQ);
    if (!wait_entry(p, en, rs.qk)) return;
    const int job = *reinterpret_cast<volatile int32_t*>(&en->job);
    if (job < 0) { ++rs.qk; break; }
    const int wj = en->wj;
    const int u = en->unit, rb = en->rb, isD = en->isD, pos0 = en->pos0, nt = en->nt;
    ++rs.qk;
    if (!ok) continue;
    ++n_jobs;
    const uint32_t gc = isD ? 0u : rs.gcount++;
    const int b = wj % NACC;
    const unsigned long long tw0 = pclock(prof);
    if (!wait_mbar(accf_bar(smem, pipe, b), (uint32_t)(wj / NACC) & 1u, p.sync, p.timeout_ns, DEV_TIMEOUT_PIPE, wj)) {
      ok = false;
      continue;
    }
    const unsigned long long tk0 = pclock(prof);
    t_wait += tk0 - tw0;
    tc_fence_after();
    const uint32_t tacc = tmem + ((uint32_t)(32 * q) << 16) + pipe_acc<U>(pipe, b);
    if (!isD) {
      float av[U];
      // block amax of warps q and q ^ 1 meet in shared memory; the exchange
      // buffer alternates so that a warp one job ahead cannot overwrite it
      const int xb = (int)(gc & 1u);
      float* xc = xch_buf(smem, pipe, xb, U);
#pragma unroll
      for (int j = 0; j < U; ++j) {
        av[j] = 0.f;
        if (j < nt) {
          float v[NTERM];
          tmem_ld8(tacc + j * NTERM, v);
          float sum = v[NTERM - 1];
#pragma unroll
          for (int k = NTERM - 2; k >= 0; --k) sum += v[k];
          const float other = __shfl_xor_sync(FULL, sum, 16);
          const float g = lane < 16 ? sum : other, up = lane < 16 ? other : sum;
          const float a = g / (1.0f + expf(-g)) * up;
          av[j] = a;
          float am = fabsf(a);
#pragma unroll
          for (int o = 8; o > 0; o >>= 1) am = fmaxf(am, __shfl_xor_sync(FULL, am, o));
          if (lane == 0) xc[j * 4 + q] = am;
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(xch_bar(smem, pipe, xb));
      if (!wait_mbar(xch_bar(smem, pipe, xb), (gc >> 1) & 1u, p.sync, p.timeout_ns, DEV_TIMEOUT_PIPE, wj)) {
        ok = false;
        continue;
      }
      const int i0 = rb * GU_I_ROWS, sD = i0 / KS, kk = (i0 % KS) / 64, kc = q >> 1;
#pragma unroll
      for (int j = 0; j < U; ++j) {
        if (j < nt) {
          const int s0 = term0_exp(fmaxf(xc[j * 4 + q], xc[j * 4 + (q ^ 1)]));
          const uint32_t word = term_word<16>(e2m1_terms(av[j], s0), lane);
          uint8_t* img = p.aimg + ((int64_t)sD * p.TK + pos0 + j) * IMG_BYTES;
          if (lane < 16)
            *reinterpret_cast<uint32_t*>(img + kk * 256 + kc * 128 + (lane >> 1) * 16 + (q & 1) * 8 +
                                         (lane & 1) * 4) = word;
          if ((q & 1) == 0 && lane < NTERM) {
            const uint8_t e8 = (uint8_t)(term_exp(s0, lane) + 127);
            img[IMG_CODE_BYTES + lane * 16 + 2 * kk + kc] = e8;
            // big units: positions 4..7 also at bytes 4..7 of position j - 4's scale rows
            if (U == NT_BIG && j >= NT_MAX) img[IMG_CODE_BYTES + lane * 16 + 4 + 2 * kk + kc - NT_MAX * IMG_BYTES] = e8;
          }
        }
      }
      __syncwarp();
      if (lane == 0) {
        fence_proxy_async_global();
        __threadfence();
        red_release_add_u32(ready + u, 1u);
      }
    } else {
      const int h0 = rb * JOB_ROWS;
#pragma unroll
      for (int j = 0; j < (U > ND_MAX ? U : ND_MAX); ++j) {
        if (j < nt) {
          float v[NTERM];
          tmem_ld8(tacc + j * NTERM, v);
          float sum = v[NTERM - 1];
#pragma unroll
          for (int k = NTERM - 2; k >= 0; --k) sum += v[k];
          p.ypair[(int64_t)(pos0 + j) * p.H + h0 + 32 * q + lane] = sum * ld_tab(cx.wpos + pos0 + j, cx.global);
        }
      }
    }
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(acce_bar(smem, pipe, b));
    t_work += pclock(prof) - tk0;
  }
  if (prof && lane == 0) {
    atomicAdd(p.prof + PF_EPI_WAIT, t_wait);
    atomicAdd(p.prof + PF_EPI_WORK, t_work);
    atomicAdd(p.prof + PF_EPI_TOTAL, pclock(prof) - t_begin);
    if (q == 0) atomicAdd(p.prof + PF_JOBS, n_jobs);
  }
}

// ---- phase C, large T*K: one pipeline over tiles -------------------------------------------
// Tensor memory: NACCV accumulator sets of R accumulators of ACCW columns
// (accumulator r of set b at (b R + r) ACCW), then NSF scale-factor buffers
// of 4 R + 4 columns (A: 4 per row block, then B: 4 per 128 B rows).
template <int TM>
__device__ __forceinline__ uint32_t lt_acc(int b, int r) {
  return (uint32_t)(b * TileCfg<TM>::R + r) * TileCfg<TM>::ACCW;
}
template <int TM>
__device__ __forceinline__ uint32_t lt_sf(int i) {
  using C = TileCfg<TM>;
  return (uint32_t)(C::NACCV * C::R * C::ACCW + i * (4 * C::R + 4 * LT_SF_BLOCKS));
}
static_assert(LT_NACC * LT_ACC_COLS + NSF * (4 + 4 * LT_SF_BLOCKS) <= TMEM_COLS, "tensor memory (tiles)");
static_assert(LTA_NACC * LTA_R * LTA_ACC_COLS + NSF * (4 * LTA_R + 4 * LT_SF_BLOCKS) <= TMEM_COLS,
              "tensor memory (tile pairs)");

// MMA issuer of the tile stream (one thread): per stage the weight scales of
// the job's R row blocks and the tile's 1-2 scale blocks go to tensor memory,
// then per row block two MMAs (K = 64 each, N = 8 per position of the tile)
// accumulate into that row block's accumulator.
template <int TM>
__device__ void stream_mma_lt(const EngineParams& p, uint8_t* smem, uint32_t tmem, RoleState& rs) {
  using C = TileCfg<TM>;
  JobEntry* jq = job_queue(smem, 0);
  const uint32_t ring0 = smem_u32(smem + OFF_RING);
  const bool prof = p.prof != nullptr;
  unsigned long long t_full = 0, t_issue = 0, t_acc = 0;
  bool ok = true;
  for (;;) {
    JobEntry* en = jq + (rs.qk % JQ);
    if (!wait_entry(p, en, rs.qk)) return;
    const int job = *reinterpret_cast<volatile int32_t*>(&en->job);
    if (job < 0) { ++rs.qk; break; }
    const int s0 = en->s0, nc = en->nc, nt = en->nt, wj = en->wj;
    ++rs.qk;
    if (!ok) continue;
    const int b = wj % C::NACCV;
    const uint32_t use = (uint32_t)(wj / C::NACCV);
    const unsigned long long ta0 = pclock(prof);
    if (use > 0 &&
        !wait_mbar(acce_bar(smem, 0, b), (use - 1) & 1u, p.sync, p.timeout_ns, DEV_TIMEOUT_PIPE, wj)) {
      ok = false;
      continue;
    }
    t_acc += pclock(prof) - ta0;
    tc_fence_after();
    const int n = lt_cols(nt), nblk = (n + 127) / 128;
    const uint32_t idesc0 = mxf4_idesc(n, 0u), idesc1 = mxf4_idesc(n, 2u);
    for (int c = 0; c < nc; ++c) {
      const uint32_t s = (uint32_t)s0 + c;
      const int slot = (int)(s % C::NS);
      const unsigned long long tf0 = pclock(prof);
      if (!wait_mbar(full_bar(smem, 0, slot), (s / C::NS) & 1u, p.sync, p.timeout_ns, DEV_TIMEOUT_PIPE, s)) {
        ok = false;
        break;
      }
      const unsigned long long tm0 = pclock(prof);
      t_full += tm0 - tf0;
      const uint32_t sa = ring0 + (uint32_t)slot * C::SLOTB, sb = sa + C::R * STAGE_A_BYTES;
      const uint32_t tsf = tmem + lt_sf<TM>((int)(rs.sfc++ % NSF));
      const uint32_t tsb = tsf + 4 * C::R;  // B scale columns
#pragma unroll
      for (int r = 0; r < C::R; ++r)
        tmem_cp_sf(tsf + 4 * r, smem_desc(sa + r * STAGE_A_BYTES + STAGE_CODE_BYTES, 0, 128));
      for (int q = 0; q < nblk; ++q) tmem_cp_sf(tsb + 4 * q, smem_desc(sb + q * 512, 0, 128));
      const uint32_t bc = sb + LT_SF_BYTES;
#pragma unroll
      for (int r = 0; r < C::R; ++r) {
        const uint32_t tacc = tmem + lt_acc<TM>(b, r), ar = sa + r * STAGE_A_BYTES, tsa = tsf + 4 * r;
        mma_mxf4(tacc, smem_desc(ar, 128, 256), smem_desc(bc, 128, IMG_CODE_BYTES), idesc0, tsa, tsb,
                 c > 0 ? 1u : 0u);
        mma_mxf4(tacc, smem_desc(ar + 4096, 128, 256), smem_desc(bc + 256, 128, IMG_CODE_BYTES), idesc1,
                 tsa | (2u << 30), tsb | (2u << 30), 1u);
      }
      tc_commit(empty_bar(smem, 0, slot));
      t_issue += pclock(prof) - tm0;
    }
    if (ok) tc_commit(accf_bar(smem, 0, b));
  }
  if (prof) {
    atomicAdd(p.prof + PF_MMA_FULL, t_full);
    atomicAdd(p.prof + PF_MMA_ISSUE, t_issue);
    atomicAdd(p.prof + PF_MMA_ACC, t_acc);
  }
}

// Epilogue of the tile stream (warps 4..7, warp q reading tensor-memory lanes
// 32q..32q+31): as stream_epilogue, over up to LT_MAX positions; the SwiGLU
// term images are written into the tile images of the down jobs.
// Sum of position j's LT_NTERM accumulator columns (this warp's 32 rows):
// the eight columns from the aligned group holding the first, and the next
// group when the terms cross into it; terms summed last to first.
__device__ __forceinline__ float lt_position_sum(uint32_t tacc, int j) {
  const int c0 = LT_NTERM * j, g0 = c0 & ~7;
  float v[16];
  tmem_ld8(tacc + g0, *reinterpret_cast<float(*)[8]>(v));
  if (c0 + LT_NTERM > g0 + 8) tmem_ld8(tacc + g0 + 8, *reinterpret_cast<float(*)[8]>(v + 8));
  float sum = 0.f;
#pragma unroll
  for (int k = LT_NTERM - 1; k >= 0; --k) {
    float t = 0.f;
#pragma unroll
    for (int i = 0; i < 16; ++i)
      if (i == c0 - g0 + k) t = v[i];
    sum = k == LT_NTERM - 1 ? t : sum + t;
  }
  return sum;
}
// Eight epilogue warps in two sets (warps 4..7 and 8..11, each covering the
// four accumulator lane quadrants), each with its own amax exchange buffers
// and barriers.  Tiles (one row block per job): set `set` handles positions
// set, set + 2, ...  Tile pairs: set `set` handles every position of row
// block rb + set (its own accumulator).
template <int TM>
__device__ void stream_epilogue_lt(const EngineParams& p, uint8_t* smem, const StreamCtx& cx, uint32_t tmem,
                                   int set, RoleState& rs) {
  using C = TileCfg<TM>;
  static_assert(C::R == 1 || C::R == 2, "one row block per epilogue set");
  const int J0 = C::R == 1 ? set : 0, JS = C::R == 1 ? 2 : 1, rs_ = C::R == 1 ? 0 : set;
  const int lane = threadIdx.x & 31, q = (threadIdx.x >> 5) & 3;
  JobEntry* jq = job_queue(smem, 0);
  uint32_t* ready = p.sync + SY_READY;
  const int nsd = p.I / KS;
  const bool prof = p.prof != nullptr;
  unsigned long long t_wait = 0, t_work = 0, n_jobs = 0;
  const unsigned long long t_begin = pclock(prof);
  bool ok = true;
  float av[LT_MAX];
  for (;;) {
    JobEntry* en = jq + (rs.qk % JQ);
    if (!wait_entry(p, en, rs.qk)) return;
    const int job = *reinterpret_cast<volatile int32_t*>(&en->job);
    if (job < 0) { ++rs.qk; break; }
    const int wj = en->wj;
    const int u = en->unit, rb = en->rb, isD = en->isD, pos0 = en->pos0, nt = en->nt;
    ++rs.qk;
    if (!ok) continue;
    ++n_jobs;
    const uint32_t gc = isD ? 0u : rs.gcount++;
    const int b = wj % C::NACCV;
    const unsigned long long tw0 = pclock(prof);
    if (!wait_mbar(accf_bar(smem, 0, b), (uint32_t)(wj / C::NACCV) & 1u, p.sync, p.timeout_ns, DEV_TIMEOUT_PIPE, wj)) {
      ok = false;
      continue;
    }
    const unsigned long long tk0 = pclock(prof);
    t_wait += tk0 - tw0;
    tc_fence_after();
    const uint32_t tacc = tmem + ((uint32_t)(32 * q) << 16) + lt_acc<TM>(b, rs_);
    const int rbe = rb + rs_;  // this set's row block
    if (!isD) {
      const int xb = (int)(gc & 1u);
      float* xc = reinterpret_cast<float*>(smem + OFF_XCH) + (set * 2 + xb) * LT_MAX * 4;
      for (int j = J0; j < nt; j += JS) {
        const float sum = lt_position_sum(tacc, j);
        const float other = __shfl_xor_sync(FULL, sum, 16);
        const float g = lane < 16 ? sum : other, up = lane < 16 ? other : sum;
        const float a = g / (1.0f + expf(-g)) * up;
        av[j] = a;
        float am = fabsf(a);
#pragma unroll
        for (int o = 8; o > 0; o >>= 1) am = fmaxf(am, __shfl_xor_sync(FULL, am, o));
        if (lane == 0) xc[j * 4 + q] = am;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(xch_bar(smem, set, xb));
      if (!wait_mbar(xch_bar(smem, set, xb), (gc >> 1) & 1u, p.sync, p.timeout_ns, DEV_TIMEOUT_PIPE, wj)) {
        ok = false;
        continue;
      }
      const int i0 = rbe * GU_I_ROWS, sD = i0 / KS, kk = (i0 % KS) / 64, kc = q >> 1;
      uint8_t* img = p.atl + ((int64_t)u * nsd + sD) * LT_IMG_BYTES;
      for (int j = J0; j < nt; j += JS) {
        const int s0 = term0_exp(fmaxf(xc[j * 4 + q], xc[j * 4 + (q ^ 1)]));
        const uint32_t word = term_word<16>(e2m1_terms<LT_NTERM>(av[j], s0), lane);
        if (lane < 2 * LT_NTERM)  // lane l: term l / 2, elements 8 (l % 2) .. + 7 of this warp's 16
          *reinterpret_cast<uint32_t*>(img + lt_row_offset(LT_NTERM * j + (lane >> 1)) + kk * 256 + kc * 128 +
                                       (q & 1) * 8 + (lane & 1) * 4) = word;
        if ((q & 1) == 0 && lane < LT_NTERM)
          img[lt_sf_offset(LT_NTERM * j + lane, 2 * kk + kc)] = (uint8_t)(term_exp(s0, lane) + 127);
      }
      __syncwarp();
      if (lane == 0) {
        fence_proxy_async_global();
        __threadfence();
        red_release_add_u32(ready + u, 1u);
      }
    } else {
      const int h0 = rbe * JOB_ROWS;
      for (int j = J0; j < nt; j += JS) {
        const float sum = lt_position_sum(tacc, j);
        p.ypair[(int64_t)(pos0 + j) * p.H + h0 + 32 * q + lane] = sum * ld_tab(cx.wpos + pos0 + j, cx.global);
      }
    }
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(acce_bar(smem, 0, b));
    t_work += pclock(prof) - tk0;
  }
  if (prof && lane == 0) {
    atomicAdd(p.prof + PF_EPI_WAIT, t_wait);
    atomicAdd(p.prof + PF_EPI_WORK, t_work);
    atomicAdd(p.prof + PF_EPI_TOTAL, pclock(prof) - t_begin);
    if (q == 0) atomicAdd(p.prof + PF_JOBS, n_jobs);
  }
}

// ---- phase C, large T*K, E4M3 tiles on kind::mxf8f6f4 -----------------------------------------
// Ring slot (ET_SLOT_BYTES): the packed weight stage (STAGE_A_BYTES, from the
// producer), the tile's B image (from the producer), and the weight codes in
// the kind's 16-byte-chunk form (ET_U_BYTES, from the converter warps; the
// MMA still takes the weight scales from the packed stage).  Barriers: full
// (0, slot) = the producer's copies, full (1, slot) = the converted codes (two
// converter warps), empty (0, slot) = the MMAs done with the whole slot.
// Tensor memory: 2 accumulators of ET_ACC_COLS, then NSF scale buffers of 12
// columns (A: 4, B: 4 per 128 rows).
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, const EngineParams& p, uint32_t info);
__device__ __forceinline__ uint32_t et_acc(int b) { return (uint32_t)b * ET_ACC_COLS; }
__device__ __forceinline__ uint32_t et_sf(int i) { return (uint32_t)(2 * ET_ACC_COLS + i * (4 + 4 * LT_SF_BLOCKS)); }
__device__ __forceinline__ uint8_t* et_slot(uint8_t* smem, int slot) { return smem + OFF_RING + (size_t)slot * ET_SLOT_BYTES; }
constexpr int ET_U_OFF = STAGE_A_BYTES + ET_AB_BYTES;
static_assert(ET_U_OFF % 128 == 0 && (size_t)ET_NSLOT * ET_SLOT_BYTES <= RING_BYTES, "E4M3 ring layout");

// Converter warps (2 and 3): each packed 16-byte chunk (32 E2M1 codes of one
// weight row: row m, K half kk, 32-element chunk c of the packed stage) becomes
// the two 16-element chunks of K slice 2 kk + c in the kind's form: 8 packed
// bytes, then 8 zero bytes.
__device__ void stream_convert_e(const EngineParams& p, uint8_t* smem, int wl, RoleState& rs) {
  const int lane = threadIdx.x & 31, tid = 32 * wl + lane;
  JobEntry* jq = job_queue(smem, 0);
  bool ok = true;
  for (;;) {
    JobEntry* en = jq + (rs.qk % JQ);
    if (!wait_entry(p, en, rs.qk)) return;
    const int job = *reinterpret_cast<volatile int32_t*>(&en->job);
    if (job < 0) { ++rs.qk; break; }
    const int s0 = en->s0, nc = en->nc;
    ++rs.qk;
    if (!ok) continue;
    for (int c = 0; c < nc; ++c) {
      const uint32_t s = (uint32_t)s0 + c;
      const int slot = (int)(s % ET_NSLOT);
      if (!warp_wait(full_bar(smem, 0, slot), (s / ET_NSLOT) & 1u, p, s)) { ok = false; break; }
      const uint8_t* raw = et_slot(smem, slot);
      uint8_t* u = et_slot(smem, slot) + ET_U_OFF;
#pragma unroll 4
      for (int i = tid; i < 128 * 4; i += 64) {
        const int m = i >> 2, q = i & 3, kk = q >> 1, kc = q & 1;
        const uint4 w = *reinterpret_cast<const uint4*>(raw + kk * 4096 + (m >> 3) * 256 + kc * 128 + (m & 7) * 16);
        uint8_t* d = u + q * 4096 + (m >> 3) * 256 + (m & 7) * 16;
        *reinterpret_cast<uint4*>(d) = make_uint4(w.x, w.y, 0u, 0u);
        *reinterpret_cast<uint4*>(d + 128) = make_uint4(w.z, w.w, 0u, 0u);
      }
      fence_proxy_async_smem();  // read by the tensor cores (async proxy)
      __syncwarp();
      if (lane == 0) mbar_arrive(full_bar(smem, 1, slot));
    }
  }
}

// MMA issuer of the E4M3 tiles (one thread): per stage the weight scales and
// the tile's 1-2 scale blocks go to tensor memory, then four MMAs (K = 32
// each, scale byte i of the stage's block column) accumulate.
__device__ void stream_mma_e(const EngineParams& p, uint8_t* smem, uint32_t tmem, RoleState& rs) {
  JobEntry* jq = job_queue(smem, 0);
  const bool prof = p.prof != nullptr;
  unsigned long long t_full = 0, t_issue = 0, t_acc = 0;
  bool ok = true;
  for (;;) {
    JobEntry* en = jq + (rs.qk % JQ);
    if (!wait_entry(p, en, rs.qk)) return;
    const int job = *reinterpret_cast<volatile int32_t*>(&en->job);
    if (job < 0) { ++rs.qk; break; }
    const int s0 = en->s0, nc = en->nc, nt = en->nt, wj = en->wj, isD = en->isD;
    ++rs.qk;
    if (!ok) continue;
    const int b = wj & 1;
    const uint32_t use = (uint32_t)(wj >> 1);
    const unsigned long long ta0 = pclock(prof);
    if (use > 0 &&
        !wait_mbar(acce_bar(smem, 0, b), (use - 1) & 1u, p.sync, p.timeout_ns, DEV_TIMEOUT_PIPE, wj)) {
      ok = false;
      continue;
    }
    t_acc += pclock(prof) - ta0;
    tc_fence_after();
    const uint32_t tacc = tmem + et_acc(b);
    const int n = et_cols(nt, isD ? ET_ATERMS : ET_XTERMS), nblk = (n + 127) / 128;
    for (int c = 0; c < nc; ++c) {
      const uint32_t s = (uint32_t)s0 + c;
      const int slot = (int)(s % ET_NSLOT);
      const unsigned long long tf0 = pclock(prof);
      if (!wait_mbar(full_bar(smem, 0, slot), (s / ET_NSLOT) & 1u, p.sync, p.timeout_ns, DEV_TIMEOUT_PIPE, s) ||
          !wait_mbar(full_bar(smem, 1, slot), (s / ET_NSLOT) & 1u, p.sync, p.timeout_ns, DEV_TIMEOUT_PIPE, s)) {
        ok = false;
        break;
      }
      const unsigned long long tm0 = pclock(prof);
      t_full += tm0 - tf0;
      tc_fence_after();
      const uint32_t sa = smem_u32(et_slot(smem, slot)), sb = sa + STAGE_A_BYTES, su = sa + ET_U_OFF;
      const uint32_t tsf = tmem + et_sf((int)(rs.sfc++ % NSF)), tsb = tsf + 4;
      tmem_cp_sf(tsf, smem_desc(sa + STAGE_CODE_BYTES, 0, 128));
      for (int q = 0; q < nblk; ++q) tmem_cp_sf(tsb + 4 * q, smem_desc(sb + q * 512, 0, 128));
#pragma unroll
      for (int i = 0; i < 4; ++i)
        mma_mxf8(tacc, smem_desc(su + i * 4096, 128, 256), smem_desc(sb + LT_SF_BYTES + i * n * 32, 128, 256),
                 mxf8_idesc(n, (uint32_t)i), tsf | ((uint32_t)i << 30), tsb | ((uint32_t)i << 30),
                 (c > 0 || i > 0) ? 1u : 0u);
      tc_commit(empty_bar(smem, 0, slot));
      t_issue += pclock(prof) - tm0;
    }
    if (ok) tc_commit(accf_bar(smem, 0, b));
  }
  if (prof) {
    atomicAdd(p.prof + PF_MMA_FULL, t_full);
    atomicAdd(p.prof + PF_MMA_ISSUE, t_issue);
    atomicAdd(p.prof + PF_MMA_ACC, t_acc);
  }
}

// Sum of position j's NT accumulator columns (this warp's 32 rows), the
// eight-column group holding the first and the next one when the terms cross
// into it; terms summed last to first.
template <int NT>
__device__ __forceinline__ float et_position_sum(uint32_t tacc, int j) {
  const int c0 = NT * j, g0 = c0 & ~7;
  float v[16];
  tmem_ld8(tacc + g0, *reinterpret_cast<float(*)[8]>(v));
  if (c0 + NT > g0 + 8) tmem_ld8(tacc + g0 + 8, *reinterpret_cast<float(*)[8]>(v + 8));
  float sum = 0.f;
#pragma unroll
  for (int k = NT - 1; k >= 0; --k) {
    float t = 0.f;
#pragma unroll
    for (int i = 0; i < 16; ++i)
      if (i == c0 - g0 + k) t = v[i];
    sum = k == NT - 1 ? t : sum + t;
  }
  return sum;
}

// Epilogue of the E4M3 tiles: eight warps in two sets (positions set, set + 2,
// ...), warp q reading accumulator rows 32 q .. 32 q + 31.  Gate/up: SwiGLU
// of the gate and up rows (lanes l, l + 16), the block amax shared with warp
// q ^ 1, ET_ATERMS E4M3 terms of the output written into the tile's down
// image (row n = 3 j + k, this warp's 16 elements at 16 (q % 2) of block
// 2 kk + q / 2); down: the position's column sum times the routing weight.
__device__ void stream_epilogue_e(const EngineParams& p, uint8_t* smem, const StreamCtx& cx, uint32_t tmem,
                                  int set, RoleState& rs) {
  const int lane = threadIdx.x & 31, q = (threadIdx.x >> 5) & 3;
  JobEntry* jq = job_queue(smem, 0);
  uint32_t* ready = p.sync + SY_READY;
  const int nsd = p.I / KS;
  const bool prof = p.prof != nullptr;
  unsigned long long t_wait = 0, t_work = 0, n_jobs = 0;
  const unsigned long long t_begin = pclock(prof);
  bool ok = true;
  float av[ET_MAX];
  for (;;) {
    JobEntry* en = jq + (rs.qk % JQ);
    if (!wait_entry(p, en, rs.qk)) return;
    const int job = *reinterpret_cast<volatile int32_t*>(&en->job);
    if (job < 0) { ++rs.qk; break; }
    const int wj = en->wj;
    const int u = en->unit, rb = en->rb, isD = en->isD, pos0 = en->pos0, nt = en->nt;
    ++rs.qk;
    if (!ok) continue;
    ++n_jobs;
    const uint32_t gc = isD ? 0u : rs.gcount++;
    const int b = wj & 1;
    const unsigned long long tw0 = pclock(prof);
    if (!wait_mbar(accf_bar(smem, 0, b), (uint32_t)(wj >> 1) & 1u, p.sync, p.timeout_ns, DEV_TIMEOUT_PIPE, wj)) {
      ok = false;
      continue;
    }
    const unsigned long long tk0 = pclock(prof);
    t_wait += tk0 - tw0;
    tc_fence_after();
    const uint32_t tacc = tmem + ((uint32_t)(32 * q) << 16) + et_acc(b);
    if (!isD) {
      const int xb = (int)(gc & 1u);
      float* xc = reinterpret_cast<float*>(smem + OFF_XCH) + (set * 2 + xb) * ET_MAX * 4;
      for (int j = set; j < nt; j += 2) {
        const float sum = et_position_sum<ET_XTERMS>(tacc, j);
        const float other = __shfl_xor_sync(FULL, sum, 16);
        const float g = lane < 16 ? sum : other, up = lane < 16 ? other : sum;
        const float a = g / (1.0f + expf(-g)) * up;
        av[j] = a;
        float am = fabsf(a);
#pragma unroll
        for (int o = 8; o > 0; o >>= 1) am = fmaxf(am, __shfl_xor_sync(FULL, am, o));
        if (lane == 0) xc[j * 4 + q] = am;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(xch_bar(smem, set, xb));
      if (!wait_mbar(xch_bar(smem, set, xb), (gc >> 1) & 1u, p.sync, p.timeout_ns, DEV_TIMEOUT_PIPE, wj)) {
        ok = false;
        continue;
      }
      const int i0 = rb * GU_I_ROWS, sD = i0 / KS, blk = 2 * ((i0 % KS) / 64) + (q >> 1);
      const int N = et_cols(nt, ET_ATERMS);
      uint8_t* img = p.ate + ((int64_t)u * nsd + sD) * ET_AB_BYTES;
      const int e0 = 32 * blk + 16 * (q & 1);  // this warp's first element of the stage
      for (int j = set; j < nt; j += 2) {
        const int s0 = et_term0_exp(fmaxf(xc[j * 4 + q], xc[j * 4 + (q ^ 1)]));
        float r = av[j];
#pragma unroll
        for (int k = 0; k < ET_ATERMS; ++k) {
          const uint32_t c = et_term(r, s0, k);
          // lanes 4 w .. 4 w + 3 (w < 4) pack their bytes into one word: elements e0 + 4 w .. + 3
          const uint32_t c1 = __shfl_down_sync(FULL, c, 1), c2 = __shfl_down_sync(FULL, c, 2),
                         c3 = __shfl_down_sync(FULL, c, 3);
          if (lane < 16 && (lane & 3) == 0)
            *reinterpret_cast<uint32_t*>(img + et_code_offset(ET_ATERMS * j + k, e0 + lane, N)) =
                c | (c1 << 8) | (c2 << 16) | (c3 << 24);
        }
        if ((q & 1) == 0 && lane < ET_ATERMS)
          img[lt_sf_offset(ET_ATERMS * j + lane, blk)] = (uint8_t)(s0 - ET_STEP * lane + 127);
      }
      __syncwarp();
      if (lane == 0) {
        fence_proxy_async_global();
        __threadfence();
        red_release_add_u32(ready + u, 1u);
      }
    } else {
      const int h0 = rb * JOB_ROWS;
      for (int j = set; j < nt; j += 2) {
        const float sum = et_position_sum<ET_ATERMS>(tacc, j);
        p.ypair[(int64_t)(pos0 + j) * p.H + h0 + 32 * q + lane] = sum * ld_tab(cx.wpos + pos0 + j, cx.global);
      }
    }
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(acce_bar(smem, 0, b));
    t_work += pclock(prof) - tk0;
  }
  if (prof && lane == 0) {
    atomicAdd(p.prof + PF_EPI_WAIT, t_wait);
    atomicAdd(p.prof + PF_EPI_WORK, t_work);
    atomicAdd(p.prof + PF_EPI_TOTAL, pclock(prof) - t_begin);
    if (q == 0) atomicAdd(p.prof + PF_JOBS, n_jobs);
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
    const float4 v = __ldcg(reinterpret_cast<const float4*>(p.ypair + (int64_t)pos * p.H + h));
    s.x += v.x; s.y += v.y; s.z += v.z; s.w += v.w;
  }
  return s;
}

// ---- bf16 tile stream roles ---------------------------------------------------------------
// Three rings in the ring area: FT_RA raw weight half-stages, FT_NB B blocks,
// FT_AB dequantised A blocks.  Barriers (pipe 0 / pipe 1 arrays):
//   rawfull[i] = full(0, i)      producer's copies        rawempty[i] = empty(0, i)  converter warps
//   bfull[i]   = full(1, i)      producer's copy          bempty[i]   = empty(1, i)  MMA commit
//   afull[i]   = full(1, NB + i) converter warps          aempty[i]   = empty(1, NB + i)  MMA commit
// and accf/acce(0, 0..1) between the MMA issuer and the epilogue warps.
__device__ __forceinline__ uint8_t* ft_raw(uint8_t* smem, int i) { return smem + OFF_RING + (size_t)i * FT_RAW_BYTES; }
__device__ __forceinline__ uint8_t* ft_b(uint8_t* smem, int i) {
  return smem + OFF_RING + (size_t)FT_RA * FT_RAW_BYTES + (size_t)i * FT_TERM_BYTES;
}
__device__ __forceinline__ uint8_t* ft_a(uint8_t* smem, int i) {
  return smem + OFF_RING + (size_t)FT_RA * FT_RAW_BYTES + (size_t)FT_NB * FT_TERM_BYTES + (size_t)i * FT_A_BYTES;
}
__device__ __forceinline__ uint64_t* rawfull_bar(uint8_t* smem, int i) { return full_bar(smem, 0, i); }
__device__ __forceinline__ uint64_t* rawempty_bar(uint8_t* smem, int i) { return empty_bar(smem, 0, i); }
__device__ __forceinline__ uint64_t* bfull_bar(uint8_t* smem, int i) { return full_bar(smem, 1, i); }
__device__ __forceinline__ uint64_t* bempty_bar(uint8_t* smem, int i) { return empty_bar(smem, 1, i); }
__device__ __forceinline__ uint64_t* afull_bar(uint8_t* smem, int i) { return full_bar(smem, 1, FT_NB + i); }
__device__ __forceinline__ uint64_t* aempty_bar(uint8_t* smem, int i) { return empty_bar(smem, 1, FT_NB + i); }
static_assert((size_t)FT_RA * FT_RAW_BYTES + (size_t)FT_NB * FT_TERM_BYTES + (size_t)FT_AB * FT_A_BYTES <= RING_BYTES,
              "bf16 tile rings");
static_assert(FT_RAW_BYTES % 128 == 0 && FT_TERM_BYTES % 128 == 0 && FT_A_BYTES % 128 == 0, "ring alignment");

// kind::f16 instruction descriptor: bf16 A and B (K-major), fp32 D, M = 128.
__device__ __forceinline__ uint32_t f16_idesc(int n) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(n >> 3) << 17) | ((uint32_t)(128 >> 4) << 24);
}
__device__ __forceinline__ void mma_bf16(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                         uint32_t accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n"
      ::"r"(tmem_d), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Bounded wait of lane 0 for a ring barrier's phase, shared with the warp.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, const EngineParams& p, uint32_t info) {
  int ok = 1;
  if ((threadIdx.x & 31) == 0) ok = wait_mbar(bar, parity, p.sync, p.timeout_ns, DEV_TIMEOUT_PIPE, info);
  return __shfl_sync(FULL, ok, 0) != 0;
}

// Producer warp of the bf16 tile stream: jobs -> queue entries (s0: first raw
// half-stage sequence number, b0: first B block sequence number) -> copies.
// Lane 0 issues; a down half-stage has two B blocks (the SwiGLU terms).
__device__ void stream_producer_f16(const EngineParams& p, const LayerPtrs& lp, uint8_t* smem,
                                    const StreamCtx& cx, RoleState& rs) {
  const int lane = threadIdx.x & 31;
  JobEntry* jq = job_queue(smem, 0);
  uint32_t* ready = p.sync + SY_READY;
  const int gub = p.I / GU_I_ROWS, db = p.H / JOB_ROWS;
  const int64_t n_gu = (int64_t)cx.n_units * gub, n_all = n_gu + (int64_t)cx.n_dunits * db;
  const int nh_gu = p.H / FT_HK, nh_d = p.I / FT_HK;
  const uint32_t need = (uint32_t)gub * 4u;
  const uint32_t seq_start = rs.seq, b_start = rs.sfc;
  bool ok = true;
  unsigned long long t_empty = 0, t_ready = 0;
  const unsigned long long t_begin = clock64();
  fence_proxy_async_global();
  const int64_t jbase = gridDim.x;
  long long next = blockIdx.x;
  for (;;) {
    const int64_t j = __shfl_sync(FULL, next, 0);
    if (j >= n_all || !ok) {
      if (lane == 0) {
        JobEntry* en = jq + (rs.qk % JQ);
        en->job = -1; en->s0 = (int32_t)rs.seq; en->nc = 0; en->pad = (int32_t)rs.sfc;
        __threadfence_block();
        *reinterpret_cast<volatile int32_t*>(&en->flag) = rs.qk + 1;
      }
      ++rs.qk;
      break;
    }
    if (lane == 0) next = jbase + atomicAdd(p.sync + SY_JOBS, 1u);
    const bool isD = j >= n_gu;
    const int64_t jj = isD ? j - n_gu : j;
    const int per = isD ? db : gub;
    const int u = (int)(jj / per), rb = (int)(jj % per);
    const int4 ur = ld_tab(reinterpret_cast<const int4*>((isD ? cx.dunits : cx.units) + (int64_t)u * 4), cx.global);
    const int e = ur.x, pos0 = ur.y, nt = ur.z;
    const int nh = isD ? nh_d : nh_gu;
    if (isD) {
      const int gu = ur.w;
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
      if (!ok) continue;
      fence_proxy_async_global();  // the SwiGLU terms were written by generic stores of other CTAs
    }
    if (lane == 0) {
      JobEntry* en = jq + (rs.qk % JQ);
      en->job = (int32_t)j; en->s0 = (int32_t)rs.seq; en->nc = nh; en->unit = u; en->rb = rb;
      en->isD = isD; en->e = e; en->pos0 = pos0; en->nt = nt; en->wj = rs.wj; en->pad = (int32_t)rs.sfc;
      __threadfence_block();
      *reinterpret_cast<volatile int32_t*>(&en->flag) = rs.qk + 1;
    }
    ++rs.qk;
    ++rs.wj;
    const uint8_t* wbase = isD ? lp.w_d + ((int64_t)e * db + rb) * (nh / 2) * STAGE_A_BYTES
                               : lp.w_gu + ((int64_t)e * gub + rb) * (nh / 2) * STAGE_A_BYTES;
    const int n16 = (nt + 15) & ~15;
    const uint32_t bbytes = (uint32_t)n16 * FT_HK * 2u;
    const int terms = isD ? 2 : 1;
    for (int h = 0; h < nh && ok; ++h) {
      // raw half-stage: codes of half h % 2 of stage h / 2, and that stage's scales
      const uint32_t r = rs.seq;
      const int ri = (int)(r % FT_RA);
      const unsigned long long te0 = clock64();
      if (r >= (uint32_t)FT_RA)
        if (!warp_wait(rawempty_bar(smem, ri), ((r / FT_RA) + 1) & 1u, p, r)) { ok = false; break; }
      if (lane == 0) {
        uint64_t* fb = rawfull_bar(smem, ri);
        const uint8_t* src = wbase + (int64_t)(h >> 1) * STAGE_A_BYTES;
        mbar_arrive_expect_tx(fb, FT_RAW_BYTES);
        bulk_g2s(ft_raw(smem, ri), src + (h & 1) * 4096, 4096, fb);
        bulk_g2s(ft_raw(smem, ri) + 4096, src + STAGE_CODE_BYTES, 512, fb);
      }
      ++rs.seq;
      for (int t = 0; t < terms; ++t) {
        const uint32_t bq = rs.sfc;
        const int bi = (int)(bq % FT_NB);
        if (bq >= (uint32_t)FT_NB)
          if (!warp_wait(bempty_bar(smem, bi), ((bq / FT_NB) + 1) & 1u, p, bq)) { ok = false; break; }
        if (lane == 0) {
          uint64_t* fb = bfull_bar(smem, bi);
          const uint8_t* src = isD ? p.atf + (((int64_t)u * nh_d + h) * 2 + t) * FT_TERM_BYTES
                                   : p.xtf + ((int64_t)u * nh_gu + h) * FT_TERM_BYTES;
          mbar_arrive_expect_tx(fb, bbytes);
          bulk_g2s(ft_b(smem, bi), src, bbytes, fb);
        }
        ++rs.sfc;
      }
      t_empty += clock64() - te0;
    }
  }
  if (p.prof && lane == 0) {
    atomicAdd(p.prof + PF_PROD_EMPTY, t_empty);
    atomicAdd(p.prof + PF_PROD_READY, t_ready);
    atomicAdd(p.prof + PF_PROD_TOTAL, clock64() - t_begin);
    atomicAdd(p.prof + PF_STAGES, (unsigned long long)(rs.seq - seq_start));
  }
  // let every issued copy land before the rings are reused or the CTA exits
  if (lane == 0) {
    const uint32_t nr = min(rs.seq - seq_start, (uint32_t)FT_RA);
    for (uint32_t r = rs.seq - nr; r != rs.seq; ++r) {
      const uint64_t t0 = globaltimer_ns();
      while (!mbar_try_wait(rawfull_bar(smem, (int)(r % FT_RA)), (r / FT_RA) & 1u))
        if (globaltimer_ns() - t0 > DRAIN_NS) break;
    }
    const uint32_t nb = min(rs.sfc - b_start, (uint32_t)FT_NB);
    for (uint32_t b = rs.sfc - nb; b != rs.sfc; ++b) {
      const uint64_t t0 = globaltimer_ns();
      while (!mbar_try_wait(bfull_bar(smem, (int)(b % FT_NB)), (b / FT_NB) & 1u))
        if (globaltimer_ns() - t0 > DRAIN_NS) break;
    }
  }
  __syncwarp();
}

// bf16 bits of the eight E2M1 magnitudes times 2^(sb - 127), as byte tables
// for prmt: lo[0] (magnitudes 0..3) and lo[1] (4..7) hold the low bytes,
// hi[0], hi[1] the high bytes.  Exact: every such product is a bf16 value
// (normal for sb in [2, 252], where the exponent field is added directly).
__device__ __forceinline__ void e2m1_bf16_tables(uint32_t sb, uint32_t (&lo)[2], uint32_t (&hi)[2]) {
  uint32_t v[4];  // bf16 pairs (magnitude 2i in the low half, 2i + 1 in the high half)
  if (sb >= 2u && sb <= 252u) {
    const uint32_t d = (sb - 127u) << 7;  // added to each exponent field (two's complement)
    const uint32_t dd = (d << 16) | (d & 0xFFFFu);
    // magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6 at 2^0: 0x0000 0x3F00 0x3F80 0x3FC0 0x4000 0x4040 0x4080 0x40C0
    v[0] = (0x3F00u + d) << 16;
    v[1] = __vadd2(0x3FC03F80u, dd);
    v[2] = __vadd2(0x40404000u, dd);
    v[3] = __vadd2(0x40C04080u, dd);
  } else {
    const float sc = sb == 0u ? __int_as_float(0x00400000) : sb == 255u ? __int_as_float(0x7FC00000)
                                                                         : __int_as_float((int)(sb << 23));
    const float mag[8] = {0.f, 0.5f, 1.f, 1.5f, 2.f, 3.f, 4.f, 6.f};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint32_t a = __bfloat16_as_ushort(__float2bfloat16_rn(mag[2 * i] * sc));
      const uint32_t b = __bfloat16_as_ushort(__float2bfloat16_rn(mag[2 * i + 1] * sc));
      v[i] = a | (b << 16);
    }
  }
  lo[0] = __byte_perm(v[0], v[1], 0x6420);
  hi[0] = __byte_perm(v[0], v[1], 0x7531);
  lo[1] = __byte_perm(v[2], v[3], 0x6420);
  hi[1] = __byte_perm(v[2], v[3], 0x7531);
}
// Four E2M1 codes (16 bits, element i in bits 4i..4i+3) -> two bf16x2 words.
__device__ __forceinline__ void e2m1x4_bf16(uint32_t c16, const uint32_t (&lo)[2], const uint32_t (&hi)[2],
                                            uint32_t& w0, uint32_t& w1) {
  const uint32_t sel = c16 & 0x7777u;
  const uint32_t l4 = __byte_perm(lo[0], lo[1], sel), h4 = __byte_perm(hi[0], hi[1], sel);
  w0 = __byte_perm(l4, h4, 0x5140) | ((c16 << 12) & 0x8000u) | ((c16 << 24) & 0x80000000u);
  w1 = __byte_perm(l4, h4, 0x7362) | ((c16 << 4) & 0x8000u) | ((c16 << 16) & 0x80000000u);
}

// Converter warps: each raw weight half-stage (128 rows x 64 K of codes, the
// stage's scales) becomes a bf16 A block in the kind::f16 K-major layout.  An
// item is one row's 32-element block: 16 bytes of codes and its scale in, 64
// bytes of bf16 out.
__device__ void stream_convert_f16(const EngineParams& p, uint8_t* smem, int ci, RoleState& rs) {
  const int lane = threadIdx.x & 31;
  JobEntry* jq = job_queue(smem, 0);
  bool ok = true;
  for (;;) {
    JobEntry* en = jq + (rs.qk % JQ);
    if (!wait_entry(p, en, rs.qk)) return;
    const int job = *reinterpret_cast<volatile int32_t*>(&en->job);
    if (job < 0) { ++rs.qk; break; }
    const int s0 = en->s0, nh = en->nc;
    ++rs.qk;
    if (!ok) continue;
    for (int h = 0; h < nh; ++h) {
      const uint32_t r = (uint32_t)s0 + h;
      const int ri = (int)(r % FT_RA), ai = (int)(r % FT_AB);
      if (!warp_wait(rawfull_bar(smem, ri), (r / FT_RA) & 1u, p, r) ||
          (r >= (uint32_t)FT_AB && !warp_wait(aempty_bar(smem, ai), ((r / FT_AB) + 1) & 1u, p, r))) {
        ok = false;
        break;
      }
      const uint8_t* raw = ft_raw(smem, ri);
      uint8_t* out = ft_a(smem, ai);
      const int kb0 = 2 * (h & 1);  // scale blocks of this half
      for (int it = ci * 32 + lane; it < 256; it += FT_CONV_WARPS * 32) {
        const int m = it & 127, blk = it >> 7;
        const uint4 cw = *reinterpret_cast<const uint4*>(raw + (m >> 3) * 256 + blk * 128 + (m & 7) * 16);
        const uint32_t sb = raw[4096 + (m & 31) * 16 + (m >> 5) * 4 + kb0 + blk];
        uint32_t lo[2], hi[2];
        e2m1_bf16_tables(sb, lo, hi);
        const uint32_t w[4] = {cw.x, cw.y, cw.z, cw.w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {  // elements 32 blk + 8 q .. + 7 of the half: chunk j = 4 blk + q
          uint4 o;
          e2m1x4_bf16(w[q] & 0xFFFFu, lo, hi, o.x, o.y);
          e2m1x4_bf16(w[q] >> 16, lo, hi, o.z, o.w);
          const int jc = 4 * blk + q;
          *reinterpret_cast<uint4*>(out + (jc >> 1) * 4096 + (m >> 3) * 256 + (jc & 1) * 128 + (m & 7) * 16) = o;
        }
      }
      fence_proxy_async_smem();  // the bf16 block is read by the tensor cores (async proxy)
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(afull_bar(smem, ai));
        mbar_arrive(rawempty_bar(smem, ri));
      }
    }
  }
}

// MMA issuer of the bf16 tile stream: per half-stage and B block 4 MMAs of
// K = 16 (M = 128, N = n16) into the job's accumulator.
__device__ void stream_mma_f16(const EngineParams& p, uint8_t* smem, uint32_t tmem, RoleState& rs) {
  JobEntry* jq = job_queue(smem, 0);
  const bool prof = p.prof != nullptr;
  unsigned long long t_full = 0, t_issue = 0, t_acc = 0;
  bool ok = true;
  for (;;) {
    JobEntry* en = jq + (rs.qk % JQ);
    if (!wait_entry(p, en, rs.qk)) return;
    const int job = *reinterpret_cast<volatile int32_t*>(&en->job);
    if (job < 0) { ++rs.qk; break; }
    const int s0 = en->s0, nh = en->nc, nt = en->nt, wj = en->wj, isD = en->isD, b0 = en->pad;
    ++rs.qk;
    if (!ok) continue;
    const int b = wj & 1;
    const uint32_t use = (uint32_t)(wj >> 1);
    const unsigned long long ta0 = pclock(prof);
    if (use > 0 && !wait_mbar(acce_bar(smem, 0, b), (use - 1) & 1u, p.sync, p.timeout_ns, DEV_TIMEOUT_PIPE, wj)) {
      ok = false;
      continue;
    }
    t_acc += pclock(prof) - ta0;
    tc_fence_after();
    const uint32_t tacc = tmem + (uint32_t)(b * FT_ACC_COLS);
    const int n16 = (nt + 15) & ~15, terms = isD ? 2 : 1;
    const uint32_t idesc = f16_idesc(n16);
    for (int h = 0; h < nh && ok; ++h) {
      const uint32_t r = (uint32_t)s0 + h;
      const int ai = (int)(r % FT_AB);
      const unsigned long long tf0 = pclock(prof);
      if (!wait_mbar(afull_bar(smem, ai), (r / FT_AB) & 1u, p.sync, p.timeout_ns, DEV_TIMEOUT_PIPE, r)) {
        ok = false;
        break;
      }
      t_full += pclock(prof) - tf0;
      const uint32_t sa = smem_u32(ft_a(smem, ai));
      for (int t = 0; t < terms; ++t) {
        const uint32_t bq = (uint32_t)b0 + h * terms + t;
        const int bi = (int)(bq % FT_NB);
        const unsigned long long tb0 = pclock(prof);
        if (!wait_mbar(bfull_bar(smem, bi), (bq / FT_NB) & 1u, p.sync, p.timeout_ns, DEV_TIMEOUT_PIPE, bq)) {
          ok = false;
          break;
        }
        const unsigned long long tm0 = pclock(prof);
        t_full += tm0 - tb0;
        tc_fence_after();
        const uint32_t sb = smem_u32(ft_b(smem, bi));
#pragma unroll
        for (int k16 = 0; k16 < FT_HK / 16; ++k16)
          mma_bf16(tacc, smem_desc(sa + k16 * 4096, 128, 256), smem_desc(sb + k16 * n16 * 32, 128, 256), idesc,
                   (h > 0 || t > 0 || k16 > 0) ? 1u : 0u);
        tc_commit(bempty_bar(smem, bi));
        t_issue += pclock(prof) - tm0;
      }
      if (!ok) break;
      tc_commit(aempty_bar(smem, ai));
    }
    if (ok) tc_commit(accf_bar(smem, 0, b));
  }
  if (prof) {
    atomicAdd(p.prof + PF_MMA_FULL, t_full);
    atomicAdd(p.prof + PF_MMA_ISSUE, t_issue);
    atomicAdd(p.prof + PF_MMA_ACC, t_acc);
  }
}

// Epilogue warps of the bf16 tile stream (warp q reads accumulator rows
// 32 q..32 q + 31).  Gate/up: SwiGLU of the gate and up rows (lanes l and
// l + 16), written as two bf16 terms into the tile's down B blocks.  Down:
// each position's column times its routing weight.
__device__ void stream_epilogue_f16(const EngineParams& p, uint8_t* smem, const StreamCtx& cx, uint32_t tmem,
                                    RoleState& rs) {
  const int lane = threadIdx.x & 31, q = (threadIdx.x >> 5) & 3;
  JobEntry* jq = job_queue(smem, 0);
  uint32_t* ready = p.sync + SY_READY;
  const int nhd = p.I / FT_HK;
  const bool prof = p.prof != nullptr;
  unsigned long long t_wait = 0, t_work = 0, n_jobs = 0;
  const unsigned long long t_begin = pclock(prof);
  bool ok = true;
  for (;;) {
    JobEntry* en = jq + (rs.qk % JQ);
    if (!wait_entry(p, en, rs.qk)) return;
    const int job = *reinterpret_cast<volatile int32_t*>(&en->job);
    if (job < 0) { ++rs.qk; break; }
    const int wj = en->wj;
    const int u = en->unit, rb = en->rb, isD = en->isD, pos0 = en->pos0, nt = en->nt;
    ++rs.qk;
    if (!ok) continue;
    ++n_jobs;
    const int b = wj & 1;
    const unsigned long long tw0 = pclock(prof);
    if (!wait_mbar(accf_bar(smem, 0, b), (uint32_t)(wj >> 1) & 1u, p.sync, p.timeout_ns, DEV_TIMEOUT_PIPE, wj)) {
      ok = false;
      continue;
    }
    const unsigned long long tk0 = pclock(prof);
    t_wait += tk0 - tw0;
    tc_fence_after();
    const uint32_t tacc = tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)(b * FT_ACC_COLS);
    const int n16 = (nt + 15) & ~15;
    if (!isD) {
      // rows 32 q + l: gate of I row i0 + 16 q + l for l < 16, up of the same row for l >= 16
      const int i = rb * GU_I_ROWS + 16 * q + (lane & 15);
      const int hD = i / FT_HK, k = i % FT_HK;
      uint8_t* dst = p.atf + ((int64_t)u * nhd + hD) * 2 * FT_TERM_BYTES;
      for (int j0 = 0; j0 < nt; j0 += 8) {
        float v[8];
        tmem_ld8(tacc + j0, v);
#pragma unroll
        for (int jj = 0; jj < 8; ++jj) {
          const float other = __shfl_xor_sync(FULL, v[jj], 16);
          const int j = j0 + jj;
          if (lane < 16 && j < nt) {
            const float g = v[jj], up = other;
            const float a = g / (1.0f + expf(-g)) * up;
            const __nv_bfloat16 h0 = __float2bfloat16_rn(a);
            const __nv_bfloat16 h1 = __float2bfloat16_rn(a - __bfloat162float(h0));
            *reinterpret_cast<__nv_bfloat16*>(dst + ft_b_offset(j, k, n16)) = h0;
            *reinterpret_cast<__nv_bfloat16*>(dst + FT_TERM_BYTES + ft_b_offset(j, k, n16)) = h1;
          }
        }
      }
      __syncwarp();
      if (lane == 0) {
        fence_proxy_async_global();
        __threadfence();
        red_release_add_u32(ready + u, 1u);
      }
    } else {
      const int hrow = rb * JOB_ROWS + 32 * q + lane;
      for (int j0 = 0; j0 < nt; j0 += 8) {
        float v[8];
        tmem_ld8(tacc + j0, v);
#pragma unroll
        for (int jj = 0; jj < 8; ++jj) {
          const int j = j0 + jj;
          if (j < nt) p.ypair[(int64_t)(pos0 + j) * p.H + hrow] = v[jj] * ld_tab(cx.wpos + pos0 + j, cx.global);
        }
      }
    }
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(acce_bar(smem, 0, b));
    t_work += pclock(prof) - tk0;
  }
  if (prof && lane == 0) {
    atomicAdd(p.prof + PF_EPI_WAIT, t_wait);
    atomicAdd(p.prof + PF_EPI_WORK, t_work);
    atomicAdd(p.prof + PF_EPI_TOTAL, pclock(prof) - t_begin);
    if (q == 0) atomicAdd(p.prof + PF_JOBS, n_jobs);
  }
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

// I-sharded layer, last step: the fused one-shot all-reduce (see AllReduce in
// engine.cuh).  This rank's fp32 partial (the slot-order combine) goes to slot
// epoch % 2 of its own region; after a grid barrier CTA 0 publishes the epoch
// to every rank (system-scope release); every CTA waits, bounded, until every
// rank's epoch is in its own region (system-scope acquire), then sums its
// share of [T][H] over the ranks in rank order -- the same operations on
// every rank, so every rank's y is bit-identical -- and rounds to bf16.
// Returns false (every thread of the CTA) on a timeout or a recorded error.
__device__ bool phase_allreduce_out(const EngineParams& p, const int32_t* inv, int layer) {
  const int64_t gt = (int64_t)blockIdx.x * THREADS + threadIdx.x;
  const int64_t gs = (int64_t)gridDim.x * THREADS;
  const int H4 = p.H / 4, world = p.ar.world, rank = p.ar.rank;
  const uint32_t epoch = p.ar.epoch;
  const int64_t slot = (int64_t)(epoch & 1u) * p.ar.slot_floats;
  float* mine = reinterpret_cast<float*>(p.ar.region[rank] + AR_FLAG_BYTES) + slot;
  for (int64_t g = gt; g < (int64_t)p.T * H4; g += gs) {
    const int t = (int)(g / H4), h = (int)(g % H4) * 4;
    *reinterpret_cast<float4*>(mine + (int64_t)t * p.H + h) = combine4(p, inv, t, h);
  }
  if (!grid_barrier(p.sync, p.timeout_ns, 10 * layer + 8)) return false;
  if (blockIdx.x == 0 && (int)threadIdx.x < world) {
    // the barrier acquired every CTA's partial; make it visible system-wide
    // before the epoch
    __threadfence_system();
    st_release_sys_u32(reinterpret_cast<uint32_t*>(p.ar.region[threadIdx.x]) + rank, epoch);
  }
  int ok = 1;
  if (threadIdx.x == 0) {
    const uint32_t* flags = reinterpret_cast<const uint32_t*>(p.ar.region[rank]);
    const uint64_t t0 = globaltimer_ns();
    for (int r = 0; r < world && ok; ++r) {
      uint32_t spins = 0;
      while (ld_acquire_sys_u32(flags + r) < epoch) {
        if ((++spins & 15u) == 0u) {
          if (error_set(p.sync)) { ok = 0; break; }
          if (globaltimer_ns() - t0 > p.timeout_ns) { set_error(p.sync, DEV_TIMEOUT_PEER, (uint32_t)r); ok = 0; break; }
        }
        __nanosleep(64);
      }
    }
  }
  if (!__syncthreads_and(ok)) return false;
  __nv_bfloat16* dump = p.layer_io ? p.layer_io + (int64_t)p.L * p.T * p.H : nullptr;
  for (int64_t g = gt; g < (int64_t)p.T * H4; g += gs) {
    const int t = (int)(g / H4), h = (int)(g % H4) * 4;
    const int64_t off = slot + (int64_t)t * p.H + h;
    float4 s = ld_volatile_f4(reinterpret_cast<const float*>(p.ar.region[0] + AR_FLAG_BYTES) + off);
    for (int r = 1; r < world; ++r) {
      const float4 v = ld_volatile_f4(reinterpret_cast<const float*>(p.ar.region[r] + AR_FLAG_BYTES) + off);
      s.x += v.x; s.y += v.y; s.z += v.z; s.w += v.w;
    }
    store_bf16x4(p.y_out + (int64_t)t * p.H + h, s);
    if (dump) store_bf16x4(dump + (int64_t)t * p.H + h, s);
  }
  return true;
}

// RMSNorm between chained layers: y = bf16(combine); x_next = bf16(y * r),
// r = 1 / sqrt(mean(y^2) + eps).  A token's H values are cut into RMS_CHUNKS
// chunks.  The sum of squares of a chunk is reduced in a fixed order (each
// thread one float4, then the warp, then the warps in order), and a token's
// sum is its chunk sums added in chunk order, so the result does not depend
// on how chunks are spread over CTAs.  The engine spreads the T * RMS_CHUNKS
// chunks over the whole grid (partial sums, a grid barrier, then the scaling
// of each chunk); the operator-by-operator launch runs all chunks of a token
// in one CTA.  Both give the same bits.
constexpr int RMS_CHUNKS = 8;
static_assert(8192 / RMS_CHUNKS / 4 <= THREADS, "one float4 of a chunk per thread");

// The bf16-rounded combine of this thread's float4 of chunk c of token t (zero
// past the chunk): the k slot loads are issued before the adds, which stay in
// slot order.  (Scalar arguments: out-of-line callers must not take the
// kernel's parameter block by reference.)
__device__ __forceinline__ float4 rms_chunk_values(const float* ypair, const int32_t* inv, int K, int H, int t,
                                                   int c, bool& mine) {
  const int cl4 = H / RMS_CHUNKS / 4;
  mine = (int)threadIdx.x < cl4;
  float4 s = make_float4(0.f, 0.f, 0.f, 0.f);
  if (mine) {
    const int h = c * (H / RMS_CHUNKS) + 4 * (int)threadIdx.x;
    for (int s0 = 0; s0 < K; s0 += 8) {
      float4 v[8];
#pragma unroll
      for (int i = 0; i < 8; ++i)
        if (s0 + i < K) v[i] = __ldcg(reinterpret_cast<const float4*>(ypair + (int64_t)inv[t * K + s0 + i] * H + h));
#pragma unroll
      for (int i = 0; i < 8; ++i)
        if (s0 + i < K) { s.x += v[i].x; s.y += v[i].y; s.z += v[i].z; s.w += v[i].w; }
    }
    s.x = __bfloat162float(__float2bfloat16_rn(s.x));
    s.y = __bfloat162float(__float2bfloat16_rn(s.y));
    s.z = __bfloat162float(__float2bfloat16_rn(s.z));
    s.w = __bfloat162float(__float2bfloat16_rn(s.w));
  }
  return s;
}

// Sum of squares of the values v (this thread's part of one chunk), fixed
// reduction order; every thread of the CTA gets the result.
__device__ float rms_chunk_ss(float4 v, float* red) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  float ss = v.x * v.x + v.y * v.y + v.z * v.z + v.w * v.w;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(FULL, ss, o);
  __syncthreads();  // red is free
  if (lane == 0) red[warp] = ss;
  __syncthreads();
  float tot = 0.f;
#pragma unroll
  for (int w = 0; w < WARPS; ++w) tot += red[w];
  return tot;
}

// x_next chunk = bf16(v * 1 / sqrt(tot / H + eps)).
__device__ __forceinline__ void rms_chunk_store(__nv_bfloat16* xnext, int H, float eps, int t, int c, float4 v,
                                                bool mine, float tot) {
  const float r = 1.0f / sqrtf(tot / (float)H + eps);
  if (mine)
    store_bf16x4(xnext + (int64_t)t * H + c * (H / RMS_CHUNKS) + 4 * (int)threadIdx.x,
                 make_float4(v.x * r, v.y * r, v.z * r, v.w * r));
}

// Engine: the chunk sums of squares of every (token, chunk) task, spread over
// the grid, into part[t * RMS_CHUNKS + c]; a grid barrier; then each token's
// sum from its chunk sums in chunk order and the scaled bf16 values of every
// task's chunk.  A CTA's first task keeps its values in registers across the
// barrier; further tasks (more than one per CTA) recompute them.  Returns
// false on a barrier timeout or a recorded error.
__device__ bool phase_rms(const float* ypair, const int32_t* inv, int K, int H, int T, float eps,
                                       __nv_bfloat16* xnext, float* part, float* red, uint32_t* sync,
                                       uint64_t timeout_ns, uint32_t where) {
  const int ntask = T * RMS_CHUNKS;
  float4 v0 = make_float4(0.f, 0.f, 0.f, 0.f);
  bool mine0 = false;
  for (int task = blockIdx.x; task < ntask; task += gridDim.x) {
    bool mine;
    const float4 v = rms_chunk_values(ypair, inv, K, H, task / RMS_CHUNKS, task % RMS_CHUNKS, mine);
    const float ss = rms_chunk_ss(v, red);
    if (threadIdx.x == 0) part[task] = ss;
    if (task == (int)blockIdx.x) { v0 = v; mine0 = mine; }
  }
  if (!grid_barrier(sync, timeout_ns, where)) return false;
  for (int task = blockIdx.x; task < ntask; task += gridDim.x) {
    const int t = task / RMS_CHUNKS, c = task % RMS_CHUNKS;
    float tot = 0.f;
#pragma unroll
    for (int q = 0; q < RMS_CHUNKS; ++q) tot += __ldcg(part + t * RMS_CHUNKS + q);
    bool mine = mine0;
    float4 v = v0;
    if (task != (int)blockIdx.x) v = rms_chunk_values(ypair, inv, K, H, t, c, mine);
    rms_chunk_store(xnext, H, eps, t, c, v, mine, tot);
  }
  return true;
}

// Operator-by-operator launch: every chunk of a token in one CTA (tokens over
// the CTAs), the same arithmetic in the same order as phase_rms.
__device__ void phase_combine_rmsnorm(const EngineParams& p, const int32_t* inv, uint8_t* smem) {
  CtaTables& tb = tables(smem);
  for (int t = blockIdx.x; t < p.T; t += gridDim.x) {
    float tot = 0.f;
    for (int c = 0; c < RMS_CHUNKS; ++c) {
      bool mine;
      tot += rms_chunk_ss(rms_chunk_values(p.ypair, inv, p.K, p.H, t, c, mine), tb.red);
    }
    for (int c = 0; c < RMS_CHUNKS; ++c) {
      bool mine;
      const float4 v = rms_chunk_values(p.ypair, inv, p.K, p.H, t, c, mine);
      rms_chunk_store(p.xnext, p.H, p.rms_eps, t, c, v, mine, tot);
    }
    __syncthreads();
  }
}

// L2 prefetch of this CTA's 1/gridDim share of `bytes` (a multiple of 16) at
// `base` (16-byte aligned), in bulk prefetches of at most 16 KB.
__device__ void prefetch_share(const void* base, size_t bytes) {
  const size_t share = ((bytes + gridDim.x - 1) / gridDim.x + 15) & ~size_t(15);
  const size_t b0 = (size_t)blockIdx.x * share;
  if (b0 >= bytes) return;
  const size_t b1 = b0 + share < bytes ? b0 + share : bytes;
  for (size_t o = b0; o < b1; o += 16384) {
    const size_t n = b1 - o < 16384 ? b1 - o : 16384;
    prefetch_l2_bulk(static_cast<const uint8_t*>(base) + o, (uint32_t)n);
  }
}

// All layers; returns early (every thread of the CTA together) when a grid
// barrier reports an error, or after routing in route-only mode.
// MODE 0: pipeline stream, one layer, plain combine (the decode kernel); MODE 5:
// pipeline stream with chained layers (RMSNorm) or the fused all-reduce; MODE 1:
// E2M1 term tiles (kind::mxf4); MODE 4: E2M1 term tile pairs (two row blocks per
// job); MODE 6: E4M3 term tiles (kind::mxf8f6f4); MODE 2: bf16 tiles
// (kind::f16).  The tile modes run only above SMALL_PAIRS.
template <int MODE>
__device__ void run_layers(const EngineParams& p, uint8_t* smem, uint32_t tmem, RoleState& rs,
                           bool stamp) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  constexpr bool PIPE = MODE == 0 || MODE == 5 || MODE == 7;  // pipeline stream (MODE 7: big units)
  // MODE 0 is launched only for T*K <= SMALL_PAIRS: its routing is always per CTA
  const bool small = PIPE && MODE != 7 && (MODE == 0 || p.TK <= SMALL_PAIRS);
  CtaTables& tb = tables(smem);
  for (int layer = 0; layer < p.L; ++layer) {
    const LayerPtrs& lp = p.layers[layer];
    const __nv_bfloat16* x = layer == 0 ? p.x_in : p.xnext;
    uint64_t* st = stamp ? p.stamps + 1 + layer * STAMPS_PER_LAYER : nullptr;
    // the fp64 MMA router wherever the routing is grid-wide (T*K > SMALL_PAIRS):
    // from a few dozen tokens its 8-token tiles are full enough to pay
    if constexpr (!PIPE) phase_router_tiles(x, lp.router_w, p.logits, p.sync, p.T, p.H, p.E, p.TK, p.HS, smem);
    else if (MODE != 0 && !small) phase_router_tiles(x, lp.router_w, p.logits, p.sync, p.T, p.H, p.E, p.TK, p.HS, smem);
    else phase_router<MODE == 5 ? 10 : 2, MODE == 5>(p, lp, x, smem);
    if (st) st[0] = globaltimer_ns();
    StreamCtx cx;
    const int32_t* inv;
    if (small) {
      if (!route_barrier(p, lp, x, layer, smem, 10 * layer + 1, st ? st + 1 : nullptr)) return;
      if (p.route_only) return;
      if (st) st[3] = globaltimer_ns();
      cx = StreamCtx{tb.units, tb.dunits, tb.tokpos, tb.wpos, tb.n_units, tb.n_dunits, false};
      inv = tb.inv;
    } else {
      if constexpr (MODE == 6) phase_images_e4m3(p, x, layer);
      else if constexpr (MODE == 1 || MODE == 4) phase_images<LT_NTERM>(p, x, layer);
      else if constexpr (MODE != 2) phase_images(p, x, layer);  // the bf16 tiles gather x itself
      if (st) st[1] = globaltimer_ns();
      if (!grid_barrier(p.sync, p.timeout_ns, 10 * layer + 1)) return;
      if (st) st[2] = globaltimer_ns();
      phase_topk_large(p, lp);
      if (!grid_barrier(p.sync, p.timeout_ns, 10 * layer + 2)) return;
      if (st) st[3] = globaltimer_ns();
      if constexpr (MODE == 2) phase_permute_f16(p, smem);
      else phase_permute_large(p, smem, MODE == 6 ? ET_MAX : MODE == 4 ? LTA_MAX : MODE == 1 ? LT_MAX : MODE == 7 ? NT_BIG : NT_MAX);
      if (!grid_barrier(p.sync, p.timeout_ns, 10 * layer + 3)) return;
      if (p.route_only) return;
      if constexpr (MODE == 1 || MODE == 4) {
        phase_tile_gather(p);
        if (!grid_barrier(p.sync, p.timeout_ns, 10 * layer + 6)) return;
      } else if constexpr (MODE == 7) {
        phase_pos_gather(p);
        if (!grid_barrier(p.sync, p.timeout_ns, 10 * layer + 6)) return;
      } else if constexpr (MODE == 6) {
        phase_tile_gather_e4m3(p);
        if (!grid_barrier(p.sync, p.timeout_ns, 10 * layer + 6)) return;
      } else if constexpr (MODE == 2) {
        phase_tile_gather_f16(p, x);
        if (!grid_barrier(p.sync, p.timeout_ns, 10 * layer + 6)) return;
      }
      cx = StreamCtx{p.units, p.dunits, p.tokpos, p.wpos, (int)ld_cg_u32(p.n_units), (int)ld_cg_u32(p.n_units + 1), true};
      inv = p.inv;
    }
    if (st) st[4] = globaltimer_ns();
    // the next layer's router weights go to L2 while this layer streams (its
    // expert weights are evict-first, so they stay): every CTA prefetches its
    // share, a few tens of KB, without waiting for it
    if (layer + 1 < p.L && threadIdx.x == 32 * (WARPS - 1))
      prefetch_share(p.layers[layer + 1].router_w, (size_t)p.E * p.H * 4);
    fence_proxy_async_smem();  // the ring held routing scratch written by generic stores
    __syncthreads();
    if constexpr (PIPE) {  // two pipelines per CTA, units of <= NT_MAX (MODE 7: NT_BIG) positions
      constexpr int U = MODE == 7 ? NT_BIG : NT_MAX;
      if (warp < EPI_WARP0) {
        const int pipe = warp >> 1;
        if ((warp & 1) == 0) {
          stream_producer<MODE == 7 ? 7 : 0>(p, lp, smem, cx, pipe, rs);
        } else {
          if (lane == 0) stream_mma<U>(p, smem, tmem, pipe, rs);
          __syncwarp();
        }
      } else {
        stream_epilogue<U>(p, smem, cx, tmem, (warp - EPI_WARP0) / 4, rs);
      }
    } else if constexpr (MODE == 1 || MODE == 4) {  // one pipeline per CTA over tiles (pairs)
      if (warp == 0) {
        stream_producer<MODE>(p, lp, smem, cx, 0, rs);
      } else if (warp == 1) {
        if (lane == 0) stream_mma_lt<MODE>(p, smem, tmem, rs);
        __syncwarp();
      } else if (warp >= EPI_WARP0) {
        stream_epilogue_lt<MODE>(p, smem, cx, tmem, warp >= EPI_WARP0 + 4 ? 1 : 0, rs);
      }
    } else if constexpr (MODE == 6) {  // E4M3 tiles: producer, MMA issuer, two converter warps, eight epilogue warps
      if (warp == 0) {
        stream_producer<6>(p, lp, smem, cx, 0, rs);
      } else if (warp == 1) {
        if (lane == 0) stream_mma_e(p, smem, tmem, rs);
        __syncwarp();
      } else if (warp < EPI_WARP0) {
        stream_convert_e(p, smem, warp - 2, rs);
      } else {
        stream_epilogue_e(p, smem, cx, tmem, warp >= EPI_WARP0 + 4 ? 1 : 0, rs);
      }
    } else {  // bf16 tiles: producer, MMA issuer, six converter warps, four epilogue warps
      if (warp == 0) {
        stream_producer_f16(p, lp, smem, cx, rs);
      } else if (warp == 1) {
        if (lane == 0) stream_mma_f16(p, smem, tmem, rs);
        __syncwarp();
      } else if (warp >= EPI_WARP0 && warp < EPI_WARP0 + 4) {
        stream_epilogue_f16(p, smem, cx, tmem, rs);
      } else {
        stream_convert_f16(p, smem, warp < EPI_WARP0 ? warp - 2 : warp - 6, rs);
      }
    }
    if (!grid_barrier(p.sync, p.timeout_ns, 10 * layer + 4)) return;
    if (st) st[5] = globaltimer_ns();
    // every producer has passed its image wait and every CTA has counted
    // itself: the count restarts for the next layer or launch
    if (blockIdx.x == 0 && threadIdx.x == 0) { p.sync[SY_XDONE] = 0u; p.sync[SY_IMGQ] = 0u; }
    // MODE 0 runs single layers without the all-reduce (launch rule), so the
    // decode kernel carries neither the RMSNorm nor the all-reduce code
    if (MODE != 0 && layer + 1 < p.L) {
      // the partial logits are not read again in this layer: they hold the
      // chunk sums of squares until the next layer's router overwrites them
      if (!phase_rms(p.ypair, inv, p.K, p.H, p.T, p.rms_eps, p.xnext, reinterpret_cast<float*>(p.logits),
                     tb.red, p.sync, p.timeout_ns, 10 * layer + 7))
        return;
      if (!grid_barrier(p.sync, p.timeout_ns, 10 * layer + 5)) return;
    } else if (MODE != 0 && p.ar.world > 0) {
      if (!phase_allreduce_out(p, inv, layer)) return;
    } else {
      phase_combine_out(p, inv);
    }
    if (st) st[6] = globaltimer_ns();
  }
}

// One operator of one layer per launch (MODE 3): the same phases as the
// engine's small-T*K layer, with a kernel boundary instead of each grid-wide
// wait.  The tables come from global memory; the down jobs start only after
// every gate/up job has finished (their own launch).  Under programmatic
// dependent launch a grid waits for its predecessor before it touches
// anything, and lets its successor be scheduled right after that.
template <int SPLIT>
__device__ void op_stream(const EngineParams& p, const LayerPtrs& lp, uint8_t* smem, uint32_t tmem,
                          RoleState& rs) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const StreamCtx cx{p.units, p.dunits, p.tokpos, p.wpos, (int)ld_cg_u32(p.n_units),
                     (int)ld_cg_u32(p.n_units + 1), true};
  if (warp < EPI_WARP0) {
    const int pipe = warp >> 1;
    if ((warp & 1) == 0) {
      stream_producer<0, SPLIT>(p, lp, smem, cx, pipe, rs);
    } else {
      if (lane == 0) stream_mma(p, smem, tmem, pipe, rs);
      __syncwarp();
    }
  } else {
    stream_epilogue(p, smem, cx, tmem, (warp - EPI_WARP0) / 4, rs);
  }
}

__device__ void run_op(const EngineParams& p, uint8_t* smem, uint32_t tmem, RoleState& rs) {
  const int layer = p.op_layer;
  const LayerPtrs& lp = p.layers[layer];
  const __nv_bfloat16* x = layer == 0 ? p.x_in : p.xnext;
  grid_dependency_wait();
  grid_launch_dependents();
  switch (p.op) {
    case OP_ROUTER: phase_router(p, lp, x, smem); break;
    case OP_ROUTE:
      if (threadIdx.x == 0) p.sync[SY_JOBS2] = 0u;
      phase_route_small(p, lp, smem);
      break;
    case OP_IMAGES: phase_images(p, x, layer); break;
    case OP_GATEUP: op_stream<1>(p, lp, smem, tmem, rs); break;
    case OP_DOWN: op_stream<2>(p, lp, smem, tmem, rs); break;
    case OP_COMBINE:
      if (layer + 1 < p.L) phase_combine_rmsnorm(p, p.inv, smem);
      else phase_combine_out(p, p.inv);
      break;
    default: break;
  }
}

// Seven instances: MODE 0, 1, 2, 4, 5, 6 (see run_layers), each holding only
// its own stream code, and MODE 3, one operator per launch (run_op).
template <int MODE>
__global__ void __launch_bounds__(THREADS, 1) engine_kernel(const EngineParams p) {
  extern __shared__ __align__(1024) uint8_t smem[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int pp = 0; pp < NPIPE; ++pp) {
      for (int i = 0; i < NSLOT; ++i) {
        // bf16 tiles: a raw slot is free once every converter warp has read
        // it (rawempty_bar), an A block is full once every converter warp
        // has written it (afull_bar)
        // E4M3 tiles: pipe 1's full barriers announce the converted weight codes (two warps)
        mbar_init(full_bar(smem, pp, i), MODE == 2 && pp == 1 && i >= FT_NB ? FT_CONV_WARPS
                                         : MODE == 6 && pp == 1 ? 2 : 1);
        mbar_init(empty_bar(smem, pp, i), MODE == 2 && pp == 0 ? FT_CONV_WARPS : 1);
      }
      for (int i = 0; i < NACC; ++i) {
        mbar_init(accf_bar(smem, pp, i), 1);
        mbar_init(acce_bar(smem, pp, i), (MODE == 1 || MODE == 4 || MODE == 6) && pp == 0 ? 8 : 4);  // tiles: eight epilogue warps
      }
      for (int i = 0; i < 2; ++i) mbar_init(xch_bar(smem, pp, i), 4);
      mbar_init(drain_bar(smem, pp), 1);
    }
    fence_mbar_init();
  }
  for (int i = threadIdx.x; i < NPIPE * JQ; i += THREADS) job_queue(smem, 0)[i].flag = 0;
  const bool use_tmem = !p.route_only && (MODE != 3 || p.op == OP_GATEUP || p.op == OP_DOWN);
  if (use_tmem && warp == 1) {
    tmem_alloc(tmem_base_word(smem), TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = use_tmem ? *tmem_base_word(smem) : 0u;
  const bool stamp = MODE != 3 && p.stamps != nullptr && blockIdx.x == 0 && threadIdx.x == 0;
  if (stamp) p.stamps[0] = globaltimer_ns();
  RoleState rs;
  if constexpr (MODE == 3) run_op(p, smem, tmem, rs);
  else run_layers<MODE>(p, smem, tmem, rs, stamp);
  if (use_tmem) {
    // free tensor memory only once every MMA this CTA issued has completed
    if (warp < EPI_WARP0 && (warp & 1) && lane == 0) {
      uint64_t* db = drain_bar(smem, warp >> 1);
      tc_commit(db);
      const uint64_t t0 = globaltimer_ns();
      while (!mbar_try_wait(db, 0u)) {
        if (globaltimer_ns() - t0 > DRAIN_NS) { set_error(p.sync, DEV_TIMEOUT_PIPE, 0xFFFFu); break; }
      }
    }
    __syncwarp();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem, TMEM_COLS);
  }
}

}  // namespace

size_t engine_smem_bytes() { return SMEM_BYTES; }

int engine_max_grid(int device, int* err) {
  int per_sm = ~0u >> 1, sms = 0;
  for (const void* k : {(const void*)engine_kernel<0>, (const void*)engine_kernel<1>, (const void*)engine_kernel<2>,
                        (const void*)engine_kernel<3>, (const void*)engine_kernel<4>, (const void*)engine_kernel<5>,
                        (const void*)engine_kernel<6>, (const void*)engine_kernel<7>}) {
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM_BYTES);
    if (e != cudaSuccess) { *err = (int)e; return 0; }
    int n = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, k, THREADS, SMEM_BYTES);
    if (e != cudaSuccess) { *err = (int)e; return 0; }
    per_sm = n < per_sm ? n : per_sm;
  }
  cudaError_t e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, device);
  if (e != cudaSuccess) { *err = (int)e; return 0; }
  *err = 0;
  return per_sm * sms;
}

cudaError_t engine_launch(const EngineParams& p, int grid, cudaStream_t s) {
  void* args[] = {const_cast<EngineParams*>(&p)};
  // MODE 0's launch rule: routing per CTA (T*K <= SMALL_PAIRS), one layer, no
  // all-reduce (or routing only); big units (MODE 7) for grid-wide routing
  // with at least BIG_MIN_PER_EXPERT positions per expert; every other
  // pipeline launch takes MODE 5
  const bool plain = p.TK <= SMALL_PAIRS && ((p.L == 1 && p.ar.world == 0) || p.route_only);
  const void* pipe_k = plain                                         ? (const void*)engine_kernel<0>
                       : !p.route_only && use_big_units(p.TK, p.E) ? (const void*)engine_kernel<7>
                                                                     : (const void*)engine_kernel<5>;
  const void* k = !use_tiles(p.TK, p.E) || p.route_only ? pipe_k
                  : p.large == LARGE_F16                  ? (const void*)engine_kernel<2>
                  : p.large == LARGE_MXF8                 ? (const void*)engine_kernel<6>
                  : use_tile_pairs(p.TK, p.E, p.H)         ? (const void*)engine_kernel<4>
                                                          : (const void*)engine_kernel<1>;
  return cudaLaunchCooperativeKernel(k, dim3(grid), dim3(THREADS), args, SMEM_BYTES, s);
}

cudaError_t engine_launch_ops(const EngineParams& p0, int grid, bool pdl, cudaStream_t s) {
  EngineParams p = p0;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.blockDim = dim3(THREADS);
  cfg.dynamicSmemBytes = SMEM_BYTES;
  cfg.stream = s;
  cfg.attrs = pdl ? attr : nullptr;
  cfg.numAttrs = pdl ? 1 : 0;
  for (int l = 0; l < p0.L; ++l) {
    for (int op = OP_ROUTER; op <= OP_COUNT; ++op) {
      p.op = op;
      p.op_layer = l;
      // routing is one CTA's work; an RMSNorm combine takes one CTA per token
      const int g = op == OP_ROUTE ? 1 : (op == OP_COMBINE && l + 1 < p0.L ? (p0.T < grid ? p0.T : grid) : grid);
      cfg.gridDim = dim3(g);
      const cudaError_t e = cudaLaunchKernelEx(&cfg, engine_kernel<3>, p);
      if (e != cudaSuccess) return e;
    }
  }
  return cudaSuccess;
}

}  // namespace moe
