// Speculative-verify acceptance step (rejection sampling over verify blocks),
// one cooperative launch.  The contract is in include/spec_verify.h.
//
// Four phases, separated by bounded grid-wide barriers (the last one only
// above 16 blocks):
//   rows     every (block, row, 512-entry segment): the segment's max m and
//            z = sum exp(l - m) (fp64), one warp each;
//   decide   every block (one CTA): each row's max M and Z = sum z exp(m - M)
//            (a warp per row, the statistics read once), then the block's
//            acceptance tests (one lane per draft, inputs loaded before the
//            rows' work); it records n and the drawn row's normalisers;
//   weights  every (block, 256-entry segment) of the row the block draws
//            from: the weights' segment sum (each lane 8 consecutive entries,
//            lane sums scanned in a fixed order);
//   draw     every block, one warp each (up to 16 blocks on the last CTA to
//            finish its weight sums, the other CTAs exiting; else after a
//            third barrier on every CTA): the segment, then the entry, whose
//            cumulative weight first exceeds u * total.  The crossing
//            segment's weights are recomputed exactly as before, so its lane
//            sums and scan are bit-identical.
#include "spec_verify.h"

#include <cuda_runtime.h>
#include <math.h>

#include "ptx.cuh"

namespace {

using namespace moe;

constexpr unsigned FULL = 0xFFFFFFFFu;
constexpr int SV_THREADS = 512, SV_WARPS = SV_THREADS / 32;
constexpr int SEG = 512;        // vocabulary entries per statistics segment
constexpr int LPL = SEG / 32;   // ... per lane
constexpr int SEGC = 256;       // vocabulary entries per weight segment
constexpr int LPC = SEGC / 32;  // ... per lane
constexpr int SBR = 24;         // segment sums per lane loaded together in the draw
constexpr uint64_t SV_TIMEOUT_NS = 2000000000ull;

// workspace header (uint32 words), then %globaltimer stamps at byte 64
enum : int { W_COUNT = 0, W_GEN = 1, W_ERROR = 2, W_INFO = 3, W_DONE = 4 };
constexpr size_t STAMP_OFF = 64, HEADER_BYTES = 256;
enum : int { MODE_BONUS = 0, MODE_RESIDUAL = 1 };

struct Meta {  // one per block, written by its decision
  int n, mode, pad0, pad1;
  double Mt, iZt;  // target row n: max, 1 / sum of exp
  double Md, iZd;  // draft row n (residual mode)
};

struct SvParams {
  const float* lt;   // [B][G+1][V]
  const float* ld;   // [B][G][V]
  const int32_t* d;  // [B][G]
  const double* r;   // [B][G]
  const double* u;   // [B]
  int B, G, V, nseg, nsegc;
  int32_t* n_out;    // [B]
  int32_t* tok_out;  // [B][G+1]
  uint32_t* hdr;     // W_*
  double2* stat;     // [B][2G+1][nseg] (segment max, sum of exp)
  Meta* meta;        // [B]
  double* segw;      // [B][nsegc] weight sums of the drawn row
  double* segf;      // [B][nsegc] target-row sums (residual-mode fallback)
  double exp2tab[32];  // 2^(j/32), correctly rounded (host long double)
};

struct Layout {
  size_t stat, meta, segw, segf, total;
};

inline size_t up16(size_t x) { return (x + 15) & ~(size_t)15; }

inline Layout layout(int B, int G, int V) {
  const size_t R = 2 * (size_t)G + 1, ns = (size_t)(V + SEG - 1) / SEG, nc = (size_t)(V + SEGC - 1) / SEGC;
  Layout L{};
  size_t o = HEADER_BYTES;
  L.stat = o; o += (size_t)B * R * ns * sizeof(double2);
  L.meta = o; o += (size_t)B * sizeof(Meta);
  L.segw = o; o += up16((size_t)B * nc * sizeof(double));
  L.segf = o; o += up16((size_t)B * nc * sizeof(double));
  L.total = o;
  return L;
}

__device__ __forceinline__ const float* row_ptr(const SvParams& p, int b, int row) {
  return row <= p.G ? p.lt + ((size_t)b * (p.G + 1) + row) * p.V
                    : p.ld + ((size_t)b * p.G + (row - p.G - 1)) * p.V;
}

__device__ __forceinline__ bool sv_error(const uint32_t* hdr) { return ld_volatile_u32(hdr + W_ERROR) != 0u; }

__device__ __forceinline__ uint64_t* stamps(const SvParams& p) {
  return reinterpret_cast<uint64_t*>(reinterpret_cast<uint8_t*>(p.hdr) + STAMP_OFF);
}

// Bounded grid-wide barrier (generation counter); false on timeout or a
// recorded error, for every thread of the CTA.
__device__ bool sv_grid_sync(uint32_t* hdr, uint32_t where) {
  __syncthreads();
  int ok = 1;
  if (threadIdx.x == 0) {
    const uint32_t gen = ld_volatile_u32(hdr + W_GEN);
    const uint32_t prev = atom_add_acq_rel_u32(hdr + W_COUNT, 1u);
    if (prev == gridDim.x - 1) {
      *reinterpret_cast<volatile uint32_t*>(hdr + W_COUNT) = 0u;
      st_release_u32(hdr + W_GEN, gen + 1);
    } else {
      const uint64_t t0 = globaltimer_ns();
      uint32_t spins = 0;
      while (ld_acquire_u32(hdr + W_GEN) == gen) {
        if ((++spins & 15u) == 0u) {
          if (sv_error(hdr)) { ok = 0; break; }
          if (globaltimer_ns() - t0 > SV_TIMEOUT_NS) {
            if (atomicCAS(hdr + W_ERROR, 0u, 1u) == 0u) atomicExch(hdr + W_INFO, where);
            ok = 0;
            break;
          }
        }
        __nanosleep(32);
      }
      __threadfence();
    }
    if (ok && sv_error(hdr)) ok = 0;
  }
  return __syncthreads_and(ok) != 0;
}

// exp(d) in fp64, after Tang's table-driven method (P. T. P. Tang, "Table-driven
// implementation of the exponential function in IEEE floating-point
// arithmetic", ACM TOMS 15(2), 1989): d = (32 m + j) ln2/32 + r with
// |r| <= ln2/64, so exp(d) = 2^m * 2^(j/32) * exp(r).  exp(r) - 1 is its Taylor
// polynomial to degree 6 (truncation below 4e-18), ln2/32 is a double-double,
// and 2^(j/32) comes correctly rounded from a 32-entry table in shared memory.
// Error about 1 ulp.  Arguments here are l - max <= 0; below -708 (and for
// -inf) it returns 0: such a term is under 2^-1021 of the row's largest, 1.
// Branch-free, so that many calls schedule as straight-line code.
__device__ __forceinline__ double sv_exp(double d, const double* tab) {
  constexpr double INV_L = 0x1.71547652b82fep+5;         // 32 / ln2
  constexpr double L_HI = 0x1.62e42fefa39efp-1 / 32.0;   // ln2 / 32, leading part
  constexpr double L_LO = 0x1.abc9e3b39803fp-56 / 32.0;  // ln2 / 32 - L_HI
  constexpr double SHIFT = 0x1.8p52;                     // rounds to an integer in the low bits
  const double t = fma(d, INV_L, SHIFT);
  const int N = __double2loint(t);
  const double Nd = t - SHIFT;
  double r = fma(-Nd, L_HI, d);
  r = fma(-Nd, L_LO, r);
  double q = fma(r, 1.0 / 720.0, 1.0 / 120.0);
  q = fma(q, r, 1.0 / 24.0);
  q = fma(q, r, 1.0 / 6.0);
  q = fma(q, r, 0.5);
  q = fma(q, r, 1.0);
  q *= r;  // exp(r) - 1
  const double T = tab[N & 31];
  const double e = fma(T, q, T);  // 2^(j/32) exp(r), in [0.98, 2.03)
  // times 2^m, m = floor(N / 32): added to the exponent field (stays normal
  // above -708); below, and for -inf or NaN, the select gives 0 (no branch:
  // the arithmetic above is then meaningless but harmless)
  const double res = __hiloint2double(__double2hiint(e) + ((N >> 5) << 20), __double2loint(e));
  return d > -708.0 ? res : 0.0;
}

__device__ __forceinline__ double warp_incl_scan(double v, int lane) {
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const double y = __shfl_up_sync(FULL, v, o);
    if (lane >= o) v += y;
  }
  return v;
}

// ---- rows: segment statistics, row normalisers, decisions ----------------------

__device__ __forceinline__ void seg_load(const SvParams& p, int64_t task, int R, int lane, float (&v)[LPL]) {
  const int s = (int)(task % p.nseg);
  const int64_t br = task / p.nseg;
  const float* src = row_ptr(p, (int)(br / R), (int)(br % R));
  const int j0 = s * SEG;
#pragma unroll
  for (int k = 0; k < LPL; ++k) {
    const int j = j0 + lane + 32 * k;
    v[k] = j < p.V ? __ldg(src + j) : -INFINITY;
  }
}

// Rows br0 and (if br1 >= 0) br1: M = max over the row's segments, then
// Z = sum z exp(m - M), each lane over its segments in order, the lanes summed
// in a fixed tree.  Up to 32*SBF segments per row stay in registers between
// the two passes, and both rows' loads are in flight together.
constexpr int SBF = 10;

__device__ __forceinline__ void row_mz(const double2 (&v)[SBF], const double* tab, double2& out) {
  double M = -INFINITY, Z = 0.0;
#pragma unroll
  for (int k = 0; k < SBF; ++k) M = fmax(M, v[k].x);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) M = fmax(M, __shfl_xor_sync(FULL, M, o));
#pragma unroll
  for (int k = 0; k < SBF; ++k)
    if (v[k].y > 0.0) Z += v[k].y * sv_exp(v[k].x - M, tab);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) Z += __shfl_xor_sync(FULL, Z, o);
  out = make_double2(M, Z);
}

__device__ double2 row_finalize_loop(const SvParams& p, int64_t br, int lane, const double* tab) {
  const double2* st = p.stat + br * p.nseg;
  double M = -INFINITY, Z = 0.0;
  for (int s = lane; s < p.nseg; s += 32) M = fmax(M, __ldcg(&st[s].x));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) M = fmax(M, __shfl_xor_sync(FULL, M, o));
  for (int s = lane; s < p.nseg; s += 32) {
    const double2 v = __ldcg(st + s);
    if (v.y > 0.0) Z += v.y * sv_exp(v.x - M, tab);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) Z += __shfl_xor_sync(FULL, Z, o);
  return make_double2(M, Z);
}

__device__ void rows_finalize(const SvParams& p, int64_t br0, int64_t br1, int lane, const double* tab,
                              double2& out0, double2& out1) {
  if (p.nseg > 32 * SBF) {
    out0 = row_finalize_loop(p, br0, lane, tab);
    if (br1 >= 0) out1 = row_finalize_loop(p, br1, lane, tab);
    return;
  }
  double2 v0[SBF], v1[SBF];
#pragma unroll
  for (int k = 0; k < SBF; ++k) {
    const int s = lane + 32 * k;
    v0[k] = s < p.nseg ? __ldcg(p.stat + br0 * p.nseg + s) : make_double2(-INFINITY, 0.0);
    v1[k] = br1 >= 0 && s < p.nseg ? __ldcg(p.stat + br1 * p.nseg + s) : make_double2(-INFINITY, 0.0);
  }
  row_mz(v0, tab, out0);
  if (br1 >= 0) row_mz(v1, tab, out1);
}

// The inputs of draft `lane`'s acceptance test in block b.
struct TestIn {
  int d;
  float lp, lq;
  double r;
};

__device__ __forceinline__ TestIn test_load(const SvParams& p, int b, int lane) {
  TestIn in{-1, 0.f, 0.f, 0.0};
  if (lane < p.G) {
    in.d = p.d[(size_t)b * p.G + lane];
    in.r = p.r[(size_t)b * p.G + lane];
    if (in.d >= 0 && in.d < p.V) {
      in.lp = p.lt[((size_t)b * (p.G + 1) + lane) * p.V + in.d];
      in.lq = p.ld[((size_t)b * p.G + lane) * p.V + in.d];
    }
  }
  return in;
}

// The acceptance tests of block b, draft i on lane i (G <= 16): accepted when
// r * q(d) < p(d).  n = the first rejection (G if none).  rows: the block's
// (M, Z) per row, in shared memory.
__device__ void decide(const SvParams& p, int b, int lane, const double* tab, const TestIn& in,
                       const double2* rows) {
  bool acc = true;
  if (lane < p.G) {
    acc = false;
    if (in.d >= 0 && in.d < p.V) {
      const double2 sp = rows[lane], sq = rows[p.G + 1 + lane];
      const double pd = sv_exp((double)in.lp - sp.x, tab) / sp.y;
      const double qd = sv_exp((double)in.lq - sq.x, tab) / sq.y;
      acc = in.r * qd < pd;
    }
  }
  const unsigned rej = __ballot_sync(FULL, !acc);
  const int n = rej ? __ffs(rej) - 1 : p.G;
  if (lane <= p.G) p.tok_out[(size_t)b * (p.G + 1) + lane] = lane < n ? in.d : -1;  // [n]: the draw
  if (lane == 0) {
    Meta m{};
    m.n = n;
    m.mode = n < p.G ? MODE_RESIDUAL : MODE_BONUS;
    m.Mt = rows[n].x;
    m.iZt = 1.0 / rows[n].y;
    if (m.mode == MODE_RESIDUAL) {
      m.Md = rows[p.G + 1 + n].x;
      m.iZd = 1.0 / rows[p.G + 1 + n].y;
    }
    p.meta[b] = m;
    p.n_out[b] = n;
    if (b == 0) stamps(p)[3] = globaltimer_ns();
  }
  __syncwarp();
}

// NT statistics segments per warp and iteration, the loads of all in flight.
constexpr int NT = 3;

__device__ void phase_rows(const SvParams& p, const double* tab) {
  const int lane = threadIdx.x & 31;
  // consecutive tasks on consecutive CTAs: every SM gets an even share
  const int64_t gw = (int64_t)(threadIdx.x >> 5) * gridDim.x + blockIdx.x;
  const int64_t nw = (int64_t)gridDim.x * SV_WARPS;
  const int R = 2 * p.G + 1;
  const int64_t ntask = (int64_t)p.B * R * p.nseg;
  for (int64_t t0 = gw; t0 < ntask; t0 += NT * nw) {
    float v[NT][LPL];
#pragma unroll
    for (int i = 0; i < NT; ++i) {
      if (t0 + i * nw < ntask) seg_load(p, t0 + i * nw, R, lane, v[i]);
      else
#pragma unroll
        for (int k = 0; k < LPL; ++k) v[i][k] = -INFINITY;
    }
    // the NT segments side by side: maxima, then every exp, then the sums
    float m[NT];
#pragma unroll
    for (int i = 0; i < NT; ++i) {
      m[i] = v[i][0];
#pragma unroll
      for (int k = 1; k < LPL; ++k) m[i] = fmaxf(m[i], v[i][k]);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
#pragma unroll
      for (int i = 0; i < NT; ++i) m[i] = fmaxf(m[i], __shfl_xor_sync(FULL, m[i], o));
    double z[NT];
#pragma unroll
    for (int i = 0; i < NT; ++i) {
      z[i] = 0.0;
      if (m[i] != -INFINITY) {
        const double md = (double)m[i];
#pragma unroll
        for (int k = 0; k < LPL; ++k) z[i] += sv_exp((double)v[i][k] - md, tab);
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
#pragma unroll
      for (int i = 0; i < NT; ++i) z[i] += __shfl_xor_sync(FULL, z[i], o);
    if (lane == 0) {
#pragma unroll
      for (int i = 0; i < NT; ++i)
        if (t0 + i * nw < ntask) p.stat[t0 + i * nw] = make_double2((double)m[i], z[i]);
    }
  }
}

// Every block on one CTA: its rows' normalisers (row r on warp (r + 1) % 16,
// so that warp 0 has at most one), then its acceptance tests on warp 0, whose
// loads were issued before the rows' work.
__device__ void phase_decide(const SvParams& p, const double* tab, double2* rows) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int R = 2 * p.G + 1;
  for (int b = blockIdx.x; b < p.B; b += gridDim.x) {
    TestIn in{};
    if (warp == 0) in = test_load(p, b, lane);
    for (int row = (warp + SV_WARPS - 1) % SV_WARPS; row < R; row += 2 * SV_WARPS) {
      const int row1 = row + SV_WARPS < R ? row + SV_WARPS : -1;
      double2 s0, s1;
      rows_finalize(p, (int64_t)b * R + row, row1 >= 0 ? (int64_t)b * R + row1 : -1, lane, tab, s0, s1);
      if (lane == 0) {
        rows[row] = s0;
        if (row1 >= 0) rows[row1] = s1;
      }
    }
    __syncthreads();
    if (warp == 0) decide(p, b, lane, tab, in, rows);
    __syncthreads();
  }
}

// ---- draws: weight segments, then the draw -------------------------------------

__device__ __forceinline__ Meta load_meta(const SvParams& p, int b) {
  const double2* src = reinterpret_cast<const double2*>(p.meta + b);
  const int4 h = __ldcg(reinterpret_cast<const int4*>(src));
  const double2 t = __ldcg(src + 1), q = __ldcg(src + 2);
  Meta m{};
  m.n = h.x;
  m.mode = h.y;
  m.Mt = t.x;
  m.iZt = t.y;
  m.Md = q.x;
  m.iZd = q.y;
  return m;
}

// Weights of entries s*SEGC + LPC*lane + k (k < LPC) of block b's drawn row.
// Residual mode: w = max(0, p - q) and f = exp(l - M) of the target row (the
// fallback's weights).  Bonus mode: w = exp(l - M) of the target row, f = 0.
__device__ __forceinline__ void seg_weights(const SvParams& p, int b, const Meta& m, int s, int lane,
                                            const double* tab, double (&w)[LPC], double (&f)[LPC]) {
  const bool res = m.mode == MODE_RESIDUAL;
  const float* tr = row_ptr(p, b, m.n);
  const float* qr = res ? row_ptr(p, b, p.G + 1 + m.n) : tr;
  const int j0 = s * SEGC + LPC * lane;
  float lt[LPC], lq[LPC];
#pragma unroll
  for (int k = 0; k < LPC; ++k) {
    const int j = j0 + k;
    lt[k] = j < p.V ? __ldg(tr + j) : -INFINITY;
    lq[k] = res && j < p.V ? __ldg(qr + j) : -INFINITY;
  }
#pragma unroll
  for (int k = 0; k < LPC; ++k) {
    const double et = sv_exp((double)lt[k] - m.Mt, tab);
    if (res) {
      const double eq = sv_exp((double)lq[k] - m.Md, tab);
      w[k] = fmax(et * m.iZt - eq * m.iZd, 0.0);
      f[k] = et;
    } else {
      w[k] = et;
      f[k] = 0.0;
    }
  }
}

// The lane holding the crossing: the first lane whose inclusive sum exceeds
// t; if rounding left none, or the lane holds no weight, the nearest lane with
// weight (below first).
__device__ __forceinline__ int crossing_lane(double incl_plus_base, double t, double own) {
  const unsigned over = __ballot_sync(FULL, incl_plus_base > t);
  const unsigned pos = __ballot_sync(FULL, own > 0.0);
  int L = over ? __ffs(over) - 1 : 31;
  if (pos && !((pos >> L) & 1u)) {
    const unsigned below = pos & (L == 31 ? FULL : (2u << L) - 1u);
    L = below ? 31 - __clz(below) : __ffs(pos) - 1;
  }
  return L;  // with no weight anywhere (possible only for non-finite inputs): any lane
}

// Sum of the segment weights W[s_lo, s_hi) in index order; loads in batches
// of SBR, all in flight together.
__device__ __forceinline__ double range_sum(const double* W, int s_lo, int s_hi) {
  double c = 0.0;
  for (int s0 = s_lo; s0 < s_hi; s0 += SBR) {
    double v[SBR];
#pragma unroll
    for (int k = 0; k < SBR; ++k) v[k] = s0 + k < s_hi ? __ldcg(W + s0 + k) : 0.0;
#pragma unroll
    for (int k = 0; k < SBR; ++k) c += v[k];
  }
  return c;
}

// The draw of block b (one warp): lane l owns consecutive segments; the lane
// whose range crosses t = u * S walks it; then the crossing segment's weights
// are recomputed and the crossing lane walks its LPC entries.
__device__ void draw(const SvParams& p, int b, const Meta& m, int lane, const double* tab) {
  const int spl = (p.nsegc + 31) / 32;
  const int s_lo = min(lane * spl, p.nsegc), s_hi = min(s_lo + spl, p.nsegc);
  const double* W = p.segw + (size_t)b * p.nsegc;
  double c = range_sum(W, s_lo, s_hi);
  double incl = warp_incl_scan(c, lane);
  double S = __shfl_sync(FULL, incl, 31);
  const bool fallback = m.mode == MODE_RESIDUAL && !(S > 0.0);  // no residual weight: draw from p
  if (fallback) {
    W = p.segf + (size_t)b * p.nsegc;
    c = range_sum(W, s_lo, s_hi);
    incl = warp_incl_scan(c, lane);
    S = __shfl_sync(FULL, incl, 31);
  }
  const double t = p.u[b] * S;
  const int L = crossing_lane(incl, t, c);
  double before = __shfl_up_sync(FULL, incl, 1);
  if (lane == 0) before = 0.0;
  before = __shfl_sync(FULL, before, L);
  int sstar = -1;
  double base = 0.0;
  if (lane == L) {
    double acc = before, last_acc = before;
    int last = -1;
    for (int s0 = s_lo; s0 < s_hi && sstar < 0; s0 += SBR) {
      double v[SBR];
#pragma unroll
      for (int k = 0; k < SBR; ++k) v[k] = s0 + k < s_hi ? __ldcg(W + s0 + k) : 0.0;
#pragma unroll
      for (int k = 0; k < SBR; ++k) {
        if (sstar < 0 && v[k] > 0.0) {
          if (acc + v[k] > t) {
            sstar = s0 + k;
            base = acc;
          } else {
            last = s0 + k;
            last_acc = acc;
          }
        }
        acc += v[k];
      }
    }
    if (sstar < 0) {
      sstar = last;
      base = last_acc;
    }
  }
  sstar = __shfl_sync(FULL, sstar, L);
  base = __shfl_sync(FULL, base, L);
  if (sstar < 0) sstar = 0;  // no weight at all: only for non-finite inputs; keeps the loads in range
  double w[LPC], f[LPC];
  seg_weights(p, b, m, sstar, lane, tab, w, f);
  double sig = 0.0;
#pragma unroll
  for (int k = 0; k < LPC; ++k) sig += fallback ? f[k] : w[k];
  const double inc2 = warp_incl_scan(sig, lane);
  const int L2 = crossing_lane(base + inc2, t, sig);
  double pre = __shfl_up_sync(FULL, inc2, 1);
  if (lane == 0) pre = 0.0;
  if (lane == L2) {
    double acc = base + pre;
    int j = -1, last = -1;
#pragma unroll
    for (int k = 0; k < LPC; ++k) {
      const double x = fallback ? f[k] : w[k];
      if (j < 0 && x > 0.0) {
        if (acc + x > t) j = k;
        else last = k;
      }
      acc += x;
    }
    if (j < 0) j = last < 0 ? 0 : last;
    p.tok_out[(size_t)b * (p.G + 1) + m.n] = sstar * SEGC + LPC * lane + j;
  }
  __syncwarp();
}

// Weight segment sums of every block's drawn row.
__device__ void phase_weights(const SvParams& p, const double* tab) {
  const int lane = threadIdx.x & 31;
  // consecutive tasks on consecutive CTAs: few tasks spread over every SM
  const int64_t gw = (int64_t)(threadIdx.x >> 5) * gridDim.x + blockIdx.x;
  const int64_t nw = (int64_t)gridDim.x * SV_WARPS;
  const int64_t ntask = (int64_t)p.B * p.nsegc;
  for (int64_t task = gw; task < ntask; task += nw) {
    const int b = (int)(task / p.nsegc), s = (int)(task % p.nsegc);
    const Meta m = load_meta(p, b);
    double w[LPC], f[LPC];
    seg_weights(p, b, m, s, lane, tab, w, f);
    double sw = 0.0, sf = 0.0;
#pragma unroll
    for (int k = 0; k < LPC; ++k) {
      sw += w[k];
      sf += f[k];
    }
    sw = warp_incl_scan(sw, lane);
    sf = warp_incl_scan(sf, lane);
    if (lane == 31) {
      p.segw[task] = sw;
      p.segf[task] = sf;
    }
  }
}

// The draws, one warp per block.  Up to SV_WARPS blocks: every CTA counts
// itself done with its weight sums, and the last one to do so draws every
// block while the others exit.  More blocks: after a grid-wide barrier, on
// every CTA.  True on the CTA(s) that drew.
__device__ bool phase_draw(const SvParams& p, const double* tab) {
  const int lane = threadIdx.x & 31;
  if (p.B > SV_WARPS) {
    if (!sv_grid_sync(p.hdr, 3)) return false;
    if (blockIdx.x == 0 && threadIdx.x == 0) stamps(p)[6] = globaltimer_ns();
    const int64_t gw = (int64_t)(threadIdx.x >> 5) * gridDim.x + blockIdx.x;
    for (int64_t b = gw; b < p.B; b += (int64_t)gridDim.x * SV_WARPS)
      draw(p, (int)b, load_meta(p, (int)b), lane, tab);
    return blockIdx.x == 0;
  }
  __shared__ int last;
  __syncthreads();
  if (threadIdx.x == 0) last = atom_add_acq_rel_u32(p.hdr + W_DONE, 1u) == gridDim.x - 1;
  __syncthreads();
  if (!last) return false;
  if (threadIdx.x == 0) {
    p.hdr[W_DONE] = 0u;  // every CTA has counted itself
    stamps(p)[6] = globaltimer_ns();
  }
  __threadfence();
  for (int b = threadIdx.x >> 5; b < p.B; b += SV_WARPS) draw(p, b, load_meta(p, b), lane, tab);
  return true;
}

__global__ void __launch_bounds__(SV_THREADS, 1) spec_verify_kernel(const SvParams p) {
  __shared__ double tab[32];
  __shared__ double2 rows[2 * SPEC_MAX_GAMMA + 1];
  if (threadIdx.x < 32) tab[threadIdx.x] = p.exp2tab[threadIdx.x];
  __syncthreads();
  uint64_t* st = blockIdx.x == 0 && threadIdx.x == 0 ? stamps(p) : nullptr;
  if (st) st[0] = globaltimer_ns();
  phase_rows(p, tab);
  if (st) st[1] = globaltimer_ns();
  if (!sv_grid_sync(p.hdr, 1)) return;
  if (st) st[2] = globaltimer_ns();
  phase_decide(p, tab, rows);  // stamp 3: block 0 decided
  if (!sv_grid_sync(p.hdr, 2)) return;
  if (st) st[4] = globaltimer_ns();
  phase_weights(p, tab);
  if (st) st[5] = globaltimer_ns();
  if (phase_draw(p, tab)) {  // stamp 6: the drawing CTA starts
    __syncthreads();
    if (threadIdx.x == 0) stamps(p)[7] = globaltimer_ns();
  }
}

struct ExpTable {
  double v[32];
};

__global__ void spec_exp_kernel(const double* x, double* y, int64_t n, const ExpTable t) {
  __shared__ double tab[32];
  if (threadIdx.x < 32) tab[threadIdx.x] = t.v[threadIdx.x];
  __syncthreads();
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x)
    y[i] = sv_exp(x[i], tab);
}

// 2^(j/32), j < 32, rounded to double from long double (64-bit significand):
// correctly rounded.
void exp2_table(double* out) {
  for (int j = 0; j < 32; ++j) out[j] = (double)exp2l((long double)j / 32.0L);
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

// CTAs per launch on this device (cooperative: all co-resident), 0 on error.
int sv_grid(int dev) {
  static int cached[64] = {};
  if (dev >= 0 && dev < 64 && cached[dev] > 0) return cached[dev];
  int per_sm = 0, sms = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, spec_verify_kernel, SV_THREADS, 0) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || per_sm < 1)
    return 0;
  const int g = (per_sm < 2 ? per_sm : 2) * sms;
  if (dev >= 0 && dev < 64) cached[dev] = g;
  return g;
}

}  // namespace

extern "C" {

int64_t spec_verify_workspace_bytes(int32_t B, int32_t G, int32_t V) {
  if (B <= 0 || G < 0 || G > SPEC_MAX_GAMMA || V <= 0 || V > SPEC_MAX_VOCAB) return -1;
  return (int64_t)layout(B, G, V).total;
}

int32_t spec_verify(const float* target_logits, const float* draft_logits, const int32_t* draft_tokens,
                    const double* r_accept, const double* u_sample, int32_t B, int32_t G, int32_t V,
                    int32_t* n_accepted, int32_t* tokens_out, void* workspace, int64_t workspace_bytes,
                    void* stream) {
  if (B < 0) return MOE_ERR_INVALID_ARG;
  if (B == 0) return MOE_OK;
  const int64_t need = spec_verify_workspace_bytes(B, G, V);
  if (need < 0 || !target_logits || !u_sample || !n_accepted || !tokens_out || !workspace ||
      workspace_bytes < need || (G > 0 && (!draft_logits || !draft_tokens || !r_accept)))
    return MOE_ERR_INVALID_ARG;
  if (!aligned(target_logits, 4) || !aligned(draft_logits, 4) || !aligned(draft_tokens, 4) ||
      !aligned(r_accept, 8) || !aligned(u_sample, 8) || !aligned(n_accepted, 4) || !aligned(tokens_out, 4) ||
      !aligned(workspace, 16))
    return MOE_ERR_INVALID_ARG;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return MOE_ERR_DEVICE;
  }
  const int grid = sv_grid(dev);
  if (grid <= 0) {
    cudaGetLastError();
    return MOE_ERR_DEVICE;
  }
  const Layout L = layout(B, G, V);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  SvParams p{};
  p.lt = target_logits; p.ld = draft_logits; p.d = draft_tokens; p.r = r_accept; p.u = u_sample;
  p.B = B; p.G = G; p.V = V; p.nseg = (V + SEG - 1) / SEG; p.nsegc = (V + SEGC - 1) / SEGC;
  p.n_out = n_accepted; p.tok_out = tokens_out;
  p.hdr = reinterpret_cast<uint32_t*>(ws);
  p.stat = reinterpret_cast<double2*>(ws + L.stat);
  p.meta = reinterpret_cast<Meta*>(ws + L.meta);
  p.segw = reinterpret_cast<double*>(ws + L.segw);
  p.segf = reinterpret_cast<double*>(ws + L.segf);
  exp2_table(p.exp2tab);
  void* args[] = {&p};
  return cudaLaunchCooperativeKernel((const void*)spec_verify_kernel, dim3(grid), dim3(SV_THREADS), args, 0,
                                     static_cast<cudaStream_t>(stream)) == cudaSuccess
             ? MOE_OK
             : MOE_ERR_CUDA;
}

int32_t spec_exp(const double* x, double* y, int64_t n, void* stream) {
  if (n < 0 || (n > 0 && (!x || !y || !aligned(x, 8) || !aligned(y, 8)))) return MOE_ERR_INVALID_ARG;
  if (n == 0) return MOE_OK;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return MOE_ERR_DEVICE;
  }
  ExpTable t;
  exp2_table(t.v);
  const int64_t blocks = (n + 255) / 256;
  spec_exp_kernel<<<(unsigned)(blocks < 4096 ? blocks : 4096), 256, 0, static_cast<cudaStream_t>(stream)>>>(x, y, n,
                                                                                                          t);
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

int32_t spec_verify_status(void* workspace, void* stream) {
  if (!workspace || !aligned(workspace, 16)) return MOE_ERR_INVALID_ARG;
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return MOE_ERR_CUDA;
  uint32_t words[8] = {};
  if (cudaMemcpy(words, workspace, sizeof(words), cudaMemcpyDeviceToHost) != cudaSuccess) return MOE_ERR_CUDA;
  if (words[W_ERROR] == 0u) return MOE_OK;
  if (cudaMemset(workspace, 0, sizeof(words)) != cudaSuccess) return MOE_ERR_CUDA;
  return MOE_ERR_TIMEOUT;
}

}  // extern "C"
