// Shared definitions between the C-ABI layer and the CUDA kernels of the
// MXFP4 MoE expert feed-forward.
#pragma once
#include <stdint.h>
#include <cuda_runtime.h>
#include <cuda_bf16.h>

namespace moe {

// ---- streaming layout -------------------------------------------------------------
// The weight stream is cut into jobs of 64 weight rows x the whole contraction
// dimension: a gate/up job holds 32 gate rows and the same 32 up rows of one
// expert (one 32-row block of the intermediate dimension), a down job 64 rows
// of Wd.  A job is streamed in stages of KC = 128 K elements (four MX blocks);
// the stage layout (see quantize.cu) is the mma.m16n8k16 A-fragment order, so
// a lane turns its 16 bytes per half-stage straight into f16 fragments.
constexpr int KC = 128;                                  // K elements per stage
constexpr int KB = KC / 32;                              // MX blocks per stage
constexpr int STAGE_ROWS = 64;                           // weight rows per stage
constexpr int STAGE_CODE_BYTES = STAGE_ROWS * KC / 2;    // 4096
constexpr int STAGE_W_BYTES = STAGE_CODE_BYTES + STAGE_ROWS * KB;  // 4352
constexpr int NT_MAX = 8;                                // tokens per gate/up unit (one MMA n-tile)
constexpr int ND_MAX = 4;                                // pairs per down unit (hi+lo: one n-tile)
// activations of one K chunk, per (token, expert) pair of the down projection:
// 4 block exponents q (padded to 16 bytes), then the hi and lo f16 halves of
// the SwiGLU output in fragment order.  Consumer lanes read activation
// fragments straight from L2; the ring carries weight stages only.
constexpr int A16_HDR = 16;
constexpr int A16_CHUNK_BYTES = A16_HDR + KC * 2 * 2;    // 528
constexpr int SLOT_BYTES = STAGE_W_BYTES;                // 4352
constexpr int MAX_HSPLIT = 8;                            // router dot products split along H

constexpr int MAX_LAYERS = 16;
constexpr int MAX_EXPERTS = 512;
constexpr int NCW = 8;                                   // consumer (MMA) warps per CTA
constexpr int WARPS = NCW + 1;                           // + one producer warp
constexpr int THREADS = WARPS * 32;
constexpr int NSLOT = 40;                                // stage ring slots per CTA
constexpr int PRODUCER_BATCH = 16;                       // stages per bulk-copy instruction
constexpr int JQ = 32;                                   // job queue entries per CTA
constexpr int PART_LD = 68;                              // partial-sum column stride (floats)
constexpr int PART_COLS = 8;                             // one n-tile
constexpr int SMALL_PAIRS = 256;                         // T*k up to this: routing done per CTA
constexpr int STAMPS_PER_LAYER = 7;  // x converted, logits (CTA 0), prepared, top-k, routed, streamed, combined

// sync word layout (uint32)
enum : int {
  SY_BAR_COUNT = 0, SY_BAR_GEN = 1, SY_JOBS = 2, SY_ERROR = 3, SY_ERRINFO = 4,
  SY_READY = 8,  // ready[unit] from here
};
// device-side error codes (status word)
enum : uint32_t {
  DEV_OK = 0, DEV_TIMEOUT_BARRIER = 1, DEV_TIMEOUT_PIPE = 2, DEV_TIMEOUT_READY = 3,
  DEV_TIMEOUT_QUEUE = 4,
};

// Upper bounds of the unit tables for T*K pairs over E experts.
__host__ __device__ inline int max_units(int E, int64_t TK) { return (int)((E < TK ? E : TK) + TK / NT_MAX + 1); }
__host__ __device__ inline int max_dunits(int E, int64_t TK) { return (int)((E < TK ? E : TK) + TK / ND_MAX + 1); }

// Router split of H: about 1024 elements per part, each part a multiple of KC.
inline int router_hsplit(int H) {
  int hs = H % 1024 == 0 ? H / 1024 : 1;
  return hs > MAX_HSPLIT ? (H % (MAX_HSPLIT * KC) == 0 ? MAX_HSPLIT : 1) : hs;
}

struct LayerPtrs {
  const uint8_t* w_gu;  // gate/up stages  [E][I/32][H/KC][STAGE_W_BYTES]
  const uint8_t* w_d;   // down stages     [E][H/64][I/KC][STAGE_W_BYTES]
  const float* router_w;  // [E][H]
  const float* router_b;  // [E] or null
};

struct EngineParams {
  int H, I, E, K, T, TK, L;  // hidden, inter, experts, top_k, tokens, T*K, layers to run
  int HS;                    // router H split (H/HS a multiple of KC)
  int route_only;            // 1: stop after routing of layer 0, export maps
  float rms_eps;
  uint64_t timeout_ns;
  LayerPtrs layers[MAX_LAYERS];
  const __nv_bfloat16* x_in;  // [T][H]
  __nv_bfloat16* y_out;       // [T][H] (null in route-only mode)
  __nv_bfloat16* layer_io;    // null or [L+1][T][H]
  // workspace (handle-owned)
  double* logits;             // [HS][T][E] partial logits
  uint8_t* xh;                // [T][H] f16, fragment order within 32-blocks
  float* pxf;                 // [T] power-of-two scale of each token's xh
  __nv_bfloat16* xnext;       // [T][H]
  int32_t* idx;               // [TK]
  float* wts;                 // [TK]
  int32_t* counts;            // [E]
  int32_t* offsets;           // [E+1]
  int32_t* perm;              // [TK]
  int32_t* inv;               // [TK]
  int32_t* tokpos;            // [TK] token of each permuted position
  float* wpos;                // [TK] routing weight of each permuted position
  int32_t* units;             // [Umax][4] gate/up units (expert, pos0, nt <= 8, 0)
  int32_t* dunits;            // [Dmax][4] down units (expert, pos0, nt <= 4, gate/up unit)
  int32_t* n_units;           // [2] gate/up units, down units
  uint8_t* a16;               // [I/KC][TK][A16_CHUNK_BYTES]  SwiGLU output, hi/lo f16
  float* ypair;               // [TK][H]
  uint32_t* sync;             // see SY_*
  uint64_t* stamps;           // null or [1 + MAX_LAYERS * STAMPS_PER_LAYER] %globaltimer ns (CTA 0)
  unsigned long long* prof;   // null or [PROF_COUNTERS] summed SM-clock cycles (stream phase)
};

// stream-phase profile counters (cycles summed over CTAs / warps)
enum : int {
  PF_PROD_EMPTY = 0, PF_PROD_READY, PF_PROD_TOTAL, PF_STAGES,
  PF_CONS_FULL, PF_CONS_MMA, PF_CONS_BAR, PF_CONS_EPI, PF_CONS_QUEUE, PF_CONS_TOTAL, PF_JOBS,
  PROF_COUNTERS
};

size_t engine_smem_bytes();
cudaError_t engine_launch(const EngineParams& p, int grid, cudaStream_t s);
int engine_max_grid(int device, int* err);

cudaError_t quantize_launch(const void* w, int64_t rows, int64_t K, uint8_t* codes,
                            uint8_t* scales, cudaStream_t s);
// Repack canonical codes [E][N][K/2] + scales [E][N][K/32] into streaming stages.
cudaError_t repack_gu_launch(const uint8_t* gc, const uint8_t* gs, const uint8_t* uc,
                             const uint8_t* us, int E, int I, int H, uint8_t* out, cudaStream_t s);
cudaError_t repack_d_launch(const uint8_t* dc, const uint8_t* ds, int E, int H, int I,
                            uint8_t* out, cudaStream_t s);

}  // namespace moe
