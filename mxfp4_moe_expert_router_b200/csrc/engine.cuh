// Shared definitions between the C-ABI layer and the CUDA kernels of the
// MXFP4 MoE expert feed-forward.
#pragma once
#include <stdint.h>
#include <cuda_runtime.h>
#include <cuda_bf16.h>

namespace moe {

// ---- streaming layout -------------------------------------------------------------
// One pipeline stage covers KC elements of the contraction dimension for 32
// weight rows: the codes of 4 MX blocks laid out [block][row][16 B], then the
// 32 rows' 4 scale bytes [row][4 B].  A gate/up stage holds 16 gate rows
// (lanes 0-15) then the same 16 up rows (lanes 16-31); a down stage holds 32
// consecutive rows of Wd.  Stages of one (expert, row block) are contiguous
// over the K chunks, so a warp streams one contiguous byte range per job.
constexpr int KC = 128;                          // K elements per stage
constexpr int KB = KC / 32;                      // MX blocks per stage
constexpr int ROWS = 32;                         // weight rows per stage (= lanes)
constexpr int STAGE_CODE_BYTES = ROWS * KC / 2;  // 2048
constexpr int STAGE_W_BYTES = STAGE_CODE_BYTES + ROWS * KB;  // 2176
constexpr int GU_ROWS = 16;                      // gate (and up) rows per gate/up job
constexpr int NT_MAX = 8;                        // tokens per job (a "unit" of a segment)
constexpr int X_SLICE_BYTES = KC * 4;            // one token's fp32 activations per stage

constexpr int MAX_LAYERS = 16;
constexpr int MAX_EXPERTS = 512;
constexpr int THREADS = 256;                     // 8 warps per CTA
constexpr int WARPS = THREADS / 32;
constexpr int RING_BYTES = 24576;                // per-warp stage ring
constexpr int NBAR = 16;                         // stages in flight per warp (max)
constexpr int JQ = 32;                           // per-warp job queue entries
constexpr int SMALL_PAIRS = 256;                 // T*k up to this: routing done per CTA

// sync word layout (uint32)
enum : int {
  SY_BAR_COUNT = 0, SY_BAR_GEN = 1, SY_JOBS = 2, SY_ERROR = 3, SY_ERRINFO = 4,
  SY_READY = 8,  // ready[unit] from here
};
// device-side error codes (status word)
enum : uint32_t {
  DEV_OK = 0, DEV_TIMEOUT_BARRIER = 1, DEV_TIMEOUT_PIPE = 2, DEV_TIMEOUT_READY = 3,
};

struct LayerPtrs {
  const uint8_t* w_gu;  // gate/up stages  [E][I/16][H/KC][STAGE_W_BYTES]
  const uint8_t* w_d;   // down stages     [E][H/32][I/KC][STAGE_W_BYTES]
  const float* router_w;  // [E][H]
  const float* router_b;  // [E] or null
};

struct EngineParams {
  int H, I, E, K, T, TK, L;  // hidden, inter, experts, top_k, tokens, T*K, layers to run
  int route_only;            // 1: stop after routing of layer 0, export maps
  float rms_eps;
  uint64_t timeout_ns;
  LayerPtrs layers[MAX_LAYERS];
  const __nv_bfloat16* x_in;  // [T][H]
  __nv_bfloat16* y_out;       // [T][H] (null in route-only mode)
  __nv_bfloat16* layer_io;    // null or [L+1][T][H]
  // workspace (handle-owned)
  double* logits;             // [T][E]
  float* xf;                  // [T][H]
  __nv_bfloat16* xnext;       // [T][H]
  int32_t* idx;               // [TK]
  float* wts;                 // [TK]
  int32_t* counts;            // [E]
  int32_t* offsets;           // [E+1]
  int32_t* perm;              // [TK]
  int32_t* inv;               // [TK]
  int32_t* tokpos;            // [TK] token of each permuted position
  float* wpos;                // [TK] routing weight of each permuted position
  int32_t* units;             // [Umax][4] (expert, pos0, nt, 0)
  int32_t* n_units;           // [1]
  float* abuf;                // [I/KC][TK][KC]
  float* ypair;               // [TK][H]
  uint32_t* sync;             // see SY_*
  // route-only exports (device, caller-owned)
  int32_t* o_idx; float* o_w; int32_t* o_counts; int32_t* o_offsets; int32_t* o_perm; int32_t* o_inv;
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
