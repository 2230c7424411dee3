// Shared definitions between the C-ABI layer and the CUDA kernels of the
// MXFP4 MoE expert feed-forward.
#pragma once
#include <stdint.h>
#include <cuda_runtime.h>
#include <cuda_bf16.h>

namespace moe {

// ---- streaming layout -------------------------------------------------------------
// The weight stream is cut into jobs of 128 weight rows (the M of one
// block-scaled tensor-core MMA) x the whole contraction dimension: a gate/up
// job holds 64 gate rows and the same 64 up rows of one expert, a down job 128
// rows of Wd.  A job is streamed in stages of KS = 128 K elements (four MX
// blocks).  A stage is laid out exactly as the MMA reads it from shared
// memory: E2M1 codes as K-major 8-row x 16-byte core matrices (two MMAs of
// K = 64), then the E8M0 scales in the scale-factor copy layout (row m at byte
// (m % 32) * 16 + (m / 32) * 4 + block).  Row m of a gate/up job is, with
// q = m / 32 and l = m % 32, gate (l < 16) or up (l >= 16) of intermediate row
// 16 q + (l % 16), so that both halves of a SwiGLU meet in one warp.
constexpr int KS = 128;                                  // K elements per stage
constexpr int KB = KS / 32;                              // MX blocks per stage
constexpr int JOB_ROWS = 128;                            // weight rows per job
constexpr int GU_I_ROWS = JOB_ROWS / 2;                  // intermediate rows per gate/up job
constexpr int STAGE_CODE_BYTES = JOB_ROWS * KS / 2;      // 8192
constexpr int STAGE_A_BYTES = STAGE_CODE_BYTES + JOB_ROWS * KB;  // 8704
// Activations enter the MMA as B operands: each column group (a token of a
// gate/up unit, a (token, expert) pair of a down unit) is 8 MMA columns, the
// terms v = sum_k c_k 2^s_k (c_k E2M1, one E8M0 exponent per term and block)
// of an exact E2M1 expansion.  Per stage and group: 8 rows x 64 bytes of codes
// (two K = 64 halves of 2 x 16-byte chunks) and 8 rows x 16 bytes of scales
// (bytes 0..3 = the four blocks, 4..15 zero).
constexpr int NTERM = 8;
constexpr int IMG_CODE_BYTES = NTERM * KS / 2;           // 512
constexpr int IMG_BYTES = IMG_CODE_BYTES + NTERM * 16;   // 640
constexpr int NT_MAX = 4;                                // tokens per gate/up unit (N <= 32)
constexpr int ND_MAX = 4;                                // pairs per down unit
constexpr int SLOT_BYTES = STAGE_A_BYTES + NT_MAX * IMG_BYTES;  // 11264
constexpr int MAX_HSPLIT = 8;                            // router dot products split along H

constexpr int MAX_LAYERS = 16;
constexpr int MAX_EXPERTS = 512;
// The weight stream runs as NPIPE independent pipelines per CTA, each with its
// own job queue, stage ring, tensor-memory accumulators and roles: warp 2p is
// pipeline p's producer, warp 2p + 1 its MMA issuer, warps 4 + 4p .. 7 + 4p its
// epilogue (one warp per 32-lane tensor-memory sub-partition).  A single
// thread issues tcgen05 instructions at a few hundred cycles per stage, so two
// issuers are needed to keep up with HBM.
constexpr int NPIPE = 2;
constexpr int WARPS = 12;
constexpr int THREADS = WARPS * 32;
constexpr int EPI_WARP0 = 4;
constexpr int NSLOT = 9;                                 // stage ring slots per pipeline
constexpr int PRODUCER_BATCH = 8;                        // most stages per bulk-copy round
constexpr int JQ = 32;                                   // job queue entries per pipeline
constexpr int NACC = 2;                                  // accumulator buffers per pipeline
constexpr int ACC_COLS = NT_MAX * NTERM;                 // 32 columns per buffer
constexpr int NSF = 4;                                   // scale-factor buffers per pipeline
constexpr int SF_COLS = 8;                               // A (4 columns) + B (4 columns)
constexpr int TMEM_COLS = 512;                          // the whole tensor memory of the SM
static_assert(NPIPE * (NACC * ACC_COLS + NSF * SF_COLS) <= TMEM_COLS, "tensor memory budget");
// a batch's stages must occupy distinct slots whose previous use is already issued
static_assert(PRODUCER_BATCH <= NSLOT && PRODUCER_BATCH < 32, "producer batch");
constexpr int SMALL_PAIRS = 256;                         // T*K up to this: routing done per CTA
// Big units (grid-wide routing without tiles, at least BIG_MIN_PER_EXPERT
// positions per expert on average): units of up to NT_BIG positions, so that
// an expert hit by 5..8 positions streams its weights once.  The B operand is
// a unit's run of per-position x images (one bulk copy per stage) in which
// positions 4..7 also have their scale bytes at bytes 4..7 of the scale rows
// of positions 0..3: one 32-row scale-factor copy then fills the B scale
// columns 4 (B rows 0..31) and 5 (rows 32..63), and the stage takes the same
// two MMAs (N = 8 nt <= 64) as a unit of NT_MAX.
constexpr int NT_BIG = 8;
constexpr int BIG_MIN_PER_EXPERT = 4;
constexpr int SLOT_BYTES_BIG = STAGE_A_BYTES + NT_BIG * IMG_BYTES;  // 13824
constexpr int NSLOT_BIG = 7;                             // per pipeline
constexpr int ACC_COLS_BIG = NT_BIG * NTERM;             // 64 columns per buffer
static_assert(NPIPE * (NACC * ACC_COLS_BIG + NSF * SF_COLS) <= TMEM_COLS, "tensor memory budget (big units)");
static_assert(NSLOT_BIG <= NSLOT, "big-unit ring barriers");
static_assert(NT_BIG == 2 * NT_MAX, "positions 4..7 pair with positions 0..3");

// ---- large T*K: tile stream --------------------------------------------------------------
// With many tokens per expert (T*K >= LT_MIN_PER_EXPERT * E) a unit ("tile")
// holds up to LT_MAX consecutive positions of one expert's segment and one MMA
// covers all of them.  The tile stream carries LT_NTERM E2M1 terms of each
// activation (the first LT_NTERM of the NTERM-term expansion; the residual is
// below 2^-15 of the block maximum), so B row n = LT_NTERM * tl + k holds term
// k of position tl, and N = lt_cols(nt) (rounded up to 8, at most 192).  Per
// (tile, 128-K stage) the B operand is one image: LT_SF_BLOCKS blocks of 512
// bytes in the scale-factor copy layout (the scale of row n sits in block
// n / 128, row n % 32, bytes 4 ((n / 32) % 4) + block index: lt_sf_offset),
// then the codes in 8-row groups of 512 bytes, row n at
// lt_row_offset(n) + 256 kk + 128 kc for its four 16-byte chunks.  One bulk
// copy of LT_SF_BYTES + lt_cols(nt) * 64 bytes brings a tile's B operand.
constexpr int LT_NTERM = 5;
constexpr int LT_MAX = 38;
constexpr int LT_MIN_PER_EXPERT = 8;                     // T*K / E from which tiles are used
constexpr int LT_SF_BLOCKS = 2;                          // 32-row copies covering N <= 256
constexpr int LT_SF_BYTES = LT_SF_BLOCKS * 512;
constexpr int LT_ACC_COLS = 192;                         // accumulator columns (B rows) at most
constexpr int LT_CODE_BYTES = LT_ACC_COLS / 8 * IMG_CODE_BYTES;  // 12288
constexpr int LT_IMG_BYTES = LT_SF_BYTES + LT_CODE_BYTES;  // 13312
constexpr int LT_SLOT_BYTES = STAGE_A_BYTES + LT_IMG_BYTES;       // 22016
constexpr int LT_NSLOT = 9;                              // one pipeline
constexpr int LT_NACC = 2;
constexpr int LT_SF_COLS = 4 + 4 * LT_SF_BLOCKS;         // 12
static_assert(((LT_NTERM * LT_MAX + 7) & ~7) <= LT_ACC_COLS, "tile columns");
static_assert(LT_NTERM <= NTERM, "tile terms are a prefix of the expansion");
static_assert(LT_NACC * LT_ACC_COLS + NSF * LT_SF_COLS <= TMEM_COLS, "tensor memory budget (tiles)");
static_assert(LT_NSLOT <= NPIPE * NSLOT, "tile ring barriers");
static_assert(LT_ACC_COLS <= 128 * LT_SF_BLOCKS, "tile scale-factor blocks");
// Tile pairs: with few positions per expert (T*K <= LTA_PER_EXPERT * E) a
// tile holds at most LTA_MAX positions (N <= 96) and a job covers LTA_R = 2
// consecutive row blocks that share every B stage: per stage the producer
// brings the two 8704-byte weight stages and one B image, and the MMA issuer
// accumulates into one tensor-memory accumulator per row block.  More of the
// bytes in flight are then weights (the B image is read once per two row
// blocks), which is what the stream is short of at these sizes.  Needs H % 256
// == 0 (down jobs of 2 x 128 rows of H).
constexpr int LTA_MAX = 22;
constexpr int LTA_R = 2;
constexpr int LTA_NACC = 2;                              // accumulator sets (of LTA_R accumulators)
constexpr int LTA_PER_EXPERT = 24;
constexpr int LTA_ACC_COLS = 112;                        // accumulator columns per row block at most
constexpr int LTA_B_BYTES = LT_SF_BYTES + LTA_ACC_COLS / 8 * IMG_CODE_BYTES;  // 8192
constexpr int LTA_SLOT_BYTES = LTA_R * STAGE_A_BYTES + LTA_B_BYTES;           // 25600
constexpr int LTA_NSLOT = 7;
static_assert(((LT_NTERM * LTA_MAX + 7) & ~7) <= LTA_ACC_COLS && LTA_ACC_COLS <= 128, "tile pair columns");
static_assert(LTA_NACC * LTA_R * LTA_ACC_COLS + NSF * (4 * LTA_R + 4) <= TMEM_COLS, "tensor memory budget (tile pairs)");
static_assert(LTA_NSLOT <= NPIPE * NSLOT, "tile pair ring barriers");
// B rows (= accumulator columns) of a tile of nt positions.
__host__ __device__ constexpr int lt_cols(int nt) { return (LT_NTERM * nt + 7) & ~7; }
// Byte offset in a tile image of B row n's first 16-byte chunk.
__host__ __device__ constexpr int lt_row_offset(int n) { return LT_SF_BYTES + (n / 8) * IMG_CODE_BYTES + (n % 8) * 16; }
// Byte offset in a tile image of the scale of B row n, 32-element block kb.
__host__ __device__ constexpr int lt_sf_offset(int n, int kb) {
  return (n / 128) * 512 + (n % 32) * 16 + 4 * ((n / 32) % 4) + kb;
}
// ---- large T*K: bf16 tile stream (kind::f16 on dequantised weights) ----------------------
// The same tile jobs, with x in bf16 as the B operand (one term, exact) and
// the MXFP4 weights dequantised to bf16 in shared memory by converter warps.
// A tile holds up to FT_MAX positions (balanced split of an expert's
// segment), padded to n16 (a multiple of 16) B rows, so one MMA has N = n16.
// K runs in half-stages of 64: per half-stage the producer brings the half of
// the packed weight stage (4096 bytes of codes + the stage's 512 scale bytes)
// into the raw ring and the B block(s) into the B ring; a converter pass
// turns the raw half into a bf16 A block; the MMA issuer runs 4 MMAs of
// K = 16 per B block.  B blocks are K-major without swizzle: for K slice k16
// [n16 / 8 row groups][2 core matrices along K][8 rows][16 bytes], slices
// n16 * 32 bytes apart (ft_b_offset).  The down projection's B is the SwiGLU
// output as two bf16 terms (leading term, then the remainder), two B blocks
// per half-stage accumulated into the same accumulator.
constexpr int FT_MAX = 128;
constexpr int FT_HK = 64;                                 // K per half-stage
constexpr int FT_TERM_BYTES = FT_MAX * FT_HK * 2;         // one B block at most: 16384
constexpr int FT_RAW_BYTES = 4096 + 512;                  // codes of a half-stage + the stage's scales
constexpr int FT_RA = 8;                                  // raw weight ring
constexpr int FT_NB = 6;                                  // B ring
constexpr int FT_AB = 3;                                  // dequantised A blocks
constexpr int FT_A_BYTES = 128 * FT_HK * 2;               // 16384
constexpr int FT_ACC_COLS = FT_MAX;                       // accumulator columns per job
constexpr int FT_CONV_WARPS = 6;                          // warps 2, 3, 8..11
static_assert(FT_RA <= NSLOT && FT_NB + FT_AB <= NSLOT, "bf16 tile barriers");
static_assert(2 * FT_ACC_COLS <= TMEM_COLS, "tensor memory budget (bf16 tiles)");
// Byte offset of element k (< FT_HK) of B row r in a block of `rows` rows.
__host__ __device__ constexpr int ft_b_offset(int r, int k, int rows) {
  return (k / 16) * rows * 32 + (r / 8) * 256 + ((k % 16) / 8) * 128 + (r % 8) * 16 + (k % 8) * 2;
}
// Tiles of the bf16 stream (at most FT_MAX positions each, balanced).
__host__ __device__ inline int max_ftiles(int E, int64_t TK) { return (int)((E < TK ? E : TK) + TK / FT_MAX + 1); }
// Large-T*K stream kind: 1 = E2M1 term tiles on kind::mxf4, 2 = bf16 tiles on kind::f16.
// ---- large T*K: E4M3 term tiles on kind::mxf8f6f4 ---------------------------------------
// The block-scaled kind that takes E2M1 weights and E4M3 activations.  Each
// activation value is an exact-to-fp32-rounding sum of block-scaled E4M3
// terms with fixed exponent steps: s_0 = the least s with amax <= 448 * 2^s
// for the 32-element block, s_k = s_0 - 4 k, each term rounding the remaining
// residual to nearest.  x takes ET_XTERMS = 2 terms (bf16 has 8 significant
// bits: exact except for about 6e-5 of the values, worst residual 3e-7 of the
// block max), the SwiGLU output ET_ATERMS = 3 (residual below 6e-5 of the
// block max).  A tile holds at most ET_MAX positions; its B rows are
// n = terms * tl + k, N rounded up to 16.
// The weights stay packed MXFP4 in HBM and in the ring; two converter warps
// rewrite each stage's codes into the kind's shared-memory form for 4-bit
// data, 16 elements per 16-byte chunk: 8 packed bytes (element 2j in the low
// nibble of byte j), then 8 zero bytes.  8-bit operands are K-major 8-row x
// 16-byte core matrices; an MMA covers K = 32 (one scale block, selected by
// the scale-factor byte index).
// Per-token x images: [H/KS][T][ET_XIMG] bytes: term k's 128 codes at k * 128,
// its 4 block scales at 256 + 4 k.  Tile images (B operand of one stage):
// the scale-factor block (LT_SF_BYTES, lt_sf_offset layout), then the codes of
// K slice i (32 elements) at LT_SF_BYTES + i * N * 32 as [N/8][2][8][16].
constexpr int ET_XTERMS = 2, ET_ATERMS = 3;
constexpr int ET_STEP = 4;                               // exponent step between terms
constexpr int ET_MAX = 64;
constexpr int ET_XIMG = 272;                             // per-token x image bytes per stage
constexpr int ET_ACC_COLS = 192;                         // 3 terms x 64 positions
constexpr int ET_XB_BYTES = LT_SF_BYTES + 4 * 128 * 32;  // gate/up B image at most (N <= 128)
constexpr int ET_AB_BYTES = LT_SF_BYTES + 4 * ET_ACC_COLS * 32;  // down B image at most (N <= 192)
constexpr int ET_U_BYTES = 128 * KS;                     // a stage's codes in the 16-byte-chunk form
constexpr int ET_SLOT_BYTES = STAGE_A_BYTES + ET_AB_BYTES + ET_U_BYTES;  // raw stage, B image, converted A
constexpr int ET_NSLOT = 4;
static_assert(ET_ATERMS * ET_MAX <= ET_ACC_COLS && ET_XTERMS * ET_MAX <= 128, "E4M3 tile columns");
static_assert(2 * ET_ACC_COLS + NSF * (4 + 4 * LT_SF_BLOCKS) <= TMEM_COLS, "tensor memory (E4M3 tiles)");
static_assert(ET_SLOT_BYTES % 128 == 0 && ET_NSLOT <= NPIPE * NSLOT, "E4M3 tile ring");
// B rows of a tile of nt positions with `terms` terms per position (a multiple of 16).
__host__ __device__ constexpr int et_cols(int nt, int terms) { return (terms * nt + 15) & ~15; }
// Byte offset in an E4M3 tile image of element e (0..127 of the stage) of B row n, N rows.
__host__ __device__ constexpr int et_code_offset(int n, int e, int N) {
  return LT_SF_BYTES + (e / 32) * N * 32 + (n / 8) * 256 + ((e % 32) / 16) * 128 + (n % 8) * 16 + (e % 16);
}
__host__ __device__ constexpr int et_img_bytes(int N) { return LT_SF_BYTES + 4 * N * 32; }
// Tiles of the E4M3 stream (at most ET_MAX positions each).
__host__ __device__ inline int max_etiles(int E, int64_t TK) { return (int)((E < TK ? E : TK) + TK / ET_MAX + 1); }

enum : int { LARGE_MXF4 = 1, LARGE_F16 = 2, LARGE_MXF8 = 3 };

// Whether a launch of T*K pairs over E experts streams tiles.
__host__ __device__ inline bool use_tiles(int64_t TK, int E) {
  return TK > SMALL_PAIRS && TK >= (int64_t)LT_MIN_PER_EXPERT * E;
}
// Whether a launch without tiles and with grid-wide routing takes big units.
__host__ __device__ inline bool use_big_units(int64_t TK, int E) {
  return TK > SMALL_PAIRS && !use_tiles(TK, E) && TK >= (int64_t)BIG_MIN_PER_EXPERT * E;
}
// The largest T*K up to TKmax that takes big units (0: none), which sizes
// the per-position x images.
__host__ __device__ inline int64_t max_big_pairs(int64_t TKmax, int E) {
  const int64_t below = (int64_t)LT_MIN_PER_EXPERT * E - 1;  // the largest T*K without tiles
  const int64_t n = TKmax < below ? TKmax : below;
  return use_big_units(n, E) ? n : 0;
}
// Whether its tiles are streamed as tile pairs (two row blocks per job).
__host__ __device__ inline bool use_tile_pairs(int64_t TK, int E, int H) {
  return use_tiles(TK, E) && H % (LTA_R * JOB_ROWS) == 0 && TK <= (int64_t)LTA_PER_EXPERT * E;
}
constexpr int STAMPS_PER_LAYER = 7;  // router, x images, routing wait, top-k / tables, permutation, stream, combine (CTA 0)

// sync word layout (uint32)
enum : int {
  SY_BAR_COUNT = 0, SY_BAR_GEN = 1, SY_JOBS = 2, SY_ERROR = 3, SY_ERRINFO = 4,
  SY_XDONE = 5,  // CTAs whose x term images of this layer are written (small T*K)
  SY_JOBS2 = 6,  // down-job counter of the operator-by-operator launches
  SY_IMGQ = 7,   // x image tasks claimed (small T*K)
  SY_READY = 8,  // ready[unit] from here
};
// device-side error codes (status word)
enum : uint32_t {
  DEV_OK = 0, DEV_TIMEOUT_BARRIER = 1, DEV_TIMEOUT_PIPE = 2, DEV_TIMEOUT_READY = 3,
  DEV_TIMEOUT_QUEUE = 4, DEV_TIMEOUT_IMAGES = 5, DEV_TIMEOUT_PEER = 6,
};

// Upper bounds of the unit tables for T*K pairs over E experts.
__host__ __device__ inline int max_units(int E, int64_t TK) { return (int)((E < TK ? E : TK) + TK / NT_MAX + 1); }
// Tiles of the large path (at most LT_MAX, or LTA_MAX for tile pairs, positions each).
__host__ __device__ inline int max_tiles(int E, int64_t TK) { return (int)((E < TK ? E : TK) + TK / LTA_MAX + 1); }
__host__ __device__ inline int max_dunits(int E, int64_t TK) { return (int)((E < TK ? E : TK) + TK / ND_MAX + 1); }

// Router split of H into HS parts of H / HS elements (a multiple of 8).
inline int router_hsplit(int H) { return H % (8 * MAX_HSPLIT) == 0 ? MAX_HSPLIT : 1; }

struct LayerPtrs {
  const uint8_t* w_gu;  // gate/up stages  [E][I/64][H/KS][STAGE_A_BYTES]
  const uint8_t* w_d;   // down stages     [E][H/128][I/KS][STAGE_A_BYTES]
  const float* router_w;  // [E][H]
  const float* router_b;  // [E] or null
};

// ---- I-sharded layer with the fused one-shot all-reduce --------------------------------
// Every rank owns one region in its own memory: MAX_RANKS epoch words (the
// flag rank r last published into this region, at word r), padded to
// AR_FLAG_BYTES, then two slots of [max_tokens][H] fp32 partial outputs.
// A call of epoch e (1, 2, ... on every rank alike) writes this rank's
// partial into slot e % 2 of its own region, publishes e into word `rank` of
// every rank's region, waits until its own region holds e (or more) from
// every rank, then sums the ranks' slot e % 2 in rank order (peer loads) and
// rounds to bf16.  Two slots suffice: a rank can write slot e % 2 again only
// at epoch e + 2, after every rank has published epoch e + 1, which each does
// only after it finished reading epoch e.
constexpr int MAX_RANKS = 8;
constexpr int AR_FLAG_BYTES = 256;
struct AllReduce {
  int rank, world;            // world == 0: not an I-sharded call
  uint32_t epoch;
  int64_t slot_floats;        // floats per partial slot (max_tokens * H)
  uint8_t* region[MAX_RANKS]; // every rank's region, as this GPU addresses it (own: local)
};
__host__ __device__ inline size_t ar_region_bytes(int64_t max_tokens, int H) {
  return AR_FLAG_BYTES + 2 * (size_t)max_tokens * H * 4;
}

struct EngineParams {
  int H, I, E, K, T, TK, L;  // hidden, inter, experts, top_k, tokens, T*K, layers to run
  int HS;                    // router H split (H/HS a multiple of 8)
  int route_only;            // 1: stop after routing of layer 0, export maps
  float rms_eps;
  uint64_t timeout_ns;
  LayerPtrs layers[MAX_LAYERS];
  const __nv_bfloat16* x_in;  // [T][H]
  __nv_bfloat16* y_out;       // [T][H] (null in route-only mode)
  __nv_bfloat16* layer_io;    // null or [L+1][T][H]
  // workspace (handle-owned)
  double* logits;             // [HS][T][E] partial logits
  uint8_t* xt;                // [H/KS][T][IMG_BYTES] E2M1 term images of x
  __nv_bfloat16* xnext;       // [T][H]
  int32_t* idx;               // [TK]
  float* wts;                 // [TK]
  int32_t* counts;            // [E]
  int32_t* offsets;           // [E+1]
  int32_t* perm;              // [TK]
  int32_t* inv;               // [TK]
  int32_t* tokpos;            // [TK] token of each permuted position
  float* wpos;                // [TK] routing weight of each permuted position
  int32_t* units;             // [Umax][4] gate/up units (expert, pos0, nt <= NT_MAX or NT_BIG, 0)
  int32_t* dunits;            // [Dmax][4] down units (expert, pos0, nt, gate/up unit): the gate/up ranges
  int32_t* n_units;           // [2] gate/up units, down units
  uint8_t* aimg;              // [I/KS][TK][IMG_BYTES] E2M1 term images of the SwiGLU output
  uint8_t* xp;                // big units: [H/KS][TK][IMG_BYTES] x images per permuted position
  uint8_t* xtl;               // large T*K: [tiles][H/KS][LT_IMG_BYTES] x term images per tile
  uint8_t* atl;               // large T*K: [tiles][I/KS][LT_IMG_BYTES] SwiGLU term images per tile
  uint8_t* xtf;               // bf16 tiles: [tiles][H/FT_HK][FT_TERM_BYTES] x per tile
  uint8_t* atf;               // bf16 tiles: [tiles][I/FT_HK][2][FT_TERM_BYTES] SwiGLU output terms per tile
  uint8_t* xe;                // E4M3 tiles: [H/KS][T][ET_XIMG] per-token x term images
  uint8_t* xte;               // E4M3 tiles: [tiles][H/KS][ET_XB_BYTES] x tile images
  uint8_t* ate;               // E4M3 tiles: [tiles][I/KS][ET_AB_BYTES] SwiGLU output tile images
  int large;                  // stream kind above SMALL_PAIRS with tiles: LARGE_MXF4, LARGE_F16 or LARGE_MXF8
  float* ypair;               // [TK][H]
  uint32_t* sync;             // see SY_*
  uint64_t* stamps;           // null or [1 + MAX_LAYERS * STAMPS_PER_LAYER] %globaltimer ns (CTA 0)
  unsigned long long* prof;   // null or [PROF_COUNTERS] summed SM-clock cycles (stream phase)
  AllReduce ar;               // I-sharded layer: the fused all-reduce of the last combine
  int op;                     // operator-by-operator launches: the OP_* this launch runs (0: whole engine)
  int op_layer;               // ... and its layer
};

// The operators of one layer when every step is its own launch (small T*K):
// router partial logits, routing (one CTA), x term images, gate/up jobs, down
// jobs, combine.
enum : int { OP_ROUTER = 1, OP_ROUTE, OP_IMAGES, OP_GATEUP, OP_DOWN, OP_COMBINE, OP_COUNT = OP_COMBINE };

// stream-phase profile counters (SM-clock cycles summed over CTAs; the
// epilogue ones also over its 8 warps)
enum : int {
  PF_PROD_EMPTY = 0, PF_PROD_READY, PF_PROD_TOTAL, PF_STAGES,
  PF_MMA_FULL, PF_MMA_ISSUE, PF_MMA_ACC, PF_EPI_WAIT, PF_EPI_WORK, PF_EPI_TOTAL, PF_JOBS,
  PROF_COUNTERS
};

size_t engine_smem_bytes();
cudaError_t engine_launch(const EngineParams& p, int grid, cudaStream_t s);
// The same layer(s) as OP_COUNT launches per layer; pdl: each launch may start
// while its predecessor drains (programmatic dependent launch).
cudaError_t engine_launch_ops(const EngineParams& p, int grid, bool pdl, cudaStream_t s);
int engine_max_grid(int device, int* err);

cudaError_t quantize_launch(const void* w, int64_t rows, int64_t K, uint8_t* codes,
                            uint8_t* scales, cudaStream_t s);
// Repack canonical codes [E][N][K/2] + scales [E][N][K/32] into streaming stages
// (rows must be a multiple of 64 for gate/up, 128 for down; K a multiple of KS).
cudaError_t repack_gu_launch(const uint8_t* gc, const uint8_t* gs, const uint8_t* uc,
                             const uint8_t* us, int E, int I, int H, uint8_t* out, cudaStream_t s);
cudaError_t repack_d_launch(const uint8_t* dc, const uint8_t* ds, int E, int H, int I,
                            uint8_t* out, cudaStream_t s);

}  // namespace moe
