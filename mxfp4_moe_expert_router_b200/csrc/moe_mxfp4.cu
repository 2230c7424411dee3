// C-ABI of the MXFP4 MoE expert feed-forward: argument validation, the handle
// (repacked weights + workspace), and the launches.  Declarations and the
// contract of every entry point are in include/moe_mxfp4.h.
#include "moe_mxfp4.h"

#include <cstdlib>
#include <cstring>
#include <new>
#include <vector>

#include "engine.cuh"
#include "partial.cuh"

using namespace moe;

struct moe_mxfp4 {
  moe_config_t cfg{};
  int device = 0;
  int grid = 0;
  uint64_t timeout_ns = 2000000000ull;
  int umax = 0;
  uint8_t* w_gu[MAX_LAYERS] = {};
  uint8_t* w_d[MAX_LAYERS] = {};
  float* router_w[MAX_LAYERS] = {};
  float* router_b[MAX_LAYERS] = {};
  double* logits = nullptr;
  uint8_t* xt = nullptr;
  uint8_t* aimg = nullptr;
  uint8_t* xtl = nullptr;  // large T*k only
  uint8_t* xp = nullptr;   // big units only
  uint8_t* atl = nullptr;
  uint8_t *xe = nullptr, *xte = nullptr, *ate = nullptr;  // large T*k only (E4M3 tiles)
  uint8_t* xtf = nullptr;  // large T*k only (bf16 tiles)
  uint8_t* atf = nullptr;
  int large = LARGE_MXF4;  // stream kind for large T*k
  __nv_bfloat16* xnext = nullptr;
  int32_t *idx = nullptr, *counts = nullptr, *offsets = nullptr, *perm = nullptr, *inv = nullptr,
          *tokpos = nullptr, *units = nullptr, *dunits = nullptr, *n_units = nullptr;
  float *wts = nullptr, *wpos = nullptr, *ypair = nullptr;
  uint32_t* sync = nullptr;
  uint64_t* stamps = nullptr;
  unsigned long long* prof = nullptr;
  bool profiling = false;
  __nv_bfloat16 *x_stage = nullptr, *y_stage = nullptr;
  // moe_forward_host_async: two staging slots, copy streams and their events
  __nv_bfloat16 *x_stage2[2] = {}, *y_stage2[2] = {};
  cudaStream_t h2d = nullptr, d2h = nullptr;
  cudaEvent_t ev_in[2] = {}, ev_k[2] = {}, ev_out[2] = {};
  uint64_t host_seq = 0;
  // I-sharded layer with the fused all-reduce: this handle's region (own
  // allocation, so that it can be exported by CUDA IPC), every rank's region
  // as this GPU addresses it, and the epoch of the last call
  uint8_t* ar_region = nullptr;
  size_t ar_bytes = 0;
  int ar_rank = -1, ar_world = 0;
  uint32_t ar_epoch = 0;
  uint8_t* ar_regions[MAX_RANKS] = {};
  std::vector<void*> allocs;
};

namespace {

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

template <class T>
bool dalloc(moe_mxfp4* h, T** out, size_t bytes) {
  void* p = nullptr;
  if (cudaMalloc(&p, bytes < 16 ? 16 : bytes) != cudaSuccess) { *out = nullptr; return false; }
  h->allocs.push_back(p);
  *out = static_cast<T*>(p);
  return true;
}

void free_all(moe_mxfp4* h) {
  for (int i = 0; i < 2; ++i) {
    if (h->ev_in[i]) cudaEventDestroy(h->ev_in[i]);
    if (h->ev_k[i]) cudaEventDestroy(h->ev_k[i]);
    if (h->ev_out[i]) cudaEventDestroy(h->ev_out[i]);
    h->ev_in[i] = h->ev_k[i] = h->ev_out[i] = nullptr;
  }
  if (h->h2d) cudaStreamDestroy(h->h2d);
  if (h->d2h) cudaStreamDestroy(h->d2h);
  h->h2d = h->d2h = nullptr;
  for (void* p : h->allocs) cudaFree(p);
  h->allocs.clear();
}

// Copy streams, events and the second staging slot of moe_forward_host_async,
// created on first use.
bool host_async_ready(moe_mxfp4* h) {
  if (h->h2d) return true;
  const size_t bytes = (size_t)h->cfg.max_tokens * h->cfg.hidden * 2;
  h->x_stage2[0] = h->x_stage;
  h->y_stage2[0] = h->y_stage;
  if (!dalloc(h, &h->x_stage2[1], bytes) || !dalloc(h, &h->y_stage2[1], bytes)) return false;
  for (int i = 0; i < 2; ++i)
    if (cudaEventCreateWithFlags(&h->ev_in[i], cudaEventDisableTiming) != cudaSuccess ||
        cudaEventCreateWithFlags(&h->ev_k[i], cudaEventDisableTiming) != cudaSuccess ||
        cudaEventCreateWithFlags(&h->ev_out[i], cudaEventDisableTiming) != cudaSuccess)
      return false;
  return cudaStreamCreateWithFlags(&h->h2d, cudaStreamNonBlocking) == cudaSuccess &&
         cudaStreamCreateWithFlags(&h->d2h, cudaStreamNonBlocking) == cudaSuccess;
}

size_t stage_bytes_gu(const moe_config_t& c) {
  return (size_t)c.num_experts * (c.inter / GU_I_ROWS) * (c.hidden / KS) * STAGE_A_BYTES;
}
size_t stage_bytes_d(const moe_config_t& c) {
  return (size_t)c.num_experts * (c.hidden / JOB_ROWS) * (c.inter / KS) * STAGE_A_BYTES;
}

int32_t validate_cfg(const moe_config_t* c) {
  if (!c) return MOE_ERR_INVALID_ARG;
  if (c->hidden <= 0 || c->inter <= 0 || c->num_experts <= 0 || c->top_k <= 0 ||
      c->max_tokens <= 0 || c->num_layers <= 0 || c->top_k > c->num_experts ||
      !(c->rms_eps >= 0.f))
    return MOE_ERR_INVALID_ARG;
  if (c->hidden % KS || c->inter % KS || c->hidden > 8192 || c->num_experts > MAX_EXPERTS ||
      c->top_k > 32 || c->num_layers > MAX_LAYERS)
    return MOE_ERR_UNSUPPORTED_SHAPE;
  if ((int64_t)c->max_tokens * c->top_k > (int64_t)1 << 28) return MOE_ERR_UNSUPPORTED_SHAPE;
  return MOE_OK;
}

// x_stage / y_stage double as slot 0 of moe_forward_host_async.  Before another
// call writes them, `s` waits for that slot's last copy in, layers and copy out
// (events that were never recorded are complete).
cudaError_t wait_async_slot0(const moe_mxfp4* h, cudaStream_t s) {
  if (!h->h2d) return cudaSuccess;
  cudaError_t e = cudaStreamWaitEvent(s, h->ev_in[0], 0);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(s, h->ev_k[0], 0);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(s, h->ev_out[0], 0);
  return e;
}

EngineParams base_params(const moe_mxfp4* h, int T) {
  EngineParams p{};
  p.H = h->cfg.hidden; p.I = h->cfg.inter; p.E = h->cfg.num_experts; p.K = h->cfg.top_k;
  p.T = T; p.TK = T * h->cfg.top_k; p.L = h->cfg.num_layers;
  p.rms_eps = h->cfg.rms_eps;
  p.HS = router_hsplit(h->cfg.hidden);
  p.timeout_ns = h->timeout_ns;
  for (int l = 0; l < h->cfg.num_layers; ++l)
    p.layers[l] = LayerPtrs{h->w_gu[l], h->w_d[l], h->router_w[l], h->router_b[l]};
  p.logits = h->logits; p.xt = h->xt; p.xnext = h->xnext;
  p.idx = h->idx; p.wts = h->wts; p.counts = h->counts; p.offsets = h->offsets;
  p.perm = h->perm; p.inv = h->inv; p.tokpos = h->tokpos; p.wpos = h->wpos;
  p.units = h->units; p.dunits = h->dunits; p.n_units = h->n_units; p.aimg = h->aimg;
  p.xtl = h->xtl; p.atl = h->atl; p.xp = h->xp;
  p.xtf = h->xtf; p.atf = h->atf; p.large = h->large;
  p.xe = h->xe; p.xte = h->xte; p.ate = h->ate;
  p.ypair = h->ypair;
  p.sync = h->sync;
  p.stamps = h->stamps;
  p.prof = h->profiling ? h->prof : nullptr;
  return p;
}

}  // namespace

extern "C" {

const char* moe_status_str(int32_t s) {
  switch (s) {
    case MOE_OK: return "ok";
    case MOE_ERR_INVALID_ARG: return "invalid argument";
    case MOE_ERR_UNSUPPORTED_SHAPE: return "unsupported shape";
    case MOE_ERR_OOM: return "device out of memory";
    case MOE_ERR_CUDA: return "CUDA error";
    case MOE_ERR_TIMEOUT: return "device-side wait timed out";
    case MOE_ERR_DEVICE: return "no usable device";
    default: return "unknown status";
  }
}

int32_t mxfp4_quantize(const void* w_bf16, int64_t rows, int64_t K, uint8_t* codes,
                       uint8_t* scales, void* stream) {
  if (rows < 0 || K <= 0 || K % 32) return MOE_ERR_INVALID_ARG;
  if (rows == 0) return MOE_OK;
  if (!w_bf16 || !codes || !scales || !aligned16(w_bf16) || !aligned16(codes))
    return MOE_ERR_INVALID_ARG;
  return quantize_launch(w_bf16, rows, K, codes, scales, static_cast<cudaStream_t>(stream)) ==
                 cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

int32_t moe_mxfp4_create(const moe_config_t* cfg, const uint8_t* const* gate_codes,
                         const uint8_t* const* gate_scales, const uint8_t* const* up_codes,
                         const uint8_t* const* up_scales, const uint8_t* const* down_codes,
                         const uint8_t* const* down_scales, const float* const* router_w,
                         const float* const* router_bias, void* stream, moe_mxfp4_t** out) {
  if (!out) return MOE_ERR_INVALID_ARG;
  *out = nullptr;
  int32_t st = validate_cfg(cfg);
  if (st != MOE_OK) return st;
  if (!gate_codes || !gate_scales || !up_codes || !up_scales || !down_codes || !down_scales ||
      !router_w)
    return MOE_ERR_INVALID_ARG;
  const int L = cfg->num_layers;
  for (int l = 0; l < L; ++l) {
    if (!gate_codes[l] || !gate_scales[l] || !up_codes[l] || !up_scales[l] || !down_codes[l] ||
        !down_scales[l] || !router_w[l])
      return MOE_ERR_INVALID_ARG;
    if (!aligned16(gate_codes[l]) || !aligned16(up_codes[l]) || !aligned16(down_codes[l]) ||
        !aligned16(router_w[l]))
      return MOE_ERR_INVALID_ARG;
  }
  int dev = 0, ndev = 0, major = 0, minor = 0;
  if (cudaGetDeviceCount(&ndev) != cudaSuccess || ndev == 0) { cudaGetLastError(); return MOE_ERR_DEVICE; }
  if (cudaGetDevice(&dev) != cudaSuccess) return MOE_ERR_DEVICE;
  cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
  cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
  if (major != 10 || minor != 0) return MOE_ERR_DEVICE;  // built for sm_100a only

  moe_mxfp4* h = new (std::nothrow) moe_mxfp4();
  if (!h) return MOE_ERR_OOM;
  h->cfg = *cfg;
  h->device = dev;
  if (const char* env = std::getenv("MOE_TIMEOUT_NS")) {
    const unsigned long long v = std::strtoull(env, nullptr, 10);
    if (v > 0) h->timeout_ns = v;
  }
  int gerr = 0;
  const int maxg = engine_max_grid(dev, &gerr);
  int sms = 0;
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (gerr || maxg < 1 || sms < 1) { delete h; return MOE_ERR_DEVICE; }
  h->grid = maxg < sms ? maxg : sms;

  const int H = cfg->hidden, I = cfg->inter, E = cfg->num_experts, K = cfg->top_k;
  const int64_t Tm = cfg->max_tokens, TKm = Tm * K;
  h->umax = max_units(E, TKm);
  const int dmax = max_dunits(E, TKm);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  bool ok = true;
  for (int l = 0; l < L && ok; ++l) {
    ok = dalloc(h, &h->w_gu[l], stage_bytes_gu(*cfg)) && dalloc(h, &h->w_d[l], stage_bytes_d(*cfg)) &&
         dalloc(h, &h->router_w[l], (size_t)E * H * 4);
    if (ok && router_bias && router_bias[l]) ok = dalloc(h, &h->router_b[l], (size_t)E * 4);
  }
  const int HS = router_hsplit(H);
  ok = ok && dalloc(h, &h->logits, (size_t)HS * Tm * E * 8) && dalloc(h, &h->xt, (size_t)(H / KS) * Tm * IMG_BYTES) &&
       dalloc(h, &h->xnext, (size_t)Tm * H * 2) && dalloc(h, &h->idx, (size_t)TKm * 4) &&
       dalloc(h, &h->wts, (size_t)TKm * 4) && dalloc(h, &h->counts, (size_t)E * 4) &&
       dalloc(h, &h->offsets, (size_t)(E + 1) * 4) && dalloc(h, &h->perm, (size_t)TKm * 4) &&
       dalloc(h, &h->inv, (size_t)TKm * 4) && dalloc(h, &h->tokpos, (size_t)TKm * 4) &&
       dalloc(h, &h->wpos, (size_t)TKm * 4) && dalloc(h, &h->units, (size_t)h->umax * 16) &&
       dalloc(h, &h->dunits, (size_t)dmax * 16) &&
       dalloc(h, &h->n_units, 16) &&
       dalloc(h, &h->aimg, (size_t)(I / KS) * TKm * IMG_BYTES) &&
       dalloc(h, &h->ypair, (size_t)TKm * H * 4) &&
       dalloc(h, &h->sync, (size_t)(SY_READY + h->umax) * 4) &&
       dalloc(h, &h->stamps, (size_t)(1 + MAX_LAYERS * STAMPS_PER_LAYER) * 8) &&
       dalloc(h, &h->prof, (size_t)PROF_COUNTERS * 8) &&
       dalloc(h, &h->x_stage, (size_t)Tm * H * 2) && dalloc(h, &h->y_stage, (size_t)Tm * H * 2);
  if (ok && max_big_pairs(TKm, E) > 0)  // per-position x images of the big units
    ok = dalloc(h, &h->xp, (size_t)(H / KS) * max_big_pairs(TKm, E) * IMG_BYTES);
  if (ok && use_tiles(TKm, E)) {  // tile images of the large-T*k stream
    const size_t tiles = (size_t)max_tiles(E, TKm);
    ok = dalloc(h, &h->xtl, tiles * (H / KS) * LT_IMG_BYTES) && dalloc(h, &h->atl, tiles * (I / KS) * LT_IMG_BYTES);
    const size_t ftiles = (size_t)max_ftiles(E, TKm);
    ok = ok && dalloc(h, &h->xtf, ftiles * (H / FT_HK) * FT_TERM_BYTES) &&
         dalloc(h, &h->atf, ftiles * (I / FT_HK) * 2 * FT_TERM_BYTES);
    const size_t etiles = (size_t)max_etiles(E, TKm);
    ok = ok && dalloc(h, &h->xe, (size_t)(H / KS) * Tm * ET_XIMG) &&
         dalloc(h, &h->xte, etiles * (H / KS) * ET_XB_BYTES) && dalloc(h, &h->ate, etiles * (I / KS) * ET_AB_BYTES);
  }
  if (!ok) { free_all(h); delete h; cudaGetLastError(); return MOE_ERR_OOM; }

  // term images: the scale rows' padding bytes 4..15 are read by the
  // scale-factor copies and must stay zero; the kernels never write them
  cudaError_t e = cudaMemsetAsync(h->sync, 0, (size_t)(SY_READY + h->umax) * 4, s);
  if (e == cudaSuccess) e = cudaMemsetAsync(h->xt, 0, (size_t)(H / KS) * Tm * IMG_BYTES, s);
  if (e == cudaSuccess) e = cudaMemsetAsync(h->aimg, 0, (size_t)(I / KS) * TKm * IMG_BYTES, s);
  for (int l = 0; l < L && e == cudaSuccess; ++l) {
    e = repack_gu_launch(gate_codes[l], gate_scales[l], up_codes[l], up_scales[l], E, I, H,
                         h->w_gu[l], s);
    if (e == cudaSuccess) e = repack_d_launch(down_codes[l], down_scales[l], E, H, I, h->w_d[l], s);
    if (e == cudaSuccess)
      e = cudaMemcpyAsync(h->router_w[l], router_w[l], (size_t)E * H * 4, cudaMemcpyDeviceToDevice, s);
    if (e == cudaSuccess && h->router_b[l])
      e = cudaMemcpyAsync(h->router_b[l], router_bias[l], (size_t)E * 4, cudaMemcpyDeviceToDevice, s);
  }
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) { free_all(h); delete h; cudaGetLastError(); return MOE_ERR_CUDA; }
  *out = h;
  return MOE_OK;
}

int32_t moe_route(moe_mxfp4_t* h, int32_t layer, const void* x_bf16, int32_t T,
                  int32_t* topk_idx, float* topk_w, int32_t* counts, int32_t* offsets,
                  int32_t* perm, int32_t* inv_perm, void* stream) {
  if (!h || layer < 0 || layer >= h->cfg.num_layers || T < 0 || T > h->cfg.max_tokens)
    return MOE_ERR_INVALID_ARG;
  if (T == 0) return MOE_OK;
  if (!x_bf16 || !topk_idx || !topk_w || !counts || !offsets || !perm || !inv_perm ||
      !aligned16(x_bf16))
    return MOE_ERR_INVALID_ARG;
  EngineParams p = base_params(h, T);
  p.L = 1;
  p.layers[0] = p.layers[layer];
  p.route_only = 1;
  p.x_in = static_cast<const __nv_bfloat16*>(x_bf16);
  p.idx = topk_idx; p.wts = topk_w; p.counts = counts; p.offsets = offsets; p.perm = perm;
  p.inv = inv_perm;
  return engine_launch(p, h->grid, static_cast<cudaStream_t>(stream)) == cudaSuccess ? MOE_OK
                                                                                     : MOE_ERR_CUDA;
}

int32_t moe_forward(moe_mxfp4_t* h, const void* x_bf16, int32_t T, void* y_bf16,
                    void* layer_io_bf16, void* stream) {
  if (!h || T < 0 || T > h->cfg.max_tokens) return MOE_ERR_INVALID_ARG;
  if (T == 0) return MOE_OK;
  if (!x_bf16 || !y_bf16 || !aligned16(x_bf16) || !aligned16(y_bf16) ||
      (layer_io_bf16 && !aligned16(layer_io_bf16)))
    return MOE_ERR_INVALID_ARG;
  const size_t bytes = (size_t)T * h->cfg.hidden * 2;
  const char* xa = static_cast<const char*>(x_bf16);
  const char* ya = static_cast<const char*>(y_bf16);
  if (xa < ya + bytes && ya < xa + bytes) return MOE_ERR_INVALID_ARG;
  EngineParams p = base_params(h, T);
  p.x_in = static_cast<const __nv_bfloat16*>(x_bf16);
  p.y_out = static_cast<__nv_bfloat16*>(y_bf16);
  p.layer_io = static_cast<__nv_bfloat16*>(layer_io_bf16);
  return engine_launch(p, h->grid, static_cast<cudaStream_t>(stream)) == cudaSuccess ? MOE_OK
                                                                                     : MOE_ERR_CUDA;
}

int32_t moe_forward_ops(moe_mxfp4_t* h, const void* x_bf16, int32_t T, void* y_bf16,
                        void* layer_io_bf16, int32_t flags, void* stream) {
  if (!h || T < 0 || T > h->cfg.max_tokens || (flags & ~MOE_OPS_PDL)) return MOE_ERR_INVALID_ARG;
  if (T == 0) return MOE_OK;
  if (!x_bf16 || !y_bf16 || !aligned16(x_bf16) || !aligned16(y_bf16) ||
      (layer_io_bf16 && !aligned16(layer_io_bf16)))
    return MOE_ERR_INVALID_ARG;
  if ((int64_t)T * h->cfg.top_k > SMALL_PAIRS) return MOE_ERR_UNSUPPORTED_SHAPE;
  const size_t bytes = (size_t)T * h->cfg.hidden * 2;
  const char* xa = static_cast<const char*>(x_bf16);
  const char* ya = static_cast<const char*>(y_bf16);
  if (xa < ya + bytes && ya < xa + bytes) return MOE_ERR_INVALID_ARG;
  EngineParams p = base_params(h, T);
  p.stamps = nullptr;
  p.x_in = static_cast<const __nv_bfloat16*>(x_bf16);
  p.y_out = static_cast<__nv_bfloat16*>(y_bf16);
  p.layer_io = static_cast<__nv_bfloat16*>(layer_io_bf16);
  return engine_launch_ops(p, h->grid, (flags & MOE_OPS_PDL) != 0, static_cast<cudaStream_t>(stream)) == cudaSuccess
             ? MOE_OK
             : MOE_ERR_CUDA;
}

int32_t moe_forward_partial(moe_mxfp4_t* h, const void* x_bf16, int32_t T, float* y_f32, void* stream) {
  if (!h || T < 0 || T > h->cfg.max_tokens) return MOE_ERR_INVALID_ARG;
  if (T == 0) return MOE_OK;
  if (!x_bf16 || !y_f32 || !aligned16(x_bf16) || !aligned16(y_f32)) return MOE_ERR_INVALID_ARG;
  if (h->cfg.num_layers != 1) return MOE_ERR_UNSUPPORTED_SHAPE;
  const int32_t st = moe_forward(h, x_bf16, T, h->y_stage, nullptr, stream);
  if (st != MOE_OK) return st;
  return combine_f32_launch(h->ypair, h->inv, T, h->cfg.top_k, h->cfg.hidden, y_f32,
                            static_cast<cudaStream_t>(stream)) == cudaSuccess
             ? MOE_OK
             : MOE_ERR_CUDA;
}

int32_t moe_ishard_region(moe_mxfp4_t* h, void** base_out, uint64_t* bytes_out) {
  if (!h || !base_out || !bytes_out) return MOE_ERR_INVALID_ARG;
  if (h->cfg.num_layers != 1) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (!h->ar_region) {
    const size_t bytes = ar_region_bytes(h->cfg.max_tokens, h->cfg.hidden);
    void* p = nullptr;
    if (cudaMalloc(&p, bytes) != cudaSuccess) { cudaGetLastError(); return MOE_ERR_OOM; }
    if (cudaMemset(p, 0, bytes) != cudaSuccess || cudaDeviceSynchronize() != cudaSuccess) {
      cudaFree(p);
      cudaGetLastError();
      return MOE_ERR_CUDA;
    }
    h->allocs.push_back(p);
    h->ar_region = static_cast<uint8_t*>(p);
    h->ar_bytes = bytes;
  }
  *base_out = h->ar_region;
  *bytes_out = h->ar_bytes;
  return MOE_OK;
}

int32_t moe_ishard_ipc_handle(moe_mxfp4_t* h, void* handle_out) {
  if (!h || !handle_out) return MOE_ERR_INVALID_ARG;
  void* base = nullptr;
  uint64_t bytes = 0;
  const int32_t st = moe_ishard_region(h, &base, &bytes);
  if (st != MOE_OK) return st;
  cudaIpcMemHandle_t ipc;
  static_assert(sizeof(ipc) == MOE_IPC_HANDLE_BYTES, "IPC handle size");
  if (cudaIpcGetMemHandle(&ipc, base) != cudaSuccess) { cudaGetLastError(); return MOE_ERR_CUDA; }
  std::memcpy(handle_out, &ipc, sizeof(ipc));
  return MOE_OK;
}

int32_t moe_ishard_ipc_open(const void* handle, void** base_out) {
  if (!handle || !base_out) return MOE_ERR_INVALID_ARG;
  cudaIpcMemHandle_t ipc;
  std::memcpy(&ipc, handle, sizeof(ipc));
  void* p = nullptr;
  if (cudaIpcOpenMemHandle(&p, ipc, cudaIpcMemLazyEnablePeerAccess) != cudaSuccess) {
    cudaGetLastError();
    *base_out = nullptr;
    return MOE_ERR_CUDA;
  }
  *base_out = p;
  return MOE_OK;
}

int32_t moe_ishard_ipc_close(void* base) {
  if (!base) return MOE_ERR_INVALID_ARG;
  if (cudaIpcCloseMemHandle(base) != cudaSuccess) { cudaGetLastError(); return MOE_ERR_CUDA; }
  return MOE_OK;
}

int32_t moe_ishard_attach(moe_mxfp4_t* h, int32_t rank, int32_t world, void* const* regions) {
  if (!h || !regions || world < 1 || world > MAX_RANKS || rank < 0 || rank >= world) return MOE_ERR_INVALID_ARG;
  if (h->cfg.num_layers != 1) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (!h->ar_region || regions[rank] != h->ar_region) return MOE_ERR_INVALID_ARG;
  for (int r = 0; r < world; ++r)
    if (!regions[r] || !aligned16(regions[r])) return MOE_ERR_INVALID_ARG;
  // epochs restart at 1: clear the epoch words the peers publish into
  if (cudaMemset(h->ar_region, 0, AR_FLAG_BYTES) != cudaSuccess || cudaDeviceSynchronize() != cudaSuccess) {
    cudaGetLastError();
    return MOE_ERR_CUDA;
  }
  for (int r = 0; r < MAX_RANKS; ++r) h->ar_regions[r] = r < world ? static_cast<uint8_t*>(regions[r]) : nullptr;
  h->ar_rank = rank;
  h->ar_world = world;
  h->ar_epoch = 0;
  return MOE_OK;
}

int32_t moe_forward_ishard(moe_mxfp4_t* h, const void* x_bf16, int32_t T, void* y_bf16, void* stream) {
  if (!h || T < 0 || T > h->cfg.max_tokens) return MOE_ERR_INVALID_ARG;
  if (h->ar_world < 1) return MOE_ERR_INVALID_ARG;  // not attached
  if (T == 0) return MOE_OK;
  if (!x_bf16 || !y_bf16 || !aligned16(x_bf16) || !aligned16(y_bf16)) return MOE_ERR_INVALID_ARG;
  const size_t bytes = (size_t)T * h->cfg.hidden * 2;
  const char* xa = static_cast<const char*>(x_bf16);
  const char* ya = static_cast<const char*>(y_bf16);
  if (xa < ya + bytes && ya < xa + bytes) return MOE_ERR_INVALID_ARG;
  EngineParams p = base_params(h, T);
  p.x_in = static_cast<const __nv_bfloat16*>(x_bf16);
  p.y_out = static_cast<__nv_bfloat16*>(y_bf16);
  p.ar.rank = h->ar_rank;
  p.ar.world = h->ar_world;
  p.ar.epoch = h->ar_epoch + 1;
  p.ar.slot_floats = (int64_t)h->cfg.max_tokens * h->cfg.hidden;
  for (int r = 0; r < MAX_RANKS; ++r) p.ar.region[r] = h->ar_regions[r];
  if (engine_launch(p, h->grid, static_cast<cudaStream_t>(stream)) != cudaSuccess) return MOE_ERR_CUDA;
  h->ar_epoch = p.ar.epoch;
  return MOE_OK;
}

int32_t moe_round_bf16(const float* in_f32, void* out_bf16, int64_t n, void* stream) {
  if (n < 0 || (n > 0 && (!in_f32 || !out_bf16 || (reinterpret_cast<uintptr_t>(in_f32) & 3u) ||
                          (reinterpret_cast<uintptr_t>(out_bf16) & 1u))))
    return MOE_ERR_INVALID_ARG;
  if (n == 0) return MOE_OK;
  return round_bf16_launch(in_f32, static_cast<__nv_bfloat16*>(out_bf16), n, static_cast<cudaStream_t>(stream)) ==
                 cudaSuccess
             ? MOE_OK
             : MOE_ERR_CUDA;
}

int32_t moe_set_large_kind(moe_mxfp4_t* h, int32_t kind) {
  if (!h || (kind != LARGE_MXF4 && kind != LARGE_F16 && kind != LARGE_MXF8)) return MOE_ERR_INVALID_ARG;
  h->large = kind;
  return MOE_OK;
}

int32_t moe_status(moe_mxfp4_t* h, void* stream) {
  if (!h) return MOE_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(s) != cudaSuccess) return MOE_ERR_CUDA;
  if (h->h2d && (cudaStreamSynchronize(h->h2d) != cudaSuccess || cudaStreamSynchronize(h->d2h) != cudaSuccess))
    return MOE_ERR_CUDA;
  uint32_t words[SY_READY] = {};
  if (cudaMemcpy(words, h->sync, sizeof(words), cudaMemcpyDeviceToHost) != cudaSuccess)
    return MOE_ERR_CUDA;
  if (words[SY_ERROR] == DEV_OK) return MOE_OK;
  if (cudaMemset(h->sync, 0, sizeof(words)) != cudaSuccess) return MOE_ERR_CUDA;
  return MOE_ERR_TIMEOUT;
}

int32_t moe_forward_host(moe_mxfp4_t* h, const void* x_host, int32_t T, void* y_host,
                         void* stream) {
  if (!h || T < 0 || T > h->cfg.max_tokens) return MOE_ERR_INVALID_ARG;
  if (T == 0) return MOE_OK;
  if (!x_host || !y_host) return MOE_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const size_t bytes = (size_t)T * h->cfg.hidden * 2;
  if (wait_async_slot0(h, s) != cudaSuccess ||
      cudaMemcpyAsync(h->x_stage, x_host, bytes, cudaMemcpyHostToDevice, s) != cudaSuccess)
    return MOE_ERR_CUDA;
  int32_t st = moe_forward(h, h->x_stage, T, h->y_stage, nullptr, stream);
  if (st != MOE_OK) return st;
  if (cudaMemcpyAsync(y_host, h->y_stage, bytes, cudaMemcpyDeviceToHost, s) != cudaSuccess)
    return MOE_ERR_CUDA;
  return moe_status(h, stream);
}

int32_t moe_forward_host_async(moe_mxfp4_t* h, const void* x_host, int32_t T, void* y_host,
                               void* stream) {
  if (!h || T < 0 || T > h->cfg.max_tokens) return MOE_ERR_INVALID_ARG;
  if (T == 0) return MOE_OK;
  if (!x_host || !y_host) return MOE_ERR_INVALID_ARG;
  if (!host_async_ready(h)) return MOE_ERR_CUDA;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int k = (int)(h->host_seq & 1u);
  const size_t bytes = (size_t)T * h->cfg.hidden * 2;
  // slot k was last used two calls ago: its input is free once that call's
  // layers ran, its output once that call's copy back finished
  if (cudaStreamWaitEvent(h->h2d, h->ev_k[k], 0) != cudaSuccess ||
      cudaMemcpyAsync(h->x_stage2[k], x_host, bytes, cudaMemcpyHostToDevice, h->h2d) != cudaSuccess ||
      cudaEventRecord(h->ev_in[k], h->h2d) != cudaSuccess ||
      cudaStreamWaitEvent(s, h->ev_in[k], 0) != cudaSuccess ||
      cudaStreamWaitEvent(s, h->ev_out[k], 0) != cudaSuccess)
    return MOE_ERR_CUDA;
  const int32_t st = moe_forward(h, h->x_stage2[k], T, h->y_stage2[k], nullptr, stream);
  if (st != MOE_OK) return st;
  if (cudaEventRecord(h->ev_k[k], s) != cudaSuccess ||
      cudaStreamWaitEvent(h->d2h, h->ev_k[k], 0) != cudaSuccess ||
      cudaMemcpyAsync(y_host, h->y_stage2[k], bytes, cudaMemcpyDeviceToHost, h->d2h) != cudaSuccess ||
      cudaEventRecord(h->ev_out[k], h->d2h) != cudaSuccess)
    return MOE_ERR_CUDA;
  ++h->host_seq;
  return MOE_OK;
}

int32_t moe_host_join(moe_mxfp4_t* h, void* stream) {
  if (!h) return MOE_ERR_INVALID_ARG;
  if (!h->h2d) return MOE_OK;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  for (int k = 0; k < 2; ++k)
    if (cudaStreamWaitEvent(s, h->ev_out[k], 0) != cudaSuccess) return MOE_ERR_CUDA;
  return MOE_OK;
}

int32_t moe_phase_ns(moe_mxfp4_t* h, uint64_t* ns_out, int32_t max_n, void* stream) {
  if (!h || !ns_out || max_n < 0) return MOE_ERR_INVALID_ARG;
  const int n = h->cfg.num_layers * STAMPS_PER_LAYER;
  uint64_t raw[1 + MAX_LAYERS * STAMPS_PER_LAYER];
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess ||
      cudaMemcpy(raw, h->stamps, (size_t)(1 + n) * 8, cudaMemcpyDeviceToHost) != cudaSuccess)
    return MOE_ERR_CUDA;
  for (int i = 0; i < n && i < max_n; ++i) ns_out[i] = raw[i + 1] - raw[i];
  return MOE_OK;
}

int32_t moe_stream_profile(moe_mxfp4_t* h, int32_t enable, uint64_t* out, int32_t max_n,
                           void* stream) {
  if (!h || max_n < 0 || (max_n > 0 && !out)) return MOE_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(s) != cudaSuccess) return MOE_ERR_CUDA;
  if (max_n > 0) {
    uint64_t raw[PROF_COUNTERS];
    if (cudaMemcpy(raw, h->prof, sizeof(raw), cudaMemcpyDeviceToHost) != cudaSuccess) return MOE_ERR_CUDA;
    for (int i = 0; i < PROF_COUNTERS && i < max_n; ++i) out[i] = raw[i];
  }
  if (cudaMemset(h->prof, 0, (size_t)PROF_COUNTERS * 8) != cudaSuccess) return MOE_ERR_CUDA;
  h->profiling = enable != 0;
  return MOE_OK;
}

int32_t moe_set_timeout_ns(moe_mxfp4_t* h, uint64_t ns) {
  if (!h || ns == 0) return MOE_ERR_INVALID_ARG;
  h->timeout_ns = ns;
  return MOE_OK;
}

int32_t moe_engine_grid(const moe_mxfp4_t* h) { return h ? h->grid : 0; }

void moe_mxfp4_destroy(moe_mxfp4_t* h) {
  if (!h) return;
  if (h->h2d) {  // copies of moe_forward_host_async still in flight
    cudaStreamSynchronize(h->h2d);
    cudaStreamSynchronize(h->d2h);
  }
  free_all(h);
  delete h;
}

}  // extern "C"
