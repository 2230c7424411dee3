// moe_route_static: routing (router logits, top-k, renormalised weights,
// per-expert permutation) without a handle and without any device allocation.
//
// Who needs it: callers that cannot call cudaMalloc -- code running while a
// caching allocator owns all free memory, a process under a fixed memory
// budget that was reserved up front, or a runtime that forbids allocation on
// its serving path -- but still want the router of this library.  The regular
// moe_route needs a handle, and moe_mxfp4_create allocates.
//
// The working memory the routing kernel needs beyond its inputs and outputs
// (fp64 partial logits, the unit table, barrier and status words)
// lives in one file-scope __device__ array of MOE_ROUTE_STATIC_SCRATCH_BYTES.
// Every device that loads this library holds that array until the process
// exits.  All calls share it: two calls whose kernels overlap on the GPU (on
// different streams, or from different host threads) race on it and give
// wrong results; serialise them.  Each call clears the words that must start
// at zero; everything else is fully rewritten before it is read.
#include "moe_mxfp4.h"

#include <cstdlib>
#include <mutex>

#include "engine.cuh"

using namespace moe;

namespace {

constexpr size_t kScratchBytes = MOE_ROUTE_STATIC_SCRATCH_BYTES;
__device__ __align__(256) unsigned char g_route_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_setup_mutex;
void* g_scratch_ptr[kMaxDevices] = {};
int g_grid[kMaxDevices] = {};

size_t align256(size_t v) { return (v + 255) & ~size_t(255); }

struct Layout {
  size_t logits, units, dunits, n_units, tokpos, wpos, sync, total;
  int umax;
};

// Offsets of every scratch region the routing-only engine launch touches.
Layout layout_for(int T, int H, int E, int K) {
  Layout l{};
  const int64_t TK = (int64_t)T * K;
  l.umax = max_units(E, TK);
  size_t o = 0;
  l.sync = o;    o = align256(o + (size_t)(SY_READY + l.umax) * 4);
  l.logits = o;  o = align256(o + (size_t)router_hsplit(H) * T * E * 8);
  l.units = o;   o = align256(o + (size_t)l.umax * 16);
  l.dunits = o;  o = align256(o + (size_t)max_dunits(E, TK) * 16);
  l.n_units = o; o = align256(o + 16);
  l.tokpos = o;  o = align256(o + (size_t)TK * 4);
  l.wpos = o;    o = align256(o + (size_t)TK * 4);
  l.total = o;
  return l;
}

// Once per device, with that device current: the device address of the
// scratch array (the host-side symbol is only a stand-in) and the engine grid.
int32_t setup_device(int dev, void** scratch, int* grid) {
  if (dev < 0 || dev >= kMaxDevices) return MOE_ERR_DEVICE;
  std::lock_guard<std::mutex> lock(g_setup_mutex);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_route_scratch) != cudaSuccess || !p) {
      cudaGetLastError();
      return MOE_ERR_CUDA;
    }
    int err = 0, sms = 0;
    const int maxg = engine_max_grid(dev, &err);
    if (err || maxg < 1 || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
      cudaGetLastError();
      return MOE_ERR_DEVICE;
    }
    g_grid[dev] = maxg < sms ? maxg : sms;
    g_scratch_ptr[dev] = p;
  }
  *scratch = g_scratch_ptr[dev];
  *grid = g_grid[dev];
  return MOE_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

extern "C" MOE_API int32_t moe_route_static(const void* x_bf16, int32_t T, int32_t hidden,
                                            const float* router_w, const float* router_bias,
                                            int32_t num_experts, int32_t top_k, int32_t* topk_idx,
                                            float* topk_w, int32_t* counts, int32_t* offsets,
                                            int32_t* perm, int32_t* inv_perm, void* stream) {
  if (T < 0 || hidden <= 0 || num_experts <= 0 || top_k <= 0 || top_k > num_experts)
    return MOE_ERR_INVALID_ARG;
  if (hidden % KS || hidden > 8192 || num_experts > MAX_EXPERTS || top_k > 32)
    return MOE_ERR_UNSUPPORTED_SHAPE;
  if (T == 0) return MOE_OK;
  if (!x_bf16 || !router_w || !topk_idx || !topk_w || !counts || !offsets || !perm || !inv_perm ||
      !aligned16(x_bf16) || !aligned16(router_w))
    return MOE_ERR_INVALID_ARG;
  const Layout lay = layout_for(T, hidden, num_experts, top_k);
  if ((int64_t)T * top_k > (int64_t)1 << 28 || lay.total > kScratchBytes) return MOE_ERR_UNSUPPORTED_SHAPE;

  int dev = 0, major = 0, minor = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) { cudaGetLastError(); return MOE_ERR_DEVICE; }
  cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
  cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
  if (major != 10 || minor != 0) return MOE_ERR_DEVICE;
  void* base = nullptr;
  int grid = 0;
  int32_t st = setup_device(dev, &base, &grid);
  if (st != MOE_OK) return st;

  unsigned char* s = static_cast<unsigned char*>(base);
  EngineParams p{};
  p.H = hidden; p.I = KS; p.E = num_experts; p.K = top_k; p.T = T; p.TK = T * top_k; p.L = 1;
  p.HS = router_hsplit(hidden);
  p.route_only = 1;
  p.timeout_ns = 2000000000ull;
  if (const char* env = std::getenv("MOE_TIMEOUT_NS")) {
    const unsigned long long v = std::strtoull(env, nullptr, 10);
    if (v > 0) p.timeout_ns = v;
  }
  p.layers[0] = LayerPtrs{nullptr, nullptr, router_w, router_bias};
  p.x_in = static_cast<const __nv_bfloat16*>(x_bf16);
  p.logits = reinterpret_cast<double*>(s + lay.logits);
  p.units = reinterpret_cast<int32_t*>(s + lay.units);
  p.dunits = reinterpret_cast<int32_t*>(s + lay.dunits);
  p.n_units = reinterpret_cast<int32_t*>(s + lay.n_units);
  p.tokpos = reinterpret_cast<int32_t*>(s + lay.tokpos);
  p.wpos = reinterpret_cast<float*>(s + lay.wpos);
  p.sync = reinterpret_cast<uint32_t*>(s + lay.sync);
  p.idx = topk_idx; p.wts = topk_w; p.counts = counts; p.offsets = offsets; p.perm = perm;
  p.inv = inv_perm;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  // barrier, job and status words must start at zero (a previous call that
  // timed out may have left them set)
  if (cudaMemsetAsync(p.sync, 0, SY_READY * sizeof(uint32_t), cs) != cudaSuccess) return MOE_ERR_CUDA;
  return engine_launch(p, grid, cs) == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

// The status word of the routing kernel sits at the start of the array (the
// sync region is at offset 0 for every size), so its address does not depend
// on the sizes of the last call.
extern "C" MOE_API int32_t moe_route_static_status(void* stream) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) { cudaGetLastError(); return MOE_ERR_DEVICE; }
  if (dev < 0 || dev >= kMaxDevices) return MOE_ERR_DEVICE;
  void* base = nullptr;
  {
    std::lock_guard<std::mutex> lock(g_setup_mutex);
    base = g_scratch_ptr[dev];
  }
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(cs) != cudaSuccess) { cudaGetLastError(); return MOE_ERR_CUDA; }
  if (!base) return MOE_OK;  // no call on this device yet
  uint32_t* sync = static_cast<uint32_t*>(base);
  uint32_t words[2] = {};
  static_assert(SY_ERRINFO == SY_ERROR + 1, "status and info words are adjacent");
  if (cudaMemcpyAsync(words, sync + SY_ERROR, sizeof(words), cudaMemcpyDeviceToHost, cs) != cudaSuccess ||
      cudaStreamSynchronize(cs) != cudaSuccess) {
    cudaGetLastError();
    return MOE_ERR_CUDA;
  }
  if (words[0] == DEV_OK) return MOE_OK;
  if (cudaMemsetAsync(sync, 0, SY_READY * sizeof(uint32_t), cs) != cudaSuccess ||
      cudaStreamSynchronize(cs) != cudaSuccess) {
    cudaGetLastError();
    return MOE_ERR_CUDA;
  }
  return MOE_ERR_TIMEOUT;
}
