// moe_route_noalloc: the router (moe_route) for callers that cannot provide a
// device workspace.
//
// Some callers own no device memory of their own: a plug-in whose host
// framework hands it only the input and output tensors (no workspace hook,
// no allocator it may call), or code running where a device allocation is not
// allowed or would break a memory plan fixed in advance. This entry point
// needs nothing beyond its inputs and outputs: the router's split-K partial
// sums live in the file-scope device array below instead of the caller's
// workspace. It computes what moe_route computes, but not with the same
// kernels: the logits come from a split-K CUDA-core GEMV of its own
// (k_dense_gemv, K split as router_splits below decides), and only the top-k
// launch (k_topk) is shared with moe_route. moe_route sums the logits on
// other kernels (a tensor-core row GEMV for one token, the tcgen05 GEMM for
// more), in another order, so the two agree to fp32 rounding of the logits:
// the selected experts are the same except where two router logits are a
// near tie, and the weights agree to the same rounding.
//
// Limits and rules:
// * the scratch holds kNoAllocScratchFloats fp32 values (4 MiB); shapes whose
//   partial sums need more (S * T * E floats) are rejected with
//   MOE_ERR_UNSUPPORTED_SHAPE before anything is enqueued;
// * every GPU that loads this library holds the 4 MiB until the process exits;
// * the array is shared by all calls on a device and keeps the last call's
//   contents; every element a call reads was written earlier in that same
//   call, so nothing needs clearing, but calls whose work overlaps on the
//   GPU (different streams without ordering) race on it;
// * the first call on each device looks up the array's device address
//   (cudaGetSymbolAddress, with that device current); make that first call
//   before capturing a stream into a CUDA graph;
// * no cudaMalloc, cudaFree or other allocating call is made.
#include <cuda_runtime.h>

#include <mutex>

#include "common.cuh"
#include "kernels.h"

namespace {

constexpr size_t kNoAllocScratchFloats = (size_t)1 << 20;   // 4 MiB of fp32

static __device__ __align__(256) float g_router_scratch[kNoAllocScratchFloats];

std::mutex g_noalloc_mu;
float* g_scratch_ptr[64] = {};

// Device address of g_router_scratch on the current device (looked up once).
moe_status scratch_address(float** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64)
    return moe::record_error(MOE_ERR_CUDA, "moe_route_noalloc: cudaGetDevice failed");
  std::lock_guard<std::mutex> lk(g_noalloc_mu);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_router_scratch);
    if (e != cudaSuccess || !p)
      return moe::record_error(MOE_ERR_CUDA, "moe_route_noalloc: cudaGetSymbolAddress failed");
    g_scratch_ptr[dev] = static_cast<float*>(p);
  }
  *out = g_scratch_ptr[dev];
  return MOE_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// K splits of this entry point's router GEMV: enough warps to cover 148 SMs at
// about 4 per SM, whole 32-element steps, at least 8 per split, at most 16
// splits. The split-K partials are summed by k_topk in split order, so every
// call on the same inputs gives the same bits.
int router_splits(int N, int T, int K) {
  const long warps = (long)((N + 15) / 16) * ((T + 31) / 32);
  const int ksteps = K / 32;
  int S = 1;
  for (int c = 1; c <= ksteps && c <= 16; ++c) {
    if (ksteps % c) continue;
    if (ksteps / c < 8) break;
    S = c;
    if (warps * c >= 148L * 4) break;
  }
  return S;
}

}  // namespace

extern "C" moe_status moe_route_noalloc(const moe_dims* dims, const uint16_t* x,
                                        const uint16_t* w_router, int32_t* topk_idx,
                                        float* topk_w, float* logits, void* stream) {
  if (moe_workspace_size(dims) == 0) return (moe_status)(dims ? MOE_ERR_UNSUPPORTED_SHAPE : MOE_ERR_INVALID_ARG);
  const void* ptrs[4] = {x, w_router, topk_idx, topk_w};
  const char* names[4] = {"x", "w_router", "topk_idx", "topk_w"};
  for (int i = 0; i < 4; ++i) {
    if (!ptrs[i]) return moe::record_error(MOE_ERR_INVALID_ARG, names[i]);
    if (!aligned16(ptrs[i])) return moe::record_error(MOE_ERR_ALIGNMENT, names[i]);
  }
  if (logits && !aligned16(logits)) return moe::record_error(MOE_ERR_ALIGNMENT, "logits");
  const int S = router_splits(dims->E, dims->T, dims->H);
  if ((size_t)S * dims->T * dims->E > kNoAllocScratchFloats)
    return moe::record_error(MOE_ERR_UNSUPPORTED_SHAPE,
                             "moe_route_noalloc: S*T*E partial sums exceed the 4 MiB static scratch "
                             "(use moe_route with a workspace)");
  float* part = nullptr;
  moe_status st = scratch_address(&part);
  if (st != MOE_OK) return st;
  const cudaStream_t cs = (cudaStream_t)stream;
  moe::DenseArgs a;
  a.w[0] = a.w[1] = a.w[2] = w_router;
  a.rows[0] = dims->E; a.rows[1] = 0; a.rows[2] = 0;
  a.N = dims->E;
  a.x = x; a.x_f32 = 0;
  a.part = part;
  a.T = dims->T; a.K = dims->H; a.S = S; a.kper = dims->H / S;
  const dim3 grid((a.N + 16 * moe::kDenseWarps - 1) / (16 * moe::kDenseWarps), S, (a.T + 31) / 32);
  moe::k_dense_gemv<<<grid, 32 * moe::kDenseWarps, 0, cs>>>(a);
  moe::RouteCfg rc;
  rc.bias = nullptr;
  rc.score_fn = dims->score_fn;
  rc.n_group = dims->n_group > 1 ? dims->n_group : 1;
  rc.topk_group = dims->n_group > 1 ? dims->topk_group : 1;
  rc.scale = dims->route_scale == 0.0f ? 1.0f : dims->route_scale;
  moe::k_topk<<<dims->T, moe::kTopkThreads, 0, cs>>>(part, S, dims->T, dims->E, dims->E, dims->k, topk_idx,
                                                     topk_w, logits, nullptr, moe::TopkFuse{}, rc);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return moe::record_error(MOE_ERR_CUDA, cudaGetErrorString(e));
  return MOE_OK;
}
