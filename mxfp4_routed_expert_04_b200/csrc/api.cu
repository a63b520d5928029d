// C ABI of the routed MXFP4 MoE layer: validation, workspace plan, launch
// order. Declared in include/moe_mxfp4.h.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>
#include <stdarg.h>
#include <stdio.h>
#include <string.h>

#include <algorithm>
#include <mutex>
#include <vector>

#include "../../include/moe_mxfp4.h"
#include "kernels.h"

namespace {

thread_local char g_err[512] = "";

moe_status fail(moe_status s, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof(g_err), fmt, ap);
  va_end(ap);
  return s;
}

constexpr int kNumSMs = 148;

inline size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Token count from which the shared expert's gate/up GEMM applies SwiGLU in its
// epilogue (below it the gate, up and sigmoid-gate rows write split-K
// partial sums and a finaliser applies SwiGLU).
constexpr int kDenseSwiGLUTokens = 128;

// One token: the router and the shared expert stream contiguous ranges of
// weight rows through the tensor-core row GEMV (k_rows_bf16, no split-K) when
// both reduction lengths (H, I_shared) are powers of two in 1024..8192;
// otherwise they take the tcgen05 GEMM with a 16-token tile.
bool rows_k_ok(int K) { return K == 1024 || K == 2048 || K == 4096 || K == 8192; }
bool rows_path_for(int T, int H, int Is) { return T == 1 && rows_k_ok(H) && rows_k_ok(Is); }
constexpr size_t kRowsSmemBudget = 220 * 1024;
constexpr int kRowsFreeSMs = 8;     // SMs a side-stream row GEMV leaves to the routing chain
// one token: the router row GEMV (8.4 MB at decode1) takes 3/8 of the SMs,
// and in moe_layer the shared expert's first half (67 MB) the others from the
// start, so that both end close to when the top-k does (with all SMs for the
// router, the shared expert starts only as the router's CTAs leave)
constexpr int kLayerRouterEighths = 3;

// Token tile of the tcgen05 bf16 GEMM: the MMA's N, a multiple of 16 up to 128.
int tc_tile_tokens(int T) { return T >= 128 ? 128 : (T + 15) / 16 * 16; }

// K splits of a tcgen05 bf16 GEMM over `units` (weight units x token tiles):
// double while the SMs are covered less than four times over, each split keeps
// at least two 64-element stages and the partial sums (`split_bytes` per
// split) stay within 40 MB.
int tc_splits(long units, int K, size_t split_bytes) {
  const int ks = K / 64;
  int S = 1;
  while (S < 64 && units * S < 4L * kNumSMs && ks % (2 * S) == 0 && ks / (2 * S) >= 2 &&
         (size_t)(2 * S) * split_bytes <= (40u << 20))
    S *= 2;
  return S;
}

// 32-bit word of the 256-byte status region (cleared by moe_workspace_init)
// where the one-token launch's counters start: kRouted1SyncWords words
constexpr int kSyncWord = 16;
static_assert(4 * (kSyncWord + moe::kRouted1SyncWords) <= 256, "counters inside the status region");

struct Plan {
  int T, H, I, E, k, Is, L, W, R, mode;
  moe::RouteCfg rc;          // router variant (bias pointer filled per call)
  int S_router, S_sgu, S_sd, S_ld, S_lu;
  int Nt;                    // token tile of the tcgen05 bf16 GEMMs
  bool swiglu_tc;            // shared gate/up GEMM applies SwiGLU in its epilogue
  bool rows;                 // one token: router and shared expert on k_rows_bf16
  size_t off_hsb;            // shared expert h as a bf16 hi/lo pair [2][T, I_shared]
  size_t off_status, off_router, off_h16, off_hscale, off_h32, off_sgu, off_gl, off_sd, off_ld,
      off_ylat, off_lu, off_hsf, total;
  int max_tiles;
  size_t xop_bytes, xop_scale_off, xop_tiles_off, xop_tbase_off, xop_ntiles_off;
};

moe_status check_dims(const moe_dims* d) {
  if (!d) return fail(MOE_ERR_INVALID_ARG, "dims is NULL");
  if (d->act_mode != MOE_ACT_BF16 && d->act_mode != MOE_ACT_MXFP4)
    return fail(MOE_ERR_INVALID_ARG, "act_mode %d is not a moe_act_mode", d->act_mode);
  if (d->T < 1 || d->T > 65536) return fail(MOE_ERR_UNSUPPORTED_SHAPE, "T=%d outside [1, 65536]", d->T);
  if (d->E < 1 || d->E > 1024) return fail(MOE_ERR_UNSUPPORTED_SHAPE, "E=%d outside [1, 1024]", d->E);
  if (d->k < 1 || d->k > 32 || d->k > d->E)
    return fail(MOE_ERR_UNSUPPORTED_SHAPE, "k=%d outside [1, min(E, 32)]", d->k);
  const int dims4[4] = {d->H, d->I, d->I_shared, d->L};
  const char* names[4] = {"H", "I", "I_shared", "L"};
  for (int i = 0; i < 4; ++i) {
    if (i == 3 && d->L == 0) continue;
    if (dims4[i] < 128 || dims4[i] % 128 != 0 || dims4[i] > (1 << 16))
      return fail(MOE_ERR_UNSUPPORTED_SHAPE, "%s=%d is not a multiple of 128 in [128, 65536]",
                  names[i], dims4[i]);
  }
  if ((long)d->T * d->k > (1L << 24))
    return fail(MOE_ERR_UNSUPPORTED_SHAPE, "T*k=%ld above 2^24", (long)d->T * d->k);
  if (d->score_fn != MOE_SCORE_SOFTMAX && d->score_fn != MOE_SCORE_SIGMOID)
    return fail(MOE_ERR_INVALID_ARG, "score_fn %d is not a moe_score_fn", d->score_fn);
  if (!(d->route_scale >= 0.0f) || d->route_scale > 1e30f)
    return fail(MOE_ERR_INVALID_ARG, "route_scale must be finite and >= 0");
  if (d->n_group > 1) {
    if (d->n_group > moe::kMaxGroups || d->E % d->n_group != 0)
      return fail(MOE_ERR_UNSUPPORTED_SHAPE, "n_group=%d must divide E=%d and be <= %d", d->n_group,
                  d->E, moe::kMaxGroups);
    if (d->topk_group < 1 || d->topk_group > d->n_group ||
        (long)d->topk_group * (d->E / d->n_group) < d->k)
      return fail(MOE_ERR_UNSUPPORTED_SHAPE,
                  "topk_group=%d: needs 1 <= topk_group <= n_group and topk_group*E/n_group >= k",
                  d->topk_group);
  } else if (d->n_group < 0) {
    return fail(MOE_ERR_UNSUPPORTED_SHAPE, "n_group=%d is negative", d->n_group);
  }
  return MOE_OK;
}

moe_status make_plan(const moe_dims* d, Plan& p) {
  moe_status st = check_dims(d);
  if (st != MOE_OK) return st;
  p.T = d->T; p.H = d->H; p.I = d->I; p.E = d->E; p.k = d->k; p.Is = d->I_shared; p.L = d->L;
  p.W = d->L ? d->L : d->H;
  p.R = d->T * d->k;
  p.mode = d->act_mode;
  p.rc.bias = nullptr;
  p.rc.score_fn = d->score_fn;
  p.rc.n_group = d->n_group > 1 ? d->n_group : 1;
  p.rc.topk_group = d->n_group > 1 ? d->topk_group : 1;
  p.rc.scale = d->route_scale == 0.0f ? 1.0f : d->route_scale;
  p.Nt = tc_tile_tokens(p.T);
  p.swiglu_tc = p.T >= kDenseSwiGLUTokens;
  p.rows = rows_path_for(p.T, p.H, p.Is);
  if (p.rows) {
    p.S_router = 1;
    p.S_sgu = 1;
    p.S_sd = 1;
  } else {
    const long ntt = (p.T + p.Nt - 1) / p.Nt;
    // the router rows, the sigmoid-gate row and the latent down-projection
    // rows share one pass over x (the same splits when launched alone)
    p.S_router = tc_splits((long)((p.E + 255) / 256 + 1 + (p.L + 255) / 256) * ntt, p.H,
                           (size_t)p.T * (p.E + 1 + p.L) * 4);
    // SwiGLU epilogue: one split, the sigmoid-gate row on the GEMV
    p.S_sgu = p.swiglu_tc ? 1
                          : tc_splits((long)(2 * ((p.Is + 255) / 256) + 1) * ntt, p.H,
                                      (size_t)p.T * (2 * p.Is + 1) * 4);
    p.S_sd = tc_splits((long)((p.H + 255) / 256) * ntt, p.Is, (size_t)p.T * p.H * 4);
  }
  p.S_ld = p.L ? p.S_router : 0;
  p.S_lu = p.L ? tc_splits((long)((p.H + 255) / 256) * ((p.T + p.Nt - 1) / p.Nt), p.L,
                           (size_t)p.T * p.H * 4)
               : 0;
  size_t o = 0;
  auto take = [&](size_t bytes) { size_t r = o; o = align_up(o + bytes, 256); return r; };
  p.off_status = take(256);            // status word, then (from int kSyncWord) the one-token counters
  // + the sigmoid-gate column (+ the latent down-projection columns on the
  // tcgen05 GEMM)
  p.off_router = take((size_t)p.S_router * p.T * (p.E + 1 + (p.rows ? 0 : p.L)) * 4);
  p.off_h16 = take((size_t)p.R * p.I * 2);
  p.off_hscale = take((size_t)p.R * (p.I / 16) * 4);
  p.off_h32 = take((size_t)p.R * p.I * 4);
  p.off_sgu = take(p.swiglu_tc || p.rows ? 0 : (size_t)p.S_sgu * p.T * (2 * p.Is + 1) * 4);
  // shared expert h: a bf16 hi/lo pair [2][T, I_shared]; one token on the row
  // GEMV: fp32 [I_shared] in the same bytes
  p.off_hsb = take((size_t)2 * p.T * p.Is * 2);
  p.off_gl = take((size_t)p.T * 4);
  p.off_sd = take((size_t)p.S_sd * p.T * p.H * 4);
  p.off_ld = take(p.L ? (size_t)p.S_ld * p.T * p.L * 4 : 0);
  p.off_ylat = take(p.L ? (size_t)p.T * p.L * 4 : 0);   // bf16 pair [2][T, L]
  p.off_lu = take(p.L ? (size_t)p.S_lu * p.T * p.H * 4 : 0);
  // MXFP4 activations: tiles of at most kTileRows rows of one expert; the sum
  // over experts of ceil(rows / kTileRows) is below R / kTileRows + (experts) + 1.
  // h codes reuse the h16 region (larger); h scales are tiled.
  p.max_tiles = p.mode == MOE_ACT_MXFP4 ? p.R / moe::kTileRows + std::min(p.E, p.R) + 1 : 0;
  p.off_hsf = take((size_t)p.max_tiles * (p.I / 128) * 512);
  p.total = o;
  if (p.mode == MOE_ACT_BF16) {
    p.xop_scale_off = align_up((size_t)p.T * p.W * 2, 256);
    p.xop_bytes = p.xop_scale_off + (size_t)p.T * 4;
    p.xop_tiles_off = p.xop_tbase_off = p.xop_ntiles_off = 0;
  } else {
    p.xop_scale_off = align_up((size_t)p.R * p.W / 2, 256);
    p.xop_tiles_off = align_up(p.xop_scale_off + (size_t)p.max_tiles * (p.W / 128) * 512, 256);
    p.xop_tbase_off = align_up(p.xop_tiles_off + (size_t)p.max_tiles * 16, 256);
    p.xop_ntiles_off = align_up(p.xop_tbase_off + (size_t)p.E * 4, 256);
    p.xop_bytes = p.xop_ntiles_off + 16;
  }
  return MOE_OK;
}

template <typename T>
T* at(void* ws, size_t off) { return reinterpret_cast<T*>(static_cast<char*>(ws) + off); }

moe_status check_ws(const Plan& p, void* ws, size_t ws_bytes) {
  if (!ws) return fail(MOE_ERR_INVALID_ARG, "workspace is NULL");
  if (!aligned16(ws)) return fail(MOE_ERR_ALIGNMENT, "workspace not 16-byte aligned");
  if (ws_bytes < p.total)
    return fail(MOE_ERR_WORKSPACE_TOO_SMALL, "workspace %zu bytes < %zu needed", ws_bytes, p.total);
  return MOE_OK;
}

#define CHECK_PTR(p)                                                                   \
  do {                                                                                 \
    if (!(p)) return fail(MOE_ERR_INVALID_ARG, "%s is NULL", #p);                      \
    if (!aligned16(p)) return fail(MOE_ERR_ALIGNMENT, "%s is not 16-byte aligned", #p); \
  } while (0)

moe_status launched(const char* what) {
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return fail(MOE_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
  return MOE_OK;
}

// Launch with programmatic stream serialization: the kernel may start while
// the previous kernel of the stream is still running (every kernel of this
// library waits in pdl_wait() before it reads memory), hiding the launch gap.
template <typename... KArgs, typename... Args>
void launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                Args... args) {
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaLaunchKernelEx(&cfg, kernel, args...);
}

// per-device one-time setup: kernel attributes, the side stream and events of moe_layer
struct DeviceState {
  bool ready = false;
  int num_sms = 0;
  int gemv_ctas_per_sm = 0;
  cudaStream_t side = nullptr;
  cudaEvent_t ev_fork = nullptr, ev_shared = nullptr;
};
std::mutex g_mu;
DeviceState g_dev[64];

moe_status device_state(DeviceState** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64)
    return fail(MOE_ERR_CUDA, "cudaGetDevice failed");
  std::lock_guard<std::mutex> lk(g_mu);
  DeviceState& s = g_dev[dev];
  if (!s.ready) {
    cudaError_t e = cudaFuncSetAttribute(moe::k_permute, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)moe::permute_smem_bytes(1024, 1 << 24));
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(moe::k_mxf4_gemm<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               (int)moe::mxf4_gemm_smem_bytes(true));
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(moe::k_mxf4_gemm<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               (int)moe::mxf4_gemm_smem_bytes(false));
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(moe::k_bf16_gemm, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               moe::kBf16SmemBudget + 1024 + 256);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(moe::k_mma_gateup, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               (int)moe::mma_gateup_smem_bytes());
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(moe::k_mma_down, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               (int)moe::mma_down_smem_bytes());
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(moe::k_rows_bf16<false, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               (int)kRowsSmemBudget);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(moe::k_rows_bf16<true, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               (int)kRowsSmemBudget);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(moe::k_rows_bf16<false, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               (int)kRowsSmemBudget);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&s.num_sms, cudaDevAttrMultiProcessorCount, dev);
    if (e == cudaSuccess)
      e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&s.gemv_ctas_per_sm, moe::k_gateup_mxfp4, 32,
                                                        moe::gemv_mxfp4_smem_bytes());
    if (e == cudaSuccess && s.gemv_ctas_per_sm < 1) s.gemv_ctas_per_sm = 1;
    if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&s.side, cudaStreamNonBlocking);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&s.ev_fork, cudaEventDisableTiming);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&s.ev_shared, cudaEventDisableTiming);
    if (e != cudaSuccess) return fail(MOE_ERR_CUDA, "device setup: %s", cudaGetErrorString(e));
    s.ready = true;
  }
  *out = &s;
  return MOE_OK;
}

// ---------------------------------------------------------------------------
// launchers (arguments already validated)
// ---------------------------------------------------------------------------

// single-token row GEMV: one CTA per SM (at most max_ctas), ring depth from
// the shared-memory budget
// slots of a stage: the units of a CTA rounded up to a power of two (at most
// 16 MMA rows), so that a CTA's few rows come in whole-row stages; the slots
// set the K chunk of a stage and so the order of each row's sum
int rows_slots(long units, int grid, bool swiglu) {
  const long per = (units + grid - 1) / grid;
  int pp = 1;
  while (pp < per && pp < (swiglu ? 8 : 16)) pp <<= 1;
  return swiglu ? 2 * pp : pp;
}
moe_status launch_rows(const DeviceState& ds, moe::RowsArgs& r, bool swiglu, bool x_f32, int max_ctas,
                       cudaStream_t st, const char* what, bool pdl = true, int force_slots = 0) {
  const long units = swiglu ? r.rows[0] : (long)r.rows[0] + r.rows[1] + r.rows[2];
  const int grid = (int)std::max<long>(1, std::min<long>(units, max_ctas));
  r.slots = force_slots > 0 ? force_slots : rows_slots(units, grid, swiglu);
  r.nst = moe::rows_stages(r.K, r.slots, x_f32, kRowsSmemBudget);
  if (!r.nst) return fail(MOE_ERR_UNSUPPORTED_SHAPE, "%s: K=%d too long for the row GEMV", what, r.K);
  const size_t smem = (size_t)r.nst * moe::rows_stage_bytes(r.K, r.slots) + moe::rows_act_bytes(r.K, x_f32);
  void (*kern)(moe::RowsArgs) = swiglu ? moe::k_rows_bf16<true, false>
                                       : (x_f32 ? moe::k_rows_bf16<false, true> : moe::k_rows_bf16<false, false>);
  const dim3 block(32 * (moe::kRowsConsumers + 1));
  if (pdl) launch_pdl(kern, dim3(grid), block, smem, st, r);
  else kern<<<grid, block, smem, st>>>(r);
  return launched(what);
}

moe_status do_permute(const Plan& p, const int32_t* idx, const uint16_t* xin, int32_t* counts,
                      int32_t* offsets, int32_t* expert_list, int32_t* row_token, int32_t* row_slot,
                      int32_t* slot_row, void* x_op, void* ws, cudaStream_t st) {
  launch_pdl(moe::k_permute, dim3(1), dim3(1024), moe::permute_smem_bytes(p.E, p.R), st, idx, p.T, p.k, p.E,
             counts, offsets, expert_list, row_token, row_slot, slot_row, at<int32_t>(ws, p.off_status));
  moe_status s = launched("permute");
  if (s != MOE_OK) return s;
  if (p.mode == MOE_ACT_BF16) {
    launch_pdl(moe::k_act_to_f16, dim3(p.T), dim3(256), 0, st, xin, p.W, static_cast<__half*>(x_op),
               at<float>(x_op, p.xop_scale_off));
  } else {
    moe::k_tile_list<<<1, 1024, 0, st>>>(offsets, expert_list, at<int4>(x_op, p.xop_tiles_off),
                                         at<int32_t>(x_op, p.xop_tbase_off),
                                         at<int32_t>(x_op, p.xop_ntiles_off));
    if ((s = launched("tile list")) != MOE_OK) return s;
    moe::k_act_to_mxfp4_perm<<<p.T, 256, 0, st>>>(
        xin, p.W, p.k, idx, slot_row, offsets, expert_list, at<int32_t>(x_op, p.xop_tbase_off),
        static_cast<uint8_t*>(x_op), at<uint8_t>(x_op, p.xop_scale_off));
  }
  return launched("activation operand");
}

// CUDA-core GEMV launch shape for reduction length K (up to 8192): lanes own
// BPL = ceil(K/1024) blocks; one CTA per SM with a ring of MOE_FMA_SMEM_KB KB.
#ifndef MOE_FMA_SMEM_KB
#define MOE_FMA_SMEM_KB 224
#endif
struct FmaPlan {
  int bpl = 0;
  moe::FmaGeometry g{};
};
FmaPlan fma_plan(int K, bool gate_up) {
  FmaPlan f;
  const int kb = K / 32;
  f.bpl = kb <= 32 ? 1 : kb <= 64 ? 2 : kb <= 128 ? 4 : kb <= 256 ? 8 : 0;
  if (!f.bpl) return f;
  f.g = moe::fma_geometry(K, gate_up, (size_t)MOE_FMA_SMEM_KB * 1024);
  return f;
}
// the CUDA-core path serves single-token experts when both projections fit it
bool fma_path(const Plan& p) { return fma_plan(p.W, true).g.ok && fma_plan(p.I, false).g.ok; }

// one token: the CUDA-core path in one launch, when its down role's two h
// buffers fit beside the ring
bool routed1_path(const Plan& p) {
  if (p.T != 1 || p.k > moe::kRouted1MaxK || p.mode != MOE_ACT_BF16 || !fma_path(p)) return false;
  moe::FmaGeometry gg, gd;
  moe::routed1_geometry(p.W, p.I, (size_t)MOE_FMA_SMEM_KB * 1024, gg, gd);
  return gg.ok;
}

// One token: both projections of its experts in one launch (k_fma_routed1),
// one CTA per SM taking chunks from the counters in the status region.
moe_status launch_routed1(const DeviceState& ds, const Plan& p, const moe::FmaArgs& a, cudaStream_t st) {
  const char* what = "expert gate/up + down (cuda cores, one launch)";
  moe::FmaGeometry gg, gd;
  moe::routed1_geometry(a.W, a.I, (size_t)MOE_FMA_SMEM_KB * 1024, gg, gd);
  const int bg = fma_plan(a.W, true).bpl, bd = fma_plan(a.I, false).bpl;
  if (!gg.ok || !bg || !bd) return fail(MOE_ERR_UNSUPPORTED_SHAPE, "%s: no geometry", what);
  using K = void (*)(moe::FmaArgs, moe::FmaGeometry, moe::FmaGeometry);
  static const K table[4][4] = {
      {moe::k_fma_routed1<1, 1, 8>, moe::k_fma_routed1<1, 2, 4>, moe::k_fma_routed1<1, 4, 2>, moe::k_fma_routed1<1, 8, 1>},
      {moe::k_fma_routed1<2, 1, 8>, moe::k_fma_routed1<2, 2, 4>, moe::k_fma_routed1<2, 4, 2>, moe::k_fma_routed1<2, 8, 1>},
      {moe::k_fma_routed1<4, 1, 8>, moe::k_fma_routed1<4, 2, 4>, moe::k_fma_routed1<4, 4, 2>, moe::k_fma_routed1<4, 8, 1>},
      {moe::k_fma_routed1<8, 1, 8>, moe::k_fma_routed1<8, 2, 4>, moe::k_fma_routed1<8, 4, 2>, moe::k_fma_routed1<8, 8, 1>}};
  auto idx = [](int bpl) { return bpl == 1 ? 0 : bpl == 2 ? 1 : bpl == 4 ? 2 : 3; };
  const K kern = table[idx(bg)][idx(bd)];
  if (gd.rps != (bd == 1 ? 8 : bd == 2 ? 4 : bd == 4 ? 2 : 1))
    return fail(MOE_ERR_UNSUPPORTED_SHAPE, "%s: down rows per warp %d", what, gd.rps);
  const cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)gg.smem_bytes);
  if (e != cudaSuccess) return fail(MOE_ERR_CUDA, "%s setup: %s", what, cudaGetErrorString(e));
  const long n = std::min(p.E, p.k);
  const long chunks = n * ((a.I + gg.units - 1) / gg.units + (a.W + gd.units - 1) / gd.units);
  const int grid = (int)std::min<long>(ds.num_sms, std::max(1L, chunks));
  launch_pdl(kern, dim3((unsigned)grid), dim3(32 * moe::kRouted1Warps), gg.smem_bytes, st, a, gg, gd);
  return launched(what);
}

template <bool kGateUp>
moe_status launch_fma(const DeviceState& ds, const moe::FmaArgs& a, cudaStream_t st) {
  const int K = kGateUp ? a.W : a.I;
  const FmaPlan f = fma_plan(K, kGateUp);
  const char* what = kGateUp ? "expert gate/up (cuda cores)" : "expert down (cuda cores)";
  void (*kern)(moe::FmaArgs, moe::FmaGeometry) = nullptr;
  if (f.bpl == 1) kern = moe::k_fma_gemv<1, kGateUp, kGateUp ? 1 : 8>;
  if (f.bpl == 2) kern = moe::k_fma_gemv<2, kGateUp, kGateUp ? 1 : 4>;
  if (f.bpl == 4) kern = moe::k_fma_gemv<4, kGateUp, kGateUp ? 1 : 2>;
  if (f.bpl == 8) kern = moe::k_fma_gemv<8, kGateUp, 1>;
  if (!kern || !f.g.ok) return fail(MOE_ERR_UNSUPPORTED_SHAPE, "%s: no kernel for K=%d", what, K);
  const int threads = 32 * (moe::kFmaConsumers + 1);
  const cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)f.g.smem_bytes);
  if (e != cudaSuccess) return fail(MOE_ERR_CUDA, "%s setup: %s", what, cudaGetErrorString(e));
  // one CTA per SM, each with an equal share of the units of the single-token experts
  const long units = (long)std::min(a.E, a.R) * (kGateUp ? a.I : a.W);
  const long ctas = std::max<long>(1, std::min<long>((units + f.g.units - 1) / f.g.units, ds.num_sms));
  launch_pdl(kern, dim3((unsigned)ctas), dim3(threads), f.g.smem_bytes, st, a, f.g);
  return launched(what);
}

// cuTensorMapEncodeTiled from the driver, looked up once through the runtime
// (the library links no driver stub).
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
  });
  return fn;
}

// 2-D map over a row-major [rows, cols] matrix read in boxes of box_rows rows
// x 128 bytes with the 128-byte swizzle (a row a multiple of 16 bytes).
moe_status tile_map(CUtensorMap* m, const void* base, CUtensorMapDataType dtype, uint32_t elem_bytes,
                    uint64_t rows, uint64_t cols, uint32_t box_rows, const char* what) {
  PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
  if (!enc) return fail(MOE_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {cols * elem_bytes};
  const cuuint32_t box[2] = {128 / elem_bytes, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = enc(m, dtype, 2, const_cast<void*>(base), dims, strides, box, estr,
                         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(MOE_ERR_CUDA, "tensor map for %s: CUresult %d", what, (int)r);
  return MOE_OK;
}

// bytes [rows, row_bytes] read in unswizzled boxes of box_bytes x box_rows
moe_status byte_map(CUtensorMap* m, const void* base, uint64_t rows, uint64_t row_bytes, uint32_t box_bytes,
                    uint32_t box_rows, const char* what) {
  PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
  if (!enc) return fail(MOE_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
  const cuuint64_t dims[2] = {row_bytes, rows};
  const cuuint64_t strides[1] = {row_bytes};
  const cuuint32_t box[2] = {box_bytes, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
                         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(MOE_ERR_CUDA, "tensor map for %s: CUresult %d", what, (int)r);
  return MOE_OK;
}

// MXFP4 codes: [rows, row_bytes] bytes
moe_status code_map(CUtensorMap* m, const uint8_t* base, uint64_t rows, uint64_t row_bytes,
                    uint32_t box_rows, const char* what) {
  return tile_map(m, base, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, rows, row_bytes, box_rows, what);
}

// bf16 matrices: [rows, cols] elements
moe_status bf16_map(CUtensorMap* m, const uint16_t* base, uint64_t rows, uint64_t cols,
                    const char* what, uint32_t box_rows = 128) {
  return tile_map(m, base, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, rows, cols, box_rows, what);
}

// grid: one CTA per SM at most (the stage ring takes most of shared memory)
moe_status launch_bf16_gemm(const DeviceState& ds, moe::Bf16GemmArgs& g, cudaStream_t st,
                            const char* what, bool pdl = true) {
  long units = 0;
  for (int i = 0; i < 3; ++i)
    units += g.mode == moe::kBf16SwiGLU ? (i == 0 ? g.seg_rows[0] / 128 : 0) : (g.seg_rows[i] + 255) / 256;
  const long items = units * ((g.T + g.N - 1) / g.N) * g.S;
  const int grid = (int)std::min<long>(items, ds.num_sms);
  const size_t smem = moe::bf16_gemm_smem_bytes(g.N, g.passes);
  if (pdl) launch_pdl(moe::k_bf16_gemm, dim3(grid), dim3(moe::bf16_gemm_threads()), smem, st, g);
  else moe::k_bf16_gemm<<<grid, moe::bf16_gemm_threads(), smem, st>>>(g);
  return launched(what);
}

// x_lat[t, n] = bf16(sum_s part[s, t, n]) from the latent down-projection's
// partial sums (rows of ld floats)
moe_status round_latent(const Plan& p, const float* part, int ld, uint16_t* x_lat, cudaStream_t st) {
  launch_pdl(moe::k_round_bf16, dim3((p.L + moe::kFinThreads - 1) / moe::kFinThreads, p.T),
             dim3(moe::kFinThreads), 0, st, part, p.S_ld, p.T, p.L, ld, x_lat);
  return launched("latent round");
}

// The router logits, then top-k. The same pass over x can carry the shared
// expert's sigmoid-gate row (w_sgate) and the latent down-projection (w_ld,
// rounded to bf16 into x_lat after the top-k).
// (fuse: one token in bf16 mode, the top-k launch also writes the dispatch
// and the activation operand; moe_permute is then skipped)
// one token: the router row GEMV's CTAs, and its stage slots for the rows it
// carries in moe_layer (router, sigmoid gate, latent down); the sigmoid-gate
// row alone uses the same slots, so that it has the same bits either way
int router_ctas(const DeviceState& ds) { return std::max(1, ds.num_sms * kLayerRouterEighths / 8); }
int router_slots(const Plan& p, const DeviceState& ds) {
  const long units = (long)p.E + 1 + p.L;
  return rows_slots(units, (int)std::min<long>(units, router_ctas(ds)), false);
}

moe_status do_route(const Plan& p, const DeviceState& ds, const uint16_t* x, const uint16_t* wr,
                    const float* e_bias, int32_t* idx, float* w, float* logits, void* ws,
                    cudaStream_t st, const uint16_t* w_sgate = nullptr,
                    const uint16_t* w_ld = nullptr, uint16_t* x_lat = nullptr,
                    const moe::TopkFuse* fuse = nullptr) {
  moe::TopkFuse tf = fuse ? *fuse : moe::TopkFuse{};
  moe::RouteCfg rc = p.rc;
  rc.bias = e_bias;
  float* part = at<float>(ws, p.off_router);
  moe_status s;
  if (p.rows) {
    moe::RowsArgs r;
    memset(&r, 0, sizeof(r));
    r.w[0] = wr; r.rows[0] = p.E; r.out[0] = part;
    int seg = 1;
    if (w_sgate) { r.w[seg] = w_sgate; r.rows[seg] = 1; r.out[seg] = at<float>(ws, p.off_gl); ++seg; }
    if (w_ld) { r.w[seg] = w_ld; r.rows[seg] = p.L; r.out[seg] = at<float>(ws, p.off_ld); }
    r.x = x; r.K = p.H; r.status = at<int32_t>(ws, p.off_status);
    if (tf.x16 && p.H == tf.W) {
      // one token: the router launch writes the activation operand (its CTAs
      // hold x already, and it runs before the shared expert loads HBM)
      r.x16 = tf.x16; r.xscale = tf.xscale;
      tf.x16 = nullptr;
    }
    // (the same share of the SMs and stage geometry in moe_route and
    // moe_layer, so that both give the same bits)
    if ((s = launch_rows(ds, r, false, false, router_ctas(ds), st, "router gemv", true,
                         router_slots(p, ds))) != MOE_OK)
      return s;
    launch_pdl(moe::k_topk, dim3(p.T), dim3(moe::kTopkThreads), 0, st, (const float*)part, 1, p.T, p.E,
               p.E, p.k, idx, w, logits, (float*)nullptr, tf, rc);
    if ((s = launched("top-k")) != MOE_OK) return s;
    return w_ld ? round_latent(p, at<float>(ws, p.off_ld), p.L, x_lat, st) : MOE_OK;
  }
  // many tokens: the router rows, then the sigmoid-gate row (column E of the
  // partial sums) and the latent rows as further segments of the tcgen05 GEMM
  moe::Bf16GemmArgs g;
  memset(&g, 0, sizeof(g));
  if ((s = bf16_map(&g.map_a[0], wr, p.E, p.H, "router weights")) != MOE_OK ||
      (s = bf16_map(&g.map_b0, x, p.T, p.H, "tokens", p.Nt)) != MOE_OK ||
      (w_sgate && (s = bf16_map(&g.map_a[1], w_sgate, 1, p.H, "sigmoid-gate weights")) != MOE_OK) ||
      (w_ld && (s = bf16_map(&g.map_a[2], w_ld, p.L, p.H, "latent down weights")) != MOE_OK))
    return s;
  const int lat_col = w_sgate ? p.E + 1 : p.E;
  const int ld = lat_col + (w_ld ? p.L : 0);
  g.out = part; g.status = at<int32_t>(ws, p.off_status);
  g.mode = moe::kBf16Plain; g.K = p.H; g.T = p.T; g.S = p.S_router; g.passes = 1; g.N = p.Nt;
  g.seg_rows[0] = p.E; g.seg_rows[1] = w_sgate ? 1 : 0; g.seg_rows[2] = w_ld ? p.L : 0; g.ld = ld;
  if ((s = launch_bf16_gemm(ds, g, st, "router gemm (tcgen05)")) != MOE_OK) return s;
  launch_pdl(moe::k_topk, dim3(p.T), dim3(moe::kTopkThreads), 0, st, (const float*)part, p.S_router, p.T, p.E,
             ld, p.k, idx, w, logits, w_sgate ? at<float>(ws, p.off_gl) : (float*)nullptr, tf, rc);
  if ((s = launched("top-k")) != MOE_OK) return s;
  return w_ld ? round_latent(p, part + lat_col, ld, x_lat, st) : MOE_OK;
}

// Shared expert on the tcgen05 GEMM, first half: h = silu(Wg x) * (Wu x) as
// a bf16 hi/lo pair and the sigmoid-gate logit. Many tokens: SwiGLU in the
// gate/up epilogue, the sigmoid-gate row on the GEMV. Few tokens: the gate,
// up and sigmoid-gate rows as three segments of one split-K GEMM, SwiGLU in
// the finaliser.
moe_status do_shared_up(const Plan& p, const DeviceState& ds, const uint16_t* x, const uint16_t* w_sgate,
                        const uint16_t* ws_gate, const uint16_t* ws_up, void* ws, cudaStream_t st,
                        bool sgate_done = false, int max_ctas = 0) {
  if (p.rows) {
    moe::RowsArgs r;
    memset(&r, 0, sizeof(r));
    r.w[0] = ws_gate; r.w[1] = ws_up; r.rows[0] = p.Is; r.out[0] = at<float>(ws, p.off_hsb);
    r.x = x; r.K = p.H; r.status = at<int32_t>(ws, p.off_status);
    moe_status s = launch_rows(ds, r, true, false, max_ctas ? max_ctas : ds.num_sms, st,
                               "shared gate/up gemv", false);
    if (s != MOE_OK || sgate_done) return s;
    moe::RowsArgs g;
    memset(&g, 0, sizeof(g));
    g.w[0] = w_sgate; g.rows[0] = 1; g.out[0] = at<float>(ws, p.off_gl);
    g.x = x; g.K = p.H; g.status = r.status;
    return launch_rows(ds, g, false, false, 1, st, "shared gate gemv", true, router_slots(p, ds));
  }
  uint16_t* h_hi = at<uint16_t>(ws, p.off_hsb);
  uint16_t* h_lo = h_hi + (size_t)p.T * p.Is;
  int32_t* status = at<int32_t>(ws, p.off_status);
  moe_status s;
  moe::Bf16GemmArgs g;
  memset(&g, 0, sizeof(g));
  if ((s = bf16_map(&g.map_a[0], ws_gate, p.Is, p.H, "shared gate weights")) != MOE_OK ||
      (s = bf16_map(&g.map_a[1], ws_up, p.Is, p.H, "shared up weights")) != MOE_OK ||
      (s = bf16_map(&g.map_b0, x, p.T, p.H, "tokens", p.Nt)) != MOE_OK)
    return s;
  g.status = status;
  g.K = p.H; g.T = p.T; g.passes = 1; g.N = p.Nt;
  if (p.swiglu_tc) {
    g.mode = moe::kBf16SwiGLU; g.S = 1;
    g.seg_rows[0] = p.Is;
    g.h_hi = h_hi; g.h_lo = h_lo;
    if ((s = launch_bf16_gemm(ds, g, st, "shared gate/up gemm (tcgen05)", false)) != MOE_OK) return s;
    // the sigmoid-gate row: with the router rows in moe_layer; else alone on
    // the same GEMM geometry (tile, splits, K order) and summed in the same
    // order, so that both give the same bits (partials in the router region)
    if (!sgate_done) {
      moe::Bf16GemmArgs q;
      memset(&q, 0, sizeof(q));
      if ((s = bf16_map(&q.map_a[0], w_sgate, 1, p.H, "sigmoid-gate weights")) != MOE_OK ||
          (s = bf16_map(&q.map_b0, x, p.T, p.H, "tokens", p.Nt)) != MOE_OK)
        return s;
      float* part = at<float>(ws, p.off_router);
      q.out = part; q.status = status;
      q.mode = moe::kBf16Plain; q.K = p.H; q.T = p.T; q.S = p.S_router; q.passes = 1; q.N = p.Nt;
      q.seg_rows[0] = 1; q.ld = 1;
      if ((s = launch_bf16_gemm(ds, q, st, "sigmoid-gate gemm (tcgen05)")) != MOE_OK) return s;
      launch_pdl(moe::k_sum_column, dim3((p.T + moe::kFinThreads - 1) / moe::kFinThreads), dim3(moe::kFinThreads),
                 0, st, (const float*)part, p.S_router, p.T, 1, 0, at<float>(ws, p.off_gl));
      if ((s = launched("sigmoid-gate sum")) != MOE_OK) return s;
    }
  } else {
    if ((s = bf16_map(&g.map_a[2], w_sgate, 1, p.H, "shared sigmoid-gate weights")) != MOE_OK) return s;
    float* sgu = at<float>(ws, p.off_sgu);
    g.mode = moe::kBf16Plain; g.S = p.S_sgu;
    g.seg_rows[0] = p.Is; g.seg_rows[1] = p.Is; g.seg_rows[2] = 1; g.ld = 2 * p.Is + 1;
    g.out = sgu;
    if ((s = launch_bf16_gemm(ds, g, st, "shared gate/up gemm (tcgen05)", false)) != MOE_OK) return s;
    launch_pdl(moe::k_shared_swiglu, dim3((p.Is + moe::kFinThreads - 1) / moe::kFinThreads, p.T),
               dim3(moe::kFinThreads), 0, st, (const float*)sgu,
               p.S_sgu, p.T, p.Is, h_hi, h_lo, at<float>(ws, p.off_gl));
    if ((s = launched("shared swiglu")) != MOE_OK) return s;
  }
  return MOE_OK;
}

// Shared expert, second half: the down GEMM over both halves of h (split-K
// partial sums for the combine).
// One token on the row GEMV and no latent projection: the shared down launch
// also finishes the combine (same order of operations as k_combine).
bool combine_in_shared_down(const Plan& p) { return p.rows && p.L == 0; }

// comb (combine_in_shared_down): y_perm, slot_row, topk_w of the routed
// experts and the layer output y
moe_status do_shared_down(const Plan& p, const DeviceState& ds, const uint16_t* ws_down, void* ws,
                          cudaStream_t st, int max_ctas = 0, const float* y_perm = nullptr,
                          const int32_t* slot_row = nullptr, const float* topk_w = nullptr,
                          float* y = nullptr) {
  if (p.rows) {
    moe::RowsArgs r;
    memset(&r, 0, sizeof(r));
    r.w[0] = ws_down; r.rows[0] = p.H; r.out[0] = at<float>(ws, p.off_sd);
    r.x = at<float>(ws, p.off_hsb); r.K = p.Is; r.status = at<int32_t>(ws, p.off_status);
    if (y && combine_in_shared_down(p)) {
      r.y = y; r.y_perm = y_perm; r.slot_row = slot_row; r.topk_w = topk_w;
      r.gate_logit = at<float>(ws, p.off_gl); r.k = p.k;
    }
    return launch_rows(ds, r, false, true, max_ctas ? max_ctas : ds.num_sms, st,
                       r.y ? "shared down gemv + combine" : "shared down gemv");
  }
  uint16_t* h_hi = at<uint16_t>(ws, p.off_hsb);
  uint16_t* h_lo = h_hi + (size_t)p.T * p.Is;
  moe_status s;
  moe::Bf16GemmArgs d;
  memset(&d, 0, sizeof(d));
  if ((s = bf16_map(&d.map_a[0], ws_down, p.H, p.Is, "shared down weights")) != MOE_OK ||
      (s = bf16_map(&d.map_b0, h_hi, p.T, p.Is, "shared h (hi)", p.Nt)) != MOE_OK ||
      (s = bf16_map(&d.map_b1, h_lo, p.T, p.Is, "shared h (lo)", p.Nt)) != MOE_OK)
    return s;
  d.out = at<float>(ws, p.off_sd); d.status = at<int32_t>(ws, p.off_status);
  d.mode = moe::kBf16Plain; d.K = p.Is; d.T = p.T; d.S = p.S_sd; d.passes = 2; d.N = p.Nt;
  d.seg_rows[0] = p.H; d.ld = p.H;
  return launch_bf16_gemm(ds, d, st, "shared down gemm (tcgen05)");
}

// MXFP4 activations: gate/up (+ SwiGLU, h quantised to MXFP4) and down on the
// tensor cores, one persistent CTA per SM each; the tile list and the token
// operand come from moe_permute (inside x_op), weight scales are tiled.
// Make `st` wait for `ev` (NULL: nothing) before the next launch.
moe_status join_before(cudaEvent_t ev, cudaStream_t st) {
  if (!ev) return MOE_OK;
  const cudaError_t e = cudaStreamWaitEvent(st, ev, 0);
  return e == cudaSuccess ? MOE_OK : fail(MOE_ERR_CUDA, "join: %s", cudaGetErrorString(e));
}

// `join` (or NULL): an event the down projection waits for (moe_layer joins
// the shared expert's stream there, well after that work is done, so that the
// join never delays a launch)
moe_status do_expert_ffn_mxf4(const Plan& p, const DeviceState& ds, const void* x_op,
                              const uint8_t* wg_q, const uint8_t* wg_s, const uint8_t* wu_q,
                              const uint8_t* wu_s, const uint8_t* wd_q, const uint8_t* wd_s,
                              float* y_perm, void* ws, cudaStream_t st, cudaEvent_t join = nullptr) {
  void* xop = const_cast<void*>(x_op);
  const int4* tiles = at<int4>(xop, p.xop_tiles_off);
  const int32_t* n_tiles = at<int32_t>(xop, p.xop_ntiles_off);
  uint8_t* hq = at<uint8_t>(ws, p.off_h16);
  uint8_t* hs = at<uint8_t>(ws, p.off_hsf);
  moe_status s;
  moe::Mxf4GemmArgs g;
  memset(&g, 0, sizeof(g));
  if ((s = code_map(&g.map_a0, wg_q, (uint64_t)p.E * p.I, p.W / 2, 128, "gate weights")) != MOE_OK ||
      (s = code_map(&g.map_a1, wu_q, (uint64_t)p.E * p.I, p.W / 2, 128, "up weights")) != MOE_OK ||
      (s = code_map(&g.map_b, static_cast<const uint8_t*>(x_op), (uint64_t)p.R, p.W / 2,
                    moe::kTileRows, "token codes")) != MOE_OK)
    return s;
  g.sa0 = wg_s; g.sa1 = wu_s;
  g.bs = at<uint8_t>(xop, p.xop_scale_off);
  g.tiles = tiles; g.n_tiles = n_tiles;
  g.hq = hq; g.hs = hs;
  g.status = at<int32_t>(ws, p.off_status);
  g.K = p.W; g.M = p.I;
  const int threads = moe::mxf4_gemm_threads();
  moe::k_mxf4_gemm<true><<<ds.num_sms, threads, moe::mxf4_gemm_smem_bytes(true), st>>>(g);
  if ((s = launched("expert gate/up (tcgen05)")) != MOE_OK) return s;
  moe::Mxf4GemmArgs d;
  memset(&d, 0, sizeof(d));
  if ((s = code_map(&d.map_a0, wd_q, (uint64_t)p.E * p.W, p.I / 2, 128, "down weights")) != MOE_OK ||
      (s = code_map(&d.map_b, hq, (uint64_t)p.R, p.I / 2, moe::kTileRows, "h codes")) != MOE_OK)
    return s;
  d.map_a1 = d.map_a0;
  d.sa0 = wd_s; d.sa1 = wd_s;
  d.bs = hs;
  d.tiles = tiles; d.n_tiles = n_tiles;
  d.y = y_perm;
  d.status = g.status;
  d.K = p.I; d.M = p.W;
  if ((s = join_before(join, st)) != MOE_OK) return s;
  moe::k_mxf4_gemm<false><<<ds.num_sms, threads, moe::mxf4_gemm_smem_bytes(false), st>>>(d);
  return launched("expert down (tcgen05)");
}

moe_status do_expert_ffn(const Plan& p, const DeviceState& ds, const void* x_op,
                         const int32_t* offsets, const int32_t* expert_list,
                         const int32_t* row_token, const uint8_t* wg_q, const uint8_t* wg_s,
                         const uint8_t* wu_q, const uint8_t* wu_s, const uint8_t* wd_q,
                         const uint8_t* wd_s, float* y_perm, void* ws, cudaStream_t st,
                         cudaEvent_t join = nullptr, const void* l2_next = nullptr,
                         size_t l2_next_bytes = 0) {
  if (p.mode == MOE_ACT_MXFP4)
    return do_expert_ffn_mxf4(p, ds, x_op, wg_q, wg_s, wu_q, wu_s, wd_q, wd_s, y_perm, ws, st, join);
  const long ny = p.E < p.R ? p.E : p.R;     // most experts that can be active
  moe::GateUpArgs g;
  g.x16 = static_cast<const __half*>(x_op);
  g.xscale = reinterpret_cast<const float*>(static_cast<const char*>(x_op) + p.xop_scale_off);
  g.offsets = offsets; g.expert_list = expert_list; g.row_token = row_token;
  g.wg_q = wg_q; g.wg_s = wg_s; g.wu_q = wu_q; g.wu_s = wu_s;
  g.h16 = at<__half>(ws, p.off_h16);
  g.hscale = at<float>(ws, p.off_hscale);
  g.W = p.W; g.I = p.I; g.E = p.E; g.R = p.R;
  const size_t smem = moe::gemv_mxfp4_smem_bytes();
  const long slots = (long)ds.num_sms * ds.gemv_ctas_per_sm;
  // single-token experts on the CUDA cores
  const bool fma = fma_path(p);
  moe::FmaArgs f;
  f.x16 = g.x16; f.xscale = g.xscale; f.h32 = at<float>(ws, p.off_h32);
  f.offsets = offsets; f.expert_list = expert_list; f.row_token = row_token;
  f.wg_q = wg_q; f.wg_s = wg_s; f.wu_q = wu_q; f.wu_s = wu_s; f.wd_q = wd_q; f.wd_s = wd_s;
  f.y_perm = y_perm;
  f.l2_next = l2_next && l2_next_bytes >= 16 && aligned16(l2_next) ? l2_next : nullptr;
  f.l2_next_bytes = f.l2_next ? (uint64_t)(l2_next_bytes & ~(size_t)15) : 0;
  f.status = at<int32_t>(ws, p.off_status);
  f.sync = at<int32_t>(ws, p.off_status) + kSyncWord;
  f.W = p.W; f.I = p.I; f.E = p.E; f.R = p.R;
  g.min_tokens = fma ? 2 : 1;
  if (fma && routed1_path(p)) {
    // one token: every active expert has exactly one row; both projections in one launch
    moe_status s = join_before(join, st);
    return s != MOE_OK ? s : launch_routed1(ds, p, f, st);
  }
  // one token: its k experts are distinct, so every active expert has exactly
  // one token and the tensor-core kernels would find no work
  const bool mma = !(fma && p.T == 1);
  moe_status s = MOE_OK;
  if (fma && (s = launch_fma<true>(ds, f, st)) != MOE_OK) return s;
  // experts with 2+ tokens: CTA-wide TMA rings (W and I multiples of 512:
  // whole 512-element slices, scale rows a multiple of 16 bytes) with h as
  // fp32 rows converted to f16 with one scale per row in between; else the
  // per-warp rings with h in f16 with one scale per 16-element group
  if (mma && p.W % 512 == 0 && p.I % 512 == 0) {
    moe::MmaGateUpArgs m;
    memset(&m, 0, sizeof(m));
    const uint64_t rows = (uint64_t)p.E * p.I;
    if ((s = code_map(&m.map_gq, wg_q, rows, p.W / 2, 64, "gate weights")) != MOE_OK ||
        (s = code_map(&m.map_uq, wu_q, rows, p.W / 2, 64, "up weights")) != MOE_OK ||
        (s = byte_map(&m.map_gs, wg_s, rows, p.W / 32, 16, 64, "gate scales")) != MOE_OK ||
        (s = byte_map(&m.map_us, wu_s, rows, p.W / 32, 16, 64, "up scales")) != MOE_OK)
      return s;
    m.g = g;
    m.h32 = f.h32;
    m.status = at<int32_t>(ws, p.off_status);
    launch_pdl(moe::k_mma_gateup, dim3(ds.num_sms), dim3(32 * (moe::kMmaConsumers + 1)),
               moe::mma_gateup_smem_bytes(), st, m);
    if ((s = launched("expert gate/up (tensor cores, multi-token)")) != MOE_OK) return s;
    float* hrs = g.hscale;                               // [R] row scales in the group-scale region
    const int grid_h = (int)std::min<long>((p.R + 7) / 8, (long)ds.num_sms * 8);
    launch_pdl(moe::k_h_rowscale, dim3(grid_h), dim3(256), 0, st, (const float*)f.h32, offsets, p.E,
               p.R, p.I, g.min_tokens, g.h16, hrs);
    if ((s = launched("expert h row scales")) != MOE_OK) return s;
    if ((s = join_before(join, st)) != MOE_OK) return s;
    if (fma && (s = launch_fma<false>(ds, f, st)) != MOE_OK) return s;
    moe::MmaDownArgs d;
    memset(&d, 0, sizeof(d));
    const uint64_t drows = (uint64_t)p.E * p.W;
    if ((s = code_map(&d.map_dq, wd_q, drows, p.I / 2, 128, "down weights")) != MOE_OK ||
        (s = byte_map(&d.map_ds, wd_s, drows, p.I / 32, 16, 128, "down scales")) != MOE_OK)
      return s;
    d.h16 = g.h16; d.hrs = hrs; d.offsets = offsets; d.expert_list = expert_list;
    d.y_perm = y_perm; d.status = at<int32_t>(ws, p.off_status);
    d.W = p.W; d.I = p.I; d.E = p.E; d.R = p.R; d.min_tokens = g.min_tokens;
    launch_pdl(moe::k_mma_down, dim3(ds.num_sms), dim3(32 * (moe::kMmaConsumers + 1)),
               moe::mma_down_smem_bytes(), st, d);
    return launched("expert down (tensor cores, multi-token)");
  }
  const int grid_g = (int)std::min<long>(ny * (p.I / 16), slots);
  if (mma) {
    launch_pdl(moe::k_gateup_mxfp4, dim3(grid_g), dim3(32), smem, st, g);
    if ((s = launched("expert gate/up")) != MOE_OK) return s;
  }
  moe::DownArgs d;
  d.h16 = g.h16; d.hscale = g.hscale; d.offsets = offsets; d.expert_list = expert_list;
  d.wd_q = wd_q; d.wd_s = wd_s; d.y_perm = y_perm;
  d.W = p.W; d.I = p.I; d.E = p.E; d.R = p.R;
  d.min_tokens = g.min_tokens;
  if ((s = join_before(join, st)) != MOE_OK) return s;
  if (fma && (s = launch_fma<false>(ds, f, st)) != MOE_OK) return s;
  if (!mma) return MOE_OK;
  const int grid_d = (int)std::min<long>(ny * (p.W / 32), slots);
  launch_pdl(moe::k_down_mxfp4, dim3(grid_d), dim3(32), smem, st, d);
  return launched("expert down");
}

// The latent up-projection: W_lu [H, L] times the routed sum y_lat given as a
// bf16 pair (hi, lo), on the tcgen05 GEMM; split-K partials [S_lu, T, H].
moe_status do_latent_up(const Plan& p, const DeviceState& ds, const uint16_t* w_lat_up, void* ws,
                        cudaStream_t st) {
  uint16_t* y_hi = at<uint16_t>(ws, p.off_ylat);
  uint16_t* y_lo = y_hi + (size_t)p.T * p.L;
  moe_status s;
  moe::Bf16GemmArgs u;
  memset(&u, 0, sizeof(u));
  if ((s = bf16_map(&u.map_a[0], w_lat_up, p.H, p.L, "latent up weights")) != MOE_OK ||
      (s = bf16_map(&u.map_b0, y_hi, p.T, p.L, "latent sum (hi)", p.Nt)) != MOE_OK ||
      (s = bf16_map(&u.map_b1, y_lo, p.T, p.L, "latent sum (lo)", p.Nt)) != MOE_OK)
    return s;
  u.out = at<float>(ws, p.off_lu); u.status = at<int32_t>(ws, p.off_status);
  u.mode = moe::kBf16Plain; u.K = p.L; u.T = p.T; u.S = p.S_lu; u.passes = 2; u.N = p.Nt;
  u.seg_rows[0] = p.H; u.ld = p.H;
  return launch_bf16_gemm(ds, u, st, "latent up gemm (tcgen05)");
}

moe_status do_final(const Plan& p, const DeviceState& ds, const float* y_perm, const int32_t* slot_row,
                    const float* topk_w, const uint16_t* w_lat_up, float* y, void* ws, cudaStream_t st) {
  moe::CombineArgs c;
  memset(&c, 0, sizeof(c));
  c.slot_row = slot_row; c.topk_w = topk_w; c.k = p.k;
  c.gate_logit = at<float>(ws, p.off_gl);
  c.T = p.T;
  if (p.L) {
    // routed weighted sum at width L (as a bf16 pair), then the
    // up-projection, then + shared
    c.y_perm = y_perm;
    c.out_hi = at<uint16_t>(ws, p.off_ylat); c.out_lo = c.out_hi + (size_t)p.T * p.L;
    c.width = p.L;
    moe::k_combine<<<dim3((p.L / 4 + moe::kCombineThreads - 1) / moe::kCombineThreads, p.T),
                     moe::kCombineThreads, 0, st>>>(c);
    moe_status s = launched("latent combine");
    if (s != MOE_OK || (s = do_latent_up(p, ds, w_lat_up, ws, st)) != MOE_OK) return s;
    c.y_perm = nullptr; c.out_hi = c.out_lo = nullptr;
    c.add1 = at<float>(ws, p.off_lu); c.S1 = p.S_lu;
  } else {
    c.y_perm = y_perm;
  }
  c.add2 = at<float>(ws, p.off_sd); c.S2 = p.S_sd;
  c.out = y; c.width = p.H;
  moe::k_combine<<<dim3((p.H / 4 + moe::kCombineThreads - 1) / moe::kCombineThreads, p.T),
                   moe::kCombineThreads, 0, st>>>(c);
  return launched("combine");
}

// The latent down-projection alone: the same GEMM geometry and split order as
// when it rides along with the router rows, so that both give the same bits.
moe_status do_latent_down(const Plan& p, const DeviceState& ds, const uint16_t* x, const uint16_t* w_ld,
                          uint16_t* x_lat, void* ws, cudaStream_t st) {
  float* part = at<float>(ws, p.off_ld);
  moe_status s;
  if (p.rows) {
    moe::RowsArgs r;
    memset(&r, 0, sizeof(r));
    r.w[0] = w_ld; r.rows[0] = p.L; r.out[0] = part;
    r.x = x; r.K = p.H; r.status = at<int32_t>(ws, p.off_status);
    if ((s = launch_rows(ds, r, false, false, ds.num_sms, st, "latent down gemv")) != MOE_OK) return s;
  } else {
    moe::Bf16GemmArgs g;
    memset(&g, 0, sizeof(g));
    if ((s = bf16_map(&g.map_a[0], w_ld, p.L, p.H, "latent down weights")) != MOE_OK ||
        (s = bf16_map(&g.map_b0, x, p.T, p.H, "tokens", p.Nt)) != MOE_OK)
      return s;
    g.out = part; g.status = at<int32_t>(ws, p.off_status);
    g.mode = moe::kBf16Plain; g.K = p.H; g.T = p.T; g.S = p.S_ld; g.passes = 1; g.N = p.Nt;
    g.seg_rows[0] = p.L; g.ld = p.L;
    if ((s = launch_bf16_gemm(ds, g, st, "latent down gemm (tcgen05)")) != MOE_OK) return s;
  }
  return round_latent(p, part, p.L, x_lat, st);
}

}  // namespace

namespace moe {
// Record a status and its one-line reason for moe_last_error() (used by the
// entry points that live in other translation units).
moe_status record_error(moe_status s, const char* msg) { return fail(s, "%s", msg); }
}  // namespace moe

// ===========================================================================
// C ABI
// ===========================================================================
extern "C" {

const char* moe_status_string(moe_status s) {
  switch (s) {
    case MOE_OK: return "ok";
    case MOE_ERR_INVALID_ARG: return "invalid argument";
    case MOE_ERR_UNSUPPORTED_SHAPE: return "unsupported shape";
    case MOE_ERR_ALIGNMENT: return "pointer not 16-byte aligned";
    case MOE_ERR_WORKSPACE_TOO_SMALL: return "workspace too small";
    case MOE_ERR_CUDA: return "CUDA runtime error";
    case MOE_ERR_DEVICE_STATUS: return "device flagged a data error";
  }
  return "unknown status";
}

const char* moe_last_error(void) { return g_err; }

size_t moe_workspace_size(const moe_dims* dims) {
  Plan p;
  return make_plan(dims, p) == MOE_OK ? p.total : 0;
}

size_t moe_x_op_size(const moe_dims* dims) {
  Plan p;
  return make_plan(dims, p) == MOE_OK ? p.xop_bytes : 0;
}

moe_status moe_mxf4_layout_of(const moe_dims* dims, moe_mxf4_layout* out) {
  Plan p;
  moe_status s = make_plan(dims, p);
  if (s != MOE_OK) return s;
  if (!out) return fail(MOE_ERR_INVALID_ARG, "out is NULL");
  if (p.mode != MOE_ACT_MXFP4)
    return fail(MOE_ERR_UNSUPPORTED_SHAPE, "the layout applies to MOE_ACT_MXFP4 only");
  out->x_codes = 0;
  out->x_scales = p.xop_scale_off;
  out->tiles = p.xop_tiles_off;
  out->tile_base = p.xop_tbase_off;
  out->n_tiles = p.xop_ntiles_off;
  out->h_codes = p.off_h16;
  out->h_scales = p.off_hsf;
  out->max_tiles = p.max_tiles;
  out->tile_rows = moe::kTileRows;
  return MOE_OK;
}

moe_status moe_tile_scales(const uint8_t* src, int64_t rows, int32_t K, uint8_t* dst, void* stream) {
  if (!src || !dst) return fail(MOE_ERR_INVALID_ARG, "src or dst is NULL");
  if (!aligned16(src) || !aligned16(dst)) return fail(MOE_ERR_ALIGNMENT, "src or dst not 16-byte aligned");
  if (rows < 128 || rows % 128 != 0 || K < 128 || K % 128 != 0 || K > (1 << 16) ||
      rows > (1L << 31))
    return fail(MOE_ERR_UNSUPPORTED_SHAPE, "rows=%lld, K=%d: rows and K must be multiples of 128",
                (long long)rows, K);
  const long n = rows * (K / 128);
  const int blocks = (int)std::min<long>((n + 255) / 256, 148L * 16);
  moe::k_tile_scales<<<blocks, 256, 0, (cudaStream_t)stream>>>(src, rows, K, dst);
  return launched("tile scales");
}

moe_status moe_workspace_init(const moe_dims* dims, void* ws, size_t ws_bytes, void* stream) {
  Plan p;
  moe_status s = make_plan(dims, p);
  if (s != MOE_OK) return s;
  if ((s = check_ws(p, ws, ws_bytes)) != MOE_OK) return s;
  const cudaError_t e = cudaMemsetAsync(at<char>(ws, p.off_status), 0, 256, (cudaStream_t)stream);
  if (e != cudaSuccess) return fail(MOE_ERR_CUDA, "status clear: %s", cudaGetErrorString(e));
  return MOE_OK;
}

moe_status moe_device_status(const void* ws, int32_t* host_status, void* stream) {
  if (!ws || !host_status) return fail(MOE_ERR_INVALID_ARG, "ws or host_status is NULL");
  int32_t v = 0;
  cudaError_t e = cudaMemcpyAsync(&v, ws, sizeof(v), cudaMemcpyDeviceToHost, (cudaStream_t)stream);
  if (e == cudaSuccess) e = cudaStreamSynchronize((cudaStream_t)stream);
  if (e != cudaSuccess) return fail(MOE_ERR_CUDA, "status read: %s", cudaGetErrorString(e));
  *host_status = v;
  return v ? fail(MOE_ERR_DEVICE_STATUS, "device status word 0x%x", v) : MOE_OK;
}

moe_status moe_route(const moe_dims* dims, const uint16_t* x, const uint16_t* w_router,
                     int32_t* topk_idx, float* topk_w, float* logits, void* ws, size_t ws_bytes,
                     void* stream) {
  Plan p;
  moe_status s = make_plan(dims, p);
  if (s != MOE_OK) return s;
  CHECK_PTR(x); CHECK_PTR(w_router); CHECK_PTR(topk_idx); CHECK_PTR(topk_w);
  if (logits && !aligned16(logits)) return fail(MOE_ERR_ALIGNMENT, "logits not 16-byte aligned");
  if ((s = check_ws(p, ws, ws_bytes)) != MOE_OK) return s;
  DeviceState* ds;
  if ((s = device_state(&ds)) != MOE_OK) return s;
  return do_route(p, *ds, x, w_router, nullptr, topk_idx, topk_w, logits, ws, (cudaStream_t)stream);
}

moe_status moe_route_biased(const moe_dims* dims, const uint16_t* x, const uint16_t* w_router,
                            const float* e_bias, int32_t* topk_idx, float* topk_w, float* logits,
                            void* ws, size_t ws_bytes, void* stream) {
  Plan p;
  moe_status s = make_plan(dims, p);
  if (s != MOE_OK) return s;
  CHECK_PTR(x); CHECK_PTR(w_router); CHECK_PTR(topk_idx); CHECK_PTR(topk_w);
  if (e_bias && !aligned16(e_bias)) return fail(MOE_ERR_ALIGNMENT, "e_bias not 16-byte aligned");
  if (logits && !aligned16(logits)) return fail(MOE_ERR_ALIGNMENT, "logits not 16-byte aligned");
  if ((s = check_ws(p, ws, ws_bytes)) != MOE_OK) return s;
  DeviceState* ds;
  if ((s = device_state(&ds)) != MOE_OK) return s;
  return do_route(p, *ds, x, w_router, e_bias, topk_idx, topk_w, logits, ws, (cudaStream_t)stream);
}

moe_status moe_permute(const moe_dims* dims, const int32_t* topk_idx, const uint16_t* x_in,
                       int32_t* counts, int32_t* offsets, int32_t* expert_list, int32_t* row_token,
                       int32_t* row_slot, int32_t* slot_row, void* x_op, void* ws, size_t ws_bytes,
                       void* stream) {
  Plan p;
  moe_status s = make_plan(dims, p);
  if (s != MOE_OK) return s;
  CHECK_PTR(topk_idx); CHECK_PTR(x_in); CHECK_PTR(counts); CHECK_PTR(offsets);
  CHECK_PTR(expert_list); CHECK_PTR(row_token); CHECK_PTR(row_slot); CHECK_PTR(slot_row); CHECK_PTR(x_op);
  if ((s = check_ws(p, ws, ws_bytes)) != MOE_OK) return s;
  DeviceState* ds;
  if ((s = device_state(&ds)) != MOE_OK) return s;
  return do_permute(p, topk_idx, x_in, counts, offsets, expert_list, row_token, row_slot, slot_row,
                    x_op, ws, (cudaStream_t)stream);
}

moe_status moe_expert_ffn(const moe_dims* dims, const void* x_op, const int32_t* offsets,
                          const int32_t* expert_list, const int32_t* row_token,
                          const uint8_t* wg_q, const uint8_t* wg_s,
                          const uint8_t* wu_q, const uint8_t* wu_s, const uint8_t* wd_q,
                          const uint8_t* wd_s, float* y_perm, void* ws, size_t ws_bytes,
                          void* stream) {
  Plan p;
  moe_status s = make_plan(dims, p);
  if (s != MOE_OK) return s;
  CHECK_PTR(x_op); CHECK_PTR(offsets); CHECK_PTR(expert_list); CHECK_PTR(row_token);
  CHECK_PTR(wg_q); CHECK_PTR(wg_s); CHECK_PTR(wu_q); CHECK_PTR(wu_s); CHECK_PTR(wd_q); CHECK_PTR(wd_s);
  CHECK_PTR(y_perm);
  if ((s = check_ws(p, ws, ws_bytes)) != MOE_OK) return s;
  DeviceState* ds;
  if ((s = device_state(&ds)) != MOE_OK) return s;
  return do_expert_ffn(p, *ds, x_op, offsets, expert_list, row_token, wg_q, wg_s, wu_q, wu_s, wd_q,
                       wd_s, y_perm, ws, (cudaStream_t)stream);
}

// ---------------------------------------------------------------------------
// Routed experts streamed from host memory through an LRU cache of expert
// slots in device memory (rabbit README: routed experts stay off the
// accelerator and are fetched when needed through an LRU cache per layer; its
// feature list: per-expert early drain, an expert's matmul starts as soon as
// its own bytes have arrived).
// ---------------------------------------------------------------------------
}  // extern "C"

struct moe_expert_cache {
  int dev = 0;
  int32_t slots = 0;
  int E = 0, I = 0, W = 0;
  uint8_t* base = nullptr;              // slot 0; slot s at base + s * slot_bytes
  size_t slot_bytes = 0;
  size_t off[6] = {};                   // wg_q, wg_s, wu_q, wu_s, wd_q, wd_s inside a slot
  size_t len[6] = {};
  int32_t* one_list = nullptr;          // {1, 0}: the expert list of a one-expert problem
  cudaStream_t copy = nullptr;          // the copy engine's stream
  std::vector<int32_t> slot_expert;     // expert held by each slot (-1: none)
  std::vector<int64_t> slot_used;       // last call that used each slot (LRU order)
  std::vector<int32_t> expert_slot;     // slot of each expert (-1: not cached)
  std::vector<cudaEvent_t> loaded;      // a slot's copy has landed
  std::vector<cudaEvent_t> released;    // the last launch reading a slot has run
  int64_t calls = 0, hits = 0, misses = 0, bytes = 0;
  std::mutex mu;
};

namespace {

// Byte layout of one slot: the six arrays of one expert, each at a 256-byte
// boundary; the whole slot a multiple of 256 bytes.
size_t cache_layout(int I, int W, size_t (&off)[6], size_t (&len)[6]) {
  const size_t gq = (size_t)I * W / 2, gs = (size_t)I * W / 32;
  const size_t l[6] = {gq, gs, gq, gs, gq, gs};   // down is [W, I]: the same sizes
  size_t o = 0;
  for (int i = 0; i < 6; ++i) {
    off[i] = o;
    len[i] = l[i];
    o = align_up(o + l[i], 256);
  }
  return o;
}

const int32_t kOneList[2] = {1, 0};

}  // namespace

extern "C" {

size_t moe_expert_cache_bytes(const moe_dims* dims, int32_t slots) {
  Plan p;
  if (make_plan(dims, p) != MOE_OK || slots < 1) return 0;
  size_t off[6], len[6];
  return 256 + (size_t)slots * cache_layout(p.I, p.W, off, len);
}

moe_status moe_expert_cache_create(const moe_dims* dims, int32_t slots, void* dev_mem, size_t dev_bytes,
                                   moe_expert_cache** out) {
  Plan p;
  moe_status s = make_plan(dims, p);
  if (s != MOE_OK) return s;
  if (!out) return fail(MOE_ERR_INVALID_ARG, "out is NULL");
  *out = nullptr;
  if (p.mode != MOE_ACT_BF16)
    return fail(MOE_ERR_UNSUPPORTED_SHAPE, "expert streaming serves MOE_ACT_BF16 (decode) layers");
  if (slots < 1 || slots > 65536) return fail(MOE_ERR_UNSUPPORTED_SHAPE, "slots=%d outside [1, 65536]", slots);
  CHECK_PTR(dev_mem);
  if (((uintptr_t)dev_mem & 255u) != 0) return fail(MOE_ERR_ALIGNMENT, "dev_mem not 256-byte aligned");
  if (dev_bytes < moe_expert_cache_bytes(dims, slots))
    return fail(MOE_ERR_WORKSPACE_TOO_SMALL, "dev_mem %zu bytes < %zu needed", dev_bytes,
                moe_expert_cache_bytes(dims, slots));
  moe_expert_cache* c = new moe_expert_cache;
  cudaGetDevice(&c->dev);
  c->slots = slots;
  c->E = p.E; c->I = p.I; c->W = p.W;
  c->one_list = static_cast<int32_t*>(dev_mem);
  c->base = static_cast<uint8_t*>(dev_mem) + 256;
  c->slot_bytes = cache_layout(p.I, p.W, c->off, c->len);
  c->slot_expert.assign(slots, -1);
  c->slot_used.assign(slots, -1);
  c->expert_slot.assign(p.E, -1);
  cudaError_t e = cudaStreamCreateWithFlags(&c->copy, cudaStreamNonBlocking);
  c->loaded.assign(slots, nullptr);
  c->released.assign(slots, nullptr);
  for (int i = 0; i < slots && e == cudaSuccess; ++i) {
    e = cudaEventCreateWithFlags(&c->loaded[i], cudaEventDisableTiming);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&c->released[i], cudaEventDisableTiming);
  }
  if (e == cudaSuccess)
    e = cudaMemcpyAsync(c->one_list, kOneList, sizeof(kOneList), cudaMemcpyHostToDevice, c->copy);
  if (e == cudaSuccess) e = cudaStreamSynchronize(c->copy);
  if (e != cudaSuccess) {
    moe_expert_cache_destroy(c);
    return fail(MOE_ERR_CUDA, "expert cache setup: %s", cudaGetErrorString(e));
  }
  *out = c;
  return MOE_OK;
}

moe_status moe_expert_cache_destroy(moe_expert_cache* c) {
  if (!c) return MOE_OK;
  if (c->copy) cudaStreamSynchronize(c->copy);
  for (cudaEvent_t ev : c->loaded)
    if (ev) cudaEventDestroy(ev);
  for (cudaEvent_t ev : c->released)
    if (ev) cudaEventDestroy(ev);
  if (c->copy) cudaStreamDestroy(c->copy);
  delete c;
  return MOE_OK;
}

moe_status moe_expert_cache_stats(const moe_expert_cache* c, int64_t* hits, int64_t* misses,
                                  int64_t* bytes_copied) {
  if (!c || !hits || !misses || !bytes_copied) return fail(MOE_ERR_INVALID_ARG, "NULL argument");
  moe_expert_cache* m = const_cast<moe_expert_cache*>(c);
  std::lock_guard<std::mutex> lk(m->mu);
  *hits = c->hits;
  *misses = c->misses;
  *bytes_copied = c->bytes;
  return MOE_OK;
}

moe_status moe_expert_ffn_streamed(moe_expert_cache* c, const moe_dims* dims, const int32_t* active,
                                   int32_t n_active, const void* x_op, const int32_t* offsets,
                                   const int32_t* row_token, const uint8_t* const* host_experts,
                                   float* y_perm, void* ws, size_t ws_bytes, void* stream) {
  Plan p;
  moe_status s = make_plan(dims, p);
  if (s != MOE_OK) return s;
  if (!c) return fail(MOE_ERR_INVALID_ARG, "cache is NULL");
  if (p.E != c->E || p.I != c->I || p.W != c->W || p.mode != MOE_ACT_BF16)
    return fail(MOE_ERR_INVALID_ARG, "dims do not match the cache");
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev != c->dev)
    return fail(MOE_ERR_INVALID_ARG, "the cache belongs to device %d", c->dev);
  CHECK_PTR(x_op); CHECK_PTR(offsets); CHECK_PTR(row_token); CHECK_PTR(host_experts); CHECK_PTR(y_perm);
  if (n_active < 0 || n_active > p.E) return fail(MOE_ERR_INVALID_ARG, "n_active=%d outside [0, E]", n_active);
  if (n_active > 0) CHECK_PTR(active);
  if (n_active > c->slots)
    return fail(MOE_ERR_UNSUPPORTED_SHAPE, "%d active experts > %d cache slots", n_active, c->slots);
  for (int i = 0; i < n_active; ++i) {
    if (active[i] < 0 || active[i] >= p.E) return fail(MOE_ERR_INVALID_ARG, "active[%d]=%d outside [0, E)", i, active[i]);
    for (int j = 0; j < i; ++j)
      if (active[j] == active[i]) return fail(MOE_ERR_INVALID_ARG, "expert %d listed twice", active[i]);
    for (int a = 0; a < 6; ++a)
      if (!host_experts[(size_t)active[i] * 6 + a])
        return fail(MOE_ERR_INVALID_ARG, "host_experts[%d][%d] is NULL", active[i], a);
  }
  if ((s = check_ws(p, ws, ws_bytes)) != MOE_OK) return s;
  DeviceState* ds;
  if ((s = device_state(&ds)) != MOE_OK) return s;
  // each expert runs as a one-expert problem: offsets shifted to its pair of
  // entries, the expert list {1, 0}, the weights of its slot (extent E = 1);
  // the workspace layout stays the full plan's (rows are global row ids)
  Plan p1 = p;
  p1.E = 1;
  const cudaStream_t st = (cudaStream_t)stream;
  std::lock_guard<std::mutex> lk(c->mu);
  const int64_t call = ++c->calls;
  // 1) slots: hits keep theirs; misses take the least recently used slot
  //    that this call does not use, and are copied in list order
  std::vector<int32_t> slot_of(n_active, -1);
  std::vector<char> miss(n_active, 0);
  for (int i = 0; i < n_active; ++i) {
    const int e = active[i];
    if (c->expert_slot[e] >= 0) {
      slot_of[i] = c->expert_slot[e];
      c->slot_used[slot_of[i]] = call;
      ++c->hits;
    }
  }
  cudaError_t err = cudaSuccess;
  for (int i = 0; i < n_active && err == cudaSuccess; ++i) {
    if (slot_of[i] >= 0) continue;
    int best = -1;
    for (int t = 0; t < c->slots; ++t)
      if (c->slot_used[t] != call && (best < 0 || c->slot_used[t] < c->slot_used[best])) best = t;
    const int e = active[i];
    if (c->slot_expert[best] >= 0) c->expert_slot[c->slot_expert[best]] = -1;
    c->slot_expert[best] = e;
    c->expert_slot[e] = best;
    c->slot_used[best] = call;
    slot_of[i] = best;
    miss[i] = 1;
    ++c->misses;
    // the copy overwrites the slot only after the last launch that read it
    uint8_t* dst = c->base + (size_t)best * c->slot_bytes;
    err = cudaStreamWaitEvent(c->copy, c->released[best], 0);
    for (int a = 0; a < 6 && err == cudaSuccess; ++a) {
      err = cudaMemcpyAsync(dst + c->off[a], host_experts[(size_t)e * 6 + a], c->len[a],
                            cudaMemcpyHostToDevice, c->copy);
      c->bytes += (int64_t)c->len[a];
    }
    if (err == cudaSuccess) err = cudaEventRecord(c->loaded[best], c->copy);
  }
  if (err != cudaSuccess) return fail(MOE_ERR_CUDA, "expert copy: %s", cudaGetErrorString(err));
  // 2) each expert's FFN as soon as its own bytes have landed (cache hits at
  //    once), in list order on the caller's stream
  for (int i = 0; i < n_active; ++i) {
    const int e = active[i];
    const int t = slot_of[i];
    uint8_t* b = c->base + (size_t)t * c->slot_bytes;
    if ((err = cudaStreamWaitEvent(st, c->loaded[t], 0)) != cudaSuccess)
      return fail(MOE_ERR_CUDA, "expert wait: %s", cudaGetErrorString(err));
    if ((s = do_expert_ffn(p1, *ds, x_op, offsets + e, c->one_list, row_token, b + c->off[0],
                           b + c->off[1], b + c->off[2], b + c->off[3], b + c->off[4], b + c->off[5],
                           y_perm, ws, st)) != MOE_OK)
      return s;
    if ((err = cudaEventRecord(c->released[t], st)) != cudaSuccess)
      return fail(MOE_ERR_CUDA, "expert release: %s", cudaGetErrorString(err));
  }
  return MOE_OK;
}

moe_status moe_combine(const moe_dims* dims, const float* y_perm, const int32_t* slot_row,
                       const float* topk_w, const uint16_t* x, const uint16_t* w_sgate,
                       const uint16_t* ws_gate, const uint16_t* ws_up, const uint16_t* ws_down,
                       const uint16_t* w_lat_up, float* y, void* ws, size_t ws_bytes, void* stream) {
  Plan p;
  moe_status s = make_plan(dims, p);
  if (s != MOE_OK) return s;
  CHECK_PTR(y_perm); CHECK_PTR(slot_row); CHECK_PTR(topk_w); CHECK_PTR(x); CHECK_PTR(w_sgate);
  CHECK_PTR(ws_gate); CHECK_PTR(ws_up); CHECK_PTR(ws_down); CHECK_PTR(y);
  if (p.L) { CHECK_PTR(w_lat_up); }
  else if (w_lat_up) return fail(MOE_ERR_INVALID_ARG, "w_lat_up given but L == 0");
  if ((s = check_ws(p, ws, ws_bytes)) != MOE_OK) return s;
  const cudaStream_t st = (cudaStream_t)stream;
  DeviceState* ds;
  if ((s = device_state(&ds)) != MOE_OK) return s;
  if ((s = do_shared_up(p, *ds, x, w_sgate, ws_gate, ws_up, ws, st)) != MOE_OK) return s;
  if (combine_in_shared_down(p))
    return do_shared_down(p, *ds, ws_down, ws, st, 0, y_perm, slot_row, topk_w, y);
  if ((s = do_shared_down(p, *ds, ws_down, ws, st)) != MOE_OK) return s;
  return do_final(p, *ds, y_perm, slot_row, topk_w, w_lat_up, y, ws, st);
}

moe_status moe_latent_down(const moe_dims* dims, const uint16_t* x, const uint16_t* w_lat_down,
                           uint16_t* x_lat, void* ws, size_t ws_bytes, void* stream) {
  Plan p;
  moe_status s = make_plan(dims, p);
  if (s != MOE_OK) return s;
  if (!p.L) return fail(MOE_ERR_INVALID_ARG, "moe_latent_down needs L > 0");
  CHECK_PTR(x); CHECK_PTR(w_lat_down); CHECK_PTR(x_lat);
  if ((s = check_ws(p, ws, ws_bytes)) != MOE_OK) return s;
  DeviceState* ds;
  if ((s = device_state(&ds)) != MOE_OK) return s;
  return do_latent_down(p, *ds, x, w_lat_down, x_lat, ws, (cudaStream_t)stream);
}

moe_status moe_layer(const moe_dims* dims, const moe_layer_args* a, void* ws, size_t ws_bytes,
                     void* stream) {
  Plan p;
  moe_status s = make_plan(dims, p);
  if (s != MOE_OK) return s;
  if (!a) return fail(MOE_ERR_INVALID_ARG, "args is NULL");
  CHECK_PTR(a->x); CHECK_PTR(a->w_router);
  CHECK_PTR(a->wg_q); CHECK_PTR(a->wg_s); CHECK_PTR(a->wu_q); CHECK_PTR(a->wu_s);
  CHECK_PTR(a->wd_q); CHECK_PTR(a->wd_s);
  CHECK_PTR(a->w_sgate); CHECK_PTR(a->ws_gate); CHECK_PTR(a->ws_up); CHECK_PTR(a->ws_down);
  CHECK_PTR(a->topk_idx); CHECK_PTR(a->topk_w); CHECK_PTR(a->counts); CHECK_PTR(a->offsets);
  CHECK_PTR(a->expert_list);
  CHECK_PTR(a->row_token); CHECK_PTR(a->row_slot); CHECK_PTR(a->slot_row); CHECK_PTR(a->x_op);
  CHECK_PTR(a->y_perm); CHECK_PTR(a->y);
  if (p.L) { CHECK_PTR(a->w_lat_down); CHECK_PTR(a->w_lat_up); CHECK_PTR(a->x_lat); }
  if ((s = check_ws(p, ws, ws_bytes)) != MOE_OK) return s;
  DeviceState* ds;
  if ((s = device_state(&ds)) != MOE_OK) return s;
  std::lock_guard<std::mutex> lk(g_mu);
  const cudaStream_t st = (cudaStream_t)stream;
  cudaError_t e = cudaEventRecord(ds->ev_fork, st);
  if (e != cudaSuccess) return fail(MOE_ERR_CUDA, "fork: %s", cudaGetErrorString(e));
  // main stream first: the router's CTAs are queued before the shared expert's
  // (one token or the SwiGLU-epilogue GEMM: the sigmoid-gate row rides along
  // with the router rows; the latent down-projection always does)
  const bool sgate_with_router = p.rows || p.swiglu_tc;
  // one token, bf16 activations, no latent projection: the top-k launch also
  // writes the dispatch and the activation operand (what moe_permute writes)
  const bool fused_dispatch = p.T == 1 && p.mode == MOE_ACT_BF16 && p.L == 0;
  moe::TopkFuse tf{};
  if (fused_dispatch) {
    tf.counts = a->counts; tf.offsets = a->offsets; tf.expert_list = a->expert_list;
    tf.row_token = a->row_token; tf.row_slot = a->row_slot; tf.slot_row = a->slot_row;
    tf.x = a->x; tf.W = p.W;
    tf.x16 = static_cast<__half*>(a->x_op); tf.xscale = at<float>(a->x_op, p.xop_scale_off);
  }
  if (a->e_bias && !aligned16(a->e_bias)) return fail(MOE_ERR_ALIGNMENT, "e_bias not 16-byte aligned");
  const int router_sms = p.rows ? router_ctas(*ds) : 0;
  if ((s = do_route(p, *ds, a->x, a->w_router, a->e_bias, a->topk_idx, a->topk_w, nullptr, ws, st,
                    sgate_with_router ? a->w_sgate : nullptr, p.L ? a->w_lat_down : nullptr,
                    a->x_lat, fused_dispatch ? &tf : nullptr)) != MOE_OK)
    return s;
  // side stream: the first half of the shared expert (it streams its weights
  // while the routing chain runs)
  if ((e = cudaStreamWaitEvent(ds->side, ds->ev_fork, 0)) != cudaSuccess)
    return fail(MOE_ERR_CUDA, "fork: %s", cudaGetErrorString(e));
  // (the row GEMV leaves a few SMs to the routing chain's small kernels)
  if ((s = do_shared_up(p, *ds, a->x, a->w_sgate, a->ws_gate, a->ws_up, ws, ds->side, sgate_with_router,
                        ds->num_sms - (router_sms ? router_sms : kRowsFreeSMs))) != MOE_OK)
    return s;
  if ((e = cudaEventRecord(ds->ev_shared, ds->side)) != cudaSuccess)
    return fail(MOE_ERR_CUDA, "event: %s", cudaGetErrorString(e));
  // main stream: dispatch, experts, combine
  if (!fused_dispatch &&
      (s = do_permute(p, a->topk_idx, p.L ? a->x_lat : a->x, a->counts, a->offsets, a->expert_list,
                      a->row_token, a->row_slot, a->slot_row, a->x_op, ws, st)) != MOE_OK)
    return s;
  // the routed experts follow the dispatch directly (their CTAs take the SMs
  // the shared expert's first half leaves); the shared stream joins before the
  // shared down projection, the first reader of its output (a joined launch
  // loses the early start of programmatic serialisation, a few microseconds,
  // wherever the join sits)
  // (one token: as the routed launch's chunks run out, its CTAs prefetch the
  // shared down weights, which the next launch reads, into L2)
  const bool sd_next = combine_in_shared_down(p);
  if ((s = do_expert_ffn(p, *ds, a->x_op, a->offsets, a->expert_list, a->row_token, a->wg_q,
                         a->wg_s, a->wu_q, a->wu_s, a->wd_q, a->wd_s, a->y_perm, ws, st, nullptr,
                         sd_next ? a->ws_down : nullptr, sd_next ? (size_t)p.H * p.Is * 2 : 0)) != MOE_OK)
    return s;
  if ((s = join_before(ds->ev_shared, st)) != MOE_OK) return s;
  if (combine_in_shared_down(p))
    return do_shared_down(p, *ds, a->ws_down, ws, st, 0, a->y_perm, a->slot_row, a->topk_w, a->y);
  if ((s = do_shared_down(p, *ds, a->ws_down, ws, st)) != MOE_OK) return s;
  return do_final(p, *ds, a->y_perm, a->slot_row, a->topk_w, a->w_lat_up, a->y, ws, st);
}

}  // extern "C"
