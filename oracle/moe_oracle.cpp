// Plain CPU oracle of the routed MXFP4 Mixture-of-Experts FFN layer, in C++17
// with float64 arithmetic.
//
// TEST INFRASTRUCTURE. Only tests/, __graft_entry__.smoke() and the CPU legs of
// bench.py (cpu_baseline and --impl reference) load this library, through the
// ctypes shim in oracle/__init__.py. The product (the CUDA library and its
// binding) never includes, links or calls it, and this file includes nothing
// of the product: the two share no code, header, table or helper.
//
// What it computes is the definition of the layer, written out step by step in
// the order of the pages, one function per step, so that a reader can check
// each against its source and the CUDA path can be compared stage by stage:
//
//   a1 router        logits[t, e] = sum_h x[t, h] Wr[e, h]
//   a2 top-k         softmax top-k, renormalised over the selected experts
//                    (variants: sigmoid scores with a selection bias, and
//                    group-limited selection)
//   a3 permute       (token, slot) pairs grouped by expert, ascending token
//   a4 quantise      OCP MXFP4 conversion of activations (MXFP4 mode only)
//   a5-a7 expert     y = Wd (silu(Wg x) * (Wu x)) on MXFP4 weights
//   a8 shared        sigmoid(w_sg . x) * Wsd (silu(Wsg x) * (Wsu x)), bf16
//   a9 combine       y[t] = sum_j w[t, j] Y[row of (t, j)] + s[t]
//   a10 latent       x_lat = bf16(W_ld x); routed experts at width L; W_lu
//
// Sources (the pages describe the layer by its shape only):
// * rabbit README (ferrumox/rabbit), model table, row "MoE routing": softmax
//   routing to 10 of 512 experts plus a gated shared expert (Qwen3.8-Max); "Stable LatentMoE"
//   (Kimi K3), "grouped routing" (Kimi Linear), "noaux_tc sigmoid" (GLM-5.2).
//   Row "native quantization read": routed experts in OCP MXFP4.
// * rabbit README, phase breakdown: the "expert matmul" phase is this layer's
//   routed expert products.
// * "Ran Moonshot's 2.8T-parameter Kimi K3 on a GPU-less mini-PC",
//   architecture paragraph: Stable LatentMoE, the routed experts compute in a
//   narrower latent width; 896 experts per layer.
// Number formats follow the OCP Microscaling Formats (MX) v1.0 specification,
// section 5 (MXFP4: E2M1 elements, one E8M0 scale per 32 elements). Every
// other choice is a reading, stated beside the function that takes it.
//
// Arithmetic rules: every value is decoded exactly into a double; every sum
// runs in one fixed order (ascending index) inside one thread, so results do
// not depend on the thread count. Threads split only independent outputs.
// Compiled without fast-math and with floating-point contraction off.
#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <functional>
#include <numeric>
#include <thread>
#include <vector>

namespace {

int g_threads = 0;   // 0: all hardware threads

int thread_count() {
  if (g_threads > 0) return g_threads;
  const unsigned h = std::thread::hardware_concurrency();
  return h ? (int)h : 1;
}

// Runs body(i) for i in [0, n), split into contiguous chunks over the threads.
// Each i is independent; no reduction crosses threads.
void parallel_for(int64_t n, const std::function<void(int64_t)>& body) {
  const int nt = (int)std::min<int64_t>(thread_count(), n);
  if (nt <= 1) {
    for (int64_t i = 0; i < n; ++i) body(i);
    return;
  }
  std::vector<std::thread> pool;
  pool.reserve(nt);
  for (int t = 0; t < nt; ++t) {
    const int64_t lo = n * t / nt, hi = n * (t + 1) / nt;
    pool.emplace_back([lo, hi, &body] {
      for (int64_t i = lo; i < hi; ++i) body(i);
    });
  }
  for (auto& th : pool) th.join();
}

// ---------------------------------------------------------------------------
// number formats (OCP MX v1.0, section 5.3)
// ---------------------------------------------------------------------------

// E2M1: bit 3 sign, bits 2..1 exponent (bias 1), bit 0 mantissa; exponent
// field 0 is subnormal (0 and 0.5). Magnitudes of the low three bits:
const double kE2M1[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};

double e2m1(uint8_t code) {
  const double m = kE2M1[code & 7];
  return (code & 8) ? -m : m;
}

// E8M0: 2^(c - 127) for c in 0..254; 255 is NaN. No sign, no zero.
double e8m0(uint8_t code) {
  if (code == 255) return std::nan("");
  return std::ldexp(1.0, (int)code - 127);
}

// Element k of an MXFP4 row: q holds two codes per byte, element 2j in the
// LOW nibble of byte j (reading: the pages do not give the nibble order).
uint8_t nibble(const uint8_t* qrow, int64_t k) {
  const uint8_t b = qrow[k >> 1];
  return (k & 1) ? (uint8_t)(b >> 4) : (uint8_t)(b & 0xF);
}

// Dense value of row n of an MXFP4 matrix [N, K] (K a multiple of 32).
void decode_row(const uint8_t* q, const uint8_t* s, int64_t K, int64_t n, double* out) {
  const uint8_t* qrow = q + n * (K / 2);
  const uint8_t* srow = s + n * (K / 32);
  for (int64_t k = 0; k < K; ++k) out[k] = e2m1(nibble(qrow, k)) * e8m0(srow[k / 32]);
}

double bf16(uint16_t bits) {
  const uint32_t u = (uint32_t)bits << 16;
  float f;
  std::memcpy(&f, &u, 4);
  return (double)f;
}

// Nearest bf16 to a double, ties to even, in one rounding step. bf16 keeps 8
// significant bits: the spacing of values in [2^(e-1), 2^e) is 2^(e-8), never
// below 2^-133 (the subnormal spacing). Scaling by a power of two is exact and
// nearbyint rounds half to even (default rounding mode); the result is then a
// bf16 value exactly (or overflows to infinity).
uint16_t round_bf16(double v) {
  if (std::isnan(v)) return 0x7FC0;
  int e = 0;
  std::frexp(v, &e);
  const int ulp = std::max(e - 8, -133);
  const double r = std::ldexp(std::nearbyint(std::ldexp(v, -ulp)), ulp);
  const float f = (float)r;   // exact (a bf16 value), or +-inf beyond the range
  uint32_t u;
  std::memcpy(&u, &f, 4);
  return (uint16_t)(u >> 16);
}

double silu(double z) { return z / (1.0 + std::exp(-z)); }
double sigmoid(double z) { return 1.0 / (1.0 + std::exp(-z)); }

// One block of the OCP MX v1.0 conversion (section 6.3) to MXFP4:
// amax = max |v|; X = floor(log2 amax) - 2 (2 = the largest E2M1 exponent);
// scale code 127 + X clamped to 0..254 (an all-zero block: code 0); each
// v / 2^X rounded to the nearest E2M1 magnitude with ties to the even code,
// magnitudes of 6 or more saturating to 6; the sign bit is v's sign bit.
void quantize_block(const double* v, uint8_t* codes, uint8_t* scale) {
  double amax = 0.0;
  for (int i = 0; i < 32; ++i) amax = std::max(amax, std::fabs(v[i]));
  int sc = 0;
  if (amax > 0.0) {
    int e = 0;
    std::frexp(amax, &e);              // amax = f 2^e, f in [0.5, 1): floor(log2) = e - 1
    sc = std::min(254, std::max(0, 127 + (e - 1) - 2));
  }
  *scale = (uint8_t)sc;
  const double unit = std::ldexp(1.0, sc - 127);
  for (int i = 0; i < 32; ++i) {
    const double s = std::fabs(v[i]) / unit;   // exact: division by a power of two
    int c = 0;
    if (s >= 6.0) {
      c = 7;
    } else if (s > 0.0) {
      int hi = 0;
      while (kE2M1[hi] < s) ++hi;              // first magnitude >= s (hi >= 1)
      const int lo = hi - 1;
      const double d_lo = s - kE2M1[lo], d_hi = kE2M1[hi] - s;
      c = (d_hi < d_lo || (d_hi == d_lo && (hi % 2) == 0)) ? hi : lo;
    }
    codes[i] = (uint8_t)(c | (std::signbit(v[i]) ? 8 : 0));
  }
}

// out[r, n] = sum_k W[n, k] x[r, k] for an MXFP4 matrix W [N, K] and float64
// rows x [R, K]: each row of W is decoded once (exactly), then every sum runs
// over k in ascending order.
void mxfp4_matmul(const uint8_t* q, const uint8_t* s, int64_t N, int64_t K, const double* x,
                  int64_t R, double* out) {
  parallel_for(N, [&](int64_t n) {
    std::vector<double> w(K);
    decode_row(q, s, K, n, w.data());
    for (int64_t r = 0; r < R; ++r) {
      const double* xr = x + r * K;
      double acc = 0.0;
      for (int64_t k = 0; k < K; ++k) acc += w[k] * xr[k];
      out[r * N + n] = acc;
    }
  });
}

// out[r, n] = sum_k W[n, k] x[r, k] for a bf16 matrix W [N, K].
void bf16_matmul(const uint16_t* W, int64_t N, int64_t K, const double* x, int64_t R, double* out) {
  parallel_for(N, [&](int64_t n) {
    std::vector<double> w(K);
    for (int64_t k = 0; k < K; ++k) w[k] = bf16(W[n * K + k]);
    for (int64_t r = 0; r < R; ++r) {
      const double* xr = x + r * K;
      double acc = 0.0;
      for (int64_t k = 0; k < K; ++k) acc += w[k] * xr[k];
      out[r * N + n] = acc;
    }
  });
}

std::vector<double> bf16_rows(const uint16_t* bits, int64_t n) {
  std::vector<double> v(n);
  for (int64_t i = 0; i < n; ++i) v[i] = bf16(bits[i]);
  return v;
}

// Order of experts for selection: larger score first, equal scores by lower
// expert index first (reading: the lowest index wins a tie).
void rank_desc(const double* score, int n, std::vector<int>& order) {
  order.resize(n);
  std::iota(order.begin(), order.end(), 0);
  std::stable_sort(order.begin(), order.end(),
                   [&](int a, int b) { return score[a] > score[b]; });
}

}  // namespace

extern "C" {

// Routing near-tie flags (bits of flags[t]).
enum { kTieSet = 1, kTieOrder = 2, kTieGroup = 4 };

void moe_o_set_threads(int n) { g_threads = n; }
int moe_o_threads(void) { return thread_count(); }

// --- number formats ----------------------------------------------------------

void moe_o_e2m1_decode(const uint8_t* codes, int64_t n, double* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = e2m1(codes[i]);
}

void moe_o_e8m0_decode(const uint8_t* codes, int64_t n, double* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = e8m0(codes[i]);
}

void moe_o_mxfp4_dequant(const uint8_t* q, const uint8_t* s, int64_t N, int64_t K, double* out) {
  for (int64_t n = 0; n < N; ++n) decode_row(q, s, K, n, out + n * K);
}

// codes [n] unpacked (one per byte) and their scales [n/32] -> values [n].
void moe_o_mxfp4_values(const uint8_t* codes, const uint8_t* scales, int64_t n, double* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = e2m1(codes[i]) * e8m0(scales[i / 32]);
}

// Element codes [n] -> bytes [n/2], element 2j in the low nibble of byte j.
void moe_o_mxfp4_pack(const uint8_t* codes, int64_t n, uint8_t* out) {
  for (int64_t j = 0; j < n / 2; ++j)
    out[j] = (uint8_t)((codes[2 * j] & 0xF) | ((codes[2 * j + 1] & 0xF) << 4));
}

void moe_o_bf16_decode(const uint16_t* bits, int64_t n, double* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = bf16(bits[i]);
}

void moe_o_round_bf16(const double* v, int64_t n, uint16_t* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = round_bf16(v[i]);
}

void moe_o_silu(const double* z, int64_t n, double* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = silu(z[i]);
}

void moe_o_sigmoid(const double* z, int64_t n, double* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = sigmoid(z[i]);
}

// a4: MXFP4 quantisation of rows v [rows, K] (K a multiple of 32): unpacked
// codes [rows, K] and scale codes [rows, K/32].
void moe_o_mxfp4_quantize(const double* v, int64_t rows, int64_t K, uint8_t* codes,
                          uint8_t* scales) {
  for (int64_t r = 0; r < rows; ++r)
    for (int64_t b = 0; b < K / 32; ++b)
      quantize_block(v + r * K + 32 * b, codes + r * K + 32 * b, scales + r * (K / 32) + b);
}

void moe_o_mxfp4_matmul(const uint8_t* q, const uint8_t* s, int64_t N, int64_t K,
                        const double* x, int64_t R, double* out) {
  mxfp4_matmul(q, s, N, K, x, R, out);
}

void moe_o_bf16_matmul(const uint16_t* W, int64_t N, int64_t K, const double* x, int64_t R,
                       double* out) {
  bf16_matmul(W, N, K, x, R, out);
}

// --- a1: router -----------------------------------------------------------------
// logits[t, e] = sum_h x[t, h] Wr[e, h] from the bf16 inputs.
void moe_o_router_logits(const uint16_t* x, const uint16_t* wr, int T, int H, int E,
                         double* logits) {
  const std::vector<double> xd = bf16_rows(x, (int64_t)T * H);
  bf16_matmul(wr, E, H, xd.data(), T, logits);
}

// --- a2: top-k selection and weights ------------------------------------------------
// score_fn 0 (softmax; rabbit README, the softmax router keeping 10 of 512): the scores are
// the logits themselves for selection (the softmax is monotone, so ranking by
// logit ranks by probability), and w_j = exp(l_j - m) / sum_sel exp(l_i - m),
// m the largest selected logit: the full softmax renormalised over the
// selected experts (its denominator cancels).
// score_fn 1 (sigmoid; reading of GLM-5.2's "noaux_tc sigmoid"): s_e =
// sigmoid(l_e); selection ranks s_e + bias[e] (the bias steers selection only,
// the auxiliary-loss-free balancing term); w_j = s_j / sum_sel s_i.
// Both: w is multiplied by `scale` (1 for the plain softmax router).
// Group-limited selection (reading of "grouped routing"; n_group > 1): the E
// experts form n_group consecutive groups of E / n_group; a group's score is
// the sum of the two largest expert scores in it (the one score when a group
// has one expert), the expert score being the softmax probability (softmax;
// computed as exp(l_e - max_e' l_e'), the common denominator dropped) or the
// biased sigmoid score s_e + bias[e] (sigmoid); the topk_group best groups
// are kept (ties: lower group first) and the top k is taken among their
// experts only, ranked as above.
// Near-tie flags: kTieSet when the k-th and (k+1)-th selection scores among
// the eligible experts differ by less than near_tie (the selected SET then
// depends on rounding); kTieOrder when two adjacent selected scores do (only
// the slot ORDER does); kTieGroup when the topk_group-th and next group
// scores do.
// idx_in (nullable): a given selection [T, k] whose weights are wanted instead.
int moe_o_route(const double* logits, const double* bias, int T, int E, int k, int score_fn,
                int n_group, int topk_group, double scale, double near_tie,
                const int32_t* idx_in, int32_t* idx, double* w, uint8_t* flags) {
  if (k < 1 || k > E || (score_fn != 0 && score_fn != 1)) return 1;
  if (n_group < 1) n_group = 1;
  if (E % n_group || topk_group < 1 || topk_group > n_group) return 2;
  if (n_group > 1 && (int64_t)topk_group * (E / n_group) < k) return 3;
  const int gsize = E / n_group;
  for (int t = 0; t < T; ++t) {
    const double* l = logits + (int64_t)t * E;
    std::vector<double> sc(E), choice(E);
    for (int e = 0; e < E; ++e) {
      sc[e] = score_fn == 0 ? l[e] : sigmoid(l[e]);
      choice[e] = sc[e] + (score_fn == 1 && bias ? bias[e] : 0.0);
    }
    uint8_t f = 0;
    std::vector<char> eligible(E, 1);
    if (n_group > 1) {
      std::vector<double> gval(E);
      double lmax = -INFINITY;
      for (int e = 0; e < E; ++e) lmax = std::max(lmax, l[e]);
      for (int e = 0; e < E; ++e) gval[e] = score_fn == 0 ? std::exp(l[e] - lmax) : choice[e];
      std::vector<double> gscore(n_group);
      std::vector<int> ord;
      for (int g = 0; g < n_group; ++g) {
        rank_desc(gval.data() + (int64_t)g * gsize, gsize, ord);
        gscore[g] = gval[g * gsize + ord[0]] + (gsize > 1 ? gval[g * gsize + ord[1]] : 0.0);
      }
      std::vector<int> gord;
      rank_desc(gscore.data(), n_group, gord);
      std::fill(eligible.begin(), eligible.end(), 0);
      for (int i = 0; i < topk_group; ++i)
        for (int e = 0; e < gsize; ++e) eligible[gord[i] * gsize + e] = 1;
      if (topk_group < n_group &&
          gscore[gord[topk_group - 1]] - gscore[gord[topk_group]] < near_tie)
        f |= kTieGroup;
    }
    // ranking of the eligible experts
    std::vector<double> masked(E);
    for (int e = 0; e < E; ++e) masked[e] = eligible[e] ? choice[e] : -INFINITY;
    std::vector<int> ord;
    rank_desc(masked.data(), E, ord);
    int n_elig = 0;
    for (int e = 0; e < E; ++e) n_elig += eligible[e];
    int32_t* it = idx + (int64_t)t * k;
    for (int j = 0; j < k; ++j) it[j] = ord[j];
    if (k < n_elig && masked[ord[k - 1]] - masked[ord[k]] < near_tie) f |= kTieSet;
    for (int j = 0; j + 1 < k; ++j)
      if (masked[ord[j]] - masked[ord[j + 1]] < near_tie) f |= kTieOrder;
    flags[t] = f;
    // weights of the oracle's selection, or of the given one
    const int32_t* sel = idx_in ? idx_in + (int64_t)t * k : it;
    double* wt = w + (int64_t)t * k;
    if (score_fn == 0) {
      double m = -INFINITY;
      for (int j = 0; j < k; ++j) m = std::max(m, l[sel[j]]);
      double sum = 0.0;
      for (int j = 0; j < k; ++j) {
        wt[j] = std::exp(l[sel[j]] - m);
        sum += wt[j];
      }
      for (int j = 0; j < k; ++j) wt[j] = wt[j] / sum * scale;
    } else {
      double sum = 0.0;
      for (int j = 0; j < k; ++j) sum += sc[sel[j]];
      for (int j = 0; j < k; ++j) wt[j] = sc[sel[j]] / sum * scale;
    }
  }
  return 0;
}

// --- a3: permutation --------------------------------------------------------------
// Groups the T*k (token, slot) pairs by expert: counts[e], offsets (exclusive
// prefix sum, E+1 entries), rows ordered by expert and, inside an expert, by
// ascending token (reading: the pages never describe the dispatch; "stable by
// token" is the plainest order; a token holds an expert at most once).
// Returns 1 when an index is outside [0, E) (nothing written then).
int moe_o_permute(const int32_t* idx, int T, int k, int E, int32_t* counts, int32_t* offsets,
                  int32_t* row_token, int32_t* row_slot, int32_t* slot_row) {
  for (int64_t p = 0; p < (int64_t)T * k; ++p)
    if (idx[p] < 0 || idx[p] >= E) return 1;
  for (int e = 0; e < E; ++e) counts[e] = 0;
  for (int64_t p = 0; p < (int64_t)T * k; ++p) counts[idx[p]]++;
  offsets[0] = 0;
  for (int e = 0; e < E; ++e) offsets[e + 1] = offsets[e] + counts[e];
  std::vector<int32_t> fill(offsets, offsets + E);
  for (int t = 0; t < T; ++t)
    for (int j = 0; j < k; ++j) {
      const int e = idx[(int64_t)t * k + j];
      const int32_t r = fill[e]++;
      row_token[r] = t;
      row_slot[r] = j;
      slot_row[(int64_t)t * k + j] = r;
    }
  return 0;
}

// --- a5-a7: one routed expert on its rows ------------------------------------------
// x [n, W] float64 rows of this expert; Wg, Wu [I, W] and Wd [W, I] MXFP4.
//   g = Wg x, u = Wu x, h = silu(g) * u, y = Wd h
// act 0 ("exact"): x and h enter their products unrounded (decode: bf16 x is
//   exact; h keeps full precision).
// act 1 ("mxfp4"): x and h are each quantised to MXFP4 (a4, 32-element
//   blocks along the contraction) before their products (prefill with MXFP4
//   activations).
// Reading: the activation is SwiGLU, silu(z) = z / (1 + e^-z), for every
// model (the Kimi K3 page names "SituAndMul" without defining it).
// Outputs: y [n, W]; h [n, I] as it entered the down projection; h_raw
// [n, I] (nullable) = silu(g) * u before any rounding.
int moe_o_expert_ffn(const double* x, int n, int W, int I, const uint8_t* wg_q,
                     const uint8_t* wg_s, const uint8_t* wu_q, const uint8_t* wu_s,
                     const uint8_t* wd_q, const uint8_t* wd_s, int act, double* y, double* h,
                     double* h_raw) {
  if (act != 0 && act != 1) return 1;
  std::vector<double> xin(x, x + (int64_t)n * W);
  if (act == 1) {
    std::vector<uint8_t> c((size_t)n * W), s((size_t)n * W / 32);
    moe_o_mxfp4_quantize(x, n, W, c.data(), s.data());
    moe_o_mxfp4_values(c.data(), s.data(), (int64_t)n * W, xin.data());
  }
  std::vector<double> g((size_t)n * I), u((size_t)n * I);
  mxfp4_matmul(wg_q, wg_s, I, W, xin.data(), n, g.data());
  mxfp4_matmul(wu_q, wu_s, I, W, xin.data(), n, u.data());
  for (int64_t i = 0; i < (int64_t)n * I; ++i) h[i] = silu(g[i]) * u[i];
  if (h_raw) std::copy(h, h + (int64_t)n * I, h_raw);
  if (act == 1) {
    std::vector<uint8_t> c((size_t)n * I), s((size_t)n * I / 32);
    moe_o_mxfp4_quantize(h, n, I, c.data(), s.data());
    moe_o_mxfp4_values(c.data(), s.data(), (int64_t)n * I, h);
  }
  mxfp4_matmul(wd_q, wd_s, W, I, h, n, y);
  return 0;
}

// --- a8: gated shared expert ----------------------------------------------------------
// s[t] = sigmoid(x[t] . w_sg) * Wsd (silu(Wsg x[t]) * (Wsu x[t])), bf16 weights.
// Reading: the gate is one sigmoid scalar per token from a weight vector w_sg
// (the pages only call it a gated shared expert); the shared expert always runs.
void moe_o_shared_expert(const uint16_t* x, int T, int H, int Is, const uint16_t* ws_gate,
                         const uint16_t* ws_up, const uint16_t* ws_down, const uint16_t* w_sgate,
                         double* s, double* gate) {
  const std::vector<double> xd = bf16_rows(x, (int64_t)T * H);
  std::vector<double> glogit(T);
  bf16_matmul(w_sgate, 1, H, xd.data(), T, glogit.data());
  std::vector<double> g((size_t)T * Is), u((size_t)T * Is), h((size_t)T * Is);
  bf16_matmul(ws_gate, Is, H, xd.data(), T, g.data());
  bf16_matmul(ws_up, Is, H, xd.data(), T, u.data());
  for (int64_t i = 0; i < (int64_t)T * Is; ++i) h[i] = silu(g[i]) * u[i];
  bf16_matmul(ws_down, H, Is, h.data(), T, s);
  for (int t = 0; t < T; ++t) {
    gate[t] = sigmoid(glogit[t]);
    for (int c = 0; c < H; ++c) s[(int64_t)t * H + c] *= gate[t];
  }
}

// --- a9 (+ a10 up): combine -----------------------------------------------------------
// acc[t] = sum_j w[t, j] * y_perm[slot_row[t, j]] (slots in order j = 0..k-1),
// at width W; latent layers map it once: acc = W_lu acc (W_lu [H, L] bf16);
// then y[t] = acc[t] + shared[t] (shared nullable).
void moe_o_combine(const double* y_perm, int W, const int32_t* slot_row, const double* w, int T,
                   int k, const double* shared, const uint16_t* w_lat_up, int H, double* y) {
  std::vector<double> acc((size_t)T * W, 0.0);
  for (int t = 0; t < T; ++t)
    for (int j = 0; j < k; ++j) {
      const double wj = w[(int64_t)t * k + j];
      const double* row = y_perm + (int64_t)slot_row[(int64_t)t * k + j] * W;
      for (int c = 0; c < W; ++c) acc[(int64_t)t * W + c] += wj * row[c];
    }
  const int out_w = w_lat_up ? H : W;
  if (w_lat_up) {
    bf16_matmul(w_lat_up, H, W, acc.data(), T, y);
  } else {
    std::copy(acc.begin(), acc.end(), y);
  }
  if (shared)
    for (int64_t i = 0; i < (int64_t)T * out_w; ++i) y[i] += shared[i];
}

// --- a10: latent down-projection --------------------------------------------------------
// x_lat = bf16_rne(W_ld x) [T, L] (reading: a dense bf16 matrix [L, H] whose
// result is rounded to bf16, the experts' input type, before the experts).
void moe_o_latent_down(const uint16_t* x, int T, int H, const uint16_t* w_lat_down, int L,
                       uint16_t* x_lat) {
  const std::vector<double> xd = bf16_rows(x, (int64_t)T * H);
  std::vector<double> v((size_t)T * L);
  bf16_matmul(w_lat_down, L, H, xd.data(), T, v.data());
  for (int64_t i = 0; i < (int64_t)T * L; ++i) x_lat[i] = round_bf16(v[i]);
}

// --- the whole layer ----------------------------------------------------------------------
typedef struct {
  int32_t T, H, I, E, k, I_shared, L;
  int32_t act;          // 0 exact, 1 MXFP4 activations
  int32_t score_fn;     // 0 softmax, 1 sigmoid
  int32_t n_group, topk_group;
  double route_scale;
  double near_tie;
} moe_o_dims;

typedef struct {
  const uint16_t *x, *w_router;
  const double* e_bias;                        // [E] or NULL
  const uint16_t *w_sgate, *ws_gate, *ws_up, *ws_down;
  const uint16_t *w_lat_down, *w_lat_up;       // NULL unless L > 0
  // per-expert weight tables [E]: NULL for an expert no token selects
  const uint8_t* const* wg_q;
  const uint8_t* const* wg_s;
  const uint8_t* const* wu_q;
  const uint8_t* const* wu_s;
  const uint8_t* const* wd_q;
  const uint8_t* const* wd_s;
  const int32_t* idx_override;                 // [T, k] or NULL
} moe_o_inputs;

typedef struct {
  double* logits;                // [T, E]
  int32_t* idx;                  // [T, k]
  double* w;                     // [T, k]
  uint8_t* flags;                // [T]
  int32_t *counts, *offsets, *row_token, *row_slot, *slot_row;
  uint16_t* x_lat;               // [T, L] (latent layers)
  double* y_perm;                // [T*k, W]
  double* h_perm;                // [T*k, I]
  double* shared;                // [T, H]
  double* gate;                  // [T]
  double* y;                     // [T, H]
} moe_o_outputs;

// Returns 0; 1-3 for a bad routing configuration; 4 for an index outside
// [0, E); 5 for a selected expert whose weights were not given.
int moe_o_layer(const moe_o_dims* d, const moe_o_inputs* in, const moe_o_outputs* out) {
  const int T = d->T, E = d->E, k = d->k, H = d->H;
  const int W = d->L ? d->L : H;
  moe_o_router_logits(in->x, in->w_router, T, H, E, out->logits);
  int st = moe_o_route(out->logits, in->e_bias, T, E, k, d->score_fn, d->n_group, d->topk_group,
                       d->route_scale, d->near_tie, in->idx_override, out->idx, out->w, out->flags);
  if (st) return st;
  if (in->idx_override)
    std::copy(in->idx_override, in->idx_override + (int64_t)T * k, out->idx);
  if (moe_o_permute(out->idx, T, k, E, out->counts, out->offsets, out->row_token, out->row_slot,
                    out->slot_row))
    return 4;
  std::vector<double> xin;
  if (d->L) {
    moe_o_latent_down(in->x, T, H, in->w_lat_down, d->L, out->x_lat);
    xin = bf16_rows(out->x_lat, (int64_t)T * d->L);
  } else {
    xin = bf16_rows(in->x, (int64_t)T * H);
  }
  for (int e = 0; e < E; ++e) {
    const int r0 = out->offsets[e], n = out->offsets[e + 1] - r0;
    if (n == 0) continue;
    if (!in->wg_q[e] || !in->wg_s[e] || !in->wu_q[e] || !in->wu_s[e] || !in->wd_q[e] ||
        !in->wd_s[e])
      return 5;
    std::vector<double> rows((size_t)n * W);
    for (int i = 0; i < n; ++i)
      std::copy(xin.begin() + (int64_t)out->row_token[r0 + i] * W,
                xin.begin() + (int64_t)(out->row_token[r0 + i] + 1) * W,
                rows.begin() + (int64_t)i * W);
    moe_o_expert_ffn(rows.data(), n, W, d->I, in->wg_q[e], in->wg_s[e], in->wu_q[e],
                     in->wu_s[e], in->wd_q[e], in->wd_s[e], d->act,
                     out->y_perm + (int64_t)r0 * W, out->h_perm + (int64_t)r0 * d->I, nullptr);
  }
  moe_o_shared_expert(in->x, T, H, d->I_shared, in->ws_gate, in->ws_up, in->ws_down,
                      in->w_sgate, out->shared, out->gate);
  moe_o_combine(out->y_perm, W, out->slot_row, out->w, T, k, out->shared,
                d->L ? in->w_lat_up : nullptr, H, out->y);
  return 0;
}

}  // extern "C"
