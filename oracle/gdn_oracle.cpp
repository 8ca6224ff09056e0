// CPU oracle for the Gated DeltaNet (GDN) token mixer: float64, token by token.
//
// TEST INFRASTRUCTURE ONLY.  Nothing on the product path may include, link,
// load or call this file; it is used by tests/, by the smoke check and by the
// benchmark's CPU-baseline leg.  It shares no code with the CUDA library.
//
// What it computes is the plain definition of the mixer, one token at a time,
// in the order the stages are named by the reference pages:
//   * "causal depthwise Conv1D, Gated DeltaNet recurrence, and recurrent-state
//     cache" -- DS4Server issue #88 ("Add a performance-parity Qwen3.8-27B Q4
//     and Q8 text backend on Metal"), section Scope;
//   * "16-key/48-value-head GDN geometry, convolution width 4, fp32 recurrent
//     state, sigmoid output gate, and exact L2-normalization epsilon
//     placement" and "zero-centered norms" -- DS4Server issue #95 ("Implement
//     the Qwen3.8 Flash Next Rust and Metal text core"), section
//     Implementation;
//   * "BF16 width-4 convolution history, fp32 Gated DeltaNet recurrence" and
//     "zero-centered grouped RMS" -- issue #95, implementation comment.
// The pages name these stages but print no formula.  The formulas below are
// the standard Gated DeltaNet ones; each reading the pages leave open is
// stated where it is used (epsilon inside the square root of the sum, the
// last conv tap on the current token, contiguous key-head groups, norm
// weight applied as 1 + w, norm before the sigmoid gate).
//
// Every input arrives as float32 holding the exact value of its stored dtype
// (bf16 or fp32); every operation here is float64 with the host libm.

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <thread>
#include <vector>

extern "C" {

struct gdn_ref_geometry {
  int32_t num_k_heads;  // Hk
  int32_t num_v_heads;  // Hv, a multiple of Hk
  int32_t head_k_dim;   // dk
  int32_t head_v_dim;   // dv
  int32_t conv_width;   // W
  double l2_eps;        // epsilon inside the L2 norm's square root
  double norm_eps;      // epsilon inside the RMSNorm's square root
  double q_scale;       // factor on the normalised query
};

// softplus(x) = log(1 + e^x) in its overflow-free form.
static double softplus(double x) { return std::max(x, 0.0) + std::log1p(std::exp(-std::fabs(x))); }
static double sigmoid(double x) { return 1.0 / (1.0 + std::exp(-x)); }
static double silu(double y) { return y / (1.0 + std::exp(-y)); }

// Gates of one token and value head: g = -exp(A_log) * softplus(a + dt_bias),
// alpha = exp(g) (the decay), beta = sigmoid(b) (the write strength).
void gdn_ref_gates(double a, double dt_bias, double A_log, double b, double* g, double* alpha, double* beta) {
  const double gg = -std::exp(A_log) * softplus(a + dt_bias);
  *g = gg;
  *alpha = std::exp(gg);
  *beta = sigmoid(b);
}

// out = scale * x / sqrt(sum(x^2) + eps): the epsilon sits inside the square
// root of the sum (issue #95, "exact L2-normalization epsilon placement").
void gdn_ref_l2norm(const double* x, int32_t n, double eps, double scale, double* out) {
  double s = 0.0;
  for (int32_t i = 0; i < n; ++i) s += x[i] * x[i];
  const double r = scale / std::sqrt(s + eps);
  for (int32_t i = 0; i < n; ++i) out[i] = x[i] * r;
}

// Zero-centred RMSNorm over one value head's output, then the sigmoid output
// gate: out_j = o_j / sqrt(mean(o^2) + eps) * (1 + w_j) * sigmoid(z_j).
void gdn_ref_output(const double* o, const double* z, const double* w, int32_t dv, double eps, double* out) {
  double s = 0.0;
  for (int32_t j = 0; j < dv; ++j) s += o[j] * o[j];
  const double r = 1.0 / std::sqrt(s / dv + eps);
  for (int32_t j = 0; j < dv; ++j) out[j] = o[j] * r * (1.0 + w[j]) * sigmoid(z[j]);
}

// One step of the gated delta rule on a dk x dv state S (row-major S[i*dv+j]):
//   S <- alpha * S;  r = S^T k;  delta = beta * (v - r);  S <- S + k delta^T;
//   o = S^T q.
void gdn_ref_delta_step(double* S, const double* k, const double* v, const double* q, double alpha, double beta,
                        int32_t dk, int32_t dv, double* o) {
  std::vector<double> r(dv, 0.0), delta(dv);
  for (int32_t i = 0; i < dk * dv; ++i) S[i] *= alpha;
  for (int32_t i = 0; i < dk; ++i)
    for (int32_t j = 0; j < dv; ++j) r[j] += S[i * dv + j] * k[i];
  for (int32_t j = 0; j < dv; ++j) delta[j] = beta * (v[j] - r[j]);
  for (int32_t i = 0; i < dk; ++i)
    for (int32_t j = 0; j < dv; ++j) S[i * dv + j] += k[i] * delta[j];
  for (int32_t j = 0; j < dv; ++j) o[j] = 0.0;
  for (int32_t i = 0; i < dk; ++i)
    for (int32_t j = 0; j < dv; ++j) o[j] += S[i * dv + j] * q[i];
}

// Causal depthwise conv of channel c at local position p of a sequence, then
// SiLU.  The history holds the W-1 raw inputs before the sequence, oldest
// first; the last tap w[c][W-1] multiplies the current token.
static double conv_silu(const float* conv_w, int32_t W, const float* hist /*[W-1][C]*/, const float* x /*[len][C]*/,
                        int64_t C, int64_t c, int64_t p) {
  double y = 0.0;
  for (int32_t j = 0; j < W; ++j) {
    const int64_t m = p + j - (W - 1);  // position of this tap, relative to the sequence start
    const double xv = (m < 0) ? (double)hist[(m + (W - 1)) * C + c] : (double)x[m * C + c];
    y += (double)conv_w[c * W + j] * xv;
  }
  return silu(y);
}

// New conv history of every sequence: the last W-1 raw inputs of
// [history, x], copied unchanged (so bf16 history stays bf16 bytes).
void gdn_ref_conv_history(int64_t C, int32_t W, const float* x, const int64_t* cu_seqlens, int32_t N,
                          const float* hist_in, float* hist_out) {
  for (int32_t n = 0; n < N; ++n) {
    const int64_t len = cu_seqlens[n + 1] - cu_seqlens[n];
    const float* xs = x + cu_seqlens[n] * C;
    const float* hin = hist_in + (int64_t)n * (W - 1) * C;
    float* hout = hist_out + (int64_t)n * (W - 1) * C;
    for (int32_t i = 0; i < W - 1; ++i) {
      const int64_t m = len + i - (W - 1);  // source position relative to the sequence start
      for (int64_t c = 0; c < C; ++c) hout[i * C + c] = (m < 0) ? hin[(m + (W - 1)) * C + c] : xs[m * C + c];
    }
  }
}

// Standalone conv prefill: y[t][c] = SiLU(conv) for every channel, plus the
// new history.
int32_t gdn_ref_conv_prefill(int64_t C, int32_t W, const float* conv_w, const float* x, const int64_t* cu_seqlens,
                             int32_t N, const float* hist_in, double* y, float* hist_out) {
  for (int32_t n = 0; n < N; ++n) {
    const int64_t len = cu_seqlens[n + 1] - cu_seqlens[n];
    const float* xs = x + cu_seqlens[n] * C;
    const float* hin = hist_in + (int64_t)n * (W - 1) * C;
    for (int64_t p = 0; p < len; ++p)
      for (int64_t c = 0; c < C; ++c) y[(cu_seqlens[n] + p) * C + c] = conv_silu(conv_w, W, hin, xs, C, c, p);
  }
  gdn_ref_conv_history(C, W, x, cu_seqlens, N, hist_in, hist_out);
  return 0;
}

// One (sequence n, value head h) of a prefill: walk the tokens in order.
static void prefill_task(const gdn_ref_geometry& g, const float* conv_w, const float* A_log, const float* dt_bias,
                         const float* norm_w, const float* qkv, const float* z, const float* a, const float* b,
                         const int64_t* cu, int32_t n, int32_t h, const float* hist_in, double* state, double* o) {
  const int32_t Hk = g.num_k_heads, Hv = g.num_v_heads, dk = g.head_k_dim, dv = g.head_v_dim, W = g.conv_width;
  const int32_t G = Hv / Hk;
  const int32_t kh = h / G;  // value heads G*kh .. G*kh+G-1 share key head kh
  const int64_t C = 2LL * Hk * dk + (int64_t)Hv * dv;
  const int64_t q0 = (int64_t)kh * dk, k0 = (int64_t)Hk * dk + (int64_t)kh * dk,
                v0 = 2LL * Hk * dk + (int64_t)h * dv;
  const int64_t len = cu[n + 1] - cu[n];
  const float* xs = qkv + cu[n] * C;
  const float* hin = hist_in + (int64_t)n * (W - 1) * C;

  // S[i][j] = state[n][h][j][i] (the state is stored transposed, [dv][dk]).
  double* st = state + ((int64_t)n * Hv + h) * dv * dk;
  std::vector<double> S((size_t)dk * dv);
  for (int32_t i = 0; i < dk; ++i)
    for (int32_t j = 0; j < dv; ++j) S[(size_t)i * dv + j] = st[(int64_t)j * dk + i];

  std::vector<double> qu(dk), ku(dk), vu(dv), qh(dk), khat(dk), ov(dv), zv(dv), wv(dv), out(dv);
  for (int32_t j = 0; j < dv; ++j) wv[j] = norm_w[j];
  for (int64_t p = 0; p < len; ++p) {
    const int64_t t = cu[n] + p;
    for (int32_t i = 0; i < dk; ++i) qu[i] = conv_silu(conv_w, W, hin, xs, C, q0 + i, p);
    for (int32_t i = 0; i < dk; ++i) ku[i] = conv_silu(conv_w, W, hin, xs, C, k0 + i, p);
    for (int32_t j = 0; j < dv; ++j) vu[j] = conv_silu(conv_w, W, hin, xs, C, v0 + j, p);
    gdn_ref_l2norm(qu.data(), dk, g.l2_eps, g.q_scale, qh.data());
    gdn_ref_l2norm(ku.data(), dk, g.l2_eps, 1.0, khat.data());
    double gg, alpha, beta;
    gdn_ref_gates(a[t * Hv + h], dt_bias[h], A_log[h], b[t * Hv + h], &gg, &alpha, &beta);
    gdn_ref_delta_step(S.data(), khat.data(), vu.data(), qh.data(), alpha, beta, dk, dv, ov.data());
    for (int32_t j = 0; j < dv; ++j) zv[j] = z[t * (int64_t)Hv * dv + (int64_t)h * dv + j];
    gdn_ref_output(ov.data(), zv.data(), wv.data(), dv, g.norm_eps, out.data());
    for (int32_t j = 0; j < dv; ++j) o[t * (int64_t)Hv * dv + (int64_t)h * dv + j] = out[j];
  }
  for (int32_t i = 0; i < dk; ++i)
    for (int32_t j = 0; j < dv; ++j) st[(int64_t)j * dk + i] = S[(size_t)i * dv + j];
}

// Prefill over packed sequences (cu_seqlens [N+1]).  Heads with
// head_mask[h] == 0 are skipped (their outputs and states are left as they
// are), so a caller can sample value heads of a large problem.  state is
// float64 [N][Hv][dv][dk], read and written in place; o is float64
// [T][Hv*dv]; hist_out receives the new conv history (float32 copies).
int32_t gdn_ref_prefill(const gdn_ref_geometry* geo, const float* conv_w, const float* A_log, const float* dt_bias,
                        const float* norm_w, const float* qkv, const float* z, const float* a, const float* b,
                        const int64_t* cu_seqlens, int32_t N, const uint8_t* head_mask, const float* hist_in,
                        double* state, double* o, float* hist_out, int32_t num_threads) {
  const gdn_ref_geometry g = *geo;
  if (g.num_k_heads <= 0 || g.num_v_heads % g.num_k_heads != 0 || g.conv_width < 1) return -1;
  std::vector<std::pair<int32_t, int32_t>> tasks;
  for (int32_t n = 0; n < N; ++n)
    for (int32_t h = 0; h < g.num_v_heads; ++h)
      if (!head_mask || head_mask[h]) tasks.emplace_back(n, h);
  std::atomic<size_t> next{0};
  auto worker = [&]() {
    for (size_t i = next++; i < tasks.size(); i = next++)
      prefill_task(g, conv_w, A_log, dt_bias, norm_w, qkv, z, a, b, cu_seqlens, tasks[i].first, tasks[i].second,
                   hist_in, state, o);
  };
  const int32_t nt = std::max<int32_t>(1, std::min<int32_t>(num_threads, (int32_t)tasks.size()));
  std::vector<std::thread> pool;
  for (int32_t i = 1; i < nt; ++i) pool.emplace_back(worker);
  worker();
  for (auto& th : pool) th.join();
  const int64_t C = 2LL * g.num_k_heads * g.head_k_dim + (int64_t)g.num_v_heads * g.head_v_dim;
  if (hist_out) gdn_ref_conv_history(C, g.conv_width, qkv, cu_seqlens, N, hist_in, hist_out);
  return 0;
}

// One decode step: every sequence advances by exactly one token, i.e. a
// prefill whose sequences all have length 1.
int32_t gdn_ref_decode_step(const gdn_ref_geometry* geo, const float* conv_w, const float* A_log,
                            const float* dt_bias, const float* norm_w, const float* qkv, const float* z,
                            const float* a, const float* b, int32_t N, const uint8_t* head_mask,
                            const float* hist_in, double* state, double* o, float* hist_out, int32_t num_threads) {
  std::vector<int64_t> cu(N + 1);
  for (int32_t n = 0; n <= N; ++n) cu[n] = n;
  return gdn_ref_prefill(geo, conv_w, A_log, dt_bias, norm_w, qkv, z, a, b, cu.data(), N, head_mask, hist_in, state,
                         o, hist_out, num_threads);
}

// Dense projection of a linear layer ("GDN projection" primitive, issue #95,
// Verification; the BF16 projection kernels of its implementation comment):
//   y[i][c] = sum_k x[rows[i]][k] * w[c][k]
// for the R listed rows of x [M][K]; w [N][K] holds the layer's weight (output
// features x input features).  Every product and sum is float64, k ascending.
void gdn_ref_project(const float* x, int64_t K, const float* w, int64_t N, const int64_t* rows, int64_t R,
                     double* y, int32_t num_threads) {
  std::atomic<int64_t> next{0};
  auto worker = [&]() {
    for (int64_t i = next++; i < R; i = next++) {
      const float* xr = x + rows[i] * K;
      for (int64_t c = 0; c < N; ++c) {
        const float* wc = w + c * K;
        double s = 0.0;
        for (int64_t k = 0; k < K; ++k) s += (double)xr[k] * (double)wc[k];
        y[i * N + c] = s;
      }
    }
  };
  const int32_t nt = (int32_t)std::max<int64_t>(1, std::min<int64_t>(num_threads, R));
  std::vector<std::thread> pool;
  for (int32_t t = 1; t < nt; ++t) pool.emplace_back(worker);
  worker();
  for (auto& th : pool) th.join();
}

}  // extern "C"
