// Plain fp64 CPU oracle for the gated delta-rule (Gated DeltaNet) layer.
//
// TEST INFRASTRUCTURE ONLY. Nothing in the product path may link, load or call
// this file; only the tests, the smoke check and the bench's CPU-baseline leg do.
// It shares no code, header or constant with the CUDA library.
//
// Sources (page titles and sections):
//  * llama.cpp compare b7429..b7432, "Optimization: Qwen3 next autoregressive pass",
//    src/models/qwen3next.cpp, build_delta_net_autoregressive: the single-token step
//    S <- e^g S ; kv = S^T k ; delta = beta (v - kv) ; S <- S + k delta^T ; o = S^T q.
//  * same page, the removed single-chunk path (the PyTorch-style comments) and
//    build_delta_net_chunking: the chunked (WY/UT) form used by oracle_chunked.
//  * ik_llama.cpp src/llama-delta-net.cpp, build_layer_attn_linear_core: the front
//    (ggml_ssm_conv over [conv_state; x], SiLU over the whole conv output, q|k|v
//    split, L2 norm of q and k, grouped GQA repeat, gate = softplus(a + dt_bias)*ssm_a).
//
// Readings where the pages leave a step open (each also listed in the design notes):
//  * L2 norm: x / sqrt(sum x^2 + eps).
//  * softplus(x) = max(x,0) + log1p(exp(-|x|)) (exact, no threshold switch).
//  * ssm_a = -exp(A_log).
//  * conv: cross-correlation, tap d_conv-1 on the current token, no bias, state rows
//    ordered oldest -> newest; the new state is the last d_conv-1 rows of [state; x].
//  * GQA grouped: v-head h reads k-head h / (H_v / H_k).
//  * reset[n] != 0: the sequence starts from a zero recurrent state and zero conv state.
//  * d_conv == 0: no conv and no SiLU; x is the q|k|v stream as given.
//
// Every function here is plain loops in double precision, one (sequence, head) unit at a
// time; units are spread over std::thread workers, each unit computed by exactly one
// worker in a fixed order, so results do not depend on the thread count.

#include <cmath>
#include <cstdint>
#include <cstring>
#include <thread>
#include <vector>
#include <functional>
#include <algorithm>

namespace {

void run_units(int n_units, int n_threads, const std::function<void(int)>& fn) {
  if (n_threads <= 1 || n_units <= 1) {
    for (int u = 0; u < n_units; ++u) fn(u);
    return;
  }
  n_threads = std::min(n_threads, n_units);
  std::vector<std::thread> pool;
  pool.reserve(n_threads);
  for (int w = 0; w < n_threads; ++w) {
    pool.emplace_back([&, w]() {
      for (int u = w; u < n_units; u += n_threads) fn(u);
    });
  }
  for (auto& th : pool) th.join();
}

double sigmoid(double x) { return 1.0 / (1.0 + std::exp(-x)); }
double softplus(double x) { return std::max(x, 0.0) + std::log1p(std::exp(-std::fabs(x))); }

}  // namespace

extern "C" {

// Front: causal depthwise conv over [conv_state; x], SiLU, q|k|v split, L2 norm of q and k,
// q scale, gates. Per sequence n (tokens cu_seqlens[n] .. cu_seqlens[n+1]-1).
//   x          [T_total][conv_dim], conv_dim = 2*H_k*d_k + H_v*d_v, channel order q|k|v
//   conv_w     [conv_dim][d_conv]          (ignored when d_conv == 0)
//   conv_state [n_seqs][d_conv-1][conv_dim] per sequence (already gathered by slot);
//              read as the initial state, overwritten with the final state.
//   a, b       [T_total][H_v];  A_log, dt_bias [H_v]
//   outputs q,k [T_total][H_k][d_k], v [T_total][H_v][d_v], g, beta [T_total][H_v]
int oracle_front(int64_t T_total, int n_seqs, const int32_t* cu_seqlens, const uint8_t* reset,
                 int H_k, int H_v, int d_k, int d_v, int d_conv,
                 const double* x, const double* conv_w, double* conv_state,
                 const double* a, const double* b, const double* A_log, const double* dt_bias,
                 double eps, double q_scale,
                 double* q, double* k, double* v, double* g, double* beta, int n_threads) {
  const int64_t conv_dim = 2LL * H_k * d_k + (int64_t)H_v * d_v;
  const int n_state_rows = d_conv > 0 ? d_conv - 1 : 0;
  run_units(n_seqs, n_threads, [&](int n) {
    const int64_t t0 = cu_seqlens[n], t1 = cu_seqlens[n + 1];
    const int64_t len = t1 - t0;
    // x_ext = [state rows (oldest first); x rows of this sequence]
    std::vector<double> x_ext((size_t)(n_state_rows + len) * conv_dim, 0.0);
    double* st = conv_state + (int64_t)n * n_state_rows * conv_dim;
    const bool rst = reset != nullptr && reset[n] != 0;
    for (int r = 0; r < n_state_rows; ++r)
      for (int64_t c = 0; c < conv_dim; ++c)
        x_ext[(size_t)r * conv_dim + c] = rst ? 0.0 : st[(int64_t)r * conv_dim + c];
    for (int64_t t = 0; t < len; ++t)
      for (int64_t c = 0; c < conv_dim; ++c)
        x_ext[(size_t)(n_state_rows + t) * conv_dim + c] = x[(t0 + t) * conv_dim + c];

    std::vector<double> u(conv_dim);
    for (int64_t t = 0; t < len; ++t) {
      const int64_t tt = t0 + t;
      for (int64_t c = 0; c < conv_dim; ++c) {
        if (d_conv > 0) {
          double y = 0.0;
          for (int j = 0; j < d_conv; ++j)  // tap j reads row t + j of x_ext; tap d_conv-1 = current
            y += conv_w[c * d_conv + j] * x_ext[(size_t)(t + j) * conv_dim + c];
          u[c] = y * sigmoid(y);  // SiLU
        } else {
          u[c] = x_ext[(size_t)t * conv_dim + c];
        }
      }
      for (int h = 0; h < H_k; ++h) {
        const double* qh = &u[(int64_t)h * d_k];
        const double* kh = &u[(int64_t)H_k * d_k + (int64_t)h * d_k];
        double sq = 0.0, sk = 0.0;
        for (int i = 0; i < d_k; ++i) { sq += qh[i] * qh[i]; sk += kh[i] * kh[i]; }
        const double nq = 1.0 / std::sqrt(sq + eps), nk = 1.0 / std::sqrt(sk + eps);
        for (int i = 0; i < d_k; ++i) {
          q[(tt * H_k + h) * d_k + i] = qh[i] * nq * q_scale;
          k[(tt * H_k + h) * d_k + i] = kh[i] * nk;
        }
      }
      for (int h = 0; h < H_v; ++h)
        for (int j = 0; j < d_v; ++j)
          v[(tt * H_v + h) * d_v + j] = u[2LL * H_k * d_k + (int64_t)h * d_v + j];
      for (int h = 0; h < H_v; ++h) {
        const double ssm_a = -std::exp(A_log[h]);
        g[tt * H_v + h] = ssm_a * softplus(a[tt * H_v + h] + dt_bias[h]);
        beta[tt * H_v + h] = sigmoid(b[tt * H_v + h]);
      }
    }
    // new conv state: the last n_state_rows rows of x_ext
    for (int r = 0; r < n_state_rows; ++r)
      for (int64_t c = 0; c < conv_dim; ++c)
        st[(int64_t)r * conv_dim + c] = x_ext[(size_t)(len + r) * conv_dim + c];
  });
  return 0;
}

// Sequential per-token recurrence (the definition). Per sequence n and v-head h, with
// k-head hk = h / (H_v/H_k), for each token t in order:
//   S <- exp(g_t) S ;  r = S^T k_t ;  S <- S + beta_t k_t (v_t - r)^T ;  o_t = S^T q_t
//   S  [n_seqs][H_v][d_k][d_v] (row-major, d_v contiguous): initial in, final out.
int oracle_recurrence(int64_t T_total, int n_seqs, const int32_t* cu_seqlens,
                      int H_k, int H_v, int d_k, int d_v,
                      const double* q, const double* k, const double* v,
                      const double* g, const double* beta,
                      double* S, double* o, int n_threads) {
  (void)T_total;
  const int ratio = H_v / H_k;
  run_units(n_seqs * H_v, n_threads, [&](int unit) {
    const int n = unit / H_v, h = unit % H_v, hk = h / ratio;
    double* Sh = S + ((int64_t)n * H_v + h) * d_k * d_v;
    std::vector<double> r(d_v);
    for (int64_t t = cu_seqlens[n]; t < cu_seqlens[n + 1]; ++t) {
      const double* kt = k + (t * H_k + hk) * d_k;
      const double* qt = q + (t * H_k + hk) * d_k;
      const double* vt = v + (t * H_v + h) * d_v;
      const double decay = std::exp(g[t * H_v + h]);
      const double bt = beta[t * H_v + h];
      for (int64_t e = 0; e < (int64_t)d_k * d_v; ++e) Sh[e] *= decay;
      for (int j = 0; j < d_v; ++j) {
        double acc = 0.0;
        for (int i = 0; i < d_k; ++i) acc += Sh[(int64_t)i * d_v + j] * kt[i];
        r[j] = acc;
      }
      for (int i = 0; i < d_k; ++i)
        for (int j = 0; j < d_v; ++j)
          Sh[(int64_t)i * d_v + j] += kt[i] * bt * (vt[j] - r[j]);
      double* ot = o + (t * H_v + h) * d_v;
      for (int j = 0; j < d_v; ++j) {
        double acc = 0.0;
        for (int i = 0; i < d_k; ++i) acc += Sh[(int64_t)i * d_v + j] * qt[i];
        ot[j] = acc;
      }
    }
  });
  return 0;
}

// Chunked restatement in fp64, following the chunk math of the removed single-chunk path
// of the qwen3next page step by step (chunk length C; the last chunk of a sequence may be
// shorter). Same arguments as oracle_recurrence plus C. Used only to pin the identity
// "chunked == recurrent"; the GPU is compared against oracle_recurrence.
int oracle_chunked(int64_t T_total, int n_seqs, const int32_t* cu_seqlens,
                   int H_k, int H_v, int d_k, int d_v,
                   const double* q, const double* k, const double* v,
                   const double* g, const double* beta,
                   double* S, double* o, int C, int n_threads) {
  (void)T_total;
  if (C <= 0) return -1;
  const int ratio = H_v / H_k;
  run_units(n_seqs * H_v, n_threads, [&](int unit) {
    const int n = unit / H_v, h = unit % H_v, hk = h / ratio;
    double* Sh = S + ((int64_t)n * H_v + h) * d_k * d_v;
    std::vector<double> gc(C), A((size_t)C * C), U((size_t)C * d_v), W((size_t)C * d_k),
        P((size_t)C * C), vn((size_t)C * d_v), Snew((size_t)d_k * d_v);
    for (int64_t c0 = cu_seqlens[n]; c0 < cu_seqlens[n + 1]; c0 += C) {
      const int L = (int)std::min<int64_t>(C, cu_seqlens[n + 1] - c0);
      auto K = [&](int i, int d) { return k[((c0 + i) * H_k + hk) * d_k + d]; };
      auto Q = [&](int i, int d) { return q[((c0 + i) * H_k + hk) * d_k + d]; };
      auto V = [&](int i, int j) { return v[((c0 + i) * H_v + h) * d_v + j]; };
      auto B = [&](int i) { return beta[(c0 + i) * H_v + h]; };
      // g_cumsum within the chunk
      double run = 0.0;
      for (int i = 0; i < L; ++i) { run += g[(c0 + i) * H_v + h]; gc[i] = run; }
      // attn = -((k_beta @ k^T) * decay_mask) on the strictly lower triangle
      for (int i = 0; i < L; ++i)
        for (int j = 0; j < L; ++j) {
          double val = 0.0;
          if (j < i) {
            double kk = 0.0;
            for (int d = 0; d < d_k; ++d) kk += B(i) * K(i, d) * K(j, d);
            val = -kk * std::exp(gc[i] - gc[j]);
          }
          A[(size_t)i * C + j] = val;
        }
      // row recursion: attn[i, :i] += sum_m attn[i, m] * attn[m, :i]  (rows m < i already
      // updated), then attn += I.  Result: T = (I - A)^{-1}.
      for (int i = 1; i < L; ++i) {
        std::vector<double> row(i);
        for (int j = 0; j < i; ++j) row[j] = A[(size_t)i * C + j];
        for (int j = 0; j < i; ++j) {
          double acc = 0.0;
          for (int m = 0; m < i; ++m) acc += row[m] * A[(size_t)m * C + j];
          A[(size_t)i * C + j] = row[j] + acc;
        }
      }
      for (int i = 0; i < L; ++i) A[(size_t)i * C + i] += 1.0;
      // value = attn @ (v * beta);  k_cumdecay = attn @ (k * beta * exp(g_cum))
      for (int i = 0; i < L; ++i) {
        for (int j = 0; j < d_v; ++j) {
          double acc = 0.0;
          for (int m = 0; m < L; ++m) acc += A[(size_t)i * C + m] * V(m, j) * B(m);
          U[(size_t)i * d_v + j] = acc;
        }
        for (int d = 0; d < d_k; ++d) {
          double acc = 0.0;
          for (int m = 0; m < L; ++m) acc += A[(size_t)i * C + m] * K(m, d) * B(m) * std::exp(gc[m]);
          W[(size_t)i * d_k + d] = acc;
        }
      }
      // intra-chunk scores: (q @ k^T) * decay_mask, lower triangle including the diagonal
      for (int i = 0; i < L; ++i)
        for (int j = 0; j < L; ++j) {
          double val = 0.0;
          if (j <= i) {
            double qk = 0.0;
            for (int d = 0; d < d_k; ++d) qk += Q(i, d) * K(j, d);
            val = qk * std::exp(gc[i] - gc[j]);
          }
          P[(size_t)i * C + j] = val;
        }
      // v_new = value - k_cumdecay @ S
      for (int i = 0; i < L; ++i)
        for (int j = 0; j < d_v; ++j) {
          double acc = 0.0;
          for (int d = 0; d < d_k; ++d) acc += W[(size_t)i * d_k + d] * Sh[(int64_t)d * d_v + j];
          vn[(size_t)i * d_v + j] = U[(size_t)i * d_v + j] - acc;
        }
      // o = (q * exp(g_cum)) @ S + attn @ v_new
      for (int i = 0; i < L; ++i)
        for (int j = 0; j < d_v; ++j) {
          double inter = 0.0;
          for (int d = 0; d < d_k; ++d) inter += Q(i, d) * std::exp(gc[i]) * Sh[(int64_t)d * d_v + j];
          double intra = 0.0;
          for (int m = 0; m < L; ++m) intra += P[(size_t)i * C + m] * vn[(size_t)m * d_v + j];
          o[((c0 + i) * H_v + h) * d_v + j] = inter + intra;
        }
      // S = S * exp(g_last) + (k * exp(g_last - g_cum))^T @ v_new
      const double gl = gc[L - 1];
      for (int d = 0; d < d_k; ++d)
        for (int j = 0; j < d_v; ++j) {
          double acc = 0.0;
          for (int m = 0; m < L; ++m) acc += K(m, d) * std::exp(gl - gc[m]) * vn[(size_t)m * d_v + j];
          Snew[(size_t)d * d_v + j] = Sh[(int64_t)d * d_v + j] * std::exp(gl) + acc;
        }
      std::memcpy(Sh, Snew.data(), sizeof(double) * d_k * d_v);
    }
  });
  return 0;
}

int oracle_version(void) { return 1; }

}  // extern "C"
