// Plain fp64 CPU oracle for central-difference random-vector gradient
// estimation (CD-RGE) on multi-layer LSTMs, in C++17 with std::thread.
//
// TEST INFRASTRUCTURE ONLY.  Only tests/, __graft_entry__.smoke() and the
// cpu_baseline / --impl reference legs of bench.py may load it.  It shares no
// code with the CUDA library (no header, helper, table or generator) and is an
// implementation of the method independent of the numpy oracle next to it.
//
// Sources ("Scaling Recurrent Neural Networks to a Billion Parameters with
// Zero-Order Optimization", Chaubard & Kochenderfer):
//   pith.science review, "What carries the argument": the update
//     Theta' = Theta - 1/(2 n_pert) sum_i (L(Theta + eps p_i) - L(Theta - eps p_i)) p_i,
//     Rademacher p_i, eta tied to eps; each probe costs two complete forwards.
//   alex-wiki source page, "Method": g_hat = 1/K sum_i (L+_i - L-_i)/(2 eps) u_i,
//     theta' = theta - eta g_hat; reconstructible random seeds.
//   pith.science review, "Circularity Check": the forward difference
//     (L(theta + eps u) - L(theta))/eps u over an antithetic set.
//
// Readings where the pages are silent (the same as the numpy oracle's):
//   1. textbook LSTM, gate blocks i, f, g, o; one bias per layer; h0 = c0 = 0;
//      embedding in front, a linear output layer on the top layer's h;
//   2. natural-log softmax cross-entropy at every step, mean over targets >= 0
//      (0 when nothing is scored);
//   3. every parameter is perturbed; the zero padding between segments is not
//      a parameter;
//   4. p_ij from Philox4x32-10 (Salmon, Moraes, Dror & Shaw, SC'11) with key
//      (seed lo, seed hi), counter (q lo, q hi, i, 0), q = j >> 7; element j
//      reads word (j >> 5) & 3 at bit (e >> 1) + 16 (e & 1), e = j & 31;
//      bit 1 means p = -1;
//   5. eps and eta are fp32 values promoted exactly to double.
//
// Nothing is materialised per probe: every perturbed weight is formed as
// (double)theta_j + s eps p_ij where the forward reads it, so the oracle runs
// models whose fp64 copy would not fit in host memory.  All arithmetic is
// fp64.  Parity: pinned by tests/test_oracle_native.py (known-answer Philox
// vectors, torch fp64 LSTM + cross-entropy, the numpy oracle, closed forms).
#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <thread>
#include <vector>

namespace {

// ---------------------------------------------------------------------------
// Probe signs
// ---------------------------------------------------------------------------
struct Words {
  uint32_t w[4];
};

// Philox4x32-10: ten rounds of
//   (c0, c1, c2, c3) -> (hi(B c2) ^ c1 ^ k0, lo(B c2), hi(A c0) ^ c3 ^ k1, lo(A c0))
// with A = 0xD2511F53, B = 0xCD9E8D57; between rounds the key grows by the
// Weyl increments 0x9E3779B9 (k0) and 0xBB67AE85 (k1).  x: counter in, output out.
void philox_rounds(uint32_t x[4], uint32_t key0, uint32_t key1) {
  for (int round = 0; round < 10; ++round) {
    if (round > 0) {
      key0 += 0x9E3779B9u;
      key1 += 0xBB67AE85u;
    }
    const uint64_t prodA = (uint64_t)0xD2511F53u * x[0];
    const uint64_t prodB = (uint64_t)0xCD9E8D57u * x[2];
    const uint32_t y[4] = {(uint32_t)(prodB >> 32) ^ x[1] ^ key0, (uint32_t)prodB,
                           (uint32_t)(prodA >> 32) ^ x[3] ^ key1, (uint32_t)prodA};
    for (int i = 0; i < 4; ++i) x[i] = y[i];
  }
}

// The four sign words of 128-element block q of a probe: counter
// (q lo, q hi, probe, 0), key (seed lo, seed hi).
Words philox_block(uint64_t seed, uint32_t probe, uint64_t q) {
  Words w{{(uint32_t)q, (uint32_t)(q >> 32), probe, 0u}};
  philox_rounds(w.w, (uint32_t)seed, (uint32_t)(seed >> 32));
  return w;
}

// Bit of element x (0..127) of a block inside its word.
inline int bit_in_word(int x) {
  const int e = x & 31;
  return (e >> 1) + 16 * (e & 1);
}

// p_{probe, j} for j in [j0, j0 + n) as +-1.0 into out[0..n).
void signs(uint64_t seed, uint32_t probe, int64_t j0, int64_t n, double* out) {
  int64_t j = j0;
  while (j < j0 + n) {
    const uint64_t q = (uint64_t)j >> 7;
    const Words w = philox_block(seed, probe, q);
    const int64_t block_end = std::min<int64_t>((int64_t)(q + 1) << 7, j0 + n);
    for (; j < block_end; ++j) {
      const int x = (int)(j & 127);
      const uint32_t bit = (w.w[x >> 5] >> bit_in_word(x)) & 1u;
      out[j - j0] = bit ? -1.0 : 1.0;
    }
  }
}

// ---------------------------------------------------------------------------
// Parameter layout: E[V x E]; per layer W_l[4H x (in_l + H)], b_l[4H];
// W_out[V x H]; b_out[V]; each segment starts on a multiple of 128.
// ---------------------------------------------------------------------------
struct Layout {
  int V = 0, E = 0, H = 0, L = 0;
  int64_t offE = 0, offWout = 0, offbout = 0, d_pad = 0;
  std::vector<int64_t> offW, offb;
  std::vector<int64_t> seg_off, seg_len;
};

Layout make_layout(int V, int E, int H, int L) {
  Layout m;
  m.V = V;
  m.E = E;
  m.H = H;
  m.L = L;
  int64_t off = 0;
  auto take = [&](int64_t len) {
    const int64_t at = off;
    m.seg_off.push_back(at);
    m.seg_len.push_back(len);
    off += len;
    off = (off + 127) / 128 * 128;
    return at;
  };
  m.offE = take((int64_t)V * E);
  for (int l = 0; l < L; ++l) {
    const int64_t in = l == 0 ? E : H;
    m.offW.push_back(take(4LL * H * (in + H)));
    m.offb.push_back(take(4LL * H));
  }
  m.offWout = take((int64_t)V * H);
  m.offbout = take((int64_t)V);
  m.d_pad = off;
  return m;
}

// Run body(begin, end) over [0, n) on up to `threads` std::threads.
template <class F>
void parallel_for(int64_t n, int threads, F&& body) {
  if (n <= 0) return;
  const int nt = (int)std::max<int64_t>(1, std::min<int64_t>(threads, n));
  if (nt == 1) {
    body((int64_t)0, n);
    return;
  }
  std::vector<std::thread> pool;
  pool.reserve(nt);
  for (int t = 0; t < nt; ++t) {
    const int64_t b = n * t / nt, e = n * (t + 1) / nt;
    pool.emplace_back([=, &body] { body(b, e); });
  }
  for (auto& th : pool) th.join();
}

// One perturbed point Theta + s eps p_probe, read element by element.
struct Point {
  const float* theta;
  uint64_t seed;
  uint32_t probe;
  double s_eps;  // s * eps (0 for the unperturbed point)
  // out[k] = theta_j + s eps p_j for j = j0 + k, k < n
  void read(int64_t j0, int64_t n, double* out) const {
    if (s_eps == 0.0) {
      for (int64_t k = 0; k < n; ++k) out[k] = (double)theta[j0 + k];
      return;
    }
    const double step[2] = {s_eps, -s_eps};  // sign bit 0: p = +1, 1: p = -1
    int64_t j = j0;
    const int64_t end = j0 + n;
    while (j < end) {
      const uint64_t q = (uint64_t)j >> 7;
      const Words w = philox_block(seed, probe, q);
      const int64_t block_end = std::min<int64_t>((int64_t)(q + 1) << 7, end);
      for (; j < block_end; ++j) {
        const int x = (int)(j & 127);
        const uint32_t bit = (w.w[x >> 5] >> bit_in_word(x)) & 1u;
        out[j - j0] = (double)theta[j] + step[bit];
      }
    }
  }
};

inline double sigmoid(double x) { return 1.0 / (1.0 + std::exp(-x)); }

// Complete forward of rows [tokens/targets: nb x T] at one perturbed point:
// embedding -> L LSTM layers -> linear -> softmax cross-entropy at every step.
// row_loss[b] = sum over scored steps of the row's cross-entropy,
// row_count[b] = number of scored steps.
void forward(const Layout& m, const Point& pt, const int32_t* tokens, const int32_t* targets,
             int nb, int T, int threads, double* row_loss, int64_t* row_count) {
  const int H = m.H, E = m.E, V = m.V, L = m.L;
  std::vector<std::vector<double>> h(L, std::vector<double>((size_t)nb * H, 0.0));
  std::vector<std::vector<double>> c(L, std::vector<double>((size_t)nb * H, 0.0));
  std::vector<double> x((size_t)nb * std::max(E, H));
  std::vector<double> G((size_t)nb * 4 * H);
  std::vector<double> z((size_t)nb * V);
  std::vector<double> row;
  for (int b = 0; b < nb; ++b) {
    row_loss[b] = 0.0;
    row_count[b] = 0;
  }
  for (int t = 0; t < T; ++t) {
    // x_t = E[token] (perturbed)
    for (int b = 0; b < nb; ++b) {
      const int tok = tokens[(int64_t)b * T + t];
      pt.read(m.offE + (int64_t)tok * E, E, &x[(size_t)b * E]);
    }
    int in = E;
    for (int l = 0; l < L; ++l) {
      const int K = in + H;
      // a[k][b] = [x_t | h_{t-1}] (column layout so the row loop below runs
      // over independent batch rows)
      std::vector<double> a((size_t)K * nb);
      for (int b = 0; b < nb; ++b) {
        for (int k = 0; k < in; ++k) a[(size_t)k * nb + b] = x[(size_t)b * in + k];
        for (int k = 0; k < H; ++k) a[(size_t)(in + k) * nb + b] = h[l][(size_t)b * H + k];
      }
      // G[b][r] = b_l[r] + sum_k a[k][b] W_l[r][k]
      const int64_t offW = m.offW[l], offb = m.offb[l];
      const int64_t macs = 4LL * H * K * nb;
      parallel_for(4LL * H, macs >= (1 << 22) ? threads : 1, [&](int64_t r0, int64_t r1) {
        std::vector<double> w(K), acc(nb);
        double bias;
        for (int64_t r = r0; r < r1; ++r) {
          pt.read(offW + r * K, K, w.data());
          pt.read(offb + r, 1, &bias);
          for (int b = 0; b < nb; ++b) acc[b] = 0.0;
          for (int k = 0; k < K; ++k) {
            const double wk = w[k];
            const double* ak = &a[(size_t)k * nb];
            for (int b = 0; b < nb; ++b) acc[b] += ak[b] * wk;
          }
          for (int b = 0; b < nb; ++b) G[(size_t)b * 4 * H + r] = acc[b] + bias;
        }
      });
      // gates i, f, g, o and the state update
      for (int b = 0; b < nb; ++b) {
        const double* g = &G[(size_t)b * 4 * H];
        for (int u = 0; u < H; ++u) {
          const double ig = sigmoid(g[u]);
          const double fg = sigmoid(g[H + u]);
          const double gg = std::tanh(g[2 * H + u]);
          const double og = sigmoid(g[3 * H + u]);
          double& cs = c[l][(size_t)b * H + u];
          cs = fg * cs + ig * gg;
          h[l][(size_t)b * H + u] = og * std::tanh(cs);
        }
      }
      for (size_t i = 0; i < (size_t)nb * H; ++i) x[i] = h[l][i];
      in = H;
    }
    // logits z[b][v] = b_out[v] + sum_k h_top[b][k] W_out[v][k]
    row.resize(H);
    for (int v = 0; v < V; ++v) {
      double bias;
      pt.read(m.offWout + (int64_t)v * H, H, row.data());
      pt.read(m.offbout + v, 1, &bias);
      for (int b = 0; b < nb; ++b) {
        double s = 0.0;
        for (int k = 0; k < H; ++k) s += x[(size_t)b * H + k] * row[k];
        z[(size_t)b * V + v] = s + bias;
      }
    }
    for (int b = 0; b < nb; ++b) {
      const int tg = targets[(int64_t)b * T + t];
      if (tg < 0) continue;
      const double* zb = &z[(size_t)b * V];
      double mx = zb[0];
      for (int v = 1; v < V; ++v) mx = std::max(mx, zb[v]);
      double se = 0.0;
      for (int v = 0; v < V; ++v) se += std::exp(zb[v] - mx);
      row_loss[b] += mx + std::log(se) - zb[tg];
      row_count[b] += 1;
    }
  }
}

int check_inputs(const Layout& m, const int32_t* tokens, const int32_t* targets, int B, int T) {
  for (int64_t i = 0; i < (int64_t)B * T; ++i) {
    if (tokens[i] < 0 || tokens[i] >= m.V) return 2;
    if (targets[i] < -1 || targets[i] >= m.V) return 2;
  }
  return 0;
}

}  // namespace

extern "C" {

// Padded length of theta for the spec.
int64_t zoo_d_pad(int V, int E, int H, int L) { return make_layout(V, E, H, L).d_pad; }

// The raw Philox4x32-10 block of counter (c0, c1, c2, c3) and key (k0, k1)
// (for checking against published known-answer vectors).
void zoo_philox4x32_10(uint32_t c0, uint32_t c1, uint32_t c2, uint32_t c3, uint32_t k0,
                       uint32_t k1, uint32_t* out) {
  uint32_t x[4] = {c0, c1, c2, c3};
  philox_rounds(x, k0, k1);
  for (int i = 0; i < 4; ++i) out[i] = x[i];
}

// Philox words of blocks q0 .. q0 + n - 1 of one probe: out[4 k + w].
void zoo_sign_words(uint64_t seed, uint32_t probe, uint64_t q0, int64_t n, uint32_t* out) {
  for (int64_t k = 0; k < n; ++k) {
    const Words w = philox_block(seed, probe, q0 + (uint64_t)k);
    for (int i = 0; i < 4; ++i) out[4 * k + i] = w.w[i];
  }
}

// p_{probe, j} for j in [j0, j0 + n) as int8 +-1.
void zoo_signs(uint64_t seed, uint32_t probe, int64_t j0, int64_t n, int8_t* out) {
  std::vector<double> s((size_t)n);
  signs(seed, probe, j0, n, s.data());
  for (int64_t k = 0; k < n; ++k) out[k] = s[k] > 0 ? 1 : -1;
}

// Per-row losses of probes probes[0..n_probes) at both signs over batch rows
// rows[0..n_rows) (all B rows if rows is null):
//   row_loss[(2 p + s) n_rows + r] for s = 0 (+eps), 1 (-eps);
//   row_count[r] = scored steps of row r.
// eps == 0 evaluates the unperturbed point (both signs equal L(theta)).
// Returns 0, or 1 (bad spec / arguments), 2 (token or target out of range).
int zoo_probe_row_losses(const float* theta, int V, int E, int H, int L, uint64_t seed,
                         const int32_t* probes, int n_probes, float eps, const int32_t* tokens,
                         const int32_t* targets, int B, int T, const int32_t* rows, int n_rows,
                         int threads, double* row_loss, int64_t* row_count) {
  if (!theta || V < 2 || E < 1 || H < 1 || L < 1 || B < 1 || T < 1 || n_probes < 0 ||
      threads < 1)
    return 1;
  const Layout m = make_layout(V, E, H, L);
  if (check_inputs(m, tokens, targets, B, T)) return 2;
  const int nb = rows ? n_rows : B;
  std::vector<int32_t> tok((size_t)nb * T), tgt((size_t)nb * T);
  for (int r = 0; r < nb; ++r) {
    const int b = rows ? rows[r] : r;
    if (b < 0 || b >= B) return 1;
    std::memcpy(&tok[(size_t)r * T], tokens + (int64_t)b * T, sizeof(int32_t) * T);
    std::memcpy(&tgt[(size_t)r * T], targets + (int64_t)b * T, sizeof(int32_t) * T);
  }
  const double e = (double)eps;
  const int units = 2 * n_probes;
  // per-unit work; small models run whole units in parallel, large ones
  // split each unit's gate rows over the threads
  double macs = (double)V * H;
  for (int l = 0; l < L; ++l) macs += 4.0 * H * ((l == 0 ? E : H) + H);
  macs *= (double)nb * T;
  const bool by_unit = macs < 5e7 && units > 1;
  std::vector<std::vector<int64_t>> counts(units, std::vector<int64_t>(nb));
  auto run_unit = [&](int u, int th) {
    const Point pt{theta, seed, (uint32_t)probes[u / 2], (u & 1) ? -e : e};
    forward(m, pt, tok.data(), tgt.data(), nb, T, th, row_loss + (size_t)u * nb,
            counts[u].data());
  };
  if (by_unit) {
    std::atomic<int> next{0};
    parallel_for(std::min(threads, units), threads, [&](int64_t, int64_t) {
      for (int u = next++; u < units; u = next++) run_unit(u, 1);
    });
  } else {
    for (int u = 0; u < units; ++u) run_unit(u, threads);
  }
  if (row_count) {
    if (units > 0) {
      for (int r = 0; r < nb; ++r) row_count[r] = counts[0][r];
    } else {
      for (int r = 0; r < nb; ++r) {
        row_count[r] = 0;
        for (int t = 0; t < T; ++t) row_count[r] += tgt[(size_t)r * T + t] >= 0;
      }
    }
  }
  return 0;
}

// c_i = eta (L+_i - L-_i) / (2 eps n_pert)  (alex-wiki "Method").
void zoo_coefficients(const double* lp, const double* lm, int n, float eps, float eta,
                      double* out) {
  for (int i = 0; i < n; ++i) out[i] = (double)eta * (lp[i] - lm[i]) / (2.0 * (double)eps * n);
}

// Forward-difference coefficients c_i = eta (L+_i - L0) / (eps n_pert).
void zoo_coefficients_forward(const double* lp, double l0, int n, float eps, float eta,
                              double* out) {
  for (int i = 0; i < n; ++i) out[i] = (double)eta * (lp[i] - l0) / ((double)eps * n);
}

int zoo_update_range(const float* theta, int V, int E, int H, int L, uint64_t seed, int n_pert,
                     const double* coeffs, int64_t j0, int64_t j1, int threads, double* out);

// theta'_j = theta_j - sum_i c_i p_ij for the elements index[0..n_index), or
// for all d_pad elements when index is null (padding copied unchanged).
// out: fp64 [n_index] or [d_pad].  Returns 1 on bad arguments.
int zoo_update(const float* theta, int V, int E, int H, int L, uint64_t seed, int n_pert,
               const double* coeffs, const int64_t* index, int64_t n_index, int threads,
               double* out) {
  if (!theta || !coeffs || !out || n_pert < 0 || threads < 1) return 1;
  const Layout m = make_layout(V, E, H, L);
  if (index) {
    for (int64_t k = 0; k < n_index; ++k)
      if (index[k] < 0 || index[k] >= m.d_pad) return 1;
    parallel_for(n_index, n_index >= 4096 ? threads : 1, [&](int64_t k0, int64_t k1) {
      for (int64_t k = k0; k < k1; ++k) {
        const int64_t j = index[k];
        double acc = 0.0, p;
        for (int i = 0; i < n_pert; ++i) {
          signs(seed, (uint32_t)i, j, 1, &p);
          acc += coeffs[i] * p;
        }
        out[k] = (double)theta[j] - acc;
      }
    });
    return 0;
  }
  return zoo_update_range(theta, V, E, H, L, seed, n_pert, coeffs, 0, m.d_pad, threads, out);
}

// theta'_j for the contiguous elements j0 <= j < j1 (out: fp64 [j1 - j0];
// padding copied unchanged).  Returns 1 on bad arguments.
int zoo_update_range(const float* theta, int V, int E, int H, int L, uint64_t seed, int n_pert,
                     const double* coeffs, int64_t j0_all, int64_t j1_all, int threads,
                     double* out) {
  const Layout m = make_layout(V, E, H, L);
  if (!theta || !coeffs || !out || n_pert < 0 || threads < 1 || j0_all < 0 || j1_all > m.d_pad ||
      j0_all > j1_all)
    return 1;
  for (int64_t j = j0_all; j < j1_all; ++j) out[j - j0_all] = (double)theta[j];
  for (size_t s = 0; s < m.seg_off.size(); ++s) {
    const int64_t off = std::max(m.seg_off[s], j0_all);
    const int64_t len = std::min(m.seg_off[s] + m.seg_len[s], j1_all) - off;
    if (len <= 0) continue;
    const int64_t nblk = (len + 4095) / 4096;
    parallel_for(nblk, nblk >= 4 ? threads : 1, [&](int64_t b0, int64_t b1) {
      std::vector<double> p(4096);
      for (int64_t blk = b0; blk < b1; ++blk) {
        const int64_t j0 = off + blk * 4096;
        const int64_t n = std::min<int64_t>(4096, off + len - j0);
        for (int i = 0; i < n_pert; ++i) {
          signs(seed, (uint32_t)i, j0, n, p.data());
          for (int64_t k = 0; k < n; ++k) out[j0 - j0_all + k] -= coeffs[i] * p[k];
        }
      }
    });
  }
  return 0;
}

// Gram matrix of the probes over the real parameters:
// G[a][b] = sum_j p_{probes[a], j} p_{probes[b], j} = d_real - 2 #(j : signs differ).
int zoo_probe_gram(int V, int E, int H, int L, uint64_t seed, const int32_t* probes, int n,
                   int threads, double* gram) {
  if (n < 0 || threads < 1) return 1;
  const Layout m = make_layout(V, E, H, L);
  int64_t d_real = 0;
  for (int64_t len : m.seg_len) d_real += len;
  std::vector<std::vector<int64_t>> diff_parts(threads, std::vector<int64_t>((size_t)n * n, 0));
  for (size_t s = 0; s < m.seg_off.size(); ++s) {
    const int64_t q0 = m.seg_off[s] >> 7;
    const int64_t nq = (m.seg_len[s] + 127) >> 7;
    const int64_t len = m.seg_len[s];
    std::atomic<int> slot{0};
    parallel_for(nq, nq >= 64 ? threads : 1, [&](int64_t a0, int64_t a1) {
      std::vector<int64_t>& diff = diff_parts[slot++];
      std::vector<Words> w(n);
      for (int64_t qq = a0; qq < a1; ++qq) {
        // bits of the block that hold real elements (a segment's last block
        // may be partly padding)
        uint32_t mask[4] = {0u, 0u, 0u, 0u};
        const int64_t n_real = std::min<int64_t>(128, len - qq * 128);
        for (int x = 0; x < n_real; ++x) mask[x >> 5] |= 1u << bit_in_word(x);
        for (int a = 0; a < n; ++a) w[a] = philox_block(seed, (uint32_t)probes[a], q0 + qq);
        for (int a = 0; a < n; ++a)
          for (int b = a + 1; b < n; ++b) {
            int64_t d = 0;
            for (int i = 0; i < 4; ++i)
              d += __builtin_popcount((w[a].w[i] ^ w[b].w[i]) & mask[i]);
            diff[(size_t)a * n + b] += d;
          }
      }
    });
  }
  for (int a = 0; a < n; ++a)
    for (int b = 0; b < n; ++b) {
      if (a == b) {
        gram[(size_t)a * n + b] = (double)d_real;
        continue;
      }
      const int lo = std::min(a, b), hi = std::max(a, b);
      int64_t d = 0;
      for (auto& part : diff_parts) d += part[(size_t)lo * n + hi];
      gram[(size_t)a * n + b] = (double)(d_real - 2 * d);
    }
  return 0;
}

}  // extern "C"
