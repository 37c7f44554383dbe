// Offline weight transform on the host, in float64.
//
// SVDQuant (paperlayer.ai summary of arXiv 2411.05007v4):
//  * smoothing (§4.2; App. D, following SmoothQuant): per input channel j,
//    lam_j = act_absmax_j^alpha / max_n |W_nj|^(1-alpha); lam_j = 1 when either
//    maximum is 0.  The runtime multiplies activations by inv_lam = fp32(1/lam);
//    the smoothed weight is W_hat = W diag(1/inv_lam).
//  * low-rank split (§4.2): the top-r singular triplets of W_hat.  Computed by
//    randomized subspace iteration with Rayleigh-Ritz (Halko, Martinsson and
//    Tropp, "Finding structure with randomness", 2011, Alg. 4.4 + 5.1): a
//    Gaussian start of r + p columns, q rounds of W_hat^T / W_hat products with
//    re-orthonormalization, then the exact SVD of the small projected matrix
//    through the eigen-decomposition of B B^T (cyclic Jacobi).
//  * factors: L1 = U_r S_r (K x r), L2 = V_r^T (r x N); stored as
//    L1' = bf16(diag(inv_lam) L1) and L2b = bf16(L2); the residual absorbs the
//    factor rounding: R = W_hat - (diag(1/inv_lam) L1' L2b)^T.
//  * refinement (§4.2: the split can be refined over several iterations; the
//    formula is a reading): with Q(R) = alpha_w * (R / alpha_w quantized to
//    NVFP4 and dequantized), L_{t+1} = SVD_r(W_hat - Q(W_hat - L_t)); the split
//    with the smallest ||R - Q(R)||_F among the iterations tried is kept.
#include <algorithm>
#include <cmath>
#include <cstring>
#include <functional>
#include <random>
#include <thread>
#include <vector>

#include "svdq_internal.h"

namespace svdq {

uint16_t f32_to_bf16_rne(float x) {
  uint32_t u;
  std::memcpy(&u, &x, 4);
  if ((u & 0x7F800000u) == 0x7F800000u) return static_cast<uint16_t>(u >> 16);  // inf/nan
  u += 0x7FFFu + ((u >> 16) & 1u);
  return static_cast<uint16_t>(u >> 16);
}

float bf16_to_f32(uint16_t b) {
  const uint32_t u = static_cast<uint32_t>(b) << 16;
  float f;
  std::memcpy(&f, &u, 4);
  return f;
}

float weight_factor(const float* R, size_t n) {
  double m = 0.0;
  for (size_t i = 0; i < n; ++i) m = std::max(m, std::fabs(static_cast<double>(R[i])));
  if (m == 0.0) return 1.0f;
  int e = 0;
  const double frac = std::frexp(m / (6.0 * 448.0), &e);  // m' = frac * 2^e, frac in [0.5, 1)
  const int c = frac == 0.5 ? e - 1 : e;                  // ceil(log2(m'))
  return static_cast<float>(std::ldexp(1.0, c));
}

// INT4 codec (SVDQuant App. D: groups of 64 with 16-bit scales; §3: qmax 7):
// s = bf16(fp32(amax / 7)), q = clamp(rint(fp32(v * fp32(1 / s))), -7, 7) with
// round-half-even, two's-complement nibbles, per 8 elements one little-endian
// word with the even elements in nibbles 0-3 and the odd ones in nibbles 4-7.
// IEEE fp32 host arithmetic (no contraction across the steps).
void int4_encode_rows(const float* R, int rows, int K, int rows_pad, uint8_t* codes, uint16_t* scales) {
  const int G = K / 64;
  for (int n = 0; n < rows; ++n) {
    const float* v = R + static_cast<size_t>(n) * K;
    uint8_t* c = codes + static_cast<size_t>(n) * (K / 2);
    for (int g = 0; g < G; ++g) {
      float amax = 0.0f;
      for (int j = 0; j < 64; ++j) amax = std::max(amax, std::fabs(v[64 * g + j]));
      volatile float q7 = amax / 7.0f;  // one fp32 rounding before the bf16 one
      const uint16_t sb = f32_to_bf16_rne(q7);
      scales[static_cast<size_t>(g) * rows_pad + n] = sb;
      const float sv = bf16_to_f32(sb);
      volatile float r = sv > 0.0f ? 1.0f / sv : 0.0f;
      for (int j = 0; j < 64; j += 8) {
        uint32_t word = 0;
        for (int e = 0; e < 8; ++e) {
          volatile float t = v[64 * g + j + e] * r;
          const int q = std::min(7, std::max(-7, static_cast<int>(std::nearbyint(t))));
          word |= (static_cast<uint32_t>(q) & 0xFu) << (4 * ((e & 1) ? 4 + (e >> 1) : (e >> 1)));
        }
        for (int b = 0; b < 4; ++b) c[32 * g + j / 2 + b] = static_cast<uint8_t>(word >> (8 * b));
      }
    }
  }
}

namespace {

void parallel_for(long n, const std::function<void(long, long)>& body) {
  const long hw = std::max(1u, std::thread::hardware_concurrency());
  const long nt = std::max(1L, std::min(hw, n / 4 + 1));
  if (nt == 1) {
    body(0, n);
    return;
  }
  std::vector<std::thread> ts;
  const long chunk = (n + nt - 1) / nt;
  for (long t = 0; t < nt; ++t) {
    const long b = t * chunk, e = std::min(n, b + chunk);
    if (b < e) ts.emplace_back(body, b, e);
  }
  for (auto& t : ts) t.join();
}

// Y[N x l] = A[N x K] * X[K x l]   (all row-major)
void mul_a_x(const std::vector<double>& A, int N, int K, const std::vector<double>& X, int l,
             std::vector<double>& Y) {
  Y.assign(static_cast<size_t>(N) * l, 0.0);
  parallel_for(N, [&](long b, long e) {
    std::vector<double> acc(l);
    for (long n = b; n < e; ++n) {
      std::fill(acc.begin(), acc.end(), 0.0);
      const double* a = &A[static_cast<size_t>(n) * K];
      for (int k = 0; k < K; ++k) {
        const double w = a[k];
        const double* x = &X[static_cast<size_t>(k) * l];
        for (int j = 0; j < l; ++j) acc[j] += w * x[j];
      }
      std::copy(acc.begin(), acc.end(), &Y[static_cast<size_t>(n) * l]);
    }
  });
}

// Z[K x l] = A^T[K x N] * Q[N x l]
void mul_at_q(const std::vector<double>& A, int N, int K, const std::vector<double>& Q, int l,
              std::vector<double>& Z) {
  Z.assign(static_cast<size_t>(K) * l, 0.0);
  parallel_for(K, [&](long b, long e) {
    for (int n = 0; n < N; ++n) {
      const double* a = &A[static_cast<size_t>(n) * K];
      const double* q = &Q[static_cast<size_t>(n) * l];
      for (long k = b; k < e; ++k) {
        const double w = a[k];
        if (w == 0.0) continue;
        double* z = &Z[static_cast<size_t>(k) * l];
        for (int j = 0; j < l; ++j) z[j] += w * q[j];
      }
    }
  });
}

// Orthonormalizes the l columns of a row-major [rows x l] matrix in place
// (modified Gram-Schmidt, applied twice for stability).
void orthonormalize(std::vector<double>& M, int rows, int l) {
  std::vector<double> c(static_cast<size_t>(l) * rows);
  for (int i = 0; i < rows; ++i)
    for (int j = 0; j < l; ++j) c[static_cast<size_t>(j) * rows + i] = M[static_cast<size_t>(i) * l + j];
  for (int pass = 0; pass < 2; ++pass) {
    for (int j = 0; j < l; ++j) {
      double* cj = &c[static_cast<size_t>(j) * rows];
      for (int p = 0; p < j; ++p) {
        const double* cp = &c[static_cast<size_t>(p) * rows];
        double d = 0.0;
        for (int i = 0; i < rows; ++i) d += cp[i] * cj[i];
        for (int i = 0; i < rows; ++i) cj[i] -= d * cp[i];
      }
      double nrm = 0.0;
      for (int i = 0; i < rows; ++i) nrm += cj[i] * cj[i];
      nrm = std::sqrt(nrm);
      const double inv = nrm > 0.0 ? 1.0 / nrm : 0.0;
      for (int i = 0; i < rows; ++i) cj[i] *= inv;
    }
  }
  for (int i = 0; i < rows; ++i)
    for (int j = 0; j < l; ++j) M[static_cast<size_t>(i) * l + j] = c[static_cast<size_t>(j) * rows + i];
}

// Cyclic Jacobi eigen-decomposition of a symmetric [n x n] matrix G (row-major).
// On return d holds the eigenvalues (descending) and E the matching
// eigenvectors as columns.
void jacobi_eigen(std::vector<double> G, int n, std::vector<double>& d, std::vector<double>& E) {
  E.assign(static_cast<size_t>(n) * n, 0.0);
  for (int i = 0; i < n; ++i) E[static_cast<size_t>(i) * n + i] = 1.0;
  auto g = [&](int i, int j) -> double& { return G[static_cast<size_t>(i) * n + j]; };
  for (int sweep = 0; sweep < 100; ++sweep) {
    double off = 0.0, diag = 0.0;
    for (int i = 0; i < n; ++i) {
      diag += g(i, i) * g(i, i);
      for (int j = i + 1; j < n; ++j) off += g(i, j) * g(i, j);
    }
    if (off <= 1e-30 * diag || off == 0.0) break;
    for (int p = 0; p < n; ++p) {
      for (int q = p + 1; q < n; ++q) {
        const double apq = g(p, q);
        if (std::fabs(apq) < 1e-300) continue;
        const double theta = (g(q, q) - g(p, p)) / (2.0 * apq);
        const double t = (theta >= 0 ? 1.0 : -1.0) / (std::fabs(theta) + std::sqrt(theta * theta + 1.0));
        const double c = 1.0 / std::sqrt(t * t + 1.0), s = t * c;
        for (int k = 0; k < n; ++k) {  // G <- J^T G J
          const double gkp = g(k, p), gkq = g(k, q);
          g(k, p) = c * gkp - s * gkq;
          g(k, q) = s * gkp + c * gkq;
        }
        for (int k = 0; k < n; ++k) {
          const double gpk = g(p, k), gqk = g(q, k);
          g(p, k) = c * gpk - s * gqk;
          g(q, k) = s * gpk + c * gqk;
        }
        for (int k = 0; k < n; ++k) {
          double* e = &E[static_cast<size_t>(k) * n];
          const double ekp = e[p], ekq = e[q];
          e[p] = c * ekp - s * ekq;
          e[q] = s * ekp + c * ekq;
        }
      }
    }
  }
  std::vector<int> order(n);
  for (int i = 0; i < n; ++i) order[i] = i;
  std::sort(order.begin(), order.end(), [&](int a, int b) { return g(a, a) > g(b, b); });
  d.resize(n);
  std::vector<double> Es(static_cast<size_t>(n) * n);
  for (int j = 0; j < n; ++j) {
    d[j] = g(order[j], order[j]);
    for (int k = 0; k < n; ++k) Es[static_cast<size_t>(k) * n + j] = E[static_cast<size_t>(k) * n + order[j]];
  }
  E.swap(Es);
}

// Top-r split of A (N x K) by randomized subspace iteration, 16-bit factors
// (the smoothing multipliers folded into L1'), and the residual of W_hat that
// the stored factors leave, R = W_hat - (diag(1/inv_lam) L1' L2b)^T in fp32.
void split_round_residual(const std::vector<double>& Wh, const std::vector<double>& A, int N, int K,
                          const svdq_prepare_opts& o, const std::vector<float>& inv_lam, std::vector<uint16_t>* L1p_out,
                          std::vector<uint16_t>* L2_out, std::vector<float>* R_out) {
  const int r = o.rank;
  (*L1p_out).assign(static_cast<size_t>(K) * r, 0);
  (*L2_out).assign(static_cast<size_t>(r) * N, 0);
  std::vector<double> L1s(static_cast<size_t>(K) * r, 0.0), L2d(static_cast<size_t>(r) * N, 0.0);
  if (r > 0) {
    // ---- randomized subspace iteration
    const int l = std::min(r + std::max(0, o.oversample), std::min(N, K));
    std::mt19937_64 gen(o.seed);
    std::normal_distribution<double> nd(0.0, 1.0);
    std::vector<double> Om(static_cast<size_t>(K) * l);
    for (auto& v : Om) v = nd(gen);
    std::vector<double> Y, Z, Q;
    mul_a_x(A, N, K, Om, l, Y);
    orthonormalize(Y, N, l);
    for (int it = 0; it < std::max(0, o.power_iters); ++it) {
      mul_at_q(A, N, K, Y, l, Z);
      orthonormalize(Z, K, l);
      mul_a_x(A, N, K, Z, l, Y);
      orthonormalize(Y, N, l);
    }
    Q.swap(Y);                       // N x l, orthonormal columns
    mul_at_q(A, N, K, Q, l, Z);     // Z = A^T Q = B^T  (K x l)
    // ---- Rayleigh-Ritz: eigen-decomposition of B B^T = Z^T Z (l x l)
    std::vector<double> G(static_cast<size_t>(l) * l, 0.0);
    for (int a = 0; a < l; ++a)
      for (int b = a; b < l; ++b) {
        double s = 0.0;
        for (int k = 0; k < K; ++k) s += Z[static_cast<size_t>(k) * l + a] * Z[static_cast<size_t>(k) * l + b];
        G[static_cast<size_t>(a) * l + b] = G[static_cast<size_t>(b) * l + a] = s;
      }
    std::vector<double> d, E;
    jacobi_eigen(G, l, d, E);
    // L2 = (Q E_r)^T, L1 = B^T E_r = Z E_r
    for (int i = 0; i < r; ++i) {
      for (int n = 0; n < N; ++n) {
        double s = 0.0;
        for (int a = 0; a < l; ++a) s += Q[static_cast<size_t>(n) * l + a] * E[static_cast<size_t>(a) * l + i];
        L2d[static_cast<size_t>(i) * N + n] = s;
      }
      for (int k = 0; k < K; ++k) {
        double s = 0.0;
        for (int a = 0; a < l; ++a) s += Z[static_cast<size_t>(k) * l + a] * E[static_cast<size_t>(a) * l + i];
        L1s[static_cast<size_t>(k) * r + i] = s;
      }
    }
    // ---- 16-bit factors; the residual uses them as the runtime does
    for (int k = 0; k < K; ++k)
      for (int i = 0; i < r; ++i) {
        const double v = static_cast<double>(inv_lam[k]) * L1s[static_cast<size_t>(k) * r + i];
        const uint16_t b = f32_to_bf16_rne(static_cast<float>(v));
        (*L1p_out)[static_cast<size_t>(k) * r + i] = b;
        L1s[static_cast<size_t>(k) * r + i] = static_cast<double>(bf16_to_f32(b)) / static_cast<double>(inv_lam[k]);
      }
    for (size_t i = 0; i < L2d.size(); ++i) {
      const uint16_t b = f32_to_bf16_rne(static_cast<float>(L2d[i]));
      (*L2_out)[i] = b;
      L2d[i] = bf16_to_f32(b);
    }
  }
  (*R_out).resize(static_cast<size_t>(N) * K);
  parallel_for(N, [&](long b, long e) {
    std::vector<double> l2n(std::max(r, 1));
    for (long n = b; n < e; ++n) {
      for (int i = 0; i < r; ++i) l2n[i] = L2d[static_cast<size_t>(i) * N + n];
      for (int k = 0; k < K; ++k) {
        double low = 0.0;
        const double* l1 = &L1s[static_cast<size_t>(k) * r];
        for (int i = 0; i < r; ++i) low += l1[i] * l2n[i];
        (*R_out)[static_cast<size_t>(n) * K + k] = static_cast<float>(Wh[static_cast<size_t>(n) * K + k] - low);
      }
    }
  });
}

// NVFP4 round trip of one fp32 value set as the runtime sees it:
// E4M3 (round to nearest even, saturating) of a non-negative x, as a value.
double e4m3_rne_sat(double x) {
  if (x >= 448.0) return 448.0;
  if (x < 0.015625) return std::nearbyint(x * 512.0) / 512.0;  // subnormals: steps of 2^-9
  int ex = 0;
  std::frexp(x, &ex);                                             // x = f 2^ex, f in [0.5, 1)
  const double step = std::ldexp(1.0, ex - 4);                   // 3 mantissa bits
  return std::nearbyint(x / step) * step;
}
// E2M1 (round to nearest even on {0, .5, 1, 1.5, 2, 3, 4, 6}, saturating), as a value.
double e2m1_rne_sat(double v) {
  const double a = std::fabs(v);
  double q;
  if (a >= 6.0) q = 6.0;
  else if (a < 2.0) q = std::nearbyint(a * 2.0) / 2.0;
  else if (a < 4.0) q = std::nearbyint(a);
  else q = std::nearbyint(a / 2.0) * 2.0;
  return v < 0 ? -q : q;
}

// ||R - Q(R)||_F with Q(R) = alpha_w * NVFP4 round trip of R / alpha_w (groups of
// 16 along K: s = E4M3(fp32(amax / 6)), codes E2M1(fp32(v * fp32(1 / s))));
// writes Q(R) (float64, N x K) to *Q if given.
double fake_quant_error(const std::vector<float>& R, int N, int K, std::vector<double>* Q) {
  const float aw = weight_factor(R.data(), R.size());
  if (Q) Q->assign(R.size(), 0.0);
  std::vector<double> part(static_cast<size_t>(N), 0.0);
  parallel_for(N, [&](long b, long e) {
    for (long n = b; n < e; ++n) {
      double acc = 0.0;
      for (int g = 0; g < K; g += 16) {
        const float* row = &R[static_cast<size_t>(n) * K + g];
        float v[16], amax = 0.0f;
        for (int i = 0; i < 16; ++i) {
          v[i] = row[i] / aw;  // exact: aw is a power of two
          amax = std::max(amax, std::fabs(v[i]));
        }
        const double s = e4m3_rne_sat(static_cast<double>(amax / 6.0f));
        const float rs = s > 0.0 ? 1.0f / static_cast<float>(s) : 0.0f;
        for (int i = 0; i < 16; ++i) {
          const double deq = s > 0.0 ? e2m1_rne_sat(static_cast<double>(v[i] * rs)) * s * aw : 0.0;
          const double d = static_cast<double>(row[i]) - deq;
          acc += d * d;
          if (Q) (*Q)[static_cast<size_t>(n) * K + g + i] = deq;
        }
      }
      part[n] = acc;
    }
  });
  double tot = 0.0;
  for (double x : part) tot += x;
  return std::sqrt(tot);
}

}  // namespace

svdq_status host_prepare_split(const uint16_t* W_bf16, const float* act_absmax, int N, int K,
                               const svdq_prepare_opts& o, HostSplit* out) {
  const int r = o.rank;
  // ---- smoothing
  std::vector<double> wmax(K, 0.0);
  for (int n = 0; n < N; ++n)
    for (int k = 0; k < K; ++k)
      wmax[k] = std::max(wmax[k], std::fabs(static_cast<double>(bf16_to_f32(W_bf16[static_cast<size_t>(n) * K + k]))));
  out->inv_lam.resize(K);
  for (int k = 0; k < K; ++k) {
    const double ax = act_absmax[k];
    double lam = 1.0;
    if (ax > 0.0 && wmax[k] > 0.0) lam = std::pow(ax, static_cast<double>(o.alpha)) / std::pow(wmax[k], 1.0 - o.alpha);
    const float lam32 = static_cast<float>(lam);
    out->inv_lam[k] = static_cast<float>(1.0 / static_cast<double>(lam32));
  }
  std::vector<double> Wh(static_cast<size_t>(N) * K);
  parallel_for(N, [&](long b, long e) {
    for (long n = b; n < e; ++n)
      for (int k = 0; k < K; ++k)
        Wh[static_cast<size_t>(n) * K + k] =
            static_cast<double>(bf16_to_f32(W_bf16[static_cast<size_t>(n) * K + k])) /
            static_cast<double>(out->inv_lam[k]);
  });

  const int iters = std::max(1, o.refine_iters);
  std::vector<double> A = Wh;  // matrix whose top-r split is taken (W_hat, then W_hat - Q(R_t))
  std::vector<double> Q;
  out->refine_err.clear();
  for (int t = 0; t < iters; ++t) {
    std::vector<uint16_t> L1p, L2;
    std::vector<float> R;
    split_round_residual(Wh, A, N, K, o, out->inv_lam, &L1p, &L2, &R);
    const double err = fake_quant_error(R, N, K, t + 1 < iters ? &Q : nullptr);
    out->refine_err.push_back(err);
    if (t == 0 || err < *std::min_element(out->refine_err.begin(), out->refine_err.end() - 1)) {
      out->L1p.swap(L1p);
      out->L2.swap(L2);
      out->R.swap(R);
    }
    if (t + 1 < iters)
      parallel_for(N, [&](long b, long e) {
        for (size_t i = static_cast<size_t>(b) * K; i < static_cast<size_t>(e) * K; ++i) A[i] = Wh[i] - Q[i];
      });
  }
  return SVDQ_OK;
}

}  // namespace svdq
