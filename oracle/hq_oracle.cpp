/*
 * hq_oracle.cpp -- plain fp64 CPU oracle for the HadaNorm Hadamard-domain
 * quantized linear layer.  TEST INFRASTRUCTURE ONLY (tests, smoke check,
 * benchmark CPU-baseline leg).  Shares no code with the CUDA library.
 *
 * Each step is written out in the order and notation of the pages:
 *   HadaNorm review, Eq. (1):  X~ = X diag(sigma^-1) H - mu,
 *                              W~ = H^T diag(sigma) W,  b~ = b + mu W~.
 *   HadaNorm review, Eq. (3):  sigma_i = max|X_i|^a / max|W_i|^(1-a).
 *   HaTQ Sec. III-C, Eq. (7)-(8): H = H~ / sqrt(m), y_i = sum_j H~_ij x_j / sqrt(m).
 *   HaTQ Supplement Eq. (34):  Sylvester doubling.
 *   HaTQ Sec. III-A, Eq. (3):  x_int = clamp(round(x/s), -q, q), s = |x|_inf / q,
 *                              q = 2^(b-1) - 1.
 *   HaTQ Sec. IV-B, Eq. (14), (18): integer accumulation, accumulator scale
 *                              s_x * s_w.
 *   Data-free 4-bit blog, "Hadamard rotation", step 7: H block-diagonal,
 *                              one block per group.
 *   HaTQ Sec. IV-B, Eq. (15)-(17), supplement Eq. (40)-(41): the weight-only
 *                              form, W rotated along the output channels and
 *                              the output basis restored after accumulation.
 * No fast transform is used: the block Hadamard product is a dense sum over
 * the popcount-sign entries, and the GEMM is a triple loop.
 */
#include "hq_oracle.h"

#include <cmath>
#include <cstring>
#include <thread>
#include <vector>

namespace {

/* Runs body(i) for i in [0, count) split over nthreads std::threads.  Rows
 * are independent, so the split does not change any arithmetic. */
template <class F>
void parallel_rows(int64_t count, int nthreads, F body) {
  if (nthreads <= 1 || count < 2) {
    for (int64_t i = 0; i < count; ++i) body(i);
    return;
  }
  if (nthreads > count) nthreads = (int)count;
  std::vector<std::thread> pool;
  for (int w = 0; w < nthreads; ++w) {
    pool.emplace_back([=]() {
      for (int64_t i = w; i < count; i += nthreads) body(i);
    });
  }
  for (auto& th : pool) th.join();
}

bool is_pow2(int64_t n) { return n > 0 && (n & (n - 1)) == 0; }

int64_t qmax_for_bits(int bits) { return (int64_t(1) << (bits - 1)) - 1; }

double clampd(double v, double lo, double hi) {
  return v < lo ? lo : (v > hi ? hi : v);
}

/* Dense normalized Hadamard block H_n = H~_n / sqrt(n) (HaTQ Eq. (7)), entries
 * from the popcount formula, row-major [n*n].  The block-diagonal H of the
 * layer is diag(H_n, ..., H_n): H[j,k] = H_n[j mod n, k mod n] when j and k
 * lie in the same block, 0 otherwise. */
std::vector<double> dense_block(int64_t n) {
  std::vector<double> h(size_t(n * n));
  const double inv = 1.0 / std::sqrt(double(n));
  for (int64_t j = 0; j < n; ++j)
    for (int64_t k = 0; k < n; ++k)
      h[size_t(j * n + k)] = double(hqo_hadamard_entry(j, k)) * inv;
  return h;
}

}  // namespace

extern "C" {

int hqo_hadamard_entry(int64_t j, int64_t k) {
  uint64_t v = uint64_t(j) & uint64_t(k);
  int parity = 0;
  while (v) {
    parity ^= int(v & 1u);
    v >>= 1;
  }
  return parity ? -1 : 1;
}

int hqo_sylvester(int64_t n, int8_t* out) {
  if (!is_pow2(n) || out == nullptr) return -1;
  out[0] = 1;
  for (int64_t m = 1; m < n; m *= 2) {
    /* out currently holds H_m in its top-left m x m corner, row stride n. */
    for (int64_t r = 0; r < m; ++r) {
      for (int64_t c = 0; c < m; ++c) {
        int8_t h = out[r * n + c];
        out[r * n + (c + m)] = h;
        out[(r + m) * n + c] = h;
        out[(r + m) * n + (c + m)] = int8_t(-h);
      }
    }
  }
  return 0;
}

double hqo_bf16_to_f64(uint16_t b) {
  uint32_t u = uint32_t(b) << 16;
  float f;
  std::memcpy(&f, &u, sizeof(f));
  return double(f);
}

double hqo_rne(double x) {
  double f = std::floor(x);
  double diff = x - f;
  if (diff > 0.5) return f + 1.0;
  if (diff < 0.5) return f;
  /* exact tie: pick the even neighbour */
  return (std::fmod(f, 2.0) == 0.0) ? f : f + 1.0;
}

uint16_t hqo_f64_to_bf16(double x) {
  if (std::isnan(x)) return 0x7FC0;
  uint16_t sign = std::signbit(x) ? 0x8000 : 0x0000;
  double a = std::fabs(x);
  if (a == 0.0) return sign;
  /* a = f * 2^e with f in [0.5, 1); bf16 keeps 8 significant bits. */
  int e;
  (void)std::frexp(a, &e);
  /* bf16 normal range: exponents of the form 2^(e-1) with e-1 in [-126, 127];
   * subnormals keep fewer bits (step 2^-133). */
  int unbiased = e - 1;
  double step;
  if (unbiased >= -126) {
    step = std::ldexp(1.0, unbiased - 7);
  } else {
    step = std::ldexp(1.0, -133);
  }
  double r = hqo_rne(a / step) * step;
  if (r >= std::ldexp(1.0, 128)) return uint16_t(sign | 0x7F80); /* overflow */
  /* r is exactly representable in bf16, hence in float: take the top bits. */
  float rf = float(r);
  uint32_t u;
  std::memcpy(&u, &rf, sizeof(u));
  return uint16_t(sign | ((u >> 16) & 0x7FFF));
}

int hqo_col_absmax(const uint16_t* M, int64_t R, int64_t C, double* out) {
  if (M == nullptr || out == nullptr || R < 0 || C <= 0) return -1;
  for (int64_t c = 0; c < C; ++c) out[c] = 0.0;
  for (int64_t r = 0; r < R; ++r) {
    for (int64_t c = 0; c < C; ++c) {
      double v = std::fabs(hqo_bf16_to_f64(M[r * C + c]));
      if (v > out[c]) out[c] = v;
    }
  }
  return 0;
}

int hqo_channel_mean(const uint16_t* M, int64_t R, int64_t C, double* out) {
  if (M == nullptr || out == nullptr || R <= 0 || C <= 0) return -1;
  for (int64_t c = 0; c < C; ++c) {
    double sum = 0.0;
    for (int64_t r = 0; r < R; ++r) sum += hqo_bf16_to_f64(M[r * C + c]);
    out[c] = sum / double(R);
  }
  return 0;
}

int hqo_sigma(int64_t K, const double* amax_x, const double* amax_w,
              double alpha, double* sigma) {
  if (K <= 0 || amax_x == nullptr || amax_w == nullptr || sigma == nullptr)
    return -1;
  for (int64_t k = 0; k < K; ++k) {
    if (amax_x[k] > 0.0 && amax_w[k] > 0.0) {
      sigma[k] = std::pow(amax_x[k], alpha) / std::pow(amax_w[k], 1.0 - alpha);
    } else {
      sigma[k] = 1.0;
    }
  }
  return 0;
}

int hqo_quantize_act(int64_t K, int64_t n, int bits, int gran, int centering,
                     const uint16_t* X, int64_t T, const double* sigma,
                     const double* shift, double static_scale, const int64_t* rows, int64_t nrows,
                     int8_t* codes, double* scale, double* mean, double* tie,
                     double* Z, int nthreads) {
  if (K <= 0 || !is_pow2(n) || K % n != 0 || bits < 2 || bits > 8) return -1;
  if (gran < 0 || gran > 2 || centering < 0 || centering > 2) return -1;
  if (X == nullptr || T < 0 || nrows < 0 || codes == nullptr ||
      scale == nullptr || mean == nullptr)
    return -1;
  if (rows == nullptr && nrows != T) return -1;
  if (rows != nullptr) {
    for (int64_t i = 0; i < nrows; ++i)
      if (rows[i] < 0 || rows[i] >= T) return -1;
  }
  const double q = double(qmax_for_bits(bits));
  const std::vector<double> Hn = dense_block(n);

  /* Step 1 for one row: Y = X diag(sigma^-1); with centering 2 the row's
   * mean mu is subtracted from Y here, before the rotation; Z = Y H; with
   * centering 1 the mean m of Z is what is subtracted after it.  `zshift`
   * is the value removed from Z (m, or 0), `mean_out` the row's reported
   * mean (m for centering 1, mu for centering 2, else 0). */
  auto transform_row = [&](int64_t t, std::vector<double>& V, double& zshift,
                           double& mean_out) {
    std::vector<double> Y(K);
    for (int64_t j = 0; j < K; ++j) {
      double s = sigma ? sigma[j] : 1.0;
      Y[j] = hqo_bf16_to_f64(X[t * K + j]) / s;
      if (shift) Y[j] -= shift[j]; /* the per-channel mean over tokens */
    }
    mean_out = 0.0;
    if (centering == 2) {
      double sum = 0.0;
      for (int64_t j = 0; j < K; ++j) sum += Y[j];
      mean_out = sum / double(K);
      for (int64_t j = 0; j < K; ++j) Y[j] -= mean_out;
    }
    V.assign(K, 0.0);
    for (int64_t k = 0; k < K; ++k) {
      int64_t b0 = (k / n) * n; /* H is block diagonal: only j in k's block */
      double acc = 0.0;
      for (int64_t j = b0; j < b0 + n; ++j)
        acc += Y[j] * Hn[size_t((j - b0) * n + (k - b0))];
      V[k] = acc;
    }
    zshift = 0.0;
    if (centering == 1) {
      double sum = 0.0;
      for (int64_t k = 0; k < K; ++k) sum += V[k];
      zshift = sum / double(K);
      mean_out = zshift;
    }
  };

  /* Per-tensor dynamic scale: max |Z - m| over every row of the tensor. */
  double tensor_scale = 0.0, tensor_max = 0.0;
  if (gran == 1) {
    std::vector<double> row_max(T, 0.0);
    parallel_rows(T, nthreads, [&](int64_t t) {
      std::vector<double> V;
      double m, mu;
      transform_row(t, V, m, mu);
      double a = 0.0;
      for (int64_t k = 0; k < K; ++k) a = std::fmax(a, std::fabs(V[k] - m));
      row_max[t] = a;
    });
    double a = 0.0;
    for (int64_t t = 0; t < T; ++t) a = std::fmax(a, row_max[t]);
    tensor_max = a;
    tensor_scale = a / q;
  } else if (gran == 2) {
    tensor_scale = static_scale;
  }

  parallel_rows(nrows, nthreads, [&](int64_t i) {
    int64_t t = rows ? rows[i] : i;
    std::vector<double> V;
    double m, mu;
    transform_row(t, V, m, mu);
    if (Z) {
      for (int64_t k = 0; k < K; ++k) Z[i * K + k] = V[k];
    }
    for (int64_t k = 0; k < K; ++k) V[k] -= m; /* V = Z - mu */
    /* s = a / q with a = max |V| (dynamic), or the given s (static).  The
     * scaled value V / s is formed as V * q / a for a dynamic scale: the same
     * number, one rounding instead of two, so a value that lies exactly on a
     * rounding tie stays on it (unrotated bf16 inputs do). */
    double s, a = 0.0;
    if (gran == 0) {
      for (int64_t k = 0; k < K; ++k) a = std::fmax(a, std::fabs(V[k]));
      s = a / q;
    } else {
      s = tensor_scale;
      a = tensor_max;
    }
    scale[i] = s;
    mean[i] = mu;
    for (int64_t k = 0; k < K; ++k) {
      double c = 0.0, d = 0.5;
      if (s > 0.0) {
        double x = gran == 2 ? V[k] / s : (V[k] * q) / a;
        c = clampd(hqo_rne(x), -q, q);
        double ax = std::fabs(x);
        d = std::fabs(ax - std::floor(ax) - 0.5);
      }
      codes[i * K + k] = int8_t(c);
      if (tie) tie[i * K + k] = d;
    }
  });
  return 0;
}

int hqo_prepare_weights(int64_t K, int64_t N, int64_t n, int bits,
                        const uint16_t* W, const uint16_t* bias,
                        const double* sigma, const double* shift, int8_t* w_codes, double* w_scale,
                        double* colsum, double* corr_pre, double* bias_out,
                        double* tie, double* Wt, int nthreads) {
  if (K <= 0 || N <= 0 || !is_pow2(n) || K % n != 0 || bits < 2 || bits > 8)
    return -1;
  if (W == nullptr || w_codes == nullptr || w_scale == nullptr ||
      colsum == nullptr || bias_out == nullptr)
    return -1;
  const double q = double(qmax_for_bits(bits));
  const std::vector<double> Hn = dense_block(n);
  parallel_rows(N, nthreads, [&](int64_t c) {
    /* W~_math[k,c] = sum_j (H^T)[k,j] sigma_j W_math[j,c]
     *             = sum_j H[j,k] sigma_j W[c,j]                             */
    std::vector<double> wt(K);
    for (int64_t k = 0; k < K; ++k) {
      int64_t b0 = (k / n) * n;
      double acc = 0.0;
      for (int64_t j = b0; j < b0 + n; ++j) {
        double s = sigma ? sigma[j] : 1.0;
        acc += Hn[size_t((j - b0) * n + (k - b0))] * s *
               hqo_bf16_to_f64(W[c * K + j]);
      }
      wt[k] = acc;
    }
    double sum = 0.0, a = 0.0;
    for (int64_t k = 0; k < K; ++k) {
      sum += wt[k];
      a = std::fmax(a, std::fabs(wt[k]));
    }
    colsum[c] = sum;
    if (corr_pre) {
      /* the correction of centering before the rotation: sum_k sigma_k W[c,k] */
      double cp = 0.0;
      for (int64_t k = 0; k < K; ++k) cp += (sigma ? sigma[k] : 1.0) * hqo_bf16_to_f64(W[c * K + k]);
      corr_pre[c] = cp;
    }
    double s = a / q;
    w_scale[c] = s;
    for (int64_t k = 0; k < K; ++k) {
      double code = 0.0, d = 0.5;
      if (s > 0.0) {
        double x = (wt[k] * q) / a; /* = wt / s, one rounding (see hqo_quantize_act) */
        code = clampd(hqo_rne(x), -q, q);
        double ax = std::fabs(x);
        d = std::fabs(ax - std::floor(ax) - 0.5);
      }
      w_codes[c * K + k] = int8_t(code);
      if (tie) tie[c * K + k] = d;
      if (Wt) Wt[c * K + k] = wt[k];
    }
    bias_out[c] = bias ? hqo_bf16_to_f64(bias[c]) : 0.0;
    if (shift) {
      /* the removed per-channel mean, mu diag(sigma) W in the pages'
       * orientation, is the same for every token: a bias term */
      double cs = 0.0;
      for (int64_t k = 0; k < K; ++k)
        cs += shift[k] * (sigma ? sigma[k] : 1.0) * hqo_bf16_to_f64(W[c * K + k]);
      bias_out[c] += cs;
    }
  });
  return 0;
}

int hqo_gemm_acc(const int8_t* A, const int8_t* B, int64_t M, int64_t N,
                 int64_t K, const int64_t* rows, int64_t nrows, int64_t* acc,
                 int nthreads) {
  if (A == nullptr || B == nullptr || acc == nullptr || M < 0 || N <= 0 ||
      K <= 0 || nrows < 0)
    return -1;
  if (rows == nullptr && nrows != M) return -1;
  if (rows != nullptr) {
    for (int64_t i = 0; i < nrows; ++i)
      if (rows[i] < 0 || rows[i] >= M) return -1;
  }
  parallel_rows(nrows, nthreads, [&](int64_t i) {
    int64_t t = rows ? rows[i] : i;
    for (int64_t c = 0; c < N; ++c) {
      int64_t s = 0;
      for (int64_t k = 0; k < K; ++k)
        s += int64_t(A[t * K + k]) * int64_t(B[c * K + k]);
      acc[i * N + c] = s;
    }
  });
  return 0;
}

int hqo_epilogue(const int64_t* acc, int64_t nrows, int64_t N,
                 const double* sx, const double* m, const double* sw,
                 const double* b, const double* colsum, double* y,
                 uint16_t* y_bf16) {
  if (acc == nullptr || sx == nullptr || sw == nullptr || nrows < 0 || N <= 0)
    return -1;
  if (m != nullptr && colsum == nullptr) return -1;
  for (int64_t i = 0; i < nrows; ++i) {
    for (int64_t c = 0; c < N; ++c) {
      /* Q(X~) Q(W~) + b~ with b~ = b + mu W~ (mu_t = m_t on every channel) */
      double v = sx[i] * sw[c] * double(acc[i * N + c]);
      v += b ? b[c] : 0.0;
      if (m) v += m[i] * colsum[c];
      if (y) y[i * N + c] = v;
      if (y_bf16) y_bf16[i * N + c] = hqo_f64_to_bf16(v);
    }
  }
  return 0;
}

int hqo_exact_linear(const uint16_t* X, const uint16_t* W, const uint16_t* bias,
                     int64_t T, int64_t K, int64_t N, const int64_t* rows,
                     int64_t nrows, double* y, int nthreads) {
  if (X == nullptr || W == nullptr || y == nullptr || T < 0 || K <= 0 ||
      N <= 0 || nrows < 0)
    return -1;
  if (rows == nullptr && nrows != T) return -1;
  if (rows != nullptr) {
    for (int64_t i = 0; i < nrows; ++i)
      if (rows[i] < 0 || rows[i] >= T) return -1;
  }
  parallel_rows(nrows, nthreads, [&](int64_t i) {
    int64_t t = rows ? rows[i] : i;
    for (int64_t c = 0; c < N; ++c) {
      double s = 0.0;
      for (int64_t k = 0; k < K; ++k)
        s += hqo_bf16_to_f64(X[t * K + k]) * hqo_bf16_to_f64(W[c * K + k]);
      y[i * N + c] = s + (bias ? hqo_bf16_to_f64(bias[c]) : 0.0);
    }
  });
  return 0;
}

int hqo_prepare_weights_wh(int64_t K, int64_t N, int64_t n_out, int bits,
                           const uint16_t* W, const uint16_t* bias,
                           const double* sigma, int8_t* w_codes, double* w_scale,
                           double* b_bar, double* tie, double* Wbar, int nthreads) {
  if (K <= 0 || N <= 0 || !is_pow2(n_out) || N % n_out != 0 || bits < 2 || bits > 8)
    return -1;
  if (W == nullptr || w_codes == nullptr || w_scale == nullptr || b_bar == nullptr) return -1;
  const double q = double(qmax_for_bits(bits));
  const std::vector<double> Hn = dense_block(n_out);
  const double inv_sqrt_m = 1.0 / std::sqrt(double(n_out));
  parallel_rows(N, nthreads, [&](int64_t c) {
    /* S[c,k] = sum_j H~_out[c,j] sigma_k W[j,k] with the +-1 entries, j over
     * c's block of N; Wbar = S / sqrt(n_out).  The codes depend only on
     * Wbar / max|Wbar| = S / max|S|, formed from S so that the normalization
     * does not move a value that lies exactly on a rounding tie. */
    const int64_t c0 = (c / n_out) * n_out;
    std::vector<double> su(K);
    for (int64_t k = 0; k < K; ++k) {
      const double s = sigma ? sigma[k] : 1.0;
      double acc = 0.0;
      for (int64_t j = c0; j < c0 + n_out; ++j)
        acc += double(hqo_hadamard_entry(c - c0, j - c0)) * s * hqo_bf16_to_f64(W[j * K + k]);
      su[k] = acc;
    }
    double au = 0.0;
    for (int64_t k = 0; k < K; ++k) au = std::fmax(au, std::fabs(su[k]));
    const double sc = (au * inv_sqrt_m) / q; /* max|Wbar| / q */
    w_scale[c] = sc;
    for (int64_t k = 0; k < K; ++k) {
      double code = 0.0, d = 0.5;
      if (au > 0.0) {
        const double x = (su[k] * q) / au; /* = Wbar / w_scale */
        code = clampd(hqo_rne(x), -q, q);
        const double ax = std::fabs(x);
        d = std::fabs(ax - std::floor(ax) - 0.5);
      }
      w_codes[c * K + k] = int8_t(code);
      if (tie) tie[c * K + k] = d;
      if (Wbar) Wbar[c * K + k] = su[k] * inv_sqrt_m;
    }
    /* b_bar[c] = sum_j b[j] H_out[j,c] */
    double bb = 0.0;
    if (bias) {
      for (int64_t j = c0; j < c0 + n_out; ++j)
        bb += hqo_bf16_to_f64(bias[j]) * Hn[size_t((j - c0) * n_out + (c - c0))];
    }
    b_bar[c] = bb;
  });
  return 0;
}

int hqo_output_rotation(const double* M, int64_t rows, int64_t N, int64_t n_out,
                        double* out) {
  if (M == nullptr || out == nullptr || rows < 0 || N <= 0 || !is_pow2(n_out) ||
      N % n_out != 0)
    return -1;
  const std::vector<double> Hn = dense_block(n_out);
  for (int64_t i = 0; i < rows; ++i) {
    for (int64_t c = 0; c < N; ++c) {
      const int64_t c0 = (c / n_out) * n_out;
      double acc = 0.0;
      for (int64_t j = c0; j < c0 + n_out; ++j)
        acc += M[i * N + j] * Hn[size_t((j - c0) * n_out + (c - c0))];
      out[i * N + c] = acc;
    }
  }
  return 0;
}

int hqo_epilogue_wh(const int64_t* acc, int64_t nrows, int64_t N, int64_t n_out,
                    const double* sx, const double* sw, const double* b_bar,
                    double* y, uint16_t* y_bf16) {
  if (acc == nullptr || sx == nullptr || sw == nullptr || nrows < 0 || N <= 0 ||
      !is_pow2(n_out) || N % n_out != 0)
    return -1;
  std::vector<double> A(static_cast<size_t>(N)), Y(static_cast<size_t>(N));
  for (int64_t i = 0; i < nrows; ++i) {
    /* the bracket of Eq. (41): dequantized Q(X) Q(Wbar)^T plus b_bar */
    for (int64_t j = 0; j < N; ++j)
      A[size_t(j)] = sx[i] * sw[j] * double(acc[i * N + j]) + (b_bar ? b_bar[j] : 0.0);
    /* back to the original output basis: times (T_out)^T = H_out */
    if (hqo_output_rotation(A.data(), 1, N, n_out, Y.data()) != 0) return -1;
    for (int64_t c = 0; c < N; ++c) {
      if (y) y[i * N + c] = Y[size_t(c)];
      if (y_bf16) y_bf16[i * N + c] = hqo_f64_to_bf16(Y[size_t(c)]);
    }
  }
  return 0;
}

int hqo_pack_i4(const int8_t* codes, int64_t count, uint8_t* out) {
  if (count < 0 || count % 2 != 0 || (count > 0 && (codes == nullptr || out == nullptr)))
    return -1;
  for (int64_t j = 0; j < count / 2; ++j) {
    const int lo = codes[2 * j], hi = codes[2 * j + 1];
    if (lo < -8 || lo > 7 || hi < -8 || hi > 7) return -1;
    /* a 4-bit two's-complement value v is stored as v mod 16 */
    const int lo4 = lo < 0 ? lo + 16 : lo;
    const int hi4 = hi < 0 ? hi + 16 : hi;
    out[j] = uint8_t(lo4 + 16 * hi4);
  }
  return 0;
}

int hqo_unpack_i4(const uint8_t* packed, int64_t count, int8_t* codes) {
  if (count < 0 || count % 2 != 0 || (count > 0 && (codes == nullptr || packed == nullptr)))
    return -1;
  for (int64_t j = 0; j < count / 2; ++j) {
    const int lo4 = packed[j] % 16, hi4 = packed[j] / 16;
    codes[2 * j] = int8_t(lo4 >= 8 ? lo4 - 16 : lo4);
    codes[2 * j + 1] = int8_t(hi4 >= 8 ? hi4 - 16 : hi4);
  }
  return 0;
}

}  /* extern "C" */

/* ---------------------------------------------------------------------------
 * Group-wise form with a low-rank branch (see hq_oracle.h). */

namespace {
/* The symmetric quantizer of one group of values: s = max |v| / q, codes
 * rne(v q / max) (one rounding), clamp; s = 0 gives zero codes. */
void quantize_group(const double* v, int64_t g, double q, int8_t* codes, double* scale,
                    double* tie) {
  double a = 0.0;
  for (int64_t i = 0; i < g; ++i) a = std::fmax(a, std::fabs(v[i]));
  *scale = a / q;
  for (int64_t i = 0; i < g; ++i) {
    double c = 0.0, d = 0.5;
    if (a > 0.0) {
      const double x = (v[i] * q) / a;
      c = clampd(hqo_rne(x), -q, q);
      const double ax = std::fabs(x);
      d = std::fabs(ax - std::floor(ax) - 0.5);
    }
    codes[i] = int8_t(c);
    if (tie) tie[i] = d;
  }
}
}  // namespace

extern "C" {

int hqo_gw_prepare_weights(int64_t K, int64_t N, int64_t g, int bits, int64_t rank,
                           const uint16_t* W, const uint16_t* bias, const double* sigma,
                           const double* L1, const double* L2, uint16_t* l1s, uint16_t* l2b,
                           int8_t* w_codes, double* w_gscale, double* bias_out, double* tie,
                           double* Rh, int nthreads) {
  if (K <= 0 || N <= 0 || !is_pow2(g) || K % g != 0 || bits < 2 || bits > 8 || rank < 0)
    return -1;
  if (W == nullptr || w_codes == nullptr || w_gscale == nullptr || bias_out == nullptr)
    return -1;
  if (rank > 0 && (L1 == nullptr || L2 == nullptr || l1s == nullptr || l2b == nullptr)) return -1;
  const double q = double(qmax_for_bits(bits));
  const std::vector<double> Hg = dense_block(g);
  const int64_t G = K / g;
  /* the 16-bit factors: l2 = bf16(L2), l1 = bf16(L1 diag(sigma^-1)) */
  for (int64_t r = 0; r < rank; ++r)
    for (int64_t k = 0; k < K; ++k)
      l1s[r * K + k] = hqo_f64_to_bf16(L1[r * K + k] / (sigma ? sigma[k] : 1.0));
  for (int64_t i = 0; i < N * rank; ++i) l2b[i] = hqo_f64_to_bf16(L2[i]);
  parallel_rows(N, nthreads, [&](int64_t c) {
    /* R[c,k] = W[c,k] sigma_k - sum_r l2[c,r] l1[r,k] sigma_k */
    std::vector<double> R(K);
    for (int64_t k = 0; k < K; ++k) {
      const double s = sigma ? sigma[k] : 1.0;
      double lr = 0.0;
      for (int64_t r = 0; r < rank; ++r)
        lr += hqo_bf16_to_f64(l2b[c * rank + r]) * hqo_bf16_to_f64(l1s[r * K + k]);
      R[k] = hqo_bf16_to_f64(W[c * K + k]) * s - lr * s;
    }
    /* R H, one g x g block per group, then the group quantizer */
    std::vector<double> v(g);
    for (int64_t j = 0; j < G; ++j) {
      for (int64_t i = 0; i < g; ++i) {
        double acc = 0.0;
        for (int64_t m = 0; m < g; ++m) acc += R[j * g + m] * Hg[size_t(m * g + i)];
        v[i] = acc;
        if (Rh) Rh[c * K + j * g + i] = acc;
      }
      quantize_group(v.data(), g, q, w_codes + c * K + j * g, w_gscale + c * G + j,
                     tie ? tie + c * K + j * g : nullptr);
    }
    bias_out[c] = bias ? hqo_bf16_to_f64(bias[c]) : 0.0;
  });
  return 0;
}

int hqo_gw_quantize_act(int64_t K, int64_t g, int bits, int64_t rank, const uint16_t* X,
                        int64_t T, const double* sigma, const uint16_t* l1s, const int64_t* rows,
                        int64_t nrows, int8_t* codes, double* gscale, uint16_t* u, double* tie,
                        double* Z, int nthreads) {
  if (K <= 0 || !is_pow2(g) || K % g != 0 || bits < 2 || bits > 8 || rank < 0) return -1;
  if (X == nullptr || T < 0 || nrows < 0 || codes == nullptr || gscale == nullptr) return -1;
  if (rank > 0 && (l1s == nullptr || u == nullptr)) return -1;
  if (rows == nullptr && nrows != T) return -1;
  if (rows != nullptr) {
    for (int64_t i = 0; i < nrows; ++i)
      if (rows[i] < 0 || rows[i] >= T) return -1;
  }
  const double q = double(qmax_for_bits(bits));
  const std::vector<double> Hg = dense_block(g);
  const int64_t G = K / g;
  parallel_rows(nrows, nthreads, [&](int64_t i) {
    const int64_t t = rows ? rows[i] : i;
    /* the 16-bit branch's down projection of the original input */
    for (int64_t r = 0; r < rank; ++r) {
      double acc = 0.0;
      for (int64_t k = 0; k < K; ++k)
        acc += hqo_bf16_to_f64(X[t * K + k]) * hqo_bf16_to_f64(l1s[r * K + k]);
      u[i * rank + r] = hqo_f64_to_bf16(acc);
    }
    /* x^ H per group, then the group quantizer */
    std::vector<double> xh(K), v(g);
    for (int64_t k = 0; k < K; ++k)
      xh[k] = hqo_bf16_to_f64(X[t * K + k]) / (sigma ? sigma[k] : 1.0);
    for (int64_t j = 0; j < G; ++j) {
      for (int64_t c = 0; c < g; ++c) {
        double acc = 0.0;
        for (int64_t m = 0; m < g; ++m) acc += xh[j * g + m] * Hg[size_t(m * g + c)];
        v[c] = acc;
        if (Z) Z[i * K + j * g + c] = acc;
      }
      quantize_group(v.data(), g, q, codes + i * K + j * g, gscale + i * G + j,
                     tie ? tie + i * K + j * g : nullptr);
    }
  });
  return 0;
}

int hqo_gw_epilogue(const int8_t* A, const int8_t* B, int64_t nrows, int64_t N, int64_t K,
                    int64_t g, const double* ascale, const double* wscale, const uint16_t* u,
                    const uint16_t* l2b, int64_t rank, const double* b, double* y,
                    uint16_t* y_bf16, int nthreads) {
  if (A == nullptr || B == nullptr || ascale == nullptr || wscale == nullptr || nrows < 0 ||
      N <= 0 || K <= 0 || !is_pow2(g) || K % g != 0 || rank < 0)
    return -1;
  if (rank > 0 && (u == nullptr || l2b == nullptr)) return -1;
  const int64_t G = K / g;
  parallel_rows(nrows, nthreads, [&](int64_t i) {
    for (int64_t c = 0; c < N; ++c) {
      double acc = 0.0;
      for (int64_t j = 0; j < G; ++j) {
        int64_t s = 0; /* the group's integer sum, exact */
        for (int64_t k = j * g; k < (j + 1) * g; ++k) s += int64_t(A[i * K + k]) * int64_t(B[c * K + k]);
        acc += ascale[i * G + j] * wscale[c * G + j] * double(s);
      }
      for (int64_t r = 0; r < rank; ++r)
        acc += hqo_bf16_to_f64(u[i * rank + r]) * hqo_bf16_to_f64(l2b[c * rank + r]);
      if (b) acc += b[c];
      if (y) y[i * N + c] = acc;
      if (y_bf16) y_bf16[i * N + c] = hqo_f64_to_bf16(acc);
    }
  });
  return 0;
}

}  /* extern "C" */

