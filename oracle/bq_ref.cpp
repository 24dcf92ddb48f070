// Reference quantizers and layers of the bit-plane quantized linear layer, in plain C++.
//
// TEST INFRASTRUCTURE ONLY. Only the tests, the smoke check and the bench's CPU legs load this
// library; the product path (the CUDA library and its binding) never does. It shares no code,
// header, table or helper with the CUDA sources.
//
// Style: plain loops in the order the definitions are written, float64 / int64 arithmetic for
// every sum and product, float32 only where a stored float32 operand takes a decision that
// turns into an integer code (sign, rounding, nearest point). OpenMP runs independent output
// rows (or vectors) in parallel; no loop is blocked, fused or reordered beyond that. Built with
// -O2 -ffp-contract=off (no fused multiply-add), so every float32 and float64 operation is a
// separately rounded IEEE operation.
//
// Conventions: W [N][K] float32 row-major, x [M][K] float32 holding bf16 values, y [M][N]
// float64, accumulators int64. Every entry point returns 0, or -1 on an argument it refuses.
//
// Pages (titles, as cited in the function comments):
//   [RaBiT]  "RaBiT框架：突破2比特量化性能瓶颈的LLM部署方案"
//   [HGF]    "1.58位LLM混合门控流优化技术解析"
//   [ABQ]    "ABQ-LLM：用于大語言模型的任意比特量化推理加速"
//   [BVSR]   "BVSR：面向分布感知的大语言模型权重量化的比特向量求和表示"
//   [BitNet] "1-bit LLM的端侧推理革命"

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <vector>

#ifdef _OPENMP
#include <omp.h>
#endif

namespace {

// sign(v) = +1 if v >= 0 else -1 ([BitNet] §2.1); -0.0 >= 0 holds, so sign(-0.0) = +1.
inline int8_t sign_pm1(double v) { return v >= 0.0 ? int8_t(1) : int8_t(-1); }

// round half to even of a float32 (the default IEEE rounding mode)
inline float rn(float v) { return std::nearbyint(v); }

// mean |a| over n values: float64 sum in index order, divided by n, stored float32
float mean_abs(const float* a, int64_t n, int64_t stride = 1) {
  if (n == 0) return 0.0f;
  double s = 0.0;
  for (int64_t i = 0; i < n; i++) s += std::fabs(double(a[i * stride]));
  return float(s / double(n));
}

float mean_abs_d(const double* a, int64_t n) {
  if (n == 0) return 0.0f;
  double s = 0.0;
  for (int64_t i = 0; i < n; i++) s += std::fabs(a[i]);
  return float(s / double(n));
}

// number of set bits of a 64-bit word, counted one bit at a time
int popcount64(uint64_t v) {
  int c = 0;
  for (int b = 0; b < 64; b++) c += int((v >> b) & 1u);
  return c;
}

constexpr int kVec = 32;                                  // BVSR vector length
constexpr int kPlanes = 4;                                // BVSR bitvectors per vector
constexpr int kGrid = 8;                                  // range grid points per side
constexpr double kRatios[4] = {1.5, 2.0, 2.5, 3.0};       // geometric ratios of the set families
constexpr int kSets = 4 * kGrid * kGrid;                  // 256 cached sets

}  // namespace

extern "C" {

int bqref_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

void bqref_set_threads(int n) {
#ifdef _OPENMP
  if (n > 0) omp_set_num_threads(n);
#else
  (void)n;
#endif
}

// ---------------------------------------------------------------------------------------------
// small helpers exposed for the pins
// ---------------------------------------------------------------------------------------------

// sign of each value ([BitNet] §2.1): out[i] = +1 if v[i] >= 0 else -1
int bqref_sign(const double* v, int64_t n, int8_t* out) {
  if (n < 0) return -1;
  for (int64_t i = 0; i < n; i++) out[i] = sign_pm1(v[i]);
  return 0;
}

// mean |a| in float64 (index order), stored float32
int bqref_mean_abs(const float* a, int64_t n, float* out) {
  if (n < 0) return -1;
  *out = mean_abs(a, n);
  return 0;
}

// nearest bfloat16 (ties to even) of each float32, returned as float32 (the storage of the
// [HGF] §2.1 correction matrices)
int bqref_bf16_round(const float* a, int64_t n, float* out) {
  for (int64_t i = 0; i < n; i++) {
    uint32_t u;
    std::memcpy(&u, &a[i], 4);
    uint64_t w = uint64_t(u);
    w = (w + 0x7FFFu + ((w >> 16) & 1u)) & 0xFFFF0000u;
    const uint32_t r = uint32_t(w);
    std::memcpy(&out[i], &r, 4);
  }
  return 0;
}

// ---------------------------------------------------------------------------------------------
// activation quantization
// ---------------------------------------------------------------------------------------------

// Per-token absmax int8 ([HGF] §1.2; [BVSR] Introduction, online input quantization):
// gamma = max_k |x|, s = 127 / gamma (float32 divide), q = clamp(rn(x * s), -127, 127) with the
// product rounded to float32; gamma = 0 gives q = 0.
int bqref_quantize_act_int8(const float* x, int64_t M, int64_t K, int8_t* q, float* gamma) {
  if (M < 0 || K < 0) return -1;
#pragma omp parallel for schedule(static)
  for (int64_t m = 0; m < M; m++) {
    const float* xr = x + m * K;
    float g = 0.0f;
    for (int64_t k = 0; k < K; k++) {
      const float a = std::fabs(xr[k]);
      if (a > g) g = a;
    }
    gamma[m] = g;
    for (int64_t k = 0; k < K; k++) {
      if (g > 0.0f) {
        const float s = 127.0f / g;
        const float v = xr[k] * s;
        float r = rn(v);
        if (r > 127.0f) r = 127.0f;
        if (r < -127.0f) r = -127.0f;
        q[m * K + k] = int8_t(r);
      } else {
        q[m * K + k] = 0;
      }
    }
  }
  return 0;
}

// x_hat = q gamma / 127 in float64 ([HGF] §1.2 dequantization)
int bqref_dequant_act_int8(const int8_t* q, const float* gamma, int64_t M, int64_t K, double* out) {
  for (int64_t m = 0; m < M; m++) {
    const double s = double(gamma[m]) / 127.0;
    for (int64_t k = 0; k < K; k++) out[m * K + k] = double(q[m * K + k]) * s;
  }
  return 0;
}

// Uniform asymmetric quantizer per row ([ABQ] §3.2 eq.(3) with the compensation term off and
// no learned clipping, §3.1 eq.(1) with alpha = beta = 1):
//   lo = min, hi = max (float32), Delta = max(hi - lo, 1e-5) / (2^bits - 1) (float32 ops),
//   z = rn(-lo / Delta) (integer, unclamped), q = clamp(rn(v / Delta) + z, 0, 2^bits - 1).
int bqref_quantize_rows_asym(const float* V, int64_t R, int64_t L, int bits, int32_t* q, float* delta,
                             int32_t* z) {
  if (R < 0 || L < 1 || bits < 1 || bits > 16) return -1;
  const int64_t qmax = (int64_t(1) << bits) - 1;
#pragma omp parallel for schedule(static)
  for (int64_t r = 0; r < R; r++) {
    const float* v = V + r * L;
    float lo = v[0], hi = v[0];
    for (int64_t i = 1; i < L; i++) {
      lo = std::min(lo, v[i]);
      hi = std::max(hi, v[i]);
    }
    float span = hi - lo;
    if (span < 1e-5f) span = 1e-5f;
    const float d = span / float(qmax);
    const int64_t zz = int64_t(rn(-lo / d));
    delta[r] = d;
    z[r] = int32_t(zz);
    for (int64_t i = 0; i < L; i++) {
      int64_t c = int64_t(rn(v[i] / d)) + zz;
      if (c < 0) c = 0;
      if (c > qmax) c = qmax;
      q[r * L + i] = int32_t(c);
    }
  }
  return 0;
}

// ---------------------------------------------------------------------------------------------
// RaBiT residual binarization ([RaBiT] §2.1-§2.2; §6 three-bit extension read as a third path)
// ---------------------------------------------------------------------------------------------

// P paths: R_0 = W; path p: B_p = sign(R_{p-1}), g_p[n] = mean_k |R_{p-1}[n,:]| (float64, stored
// float32), R_p = R_{p-1} - g_p B_p h_p (float64 from the stored float32 g_p and h_p).
// h [P][K] given (h_1 = 1 in the two-path reading). Out: B [P][N][K], g [P][N].
int bqref_rabit_pack_paths(const float* W, int64_t N, int64_t K, int P, const float* h, int8_t* B, float* g) {
  if (N < 0 || K < 1 || P < 1) return -1;
#pragma omp parallel for schedule(static)
  for (int64_t n = 0; n < N; n++) {
    std::vector<double> R(K);
    for (int64_t k = 0; k < K; k++) R[k] = double(W[n * K + k]);
    for (int p = 0; p < P; p++) {
      int8_t* Bp = B + (int64_t(p) * N + n) * K;
      for (int64_t k = 0; k < K; k++) Bp[k] = sign_pm1(R[k]);
      const float gp = mean_abs_d(R.data(), K);
      g[int64_t(p) * N + n] = gp;
      for (int64_t k = 0; k < K; k++) R[k] = R[k] - (double(gp) * double(Bp[k])) * double(h[int64_t(p) * K + k]);
    }
  }
  return 0;
}

// W_hat [N][K] = sum_p g_p B_p h_p in float64 ([RaBiT] §2.1), paths added from the first
int bqref_rabit_weight(const int8_t* B, const float* g, const float* h, int P, int64_t N, int64_t K, double* out) {
  for (int64_t n = 0; n < N; n++)
    for (int64_t k = 0; k < K; k++) {
      double s = 0.0;
      for (int p = 0; p < P; p++)
        s += (double(g[int64_t(p) * N + n]) * double(B[(int64_t(p) * N + n) * K + k])) * double(h[int64_t(p) * K + k]);
      out[n * K + k] = s;
    }
  return 0;
}

// [RaBiT] §2.3 function-aware initialization, stage 1: iterative residual SVID over two paths.
// Reading: path q approximates T_q = W - W_other by sign(T_q) (g_q h_q^T); one round updates
// path 1 then path 2; an update sets B_q = sign(T_q), then g_q[i] = sum_j |T_ij| h_q[j] /
// sum_j h_q[j]^2 (0 if that is 0), then h_q[j] = sum_i |T_ij| g_q[i] / sum_i g_q[i]^2 (kept if
// that is 0). Start g = 0, h = 1, B_1 = sign(W), B_2 = +1. float64 with sums in index order, g
// and h stored float32 after every update. Out: B [2][N][K], g [2][N], h [2][K].
int bqref_rabit_pack_svid(const float* W, int64_t N, int64_t K, int rounds, int8_t* B, float* g, float* h) {
  if (N < 1 || K < 1 || rounds < 0) return -1;
  for (int q = 0; q < 2; q++) {
    for (int64_t n = 0; n < N; n++) g[q * N + n] = 0.0f;
    for (int64_t k = 0; k < K; k++) h[q * K + k] = 1.0f;
  }
  for (int64_t i = 0; i < N * K; i++) {
    B[i] = sign_pm1(double(W[i]));
    B[N * K + i] = 1;
  }
  std::vector<double> A(size_t(N * K));
  for (int r = 0; r < rounds; r++) {
    for (int q = 0; q < 2; q++) {
      const int o = 1 - q;
      int8_t* Bq = B + int64_t(q) * N * K;
      const int8_t* Bo = B + int64_t(o) * N * K;
#pragma omp parallel for schedule(static)
      for (int64_t i = 0; i < N; i++)
        for (int64_t j = 0; j < K; j++) {
          const double wo = (double(g[o * N + i]) * double(h[o * K + j])) * double(Bo[i * K + j]);
          const double t = double(W[i * K + j]) - wo;
          Bq[i * K + j] = sign_pm1(t);
          A[size_t(i * K + j)] = std::fabs(t);
        }
      double hh = 0.0;
      for (int64_t j = 0; j < K; j++) hh += double(h[q * K + j]) * double(h[q * K + j]);
#pragma omp parallel for schedule(static)
      for (int64_t i = 0; i < N; i++) {
        if (hh > 0.0) {
          double s = 0.0;
          for (int64_t j = 0; j < K; j++) s += A[size_t(i * K + j)] * double(h[q * K + j]);
          g[q * N + i] = float(s / hh);
        } else {
          g[q * N + i] = 0.0f;
        }
      }
      double gg = 0.0;
      for (int64_t i = 0; i < N; i++) gg += double(g[q * N + i]) * double(g[q * N + i]);
      if (gg > 0.0) {
#pragma omp parallel for schedule(static)
        for (int64_t j = 0; j < K; j++) {
          double s = 0.0;
          for (int64_t i = 0; i < N; i++) s += A[size_t(i * K + j)] * double(g[q * N + i]);
          h[q * K + j] = float(s / gg);
        }
      }
    }
  }
  return 0;
}

// ||W - W_hat||^2 in float64, W_hat as in bqref_rabit_weight, summed row by row in index order
int bqref_rabit_recon_error(const float* W, const int8_t* B, const float* g, const float* h, int P, int64_t N,
                            int64_t K, double* out) {
  double tot = 0.0;
  for (int64_t n = 0; n < N; n++)
    for (int64_t k = 0; k < K; k++) {
      double w = 0.0;
      for (int p = 0; p < P; p++)
        w += (double(g[int64_t(p) * N + n]) * double(B[(int64_t(p) * N + n) * K + k])) * double(h[int64_t(p) * K + k]);
      const double d = double(W[n * K + k]) - w;
      tot += d * d;
    }
  *out = tot;
  return 0;
}

// y [M][N] = sum_k W_hat[n,k] x[m,k] in float64 with x the unquantized bf16 activations (the
// [RaBiT] §3.2 kernel applies signs to the input); acc [P][M][N] = sum_k B_p h_p x per path.
int bqref_rabit_layer(const int8_t* B, const float* g, const float* h, int P, int64_t N, int64_t K, const float* x,
                      int64_t M, double* y, double* acc) {
  if (P < 1 || N < 0 || K < 1 || M < 0) return -1;
#pragma omp parallel for schedule(static)
  for (int64_t n = 0; n < N; n++) {
    for (int64_t m = 0; m < M; m++) {
      double s = 0.0;
      for (int64_t k = 0; k < K; k++) {
        double w = 0.0;
        for (int p = 0; p < P; p++)
          w += (double(g[int64_t(p) * N + n]) * double(B[(int64_t(p) * N + n) * K + k])) * double(h[int64_t(p) * K + k]);
        s += w * double(x[m * K + k]);
      }
      y[m * N + n] = s;
      for (int p = 0; p < P; p++) {
        double a = 0.0;
        for (int64_t k = 0; k < K; k++)
          a += (double(B[(int64_t(p) * N + n) * K + k]) * double(h[int64_t(p) * K + k])) * double(x[m * K + k]);
        acc[(int64_t(p) * M + m) * N + n] = a;
      }
    }
  }
  return 0;
}

// ---------------------------------------------------------------------------------------------
// BitNet W1A8 ([BitNet] §2.1-§2.3) and ternary W1.58A8 ([HGF] §1.2, §2.1, §4.1)
// ---------------------------------------------------------------------------------------------

// W ~ alpha sign(W), alpha = mean|W| over the whole tensor (the page learns it per matrix)
int bqref_bitnet_pack(const float* W, int64_t N, int64_t K, int8_t* B, float* alpha) {
  if (N < 0 || K < 0) return -1;
  for (int64_t i = 0; i < N * K; i++) B[i] = sign_pm1(double(W[i]));
  *alpha = mean_abs(W, N * K);
  return 0;
}

// gamma = mean|W| (the page's code; its prose says absmax), T = clamp(rn(W / gamma), -1, 1)
// with W / gamma a float32 divide, ties to even; gamma = 0 gives T = 0.
int bqref_ternary_pack(const float* W, int64_t N, int64_t K, int8_t* T, float* gamma) {
  if (N < 0 || K < 0) return -1;
  const float gw = mean_abs(W, N * K);
  *gamma = gw;
  for (int64_t i = 0; i < N * K; i++) {
    if (gw > 0.0f) {
      float r = rn(W[i] / gw);
      if (r > 1.0f) r = 1.0f;
      if (r < -1.0f) r = -1.0f;
      T[i] = int8_t(r);
    } else {
      T[i] = 0;
    }
  }
  return 0;
}

// Shared by the sign and ternary layers: acc = sum_k C[n,k] q[m,k] (int64) and
// y = sum_k (s_w C[n,k]) (q[m,k] gamma[m] / 127) in float64, q the per-token int8 codes.
static void int8_code_layer(const int8_t* C, float s_w, int64_t N, int64_t K, const int8_t* q, const float* gamma,
                            int64_t M, int64_t* acc, double* y) {
#pragma omp parallel for schedule(static)
  for (int64_t n = 0; n < N; n++)
    for (int64_t m = 0; m < M; m++) {
      int64_t a = 0;
      double s = 0.0;
      const double gs = double(gamma[m]) / 127.0;
      for (int64_t k = 0; k < K; k++) {
        const int64_t c = C[n * K + k], v = q[m * K + k];
        a += c * v;
        s += (double(s_w) * double(c)) * (double(v) * gs);
      }
      acc[m * N + n] = a;
      y[m * N + n] = s;
    }
}

// y = (alpha B) (q gamma / 127) summed in float64; acc = sum_k B q (int64). Also returns the
// activation codes and scales.
int bqref_bitnet_layer(const int8_t* B, float alpha, int64_t N, int64_t K, const float* x, int64_t M, int8_t* q,
                       float* gamma, int64_t* acc, double* y) {
  if (N < 0 || K < 1 || M < 0) return -1;
  bqref_quantize_act_int8(x, M, K, q, gamma);
  int8_code_layer(B, alpha, N, K, q, gamma, M, acc, y);
  return 0;
}

// u[m,r] = SiLU(sum_k x[m,k] A[k,r]) in float64 with x unquantized ([HGF] §2.1 gated
// correction); out[m,n] = tanh(alpha) sum_r u[m,r] B[r,n]. SiLU(z) = z / (1 + exp(-z)).
int bqref_lora_correction(const float* x, int64_t M, int64_t K, const float* A, const float* Bl, int r, int64_t N,
                          float alpha, double* out) {
  if (M < 0 || K < 0 || r < 0 || N < 0) return -1;
  const double ta = std::tanh(double(alpha));
#pragma omp parallel for schedule(static)
  for (int64_t m = 0; m < M; m++) {
    std::vector<double> u(size_t(r > 0 ? r : 1));
    for (int j = 0; j < r; j++) {
      double z = 0.0;
      for (int64_t k = 0; k < K; k++) z += double(x[m * K + k]) * double(A[k * r + j]);
      u[size_t(j)] = z / (1.0 + std::exp(-z));
    }
    for (int64_t n = 0; n < N; n++) {
      double s = 0.0;
      for (int j = 0; j < r; j++) s += u[size_t(j)] * double(Bl[int64_t(j) * N + n]);
      out[m * N + n] = ta * s;
    }
  }
  return 0;
}

// acc = sum_k T q (int64); y = (gamma_w T)(q gamma_x / 127) in float64 plus, with r > 0, the
// gated correction tanh(alpha) SiLU(x A) B on the unquantized x ([HGF] §1.2, §2.1). y_t and y_l
// (nullable) receive the two terms.
int bqref_ternary_layer(const int8_t* T, float gamma_w, const float* A, const float* Bl, int r, float lora_alpha,
                        int64_t N, int64_t K, const float* x, int64_t M, int8_t* q, float* gamma, int64_t* acc,
                        double* y, double* y_t, double* y_l) {
  if (N < 0 || K < 1 || M < 0 || r < 0) return -1;
  bqref_quantize_act_int8(x, M, K, q, gamma);
  std::vector<double> yt(size_t(M * N)), yl(size_t(M * N), 0.0);
  int8_code_layer(T, gamma_w, N, K, q, gamma, M, acc, yt.data());
  if (r > 0) bqref_lora_correction(x, M, K, A, Bl, r, N, lora_alpha, yl.data());
  for (int64_t i = 0; i < M * N; i++) {
    y[i] = yt[size_t(i)] + yl[size_t(i)];
    if (y_t) y_t[i] = yt[size_t(i)];
    if (y_l) y_l[i] = yl[size_t(i)];
  }
  return 0;
}

// ---------------------------------------------------------------------------------------------
// ABQ arbitrary-bit WxAy ([ABQ] abstract, §3.1-§3.3)
// ---------------------------------------------------------------------------------------------

// [ABQ] §3.3 bit balance (W2*): symmetric five levels. Per row hi = max|W|, Delta =
// max(hi - (-hi), 1e-5) / 4 (float32), z = 2, q = clamp(rn(W / Delta) + 2, 0, 4).
int bqref_abq_pack_balanced(const float* W, int64_t N, int64_t K, int32_t* Q, float* delta, int32_t* z) {
  if (N < 0 || K < 1) return -1;
#pragma omp parallel for schedule(static)
  for (int64_t n = 0; n < N; n++) {
    float hi = 0.0f;
    for (int64_t k = 0; k < K; k++) hi = std::max(hi, std::fabs(W[n * K + k]));
    float span = hi - (-hi);
    if (span < 1e-5f) span = 1e-5f;
    const float d = span / 4.0f;
    delta[n] = d;
    z[n] = 2;
    for (int64_t k = 0; k < K; k++) {
      int64_t c = int64_t(rn(W[n * K + k] / d)) + 2;
      if (c < 0) c = 0;
      if (c > 4) c = 4;
      Q[n * K + k] = int32_t(c);
    }
  }
  return 0;
}

// [ABQ] §3.2 eq.(3) distribution compensation with gamma = 1: W' = W + a b^T, a per output row,
// b per input column, in float32 with the product a[n] b[k] rounded before the sum.
int bqref_abq_compensate(const float* W, const float* a, const float* b, int64_t N, int64_t K, float* Wc) {
  if (N < 0 || K < 0) return -1;
  for (int64_t n = 0; n < N; n++)
    for (int64_t k = 0; k < K; k++) {
      const float p = a[n] * b[k];
      Wc[n * K + k] = W[n * K + k] + p;
    }
  return 0;
}

// Activations per token with a bits (quantize_rows_asym), then
// I = sum_k (qw - zw)(qx - zx) (int64) and y = sum_k (Dw (qw - zw)) (Dx (qx - zx)) in float64.
int bqref_abq_layer(const int32_t* Q, const float* delta, const int32_t* zw, int64_t N, int64_t K, const float* x,
                    int64_t M, int a_bits, int32_t* Qx, float* dx, int32_t* zx, int64_t* I, double* y) {
  if (N < 0 || K < 1 || M < 0) return -1;
  if (bqref_quantize_rows_asym(x, M, K, a_bits, Qx, dx, zx) != 0) return -1;
#pragma omp parallel for schedule(static)
  for (int64_t n = 0; n < N; n++)
    for (int64_t m = 0; m < M; m++) {
      int64_t a = 0;
      double s = 0.0;
      for (int64_t k = 0; k < K; k++) {
        const int64_t cw = int64_t(Q[n * K + k]) - zw[n], cx = int64_t(Qx[m * K + k]) - zx[m];
        a += cw * cx;
        s += (double(delta[n]) * double(cw)) * (double(dx[m]) * double(cx));
      }
      I[m * N + n] = a;
      y[m * N + n] = s;
    }
  return 0;
}

// ---------------------------------------------------------------------------------------------
// Bit-plane identities: what the binary AND + popcount kernels compute ([ABQ] abstract;
// [BitNet] §2.3)
// ---------------------------------------------------------------------------------------------

// sum_b sum_c w_b w_c popc(W_b AND X_c) over one pair of code vectors of length n: plane b of a
// code is its bit b (codes taken modulo 2^bits, i.e. two's complement when signed), plane
// weight 2^b, the top plane -2^(bits-1) when signed; planes packed 64 elements to a word.
int bqref_bitplane_dot(const int64_t* wc, int w_bits, int w_signed, const int64_t* xc, int x_bits, int x_signed,
                       int64_t n, int64_t* out) {
  if (w_bits < 1 || w_bits > 16 || x_bits < 1 || x_bits > 16 || n < 0) return -1;
  const int64_t words = (n + 63) / 64;
  int64_t tot = 0;
  for (int b = 0; b < w_bits; b++) {
    const int64_t wb = (w_signed && b == w_bits - 1) ? -(int64_t(1) << b) : (int64_t(1) << b);
    for (int c = 0; c < x_bits; c++) {
      const int64_t xw = (x_signed && c == x_bits - 1) ? -(int64_t(1) << c) : (int64_t(1) << c);
      int64_t pc = 0;
      for (int64_t w = 0; w < words; w++) {
        uint64_t Wb = 0, Xc = 0;
        for (int64_t j = 0; j < 64 && w * 64 + j < n; j++) {
          Wb |= uint64_t((wc[w * 64 + j] >> b) & 1) << j;
          Xc |= uint64_t((xc[w * 64 + j] >> c) & 1) << j;
        }
        pc += popcount64(Wb & Xc);
      }
      tot += wb * xw * pc;
    }
  }
  *out = tot;
  return 0;
}

// plane b of each code (bit b of the code modulo 2^bits): out [bits][n] of 0/1
int bqref_planes_of(const int64_t* codes, int64_t n, int bits, uint8_t* out) {
  if (bits < 1 || bits > 16 || n < 0) return -1;
  for (int b = 0; b < bits; b++)
    for (int64_t i = 0; i < n; i++) out[int64_t(b) * n + i] = uint8_t((codes[i] >> b) & 1);
  return 0;
}

// plane weights 2^b; the top plane of a two's-complement code weighs -2^(bits-1)
int bqref_plane_weights(int bits, int is_signed, int64_t* out) {
  if (bits < 1 || bits > 16) return -1;
  for (int b = 0; b < bits; b++) out[b] = (is_signed && b == bits - 1) ? -(int64_t(1) << b) : (int64_t(1) << b);
  return 0;
}

// [BitNet] §2.3 XNOR form for +-1 vectors (bit 1 <=> +1): 2 popc(xnor(a, b)) - n
int bqref_xnor_popcount_dot(const int8_t* a, const int8_t* b, int64_t n, int64_t* out) {
  if (n < 0) return -1;
  int64_t agree = 0;
  for (int64_t w = 0; w < (n + 63) / 64; w++) {
    uint64_t A = 0, B = 0, mask = 0;
    for (int64_t j = 0; j < 64 && w * 64 + j < n; j++) {
      A |= uint64_t(a[w * 64 + j] > 0) << j;
      B |= uint64_t(b[w * 64 + j] > 0) << j;
      mask |= uint64_t(1) << j;
    }
    agree += popcount64(~(A ^ B) & mask);
  }
  *out = 2 * agree - n;
  return 0;
}

// ---------------------------------------------------------------------------------------------
// BVSR bitvector-sum weights with cached coefficient sets ([BVSR] Introduction)
// ---------------------------------------------------------------------------------------------

// Nearest-rank quantile num/den of an ascending array of n values: element ceil(num n / den) - 1
int bqref_nearest_rank(const double* sorted, int64_t n, int64_t num, int64_t den, double* out) {
  if (n < 1 || den < 1) return -1;
  const int64_t rank = (num * n + den - 1) / den;
  *out = sorted[std::max<int64_t>(rank - 1, 0)];
  return 0;
}

// The 256 cached sets of a matrix (reading of the page's geometric sets on a data-range grid):
// set s = 64 j + 8 a + b has ratio r_j in {1.5, 2, 2.5, 3} and template t_i = r^i / sum_i' r^i';
// lo_a = the (2a + 1)/16 nearest-rank quantile of the vector minima, hi_b = the (2b + 1)/16
// quantile of the vector maxima (vectors: 32 consecutive k of a row); c_i = (hi_b - lo_a) t_i,
// o = lo_a, in float64 and stored float32. table [256][5] = (c0, c1, c2, c3, o).
int bqref_bvsr_set_table(const float* W, int64_t N, int64_t K, float* table) {
  if (N < 1 || K < kVec || K % kVec != 0) return -1;
  const int64_t V = N * (K / kVec);
  std::vector<double> mins(static_cast<size_t>(V)), maxs(static_cast<size_t>(V));
  for (int64_t v = 0; v < V; v++) {
    const float* e = W + v * kVec;
    float lo = e[0], hi = e[0];
    for (int i = 1; i < kVec; i++) {
      lo = std::min(lo, e[i]);
      hi = std::max(hi, e[i]);
    }
    mins[size_t(v)] = lo;
    maxs[size_t(v)] = hi;
  }
  std::sort(mins.begin(), mins.end());
  std::sort(maxs.begin(), maxs.end());
  double los[kGrid], his[kGrid];
  for (int a = 0; a < kGrid; a++) bqref_nearest_rank(mins.data(), V, 2 * a + 1, 16, &los[a]);
  for (int b = 0; b < kGrid; b++) bqref_nearest_rank(maxs.data(), V, 2 * b + 1, 16, &his[b]);
  for (int j = 0; j < 4; j++) {
    const double r = kRatios[j];
    double pw[kPlanes], tsum = 0.0;
    for (int i = 0; i < kPlanes; i++) {
      pw[i] = 1.0;
      for (int e = 0; e < i; e++) pw[i] *= r;
      tsum += pw[i];
    }
    for (int a = 0; a < kGrid; a++)
      for (int b = 0; b < kGrid; b++) {
        const int s = 64 * j + 8 * a + b;
        const double span = his[b] - los[a];
        for (int i = 0; i < kPlanes; i++) table[s * 5 + i] = float(span * (pw[i] / tsum));
        table[s * 5 + 4] = float(los[a]);
      }
  }
  return 0;
}

int bqref_bvsr_points(const float* table, int S, double* P);

// The quantile grid of bqref_bvsr_set_table as its raw (lo_a, hi_b) pairs: grid[8a + b] =
// (lo_a, hi_b), float64 copies of float32 quantiles.
static void bvsr_grid(const float* W, int64_t N, int64_t K, double* grid) {
  const int64_t V = N * (K / kVec);
  std::vector<double> mins(static_cast<size_t>(V)), maxs(static_cast<size_t>(V));
  for (int64_t v = 0; v < V; v++) {
    const float* e = W + v * kVec;
    float lo = e[0], hi = e[0];
    for (int i = 1; i < kVec; i++) {
      lo = std::min(lo, e[i]);
      hi = std::max(hi, e[i]);
    }
    mins[size_t(v)] = lo;
    maxs[size_t(v)] = hi;
  }
  std::sort(mins.begin(), mins.end());
  std::sort(maxs.begin(), maxs.end());
  for (int a = 0; a < kGrid; a++)
    for (int b = 0; b < kGrid; b++) {
      bqref_nearest_rank(mins.data(), V, 2 * a + 1, 16, &grid[2 * (8 * a + b)]);
      bqref_nearest_rank(maxs.data(), V, 2 * b + 1, 16, &grid[2 * (8 * a + b) + 1]);
    }
}

// Templates t_i = r^i / sum_i' r^i' of family j (ratio r_j), float64.
static void bvsr_templates(int j, double t[kPlanes]) {
  double pw[kPlanes], tsum = 0.0;
  for (int i = 0; i < kPlanes; i++) {
    pw[i] = 1.0;
    for (int e = 0; e < i; e++) pw[i] *= kRatios[j];
    tsum += pw[i];
  }
  for (int i = 0; i < kPlanes; i++) t[i] = pw[i] / tsum;
}

// Set (c_0..c_3, o) of family j on the range [lo, hi]: c_i = (hi - lo) t_i and o = lo, stored
// float32 (the construction of every cached set).
static void bvsr_make_set(int j, double lo, double hi, float* row5) {
  double t[kPlanes];
  bvsr_templates(j, t);
  const double span = hi - lo;
  for (int i = 0; i < kPlanes; i++) row5[i] = float(span * t[i]);
  row5[4] = float(lo);
}

// Squared error of one vector under one set (nearest of its 16 points per element, the lowest
// code on a tie; errors added in element order, float64).
static double bvsr_vector_error(const float* w, const float* row5) {
  double P[16];
  bqref_bvsr_points(row5, 1, P);
  double err = 0.0;
  for (int e = 0; e < kVec; e++) {
    const double we = double(w[e]);
    int bc = 0;
    double bd = std::fabs(we - P[0]);
    for (int c = 1; c < 16; c++) {
      const double d = std::fabs(we - P[c]);
      if (d < bd) { bd = d; bc = c; }
    }
    const double de = we - P[bc];
    err = err + de * de;
  }
  return err;
}

// Fixed-point value of a vector extreme for the cluster sums: round-to-nearest of v 2^40 (the
// scaling is exact), so that sums of any number of them are exact and independent of order.
static int64_t bvsr_fix(float v) { return std::llrint(std::ldexp(double(v), 40)); }

// [BVSR] Introduction, coefficient cache: the sets are shared by many weight vectors through a
// selection step the page calls the coefficient cache. Clustering reading (the page gives no
// procedure; every step below is a reading):
//  1. each vector v takes its own range lo_v = min, hi_v = max and the ratio family j_v whose set
//     on that range, (c = (hi_v - lo_v) t_j, o = lo_v), gives it the least squared error (the
//     lowest j on a tie);
//  2. per family j, the points (lo_v, hi_v) of its vectors are clustered by Lloyd's k-means into
//     64 centroids, started from the 8 x 8 quantile grid of bqref_bvsr_set_table (centroid
//     8a + b = (lo_a, hi_b)); a round assigns every point to the nearest centroid (squared
//     Euclidean distance in float64, the lowest index on a tie), then moves each centroid that
//     has points to their mean, computed exactly as sum_v fix(v) / count / 2^40 with fix(v) =
//     rn(v 2^40) summed in int64 (order-independent); a centroid without points stays;
//  3. set 64 j + c is the family-j set on centroid c's range: c_i = (hi_c - lo_c) t_{j,i} and
//     o = lo_c, stored float32. With rounds = 0 this is bqref_bvsr_set_table.
// Out: table [256][5]; family [V] (nullable): j_v; assign [V] (nullable): the cluster of the last
// round (0 without rounds); centroids [4][64][2] (nullable): final (lo, hi) per family and cluster.
int bqref_bvsr_cluster_table(const float* W, int64_t N, int64_t K, int rounds, float* table, uint8_t* family,
                             uint8_t* assign, double* centroids) {
  if (N < 1 || K < kVec || K % kVec != 0 || rounds < 0) return -1;
  const int64_t V = N * (K / kVec);
  double grid[2 * kGrid * kGrid];
  bvsr_grid(W, N, K, grid);
  std::vector<float> lo(static_cast<size_t>(V)), hi(static_cast<size_t>(V));
  std::vector<uint8_t> fam(static_cast<size_t>(V)), asg(static_cast<size_t>(V), 0);
#pragma omp parallel for schedule(static)
  for (int64_t v = 0; v < V; v++) {
    const float* e = W + v * kVec;
    float l = e[0], h = e[0];
    for (int i = 1; i < kVec; i++) {
      l = std::min(l, e[i]);
      h = std::max(h, e[i]);
    }
    lo[size_t(v)] = l;
    hi[size_t(v)] = h;
    int bj = 0;
    double be = 0.0;
    for (int j = 0; j < 4; j++) {
      float row5[5];
      bvsr_make_set(j, double(l), double(h), row5);
      const double err = bvsr_vector_error(e, row5);
      if (j == 0 || err < be) { be = err; bj = j; }
    }
    fam[size_t(v)] = uint8_t(bj);
  }
  double cen[4][kGrid * kGrid][2];
  for (int j = 0; j < 4; j++)
    for (int c = 0; c < kGrid * kGrid; c++) {
      cen[j][c][0] = grid[2 * c];
      cen[j][c][1] = grid[2 * c + 1];
    }
  for (int r = 0; r < rounds; r++) {
#pragma omp parallel for schedule(static)
    for (int64_t v = 0; v < V; v++) {
      const int j = fam[size_t(v)];
      int bc = 0;
      double bd = 0.0;
      for (int c = 0; c < kGrid * kGrid; c++) {
        const double dl = double(lo[size_t(v)]) - cen[j][c][0], dh = double(hi[size_t(v)]) - cen[j][c][1];
        const double d = dl * dl + dh * dh;
        if (c == 0 || d < bd) { bd = d; bc = c; }
      }
      asg[size_t(v)] = uint8_t(bc);
    }
    int64_t sl[4][kGrid * kGrid] = {}, sh[4][kGrid * kGrid] = {}, cnt[4][kGrid * kGrid] = {};
    for (int64_t v = 0; v < V; v++) {
      const int j = fam[size_t(v)], c = asg[size_t(v)];
      sl[j][c] += bvsr_fix(lo[size_t(v)]);
      sh[j][c] += bvsr_fix(hi[size_t(v)]);
      cnt[j][c] += 1;
    }
    for (int j = 0; j < 4; j++)
      for (int c = 0; c < kGrid * kGrid; c++)
        if (cnt[j][c] > 0) {
          cen[j][c][0] = std::ldexp(double(sl[j][c]) / double(cnt[j][c]), -40);
          cen[j][c][1] = std::ldexp(double(sh[j][c]) / double(cnt[j][c]), -40);
        }
  }
  for (int j = 0; j < 4; j++)
    for (int c = 0; c < kGrid * kGrid; c++) bvsr_make_set(j, cen[j][c][0], cen[j][c][1], table + (64 * j + c) * 5);
  if (family) std::memcpy(family, fam.data(), size_t(V));
  if (assign) std::memcpy(assign, asg.data(), size_t(V));
  if (centroids) std::memcpy(centroids, cen, sizeof(cen));
  return 0;
}

// P[s][code] = o + sum of the c_i whose bit i of code is set, added in i order in float64
int bqref_bvsr_points(const float* table, int S, double* P) {
  if (S < 1) return -1;
  for (int s = 0; s < S; s++)
    for (int code = 0; code < 16; code++) {
      double acc = double(table[s * 5 + 4]);
      for (int i = 0; i < kPlanes; i++)
        if ((code >> i) & 1) acc = acc + double(table[s * 5 + i]);
      P[s * 16 + code] = acc;
    }
  return 0;
}

// Exhaustive search: for each vector and each of the 256 sets, every element takes the nearest
// of the set's 16 points (smallest |w - p|, the lowest code on a tie); the set's error is
// sum_e (w_e - p)^2 added in element order (float64); the vector takes the set of least error
// (the lowest set index on a tie). vecs [V][32] -> codes [V][32], sets [V].
int bqref_bvsr_encode(const float* vecs, int64_t V, const float* table, uint8_t* codes, uint8_t* sets) {
  if (V < 0) return -1;
  std::vector<double> P(size_t(kSets) * 16);
  bqref_bvsr_points(table, kSets, P.data());
#pragma omp parallel for schedule(dynamic, 64)
  for (int64_t v = 0; v < V; v++) {
    const float* w = vecs + v * kVec;
    double best_err = 0.0;
    int best_s = -1;
    uint8_t best_codes[kVec], cur[kVec];
    for (int s = 0; s < kSets; s++) {
      const double* ps = P.data() + size_t(s) * 16;
      double err = 0.0;
      for (int e = 0; e < kVec; e++) {
        const double we = double(w[e]);
        int bc = 0;
        double bd = std::fabs(we - ps[0]);
        for (int c = 1; c < 16; c++) {
          const double d = std::fabs(we - ps[c]);
          if (d < bd) { bd = d; bc = c; }
        }
        cur[e] = uint8_t(bc);
        const double de = we - ps[bc];
        err = err + de * de;
      }
      if (best_s < 0 || err < best_err) {
        best_err = err;
        best_s = s;
        std::memcpy(best_codes, cur, kVec);
      }
    }
    sets[v] = uint8_t(best_s);
    std::memcpy(codes + v * kVec, best_codes, kVec);
  }
  return 0;
}

// acc = sum_k code q (int64, code = sum_i 2^i b_i); y = sum_k W_hat x_hat in float64 with
// W_hat[n,k] = P[set(n, k / 32)][code(n,k)] and x_hat the per-token absmax int8 activations.
int bqref_bvsr_layer(const uint8_t* codes, const uint8_t* sets, const float* table, int64_t N, int64_t K,
                     const float* x, int64_t M, int8_t* q, float* gamma, int64_t* acc, double* y) {
  if (N < 0 || K < kVec || K % kVec != 0 || M < 0) return -1;
  std::vector<double> P(size_t(kSets) * 16);
  bqref_bvsr_points(table, kSets, P.data());
  bqref_quantize_act_int8(x, M, K, q, gamma);
#pragma omp parallel for schedule(static)
  for (int64_t n = 0; n < N; n++)
    for (int64_t m = 0; m < M; m++) {
      int64_t a = 0;
      double s = 0.0;
      const double gs = double(gamma[m]) / 127.0;
      for (int64_t k = 0; k < K; k++) {
        const int c = codes[n * K + k];
        const int set = sets[n * (K / kVec) + k / kVec];
        const int64_t v = q[m * K + k];
        a += int64_t(c) * v;
        s += P[size_t(set) * 16 + size_t(c)] * (double(v) * gs);
      }
      acc[m * N + n] = a;
      y[m * N + n] = s;
    }
  return 0;
}

// ---------------------------------------------------------------------------------------------
// size and bandwidth arithmetic, and the tolerance of the layer outputs
// ---------------------------------------------------------------------------------------------

// Memory-wall bound T <= B / (P b / 8) tokens per second ([HGF] §1.1)
double bqref_decode_tokens_per_s(double bandwidth_bytes_s, double params, double bits) {
  return bandwidth_bytes_s / (params * bits / 8.0);
}

// Storage bits per weight of the packed planes or bitvectors, scales excluded: RaBiT two sign
// planes, BitNet one, ternary two ([HGF] §4.1), ABQ w, BVSR 4 bitvectors plus one 8-bit set index
// per 32-element vector. fmt: 1 RaBiT, 2 BitNet, 3 ternary, 4 ABQ, 5 BVSR.
double bqref_weight_bits_per_param(int fmt, int w_bits) {
  switch (fmt) {
    case 1: return 2.0;
    case 2: return 1.0;
    case 3: return 2.0;
    case 4: return double(w_bits);
    case 5: return double(kPlanes) + 8.0 / double(kVec);
    default: return -1.0;
  }
}

// SiLU(z) = z / (1 + exp(-z)) ([HGF] §2.1 gate nonlinearity), float64
int bqref_silu(const double* z, int64_t n, double* out) {
  for (int64_t i = 0; i < n; i++) out[i] = z[i] / (1.0 + std::exp(-z[i]));
  return 0;
}

// max|y - y_ref| <= rel (||y_ref||_inf + 1e-6); an empty y_ref passes when y is empty too
int bqref_tolerance_ok(const double* y, int64_t ny, const double* y_ref, int64_t n, double rel) {
  if (n == 0) return ny == 0;
  double err = 0.0, mx = 0.0;
  for (int64_t i = 0; i < n; i++) {
    err = std::max(err, std::fabs(y[i] - y_ref[i]));
    mx = std::max(mx, std::fabs(y_ref[i]));
  }
  return err <= rel * (mx + 1e-6);
}

}  // extern "C"
