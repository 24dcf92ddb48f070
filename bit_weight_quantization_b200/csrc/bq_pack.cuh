// Weight quantize + pack kernels (offline step of the layer).
//
// Every quantizer decision that turns a float into a code is taken in float32
// with IEEE round-to-nearest operations (__fdiv_rn, rintf) or in float64 with
// explicitly rounded operations (__dadd_rn / __dmul_rn, no FMA contraction),
// so that the codes are reproducible bit for bit. Reductions (means) run in
// float64 and are stored as float32.
#pragma once

#include "bq_internal.cuh"

namespace bqi {

struct HeaderWords {
  uint32_t w[HW_COUNT];
};

__global__ void k_write_header(uint32_t* hdr, HeaderWords h) {
  int i = threadIdx.x;
  if (i < 64) hdr[i] = i < HW_COUNT ? h.w[i] : 0u;
}

// ---------------------------------------------------------------------------
// mean |W| over a tensor: per-row float64 sums, then one fixed-order total
// ---------------------------------------------------------------------------
__global__ void k_row_abs_sum(const float* __restrict__ W, int K, double* __restrict__ row_sum) {
  __shared__ double sh[32];
  const float* w = W + size_t(blockIdx.x) * K;
  double s = 0.0;
  for (int k = threadIdx.x * 4; k < K; k += blockDim.x * 4) {
    float4 v = *reinterpret_cast<const float4*>(w + k);
    s = __dadd_rn(s, fabs(double(v.x)));
    s = __dadd_rn(s, fabs(double(v.y)));
    s = __dadd_rn(s, fabs(double(v.z)));
    s = __dadd_rn(s, fabs(double(v.w)));
  }
  s = block_sum(s, sh);
  if (threadIdx.x == 0) row_sum[blockIdx.x] = s;
}

__global__ void k_tensor_mean(const double* __restrict__ row_sum, int N, double count,
                              uint32_t* __restrict__ hdr) {
  __shared__ double sh[32];
  double s = 0.0;
  for (int n = threadIdx.x; n < N; n += blockDim.x) s = __dadd_rn(s, row_sum[n]);
  s = block_sum(s, sh);
  if (threadIdx.x == 0) {
    float m = count > 0 ? __double2float_rn(__ddiv_rn(s, count)) : 0.f;
    hdr[HW_TSCALE] = __float_as_uint(m);
  }
}

// ---------------------------------------------------------------------------
// ABQ per-row asymmetric quantizer parameters: Delta, z, S_w = sum_k q
// ---------------------------------------------------------------------------
__device__ __forceinline__ int abq_code(float w, float delta, int z, int qmax) {
  float r = rintf(__fdiv_rn(w, delta));
  long long q = (long long)r + z;
  q = q < 0 ? 0 : q;
  q = q > qmax ? qmax : q;
  return int(q);
}

// The weight the ABQ codes quantize: W[n][k], or with distribution compensation (ca, cb not
// null) W[n][k] + ca[n] * cb[k], the product rounded before the sum (ABQ-LLM §3.2 eq.(3)).
__device__ __forceinline__ float abq_weight(float w, const float* ca, const float* cb, int n, int k) {
  return ca ? __fadd_rn(w, __fmul_rn(ca[n], cb[k])) : w;
}

// balanced (W2*, w_bits = 3): symmetric range [-max|W|, max|W|] in 4 steps, z = 2; the
// codes rn(W/Delta) + 2 then lie in 0..4 (|W/Delta| <= 2), under the same clamp.
// One block per row n < N; ca [N] and cb [K] are the optional compensation vectors.
__global__ void k_abq_rows(const float* __restrict__ W, const float* __restrict__ ca, const float* __restrict__ cb,
                           int K, int w_bits, int balanced, float* __restrict__ delta, int* __restrict__ zero,
                           int* __restrict__ sumq) {
  __shared__ float shf[32];
  __shared__ int shi[32];
  const int n = blockIdx.x;
  const float* w = W + size_t(n) * K;
  float lo = INFINITY, hi = -INFINITY;
  for (int k = threadIdx.x; k < K; k += blockDim.x) {
    float v = abq_weight(w[k], ca, cb, n, k);
    lo = fminf(lo, v);
    hi = fmaxf(hi, v);
  }
  lo = block_min(lo, shf);
  hi = block_max(hi, shf);
  const int qmax = (1 << w_bits) - 1;
  float d;
  int z;
  if (balanced) {
    const float hm = fmaxf(fabsf(lo), fabsf(hi));
    d = __fdiv_rn(fmaxf(__fsub_rn(hm, -hm), 1e-5f), 4.f);
    z = 2;
  } else {
    d = __fdiv_rn(fmaxf(__fsub_rn(hi, lo), 1e-5f), float(qmax));
    z = int(rintf(__fdiv_rn(-lo, d)));
  }
  int s = 0;
  for (int k = threadIdx.x; k < K; k += blockDim.x) s += abq_code(abq_weight(w[k], ca, cb, n, k), d, z, qmax);
  s = block_sum(s, shi);
  if (threadIdx.x == 0) {
    delta[blockIdx.x] = d;
    zero[blockIdx.x] = z;
    sumq[blockIdx.x] = s;
  }
}

// ---------------------------------------------------------------------------
// Tiled field packer for BitNet / ternary / ABQ: one thread per 32-bit word.
// ---------------------------------------------------------------------------
struct FieldPackArgs {
  const float* W;
  uint32_t* tiles;
  int N, K, KT, tile_words, nstreams;
  int field[4], shift[4], soff_words[4];
  const uint32_t* hdr;      // for the tensor scale (ternary gamma_W)
  const float* abq_delta;   // ABQ row params
  const int* abq_zero;
  const float* abq_comp_a;  // ABQ distribution compensation a [N], b [K] (null: off)
  const float* abq_comp_b;
  int w_bits;
  uint64_t total_words;
};

template <int FMT>
__global__ void k_pack_fields(FieldPackArgs a) {
  uint64_t idx = uint64_t(blockIdx.x) * blockDim.x + threadIdx.x;
  if (idx >= a.total_words) return;
  const int tw = a.tile_words;
  const uint64_t tile = idx / tw;
  const int wt = int(idx - tile * tw);
  const int rb = int(tile / a.KT), kt = int(tile - uint64_t(rb) * a.KT);
  int s = 0;
  while (s + 1 < a.nstreams && wt >= a.soff_words[s + 1]) s++;
  const int f = a.field[s];
  const int ws = wt - a.soff_words[s];      // word within stream: [u][lane][r]
  const int u = ws / 128, lane = (ws >> 2) & 31, r = ws & 3;
  const int g = lane >> 2, t = lane & 3;
  const int row = rb * 16 + g + 8 * (r & 1);
  const int nj = 8 / f;
  float gamma = 0.f;
  if (FMT == BQ_FMT_TERNARY_A8) gamma = __uint_as_float(a.hdr[HW_TSCALE]);
  float d = 0.f;
  int z = 0;
  const int qmax = (1 << a.w_bits) - 1;
  if (FMT == BQ_FMT_ABQ && row < a.N) { d = a.abq_delta[row]; z = a.abq_zero[row]; }
  uint32_t word = 0;
  for (int j = 0; j < nj; j++) {
    const int kb = 32 * (8 * kt + u * nj + j) + 16 * (r >> 1) + 4 * t;
    for (int b = 0; b < 4; b++) {
      const int k = kb + b;
      uint32_t field;
      const bool in = row < a.N && k < a.K;
      const float w = in ? a.W[size_t(row) * a.K + k] : 0.f;
      if (FMT == BQ_FMT_BITNET_W1A8) {
        field = in ? (w >= 0.f ? 0u : 1u) : 0u;               // bit set <=> sign -1
      } else if (FMT == BQ_FMT_TERNARY_A8) {
        int T = 0;
        if (in && gamma > 0.f) {
          float q = rintf(__fdiv_rn(w, gamma));
          T = q > 1.f ? 1 : (q < -1.f ? -1 : int(q));
        }
        field = uint32_t(T + 1);                              // {0,1,2}
      } else {                                                // ABQ
        int q = in ? abq_code(abq_weight(w, a.abq_comp_a, a.abq_comp_b, row, k), d, z, qmax) : 0;
        field = (uint32_t(q) >> a.shift[s]) & ((1u << f) - 1u);
      }
      word |= field << (8 * b + f * j);
    }
  }
  a.tiles[idx] = word;
}

// ---------------------------------------------------------------------------
// RaBiT: B1 = sign(W), g1 = mean|W|, R1 = W - g1 B1 (h1 = 1), B2 = sign(R1),
// g2 = mean|R1|; one block per row.
// ---------------------------------------------------------------------------
__global__ void k_rabit_pack(const float* __restrict__ W, int N_pad, int K, int K_pad,
                             uint32_t* __restrict__ planes, float* __restrict__ g) {
  __shared__ double sh[32];
  const int n = blockIdx.x;
  const float* w = W + size_t(n) * K;
  double s1 = 0.0;
  for (int k = threadIdx.x; k < K; k += blockDim.x) s1 = __dadd_rn(s1, fabs(double(w[k])));
  s1 = block_sum(s1, sh);
  const float g1 = __double2float_rn(__ddiv_rn(s1, double(K)));
  const double g1d = double(g1);
  const int W32 = K_pad / 32;
  double s2 = 0.0;
  for (int wd = threadIdx.x; wd < W32; wd += blockDim.x) {
    uint32_t p1 = 0, p2 = 0;
    for (int j = 0; j < 32; j++) {
      const int k = wd * 32 + j;
      if (k >= K) break;
      const float v = w[k];
      const bool neg1 = !(v >= 0.f);
      const double r1 = __dsub_rn(double(v), neg1 ? -g1d : g1d);
      const bool neg2 = !(r1 >= 0.0);
      s2 = __dadd_rn(s2, fabs(r1));
      p1 |= uint32_t(neg1) << j;
      p2 |= uint32_t(neg2) << j;
    }
    planes[size_t(n) * W32 + wd] = p1;
    planes[(size_t(N_pad) + n) * W32 + wd] = p2;
  }
  s2 = block_sum(s2, sh);
  if (threadIdx.x == 0) {
    g[n] = g1;
    g[N_pad + n] = __double2float_rn(__ddiv_rn(s2, double(K)));
  }
}

// h1 = 1, h2 (and h3 for three paths, when h3 is not null) copied; 0 on the padding columns.
__global__ void k_rabit_h(const float* __restrict__ h2, const float* __restrict__ h3, int K, int K_pad,
                          float* __restrict__ h1_out, float* __restrict__ h2_out, float* __restrict__ h3_out) {
  int k = blockIdx.x * blockDim.x + threadIdx.x;
  if (k >= K_pad) return;
  h1_out[k] = k < K ? 1.f : 0.f;
  h2_out[k] = k < K ? h2[k] : 0.f;
  if (h3) h3_out[k] = k < K ? h3[k] : 0.f;
}

// RaBiT with P paths: R_0 = W; path p takes B_p = sign(R_{p-1}) and g_p = mean_k |R_{p-1}|
// (float64 sum, stored float32), then R_p = R_{p-1} - g_p B_p h_p in float64 from the stored
// g_p and h_p (their float64 product is exact). One block per row n < N; pass p replays the
// earlier paths from W, so no residual is stored. h: the packed h_p [P][K_pad] (h1 = 1).
template <int P>
__global__ void k_rabit_pack_paths(const float* __restrict__ W, const float* __restrict__ h, int N_pad, int K,
                                   int K_pad, uint32_t* __restrict__ planes, float* __restrict__ g) {
  __shared__ double sh[32];
  __shared__ float gs[P];
  const int n = blockIdx.x;
  const float* w = W + size_t(n) * K;
  const int W32 = K_pad / 32;
  for (int p = 0; p < P; p++) {
    double s = 0.0;
    for (int wd = threadIdx.x; wd < W32; wd += blockDim.x) {
      uint32_t bits = 0;
      for (int j = 0; j < 32; j++) {
        const int k = wd * 32 + j;
        if (k >= K) break;
        double r = double(w[k]);
        for (int q = 0; q < p; q++) {
          const double gh = __dmul_rn(double(gs[q]), double(h[size_t(q) * K_pad + k]));
          r = __dsub_rn(r, r >= 0.0 ? gh : -gh);
        }
        s = __dadd_rn(s, fabs(r));
        bits |= uint32_t(!(r >= 0.0)) << j;
      }
      planes[(size_t(p) * N_pad + n) * W32 + wd] = bits;
    }
    s = block_sum(s, sh);
    if (threadIdx.x == 0) {
      const float gp = __double2float_rn(__ddiv_rn(s, double(K)));
      gs[p] = gp;
      g[size_t(p) * N_pad + n] = gp;
    }
    __syncthreads();
  }
}

// ---------------------------------------------------------------------------
// RaBiT iterative residual SVID (pack option). Path q's target is T = W - (g_o h_o) B_o
// from the other path's float32 g, h and sign plane; B_q = sign(T); one alternating
// least-squares step of |T| ~ g_q h_q^T: g_q[i] = sum_j |T_ij| h_q[j] / sum_j h_q[j]^2, then
// h_q[j] = sum_i |T_ij| g_q[i] / sum_i g_q[i]^2. float64, every sum in index order (one
// thread per row or column, the norms by one thread per block), results rounded to float32.
// ---------------------------------------------------------------------------
__device__ __forceinline__ double svid_target(float w, float go, float ho, uint32_t word_o, int j) {
  const double wo = __dmul_rn(double(go), double(ho));
  return __dsub_rn(double(w), ((word_o >> j) & 1u) ? -wo : wo);
}

// start: planes 0 (+1), g = 0, h = 1 on the real columns (0 on padding)
__global__ void k_svid_init(int N_pad, int K, int K_pad, uint32_t* __restrict__ planes, float* __restrict__ g,
                            float* __restrict__ h1, float* __restrict__ h2) {
  const uint64_t i = uint64_t(blockIdx.x) * blockDim.x + threadIdx.x;
  const uint64_t nw = 2ull * N_pad * (K_pad / 32);
  if (i < nw) planes[i] = 0u;
  if (i < uint64_t(2) * N_pad) g[i] = 0.f;
  if (i < uint64_t(K_pad)) { h1[i] = i < uint64_t(K) ? 1.f : 0.f; h2[i] = i < uint64_t(K) ? 1.f : 0.f; }
}

// sum_{i < n} v[i]^2 in index order (float64), by thread 0, shared with the block
__device__ __forceinline__ double svid_sq_norm(const float* __restrict__ v, int n, double* sh) {
  if (threadIdx.x == 0) {
    double s = 0.0;
    for (int i = 0; i < n; i++) s = __dadd_rn(s, __dmul_rn(double(v[i]), double(v[i])));
    *sh = s;
  }
  __syncthreads();
  return *sh;
}

// one thread per row: the sign plane of path q and g_q
__global__ void k_svid_rows(const float* __restrict__ W, int N, int K, int K_pad, const uint32_t* __restrict__ plane_o,
                            const float* __restrict__ g_o, const float* __restrict__ h_o, uint32_t* __restrict__ plane_q,
                            const float* __restrict__ h_q, float* __restrict__ g_q) {
  __shared__ double hh_s;
  const double hh = svid_sq_norm(h_q, K, &hh_s);
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= N) return;
  const int W32 = K_pad / 32;
  const float* w = W + size_t(i) * K;
  const float go = g_o[i];
  double acc = 0.0;
  for (int wd = 0; wd < W32; wd++) {
    const uint32_t word_o = plane_o[size_t(i) * W32 + wd];
    uint32_t bits = 0;
    for (int j = 0; j < 32; j++) {
      const int k = wd * 32 + j;
      if (k >= K) break;
      const double t = svid_target(w[k], go, h_o[k], word_o, j);
      bits |= uint32_t(!(t >= 0.0)) << j;
      acc = __dadd_rn(acc, __dmul_rn(fabs(t), double(h_q[k])));
    }
    plane_q[size_t(i) * W32 + wd] = bits;
  }
  g_q[i] = hh > 0.0 ? __double2float_rn(__ddiv_rn(acc, hh)) : 0.f;
}

// one thread per column: h_q (unchanged when g_q is all zero)
__global__ void k_svid_cols(const float* __restrict__ W, int N, int K, int K_pad, const uint32_t* __restrict__ plane_o,
                            const float* __restrict__ g_o, const float* __restrict__ h_o, const float* __restrict__ g_q,
                            float* __restrict__ h_q) {
  __shared__ double gg_s;
  const double gg = svid_sq_norm(g_q, N, &gg_s);
  const int k = blockIdx.x * blockDim.x + threadIdx.x;
  if (k >= K || !(gg > 0.0)) return;
  const int W32 = K_pad / 32, wd = k / 32, j = k % 32;
  const float ho = h_o[k];
  double acc = 0.0;
  for (int i = 0; i < N; i++) {
    const double t = svid_target(W[size_t(i) * K + k], g_o[i], ho, plane_o[size_t(i) * W32 + wd], j);
    acc = __dadd_rn(acc, __dmul_rn(fabs(t), double(g_q[i])));
  }
  h_q[k] = __double2float_rn(__ddiv_rn(acc, gg));
}

// ---------------------------------------------------------------------------
// Ternary LoRA matrices to bf16: A [K][r] -> [K_pad][r], B [r][N] -> B^T [N_pad][r]
// ---------------------------------------------------------------------------
__global__ void k_lora_to_bf16(const float* __restrict__ A, const float* __restrict__ B, int N, int K,
                               int N_pad, int K_pad, int r, uint16_t* __restrict__ A16,
                               uint16_t* __restrict__ Bt16) {
  uint64_t i = uint64_t(blockIdx.x) * blockDim.x + threadIdx.x;
  const uint64_t na = uint64_t(K_pad) * r, nb = uint64_t(N_pad) * r;
  if (i < na) {
    int k = int(i / r), c = int(i % r);
    A16[i] = k < K ? float_to_bf16_bits(A[size_t(k) * r + c]) : 0;
  } else if (i < na + nb) {
    uint64_t j = i - na;
    int n = int(j / r), c = int(j % r);
    Bt16[j] = n < N ? float_to_bf16_bits(B[size_t(c) * N + n]) : 0;
  }
}

// ---------------------------------------------------------------------------
// BVSR: per-vector min/max keys, nearest-rank quantiles by a 32-step bitwise
// selection, the 256-set table, then the exhaustive search per vector.
// ---------------------------------------------------------------------------
__global__ void k_bvsr_minmax(const float* __restrict__ W, int K, uint64_t V, uint32_t* __restrict__ kmin,
                              uint32_t* __restrict__ kmax) {
  uint64_t v = uint64_t(blockIdx.x) * blockDim.x + threadIdx.x;
  if (v >= V) return;
  const int vpr = K / 32;
  const uint64_t n = v / vpr, kv = v % vpr;
  const float4* p = reinterpret_cast<const float4*>(W + n * K + kv * 32);
  float lo = INFINITY, hi = -INFINITY;
#pragma unroll
  for (int i = 0; i < 8; i++) {
    float4 q = p[i];
    lo = fminf(fminf(lo, q.x), fminf(q.y, fminf(q.z, q.w)));
    hi = fmaxf(fmaxf(hi, q.x), fmaxf(q.y, fmaxf(q.z, q.w)));
  }
  kmin[v] = float_key(lo);
  kmax[v] = float_key(hi);
}

// target t < 8: (2t+1)/16 quantile of the minima; t >= 8: (2(t-8)+1)/16 of the maxima
__device__ __forceinline__ uint64_t bvsr_rank(int t, uint64_t V) {
  uint64_t num = 2 * (t & 7) + 1;
  uint64_t r = (num * V + 15) / 16;
  return r < 1 ? 1 : r;
}

__device__ __forceinline__ uint32_t bvsr_answer(const uint32_t* counts, int t, uint64_t V, int from_bit) {
  uint32_t ans = 0;
  const uint64_t rk = bvsr_rank(t, V);
  for (int b = 31; b >= from_bit; b--)
    if (uint64_t(counts[b * 16 + t]) < rk) ans |= 1u << b;
  return ans;
}

// counts[bit][t] = #{keys <= ans_t(bits above) | (2^bit - 1)}
__global__ void k_bvsr_count(const uint32_t* __restrict__ kmin, const uint32_t* __restrict__ kmax,
                             uint64_t V, uint32_t* __restrict__ counts, int bit) {
  __shared__ uint32_t thr_sh[16];
  if (threadIdx.x < 16) thr_sh[threadIdx.x] = bvsr_answer(counts, threadIdx.x, V, bit + 1) | ((1u << bit) - 1u);
  __syncthreads();
  uint32_t thr[16];
#pragma unroll
  for (int t = 0; t < 16; t++) thr[t] = thr_sh[t];
  uint32_t c[16];
#pragma unroll
  for (int t = 0; t < 16; t++) c[t] = 0;
  for (uint64_t v = uint64_t(blockIdx.x) * blockDim.x + threadIdx.x; v < V;
       v += uint64_t(gridDim.x) * blockDim.x) {
    const uint32_t a = kmin[v], b = kmax[v];
#pragma unroll
    for (int t = 0; t < 8; t++) c[t] += a <= thr[t];
#pragma unroll
    for (int t = 8; t < 16; t++) c[t] += b <= thr[t];
  }
#pragma unroll
  for (int t = 0; t < 16; t++) {
    uint32_t s = warp_sum(c[t]);
    if ((threadIdx.x & 31) == 0 && s) atomicAdd(&counts[bit * 16 + t], s);
  }
}

// Table row of a set of family j on the range [lo, hi] (set s = 64j + c): c_i = (hi - lo) t_i with
// t_i = r^i / sum r^i' (float64, stored float32), o = lo; then the kernel's derived constants
// sc = (hi - lo) / sum R, the family index and the integer templates R_0..R_3 as bytes of one
// word: {8,12,18,27} {1,2,4,8} {8,20,50,125} {1,3,9,27}.
__device__ __forceinline__ void bvsr_set_row(float* row, int j, double lo, double hi) {
  const double r = 1.5 + 0.5 * j;
  const double pw[4] = {1.0, r, r * r, r * r * r};
  const double tsum = __dadd_rn(__dadd_rn(__dadd_rn(pw[0], pw[1]), pw[2]), pw[3]);
  const double span = __dsub_rn(hi, lo);
  for (int i = 0; i < 4; i++) row[i] = __double2float_rn(__dmul_rn(span, __ddiv_rn(pw[i], tsum)));
  row[4] = __double2float_rn(lo);
  const double rsum[4] = {65.0, 15.0, 203.0, 40.0};
  row[5] = __double2float_rn(__ddiv_rn(span, rsum[j]));
  row[6] = float(j);
  const uint32_t rword[4] = {0x1B120C08u, 0x08040201u, 0x7D321408u, 0x1B090301u};
  row[7] = __uint_as_float(rword[j]);
}
__device__ __forceinline__ void bvsr_write_set(float* table, int s, double lo, double hi) {
  bvsr_set_row(table + s * kBvsrTableStride, s >> 6, lo, hi);
}

// One block of 256 threads: set s = 64j + 8a + b on the quantile grid (lo_a, hi_b). With
// `grid` (the clustering pack) also the grid itself, grid[8a + b] = (lo_a, hi_b) in float64.
__global__ void k_bvsr_table(const uint32_t* counts_in, uint64_t V, float* table, double* grid) {
  __shared__ uint32_t cnt[32 * 16];
  __shared__ float lo[8], hi[8];
  for (int i = threadIdx.x; i < 32 * 16; i += blockDim.x) cnt[i] = counts_in[i];
  __syncthreads();   // every read of the counts (which share the table's memory) is done
  if (threadIdx.x < 16) {
    const float v = key_float(bvsr_answer(cnt, threadIdx.x, V, 0));
    if (threadIdx.x < 8) lo[threadIdx.x] = v; else hi[threadIdx.x - 8] = v;
  }
  __syncthreads();
  const int s = threadIdx.x, a = (s >> 3) & 7, b = s & 7;
  bvsr_write_set(table, s, double(lo[a]), double(hi[b]));
  if (grid && s < 64) {
    grid[2 * s] = double(lo[a]);
    grid[2 * s + 1] = double(hi[b]);
  }
}

// Points of set s, o + c0 b0 + c1 b1 + c2 b2 + c3 b3 summed left to right in float64.
__device__ __forceinline__ void bvsr_points(const float* __restrict__ row, double P[16]) {
  const double o = row[4], c0 = row[0], c1 = row[1], c2 = row[2], c3 = row[3];
#pragma unroll
  for (int code = 0; code < 16; code++) {
    double acc = o;
    if (code & 1) acc = __dadd_rn(acc, c0);
    if (code & 2) acc = __dadd_rn(acc, c1);
    if (code & 4) acc = __dadd_rn(acc, c2);
    if (code & 8) acc = __dadd_rn(acc, c3);
    P[code] = acc;
  }
}

// nearest point: smallest |w - p|, lowest code on an exact tie
__device__ __forceinline__ int bvsr_nearest(double w, const double P[16], double* p_out) {
  double best = INFINITY, bp = P[0];
  int bc = 0;
#pragma unroll
  for (int code = 0; code < 16; code++) {
    const double d = fabs(__dsub_rn(w, P[code]));
    if (d < best) { best = d; bc = code; bp = P[code]; }
  }
  *p_out = bp;
  return bc;
}

// One block of 256 threads (thread = set) per vector, grid-stride over vectors.
__global__ void __launch_bounds__(256) k_bvsr_search(const float* __restrict__ W, int K, int KT, uint64_t V,
                                                     const float* __restrict__ table, uint32_t* __restrict__ tiles32) {
  __shared__ float wv[32];
  __shared__ double red_e[8];
  __shared__ int red_s[8];
  __shared__ int s_best_sh;
  const int s = threadIdx.x, lane = s & 31, warp = s >> 5;
  double P[16];
  bvsr_points(table + s * kBvsrTableStride, P);
  const int vpr = K / 32;
  for (uint64_t v = blockIdx.x; v < V; v += gridDim.x) {
    const uint64_t n = v / vpr;
    const int kv = int(v % vpr);
    __syncthreads();
    if (s < 32) wv[s] = W[n * K + uint64_t(kv) * 32 + s];
    __syncthreads();
    double err = 0.0;
    for (int e = 0; e < 32; e++) {
      const double w = double(wv[e]);
      double p;
      bvsr_nearest(w, P, &p);
      const double de = __dsub_rn(w, p);
      err = __dadd_rn(err, __dmul_rn(de, de));
    }
    // argmin over sets, lowest index on a tie
    int sb = s;
    double eb = err;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const double e2 = __shfl_xor_sync(0xffffffffu, eb, o);
      const int s2 = __shfl_xor_sync(0xffffffffu, sb, o);
      if (e2 < eb || (e2 == eb && s2 < sb)) { eb = e2; sb = s2; }
    }
    if (lane == 0) { red_e[warp] = eb; red_s[warp] = sb; }
    __syncthreads();
    if (warp == 0) {
      eb = lane < 8 ? red_e[lane] : INFINITY;
      sb = lane < 8 ? red_s[lane] : 0x7fffffff;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        const double e2 = __shfl_xor_sync(0xffffffffu, eb, o);
        const int s2 = __shfl_xor_sync(0xffffffffu, sb, o);
        if (e2 < eb || (e2 == eb && s2 < sb)) { eb = e2; sb = s2; }
      }
      if (lane == 0) s_best_sh = sb;
    }
    __syncthreads();
    if (warp == 0) {
      const int sbest = s_best_sh;
      double Pb[16];
      bvsr_points(table + sbest * kBvsrTableStride, Pb);
      double p;
      const int code = bvsr_nearest(double(wv[lane]), Pb, &p);
      // tile position of element e = lane of vector (n, kv): word 2(j & 1) + (e >> 4) of lane
      // 4g + t in block j >> 1, nibble b of its low (row g) or high (row g + 8) half
      const int rb = int(n >> 4), rho = int(n & 15), g = rho & 7, rbit = rho >> 3;
      const int kt = kv >> 3, j = kv & 7;
      const int e = lane, hk = e >> 4, t = (e >> 2) & 3, b = e & 3;
      const uint64_t tile_w = (uint64_t(rb) * KT + kt) * (kBvsrTileBytes / 4);
      const uint64_t word = tile_w + uint64_t((j >> 1) * 32 + 4 * g + t) * 4 + 2 * (j & 1) + hk;
      uint32_t val = uint32_t(code) << (16 * rbit + 4 * b);
      val |= __shfl_xor_sync(0xffffffffu, val, 1);
      val |= __shfl_xor_sync(0xffffffffu, val, 2);
      if (b == 0 && val) atomicOr(&tiles32[word], val);  // rows g and g + 8 share the word
      // set index of (row rho, vector j of the tile) at byte 2048 + 8 rho + j of the tile
      if (lane == 0) reinterpret_cast<uint8_t*>(tiles32 + tile_w)[2048 + rho * 8 + j] = uint8_t(sbest);
    }
  }
}

// ---------------------------------------------------------------------------
// BVSR coefficient cache, clustering reading ("BVSR" page, Introduction): per-vector ratio
// family on the vector's own range, then per family Lloyd k-means of the vectors' (min, max)
// into 64 centroids started from the quantile grid; centroid means are exact (fixed-point
// int64 sums of rn(v 2^40), so the atomic accumulation order does not matter).
// ---------------------------------------------------------------------------
constexpr double kBvsrFix = 1099511627776.0;              // 2^40
constexpr double kBvsrUnfix = 9.094947017729282379150390625e-13;  // 2^-40

// Per vector (4 threads, one per family): the family j whose set on the vector's own range
// [min, max] (bvsr_write_set's c_i and o) gives the least squared error (nearest of 16 points per
// element, the lowest code on a tie, errors added in element order); the lowest j on a tie.
__global__ void __launch_bounds__(256) k_bvsr_family(const float* __restrict__ W, int K, uint64_t V,
                                                     uint8_t* __restrict__ fam) {
  const uint64_t gid = uint64_t(blockIdx.x) * blockDim.x + threadIdx.x;
  const uint64_t v = gid >> 2;
  const int j = int(gid & 3);
  const bool live = v < V;
  const int vpr = K / 32;
  double err = INFINITY;
  if (live) {
    const float* w = W + (v / vpr) * uint64_t(K) + uint64_t(v % vpr) * 32;
    float lo = w[0], hi = w[0];
    for (int e = 1; e < 32; e++) { lo = fminf(lo, w[e]); hi = fmaxf(hi, w[e]); }
    float row[kBvsrTableStride];
    bvsr_set_row(row, j, double(lo), double(hi));
    double P[16];
    bvsr_points(row, P);
    err = 0.0;
    for (int e = 0; e < 32; e++) {
      const double we = double(w[e]);
      double p;
      bvsr_nearest(we, P, &p);
      const double de = __dsub_rn(we, p);
      err = __dadd_rn(err, __dmul_rn(de, de));
    }
  }
  // lowest error among the vector's 4 lanes, the lowest family on a tie
  int bj = j;
  double be = err;
#pragma unroll
  for (int o = 1; o < 4; o <<= 1) {
    const double e2 = __shfl_xor_sync(0xffffffffu, be, o);
    const int j2 = __shfl_xor_sync(0xffffffffu, bj, o);
    if (e2 < be || (e2 == be && j2 < bj)) { be = e2; bj = j2; }
  }
  if (live && j == 0) fam[v] = uint8_t(bj);
}

// One k-means round's assignment: each vector to the nearest of its family's 64 centroids
// (squared distance in float64, the lowest index on a tie), adding rn(v 2^40) of its min and
// max and a count to that cluster's int64 sums (acc [256][3], zeroed before the round).
__global__ void __launch_bounds__(256) k_bvsr_assign(const uint32_t* __restrict__ kmin,
                                                     const uint32_t* __restrict__ kmax,
                                                     const uint8_t* __restrict__ fam, uint64_t V,
                                                     const double* __restrict__ cen,
                                                     unsigned long long* __restrict__ acc) {
  const uint64_t v = uint64_t(blockIdx.x) * blockDim.x + threadIdx.x;
  if (v >= V) return;
  const int j = fam[v];
  const double lo = double(key_float(kmin[v])), hi = double(key_float(kmax[v]));
  const double* c = cen + 2 * 64 * j;
  int bc = 0;
  double bd = 0.0;
  for (int k = 0; k < 64; k++) {
    const double dl = __dsub_rn(lo, c[2 * k]), dh = __dsub_rn(hi, c[2 * k + 1]);
    const double d = __dadd_rn(__dmul_rn(dl, dl), __dmul_rn(dh, dh));
    if (k == 0 || d < bd) { bd = d; bc = k; }
  }
  unsigned long long* a = acc + 3 * (64 * j + bc);
  atomicAdd(&a[0], (unsigned long long)__double2ll_rn(__dmul_rn(lo, kBvsrFix)));
  atomicAdd(&a[1], (unsigned long long)__double2ll_rn(__dmul_rn(hi, kBvsrFix)));
  atomicAdd(&a[2], 1ull);
}

// Centroid update (256 threads, one per cluster of the four families): the exact mean of the
// round's members, sum / count / 2^40 in float64; a cluster without members keeps its centroid.
__global__ void k_bvsr_update(const unsigned long long* __restrict__ acc, double* __restrict__ cen) {
  const int s = threadIdx.x;
  const long long n = (long long)acc[3 * s + 2];
  if (n <= 0) return;
  const double dn = __ll2double_rn(n);
  cen[2 * s] = __dmul_rn(__ddiv_rn(__ll2double_rn((long long)acc[3 * s]), dn), kBvsrUnfix);
  cen[2 * s + 1] = __dmul_rn(__ddiv_rn(__ll2double_rn((long long)acc[3 * s + 1]), dn), kBvsrUnfix);
}

// The clustered table: set s = 64j + c on centroid c of family j (256 threads).
__global__ void k_bvsr_cluster_sets(const double* __restrict__ cen, float* __restrict__ table) {
  const int s = threadIdx.x;
  bvsr_write_set(table, s, cen[2 * s], cen[2 * s + 1]);
}

// Every family starts from the same quantile grid: copy grid [64][2] into families 1..3.
__global__ void k_bvsr_grid_families(double* cen) {
  const int i = threadIdx.x;  // 0 .. 127
  for (int j = 1; j < 4; j++) cen[2 * 64 * j + i] = cen[i];
}

}  // namespace bqi
