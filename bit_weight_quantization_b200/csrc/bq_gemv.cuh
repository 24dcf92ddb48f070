// The layer: y = sum_k scales (.) (B_k . x) over packed weight bit-fields.
//
// Tensor-core formulation. On sm_100a the binary AND+popcount MMA is not a
// native tensor-core operation, while the int8 m16n8k32 MMA is; so a weight
// tile (16 rows x 256 k) is kept as bit-fields laid out in the A-fragment order:
// one AND with the mask of field j turns a lane's 16 bytes into the four A
// registers of one MMA whose bytes are field_value << (f*j). The int8 codes of
// the activations (whose two's-complement bits are the activation bit-planes)
// are the B operand, one token per B column. Each field position j keeps its
// own int32 accumulator; at the end sum_j acc_j >> (f*j) is exactly
// sum_k field_k * q_k, i.e. sum_b sum_c 2^(b+c) popc(W_b & X_c) over the
// planes of the stream.
//
// Work split: CTA = one 16-row block x one group of 8 tokens, its NW warps
// split the k-tiles; partial sums meet in shared memory, warp 0 runs the
// fused epilogue (scales, zero points, LoRA term). No cross-CTA reduction.
#pragma once

#include "bq_internal.cuh"

namespace bqi {

__device__ unsigned int g_bq_device_error;

struct GemvArgs {
  const uint8_t* tiles;
  const uint32_t* pk_hdr;
  const float* row_delta;    // ABQ Delta_w [N_pad]
  const int* row_zero;       // ABQ z_w
  const int* row_sum;        // ABQ S_w
  const uint16_t* lora_bt;   // ternary B^T bf16 [N_pad][r]
  const float* bvsr_table;   // [256][8]
  const uint8_t* bvsr_idx;   // [N_pad][K_pad/32]
  const uint32_t* rabit_planes;
  const float* rabit_g;      // g1 [N_pad], g2 [N_pad]
  const uint32_t* act_hdr;
  const uint8_t* act_codes;
  const uint32_t* act_tok;
  const float* act_u;
  const int* act_gsum;
  const float* act_xt;
  float* y;
  long long* acc;
  int N, K, N_pad, K_pad, KT, M, tile_bytes, rank, fmt, shift0, shift1, shift2;
};

// the act buffer must come from bq_quantize_act for this layer and M
__device__ __forceinline__ bool act_header_ok(const GemvArgs& a) {
  const uint32_t* h = a.act_hdr;
  return h[AW_MAGIC] == kActMagic && h[AW_FMT] == uint32_t(a.fmt) && h[AW_M] == uint32_t(a.M) &&
         h[AW_K] == uint32_t(a.K);
}

template <bool BSIGNED>
__device__ __forceinline__ void mma_u8(int (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                       uint32_t b0, uint32_t b1) {
  if (BSIGNED)
    asm("mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};\n"
        : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
  else
    asm("mma.sync.aligned.m16n8k32.row.col.s32.u8.u8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};\n"
        : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint4 ldg_stream(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

// B-operand word (mu, h) of this lane's 16 act words (4 uint4, words 2mu+h)
__device__ __forceinline__ uint32_t bword(const uint4 (&b)[4], int mu, int h) {
  const uint4& v = b[mu >> 1];
  return (mu & 1) ? (h ? v.w : v.z) : (h ? v.y : v.x);
}

// One stream of field width F: w[F] uint4 of this lane for the tile, acc[8/F][4].
template <int F, bool BSIGNED, int WN, int AN>
__device__ __forceinline__ void stream_mma(const uint4 (&w)[WN], const uint4 (&b)[4], int (&acc)[AN][4]) {
  static_assert(WN == F && AN == 8 / F, "stream register shapes");
#pragma unroll
  for (int u = 0; u < F; u++) {
#pragma unroll
    for (int j = 0; j < AN; j++) {
      constexpr uint32_t base = (F == 8) ? 0xFFu : ((1u << F) - 1u);
      const uint32_t m = (base << (F * j)) * 0x01010101u;
      const int mu = u * AN + j;
      mma_u8<BSIGNED>(acc[j], w[u].x & m, w[u].y & m, w[u].z & m, w[u].w & m, bword(b, mu, 0), bword(b, mu, 1));
    }
  }
}

// sum_j acc_j >> (F j) is the exact per-stream sum; shifted into the code's bit position
template <int F, int AN>
__device__ __forceinline__ void fold_stream(const int (&acc)[AN][4], int (&p)[4], int shift) {
#pragma unroll
  for (int c = 0; c < 4; c++) {
    int s = 0;
#pragma unroll
    for (int j = 0; j < AN; j++) s += acc[j][c] >> (F * j);
    p[c] += s * (1 << shift);
  }
}

template <int FMT, int F0, int F1, int F2, int NW>
__global__ void __launch_bounds__(NW * 32) k_gemv_mma(GemvArgs a) {
  constexpr bool BSIGNED = FMT != BQ_FMT_ABQ;
  __shared__ int red[NW > 1 ? NW - 1 : 1][32][4];
  __shared__ int bad;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int g = lane >> 2, t = lane & 3;
  const int rb = blockIdx.x, tg = blockIdx.y;
  if (threadIdx.x == 0) {
    bad = act_header_ok(a) ? 0 : 1;
    if (bad) atomicOr(&g_bq_device_error, 1u);
  }
  __syncthreads();
  if (bad) return;

  constexpr int W0 = F0 > 0 ? F0 : 1, A0 = F0 > 0 ? 8 / F0 : 1;
  constexpr int W1 = F1 > 0 ? F1 : 1, A1 = F1 > 0 ? 8 / F1 : 1;
  constexpr int W2 = F2 > 0 ? F2 : 1, A2 = F2 > 0 ? 8 / F2 : 1;
  uint4 w0[W0], w1[W1], w2[W2];
  int c0[A0][4], c1[A1][4], c2[A2][4];
#pragma unroll
  for (int j = 0; j < A0; j++) c0[j][0] = c0[j][1] = c0[j][2] = c0[j][3] = 0;
#pragma unroll
  for (int j = 0; j < A1; j++) c1[j][0] = c1[j][1] = c1[j][2] = c1[j][3] = 0;
#pragma unroll
  for (int j = 0; j < A2; j++) c2[j][0] = c2[j][1] = c2[j][2] = c2[j][3] = 0;

  const int tok_b = tg * 8 + g;                  // this lane's B column (token)
  const bool has_tok = tok_b < a.M;
  const uint4* actp = reinterpret_cast<const uint4*>(a.act_codes) + (size_t(has_tok ? tok_b : 0) * a.KT) * 16 + t * 4;
  const uint8_t* tbase = a.tiles + size_t(rb) * a.KT * a.tile_bytes + lane * 16;

  for (int kt = warp; kt < a.KT; kt += NW) {
    const uint8_t* tp = tbase + size_t(kt) * a.tile_bytes;
    if constexpr (F0 > 0) {
#pragma unroll
      for (int u = 0; u < F0; u++) w0[u] = ldg_stream(tp + u * 512);
    }
    if constexpr (F1 > 0) {
#pragma unroll
      for (int u = 0; u < F1; u++) w1[u] = ldg_stream(tp + (F0 + u) * 512);
    }
    if constexpr (F2 > 0) {
#pragma unroll
      for (int u = 0; u < F2; u++) w2[u] = ldg_stream(tp + (F0 + F1 + u) * 512);
    }
    uint4 b[4];
#pragma unroll
    for (int i = 0; i < 4; i++) b[i] = has_tok ? __ldg(actp + size_t(kt) * 16 + i) : make_uint4(0, 0, 0, 0);
    if constexpr (F0 > 0) stream_mma<F0, BSIGNED>(w0, b, c0);
    if constexpr (F1 > 0) stream_mma<F1, BSIGNED>(w1, b, c1);
    if constexpr (F2 > 0) stream_mma<F2, BSIGNED>(w2, b, c2);
  }

  int p[4] = {0, 0, 0, 0};
  if constexpr (F0 > 0) fold_stream<F0>(c0, p, a.shift0);
  if constexpr (F1 > 0) fold_stream<F1>(c1, p, a.shift1);
  if constexpr (F2 > 0) fold_stream<F2>(c2, p, a.shift2);

  if (NW > 1) {
    if (warp > 0)
#pragma unroll
      for (int c = 0; c < 4; c++) red[warp - 1][lane][c] = p[c];
    __syncthreads();
    if (warp != 0) return;
    for (int w = 0; w < NW - 1; w++)
#pragma unroll
      for (int c = 0; c < 4; c++) p[c] += red[w][lane][c];
  }

  // fused epilogue: lane holds (row g | g+8) x (token 2t | 2t+1)
  const float tscale = __uint_as_float(a.pk_hdr[HW_TSCALE]);
#pragma unroll
  for (int c = 0; c < 4; c++) {
    const int row = rb * 16 + g + 8 * (c >> 1);
    const int tok = tg * 8 + 2 * t + (c & 1);
    if (row >= a.N || tok >= a.M) continue;
    const uint32_t* tk = a.act_tok + 4 * tok;
    long long acc;
    float yv;
    if (FMT == BQ_FMT_BITNET_W1A8) {
      // p = sum_k neg_k q_k  ->  sum_k sign_k q_k = sum q - 2p
      acc = (long long)int(tk[1]) - 2ll * p[c];
      yv = __fmul_rn(tscale, __fdiv_rn(__uint_as_float(tk[0]), 127.f)) * float(acc);
    } else if (FMT == BQ_FMT_TERNARY_A8) {
      // p = sum_k (T_k + 1) q_k  ->  sum_k T_k q_k = p - sum q
      acc = (long long)p[c] - (long long)int(tk[1]);
      yv = __fmul_rn(tscale, __fdiv_rn(__uint_as_float(tk[0]), 127.f)) * float(acc);
      if (a.rank > 0) {
        const float* u = a.act_u + size_t(tok) * a.rank;
        const uint16_t* bt = a.lora_bt + size_t(row) * a.rank;
        float l = 0.f;
        for (int r = 0; r < a.rank; r++) l = fmaf(u[r], bf16_bits_to_float(bt[r]), l);
        yv += tanhf(__uint_as_float(a.pk_hdr[HW_LORA_ALPHA])) * l;
      }
    } else {
      // ABQ: I = P - z_x S_w - z_w S_x + K z_w z_x
      const long long zx = int(tk[1]), sx = int(tk[2]);
      const long long zw = a.row_zero[row], sw = a.row_sum[row];
      acc = (long long)p[c] - zx * sw - zw * sx + (long long)a.K * zw * zx;
      yv = __fmul_rn(a.row_delta[row], __uint_as_float(tk[0])) * float(acc);
    }
    a.y[size_t(tok) * a.N + row] = yv;
    if (a.acc) a.acc[size_t(tok) * a.N + row] = acc;
  }
}

// ---------------------------------------------------------------------------
// BVSR: four 1-bit planes; every 32-k MMA block is one vector per row, with its
// own coefficient set, so each tile folds its planes immediately:
//   y += (gamma_x/127) [ sc_s (sum_i R_i T_i) + o_s S_v ],  T_i = acc_i >> j
// (c_i = sc_s R_i for the integer ratio templates R of set s).
// ---------------------------------------------------------------------------
template <int NW>
__global__ void __launch_bounds__(NW * 32) k_gemv_bvsr(GemvArgs a) {
  __shared__ float tab_sc[kBvsrSets], tab_o[kBvsrSets];
  __shared__ uint32_t tab_r[kBvsrSets];
  __shared__ float redf[NW > 1 ? NW - 1 : 1][32][4];
  __shared__ long long redl[NW > 1 ? NW - 1 : 1][32][4];
  __shared__ int bad;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int g = lane >> 2, t = lane & 3;
  const int rb = blockIdx.x, tg = blockIdx.y;
  if (threadIdx.x == 0) {
    bad = act_header_ok(a) ? 0 : 1;
    if (bad) atomicOr(&g_bq_device_error, 1u);
  }
  for (int s = threadIdx.x; s < kBvsrSets; s += blockDim.x) {
    const float* row = a.bvsr_table + s * kBvsrTableStride;
    tab_sc[s] = row[5];
    tab_o[s] = row[4];
    const int j = int(row[6]);
    // integer templates R_i (ratio 1.5, 2, 2.5, 3), one byte each
    const uint32_t R[4] = {0x1B120C08u, 0x08040201u, 0x7D321408u, 0x1B090301u};
    tab_r[s] = R[j & 3];
  }
  __syncthreads();
  if (bad) return;

  const int tok_b = tg * 8 + g;
  const bool has_tok = tok_b < a.M;
  const uint4* actp = reinterpret_cast<const uint4*>(a.act_codes) + (size_t(has_tok ? tok_b : 0) * a.KT) * 16 + t * 4;
  const uint8_t* tbase = a.tiles + size_t(rb) * a.KT * 2048 + lane * 16;
  const int VPR = a.K_pad / 32;
  const int row0 = rb * 16 + g, row1 = row0 + 8;
  const int tokc[2] = {tg * 8 + 2 * t, tg * 8 + 2 * t + 1};
  float yacc[4] = {0.f, 0.f, 0.f, 0.f};
  long long cacc[4] = {0, 0, 0, 0};

  for (int kt = warp; kt < a.KT; kt += NW) {
    const uint8_t* tp = tbase + size_t(kt) * 2048;
    uint4 w[4];
#pragma unroll
    for (int i = 0; i < 4; i++) w[i] = ldg_stream(tp + i * 512);
    uint4 b[4];
#pragma unroll
    for (int i = 0; i < 4; i++) b[i] = has_tok ? __ldg(actp + size_t(kt) * 16 + i) : make_uint4(0, 0, 0, 0);
    const uint2 i0 = *reinterpret_cast<const uint2*>(a.bvsr_idx + size_t(row0) * VPR + kt * 8);
    const uint2 i1 = *reinterpret_cast<const uint2*>(a.bvsr_idx + size_t(row1) * VPR + kt * 8);
    int gs[2][8];
#pragma unroll
    for (int h = 0; h < 2; h++) {
      if (tokc[h] < a.M) {
        const int4* gp = reinterpret_cast<const int4*>(a.act_gsum + size_t(tokc[h]) * VPR + kt * 8);
        const int4 x0 = gp[0], x1 = gp[1];
        gs[h][0] = x0.x; gs[h][1] = x0.y; gs[h][2] = x0.z; gs[h][3] = x0.w;
        gs[h][4] = x1.x; gs[h][5] = x1.y; gs[h][6] = x1.z; gs[h][7] = x1.w;
      } else {
#pragma unroll
        for (int j = 0; j < 8; j++) gs[h][j] = 0;
      }
    }
#pragma unroll
    for (int j = 0; j < 8; j++) {
      const uint32_t m = (1u << j) * 0x01010101u;
      int d[4][4];
#pragma unroll
      for (int i = 0; i < 4; i++) {
        d[i][0] = d[i][1] = d[i][2] = d[i][3] = 0;
        mma_u8<true>(d[i], w[i].x & m, w[i].y & m, w[i].z & m, w[i].w & m, bword(b, j, 0), bword(b, j, 1));
      }
      const int s0 = int(((j < 4 ? i0.x : i0.y) >> (8 * (j & 3))) & 0xFFu);
      const int s1 = int(((j < 4 ? i1.x : i1.y) >> (8 * (j & 3))) & 0xFFu);
#pragma unroll
      for (int c = 0; c < 4; c++) {
        const int s = (c >> 1) ? s1 : s0;
        const uint32_t R = tab_r[s];
        const int E = (int(R & 0xFF) * d[0][c] + int((R >> 8) & 0xFF) * d[1][c] +
                       int((R >> 16) & 0xFF) * d[2][c] + int(R >> 24) * d[3][c]) >> j;
        yacc[c] = fmaf(tab_sc[s], float(E), fmaf(tab_o[s], float(gs[c & 1][j]), yacc[c]));
        if (a.acc) cacc[c] += (d[0][c] + 2 * d[1][c] + 4 * d[2][c] + 8 * d[3][c]) >> j;
      }
    }
  }

  if (NW > 1) {
    if (warp > 0)
#pragma unroll
      for (int c = 0; c < 4; c++) { redf[warp - 1][lane][c] = yacc[c]; redl[warp - 1][lane][c] = cacc[c]; }
    __syncthreads();
    if (warp != 0) return;
    for (int w = 0; w < NW - 1; w++)
#pragma unroll
      for (int c = 0; c < 4; c++) { yacc[c] += redf[w][lane][c]; cacc[c] += redl[w][lane][c]; }
  }
#pragma unroll
  for (int c = 0; c < 4; c++) {
    const int row = rb * 16 + g + 8 * (c >> 1);
    const int tok = tokc[c & 1];
    if (row >= a.N || tok >= a.M) continue;
    const float gx = __uint_as_float(a.act_tok[4 * tok]);
    a.y[size_t(tok) * a.N + row] = __fdiv_rn(gx, 127.f) * yacc[c];
    if (a.acc) a.acc[size_t(tok) * a.N + row] = cacc[c];
  }
}

// ---------------------------------------------------------------------------
// RaBiT: fp32 sign-apply, y = g1 sum_k (-1)^B1 x~1 + g2 sum_k (-1)^B2 x~2 with
// x~p = h_p x; the sign bit of x~ is flipped by XOR with the plane bit.
// One warp per row; lane l takes k = 32w + l.
// ---------------------------------------------------------------------------
template <int NW>
__global__ void __launch_bounds__(NW * 32) k_gemv_rabit(GemvArgs a) {
  __shared__ int bad;
  if (threadIdx.x == 0) {
    bad = act_header_ok(a) ? 0 : 1;
    if (bad) atomicOr(&g_bq_device_error, 1u);
  }
  __syncthreads();
  if (bad) return;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int row = blockIdx.x * NW + warp;
  if (row >= a.N) return;
  const int W32 = a.K_pad / 32;
  const uint32_t* p1 = a.rabit_planes + size_t(row) * W32;
  const uint32_t* p2 = a.rabit_planes + (size_t(a.N_pad) + row) * W32;
  for (int m = 0; m < a.M; m++) {
    const float* x1 = a.act_xt + size_t(m) * a.K_pad;
    const float* x2 = a.act_xt + (size_t(a.M) + m) * a.K_pad;
    float acc1 = 0.f, acc2 = 0.f;
    for (int wd = 0; wd < W32; wd++) {
      const uint32_t b1 = __ldg(p1 + wd), b2 = __ldg(p2 + wd);
      const int k = wd * 32 + lane;
      acc1 += __uint_as_float(__float_as_uint(__ldg(x1 + k)) ^ (((b1 >> lane) & 1u) << 31));
      acc2 += __uint_as_float(__float_as_uint(__ldg(x2 + k)) ^ (((b2 >> lane) & 1u) << 31));
    }
    acc1 = warp_sum(acc1);
    acc2 = warp_sum(acc2);
    if (lane == 0) a.y[size_t(m) * a.N + row] = fmaf(a.rabit_g[row], acc1, a.rabit_g[a.N_pad + row] * acc2);
  }
}

}  // namespace bqi
