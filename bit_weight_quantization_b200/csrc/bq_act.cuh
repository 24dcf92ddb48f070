// Online activation quantization (one call per layer input).
//
// Grid (slices, M): every block re-reduces its token's whole row (max|x| or
// min/max) from L2, which is cheap next to a cross-block exchange, keeping the
// row in shared memory for the later passes, then codes its own slice of
// k-tiles into the B-operand fragment order. Block slice 0 also writes the
// per-token parameters, the sums and the LoRA input u.
#pragma once

#include "bq_internal.cuh"

namespace bqi {

constexpr int kActRowSmemMax = 16384;  // elements of a row kept in shared memory (32 KB, no opt-in)

struct ActArgs {
  const uint16_t* x;        // bf16 [M][K]
  uint8_t* act;             // act buffer base
  int M, K, K_pad, KT, a_bits, rank, fmt, tiles_per_slice;
  int x_smem;               // the row is kept in dynamic shared memory (K_pad * 2 bytes)
  uint64_t off_codes, off_tok, off_gsum, off_u, off_xt, off_ct, total;
  const uint16_t* lora_A;   // ternary: bf16 [K_pad][r]
  const float* h;           // RaBiT: h_p at h + p K_pad, p < rabit_paths(fmt)
};

__device__ __forceinline__ void act_write_header(const ActArgs& a) {
  uint32_t* h = reinterpret_cast<uint32_t*>(a.act);
  for (int i = threadIdx.x; i < 64; i += blockDim.x) {
    uint32_t v = 0;
    switch (i) {
      case AW_MAGIC: v = kActMagic; break;
      case AW_VERSION: v = kVersion; break;
      case AW_FMT: v = uint32_t(a.fmt); break;
      case AW_M: v = uint32_t(a.M); break;
      case AW_K: v = uint32_t(a.K); break;
      case AW_KPAD: v = uint32_t(a.K_pad); break;
      case AW_ABITS: v = uint32_t(a.a_bits); break;
      case AW_LORA_RANK: v = uint32_t(a.rank); break;
      case AW_TOTAL: v = uint32_t(a.total); break;
      case AW_TOTAL + 1: v = uint32_t(a.total >> 32); break;
      case AW_OFF_CODES: v = uint32_t(a.off_codes); break;
      case AW_OFF_CODES + 1: v = uint32_t(a.off_codes >> 32); break;
      case AW_OFF_TOK: v = uint32_t(a.off_tok); break;
      case AW_OFF_TOK + 1: v = uint32_t(a.off_tok >> 32); break;
      case AW_OFF_GSUM: v = uint32_t(a.off_gsum); break;
      case AW_OFF_GSUM + 1: v = uint32_t(a.off_gsum >> 32); break;
      case AW_OFF_U: v = uint32_t(a.off_u); break;
      case AW_OFF_U + 1: v = uint32_t(a.off_u >> 32); break;
      case AW_OFF_XT: v = uint32_t(a.off_xt); break;
      case AW_OFF_XT + 1: v = uint32_t(a.off_xt >> 32); break;
      case AW_OFF_CT: v = uint32_t(a.off_ct); break;
      case AW_OFF_CT + 1: v = uint32_t(a.off_ct >> 32); break;
      default: break;
    }
    h[i] = v;
  }
}


__device__ __forceinline__ void load4(const uint16_t* xr, int k, int K, float v[4]) {
  if (k + 3 < K) {
    const uint2 p = *reinterpret_cast<const uint2*>(xr + k);
    v[0] = __uint_as_float(p.x << 16);
    v[1] = __uint_as_float(p.x & 0xFFFF0000u);
    v[2] = __uint_as_float(p.y << 16);
    v[3] = __uint_as_float(p.y & 0xFFFF0000u);
  } else {
    for (int b = 0; b < 4; b++) v[b] = k + b < K ? bf16_bits_to_float(xr[k + b]) : 0.f;
  }
}

// four bf16 of the row at k from the block's shared copy (filled by the scale pass) or from x
__device__ __forceinline__ void load4_row(const uint16_t* xr, const uint2* xs, int k, int K, float v[4]) {
  if (xs && k + 3 < K) {
    const uint2 p = xs[k >> 2];
    v[0] = __uint_as_float(p.x << 16);
    v[1] = __uint_as_float(p.x & 0xFFFF0000u);
    v[2] = __uint_as_float(p.y << 16);
    v[3] = __uint_as_float(p.y & 0xFFFF0000u);
  } else {
    load4(xr, k, K, v);
  }
}
// the scale pass: four bf16 from x, also kept in the block's shared copy
__device__ __forceinline__ void load4_keep(const uint16_t* xr, uint2* xs, int k, int K, float v[4]) {
  if (k + 3 < K) {
    const uint2 p = *reinterpret_cast<const uint2*>(xr + k);
    if (xs) xs[k >> 2] = p;
    v[0] = __uint_as_float(p.x << 16);
    v[1] = __uint_as_float(p.x & 0xFFFF0000u);
    v[2] = __uint_as_float(p.y << 16);
    v[3] = __uint_as_float(p.y & 0xFFFF0000u);
  } else {
    load4(xr, k, K, v);
  }
}

// absmax int8: gamma = max|x|, s = 127/gamma, q = clamp(rn(x*s), -127, 127); gamma = 0 -> q = 0
__device__ __forceinline__ int q_a8(float x, float s) {
  float q = rintf(__fmul_rn(x, s));
  q = fminf(fmaxf(q, -127.f), 127.f);
  return int(q);
}
// asymmetric a-bit: q = clamp(rn(x/Delta) + z, 0, 2^a - 1)
__device__ __forceinline__ int q_asym(float x, float d, int z, int qmax) {
  long long q = (long long)rintf(__fdiv_rn(x, d)) + z;
  q = q < 0 ? 0 : q;
  q = q > qmax ? qmax : q;
  return int(q);
}

// Up to 1024 threads a block. A block that codes its token's whole row (one slice) takes the
// code sum from that pass; otherwise slice 0 codes the row once more for it (for ABQ a
// correctly rounded divide per element on that block's critical path).
template <int FMT>
__global__ void __launch_bounds__(1024) k_act_quant(ActArgs a) {
  __shared__ float shf[32], shf2[32];
  __shared__ int shi[32];
  extern __shared__ uint2 act_xs[];  // the token's row (when a.x_smem): one global read of it
  uint2* xs = a.x_smem ? act_xs : nullptr;
  const int m = blockIdx.y, slice = blockIdx.x;
  const uint16_t* xr = a.x + size_t(m) * a.K;
  pdl_trigger();
  pdl_wait();   // x (and this act buffer) may belong to the previous kernel
  if (slice == 0 && m == 0) act_write_header(a);

  // --- per-token scale (whole row) ---
  float scale = 0.f, delta = 0.f;
  int zero = 0;
  const int qmax = (1 << a.a_bits) - 1;
  if (FMT == BQ_FMT_ABQ) {
    float lo = INFINITY, hi = -INFINITY;
    for (int k = threadIdx.x * 4; k < a.K; k += blockDim.x * 4) {
      float v[4];
      load4_keep(xr, xs, k, a.K, v);
      for (int b = 0; b < 4; b++) if (k + b < a.K) { lo = fminf(lo, v[b]); hi = fmaxf(hi, v[b]); }
    }
    // one block-wide reduction for both: max of (-lo, hi)
    {
      float nlo = warp_max(-lo), whi = warp_max(hi);
      const int lane = threadIdx.x & 31, w = threadIdx.x >> 5, nw = blockDim.x >> 5;
      __syncthreads();
      if (lane == 0) { shf[w] = nlo; shf2[w] = whi; }
      __syncthreads();
      nlo = lane < nw ? shf[lane] : -INFINITY;
      whi = lane < nw ? shf2[lane] : -INFINITY;
      lo = -warp_max(nlo);
      hi = warp_max(whi);
    }
    delta = __fdiv_rn(fmaxf(__fsub_rn(hi, lo), 1e-5f), float(qmax));
    zero = int(rintf(__fdiv_rn(-lo, delta)));
  } else {
    float mx = 0.f;
    for (int k = threadIdx.x * 4; k < a.K; k += blockDim.x * 4) {
      float v[4];
      load4_keep(xr, xs, k, a.K, v);
      for (int b = 0; b < 4; b++) mx = fmaxf(mx, fabsf(v[b]));
    }
    mx = block_max(mx, shf);
    scale = mx;                                            // gamma_x
    delta = mx > 0.f ? __fdiv_rn(127.f, mx) : 0.f;         // s = 127/gamma
  }

  // --- codes for this slice of k-tiles ---
  uint32_t* codes = reinterpret_cast<uint32_t*>(a.act + a.off_codes) + size_t(m) * a.KT * 64;
  int* gsum = reinterpret_cast<int*>(a.act + a.off_gsum) + size_t(m) * (a.K_pad / 32);
  const int kt0 = slice * a.tiles_per_slice;
  const int kt1 = min(a.KT, kt0 + a.tiles_per_slice);
  const bool whole_row = kt0 == 0 && kt1 == a.KT;  // this block codes the whole row
  int row_sum = 0;                                 // this thread's share of the code sum
  for (int q4 = kt0 * 64 + threadIdx.x; q4 < kt1 * 64; q4 += blockDim.x) {
    const int k = q4 * 4;
    float v[4];
    load4_row(xr, xs, k, a.K, v);
    uint32_t word = 0;
    int qs = 0;
    for (int b = 0; b < 4; b++) {
      int q = 0;
      if (k + b < a.K) q = FMT == BQ_FMT_ABQ ? q_asym(v[b], delta, zero, qmax) : q_a8(v[b], delta);
      qs += q;
      word |= (uint32_t(q) & 0xFFu) << (8 * b);
    }
    row_sum += qs;
    const int kt = k >> 8;
    codes[kt * 64 + code_word_in_tile(k & 255)] = word;
    if (a.off_ct) {  // the tensor-core copy: [KT][16 k-units][Mp / 8][8 tokens][16 bytes]
      // within each 32-k chunk a code sits at the MMA's k position p of the weight operand in
      // tensor memory: k' = k % 32 at p = 8 ((k' % 16) / 4) + 4 (k' / 16) + k' % 4, i.e. k-unit
      // 2 (chunk) + p / 16, byte p % 16 (a word of four codes stays together)
      const int Mp = tc_tokens(a.M), kk = k & 255, kp = kk & 31;
      const int p = 8 * ((kp & 15) >> 2) + 4 * (kp >> 4) + (kp & 3);
      uint8_t* ct = a.act + a.off_ct + size_t(kt) * Mp * 256 + (2 * (kk >> 5) + (p >> 4)) * (Mp * 16) + (p & 15);
      *reinterpret_cast<uint32_t*>(ct + (m >> 3) * 128 + (m & 7) * 16) = word;
      if (m < Mp - a.M) {  // token M + m pads the MMA's N to a multiple of 16 (Mp - M < 16 <= M)
        const int mp = a.M + m;
        *reinterpret_cast<uint32_t*>(ct + (mp >> 3) * 128 + (mp & 7) * 16) = 0u;
      }
    }
    if (FMT == BQ_FMT_BVSR4) {
      // 8 consecutive threads cover one 32-element vector (blockDim and 64 are multiples of 8)
      qs += __shfl_xor_sync(0xffffffffu, qs, 1);
      qs += __shfl_xor_sync(0xffffffffu, qs, 2);
      qs += __shfl_xor_sync(0xffffffffu, qs, 4);
      if ((q4 & 7) == 0) gsum[k >> 5] = qs;
    }
  }

  // --- ternary: partial dot products of x and A over this slice's k-tiles (the LoRA input
  //     u = SiLU(sum of partials) is formed by the layer kernel) ---
  if (FMT == BQ_FMT_TERNARY_A8 && a.rank > 0) {
    float* up = reinterpret_cast<float*>(a.act + a.off_u);
    const int nw = blockDim.x >> 5, lane = threadIdx.x & 31;
    const int nc = a.rank / 8;  // 8-rank chunks
    for (int i = threadIdx.x >> 5; i < (kt1 - kt0) * nc; i += nw) {
      const int kt = kt0 + i / nc, rc = (i % nc) * 8;
      lora_tile_partial_warp(xr, a.lora_A, a.K, a.rank, kt, rc, lane, up + (size_t(kt) * a.M + m) * a.rank);
    }
  }

  if (slice != 0) return;
  // --- per-token parameters: sum of codes over the whole row (the codes pass already summed
  //     them when this block coded the whole row; padding k hold code 0) ---
  int s = row_sum;
  if (!whole_row) {
    s = 0;
    for (int k = threadIdx.x * 4; k < a.K; k += blockDim.x * 4) {
      float v[4];
      load4_row(xr, xs, k, a.K, v);
      for (int b = 0; b < 4; b++)
        if (k + b < a.K) s += FMT == BQ_FMT_ABQ ? q_asym(v[b], delta, zero, qmax) : q_a8(v[b], delta);
    }
  }
  s = block_sum(s, shi);
  uint32_t* tok = reinterpret_cast<uint32_t*>(a.act + a.off_tok) + 4 * m;
  if (threadIdx.x == 0) {
    if (FMT == BQ_FMT_ABQ) {
      tok[0] = __float_as_uint(delta); tok[1] = uint32_t(zero); tok[2] = uint32_t(s); tok[3] = 0;
    } else {
      tok[0] = __float_as_uint(scale); tok[1] = uint32_t(s); tok[2] = 0; tok[3] = 0;
    }
  }
}
// RaBiT: xt_p = h_p * x in float32 for each path p, no quantization.
__global__ void k_act_rabit(ActArgs a) {
  const int m = blockIdx.y;
  pdl_trigger();
  pdl_wait();
  if (blockIdx.x == 0 && m == 0) act_write_header(a);
  const int k = blockIdx.x * blockDim.x + threadIdx.x;
  if (k >= a.K_pad) return;
  float* xt = reinterpret_cast<float*>(a.act + a.off_xt);
  const float x = k < a.K ? bf16_bits_to_float(a.x[size_t(m) * a.K + k]) : 0.f;
  const int P = rabit_paths(a.fmt);
  for (int p = 0; p < P; p++)
    xt[(size_t(p) * a.M + m) * a.K_pad + k] = k < a.K ? __fmul_rn(a.h[size_t(p) * a.K_pad + k], x) : 0.f;
}

}  // namespace bqi
