// The layer: y = sum_k scales (.) (B_k . x) over packed weight bit-fields.
//
// Tensor-core formulation. On sm_100a the binary AND+popcount MMA is not a
// native tensor-core operation, while the int8 m16n8k32 MMA is; so a weight
// tile (16 rows x 256 k) is kept as bit-fields laid out in the A-fragment order:
// one AND with the mask of field j turns a lane's 16 bytes into the four A
// registers of one MMA whose bytes are field_value << (f*j). The int8 codes of
// the activations (whose two's-complement bits are the activation bit-planes)
// are the B operand, one token per B column. Each field position j keeps its
// own int32 accumulator; sum_j acc_j >> (f*j) is exactly sum_k field_k * q_k,
// i.e. sum_b sum_c 2^(b+c) popc(W_b & X_c) over the planes of the stream.
//
// Data movement. A CTA owns one 16-row block and up to 8 tokens; its warps
// split the k-tiles. At entry each warp starts one bulk (TMA) copy of its
// contiguous weight slab into shared memory (double-buffered rounds when the
// slab is large), completing on an mbarrier. The kernel is launched with
// programmatic dependent launch: it lets the next launch in the stream start at
// once, and issues only the weight copies (constant data) before
// griddepcontrol.wait; activations are read after it. The fused variant
// (bq_linear) runs the activation quantization in the prologue. Partial sums
// meet in shared memory and warp 0 runs the fused epilogue.
#pragma once

#include "bq_internal.cuh"

namespace bqi {

__device__ unsigned int g_bq_device_error;
constexpr unsigned int kErrActHeader = 1u;    // act buffer does not match the layer/M
constexpr unsigned int kErrCopyTimeout = 2u;  // a bulk copy did not complete within the wait bound
constexpr uint32_t kMaxSpin = 1u << 22;       // try_wait rounds before a wait is abandoned

// ---------------------------------------------------------------------------
// PTX wrappers: shared addresses, mbarrier, bulk copy, PDL
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;\n" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
}
__device__ __forceinline__ void fence_proxy_async() {
  asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;\n" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}
// global -> shared bulk copy; dst and src 16-byte aligned, bytes a multiple of 16
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];\n" ::"r"(
          smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
// bounded wait: false (and the device error word raised) if the phase never completes
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity) {
  for (uint32_t i = 0; i < kMaxSpin; i++)
    if (mbar_try_wait(bar, parity)) return true;
  atomicOr(&g_bq_device_error, kErrCopyTimeout);
  return false;
}

__device__ __forceinline__ uint4 lds128(const void* p) { return *reinterpret_cast<const uint4*>(p); }

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

// One layer of a group that shares its input x (same format, K and bit widths): global row
// blocks [previous rb_end, rb_end) are its row blocks 0, 1, ...
constexpr int kMaxGroup = 4;
struct GroupLayer {
  const uint8_t* tiles;
  const uint32_t* hdr;
  const float* row_delta;   // ABQ Delta_w [N_pad]
  const int* row_zero;      // ABQ z_w
  const int* row_sum;       // ABQ S_w
  float* y;                 // [M][N]
  long long* acc;           // [M][N] or null
  int N, rb_end;
};

struct LayerArgs {
  GroupLayer gl[kMaxGroup];
  int n_grp;
  // packed weights (the single layer, or the group's first)
  const uint32_t* pk_hdr;
  const uint16_t* lora_bt;  // ternary B^T bf16 [N_pad][r]
  const float* bvsr_table;  // [256][8]
  const uint32_t* rabit_planes;
  const float* rabit_g;     // g_p [P][N_pad]
  const float* rabit_h;     // h_p [P][K_pad]
  // activations: x (fused) or the act buffer
  const uint16_t* x;
  const uint32_t* act_hdr;
  const uint8_t* act_codes;
  const uint32_t* act_tok;
  const int* act_gsum;
  const float* act_xt;
  const float* u_part;      // ternary: partial x.A per 256-k tile [KT][M][r] (act buffer or workspace)
  unsigned long long act_total;  // unfused: the act buffer's size for this layer and M
  float* y;
  long long* acc;
  int N, K, N_pad, K_pad, KT, RB, M, tile_bytes, rank, fmt, a_bits, shift0, shift1, shift2;
  // work split and shared-memory carve, computed on the host:
  //   T  k-tiles per warp per row block,  C  tiles per ring chunk,  S  ring stages,
  //   tpc tokens per CTA, TG token groups, CPG CTAs per token group,
  //   WPR warps sharing one row block (the k-split), a power of two dividing NW
  int T, C, S, tpc, TG, CPG, WPR, cstride, J;
  uint32_t off_ring, off_codes, off_tok, off_u, off_gsum, off_tab, off_red, off_lbt, off_bar, smem_bytes;
  int lbt_smem;             // ternary: the CTA's B^T rows are copied to off_lbt (else read from global)
};

// ---------------------------------------------------------------------------
// activation staging into shared memory
// ---------------------------------------------------------------------------
constexpr int kMaxXChunks = 16;   // 16-byte chunks of x held in registers per thread
// shared token area (words): [16][4] per-token parameters (at most 16 tokens a CTA: BVSR from
// an act buffer; 8 otherwise), then tanh(alpha) and the group members' weight scales
constexpr int kMaxTpc = 16;
constexpr int kTokAlpha = 4 * kMaxTpc, kTokWScale = kTokAlpha + 1, kTokWords = kTokWScale + 8;

// asymmetric a-bit code: clamp(rn(x / Delta) + z, 0, 2^a - 1)
__device__ __forceinline__ int quant_asym(float x, float d, int z, int qmax) {
  long long q = (long long)rintf(__fdiv_rn(x, d)) + z;
  q = q < 0 ? 0 : q;
  return int(q > qmax ? qmax : q);
}

// Reduce v over the TPT consecutive threads of a token group (TPT a power of two, 16..1024):
// butterfly within the warp, then, for groups wider than a warp, one exchange through
// sh[warp] (each call needs its own sh). Every thread of the block calls it; every
// thread gets its group's result.
// The up to 8 warp values are read back with two 16-byte loads issued together (sh is
// 16-byte aligned, T is 4 bytes), so the exchange costs one shared-memory latency.
template <typename T, typename Op>
__device__ __forceinline__ T group_reduce(T v, int TPT, T* sh, Op op) {
  static_assert(sizeof(T) == 4, "32-bit values");
  for (int o = min(16, TPT / 2); o > 0; o >>= 1) v = op(v, __shfl_xor_sync(0xffffffffu, v, o));
  if (TPT > 32) {
    const int warp = threadIdx.x >> 5, wpg = TPT / 32, g0 = (warp / wpg) * wpg;
    if ((threadIdx.x & 31) == 0) sh[warp] = v;
    __syncthreads();
    const uint4 q0 = *reinterpret_cast<const uint4*>(sh), q1 = *reinterpret_cast<const uint4*>(sh + 4);
    const uint32_t u[8] = {q0.x, q0.y, q0.z, q0.w, q1.x, q1.y, q1.z, q1.w};
    T e[8];
#pragma unroll
    for (int w = 0; w < 8; w++) memcpy(&e[w], &u[w], 4);
    T r = e[0];
#pragma unroll
    for (int w = 1; w < 8; w++)
      if (w == g0) r = e[w];
#pragma unroll
    for (int w = 1; w < 8; w++)
      if (w > g0 && w < g0 + wpg) r = op(r, e[w]);  // warps g0, g0 + 1, ... in order
    v = r;
  }
  return v;
}

// Round-to-nearest-even of a float32 product p with |p| < 2^22: adding 1.5*2^23 leaves the
// integer in the low mantissa bits (the byte of the two's-complement code in the low byte).
__device__ __forceinline__ uint32_t rn_biased(float p) { return __float_as_uint(__fadd_rn(p, 12582912.0f)); }
constexpr uint32_t kRnBias = 0x4B400000u;

// L2 prefetch of this CTA's x rows, issued before griddepcontrol.wait. It only warms L2
// (the coherent point for the previous kernel's writes); every read of x happens after the wait.
__device__ __forceinline__ void prefetch_x(const LayerArgs& a, int m0, int mg, int NT) {
  const char* base = reinterpret_cast<const char*>(a.x + size_t(m0) * a.K);
  const int lines = (mg * a.K * 2 + 127) / 128;
  for (int i = threadIdx.x; i < lines; i += NT) asm volatile("prefetch.global.L2 [%0];" ::"l"(base + size_t(i) * 128));
}

// Token part of the output scale (slot 3 of its parameters): gamma/127 for the A8 formats
// (the epilogue multiplies BitNet alpha or ternary gamma_W in), ABQ Delta_x (times Delta_w
// per row in the epilogue).
template <int FMT>
__device__ __forceinline__ uint32_t token_scale(uint32_t word0) {
  const float g0 = __uint_as_float(word0);
  return __float_as_uint(FMT == BQ_FMT_ABQ ? g0 : __fdiv_rn(g0, 127.f));
}

// The group member holding global row block rb, and rb's index inside that member.
__device__ __forceinline__ int member_of(const LayerArgs& a, int rb, int& lrb) {
  int l = 0;
#pragma unroll
  for (int i = 0; i < kMaxGroup - 1; i++)
    if (i + 1 < a.n_grp && rb >= a.gl[i].rb_end) l = i + 1;
  lrb = rb - (l > 0 ? a.gl[l - 1].rb_end : 0);
  return l;
}

// Fused: each token of this CTA is quantized by a group of TPT threads that hold the
// token's x in registers (J 16-byte chunks each, loaded at once): per-token scale over
// the whole row, codes into the fragment-order image (token stride cstride), sum of
// codes, BVSR vector sums. Token parameters: A8 {gamma, sum q}; ABQ {Delta, z, sum q}.
template <int FMT, int NW>
__device__ void stage_quantize(const LayerArgs& a, uint8_t* smem, int m0, int mg) {
  constexpr int NT = NW * 32;
  const int tid = threadIdx.x, K = a.K;
  float* sh_lo = reinterpret_cast<float*>(smem + a.off_red);   // three separate exchange slots
  float* sh_hi = sh_lo + 32;
  int* sh_sum = reinterpret_cast<int*>(sh_lo + 64);
  int mgp = 1;
  while (mgp < mg) mgp <<= 1;
  const int TPT = NT / mgp;
  const int m = tid / TPT, lt = tid - m * TPT;
  const bool active = m < mg;
  const int nch = K / 8, npad = a.K_pad / 8;
  const uint4* xr = reinterpret_cast<const uint4*>(a.x + size_t(m0 + (active ? m : 0)) * K);
  uint4 xv[kMaxXChunks];
#pragma unroll
  for (int j = 0; j < kMaxXChunks; j++) {
    const int c = lt + j * TPT;
    xv[j] = (active && j < a.J && c < nch) ? __ldg(xr + c) : make_uint4(0, 0, 0, 0);
  }
  // pass 1: max|x| (A8) or min/max (ABQ); chunks beyond K are not real elements
  float p0 = FMT == BQ_FMT_ABQ ? INFINITY : 0.f, p1 = -INFINITY;
#pragma unroll
  for (int j = 0; j < kMaxXChunks; j++) {
    const int c = lt + j * TPT;
    if (active && j < a.J && c < nch) {
      const uint32_t w[4] = {xv[j].x, xv[j].y, xv[j].z, xv[j].w};
#pragma unroll
      for (int h = 0; h < 4; h++) {
        const float lo = __uint_as_float(w[h] << 16), hi = __uint_as_float(w[h] & 0xFFFF0000u);
        if (FMT == BQ_FMT_ABQ) { p0 = fminf(p0, fminf(lo, hi)); p1 = fmaxf(p1, fmaxf(lo, hi)); }
        else p0 = fmaxf(p0, fmaxf(fabsf(lo), fabsf(hi)));
      }
    }
  }
  float sc = 0.f, d = 1.f;
  int z = 0;
  const int qmax = (1 << a.a_bits) - 1;
  if (FMT == BQ_FMT_ABQ) {
    p0 = group_reduce(p0, TPT, sh_lo, [](float x, float y) { return fminf(x, y); });
    p1 = group_reduce(p1, TPT, sh_hi, [](float x, float y) { return fmaxf(x, y); });
    d = __fdiv_rn(fmaxf(__fsub_rn(p1, p0), 1e-5f), float(qmax));
    z = int(rintf(__fdiv_rn(-p0, d)));
  } else {
    p0 = group_reduce(p0, TPT, sh_lo, [](float x, float y) { return fmaxf(x, y); });
    sc = p0 > 0.f ? __fdiv_rn(127.f, p0) : 0.f;  // 127/gamma; gamma = 0 gives q = 0
  }
  // pass 2: codes, sums. A8: q = rn(x * sc) (|x sc| <= 127 so no clamp is reached);
  // ABQ: q = clamp(rn(x / Delta) + z, 0, 2^a - 1).
  uint32_t* cw = reinterpret_cast<uint32_t*>(smem + a.off_codes + size_t(active ? m : 0) * a.cstride);
  int* gsum = reinterpret_cast<int*>(smem + a.off_gsum);
  const int VPR = a.K_pad / 32;
  uint32_t qsum = 0;  // A8: sum of codes, from the biased floats, modulo 2^32
#pragma unroll
  for (int j = 0; j < kMaxXChunks; j++) {
    if (j >= a.J) break;
    const int c = lt + j * TPT;
    const int k = c * 8;
    uint32_t word0 = 0, word1 = 0;
    int qs = 0;
    if (active && c < nch) {
      const uint32_t w[4] = {xv[j].x, xv[j].y, xv[j].z, xv[j].w};
      uint32_t q8[8];
#pragma unroll
      for (int e = 0; e < 8; e++) {
        const float xf = __uint_as_float((e & 1) ? (w[e >> 1] & 0xFFFF0000u) : (w[e >> 1] << 16));
        if (FMT == BQ_FMT_ABQ) {
          const int q = quant_asym(xf, d, z, qmax);
          qs += q;
          q8[e] = uint32_t(q);
        } else {
          q8[e] = rn_biased(__fmul_rn(xf, sc));
          qs += int(q8[e] - kRnBias);
        }
      }
      word0 = __byte_perm(__byte_perm(q8[0], q8[1], 0x0040), __byte_perm(q8[2], q8[3], 0x0040), 0x5410);
      word1 = __byte_perm(__byte_perm(q8[4], q8[5], 0x0040), __byte_perm(q8[6], q8[7], 0x0040), 0x5410);
    }
    if (active && c < npad) {
      cw[(k >> 8) * 64 + code_word_in_tile(k & 255)] = word0;
      cw[((k + 4) >> 8) * 64 + code_word_in_tile((k + 4) & 255)] = word1;
    }
    qsum += uint32_t(qs);
    if (FMT == BQ_FMT_BVSR4) {  // 4 consecutive threads cover one 32-element vector
      qs += __shfl_xor_sync(0xffffffffu, qs, 1);
      qs += __shfl_xor_sync(0xffffffffu, qs, 2);
      if (active && c < npad && (c & 3) == 0) gsum[m * VPR + (c >> 2)] = qs;
    }
  }
  const int total = group_reduce(int(qsum), TPT, sh_sum, [](int x, int y) { return x + y; });
  uint32_t* tok = reinterpret_cast<uint32_t*>(smem + a.off_tok);
  if (active && lt == 0) {
    if (FMT == BQ_FMT_ABQ) {
      tok[4 * m + 0] = __float_as_uint(d); tok[4 * m + 1] = uint32_t(z); tok[4 * m + 2] = uint32_t(total);
    } else {
      tok[4 * m + 0] = __float_as_uint(p0); tok[4 * m + 1] = uint32_t(total);
    }
    tok[4 * m + 3] = token_scale<FMT>(tok[4 * m + 0]);
  }
}

// One token per CTA (decode): the same arithmetic as stage_quantize, with all 256 threads on
// the one token and JM (a compile-time bound on the 16-byte chunks a thread holds) unrolled.
// A8 formats: max|x| compares the bf16 bit patterns of |x| as integers (exact for
// non-negative values); ABQ: min and max in one exchange. Code sums add the packed bytes by
// dp4a; BVSR vector sums combine 4 neighbouring threads (32 elements).
template <int FMT, int NW, int JM>
__device__ void stage_quantize_1tok(const LayerArgs& a, uint8_t* smem, int m0) {
  constexpr int NT = NW * 32;
  constexpr bool ABQ = FMT == BQ_FMT_ABQ;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nch = a.K / 8, npad = a.K_pad / 8;
  const uint4* xr = reinterpret_cast<const uint4*>(a.x + size_t(m0) * a.K);
  uint4 xv[JM];
#pragma unroll
  for (int j = 0; j < JM; j++) {
    const int c = tid + j * NT;
    xv[j] = c < nch ? __ldg(xr + c) : make_uint4(0, 0, 0, 0);
  }
  float* shf = reinterpret_cast<float*>(smem + a.off_red);  // [0, 32) and [32, 64): the two exchanges
  float sc = 0.f, d = 1.f;
  int z = 0;
  uint32_t w0 = 0;  // token word 0: gamma (A8) or Delta (ABQ)
  const int qmax = (1 << a.a_bits) - 1;
  if constexpr (!ABQ) {
    uint32_t mb = 0;  // f32 bit pattern of max |x| (bf16 values widened)
#pragma unroll
    for (int j = 0; j < JM; j++) {
      const uint32_t w[4] = {xv[j].x, xv[j].y, xv[j].z, xv[j].w};
#pragma unroll
      for (int h = 0; h < 4; h++) mb = max(mb, max(w[h] & 0x7FFF0000u, (w[h] << 16) & 0x7FFF0000u));
    }
    mb = group_reduce(mb, NT, reinterpret_cast<uint32_t*>(shf), [](uint32_t x, uint32_t y) { return max(x, y); });
    const float gmax = __uint_as_float(mb);
    sc = gmax > 0.f ? __fdiv_rn(127.f, gmax) : 0.f;  // 127/gamma; gamma = 0 gives q = 0
    w0 = mb;
  } else {
    float lo = INFINITY, hi = -INFINITY;  // over the real elements only
#pragma unroll
    for (int j = 0; j < JM; j++) {
      if (tid + j * NT >= nch) continue;
      const uint32_t w[4] = {xv[j].x, xv[j].y, xv[j].z, xv[j].w};
#pragma unroll
      for (int h = 0; h < 4; h++) {
        const float e0 = __uint_as_float(w[h] << 16), e1 = __uint_as_float(w[h] & 0xFFFF0000u);
        lo = fminf(lo, fminf(e0, e1));
        hi = fmaxf(hi, fmaxf(e0, e1));
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      lo = fminf(lo, __shfl_xor_sync(0xffffffffu, lo, o));
      hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, o));
    }
    if (lane == 0) { shf[warp] = lo; shf[32 + warp] = hi; }
    __syncthreads();
    const float4 l0 = *reinterpret_cast<const float4*>(shf), l1 = *reinterpret_cast<const float4*>(shf + 4);
    const float4 h0 = *reinterpret_cast<const float4*>(shf + 32), h1 = *reinterpret_cast<const float4*>(shf + 36);
    lo = fminf(fminf(fminf(l0.x, l0.y), fminf(l0.z, l0.w)), fminf(fminf(l1.x, l1.y), fminf(l1.z, l1.w)));
    hi = fmaxf(fmaxf(fmaxf(h0.x, h0.y), fmaxf(h0.z, h0.w)), fmaxf(fmaxf(h1.x, h1.y), fmaxf(h1.z, h1.w)));
    d = __fdiv_rn(fmaxf(__fsub_rn(hi, lo), 1e-5f), float(qmax));
    z = int(rintf(__fdiv_rn(-lo, d)));
    w0 = __float_as_uint(d);
  }
  uint32_t* cw = reinterpret_cast<uint32_t*>(smem + a.off_codes);
  int* gsum = reinterpret_cast<int*>(smem + a.off_gsum);
  int qsum = 0;
#pragma unroll
  for (int j = 0; j < JM; j++) {
    const int c = tid + j * NT;
    if (j * NT >= npad) break;  // uniform: no thread has chunks left
    uint32_t word0 = 0, word1 = 0;
    if (c < nch) {
      const uint32_t w[4] = {xv[j].x, xv[j].y, xv[j].z, xv[j].w};
      uint32_t q8[8];
#pragma unroll
      for (int e = 0; e < 8; e++) {
        const float xf = __uint_as_float((e & 1) ? (w[e >> 1] & 0xFFFF0000u) : (w[e >> 1] << 16));
        q8[e] = ABQ ? uint32_t(quant_asym(xf, d, z, qmax)) : rn_biased(__fmul_rn(xf, sc));
      }
      word0 = __byte_perm(__byte_perm(q8[0], q8[1], 0x0040), __byte_perm(q8[2], q8[3], 0x0040), 0x5410);
      word1 = __byte_perm(__byte_perm(q8[4], q8[5], 0x0040), __byte_perm(q8[6], q8[7], 0x0040), 0x5410);
    }
    int qs = ABQ ? int(__dp4a(word0, 0x01010101u, __dp4a(word1, 0x01010101u, 0u)))
                 : __dp4a(int(word0), 0x01010101, __dp4a(int(word1), 0x01010101, 0));
    qsum += qs;
    if (c < npad) {  // chunks past K hold code 0
      const int k = c * 8;
      cw[(k >> 8) * 64 + code_word_in_tile(k & 255)] = word0;
      cw[((k + 4) >> 8) * 64 + code_word_in_tile((k + 4) & 255)] = word1;
    }
    if (FMT == BQ_FMT_BVSR4) {  // 4 consecutive threads cover one 32-element vector
      qs += __shfl_xor_sync(0xffffffffu, qs, 1);
      qs += __shfl_xor_sync(0xffffffffu, qs, 2);
      if (c < npad && (c & 3) == 0) gsum[c >> 2] = qs;
    }
  }
  int* shs = reinterpret_cast<int*>(smem + a.off_red) + 64;
  const int total = group_reduce(qsum, NT, shs, [](int x, int y) { return x + y; });
  if (tid == 0) {
    uint32_t* tok = reinterpret_cast<uint32_t*>(smem + a.off_tok);
    tok[0] = w0;
    tok[1] = ABQ ? uint32_t(z) : uint32_t(total);
    tok[2] = ABQ ? uint32_t(total) : 0u;
    tok[3] = token_scale<FMT>(w0);
  }
}

// Rows too long to hold in registers (more than kMaxXChunks chunks a thread, K > 32768 for
// one token): the same arithmetic as stage_quantize, reading x twice (once for the scale,
// once to code it).
template <int FMT, int NW>
__device__ void stage_quantize_reload(const LayerArgs& a, uint8_t* smem, int m0, int mg) {
  constexpr int NT = NW * 32;
  const int tid = threadIdx.x, K = a.K;
  float* sh_lo = reinterpret_cast<float*>(smem + a.off_red);
  float* sh_hi = sh_lo + 32;
  int* sh_sum = reinterpret_cast<int*>(sh_lo + 64);
  int mgp = 1;
  while (mgp < mg) mgp <<= 1;
  const int TPT = NT / mgp;
  const int m = tid / TPT, lt = tid - m * TPT;
  const bool active = m < mg;
  const int nch = K / 8, npad = a.K_pad / 8;
  const uint4* xr = reinterpret_cast<const uint4*>(a.x + size_t(m0 + (active ? m : 0)) * K);
  float p0 = FMT == BQ_FMT_ABQ ? INFINITY : 0.f, p1 = -INFINITY;
  for (int c = lt; active && c < nch; c += TPT) {
    const uint4 v = __ldg(xr + c);
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int h = 0; h < 4; h++) {
      const float lo = __uint_as_float(w[h] << 16), hi = __uint_as_float(w[h] & 0xFFFF0000u);
      if (FMT == BQ_FMT_ABQ) { p0 = fminf(p0, fminf(lo, hi)); p1 = fmaxf(p1, fmaxf(lo, hi)); }
      else p0 = fmaxf(p0, fmaxf(fabsf(lo), fabsf(hi)));
    }
  }
  float sc = 0.f, d = 1.f;
  int z = 0;
  const int qmax = (1 << a.a_bits) - 1;
  if (FMT == BQ_FMT_ABQ) {
    p0 = group_reduce(p0, TPT, sh_lo, [](float x, float y) { return fminf(x, y); });
    p1 = group_reduce(p1, TPT, sh_hi, [](float x, float y) { return fmaxf(x, y); });
    d = __fdiv_rn(fmaxf(__fsub_rn(p1, p0), 1e-5f), float(qmax));
    z = int(rintf(__fdiv_rn(-p0, d)));
  } else {
    p0 = group_reduce(p0, TPT, sh_lo, [](float x, float y) { return fmaxf(x, y); });
    sc = p0 > 0.f ? __fdiv_rn(127.f, p0) : 0.f;
  }
  uint32_t* cw = reinterpret_cast<uint32_t*>(smem + a.off_codes + size_t(active ? m : 0) * a.cstride);
  int* gsum = reinterpret_cast<int*>(smem + a.off_gsum);
  const int VPR = a.K_pad / 32;
  uint32_t qsum = 0;
  for (int c0 = 0; c0 < npad; c0 += TPT) {  // uniform trip count (the BVSR sums shuffle)
    const int c = c0 + lt;
    uint32_t word0 = 0, word1 = 0;
    int qs = 0;
    if (active && c < nch) {
      const uint4 v = __ldg(xr + c);
      const uint32_t w[4] = {v.x, v.y, v.z, v.w};
      uint32_t q8[8];
#pragma unroll
      for (int e = 0; e < 8; e++) {
        const float xf = __uint_as_float((e & 1) ? (w[e >> 1] & 0xFFFF0000u) : (w[e >> 1] << 16));
        if (FMT == BQ_FMT_ABQ) {
          const int q = quant_asym(xf, d, z, qmax);
          qs += q;
          q8[e] = uint32_t(q);
        } else {
          q8[e] = rn_biased(__fmul_rn(xf, sc));
          qs += int(q8[e] - kRnBias);
        }
      }
      word0 = __byte_perm(__byte_perm(q8[0], q8[1], 0x0040), __byte_perm(q8[2], q8[3], 0x0040), 0x5410);
      word1 = __byte_perm(__byte_perm(q8[4], q8[5], 0x0040), __byte_perm(q8[6], q8[7], 0x0040), 0x5410);
    }
    if (active && c < npad) {
      const int k = c * 8;
      cw[(k >> 8) * 64 + code_word_in_tile(k & 255)] = word0;
      cw[((k + 4) >> 8) * 64 + code_word_in_tile((k + 4) & 255)] = word1;
    }
    qsum += uint32_t(qs);
    if (FMT == BQ_FMT_BVSR4) {  // 4 consecutive threads cover one 32-element vector
      qs += __shfl_xor_sync(0xffffffffu, qs, 1);
      qs += __shfl_xor_sync(0xffffffffu, qs, 2);
      if (active && c < npad && (c & 3) == 0) gsum[m * VPR + (c >> 2)] = qs;
    }
  }
  const int total = group_reduce(int(qsum), TPT, sh_sum, [](int x, int y) { return x + y; });
  uint32_t* tok = reinterpret_cast<uint32_t*>(smem + a.off_tok);
  if (active && lt == 0) {
    if (FMT == BQ_FMT_ABQ) {
      tok[4 * m + 0] = __float_as_uint(d); tok[4 * m + 1] = uint32_t(z); tok[4 * m + 2] = uint32_t(total);
    } else {
      tok[4 * m + 0] = __float_as_uint(p0); tok[4 * m + 1] = uint32_t(total);
    }
    tok[4 * m + 3] = token_scale<FMT>(tok[4 * m + 0]);
  }
}

// The act buffer was written for this layer and M: every header word its layout depends on
// (the format, M, K, activation bits, correction rank) and its total size agree, so every
// section read below lies inside it.
__device__ __forceinline__ bool act_header_ok(const uint32_t* h, const LayerArgs& a) {
  return h[AW_MAGIC] == kActMagic && h[AW_VERSION] == kVersion && h[AW_FMT] == uint32_t(a.fmt) &&
         h[AW_M] == uint32_t(a.M) && h[AW_K] == uint32_t(a.K) && h[AW_ABITS] == uint32_t(a.a_bits) &&
         h[AW_LORA_RANK] == uint32_t(a.rank) && h[AW_TOTAL] == uint32_t(a.act_total) &&
         h[AW_TOTAL + 1] == uint32_t(a.act_total >> 32);
}

// Unfused: this CTA's tokens from the act buffer (after checking its header): the codes
// by one bulk copy per token, token parameters and BVSR sums by plain loads.
template <int FMT, int NW>
__device__ bool stage_copy(const LayerArgs& a, uint8_t* smem, int m0, int mg, uint64_t* xbar) {
  constexpr int NT = NW * 32;
  int* bad = reinterpret_cast<int*>(smem + a.off_red);
  const int tid = threadIdx.x;
  if (tid == 0) {
    const int b = !act_header_ok(a.act_hdr, a);
    *bad = b;
    if (b) {
      atomicOr(&g_bq_device_error, kErrActHeader);
    } else {
      const uint32_t per = uint32_t(a.KT) * 256u;
      mbar_expect_tx(xbar, per * uint32_t(mg));
      for (int m = 0; m < mg; m++)
        bulk_g2s(smem + a.off_codes + size_t(m) * a.cstride, a.act_codes + size_t(m0 + m) * per, per, xbar);
    }
  }
  __syncthreads();
  if (*bad) return false;
  uint32_t* tok = reinterpret_cast<uint32_t*>(smem + a.off_tok);
  if (tid < 4 * mg) tok[tid] = (tid & 3) == 3 ? token_scale<FMT>(a.act_tok[4 * m0 + tid - 3]) : a.act_tok[4 * m0 + tid];
  if (FMT == BQ_FMT_BVSR4) {
    const int VPR = a.K_pad / 32;
    int* gsum = reinterpret_cast<int*>(smem + a.off_gsum);
    for (int i = tid; i < mg * VPR; i += NT) gsum[i] = a.act_gsum[size_t(m0) * VPR + i];
  }
  return mbar_wait_bounded(xbar, 0);
}

// Ternary: u[m][r] = SiLU(sum over k-tiles of the partial dot products of x and A),
// summed in tile order, into shared memory.
__device__ void stage_lora_u(const LayerArgs& a, uint8_t* smem, int m0, int mg, int NT) {
  float* us = reinterpret_cast<float*>(smem + a.off_u);
  for (int i = threadIdx.x; i < mg * a.rank; i += NT) {
    const int m = i / a.rank, r = i - m * a.rank;
    const float* up = a.u_part + size_t(m0 + m) * a.rank + r;
    const size_t st = size_t(a.M) * a.rank;
    float zsum = 0.f;
    for (int kt = 0; kt < a.KT; kt += 8) {  // loads of 8 tiles in flight, summed in tile order
      float v[8];
#pragma unroll
      for (int e = 0; e < 8; e++) v[e] = kt + e < a.KT ? up[(kt + e) * st] : 0.f;
#pragma unroll
      for (int e = 0; e < 8; e++)
        if (kt + e < a.KT) zsum += v[e];
    }
    us[i] = zsum / (1.f + expf(-zsum));
  }
}

// Per-row ABQ parameters of a row block's rows g and g + 8 (Delta_w, z_w, S_w), loaded
// ahead of the block's tiles so the epilogue does not wait on them.
struct RowP {
  float d[2];
  int z[2], s[2];
};
template <int FMT>
__device__ __forceinline__ void load_rowp(const LayerArgs& a, int rb, int lane, RowP& rp) {
  if constexpr (FMT == BQ_FMT_ABQ) {
    int lrb;
    const GroupLayer& m = a.gl[member_of(a, rb, lrb)];
#pragma unroll
    for (int h = 0; h < 2; h++) {
      const int row = lrb * 16 + (lane >> 2) + 8 * h;  // < N_pad: the arrays are padded
      rp.d[h] = __ldg(m.row_delta + row);
      rp.z[h] = __ldg(m.row_zero + row);
      rp.s[h] = __ldg(m.row_sum + row);
    }
  }
}

// Fused epilogue for one 16-row block: lane holds (row g | g+8) x (token 2t | 2t+1).
// tok[4m + 3] holds the token's output scale (alpha gamma/127, gamma_W gamma/127,
// gamma/127 or Delta_x).
template <int FMT>
__device__ __forceinline__ void layer_epilogue(const LayerArgs& a, const uint8_t* smem, const uint32_t* tok, int rb,
                                               int m0, int mg, int lane, const RowP& rp, const uint8_t* lbt,
                                               const long long (&pl)[4], const float (&yl)[4]) {
  const int g = lane >> 2, t = lane & 3;
  // ternary: the LoRA term sum_r u[token][r] B^T[row][r] of this lane's 4 outputs, rank in
  // steps of 8 (u and both B^T rows loaded once for all four), each sum in rank order
  float lv[4] = {0.f, 0.f, 0.f, 0.f};
  if (FMT == BQ_FMT_TERNARY_A8 && a.rank > 0) {
    const float* u0 = reinterpret_cast<const float*>(smem + a.off_u) + size_t(2 * t) * a.rank;
    const float* u1 = u0 + a.rank;
    const bool v0 = 2 * t < mg, v1 = 2 * t + 1 < mg;
    const int r0 = rb * 16 + g;
    const uint4* bt0 = a.lbt_smem ? reinterpret_cast<const uint4*>(lbt + size_t(g) * a.rank * 2)
                                  : reinterpret_cast<const uint4*>(a.lora_bt + size_t(r0) * a.rank);
    const uint4* bt1 = bt0 + a.rank;  // row + 8: 8 rows of rank bf16 = rank uint4 further
    for (int q8 = 0; q8 < a.rank / 8; q8++) {
      const uint4 b0 = bt0[q8], b1 = bt1[q8];
      const float4 ua = v0 ? *reinterpret_cast<const float4*>(u0 + q8 * 8) : make_float4(0.f, 0.f, 0.f, 0.f);
      const float4 ub = v0 ? *reinterpret_cast<const float4*>(u0 + q8 * 8 + 4) : make_float4(0.f, 0.f, 0.f, 0.f);
      const float4 uc = v1 ? *reinterpret_cast<const float4*>(u1 + q8 * 8) : make_float4(0.f, 0.f, 0.f, 0.f);
      const float4 ud = v1 ? *reinterpret_cast<const float4*>(u1 + q8 * 8 + 4) : make_float4(0.f, 0.f, 0.f, 0.f);
      const float uu0[8] = {ua.x, ua.y, ua.z, ua.w, ub.x, ub.y, ub.z, ub.w};
      const float uu1[8] = {uc.x, uc.y, uc.z, uc.w, ud.x, ud.y, ud.z, ud.w};
      const uint32_t h0[4] = {b0.x, b0.y, b0.z, b0.w}, h1[4] = {b1.x, b1.y, b1.z, b1.w};
#pragma unroll
      for (int e = 0; e < 8; e++) {
        const float w0 = __uint_as_float((e & 1) ? (h0[e >> 1] & 0xFFFF0000u) : (h0[e >> 1] << 16));
        const float w1 = __uint_as_float((e & 1) ? (h1[e >> 1] & 0xFFFF0000u) : (h1[e >> 1] << 16));
        lv[0] = fmaf(uu0[e], w0, lv[0]);
        lv[1] = fmaf(uu1[e], w0, lv[1]);
        lv[2] = fmaf(uu0[e], w1, lv[2]);
        lv[3] = fmaf(uu1[e], w1, lv[3]);
      }
    }
  }
  int lrb;
  const int l = member_of(a, rb, lrb);
  const GroupLayer& mb = a.gl[l];
  const float tw = __uint_as_float(reinterpret_cast<const uint32_t*>(smem + a.off_tok)[kTokWScale + l]);
#pragma unroll
  for (int c = 0; c < 4; c++) {
    const int row = lrb * 16 + g + 8 * (c >> 1);
    const int tl = 2 * t + (c & 1);
    if (row >= mb.N || tl >= mg) continue;
    const uint32_t* tk = tok + 4 * tl;
    const float scale = (FMT == BQ_FMT_BITNET_W1A8 || FMT == BQ_FMT_TERNARY_A8)
                            ? __fmul_rn(tw, __uint_as_float(tk[3]))  // alpha or gamma_W times gamma/127
                            : __uint_as_float(tk[3]);
    long long acc;
    float yv;
    if (FMT == BQ_FMT_BITNET_W1A8) {
      // p = sum_k neg_k q_k  ->  sum_k sign_k q_k = sum q - 2p
      acc = (long long)int(tk[1]) - 2ll * pl[c];
      yv = scale * float(acc);
    } else if (FMT == BQ_FMT_TERNARY_A8) {
      // p = sum_k (T_k + 1) q_k  ->  sum_k T_k q_k = p - sum q
      acc = pl[c] - (long long)int(tk[1]);
      yv = scale * float(acc);
      if (a.rank > 0) yv += __uint_as_float(reinterpret_cast<const uint32_t*>(smem + a.off_tok)[kTokAlpha]) * lv[c];
    } else if (FMT == BQ_FMT_ABQ) {
      // I = P - z_x S_w - z_w S_x + K z_w z_x
      const long long zx = int(tk[1]), sx = int(tk[2]);
      const long long zw = rp.z[c >> 1], sw = rp.s[c >> 1];
      acc = pl[c] - zx * sw - zw * sx + (long long)a.K * zw * zx;
      yv = __fmul_rn(rp.d[c >> 1], scale) * float(acc);
    } else {
      acc = pl[c];
      yv = scale * yl[c];
    }
    mb.y[size_t(m0 + tl) * mb.N + row] = yv;
    if (mb.acc) mb.acc[size_t(m0 + tl) * mb.N + row] = acc;
  }
}

// Exact float of an integer |v| < 2^22 by the 1.5 * 2^23 bias (two full-rate ops).
__device__ __forceinline__ float small_int_to_float(int v) {
  return __fsub_rn(__int_as_float(int(kRnBias) + v), 12582912.0f);
}

// prmt.b32 in its default mode: byte i of the result is byte (s >> 4i) & 7 of the pair
// {a (bytes 0-3), b (bytes 4-7)}, or, when bit 3 of that selector nibble is set, the sign
// bit of that byte copied over all eight bits. Only the low 16 bits of s are read.
__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
  return d;
}

// Per family of coefficient sets (set index >> 6, one geometric ratio each), from its integer
// template R_0..R_3 (proportional to r^i): lo/hi = the bytes L3(c) = R_0 b_0 + R_1 b_1 + R_2 b_2
// for c = 0..3 / 4..7 (b_i the bits of c), r3 = R_3 in every byte. All entries are below 128.
struct BvsrFam {
  uint32_t lo, hi, r3, pad;
};

// One BVSR tile (16 rows x 8 vectors of 32 k) for this lane's outputs. For vector j the lane
// holds two words: the 4-bit codes of A registers a0 (row g) and a1 (row g + 8) in the low and
// high half of the first, a2 and a3 in the second, nibble b of a half being byte b of the
// register. With the set's integer template, L(c) = sum_i R_i b_i(c) = L3(c & 7) + R_3 [c >= 8]
// (at most 203, one u8 byte), and E = sum_k L(code_k) q_k comes exactly from one int8 MMA on
// the byte sums of L3(c & 7) (the family table selected by the code with its bit 3 cleared)
// and R_3 [c >= 8] (R_3 selected with bit 3 flipped, so that codes below 8 copy the sign of
// R_3 < 128, i.e. 0); no byte of the sum carries, as L(c) < 256. Per row and vector the set s
// gives o and sc = span / sum R (table words
// 4, 5): y += sc E + o S_v, S_v the vector's code sum. TWO (warp-uniform): the CTA holds more
// than one token, so outputs c = 1, 3 (token 2t + 1) are live too; with one token only c = 0, 2.
// want_acc adds sum_k code_k q_k (a third MMA on the code bytes).
// The tile's four vector pairs (the weight words and the act codes of a pair are one 16-byte
// load each) are unrolled into one block, so that the loads and MMAs of later pairs overlap the
// float epilogue of earlier ones; the tile's set bytes for rows g and g + 8 are i0, i1 (byte j
// of the pair of words).
// G2: the CTA holds a second group of 8 tokens (8..15, BVSR from an act buffer only): its codes
// bp2, code sums gs_row2 and flags tok2/tok3 go through a second MMA on the same decoded A
// operand, into yacc2 / cacc2.
template <bool G2>
__device__ __forceinline__ void bvsr_tile(const uint8_t* tp, const uint8_t* bp, bool has_tok, uint2 i0, uint2 i1,
                                          const float* tab, const BvsrFam* fam, const int* gs_row, int VPR,
                                          bool TWO, bool tok0, bool tok1, bool want_acc, float (&yacc)[4],
                                          long long (&cacc)[4], const uint8_t* bp2, bool has_tok2,
                                          const int* gs_row2, bool tok2, bool tok3, float (&yacc2)[4],
                                          long long (&cacc2)[4]) {
#pragma unroll
  for (int jp = 0; jp < 4; jp++) {
    const uint4 q = lds128(tp + jp * 512);
    const uint4 bq = has_tok ? lds128(bp + jp * 16) : make_uint4(0, 0, 0, 0);
    const uint4 bq2 = G2 && has_tok2 ? lds128(bp2 + jp * 16) : make_uint4(0, 0, 0, 0);
    const uint32_t iw0 = jp < 2 ? i0.x : i0.y, iw1 = jp < 2 ? i1.x : i1.y;
#pragma unroll
    for (int v = 0; v < 2; v++) {
      const int j = 2 * jp + v;
      const uint32_t w0 = v ? q.z : q.x, w1 = v ? q.w : q.y;
      const uint32_t b0 = v ? bq.z : bq.x, b1 = v ? bq.w : bq.y;
      const uint32_t sel[4] = {w0, w0 >> 16, w1, w1 >> 16};  // a0 (row g), a1 (g + 8), a2 (g), a3 (g + 8)
      const int s0 = int(__byte_perm(iw0, 0, 0x4440u | uint32_t(j & 3)));
      const int s1 = int(__byte_perm(iw1, 0, 0x4440u | uint32_t(j & 3)));
      const BvsrFam f0 = fam[s0 >> 6], f1 = fam[s1 >> 6];
      uint32_t a1[4];
#pragma unroll
      for (int r = 0; r < 4; r++) {
        const BvsrFam& f = (r & 1) ? f1 : f0;
        a1[r] = prmt(f.lo, f.hi, sel[r] & 0x7777u) + prmt(f.r3, f.r3, sel[r] ^ 0x8888u);
      }
      int d1[4] = {0, 0, 0, 0};
      mma_u8<true>(d1, a1[0], a1[1], a1[2], a1[3], b0, b1);
      int e1[4] = {0, 0, 0, 0};
      if (G2) mma_u8<true>(e1, a1[0], a1[1], a1[2], a1[3], v ? bq2.z : bq2.x, v ? bq2.w : bq2.y);
      if (want_acc) {  // the code bytes: c & 7 plus 8 [c >= 8]
        uint32_t a3[4];
#pragma unroll
        for (int r = 0; r < 4; r++)
          a3[r] = prmt(0x03020100u, 0x07060504u, sel[r] & 0x7777u) + prmt(0x08080808u, 0x08080808u, sel[r] ^ 0x8888u);
        int d3[4] = {0, 0, 0, 0};
        mma_u8<true>(d3, a3[0], a3[1], a3[2], a3[3], b0, b1);
#pragma unroll
        for (int c = 0; c < 4; c++) cacc[c] += d3[c];
        if (G2) {
          int e3[4] = {0, 0, 0, 0};
          mma_u8<true>(e3, a3[0], a3[1], a3[2], a3[3], v ? bq2.z : bq2.x, v ? bq2.w : bq2.y);
#pragma unroll
          for (int c = 0; c < 4; c++) cacc2[c] += e3[c];
        }
      }
      const float2 os[2] = {*reinterpret_cast<const float2*>(tab + s0 * kBvsrTableStride + 4),
                            *reinterpret_cast<const float2*>(tab + s1 * kBvsrTableStride + 4)};
      const float gsf[2] = {tok0 ? small_int_to_float(gs_row[j]) : 0.f,
                            TWO && tok1 ? small_int_to_float(gs_row[VPR + j]) : 0.f};
#pragma unroll
      for (int h = 0; h < 2; h++) {  // row g (h = 0) or g + 8
#pragma unroll
        for (int qq = 0; qq < 2; qq++) {
          if (qq == 1 && !TWO) break;  // warp-uniform
          const int c = 2 * h + qq;
          yacc[c] = fmaf(os[h].y, small_int_to_float(d1[c]), fmaf(os[h].x, gsf[qq], yacc[c]));
        }
      }
      if (G2) {
        const float gsf2[2] = {tok2 ? small_int_to_float(gs_row2[j]) : 0.f, tok3 ? small_int_to_float(gs_row2[VPR + j]) : 0.f};
#pragma unroll
        for (int c = 0; c < 4; c++)
          yacc2[c] = fmaf(os[c >> 1].y, small_int_to_float(e1[c]), fmaf(os[c >> 1].x, gsf2[c & 1], yacc2[c]));
      }
    }
  }
}

// ---------------------------------------------------------------------------
// The layer kernel for the tiled formats (BitNet, ternary, ABQ, BVSR).
// Persistent: CTA c serves token group c % TG and row blocks c / TG + i*CPG. Its
// warps form G = NW/WPR groups of WPR warps; group gr takes the CTA's row blocks
// gr, gr + G, ..., and warp w of a group owns k-tiles [w*T, w*T + T) of each. A
// warp's tiles stream through its own S-stage ring of C-tile chunks (bulk copies on
// per-stage mbarriers). A group's partial sums meet in shared memory behind that
// group's named barrier (none when WPR = 1) and one of its warps runs the fused
// epilogue: after the prologue there is no block-wide synchronization.
// ---------------------------------------------------------------------------
// Two CTAs per SM (at most 128 registers a thread): the next launch's CTA must fit beside
// this one to prefetch its weights. BVSR from an act buffer (up to 16 tokens, two MMA groups)
// runs one CTA per SM and takes the registers of a whole half of the file.
// T1: every CTA holds one token (tpc = 1); the kernel then carries only the one-token staging.
template <int FMT, int F0, int F1, int F2, int NW, bool FUSED, bool T1>
__global__ void __launch_bounds__(NW * 32, (FMT == BQ_FMT_BVSR4 && !FUSED) ? 1 : 2) k_layer(const __grid_constant__ LayerArgs a) {
  extern __shared__ __align__(128) uint8_t smem[];
  constexpr bool BSIGNED = FMT != BQ_FMT_ABQ;
  constexpr bool BVSR = FMT == BQ_FMT_BVSR4;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, g = lane >> 2, t = lane & 3;
  const int tg = blockIdx.x % a.TG, cg = blockIdx.x / a.TG;
  const int m0 = tg * a.tpc, mg = min(a.tpc, a.M - m0);
  const int n_items = cg < a.RB ? (a.RB - cg + a.CPG - 1) / a.CPG : 0;  // row blocks of this CTA
  const int WPR = a.WPR, G = NW / WPR;
  const int grp = warp / WPR, wg = warp - grp * WPR;
  const int n_gitems = grp < n_items ? (n_items - grp + G - 1) / G : 0;  // row blocks of this group
  const bool LBT = FMT == BQ_FMT_TERNARY_A8 && a.rank > 0 && a.lbt_smem && n_items > 0;

  // Let the next launch in the stream start; it only prefetches its own weights
  // before its griddepcontrol.wait.
  pdl_trigger();

  // ---- weight ring. Packed weights are written only by the pack kernels, which
  //      never trigger their dependents early, so they are complete here.
  //      This warp's chunks: e = gi * cpw + ci (gi-th row block of the group, ci < cpw),
  //      each non-empty; chunk e uses ring stage e mod S in phase (e / S) mod 2. ----
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + a.off_bar);
  uint64_t* wbar = bars + warp * a.S;
  uint64_t* tbar = bars + NW * a.S;  // BVSR coefficient table
  uint64_t* xbar = tbar + 1;         // activation codes (unfused path)
  uint64_t* lbar = tbar + 2;         // ternary B^T rows
  const int kt_begin = wg * a.T;
  const int nt = max(0, min(a.KT, kt_begin + a.T) - kt_begin);
  const int cpw = (nt + a.C - 1) / a.C;
  const int n_my = n_gitems * cpw;
  auto chunk_tiles = [&](int e) { return min(a.C, nt - (e % cpw) * a.C); };
  auto rb_of = [&](int gi) { return cg + (grp + gi * G) * a.CPG; };
  auto lbt_of = [&](int gi) { return smem + a.off_lbt + size_t(grp + gi * G) * 32 * a.rank; };
  uint8_t* ring = smem + a.off_ring + size_t(warp) * a.S * a.C * a.tile_bytes;
  auto issue = [&](int e) {
    const int st = e % a.S;
    const int kt = kt_begin + (e % cpw) * a.C;
    const uint32_t bytes = uint32_t(chunk_tiles(e)) * uint32_t(a.tile_bytes);
    int lrb;
    const uint8_t* tiles = a.gl[member_of(a, rb_of(e / cpw), lrb)].tiles;
    mbar_expect_tx(&wbar[st], bytes);
    bulk_g2s(ring + size_t(st) * a.C * a.tile_bytes, tiles + (size_t(lrb) * a.KT + kt) * a.tile_bytes, bytes,
             &wbar[st]);
  };
  const int first = min(n_my, a.S);
  if (lane == 0) {
    for (int st = 0; st < a.S; st++) mbar_init(&wbar[st], 1);
    if (warp == 0) { mbar_init(tbar, 1); mbar_init(xbar, 1); mbar_init(lbar, 1); }
    fence_mbar_init();
    for (int e = 0; e < first; e++) issue(e);
    if (BVSR && warp == 0) {
      mbar_expect_tx(tbar, kBvsrSets * kBvsrTableStride * 4);
      bulk_g2s(smem + a.off_tab, a.bvsr_table, kBvsrSets * kBvsrTableStride * 4, tbar);
    }
    if (LBT && warp == 0) {  // the B^T rows of this CTA's row blocks (16 rows x rank bf16 each)
      const uint32_t per = 32u * uint32_t(a.rank);
      mbar_expect_tx(lbar, per * uint32_t(n_items));
      for (int i = 0; i < n_items; i++)
        bulk_g2s(smem + a.off_lbt + size_t(i) * per, a.lora_bt + size_t(cg + i * a.CPG) * 16 * a.rank, per, lbar);
    }
  }
  if constexpr (FUSED) prefetch_x(a, m0, mg, NW * 32);
  int* fail = reinterpret_cast<int*>(smem + a.off_bar) + 2 * (NW * a.S + 3);  // a copy wait was abandoned
  if (tid == 0) {
    *fail = 0;
    uint32_t* tw = reinterpret_cast<uint32_t*>(smem + a.off_tok);
    for (int l = 0; l < a.n_grp; l++) tw[kTokWScale + l] = a.gl[l].hdr[HW_TSCALE];
    if (FMT == BQ_FMT_TERNARY_A8) tw[kTokAlpha] = __float_as_uint(tanhf(__uint_as_float(a.pk_hdr[HW_LORA_ALPHA])));
  }
  RowP rp;
  if (n_gitems > 0) load_rowp<FMT>(a, rb_of(0), lane, rp);
  __syncthreads();

  // ---- activations (they may be produced by the previous kernel) ----
  pdl_wait();
  bool ok = true;
  const uint32_t* tokp = reinterpret_cast<const uint32_t*>(smem + a.off_tok);
  if constexpr (FUSED) {
    if (a.J == 0) {
      stage_quantize_reload<FMT, NW>(a, smem, m0, mg);  // rows too long for registers
    } else if constexpr (T1) {
      if (a.J <= 2) stage_quantize_1tok<FMT, NW, 2>(a, smem, m0);
      else if (a.J <= 4) stage_quantize_1tok<FMT, NW, 4>(a, smem, m0);
      else if (a.J <= 8) stage_quantize_1tok<FMT, NW, 8>(a, smem, m0);
      else stage_quantize<FMT, NW>(a, smem, m0, mg);
    } else {
      stage_quantize<FMT, NW>(a, smem, m0, mg);
    }
  } else {
    ok = stage_copy<FMT, NW>(a, smem, m0, mg, xbar);
  }
  __syncthreads();
  if (FMT == BQ_FMT_TERNARY_A8 && a.rank > 0) {
    if (ok) stage_lora_u(a, smem, m0, mg, NW * 32);
    __syncthreads();
  }
  if (BVSR) {
    if (!mbar_wait_bounded(tbar, 0)) ok = false;
    // the four families' lookup tables, from the templates of sets 0, 64, 128, 192 (word 7)
    if (tid < 4 && ok) {
      const uint32_t R = reinterpret_cast<const uint32_t*>(smem + a.off_tab)[(64 * tid) * kBvsrTableStride + 7];
      const uint32_t r0 = R & 0xFFu, r1 = (R >> 8) & 0xFFu, r2 = (R >> 16) & 0xFFu, r3 = R >> 24;
      BvsrFam* fw = reinterpret_cast<BvsrFam*>(smem + a.off_tab + kBvsrSets * kBvsrTableStride * 4);
      fw[tid].lo = (r0 << 8) | (r1 << 16) | ((r0 + r1) << 24);
      fw[tid].hi = r2 | ((r2 + r0) << 8) | ((r2 + r1) << 16) | ((r2 + r1 + r0) << 24);
      fw[tid].r3 = r3 * 0x01010101u;
      fw[tid].pad = 0;
    }
    __syncthreads();
  }
  if (LBT && !mbar_wait_bounded(lbar, 0)) ok = false;

  const bool has_tok = g < mg;
  const uint8_t* bsrc = smem + a.off_codes + size_t(has_tok ? g : 0) * a.cstride + t * 64;
  // BVSR with more than 8 tokens in the CTA (from an act buffer): tokens 8..15 are a second MMA
  // group on the same decoded weights (warp-uniform)
  const bool TG2 = BVSR && !FUSED && mg > 8;
  const bool has_tok2 = TG2 && 8 + g < mg;
  const uint8_t* bsrc2 = smem + a.off_codes + size_t(has_tok2 ? 8 + g : 0) * a.cstride + t * 64;
  const int VPR = a.K_pad / 32;
  const int* gsum = reinterpret_cast<const int*>(smem + a.off_gsum);
  const float* tab = reinterpret_cast<const float*>(smem + a.off_tab);
  const BvsrFam* fam = reinterpret_cast<const BvsrFam*>(smem + a.off_tab + kBvsrSets * kBvsrTableStride * 4);
  const bool want_acc = a.gl[0].acc != nullptr;  // BVSR (never grouped)
  long long* redl = reinterpret_cast<long long*>(smem + a.off_red);                // [G][2][WPR][32][4]
  float* redf = reinterpret_cast<float*>(smem + a.off_red + 2 * NW * 32 * 4 * 8);  // same shape
  // the second token group's exchange (BVSR, more than 8 tokens) follows, in the same layout
  long long* redl2 = reinterpret_cast<long long*>(smem + a.off_red + 2 * NW * 32 * 4 * 12);
  float* redf2 = reinterpret_cast<float*>(smem + a.off_red + 2 * NW * 32 * 4 * 20);
  bool copies_ok = true;
  int waited = 0, issued = first;  // chunks this warp has waited for / has issued

  constexpr int W0 = F0 > 0 ? F0 : 1, A0 = F0 > 0 ? 8 / F0 : 1;
  constexpr int W1 = F1 > 0 ? F1 : 1, A1 = F1 > 0 ? 8 / F1 : 1;
  constexpr int W2 = F2 > 0 ? F2 : 1, A2 = F2 > 0 ? 8 / F2 : 1;
  int c0[A0][4], c1[A1][4], c2[A2][4];
  float yacc[4], yacc2[4];
  long long cacc[4], cacc2[4];

  for (int gi = 0; gi < n_gitems; gi++) {
    if (gi > 0) load_rowp<FMT>(a, rb_of(gi), lane, rp);
#pragma unroll
    for (int j = 0; j < A0; j++) c0[j][0] = c0[j][1] = c0[j][2] = c0[j][3] = 0;
#pragma unroll
    for (int j = 0; j < A1; j++) c1[j][0] = c1[j][1] = c1[j][2] = c1[j][3] = 0;
#pragma unroll
    for (int j = 0; j < A2; j++) c2[j][0] = c2[j][1] = c2[j][2] = c2[j][3] = 0;
#pragma unroll
    for (int c = 0; c < 4; c++) { yacc[c] = 0.f; cacc[c] = 0; yacc2[c] = 0.f; cacc2[c] = 0; }
    for (int ci = 0; ci < cpw; ci++) {
      const int e = gi * cpw + ci;
      const int cnt = chunk_tiles(e);
      const int st = e % a.S;
      if (copies_ok) {
        const bool got = mbar_wait_bounded(&wbar[st], uint32_t((e / a.S) & 1));
        copies_ok = __all_sync(0xffffffffu, got);
        if (copies_ok) waited = e + 1;
        else *fail = 1;
      }
      // BVSR refills the previous chunk's stage here, after this chunk's wait, rather than
      // straight after computing it: the same chunks are in flight, and the copy issue (which
      // stalls behind the shared-memory traffic of a BVSR tile) no longer sits between a
      // chunk's compute and the next wait
      if (BVSR && copies_ok && e >= 1 && e - 1 + a.S < n_my) {
        if (lane == 0) {
          fence_proxy_async();  // the previous stage's shared reads, before the last __syncwarp, are done
          issue(e - 1 + a.S);
        }
        issued = e - 1 + a.S + 1;
      }
      if (copies_ok && ok) {
        const uint8_t* sbase = ring + size_t(st) * a.C * a.tile_bytes + lane * 16;
        const int ktc = kt_begin + ci * a.C;
        for (int i = 0; i < cnt; i++) {
          const int kt = ktc + i;
          const uint8_t* tp = sbase + size_t(i) * a.tile_bytes;
          if constexpr (!BVSR) {
            uint4 b[4];
#pragma unroll
            for (int qq = 0; qq < 4; qq++) b[qq] = has_tok ? lds128(bsrc + kt * 256 + qq * 16) : make_uint4(0, 0, 0, 0);
            uint4 w0[W0], w1[W1], w2[W2];
            if constexpr (F0 > 0) {
#pragma unroll
              for (int u = 0; u < F0; u++) w0[u] = lds128(tp + u * 512);
              stream_mma<F0, BSIGNED>(w0, b, c0);
            }
            if constexpr (F1 > 0) {
#pragma unroll
              for (int u = 0; u < F1; u++) w1[u] = lds128(tp + (F0 + u) * 512);
              stream_mma<F1, BSIGNED>(w1, b, c1);
            }
            if constexpr (F2 > 0) {
#pragma unroll
              for (int u = 0; u < F2; u++) w2[u] = lds128(tp + (F0 + F1 + u) * 512);
              stream_mma<F2, BSIGNED>(w2, b, c2);
            }
          } else {
            const uint8_t* tidx = tp - lane * 16 + 2048;
            const uint2 i0 = *reinterpret_cast<const uint2*>(tidx + g * 8);
            const uint2 i1 = *reinterpret_cast<const uint2*>(tidx + (g + 8) * 8);
            const int* gs0 = gsum + size_t(2 * t) * VPR + kt * 8;
            if (!FUSED && TG2)
              bvsr_tile<true>(tp, bsrc + kt * 256, has_tok, i0, i1, tab, fam, gs0, VPR, true, 2 * t < mg, 2 * t + 1 < mg,
                              want_acc, yacc, cacc, bsrc2 + kt * 256, has_tok2, gs0 + size_t(8) * VPR, 8 + 2 * t < mg,
                              9 + 2 * t < mg, yacc2, cacc2);
            else
              bvsr_tile<false>(tp, bsrc + kt * 256, has_tok, i0, i1, tab, fam, gs0, VPR, mg > 1, 2 * t < mg,
                               2 * t + 1 < mg, want_acc, yacc, cacc, bsrc2, false, gs0, false, false, yacc2, cacc2);
          }
        }
      }
      __syncwarp();
      if (!BVSR && copies_ok && e + a.S < n_my) {
        if (lane == 0) {
          fence_proxy_async();  // this stage's shared reads are done before the copy overwrites it
          issue(e + a.S);
        }
        issued = e + a.S + 1;
      }
    }

    // ---- end of a row block: the group's sum and the fused epilogue ----
    long long p[4];
    if constexpr (!BVSR) {
      int pi[4] = {0, 0, 0, 0};
      if constexpr (F0 > 0) fold_stream<F0>(c0, pi, a.shift0);
      if constexpr (F1 > 0) fold_stream<F1>(c1, pi, a.shift1);
      if constexpr (F2 > 0) fold_stream<F2>(c2, pi, a.shift2);
#pragma unroll
      for (int c = 0; c < 4; c++) p[c] = pi[c];
    } else {
#pragma unroll
      for (int c = 0; c < 4; c++) p[c] = cacc[c];
    }
    const int rb = rb_of(gi);
    long long p2[4];
#pragma unroll
    for (int c = 0; c < 4; c++) p2[c] = cacc2[c];
    if (WPR == 1) {
      if (ok && !*fail) {
        layer_epilogue<FMT>(a, smem, tokp, rb, m0, mg, lane, rp, lbt_of(gi), p, yacc);
        if (TG2) layer_epilogue<FMT>(a, smem, tokp + 32, rb, m0 + 8, mg - 8, lane, rp, lbt_of(gi), p2, yacc2);
      }
      continue;
    }
    const int buf = gi & 1;
    const size_t slot = ((size_t(grp) * 2 + buf) * WPR + wg) * 32 + lane;
#pragma unroll
    for (int c = 0; c < 4; c++) redl[slot * 4 + c] = p[c];
    if (BVSR) {
#pragma unroll
      for (int c = 0; c < 4; c++) redf[slot * 4 + c] = yacc[c];
    }
    if (TG2) {
#pragma unroll
      for (int c = 0; c < 4; c++) { redl2[slot * 4 + c] = p2[c]; redf2[slot * 4 + c] = yacc2[c]; }
    }
    asm volatile("bar.sync %0, %1;\n" ::"r"(1 + grp), "r"(WPR * 32) : "memory");
    if (wg != gi % WPR || !ok || *fail) continue;
    long long pl[4] = {0, 0, 0, 0}, pl2[4] = {0, 0, 0, 0};
    float yl[4] = {0.f, 0.f, 0.f, 0.f}, yl2[4] = {0.f, 0.f, 0.f, 0.f};
    for (int w = 0; w < WPR; w++) {  // in warp order
      const size_t s2 = ((size_t(grp) * 2 + buf) * WPR + w) * 32 + lane;
      const longlong2 v0 = *reinterpret_cast<const longlong2*>(redl + s2 * 4);
      const longlong2 v1 = *reinterpret_cast<const longlong2*>(redl + s2 * 4 + 2);
      pl[0] += v0.x; pl[1] += v0.y; pl[2] += v1.x; pl[3] += v1.y;
      if (BVSR) {
        const float4 f = *reinterpret_cast<const float4*>(redf + s2 * 4);
        yl[0] += f.x; yl[1] += f.y; yl[2] += f.z; yl[3] += f.w;
      }
      if (TG2) {
#pragma unroll
        for (int c = 0; c < 4; c++) { pl2[c] += redl2[s2 * 4 + c]; yl2[c] += redf2[s2 * 4 + c]; }
      }
    }
    layer_epilogue<FMT>(a, smem, tokp, rb, m0, mg, lane, rp, lbt_of(gi), pl, yl);
    if (TG2) layer_epilogue<FMT>(a, smem, tokp + 32, rb, m0 + 8, mg - 8, lane, rp, lbt_of(gi), pl2, yl2);
  }
  // copies issued but never waited for (an abandoned wait) must land before the block exits
  if (!copies_ok)
    for (int e = waited; e < issued; e++) (void)mbar_wait_bounded(&wbar[e % a.S], uint32_t((e / a.S) & 1));
}

// ---------------------------------------------------------------------------
// Ternary LoRA input (fused path): partial dot products of the unquantized bf16 x
// with A over each 256-k tile, out[kt][m][r], one warp per (kt, m, 8-rank chunk) (the act
// kernel computes the same partials with the same warp routine for the unfused path).
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) k_lora_partial(const uint16_t* __restrict__ x, const uint16_t* __restrict__ A,
                                                      int M, int K, int KT, int rank, float* __restrict__ out) {
  pdl_trigger();
  pdl_wait();
  const int nc = rank / 8;  // 8-rank chunks
  const int wid = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (wid >= KT * M * nc) return;
  const int kt = wid / (M * nc), r2 = wid - kt * M * nc, m = r2 / nc, rc = (r2 - m * nc) * 8;
  lora_tile_partial_warp(x + size_t(m) * K, A, K, rank, kt, rc, threadIdx.x & 31, out + (size_t(kt) * M + m) * rank);
}

// ---------------------------------------------------------------------------
// RaBiT with P paths: fp32 sign-apply, y = sum_p g_p sum_k (-1)^B_p h_p x; the
// sign bit of h_p x is flipped by XOR with the plane bit. One warp per row,
// lane l takes k = 32w + l. Fused: reads x and h; else the act buffer's h_p x.
// The scales combine from the last path down: y = fma(g1, acc1, fma(g2, acc2, g3 acc3)).
// ---------------------------------------------------------------------------
template <int NW, bool FUSED, int P>
__global__ void __launch_bounds__(NW * 32) k_rabit(LayerArgs a) {
  __shared__ int bad;
  pdl_trigger();
  pdl_wait();
  if (!FUSED) {
    if (threadIdx.x == 0) {
      bad = !act_header_ok(a.act_hdr, a);
      if (bad) atomicOr(&g_bq_device_error, kErrActHeader);
    }
    __syncthreads();
    if (bad) return;
  }
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int row = blockIdx.x * NW + warp;
  if (row >= a.N) return;
  const int W32 = a.K_pad / 32;
  const uint32_t* pl = a.rabit_planes + size_t(row) * W32;   // path p: + p N_pad W32
  const size_t pstride = size_t(a.N_pad) * W32;
  // 128-k chunks: lane l owns k = 128c + 4l .. 4l + 3, i.e. bits 4(l & 7) .. + 3 of the chunk's
  // plane word l >> 3. Per chunk and path the warp makes one 16-byte load of the four plane words
  // (the same address for every lane), one float4 of h (or of h x, unfused) and one 8-byte load
  // of four bf16 of x: 128-bit, coalesced loads. K is a multiple of 128, so a chunk lies wholly
  // below K or wholly in the padding (x read as 0 there).
  const int sh = 4 * (lane & 7), wsel = lane >> 3;
  for (int m = 0; m < a.M; m++) {
    float acc[P];
#pragma unroll
    for (int p = 0; p < P; p++) acc[p] = 0.f;
    // four chunks at a time: every load of the four issued before the first use
    for (int c0 = 0; c0 < W32 / 4; c0 += 4) {
      uint4 wv[4][P];
      float4 hv[4][P];
      uint2 xb[4];
#pragma unroll
      for (int cc = 0; cc < 4; cc++) {
        const int c = c0 + cc, k = 128 * c + 4 * lane;
        if (c >= W32 / 4) break;
        xb[cc] = FUSED && 128 * c < a.K ? __ldg(reinterpret_cast<const uint2*>(a.x + size_t(m) * a.K + k)) : make_uint2(0, 0);
#pragma unroll
        for (int p = 0; p < P; p++) {
          wv[cc][p] = __ldg(reinterpret_cast<const uint4*>(pl + p * pstride) + c);
          hv[cc][p] = FUSED ? __ldg(reinterpret_cast<const float4*>(a.rabit_h + size_t(p) * a.K_pad + k))
                            : __ldg(reinterpret_cast<const float4*>(a.act_xt + (size_t(p) * a.M + m) * a.K_pad + k));
        }
      }
#pragma unroll
      for (int cc = 0; cc < 4; cc++) {
        if (c0 + cc >= W32 / 4) break;
        const float xv[4] = {bf16_bits_to_float(uint16_t(xb[cc].x & 0xFFFFu)), bf16_bits_to_float(uint16_t(xb[cc].x >> 16)),
                             bf16_bits_to_float(uint16_t(xb[cc].y & 0xFFFFu)), bf16_bits_to_float(uint16_t(xb[cc].y >> 16))};
#pragma unroll
        for (int p = 0; p < P; p++) {
          const uint4 w4 = wv[cc][p];
          const uint32_t wd = wsel == 0 ? w4.x : wsel == 1 ? w4.y : wsel == 2 ? w4.z : w4.w;
          const float4 h4 = hv[cc][p];
          const float xp[4] = {FUSED ? __fmul_rn(h4.x, xv[0]) : h4.x, FUSED ? __fmul_rn(h4.y, xv[1]) : h4.y,
                               FUSED ? __fmul_rn(h4.z, xv[2]) : h4.z, FUSED ? __fmul_rn(h4.w, xv[3]) : h4.w};
#pragma unroll
          for (int jj = 0; jj < 4; jj++)
            acc[p] += __uint_as_float(__float_as_uint(xp[jj]) ^ (((wd >> (sh + jj)) & 1u) << 31));
        }
      }
    }
#pragma unroll
    for (int p = 0; p < P; p++) acc[p] = warp_sum(acc[p]);
    if (lane == 0) {
      float yv = a.rabit_g[size_t(P - 1) * a.N_pad + row] * acc[P - 1];
#pragma unroll
      for (int p = P - 2; p >= 0; p--) yv = fmaf(a.rabit_g[size_t(p) * a.N_pad + row], acc[p], yv);
      a.y[size_t(m) * a.N + row] = yv;
    }
  }
}

}  // namespace bqi
