// Internal definitions shared by the pack, activation and GEMV kernels:
// header word indices, the byte layouts of the packed-weight and activation
// buffers (documented in include/bq.h), and small device helpers.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cmath>

#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "bq.h"

namespace bqi {

constexpr uint32_t kPkMagic = 0x4B505142u;   // 'BQPK'
constexpr uint32_t kActMagic = 0x43415142u;  // 'BQAC'
constexpr uint32_t kVersion = 1;

// packed-buffer header words
enum : int {
  HW_MAGIC = 0, HW_VERSION = 1, HW_FMT = 2, HW_N = 3, HW_K = 4, HW_NPAD = 5, HW_KPAD = 6,
  HW_WBITS = 7, HW_ABITS = 8, HW_NSTREAMS = 9, HW_FIELD = 10, HW_SHIFT = 14, HW_TILEBYTES = 18,
  HW_LORA_RANK = 19, HW_LORA_ALPHA = 20, HW_TSCALE = 21, HW_TOTAL = 22, HW_OFF_TILES = 24,
  HW_OFF_ROWS = 26, HW_OFF_AUX = 28, HW_OFF_AUX2 = 30, HW_COUNT = 32
};
// activation-buffer header words
enum : int {
  AW_MAGIC = 0, AW_VERSION = 1, AW_FMT = 2, AW_M = 3, AW_K = 4, AW_KPAD = 5, AW_ABITS = 6,
  AW_LORA_RANK = 7, AW_TOTAL = 8, AW_OFF_CODES = 10, AW_OFF_TOK = 12, AW_OFF_GSUM = 14,
  AW_OFF_U = 16, AW_OFF_XT = 18, AW_OFF_CT = 20, AW_COUNT = 22
};

constexpr int kBvsrSets = 256;
constexpr int kBvsrTableStride = 8;  // words per set: c0 c1 c2 c3 o sc ratio_index, R bytes (u32)
constexpr int kBvsrTileBytes = 4 * 512 + 16 * 8;
// after the table: clustering centroids f64 [256][2] and their int64 sums [256][3]
constexpr int kBvsrPackScratch = kBvsrSets * 2 * 8 + kBvsrSets * 3 * 8;

struct PkLayout {
  int fmt, N, K, N_pad, K_pad, RB, KT, w_bits, a_bits, nstreams;
  int field[4], shift[4];
  int tile_bytes, rank;
  float lora_alpha;
  uint64_t off_tiles, off_rows, off_aux, off_aux2, total;
};

struct ActLayout {
  int fmt, M, K, K_pad, KT, a_bits, rank;
  uint64_t off_codes, off_tok, off_gsum, off_u, off_xt, off_ct, total;
};

// ABQ with 16..64 tokens runs on the tensor cores, whose act buffer also holds the codes in
// the MMA's operand layout: per k-tile one contiguous block of Mp = M rounded up to 16 tokens
// (the padding tokens' codes zero).
constexpr int kTcMinM = 16, kTcMaxM = 64;
inline bool tc_layer(int fmt, int w_bits, int M) {
  return fmt == BQ_FMT_ABQ && w_bits >= 1 && w_bits <= 8 && M >= kTcMinM && M <= kTcMaxM;
}
__host__ __device__ inline int tc_tokens(int M) { return (M + 15) / 16 * 16; }

inline uint64_t align256(uint64_t x) { return (x + 255) & ~uint64_t(255); }

// Paths of a RaBiT format (0 for the tiled formats).
__host__ __device__ inline int rabit_paths(int fmt) {
  return fmt == BQ_FMT_RABIT2 ? 2 : fmt == BQ_FMT_RABIT3 ? 3 : 0;
}

// Returns false for an unknown format or bit width.
inline bool make_pk_layout(int fmt, int N, int K, int w_bits, int a_bits, int rank, float alpha,
                           PkLayout* L) {
  PkLayout l{};
  l.fmt = fmt; l.N = N; l.K = K;
  l.N_pad = (N + 15) / 16 * 16;
  l.K_pad = (K + 255) / 256 * 256;
  l.RB = l.N_pad / 16; l.KT = l.K_pad / 256;
  uint64_t tiles = 0, rows = 0, aux = 0, aux2 = 0;
  switch (fmt) {
    case BQ_FMT_RABIT2:
      l.w_bits = 2; l.a_bits = 16; l.nstreams = 2;
      l.field[0] = l.field[1] = 1; l.shift[0] = 0; l.shift[1] = 1;
      l.tile_bytes = 0;
      tiles = 2ull * l.N_pad * (l.K_pad / 8);
      rows = 2ull * l.N_pad * 4; aux = uint64_t(l.K_pad) * 4; aux2 = uint64_t(l.K_pad) * 4;
      break;
    case BQ_FMT_RABIT3:  // h2, h3 follow h1 (4 K_pad is a multiple of 256: no gaps)
      l.w_bits = 3; l.a_bits = 16; l.nstreams = 3;
      for (int s = 0; s < 3; s++) { l.field[s] = 1; l.shift[s] = s; }
      l.tile_bytes = 0;
      tiles = 3ull * l.N_pad * (l.K_pad / 8);
      rows = 3ull * l.N_pad * 4; aux = uint64_t(l.K_pad) * 4; aux2 = 2ull * l.K_pad * 4;
      break;
    case BQ_FMT_BITNET_W1A8:
      l.w_bits = 1; l.a_bits = 8; l.nstreams = 1; l.field[0] = 1; l.tile_bytes = 512;
      break;
    case BQ_FMT_TERNARY_A8:
      l.w_bits = 2; l.a_bits = 8; l.nstreams = 1; l.field[0] = 2; l.tile_bytes = 1024;
      l.rank = rank; l.lora_alpha = alpha;
      aux = uint64_t(l.K_pad) * rank * 2; aux2 = uint64_t(l.N_pad) * rank * 2;
      break;
    case BQ_FMT_ABQ: {
      if (w_bits < 1 || w_bits > 8 || a_bits < 1 || a_bits > 8) return false;
      l.w_bits = w_bits; l.a_bits = a_bits;
      int rem = w_bits, sh = 0;
      while (rem > 0) {  // fields of 8/4/2/1 bits from the low end of the code
        int f = rem >= 8 ? 8 : rem >= 4 ? 4 : rem >= 2 ? 2 : 1;
        l.field[l.nstreams] = f; l.shift[l.nstreams] = sh; l.nstreams++;
        rem -= f; sh += f;
      }
      l.tile_bytes = 512 * w_bits;
      rows = 3ull * l.N_pad * 4;
      break;
    }
    case BQ_FMT_BVSR4:
      // one stream of 4-bit codes in the nibble order of the BVSR tile (not the generic
      // field order), then the 16 x 8 set indices
      l.w_bits = 4; l.a_bits = 8; l.nstreams = 1; l.field[0] = 4; l.shift[0] = 0;
      l.tile_bytes = kBvsrTileBytes;
      aux = uint64_t(kBvsrSets) * kBvsrTableStride * 4 + kBvsrPackScratch;
      break;
    default:
      return false;
  }
  if (!rabit_paths(fmt)) tiles = uint64_t(l.RB) * l.KT * l.tile_bytes;
  l.off_tiles = 256;
  l.off_rows = align256(l.off_tiles + tiles);
  l.off_aux = align256(l.off_rows + rows);
  l.off_aux2 = align256(l.off_aux + aux);
  l.total = align256(l.off_aux2 + aux2);
  *L = l;
  return true;
}

inline ActLayout make_act_layout(const PkLayout& L, int M) {
  ActLayout a{};
  a.fmt = L.fmt; a.M = M; a.K = L.K; a.K_pad = L.K_pad; a.KT = L.KT; a.a_bits = L.a_bits;
  a.rank = L.fmt == BQ_FMT_TERNARY_A8 ? L.rank : 0;
  uint64_t codes = rabit_paths(L.fmt) ? 0 : uint64_t(M) * L.KT * 256;
  uint64_t tok = uint64_t(M) * 16;
  uint64_t gsum = L.fmt == BQ_FMT_BVSR4 ? uint64_t(M) * (L.K_pad / 32) * 4 : 0;
  uint64_t u = uint64_t(L.KT) * M * a.rank * 4;   // LoRA partials [KT][M][r]
  uint64_t xt = uint64_t(rabit_paths(L.fmt)) * M * L.K_pad * 4;
  // the same codes, [KT][16 k-units][Mp / 8][8 tokens][16 bytes]
  uint64_t ct = tc_layer(L.fmt, L.w_bits, M) ? uint64_t(tc_tokens(M)) * L.KT * 256 : 0;
  a.off_codes = 256;
  a.off_tok = align256(a.off_codes + codes);
  a.off_gsum = align256(a.off_tok + tok);
  a.off_u = align256(a.off_gsum + gsum);
  a.off_xt = align256(a.off_u + u);
  a.off_ct = ct ? align256(a.off_xt + xt) : 0;
  a.total = ct ? align256(a.off_ct + ct) : align256(a.off_xt + xt);
  return a;
}

inline bool layout_from_layer(const bq_layer* y, PkLayout* L) {
  return make_pk_layout(y->fmt, y->N, y->K, y->w_bits, y->a_bits, y->lora_rank, 0.f, L);
}

// ---------------------------------------------------------------------------
// device helpers
// ---------------------------------------------------------------------------

// Programmatic dependent launch: let the next kernel in the stream launch, and
// wait until the previous one has completed and its writes are visible.
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory"); }
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;\n" ::: "memory"); }

// Position (in 32-bit words) of the 4 activation codes k_in .. k_in+3 inside a
// token's 256-k tile in B-fragment order: k_in = 32mu + 16h + 4t + b -> word 16t + 2mu + h.
__device__ __forceinline__ int code_word_in_tile(int kin) {
  const int mu = kin >> 5, h = (kin >> 4) & 1, t = (kin >> 2) & 3;
  return 16 * t + 2 * mu + h;
}

// Ternary LoRA input, one 256-k tile and 8 ranks [rc, rc + 8), by one warp: out[i] = sum
// over the tile's k of x_k A[k][rc + i] (K % 128 == 0, so a lane's 8 k's are all inside K
// or all past it). Lane l takes k = 256 kt + 8l .. 8l + 7 and sums its 8 products in k
// order; the 32 lane sums meet in a fixed xor-butterfly, so every caller gets the same bits.
__device__ __forceinline__ void lora_tile_partial_warp(const uint16_t* xr, const uint16_t* A, int K, int rank,
                                                       int kt, int rc, int lane, float* out) {
  const int k0 = kt * 256 + lane * 8;
  const bool in = k0 < K;
  const uint4 xq = in ? *reinterpret_cast<const uint4*>(xr + k0) : make_uint4(0, 0, 0, 0);
  uint4 aq[8];
#pragma unroll
  for (int e = 0; e < 8; e++)
    aq[e] = in ? *reinterpret_cast<const uint4*>(A + size_t(k0 + e) * rank + rc) : make_uint4(0, 0, 0, 0);
  const uint32_t xw[4] = {xq.x, xq.y, xq.z, xq.w};
  float acc[8];
#pragma unroll
  for (int i = 0; i < 8; i++) acc[i] = 0.f;
#pragma unroll
  for (int e = 0; e < 8; e++) {
    const float xv = __uint_as_float((e & 1) ? (xw[e >> 1] & 0xFFFF0000u) : (xw[e >> 1] << 16));
    const uint32_t w[4] = {aq[e].x, aq[e].y, aq[e].z, aq[e].w};
#pragma unroll
    for (int i = 0; i < 8; i++)
      acc[i] = fmaf(xv, __uint_as_float((i & 1) ? (w[i >> 1] & 0xFFFF0000u) : (w[i >> 1] << 16)), acc[i]);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1)
#pragma unroll
    for (int i = 0; i < 8; i++) acc[i] += __shfl_xor_sync(0xffffffffu, acc[i], o);
  if (lane < 8) {
    float v = acc[0];
#pragma unroll
    for (int i = 1; i < 8; i++) v = lane == i ? acc[i] : v;
    out[rc + lane] = v;
  }
}

// Order-preserving map of a float to uint32 (total order on non-NaN values).
__device__ __forceinline__ uint32_t float_key(float f) {
  uint32_t b = __float_as_uint(f);
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}
__device__ __forceinline__ float key_float(uint32_t k) {
  uint32_t b = (k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k;
  return __uint_as_float(b);
}

__device__ __forceinline__ float bf16_bits_to_float(uint16_t h) {
  return __uint_as_float(uint32_t(h) << 16);
}

// Round a float to bf16 (nearest, ties to even) and return the 16-bit storage.
__device__ __forceinline__ uint16_t float_to_bf16_bits(float f) {
  uint32_t u = __float_as_uint(f);
  u += 0x7FFFu + ((u >> 16) & 1u);
  return uint16_t(u >> 16);
}

template <typename T>
__device__ __forceinline__ T warp_sum(T v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ float warp_min(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fminf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// Block-wide reductions for blockDim.x a multiple of 32 (<= 1024). `sh` needs 32 slots.
template <typename T>
__device__ T block_sum(T v, T* sh) {
  int lane = threadIdx.x & 31, w = threadIdx.x >> 5, nw = blockDim.x >> 5;
  v = warp_sum(v);
  __syncthreads();
  if (lane == 0) sh[w] = v;
  __syncthreads();
  T r = T(0);
  if (w == 0) {
    r = lane < nw ? sh[lane] : T(0);
    r = warp_sum(r);
    if (lane == 0) sh[0] = r;
  }
  __syncthreads();
  return sh[0];
}
__device__ inline float block_max(float v, float* sh) {
  int lane = threadIdx.x & 31, w = threadIdx.x >> 5, nw = blockDim.x >> 5;
  v = warp_max(v);
  __syncthreads();
  if (lane == 0) sh[w] = v;
  __syncthreads();
  if (w == 0) {
    float r = lane < nw ? sh[lane] : -INFINITY;
    r = warp_max(r);
    if (lane == 0) sh[0] = r;
  }
  __syncthreads();
  return sh[0];
}
__device__ inline float block_min(float v, float* sh) {
  int lane = threadIdx.x & 31, w = threadIdx.x >> 5, nw = blockDim.x >> 5;
  v = warp_min(v);
  __syncthreads();
  if (lane == 0) sh[w] = v;
  __syncthreads();
  if (w == 0) {
    float r = lane < nw ? sh[lane] : INFINITY;
    r = warp_min(r);
    if (lane == 0) sh[0] = r;
  }
  __syncthreads();
  return sh[0];
}

}  // namespace bqi
