// ABQ layer for 16..64 tokens on the fifth-generation tensor cores: tcgen05.mma kind::i8
// (u8 x u8 -> s32) with the accumulators in tensor memory.
//
// ABQ page §3.2 eq.(3): with codes q_w (w bits) and q_x (a bits), P = sum_k q_w q_x is a dense
// integer contraction of M tokens against N rows, the case where the tensor cores do the work
// (the pages' binary tensor-core decomposition is the same sum taken bit-plane by bit-plane).
//
// One CTA computes 128 weight rows (eight 16-row blocks, the MMA's M) for all tokens (the MMA's
// N, M rounded up to a multiple of 16). Per 256-k tile: bulk copies bring the eight packed tiles
// (bit-field streams in the A-fragment order of the int8 m16n8k32 MMA) and the tile's act codes
// of all tokens (the act buffer's tile-major copy, B-fragment order per token) into one of
// three raw stages; the eight warps re-lay both into the canonical K-major layout of the MMA
// operands (8-row x 16-byte core matrices, no swizzle), assembling each weight code byte from
// its streams' fields (code = sum_s field_s << shift_s); one thread issues the tile's eight MMAs
// (K = 32 each) and
// commits them to an mbarrier, which frees the operand buffer for the next tile. After the last
// tile the warps read the accumulators from tensor memory (tcgen05.ld, warps w and w + 4 the
// two column halves of lanes 32w .. 32w + 31) and run the ABQ zero-point epilogue. Every wait
// is bounded: on expiry the device error word is raised, no further MMA is issued, outstanding
// copies and MMAs are waited for, and the tensor memory is freed.
#pragma once

#include "bq_gemv.cuh"

namespace bqi {

constexpr int kTcRows = 128;                 // weight rows per CTA
constexpr int kTcRb = kTcRows / 16;          // row blocks per CTA
constexpr int kTcMaxN = 64;                  // tokens (MMA N) at most
constexpr int kTcThreads = 256;
constexpr int kTcStages = 3;                 // raw stages
constexpr int kTcColsAlloc = 64;             // tensor-memory columns (one per token)
// shared memory carve (bytes)
constexpr uint32_t kTcRawA = kTcRb * 4096;                 // one raw stage of weight tiles (8-bit at most)
constexpr uint32_t kTcRawB = kTcMaxN * 256;                // one raw stage of act codes
constexpr uint32_t kTcCanA = kTcRows * 256;                // canonical A of one k-tile (32 KB)
constexpr uint32_t kTcCanB = kTcMaxN * 256;                // canonical B of one k-tile (16 KB)
constexpr uint32_t kTcOffRawA = 0;
constexpr uint32_t kTcOffRawB = kTcOffRawA + kTcStages * kTcRawA;
constexpr uint32_t kTcOffCanA = kTcOffRawB + kTcStages * kTcRawB;
constexpr uint32_t kTcOffCanB = kTcOffCanA + kTcCanA;
constexpr uint32_t kTcOffBar = kTcOffCanB + kTcCanB;       // full[3], mma, then words
constexpr uint32_t kTcSmem = kTcOffBar + 128;
// canonical strides: A core matrix rows 16 B apart, 8-row groups 128 B apart, 16-byte k-units
// 2048 B apart (16 row groups); B likewise with 8 token groups per k-unit (1024 B)
constexpr uint32_t kTcLboA = 2048, kTcSboA = 128, kTcLboB = 1024, kTcSboB = 128;

struct TcArgs {
  const uint8_t* tiles;      // packed tiles [RB][KT][tile_bytes]
  const float* row_delta;    // Delta_w [N_pad]
  const int* row_zero;       // z_w
  const int* row_sum;        // S_w
  const uint32_t* act_hdr;
  const uint8_t* act_codes;  // tile-major [KT][M][256]
  const uint32_t* act_tok;   // [M][4]: Delta_x, z_x, S_x
  unsigned long long act_total;
  float* y;                  // [M][N]
  long long* acc;            // [M][N] or null
  int N, K, KT, RB, M, Nmma, a_bits, tile_bytes;
};

__device__ __forceinline__ bool tc_header_ok(const uint32_t* h, const TcArgs& a) {
  return h[AW_MAGIC] == kActMagic && h[AW_VERSION] == kVersion && h[AW_FMT] == uint32_t(BQ_FMT_ABQ) &&
         h[AW_M] == uint32_t(a.M) && h[AW_K] == uint32_t(a.K) && h[AW_ABITS] == uint32_t(a.a_bits) &&
         h[AW_LORA_RANK] == 0u && h[AW_TOTAL] == uint32_t(a.act_total) &&
         h[AW_TOTAL + 1] == uint32_t(a.act_total >> 32);
}

// Shared-memory matrix descriptor of a K-major operand without swizzle: start address, the byte
// distance between the two 16-byte k-units of one MMA (leading) and between 8-row groups
// (stride), all in 16-byte units; version 1 (bits 46-47); layout type 0 (no swizzle).
__device__ __forceinline__ uint64_t tc_smem_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  return uint64_t((saddr >> 4) & 0x3FFFu) | (uint64_t((lbo >> 4) & 0x3FFFu) << 16) |
         (uint64_t((sbo >> 4) & 0x3FFFu) << 32) | (uint64_t(1) << 46);
}

// Instruction descriptor of kind::i8: s32 accumulators (bits 4-5 = 2), u8 A and B (bits 7-9 and
// 10-12 = 0), both K-major, N >> 3 in bits 17-22, M >> 4 in bits 24-28.
__host__ __device__ constexpr uint32_t tc_instr_desc(int nmma, int mmma) {
  return (2u << 4) | (uint32_t(nmma >> 3) << 17) | (uint32_t(mmma >> 4) << 24);
}

__device__ __forceinline__ void tc_mma(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t idesc, int accum) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;\n}\n" ::"r"(tmem_d),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accum)
      : "memory");
}
__device__ __forceinline__ void tc_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n" ::"r"(smem_u32(bar))
               : "memory");
}
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;\n" ::: "memory"); }
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;\n" ::: "memory"); }

// 32 lanes x 32 columns of 32 bits from tensor memory (warp w reads lanes 32 (w % 4) .. + 31)
__device__ __forceinline__ void tc_ld32(uint32_t taddr, uint32_t (&v)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];\n"
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
        "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15]),
        "=r"(v[16]), "=r"(v[17]), "=r"(v[18]), "=r"(v[19]), "=r"(v[20]), "=r"(v[21]), "=r"(v[22]), "=r"(v[23]),
        "=r"(v[24]), "=r"(v[25]), "=r"(v[26]), "=r"(v[27]), "=r"(v[28]), "=r"(v[29]), "=r"(v[30]), "=r"(v[31])
      : "r"(taddr)
      : "memory");
  asm volatile("tcgen05.wait::ld.sync.aligned;\n" ::: "memory");
}

// Field f (bits) of 32-k chunk kc for the four words of this lane's 16 bytes of a stream of width F:
// the chunk is field kc % (8/F) of uint4 kc / (8/F); the field values land at bit offset SH.
template <int F, int SH>
__device__ __forceinline__ void tc_stream_fields(const uint8_t* base, int kc, int lane, uint32_t (&w4)[4]) {
  constexpr int per = 8 / F;
  constexpr uint32_t mask = ((1u << F) - 1u) * 0x01010101u;
  const uint4 v = *reinterpret_cast<const uint4*>(base + ((kc / per) * 32 + lane) * 16);
  const uint32_t sh = uint32_t(F * (kc % per));
  w4[0] |= ((v.x >> sh) & mask) << SH;
  w4[1] |= ((v.y >> sh) & mask) << SH;
  w4[2] |= ((v.z >> sh) & mask) << SH;
  w4[3] |= ((v.w >> sh) & mask) << SH;
}

// F0, F1, F2: the field widths of the layer's bit-field streams (0 = no such stream), from the
// low end of the code: W8 [8], W4 [4], W6 [4, 2], W7 [4, 2, 1], ...
template <int F0, int F1, int F2>
__global__ void __launch_bounds__(kTcThreads, 1) k_abq_tc(const __grid_constant__ TcArgs a) {
  extern __shared__ __align__(128) uint8_t tc_smem[];  // operands need 16-byte alignment (no swizzle)
  uint8_t* smem = tc_smem;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int rb0 = blockIdx.x * kTcRb;
  const int nrb = min(kTcRb, a.RB - rb0);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kTcOffBar);  // raw stage s filled
  uint64_t* mmab = full + kTcStages;                                // the operand buffer's MMAs done
  uint32_t* words = reinterpret_cast<uint32_t*>(mmab + 1);          // [0] tmem address, [1] failure, [2] bad header
  const uint32_t tb = uint32_t(a.tile_bytes);
  const uint32_t wbytes = uint32_t(nrb) * tb, cbytes = uint32_t(a.M) * 256u;

  pdl_trigger();
  if (tid == 0) {
    for (int st = 0; st < kTcStages; st++) mbar_init(&full[st], 1);
    mbar_init(mmab, 1);
    fence_mbar_init();
    words[1] = 0;
    words[2] = 0;
  }
  if (warp == 0) {  // tensor-memory accumulators: 128 lanes x 64 columns
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;\n" ::"r"(smem_u32(words)),
                 "r"(kTcColsAlloc)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;\n" ::: "memory");
  }
  // the padding tokens' operand rows stay zero
  for (uint32_t i = tid; i < kTcCanB / 16; i += kTcThreads)
    reinterpret_cast<uint4*>(smem + kTcOffCanB)[i] = make_uint4(0, 0, 0, 0);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = words[0];

  auto issue_w = [&](int kt, int s) {  // weights are constant: fetched before the dependency wait too
    for (int r = 0; r < nrb; r++)
      bulk_g2s(smem + kTcOffRawA + s * kTcRawA + r * tb, a.tiles + (size_t(rb0 + r) * a.KT + kt) * tb, tb, &full[s]);
  };
  auto issue_c = [&](int kt, int s) {  // one contiguous copy: tile kt of every token
    bulk_g2s(smem + kTcOffRawB + s * kTcRawB, a.act_codes + size_t(kt) * a.M * 256, cbytes, &full[s]);
  };
  const int first = min(kTcStages, a.KT);
  int issued = 0;  // k-tiles whose copies were issued (tile kt uses stage kt % 3)
  if (tid == 0) {
    for (int kt = 0; kt < first; kt++) {
      mbar_expect_tx(&full[kt], wbytes + cbytes);
      issue_w(kt, kt);
    }
  }
  pdl_wait();  // the act buffer may be the previous kernel's output
  if (tid == 0) {
    if (!tc_header_ok(a.act_hdr, a)) {
      words[2] = 1;
      atomicOr(&g_bq_device_error, kErrActHeader);
    }
    // the code copies complete the first stages' transactions even when the header is bad, so
    // that no copy is left in flight; a bad header only stops the MMAs and the outputs
    for (int kt = 0; kt < first; kt++) issue_c(kt, kt);
    issued = first;
  }
  __syncthreads();
  const bool bad = words[2] != 0;
  const uint32_t idesc = tc_instr_desc(a.Nmma, kTcRows);
  const uint32_t ca = smem_u32(smem + kTcOffCanA), cb = smem_u32(smem + kTcOffCanB);
  int committed = 0;  // tiles whose MMAs were committed (commit kt completes phase kt of mmab)

  for (int kt = 0; kt < a.KT; kt++) {
    const int s = kt % kTcStages;
    bool ok = mbar_wait_bounded(&full[s], uint32_t((kt / kTcStages) & 1));
    if (kt >= 1 && ok) ok = mbar_wait_bounded(mmab, uint32_t((kt - 1) & 1));  // operand buffer free
    if (!ok) words[1] = 1;
    __syncthreads();
    if (words[1]) break;
    {  // re-layout: raw stage s -> the operand buffer
      const uint8_t* ra = smem + kTcOffRawA + s * kTcRawA;
      uint8_t* can_a = smem + kTcOffCanA;
      const int g = lane >> 2, t = lane & 3;
      const int kc = warp;  // this warp's 32-k chunk of the tile
      for (int rbl = 0; rbl < nrb; rbl++) {
        // word w of a lane holds row g + 8(w & 1) of the block at k = 32kc + 16(w >> 1) + 4t + b;
        // stream s keeps that chunk as field kc % (8/f) of its uint4 kc / (8/f)
        uint32_t w4[4] = {0u, 0u, 0u, 0u};
        const uint8_t* tile = ra + rbl * tb;
        tc_stream_fields<F0, 0>(tile, kc, lane, w4);
        if constexpr (F1 > 0) tc_stream_fields<F1, F0>(tile + 512 * F0, kc, lane, w4);
        if constexpr (F2 > 0) tc_stream_fields<F2, F0 + F1>(tile + 512 * (F0 + F1), kc, lane, w4);
#pragma unroll
        for (int w = 0; w < 4; w++) {
          const uint32_t off = uint32_t(2 * kc + (w >> 1)) * kTcLboA + uint32_t(2 * rbl + (w & 1)) * kTcSboA +
                               uint32_t(g) * 16 + uint32_t(t) * 4;
          *reinterpret_cast<uint32_t*>(can_a + off) = w4[w];
        }
      }
      const uint8_t* rbraw = smem + kTcOffRawB + s * kTcRawB;
      uint8_t* can_b = smem + kTcOffCanB;
      for (int idx = tid; idx < a.M * 16; idx += kTcThreads) {  // (token, 16-byte chunk c)
        const int n = idx >> 4, c = idx & 15;
        const uint4 v = *reinterpret_cast<const uint4*>(rbraw + n * 256 + c * 16);
        const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
        const int tt = c >> 2, cc = c & 3;
#pragma unroll
        for (int q = 0; q < 4; q++) {  // byte 64t + 8mu + 4h + b: mu = 2cc + q / 2, h = q % 2
          const int j = 2 * (2 * cc + (q >> 1)) + (q & 1);
          const uint32_t off = uint32_t(j) * kTcLboB + uint32_t(n >> 3) * kTcSboB + uint32_t(n & 7) * 16 + uint32_t(tt) * 4;
          *reinterpret_cast<uint32_t*>(can_b + off) = w4[q];
        }
      }
    }
    fence_proxy_async();  // the operand writes become visible to the tensor cores
    tc_fence_before();
    __syncthreads();
    if (tid == 0) {
      tc_fence_after();
      if (!bad) {
#pragma unroll
        for (int i = 0; i < 8; i++)
          tc_mma(tmem, tc_smem_desc(ca + i * 2 * kTcLboA, kTcLboA, kTcSboA),
                 tc_smem_desc(cb + i * 2 * kTcLboB, kTcLboB, kTcSboB), idesc, kt > 0 || i > 0);
      }
      tc_commit(mmab);
      committed = kt + 1;
      if (kt + kTcStages < a.KT) {  // raw stage s is free again (every thread passed the barrier)
        fence_proxy_async();
        mbar_expect_tx(&full[s], wbytes + cbytes);
        issue_w(kt + kTcStages, s);
        issue_c(kt + kTcStages, s);
        issued = kt + kTcStages + 1;
      }
    }
  }
  // drain: every issued copy landed and the last committed MMA group completed
  if (tid == 0) {
    if (committed > 0 && !mbar_wait_bounded(mmab, uint32_t((committed - 1) & 1))) words[1] = 1;
    for (int kt = committed; kt < issued; kt++)
      (void)mbar_wait_bounded(&full[kt % kTcStages], uint32_t((kt / kTcStages) & 1));
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (!bad && !words[1]) {
    // epilogue: warp w holds rows 32 (w % 4) + lane of the CTA's 128 and tokens 32 (w / 4) ..
    uint32_t v[32];
    const int lq = warp & 3, half = warp >> 2;
    tc_ld32(tmem + (uint32_t(32 * lq) << 16) + uint32_t(32 * half), v);
    const int row = rb0 * 16 + 32 * lq + lane;
    if (row < a.N) {
      const float dw = __ldg(a.row_delta + row);
      const long long zw = __ldg(a.row_zero + row), sw = __ldg(a.row_sum + row);
#pragma unroll
      for (int i = 0; i < 32; i++) {
        const int m = 32 * half + i;
        if (m >= a.M) break;
        const float dx = __uint_as_float(__ldg(a.act_tok + 4 * m));
        const long long zx = int(__ldg(a.act_tok + 4 * m + 1)), sx = int(__ldg(a.act_tok + 4 * m + 2));
        // I = P - z_x S_w - z_w S_x + K z_w z_x
        const long long I = (long long)int(v[i]) - zx * sw - zw * sx + (long long)a.K * zw * zx;
        a.y[size_t(m) * a.N + row] = __fmul_rn(dw, dx) * float(I);
        if (a.acc) a.acc[size_t(m) * a.N + row] = I;
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;\n" ::"r"(tmem), "r"(kTcColsAlloc) : "memory");
  }
}

}  // namespace bqi
