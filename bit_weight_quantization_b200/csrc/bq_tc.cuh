// ABQ layer for 16..64 tokens on the fifth-generation tensor cores: tcgen05.mma kind::i8
// (u8 x u8 -> s32) with the accumulators in tensor memory.
//
// ABQ page §3.2 eq.(3): with codes q_w (w bits) and q_x (a bits), P = sum_k q_w q_x is a dense
// integer contraction of M tokens against N rows, the case where the tensor cores do the work
// (the pages' binary tensor-core decomposition is the same sum taken bit-plane by bit-plane).
//
// One CTA computes 128 weight rows (eight 16-row blocks, the MMA's M) for all tokens (the MMA's
// N = Mp, M rounded up to a multiple of 16) over a range of the 256-k tiles; a cluster of CS
// CTAs splits the tiles of one 128-row group, and each CTA then sums one slice of the tokens
// over the cluster's partial products through distributed shared memory (integer adds: exact
// in any order) and writes that slice's outputs.
//
// Warp roles, coupled only by mbarriers. The producer warp fills a ring of stages sized to the
// shared memory: per tile one TMA tensor copy of the eight packed weight tiles (bit-field
// streams in the A-fragment order of the int8 m16n8k32 MMA; rows past the layer read as zero)
// and one bulk copy of the act buffer's tensor-core block of the tile (already in the
// canonical K-major operand layout, read by the MMA in place). Eight re-layout warps, one per
// 16-row block, assemble each code byte from its streams' fields (code = sum_s field_s <<
// shift_s) and store the fragment words straight into one of two weight operand buffers in
// tensor memory (tcgen05.st 16x256b writes the m16n8 fragment pattern, so the words need no
// shuffling; the k order this gives within each 32-k chunk is the act copy's order too), then
// arrive on the buffer's "ready" barrier. The MMA warp issues the tile's eight MMAs (K = 32
// each, A from tensor memory, B from shared memory) and commits them to the stage's "empty"
// barrier, on which the producer refills the stage and the re-layout warps reuse the tile's
// operand buffer two tiles later. After the last tile the re-layout warps read the
// accumulators from tensor memory (tcgen05.ld, warps w and w + 4 the two column halves of lanes
// 32w .. 32w + 31) and run the ABQ zero-point epilogue. Every wait is bounded and also ends
// when another role has stopped: on expiry the device error word is raised, no further MMA is
// issued, outstanding copies and MMAs are waited for, every CTA of the cluster still takes both
// cluster barriers, and the tensor memory is freed. An act buffer whose header does not match
// the layer is not read past its header (no code copy, no token words, no MMA, no output).
#pragma once

#include "bq_gemv.cuh"

namespace bqi {

constexpr int kTcRows = 128;                 // weight rows per CTA
constexpr int kTcRb = kTcRows / 16;          // row blocks per CTA
constexpr int kTcMaxN = 64;                  // tokens (MMA N) at most
constexpr int kTcLayoutWarps = 8;           // re-layout / epilogue warps
constexpr int kTcProducerWarp = kTcLayoutWarps, kTcMmaWarp = kTcLayoutWarps + 1;
constexpr int kTcThreads = (kTcLayoutWarps + 2) * 32;
constexpr int kTcMaxStages = 8;
constexpr int kTcMaxCluster = 8;             // portable cluster size
// tensor memory: the accumulators (one column per token) in columns 0..63, and two A operand
// buffers of one k-tile each (128 rows x 256 codes, four codes a column) at columns 64 and 128
constexpr int kTcColsAlloc = 256;
constexpr uint32_t kTcColA = 64, kTcColsA = 64;
constexpr uint32_t kTcOffStages = 0;
// after the stages: full[8] (0), empty[8] (64), ready[2] (144), words[8] (160),
// and the token parameters Delta_x, z_x, S_x - K z_x [3][64] (256)
constexpr uint32_t kTcBarBytes = 1024;
constexpr uint32_t kTcSmemMax = 227 * 1024;
// canonical strides of B (K-major, no swizzle): 8-token groups 128 B apart, 16-byte k-units
// Mp * 16 B apart
constexpr uint32_t kTcSboB = 128;

// The packed weight tiles as a 3-D uint8 tensor for the TMA: x = 256 bytes, y = 256-byte
// chunks along a row block's tiles (KT tile_bytes / 256), z = row blocks; a box of
// (256, tile_bytes / 256, 8) is one k-tile of eight row blocks, laid out in shared memory as
// the eight tiles back to back. The map is opaque (CUtensorMap, 128 bytes, 64-byte aligned).
struct alignas(64) TcTensorMap {
  unsigned long long opaque[16];
};

struct TcArgs {
  TcTensorMap wmap;          // the packed weight tiles (see TcTensorMap)
  const float* row_delta;    // Delta_w [N_pad]
  const int* row_zero;       // z_w
  const int* row_sum;        // S_w
  const uint32_t* act_hdr;
  const uint8_t* act_codes;  // tensor-core copy [KT][16 k-units][Mp/8][8 tokens][16 B]
  const uint32_t* act_tok;   // [M][4]: Delta_x, z_x, S_x
  unsigned long long act_total;
  float* y;                  // [M][N]
  long long* acc;            // [M][N] or null
  int N, K, KT, RB, M, Mp, a_bits, tile_bytes;
  int stages, stage_bytes, CS;  // ring stages, bytes per stage (weights then codes), cluster size
};

// Ring stages that fit next to the two operand buffers, for weight tiles of tile_bytes and Mp tokens.
__host__ __device__ inline int tc_stages(int tile_bytes, int Mp) {
  const int stage = kTcRb * tile_bytes + Mp * 256;
  const int s = int((kTcSmemMax - kTcOffStages - kTcBarBytes) / uint32_t(stage));
  return s < kTcMaxStages ? s : kTcMaxStages;
}

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

__device__ __forceinline__ void tc_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n" ::"r"(smem_u32(bar))
               : "memory");
}
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;\n" ::: "memory"); }
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;\n" ::: "memory"); }

// 16 lanes x 8 columns into tensor memory in the m16n8 fragment pattern: thread 4g + t writes
// r0, r1 to lane g, columns 2t and 2t + 1, and r2, r3 to lane g + 8, the same columns
__device__ __forceinline__ void tc_st16(uint32_t taddr, uint32_t r0, uint32_t r1, uint32_t r2, uint32_t r3) {
  asm volatile("tcgen05.st.sync.aligned.16x256b.x1.b32 [%0], {%1, %2, %3, %4};\n" ::"r"(taddr), "r"(r0), "r"(r1),
               "r"(r2), "r"(r3)
               : "memory");
}
__device__ __forceinline__ void tc_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;\n" ::: "memory"); }
// the MMA with A from tensor memory (a_tmem) and B from shared memory
__device__ __forceinline__ void tc_mma_ta(uint32_t tmem_d, uint32_t tmem_a, uint64_t bdesc, uint32_t idesc, int accum) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::i8 [%0], [%1], %2, %3, p;\n}\n" ::"r"(tmem_d),
      "r"(tmem_a), "l"(bdesc), "r"(idesc), "r"(accum)
      : "memory");
}

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

// one box of a 3-D tensor map into shared memory, completing bytes on bar (no multicast)
__device__ __forceinline__ void tma_load_3d(void* dst, const TcTensorMap* map, int x, int y, int z, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], [%5];\n"
      ::"r"(smem_u32(dst)), "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(smem_u32(bar))
      : "memory");
}

// distributed shared memory of a cluster
__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;\n" : "=r"(r));
  return r;
}
__device__ __forceinline__ uint32_t dsmem_map(uint32_t saddr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;\n" : "=r"(r) : "r"(saddr), "r"(rank));
  return r;
}
__device__ __forceinline__ uint32_t dsmem_ld(uint32_t raddr) {
  uint32_t v;
  asm volatile("ld.shared::cluster.u32 %0, [%1];\n" : "=r"(v) : "r"(raddr) : "memory");
  return v;
}
// every thread of every CTA of the cluster arrives (release) and waits (acquire); the CTAs of a
// cluster are co-scheduled, and each one passes exactly two of these on every path
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\nbarrier.cluster.wait.acquire.aligned;\n" ::: "memory");
}

// lowers the barrier's pending transaction count by bytes that will never be copied
__device__ __forceinline__ void mbar_complete_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.complete_tx.shared::cta.b64 [%0], %1;\n" ::"r"(smem_u32(bar)), "r"(bytes) : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];\n" ::"r"(smem_u32(bar)) : "memory");
}

// bounded wait that also gives up once another role of the block has stopped (*stop != 0)
__device__ __forceinline__ bool tc_wait(uint64_t* bar, uint32_t parity, const uint32_t* stop) {
  for (uint32_t i = 0; i < kMaxSpin; i++) {
    if (mbar_try_wait(bar, parity)) return true;
    if (*reinterpret_cast<const volatile uint32_t*>(stop)) return false;
  }
  atomicOr(&g_bq_device_error, kErrCopyTimeout);
  return false;
}

// The token parameters and this thread's row parameters of the epilogue.
struct TcTok {
  const float* dx;  // Delta_x per token (shared)
  const int* zx;    // z_x
  const int* t;     // S_x - K z_x (mod 2^32)
  float dw;
  uint32_t zw, sw;
};

// y (and the integer accumulators when asked) of tokens m0, m0 + step, ... (< M) of one row,
// from registers.
template <int T>
__device__ __forceinline__ void tc_store_outputs(const TcArgs& a, int row, int m0, int step, const float (&yv)[T],
                                                 const uint32_t (&iv)[T]) {
#pragma unroll
  for (int j = 0; j < T; j++) {
    const int m = m0 + step * j;
    if (m < a.M) {
      a.y[size_t(m) * a.N + row] = yv[j];
      if (a.acc) a.acc[size_t(m) * a.N + row] = (long long)int(iv[j]);
    }
  }
}

// Tokens m = r0, r0 + 2 CSV, ... (< M) of row rl: the cluster's CSV partial products summed in
// CTA order, every remote load issued before the first sum (so their latencies overlap), then
// y = Delta_w Delta_x I with I = P - z_x S_w - z_w (S_x - K z_x) in wrapping int32, then stored.
template <int CSV>
__device__ __forceinline__ void tc_cluster_out(const TcArgs& a, const uint32_t* part, int rl, int row, int r0,
                                               const TcTok& tk) {
  constexpr int T = (kTcMaxN + 2 * CSV - 1) / (2 * CSV);  // tokens one thread can hold
  uint32_t L[T][CSV];
#pragma unroll
  for (int j = 0; j < T; j++) {
    const int m = r0 + 2 * CSV * j;
    const uint32_t addr = smem_u32(part + min(m, kTcMaxN - 1) * kTcRows + rl);
#pragma unroll
    for (int c = 0; c < CSV; c++) L[j][c] = m < a.M ? dsmem_ld(dsmem_map(addr, uint32_t(c))) : 0u;
  }
  float yv[T];
  uint32_t iv[T];
#pragma unroll
  for (int j = 0; j < T; j++) {
    const int m = min(r0 + 2 * CSV * j, kTcMaxN - 1);  // tokens past M are computed and not stored
    uint32_t P = 0;
#pragma unroll
    for (int c = 0; c < CSV; c++) P += L[j][c];
    iv[j] = uint32_t(int(P - uint32_t(tk.zx[m]) * tk.sw - tk.zw * uint32_t(tk.t[m])));
    yv[j] = __fmul_rn(tk.dw, tk.dx[m]) * float(int(iv[j]));
  }
  tc_store_outputs<T>(a, row, r0, 2 * CSV, yv, iv);
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
  const int CS = a.CS, S = a.stages;
  const uint32_t rank = CS > 1 ? cluster_rank() : 0u;
  const int rb0 = (blockIdx.x / CS) * kTcRb;
  const int kt0 = int(rank) * a.KT / CS, nt = (int(rank) + 1) * a.KT / CS - kt0;  // this CTA's tiles
  uint8_t* stages = smem + kTcOffStages;
  uint8_t* region = stages + size_t(S) * a.stage_bytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(region);         // stage filled
  uint64_t* empty = reinterpret_cast<uint64_t*>(region + 64);   // stage's MMAs done
  uint64_t* ready = reinterpret_cast<uint64_t*>(region + 144);  // operand buffer written
  // words: [0] tmem address, [1] a role stopped, [2] bad header, [3] this CTA failed,
  // [4] tiles whose copies were issued, [5] tiles whose MMAs were committed
  uint32_t* words = reinterpret_cast<uint32_t*>(region + 160);
  float* tok_dx = reinterpret_cast<float*>(region + 256);
  int* tok_zx = reinterpret_cast<int*>(region + 256 + 4 * kTcMaxN);
  int* tok_t = reinterpret_cast<int*>(region + 256 + 8 * kTcMaxN);  // S_x - K z_x (mod 2^32)
  const uint32_t tb = uint32_t(a.tile_bytes);
  const uint32_t raw_a = uint32_t(kTcRb) * tb;  // a stage: the weight box, then the codes
  const uint32_t cbytes = uint32_t(a.Mp) * 256u;

  pdl_trigger();
  if (tid == 0) {
    for (int st = 0; st < S; st++) {
      mbar_init(&full[st], 1);
      mbar_init(&empty[st], 1);
    }
    for (int b = 0; b < 2; b++) mbar_init(&ready[b], kTcLayoutWarps);
    fence_mbar_init();
    for (int i = 1; i < 8; i++) words[i] = 0;
  }
  if (warp == 0) {  // tensor-memory accumulators: 128 lanes x 64 columns
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;\n" ::"r"(smem_u32(words)),
                 "r"(kTcColsAlloc)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;\n" ::: "memory");
  }
  // the row this thread writes in the epilogue (row tid % 128 of the CTA's 128) and its
  // constant weight parameters
  const int row = rb0 * 16 + (tid & 127);
  float dw = 0.f;
  uint32_t zw = 0, sw = 0;
  if (warp < kTcLayoutWarps && row < a.N) {
    dw = __ldg(a.row_delta + row);
    zw = uint32_t(__ldg(a.row_zero + row));
    sw = uint32_t(__ldg(a.row_sum + row));
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = words[0];

  auto stage_of = [&](int j) { return stages + size_t(j % S) * a.stage_bytes; };
  auto issue_w = [&](int j) {  // weights are constant: fetched before the dependency wait too
    tma_load_3d(stage_of(j), &a.wmap, 0, (kt0 + j) * int(tb / 256u), rb0, &full[j % S]);
  };
  auto issue_c = [&](int j) {  // one contiguous copy: the tile's codes of every token
    bulk_g2s(stage_of(j) + raw_a, a.act_codes + size_t(kt0 + j) * cbytes, cbytes, &full[j % S]);
  };
  const int first = min(S, nt);
  const bool producer = warp == kTcProducerWarp && lane == 0;
  if (producer) {
    for (int j = 0; j < first; j++) {
      mbar_expect_tx(&full[j], raw_a + cbytes);
      issue_w(j);
    }
  }
  pdl_wait();  // the act buffer may be the previous kernel's output
  if (producer) {
    // nothing past the header is read unless it matches this layer (every section then lies
    // inside the buffer); a bad header completes the first stages' transactions without the
    // codes, and every role skips its loop
    if (!tc_header_ok(a.act_hdr, a)) {
      words[2] = 1;
      atomicOr(&g_bq_device_error, kErrActHeader);
      for (int j = 0; j < first; j++) mbar_complete_tx(&full[j], cbytes);
    } else {
      for (int j = 0; j < first; j++) issue_c(j);
    }
  }
  __syncthreads();
  const bool bad = words[2] != 0;
  if (!bad) {
    for (int m = tid; m < a.M; m += kTcThreads) {
      const int zx = int(a.act_tok[4 * m + 1]);
      tok_dx[m] = __uint_as_float(a.act_tok[4 * m]);
      tok_zx[m] = zx;
      tok_t[m] = int(a.act_tok[4 * m + 2] - uint32_t(a.K) * uint32_t(zx));
    }
  }
  uint32_t* stop = &words[1];

  if (producer) {
    int issued = first;
    // stage j % S is free again once the MMAs of tile j - S are done (use j / S - 1 of the stage)
    for (int j = first; j < nt && !bad; j++) {
      if (!tc_wait(&empty[j % S], uint32_t((j / S - 1) & 1), stop)) {
        *reinterpret_cast<volatile uint32_t*>(stop) = 1u;
        break;
      }
      mbar_expect_tx(&full[j % S], raw_a + cbytes);
      issue_w(j);
      issue_c(j);
      issued = j + 1;
    }
    words[4] = uint32_t(issued);
  } else if (warp == kTcMmaWarp) {
    if (lane == 0) {
      const uint32_t idesc = tc_instr_desc(a.Mp, kTcRows);
      const uint32_t lbo_b = uint32_t(a.Mp) * 16u;
      int committed = 0;
      for (int j = 0; j < nt && !bad; j++) {
        const int buf = j & 1;
        if (!tc_wait(&ready[buf], uint32_t((j >> 1) & 1), stop)) {
          *reinterpret_cast<volatile uint32_t*>(stop) = 1u;
          break;
        }
        tc_fence_after();
        const uint32_t ta = tmem + kTcColA + uint32_t(buf) * kTcColsA, cb = smem_u32(stage_of(j) + raw_a);
#pragma unroll
        for (int i = 0; i < 8; i++)  // chunk i: A columns 8i .. 8i + 7, B k-units 2i, 2i + 1
          tc_mma_ta(tmem, ta + 8u * uint32_t(i), tc_smem_desc(cb + i * 2 * lbo_b, lbo_b, kTcSboB), idesc, j > 0 || i > 0);
        tc_commit(&empty[j % S]);
        committed = j + 1;
      }
      words[5] = uint32_t(committed);
    }
  } else if (warp < kTcLayoutWarps) {
    // warp w takes row block b = 2 (w % 4) + w / 4 of every tile: tensor-memory lanes 16b .. 16b + 15,
    // inside its quarter of the lanes (32 (w % 4) .. + 31)
    const int rbl = 2 * (warp & 3) + (warp >> 2);
    const uint32_t lane_base = uint32_t(16 * rbl) << 16;
    for (int j = 0; j < nt && !bad; j++) {
      const int buf = j & 1;
      bool ok = tc_wait(&full[j % S], uint32_t((j / S) & 1), stop);
      // operand buffer j % 2 is free once the MMAs of tile j - 2 are done (its stage's empty phase;
      // that stage's next use needs this warp's arrival for a later tile, so the phase cannot alias)
      if (j >= 2 && ok) ok = tc_wait(&empty[(j - 2) % S], uint32_t(((j - 2) / S) & 1), stop);
      if (!__all_sync(0xffffffffu, ok)) {
        if (lane == 0) *reinterpret_cast<volatile uint32_t*>(stop) = 1u;
        break;
      }
      tc_fence_after();
      const uint8_t* tile = stage_of(j) + rbl * tb;
      const uint32_t ta = tmem + lane_base + kTcColA + uint32_t(buf) * kTcColsA;
#pragma unroll
      for (int kc = 0; kc < 8; kc++) {
        // word w of lane 4g + t holds row g + 8(w & 1) of the block at k = 32kc + 16(w >> 1) + 4t + b
        // (stream s keeps that chunk as field kc % (8/f) of its uint4 kc / (8/f)). The store puts
        // words 0, 2 (row g) and 1, 3 (row g + 8) in columns 8kc + 2t and 8kc + 2t + 1: the MMA's
        // k position 4c + b of column c holds k = 32kc + 16 (c & 1) + 4 (c >> 1) + b, and the act
        // buffer's tensor-core copy orders the codes the same way
        uint32_t w4[4] = {0u, 0u, 0u, 0u};
        tc_stream_fields<F0, 0>(tile, kc, lane, w4);
        if constexpr (F1 > 0) tc_stream_fields<F1, F0>(tile + 512 * F0, kc, lane, w4);
        if constexpr (F2 > 0) tc_stream_fields<F2, F0 + F1>(tile + 512 * (F0 + F1), kc, lane, w4);
        tc_st16(ta + 8u * uint32_t(kc), w4[0], w4[2], w4[1], w4[3]);
      }
      tc_wait_st();
      tc_fence_before();  // the operand writes become visible to the MMA issued after the arrive
      __syncwarp();
      if (lane == 0) mbar_arrive(&ready[buf]);
    }
  }
  __syncthreads();  // every role has left its loop
  // drain: the last commit of every stage (commits track all earlier MMAs) and every issued
  // copy, so that nothing is pending on this block's shared memory or tensor memory when it exits
  if (tid == 0) {
    const int committed = int(words[5]), issued = int(words[4]);
    bool ok = true;
    for (int j = max(0, committed - S); j < committed; j++)
      ok = mbar_wait_bounded(&empty[j % S], uint32_t((j / S) & 1)) && ok;
    for (int j = max(0, issued - S); j < issued; j++)
      ok = mbar_wait_bounded(&full[j % S], uint32_t((j / S) & 1)) && ok;
    words[3] = (bad || !ok || words[1] != 0 || committed != nt) ? 1u : 0u;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const bool layout_warp = warp < kTcLayoutWarps;
  // re-layout warp w holds rows 32 (w % 4) + lane of the CTA's 128 and tokens 32 (w / 4) .. + 31
  const int lq = warp & 3, half = (warp >> 2) & 1;
  const int rl = 32 * lq + lane;
  uint32_t v[32];
  if (layout_warp) tc_ld32(tmem + (uint32_t(32 * lq) << 16) + uint32_t(32 * half), v);
  // y = Delta_w Delta_x I with I = P - z_x S_w - z_w (S_x - K z_x); I fits in int32 whenever the
  // layer's int32 accumulators do, so the wrapping 32-bit arithmetic gives it exactly
  if (CS == 1) {  // rl is tid % 128: this thread's row
    if (layout_warp && words[3] == 0 && row < a.N) {
      // every output first, then every store: a store between them would keep the compiler from
      // issuing the next token's shared loads early (it cannot tell the two pointers apart)
      float yv[32];
#pragma unroll
      for (int i = 0; i < 32; i++) {
        const int m = 32 * half + i;  // < kTcMaxN; tokens past M are computed and not stored
        v[i] = uint32_t(int(v[i] - uint32_t(tok_zx[m]) * sw - zw * uint32_t(tok_t[m])));
        yv[i] = __fmul_rn(dw, tok_dx[m]) * float(int(v[i]));
      }
      tc_store_outputs<32>(a, row, 32 * half, 1, yv, v);
    }
  } else {
    // reduce-scatter over the cluster: every CTA leaves its partial products at the start of its
    // (now idle) stage ring, [token][128 rows] (M x 512 bytes, within the ring's >= 3 stages of at
    // least Mp x 256 bytes each); CTA r sums tokens m = r, r + CS, ... over all CTAs and writes them
    uint32_t* part = reinterpret_cast<uint32_t*>(smem);
    if (layout_warp) {
#pragma unroll
      for (int i = 0; i < 32; i++) part[(32 * half + i) * kTcRows + rl] = v[i];
    }
    cluster_sync_all();
    uint32_t failed = 0;
    for (int c = 0; c < CS; c++) failed |= dsmem_ld(dsmem_map(smem_u32(&words[3]), uint32_t(c)));
    if (layout_warp && failed == 0 && row < a.N) {
      const TcTok tk{tok_dx, tok_zx, tok_t, dw, zw, sw};
      const int r0 = int(rank) + CS * (tid >> 7);  // the first of this thread's tokens
      switch (CS) {
        case 2: tc_cluster_out<2>(a, part, rl, row, r0, tk); break;
        case 3: tc_cluster_out<3>(a, part, rl, row, r0, tk); break;
        case 4: tc_cluster_out<4>(a, part, rl, row, r0, tk); break;
        case 5: tc_cluster_out<5>(a, part, rl, row, r0, tk); break;
        case 6: tc_cluster_out<6>(a, part, rl, row, r0, tk); break;
        case 7: tc_cluster_out<7>(a, part, rl, row, r0, tk); break;
        default: tc_cluster_out<8>(a, part, rl, row, r0, tk); break;
      }
    }
    cluster_sync_all();  // no CTA leaves while another may still read its partial products
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;\n" ::"r"(tmem), "r"(kTcColsAlloc) : "memory");
  }
}

}  // namespace bqi
