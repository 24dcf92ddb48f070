// C ABI: host-side validation, buffer layouts and kernel launches.
#pragma once

#include <cuda.h>  // CUcontext and CUresult types only; the driver calls are resolved at run time
#include <mutex>
#include <algorithm>
#include <cstring>

#include "bq_act.cuh"
#include "bq_gemv.cuh"
#include "bq_internal.cuh"
#include "bq_pack.cuh"
#include "bq_tc.cuh"

namespace bqi {

inline bool aligned(const void* p, size_t n) { return (reinterpret_cast<uintptr_t>(p) % n) == 0; }

inline bq_status check_nk(int N, int K) {
  if (N < 1 || N > BQ_MAX_N || K < 128 || K > BQ_MAX_K || K % 128 != 0) return BQ_ERR_SIZE;
  return BQ_OK;
}

// need_ptrs: the pack call reads the device pointers; the size query does not.
inline bq_status check_desc(const bq_pack_desc* d, int K, bool need_ptrs) {
  if (!d) return BQ_ERR_INVALID_ARG;
  if (d->fmt != BQ_FMT_RABIT2 && d->rabit_svid_rounds != 0) return BQ_ERR_INVALID_ARG;
  if (d->abq_bit_balance != 0 && (d->fmt != BQ_FMT_ABQ || d->abq_bit_balance != 1 || d->w_bits != 3))
    return BQ_ERR_INVALID_ARG;
  if (d->fmt != BQ_FMT_ABQ && (d->abq_comp_a || d->abq_comp_b)) return BQ_ERR_INVALID_ARG;
  if (d->fmt != BQ_FMT_RABIT3 && d->h3) return BQ_ERR_INVALID_ARG;
  if (d->bvsr_cluster_rounds != 0 && (d->fmt != BQ_FMT_BVSR4 || d->bvsr_cluster_rounds < 0 ||
                                      d->bvsr_cluster_rounds > 100))
    return BQ_ERR_INVALID_ARG;
  switch (d->fmt) {
    case BQ_FMT_RABIT2:
      if (d->rabit_svid_rounds < 0 || d->rabit_svid_rounds > 1000) return BQ_ERR_INVALID_ARG;
      if (need_ptrs && d->rabit_svid_rounds == 0 && (!d->h2 || !aligned(d->h2, 4))) return BQ_ERR_INVALID_ARG;
      return BQ_OK;
    case BQ_FMT_RABIT3:  // the residual recursion only; h2 and h3 given
      if (need_ptrs && (!d->h2 || !aligned(d->h2, 4) || !d->h3 || !aligned(d->h3, 4))) return BQ_ERR_INVALID_ARG;
      return BQ_OK;
    case BQ_FMT_BITNET_W1A8:
      return BQ_OK;
    case BQ_FMT_TERNARY_A8:
      if (d->lora_rank < 0 || d->lora_rank > BQ_MAX_LORA_RANK || d->lora_rank % 8 != 0) return BQ_ERR_INVALID_ARG;
      if (need_ptrs && d->lora_rank > 0 &&
          (!d->lora_A || !d->lora_B || !aligned(d->lora_A, 4) || !aligned(d->lora_B, 4)))
        return BQ_ERR_INVALID_ARG;
      if (!std::isfinite(d->lora_alpha)) return BQ_ERR_INVALID_ARG;
      return BQ_OK;
    case BQ_FMT_ABQ: {
      if (d->w_bits < 1 || d->w_bits > 8 || d->a_bits < 1 || d->a_bits > 8) return BQ_ERR_INVALID_ARG;
      const long long bound = ((1ll << d->w_bits) - 1) * ((1ll << d->a_bits) - 1) * (long long)K;
      if (bound >= (1ll << 31)) return BQ_ERR_SIZE;
      if (need_ptrs && (!d->abq_comp_a != !d->abq_comp_b || !aligned(d->abq_comp_a, 4) ||
                        !aligned(d->abq_comp_b, 4)))
        return BQ_ERR_INVALID_ARG;
      return BQ_OK;
    }
    case BQ_FMT_BVSR4:
      return BQ_OK;
    default:
      return BQ_ERR_INVALID_ARG;
  }
}

inline bool desc_layout(const bq_pack_desc* d, int N, int K, PkLayout* L) {
  const int rank = d->fmt == BQ_FMT_TERNARY_A8 ? d->lora_rank : 0;
  return make_pk_layout(d->fmt, N, K, d->w_bits, d->a_bits, rank, d->lora_alpha, L);
}

inline HeaderWords header_words(const PkLayout& L) {
  HeaderWords h{};
  h.w[HW_MAGIC] = kPkMagic;
  h.w[HW_VERSION] = kVersion;
  h.w[HW_FMT] = L.fmt;
  h.w[HW_N] = L.N;
  h.w[HW_K] = L.K;
  h.w[HW_NPAD] = L.N_pad;
  h.w[HW_KPAD] = L.K_pad;
  h.w[HW_WBITS] = L.w_bits;
  h.w[HW_ABITS] = L.a_bits;
  h.w[HW_NSTREAMS] = L.nstreams;
  for (int s = 0; s < 4; s++) {
    h.w[HW_FIELD + s] = s < L.nstreams ? L.field[s] : 0;
    h.w[HW_SHIFT + s] = s < L.nstreams ? L.shift[s] : 0;
  }
  h.w[HW_TILEBYTES] = L.tile_bytes;
  h.w[HW_LORA_RANK] = L.rank;
  std::memcpy(&h.w[HW_LORA_ALPHA], &L.lora_alpha, 4);
  h.w[HW_TSCALE] = 0;
  const uint64_t q[5] = {L.total, L.off_tiles, L.off_rows, L.off_aux, L.off_aux2};
  const int at[5] = {HW_TOTAL, HW_OFF_TILES, HW_OFF_ROWS, HW_OFF_AUX, HW_OFF_AUX2};
  for (int i = 0; i < 5; i++) {
    h.w[at[i]] = uint32_t(q[i]);
    h.w[at[i] + 1] = uint32_t(q[i] >> 32);
  }
  return h;
}

inline bq_status launch_status() {
  return cudaGetLastError() == cudaSuccess ? BQ_OK : BQ_ERR_CUDA;
}

inline unsigned blocks_for(uint64_t n, unsigned threads) { return unsigned((n + threads - 1) / threads); }

inline bq_status check_layer(const bq_layer* y, PkLayout* L) {
  if (!y || !y->packed || !aligned(y->packed, 256)) return BQ_ERR_INVALID_ARG;
  if (check_nk(y->N, y->K) != BQ_OK) return BQ_ERR_SIZE;
  // the same rules as the pack: a ternary rank in 0..64 and a multiple of 8 (the correction
  // rows are loaded 16 bytes at a time), no rank elsewhere, ABQ sums exact in int32
  if (y->fmt == BQ_FMT_TERNARY_A8 ? (y->lora_rank < 0 || y->lora_rank > BQ_MAX_LORA_RANK || y->lora_rank % 8 != 0)
                                  : y->lora_rank != 0)
    return BQ_ERR_INVALID_ARG;
  if (!layout_from_layer(y, L)) return BQ_ERR_INVALID_ARG;
  if (L->fmt == BQ_FMT_ABQ && ((1ll << L->w_bits) - 1) * ((1ll << L->a_bits) - 1) * (long long)L->K >= (1ll << 31))
    return BQ_ERR_INVALID_ARG;
  if (L->N_pad != y->N_pad || L->K_pad != y->K_pad || L->total > y->packed_bytes) return BQ_ERR_BAD_PACKED;
  return BQ_OK;
}


template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                              Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, args...);
}

// bq_linear runs an ABQ layer of more than one token as activation quantization into its
// workspace (an act buffer) followed by the layer from that buffer: the per-token asymmetric
// codes take a correctly rounded divide per element, which every CTA of the fused kernel would
// otherwise repeat for its tokens.
// bq_linear quantizes the activations once into an act buffer and runs the layer from it:
// ABQ from 2 tokens (its per-element divides would otherwise repeat in every CTA), and BVSR from
// 16 (the code image holds 8 tokens a CTA where the fused staging holds 4: 5120x5120 at M = 16
// 32.5 -> 24.4 us, at M = 64 199 -> 116 us; at M = 4 the fused call is faster, 14.6 vs 17.7 us)
constexpr int kBvsrViaActM = 16;
inline bool linear_via_act(const PkLayout& L, int M) {
  return (L.fmt == BQ_FMT_ABQ && M >= 2) || (L.fmt == BQ_FMT_BVSR4 && M >= kBvsrViaActM);
}

// bq_linear scratch: the ternary LoRA partial dot products [KT][M][r] (f32), or the act buffer
// of an ABQ layer of more than one token
inline uint64_t linear_workspace(const PkLayout& L, int M) {
  if (linear_via_act(L, M)) return align256(make_act_layout(L, M).total);
  return L.fmt == BQ_FMT_TERNARY_A8 && L.rank > 0 ? align256(uint64_t(L.KT) * M * L.rank * 4) : 0;
}

// Every field of LayerArgs that depends only on the layer, M and the outputs.
inline GroupLayer group_layer(const PkLayout& L, const void* packed, float* y, int64_t* acc, int rb_begin) {
  const uint8_t* P = static_cast<const uint8_t*>(packed);
  GroupLayer m{};
  m.tiles = P + L.off_tiles;
  m.hdr = reinterpret_cast<const uint32_t*>(P);
  m.row_delta = reinterpret_cast<const float*>(P + L.off_rows);
  m.row_zero = reinterpret_cast<const int*>(P + L.off_rows) + L.N_pad;
  m.row_sum = reinterpret_cast<const int*>(P + L.off_rows) + 2 * L.N_pad;
  m.y = y;
  m.acc = reinterpret_cast<long long*>(acc);
  m.N = L.N;
  m.rb_end = rb_begin + L.RB;
  return m;
}

inline LayerArgs layer_args(const PkLayout& L, const void* packed, int M, float* y, int64_t* acc) {
  const uint8_t* P = static_cast<const uint8_t*>(packed);
  LayerArgs g{};
  g.gl[0] = group_layer(L, packed, y, acc, 0);
  g.n_grp = 1;
  g.pk_hdr = reinterpret_cast<const uint32_t*>(P);
  g.lora_bt = reinterpret_cast<const uint16_t*>(P + L.off_aux2);
  g.bvsr_table = reinterpret_cast<const float*>(P + L.off_aux);
  g.rabit_planes = reinterpret_cast<const uint32_t*>(P + L.off_tiles);
  g.rabit_g = reinterpret_cast<const float*>(P + L.off_rows);
  g.rabit_h = reinterpret_cast<const float*>(P + L.off_aux);
  g.y = y;
  g.acc = reinterpret_cast<long long*>(acc);
  g.N = L.N; g.K = L.K; g.N_pad = L.N_pad; g.K_pad = L.K_pad; g.KT = L.KT; g.M = M;
  g.RB = L.RB;
  g.tile_bytes = L.tile_bytes; g.rank = L.fmt == BQ_FMT_TERNARY_A8 ? L.rank : 0; g.fmt = L.fmt;
  g.a_bits = L.a_bits;
  g.shift0 = L.shift[0]; g.shift1 = L.shift[1]; g.shift2 = L.shift[2];
  return g;
}

inline uint32_t align128(uint64_t x) { return uint32_t((x + 127) & ~uint64_t(127)); }

// Unique id of the calling thread's current CUDA context (cuCtxGetId), or 0 when there is
// none or the driver cannot tell. Context ids are never reused within a process, so a context
// created after cudaDeviceReset, or another context on the same device, has a new id. The two
// driver entry points are resolved once through the runtime, so the library does not link the
// driver library (it still loads on a machine without one).
inline unsigned long long current_context_id() {
  typedef CUresult (*GetCurrent)(CUcontext*);
  typedef CUresult (*GetId)(CUcontext, unsigned long long*);
  static GetCurrent get_current = nullptr;
  static GetId get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<GetCurrent>(f);
    f = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<GetId>(f);
    (void)cudaGetLastError();
  });
  CUcontext c = nullptr;
  unsigned long long id = 0;
  if (!get_current || !get_id || get_current(&c) != CUDA_SUCCESS || !c || get_id(c, &id) != CUDA_SUCCESS) return 0;
  return id;
}

inline int sm_count() {
  static int n = [] {
    int dev = 0, v = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v <= 0) {
      cudaGetLastError();  // no device visible: plan for a B200's 148 SMs
      v = 148;
    }
    return v;
  }();
  return n;
}

inline int pow2ceil(int v) {
  int p = 1;
  while (p < v) p <<= 1;
  return p;
}

// Work split and shared-memory carve of the persistent k_layer (NW = 8 warps):
//  - tokens per CTA (tpc): fused, each token group of 256/pow2(tpc) threads holds its x
//    in at most 16 16-byte chunks per thread; unfused, the code image fits in 96 KB;
//  - about one CTA per SM, CPG CTAs per token group striding over the row blocks;
//  - the weight ring gets what is left (at most 96 KB; a CTA whose weight slab exceeds 128 KB
//    takes the whole SM), split among the warps that have row
//    blocks: S (2..4) stages of C tiles per such warp.
// Returns false when the layer does not fit this kernel.
inline bool plan_layer(const PkLayout& L, int M, bool fused, LayerArgs* g) {
  constexpr int NW = 8, NT = NW * 32;
  const int VPR = L.K_pad / 32;
  const bool bvsr = L.fmt == BQ_FMT_BVSR4;
  const int rank = L.fmt == BQ_FMT_TERNARY_A8 ? L.rank : 0;
  const int npad = L.K_pad / 8;
  g->cstride = L.KT * 256 + 16;
  // BVSR from an act buffer takes up to 16 tokens a CTA (two MMA groups on each decoded weight
  // fragment, so the layer is decoded once per 16 tokens); everything else at most 8
  int tpc = std::min(bvsr && !fused ? bqi::kMaxTpc : 8, M);
  if (fused) {
    auto J = [&](int t) { return (npad + NT / pow2ceil(t) - 1) / (NT / pow2ceil(t)); };
    while (tpc > 1 && J(tpc) > kMaxXChunks) tpc--;
    g->J = J(tpc) > kMaxXChunks ? 0 : J(tpc);  // 0 (then tpc = 1): the staging reads x twice
  } else {
    while (tpc > 1 && uint64_t(tpc) * g->cstride > 96 * 1024) tpc--;
    g->J = 0;
  }
  g->tpc = tpc;
  g->TG = (M + tpc - 1) / tpc;
  // BVSR tiles are long latency-bound instruction chains (about 400 instructions a 2176-byte
  // tile): at one token per CTA, two CTAs of the same launch share each SM so that 16 warps
  // hide each other's latency; the other formats (and multi-token or act-buffer BVSR, whose code
  // image is large and whose kernel takes more registers) keep about one CTA per SM.
  const int ctas_per_sm = bvsr && tpc == 1 && fused ? 2 : 1;
  g->CPG = std::max(1, std::min(L.RB, (ctas_per_sm * sm_count() + g->TG - 1) / g->TG));
  // Warps sharing a row block (the k-split), a power of two: the one with the least modelled
  // time. Warp w issues on SM sub-partition w % 4, where the MMA and field-mask issue of a
  // tile costs about tile_c cycles (measured: ~145 per 8-MMA stream, ~900 for a BVSR tile);
  // each row block a warp group finishes costs about epi_c cycles (split-K exchange and
  // epilogue: ~1000 measured with a split, ~300 without). Ties go to the wider split.
  // A BVSR tile is a latency-bound chain, so groups of fewer than 4 warps leave a CTA of one row
  // block mostly idle whatever the model says (5120x13824: 2-warp groups 38.9 us, 4-warp 28.6).
  const int ipc = (L.RB + g->CPG - 1) / g->CPG;
  const long long tile_c = bvsr ? 900 : 145ll * L.nstreams;
  int wpr = 1;
  long long best = -1;
  for (int w = NW; w >= (bvsr ? 4 : 1); w /= 2) {
    const int G = NW / w, T = (L.KT + w - 1) / w;
    long long load[4] = {0, 0, 0, 0};
    int max_items = 0;
    for (int v = 0; v < NW; v++) {
      const int gr = v / w, wg = v % w;
      const int items = gr < ipc ? (ipc - gr + G - 1) / G : 0;
      const int nt = std::max(0, std::min(L.KT, wg * T + T) - wg * T);
      load[v % 4] += (long long)items * nt * tile_c;
      max_items = std::max(max_items, items);
    }
    const long long cost = std::max(std::max(load[0], load[1]), std::max(load[2], load[3])) +
                           (long long)max_items * (w > 1 ? 1000 : 300);
    if (best < 0 || cost < best) { best = cost; wpr = w; }
  }
  g->WPR = wpr;
  g->T = (L.KT + wpr - 1) / wpr;
  uint64_t off = 0;
  auto take = [&](uint64_t bytes) {
    const uint32_t o = uint32_t(off);
    off = align128(off + bytes);
    return o;
  };
  g->off_codes = take(uint64_t(tpc) * g->cstride);
  g->off_tok = take(bqi::kTokWords * 4);  // per-token words, tanh(alpha), weight scale
  g->off_u = take(rank > 0 ? uint64_t(tpc) * rank * 4 : 16);
  g->off_gsum = take(bvsr ? uint64_t(tpc) * VPR * 4 : 16);
  g->off_tab = take(bvsr ? uint64_t(kBvsrSets) * kBvsrTableStride * 4 + 4 * 16 : 16);  // + the family tables
  // split-K exchange [G][2][WPR][32][4] of int64 (+ f32 for BVSR) when warps share a row
  // block; at least the staging reductions' 3 x 32 words
  g->off_red = take(wpr > 1 ? 2ull * NW * 32 * 4 * (bvsr ? 12 : 8) * (tpc > 8 ? 2 : 1) : 512);
  // ternary: the B^T rows of the CTA's row blocks (32 rank bytes each) when they fit in 32 KB
  const uint64_t lbt = uint64_t(ipc) * 32 * rank;
  g->lbt_smem = rank > 0 && lbt <= 32 * 1024;
  g->off_lbt = take(g->lbt_smem ? lbt : 16);
  const uint64_t fixed = off + 1024;  // + barriers
  // The ring takes up to 96 KB. Most layers then leave room for a second CTA on the SM, so
  // the next launch's CTA is resident, and prefetching its weights, while this one computes;
  // a layer whose ring and fixed part exceed half of the SM runs alone. (Capping every
  // layer at half an SM measured slower on mixed-shape layer sequences.)
  const uint64_t limit = ctas_per_sm == 2 ? 112 * 1024 : 220 * 1024;  // two CTAs share the SM's 228 KB
  // A layer whose weight slab per CTA is large (more than 128 KB) streams most of it after the
  // wait whatever the ring: it gets the whole SM for its ring (one CTA per SM, more bytes in
  // flight) instead of leaving room for the next launch's CTA.
  const bool big = uint64_t(ipc) * L.KT * L.tile_bytes > 128 * 1024 && ctas_per_sm == 1;
  const uint64_t budget = std::min<uint64_t>(big ? limit : 96 * 1024, fixed < limit ? limit - fixed : 0);
  // The ring is split among the warps that have row blocks: groups 0 .. min(G, ipc) - 1, i.e.
  // warps 0 .. active - 1 (a CTA never holds more than ipc row blocks); idle warps get none.
  const int active = std::min(NW / wpr, ipc) * wpr;
  const uint64_t per_warp = budget / uint64_t(std::max(1, active));
  if (per_warp < 2ull * L.tile_bytes) return false;
  g->S = int(std::min<uint64_t>(4, std::max<uint64_t>(2, per_warp / L.tile_bytes)));
  g->C = int(std::max<uint64_t>(1, std::min<uint64_t>(g->T, per_warp / (uint64_t(g->S) * L.tile_bytes))));
  // BVSR: the same four tiles in flight as two chunks of two (half the copy issues, each of which
  // stalls its warp for ~0.3 us behind the other warps' shared-memory traffic)
  if (bvsr && g->S == 4 && g->C == 1 && g->T >= 2) { g->S = 2; g->C = 2; }
  g->off_ring = take(uint64_t(std::max(1, active)) * g->S * g->C * L.tile_bytes);
  g->off_bar = take(uint64_t(NW * g->S + 3) * 8 + 16);
  g->smem_bytes = uint32_t(off);
  g->RB = L.RB;
  return true;
}

// One instantiation per kernel, so the statics below track that kernel's raised dynamic
// shared-memory limit in the context that raised it; a launch in another context (another
// device, or a context created after a reset) raises it again there.
template <int FMT, int F0, int F1, int F2, int NW, bool FUSED, bool T1>
inline cudaError_t launch_tiled_nw(const LayerArgs& g, dim3 grid, cudaStream_t s) {
  auto k = k_layer<FMT, F0, F1, F2, NW, FUSED, T1>;
  static std::mutex mu;
  static unsigned long long limit_ctx = 0;
  static uint32_t smem_limit = 48 * 1024;
  if (g.smem_bytes > 48 * 1024) {
    const unsigned long long ctx = current_context_id();
    std::lock_guard<std::mutex> lock(mu);
    if (ctx == 0 || ctx != limit_ctx || g.smem_bytes > smem_limit) {
      const cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, int(g.smem_bytes));
      if (e != cudaSuccess) {
        (void)cudaGetLastError();  // leave no stale error behind
        return e;
      }
      if (ctx != limit_ctx) smem_limit = 48 * 1024;
      limit_ctx = ctx;
      smem_limit = std::max(smem_limit, g.smem_bytes);
    }
  }
  return launch_pdl(k, grid, dim3(NW * 32), g.smem_bytes, s, g);
}

template <int FMT, int F0, int F1, int F2, bool FUSED>
inline cudaError_t launch_tiled(const LayerArgs& g, int NW, dim3 grid, cudaStream_t s) {
  (void)NW;
  if (FUSED && g.tpc == 1) return launch_tiled_nw<FMT, F0, F1, F2, 8, FUSED, FUSED>(g, grid, s);
  return launch_tiled_nw<FMT, F0, F1, F2, 8, FUSED, false>(g, grid, s);
}

template <bool FUSED>
inline cudaError_t launch_fmt(const PkLayout& L, const LayerArgs& g, int NW, dim3 grid, cudaStream_t s) {
  switch (L.fmt) {
    case BQ_FMT_BITNET_W1A8: return launch_tiled<BQ_FMT_BITNET_W1A8, 1, 0, 0, FUSED>(g, NW, grid, s);
    case BQ_FMT_TERNARY_A8: return launch_tiled<BQ_FMT_TERNARY_A8, 2, 0, 0, FUSED>(g, NW, grid, s);
    case BQ_FMT_BVSR4: return launch_tiled<BQ_FMT_BVSR4, 1, 1, 1, FUSED>(g, NW, grid, s);
    case BQ_FMT_ABQ:
      switch (L.w_bits) {
        case 1: return launch_tiled<BQ_FMT_ABQ, 1, 0, 0, FUSED>(g, NW, grid, s);
        case 2: return launch_tiled<BQ_FMT_ABQ, 2, 0, 0, FUSED>(g, NW, grid, s);
        case 3: return launch_tiled<BQ_FMT_ABQ, 2, 1, 0, FUSED>(g, NW, grid, s);
        case 4: return launch_tiled<BQ_FMT_ABQ, 4, 0, 0, FUSED>(g, NW, grid, s);
        case 5: return launch_tiled<BQ_FMT_ABQ, 4, 1, 0, FUSED>(g, NW, grid, s);
        case 6: return launch_tiled<BQ_FMT_ABQ, 4, 2, 0, FUSED>(g, NW, grid, s);
        case 7: return launch_tiled<BQ_FMT_ABQ, 4, 2, 1, FUSED>(g, NW, grid, s);
        case 8: return launch_tiled<BQ_FMT_ABQ, 8, 0, 0, FUSED>(g, NW, grid, s);
        default: return cudaErrorInvalidValue;
      }
    default: return cudaErrorInvalidValue;
  }
}

// ABQ with 16..64 tokens (from an act buffer) runs on the tensor cores.
inline bool tc_eligible(const PkLayout& L, int M) { return tc_layer(L.fmt, L.w_bits, M); }

// The packed weight tiles of a layer as the tensor-core kernel's 3-D TMA map (TcTensorMap).
// cuTensorMapEncodeTiled is a host-side encode (no device work), resolved once through the
// runtime like the context query above.
inline bool encode_weight_map(const PkLayout& L, const void* tiles, TcTensorMap* out) {
  typedef CUresult (*EncodeTiled)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
  static_assert(sizeof(TcTensorMap) == sizeof(CUtensorMap), "tensor map size");
  static EncodeTiled encode = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      encode = reinterpret_cast<EncodeTiled>(f);
    (void)cudaGetLastError();
  });
  if (!encode) return false;
  const cuuint64_t dims[3] = {256u, cuuint64_t(L.KT) * L.tile_bytes / 256u, cuuint64_t(L.RB)};
  const cuuint64_t strides[2] = {256u, cuuint64_t(L.KT) * L.tile_bytes};  // bytes, dims 1 and 2
  const cuuint32_t box[3] = {256u, cuuint32_t(L.tile_bytes / 256), cuuint32_t(kTcRb)};
  const cuuint32_t estr[3] = {1u, 1u, 1u};
  CUtensorMap m;
  if (encode(&m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(tiles), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return false;
  std::memcpy(out, &m, sizeof(m));
  return true;
}

// Cluster size for G row groups of 128 and KT tiles: the split of the tiles that minimises
// waves x (tiles per CTA + kTcFixedTiles), where a wave is as many clusters as the device holds
// at once (max_clusters[cs], from the occupancy query) and kTcFixedTiles is a CTA's fixed cost
// (first copies, epilogue, cluster reduction) in tiles; ties go to the smaller cluster.
constexpr int kTcFixedTiles = 4;
inline int tc_cluster_size(int G, int KT, const int* max_clusters) {
  int best = 1;
  long long best_cost = -1;
  for (int cs = 1; cs <= kTcMaxCluster && cs <= KT; cs++) {
    if (max_clusters[cs] <= 0) continue;
    const long long waves = (G + max_clusters[cs] - 1) / max_clusters[cs];
    const long long cost = waves * ((KT + cs - 1) / cs + kTcFixedTiles);
    if (best_cost < 0 || cost < best_cost) { best = cs; best_cost = cost; }
  }
  return best;
}

// One instantiation per stream layout, so the statics below track that kernel's shared-memory
// limit and cluster occupancy in the context that set them.
template <int F0, int F1, int F2>
inline bq_status launch_abq_tc_f(const PkLayout& L, TcArgs t, cudaStream_t s) {
  auto k = k_abq_tc<F0, F1, F2>;
  static std::mutex mu;
  static unsigned long long set_ctx = 0;
  static int max_clusters[kTcMaxN / 16 + 1][kTcMaxCluster + 1];  // [Mp / 16][cluster size]
  const int G = (L.RB + kTcRb - 1) / kTcRb;
  const uint32_t smem = kTcOffStages + uint32_t(t.stages) * uint32_t(t.stage_bytes) + kTcBarBytes;
  int cs = 1;
  {
    const unsigned long long ctx = current_context_id();
    std::lock_guard<std::mutex> lock(mu);
    if (ctx == 0 || ctx != set_ctx) {
      if (cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, int(kTcSmemMax)) != cudaSuccess) {
        (void)cudaGetLastError();
        return BQ_ERR_CUDA;
      }
      for (auto& r : max_clusters)
        for (int& c : r) c = -1;
      set_ctx = ctx;
    }
    int* mc = max_clusters[t.Mp / 16];
    if (mc[1] < 0) {
      int dev = 0, sms = 0;
      if (cudaGetDevice(&dev) != cudaSuccess ||
          cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
        (void)cudaGetLastError();
        return BQ_ERR_CUDA;
      }
      for (int c = 1; c <= kTcMaxCluster; c++) {
        cudaLaunchConfig_t q = {};
        q.gridDim = dim3(unsigned(c));
        q.blockDim = dim3(kTcThreads);
        q.dynamicSmemBytes = smem;
        cudaLaunchAttribute at[1];
        at[0].id = cudaLaunchAttributeClusterDimension;
        at[0].val.clusterDim.x = unsigned(c);
        at[0].val.clusterDim.y = 1;
        at[0].val.clusterDim.z = 1;
        q.attrs = at;
        q.numAttrs = 1;
        int n = 0;
        if (cudaOccupancyMaxActiveClusters(&n, k, &q) != cudaSuccess) {
          (void)cudaGetLastError();
          n = c == 1 ? sms : 0;  // without the query: no clusters, one CTA per SM
        }
        mc[c] = n;
      }
    }
    cs = tc_cluster_size(G, L.KT, mc);
  }
  t.CS = cs;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(unsigned(G * cs));
  cfg.blockDim = dim3(kTcThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute at[2];
  at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[0].val.programmaticStreamSerializationAllowed = 1;
  at[1].id = cudaLaunchAttributeClusterDimension;
  at[1].val.clusterDim.x = unsigned(cs);
  at[1].val.clusterDim.y = 1;
  at[1].val.clusterDim.z = 1;
  cfg.attrs = at;
  cfg.numAttrs = cs > 1 ? 2 : 1;
  return cudaLaunchKernelEx(&cfg, k, t) == cudaSuccess ? BQ_OK : BQ_ERR_CUDA;
}

inline bq_status launch_abq_tc(const PkLayout& L, const void* packed, const void* act, int M, float* y,
                               int64_t* acc, cudaStream_t s) {
  const uint8_t* P = static_cast<const uint8_t*>(packed);
  const uint8_t* Ab = static_cast<const uint8_t*>(act);
  const ActLayout A = make_act_layout(L, M);
  TcArgs t{};
  if (!encode_weight_map(L, P + L.off_tiles, &t.wmap)) return BQ_ERR_CUDA;
  t.row_delta = reinterpret_cast<const float*>(P + L.off_rows);
  t.row_zero = reinterpret_cast<const int*>(P + L.off_rows + 4ull * L.N_pad);
  t.row_sum = reinterpret_cast<const int*>(P + L.off_rows + 8ull * L.N_pad);
  t.act_hdr = reinterpret_cast<const uint32_t*>(Ab);
  t.act_codes = Ab + A.off_ct;
  t.act_tok = reinterpret_cast<const uint32_t*>(Ab + A.off_tok);
  t.act_total = A.total;
  t.y = y;
  t.acc = reinterpret_cast<long long*>(acc);
  t.N = L.N; t.K = L.K; t.KT = L.KT; t.RB = L.RB; t.M = M; t.Mp = tc_tokens(M); t.a_bits = L.a_bits;
  t.tile_bytes = L.tile_bytes;
  t.stages = tc_stages(L.tile_bytes, t.Mp);
  t.stage_bytes = kTcRb * L.tile_bytes + t.Mp * 256;
  t.CS = 1;
  if (t.stages < 3) return BQ_ERR_UNSUPPORTED;
  switch (L.w_bits) {  // the fields of 8/4/2/1 bits from the low end of the code
    case 1: return launch_abq_tc_f<1, 0, 0>(L, t, s);
    case 2: return launch_abq_tc_f<2, 0, 0>(L, t, s);
    case 3: return launch_abq_tc_f<2, 1, 0>(L, t, s);
    case 4: return launch_abq_tc_f<4, 0, 0>(L, t, s);
    case 5: return launch_abq_tc_f<4, 1, 0>(L, t, s);
    case 6: return launch_abq_tc_f<4, 2, 0>(L, t, s);
    case 7: return launch_abq_tc_f<4, 2, 1>(L, t, s);
    case 8: return launch_abq_tc_f<8, 0, 0>(L, t, s);
    default: return BQ_ERR_UNSUPPORTED;
  }
}

inline bq_status launch_layer(const PkLayout& L, LayerArgs& g, bool fused, cudaStream_t s) {
  cudaError_t e;
  if (rabit_paths(L.fmt)) {
    const dim3 grid(unsigned((L.N + 7) / 8));
    if (rabit_paths(L.fmt) == 2)
      e = fused ? launch_pdl(k_rabit<8, true, 2>, grid, dim3(256), 0, s, g)
                : launch_pdl(k_rabit<8, false, 2>, grid, dim3(256), 0, s, g);
    else
      e = fused ? launch_pdl(k_rabit<8, true, 3>, grid, dim3(256), 0, s, g)
                : launch_pdl(k_rabit<8, false, 3>, grid, dim3(256), 0, s, g);
  } else {
    if (!plan_layer(L, g.M, fused, &g)) return BQ_ERR_UNSUPPORTED;
    const dim3 grid(unsigned(g.TG * g.CPG));
    e = fused ? launch_fmt<true>(L, g, 8, grid, s) : launch_fmt<false>(L, g, 8, grid, s);
  }
  return e == cudaSuccess ? BQ_OK : BQ_ERR_CUDA;
}

}  // namespace bqi

using namespace bqi;

extern "C" {

const char* bq_status_str(bq_status s) {
  switch (s) {
    case BQ_OK: return "ok";
    case BQ_ERR_INVALID_ARG: return "invalid argument";
    case BQ_ERR_UNSUPPORTED: return "unsupported";
    case BQ_ERR_SIZE: return "size out of range or buffer too small";
    case BQ_ERR_CUDA: return "CUDA error";
    case BQ_ERR_BAD_PACKED: return "bad packed buffer";
    case BQ_ERR_DEVICE_CHECK: return "device-side check failed";
    default: return "unknown status";
  }
}

int32_t bq_version(void) { return BQ_ABI_VERSION; }

bq_status bq_packed_bytes(const bq_pack_desc* desc, int32_t N, int32_t K, size_t* bytes) {
  if (!bytes) return BQ_ERR_INVALID_ARG;
  bq_status st = check_nk(N, K);
  if (st != BQ_OK) return st;
  if ((st = check_desc(desc, K, false)) != BQ_OK) return st;
  PkLayout L;
  if (!desc_layout(desc, N, K, &L)) return BQ_ERR_INVALID_ARG;
  *bytes = size_t(L.total);
  return BQ_OK;
}

bq_status bq_pack_weights(const bq_pack_desc* desc, const float* W, int32_t N, int32_t K, void* packed,
                          size_t packed_bytes, void* stream, bq_layer* layer) {
  bq_status st = check_nk(N, K);
  if (st != BQ_OK) return st;
  if ((st = check_desc(desc, K, true)) != BQ_OK) return st;
  if (!W || !aligned(W, 16) || !packed || !aligned(packed, 256) || !layer) return BQ_ERR_INVALID_ARG;
  PkLayout L;
  if (!desc_layout(desc, N, K, &L)) return BQ_ERR_INVALID_ARG;
  if (packed_bytes < L.total) return BQ_ERR_SIZE;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  uint8_t* P = static_cast<uint8_t*>(packed);
  uint32_t* hdr = reinterpret_cast<uint32_t*>(P);
  if (cudaMemsetAsync(P, 0, L.total, s) != cudaSuccess) return BQ_ERR_CUDA;
  k_write_header<<<1, 64, 0, s>>>(hdr, header_words(L));

  FieldPackArgs fa{};
  fa.W = W; fa.tiles = reinterpret_cast<uint32_t*>(P + L.off_tiles);
  fa.N = N; fa.K = K; fa.KT = L.KT; fa.tile_words = L.tile_bytes / 4; fa.nstreams = L.nstreams;
  int soff = 0;
  for (int i = 0; i < 4; i++) {
    fa.field[i] = L.field[i]; fa.shift[i] = L.shift[i]; fa.soff_words[i] = soff;
    if (i < L.nstreams) soff += 128 * L.field[i];
  }
  fa.hdr = hdr; fa.w_bits = L.w_bits;
  fa.total_words = uint64_t(L.RB) * L.KT * (L.tile_bytes / 4);

  switch (L.fmt) {
    case BQ_FMT_BITNET_W1A8:
    case BQ_FMT_TERNARY_A8: {
      double* rs = reinterpret_cast<double*>(P + L.off_tiles);   // scratch, overwritten below
      k_row_abs_sum<<<N, 256, 0, s>>>(W, K, rs);
      k_tensor_mean<<<1, 1024, 0, s>>>(rs, N, double(N) * double(K), hdr);
      if (L.fmt == BQ_FMT_BITNET_W1A8)
        k_pack_fields<BQ_FMT_BITNET_W1A8><<<blocks_for(fa.total_words, 256), 256, 0, s>>>(fa);
      else
        k_pack_fields<BQ_FMT_TERNARY_A8><<<blocks_for(fa.total_words, 256), 256, 0, s>>>(fa);
      if (L.fmt == BQ_FMT_TERNARY_A8 && L.rank > 0) {
        const uint64_t n = uint64_t(L.K_pad + L.N_pad) * L.rank;
        k_lora_to_bf16<<<blocks_for(n, 256), 256, 0, s>>>(
            desc->lora_A, desc->lora_B, N, K, L.N_pad, L.K_pad, L.rank, reinterpret_cast<uint16_t*>(P + L.off_aux),
            reinterpret_cast<uint16_t*>(P + L.off_aux2));
      }
      break;
    }
    case BQ_FMT_ABQ: {
      float* delta = reinterpret_cast<float*>(P + L.off_rows);
      int* zero = reinterpret_cast<int*>(P + L.off_rows) + L.N_pad;
      int* sumq = reinterpret_cast<int*>(P + L.off_rows) + 2 * L.N_pad;
      k_abq_rows<<<N, 256, 0, s>>>(W, desc->abq_comp_a, desc->abq_comp_b, K, L.w_bits, desc->abq_bit_balance,
                                   delta, zero, sumq);
      fa.abq_delta = delta; fa.abq_zero = zero;
      fa.abq_comp_a = desc->abq_comp_a; fa.abq_comp_b = desc->abq_comp_b;
      k_pack_fields<BQ_FMT_ABQ><<<blocks_for(fa.total_words, 256), 256, 0, s>>>(fa);
      break;
    }
    case BQ_FMT_RABIT2: {
      uint32_t* planes = reinterpret_cast<uint32_t*>(P + L.off_tiles);
      float* g = reinterpret_cast<float*>(P + L.off_rows);
      float* h1 = reinterpret_cast<float*>(P + L.off_aux);
      float* h2 = reinterpret_cast<float*>(P + L.off_aux2);
      if (desc->rabit_svid_rounds == 0) {
        k_rabit_pack<<<N, 256, 0, s>>>(W, L.N_pad, K, L.K_pad, planes, g);
        k_rabit_h<<<blocks_for(L.K_pad, 256), 256, 0, s>>>(desc->h2, nullptr, K, L.K_pad, h1, h2, nullptr);
        break;
      }
      const uint64_t W32 = L.K_pad / 32;
      const uint64_t init = std::max<uint64_t>(2ull * L.N_pad * W32, std::max<uint64_t>(2ull * L.N_pad, L.K_pad));
      k_svid_init<<<blocks_for(init, 256), 256, 0, s>>>(L.N_pad, K, L.K_pad, planes, g, h1, h2);
      uint32_t* pl[2] = {planes, planes + size_t(L.N_pad) * W32};
      float* gp[2] = {g, g + L.N_pad};
      float* hp[2] = {h1, h2};
      for (int r = 0; r < desc->rabit_svid_rounds; r++)
        for (int q = 0; q < 2; q++) {
          const int o = 1 - q;
          k_svid_rows<<<blocks_for(N, 128), 128, 0, s>>>(W, N, K, L.K_pad, pl[o], gp[o], hp[o], pl[q], hp[q], gp[q]);
          k_svid_cols<<<blocks_for(K, 128), 128, 0, s>>>(W, N, K, L.K_pad, pl[o], gp[o], hp[o], gp[q], hp[q]);
        }
      break;
    }
    case BQ_FMT_RABIT3: {  // h first: the recursion reads the packed h_p
      uint32_t* planes = reinterpret_cast<uint32_t*>(P + L.off_tiles);
      float* g = reinterpret_cast<float*>(P + L.off_rows);
      float* h = reinterpret_cast<float*>(P + L.off_aux);
      k_rabit_h<<<blocks_for(L.K_pad, 256), 256, 0, s>>>(desc->h2, desc->h3, K, L.K_pad, h, h + L.K_pad,
                                                        h + 2 * size_t(L.K_pad));
      k_rabit_pack_paths<3><<<N, 256, 0, s>>>(W, h, L.N_pad, K, L.K_pad, planes, g);
      break;
    }
    case BQ_FMT_BVSR4: {
      const uint64_t V = uint64_t(N) * (K / 32);
      uint32_t* kmin = reinterpret_cast<uint32_t*>(P + L.off_tiles);   // scratch in the tile region
      uint32_t* kmax = kmin + V;
      uint32_t* counts = reinterpret_cast<uint32_t*>(P + L.off_aux);   // scratch in the table region
      float* table = reinterpret_cast<float*>(P + L.off_aux);
      k_bvsr_minmax<<<blocks_for(V, 256), 256, 0, s>>>(W, K, V, kmin, kmax);
      const unsigned cb = unsigned(std::min<uint64_t>(blocks_for(V, 256), 148ull * 8));
      for (int bit = 31; bit >= 0; bit--) k_bvsr_count<<<cb, 256, 0, s>>>(kmin, kmax, V, counts, bit);
      const int rounds = desc->bvsr_cluster_rounds;
      double* cen = rounds > 0 ? reinterpret_cast<double*>(P + L.off_aux + kBvsrSets * kBvsrTableStride * 4) : nullptr;
      k_bvsr_table<<<1, 256, 0, s>>>(counts, V, table, cen);
      if (rounds > 0) {  // the clustering reading of the coefficient cache
        unsigned long long* acc = reinterpret_cast<unsigned long long*>(cen + 2 * kBvsrSets);
        uint8_t* fam = reinterpret_cast<uint8_t*>(kmax + V);  // scratch in the tile region (9 V <= 17 V bytes)
        k_bvsr_grid_families<<<1, 128, 0, s>>>(cen);
        k_bvsr_family<<<blocks_for(4 * V, 256), 256, 0, s>>>(W, K, V, fam);
        for (int r = 0; r < rounds; r++) {
          if (cudaMemsetAsync(acc, 0, kBvsrSets * 3 * 8, s) != cudaSuccess) return BQ_ERR_CUDA;
          k_bvsr_assign<<<blocks_for(V, 256), 256, 0, s>>>(kmin, kmax, fam, V, cen, acc);
          k_bvsr_update<<<1, 256, 0, s>>>(acc, cen);
        }
        k_bvsr_cluster_sets<<<1, 256, 0, s>>>(cen, table);
      }
      if (cudaMemsetAsync(P + L.off_tiles, 0, L.off_rows - L.off_tiles, s) != cudaSuccess) return BQ_ERR_CUDA;
      const unsigned sb = unsigned(std::min<uint64_t>(V, 148ull * 16));
      k_bvsr_search<<<sb, 256, 0, s>>>(W, K, L.KT, V, table, reinterpret_cast<uint32_t*>(P + L.off_tiles));
      break;
    }
    default:
      return BQ_ERR_INVALID_ARG;
  }
  if ((st = launch_status()) != BQ_OK) return st;
  layer->fmt = L.fmt; layer->N = N; layer->K = K; layer->N_pad = L.N_pad; layer->K_pad = L.K_pad;
  layer->w_bits = L.w_bits; layer->a_bits = L.a_bits; layer->lora_rank = L.rank;
  layer->packed_bytes = packed_bytes; layer->packed = packed;
  return BQ_OK;
}

bq_status bq_packed_validate(const void* packed_host, size_t bytes, const void* packed_dev, bq_layer* layer) {
  if (!packed_host || bytes < 256 || !layer || !packed_dev || !aligned(packed_dev, 256)) return BQ_ERR_INVALID_ARG;
  uint32_t h[64];
  std::memcpy(h, packed_host, 256);
  if (h[HW_MAGIC] != kPkMagic || h[HW_VERSION] != kVersion) return BQ_ERR_BAD_PACKED;
  const int fmt = int(h[HW_FMT]), N = int(h[HW_N]), K = int(h[HW_K]);
  if (check_nk(N, K) != BQ_OK) return BQ_ERR_BAD_PACKED;
  const int rank = int(h[HW_LORA_RANK]);
  if (rank < 0 || rank > BQ_MAX_LORA_RANK) return BQ_ERR_BAD_PACKED;
  float alpha;
  std::memcpy(&alpha, &h[HW_LORA_ALPHA], 4);
  PkLayout L;
  if (!make_pk_layout(fmt, N, K, int(h[HW_WBITS]), int(h[HW_ABITS]), rank, alpha, &L)) return BQ_ERR_BAD_PACKED;
  const uint64_t total = uint64_t(h[HW_TOTAL]) | (uint64_t(h[HW_TOTAL + 1]) << 32);
  const uint64_t offs[4] = {L.off_tiles, L.off_rows, L.off_aux, L.off_aux2};
  const int at[4] = {HW_OFF_TILES, HW_OFF_ROWS, HW_OFF_AUX, HW_OFF_AUX2};
  for (int i = 0; i < 4; i++)
    if ((uint64_t(h[at[i]]) | (uint64_t(h[at[i] + 1]) << 32)) != offs[i]) return BQ_ERR_BAD_PACKED;
  if (total != L.total || int(h[HW_NPAD]) != L.N_pad || int(h[HW_KPAD]) != L.K_pad ||
      int(h[HW_TILEBYTES]) != L.tile_bytes || int(h[HW_NSTREAMS]) != L.nstreams)
    return BQ_ERR_BAD_PACKED;
  // every word the writer derives from the layout must agree with it: the kernels take bit
  // widths, fields and the correction rank from the layout, and load the correction rows 16
  // bytes at a time (a rank that is not a multiple of 8 would misalign them)
  const HeaderWords want = header_words(L);
  for (int w = HW_WBITS; w <= HW_LORA_RANK; w++)
    if (w != HW_TILEBYTES && h[w] != want.w[w]) return BQ_ERR_BAD_PACKED;
  if (fmt == BQ_FMT_TERNARY_A8 && (rank % 8 != 0 || !std::isfinite(alpha))) return BQ_ERR_BAD_PACKED;
  if (fmt != BQ_FMT_TERNARY_A8 && h[HW_LORA_ALPHA] != 0u) return BQ_ERR_BAD_PACKED;
  // the tensor scale: mean|W| for BitNet and ternary (finite, >= 0), unused (0) otherwise
  float tscale;
  std::memcpy(&tscale, &h[HW_TSCALE], 4);
  if (fmt == BQ_FMT_BITNET_W1A8 || fmt == BQ_FMT_TERNARY_A8) {
    if (!std::isfinite(tscale) || !(tscale >= 0.f)) return BQ_ERR_BAD_PACKED;
  } else if (h[HW_TSCALE] != 0u) {
    return BQ_ERR_BAD_PACKED;
  }
  for (int w = HW_OFF_AUX2 + 2; w < 64; w++)  // reserved
    if (h[w] != 0u) return BQ_ERR_BAD_PACKED;
  if (fmt == BQ_FMT_ABQ) {
    const long long bound = ((1ll << L.w_bits) - 1) * ((1ll << L.a_bits) - 1) * (long long)K;
    if (bound >= (1ll << 31)) return BQ_ERR_BAD_PACKED;
  }
  layer->fmt = fmt; layer->N = N; layer->K = K; layer->N_pad = L.N_pad; layer->K_pad = L.K_pad;
  layer->w_bits = L.w_bits; layer->a_bits = L.a_bits; layer->lora_rank = L.rank;
  layer->packed_bytes = total; layer->packed = packed_dev;
  return BQ_OK;
}

bq_status bq_act_bytes(const bq_layer* layer, int32_t M, size_t* bytes) {
  PkLayout L;
  bq_status st = check_layer(layer, &L);
  if (st != BQ_OK) return st;
  if (!bytes) return BQ_ERR_INVALID_ARG;
  if (M < 0 || M > BQ_MAX_M) return BQ_ERR_SIZE;
  *bytes = size_t(make_act_layout(L, M).total);
  return BQ_OK;
}

bq_status bq_quantize_act(const bq_layer* layer, const void* x_bf16, int32_t M, void* act, size_t act_bytes,
                          void* stream) {
  PkLayout L;
  bq_status st = check_layer(layer, &L);
  if (st != BQ_OK) return st;
  if (M < 0 || M > BQ_MAX_M) return BQ_ERR_SIZE;
  if (M == 0) return BQ_OK;
  if (!x_bf16 || !aligned(x_bf16, 16) || !act || !aligned(act, 256)) return BQ_ERR_INVALID_ARG;
  const ActLayout A = make_act_layout(L, M);
  if (act_bytes < A.total) return BQ_ERR_SIZE;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const uint8_t* P = static_cast<const uint8_t*>(layer->packed);
  ActArgs a{};
  a.x = static_cast<const uint16_t*>(x_bf16);
  a.act = static_cast<uint8_t*>(act);
  a.M = M; a.K = L.K; a.K_pad = L.K_pad; a.KT = L.KT; a.a_bits = L.a_bits; a.rank = A.rank; a.fmt = L.fmt;
  a.off_codes = A.off_codes; a.off_tok = A.off_tok; a.off_gsum = A.off_gsum; a.off_u = A.off_u; a.off_xt = A.off_xt;
  a.off_ct = A.off_ct;
  a.total = A.total;
  a.lora_A = reinterpret_cast<const uint16_t*>(P + L.off_aux);
  a.h = reinterpret_cast<const float*>(P + L.off_aux);
  if (rabit_paths(L.fmt)) {
    return launch_pdl(k_act_rabit, dim3(blocks_for(L.K_pad, 256), M), dim3(256), 0, s, a) == cudaSuccess
               ? BQ_OK : BQ_ERR_CUDA;
  }
  // each token's row splits over up to 148 / M blocks of 1024 threads; a row of at most 16 K
  // elements stays in the block's shared memory after the scale pass (read from x once)
  const int slices_target = std::max(1, std::min(L.KT, (148 + M - 1) / M));
  a.tiles_per_slice = (L.KT + slices_target - 1) / slices_target;
  const int slices = (L.KT + a.tiles_per_slice - 1) / a.tiles_per_slice;
  const dim3 grid(slices, M), block(1024);
  a.x_smem = L.K_pad <= kActRowSmemMax ? 1 : 0;
  const size_t xs_bytes = a.x_smem ? size_t(L.K_pad) * 2 : 0;
  cudaError_t e;
  switch (L.fmt) {
    case BQ_FMT_BITNET_W1A8: e = launch_pdl(k_act_quant<BQ_FMT_BITNET_W1A8>, grid, block, xs_bytes, s, a); break;
    case BQ_FMT_TERNARY_A8: e = launch_pdl(k_act_quant<BQ_FMT_TERNARY_A8>, grid, block, xs_bytes, s, a); break;
    case BQ_FMT_ABQ: e = launch_pdl(k_act_quant<BQ_FMT_ABQ>, grid, block, xs_bytes, s, a); break;
    case BQ_FMT_BVSR4: e = launch_pdl(k_act_quant<BQ_FMT_BVSR4>, grid, block, xs_bytes, s, a); break;
    default: return BQ_ERR_INVALID_ARG;
  }
  return e == cudaSuccess ? BQ_OK : BQ_ERR_CUDA;
}

bq_status bq_gemm(const bq_layer* layer, const void* act, int32_t M, float* y, int64_t* acc_dbg, void* stream) {
  PkLayout L;
  bq_status st = check_layer(layer, &L);
  if (st != BQ_OK) return st;
  if (M < 0 || M > BQ_MAX_M) return BQ_ERR_SIZE;
  if (M == 0) return BQ_OK;
  if (!act || !aligned(act, 256) || !y || !aligned(y, 4) || (acc_dbg && !aligned(acc_dbg, 8)))
    return BQ_ERR_INVALID_ARG;
  if (rabit_paths(L.fmt) && acc_dbg) return BQ_ERR_UNSUPPORTED;
  if (tc_eligible(L, M)) return launch_abq_tc(L, layer->packed, act, M, y, acc_dbg, reinterpret_cast<cudaStream_t>(stream));
  const uint8_t* Ab = static_cast<const uint8_t*>(act);
  const ActLayout A = make_act_layout(L, M);
  LayerArgs g = layer_args(L, layer->packed, M, y, acc_dbg);
  g.act_hdr = reinterpret_cast<const uint32_t*>(Ab);
  g.act_codes = Ab + A.off_codes;
  g.act_tok = reinterpret_cast<const uint32_t*>(Ab + A.off_tok);
  g.u_part = reinterpret_cast<const float*>(Ab + A.off_u);
  g.act_gsum = reinterpret_cast<const int*>(Ab + A.off_gsum);
  g.act_xt = reinterpret_cast<const float*>(Ab + A.off_xt);
  g.act_total = A.total;
  return launch_layer(L, g, false, reinterpret_cast<cudaStream_t>(stream));
}

bq_status bq_linear_workspace_bytes(const bq_layer* layer, int32_t M, size_t* bytes) {
  PkLayout L;
  bq_status st = check_layer(layer, &L);
  if (st != BQ_OK) return st;
  if (!bytes) return BQ_ERR_INVALID_ARG;
  if (M < 0 || M > BQ_MAX_M) return BQ_ERR_SIZE;
  *bytes = size_t(linear_workspace(L, M));
  return BQ_OK;
}

bq_status bq_linear(const bq_layer* layer, const void* x_bf16, int32_t M, float* y, int64_t* acc_dbg,
                    void* workspace, size_t workspace_bytes, void* stream) {
  PkLayout L;
  bq_status st = check_layer(layer, &L);
  if (st != BQ_OK) return st;
  if (M < 0 || M > BQ_MAX_M) return BQ_ERR_SIZE;
  if (M == 0) return BQ_OK;
  if (!x_bf16 || !aligned(x_bf16, 16) || !y || !aligned(y, 4) || (acc_dbg && !aligned(acc_dbg, 8)))
    return BQ_ERR_INVALID_ARG;
  if (rabit_paths(L.fmt) && acc_dbg) return BQ_ERR_UNSUPPORTED;
  const uint64_t need = linear_workspace(L, M);
  if (need > 0 && (!workspace || !aligned(workspace, 256))) return BQ_ERR_INVALID_ARG;
  if (workspace_bytes < need) return BQ_ERR_SIZE;
  if (linear_via_act(L, M)) {
    st = bq_quantize_act(layer, x_bf16, M, workspace, workspace_bytes, stream);
    return st != BQ_OK ? st : bq_gemm(layer, workspace, M, y, acc_dbg, stream);
  }
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const uint8_t* P = static_cast<const uint8_t*>(layer->packed);
  LayerArgs g = layer_args(L, layer->packed, M, y, acc_dbg);
  g.x = static_cast<const uint16_t*>(x_bf16);
  if (L.fmt == BQ_FMT_TERNARY_A8 && L.rank > 0) {
    float* up = static_cast<float*>(workspace);
    if (launch_pdl(k_lora_partial, dim3((L.KT * M * (L.rank / 8) + 7) / 8), dim3(256), 0, s, g.x,
                   reinterpret_cast<const uint16_t*>(P + L.off_aux), M, L.K, L.KT, L.rank, up) != cudaSuccess)
      return BQ_ERR_CUDA;
    g.u_part = up;
  }
  return launch_layer(L, g, true, s);
}

// Scratch of bq_linear_static_scratch (one copy per device context).
static __device__ __align__(256) uint8_t g_bq_static_scratch[BQ_STATIC_SCRATCH_BYTES];

namespace {
constexpr int kMaxDevices = 64;

// Device address of the scratch array in the current context. The address belongs to the
// context the library's module was loaded into, so it is cached per device together with that
// context's id, and looked up again (cudaGetSymbolAddress, with the device current) whenever
// the current context is not the one it was looked up in: after cudaDeviceReset, or under
// another context on the same device. Without a context id (none current yet, or a driver that
// cannot tell) it is looked up on every call.
bq_status static_scratch(void** out) {
  static std::mutex mu;
  static void* addr[kMaxDevices] = {};
  static unsigned long long ctx_of[kMaxDevices] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    (void)cudaGetLastError();
    return BQ_ERR_CUDA;
  }
  if (dev < 0 || dev >= kMaxDevices) return BQ_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(mu);
  const unsigned long long ctx = current_context_id();
  if (!addr[dev] || ctx == 0 || ctx != ctx_of[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_bq_static_scratch) != cudaSuccess || !p) {
      (void)cudaGetLastError();
      return BQ_ERR_CUDA;
    }
    addr[dev] = p;
    ctx_of[dev] = current_context_id();  // the lookup makes the device's context current
  }
  *out = addr[dev];
  return BQ_OK;
}
}  // namespace

bq_status bq_linear_static_scratch(const bq_layer* layer, const void* x_bf16, int32_t M, float* y,
                                   int64_t* acc_dbg, void* stream) {
  size_t need = 0;
  bq_status st = bq_linear_workspace_bytes(layer, M, &need);
  if (st != BQ_OK) return st;
  if (need > BQ_STATIC_SCRATCH_BYTES) return BQ_ERR_SIZE;
  void* ws = nullptr;
  st = static_scratch(&ws);
  if (st != BQ_OK) return st;
  return bq_linear(layer, x_bf16, M, y, acc_dbg, need > 0 ? ws : nullptr, need, stream);
}

bq_status bq_linear_group(const bq_layer* layers, int32_t n_layers, const void* x_bf16, int32_t M,
                          float* const* y, int64_t* const* acc_dbg, void* stream) {
  static_assert(BQ_MAX_GROUP == kMaxGroup, "group size");
  if (!layers || !y || n_layers < 1 || n_layers > BQ_MAX_GROUP) return BQ_ERR_INVALID_ARG;
  if (n_layers == 1) return bq_linear(&layers[0], x_bf16, M, y[0], acc_dbg ? acc_dbg[0] : nullptr, nullptr, 0, stream);
  PkLayout Ls[BQ_MAX_GROUP];
  for (int i = 0; i < n_layers; i++) {
    const bq_status st = check_layer(&layers[i], &Ls[i]);
    if (st != BQ_OK) return st;
    if (!y[i] || !aligned(y[i], 4) || (acc_dbg && acc_dbg[i] && !aligned(acc_dbg[i], 8))) return BQ_ERR_INVALID_ARG;
    if (Ls[i].fmt != Ls[0].fmt || Ls[i].K != Ls[0].K || Ls[i].w_bits != Ls[0].w_bits ||
        Ls[i].a_bits != Ls[0].a_bits)
      return BQ_ERR_INVALID_ARG;
  }
  const PkLayout& L0 = Ls[0];
  const bool groupable = L0.fmt == BQ_FMT_BITNET_W1A8 || L0.fmt == BQ_FMT_ABQ ||
                         (L0.fmt == BQ_FMT_TERNARY_A8 && L0.rank == 0);
  for (int i = 1; i < n_layers; i++)
    if (Ls[i].rank != L0.rank) return BQ_ERR_INVALID_ARG;
  if (!groupable) return BQ_ERR_UNSUPPORTED;
  if (M < 0 || M > BQ_MAX_M) return BQ_ERR_SIZE;
  if (M == 0) return BQ_OK;
  if (!x_bf16 || !aligned(x_bf16, 16)) return BQ_ERR_INVALID_ARG;
  LayerArgs g = layer_args(L0, layers[0].packed, M, y[0], acc_dbg ? acc_dbg[0] : nullptr);
  g.x = static_cast<const uint16_t*>(x_bf16);
  int rb = L0.RB;
  for (int i = 1; i < n_layers; i++) {
    g.gl[i] = group_layer(Ls[i], layers[i].packed, y[i], acc_dbg ? acc_dbg[i] : nullptr, rb);
    rb += Ls[i].RB;
  }
  g.n_grp = n_layers;
  PkLayout Lg = L0;  // the work split sees the group's row blocks as one layer
  Lg.RB = rb;
  return launch_layer(Lg, g, true, reinterpret_cast<cudaStream_t>(stream));
}

bq_status bq_linear_plan(const bq_layer* layer, int32_t M, int32_t fused, bq_plan_info* info) {
  PkLayout L;
  bq_status st = check_layer(layer, &L);
  if (st != BQ_OK) return st;
  if (!info) return BQ_ERR_INVALID_ARG;
  if (M < 1 || M > BQ_MAX_M) return BQ_ERR_SIZE;
  if (rabit_paths(L.fmt)) return BQ_ERR_UNSUPPORTED;
  LayerArgs g{};
  if (!plan_layer(L, M, fused != 0 && !linear_via_act(L, M), &g)) return BQ_ERR_UNSUPPORTED;
  info->tokens_per_cta = g.tpc;
  info->token_groups = g.TG;
  info->ctas_per_group = g.CPG;
  info->warps_per_row_block = g.WPR;
  info->tiles_per_warp = g.T;
  info->ring_stages = g.S;
  info->tiles_per_stage = g.C;
  info->x_chunks_per_thread = g.J;
  info->shared_bytes = g.smem_bytes;
  return BQ_OK;
}

bq_status bq_gemv(const bq_layer* layer, const void* act, float* y, int64_t* acc_dbg, void* stream) {
  return bq_gemm(layer, act, 1, y, acc_dbg, stream);
}

bq_status bq_device_check(void) {
  if (cudaDeviceSynchronize() != cudaSuccess) return BQ_ERR_CUDA;
  unsigned int v = 0;
  if (cudaMemcpyFromSymbol(&v, g_bq_device_error, sizeof(v)) != cudaSuccess) return BQ_ERR_CUDA;
  if (v) {
    const unsigned int z = 0;
    if (cudaMemcpyToSymbol(g_bq_device_error, &z, sizeof(z)) != cudaSuccess) return BQ_ERR_CUDA;
    return BQ_ERR_DEVICE_CHECK;
  }
  return BQ_OK;
}

}  // extern "C"
