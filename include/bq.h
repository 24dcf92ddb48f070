/*
 * bq.h -- C ABI of the bit-plane quantized linear layer for NVIDIA B200 (sm_100a).
 *
 * One computation, y = sum_k scales (.) (B_k . x), for five weight formats (RaBiT in a
 * two-path and a three-path variant)
 * whose weights are stored as binary planes or bitvectors B_k:
 *
 *   BQ_FMT_RABIT2       RaBiT two-path residual binarization, W_hat = g1 B1 h1 + g2 B2 h2
 *                       ("RaBiT框架" page, §2.1 equation and §2.2 forward()).
 *   BQ_FMT_RABIT3       the same residual recursion with a third path, g3 B3 h3: the 3-bit
 *                       extension the "RaBiT框架" page lists in §6, read as one more residual
 *                       path (one bit per path).
 *   BQ_FMT_BITNET_W1A8  BitNet sign weights alpha*sign(W), alpha = mean|W| per tensor
 *                       ("1-bit LLM的端侧推理革命" page, §2.1-§2.3).
 *   BQ_FMT_TERNARY_A8   1.58-bit absmean ternary weights packed 2 bits/weight, with the
 *                       gated rank-r correction tanh(alpha) SiLU(xA) B fused in
 *                       ("1.58位LLM混合门控流" page, §1.2, §2.1, §4.1).
 *   BQ_FMT_ABQ          ABQ-style arbitrary-bit WxAy: per-row / per-token asymmetric codes,
 *                       the product decomposed over weight bit-planes
 *                       ("ABQ-LLM" page, abstract and §3.2 eq.(3)).
 *   BQ_FMT_BVSR4        BVSR 4-bit bitvector sums with 256 cached coefficient sets
 *                       ("BVSR" page, Introduction).
 *
 * Calls (the problem the pages state: pack offline, quantize activations online,
 * then GEMV for decode or a small-M GEMM):
 *   bq_packed_bytes / bq_pack_weights   quantize + pack W into a self-describing buffer
 *   bq_act_bytes / bq_quantize_act      per-token activation quantization
 *   bq_gemv (M = 1) / bq_gemm (M >= 1)  the layer, fused scale/zero-point/LoRA epilogue
 *   bq_linear                           activation quantization + layer in one kernel (decode)
 *   bq_linear_group                     up to 4 layers sharing their input x, one launch
 *   bq_linear_static_scratch            bq_linear with a fixed library scratch array
 *   bq_linear_plan                      the work split of bq_linear / bq_gemm (host only)
 * Pack options (bq_pack_desc): RaBiT iterative residual SVID initialisation of g and h
 * (rabit_svid_rounds, "RaBiT框架" page §2.3); ABQ bit-balance W2* (abq_bit_balance,
 * "ABQ-LLM" page §3.3); ABQ distribution compensation W + a b^T (abq_comp_a, abq_comp_b,
 * "ABQ-LLM" page §3.2 eq.(3)).
 *
 * Ownership: the caller allocates every buffer (device memory for packed, act, W, x, y);
 * sizes come from the *_bytes queries. The library never allocates (its one static
 * scratch array aside, see bq_linear_static_scratch), frees or synchronizes (bq_packed_validate and bq_device_check excepted, which touch host memory
 * or read one device word). All work is enqueued on the caller's stream (a cudaStream_t
 * passed as void*; NULL = legacy default stream).
 *
 * Errors: arguments are validated on the host before anything is enqueued; on error
 * nothing runs and a status is returned. A failed launch returns BQ_ERR_CUDA.
 * The kernels check the act-buffer header against the layer (version, format, M, K,
 * activation bits, correction rank and total size, so that every section they read lies
 * inside the buffer) before reading anything else from it; on a mismatch they write no
 * output and raise a device error word that bq_device_check reports.
 * No exception crosses this ABI, and there is no CPU fallback: every step runs on the GPU.
 *
 * ------------------------------------------------------------------------------------
 * Packed weight buffer (device, 256-byte aligned), little-endian, version 1.
 * Header: 64 x 32-bit words (256 bytes):
 *   0 magic 0x4B505142 ('BQPK')  1 version  2 format  3 N  4 K  5 N_pad (N rounded up to 16)
 *   6 K_pad (K rounded up to 256)  7 w_bits  8 a_bits  9 n_streams
 *   10..13 field width f_s of stream s (bits per weight)  14..17 shift of stream s
 *   18 tile_bytes  19 lora_rank  20 lora_alpha (f32)  21 tensor_scale (f32: BitNet alpha,
 *   ternary gamma_W)  22-23 total_bytes (u64)  24-25 off_tiles  26-27 off_rows
 *   28-29 off_aux  30-31 off_aux2 (u64 byte offsets from the buffer start)
 * Tiled weights (formats 2-5). Tile (rb, kt) covers rows 16rb..16rb+15 and
 *   k = 256kt..256kt+255, at off_tiles + (rb*(K_pad/256) + kt)*tile_bytes. Inside a tile
 *   the streams follow one another; stream s (field width f) takes 512*f bytes laid out
 *   as [u < f][lane < 32][4 words]. In word r (0..3) of uint4 u of lane = 4g+t, the f-bit
 *   field j (bits f*j .. f*j+f-1) of byte b holds the weight at
 *       row = 16rb + g + 8(r & 1),
 *       k   = 32(8kt + u*(8/f) + j) + 16(r >> 1) + 4t + b.
 *   This is the A-operand fragment order of the int8 m16n8k32 tensor-core MMA: one AND
 *   with the mask of field j turns four packed words into the four A registers of one MMA.
 *   Padding rows/columns hold zero fields (ternary: field 1, i.e. T = 0).
 *   Streams: BitNet 1 x f=1 (bit set <=> sign -1). Ternary 1 x f=2 (field = T+1 in {0,1,2}).
 *   ABQ: w_bits split into fields of 8/4/2/1 bits from the low end (2:[2] 4:[4] 6:[4,2]
 *   8:[8], shift = bit offset in the code). BVSR: one stream (n_streams 1, f = 4, shift 0)
 *   of 4-bit codes (code = sum_i 2^i b_i over the four bitvectors) in its own nibble order:
 *   2048 bytes as 4 blocks i of [lane < 32][4 words]; word 2v + h of lane 4g+t in block i
 *   holds vector j = 2i + v of the tile, nibble b of its low half the code of row 16rb + g
 *   and nibble b of its high half that of row 16rb + g + 8, at k = 256kt + 32j + 16h + 4t + b
 *   (the four halves of a lane's two words are the four A registers of the vector's MMA, one
 *   nibble per byte). Each BVSR tile ends with 128 bytes of set indices: byte 2048 + 8g + j
 *   (g < 16) is the set of row 16rb + g, vector 8kt + j (a vector is 32 contiguous k), so
 *   tile_bytes = 2176.
 * RaBiT (formats 1 and 6, P = 2 and 3 paths) is not tiled: bit j of uint32
 *   off_tiles + 4((p*N_pad + n)(K_pad/32) + w) is the sign of path p (0..P-1), row n,
 *   k = 32w + j (1 <=> -1).
 * Sections: RaBiT rows = g_p f32 [P][N_pad]; aux = h1[K_pad], aux2 = h2[K_pad] (format 6:
 *   h2, h3 [2][K_pad]) f32, so h_p (p = 0..P-1) starts at off_aux + 4 p K_pad.
 *   Ternary aux = A bf16 [K_pad][r], aux2 = B^T bf16 [N_pad][r].
 *   ABQ rows = Delta_w f32 [N_pad], z_w i32 [N_pad], S_w = sum_k q_w i32 [N_pad].
 *   BVSR aux = coefficient table f32 [256][8] (c0 c1 c2 c3 o; then derived kernel constants:
 *   sc = (hi-lo)/sum_i R_i, ratio index, and word 7 the integer templates R_0..R_3 as the
 *   bytes of a uint32, low byte first), then 10240 bytes of pack scratch (the clustering
 *   centroids f64 [256][2] and sums i64 [256][3]) that the layer never reads.
 *
 * Activation buffer (device, 256-byte aligned), version 1.
 * Header: 64 x 32-bit words: 0 magic 0x43415142 ('BQAC') 1 version 2 format 3 M 4 K 5 K_pad
 *   6 a_bits 7 lora_rank 8-9 total_bytes 10-11 off_codes 12-13 off_tok 14-15 off_gsum
 *   16-17 off_u 18-19 off_xt 20-21 off_ct (0 when absent).
 * codes (formats 2-5): per token m and k-tile kt, 256 bytes; byte
 *   (m*(K_pad/256) + kt)*256 + 64t + 8mu + 4h + b holds the code of k = 32(8kt+mu)+16h+4t+b
 *   (the B-operand fragment order; int8 two's complement for A8 formats, whose bits are
 *   the activation bit-planes X_c, uint8 for ABQ). Padding k hold code 0.
 * tok [M][4] words: A8 {gamma_x f32, sum_k q i32, 0, 0}; ABQ {Delta_x f32, z_x i32, S_x i32, 0}.
 * gsum (BVSR): i32 [M][K_pad/32], sum of q over each 32-element vector.
 * u (ternary): f32 [K_pad/256][M][r] partial dot products of the unquantized bf16 x with A
 *   over each 256-k tile (each in k order); the layer forms SiLU(sum over tiles).
 * xt (RaBiT): f32 [P][M][K_pad] = h_p * x (no activation quantization).
 * ct (ABQ with 16 <= M <= 64 only): the same codes in the K-major operand layout of the
 *   tensor cores' kind::i8 MMA, for Mp = M rounded up to a multiple of 16 tokens: byte
 *   kt*Mp*256 + u*Mp*16 + (m/8)*128 + (m%8)*16 + (p%16) with u = 2i + p/16 holds the code of
 *   token m at k = 256kt + 32i + k', p = 8((k'%16)/4) + 4(k'/16) + k'%4 (within each 32-k
 *   chunk the order the weight operand takes in tensor memory); tokens M .. Mp-1 hold code 0.
 *   bq_gemm on such a layer runs a tcgen05 kind::i8 GEMM (128 rows of the weights per CTA in
 *   tensor memory, the tokens as the MMA's N from shared memory, accumulators in tensor
 *   memory) that reads each k-tile's block with one copy and feeds it to the MMA in place; for
 *   few row groups a cluster of CTAs splits the k-tiles and sums the partial products through
 *   distributed shared memory.
 */
#ifndef BQ_H
#define BQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  BQ_OK = 0,
  BQ_ERR_INVALID_ARG = 1,  /* null/unaligned pointer, bad enum, inconsistent arguments */
  BQ_ERR_UNSUPPORTED = 2,  /* a combination this build does not implement */
  BQ_ERR_SIZE = 3,         /* N, K, M out of range or a buffer smaller than required */
  BQ_ERR_CUDA = 4,         /* a CUDA runtime call or kernel launch failed */
  BQ_ERR_BAD_PACKED = 5,   /* packed header failed validation */
  BQ_ERR_DEVICE_CHECK = 6  /* a kernel found an inconsistent buffer (see bq_device_check) */
} bq_status;

typedef enum {
  BQ_FMT_RABIT2 = 1,
  BQ_FMT_BITNET_W1A8 = 2,
  BQ_FMT_TERNARY_A8 = 3,
  BQ_FMT_ABQ = 4,
  BQ_FMT_BVSR4 = 5,
  BQ_FMT_RABIT3 = 6
} bq_format;

/* Limits: 1 <= N <= 1<<20, 128 <= K <= 1<<16 with K % 128 == 0, 1 <= M <= 64 (M = 0 is
 * a no-op). ABQ needs (2^w - 1)(2^a - 1) K < 2^31 so that the int32 plane sums are exact. */
#define BQ_MAX_N (1 << 20)
#define BQ_MAX_K (1 << 16)
#define BQ_MAX_M 64
#define BQ_MAX_LORA_RANK 64

/* Pack options. Device pointers are read during bq_pack_weights only. */
typedef struct {
  int32_t fmt;          /* bq_format */
  int32_t w_bits;       /* ABQ weight bits, 1..8 (ignored by the other formats) */
  int32_t a_bits;       /* ABQ activation bits, 1..8 (ignored: the A8 formats use 8) */
  int32_t lora_rank;    /* ternary: rank r of the correction, 0..64, a multiple of 8 (0 = none) */
  float lora_alpha;     /* ternary: gate alpha (finite); the correction is scaled by tanh(alpha) */
  const float* h2;      /* RaBiT, rabit_svid_rounds = 0: device f32 [K], second-path input
                           scale (h1 = 1); unused otherwise (may be NULL) */
  const float* lora_A;  /* ternary: device f32 [K][r] row-major, 4-byte aligned, rounded to bf16 */
  const float* lora_B;  /* ternary: device f32 [r][N] row-major, 4-byte aligned, rounded to bf16 */
  int32_t rabit_svid_rounds;  /* RaBiT initialisation: 0 = the residual recursion with mean|.|
                           row scales (h1 = 1, h2 given); R in 1..1000 = R rounds of the
                           iterative residual SVID ("RaBiT" page, §2.3, function-aware
                           initialisation, stage 1; its default is 20): each round fits path 1
                           to W - W2, then path 2 to W - W1, as sign(target) * (g h^T) by one
                           alternating least-squares step (g per row, then h per column), in
                           float64 with sums in index order, g and h kept in float32;
                           start g = 0, h = 1. Must be 0 for the other formats. */
  int32_t abq_bit_balance;  /* ABQ, 1 = W2* ("ABQ-LLM" page, §3.3 bit-balance strategy): the
                           symmetric five levels {-2..2} per row, Delta = max|W_row| / 2
                           (max(2 max|W|, 1e-5) / 4), z = 2, code = clamp(rn(W/Delta) + 2, 0, 4)
                           in a 3-bit field; requires w_bits = 3. The layer is the ABQ w = 3
                           layer. 0 = the asymmetric min/max codes. Must be 0 for the others. */
  const float* abq_comp_a;  /* ABQ distribution compensation ("ABQ-LLM" page, §3.2 eq.(3) with
                           gamma = 1): device f32 a [N] (one per output row) and b [K] (one per */
  const float* abq_comp_b;  /* input column). Both set: the matrix quantized is W + a b^T, each
                           element formed in f32 as W[n][k] + (a[n] * b[k]) (product rounded,
                           then the sum; no fused multiply-add), and Delta, z and the codes are
                           those of that matrix (with abq_bit_balance too: its W2* codes). The
                           layer then computes y = (W + a b^T)_hat x. Both NULL: off. One of
                           them NULL, or either set for another format: BQ_ERR_INVALID_ARG. */
  const float* h3;      /* RaBiT three paths (format 6): device f32 [K], the third path's input
                           scale (h1 = 1; h2 is required too). Format 6 runs the residual
                           recursion only (rabit_svid_rounds = 0). NULL for every other format. */
  int32_t bvsr_cluster_rounds;  /* BVSR coefficient cache ("BVSR" page, Introduction), clustering
                           reading: 0 = the 256 sets on the quantile grid; R in 1..100 = the sets
                           from R rounds of Lloyd's k-means: every vector takes the ratio family
                           whose set on its own [min, max] fits it best, and per family the
                           vectors' (min, max) points are clustered into 64 centroids started
                           from the quantile grid (exact means: int64 sums of rn(v 2^40)); set
                           64j + c spans centroid c. Must be 0 for the other formats. */
} bq_pack_desc;

/* Host-side description of a packed layer; filled by bq_pack_weights or
 * bq_packed_validate, read by every other call (so no call reads the device header
 * from the host). `packed` is the caller's device buffer. Every call checks it against
 * the pack's rules (sizes, a ternary lora_rank that is a multiple of 8 within 0..64 and 0
 * for the other formats, the ABQ int32 bound) and returns BQ_ERR_INVALID_ARG, or
 * BQ_ERR_BAD_PACKED for sizes that disagree, before anything runs. */
typedef struct {
  int32_t fmt, N, K, N_pad, K_pad, w_bits, a_bits, lora_rank;
  uint64_t packed_bytes;
  const void* packed;
} bq_layer;

/* ABI version: bumped whenever a struct layout or a call's meaning changes. A caller
 * compares bq_version() with the BQ_ABI_VERSION of the header it was built against.
 * 2: bq_pack_desc gained abq_comp_a, abq_comp_b and h3; format 6 (BQ_FMT_RABIT3).
 * 3: bq_pack_desc gained bvsr_cluster_rounds; the BVSR tile holds 4-bit codes in nibble order
 * (one stream) and its aux section 10 KB of pack scratch after the table; bq_linear on ABQ
 * with M >= 2 takes an act buffer in its workspace. The buffer version word stays 1 (a BVSR
 * buffer of the earlier layout has 4 streams in its header and is refused).
 * 4: bq_linear on BVSR with M >= 16 also takes an act buffer in its workspace. */
#define BQ_ABI_VERSION 4

const char* bq_status_str(bq_status s);
int32_t bq_version(void);

/* Bytes of the packed buffer for W [N,K] under `desc`. Host only. */
bq_status bq_packed_bytes(const bq_pack_desc* desc, int32_t N, int32_t K, size_t* bytes);

/* Quantize W (device f32 [N][K], row-major, 16-byte aligned) and write the packed buffer
 * (device, >= bq_packed_bytes, 256-byte aligned). The packed buffer also serves as the
 * pack's own scratch before it is overwritten. Weight quantizers (per format): sign with
 * sign(0)=+1 and the residual recursion (RaBiT); alpha*sign(W), alpha = mean|W| (BitNet);
 * T = clamp(rn(W/gamma),-1,1), gamma = mean|W| (ternary); per-row asymmetric codes
 * q = clamp(rn(W/Delta)+z, 0, 2^w-1) (ABQ); exhaustive MSE search over the 256 cached
 * sets (BVSR). `layer` receives the host description. Asynchronous on `stream`. */
bq_status bq_pack_weights(const bq_pack_desc* desc, const float* W, int32_t N, int32_t K,
                          void* packed, size_t packed_bytes, void* stream, bq_layer* layer);

/* Parse and check a HOST copy of a packed buffer's header (e.g. after loading a saved
 * buffer) and fill `layer` with packed_dev as its device pointer. Host only. The header must
 * be exactly what bq_pack_weights writes for its format, N, K (and ABQ w/a bits, ternary
 * rank and alpha): sizes, section offsets, bit widths, fields, shifts and rank as the layout
 * derives them (a ternary rank a multiple of 8, alpha finite); the tensor scale finite and
 * >= 0 for BitNet and ternary, 0 otherwise; the reserved words 32..63 zero. Anything else:
 * BQ_ERR_BAD_PACKED (bytes < 256, a null or unaligned pointer: BQ_ERR_INVALID_ARG). */
bq_status bq_packed_validate(const void* packed_host, size_t bytes, const void* packed_dev,
                             bq_layer* layer);

/* Bytes of the activation buffer for M tokens of `layer`. Host only. */
bq_status bq_act_bytes(const bq_layer* layer, int32_t M, size_t* bytes);

/* Quantize x (device bf16 [M][K] row-major, 16-byte aligned) per token into `act`
 * (device, >= bq_act_bytes, 256-byte aligned): absmax int8 (A8 formats, gamma = max|x|,
 * q = clamp(rn(x*127/gamma), -127, 127)), per-token asymmetric a-bit codes (ABQ),
 * h_p*x in f32 (RaBiT); plus the ternary u = SiLU(xA) and the BVSR group sums. */
bq_status bq_quantize_act(const bq_layer* layer, const void* x_bf16, int32_t M, void* act,
                          size_t act_bytes, void* stream);

/* y [M][N] f32 (device) = the layer applied to the quantized activations in `act`.
 * acc_dbg (nullable, device int64 [M][N]) receives the exact integer accumulator:
 * BitNet/ternary sum_k w q, ABQ sum_k (q_w - z_w)(q_x - z_x), BVSR sum_k code q
 * (not available for RaBiT, whose path is float). bq_gemv is bq_gemm with M = 1. */
bq_status bq_gemv(const bq_layer* layer, const void* act, float* y, int64_t* acc_dbg,
                  void* stream);
bq_status bq_gemm(const bq_layer* layer, const void* act, int32_t M, float* y,
                  int64_t* acc_dbg, void* stream);

/* Fused layer for decode: the activation quantization of bq_quantize_act runs inside the
 * layer kernel's prologue, so y [M][N] f32 comes from x (device bf16 [M][K], 16-byte
 * aligned) in one launch (two for the ternary format with a LoRA term, whose
 * partial dot products of x and A are computed first into `workspace`; and two for ABQ with
 * M >= 2 and BVSR with M >= 16, which quantize the activations once into an act buffer in
 * `workspace` and run the layer from it: ABQ's per-element divides would otherwise be repeated
 * by every CTA, and BVSR's code image holds up to 16 tokens a CTA where the fused staging holds
 * 4 at K = 5120).
 * Results are identical to bq_quantize_act + bq_gemm. `workspace` (device, 256-byte aligned) must hold
 * bq_linear_workspace_bytes(layer, M) bytes; it may be NULL when that is 0.
 * Launched with programmatic dependent launch: consecutive layer calls on one stream
 * overlap the next layer's weight fetch with the current layer. */
bq_status bq_linear_workspace_bytes(const bq_layer* layer, int32_t M, size_t* bytes);
bq_status bq_linear(const bq_layer* layer, const void* x_bf16, int32_t M, float* y, int64_t* acc_dbg,
                    void* workspace, size_t workspace_bytes, void* stream);

/* Several layers that read the same input x, in one launch: e.g. the q, k and v projections
 * of a decoder layer, or its gate and up projections. Each layer keeps its own packed buffer
 * and scales; x is quantized once (as bq_linear does) and every layer's y computed from it.
 * The pages describe one layer at a time; this is that same computation for several weight
 * matrices sharing the input, so that the fixed cost of a launch (waiting for x, quantizing
 * it, the epilogue drain) is paid once.
 *  - layers: host array of n_layers (1..BQ_MAX_GROUP) descriptors, all of one format, K,
 *    w_bits and a_bits. More than one layer is supported for BitNet, ABQ and ternary
 *    without a LoRA term; other formats return BQ_ERR_UNSUPPORTED (use bq_linear).
 *  - y: host array of n_layers device pointers, f32 [M][N_i] each. acc_dbg: NULL, or a host
 *    array of n_layers nullable device int64 [M][N_i] pointers.
 *  - Results equal separate bq_linear calls bit for bit. Same errors as bq_linear, plus
 *    BQ_ERR_INVALID_ARG for mismatched layers. */
#define BQ_MAX_GROUP 4
bq_status bq_linear_group(const bq_layer* layers, int32_t n_layers, const void* x_bf16, int32_t M,
                          float* const* y, int64_t* const* acc_dbg, void* stream);

/* bq_linear with its scratch in a fixed device array inside the library instead of a
 * caller workspace. The pages have no counterpart: this is a calling convenience, not a
 * step of the method. It is for callers that cannot allocate device memory where they
 * run a layer. Examples: a plain C host that owns only the packed layer and its x/y
 * buffers and has no allocator of its own, or a decode loop that must make no allocator
 * call between its buffers being set up and the layer running.
 * Same arguments and results as bq_linear, without workspace and workspace_bytes.
 *  - Scratch limit: BQ_STATIC_SCRATCH_BYTES (1 MiB). A call needing more, that is
 *    bq_linear_workspace_bytes(layer, M) > 1 MiB, returns BQ_ERR_SIZE and enqueues
 *    nothing. Two cases use scratch: the ternary format with a LoRA term, K_pad/256 * M *
 *    rank * 4 bytes (e.g. K = 16384, M = 64, rank = 64 is exactly 1 MiB), and ABQ with
 *    M >= 2 or BVSR with M >= 16, the act buffer of about M * K_pad bytes (e.g. ABQ K = 4096,
 *    M = 64: 263 KiB; BVSR adds M * K_pad / 8 bytes of vector sums).
 *  - Setup: the first call on a device looks up the array's device address
 *    (cudaGetSymbolAddress, with that device current) and keeps it together with the
 *    current context's id; a failure there returns BQ_ERR_CUDA. The address belongs to
 *    that context, so a call under another context (one created after cudaDeviceReset,
 *    or a second context on the same device) looks it up again for that context. Make
 *    the first call on each device, and the first call after any such change of
 *    context, before any stream capture begins.
 *  - Sharing: every call on a device uses the same array. Nothing in it has to start at
 *    zero: each call writes every scratch word before it reads it. Calls on one stream
 *    are ordered and safe; calls whose work overlaps in time (several streams, or
 *    several host threads each with its own stream) race on the array, so the caller
 *    must not overlap them.
 *  - Allocates nothing: no cudaMalloc, cudaFree or allocating library call. */
#define BQ_STATIC_SCRATCH_BYTES (1u << 20)
bq_status bq_linear_static_scratch(const bq_layer* layer, const void* x_bf16, int32_t M, float* y,
                                   int64_t* acc_dbg, void* stream);

/* The work split bq_linear (fused != 0) or bq_gemm (fused = 0) would use for `layer` and M
 * tokens, for inspection and tuning. The pages have no counterpart. Host only: nothing is
 * enqueued. BQ_ERR_UNSUPPORTED if the layer does not fit the tiled kernel, or for RaBiT
 * (not tiled). The SM count is the current device's (148 when no device is visible). */
typedef struct {
  int32_t tokens_per_cta;         /* tokens sharing a CTA's MMA columns (<= 8; BVSR from an act
                                     buffer <= 16, two MMA groups) */
  int32_t token_groups;           /* CTA groups, one per tokens_per_cta tokens */
  int32_t ctas_per_group;         /* persistent CTAs per token group (grid = product) */
  int32_t warps_per_row_block;    /* warps splitting K over one 16-row block (power of two) */
  int32_t tiles_per_warp;         /* 256-k tiles of a row block one warp handles */
  int32_t ring_stages;            /* weight-ring stages per warp */
  int32_t tiles_per_stage;        /* 256-k tiles per ring stage */
  int32_t x_chunks_per_thread;    /* fused staging: 16-byte chunks of x a thread holds
                                     (0: x is read twice; 0 for bq_gemm) */
  uint32_t shared_bytes;          /* dynamic shared memory per CTA */
} bq_plan_info;
bq_status bq_linear_plan(const bq_layer* layer, int32_t M, int32_t fused, bq_plan_info* info);

/* Synchronizes the current device, then reads and clears the device error word:
 * BQ_OK or BQ_ERR_DEVICE_CHECK. */
bq_status bq_device_check(void);

#ifdef __cplusplus
}
#endif

#endif /* BQ_H */
