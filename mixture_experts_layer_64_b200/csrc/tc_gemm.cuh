// Persistent grouped GEMM on the sm_100a tensor cores (tcgen05.mma, fp32
// accumulators in tensor memory, operands staged in shared memory by TMA or
// by a cp.async row gather).
//
// One kernel serves every contraction of the layer:
//   router logits, down-projection, shared FC1, up-projection  (dense)
//   expert FC1 (+ activation) and FC2 (+ gate scale)                (grouped)
// A problem is D[r, f] = sum_k A[src(r), k] B[wrow(g, f), k] with both
// operands K-major (B holds the weights transposed to [out, in]).
//
// Two operand arrangements:
//   token-tiled (kSwap = false): the MMA's M = 128 activation rows, N = the
//     weight tile (128 or 256 features); used when groups hold many rows.
//   weight-stationary (kSwap = true): the MMA's M = 128 weight rows
//     (features), N = the tile's rows rounded up to 16 (tiles of at most 64
//     rows); used at decode sizes, where an expert sees ~16 tokens and the
//     kernel is a stream over the expert weights.
// Gated FC1 (SwiGLU) loads the gate rows f and the linear rows f + m of the
// same feature tile and accumulates them into two TMEM accumulators, so the
// epilogue sees both halves of a feature in one thread.
//
// Warp roles (384 threads; 512 with fp8 weights):
//   warp 0      TMA producer (weights, and contiguous activation rows)
//   warp 1      TMEM allocation and the single-thread MMA issuer
//   warps 2-3   row gather of activations (gathered problems): cp.async
//               copies for token-tiled tiles, completion signalled to the MMA
//               issuer through the mbarrier; four-row TMA gathers (warp 2)
//               for weight-stationary tiles
//   warps 4-11  epilogue, two warpgroups taking alternate 32-column chunks:
//               tcgen05.ld -> epilogue math -> shared-memory staging -> TMA
//               bulk stores (plain stores for partly covered row blocks)
// With fp8 E4M3 weights (512 threads) the epilogue is one warpgroup (warps
// 4-7) and warps 8-15 widen each stage's E4M3 weight tiles to f16 in shared
// memory before the MMA issuer (f16 x f16 -> fp32, the activation rows
// arrive in f16) may use the stage; the per-output-channel scales multiply
// the fp32 accumulators in the epilogue.
// The smem ring has STAGES stages of one 64-wide K slice each; TMEM holds two
// accumulator buffers so the epilogue of tile i overlaps the MMAs of tile i+1.
#pragma once

#include "common.cuh"

namespace lmoe {

constexpr int kTcThreads = 384;
constexpr int kEpiWarps = 8;  // two warpgroups; each warp reads its TMEM lane quarter (warp % 4)
constexpr int kTcSmemBudget = 200 * 1024;
constexpr int kGatherThreads = 64;
#ifndef LMOE_TMEMA_ACC_BUFS
#define LMOE_TMEMA_ACC_BUFS 2
#endif
#ifndef LMOE_TMEMA_STAGES
#define LMOE_TMEMA_STAGES 8
#endif
#ifndef LMOE_TMEMA_S8CAP
#define LMOE_TMEMA_S8CAP 12
#endif

template <bool kSwap_, bool kGather_, bool kDual_, int kWN_, int kEpi_, bool kFp8_ = false,
          int kSwapRows_ = kSwapRowTile, bool kFp4_ = false>
struct TcCfg {
  static constexpr bool kSwap = kSwap_, kGather = kGather_, kDual = kDual_, kFp8 = kFp8_;
  static constexpr int kEpi = kEpi_;
  // weight-stationary tiles: rows per tile (the MMA's N) at most.  Up to 64
  // rows (decode) the gathered rows arrive by four-row TMA gathers; wider
  // tiles (prefill experts with up to a few hundred rows, 128 or 256 rows
  // per tile) gather them with cp.async like the token-tiled kernel.
  static constexpr int kSwapRows = kSwapRows_;
  static constexpr bool kWideSwap = kSwap && kSwapRows > kSwapRowTile;
  // activation rows gathered by cp.async threads (warps 2-3)
  static constexpr bool kCpGather = kGather && (!kSwap || kWideSwap);
  // warps 0-3: producer, MMA issuer, gather; then the epilogue warps (two
  // warpgroups, or one with fp8 weights), then (fp8) the converter warps that
  // widen the E4M3 weight tiles to bf16.  The ungated token-tiled expert FC1
  // (128 x 256 tiles, eight 32-column chunks per TMEM lane quarter) takes
  // three warpgroups, so that a warp drains three chunks of a tile, not
  // four, while the next tile's MMAs run.
  static constexpr int EPI_WARPS = kFp8 ? 4 : (!kSwap && kGather && !kDual) ? 12 : kEpiWarps;
  static constexpr int CONV_THREADS = kFp8 ? 256 : 0;
  static constexpr int THREADS = 128 + 32 * EPI_WARPS + CONV_THREADS;
  // fp8 weights: the MMA runs on f16 operands, so the FC1 output (the FC2
  // input) is written in f16; FC2 writes bf16
  static constexpr bool kF16Out = kFp8 && kEpi_ == EPI_ACT;
  static constexpr int BK = 64;                       // bf16 per 128-byte swizzled row
  static constexpr int ACT_ROWS = kSwap ? kSwapRows : 128;  // activation rows per stage
  static constexpr int W_ROWS = kSwap ? 128 : (kDual ? 128 : kWN_);
  static constexpr int NUM_W = kDual ? 2 : 1;
  static constexpr int ACT_BYTES = ACT_ROWS * BK * 2;
  static constexpr int W_BYTES = W_ROWS * BK * 2;
  // low-precision weights: block-scaled FP4 (kFp4: E2M1 code pairs, 32-byte
  // rows per 64-wide K slice, then the tile's E8M0 exponents, a 16-byte box
  // per row) or fp8 E4M3 (64-byte rows)
  static constexpr bool kFp4 = kFp4_;  // (with kFp8: fp4 reuses the widening paths)
  static constexpr int W4_CODES = kFp4 ? W_ROWS * BK / 2 : 0;  // one fp4 weight tile's codes
  static constexpr int W4_EXPS = kFp4 ? W_ROWS * 16 : 0;       // ... and its exponent box
  static constexpr int W8_BYTES = kFp4 ? W4_CODES + W4_EXPS : kFp8 ? W_ROWS * BK : 0;
  // fp8 weights on weight-stationary tiles (decode): the converter warps
  // widen each E4M3 weight tile into tensor memory, and the MMA takes its A
  // operand (the weights) from there, so the widened tiles cost no shared
  // memory bandwidth; the stage ring holds the activation rows only.
  static constexpr bool kTmemA = kSwap && kFp8;
  static constexpr int STAGE_BYTES = ACT_BYTES + (kTmemA ? 0 : NUM_W * W_BYTES);  // one stage
  // epilogue staging: one 32 x 32 box per epilogue warp (bf16 or fp32)
  static constexpr int STG_WARP = kEpi == EPI_F32_BIAS ? 4096 : 2048;
  static constexpr int STG_BYTES = kSwap ? 0 : EPI_WARPS * STG_WARP;
  static constexpr int BUDGET = kTcSmemBudget + kEpiWarps * 2048 - STG_BYTES;
  static constexpr int STAGES_RAW = BUDGET / STAGE_BYTES;
  // fp8 weights: about 5/9 of the budget as widened stages (at least 3), the
  // rest as a ring of E4M3 slots (one K slice of the NUM_W weight tiles each)
  // that a producer lane fills ahead of the stages
  static constexpr int STAGES_F8 = BUDGET * 5 / 9 / STAGE_BYTES;
  // kTmemA: fp32 accumulators of at most 64 rows (two buffers), then a ring
  // of widened A tiles (64 f16-wide K = 32 columns per weight tile), apart
  // from the deeper ring of activation-row stages in shared memory, so that
  // the rows of a K step are in place before its weights are widened
  static constexpr int A_COLS = kTmemA ? 32 * NUM_W : 0;
  static constexpr int ACC_BUFS = kTmemA ? LMOE_TMEMA_ACC_BUFS : 2;  // accumulator buffers
  static constexpr int STAGES_TA =
      kTmemA ? (512 - ACC_BUFS * kSwapRowTile * NUM_W) / A_COLS : 0;
  static constexpr int STAGES_A = kTmemA ? (STAGES_TA > 8 ? 8 : STAGES_TA) : 1;
  // kTmemA: converter warps per K step (unit).  Gated tiles: all eight
  // (warps 0-3 the gate tile, 4-7 the linear one); ungated tiles: the two
  // groups of four take alternate units, so two units widen at once.
  static constexpr int CONV_PER_UNIT = kTmemA ? (kDual ? 8 : 4) : (kFp8 ? 8 : 0);
  // fp8 / fp4: the weight slot producer has warp 3 to itself where that warp
  // gathers no rows (weight-stationary tiles, and token tiles of contiguous
  // rows), else it shares the producer warp (lane 1)
  static constexpr bool kW8Warp3 = kFp8 && (kTmemA || !kCpGather);
  static constexpr int STAGES = kTmemA ? LMOE_TMEMA_STAGES
                                : kFp8 ? (STAGES_F8 < 3 ? 3 : (STAGES_F8 > 8 ? 8 : STAGES_F8))
                                       : (STAGES_RAW > 12 ? 12 : STAGES_RAW);
  static constexpr int W8_SLOT = NUM_W * W8_BYTES;
  static constexpr int S8_RAW = kFp8 ? (BUDGET - STAGES * STAGE_BYTES) / W8_SLOT : 0;  // E4M3 slots
  static constexpr int S8_CAP = kTmemA ? LMOE_TMEMA_S8CAP : 16;
  static constexpr int S8 = S8_RAW > S8_CAP ? S8_CAP : S8_RAW;
  static constexpr int RING_BYTES = STAGES * STAGE_BYTES + S8 * W8_SLOT;
  static constexpr int ACC_N = kTmemA ? kSwapRowTile
                              : kSwap ? (kSwapRows > 128 ? kSwapRows : 128) : W_ROWS;  // fp32 columns of one accumulator
  static constexpr int ACC_COLS = ACC_N * NUM_W;      // one TMEM buffer
  static constexpr int TMEM_COLS = kTmemA ? 512 : 2 * ACC_COLS;  // double buffered (+ A stages)
  static constexpr int A_COL0 = ACC_BUFS * ACC_COLS;  // kTmemA: first column of the A stages
  static constexpr int FT = W_ROWS;                   // features per tile
  static constexpr int TABLE_BYTES = 2 * (LMOE_MAX_EXPERTS + 1) * 4;  // tile_prefix, offsets
  static constexpr int SMEM_BYTES = 1024 /*align slack*/ + RING_BYTES + STG_BYTES + 512 +
                                    TABLE_BYTES;
  static_assert(TMEM_COLS == 256 || TMEM_COLS == 512, "TMEM allocation must be a power of two");
  static_assert(!kTmemA || A_COL0 + STAGES_A * A_COLS <= 512, "tensor memory: A stages");
  static_assert(SMEM_BYTES <= 227 * 1024, "shared memory");
  static_assert(STAGES >= 3, "pipeline too shallow");
  static_assert(!kFp8 || S8 >= 2, "fp8 weight ring too shallow");
  static_assert(!kTmemA || (S8 >= 2 && STAGES_A >= 2), "tensor-memory A rings too shallow");
  static_assert(ACC_BUFS == 1 || ACC_BUFS == 2, "accumulator buffers");
  static_assert(2 * STAGES * 8 + 2 * S8 * 8 + (kTmemA ? 2 * STAGES_A * 8 : 0) + 6 * 8 + 16 <= 512,
                "barrier area");
  static_assert(!kSwap || kEpi == EPI_ACT || kEpi == EPI_SCALE_ROWS, "swap epilogues");
  static_assert(kWN_ == 128 || kWN_ == 256, "weight tile");
  static_assert(!kFp8 || kEpi == EPI_ACT || kEpi == EPI_SCALE_ROWS, "fp8 weights: expert GEMMs");
  static_assert(kSwapRows == kSwapRowTile || kSwapRows == 128 || kSwapRows == 256, "swap rows");
  static_assert(!kWideSwap || !kFp8, "wide weight-stationary tiles: bf16 weights");
  static_assert(!kFp4 || kFp8, "fp4 weights: the widening (fp8) kernel paths");
};

// ---- fp8 E4M3 weights -----------------------------------------------------------
//
// The expert kernels with fp8 weights run the MMA on f16 operands: an E4M3
// code widens to f16 in one hardware conversion per pair, and the activation
// rows arrive in f16 (the layer converts the FC1 input once per forward, and
// FC1 writes its output in f16).

// Four E4M3 codes (byte 0 first) -> four f16 with the same values, as two
// f16x2 words: one exact hardware conversion per pair (every E4M3 value,
// subnormals included, is a normal f16 or zero).
__device__ __forceinline__ void e4m3x4_to_f16x4(uint32_t w, uint32_t& lo, uint32_t& hi) {
  asm("{\n\t.reg .b16 l, h;\n\t"
      "mov.b32 {l, h}, %2;\n\t"
      "cvt.rn.f16x2.e4m3x2 %0, l;\n\t"
      "cvt.rn.f16x2.e4m3x2 %1, h;\n\t}"
      : "=r"(lo), "=r"(hi)
      : "r"(w));
}

// Widens one weight tile: W_ROWS rows of 64 E4M3 codes (64-byte rows, no
// swizzle, as TMA stored them) into W_ROWS rows of 64 f16 in the 128-byte
// swizzled K-major layout the MMA reads.  ct = this thread's index among the
// kConv converter threads; chunk c = (row, 16-byte quarter q) is handled by
// thread c mod kConv.
template <int W_ROWS, int kConv>
__device__ __forceinline__ void widen_fp8_tile(const uint8_t* src, uint8_t* dst, int ct) {
#pragma unroll
  for (int c = ct; c < W_ROWS * 4; c += kConv) {
    const int r = c >> 2, q = c & 3;
    const uint4 v = *reinterpret_cast<const uint4*>(src + r * 64 + q * 16);
    const uint32_t in[4] = {v.x, v.y, v.z, v.w};
    uint32_t out[8];
#pragma unroll
    for (int i = 0; i < 4; ++i) e4m3x4_to_f16x4(in[i], out[2 * i], out[2 * i + 1]);
    uint8_t* row = dst + r * 128;
    const int sw = r & 7;
    *reinterpret_cast<uint4*>(row + (((2 * q) ^ sw) << 4)) = make_uint4(out[0], out[1], out[2], out[3]);
    *reinterpret_cast<uint4*>(row + (((2 * q + 1) ^ sw) << 4)) =
        make_uint4(out[4], out[5], out[6], out[7]);
  }
}

// Widens row r of an E4M3 weight tile (64-byte rows of 64 codes, stored by
// TMA with the 64-byte swizzle: 16-byte chunk c of row r sits at chunk
// c ^ ((r >> 1) & 3)) into 32 words of f16 pairs, K ascending (element 2i in
// the low half of word i).  With the swizzle a warp's 32 consecutive rows
// read all 32 banks evenly.
__device__ __forceinline__ void widen_fp8_row_sw64(const uint8_t* tile, int r,
                                                   uint32_t (&out)[32]) {
  const int x = (r >> 1) & 3;
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    const uint4 v = *reinterpret_cast<const uint4*>(tile + r * 64 + ((c ^ x) << 4));
    e4m3x4_to_f16x4(v.x, out[8 * c + 0], out[8 * c + 1]);
    e4m3x4_to_f16x4(v.y, out[8 * c + 2], out[8 * c + 3]);
    e4m3x4_to_f16x4(v.z, out[8 * c + 4], out[8 * c + 5]);
    e4m3x4_to_f16x4(v.w, out[8 * c + 6], out[8 * c + 7]);
  }
}

// 2^e as an f16, for e in [-24, 15], built from the binary16 encoding: a
// normal number (biased exponent e + 15, zero mantissa) for e >= -14, else
// the subnormal with the single mantissa bit e + 24.
__device__ __forceinline__ __half pow2_half(int e) {
  const unsigned short bits =
      e >= -14 ? (unsigned short)((e + 15) << 10) : (unsigned short)(1u << (e + 24));
  return __ushort_as_half(bits);
}

// Eight E2M1 codes (four bytes, the low nibble of each byte first) as four
// words of f16 pairs, each exact (cvt.rn.f16x2.e2m1x2) and then scaled by
// the block's power of two sc (an exact f16 multiply: the exponents are
// limited so that every product is an f16 value).
__device__ __forceinline__ void e2m1x8_to_f16x8(uint32_t codes, __half2 sc, uint32_t* out) {
  uint32_t w0, w1, w2, w3;
  asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
      "mov.b32 {b0, b1, b2, b3}, %4;\n\t"
      "cvt.rn.f16x2.e2m1x2 %0, b0;\n\t"
      "cvt.rn.f16x2.e2m1x2 %1, b1;\n\t"
      "cvt.rn.f16x2.e2m1x2 %2, b2;\n\t"
      "cvt.rn.f16x2.e2m1x2 %3, b3;\n\t}"
      : "=r"(w0), "=r"(w1), "=r"(w2), "=r"(w3)
      : "r"(codes));
  const uint32_t ws[4] = {w0, w1, w2, w3};
#pragma unroll
  for (int b = 0; b < 4; ++b) {
    __half2 h = *reinterpret_cast<const __half2*>(&ws[b]);
    h = __hmul2(h, sc);
    out[b] = *reinterpret_cast<const uint32_t*>(&h);
  }
}

// Widens row r of an MXFP4 weight tile for one 64-wide K slice: 32 bytes of
// E2M1 code pairs (TMA-stored with the 32-byte swizzle: 16-byte chunk c of
// row r sits at chunk c ^ ((r >> 2) & 1)) and the row's two E8M0 block
// exponents, at byte `eoff` of its 16-byte exponent row.  Output as
// widen_fp8_row_sw64: 32 words of f16 pairs, K ascending.
__device__ __forceinline__ void widen_fp4_row_sw32(const uint8_t* codes, const uint8_t* exps, int r,
                                                   int eoff, uint32_t (&out)[32]) {
  const int x = (r >> 2) & 1;
#pragma unroll
  for (int c = 0; c < 2; ++c) {  // chunk c: K elements 32c .. 32c + 31, block c
    const uint4 v = *reinterpret_cast<const uint4*>(codes + r * 32 + ((c ^ x) << 4));
    const __half2 sc = __half2half2(pow2_half((int)exps[r * 16 + eoff + c] - 127));
    e2m1x8_to_f16x8(v.x, sc, &out[16 * c + 0]);
    e2m1x8_to_f16x8(v.y, sc, &out[16 * c + 4]);
    e2m1x8_to_f16x8(v.z, sc, &out[16 * c + 8]);
    e2m1x8_to_f16x8(v.w, sc, &out[16 * c + 12]);
  }
}

// Widens an MXFP4 weight tile (W_ROWS rows of 32 code bytes, unswizzled, and
// a 16-byte exponent row each) for one 64-wide K slice to f16 in the
// 128-byte-swizzled K-major layout of a stage, by kConv converter threads:
// chunk c = (row, 32-element block h) is handled by thread c mod kConv and
// writes the block's four 16-byte chunks.
template <int W_ROWS, int kConv>
__device__ __forceinline__ void widen_fp4_tile(const uint8_t* codes, const uint8_t* exps, int eoff,
                                               uint8_t* dst, int ct) {
#pragma unroll
  for (int c = ct; c < W_ROWS * 2; c += kConv) {
    const int r = c >> 1, hb = c & 1;
    const uint4 v = *reinterpret_cast<const uint4*>(codes + r * 32 + hb * 16);
    const __half2 sc = __half2half2(pow2_half((int)exps[r * 16 + eoff + hb] - 127));
    uint32_t out[16];
    e2m1x8_to_f16x8(v.x, sc, &out[0]);
    e2m1x8_to_f16x8(v.y, sc, &out[4]);
    e2m1x8_to_f16x8(v.z, sc, &out[8]);
    e2m1x8_to_f16x8(v.w, sc, &out[12]);
    uint8_t* row = dst + r * 128;
    const int sw = r & 7;
#pragma unroll
    for (int i = 0; i < 4; ++i)
      *reinterpret_cast<uint4*>(row + (((4 * hb + i) ^ sw) << 4)) =
          make_uint4(out[4 * i], out[4 * i + 1], out[4 * i + 2], out[4 * i + 3]);
  }
}

// ---- epilogue stores ----------------------------------------------------------

// The 16-bit output value of v: bf16, or (kF16) the bits of the f16 value in
// the same storage type -- the expert FC1 of a layer with fp8 weights writes
// its hidden rows in f16, the operand type of its FC2.
template <bool kF16>
__device__ __forceinline__ bf16 round_out(float v) {
  if constexpr (kF16) return __ushort_as_bfloat16(__half_as_ushort(__float2half_rn(v)));
  else return __float2bfloat16_rn(v);
}

// One row (token-tiled mode): 32 consecutive features [f, f+32) of row `row`.
template <int kEpi, bool kGated, bool kF16 = false>
__device__ __forceinline__ void store_row32(const GemmProblem& p, int row, int f,
                                            const float (&v0)[32], const float (&v1)[32],
                                            size_t slice_off = 0) {
  const EpiParams& e = p.epi;
  const bool full = f + 32 <= p.F;
  if (kEpi == EPI_F32_BIAS) {
    float* o = static_cast<float*>(e.out) + slice_off + (size_t)row * e.ldo + f;
    if (full) {
#pragma unroll
      for (int i = 0; i < 32; i += 4) {
        float4 q;
        q.x = v0[i] + (e.bias ? __ldg(e.bias + f + i) : 0.f);
        q.y = v0[i + 1] + (e.bias ? __ldg(e.bias + f + i + 1) : 0.f);
        q.z = v0[i + 2] + (e.bias ? __ldg(e.bias + f + i + 2) : 0.f);
        q.w = v0[i + 3] + (e.bias ? __ldg(e.bias + f + i + 3) : 0.f);
        *reinterpret_cast<float4*>(o + i) = q;
      }
    } else {
#pragma unroll
      for (int i = 0; i < 32; ++i)
        if (f + i < p.F) o[i] = v0[i] + (e.bias ? e.bias[f + i] : 0.f);
    }
    return;
  }
  float r[32];
  const bf16* res = nullptr;
  size_t orow = (size_t)row;
  if (kEpi == EPI_ACT) {
#pragma unroll
    for (int i = 0; i < 32; ++i) r[i] = apply_act(e.act, v0[i], kGated ? v1[i] : 0.f);
  } else if (kEpi == EPI_SCALE_ROWS) {
    const float s = __ldg(e.row_w + row);
#pragma unroll
    for (int i = 0; i < 32; ++i) r[i] = v0[i] * s;
  } else {  // EPI_RESID
    res = static_cast<const bf16*>(e.resid) + (size_t)row * e.ldr + f;
  }
  bf16* o = static_cast<bf16*>(e.out) + orow * e.ldo + (kEpi == EPI_ACT ? e.col0 : 0) + f;
  const int split = (kEpi == EPI_ACT) ? e.split_off : 0;
  if (full) {
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const int i = 8 * c;
      if (kEpi == EPI_RESID) {
        const uint4 rv = *reinterpret_cast<const uint4*>(res + i);
        const bf16* rb = reinterpret_cast<const bf16*>(&rv);
#pragma unroll
        for (int j = 0; j < 8; ++j) r[i + j] = __bfloat162float(rb[j]) + v0[i + j];
      }
      uint4 q, ql;
      bf16* qb = reinterpret_cast<bf16*>(&q);
      bf16* qlb = reinterpret_cast<bf16*>(&ql);
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        qb[j] = round_out<kF16>(r[i + j]);
        if (!kF16) qlb[j] = __float2bfloat16_rn(r[i + j] - __bfloat162float(qb[j]));
      }
      *reinterpret_cast<uint4*>(o + i) = q;
      if (!kF16 && split) *reinterpret_cast<uint4*>(o + split + i) = ql;
    }
  } else {
    // ragged last chunk (F not a multiple of 32): element stores, fully
    // unrolled so that r and v0 stay in registers
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      if (f + i < p.F) {
        float v = (kEpi == EPI_RESID) ? __bfloat162float(res[i]) + v0[i] : r[i];
        const bf16 hi = round_out<kF16>(v);
        o[i] = hi;
        if (!kF16 && split) o[split + i] = __float2bfloat16_rn(v - __bfloat162float(hi));
      }
    }
  }
}

// One element (weight-stationary mode): feature f of row `row`.
template <int kEpi, bool kF16 = false>
__device__ __forceinline__ void store_elem(const GemmProblem& p, int row, int f, float v0, float v1) {
  const EpiParams& e = p.epi;
  if (kEpi == EPI_ACT) {
    const float v = apply_act(e.act, v0, v1);
    const bf16 hi = round_out<kF16>(v);
    bf16* o = static_cast<bf16*>(e.out) + (size_t)row * e.ldo + e.col0 + f;
    o[0] = hi;
    if (!kF16 && e.split_off) o[e.split_off] = __float2bfloat16_rn(v - __bfloat162float(hi));
  } else {  // EPI_SCALE_ROWS
    static_cast<bf16*>(e.out)[(size_t)row * e.ldo + f] =
        __float2bfloat16_rn(v0 * __ldg(e.row_w + row));
  }
}

// ---- epilogue through shared memory and TMA stores ------------------------------
//
// A TMEM row belongs to one thread, so plain global stores from registers put
// 32 rows into every store instruction, 16 bytes each: half of a 32-byte
// sector per row per instruction, which the memory system completes with
// read-modify-writes.  Instead each epilogue warp stages its 32 rows x 32
// bf16 columns in shared memory (64-byte rows with the 64-byte swizzle, which
// keeps the row-per-thread writes free of bank conflicts) and one lane writes
// the box with a bulk tensor store.  Blocks of 32 rows that a tile only partly
// covers, and the fp32 router logits, use the plain stores.
template <int kEpi, bool kGated, bool kF16>
__device__ __forceinline__ void epi_tma_chunk32_impl(const GemmProblem& p, const CUtensorMap* tmC,
                                                uint8_t* stg, int lane, int row_base, int f,
                                                const float (&v0)[32], const float (&v1)[32]) {
  const EpiParams& e = p.epi;
  const int row = row_base + lane;
  float r[32];
  if (kEpi == EPI_ACT) {
#pragma unroll
    for (int i = 0; i < 32; ++i) r[i] = apply_act(e.act, v0[i], kGated ? v1[i] : 0.f);
  } else if (kEpi == EPI_SCALE_ROWS) {
    const float sc = __ldg(e.row_w + row);
#pragma unroll
    for (int i = 0; i < 32; ++i) r[i] = v0[i] * sc;
  } else if (kEpi == EPI_RESID) {
    const bf16* rrow = static_cast<const bf16*>(e.resid) + (size_t)row * e.ldr + f;
    if (f + 32 <= p.F) {
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const uint4 rv = reinterpret_cast<const uint4*>(rrow)[c];
        const bf16* rb = reinterpret_cast<const bf16*>(&rv);
#pragma unroll
        for (int j = 0; j < 8; ++j) r[8 * c + j] = __bfloat162float(rb[j]) + v0[8 * c + j];
      }
    } else {
#pragma unroll
      for (int i = 0; i < 32; ++i) r[i] = (f + i < p.F) ? __bfloat162float(rrow[i]) + v0[i] : 0.f;
    }
  }
  if (lane == 0) bulk_wait_read0();  // the previous box has left the buffer
  __syncwarp();
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    uint4 q;
    bf16* qb = reinterpret_cast<bf16*>(&q);
#pragma unroll
    for (int j = 0; j < 8; ++j) qb[j] = round_out<kF16>(r[8 * c + j]);
    *reinterpret_cast<uint4*>(stg + lane * 64 + ((c ^ ((lane >> 1) & 3)) << 4)) = q;
  }
  fence_proxy_async_smem();
  __syncwarp();
  if (lane == 0) {
    tma_store_2d(tmC, stg, f, row_base);
    bulk_commit();
  }
}

// fp32 output (router logits, split-K partial sums): 32 rows x 32 floats,
// 128-byte rows staged with the 128-byte swizzle (16-byte chunk c of row r at
// r * 128 + ((c ^ (r & 7)) << 4)).
__device__ __forceinline__ void epi_tma_chunk32_f32(const GemmProblem& p, const CUtensorMap* tmC,
                                                    uint8_t* stg, int lane, int row_base, int f,
                                                    const float (&v0)[32]) {
  const float* b = p.epi.bias;
  if (lane == 0) bulk_wait_read0();  // the previous box has left the buffer
  __syncwarp();
#pragma unroll
  for (int c = 0; c < 8; ++c) {
    float4 q;
    float* qf = reinterpret_cast<float*>(&q);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int i = 4 * c + j;
      qf[j] = v0[i] + ((b && f + i < p.F) ? __ldg(b + f + i) : 0.f);
    }
    *reinterpret_cast<float4*>(stg + lane * 128 + ((c ^ (lane & 7)) << 4)) = q;
  }
  fence_proxy_async_smem();
  __syncwarp();
  if (lane == 0) {
    tma_store_2d(tmC, stg, f, row_base);
    bulk_commit();
  }
}

template <int kEpi, bool kGated, bool kF16 = false>
__device__ __forceinline__ void epi_tma_chunk32(const GemmProblem& p, const CUtensorMap* tmC,
                                                uint8_t* stg, int lane, int row_base, int f,
                                                const float (&v0)[32], const float (&v1)[32]) {
  if constexpr (kEpi == EPI_F32_BIAS)
    epi_tma_chunk32_f32(p, tmC, stg, lane, row_base, f, v0);
  else
    epi_tma_chunk32_impl<kEpi, kGated, kF16>(p, tmC, stg, lane, row_base, f, v0, v1);
}

// ---- tile lookup from shared memory -----------------------------------------------
//
// Every role of a persistent CTA maps its next tile index to (group, first
// row, rows) with a binary search over the groups' tile counts.  Done on
// global memory that is ~10 dependent loads at every tile boundary, longer
// than the pipeline hides, so the grouped kernels first copy tile_prefix and
// offsets (G + 1 entries each) into shared memory.
__device__ __forceinline__ void load_tile_tables(const GemmProblem& p, int* s_tiles) {
  if (p.offsets == nullptr) return;
  for (int i = threadIdx.x; i <= p.G; i += blockDim.x) {
    s_tiles[i] = p.tile_prefix[i];
    s_tiles[LMOE_MAX_EXPERTS + 1 + i] = p.offsets[i];
  }
}

__device__ __forceinline__ void locate_row_tile_s(const GemmProblem& p, const int* s_tiles, int rt,
                                                  int& g, int& row0, int& rows) {
  if (p.offsets == nullptr) {
    g = 0;
    row0 = rt * p.row_tile;
    rows = min(p.row_tile, p.M - row0);
    return;
  }
  const int* tp = s_tiles;
  const int* off = s_tiles + LMOE_MAX_EXPERTS + 1;
  int lo = 0, hi = p.G - 1;  // largest g with tp[g] <= rt
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (tp[mid] <= rt) lo = mid; else hi = mid - 1;
  }
  g = lo;
  // (rem_of: only the group's last rows % rem_of rows)
  const int start = p.rem_of > 0 ? off[g + 1] - (off[g + 1] - off[g]) % p.rem_of : off[g];
  row0 = start + (rt - tp[g]) * p.row_tile;
  rows = min(p.row_tile, off[g + 1] - row0);
}

__device__ __forceinline__ int total_row_tiles_s(const GemmProblem& p, const int* s_tiles) {
  if (p.offsets == nullptr) return (p.M + p.row_tile - 1) / p.row_tile;
  return s_tiles[p.G];
}

// ---- the work of one CTA ---------------------------------------------------------
//
// Tile-granular: tiles blockIdx.x, blockIdx.x + gridDim.x, ...; with split-K
// tile t covers the K blocks of split t / tiles_per_split.
// Stream-K (weight-stationary decode GEMMs, p.stream_k, and at least two
// tiles per CTA): the (tile, K block) units are dealt out in equal
// contiguous ranges, one per CTA, so that the weight stream ends on every SM
// at the same time instead of in a last partial wave of whole tiles.  A
// tile whose K blocks straddle two ranges is computed in two parts: the
// "head" (its first K blocks, at the end of one CTA's range) and the "tail"
// (the rest, at the start of the next CTA's range).  Each part writes its
// fp32 accumulator to a slot; whichever arrives second adds the other's part
// and runs the epilogue.  Two fp32 terms add the same in either order, so the
// result does not depend on which part finishes first, and no CTA waits for
// another.
struct TileWalk {
  int num_tiles, tiles_per_split, KB, KBS;
  long u_end;  // stream-K: end of this CTA's unit range; -1: tile-granular
};

__device__ __forceinline__ long walk_start(const TileWalk& w) {
  if (w.u_end < 0) return blockIdx.x;
  const long total = (long)w.num_tiles * w.KB;
  const long per = (total + gridDim.x - 1) / gridDim.x;
  return min(total, (long)blockIdx.x * per);
}

// The next segment: tile tl (row tile * NT + feature tile), split ks, K
// blocks [kb0, kb1).
__device__ __forceinline__ bool walk_next(const TileWalk& w, long& it, int& tl, int& ks, int& kb0,
                                          int& kb1) {
  if (w.u_end >= 0) {
    if (it >= w.u_end) return false;
    tl = (int)(it / w.KB);
    kb0 = (int)(it - (long)tl * w.KB);
    kb1 = (int)min((long)w.KB, (long)kb0 + (w.u_end - it));
    ks = 0;
    it += kb1 - kb0;
    return true;
  }
  if (it >= w.num_tiles) return false;
  const int t = (int)it;
  ks = t / w.tiles_per_split;
  tl = t - ks * w.tiles_per_split;
  kb0 = ks * w.KBS;
  kb1 = min(w.KB, kb0 + w.KBS);
  it += gridDim.x;
  return true;
}

// ---- the kernel -----------------------------------------------------------------

template <class Cfg>
__global__ void __launch_bounds__(Cfg::THREADS, 1)
    tc_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                   const __grid_constant__ CUtensorMap tmC, const GemmProblem p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* stg_base = smem + Cfg::RING_BYTES;  // epilogue staging (1024-aligned)
  uint8_t* w8_ring = smem + Cfg::STAGES * Cfg::STAGE_BYTES;  // fp8 weights: E4M3 slots
  uint64_t* full = reinterpret_cast<uint64_t*>(stg_base + Cfg::STG_BYTES);
  uint64_t* empty = full + Cfg::STAGES;
  uint64_t* w8full = empty + Cfg::STAGES;  // fp8: an E4M3 slot has landed
  uint64_t* w8empty = w8full + Cfg::S8;    // fp8: an E4M3 slot has been widened
  uint64_t* afull = w8empty + Cfg::S8;     // kTmemA: an A stage has been widened
  uint64_t* aempty = afull + (Cfg::kTmemA ? Cfg::STAGES_A : 0);  // kTmemA: its MMAs are done
  uint64_t* tfull = aempty + (Cfg::kTmemA ? Cfg::STAGES_A : 0);
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint64_t* epibar = drain + 1;  // stream-K: the epilogue warps meet here
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(epibar + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  volatile int* sk_order = reinterpret_cast<volatile int*>(tmem_slot + 2);  // stream-K
  int* s_tiles = reinterpret_cast<int*>(stg_base + Cfg::STG_BYTES + 512);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  griddep_launch();
  const int NT = (p.F + Cfg::FT - 1) / Cfg::FT;
  const int KB = p.K / Cfg::BK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < Cfg::STAGES; ++s) {
      // the producer (its expect_tx covers the weights and the activation
      // rows, including TMA-gathered ones) + the cp.async gather threads of
      // token-tiled tiles + (fp8) one lane per converter warp
      mbar_init(&full[s], 1 + (Cfg::kCpGather ? kGatherThreads : 0) +
                              (Cfg::kTmemA ? 0 : Cfg::CONV_THREADS / 32));
      mbar_init(&empty[s], 1);
    }
    if (Cfg::kTmemA) {
      for (int a = 0; a < Cfg::STAGES_A; ++a) {
        mbar_init(&afull[a], Cfg::CONV_PER_UNIT);
        mbar_init(&aempty[a], 1);
      }
    }
    for (int j = 0; j < Cfg::S8; ++j) {
      mbar_init(&w8full[j], 1);
      mbar_init(&w8empty[j], Cfg::CONV_PER_UNIT);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], Cfg::EPI_WARPS);
    }
    mbar_init(drain, 1);
    mbar_init(epibar, Cfg::EPI_WARPS);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    if (!Cfg::kGather) prefetch_tensormap(&tmA);
    prefetch_tensormap(&tmB);
    if (Cfg::kFp4) prefetch_tensormap(&tmC);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, Cfg::TMEM_COLS);
    tmem_relinquish();
    tc_fence_before();
  }
  griddep_wait();  // the previous kernel's outputs (tile tables, activations)
  load_tile_tables(p, s_tiles);
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  // Split-K (dense problems): tile t covers K blocks [kb0, kb1) of split
  // t / tiles_per_split and writes an fp32 slice of partial sums.
  const int S = p.splits > 1 ? p.splits : 1;
  const int KBS = S > 1 ? p.kb_per_split : KB;
  const int tiles_per_split = total_row_tiles_s(p, s_tiles) * NT;
  const int num_tiles = tiles_per_split * S;
  TileWalk walk{num_tiles, tiles_per_split, KB, KBS, -1};
  // stream-K only with few waves of tiles (2 to 16 per CTA): with more, the
  // last partial wave is a small share and the contiguous per-CTA ranges
  // (each SM on its own stretch of weights) measured slower than all SMs
  // sweeping consecutive tiles together
  if (Cfg::kSwap && !Cfg::kWideSwap && p.stream_k && S == 1 && num_tiles >= 2 * (int)gridDim.x &&
      num_tiles < 16 * (int)gridDim.x) {
    const long total = (long)num_tiles * KB;
    const long per = (total + gridDim.x - 1) / gridDim.x;
    walk.u_end = min(total, (long)(blockIdx.x + 1) * per);
  }

  // The fp8 / fp4 weight slot producer: walks the (tile, K block) sequence on
  // its own and keeps the slot ring loading, limited only by the converters.
  // It runs alone in warp 3 where that warp has no other work (kW8Warp3),
  // else in lane 1 of the producer warp.
  const auto w8_producer = [&]() {
    int j = 0;
    uint32_t jph = 0;
    long wissued = 0;
    bool ok = true;
    int tl, ks, kb0, kb1;
    for (long wi = walk_start(walk); ok && walk_next(walk, wi, tl, ks, kb0, kb1);) {
      const int rt = tl / NT, ft = tl - (tl / NT) * NT;
      int g, row0, rows;
      locate_row_tile_s(p, s_tiles, rt, g, row0, rows);
      const int wrow = (int)(g * p.w_group_stride) + ft * Cfg::FT;
      for (int kb = kb0; kb < kb1; ++kb) {
        if (!mbar_wait(&w8empty[j], jph ^ 1, abort_flag, p.err)) { ok = false; break; }
        uint8_t* slot = w8_ring + j * Cfg::W8_SLOT;
        mbar_arrive_expect_tx(&w8full[j], Cfg::W8_SLOT);
        if (Cfg::kFp4) {
          // code pairs (32 bytes per row of the K slice), then the exponent
          // box holding this slice's two exponents (16-byte aligned start;
          // tmC is the exponent map in the weight-stationary kernels)
          const int ex = (kb * 2) & ~15;
          tma_load_2d(&tmB, &w8full[j], slot, kb * (Cfg::BK / 2), wrow);
          tma_load_2d(&tmC, &w8full[j], slot + Cfg::W4_CODES, ex, wrow);
          if (Cfg::kDual) {
            tma_load_2d(&tmB, &w8full[j], slot + Cfg::W8_BYTES, kb * (Cfg::BK / 2),
                        wrow + p.dual_offset);
            tma_load_2d(&tmC, &w8full[j], slot + Cfg::W8_BYTES + Cfg::W4_CODES, ex,
                        wrow + p.dual_offset);
          }
        } else {
          tma_load_2d(&tmB, &w8full[j], slot, kb * Cfg::BK, wrow);
          if (Cfg::kDual)
            tma_load_2d(&tmB, &w8full[j], slot + Cfg::W8_BYTES, kb * Cfg::BK,
                        wrow + p.dual_offset);
        }
        ++wissued;
        if (++j == Cfg::S8) { j = 0; jph ^= 1; }
      }
    }
    if (*abort_flag) {
      // let the loads in flight land before the block frees its shared memory
      for (long i = 0; i < wissued && i < Cfg::S8; ++i) {
        if (j == 0) { j = Cfg::S8; jph ^= 1; }
        --j;
        mbar_wait_drain(&w8full[j], jph);
      }
    }
  };
  if (Cfg::kW8Warp3 && warp == 3) {
    if (lane == 0) w8_producer();
  } else if (warp == 0) {
    // ---------------- TMA producer ----------------
    // Lane 0 arms the stages (activation rows, and bf16 weights); with fp8
    // weights on token tiles of gathered rows lane 1 runs the weight slot
    // producer.
    if (Cfg::kFp8 && !Cfg::kW8Warp3 && lane == 1) w8_producer();
    if (lane == 0) {
      int s = 0;
      uint32_t ph = 0;
      long armed = 0;
      int tl, ks, kb0, kb1;
      for (long wi = walk_start(walk); walk_next(walk, wi, tl, ks, kb0, kb1);) {
        const int rt = tl / NT, ft = tl - (tl / NT) * NT;
        int g, row0, rows;
        locate_row_tile_s(p, s_tiles, rt, g, row0, rows);
        const int wrow = (int)(g * p.w_group_stride) + ft * Cfg::FT;
        const int nsub = Cfg::kSwap ? (rows + 31) / 32 : 4;
        uint32_t bytes = Cfg::kFp8 ? 0u : (uint32_t)(Cfg::NUM_W * Cfg::W_BYTES);
        if (!Cfg::kGather) bytes += Cfg::kSwap ? nsub * 4096 : Cfg::ACT_BYTES;
        else if (!Cfg::kCpGather) bytes += max(16, (rows + 15) & ~15) * 128;  // TMA-gathered rows
        bool ok = true;
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait(&empty[s], ph ^ 1, abort_flag, p.err)) { ok = false; break; }
          uint8_t* st = smem + s * Cfg::STAGE_BYTES;
          uint64_t* abar = &full[s];
          mbar_arrive_expect_tx(abar, bytes);
          ++armed;
          if (!Cfg::kFp8) {
            tma_load_2d(&tmB, &full[s], st + Cfg::ACT_BYTES, kb * Cfg::BK, wrow);
            if (Cfg::kDual)
              tma_load_2d(&tmB, &full[s], st + Cfg::ACT_BYTES + Cfg::W_BYTES, kb * Cfg::BK,
                          wrow + p.dual_offset);
          }
          if (!Cfg::kGather) {
            if (Cfg::kSwap) {
              for (int sub = 0; sub < nsub; ++sub)
                tma_load_2d(&tmA, abar, st + sub * 4096, kb * Cfg::BK, row0 + sub * 32);
            } else {
              tma_load_2d(&tmA, abar, st, kb * Cfg::BK, row0);
            }
          }
          if (++s == Cfg::STAGES) { s = 0; ph ^= 1; }
        }
        if (!ok) break;
      }
      if (*abort_flag) {
        // Let every armed load land before the block frees its shared memory.
        int ss = s;
        uint32_t pp = ph;
        for (long i = 0; i < armed && i < Cfg::STAGES; ++i) {
          if (ss == 0) { ss = Cfg::STAGES; pp ^= 1; }
          --ss;
          // (with fp8 weights full may stay short of the converters'
          // arrivals; the bounded wait absorbs that)
          mbar_wait_drain(&full[ss], pp);
        }
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      int s = 0, sa = 0;  // activation stage, (kTmemA) A stage
      uint32_t ph = 0, pha = 0;
      int it = 0;
      int tl, ks, kb0, kb1;
      for (long wi = walk_start(walk); walk_next(walk, wi, tl, ks, kb0, kb1); ++it) {
        const int rt = tl / NT;
        int g, row0, rows;
        locate_row_tile_s(p, s_tiles, rt, g, row0, rows);
        const int ab = Cfg::ACC_BUFS == 2 ? (it & 1) : 0;
        const uint32_t aph = Cfg::ACC_BUFS == 2 ? (uint32_t)(it >> 1) & 1 : (uint32_t)it & 1;
        if (!mbar_wait(&tempty[ab], aph ^ 1, abort_flag, p.err)) break;
        tc_fence_after();
        const uint32_t d0 = tmem_base + ab * Cfg::ACC_COLS;
        const uint32_t d1 = d0 + Cfg::ACC_N;
        // Token-tiled gated tiles: the gate and linear weight tiles sit back to
        // back in shared memory (rows 0-127 and 128-255 of one 256-row B
        // operand) and their accumulators back to back in TMEM, so one N = 256
        // MMA computes both and reads the activation tile once.
        int n = Cfg::kDual ? 2 * Cfg::ACC_N : Cfg::ACC_N;
        if (Cfg::kSwap) n = max(16, (rows + 15) & ~15);
        // fp8 weights: both operands were widened to f16
        const uint32_t idesc = Cfg::kFp8 ? idesc_f16_f32(128, n) : idesc_bf16_f32(128, n);
        bool ok = true;
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait(&full[s], ph, abort_flag, p.err)) { ok = false; break; }
          if (Cfg::kTmemA && !mbar_wait(&afull[sa], pha, abort_flag, p.err)) { ok = false; break; }
          tc_fence_after();
          const uint8_t* st = smem + s * Cfg::STAGE_BYTES;
          const uint64_t da = smem_desc_sw128(st);
          const uint64_t dw0 = smem_desc_sw128(st + Cfg::ACT_BYTES);
          const uint64_t dw1 = smem_desc_sw128(st + Cfg::ACT_BYTES + Cfg::W_BYTES);
#pragma unroll
          for (int kk = 0; kk < Cfg::BK / 16; ++kk) {
            const uint32_t acc = (kb != kb0 || kk != 0) ? 1u : 0u;
            const uint64_t adv = (uint64_t)(kk * 32) >> 4;  // 16 bf16 = 32 bytes along K
            if (Cfg::kTmemA) {
              // the widened weights of stage s in tensor memory: 8 columns
              // (16 f16) per K step, the linear half 32 columns further
              const uint32_t a0 = tmem_base + Cfg::A_COL0 + sa * Cfg::A_COLS + kk * 8;
              tc_mma_f16_tmem_a(d0, a0, da + adv, idesc, acc);
              if (Cfg::kDual) tc_mma_f16_tmem_a(d1, a0 + 32, da + adv, idesc, acc);
            } else if (Cfg::kSwap) {
              tc_mma_bf16(d0, dw0 + adv, da + adv, idesc, acc);
              if (Cfg::kDual) tc_mma_bf16(d1, dw1 + adv, da + adv, idesc, acc);
            } else {
              tc_mma_bf16(d0, da + adv, dw0 + adv, idesc, acc);
            }
          }
          tc_commit(&empty[s]);
          if (++s == Cfg::STAGES) { s = 0; ph ^= 1; }
          if (Cfg::kTmemA) {
            tc_commit(&aempty[sa]);
            if (++sa == Cfg::STAGES_A) { sa = 0; pha ^= 1; }
          }
        }
        if (!ok) break;
        tc_commit(&tfull[ab]);
      }
      // Every MMA this thread issued has completed once `drain` flips.
      tc_commit(drain);
      mbar_wait_drain(drain, 0);
    }
  } else if (warp < 4 && Cfg::kGather && !Cfg::kCpGather) {
    // ---------------- TMA row gather (weight-stationary tiles) ----------------
    // Lane i of warp 2 brings rows 4i..4i+3 of each stage's activation tile
    // (at most 64 rows) with one gather4 (rows picked by token index; the
    // tile's padding rows repeat its first row), completing on the stage's
    // full barrier, whose expected bytes the producer has armed.  Warp 3 has
    // no work here (with fp8 / fp4 weights it runs the weight slot producer).
    // (Token-tiled tiles gather 128 rows per stage with cp.async:
    // there a four-row TMA gather cannot keep up.)
    if (warp == 2) {
      int s = 0;
      uint32_t ph = 0;
      bool ok = true;
      int tl, ks, kb0, kb1;
      for (long wi = walk_start(walk); ok && walk_next(walk, wi, tl, ks, kb0, kb1);) {
        const int rt = tl / NT;
        int g, row0, rows;
        locate_row_tile_s(p, s_tiles, rt, g, row0, rows);
        const int nload = Cfg::kSwap ? max(16, (rows + 15) & ~15) : Cfg::ACT_ROWS;
        const bool active = 4 * lane < nload;
        int src[4];
        const int first = __ldg(p.gather + row0);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int r = 4 * lane + q;
          src[q] = r < rows ? __ldg(p.gather + row0 + r) : first;
        }
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait(&empty[s], ph ^ 1, abort_flag, p.err)) { ok = false; break; }
          if (active)
            tma_gather4(&tmA, &full[s], smem + s * Cfg::STAGE_BYTES + lane * 4 * 128,
                        kb * Cfg::BK, src[0], src[1], src[2], src[3]);
          if (++s == Cfg::STAGES) { s = 0; ph ^= 1; }
        }
      }
    }
  } else if (warp < 4) {
    // ---------------- cp.async row gather (token-tiled and wide tiles) ----------------
    // Each thread copies 16-byte chunks of the tile's rows straight into the
    // 128-byte-swizzled layout, then hands the stage to the MMA issuer with an
    // mbarrier arrive that the hardware triggers when its copies have landed.
    // The thread never waits for its own copies, so all STAGES stages can be
    // in flight.  Rows past the tile's end up to the MMA's row count are
    // zero-filled.
    if (Cfg::kCpGather) {
      constexpr int RI = Cfg::ACT_ROWS / 8;  // rows per thread
      const int gt = threadIdx.x - 64;  // 0..63
      const int q = gt & 7;             // 16-byte chunk of a 128-byte row
      const int rsub = gt >> 3;         // rows rsub, rsub + 8, ...
      const uint32_t swz = (uint32_t)((q ^ rsub) * 16);
      const bf16* A = static_cast<const bf16*>(p.A);
      int s = 0;
      uint32_t ph = 0;
      bool ok = true;
      int tl, ks, kb0, kb1;
      for (long wi = walk_start(walk); ok && walk_next(walk, wi, tl, ks, kb0, kb1);) {
        const int rt = tl / NT;
        int g, row0, rows;
        locate_row_tile_s(p, s_tiles, rt, g, row0, rows);
        const int nload = Cfg::kSwap ? max(16, (rows + 15) & ~15) : 128;
        const bf16* src[RI];
#pragma unroll
        for (int i = 0; i < RI; ++i) {
          const int r = rsub + 8 * i;
          src[i] = (r < rows) ? A + (size_t)__ldg(p.gather + row0 + r) * p.lda + q * 8 : A;
        }
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait(&empty[s], ph ^ 1, abort_flag, p.err)) { ok = false; break; }
          uint8_t* act = smem + s * Cfg::STAGE_BYTES;
#pragma unroll
          for (int i = 0; i < RI; ++i) {
            const int r = rsub + 8 * i;
            if (r < nload)
              cp_async_16(act + r * 128 + swz, src[i] + kb * Cfg::BK, r < rows ? 16u : 0u);
          }
          cp_async_mbar_arrive(&full[s]);
          mbar_arrive(&full[s]);
          if (++s == Cfg::STAGES) { s = 0; ph ^= 1; }
        }
      }
      cp_async_wait<0>();
    }
  } else if (warp >= 4 + Cfg::EPI_WARPS) {
    // ---------------- fp8 weights: widen to f16 ----------------
    // Same (tile, K block) sequence as the producer: E4M3 slot j is widened
    // into stage s's weight slots, handed to the MMA issuer with a fence
    // (generic-proxy writes -> tensor-core reads) and an arrive on full, and
    // the slot goes back to the producer with an arrive on w8empty.
    if (Cfg::kTmemA) {
      // Weight-stationary tiles: converter warp w (8 of them) widens the
      // rows of its TMEM lane quarter (w % 4; a warp may only access its own
      // quarter) of weight tile w / 4 (gated: the gate and the linear tile;
      // ungated: group w / 4 takes every other unit) into A stage a of
      // tensor memory, then waits for its stores and hands the stage on.
      // Units are the walk's K steps in order; every warp advances the slot
      // and stage counters over all of them.
      const int cw = warp - (4 + Cfg::EPI_WARPS);  // 0..7
      const int qd = warp & 3;
      const int half = cw >> 2;
      const int r = qd * 32 + lane;  // this thread's weight row (TMEM lane)
      int a = 0, j = 0, par = 0;
      uint32_t pha = 0, jph = 0;
      bool ok = true;
      int tl, ks, kb0, kb1;
      for (long wi = walk_start(walk); ok && walk_next(walk, wi, tl, ks, kb0, kb1);) {
        for (int kb = kb0; kb < kb1; ++kb) {
          if (Cfg::kDual || par == half) {
            // the slot has landed and the A stage's previous MMAs are done
            if (!mbar_wait(&w8full[j], jph, abort_flag, p.err)) { ok = false; break; }
            if (!mbar_wait(&aempty[a], pha ^ 1, abort_flag, p.err)) { ok = false; break; }
            tc_fence_after();
            const uint8_t* tile =
                w8_ring + j * Cfg::W8_SLOT + (Cfg::kDual ? half : 0) * Cfg::W8_BYTES;
            const uint32_t ta = tmem_base + ((uint32_t)(qd * 32) << 16) + Cfg::A_COL0 +
                                a * Cfg::A_COLS + (Cfg::kDual ? half * 32 : 0);
            uint32_t v[32];
            if (Cfg::kFp4)
              widen_fp4_row_sw32(tile, tile + Cfg::W4_CODES, r, (kb * 2) & 15, v);
            else
              widen_fp8_row_sw64(tile, r, v);
            tmem_st_32x32(ta, v);
            tc_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
              mbar_arrive(&afull[a]);
              mbar_arrive(&w8empty[j]);
            }
          }
          par ^= 1;
          if (++a == Cfg::STAGES_A) { a = 0; pha ^= 1; }
          if (++j == Cfg::S8) { j = 0; jph ^= 1; }
        }
      }
    } else if (Cfg::kFp8) {
      const int ct = threadIdx.x - (128 + 32 * Cfg::EPI_WARPS);
      int s = 0;
      uint32_t ph = 0;
      bool ok = true;
      int j = 0;
      uint32_t jph = 0;
      int tl, ks, kb0, kb1;
      for (long wi = walk_start(walk); ok && walk_next(walk, wi, tl, ks, kb0, kb1);) {
        for (int kb = kb0; kb < kb1; ++kb) {
          // the E4M3 slot has landed and the stage's previous MMAs are done
          if (!mbar_wait(&w8full[j], jph, abort_flag, p.err)) { ok = false; break; }
          if (!mbar_wait(&empty[s], ph ^ 1, abort_flag, p.err)) { ok = false; break; }
          uint8_t* st = smem + s * Cfg::STAGE_BYTES;
          const uint8_t* slot = w8_ring + j * Cfg::W8_SLOT;
#pragma unroll
          for (int i = 0; i < Cfg::NUM_W; ++i) {
            if (Cfg::kFp4)
              widen_fp4_tile<Cfg::W_ROWS, Cfg::CONV_THREADS>(
                  slot + i * Cfg::W8_BYTES, slot + i * Cfg::W8_BYTES + Cfg::W4_CODES, (kb * 2) & 15,
                  st + Cfg::ACT_BYTES + i * Cfg::W_BYTES, ct);
            else
              widen_fp8_tile<Cfg::W_ROWS, Cfg::CONV_THREADS>(slot + i * Cfg::W8_BYTES,
                                                             st + Cfg::ACT_BYTES + i * Cfg::W_BYTES,
                                                             ct);
          }
          // each thread orders its own writes for the tensor core, then one
          // lane per warp hands the warp's part on (8 arrivals, not 256)
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            mbar_arrive(&full[s]);
            mbar_arrive(&w8empty[j]);
          }
          if (++s == Cfg::STAGES) { s = 0; ph ^= 1; }
          if (++j == Cfg::S8) { j = 0; jph ^= 1; }
        }
      }
    }
  } else {
    // ---------------- epilogue (warps 4.. : two or three warpgroups) ----------------
    const int qd = warp & 3;          // TMEM lane quarter this warp may access
    const int eg = (warp - 4) >> 2;   // warpgroup: every (EPI_WARPS / 4)-th 32-column chunk
    constexpr int kChunkStride = 32 * (Cfg::EPI_WARPS / 4);  // columns between a warp's chunks
    int it = 0;
    uint32_t sk_ph = 0;  // stream-K: phase of epibar
    int tl, ks, kb0, kb1;
    for (long wi = walk_start(walk); walk_next(walk, wi, tl, ks, kb0, kb1); ++it) {
      const int rt = tl / NT, ft = tl - (tl / NT) * NT;
      const size_t slice_off = (size_t)ks * (size_t)p.epi.slice;
      int g, row0, rows;
      locate_row_tile_s(p, s_tiles, rt, g, row0, rows);
      const int ab = Cfg::ACC_BUFS == 2 ? (it & 1) : 0;
      const uint32_t aph = Cfg::ACC_BUFS == 2 ? (uint32_t)(it >> 1) & 1 : (uint32_t)it & 1;
      if (!mbar_wait(&tfull[ab], aph, abort_flag, p.err)) break;
      tc_fence_after();
      const uint32_t tb = tmem_base + ((uint32_t)(qd * 32) << 16) + ab * Cfg::ACC_COLS;
      const int f0 = ft * Cfg::FT;
      float v0[32], v1[32];
      if (!Cfg::kSwap) {
        const int r = qd * 32 + lane;
        const bool tma = p.tma_store && rows - qd * 32 >= 32;
        uint8_t* stg = stg_base + (warp - 4) * Cfg::STG_WARP;
        const int slice_rows = ks * p.M;  // split-K: the slice's rows in the output map
        for (int c0 = 32 * eg; c0 < Cfg::ACC_N; c0 += kChunkStride) {
          tmem_ld_32x32(tb + c0, v0);
          if (Cfg::kDual) tmem_ld_32x32(tb + Cfg::ACC_N + c0, v1);
          tc_wait_ld();
          if (f0 + c0 < p.F) {
            // per-output-channel scales of the fp8 weights (fp4 weights have
            // none: their block exponents were applied while widening)
            if (Cfg::kFp8 && !Cfg::kFp4) {
              const float* sc = p.w_scale + (size_t)g * p.w_group_stride + f0 + c0;
#pragma unroll
              for (int i = 0; i < 32; ++i) {
                const bool in = f0 + c0 + i < p.F;
                v0[i] *= in ? __ldg(sc + i) : 0.f;
                if (Cfg::kDual) v1[i] *= in ? __ldg(sc + p.dual_offset + i) : 0.f;
              }
            }
            if (tma)
              epi_tma_chunk32<Cfg::kEpi, Cfg::kDual, Cfg::kF16Out>(
                  p, &tmC, stg, lane, slice_rows + row0 + qd * 32, f0 + c0, v0, v1);
            else if (r < rows)
              store_row32<Cfg::kEpi, Cfg::kDual, Cfg::kF16Out>(p, row0 + r, f0 + c0, v0, v1,
                                                               slice_off);
          }
        }
      } else {
        const int f = f0 + qd * 32 + lane;
        const int fl = qd * 32 + lane;  // this thread's feature within the tile
        float s0 = 1.f, s1 = 1.f;  // fp8 weights: this thread's output channel scales
        if (Cfg::kFp8 && !Cfg::kFp4 && f < p.F) {
          const float* sc = p.w_scale + (size_t)g * p.w_group_stride + f;
          s0 = __ldg(sc);
          if (Cfg::kDual) s1 = __ldg(sc + p.dual_offset);
        }
        // Stream-K: a tile computed in two parts (see TileWalk).  Both parts
        // write their fp32 accumulators to their slot; the second to arrive
        // adds the other's and finishes the tile.
        bool finish = true;
        const float* other = nullptr;
        if (!Cfg::kWideSwap && walk.u_end >= 0 && (kb0 > 0 || kb1 < KB)) {
          const int part = kb0 > 0 ? 1 : 0;  // 1: tail (this range's start), 0: head (its end)
          const int b = part ? (int)blockIdx.x : (int)blockIdx.x + 1;  // the range boundary
          float* mine = p.sk_part + ((size_t)b * 2 + part) * kSkSlotFloats;
          other = p.sk_part + ((size_t)b * 2 + (part ^ 1)) * kSkSlotFloats;
          for (int c0 = 32 * eg; c0 < rows; c0 += kChunkStride) {
            tmem_ld_32x32(tb + c0, v0);
            if (Cfg::kDual) tmem_ld_32x32(tb + Cfg::ACC_N + c0, v1);
            tc_wait_ld();
            const int cn = min(32, rows - c0);
#pragma unroll
            for (int c = 0; c < 32; ++c) {
              if (c < cn) {
                mine[(size_t)(c0 + c) * 256 + fl] = v0[c];
                if (Cfg::kDual) mine[(size_t)(c0 + c) * 256 + 128 + fl] = v1[c];
              }
            }
          }
          // every epilogue thread's part is written and fenced before the
          // arrival is counted (bounded waits on an mbarrier, not bar.sync,
          // so that an aborting block cannot strand the other warps)
          __threadfence();
          __syncwarp();
          if (lane == 0) mbar_arrive(epibar);
          if (!mbar_wait(epibar, sk_ph, abort_flag, p.err)) break;
          sk_ph ^= 1;
          if (threadIdx.x == 128) {  // the first epilogue thread
            const int old = atomicAdd(p.sk_count + b, 1);
            if (old == 1) p.sk_count[b] = 0;  // both parts are in: reset for the next launch
            *sk_order = old;
          }
          __syncwarp();
          if (lane == 0) mbar_arrive(epibar);
          if (!mbar_wait(epibar, sk_ph, abort_flag, p.err)) break;
          sk_ph ^= 1;
          finish = *sk_order == 1;
          if (finish) __threadfence();
        }
        if (finish) {
          for (int c0 = 32 * eg; c0 < rows; c0 += kChunkStride) {
            tmem_ld_32x32(tb + c0, v0);
            if (Cfg::kDual) tmem_ld_32x32(tb + Cfg::ACC_N + c0, v1);
            tc_wait_ld();
            const int cn = min(32, rows - c0);
            if (other) {
#pragma unroll
              for (int c = 0; c < 32; ++c) {
                if (c < cn) {
                  v0[c] += __ldcg(other + (size_t)(c0 + c) * 256 + fl);
                  if (Cfg::kDual) v1[c] += __ldcg(other + (size_t)(c0 + c) * 256 + 128 + fl);
                }
              }
            }
            if (f < p.F) {
#pragma unroll
              for (int c = 0; c < 32; ++c)
                if (c < cn)
                  store_elem<Cfg::kEpi, Cfg::kF16Out>(p, row0 + c0 + c, f, v0[c] * s0,
                                                      Cfg::kDual ? v1[c] * s1 : 0.f);
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty[ab]);
    }
    if (lane == 0) bulk_wait0();  // this warp's bulk stores are complete
  }

  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, Cfg::TMEM_COLS);
  }
}


// ==== 2-SM (CTA pair) token-tiled GEMM ==========================================
//
// The prefill contractions on CTA pairs: one tcgen05.mma.cta_group::2 of
// M = 256, N = 256 per K step, issued by the pair's leader.  Each CTA stages
// its own 128 activation rows (A is split by M) and half of the 256 weight
// rows (B is split by N), so per SM the operand traffic (L2 -> shared memory,
// shared-memory reads by the tensor core, TMA requests) is two thirds of a
// single-CTA M = 128, N = 256 tile for the same math; each CTA's TMEM holds
// its 128 rows x 256 columns.  Gated FC1: CTA 0 stages the 128 gate rows and
// CTA 1 the 128 linear rows of the same features, which puts gate and linear
// accumulators side by side in every row as in the single-CTA kernel.
//
// Synchronisation: both CTAs' TMA loads complete on the leader's `full`
// barrier (2-SM TMA); the leader's MMA commits arrive on `empty` and `tfull`
// in both CTAs (multicast commit); both CTAs' epilogue warps arrive on the
// leader's `tempty` (remote arrive).  Activations are TMA tiles of contiguous
// rows (dense GEMMs, and the expert FC2 whose input rows are already in
// expert order), or (kGather, the expert FC1 of experts with many rows) rows
// fetched by token index with cp.async by warps 2-3 of each CTA: the
// leader's gather completes on its own `full` barrier, the peer's on its
// local `gfull` barrier, and the peer's warp 1 relays each completed stage to
// the leader's `full` with a remote arrive (cp.async can only signal the
// executing CTA's barriers).

template <bool kDual_, int kEpi_, bool kGather_ = false>
struct TcPairCfg {
  static constexpr bool kDual = kDual_;
  static constexpr bool kGather = kGather_;
  static constexpr int kEpi = kEpi_;
  static constexpr int BK = 64;
  static constexpr int A_BYTES = 128 * BK * 2;   // this CTA's 128 rows
  static constexpr int B_BYTES = 128 * BK * 2;   // this CTA's half of the 256 weight rows
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int STG_WARP = kEpi == EPI_F32_BIAS ? 4096 : 2048;  // one 32 x 32 box
  static constexpr int STG_BYTES = kEpiWarps * STG_WARP;               // epilogue staging
  static constexpr int STAGES = kEpi == EPI_F32_BIAS ? 5 : 6;
  static constexpr int ACC_N = 256;              // columns of one accumulator buffer
  static constexpr int TMEM_COLS = 512;
  static constexpr int FT = kDual ? 128 : 256;   // output features per tile
  static constexpr int SMEM_BYTES = 1024 + STAGES * STAGE_BYTES + STG_BYTES + 512 +
                                    2 * (LMOE_MAX_EXPERTS + 1) * 4;
  static_assert(SMEM_BYTES <= 227 * 1024, "shared memory");
};

template <class Cfg>
__global__ void __launch_bounds__(kTcThreads, 1)
    tc_gemm_pair_kernel(const __grid_constant__ CUtensorMap tmA,
                        const __grid_constant__ CUtensorMap tmB,
                        const __grid_constant__ CUtensorMap tmC, const GemmProblem p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* stg_base = smem + Cfg::STAGES * Cfg::STAGE_BYTES;  // epilogue staging (1024-aligned)
  uint64_t* full = reinterpret_cast<uint64_t*>(stg_base + Cfg::STG_BYTES);
  uint64_t* empty = full + Cfg::STAGES;
  uint64_t* gfull = empty + Cfg::STAGES;  // kGather, peer CTA: its own gather's completion
  uint64_t* tfull = gfull + Cfg::STAGES;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int* s_tiles = reinterpret_cast<int*>(stg_base + Cfg::STG_BYTES + 512);
  static_assert(3 * Cfg::STAGES * 8 + 5 * 8 + 8 <= 512, "barrier area");

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  griddep_launch();
  const uint32_t rank = cluster_ctarank();
  const int cid = (int)cluster_id_x(), ncl = (int)cluster_count_x();
  const int NT = (p.F + Cfg::FT - 1) / Cfg::FT;
  const int KB = p.K / Cfg::BK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < Cfg::STAGES; ++s) {
      // leader: the producer's expect_tx arrive, and (kGather) its own gather
      // threads and the peer's relay
      mbar_init(&full[s], Cfg::kGather ? 2 + kGatherThreads : 1);
      mbar_init(&empty[s], 1);
      mbar_init(&gfull[s], kGatherThreads);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], 2 * kEpiWarps);  // the epilogue warps of both CTAs
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    if (!Cfg::kGather) prefetch_tensormap(&tmA);
    prefetch_tensormap(&tmB);
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_slot, Cfg::TMEM_COLS);
    tmem_relinquish_pair();
    tc_fence_before();
  }
  griddep_wait();  // the previous kernel's outputs (tile tables, activations)
  load_tile_tables(p, s_tiles);
  __syncthreads();
  cluster_sync();  // both CTAs' barriers exist before any remote arrive
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int num_tiles = total_row_tiles_s(p, s_tiles) * NT;

  if (warp == 0) {
    // ---------------- TMA producer (both CTAs) ----------------
    if (lane == 0) {
      const uint32_t full_leader = cluster_map(&full[0], 0);
      // bytes the leader's barrier counts per stage: both CTAs' TMA loads
      constexpr uint32_t kTx = Cfg::kGather ? 2 * Cfg::B_BYTES : 2 * Cfg::STAGE_BYTES;
      int s = 0;
      uint32_t ph = 0;
      long armed = 0;
      for (int t = cid; t < num_tiles; t += ncl) {
        const int rt = t / NT, ft = t - (t / NT) * NT;
        int g, row0, rows;
        locate_row_tile_s(p, s_tiles, rt, g, row0, rows);
        int wrow = (int)(g * p.w_group_stride) + ft * Cfg::FT;
        wrow += Cfg::kDual ? (rank ? p.dual_offset : 0) : (int)rank * 128;
        const int arow = row0 + (int)rank * 128;
        bool ok = true;
        for (int kb = 0; kb < KB; ++kb) {
          if (!mbar_wait_cluster(&empty[s], ph ^ 1, abort_flag, p.err)) { ok = false; break; }
          uint8_t* st = smem + s * Cfg::STAGE_BYTES;
          if (rank == 0) {
            mbar_arrive_expect_tx(&full[s], kTx);
            ++armed;
          }
          const uint32_t fb = full_leader + (uint32_t)s * 8u;
          if (!Cfg::kGather) tma_load_2d_pair(&tmA, fb, st, kb * Cfg::BK, arow);
          tma_load_2d_pair(&tmB, fb, st + Cfg::A_BYTES, kb * Cfg::BK, wrow);
          if (++s == Cfg::STAGES) { s = 0; ph ^= 1; }
        }
        if (!ok) break;
      }
      if (rank == 0 && *abort_flag) {
        int ss = s;
        uint32_t pp = ph;
        for (long i = 0; i < armed && i < Cfg::STAGES; ++i) {
          if (ss == 0) { ss = Cfg::STAGES; pp ^= 1; }
          --ss;
          mbar_wait_drain(&full[ss], pp);
        }
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer (leader only) ----------------
    if (rank == 0 && lane == 0) {
      const uint32_t idesc = idesc_bf16_f32(256, Cfg::ACC_N);
      int s = 0;
      uint32_t ph = 0;
      int it = 0;
      for (int t = cid; t < num_tiles; t += ncl, ++it) {
        const int ab = it & 1;
        const uint32_t aph = (it >> 1) & 1;
        if (!mbar_wait_cluster(&tempty[ab], aph ^ 1, abort_flag, p.err)) break;
        tc_fence_after();
        const uint32_t d0 = tmem_base + ab * Cfg::ACC_N;
        bool ok = true;
        for (int kb = 0; kb < KB; ++kb) {
          if (!mbar_wait_cluster(&full[s], ph, abort_flag, p.err)) { ok = false; break; }
          // gathered rows were written by cp.async (generic proxy): order
          // them before the tensor core's reads
          if (Cfg::kGather) fence_proxy_async_smem();
          tc_fence_after();
          const uint8_t* st = smem + s * Cfg::STAGE_BYTES;
          const uint64_t da = smem_desc_sw128(st);
          const uint64_t db = smem_desc_sw128(st + Cfg::A_BYTES);
#pragma unroll
          for (int kk = 0; kk < Cfg::BK / 16; ++kk) {
            const uint64_t adv = (uint64_t)(kk * 32) >> 4;
            tc_mma_bf16_pair(d0, da + adv, db + adv, idesc, (kb | kk) != 0);
          }
          tc_commit_pair_mc(&empty[s], 0x3);
          if (++s == Cfg::STAGES) { s = 0; ph ^= 1; }
        }
        if (!ok) break;
        tc_commit_pair_mc(&tfull[ab], 0x3);
      }
      tc_commit_pair_mc(drain, 0x1);
      mbar_wait_drain(drain, 0);
    } else if (Cfg::kGather && rank == 1 && lane == 0) {
      // ---------------- relay of the peer's gather (CTA 1) ----------------
      const uint32_t full_leader = cluster_map(&full[0], 0);
      int s = 0;
      uint32_t ph = 0;
      bool ok = true;
      for (int t = cid; t < num_tiles && ok; t += ncl) {
        for (int kb = 0; kb < KB; ++kb) {
          if (!mbar_wait(&gfull[s], ph, abort_flag, p.err)) { ok = false; break; }
          fence_proxy_async_smem();
          mbar_arrive_cluster(full_leader + (uint32_t)s * 8u);
          if (++s == Cfg::STAGES) { s = 0; ph ^= 1; }
        }
      }
    }
  } else if (warp < 4) {
    // ---------------- cp.async row gather (kGather, both CTAs) ----------------
    // This CTA's 128 rows of the 256-row tile, fetched by token index into
    // the 128-byte-swizzled A stage; rows past the tile's end are zero-filled.
    if (Cfg::kGather) {
      const int gt = threadIdx.x - 64;  // 0..63
      const int q = gt & 7;             // 16-byte chunk of a 128-byte row
      const int rsub = gt >> 3;         // rows rsub, rsub + 8, ...
      const uint32_t swz = (uint32_t)((q ^ rsub) * 16);
      const bf16* A = static_cast<const bf16*>(p.A);
      uint64_t* done_bar = rank == 0 ? full : gfull;
      int s = 0;
      uint32_t ph = 0;
      bool ok = true;
      for (int t = cid; t < num_tiles && ok; t += ncl) {
        const int rt = t / NT;
        int g, row0, rows;
        locate_row_tile_s(p, s_tiles, rt, g, row0, rows);
        const int base = (int)rank * 128;
        const bf16* src[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const int r = base + rsub + 8 * i;
          src[i] = (r < rows) ? A + (size_t)__ldg(p.gather + row0 + r) * p.lda + q * 8 : A;
        }
        for (int kb = 0; kb < KB; ++kb) {
          if (!mbar_wait_cluster(&empty[s], ph ^ 1, abort_flag, p.err)) { ok = false; break; }
          uint8_t* act = smem + s * Cfg::STAGE_BYTES;
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const int r = rsub + 8 * i;
            cp_async_16(act + r * 128 + swz, src[i] + kb * Cfg::BK, base + r < rows ? 16u : 0u);
          }
          cp_async_mbar_arrive(&done_bar[s]);
          mbar_arrive(&done_bar[s]);
          if (++s == Cfg::STAGES) { s = 0; ph ^= 1; }
        }
      }
      cp_async_wait<0>();
    }
  } else if (warp >= 4) {
    // ---------------- epilogue (warps 4..11 of both CTAs) ----------------
    const int qd = warp & 3;
    const int eg = (warp - 4) >> 2;
    const uint32_t tempty_leader = cluster_map(&tempty[0], 0);
    int it = 0;
    for (int t = cid; t < num_tiles; t += ncl, ++it) {
      const int rt = t / NT, ft = t - (t / NT) * NT;
      int g, row0, rows;
      locate_row_tile_s(p, s_tiles, rt, g, row0, rows);
      const int ab = it & 1;
      const uint32_t aph = (it >> 1) & 1;
      if (!mbar_wait_cluster(&tfull[ab], aph, abort_flag, p.err)) break;
      tc_fence_after();
      const uint32_t tb = tmem_base + ((uint32_t)(qd * 32) << 16) + ab * Cfg::ACC_N;
      const int f0 = ft * Cfg::FT;
      const int wrow = (int)rank * 128 + qd * 32;  // this warp's first row in the 256-row tile
      const int r = wrow + lane;
      const bool tma = p.tma_store && rows - wrow >= 32;
      uint8_t* stg = stg_base + (warp - 4) * Cfg::STG_WARP;
      float v0[32], v1[32];
      constexpr int NCOL = Cfg::kDual ? 128 : 256;
      for (int c0 = 32 * eg; c0 < NCOL; c0 += 64) {
        tmem_ld_32x32(tb + c0, v0);
        if (Cfg::kDual) tmem_ld_32x32(tb + 128 + c0, v1);
        tc_wait_ld();
        if (f0 + c0 < p.F) {
          if (tma)
            epi_tma_chunk32<Cfg::kEpi, Cfg::kDual>(p, &tmC, stg, lane, row0 + wrow, f0 + c0, v0,
                                                   v1);
          else if (r < rows)
            store_row32<Cfg::kEpi, Cfg::kDual>(p, row0 + r, f0 + c0, v0, v1);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(tempty_leader + (uint32_t)ab * 8u);
    }
    if (lane == 0) bulk_wait0();
  }

  __syncthreads();
  cluster_sync();  // no CTA leaves while its peer may still signal its barriers
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, Cfg::TMEM_COLS);
  }
}


// ==== weight-stationary grouped GEMM on CTA pairs ================================
//
// The prefill expert GEMMs.  Token-tiled tiles have 128 (or, on pairs, 256)
// rows, and an expert's last tile is padded to that size: with a few hundred
// rows per expert a fifth to two fifths of the tensor-core work is padding.
// Here the expert's rows are the MMA's N dimension, which only needs a
// multiple of 16: one tcgen05.mma.cta_group::2 of M = 256 weight rows
// (features; each CTA stages 128) and N = the tile's rows (each CTA stages
// half), with an expert's rows split into ceil(rows / NMAX) tiles of nearly
// equal size in units of 16.  Splitting the rows across the pair keeps the
// shared-memory operand reads at or below those of a 1-CTA 128 x 256 tile
// for N >= ~100.
//
// Gated FC1 (SwiGLU) issues two MMAs per K step, gate rows and linear rows of
// the same 256 features, into accumulators at TMEM columns [0, N) and
// [128, 128 + N): NMAX = 128 keeps two buffers in 512 columns.  Ungated
// problems use NMAX = 256.
//
// Rows reach shared memory by TMA (contiguous rows: FC2) or by the cp.async
// gather of both CTAs (FC1 reads the down-projected tokens by index).  The
// peer CTA's gather completes on its own mbarrier (cp.async can only signal
// the executing CTA's barriers), and its warp 1 relays each completed stage
// to the leader's `full` barrier with a remote arrive.
//
// Epilogue: TMEM lane = feature, column = row, so each thread holds one
// feature of 32 rows and a warp writes 64 contiguous bytes of every row.

template <bool kGather_, bool kDual_, int kEpi_>
struct TcPairWsCfg {
  static constexpr bool kGather = kGather_, kDual = kDual_;
  static constexpr int kEpi = kEpi_;
  static constexpr int BK = 64;
  static constexpr int NUM_W = kDual ? 2 : 1;
  static constexpr int NMAX = kDual ? 128 : 256;  // rows per tile (the MMA's N), at most
  static constexpr int W_BYTES = 128 * BK * 2;    // this CTA's 128 weight rows
  static constexpr int B_ROWS = NMAX / 2;         // this CTA's rows of a tile, at most
  static constexpr int B_BYTES = B_ROWS * BK * 2;
  static constexpr int STAGE_BYTES = NUM_W * W_BYTES + B_BYTES;
  static constexpr int STAGES_RAW = kTcSmemBudget / STAGE_BYTES;
  static constexpr int STAGES = STAGES_RAW > 8 ? 8 : STAGES_RAW;
  static constexpr int ACC_COLS = 256;            // one accumulator buffer
  static constexpr int TMEM_COLS = 512;
  static constexpr int FT = 256;                  // output features per tile (128 per CTA)
  static constexpr int TABLE_BYTES = 2 * (LMOE_MAX_EXPERTS + 1) * 4;
  static constexpr int SMEM_BYTES = 1024 + STAGES * STAGE_BYTES + 512 + TABLE_BYTES;
  static_assert(SMEM_BYTES <= 227 * 1024, "shared memory");
  static_assert(STAGES >= 3, "pipeline too shallow");
  static_assert(kEpi == EPI_ACT || kEpi == EPI_SCALE_ROWS, "grouped epilogues");
  static_assert(kGather || B_ROWS % 32 == 0, "row boxes of 32");
};

// Row tile rt of a grouped problem split into nearly equal tiles: group g,
// first row row0, valid rows n, and the MMA's N (n rounded up to 16; at most
// NMAX when the tile counts are ceil(rows / NMAX)).
__device__ __forceinline__ void locate_ws_tile(const GemmProblem& p, const int* s_tiles, int rt,
                                               int& g, int& row0, int& n, int& nmma) {
  const int* tp = s_tiles;
  const int* off = s_tiles + LMOE_MAX_EXPERTS + 1;
  int lo = 0, hi = p.G - 1;  // largest g with tp[g] <= rt
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (tp[mid] <= rt) lo = mid; else hi = mid - 1;
  }
  g = lo;
  const int j = rt - tp[g], nt = tp[g + 1] - tp[g];
  const int rows_g = off[g + 1] - off[g];
  const int units = (rows_g + 15) >> 4;
  const int s16 = j * units / nt, e16 = (j + 1) * units / nt;
  row0 = off[g] + 16 * s16;
  n = min(16 * e16, rows_g) - 16 * s16;
  nmma = 16 * (e16 - s16);
}

template <class Cfg>
__global__ void __launch_bounds__(kTcThreads, 1)
    tc_gemm_pair_ws_kernel(const __grid_constant__ CUtensorMap tmA,
                           const __grid_constant__ CUtensorMap tmB, const GemmProblem p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + Cfg::STAGES * Cfg::STAGE_BYTES);
  uint64_t* empty = full + Cfg::STAGES;
  uint64_t* gfull = empty + Cfg::STAGES;  // peer CTA: its own gather's completion
  uint64_t* tfull = gfull + Cfg::STAGES;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int* s_tiles = reinterpret_cast<int*>(smem + Cfg::STAGES * Cfg::STAGE_BYTES + 512);
  static_assert(3 * Cfg::STAGES * 8 + 5 * 8 + 8 <= 512, "barrier area");

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  griddep_launch();
  const uint32_t rank = cluster_ctarank();
  const int cid = (int)cluster_id_x(), ncl = (int)cluster_count_x();
  const int NT = (p.F + Cfg::FT - 1) / Cfg::FT;
  const int KB = p.K / Cfg::BK;
  constexpr int W_OFF = Cfg::NUM_W * Cfg::W_BYTES;  // rows follow the weight tile(s)

  if (threadIdx.x == 0) {
    for (int s = 0; s < Cfg::STAGES; ++s) {
      // leader: its TMA arrive + (gather) its 64 gather threads + the peer's relay
      mbar_init(&full[s], Cfg::kGather ? 2 + kGatherThreads : 1);
      mbar_init(&empty[s], 1);
      mbar_init(&gfull[s], kGatherThreads);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], 2 * kEpiWarps);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    if (!Cfg::kGather) prefetch_tensormap(&tmA);
    prefetch_tensormap(&tmB);
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_slot, Cfg::TMEM_COLS);
    tmem_relinquish_pair();
    tc_fence_before();
  }
  griddep_wait();  // the previous kernel's outputs (tile tables, activations)
  load_tile_tables(p, s_tiles);
  __syncthreads();
  cluster_sync();  // both CTAs' barriers exist before any remote arrive
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int num_tiles = s_tiles[p.G] * NT;

  if (warp == 0) {
    // ---------------- TMA producer (both CTAs) ----------------
    if (lane == 0) {
      const uint32_t full_leader = cluster_map(&full[0], 0);
      int s = 0;
      uint32_t ph = 0;
      long armed = 0;
      for (int t = cid; t < num_tiles; t += ncl) {
        const int rt = t / NT, ft = t - (t / NT) * NT;
        int g, row0, n, nmma;
        locate_ws_tile(p, s_tiles, rt, g, row0, n, nmma);
        const int hb = nmma >> 1;  // rows per CTA
        const int wrow = (int)(g * p.w_group_stride) + ft * Cfg::FT + (int)rank * 128;
        const int nsub = Cfg::kGather ? 0 : (hb + 31) / 32;
        const uint32_t bytes = 2u * (uint32_t)(W_OFF + nsub * 4096);
        bool ok = true;
        for (int kb = 0; kb < KB; ++kb) {
          if (!mbar_wait_cluster(&empty[s], ph ^ 1, abort_flag, p.err)) { ok = false; break; }
          uint8_t* st = smem + s * Cfg::STAGE_BYTES;
          if (rank == 0) {
            mbar_arrive_expect_tx(&full[s], bytes);
            ++armed;
          }
          const uint32_t fb = full_leader + (uint32_t)s * 8u;
          tma_load_2d_pair(&tmB, fb, st, kb * Cfg::BK, wrow);
          if (Cfg::kDual)
            tma_load_2d_pair(&tmB, fb, st + Cfg::W_BYTES, kb * Cfg::BK, wrow + p.dual_offset);
          for (int sub = 0; sub < nsub; ++sub)
            tma_load_2d_pair(&tmA, fb, st + W_OFF + sub * 4096, kb * Cfg::BK,
                             row0 + (int)rank * hb + sub * 32);
          if (++s == Cfg::STAGES) { s = 0; ph ^= 1; }
        }
        if (!ok) break;
      }
      if (rank == 0 && *abort_flag) {
        int ss = s;
        uint32_t pp = ph;
        for (long i = 0; i < armed && i < Cfg::STAGES; ++i) {
          if (ss == 0) { ss = Cfg::STAGES; pp ^= 1; }
          --ss;
          mbar_wait_drain(&full[ss], pp);
        }
      }
    }
  } else if (warp == 1) {
    if (rank == 0 && lane == 0) {
      // ---------------- MMA issuer (leader) ----------------
      int s = 0;
      uint32_t ph = 0;
      int it = 0;
      for (int t = cid; t < num_tiles; t += ncl, ++it) {
        const int rt = t / NT;
        int g, row0, n, nmma;
        locate_ws_tile(p, s_tiles, rt, g, row0, n, nmma);
        const uint32_t idesc = idesc_bf16_f32(256, nmma);
        const int ab = it & 1;
        const uint32_t aph = (it >> 1) & 1;
        if (!mbar_wait_cluster(&tempty[ab], aph ^ 1, abort_flag, p.err)) break;
        tc_fence_after();
        const uint32_t d0 = tmem_base + ab * Cfg::ACC_COLS;
        bool ok = true;
        for (int kb = 0; kb < KB; ++kb) {
          if (!mbar_wait_cluster(&full[s], ph, abort_flag, p.err)) { ok = false; break; }
          tc_fence_after();
          const uint8_t* st = smem + s * Cfg::STAGE_BYTES;
          const uint64_t dw0 = smem_desc_sw128(st);
          const uint64_t dw1 = smem_desc_sw128(st + Cfg::W_BYTES);
          const uint64_t db = smem_desc_sw128(st + W_OFF);
#pragma unroll
          for (int kk = 0; kk < Cfg::BK / 16; ++kk) {
            const uint32_t acc = (kb | kk) != 0;
            const uint64_t adv = (uint64_t)(kk * 32) >> 4;
            tc_mma_bf16_pair(d0, dw0 + adv, db + adv, idesc, acc);
            if (Cfg::kDual) tc_mma_bf16_pair(d0 + 128, dw1 + adv, db + adv, idesc, acc);
          }
          tc_commit_pair_mc(&empty[s], 0x3);
          if (++s == Cfg::STAGES) { s = 0; ph ^= 1; }
        }
        if (!ok) break;
        tc_commit_pair_mc(&tfull[ab], 0x3);
      }
      tc_commit_pair_mc(drain, 0x1);
      mbar_wait_drain(drain, 0);
    } else if (rank == 1 && lane == 0 && Cfg::kGather) {
      // ---------------- relay of the peer's gather (CTA 1) ----------------
      const uint32_t full_leader = cluster_map(&full[0], 0);
      int s = 0;
      uint32_t ph = 0;
      bool ok = true;
      for (int t = cid; t < num_tiles && ok; t += ncl) {
        for (int kb = 0; kb < KB; ++kb) {
          if (!mbar_wait(&gfull[s], ph, abort_flag, p.err)) { ok = false; break; }
          fence_proxy_async_smem();
          mbar_arrive_cluster(full_leader + (uint32_t)s * 8u);
          if (++s == Cfg::STAGES) { s = 0; ph ^= 1; }
        }
      }
    }
  } else if (warp < 4) {
    // ---------------- cp.async row gather (both CTAs) ----------------
    if (Cfg::kGather) {
      const int gt = threadIdx.x - 64;  // 0..63
      const int q = gt & 7;             // 16-byte chunk of a 128-byte row
      const int rsub = gt >> 3;         // rows rsub, rsub + 8, ...
      const uint32_t swz = (uint32_t)((q ^ rsub) * 16);
      const bf16* A = static_cast<const bf16*>(p.A);
      uint64_t* done_bar = rank == 0 ? full : gfull;
      constexpr int RI = Cfg::B_ROWS / 8;
      int s = 0;
      uint32_t ph = 0;
      bool ok = true;
      for (int t = cid; t < num_tiles && ok; t += ncl) {
        const int rt = t / NT;
        int g, row0, n, nmma;
        locate_ws_tile(p, s_tiles, rt, g, row0, n, nmma);
        const int hb = nmma >> 1;
        const int base = (int)rank * hb;
        const bf16* src[RI];
#pragma unroll
        for (int i = 0; i < RI; ++i) {
          const int rr = base + rsub + 8 * i;
          src[i] = (rr < n) ? A + (size_t)__ldg(p.gather + row0 + rr) * p.lda + q * 8 : A;
        }
        for (int kb = 0; kb < KB; ++kb) {
          if (!mbar_wait_cluster(&empty[s], ph ^ 1, abort_flag, p.err)) { ok = false; break; }
          uint8_t* rows_smem = smem + s * Cfg::STAGE_BYTES + W_OFF;
#pragma unroll
          for (int i = 0; i < RI; ++i) {
            const int r = rsub + 8 * i;
            if (r < hb)
              cp_async_16(rows_smem + r * 128 + swz, src[i] + kb * Cfg::BK,
                          base + r < n ? 16u : 0u);
          }
          cp_async_mbar_arrive(&done_bar[s]);
          mbar_arrive(&done_bar[s]);
          if (++s == Cfg::STAGES) { s = 0; ph ^= 1; }
        }
      }
      cp_async_wait<0>();
    }
  } else {
    // ---------------- epilogue (warps 4..11 of both CTAs) ----------------
    const int qd = warp & 3;
    const int eg = (warp - 4) >> 2;
    const uint32_t tempty_leader = cluster_map(&tempty[0], 0);
    const EpiParams& e = p.epi;
    bf16* out = static_cast<bf16*>(e.out);
    int it = 0;
    for (int t = cid; t < num_tiles; t += ncl, ++it) {
      const int rt = t / NT, ft = t - (t / NT) * NT;
      int g, row0, n, nmma;
      locate_ws_tile(p, s_tiles, rt, g, row0, n, nmma);
      const int ab = it & 1;
      const uint32_t aph = (it >> 1) & 1;
      if (!mbar_wait_cluster(&tfull[ab], aph, abort_flag, p.err)) break;
      tc_fence_after();
      const uint32_t tb = tmem_base + ((uint32_t)(qd * 32) << 16) + ab * Cfg::ACC_COLS;
      const int f = ft * Cfg::FT + (int)rank * 128 + qd * 32 + lane;
      const bool fok = f < p.F;
      float v0[32], v1[32];
      for (int c0 = 32 * eg; c0 < n; c0 += 64) {
        tmem_ld_32x32(tb + c0, v0);
        if (Cfg::kDual) tmem_ld_32x32(tb + 128 + c0, v1);
        tc_wait_ld();
        const int cn = min(32, n - c0);
        float rw = 1.f;
        if (Cfg::kEpi == EPI_SCALE_ROWS && lane < cn) rw = __ldg(e.row_w + row0 + c0 + lane);
        bf16* o = out + (size_t)(row0 + c0) * e.ldo + (Cfg::kEpi == EPI_ACT ? e.col0 : 0) + f;
#pragma unroll
        for (int c = 0; c < 32; ++c) {
          float v;
          if (Cfg::kEpi == EPI_SCALE_ROWS) v = v0[c] * __shfl_sync(0xffffffffu, rw, c);
          else v = apply_act(e.act, v0[c], Cfg::kDual ? v1[c] : 0.f);
          if (c < cn && fok) {
            const bf16 hi = __float2bfloat16_rn(v);
            o[(size_t)c * e.ldo] = hi;
            if (Cfg::kEpi == EPI_ACT && e.split_off)
              o[(size_t)c * e.ldo + e.split_off] = __float2bfloat16_rn(v - __bfloat162float(hi));
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(tempty_leader + (uint32_t)ab * 8u);
    }
  }

  __syncthreads();
  cluster_sync();  // no CTA leaves while its peer may still signal its barriers
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, Cfg::TMEM_COLS);
  }
}

}  // namespace lmoe
