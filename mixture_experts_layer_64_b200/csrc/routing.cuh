// Routing: top-k selection with renormalised gates, and the grouping of
// (token, slot) pairs by expert into a deterministic, stable permutation
// (LatentMoE paper, Section 3: the top-K index set of Eq. (1)/(2) and the
// dispatch after the down-projection).
//
//   topk_softmax_kernel   one warp per token.  Each logit becomes an
//                         order-preserving 32-bit key (-0.0 folded into +0.0);
//                         the keys that can be in the top k (at or above the
//                         k-th largest lane maximum) are sorted by (key,
//                         ~expert); a radix select takes over when too many
//                         pass.  Ties go to the lowest expert index.  The
//                         gates are exp(l_j - l_0) / sum over the k chosen.
//                         Each choice sets bit t of expert e's token bitmap.
//   group_count_kernel    one warp per expert: popcount prefix over the
//                         expert's bitmap words (also clears them for the next
//                         call); the last block to finish scans the loads
//                         into offsets and into per-expert 128-row tile counts.
//   group_rank_kernel     one thread per pair: row = offsets[e] + (tokens < t
//                         routed to e), read from the word prefix + popcount;
//                         writes row -> token, row -> pair, row -> gate and
//                         pair -> row.
// Everything is integer work on fixed inputs, so the permutation is the same
// on every run and equals "sort pairs by expert, then by token".
#pragma once

#include "common.cuh"

namespace lmoe {

__device__ __forceinline__ uint32_t orderable_bits(float v) {
  if (v == 0.0f) v = 0.0f;  // -0.0 and +0.0 compare equal: one key
  const uint32_t u = __float_as_uint(v);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float from_orderable_bits(uint32_t u) {
  return __uint_as_float((u & 0x80000000u) ? (u & 0x7FFFFFFFu) : ~u);
}

// Bitonic sort of 32 values across a warp (one per lane), descending.
template <typename V>
__device__ __forceinline__ V warp_sort_desc32(V v, int lane) {
#pragma unroll
  for (int size = 2; size <= 32; size <<= 1) {
#pragma unroll
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      const V o = __shfl_xor_sync(0xffffffffu, v, stride);
      const bool keep_hi = ((lane & stride) == 0) == ((lane & size) == 0);
      v = keep_hi ? (v > o ? v : o) : (v > o ? o : v);
    }
  }
  return v;
}

// Bitonic sort of 64 values across a warp, descending: lane L holds elements
// L (a) and L + 32 (b).  On return a holds the 32 largest in order.
__device__ __forceinline__ void warp_sort_desc64(unsigned long long& a, unsigned long long& b,
                                                 int lane) {
#pragma unroll
  for (int size = 2; size <= 64; size <<= 1) {
#pragma unroll
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      if (stride == 32) {  // a and b are partners; size 64 sorts descending
        const unsigned long long hi = a > b ? a : b, lo = a > b ? b : a;
        a = hi;
        b = lo;
      } else {
        const unsigned long long oa = __shfl_xor_sync(0xffffffffu, a, stride);
        const unsigned long long ob = __shfl_xor_sync(0xffffffffu, b, stride);
        const bool lower = (lane & stride) == 0;
        const bool keep_a = lower == ((lane & size) == 0);
        const bool keep_b = lower == (((lane + 32) & size) == 0);
        a = keep_a ? (a > oa ? a : oa) : (a > oa ? oa : a);
        b = keep_b ? (b > ob ? b : ob) : (b > ob ? ob : b);
      }
    }
  }
}

// Exclusive scans over the experts of their loads and tile counts (the
// prefixes listed at group_count_kernel), by one block of up to 256 threads;
// the counts were written by other blocks (read through L2).  NULL outputs
// are skipped; entry N of each is the total.
static __device__ __noinline__ void scan_loads_block(const int* counts, int N, int* offsets,
                                              int* tile_prefix, int* tile_prefix2,
                                              int* tile_prefix64, int* big_prefix2,
                                              int* small_prefix, int* small_prefix2,
                                              int* full_prefix2 = nullptr,
                                              int* rem_prefix = nullptr) {
  constexpr int kQ = 9;
  __shared__ int s_q[kQ][256];
  const int nt = blockDim.x;
  const int per = (N + nt - 1) / nt;
  const int lo = threadIdx.x * per, hi = min(N, lo + per);
  const auto tiles_of = [](int c, int* q) {
    q[0] = c;
    q[1] = (c + kRowTile - 1) / kRowTile;
    q[2] = (c + 2 * kRowTile - 1) / (2 * kRowTile);
    q[3] = (c + kSwapRowTile - 1) / kSwapRowTile;
    q[4] = c > kPairMinRows ? q[2] : 0;
    q[5] = c > kPairMinRows ? 0 : q[1];
    q[6] = c > kPairMinRows ? 0 : q[2];
    // pair tiles of the split FC2: the whole 256-row tiles, and the last
    // rows if more than 128 of them are left (a 256-row tile pads them no
    // worse than two 128-row tiles); at most 128 left rows take one 128-row
    // single-CTA tile instead (half the padding)
    const int r = c % (2 * kRowTile);
    q[7] = c / (2 * kRowTile) + (r > kRowTile ? 1 : 0);
    q[8] = (r > 0 && r <= kRowTile) ? 1 : 0;
  };
  int sum[kQ] = {0, 0, 0, 0, 0, 0, 0, 0, 0};
  for (int i = lo; i < hi; ++i) {
    int q[kQ];
    tiles_of(__ldcg(counts + i), q);
#pragma unroll
    for (int j = 0; j < kQ; ++j) sum[j] += q[j];
  }
#pragma unroll
  for (int j = 0; j < kQ; ++j) s_q[j][threadIdx.x] = sum[j];
  __syncthreads();
  for (int o = 1; o < nt; o <<= 1) {
    int add[kQ];
#pragma unroll
    for (int j = 0; j < kQ; ++j) add[j] = threadIdx.x >= o ? s_q[j][threadIdx.x - o] : 0;
    __syncthreads();
#pragma unroll
    for (int j = 0; j < kQ; ++j) s_q[j][threadIdx.x] += add[j];
    __syncthreads();
  }
  int run[kQ];
#pragma unroll
  for (int j = 0; j < kQ; ++j) run[j] = s_q[j][threadIdx.x] - sum[j];
  int* out[kQ] = {offsets,      tile_prefix,   tile_prefix2, tile_prefix64, big_prefix2,
                  small_prefix, small_prefix2, full_prefix2, rem_prefix};
  for (int i = lo; i < hi; ++i) {
    int q[kQ];
    tiles_of(__ldcg(counts + i), q);
#pragma unroll
    for (int j = 0; j < kQ; ++j) {
      if (out[j]) out[j][i] = run[j];
      run[j] += q[j];
    }
  }
  if (threadIdx.x == nt - 1) {
#pragma unroll
    for (int j = 0; j < kQ; ++j)
      if (out[j]) out[j][N] = s_q[j][nt - 1];
  }
  __syncthreads();
}

// The sorted row of pair pidx = t * k + j: offsets[e] + the number of tokens
// below t routed to e (word prefix + popcount of the lower bits), and the
// maps between rows, tokens, pairs and gates.  debug: range checks that flag
// LMOE_DEVERR_RANGE and skip the pair.
__device__ __forceinline__ void rank_pair(long pidx, const int* idx, const float* w,
                                          const uint2* wp, const int* offsets, int T, int k, int N,
                                          int W, int* row_tok, int* row_slot, float* row_w,
                                          int* slot_row, int debug, int* err) {
  const int t = (int)(pidx / k);
  const int e = idx[pidx];
  if (debug && (e < 0 || e >= N)) {
    set_error(err, LMOE_DEVERR_RANGE);
    return;
  }
  const uint2 x = wp[(size_t)e * W + (t >> 5)];
  const int rank = (int)x.x + __popc(x.y & ((1u << (t & 31)) - 1u));
  const int row = offsets[e] + rank;
  if (debug && (row < 0 || row >= T * k)) {
    set_error(err, LMOE_DEVERR_RANGE);
    return;
  }
  if (row_tok) row_tok[row] = t;
  if (slot_row) slot_row[pidx] = row;
  row_slot[row] = (int)pidx;
  if (row_w) row_w[row] = w[pidx];
}

// logits [T, N] fp32 -> idx [T, k], w [T, k]; bitmap [N, W] gets bit t of
// token t set in the row of every chosen expert (W = ceil(T/32) words).
//
// One warp per token; lane L holds the logits of experts L, L+32, ...
// (NPL >= ceil(N/32) slots) as order-preserving 32-bit keys.
//
// Candidates: with theta the k-th largest of the 32 lane maxima, at least k
// keys are >= theta, so every one of the top k is >= theta.  When at most 64
// keys pass, they are sorted by (key, lowest expert first) and the first k
// are the answer.  Otherwise (many equal or crowded logits) a radix select
// finds the k-th largest key tau exactly (four passes over 8-bit digits, each
// a 256-bin histogram in shared memory of the keys matching the digits
// decided so far); the selection is every key above tau plus the
// lowest-indexed keys equal to tau.  Selection and order are exact integer
// operations in both branches.
//
// Variants: with sel_bias the keys are the fp32 sums logit + sel_bias[e] (the
// bias steers the choice only); the gates always come from the logits:
// renormalised over the k chosen, or (full_softmax) the softmax over all N
// logits taken at the chosen experts.
struct TopkArgs {
  const float* logits;  // [T, N]
  int T, N, k;
  const float* sel_bias;  // variants only
  int full_softmax;       // variants only
  int* idx;
  float* w;
  uint32_t* bitmap;  // [N, W]
  int W, debug;
  int* err;
  int sms;  // > 0: at most the blocks resident on this many SMs, warps striding over tokens
};

// Token t's logits, slot i of lane = expert lane + 32 i (0 past N).  Issued
// ahead of their use, so that a warp's next token loads while it ranks the
// current one.
template <int NPL>
__device__ __forceinline__ void topk_fetch(const TopkArgs& a, int t, int lane, float (&raw)[NPL]) {
  const float* lg = a.logits + (size_t)t * a.N;
#pragma unroll
  for (int i = 0; i < NPL; ++i) {
    const int e = lane + 32 * i;
    raw[i] = e < a.N ? __ldg(lg + e) : 0.f;
  }
}

template <int NPL, bool kVariant>
__device__ __forceinline__ void topk_token(const TopkArgs& a, int t, int lane,
                                           const float (&raw)[NPL], uint32_t* s_hist,
                                           unsigned long long* s_sel) {
  const int N = a.N, k = a.k;
  const float* sel_bias = kVariant ? a.sel_bias : nullptr;
  const int full_softmax = kVariant ? a.full_softmax : 0;
  const float* lg = a.logits + (size_t)t * N;
  uint32_t key[NPL];
  bool bad = false;
#pragma unroll
  for (int i = 0; i < NPL; ++i) {
    const int e = lane + 32 * i;
    key[i] = 0u;  // absent experts: 0, never above a real key and never counted
    if (e < N) {
      float v = raw[i];
      if (a.debug && !isfinite(v)) bad = true;
      if (sel_bias) v = __fadd_rn(v, __ldg(sel_bias + e));
      key[i] = orderable_bits(v);
    }
  }
  if (a.debug && __any_sync(0xffffffffu, bad) && lane == 0) set_error(a.err, LMOE_DEVERR_NONFINITE);

  uint32_t lmax = 0u;
#pragma unroll
  for (int i = 0; i < NPL; ++i) lmax = max(lmax, key[i]);
  const uint32_t theta = __shfl_sync(0xffffffffu, warp_sort_desc32(lmax, lane), k - 1);
  uint32_t sel = 0;
#pragma unroll
  for (int i = 0; i < NPL; ++i)
    if (lane + 32 * i < N && key[i] >= theta) sel |= 1u << i;
  int ncand = (int)__reduce_add_sync(0xffffffffu, (uint32_t)__popc(sel));

  if (ncand > 64 && k <= 64) {
    // A tighter lower bound on the k-th largest key: the k-th largest of the
    // lanes' two largest keys (a sub-multiset of the keys, so at most the
    // k-th largest of them all).  With k near 32 the lane maxima alone bound
    // it poorly (the k-th of 32 maxima is their smallest).
    uint32_t top2 = 0u;
    bool seen = false;  // one instance of the lane maximum skipped
#pragma unroll
    for (int i = 0; i < NPL; ++i) {
      if (lane + 32 * i < N) {
        if (!seen && key[i] == lmax) seen = true;
        else top2 = max(top2, key[i]);
      }
    }
    unsigned long long a = lmax, b = top2;
    warp_sort_desc64(a, b, lane);  // position p: lane p's a (p < 32), lane p - 32's b
    const uint32_t theta2 =
        (uint32_t)__shfl_sync(0xffffffffu, (k - 1) < 32 ? a : b, (k - 1) & 31);
    uint32_t sel2 = 0;
#pragma unroll
    for (int i = 0; i < NPL; ++i)
      if (lane + 32 * i < N && key[i] >= theta2) sel2 |= 1u << i;
    const int n2 = (int)__reduce_add_sync(0xffffffffu, (uint32_t)__popc(sel2));
    if (n2 <= 64) {
      sel = sel2;
      ncand = n2;
    }
  }

  if (ncand > 64) {
    // radix select of the k-th largest key
    uint32_t* hist = s_hist;
    uint32_t tau = 0u, tmask = 0u;
    int kk = k;  // rank of tau among the keys that match the decided digits
#pragma unroll 1
    for (int shift = 24; shift >= 0; shift -= 8) {
#pragma unroll
      for (int j = 0; j < 8; ++j) hist[lane * 8 + j] = 0u;
      __syncwarp();
#pragma unroll
      for (int i = 0; i < NPL; ++i)
        if (lane + 32 * i < N && (key[i] & tmask) == tau)
          atomicAdd(&hist[(key[i] >> shift) & 255u], 1u);
      __syncwarp();
      // lane L owns digits 255 - 8L ... 248 - 8L (descending across the warp)
      uint32_t h[8], sum = 0;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        h[j] = hist[255 - 8 * lane - j];
        sum += h[j];
      }
      uint32_t incl = sum;  // keys with digit >= this lane's lowest digit
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      const uint32_t before = incl - sum;  // keys with digit above this lane's bins
      const bool here = before < (uint32_t)kk && incl >= (uint32_t)kk;
      const int src = __ffs(__ballot_sync(0xffffffffu, here)) - 1;
      uint32_t digit = 0, above = 0;
      if (lane == src) {
        uint32_t run = before;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          if (run + h[j] >= (uint32_t)kk) {
            digit = 255 - 8 * lane - j;
            above = run;
            break;
          }
          run += h[j];
        }
      }
      digit = __shfl_sync(0xffffffffu, digit, src);
      above = __shfl_sync(0xffffffffu, above, src);
      tau |= digit << shift;
      tmask |= 255u << shift;
      kk -= (int)above;
      __syncwarp();
    }
    sel = 0;
#pragma unroll
    for (int i = 0; i < NPL; ++i)
      if (key[i] > tau) sel |= 1u << i;
    int need = kk;  // keys equal to tau still to take, lowest index first
#pragma unroll
    for (int i = 0; i < NPL; ++i) {
      if (need > 0) {
        const uint32_t tie = __ballot_sync(0xffffffffu, key[i] == tau && lane + 32 * i < N);
        if (((tie >> lane) & 1u) && __popc(tie & ((1u << lane) - 1u)) < need) sel |= 1u << i;
        need -= min(need, __popc(tie));
      }
    }
    ncand = k;
  }

  // compact the selected keys into s_sel[0..ncand) (lane-major), then sort
  const uint32_t cnt = __popc(sel);
  uint32_t incl = cnt;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  uint32_t pos = incl - cnt;
#pragma unroll
  for (int i = 0; i < NPL; ++i)
    if ((sel >> i) & 1u)
      s_sel[pos++] = ((unsigned long long)key[i] << 32) |
                          (0xFFFFFFFFu - (uint32_t)(lane + 32 * i));
  __syncwarp();
  unsigned long long v = lane < ncand ? s_sel[lane] : 0ull;
  if (ncand <= 32) {
    v = warp_sort_desc32(v, lane);
  } else {
    unsigned long long b = lane + 32 < ncand ? s_sel[lane + 32] : 0ull;
    warp_sort_desc64(v, b, lane);
  }
  const int e = (int)(0xFFFFFFFFu - (uint32_t)(v & 0xFFFFFFFFull));
  // the chosen logit of slot `lane` (the key itself unless a bias steered it)
  float val = lane < k ? from_orderable_bits((uint32_t)(v >> 32)) : -INFINITY;
  if (sel_bias && lane < k) val = __ldg(lg + e);
  float M, sum;
  if (!full_softmax) {
    M = sel_bias ? val : __shfl_sync(0xffffffffu, val, 0);  // slot 0 holds the top logit
    if (sel_bias) {
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
    }
    sum = lane < k ? expf(val - M) : 0.f;
  } else {
    // softmax over all N logits: max and sum of exp over the whole row
    M = -INFINITY;
    for (int c = lane; c < N; c += 32) M = fmaxf(M, __ldg(lg + c));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
    sum = 0.f;
    for (int c = lane; c < N; c += 32) sum += expf(__ldg(lg + c) - M);
  }
  const float ex = lane < k ? expf(val - M) : 0.f;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
  if (lane < k) {
    a.idx[(size_t)t * k + lane] = e;
    a.w[(size_t)t * k + lane] = ex / sum;
    atomicOr(a.bitmap + (size_t)e * a.W + (t >> 5), 1u << (t & 31));
  }
}

template <int NPL, bool kVariant>
__global__ void __launch_bounds__(128) topk_softmax_kernel(const TopkArgs a) {
  griddep_launch();
  griddep_wait();  // the previous kernel's outputs are visible
  __shared__ uint32_t s_hist[4][256];
  __shared__ unsigned long long s_sel[4][64];
  const int lane = threadIdx.x & 31, wib = threadIdx.x >> 5;
  // each warp takes tokens t, t + stride, ...; the next token's logits are
  // in flight while the current one is ranked
  const int stride = gridDim.x * (blockDim.x >> 5);
  int t = blockIdx.x * (blockDim.x >> 5) + wib;
  float raw[NPL];
  if (t < a.T) topk_fetch<NPL>(a, t, lane, raw);
  while (t < a.T) {
    const int tn = t + stride;
    float next[NPL];
    if (tn < a.T) topk_fetch<NPL>(a, tn, lane, next);
    topk_token<NPL, kVariant>(a, t, lane, raw, s_hist[wib], s_sel[wib]);
    if (tn < a.T) {
#pragma unroll
      for (int i = 0; i < NPL; ++i) raw[i] = next[i];
    }
    t = tn;
  }
}

// Launches topk_softmax_kernel with the smallest multiple of 4 slots per lane
// that covers N (pdl: programmatic stream serialisation).
template <int NPL, bool kVariant>
static inline cudaError_t launch_topk_npl(const TopkArgs& a, cudaStream_t st, bool pdl) {
  const auto kern = topk_softmax_kernel<NPL, kVariant>;
  int blocks = (a.T + 3) / 4;
  if (a.sms > 0 && blocks > a.sms) {
    // the blocks one wave holds (per instantiation; registers differ with NPL)
    static const int occ = [&] {
      int n = 0;
      return cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kern, 128, 0) == cudaSuccess && n > 0
                 ? n : 1;
    }();
    if (blocks > a.sms * occ) blocks = a.sms * occ;
  }
  return launch_kernel(pdl, kern, dim3(blocks), dim3(128), 0, st, a);
}

static inline cudaError_t launch_topk_args(const TopkArgs& a, cudaStream_t st, bool pdl) {
  const bool var = a.sel_bias != nullptr || a.full_softmax != 0;
  cudaError_t e = cudaSuccess;
#define LMOE_TOPK_CASE(S)                                                                   \
  case S:                                                                                   \
    e = var ? launch_topk_npl<S, true>(a, st, pdl) : launch_topk_npl<S, false>(a, st, pdl); \
    break;
  switch ((a.N + 127) / 128 * 4) {
    LMOE_TOPK_CASE(4)
    LMOE_TOPK_CASE(8)
    LMOE_TOPK_CASE(12)
    LMOE_TOPK_CASE(16)
    LMOE_TOPK_CASE(20)
    LMOE_TOPK_CASE(24)
    LMOE_TOPK_CASE(28)
    LMOE_TOPK_CASE(32)
    default:
      return cudaErrorInvalidValue;
  }
#undef LMOE_TOPK_CASE
  return e != cudaSuccess ? e : cudaGetLastError();
}

// The plain top-k launch (no fusion): logits in, indices, gates and bitmaps out.
static inline cudaError_t launch_topk(const float* logits, int T, int N, int k,
                                      const float* sel_bias, int full_softmax, int* idx, float* w,
                                      uint32_t* bitmap, int W, int debug, int* err,
                                      cudaStream_t st, bool pdl) {
  TopkArgs a;
  memset(&a, 0, sizeof a);
  a.logits = logits;
  a.T = T;
  a.N = N;
  a.k = k;
  a.sel_bias = sel_bias;
  a.full_softmax = full_softmax;
  a.idx = idx;
  a.w = w;
  a.bitmap = bitmap;
  a.W = W;
  a.debug = debug;
  a.err = err;
  return launch_topk_args(a, st, pdl);
}

// Word prefix + bits: wp[e][wd] = {set bits of expert e in words < wd, word wd}.
// Also zeroes the bitmap.  The last block scans the loads.
//
// Tile prefixes (exclusive scans over experts, entry N = the total):
//   tile_prefix      128-row tiles of every expert (single-CTA token tiles)
//   tile_prefix2     256-row tiles of every expert (CTA-pair token tiles)
//   tile_prefix64    64-row tiles of every expert (weight-stationary tiles)
//   big_prefix2      256-row tiles of the experts with > kPairMinRows rows
//   small_prefix     128-row tiles of the other experts
//   small_prefix2    256-row tiles of the other experts
// The last three split a prefill expert GEMM by load: experts with many rows
// go to the CTA-pair kernel (their last tile's padding is small against
// their rows), the rest to weight-stationary tiles of up to 128 (gated) or
// 256 rows, padded to a multiple of 16 rows.  NULL pointers skip a prefix.
static __global__ void __launch_bounds__(256) group_count_kernel(uint32_t* __restrict__ bitmap,
                                                          uint2* __restrict__ wp, int N, int W,
                                                          int* __restrict__ counts,
                                                          int* __restrict__ offsets,
                                                          int* __restrict__ tile_prefix,
                                                          int* __restrict__ tile_prefix2,
                                                          int* __restrict__ tile_prefix64,
                                                          unsigned int* done,
                                                          int* __restrict__ big_prefix2 = nullptr,
                                                          int* __restrict__ small_prefix = nullptr,
                                                          int* __restrict__ small_prefix2 = nullptr,
                                                          int* __restrict__ full_prefix2 = nullptr,
                                                          int* __restrict__ rem_prefix = nullptr) {
  griddep_launch();
  griddep_wait();  // the previous kernel's outputs are visible
  const int lane = threadIdx.x & 31;
  const int e = blockIdx.x * 8 + (threadIdx.x >> 5);
  if (e < N) {
    int running = 0;
    for (int base = 0; base < W; base += 32) {
      const int wd = base + lane;
      uint32_t bits = 0;
      if (wd < W) bits = bitmap[(size_t)e * W + wd];
      const int c = __popc(bits);
      int incl = c;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      if (wd < W) {
        wp[(size_t)e * W + wd] = make_uint2((uint32_t)(running + incl - c), bits);
        bitmap[(size_t)e * W + wd] = 0u;
      }
      running += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (lane == 0) counts[e] = running;
  }
  __threadfence();
  __syncthreads();
  __shared__ int is_last;
  if (threadIdx.x == 0) is_last = (atomicAdd(done, 1u) == gridDim.x - 1);
  __syncthreads();
  if (!is_last) return;
  __threadfence();
  scan_loads_block(counts, N, offsets, tile_prefix, tile_prefix2, tile_prefix64, big_prefix2,
                   small_prefix, small_prefix2, full_prefix2, rem_prefix);
  if (threadIdx.x == 0) *done = 0u;
}

// row(t, j) = offsets[e] + rank of t among the tokens routed to e.
static __global__ void __launch_bounds__(256) group_rank_kernel(
    const int* __restrict__ idx, const float* __restrict__ w, const uint2* __restrict__ wp,
    const int* __restrict__ offsets, int T, int k, int N, int W, int* __restrict__ row_tok,
    int* __restrict__ row_slot, float* __restrict__ row_w, int* __restrict__ slot_row, int debug,
    int* err) {
  griddep_launch();
  griddep_wait();  // the previous kernel's outputs are visible
  const long pidx = (long)blockIdx.x * blockDim.x + threadIdx.x;
  if (pidx >= (long)T * k) return;
  rank_pair(pidx, idx, w, wp, offsets, T, k, N, W, row_tok, row_slot, row_w, slot_row, debug, err);
}

}  // namespace lmoe
