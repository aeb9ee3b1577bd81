// Routing: top-k selection with renormalised gates, and the grouping of
// (token, slot) pairs by expert into a deterministic, stable permutation
// (LatentMoE paper, Section 3: the top-K index set of Eq. (1)/(2) and the
// dispatch after the down-projection).
//
//   topk_softmax_kernel   one warp per token.  Each logit becomes an
//                         order-preserving 32-bit key (-0.0 folded into +0.0);
//                         a bitwise binary search finds the k-th largest, ties
//                         go to the lowest expert index, and a bitonic sort of
//                         (key, ~expert) gives slot order.  The gates are
//                         exp(l_j - l_0) / sum over the k chosen.  Each choice
//                         sets bit t of expert e's token bitmap.
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

// logits [T, N] fp32 -> idx [T, k], w [T, k]; bitmap [N, W] gets bit t of
// token t set in the row of every chosen expert (W = ceil(T/32) words).
//
// One warp per token; lane L holds the logits of experts L, L+32, ... as
// order-preserving 32-bit keys.  The k-th largest key tau is found by a
// bitwise binary search (32 steps of per-lane counts and one warp sum); the
// selection is every key above tau plus the lowest-indexed keys equal to tau;
// a 32-lane bitonic sort of (key << 32 | ~expert) puts the k winners in slot
// order.  Selection and order are exact integer operations.
static __global__ void __launch_bounds__(256) topk_softmax_kernel(const float* __restrict__ logits,
                                                                  int T, int N, int k,
                                                                  int* __restrict__ idx,
                                                                  float* __restrict__ w,
                                                                  uint32_t* __restrict__ bitmap,
                                                                  int W, int debug, int* err) {
  __shared__ unsigned long long s_sel[8][32];
  const int lane = threadIdx.x & 31, wib = threadIdx.x >> 5;
  const int t = blockIdx.x * (blockDim.x >> 5) + wib;
  if (t >= T) return;
  const float* lg = logits + (size_t)t * N;
  uint32_t key[32];
  bool bad = false;
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    const int e = lane + 32 * i;
    key[i] = 0u;
    if (e < N) {
      const float v = __ldg(lg + e);
      if (debug && !isfinite(v)) bad = true;
      key[i] = orderable_bits(v);  // >= 1 for every non-NaN value
    }
  }
  if (debug && __any_sync(0xffffffffu, bad) && lane == 0) set_error(err, LMOE_DEVERR_NONFINITE);

  // tau: the largest value with at least k keys >= tau
  uint32_t tau = 0u;
#pragma unroll 1
  for (int b = 31; b >= 0; --b) {
    const uint32_t cand = tau | (1u << b);
    uint32_t c = 0;
#pragma unroll
    for (int i = 0; i < 32; ++i) c += key[i] >= cand ? 1u : 0u;
    if ((int)__reduce_add_sync(0xffffffffu, c) >= k) tau = cand;
  }
  uint32_t gt = 0, sel = 0;
#pragma unroll
  for (int i = 0; i < 32; ++i)
    if (key[i] > tau) {
      ++gt;
      sel |= 1u << i;
    }
  int need = k - (int)__reduce_add_sync(0xffffffffu, gt);  // ties to take, lowest index first
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    const uint32_t tie = __ballot_sync(0xffffffffu, key[i] == tau && lane + 32 * i < N);
    if (need > 0 && tie) {
      if (((tie >> lane) & 1u) && __popc(tie & ((1u << lane) - 1u)) < need) sel |= 1u << i;
      need -= min(need, __popc(tie));
    }
  }
  // compact the k selected keys into s_sel[wib][0..k) (lane-major), then sort
  const uint32_t cnt = __popc(sel);
  uint32_t incl = cnt;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  uint32_t pos = incl - cnt;
#pragma unroll
  for (int i = 0; i < 32; ++i)
    if ((sel >> i) & 1u)
      s_sel[wib][pos++] = ((unsigned long long)key[i] << 32) |
                          (0xFFFFFFFFu - (uint32_t)(lane + 32 * i));
  __syncwarp();
  unsigned long long v = lane < k ? s_sel[wib][lane] : 0ull;
  // bitonic sort, descending over the 32 lanes
#pragma unroll
  for (int size = 2; size <= 32; size <<= 1) {
#pragma unroll
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      const unsigned long long o = __shfl_xor_sync(0xffffffffu, v, stride);
      const bool desc = (lane & size) == 0;
      const bool lower = (lane & stride) == 0;
      const unsigned long long hi = v > o ? v : o, lo = v > o ? o : v;
      v = (lower == desc) ? hi : lo;
    }
  }
  const unsigned long long mine = v;
  const int e = (int)(0xFFFFFFFFu - (uint32_t)(mine & 0xFFFFFFFFull));
  const float val = from_orderable_bits((uint32_t)(mine >> 32));
  const float l0 = __shfl_sync(0xffffffffu, val, 0);
  const float ex = lane < k ? expf(val - l0) : 0.f;
  float sum = ex;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
  if (lane < k) {
    idx[(size_t)t * k + lane] = e;
    w[(size_t)t * k + lane] = ex / sum;
    atomicOr(bitmap + (size_t)e * W + (t >> 5), 1u << (t & 31));
  }
}

// Word prefix + bits: wp[e][wd] = {set bits of expert e in words < wd, word wd}.
// Also zeroes the bitmap.  The last block scans the loads.
static __global__ void __launch_bounds__(256) group_count_kernel(uint32_t* __restrict__ bitmap,
                                                          uint2* __restrict__ wp, int N, int W,
                                                          int* __restrict__ counts,
                                                          int* __restrict__ offsets,
                                                          int* __restrict__ tile_prefix,
                                                          int* __restrict__ tile_prefix2,
                                                          unsigned int* done) {
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
  // Block-wide exclusive scans of counts and of ceil(counts / 128) and
  // ceil(counts / 256) (row tiles of single CTAs and of CTA pairs).
  __shared__ int s_c[256], s_t[256], s_u[256];
  const int per = (N + 255) / 256;
  const int lo = threadIdx.x * per, hi = min(N, lo + per);
  int c_sum = 0, t_sum = 0, u_sum = 0;
  for (int i = lo; i < hi; ++i) {
    const int c = __ldcg(counts + i);
    c_sum += c;
    t_sum += (c + kRowTile - 1) / kRowTile;
    u_sum += (c + 2 * kRowTile - 1) / (2 * kRowTile);
  }
  s_c[threadIdx.x] = c_sum;
  s_t[threadIdx.x] = t_sum;
  s_u[threadIdx.x] = u_sum;
  __syncthreads();
  for (int o = 1; o < 256; o <<= 1) {
    const int a = threadIdx.x >= o ? s_c[threadIdx.x - o] : 0;
    const int b = threadIdx.x >= o ? s_t[threadIdx.x - o] : 0;
    const int d = threadIdx.x >= o ? s_u[threadIdx.x - o] : 0;
    __syncthreads();
    s_c[threadIdx.x] += a;
    s_t[threadIdx.x] += b;
    s_u[threadIdx.x] += d;
    __syncthreads();
  }
  int c_run = s_c[threadIdx.x] - c_sum, t_run = s_t[threadIdx.x] - t_sum,
      u_run = s_u[threadIdx.x] - u_sum;
  for (int i = lo; i < hi; ++i) {
    const int c = __ldcg(counts + i);
    offsets[i] = c_run;
    tile_prefix[i] = t_run;
    if (tile_prefix2) tile_prefix2[i] = u_run;
    c_run += c;
    t_run += (c + kRowTile - 1) / kRowTile;
    u_run += (c + 2 * kRowTile - 1) / (2 * kRowTile);
  }
  if (threadIdx.x == 255) {
    offsets[N] = s_c[255];
    tile_prefix[N] = s_t[255];
    if (tile_prefix2) tile_prefix2[N] = s_u[255];
    *done = 0u;
  }
}

// row(t, j) = offsets[e] + rank of t among the tokens routed to e.
static __global__ void __launch_bounds__(256) group_rank_kernel(
    const int* __restrict__ idx, const float* __restrict__ w, const uint2* __restrict__ wp,
    const int* __restrict__ offsets, int T, int k, int N, int W, int* __restrict__ row_tok,
    int* __restrict__ row_slot, float* __restrict__ row_w, int* __restrict__ slot_row, int debug,
    int* err) {
  const long pidx = (long)blockIdx.x * blockDim.x + threadIdx.x;
  if (pidx >= (long)T * k) return;
  const int t = (int)(pidx / k);
  const int e = __ldg(idx + pidx);
  if (debug && (e < 0 || e >= N)) {
    set_error(err, LMOE_DEVERR_RANGE);
    return;
  }
  const uint2 x = __ldg(wp + (size_t)e * W + (t >> 5));
  const int rank = (int)x.x + __popc(x.y & ((1u << (t & 31)) - 1u));
  const int row = __ldg(offsets + e) + rank;
  if (debug && (row < 0 || row >= T * k)) {
    set_error(err, LMOE_DEVERR_RANGE);
    return;
  }
  if (row_tok) row_tok[row] = t;
  if (slot_row) slot_row[pidx] = row;
  row_slot[row] = (int)pidx;
  if (row_w) row_w[row] = __ldg(w + pidx);
}

}  // namespace lmoe
