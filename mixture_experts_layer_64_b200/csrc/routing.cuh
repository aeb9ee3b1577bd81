// Routing: top-k selection with renormalised gates, and the grouping of
// (token, slot) pairs by expert into a deterministic, stable permutation
// (LatentMoE paper, Section 3: the top-K index set of Eq. (1)/(2) and the
// dispatch after the down-projection).
//
//   topk_softmax_kernel   one warp per token.  Each logit becomes a 64-bit key
//                         (order-preserving fp32 bits << 32 | ~expert), so one
//                         integer max picks "largest logit, then lowest
//                         index"; -0.0 is folded into +0.0 first.  k rounds of
//                         warp max (two redux.sync each) give the slots; the gates are
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
static __global__ void __launch_bounds__(256) topk_softmax_kernel(const float* __restrict__ logits, int T,
                                                           int N, int k, int* __restrict__ idx,
                                                           float* __restrict__ w,
                                                           uint32_t* __restrict__ bitmap, int W,
                                                           int debug, int* err) {
  const int lane = threadIdx.x & 31;
  const int t = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (t >= T) return;
  const float* lg = logits + (size_t)t * N;
  unsigned long long key[32];
  unsigned long long best = 0;
  bool bad = false;
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    const int e = lane + 32 * i;
    key[i] = 0;
    if (e < N) {
      const float v = __ldg(lg + e);
      if (debug && !isfinite(v)) bad = true;
      key[i] = ((unsigned long long)orderable_bits(v) << 32) | (0xFFFFFFFFu - (uint32_t)e);
      best = key[i] > best ? key[i] : best;
    }
  }
  if (debug && __any_sync(0xffffffffu, bad) && lane == 0) set_error(err, LMOE_DEVERR_NONFINITE);
  unsigned long long mine = 0;
  for (int j = 0; j < k; ++j) {
    // warp max of the 64-bit keys as two 32-bit reductions: the value bits,
    // then the inverted index among the lanes holding that value
    const uint32_t hi = (uint32_t)(best >> 32);
    const uint32_t vmax = __reduce_max_sync(0xffffffffu, hi);
    const uint32_t imax = __reduce_max_sync(0xffffffffu, hi == vmax ? (uint32_t)best : 0u);
    const unsigned long long top = ((unsigned long long)vmax << 32) | imax;
    if (lane == j) mine = top;
    const int e = (int)(0xFFFFFFFFu - (uint32_t)(top & 0xFFFFFFFFull));
    if ((e & 31) == lane) {  // the owner drops it and rescans its keys
      best = 0;
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        if (key[i] == top) key[i] = 0;
        best = key[i] > best ? key[i] : best;
      }
    }
  }
  const int e = (int)(0xFFFFFFFFu - (uint32_t)(mine & 0xFFFFFFFFull));
  const float v = from_orderable_bits((uint32_t)(mine >> 32));
  const float l0 = __shfl_sync(0xffffffffu, v, 0);
  const float ex = lane < k ? expf(v - l0) : 0.f;
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
