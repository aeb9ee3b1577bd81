// Elementwise kernels: the gate-weighted combine (Eq. (1), the sum over the
// selected experts, in latent width), the reduction of split-K partial sums,
// and the weight repack into the K-major layout the GEMMs read.
#pragma once

#include "common.cuh"

namespace lmoe {

// comb[t, c] = (resid[t, c] +) sum_{j < k} ys[slot_row[t*k + j], c], summed in
// fp32 in slot order, rounded once.  ys rows are in expert order (as the
// expert GEMMs wrote them); slot_row maps each (token, slot) pair to its row.
// Block (t, y) covers token t's columns y*blockDim*VEC, ... with a stride of
// gridDim.y*blockDim*VEC: VEC elements per thread per step (16-byte accesses).
// With add32 (fp32, row stride ldr) that addend joins the sum before the one
// rounding: the projection-skip layer adds its shared expert this way.
template <typename T>
__global__ void __launch_bounds__(256) combine_kernel(const T* __restrict__ ys,
                                                      const int* __restrict__ slot_row, int k,
                                                      int l, const T* __restrict__ resid, long ldr,
                                                      const float* __restrict__ add32,
                                                      T* __restrict__ out, long ldo) {
  griddep_launch();
  griddep_wait();  // the previous kernel's outputs are visible
  constexpr int VEC = 16 / sizeof(T);
  const int t = blockIdx.x;
  const int* rows = slot_row + (size_t)t * k;
  for (int c = (blockIdx.y * blockDim.x + threadIdx.x) * VEC; c < l;
       c += gridDim.y * blockDim.x * VEC) {
    float acc[VEC];
    if (resid) {
      const uint4 rv = *reinterpret_cast<const uint4*>(resid + (size_t)t * ldr + c);
      const T* rb = reinterpret_cast<const T*>(&rv);
#pragma unroll
      for (int v = 0; v < VEC; ++v) acc[v] = to_f32<T>(rb[v]);
    } else {
#pragma unroll
      for (int v = 0; v < VEC; ++v) acc[v] = 0.f;
    }
    if (add32) {
#pragma unroll
      for (int v = 0; v < VEC; ++v) acc[v] += add32[(size_t)t * ldr + c + v];
    }
    // the k rows in groups of 8: a group's loads are all in flight before
    // the first is added (the sum still runs in slot order)
    for (int j0 = 0; j0 < k; j0 += 8) {
      uint4 yv[8];
#pragma unroll
      for (int jj = 0; jj < 8; ++jj)
        if (j0 + jj < k)
          yv[jj] = __ldg(reinterpret_cast<const uint4*>(ys + (size_t)__ldg(rows + j0 + jj) * l + c));
#pragma unroll
      for (int jj = 0; jj < 8; ++jj) {
        if (j0 + jj < k) {
          const T* yb = reinterpret_cast<const T*>(&yv[jj]);
#pragma unroll
          for (int v = 0; v < VEC; ++v) acc[v] += to_f32<T>(yb[v]);
        }
      }
    }
    uint4 ov;
    T* ob = reinterpret_cast<T*>(&ov);
#pragma unroll
    for (int v = 0; v < VEC; ++v) ob[v] = from_f32<T>(acc[v]);
    *reinterpret_cast<uint4*>(out + (size_t)t * ldo + c) = ov;
  }
}

// Scalar fallback of combine_kernel for widths that are not a multiple of VEC.
template <typename T>
__global__ void __launch_bounds__(256) combine_scalar_kernel(const T* __restrict__ ys,
                                                             const int* __restrict__ slot_row,
                                                             int k, int l,
                                                             const T* __restrict__ resid, long ldr,
                                                             const float* __restrict__ add32,
                                                             T* __restrict__ out, long ldo) {
  griddep_launch();
  griddep_wait();  // the previous kernel's outputs are visible
  const int t = blockIdx.x;
  for (int c = threadIdx.x; c < l; c += blockDim.x) {
    float acc = resid ? to_f32<T>(resid[(size_t)t * ldr + c]) : 0.f;
    if (add32) acc += add32[(size_t)t * ldr + c];
    for (int j = 0; j < k; ++j) acc += to_f32<T>(ys[(size_t)slot_row[(size_t)t * k + j] * l + c]);
    out[(size_t)t * ldo + c] = from_f32<T>(acc);
  }
}

// Second half of a split-K dense GEMM: sums the S fp32 slices of partial
// results part[s][row][c] (c < Fp, slice = M * Fp elements apart) in slice
// order and applies the contraction's epilogue:
//   EPI_F32_BIAS  fp32 out[row][f] = sum (+ bias[f])
//   EPI_ACT       bf16 out[row][col0 + f] = act(sum_f, sum_{f + dual})
//                 (+ its rounding residue at column col0 + split_off + f)
//   EPI_RESID     bf16 out[row][f] = resid[row][f] + sum
// F is the number of output features (Fp = F, or 2F for a gated problem
// whose gate and linear rows were computed as one).  One thread per output
// element.
__global__ void __launch_bounds__(256) splitk_reduce_kernel(const float* __restrict__ part, int S,
                                                            long slice, int M, int F, int Fp,
                                                            int dual, int kind, EpiParams e) {
  griddep_launch();
  griddep_wait();  // the previous kernel's outputs are visible
  const long i = (long)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= (long)M * F) return;
  const int row = (int)(i / F), f = (int)(i - (long)row * F);
  const float* src = part + (size_t)row * Fp + f;
  float g = 0.f, u = 0.f;
  for (int s = 0; s < S; ++s) {
    g += src[(size_t)s * slice];
    if (dual) u += src[(size_t)s * slice + dual];
  }
  if (kind == EPI_F32_BIAS) {
    static_cast<float*>(e.out)[(size_t)row * e.ldo + f] = g + (e.bias ? e.bias[f] : 0.f);
  } else if (kind == EPI_ACT) {
    const float v = apply_act(e.act, g, u);
    const bf16 hi = __float2bfloat16_rn(v);
    bf16* o = static_cast<bf16*>(e.out) + (size_t)row * e.ldo + e.col0 + f;
    o[0] = hi;
    if (e.split_off) o[e.split_off] = __float2bfloat16_rn(v - __bfloat162float(hi));
  } else {  // EPI_RESID
    const float r = __bfloat162float(static_cast<const bf16*>(e.resid)[(size_t)row * e.ldr + f]);
    static_cast<bf16*>(e.out)[(size_t)row * e.ldo + f] = __float2bfloat16_rn(r + g);
  }
}

// dst[r] = src[row_tok[r]] for the R expert-sorted rows of 16-bit elements
// (cols per row): the FC1 input rows in expert order, so that the expert
// GEMM loads them as contiguous tiles instead of gathering them by token.
// One warp per row, 16-byte vectors when cols is a multiple of 8 and both
// row strides keep 16-byte alignment.
__global__ void __launch_bounds__(256) gather_rows_kernel(const uint16_t* __restrict__ src,
                                                          long lds, const int* __restrict__ row_tok,
                                                          long R, int cols,
                                                          uint16_t* __restrict__ dst, int vec) {
  griddep_launch();
  griddep_wait();  // the previous kernel's outputs are visible
  const int lane = threadIdx.x & 31;
  const long warps = (long)gridDim.x * (blockDim.x >> 5);
  for (long r = (long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); r < R; r += warps) {
    const uint16_t* s = src + (size_t)__ldg(row_tok + r) * lds;
    uint16_t* d = dst + (size_t)r * cols;
    if (vec) {
      for (int c = lane * 8; c < cols; c += 256)
        *reinterpret_cast<uint4*>(d + c) = __ldg(reinterpret_cast<const uint4*>(s + c));
    } else {
      for (int c = lane; c < cols; c += 32) d[c] = s[c];
    }
  }
}

// bf16 -> f16 for the FC1 input of a layer with fp8 expert weights (its
// expert MMAs run on f16 operands): exact for magnitudes in [2^-14, 65504],
// an absolute error below 2^-25 under that, saturating at +-65504 above.
// vec: n is a multiple of 8 and both pointers 16-byte aligned.
__global__ void __launch_bounds__(256) bf16_to_f16_kernel(const bf16* __restrict__ in,
                                                          __half* __restrict__ out, long n,
                                                          int vec) {
  griddep_launch();
  griddep_wait();  // the previous kernel's outputs are visible
  const long i0 = ((long)blockIdx.x * blockDim.x + threadIdx.x) * (vec ? 8 : 1);
  const long stride = (long)gridDim.x * blockDim.x * (vec ? 8 : 1);
  for (long i = i0; i < n; i += stride) {
    if (vec) {
      uint4 v = *reinterpret_cast<const uint4*>(in + i);
      uint32_t* w = reinterpret_cast<uint32_t*>(&v);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float lo = __uint_as_float(w[j] << 16), hi = __uint_as_float(w[j] & 0xFFFF0000u);
        uint32_t h2;
        asm("cvt.rn.satfinite.f16x2.f32 %0, %1, %2;" : "=r"(h2) : "f"(hi), "f"(lo));
        w[j] = h2;
      }
      *reinterpret_cast<uint4*>(out + i) = v;
    } else {
      const float f = __bfloat162float(in[i]);
      out[i] = __float2half_rn(fminf(fmaxf(f, -65504.f), 65504.f));
    }
  }
}

// Self-test of the bounded waits: one thread waits on an mbarrier that no
// one arrives on; after limit_ns the wait gives up, sets the device error
// word (LMOE_DEVERR_WAIT_TIMEOUT) and the kernel returns.
__global__ void wait_selftest_kernel(int* err, unsigned long long limit_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) mbar_wait(&bar, 0, &abort_flag, err, limit_ns);
}

// out[b][c][col0 + r] = in[b][r][c] for r < rows, c < cols: the [in, out]
// API layout to the K-major [out, in] layout, batched over experts, with a
// column offset so that two matrices can share one K-concatenated operand.
template <typename T>
__global__ void transpose_kernel(const T* __restrict__ in, int rows, int cols, long in_bstride,
                                 T* __restrict__ out, long ldo, int col0, long out_bstride) {
  __shared__ T tile[32][33];
  const int b = blockIdx.z;
  const int c0 = blockIdx.x * 32, r0 = blockIdx.y * 32;
  const T* src = in + (size_t)b * in_bstride;
  T* dst = out + (size_t)b * out_bstride;
  for (int i = threadIdx.y; i < 32; i += blockDim.y) {
    const int r = r0 + i, c = c0 + threadIdx.x;
    if (r < rows && c < cols) tile[i][threadIdx.x] = src[(size_t)r * cols + c];
  }
  __syncthreads();
  for (int i = threadIdx.y; i < 32; i += blockDim.y) {
    const int c = c0 + i, r = r0 + threadIdx.x;
    if (r < rows && c < cols) dst[(size_t)c * ldo + col0 + r] = tile[threadIdx.x][i];
  }
}

}  // namespace lmoe
