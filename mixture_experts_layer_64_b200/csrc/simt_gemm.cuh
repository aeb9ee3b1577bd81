// CUDA-core grouped GEMM with the same problem description and epilogues as
// the tcgen05 kernel.  It runs the fp32 layer (fp32 FMA accumulation; the
// tensor cores' tf32 mode would not meet fp32 accuracy) and any bf16
// contraction whose shape the tcgen05 kernel does not take (K not a multiple
// of 64).  Tile: 128 rows x 64 features, K slices of 16, 256 threads with an
// 8 x 4 register block each (two blocks for gated FC1).
#pragma once

#include "common.cuh"

namespace lmoe {

constexpr int kSimtTM = 128, kSimtTN = 64, kSimtTK = 16;

template <typename T, int kEpi>
__device__ __forceinline__ void simt_store(const GemmProblem& p, int row, int f, float v0, float v1) {
  const EpiParams& e = p.epi;
  if (kEpi == EPI_F32_BIAS) {
    static_cast<float*>(e.out)[(size_t)row * e.ldo + f] = v0 + (e.bias ? e.bias[f] : 0.f);
  } else if (kEpi == EPI_ACT) {
    const float v = apply_act<sizeof(T) == 4>(e.act, v0, v1);
    T* o = static_cast<T*>(e.out) + (size_t)row * e.ldo + e.col0 + f;
    const T hi = from_f32<T>(v);
    o[0] = hi;
    if (e.split_off) o[e.split_off] = from_f32<T>(v - to_f32<T>(hi));
  } else if (kEpi == EPI_SCALE_ROWS) {
    static_cast<T*>(e.out)[(size_t)row * e.ldo + f] = from_f32<T>(v0 * e.row_w[row]);
  } else {
    const T* rs = static_cast<const T*>(e.resid);
    static_cast<T*>(e.out)[(size_t)row * e.ldo + f] =
        from_f32<T>(to_f32<T>(rs[(size_t)row * e.ldr + f]) + v0);
  }
}

// One block per (row tile, feature tile); blocks beyond the device-side tile
// count return at once.
template <typename T, bool kDual, int kEpi>
__global__ void __launch_bounds__(256) simt_gemm_kernel(const GemmProblem p) {
  griddep_launch();
  griddep_wait();  // the previous kernel's outputs are visible
  __shared__ float As[kSimtTK][kSimtTM + 4];
  __shared__ float Bs[kDual ? 2 : 1][kSimtTK][kSimtTN + 4];
  const int NT = (p.F + kSimtTN - 1) / kSimtTN;
  const int rt = blockIdx.x / NT, ft = blockIdx.x - (blockIdx.x / NT) * NT;
  if (rt >= total_row_tiles(p)) return;
  int g, row0, rows;
  locate_row_tile(p, rt, g, row0, rows);
  const int f0 = ft * kSimtTN;
  const T* A = static_cast<const T*>(p.A);
  const T* B = static_cast<const T*>(p.B);
  const size_t wbase = (size_t)g * p.w_group_stride;
  const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;

  float acc0[8][4], acc1[8][4];
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc0[i][j] = acc1[i][j] = 0.f;

  for (int k0 = 0; k0 < p.K; k0 += kSimtTK) {
    // A tile: 128 rows x 16 k, 8 per thread
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int e = tid + 256 * i, r = e >> 4, kk = e & 15;
      float v = 0.f;
      if (r < rows && k0 + kk < p.K) {
        const size_t src = p.gather ? (size_t)p.gather[row0 + r] : (size_t)(row0 + r);
        v = to_f32<T>(A[src * p.lda + k0 + kk]);
      }
      As[kk][r] = v;
    }
    // B tile(s): 64 features x 16 k, 4 per thread
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int e = tid + 256 * i, c = e >> 4, kk = e & 15;
      const bool ok = (f0 + c < p.F) && (k0 + kk < p.K);
      Bs[0][kk][c] = ok ? to_f32<T>(B[(wbase + f0 + c) * p.K + k0 + kk]) : 0.f;
      if (kDual)
        Bs[kDual ? 1 : 0][kk][c] =
            ok ? to_f32<T>(B[(wbase + p.dual_offset + f0 + c) * p.K + k0 + kk]) : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < kSimtTK; ++kk) {
      float a[8], b0[4], b1[4];
#pragma unroll
      for (int i = 0; i < 8; ++i) a[i] = As[kk][ty * 8 + i];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        b0[j] = Bs[0][kk][tx * 4 + j];
        if (kDual) b1[j] = Bs[kDual ? 1 : 0][kk][tx * 4 + j];
      }
#pragma unroll
      for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          acc0[i][j] = fmaf(a[i], b0[j], acc0[i][j]);
          if (kDual) acc1[i][j] = fmaf(a[i], b1[j], acc1[i][j]);
        }
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int r = ty * 8 + i;
    if (r >= rows) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int f = f0 + tx * 4 + j;
      if (f < p.F) simt_store<T, kEpi>(p, row0 + r, f, acc0[i][j], kDual ? acc1[i][j] : 0.f);
    }
  }
}

}  // namespace lmoe
