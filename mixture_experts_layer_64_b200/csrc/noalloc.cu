// Routing without any device allocation: lmoe_route_only_noalloc.
//
// Some callers cannot call cudaMalloc: an inference server that reserves all
// of HBM up front for its own memory pool (a driver allocation would fail or
// fragment it), or code running where the implicit device synchronisation of
// cudaMalloc / cudaFree is not allowed.  They still want the routing steps
// (top-k, renormalised gates, expert grouping) without first creating a layer
// handle and reserving a workspace.  This entry point runs the same kernels as
// lmoe_route_only with their scratch (token bitmaps, word prefixes, counters)
// in one fixed-size file-scope device array instead of a workspace.
//
// The array is part of the library image: every GPU that loads the library
// holds it (LMOE_NOALLOC_SCRATCH_BYTES) until the process exits.  Every call
// shares it, so calls that overlap on the GPU (on different streams, or from
// different host threads) race; each call clears the parts that must start at
// zero before using them.
#include <cuda_runtime.h>

#include "../../include/lmoe.h"
#include "common.cuh"
#include "routing.cuh"

using namespace lmoe;

namespace {

// Layout of the scratch array for one call with W = ceil(T/32) words per
// expert: bitmap [N*W] u32 | word prefixes [N*W] uint2 | counts [N] |
// tile counts [N+1] | done counter.
constexpr size_t kMaxWords = LMOE_NOALLOC_MAX_WORDS;
constexpr size_t kBitmapBytes = kMaxWords * sizeof(uint32_t);
constexpr size_t kPrefixBytes = kMaxWords * sizeof(uint2);
constexpr size_t kCountBytes = LMOE_MAX_EXPERTS * sizeof(int);
constexpr size_t kTileBytes = (LMOE_MAX_EXPERTS + 1) * sizeof(int) + 12;  // + pad to 8
constexpr size_t kScratchBytes = kBitmapBytes + kPrefixBytes + kCountBytes + kTileBytes + 16;
static_assert(kScratchBytes <= LMOE_NOALLOC_SCRATCH_BYTES, "scratch size out of sync with lmoe.h");

}  // namespace

static __device__ __align__(256) unsigned char g_noalloc_scratch[LMOE_NOALLOC_SCRATCH_BYTES];

namespace {

// Device address of the scratch array on the current device.  In host code
// the array's name is only a host-side stand-in, so the address comes from
// cudaGetSymbolAddress with the device current.  It is looked up on every
// call (cheap once the module is loaded there), so a device reset, after
// which the module and its array may sit elsewhere, leaves no stale address.
lmoe_status scratch_for_current_device(unsigned char** out) {
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return LMOE_ERR_CUDA;
  *out = static_cast<unsigned char*>(p);
  return LMOE_OK;
}

}  // namespace

extern "C" lmoe_status lmoe_route_only_noalloc(const float* logits, int T, int N, int k, int* idx,
                                               float* w, int* offsets, int* perm, int* error_word,
                                               lmoe_stream_t stream) {
  if (N <= 0 || k <= 0 || k > N || T < 0 || !offsets) return LMOE_ERR_INVALID_ARG;
  if (T > 0 && (!logits || !idx || !w || !perm)) return LMOE_ERR_INVALID_ARG;
  if (N > LMOE_MAX_EXPERTS || k > LMOE_MAX_TOPK) return LMOE_ERR_UNSUPPORTED;
  const size_t W = ((size_t)T + 31) / 32;
  if ((size_t)N * W > kMaxWords) return LMOE_ERR_UNSUPPORTED;
  unsigned char* base = nullptr;
  lmoe_status st = scratch_for_current_device(&base);
  if (st != LMOE_OK) return st;
  cudaStream_t s = (cudaStream_t)stream;
  if (error_word && cudaMemsetAsync(error_word, 0, sizeof(int), s) != cudaSuccess)
    return LMOE_ERR_CUDA;
  if (T == 0) {
    return cudaMemsetAsync(offsets, 0, (size_t)(N + 1) * sizeof(int), s) == cudaSuccess
               ? LMOE_OK : LMOE_ERR_CUDA;
  }
  uint32_t* bitmap = reinterpret_cast<uint32_t*>(base);
  uint2* wp = reinterpret_cast<uint2*>(base + kBitmapBytes);
  int* counts = reinterpret_cast<int*>(base + kBitmapBytes + kPrefixBytes);
  int* tile_prefix = reinterpret_cast<int*>(base + kBitmapBytes + kPrefixBytes + kCountBytes);
  unsigned* done =
      reinterpret_cast<unsigned*>(base + kBitmapBytes + kPrefixBytes + kCountBytes + kTileBytes);
  // With an error word the kernels run their device checks and flag into it.
  const int debug = error_word ? 1 : 0;
  // The array keeps whatever the previous call left: clear the bitmap rows
  // this call sets bits in, and the block counter of the grouping scan.
  if (cudaMemsetAsync(bitmap, 0, (size_t)N * W * sizeof(uint32_t), s) != cudaSuccess ||
      cudaMemsetAsync(done, 0, sizeof(unsigned), s) != cudaSuccess)
    return LMOE_ERR_CUDA;
  if (launch_topk(logits, T, N, k, nullptr, 0, idx, w, bitmap, (int)W, debug, error_word, s,
                  false) != cudaSuccess)
    return LMOE_ERR_CUDA;
  group_count_kernel<<<(N + 7) / 8, 256, 0, s>>>(bitmap, wp, N, (int)W, counts, offsets,
                                                 tile_prefix, nullptr, nullptr, done);
  if (cudaGetLastError() != cudaSuccess) return LMOE_ERR_CUDA;
  const long P = (long)T * k;
  group_rank_kernel<<<(unsigned)((P + 255) / 256), 256, 0, s>>>(idx, w, wp, offsets, T, k, N,
                                                                 (int)W, nullptr, perm, nullptr,
                                                                 nullptr, debug, error_word);
  return cudaGetLastError() == cudaSuccess ? LMOE_OK : LMOE_ERR_CUDA;
}
