// Device helpers shared by the library's kernels: element types, activations,
// the epilogue parameter block, and thin inline-PTX wrappers for mbarriers,
// TMA (cp.async.bulk.tensor), cp.async and the tcgen05 tensor-core family of
// sm_100a.  Every wait on an mbarrier is bounded by wall time (globaltimer);
// on expiry it sets LMOE_DEVERR_WAIT_TIMEOUT in the device error word and
// reports failure so that the kernel can unwind instead of hanging.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/lmoe.h"

namespace lmoe {

typedef __nv_bfloat16 bf16;

enum EpiKind {
  EPI_F32_BIAS = 0,      // out_f32[r, f] = acc + bias[f]                      (router)
  EPI_ACT = 1,           // out[r, col0 + f] = act(acc) / swiglu(acc0, acc1)  (FC1, down-proj)
  EPI_SCALE_ROWS = 2,    // out[r, f] = row_w[r] * acc (rows in expert order)   (expert FC2)
  EPI_RESID = 3          // out[r, f] = resid[r, f] + acc                      (up-projection)
};
enum ActKind { ACT_NONE = -1, ACT_SILU = 0, ACT_SWIGLU = 1, ACT_RELU2 = 2 };

// Where a GEMM writes and what its epilogue mixes in.
struct EpiParams {
  void* out;              // output base (fp32 for EPI_F32_BIAS, else the layer dtype)
  long ldo;               // output row stride (elements)
  int col0;               // first output column written (EPI_ACT)
  int act;                // ActKind for EPI_ACT
  const float* bias;      // EPI_F32_BIAS, may be NULL
  const void* resid;      // EPI_RESID, row stride ldr
  long ldr;
  const float* row_w;     // EPI_SCALE_ROWS: row -> gate weight
  int split_off;          // EPI_ACT, bf16: > 0 also writes v - bf16(v) (rounded) at
                          // column col0 + split_off + f, so that hi + lo carries the
                          // value to ~16 significant bits through the next bf16 GEMM
  long slice;             // split-K partials (EPI_F32_BIAS): elements between the
                          // fp32 slices of consecutive K ranges
};

// A (possibly grouped) problem D[r, f] = sum_k A[src(r), k] * B[wrow(g, f), k]
// over the row groups [offsets[g], offsets[g+1]).  Rows are handled in tiles
// of 128 that never straddle a group; tile_prefix[g] counts the row tiles of
// the groups before g.  Without offsets the problem is one dense group of M
// rows.  Weights are K-major: group g's feature f lives in row
// g * w_group_stride + f of B (for gated FC1 the linear half starts m rows
// later: f + dual_offset).
struct GemmProblem {
  const int* offsets;     // [G+1] device, or NULL for one dense group
  const int* tile_prefix; // [G+1] device (with offsets)
  int G;
  int M;                  // rows of the dense group (offsets == NULL)
  int max_row_tiles;      // host upper bound on row tiles (grid sizing)
  int row_tile;           // rows per tile: 128, or 256 for CTA pairs (tile_prefix must match)
  const void* A;          // activations, row stride lda
  long lda;
  const int* gather;      // row -> source row of A, or NULL (identity)
  const void* B;          // K-major weights, row stride K
  long w_group_stride;
  int dual_offset;        // > 0: gated (two accumulators: f and f + dual_offset)
  int F;                  // output features
  int K;                  // reduction length
  EpiParams epi;
  int tma_store;          // token-tiled kernels: write full 32-row blocks with TMA stores
                          // (the output map is the kernel's third tensor map)
  int splits;             // dense, single-CTA token-tiled: > 1 splits K into ranges of
  int kb_per_split;       // kb_per_split 64-wide blocks, each written as an fp32 slice
  const float* w_scale;   // fp8 weights (B holds E4M3 codes): scale of weight row
                          // g * w_group_stride + f, applied to the accumulator
  int* err;               // device error word
  const uint8_t* w_exp;   // fp4 weights (B holds E2M1 code pairs, K / 2 bytes per row):
                          // E8M0 block exponents, K / 32 bytes per weight row
  int stream_k;           // weight-stationary decode tiles: stream-K work split
  float* sk_part;         // stream-K: 2 fp32 slots of kSkSlotFloats per CTA boundary
  int* sk_count;          // stream-K: one arrival counter per boundary (zero between launches)
  int rem_of;             // > 0 (grouped): the tiles cover only each group's last
                          // rows % rem_of rows (its whole rem_of-row tiles run in
                          // another launch); tile_prefix counts those tiles
};

constexpr int kRowTile = 128;
constexpr int kSwapRowTile = 64;  // rows per tile (the MMA's N, at most) of the weight-stationary kernel
// One stream-K partial accumulator of a weight-stationary tile: up to 64 rows
// x (gate, linear) x 128 features, fp32.
constexpr int kSkSlotFloats = kSwapRowTile * 2 * 128;
// Experts with more than this many rows run their prefill expert GEMMs on CTA
// pairs (256-row token tiles); the others on weight-stationary tiles whose
// row count is the expert's, rounded up to 16.  A pair tile issues its MMAs
// about a third faster than a single-CTA tile, but pads the expert's last
// tile to 256 rows: up to ~384 rows the exact-size tiles do less work.
#ifndef LMOE_PAIR_MIN_ROWS
#define LMOE_PAIR_MIN_ROWS 384
#endif
constexpr int kPairMinRows = LMOE_PAIR_MIN_ROWS;

// ---- scalar helpers ---------------------------------------------------------

template <typename T> __device__ __forceinline__ float to_f32(T v);
template <> __device__ __forceinline__ float to_f32<float>(float v) { return v; }
template <> __device__ __forceinline__ float to_f32<bf16>(bf16 v) { return __bfloat162float(v); }

template <typename T> __device__ __forceinline__ T from_f32(float v);
template <> __device__ __forceinline__ float from_f32<float>(float v) { return v; }
template <> __device__ __forceinline__ bf16 from_f32<bf16>(float v) { return __float2bfloat16_rn(v); }

// SiLU a * sigmoid(a) with the fast exponential and division intrinsics: their
// few-ulp fp32 error is far below the bf16 rounding every SiLU output gets
// (for a < -88, __expf(-a) is +inf and the quotient is 0).
__device__ __forceinline__ float silu_f(float a) { return __fdividef(a, 1.0f + __expf(-a)); }

// SiLU with the correctly rounded exponential and division (fp32 layers).
__device__ __forceinline__ float silu_precise(float a) { return a / (1.0f + expf(-a)); }

// act of one output feature; g is the gate (or only) pre-activation and u
// the linear half for SwiGLU.  kPrecise selects silu_precise.
template <bool kPrecise = false>
__device__ __forceinline__ float apply_act(int act, float g, float u) {
  switch (act) {
    case ACT_SILU: return kPrecise ? silu_precise(g) : silu_f(g);
    case ACT_SWIGLU: return (kPrecise ? silu_precise(g) : silu_f(g)) * u;
    case ACT_RELU2: return g > 0.0f ? g * g : 0.0f;
    default: return g;
  }
}

// Locates row tile `rt` in a grouped problem: group g, first row and rows.
__device__ __forceinline__ void locate_row_tile(const GemmProblem& p, int rt, int& g, int& row0,
                                                int& rows) {
  if (p.offsets == nullptr) {
    g = 0;
    row0 = rt * p.row_tile;
    rows = min(p.row_tile, p.M - row0);
    return;
  }
  int lo = 0, hi = p.G - 1;  // largest g with tile_prefix[g] <= rt
  while (lo < hi) {
    int mid = (lo + hi + 1) >> 1;
    if (__ldg(p.tile_prefix + mid) <= rt) lo = mid; else hi = mid - 1;
  }
  g = lo;
  int start = __ldg(p.offsets + g);
  const int end = __ldg(p.offsets + g + 1);
  if (p.rem_of > 0) start = end - (end - start) % p.rem_of;
  row0 = start + (rt - __ldg(p.tile_prefix + g)) * p.row_tile;
  rows = min(p.row_tile, end - row0);
}

__device__ __forceinline__ int total_row_tiles(const GemmProblem& p) {
  if (p.offsets == nullptr) return (p.M + p.row_tile - 1) / p.row_tile;
  return *((volatile const int*)(p.tile_prefix + p.G));
}

__device__ __forceinline__ void set_error(int* err, int bits) {
  if (err) atomicOr(err, bits);
}

// ---- PTX wrappers -----------------------------------------------------------

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t globaltimer() {
  uint64_t t;
  asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count)
               : "memory");
}

// ---- programmatic dependent launch ----------------------------------------------
//
// The forward's kernels are launched with programmatic stream serialisation:
// a kernel may be scheduled while its predecessor on the stream still runs,
// do its set-up that touches no global memory (barrier init, TMEM allocation,
// tensor-map prefetch), and then wait in griddep_wait until the predecessor
// has completed and its writes are visible.  Every kernel calls griddep_wait
// before its first global load or store; launched without the attribute, the
// wait returns at once.  griddep_launch lets the next kernel be scheduled once
// every CTA of this grid has issued it (all of them are then resident), so a
// waiting successor never holds resources this grid still needs.
__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void griddep_launch() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// Launches kernel `kern` on stream st, with programmatic stream serialisation
// when pdl is set (the kernel must then call griddep_wait before touching
// global memory, as every forward kernel does).
template <typename... KArgs, typename... Args>
inline cudaError_t launch_kernel(bool pdl, void (*kern)(KArgs...), dim3 grid, dim3 block,
                                 size_t smem, cudaStream_t st, Args... args) {
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kern, args...);
}

__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Wall-time limit of one mbarrier wait (ns).  No legitimate wait in these
// kernels lasts more than a few milliseconds.
constexpr uint64_t kWaitLimitNs = 2000000000ull;

// Bounded wait on `bar` reaching phase parity `parity`.  Returns false (after
// flagging the error word and the block-wide abort flag) on expiry, or
// immediately when another thread of the block has already aborted.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                          int* err, uint64_t limit_ns = kWaitLimitNs) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer();
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 255u) == 0) {
      if (*abort_flag) return false;
      if (globaltimer() - t0 > limit_ns) {
        *abort_flag = 1;
        set_error(err, LMOE_DEVERR_WAIT_TIMEOUT);
        return false;
      }
    }
  }
}

// Bounded wait that ignores the abort flag: used while draining in-flight
// asynchronous work before the block exits.
__device__ __forceinline__ bool mbar_wait_drain(uint64_t* bar, uint32_t parity) {
  const uint64_t t0 = globaltimer();
  for (uint32_t it = 0;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 255u) == 255u && globaltimer() - t0 > kWaitLimitNs) return false;
  }
}

__device__ __forceinline__ void tma_load_2d(const CUtensorMap* map, uint64_t* bar, void* smem_dst,
                                            int c0, int c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(c0), "r"(c1)
      : "memory");
}

// TMA row gather: four rows r0..r3 (any order, each a one-row box of the
// tensor map starting at column c0) land as four consecutive rows at
// smem_dst, swizzled by their shared-memory address as a four-row box would
// be; completion is counted on `bar` (4 x box bytes).
__device__ __forceinline__ void tma_gather4(const CUtensorMap* map, uint64_t* bar, void* smem_dst,
                                            int c0, int r0, int r1, int r2, int r3) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile::gather4.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5, %6, %7}], [%2];" ::"r"(smem_u32(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(c0), "r"(r0), "r"(r1),
      "r"(r2), "r"(r3)
      : "memory");
}

// Bulk tensor store of a shared-memory box to global memory (async proxy).
__device__ __forceinline__ void tma_store_2d(const CUtensorMap* map, const void* smem_src, int c0,
                                             int c1) {
  asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.tile.bulk_group [%0, {%1, %2}], [%3];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(c0), "r"(c1), "r"(smem_u32(smem_src))
               : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// wait until the sources of all committed bulk stores have been read
__device__ __forceinline__ void bulk_wait_read0() {
  asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}
// wait until all committed bulk stores have completed
__device__ __forceinline__ void bulk_wait0() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

__device__ __forceinline__ void prefetch_tensormap(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// 16-byte cp.async with zero fill of the (16 - src_bytes) tail.
__device__ __forceinline__ void cp_async_16(void* smem_dst, const void* gsrc, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(smem_dst)),
               "l"(gsrc), "r"(src_bytes)
               : "memory");
}
// Arrive on `bar` once every cp.async this thread issued so far has landed
// (the pending count is raised first, so the phase waits for the copies; the
// thread's own mbarrier.arrive is still needed to count it).
__device__ __forceinline__ void cp_async_mbar_arrive(uint64_t* bar) {
  asm volatile("cp.async.mbarrier.arrive.shared::cta.b64 [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ---- clusters (CTA pairs of the 2-SM MMA) ------------------------------------

__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ uint32_t cluster_id_x() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%clusterid.x;" : "=r"(r));
  return r;
}
__device__ __forceinline__ uint32_t cluster_count_x() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%nclusterid.x;" : "=r"(r));
  return r;
}
// shared::cluster address of the same shared variable in CTA `rank` of the cluster
__device__ __forceinline__ uint32_t cluster_map(const void* smem_ptr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_u32(smem_ptr)), "r"(rank));
  return r;
}
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::
                   : "memory");
}
// arrive on an mbarrier given by its shared::cluster address (possibly in the peer CTA)
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr)
               : "memory");
}
__device__ __forceinline__ bool mbar_try_wait_cluster(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
// Bounded wait with cluster-scope acquire (arrivals may come from the peer CTA).
__device__ __forceinline__ bool mbar_wait_cluster(uint64_t* bar, uint32_t parity,
                                                  volatile int* abort_flag, int* err) {
  if (mbar_try_wait_cluster(bar, parity)) return true;
  const uint64_t t0 = globaltimer();
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait_cluster(bar, parity)) return true;
    if ((it & 255u) == 0) {
      if (*abort_flag) return false;
      if (globaltimer() - t0 > kWaitLimitNs) {
        *abort_flag = 1;
        set_error(err, LMOE_DEVERR_WAIT_TIMEOUT);
        return false;
      }
    }
  }
}
// 2-SM TMA load into this CTA's shared memory; completion is counted on the
// mbarrier at shared::cluster address `bar_cluster` (the pair's leader).
__device__ __forceinline__ void tma_load_2d_pair(const CUtensorMap* map, uint32_t bar_cluster,
                                                 void* smem_dst, int c0, int c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.cta_group::2"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar_cluster), "r"(c0), "r"(c1)
      : "memory");
}

// tcgen05 (5th-generation tensor cores, tensor memory).
__device__ __forceinline__ void tmem_alloc(uint32_t* smem_slot, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                   smem_u32(smem_slot)),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
// D(tmem) (+)= A(smem desc) * B(smem desc)^T, bf16 inputs, fp32 accumulate.
__device__ __forceinline__ void tc_mma_bf16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                            uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// Arrive on `bar` once all previously issued tcgen05.mma of this thread finish.
__device__ __forceinline__ void tc_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   smem_u32(bar))
               : "memory");
}
// 2-SM variants: the pair's TMEM is allocated by one warp in each CTA; MMAs
// are issued by the leader and read operands from both CTAs' shared memory.
__device__ __forceinline__ void tmem_alloc_pair(uint32_t* smem_slot, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                   smem_u32(smem_slot)),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish_pair() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tc_mma_bf16_pair(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                                 uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// Arrive on `bar` (same offset) in every CTA of ctaMask once the pair's
// previously issued MMAs finish.
__device__ __forceinline__ void tc_commit_pair_mc(uint64_t* bar, uint16_t cta_mask) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 "
      "[%0], %1;" ::"r"(smem_u32(bar)),
      "h"(cta_mask)
      : "memory");
}

__device__ __forceinline__ void tc_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tc_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// D(tmem) (+)= A(tmem) * B(smem desc)^T, f16 inputs, fp32 accumulate: the A
// operand (M rows = lanes, K along the columns, two f16 per 32-bit column)
// read from tensor memory.
__device__ __forceinline__ void tc_mma_f16_tmem_a(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                                  uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// 32 lanes x 32 consecutive 32-bit columns from registers: thread i of the
// warp writes lane (taddr.lane + i), columns [taddr.col, taddr.col + 32).
__device__ __forceinline__ void tmem_st_32x32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
      "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]),
      "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]),
      "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}

// 32 lanes x 32 consecutive fp32 columns: thread i of the warp receives lane
// (taddr.lane + i), columns [taddr.col, taddr.col + 32).
__device__ __forceinline__ void tmem_ld_32x32(uint32_t taddr, float* v) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

// Shared-memory matrix descriptor of a K-major operand tile written with the
// 128-byte swizzle (rows of 64 bf16 = 128 B, 8-row atoms of 1024 B): start
// address, leading-byte offset 16 B (unused for swizzled K-major), stride
// byte offset 1024 B between 8-row groups, descriptor version 1 (sm_100),
// layout type 2 = SWIZZLE_128B.
__device__ __forceinline__ uint64_t smem_desc_sw128(const void* smem_tile) {
  const uint64_t addr = smem_u32(smem_tile);
  uint64_t desc = 0;
  desc |= (addr >> 4) & 0x3FFFull;            // bits [0,14)  start address >> 4
  desc |= (uint64_t)(16 >> 4) << 16;          // bits [16,30) leading byte offset >> 4
  desc |= (uint64_t)(1024 >> 4) << 32;        // bits [32,46) stride byte offset >> 4
  desc |= (uint64_t)1 << 46;                  // bits [46,48) version = 1
  desc |= (uint64_t)2 << 61;                  // bits [61,64) SWIZZLE_128B
  return desc;
}

// Instruction descriptor of tcgen05.mma kind::f16: bf16 A and B, fp32 D,
// both operands K-major, shape M x N.
__device__ __forceinline__ uint32_t idesc_bf16_f32(int M, int N) {
  uint32_t d = 0;
  d |= 1u << 4;                       // D format: F32
  d |= 1u << 7;                       // A format: BF16
  d |= 1u << 10;                      // B format: BF16
  d |= (uint32_t)(N >> 3) << 17;      // N >> 3
  d |= (uint32_t)(M >> 4) << 24;      // M >> 4
  return d;
}
// The same with f16 A and B (format code 0).
__device__ __forceinline__ uint32_t idesc_f16_f32(int M, int N) {
  uint32_t d = 0;
  d |= 1u << 4;                       // D format: F32
  d |= (uint32_t)(N >> 3) << 17;      // N >> 3
  d |= (uint32_t)(M >> 4) << 24;      // M >> 4
  return d;
}

}  // namespace lmoe
