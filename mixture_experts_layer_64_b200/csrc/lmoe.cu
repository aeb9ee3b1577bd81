// Host side of the LatentMoE layer library: the handle, weight repack,
// workspace, per-call kernel selection and the C ABI declared in lmoe.h.
//
// One forward pass (LatentMoE paper, Section 3, Eq. (1)/(2), plus the
// residual add) is this sequence of launches on the caller's stream:
//   1 router GEMM            logits[T,N] fp32 = x Wg + bias
//   2 top-k + softmax        idx, w, per-expert token bitmaps
//   3 grouping               word prefixes, offsets, tile counts; sorted rows
//   4 down-projection GEMM   z[T,l] = x Wdown                 (not when skipped)
//   5 shared FC1 GEMM        hs = act(x Ws1) into cat[:, l:] as bf16 hi + lo pairs
//   6 expert FC1 (grouped)   h[r] = act(z[tok(r)] W1[e])      rows gathered by token
//   7 expert FC2 (grouped)   ys[r] = w(r) * (h[r] W2[e])         rows in expert order
//   8 combine                cat[t, :l] = sum_j ys[row(t, j)] (skipped projections:
//                            out = x + sum (+ the shared expert, computed in fp32 at 5))
//   9 up-projection GEMM     out = x + [comb | hs_hi | hs_lo] [Wup ; Ws2 ; Ws2]
// Contractions run on the tcgen05 kernel (bf16) or the CUDA-core kernel
// (fp32, or shapes the tcgen05 kernel does not take).
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <string>
#include <vector>

#include "../../include/lmoe.h"
#include "common.cuh"
#include "ep.cuh"
#include "misc.cuh"
#include "routing.cuh"
#include "simt_gemm.cuh"
#include "tc_gemm.cuh"

using namespace lmoe;

namespace {

constexpr int kStages = 9;  // profiled stage count (10 boundaries)
// events per profiled forward: the 10 stage boundaries on the caller's stream,
// then the side stream's start, "down-projection done" and end
constexpr int kMarks = kStages + 4;
constexpr int kSideMark0 = kStages + 1;
const char* kStageNames[kStages] = {"router",     "topk",       "group",   "down_proj", "shared_fc1",
                                    "expert_fc1", "expert_fc2", "combine", "up_proj"};

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

}  // namespace

// The row grouping an expert GEMM runs over: G groups (experts e0 .. e0 +
// G - 1 of the weight stacks), their row offsets, and the tile counts of each
// tile size (exclusive prefixes over the groups, see group_count_kernel).
struct Grouping {
  int G = 0, e0 = 0;
  const int *offsets = nullptr, *tp128 = nullptr, *tp256 = nullptr, *tp64 = nullptr;
  const int *big256 = nullptr, *small128 = nullptr, *small256 = nullptr;
  // the split expert FC2 (LMOE_FC2_SPLIT): 256-row pair tiles of every
  // group (the last one only if more than 128 rows are left for it), and
  // one 128-row tile of the last rows % 256 of the groups where those are
  // at most 128
  const int *full256 = nullptr, *rem128 = nullptr;
};

struct lmoe_layer {
  int d, l, N, k, m, act, shared_m, dtype;
  unsigned flags;
  int m_in, ms_in, Kup, es;  // es: element size
  bool split_shared = false;  // bf16 shared hidden carried as a hi + lo pair
  bool pdl = true;            // forward kernels with programmatic dependent launch
  bool pdl_hold = false;      // the next launch follows a cross-stream wait (or opens a
                              // forward): launched with the full stream dependency
  int device = 0, num_sms = 148;
  bool weights_set = false;
  // weights, K-major
  void* Wg_t = nullptr;   // [N, d]
  float* bias = nullptr;  // [N]
  void* Wd_t = nullptr;   // [l, d]
  void* Wu_t = nullptr;   // [d, Kup]: [Wup^T | Ws2^T]
  void* Ws1_t = nullptr;  // [ms_in, d]
  void* W1_t = nullptr;   // [N * m_in, l]
  void* W2_t = nullptr;   // [N * l, m]
  // fp8 expert weights (LMOE_EXPERTS_FP8): E4M3 codes in the same K-major
  // layouts, and one fp32 scale per weight row (output channel)
  uint8_t* W1q_t = nullptr;  // [N * m_in, l]
  uint8_t* W2q_t = nullptr;  // [N * l, m]
  float* W1s = nullptr;      // [N * m_in]
  float* W2s = nullptr;      // [N * l]
  bool fp8_set = false;
  // block-scaled fp4 expert weights (LMOE_EXPERTS_FP4): E2M1 code pairs and
  // E8M0 block exponents, K-major as the caller passes them
  uint8_t* W1q4_t = nullptr;  // [N * m_in, l / 2]
  uint8_t* W1e_t = nullptr;   // [N * m_in, l / 32]
  uint8_t* W2q4_t = nullptr;  // [N * l, m / 2]
  uint8_t* W2e_t = nullptr;   // [N * l, m / 32]
  bool fp4_set = false;
  void* a16 = nullptr;       // fp8 / fp4 experts: the FC1 input rows in f16 [T, l or d]
  void* zs = nullptr;        // LMOE_SORTED_ROWS: the FC1 input rows in expert order [T*k, l or d]
  // workspace
  int max_T = 0, W = 0;
  float* logits = nullptr;
  int* idx = nullptr;
  float* w = nullptr;
  uint32_t* bitmap = nullptr;
  uint2* wp = nullptr;
  int *counts = nullptr, *offsets = nullptr, *tile_prefix = nullptr, *tile_prefix2 = nullptr;
  int* tile_prefix64 = nullptr;  // 64-row tile counts (weight-stationary kernel)
  // prefill expert GEMMs split by load: 256-row tiles of the experts with
  // more than kPairMinRows rows (CTA pairs), 128- and 256-row tiles of the
  // others (weight-stationary, single CTA)
  int *big_prefix2 = nullptr, *small_prefix = nullptr, *small_prefix2 = nullptr;
  // the expert FC2 split into whole 256-row pair tiles and 128-row tiles of
  // the rest (LMOE_FC2_SPLIT)
  int *full_prefix2 = nullptr, *rem_prefix = nullptr;
  // stream-K split of the weight-stationary decode GEMMs: two partial
  // accumulator slots and one arrival counter per boundary between CTAs
  float* sk_part = nullptr;
  int* sk_count = nullptr;
  // the forward's expert grouping (all N experts, the routing's prefixes)
  Grouping fwd_grp;
  // expert parallelism: the received rows' grouping over the local experts
  // and the expert-side workspace (lmoe_ep_reserve)
  Grouping ep_grp;
  int ep_max_rows = 0;
  int* ep_tab = nullptr;        // device: counts [N] | src_start [N+1] | roff [N] | goff [N] |
                                // offsets [N+1] | 6 tile prefixes [N+1]
  int* ep_tab_host = nullptr;   // pinned staging of the first four tables
  cudaEvent_t ep_uploaded = nullptr;  // the last upload from ep_tab_host has been read
  int *ep_perm = nullptr, *ep_inv = nullptr;  // grouped row <-> received row
  float* ep_gates = nullptr;                  // gates in grouped order
  void *ep_h = nullptr, *ep_ys = nullptr;     // FC1 output, FC2 output (grouped)
  int ep_T = -1;                              // the pending dispatch's T (-1: none)
  unsigned* done = nullptr;
  int* err = nullptr;
  int *row_tok = nullptr, *row_slot = nullptr, *slot_row = nullptr;
  float* row_w = nullptr;
  void *z = nullptr, *h = nullptr, *ys = nullptr, *cat = nullptr;
  void *x_stage = nullptr, *out_stage = nullptr;
  // host entry: a second x staging slot, a copy stream for the uploads, and
  // per slot "upload done" / "forward done reading the slot" events
  void* x_stage2 = nullptr;
  cudaStream_t copy_stream = nullptr;
  cudaEvent_t ev_up[2] = {nullptr, nullptr}, ev_used[2] = {nullptr, nullptr};
  int host_slot = 0;
  float* s32 = nullptr;  // [T, d] fp32 shared-expert output (projection-skip layers)
  float* part = nullptr;  // split-K partial sums of the dense GEMMs at small T
  size_t part_bytes = 0;
  // the stages that read only x (down-projection, shared expert FC1) run on a
  // second stream beside the router and routing steps: the stream, its own
  // split-K partial buffer, and the fork and join events
  cudaStream_t side_stream = nullptr;
  float* part_side = nullptr;
  cudaEvent_t ev_fork = nullptr, ev_side = nullptr;
  // bookkeeping
  int last_T = -1, launches = 0, expert_path = -1;
  std::string detail;
  // profiling
  std::vector<cudaEvent_t> events;
  std::vector<char> prof_side;  // per profiled forward: the side stream ran
  unsigned prof_mask = 0;       // the stages whose boundaries are recorded
  int prof_cap = 0, prof_count = 0;
  bool profiling = false;
};

namespace {

struct DevGuard {
  int prev = -1;
  bool changed = false;
  explicit DevGuard(int dev) {
    if (cudaGetDevice(&prev) == cudaSuccess && prev != dev) {
      changed = cudaSetDevice(dev) == cudaSuccess;
    }
  }
  ~DevGuard() {
    if (changed) cudaSetDevice(prev);
  }
};

lmoe_status cuda_fail(lmoe_layer* h, cudaError_t e, const char* what) {
  if (h) h->detail = std::string(what) + ": " + cudaGetErrorString(e);
  return e == cudaErrorMemoryAllocation ? LMOE_ERR_OOM : LMOE_ERR_CUDA;
}

#define LMOE_TRY(expr)               \
  do {                               \
    lmoe_status s_ = (expr);         \
    if (s_ != LMOE_OK) return s_;    \
  } while (0)

#define LMOE_CUDA(h, call)                                 \
  do {                                                     \
    cudaError_t e_ = (call);                               \
    if (e_ != cudaSuccess) return cuda_fail((h), e_, #call); \
  } while (0)

// A launch through launch_kernel (forward kernels: programmatic stream
// serialisation unless LMOE_NO_PDL).
#define LMOE_LAUNCH(h, ...)                                             \
  do {                                                                  \
    cudaError_t e_ = launch_kernel(take_pdl(h), __VA_ARGS__);           \
    if (e_ != cudaSuccess) return cuda_fail((h), e_, "kernel launch"); \
    ++(h)->launches;                                                    \
  } while (0)

#define LMOE_CHECK_LAUNCH(h)                                           \
  do {                                                                 \
    cudaError_t e_ = cudaGetLastError();                               \
    if (e_ != cudaSuccess) return cuda_fail((h), e_, "kernel launch"); \
    ++(h)->launches;                                                   \
  } while (0)

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

// Whether the next launch may use programmatic dependent launch; a pending
// hold (set after a cross-stream wait and at the start of a forward) makes
// that one launch wait for everything before it on its stream.
bool take_pdl(lmoe_layer* h) {
  const bool use = h->pdl && !h->pdl_hold;
  h->pdl_hold = false;
  return use;
}

// ---- GEMM dispatch --------------------------------------------------------------

enum GemmKind { GK_ROUTER, GK_DENSE_ACT, GK_FC1, GK_FC2, GK_UP };

struct GemmCall {
  GemmProblem p;
  GemmKind kind;
  long a_rows;  // rows of A (TMA bounds)
  long b_rows;  // rows of B (TMA bounds)
  long out_rows;  // rows of the output (TMA store bounds)
  bool swap;    // weight-stationary expert kernels
  bool pair;    // 2-SM token-tiled kernels on CTA pairs (256-row tiles)
  bool ws_pair;  // grouped: weight-stationary kernel on CTA pairs (rows on N)
  int wide;      // grouped, swap: weight-stationary tiles of up to 128 / 256 rows
                 // (0: the decode kernel's 64-row tiles)
  bool side;     // enqueued on the side stream: split-K uses the side partial buffer
  const Grouping* grp;  // grouped calls: the grouping (tile prefixes)
};

bool encode_map(CUtensorMap* map, const void* ptr, long rows, int cols, long ld, int box_rows) {
  EncodeTiledFn fn = get_encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)ld * 2};
  cuuint32_t box[2] = {64, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// fp8 E4M3 weights: rows of `cols` one-byte codes, 64-code (64-byte) boxes of
// box_rows rows, no swizzle (the converter warps re-lay them out as f16 in
// shared memory), or the 64-byte swizzle (sw64: the converters of the
// weight-stationary kernels read one row per thread into tensor memory).
bool encode_map_u8(CUtensorMap* map, const void* ptr, long rows, int cols, long ld, int box_rows,
                   bool sw64) {
  EncodeTiledFn fn = get_encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)ld};
  cuuint32_t box[2] = {64, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(ptr), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
            sw64 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_NONE,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// fp4 weights: rows of `cols` bytes (code pairs, or block exponents), boxes of
// box_cols bytes x box_rows rows, with the 32-byte swizzle (code pairs: the
// converters read one 32-byte row per thread) or none (exponents).
bool encode_map_fp4(CUtensorMap* map, const void* ptr, long rows, int cols, int box_cols,
                    int box_rows, bool sw32) {
  EncodeTiledFn fn = get_encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)cols};
  cuuint32_t box[2] = {(cuuint32_t)box_cols, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(ptr), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
            sw32 ? CU_TENSOR_MAP_SWIZZLE_32B : CU_TENSOR_MAP_SWIZZLE_NONE,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Output map of the TMA-store epilogue: 32 x 32 boxes, 64-byte swizzle for
// bf16 (64-byte rows), 128-byte swizzle for fp32 (128-byte rows).
bool encode_out_map(CUtensorMap* map, const GemmCall& c) {
  EncodeTiledFn fn = get_encode_fn();
  if (!fn) return false;
  const bool f32 = c.kind == GK_ROUTER;
  const size_t es = f32 ? 4 : 2;
  const char* base = static_cast<const char*>(c.p.epi.out) +
                     (c.kind == GK_DENSE_ACT || c.kind == GK_FC1 ? (size_t)c.p.epi.col0 * es : 0);
  cuuint64_t dims[2] = {(cuuint64_t)c.p.F, (cuuint64_t)c.out_rows};
  cuuint64_t strides[1] = {(cuuint64_t)c.p.epi.ldo * es};
  cuuint32_t box[2] = {32, 32};
  cuuint32_t estr[2] = {1, 1};
  return fn(map, f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
            const_cast<char*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
            f32 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B,
            CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Whether a token-tiled call can write its output with TMA stores.
bool tma_store_ok(const GemmCall& c) {
  const EpiParams& e = c.p.epi;
  if (c.swap || e.split_off) return false;
  const size_t es = c.kind == GK_ROUTER ? 4 : 2;
  const char* base = static_cast<const char*>(e.out) +
                     (c.kind == GK_DENSE_ACT || c.kind == GK_FC1 ? (size_t)e.col0 * es : 0);
  return aligned16(base) && ((size_t)e.ldo * es) % 16 == 0 && (c.p.F * es) % 16 == 0;
}

// Function attributes and occupancy are per device: the launch helpers
// keep what they set up per device ordinal (below kMaxDevices).
constexpr int kMaxDevices = 64;

template <class Cfg>
lmoe_status launch_tc(lmoe_layer* h, const GemmCall& c, cudaStream_t st) {
  static bool attr_done[kMaxDevices] = {};
  bool& done = attr_done[h->device % kMaxDevices];
  if (!done) {
    LMOE_CUDA(h, cudaFuncSetAttribute(tc_gemm_kernel<Cfg>,
                                      cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      Cfg::SMEM_BYTES));
    done = true;
  }
  CUtensorMap ta, tb;
  std::memset(&ta, 0, sizeof ta);
  std::memset(&tb, 0, sizeof tb);
  // activations: 32- or 128-row boxes, or (gathered rows) one-row boxes for
  // the four-row TMA gather
  if (!encode_map(&ta, c.p.A, c.a_rows, c.p.K, c.p.lda,
                  Cfg::kGather ? 1 : (Cfg::kSwap ? 32 : 128))) {
    h->detail = "cuTensorMapEncodeTiled (activations) failed";
    return LMOE_ERR_CUDA;
  }
  const bool wmap =
      Cfg::kFp4 ? encode_map_fp4(&tb, c.p.B, c.b_rows, c.p.K / 2, 32, Cfg::W_ROWS, Cfg::kTmemA)
      : Cfg::kFp8 ? encode_map_u8(&tb, c.p.B, c.b_rows, c.p.K, c.p.K, Cfg::W_ROWS, Cfg::kTmemA)
                  : encode_map(&tb, c.p.B, c.b_rows, c.p.K, c.p.K, Cfg::W_ROWS);
  if (!wmap) {
    h->detail = "cuTensorMapEncodeTiled (weights) failed";
    return LMOE_ERR_CUDA;
  }
  CUtensorMap tc;
  std::memset(&tc, 0, sizeof tc);
  GemmProblem p = c.p;
  p.tma_store = (!Cfg::kSwap && !Cfg::kFp4 && tma_store_ok(c) && encode_out_map(&tc, c)) ? 1 : 0;
  // fp4 weights: the kernel's third map holds the block exponents (its
  // epilogue then stores with plain stores)
  if (Cfg::kFp4 &&
      !encode_map_fp4(&tc, c.p.w_exp, c.b_rows, c.p.K / 32, 16, Cfg::W_ROWS, false)) {
    h->detail = "cuTensorMapEncodeTiled (fp4 exponents) failed";
    return LMOE_ERR_CUDA;
  }
  const long NT = (c.p.F + Cfg::FT - 1) / Cfg::FT;
  const long tiles = (long)c.p.max_row_tiles * NT * std::max(1, c.p.splits);
  const int grid = (int)std::max(1L, std::min<long>(h->num_sms, tiles));
  LMOE_LAUNCH(h, tc_gemm_kernel<Cfg>, dim3(grid), dim3(Cfg::THREADS), Cfg::SMEM_BYTES, st, ta, tb,
              tc, p);
  return LMOE_OK;
}

// Largest number of co-resident CTA pairs of a 2-SM kernel (cluster size 2).
template <typename Kern>
lmoe_status pair_setup(lmoe_layer* h, Kern kern, int smem_bytes, int* max_clusters) {
  LMOE_CUDA(h, cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_bytes));
  LMOE_CUDA(h, cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 0));
  cudaLaunchConfig_t q = {};
  cudaLaunchAttribute qa[1];
  qa[0].id = cudaLaunchAttributeClusterDimension;
  qa[0].val.clusterDim.x = 2;
  qa[0].val.clusterDim.y = 1;
  qa[0].val.clusterDim.z = 1;
  q.gridDim = dim3(2 * (h->num_sms / 2), 1, 1);
  q.blockDim = dim3(kTcThreads, 1, 1);
  q.dynamicSmemBytes = smem_bytes;
  q.attrs = qa;
  q.numAttrs = 1;
  LMOE_CUDA(h, cudaOccupancyMaxActiveClusters(max_clusters, kern, &q));
  if (*max_clusters < 1) {
    h->detail = "no CTA pair of the 2-SM kernel fits on the device";
    return LMOE_ERR_UNSUPPORTED;
  }
  return LMOE_OK;
}

// Launches `clusters` CTA pairs of a 2-SM kernel (programmatic stream
// serialisation unless LMOE_NO_PDL).
template <typename Kern, typename... Args>
lmoe_status pair_launch(lmoe_layer* h, Kern kern, int smem_bytes, long clusters, cudaStream_t st,
                        Args... args) {
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.gridDim = dim3((unsigned)(2 * clusters), 1, 1);
  cfg.blockDim = dim3(kTcThreads, 1, 1);
  cfg.dynamicSmemBytes = smem_bytes;
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = take_pdl(h) ? 2 : 1;
  LMOE_CUDA(h, cudaLaunchKernelEx(&cfg, kern, args...));
  ++h->launches;
  return LMOE_OK;
}

template <class Cfg>
lmoe_status launch_pair(lmoe_layer* h, const GemmCall& c, cudaStream_t st) {
  static int clusters_of[kMaxDevices] = {};
  int& max_clusters = clusters_of[h->device % kMaxDevices];
  if (max_clusters == 0)
    LMOE_TRY(pair_setup(h, tc_gemm_pair_kernel<Cfg>, Cfg::SMEM_BYTES, &max_clusters));
  CUtensorMap ta, tb;
  std::memset(&ta, 0, sizeof ta);
  std::memset(&tb, 0, sizeof tb);
  // gathered rows (kGather) are fetched by cp.async: no activation map
  if ((!Cfg::kGather && !encode_map(&ta, c.p.A, c.a_rows, c.p.K, c.p.lda, 128)) ||
      !encode_map(&tb, c.p.B, c.b_rows, c.p.K, c.p.K, 128)) {
    h->detail = "cuTensorMapEncodeTiled failed";
    return LMOE_ERR_CUDA;
  }
  const long NT = (c.p.F + Cfg::FT - 1) / Cfg::FT;
  const long tiles = (long)c.p.max_row_tiles * NT;
  const long clusters = std::max(1L, std::min<long>(max_clusters, tiles));
  CUtensorMap tc;
  std::memset(&tc, 0, sizeof tc);
  GemmProblem p = c.p;
  p.tma_store = (tma_store_ok(c) && encode_out_map(&tc, c)) ? 1 : 0;
  return pair_launch(h, tc_gemm_pair_kernel<Cfg>, Cfg::SMEM_BYTES, clusters, st, ta, tb, tc, p);
}

// Grouped expert GEMM, weight-stationary on CTA pairs: the expert's rows are
// split into ceil(rows / NMAX) tiles, whose counts are the 128- or 256-row
// tile prefix of the grouping step.
template <class Cfg>
lmoe_status launch_pair_ws(lmoe_layer* h, const GemmCall& c, cudaStream_t st) {
  static int clusters_of[kMaxDevices] = {};
  int& max_clusters = clusters_of[h->device % kMaxDevices];
  if (max_clusters == 0)
    LMOE_TRY(pair_setup(h, tc_gemm_pair_ws_kernel<Cfg>, Cfg::SMEM_BYTES, &max_clusters));
  CUtensorMap ta, tb;
  std::memset(&ta, 0, sizeof ta);
  std::memset(&tb, 0, sizeof tb);
  if ((!Cfg::kGather && !encode_map(&ta, c.p.A, c.a_rows, c.p.K, c.p.lda, 32)) ||
      !encode_map(&tb, c.p.B, c.b_rows, c.p.K, c.p.K, 128)) {
    h->detail = "cuTensorMapEncodeTiled failed";
    return LMOE_ERR_CUDA;
  }
  GemmProblem p = c.p;
  p.tile_prefix = Cfg::NMAX == 2 * kRowTile ? c.grp->tp256 : c.grp->tp128;
  p.row_tile = Cfg::NMAX;
  const long max_row_tiles = (long)c.out_rows / Cfg::NMAX + c.grp->G;
  const long NT = (c.p.F + Cfg::FT - 1) / Cfg::FT;
  const long clusters = std::max(1L, std::min<long>(max_clusters, max_row_tiles * NT));
  return pair_launch(h, tc_gemm_pair_ws_kernel<Cfg>, Cfg::SMEM_BYTES, clusters, st, ta, tb, p);
}

template <typename T, bool kDual, int kEpi>
lmoe_status launch_simt(lmoe_layer* h, const GemmCall& c, cudaStream_t st) {
  const long NT = (c.p.F + kSimtTN - 1) / kSimtTN;
  const long blocks = (long)c.p.max_row_tiles * NT;
  if (blocks <= 0) return LMOE_OK;
  LMOE_LAUNCH(h, simt_gemm_kernel<T, kDual, kEpi>, dim3((unsigned)blocks), dim3(256), 0, st, c.p);
  return LMOE_OK;
}

template <typename T>
lmoe_status dispatch_simt(lmoe_layer* h, const GemmCall& c, cudaStream_t st) {
  const bool dual = c.p.dual_offset > 0;
  switch (c.kind) {
    case GK_ROUTER: return launch_simt<T, false, EPI_F32_BIAS>(h, c, st);
    case GK_DENSE_ACT:
    case GK_FC1:
      return dual ? launch_simt<T, true, EPI_ACT>(h, c, st) : launch_simt<T, false, EPI_ACT>(h, c, st);
    case GK_FC2: return launch_simt<T, false, EPI_SCALE_ROWS>(h, c, st);
    case GK_UP: return launch_simt<T, false, EPI_RESID>(h, c, st);
  }
  return LMOE_ERR_INVALID_ARG;
}

// Whether the tcgen05 kernel can take this call: bf16, K a multiple of 64,
// 16-byte aligned rows for TMA / cp.async and for the vector epilogue.
bool tc_eligible(const lmoe_layer* h, const GemmCall& c) {
  if (h->dtype != LMOE_BF16 || (h->flags & LMOE_FORCE_SIMT)) return false;
  const GemmProblem& p = c.p;
  if (p.K % 64 != 0 || p.K <= 0) return false;
  if (p.lda % 8 != 0 || !aligned16(p.A) || !aligned16(p.B)) return false;
  if (c.kind == GK_ROUTER) {
    if (p.epi.ldo % 4 != 0 || !aligned16(p.epi.out)) return false;
  } else {
    if (p.epi.ldo % 8 != 0 || p.epi.col0 % 8 != 0 || p.epi.split_off % 8 != 0 ||
        !aligned16(p.epi.out))
      return false;
  }
  if (c.kind == GK_UP && (p.epi.ldr % 8 != 0 || !aligned16(p.epi.resid))) return false;
  return true;
}

// ---- split-K for the dense GEMMs at small T ----------------------------------
//
// At decode sizes a dense GEMM (router, down-projection, shared FC1,
// up-projection) has a handful of 128 x 128 output tiles over K = d or l:
// one CTA per tile would stream K serially while most SMs idle.  The call is
// then split over K into S ranges, each written as an fp32 slice of partial
// sums, and splitk_reduce_kernel adds the slices in a fixed order (so results
// are deterministic) and applies the epilogue.

constexpr size_t kSplitPartBytes = 32u << 20;

// Number of K ranges for a dense single-CTA call (1: no split), and the
// 64-wide K blocks per range.
float* part_buffer(const lmoe_layer* h, const GemmCall& c) {
  return c.side ? h->part_side : h->part;
}

int choose_splits(const lmoe_layer* h, const GemmCall& c, int& kbs) {
  if (c.pair || c.swap || c.p.offsets || !part_buffer(h, c)) return 1;
  const bool dual = c.p.dual_offset > 0;
  if (dual && c.p.dual_offset != c.p.F) return 1;  // gate and linear rows must be adjacent
  const int Fp = dual ? 2 * c.p.F : c.p.F;
  const int KB = c.p.K / 64;
  if (Fp % 4 != 0 || KB < 4) return 1;
  const long tiles = (long)((c.p.M + kRowTile - 1) / kRowTile) * ((Fp + 127) / 128);
  if (tiles * 4 > h->num_sms) return 1;  // fewer than 4 ranges would not pay for the reduction
  int S = (int)std::min<long>(std::min<long>(h->num_sms / tiles, KB / 2), 16);
  while (S > 1 && (size_t)S * c.p.M * Fp * sizeof(float) > h->part_bytes) --S;
  if (S < 4) return 1;
  kbs = (KB + S - 1) / S;
  return (KB + kbs - 1) / kbs;  // every range non-empty
}

lmoe_status run_split(lmoe_layer* h, const GemmCall& c, int S, int kbs, cudaStream_t st) {
  const bool dual = c.p.dual_offset > 0;
  const int Fp = dual ? 2 * c.p.F : c.p.F;
  GemmCall g = c;
  g.kind = GK_ROUTER;  // fp32 output, no bias: the partial sums
  g.p.F = Fp;
  g.p.dual_offset = 0;
  std::memset(&g.p.epi, 0, sizeof g.p.epi);
  float* part = part_buffer(h, c);
  g.p.epi.out = part;
  g.p.epi.ldo = Fp;
  g.p.epi.slice = (long)c.p.M * Fp;
  g.p.splits = S;
  g.p.kb_per_split = kbs;
  g.out_rows = (long)S * c.p.M;  // the slices stacked: rows of the output map
  LMOE_TRY((launch_tc<TcCfg<false, false, false, 128, EPI_F32_BIAS>>(h, g, st)));
  const int kind = c.kind == GK_ROUTER ? EPI_F32_BIAS : c.kind == GK_UP ? EPI_RESID : EPI_ACT;
  const long n = (long)c.p.M * c.p.F;
  LMOE_LAUNCH(h, splitk_reduce_kernel, dim3((unsigned)((n + 255) / 256)), dim3(256), 0, st,
              (const float*)part, S, g.p.epi.slice, c.p.M, c.p.F, Fp, dual ? c.p.F : 0, kind,
              c.p.epi);
  return LMOE_OK;
}

lmoe_status run_gemm(lmoe_layer* h, GemmCall c, cudaStream_t st, int* path = nullptr) {
  c.p.err = h->err;
  // The weight-stationary tensor-core kernel takes at most kSwapRowTile rows
  // (its MMA N) per tile: tiles follow the 64-row prefix.
  const auto swap_rows = [&](GemmCall& g) {
    if (g.swap && g.p.offsets && !g.wide) {
      g.p.row_tile = kSwapRowTile;
      g.p.tile_prefix = g.grp->tp64;
      g.p.max_row_tiles = (int)(g.out_rows / kSwapRowTile + g.grp->G);  // routed rows
      // the expert FC1 (the longer weight stream): stream-K over (tile, K
      // block) units when there are 2 to 16 tiles per CTA (decided in the
      // kernel from the tile count).  On FC2 it measured slower.
      g.p.stream_k = (h->sk_part && g.kind == GK_FC1) ? 1 : 0;
      g.p.sk_part = h->sk_part;
      g.p.sk_count = h->sk_count;
    }
  };
  if (c.p.w_exp) {
    // fp4 expert weights: FC1 on the weight-stationary kernel (weights widened
    // into tensor memory) at every batch size, FC2 on it or on token tiles
    // (weights widened into shared memory)
    if (!tc_eligible(h, c) || c.pair || (!c.swap && c.kind != GK_FC2)) {
      h->detail = "fp4 expert weights: no tensor-core kernel for this call";
      return LMOE_ERR_UNSUPPORTED;
    }
    if (!c.swap) {
      if (path) *path = 1;
      return launch_tc<TcCfg<false, false, false, 256, EPI_SCALE_ROWS, true, kSwapRowTile, true>>(
          h, c, st);
    }
    swap_rows(c);
    const bool dual = c.p.dual_offset > 0;
    if (path) *path = 2;
    if (c.kind == GK_FC1)
      return dual ? launch_tc<TcCfg<true, true, true, 128, EPI_ACT, true, kSwapRowTile, true>>(h, c, st)
                  : launch_tc<TcCfg<true, true, false, 128, EPI_ACT, true, kSwapRowTile, true>>(h, c, st);
    if (c.kind == GK_FC2)
      return launch_tc<TcCfg<true, false, false, 128, EPI_SCALE_ROWS, true, kSwapRowTile, true>>(h, c, st);
    return LMOE_ERR_INVALID_ARG;
  }
  if (c.p.w_scale) {
    // fp8 expert weights: the single-CTA tensor-core kernel with the E4M3
    // widening warps (weight-stationary or token-tiled)
    if (!tc_eligible(h, c) || c.pair) {
      h->detail = "fp8 expert weights need the single-CTA tensor-core kernel";
      return LMOE_ERR_UNSUPPORTED;
    }
    swap_rows(c);
    const bool dual = c.p.dual_offset > 0;
    if (path) *path = c.swap ? 2 : 1;
    if (c.kind == GK_FC1) {
      if (c.swap)
        return dual ? launch_tc<TcCfg<true, true, true, 128, EPI_ACT, true>>(h, c, st)
                    : launch_tc<TcCfg<true, true, false, 128, EPI_ACT, true>>(h, c, st);
      return dual ? launch_tc<TcCfg<false, true, true, 128, EPI_ACT, true>>(h, c, st)
                  : launch_tc<TcCfg<false, true, false, 256, EPI_ACT, true>>(h, c, st);
    }
    if (c.kind == GK_FC2)
      return c.swap ? launch_tc<TcCfg<true, false, false, 128, EPI_SCALE_ROWS, true>>(h, c, st)
                    : launch_tc<TcCfg<false, false, false, 256, EPI_SCALE_ROWS, true>>(h, c, st);
    return LMOE_ERR_INVALID_ARG;
  }
  if (c.pair && c.p.gather != nullptr && c.kind != GK_FC1) {
    // the pair kernels gather rows by index only for the expert FC1
    c.pair = false;
    c.p.row_tile = kRowTile;
    c.p.tile_prefix = c.grp ? c.grp->tp128 : nullptr;
  }
  if (!tc_eligible(h, c)) {
    if (c.pair || c.wide) {  // the CUDA-core kernel tiles by 128 rows
      c.pair = false;
      c.p.row_tile = kRowTile;
      c.p.tile_prefix = c.grp ? c.grp->tp128 : nullptr;
      if (!c.p.offsets) c.p.max_row_tiles = (c.p.M + kRowTile - 1) / kRowTile;
      else c.p.max_row_tiles = (int)((c.out_rows + kRowTile - 1) / kRowTile + c.grp->G);
    }
    if (path) *path = 0;
    return h->dtype == LMOE_F32 ? dispatch_simt<float>(h, c, st) : dispatch_simt<bf16>(h, c, st);
  }
  const bool dual = c.p.dual_offset > 0;
  if (c.ws_pair && c.p.offsets) {
    if (path) *path = 4;
    if (c.kind == GK_FC1 && c.p.gather)
      return dual ? launch_pair_ws<TcPairWsCfg<true, true, EPI_ACT>>(h, c, st)
                  : launch_pair_ws<TcPairWsCfg<true, false, EPI_ACT>>(h, c, st);
    if (c.kind == GK_FC1)  // rows already in expert order (LMOE_SORTED_ROWS)
      return dual ? launch_pair_ws<TcPairWsCfg<false, true, EPI_ACT>>(h, c, st)
                  : launch_pair_ws<TcPairWsCfg<false, false, EPI_ACT>>(h, c, st);
    if (c.kind == GK_FC2 && !c.p.gather)
      return launch_pair_ws<TcPairWsCfg<false, false, EPI_SCALE_ROWS>>(h, c, st);
  }
  if (c.swap && c.wide && c.p.offsets) {
    // weight-stationary tiles of up to 128 (gated FC1: two accumulators) or
    // 256 rows, rows gathered by cp.async (FC1) or loaded by TMA (FC2)
    if (path) *path = 2;
    if (c.kind == GK_FC1 && c.p.gather && c.wide == (dual ? 128 : 256))
      return dual ? launch_tc<TcCfg<true, true, true, 128, EPI_ACT, false, 128>>(h, c, st)
                  : launch_tc<TcCfg<true, true, false, 128, EPI_ACT, false, 256>>(h, c, st);
    if (c.kind == GK_FC1 && c.wide == (dual ? 128 : 256))  // rows in expert order
      return dual ? launch_tc<TcCfg<true, false, true, 128, EPI_ACT, false, 128>>(h, c, st)
                  : launch_tc<TcCfg<true, false, false, 128, EPI_ACT, false, 256>>(h, c, st);
    if (c.kind == GK_FC2 && !c.p.gather && !dual && c.wide == 256)
      return launch_tc<TcCfg<true, false, false, 128, EPI_SCALE_ROWS, false, 256>>(h, c, st);
    h->detail = "no wide weight-stationary kernel for this call";
    return LMOE_ERR_INVALID_ARG;
  }
  if (path) *path = c.pair ? 3 : (c.swap ? 2 : 1);
  swap_rows(c);
  if (!c.pair && !c.swap && !c.p.offsets && c.kind != GK_FC1 && c.kind != GK_FC2) {
    int kbs = 0;
    const int S = choose_splits(h, c, kbs);
    if (S > 1) return run_split(h, c, S, kbs, st);
  }
  if (c.pair) {
    switch (c.kind) {
      case GK_DENSE_ACT:
        return dual ? launch_pair<TcPairCfg<true, EPI_ACT>>(h, c, st)
                    : launch_pair<TcPairCfg<false, EPI_ACT>>(h, c, st);
      case GK_FC1:
        if (c.p.gather)
          return dual ? launch_pair<TcPairCfg<true, EPI_ACT, true>>(h, c, st)
                      : launch_pair<TcPairCfg<false, EPI_ACT, true>>(h, c, st);
        return dual ? launch_pair<TcPairCfg<true, EPI_ACT>>(h, c, st)
                    : launch_pair<TcPairCfg<false, EPI_ACT>>(h, c, st);
      case GK_FC2: return launch_pair<TcPairCfg<false, EPI_SCALE_ROWS>>(h, c, st);
      case GK_UP: return launch_pair<TcPairCfg<false, EPI_RESID>>(h, c, st);
      case GK_ROUTER: return launch_pair<TcPairCfg<false, EPI_F32_BIAS>>(h, c, st);
    }
  }
  switch (c.kind) {
    case GK_ROUTER: return launch_tc<TcCfg<false, false, false, 128, EPI_F32_BIAS>>(h, c, st);
    case GK_DENSE_ACT:
      return dual ? launch_tc<TcCfg<false, false, true, 128, EPI_ACT>>(h, c, st)
                  : launch_tc<TcCfg<false, false, false, 256, EPI_ACT>>(h, c, st);
    case GK_FC1:
      if (!c.p.gather) {  // rows already in expert order (LMOE_SORTED_ROWS)
        if (c.swap)
          return dual ? launch_tc<TcCfg<true, false, true, 128, EPI_ACT>>(h, c, st)
                      : launch_tc<TcCfg<true, false, false, 128, EPI_ACT>>(h, c, st);
        return dual ? launch_tc<TcCfg<false, false, true, 128, EPI_ACT>>(h, c, st)
                    : launch_tc<TcCfg<false, false, false, 256, EPI_ACT>>(h, c, st);
      }
      if (c.swap)
        return dual ? launch_tc<TcCfg<true, true, true, 128, EPI_ACT>>(h, c, st)
                    : launch_tc<TcCfg<true, true, false, 128, EPI_ACT>>(h, c, st);
      return dual ? launch_tc<TcCfg<false, true, true, 128, EPI_ACT>>(h, c, st)
                  : launch_tc<TcCfg<false, true, false, 256, EPI_ACT>>(h, c, st);
    case GK_FC2:
      return c.swap ? launch_tc<TcCfg<true, false, false, 128, EPI_SCALE_ROWS>>(h, c, st)
                    : launch_tc<TcCfg<false, false, false, 256, EPI_SCALE_ROWS>>(h, c, st);
    case GK_UP:
      // decode sizes: 128-wide tiles where 256-wide ones would leave more
      // than half the SMs idle (twice the CTAs, each with half the loads and
      // half the epilogue)
      if (!c.p.offsets && 2L * c.p.max_row_tiles * ((c.p.F + 255) / 256) <= h->num_sms)
        return launch_tc<TcCfg<false, false, false, 128, EPI_RESID>>(h, c, st);
      return launch_tc<TcCfg<false, false, false, 256, EPI_RESID>>(h, c, st);
  }
  return LMOE_ERR_INVALID_ARG;
}

GemmCall dense_call(GemmKind kind, int M, const void* A, long lda, const void* B, int F, int K) {
  GemmCall c;
  std::memset(&c, 0, sizeof c);
  c.kind = kind;
  c.p.M = M;
  c.p.G = 1;
  c.p.max_row_tiles = (M + kRowTile - 1) / kRowTile;
  c.p.row_tile = kRowTile;
  c.p.A = A;
  c.p.lda = lda;
  c.p.B = B;
  c.p.F = F;
  c.p.K = K;
  c.a_rows = M;
  c.b_rows = F;
  c.out_rows = M;
  c.p.epi.act = ACT_NONE;
  return c;
}

// Switches a call to CTA pairs: 256-row tiles (and their tile counts).
void make_pair(const lmoe_layer* h, GemmCall& c) {
  c.pair = true;
  c.p.row_tile = 2 * kRowTile;
  if (c.p.offsets) {
    c.p.tile_prefix = c.grp->tp256;
    const long R = (long)c.out_rows;
    c.p.max_row_tiles = (int)((R + 2 * kRowTile - 1) / (2 * kRowTile) + c.grp->G);
  } else {
    c.p.max_row_tiles = (c.p.M + 2 * kRowTile - 1) / (2 * kRowTile);
  }
}

// A grouped expert GEMM over the R rows of grouping g: the weights of the
// group's experts start at expert g.e0 of the stack B (elem_bytes each).
GemmCall grouped_call(const Grouping& g, GemmKind kind, long R, const void* A, long lda,
                      long a_rows, const int* gather, const void* B, size_t elem_bytes,
                      long stride, int F, int K) {
  GemmCall c;
  std::memset(&c, 0, sizeof c);
  c.kind = kind;
  c.grp = &g;
  c.p.offsets = g.offsets;
  c.p.tile_prefix = g.tp128;
  c.p.G = g.G;
  c.p.max_row_tiles = (int)((R + kRowTile - 1) / kRowTile + g.G);
  c.p.row_tile = kRowTile;
  c.p.A = A;
  c.p.lda = lda;
  c.p.gather = gather;
  c.p.B = static_cast<const char*>(B) + (size_t)g.e0 * stride * K * elem_bytes;
  c.p.w_group_stride = stride;
  c.p.F = F;
  c.p.K = K;
  c.a_rows = a_rows;
  c.b_rows = (long)g.G * stride;
  c.out_rows = R;
  c.p.epi.act = ACT_NONE;
  return c;
}

// A prefill expert GEMM split by load: the experts with more than
// kPairMinRows rows on CTA pairs (256-row token tiles; FC1 gathers its rows
// by token in both CTAs), the others on single-CTA weight-stationary tiles
// of the expert's rows rounded up to 16 (at most 128 rows for the gated FC1,
// whose two accumulators share the tensor memory, 256 otherwise).  Two
// launches that write disjoint rows of the output; the tile counts of each
// come from the grouping step's big / small prefixes.
lmoe_status run_split_by_load(lmoe_layer* h, const GemmCall& c, cudaStream_t st, int* path) {
  GemmCall big = c;
  make_pair(h, big);
  big.p.tile_prefix = c.grp->big256;
  LMOE_TRY(run_gemm(h, big, st));
  GemmCall small = c;
  small.pair = false;
  small.swap = true;
  const bool dual = c.kind == GK_FC1 && c.p.dual_offset > 0;
  small.wide = dual ? 128 : 256;
  small.p.row_tile = small.wide;
  small.p.tile_prefix = dual ? c.grp->small128 : c.grp->small256;
  small.p.max_row_tiles = (int)(c.out_rows / small.wide + c.grp->G);
  LMOE_TRY(run_gemm(h, small, st));
  *path = 5;
  return LMOE_OK;
}

bool use_swap(const lmoe_layer* h, long R, int G) {
  if (h->flags & LMOE_FORCE_SWAP) return true;
  if (h->flags & LMOE_FORCE_NOSWAP) return false;
  return R < 64L * G;  // fewer than 64 rows per expert on average
}

// Records boundary i of the current profiled forward if a recorded stage
// starts or ends there (boundary i of the caller's stream opens stage i and
// closes stage i - 1; side boundary kSideMark0 + j opens stage 3 + j and
// closes stage 2 + j, of which only the side stream's stages 3 and 4 count).
void prof_mark(lmoe_layer* h, cudaStream_t st, int i) {
  if (!h->profiling || h->prof_count >= h->prof_cap) return;
  const int opens = i < kSideMark0 ? i : 3 + (i - kSideMark0);
  const int closes = opens - 1;
  const bool side = i >= kSideMark0;
  const auto has = [&](int s) {
    return s >= 0 && s < kStages && (!side || s == 3 || s == 4) && ((h->prof_mask >> s) & 1u);
  };
  if (has(opens) || has(closes))
    cudaEventRecord(h->events[(size_t)h->prof_count * kMarks + i], st);
}

// ---- the routing steps ---------------------------------------------------------

// Top-k and grouping.
lmoe_status run_routing(lmoe_layer* h, const float* logits, int T, int* idx, float* w,
                        int* offsets, int* row_tok, int* row_slot, float* row_w, int* slot_row,
                        int* tile_prefix2, cudaStream_t st, bool marks) {
  const int W = (T + 31) / 32;
  const int debug = (h->flags & LMOE_DEBUG_CHECKS) ? 1 : 0;
  {
    TopkArgs a;
    std::memset(&a, 0, sizeof a);
    a.logits = logits;
    a.T = T;
    a.N = h->N;
    a.k = h->k;
    a.sel_bias = (h->flags & LMOE_ROUTE_BIAS_SELECT) ? h->bias : nullptr;
    a.full_softmax = (h->flags & LMOE_ROUTE_FULL_SOFTMAX) ? 1 : 0;
    a.idx = idx;
    a.w = w;
    a.bitmap = h->bitmap;
    a.W = W;
    a.debug = debug;
    a.err = h->err;
    a.sms = h->num_sms;  // one wave of blocks; their warps stride over the tokens
    const cudaError_t e = launch_topk_args(a, st, take_pdl(h));
    if (e != cudaSuccess) return cuda_fail(h, e, "top-k launch");
    ++h->launches;
  }
  if (marks) prof_mark(h, st, 2);
  LMOE_LAUNCH(h, group_count_kernel, dim3((h->N + 7) / 8), dim3(256), 0, st, h->bitmap, h->wp,
              h->N, W, h->counts, offsets, h->tile_prefix, tile_prefix2,
              tile_prefix2 ? h->tile_prefix64 : (int*)nullptr, h->done,
              tile_prefix2 ? h->big_prefix2 : (int*)nullptr,
              tile_prefix2 ? h->small_prefix : (int*)nullptr,
              tile_prefix2 ? h->small_prefix2 : (int*)nullptr,
              tile_prefix2 ? h->full_prefix2 : (int*)nullptr,
              tile_prefix2 ? h->rem_prefix : (int*)nullptr);
  const long P = (long)T * h->k;
  LMOE_LAUNCH(h, group_rank_kernel, dim3((unsigned)((P + 255) / 256)), dim3(256), 0, st,
              (const int*)idx, (const float*)w, (const uint2*)h->wp, (const int*)offsets, T, h->k,
              h->N, W, row_tok, row_slot, row_w, slot_row, debug, h->err);
  return LMOE_OK;
}

lmoe_status run_router(lmoe_layer* h, const void* x, float* logits, int T, cudaStream_t st) {
  GemmCall c = dense_call(GK_ROUTER, T, x, h->d, h->Wg_t, h->N, h->d);
  c.p.epi.out = logits;
  c.p.epi.ldo = h->N;
  c.p.epi.bias = (h->flags & LMOE_ROUTE_BIAS_SELECT) ? nullptr : h->bias;
  if (h->dtype == LMOE_BF16 && T >= 1024 && !(h->flags & (LMOE_FORCE_SIMT | LMOE_FORCE_NOPAIR)))
    make_pair(h, c);
  return run_gemm(h, c, st);
}

// The stages that read only x: the down-projection z = x Wdown and the shared
// expert's FC1 (with the projection-skip layout, also its FC2 in fp32), on
// stream s.  Marks m_z and m_end are recorded after the down-projection and
// at the end; on the side stream, ev_side at the end as well.
lmoe_status run_x_stages(lmoe_layer* h, const void* x, int T, bool pair_dense, bool side,
                         cudaStream_t s, int m_z, int m_end) {
  const bool skip = (h->flags & LMOE_SKIP_PROJ) != 0;
  const int d = h->d, l = h->l, ms = h->shared_m;
  if (!skip) {
    GemmCall c = dense_call(GK_DENSE_ACT, T, x, d, h->Wd_t, l, d);
    c.side = side;
    c.p.epi.out = h->z;
    c.p.epi.ldo = l;
    if (pair_dense) make_pair(h, c);
    LMOE_TRY(run_gemm(h, c, s));
  }
  prof_mark(h, s, m_z);
  if (ms > 0) {
    GemmCall c = dense_call(GK_DENSE_ACT, T, x, d, h->Ws1_t, ms, d);
    c.side = side;
    c.b_rows = h->ms_in;
    c.p.dual_offset = h->act == LMOE_ACT_SWIGLU ? ms : 0;
    c.p.epi.out = h->cat;
    c.p.epi.ldo = h->Kup;
    c.p.epi.col0 = skip ? 0 : l;
    c.p.epi.act = h->act;
    c.p.epi.split_off = h->split_shared ? ms : 0;
    if (pair_dense) make_pair(h, c);
    LMOE_TRY(run_gemm(h, c, s));
    if (skip) {
      // no up-projection GEMM to carry it: s = hs Ws2 in fp32, added by the
      // combine before the output's single rounding
      GemmCall c2 = dense_call(GK_ROUTER, T, h->cat, h->Kup, h->Wu_t, d, h->Kup);
      c2.side = side;
      c2.p.epi.out = h->s32;
      c2.p.epi.ldo = d;
      c2.p.epi.bias = nullptr;
      LMOE_TRY(run_gemm(h, c2, s));
    }
  }
  if (side) LMOE_CUDA(h, cudaEventRecord(h->ev_side, s));
  prof_mark(h, s, m_end);
  return LMOE_OK;
}

// Whether CTA pairs may be used at all, and for the dense GEMMs of T tokens.
bool pairs_allowed(const lmoe_layer* h) {
  return h->dtype == LMOE_BF16 && !(h->flags & (LMOE_FORCE_SIMT | LMOE_FORCE_NOPAIR));
}
bool pair_dense_for(const lmoe_layer* h, int T) { return pairs_allowed(h) && T >= 1024; }

// Everything before the expert GEMMs: router, top-k, grouping (on the
// caller's stream) and the x-only stages (down-projection, shared FC1; on
// the side stream, joined before returning).  Profile marks 0-5.
lmoe_status run_front(lmoe_layer* h, const void* x, int T, cudaStream_t st) {
  const bool skip = (h->flags & LMOE_SKIP_PROJ) != 0;
  const int ms = h->shared_m;
  const bool pair_dense = pair_dense_for(h, T);
  // The down-projection and the shared FC1 depend on x alone: forked onto the
  // side stream they overlap the router GEMM and the latency-bound routing
  // kernels (which fit on an SM beside a GEMM CTA).  st waits for the whole
  // side stream before the expert FC1: a shared FC1 still running beside the
  // persistent expert FC1 would hold SMs that some of its CTAs need, and
  // those CTAs' tiles would finish last.
  const bool side = h->side_stream && !(h->flags & LMOE_SINGLE_STREAM) && (!skip || ms > 0);
  if (h->profiling && h->prof_count < h->prof_cap) h->prof_side[h->prof_count] = side ? 1 : 0;
  prof_mark(h, st, 0);
  if (side) {
    LMOE_CUDA(h, cudaEventRecord(h->ev_fork, st));
    LMOE_CUDA(h, cudaStreamWaitEvent(h->side_stream, h->ev_fork, 0));
    prof_mark(h, h->side_stream, kSideMark0);
    h->pdl_hold = true;
    LMOE_TRY(run_x_stages(h, x, T, pair_dense, true, h->side_stream, kSideMark0 + 1,
                          kSideMark0 + 2));
  }
  h->pdl_hold = true;
  LMOE_TRY(run_router(h, x, h->logits, T, st));
  prof_mark(h, st, 1);
  LMOE_TRY(run_routing(h, h->logits, T, h->idx, h->w, h->offsets, h->row_tok, h->row_slot,
                       h->row_w, h->slot_row, h->tile_prefix2, st, true));
  prof_mark(h, st, 3);
  if (side) {
    LMOE_CUDA(h, cudaStreamWaitEvent(st, h->ev_side, 0));
    h->pdl_hold = true;
    prof_mark(h, st, 5);
  } else {
    LMOE_TRY(run_x_stages(h, x, T, pair_dense, false, st, 4, 5));
  }
  return LMOE_OK;
}

// The two expert GEMMs over grouping g (R rows): hbuf[r] = act(A[src(r)]
// W1[e]) with src = gather (or r), ysbuf[r] = row_w[r] * (hbuf[r] W2[e]).
// Kernels: weight-stationary below 64 rows per expert on average, else
// token-tiled (FC1 on single CTAs, FC2 on CTA pairs; or split by load).
// Profile mark 6 between the two.  Sets h->expert_path.
lmoe_status run_expert_gemms(lmoe_layer* h, const Grouping& g, const void* A, long lda, long a_rows,
                             const int* gather, long R, void* hbuf, void* ysbuf,
                             const float* row_w, cudaStream_t st) {
  const int l = h->l, m = h->m;
  const bool skip = (h->flags & LMOE_SKIP_PROJ) != 0;
  const int cols = skip ? h->d : l;
  const bool fp8 = (h->flags & LMOE_EXPERTS_FP8) != 0;
  const bool fp4 = (h->flags & LMOE_EXPERTS_FP4) != 0;
  const bool lowp = fp8 || fp4;  // f16 FC1 input and output
  // fp4 weights run on the weight-stationary kernels at every size
  const bool swap = fp4 || use_swap(h, R, g.G);
  const bool pairs_ok = pairs_allowed(h);
  // token-tiled expert GEMMs with FC1 on single CTAs and FC2 on CTA pairs,
  // or (LMOE_LOAD_SPLIT) split by load: experts with many rows on CTA pairs,
  // the rest on weight-stationary single-CTA tiles
  const bool load_split = pairs_ok && !swap && !lowp && (h->flags & LMOE_LOAD_SPLIT) &&
                          !(h->flags & LMOE_FORCE_WS_PAIR) && l % 64 == 0 && m % 64 == 0;
  const bool pair_fc2 = pairs_ok && !swap;
  // on request: the expert GEMMs weight-stationary on CTA pairs (rows on the
  // MMA's N, so an expert's last tile is padded to 16 rows, not 128 or 256)
  const bool ws_pair = pairs_ok && !swap && (h->flags & LMOE_FORCE_WS_PAIR) &&
                       !(h->flags & LMOE_FORCE_NOSWAP);
  {
    if (lowp) {
      // the fp8 / fp4 expert kernels multiply f16 operands: the FC1 input in f16
      const long n = a_rows * cols;
      const int vec = (n % 8 == 0 && aligned16(A) && aligned16(h->a16)) ? 1 : 0;
      const long work = vec ? n / 8 : n;
      const unsigned blocks = (unsigned)std::max<long>(1, std::min<long>((work + 255) / 256,
                                                                          8L * h->num_sms));
      LMOE_LAUNCH(h, bf16_to_f16_kernel, dim3(blocks), dim3(256), 0, st,
                  static_cast<const bf16*>(A), static_cast<__half*>(h->a16), n, vec);
      A = h->a16;
    }
    const bool sorted = (h->flags & LMOE_SORTED_ROWS) && h->dtype == LMOE_BF16 && !lowp && gather;
    if (sorted) {
      // the FC1 input rows copied into expert order: FC1 then loads them as
      // contiguous tiles (by TMA) like FC2 does its input
      const int vec = (cols % 8 == 0 && lda % 8 == 0 && aligned16(A) && aligned16(h->zs)) ? 1 : 0;
      const unsigned blocks =
          (unsigned)std::max<long>(1, std::min<long>((R + 7) / 8, 8L * h->num_sms));
      LMOE_LAUNCH(h, gather_rows_kernel, dim3(blocks), dim3(256), 0, st,
                  static_cast<const uint16_t*>(A), lda, gather, R, cols,
                  static_cast<uint16_t*>(h->zs), vec);
      A = h->zs;
      lda = cols;
      a_rows = R;
      gather = nullptr;
    }
    // (fp4: the weight rows hold l / 2 bytes; the expert offset g.e0 is 0,
    // expert parallelism takes no fp4 layers)
    GemmCall c = grouped_call(g, GK_FC1, R, A, lda, a_rows, gather,
                              fp4 ? (const void*)h->W1q4_t
                                  : fp8 ? (const void*)h->W1q_t : h->W1_t,
                              fp8 ? 1 : h->es, h->m_in, m, l);
    c.p.w_scale = fp8 ? h->W1s + (size_t)g.e0 * h->m_in : nullptr;
    c.p.w_exp = fp4 ? h->W1e_t : nullptr;
    c.swap = swap;
    c.ws_pair = ws_pair && !lowp;
    c.p.dual_offset = h->act == LMOE_ACT_SWIGLU ? m : 0;
    c.p.epi.out = hbuf;
    c.p.epi.ldo = m;
    c.p.epi.act = h->act;
    int path = 0;
    if (load_split) LMOE_TRY(run_split_by_load(h, c, st, &path));
    else LMOE_TRY(run_gemm(h, c, st, &path));
    h->expert_path = path;
  }
  prof_mark(h, st, 6);
  {
    GemmCall c = grouped_call(g, GK_FC2, R, hbuf, m, R, nullptr,
                              fp4 ? (const void*)h->W2q4_t
                                  : fp8 ? (const void*)h->W2q_t : h->W2_t,
                              fp8 ? 1 : h->es, l, l, m);
    c.p.w_scale = fp8 ? h->W2s + (size_t)g.e0 * l : nullptr;
    c.p.w_exp = fp4 ? h->W2e_t : nullptr;
    // fp8 / fp4 FC2 on token tiles at every size (unless weight-stationary
    // tiles are forced): one 128 x 256 MMA per K step covers 256 output
    // features where the 16-row weight-stationary tiles issue two, and at
    // decode the MMA count, not HBM, sets the pace of the widened kernels
    c.swap = swap && !(lowp && !(h->flags & LMOE_FORCE_SWAP));
    c.ws_pair = ws_pair && !lowp;
    c.p.epi.out = ysbuf;
    c.p.epi.ldo = l;
    c.p.epi.row_w = row_w;
    int path = 0;
    if (load_split) {
      LMOE_TRY(run_split_by_load(h, c, st, &path));
    } else if (pair_fc2 && !ws_pair && !lowp && (h->flags & LMOE_FC2_SPLIT) && g.full256 &&
               g.rem128) {
      // an expert's last rows past its whole 256-row tiles, when at most 128,
      // on one 128-row single-CTA tile (padding to 128 rows instead of 256);
      // everything else on CTA pairs (two launches writing disjoint rows of ys)
      GemmCall full = c;
      make_pair(h, full);
      full.p.tile_prefix = g.full256;
      full.p.max_row_tiles = (int)(R / (2 * kRowTile) + 1);
      LMOE_TRY(run_gemm(h, full, st, &path));
      GemmCall rest = c;
      rest.p.tile_prefix = g.rem128;
      rest.p.row_tile = kRowTile;
      rest.p.rem_of = 2 * kRowTile;
      rest.p.max_row_tiles = 2 * g.G;
      int p2 = 0;
      LMOE_TRY(run_gemm(h, rest, st, &p2));
    } else {
      if (pair_fc2 && !ws_pair && !lowp) make_pair(h, c);  // the pair kernels read bf16 weights
      LMOE_TRY(run_gemm(h, c, st, &path));
    }
    h->expert_path |= path << 3;
  }
  return LMOE_OK;
}

// Everything after the expert GEMMs: the gate-weighted sum of each token's k
// rows of ys (rows in the grouping's order, found through slot_row), then the
// up-projection with the shared expert and the residual (or, skipping the
// projections, the residual and the fp32 shared output in the combine).
// Profile marks 7-9.
lmoe_status run_back(lmoe_layer* h, const void* x, const void* ys, void* out, int T,
                     cudaStream_t st) {
  const bool skip = (h->flags & LMOE_SKIP_PROJ) != 0;
  const int d = h->d, l = h->l, k = h->k, ms = h->shared_m;
  prof_mark(h, st, 7);
  {
    const void* resid = skip ? x : nullptr;
    const float* add32 = (skip && ms > 0) ? h->s32 : nullptr;
    void* dst = skip ? out : h->cat;
    const long ldo = skip ? d : h->Kup;
    const int vec = 16 / h->es;
    const bool vec_ok = (l % vec == 0) && (ldo % vec == 0) && aligned16(dst) && aligned16(ys) &&
                        (!resid || (aligned16(resid) && d % vec == 0));
    const int threads = std::min(256, std::max(32, (l / vec + 31) / 32 * 32));
    // split a token's columns over blocks when T alone does not fill the GPU
    const int per_block = threads * vec;
    const int chunks = std::max(1, std::min((l + per_block - 1) / per_block,
                                            (2 * h->num_sms + T - 1) / std::max(T, 1)));
    const dim3 cgrid((unsigned)T, (unsigned)chunks);
    const long ldr = d;
    if (h->dtype == LMOE_BF16) {
      if (vec_ok)
        LMOE_LAUNCH(h, combine_kernel<bf16>, cgrid, dim3(threads), 0, st, (const bf16*)ys,
                    (const int*)h->slot_row, k, l, (const bf16*)resid, ldr, add32, (bf16*)dst, ldo);
      else
        LMOE_LAUNCH(h, combine_scalar_kernel<bf16>, dim3(T), dim3(256), 0, st, (const bf16*)ys,
                    (const int*)h->slot_row, k, l, (const bf16*)resid, ldr, add32, (bf16*)dst, ldo);
    } else {
      if (vec_ok)
        LMOE_LAUNCH(h, combine_kernel<float>, cgrid, dim3(threads), 0, st, (const float*)ys,
                    (const int*)h->slot_row, k, l, (const float*)resid, ldr, add32, (float*)dst,
                    ldo);
      else
        LMOE_LAUNCH(h, combine_scalar_kernel<float>, dim3(T), dim3(256), 0, st,
                    (const float*)ys, (const int*)h->slot_row, k, l, (const float*)resid, ldr,
                    add32, (float*)dst, ldo);
    }
  }
  prof_mark(h, st, 8);
  if (!skip) {
    GemmCall c = dense_call(GK_UP, T, h->cat, h->Kup, h->Wu_t, d, h->Kup);
    c.p.epi.out = out;
    c.p.epi.ldo = d;
    c.p.epi.resid = x;
    c.p.epi.ldr = d;
    if (pair_dense_for(h, T)) make_pair(h, c);
    LMOE_TRY(run_gemm(h, c, st));
  }
  prof_mark(h, st, 9);
  return LMOE_OK;
}

lmoe_status run_forward(lmoe_layer* h, const void* x, void* out, int T, cudaStream_t st) {
  h->launches = 0;
  const bool skip = (h->flags & LMOE_SKIP_PROJ) != 0;
  const long R = (long)T * h->k;
  LMOE_TRY(run_front(h, x, T, st));
  LMOE_TRY(run_expert_gemms(h, h->fwd_grp, skip ? x : h->z, skip ? h->d : h->l, T, h->row_tok, R,
                            h->h, h->ys, h->row_w, st));
  LMOE_TRY(run_back(h, x, h->ys, out, T, st));
  if (h->profiling && h->prof_count < h->prof_cap) ++h->prof_count;
  h->last_T = T;
  return LMOE_OK;
}

template <typename T>
void free_ptr(T*& p) {
  if (p) cudaFree((void*)p);
  p = nullptr;
}

void free_workspace(lmoe_layer* h) {
  free_ptr(h->logits);
  free_ptr(h->idx);
  free_ptr(h->w);
  free_ptr(h->bitmap);
  free_ptr(h->wp);
  free_ptr(h->counts);
  free_ptr(h->offsets);
  free_ptr(h->tile_prefix);
  free_ptr(h->tile_prefix2);
  free_ptr(h->tile_prefix64);
  free_ptr(h->big_prefix2);
  free_ptr(h->small_prefix);
  free_ptr(h->small_prefix2);
  free_ptr(h->full_prefix2);
  free_ptr(h->rem_prefix);
  free_ptr(h->sk_part);
  free_ptr(h->sk_count);
  free_ptr(h->slot_row);
  free_ptr(h->done);
  free_ptr(h->err);
  free_ptr(h->row_tok);
  free_ptr(h->row_slot);
  free_ptr(h->row_w);
  free_ptr(h->z);
  free_ptr(h->h);
  free_ptr(h->ys);
  free_ptr(h->cat);
  free_ptr(h->x_stage);
  free_ptr(h->x_stage2);
  free_ptr(h->out_stage);
  for (int i = 0; i < 2; ++i) {
    if (h->ev_up[i]) cudaEventDestroy(h->ev_up[i]);
    if (h->ev_used[i]) cudaEventDestroy(h->ev_used[i]);
    h->ev_up[i] = h->ev_used[i] = nullptr;
  }
  if (h->copy_stream) cudaStreamDestroy(h->copy_stream);
  h->copy_stream = nullptr;
  for (cudaEvent_t* e : {&h->ev_fork, &h->ev_side}) {
    if (*e) cudaEventDestroy(*e);
    *e = nullptr;
  }
  if (h->side_stream) cudaStreamDestroy(h->side_stream);
  h->side_stream = nullptr;
  free_ptr(h->part_side);
  h->host_slot = 0;
  free_ptr(h->s32);
  free_ptr(h->a16);
  free_ptr(h->zs);
  free_ptr(h->part);
  h->part_bytes = 0;
  h->max_T = 0;
}

void free_ep(lmoe_layer* h) {
  free_ptr(h->ep_tab);
  if (h->ep_tab_host) cudaFreeHost(h->ep_tab_host);
  h->ep_tab_host = nullptr;
  if (h->ep_uploaded) cudaEventDestroy(h->ep_uploaded);
  h->ep_uploaded = nullptr;
  free_ptr(h->ep_perm);
  free_ptr(h->ep_inv);
  free_ptr(h->ep_gates);
  free_ptr(h->ep_h);
  free_ptr(h->ep_ys);
  h->ep_max_rows = 0;
}

// Host tables of the received rows (see lmoe_ep_experts): per local expert
// its total rows and grouped offset; per (source, expert) block its start in
// the received order (roff, source-major) and in the grouped order (goff,
// expert-major); each source's first received row (src_start).  Returns the
// total, or -1 for a negative count.
long ep_host_tables(const int* rc, int world, int n, int* counts, int* offsets, int* src_start,
                    int* roff, int* goff) {
  long run = 0;
  for (int s = 0; s < world; ++s) {
    src_start[s] = (int)run;
    for (int e = 0; e < n; ++e) {
      if (rc[(size_t)s * n + e] < 0) return -1;
      roff[(size_t)s * n + e] = (int)run;
      run += rc[(size_t)s * n + e];
    }
  }
  src_start[world] = (int)run;
  long g = 0;
  for (int e = 0; e < n; ++e) {
    offsets[e] = (int)g;
    long c = 0;
    for (int s = 0; s < world; ++s) {
      goff[(size_t)e * world + s] = (int)(g + c);
      c += rc[(size_t)s * n + e];
    }
    counts[e] = (int)c;
    g += c;
  }
  offsets[n] = (int)g;
  return run;
}

void free_weights(lmoe_layer* h) {
  free_ptr(h->Wg_t);
  free_ptr(h->bias);
  free_ptr(h->Wd_t);
  free_ptr(h->Wu_t);
  free_ptr(h->Ws1_t);
  free_ptr(h->W1_t);
  free_ptr(h->W1q_t);
  free_ptr(h->W2q_t);
  free_ptr(h->W1q4_t);
  free_ptr(h->W1e_t);
  free_ptr(h->W2q4_t);
  free_ptr(h->W2e_t);
  h->fp4_set = false;
  free_ptr(h->W1s);
  free_ptr(h->W2s);
  h->fp8_set = false;
  free_ptr(h->W2_t);
  h->weights_set = false;
}

void destroy_events(lmoe_layer* h) {
  for (cudaEvent_t e : h->events) cudaEventDestroy(e);
  h->events.clear();
  h->prof_cap = h->prof_count = 0;
  h->profiling = false;
}

// API layout [batch][rows][cols] -> K-major [batch][cols][col0 + rows] (row stride ldo).
lmoe_status repack(lmoe_layer* h, const void* in, int rows, int cols, int batch, void* out, long ldo,
                   int col0) {
  dim3 grid((cols + 31) / 32, (rows + 31) / 32, batch), block(32, 8);
  const long ib = (long)rows * cols, ob = (long)cols * ldo;
  if (h->dtype == LMOE_BF16)
    transpose_kernel<bf16><<<grid, block>>>((const bf16*)in, rows, cols, ib, (bf16*)out, ldo, col0, ob);
  else
    transpose_kernel<float><<<grid, block>>>((const float*)in, rows, cols, ib, (float*)out, ldo, col0,
                                             ob);
  LMOE_CUDA(h, cudaGetLastError());
  return LMOE_OK;
}

bool valid_stream_call(const lmoe_layer* h, int T) { return h && T >= 0 && T <= h->max_T; }

// Weights in place: lmoe_set_weights, and with fp8 experts their codes too.
bool layer_ready(const lmoe_layer* h) {
  return h->weights_set && (!(h->flags & LMOE_EXPERTS_FP8) || h->fp8_set) &&
         (!(h->flags & LMOE_EXPERTS_FP4) || h->fp4_set);
}

}  // namespace

// ================================== C ABI ==================================

extern "C" {

const char* lmoe_status_string(lmoe_status s) {
  switch (s) {
    case LMOE_OK: return "ok";
    case LMOE_ERR_INVALID_ARG: return "invalid argument";
    case LMOE_ERR_NOT_READY: return "not ready (weights not set or workspace not reserved)";
    case LMOE_ERR_CUDA: return "CUDA error";
    case LMOE_ERR_OOM: return "out of device memory";
    case LMOE_ERR_TIMEOUT: return "device-side wait timed out";
    case LMOE_ERR_UNSUPPORTED: return "unsupported configuration";
    case LMOE_ERR_DEVICE: return "device-side check failed";
  }
  return "unknown status";
}

const char* lmoe_stage_name(int stage) {
  return (stage >= 0 && stage < kStages) ? kStageNames[stage] : "";
}

const char* lmoe_error_detail(const lmoe_layer* h) { return h ? h->detail.c_str() : ""; }

lmoe_status lmoe_create(int d, int l, int N, int k, int m, lmoe_act act, int shared_m,
                        lmoe_dtype dtype, unsigned flags, lmoe_layer** out) {
  if (!out) return LMOE_ERR_INVALID_ARG;
  *out = nullptr;
  const unsigned known = LMOE_SKIP_PROJ | LMOE_DEBUG_CHECKS | LMOE_FORCE_SIMT | LMOE_FORCE_SWAP |
                         LMOE_FORCE_NOSWAP | LMOE_FORCE_NOPAIR | LMOE_FORCE_WS_PAIR |
                         LMOE_ROUTE_FULL_SOFTMAX | LMOE_ROUTE_BIAS_SELECT | LMOE_EXPERTS_FP8 |
                         LMOE_EXPERTS_FP4 |
                         LMOE_SINGLE_STREAM | LMOE_NO_PDL | LMOE_LOAD_SPLIT |
                         LMOE_NO_STREAM_K | LMOE_SORTED_ROWS | LMOE_FC2_SPLIT;
  if (d <= 0 || l <= 0 || N <= 0 || k <= 0 || m <= 0 || shared_m < 0) return LMOE_ERR_INVALID_ARG;
  if (k > N || (flags & ~known)) return LMOE_ERR_INVALID_ARG;
  if (act != LMOE_ACT_SILU && act != LMOE_ACT_SWIGLU && act != LMOE_ACT_RELU2) return LMOE_ERR_INVALID_ARG;
  if (dtype != LMOE_F32 && dtype != LMOE_BF16) return LMOE_ERR_INVALID_ARG;
  if ((flags & LMOE_SKIP_PROJ) && l != d) return LMOE_ERR_INVALID_ARG;
  if ((flags & LMOE_FORCE_SWAP) && (flags & LMOE_FORCE_NOSWAP)) return LMOE_ERR_INVALID_ARG;
  // fp8 expert weights run on the tensor-core kernels only: bf16 layers whose
  // expert GEMMs have K (l and m) a multiple of 64
  // fp4 expert weights: bf16 layers whose K (l and m) rows of block exponents
  // are whole 16-byte boxes (K a multiple of 512); not with fp8
  if ((flags & LMOE_EXPERTS_FP4) &&
      (dtype != LMOE_BF16 || (flags & (LMOE_FORCE_SIMT | LMOE_EXPERTS_FP8)) || l % 512 != 0 ||
       m % 512 != 0))
    return LMOE_ERR_UNSUPPORTED;
  if ((flags & LMOE_EXPERTS_FP8) &&
      (dtype != LMOE_BF16 || (flags & LMOE_FORCE_SIMT) || l % 64 != 0 || m % 64 != 0))
    return LMOE_ERR_UNSUPPORTED;
  if (N > LMOE_MAX_EXPERTS || k > LMOE_MAX_TOPK) return LMOE_ERR_UNSUPPORTED;
  // 32-bit row and element indices inside the kernels
  if ((long)N * (2L * m) * l >= (1L << 31) * 8L) return LMOE_ERR_UNSUPPORTED;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return LMOE_ERR_CUDA;
  lmoe_layer* h = new lmoe_layer();
  h->d = d; h->l = l; h->N = N; h->k = k; h->m = m; h->act = act; h->shared_m = shared_m;
  h->dtype = dtype; h->flags = flags;
  h->pdl = (flags & LMOE_NO_PDL) == 0;
  h->m_in = act == LMOE_ACT_SWIGLU ? 2 * m : m;
  h->ms_in = act == LMOE_ACT_SWIGLU ? 2 * shared_m : shared_m;
  // bf16: the shared expert's hidden activations go into the up-projection as
  // hi + lo bf16 pairs (K grows by shared_m, Ws2 appears twice in the
  // K-concatenated weight), so their storage rounding no longer dominates the
  // output error of layers with a large shared contribution.
  h->split_shared = dtype == LMOE_BF16 && shared_m > 0;
  h->Kup = ((flags & LMOE_SKIP_PROJ) ? 0 : l) + shared_m * (h->split_shared ? 2 : 1);
  h->es = dtype == LMOE_BF16 ? 2 : 4;
  h->device = dev;
  int sms = 0;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess && sms > 0)
    h->num_sms = sms;
  *out = h;
  return LMOE_OK;
}

lmoe_status lmoe_set_weights(lmoe_layer* h, const void* W_g, const float* bias, const void* W_down,
                             const void* W_up, const void* W1, const void* W2, const void* Ws1,
                             const void* Ws2) {
  const bool fp8 = h && (h->flags & (LMOE_EXPERTS_FP8 | LMOE_EXPERTS_FP4));
  if (!h || !W_g || (!fp8 && (!W1 || !W2))) return LMOE_ERR_INVALID_ARG;
  const bool skip = (h->flags & LMOE_SKIP_PROJ) != 0;
  if (skip != (W_down == nullptr) || skip != (W_up == nullptr)) return LMOE_ERR_INVALID_ARG;
  if ((h->shared_m > 0) != (Ws1 != nullptr) || (h->shared_m > 0) != (Ws2 != nullptr))
    return LMOE_ERR_INVALID_ARG;
  DevGuard g(h->device);
  LMOE_CUDA(h, cudaDeviceSynchronize());
  const size_t es = h->es;
  const int d = h->d, l = h->l, N = h->N, m = h->m;
  if (!h->weights_set) {
    LMOE_CUDA(h, cudaMalloc(&h->Wg_t, (size_t)N * d * es));
    if (!fp8) {
      LMOE_CUDA(h, cudaMalloc(&h->W1_t, (size_t)N * h->m_in * l * es));
      LMOE_CUDA(h, cudaMalloc(&h->W2_t, (size_t)N * l * m * es));
    }
    if (!skip) LMOE_CUDA(h, cudaMalloc(&h->Wd_t, (size_t)l * d * es));
    if (h->Kup > 0) LMOE_CUDA(h, cudaMalloc(&h->Wu_t, (size_t)d * h->Kup * es));
    if (h->shared_m > 0) LMOE_CUDA(h, cudaMalloc(&h->Ws1_t, (size_t)h->ms_in * d * es));
  }
  free_ptr(h->bias);
  if (bias) {
    LMOE_CUDA(h, cudaMalloc(&h->bias, (size_t)N * sizeof(float)));
    LMOE_CUDA(h, cudaMemcpy(h->bias, bias, (size_t)N * sizeof(float), cudaMemcpyDeviceToDevice));
  }
  LMOE_TRY(repack(h, W_g, d, N, 1, h->Wg_t, d, 0));
  if (!fp8) {
    LMOE_TRY(repack(h, W1, l, h->m_in, N, h->W1_t, l, 0));
    LMOE_TRY(repack(h, W2, m, l, N, h->W2_t, m, 0));
  }
  if (!skip) {
    LMOE_TRY(repack(h, W_down, d, l, 1, h->Wd_t, d, 0));
    LMOE_TRY(repack(h, W_up, l, d, 1, h->Wu_t, h->Kup, 0));
  }
  if (h->shared_m > 0) {
    LMOE_TRY(repack(h, Ws1, d, h->ms_in, 1, h->Ws1_t, d, 0));
    LMOE_TRY(repack(h, Ws2, h->shared_m, d, 1, h->Wu_t, h->Kup, skip ? 0 : l));
    if (h->split_shared)
      LMOE_TRY(repack(h, Ws2, h->shared_m, d, 1, h->Wu_t, h->Kup, (skip ? 0 : l) + h->shared_m));
  }
  LMOE_CUDA(h, cudaDeviceSynchronize());
  h->weights_set = true;
  return LMOE_OK;
}

lmoe_status lmoe_set_expert_weights_fp8(lmoe_layer* h, const void* W1q, const float* W1s,
                                        const void* W2q, const float* W2s) {
  if (!h || !W1q || !W1s || !W2q || !W2s) return LMOE_ERR_INVALID_ARG;
  if (!(h->flags & LMOE_EXPERTS_FP8)) return LMOE_ERR_INVALID_ARG;
  DevGuard g(h->device);
  LMOE_CUDA(h, cudaDeviceSynchronize());
  const int l = h->l, N = h->N, m = h->m, m_in = h->m_in;
  if (!h->fp8_set) {
    LMOE_CUDA(h, cudaMalloc(&h->W1q_t, (size_t)N * m_in * l));
    LMOE_CUDA(h, cudaMalloc(&h->W2q_t, (size_t)N * l * m));
    LMOE_CUDA(h, cudaMalloc(&h->W1s, (size_t)N * m_in * sizeof(float)));
    LMOE_CUDA(h, cudaMalloc(&h->W2s, (size_t)N * l * sizeof(float)));
  }
  // codes [N][in][out] -> K-major [N][out][in], as the bf16 stacks
  {
    dim3 grid((m_in + 31) / 32, (l + 31) / 32, N), block(32, 8);
    transpose_kernel<uint8_t><<<grid, block>>>(static_cast<const uint8_t*>(W1q), l, m_in,
                                               (long)l * m_in, h->W1q_t, l, 0, (long)m_in * l);
    LMOE_CUDA(h, cudaGetLastError());
  }
  {
    dim3 grid((l + 31) / 32, (m + 31) / 32, N), block(32, 8);
    transpose_kernel<uint8_t><<<grid, block>>>(static_cast<const uint8_t*>(W2q), m, l,
                                               (long)m * l, h->W2q_t, m, 0, (long)l * m);
    LMOE_CUDA(h, cudaGetLastError());
  }
  LMOE_CUDA(h, cudaMemcpy(h->W1s, W1s, (size_t)N * m_in * sizeof(float), cudaMemcpyDeviceToDevice));
  LMOE_CUDA(h, cudaMemcpy(h->W2s, W2s, (size_t)N * l * sizeof(float), cudaMemcpyDeviceToDevice));
  LMOE_CUDA(h, cudaDeviceSynchronize());
  h->fp8_set = true;
  return LMOE_OK;
}

lmoe_status lmoe_set_expert_weights_fp4(lmoe_layer* h, const void* W1q, const void* W1e,
                                        const void* W2q, const void* W2e) {
  if (!h || !W1q || !W1e || !W2q || !W2e) return LMOE_ERR_INVALID_ARG;
  if (!(h->flags & LMOE_EXPERTS_FP4)) return LMOE_ERR_INVALID_ARG;
  DevGuard g(h->device);
  const size_t N = h->N, l = h->l, m = h->m, m_in = h->m_in;
  const size_t e1 = N * m_in * (l / 32), e2 = N * l * (m / 32);
  // every block exponent must keep code x 2^(e - 127) an f16 value
  {
    std::vector<uint8_t> ex(std::max(e1, e2));
    for (int i = 0; i < 2; ++i) {
      const size_t n = i ? e2 : e1;
      LMOE_CUDA(h, cudaMemcpy(ex.data(), i ? W2e : W1e, n, cudaMemcpyDeviceToHost));
      for (size_t j = 0; j < n; ++j)
        if (ex[j] < 127 - 23 || ex[j] > 127 + 13) {
          h->detail = "fp4 block exponent outside [2^-23, 2^13]";
          return LMOE_ERR_UNSUPPORTED;
        }
    }
  }
  LMOE_CUDA(h, cudaDeviceSynchronize());
  if (!h->fp4_set) {
    LMOE_CUDA(h, cudaMalloc(&h->W1q4_t, N * m_in * (l / 2)));
    LMOE_CUDA(h, cudaMalloc(&h->W1e_t, e1));
    LMOE_CUDA(h, cudaMalloc(&h->W2q4_t, N * l * (m / 2)));
    LMOE_CUDA(h, cudaMalloc(&h->W2e_t, e2));
  }
  LMOE_CUDA(h, cudaMemcpy(h->W1q4_t, W1q, N * m_in * (l / 2), cudaMemcpyDeviceToDevice));
  LMOE_CUDA(h, cudaMemcpy(h->W1e_t, W1e, e1, cudaMemcpyDeviceToDevice));
  LMOE_CUDA(h, cudaMemcpy(h->W2q4_t, W2q, N * l * (m / 2), cudaMemcpyDeviceToDevice));
  LMOE_CUDA(h, cudaMemcpy(h->W2e_t, W2e, e2, cudaMemcpyDeviceToDevice));
  LMOE_CUDA(h, cudaDeviceSynchronize());
  h->fp4_set = true;
  return LMOE_OK;
}

lmoe_status lmoe_reserve(lmoe_layer* h, int max_T) {
  if (!h || max_T < 1) return LMOE_ERR_INVALID_ARG;
  if (max_T <= h->max_T) return LMOE_OK;
  DevGuard g(h->device);
  LMOE_CUDA(h, cudaDeviceSynchronize());
  free_workspace(h);
  const size_t T = max_T, R = T * h->k, es = h->es;
  const size_t W = (T + 31) / 32;
  const bool skip = (h->flags & LMOE_SKIP_PROJ) != 0;
#define ALLOC(ptr, bytes) LMOE_CUDA(h, cudaMalloc((void**)&(ptr), std::max<size_t>(bytes, 16)))
  ALLOC(h->logits, T * h->N * sizeof(float));
  ALLOC(h->idx, R * sizeof(int));
  ALLOC(h->w, R * sizeof(float));
  ALLOC(h->bitmap, (size_t)h->N * W * sizeof(uint32_t));
  ALLOC(h->wp, (size_t)h->N * W * sizeof(uint2));
  ALLOC(h->counts, (size_t)h->N * sizeof(int));
  ALLOC(h->offsets, (size_t)(h->N + 1) * sizeof(int));
  ALLOC(h->tile_prefix, (size_t)(h->N + 1) * sizeof(int));
  ALLOC(h->tile_prefix2, (size_t)(h->N + 1) * sizeof(int));
  ALLOC(h->tile_prefix64, (size_t)(h->N + 1) * sizeof(int));
  ALLOC(h->big_prefix2, (size_t)(h->N + 1) * sizeof(int));
  ALLOC(h->small_prefix, (size_t)(h->N + 1) * sizeof(int));
  ALLOC(h->small_prefix2, (size_t)(h->N + 1) * sizeof(int));
  ALLOC(h->full_prefix2, (size_t)(h->N + 1) * sizeof(int));
  ALLOC(h->rem_prefix, (size_t)(h->N + 1) * sizeof(int));
  if (h->dtype == LMOE_BF16 && !(h->flags & LMOE_NO_STREAM_K)) {
    ALLOC(h->sk_part, (size_t)2 * (h->num_sms + 1) * kSkSlotFloats * sizeof(float));
    ALLOC(h->sk_count, (size_t)(h->num_sms + 1) * sizeof(int));
  }
  ALLOC(h->slot_row, R * sizeof(int));
  ALLOC(h->done, sizeof(unsigned));
  ALLOC(h->err, sizeof(int));
  ALLOC(h->row_tok, R * sizeof(int));
  ALLOC(h->row_slot, R * sizeof(int));
  ALLOC(h->row_w, R * sizeof(float));
  if (!skip) ALLOC(h->z, T * h->l * es);
  ALLOC(h->h, R * h->m * es);
  ALLOC(h->ys, R * h->l * es);
  if (h->Kup > 0) ALLOC(h->cat, T * h->Kup * es);
  ALLOC(h->x_stage, T * h->d * es);
  ALLOC(h->x_stage2, T * h->d * es);
  ALLOC(h->out_stage, T * h->d * es);
  LMOE_CUDA(h, cudaStreamCreateWithFlags(&h->copy_stream, cudaStreamNonBlocking));
  for (int i = 0; i < 2; ++i) {
    LMOE_CUDA(h, cudaEventCreateWithFlags(&h->ev_up[i], cudaEventDisableTiming));
    LMOE_CUDA(h, cudaEventCreateWithFlags(&h->ev_used[i], cudaEventDisableTiming));
  }
  if (skip && h->shared_m > 0) ALLOC(h->s32, T * h->d * sizeof(float));
  if (h->flags & (LMOE_EXPERTS_FP8 | LMOE_EXPERTS_FP4)) ALLOC(h->a16, T * (skip ? h->d : h->l) * 2);
  if (h->flags & LMOE_SORTED_ROWS) ALLOC(h->zs, R * (skip ? h->d : h->l) * 2);
  if (h->dtype == LMOE_BF16) {
    h->part_bytes = kSplitPartBytes;
    ALLOC(h->part, h->part_bytes);
    ALLOC(h->part_side, h->part_bytes);
  }
  LMOE_CUDA(h, cudaStreamCreateWithFlags(&h->side_stream, cudaStreamNonBlocking));
  for (cudaEvent_t* e : {&h->ev_fork, &h->ev_side})
    LMOE_CUDA(h, cudaEventCreateWithFlags(e, cudaEventDisableTiming));
#undef ALLOC
  LMOE_CUDA(h, cudaMemset(h->bitmap, 0, (size_t)h->N * W * sizeof(uint32_t)));
  LMOE_CUDA(h, cudaMemset(h->done, 0, sizeof(unsigned)));
  LMOE_CUDA(h, cudaMemset(h->err, 0, sizeof(int)));
  LMOE_CUDA(h, cudaMemset(h->offsets, 0, (size_t)(h->N + 1) * sizeof(int)));
  LMOE_CUDA(h, cudaMemset(h->tile_prefix, 0, (size_t)(h->N + 1) * sizeof(int)));
  LMOE_CUDA(h, cudaMemset(h->tile_prefix2, 0, (size_t)(h->N + 1) * sizeof(int)));
  LMOE_CUDA(h, cudaMemset(h->tile_prefix64, 0, (size_t)(h->N + 1) * sizeof(int)));
  LMOE_CUDA(h, cudaMemset(h->big_prefix2, 0, (size_t)(h->N + 1) * sizeof(int)));
  LMOE_CUDA(h, cudaMemset(h->small_prefix, 0, (size_t)(h->N + 1) * sizeof(int)));
  LMOE_CUDA(h, cudaMemset(h->small_prefix2, 0, (size_t)(h->N + 1) * sizeof(int)));
  LMOE_CUDA(h, cudaMemset(h->full_prefix2, 0, (size_t)(h->N + 1) * sizeof(int)));
  LMOE_CUDA(h, cudaMemset(h->rem_prefix, 0, (size_t)(h->N + 1) * sizeof(int)));
  if (h->sk_count) LMOE_CUDA(h, cudaMemset(h->sk_count, 0, (size_t)(h->num_sms + 1) * sizeof(int)));
  LMOE_CUDA(h, cudaDeviceSynchronize());
  h->max_T = max_T;
  h->W = (int)W;
  Grouping& fg = h->fwd_grp;
  fg.G = h->N;
  fg.e0 = 0;
  fg.offsets = h->offsets;
  fg.tp128 = h->tile_prefix;
  fg.tp256 = h->tile_prefix2;
  fg.tp64 = h->tile_prefix64;
  fg.big256 = h->big_prefix2;
  fg.small128 = h->small_prefix;
  fg.small256 = h->small_prefix2;
  fg.full256 = h->full_prefix2;
  fg.rem128 = h->rem_prefix;
  return LMOE_OK;
}

lmoe_status lmoe_forward(lmoe_layer* h, const void* x, void* out, int T, lmoe_stream_t stream) {
  if (!h) return LMOE_ERR_INVALID_ARG;
  if (!layer_ready(h) || h->max_T == 0) return LMOE_ERR_NOT_READY;
  if (!valid_stream_call(h, T)) return LMOE_ERR_INVALID_ARG;
  if (T == 0) return LMOE_OK;
  if (!x || !out || x == out) return LMOE_ERR_INVALID_ARG;
  DevGuard g(h->device);
  return run_forward(h, x, out, T, (cudaStream_t)stream);
}

lmoe_status lmoe_forward_host(lmoe_layer* h, const void* x_host, void* out_host, int T,
                              lmoe_stream_t stream) {
  if (!h) return LMOE_ERR_INVALID_ARG;
  if (!layer_ready(h) || h->max_T == 0) return LMOE_ERR_NOT_READY;
  if (!valid_stream_call(h, T)) return LMOE_ERR_INVALID_ARG;
  if (T == 0) return LMOE_OK;
  if (!x_host || !out_host) return LMOE_ERR_INVALID_ARG;
  DevGuard g(h->device);
  cudaStream_t st = (cudaStream_t)stream;
  const size_t bytes = (size_t)T * h->d * h->es;
  // The upload runs on the library's copy stream into one of two staging
  // slots, so that it can overlap the previous call's forward (which reads
  // the other slot); it waits until the forward that last read this slot has
  // finished.  The caller's stream waits for the upload; the download stays
  // on the caller's stream, so out_host is complete when that stream is.
  const int s = h->host_slot;
  h->host_slot ^= 1;
  void* xs = s ? h->x_stage2 : h->x_stage;
  LMOE_CUDA(h, cudaStreamWaitEvent(h->copy_stream, h->ev_used[s], 0));
  LMOE_CUDA(h, cudaMemcpyAsync(xs, x_host, bytes, cudaMemcpyHostToDevice, h->copy_stream));
  LMOE_CUDA(h, cudaEventRecord(h->ev_up[s], h->copy_stream));
  LMOE_CUDA(h, cudaStreamWaitEvent(st, h->ev_up[s], 0));
  LMOE_TRY(run_forward(h, xs, h->out_stage, T, st));
  LMOE_CUDA(h, cudaEventRecord(h->ev_used[s], st));
  LMOE_CUDA(h, cudaMemcpyAsync(out_host, h->out_stage, bytes, cudaMemcpyDeviceToHost, st));
  return LMOE_OK;
}

lmoe_status lmoe_selftest_wait_timeout(lmoe_layer* h, unsigned limit_us, lmoe_stream_t stream) {
  if (!h || limit_us == 0 || limit_us > 1000000u) return LMOE_ERR_INVALID_ARG;
  if (h->max_T == 0) return LMOE_ERR_NOT_READY;
  DevGuard g(h->device);
  wait_selftest_kernel<<<1, 32, 0, (cudaStream_t)stream>>>(h->err, 1000ull * limit_us);
  LMOE_CUDA(h, cudaGetLastError());
  return LMOE_OK;
}

lmoe_status lmoe_route_only(lmoe_layer* h, const float* logits, int T, int* idx, float* w,
                            int* offsets, int* perm, lmoe_stream_t stream) {
  if (!h) return LMOE_ERR_INVALID_ARG;
  if (h->max_T == 0) return LMOE_ERR_NOT_READY;
  if (!valid_stream_call(h, T)) return LMOE_ERR_INVALID_ARG;
  if (!offsets) return LMOE_ERR_INVALID_ARG;
  if (T > 0 && (!logits || !idx || !w || !perm)) return LMOE_ERR_INVALID_ARG;
  DevGuard g(h->device);
  cudaStream_t st = (cudaStream_t)stream;
  h->launches = 0;
  if (T == 0) {
    LMOE_CUDA(h, cudaMemsetAsync(offsets, 0, (size_t)(h->N + 1) * sizeof(int), st));
    return LMOE_OK;
  }
  h->pdl_hold = true;
  return run_routing(h, logits, T, idx, w, offsets, nullptr, perm, nullptr, nullptr, nullptr, st,
                     false);
}

lmoe_status lmoe_router_logits(lmoe_layer* h, const void* x, float* logits, int T,
                               lmoe_stream_t stream) {
  if (!h) return LMOE_ERR_INVALID_ARG;
  if (!layer_ready(h) || h->max_T == 0) return LMOE_ERR_NOT_READY;
  if (!valid_stream_call(h, T)) return LMOE_ERR_INVALID_ARG;
  if (T == 0) return LMOE_OK;
  if (!x || !logits) return LMOE_ERR_INVALID_ARG;
  DevGuard g(h->device);
  h->launches = 0;
  h->pdl_hold = true;
  return run_router(h, x, logits, T, (cudaStream_t)stream);
}

lmoe_status lmoe_stage_bytes(const lmoe_layer* h, int stage, int T, size_t* bytes) {
  if (!h || !bytes || T < 0) return LMOE_ERR_INVALID_ARG;
  const size_t t = T, R = t * h->k, es = h->es;
  const bool skip = (h->flags & LMOE_SKIP_PROJ) != 0;
  switch (stage) {
    case LMOE_STAGE_LOGITS: *bytes = t * h->N * 4; break;
    case LMOE_STAGE_IDX:
    case LMOE_STAGE_W:
    case LMOE_STAGE_PERM: *bytes = R * 4; break;
    case LMOE_STAGE_OFFSETS: *bytes = (size_t)(h->N + 1) * 4; break;
    case LMOE_STAGE_Z:
      if (skip) return LMOE_ERR_INVALID_ARG;
      *bytes = t * h->l * es;
      break;
    case LMOE_STAGE_H: *bytes = R * h->m * es; break;
    case LMOE_STAGE_YS: *bytes = R * h->l * es; break;
    case LMOE_STAGE_COMB:
      if (skip) return LMOE_ERR_INVALID_ARG;
      *bytes = t * h->l * es;
      break;
    default: return LMOE_ERR_INVALID_ARG;
  }
  return LMOE_OK;
}

lmoe_status lmoe_debug_dump(lmoe_layer* h, int stage, void* dst, size_t bytes, lmoe_stream_t stream) {
  if (!h || !dst) return LMOE_ERR_INVALID_ARG;
  if (h->last_T < 0) return LMOE_ERR_NOT_READY;
  size_t need = 0;
  LMOE_TRY(lmoe_stage_bytes(h, stage, h->last_T, &need));
  if (bytes < need) return LMOE_ERR_INVALID_ARG;
  if (need == 0) return LMOE_OK;
  const void* src = nullptr;
  size_t pitch = 0, width = 0, rows = 0;
  switch (stage) {
    case LMOE_STAGE_LOGITS: src = h->logits; break;
    case LMOE_STAGE_IDX: src = h->idx; break;
    case LMOE_STAGE_W: src = h->w; break;
    case LMOE_STAGE_OFFSETS: src = h->offsets; break;
    case LMOE_STAGE_PERM: src = h->row_slot; break;
    case LMOE_STAGE_Z: src = h->z; break;
    case LMOE_STAGE_H: src = h->h; break;
    case LMOE_STAGE_YS: src = h->ys; break;
    case LMOE_STAGE_COMB:  // the first l columns of the [T, l + shared_m] operand
      src = h->cat;
      pitch = (size_t)h->Kup * h->es;
      width = (size_t)h->l * h->es;
      rows = (size_t)h->last_T;
      break;
  }
  DevGuard g(h->device);
  if (pitch)
    LMOE_CUDA(h, cudaMemcpy2DAsync(dst, width, src, pitch, width, rows, cudaMemcpyDeviceToDevice,
                                   (cudaStream_t)stream));
  else
    LMOE_CUDA(h, cudaMemcpyAsync(dst, src, need, cudaMemcpyDeviceToDevice, (cudaStream_t)stream));
  return LMOE_OK;
}

lmoe_status lmoe_last_error(lmoe_layer* h, int* device_error_word) {
  if (!h || !device_error_word) return LMOE_ERR_INVALID_ARG;
  *device_error_word = 0;
  if (!h->err) return LMOE_OK;
  DevGuard g(h->device);
  LMOE_CUDA(h, cudaDeviceSynchronize());
  int word = 0;
  LMOE_CUDA(h, cudaMemcpy(&word, h->err, sizeof(int), cudaMemcpyDeviceToHost));
  LMOE_CUDA(h, cudaMemset(h->err, 0, sizeof(int)));
  *device_error_word = word;
  if (word & LMOE_DEVERR_WAIT_TIMEOUT) return LMOE_ERR_TIMEOUT;
  if (word) return LMOE_ERR_DEVICE;
  return LMOE_OK;
}

lmoe_status lmoe_profile_begin(lmoe_layer* h, int max_forwards) {
  return lmoe_profile_begin_stages(h, max_forwards, (1u << kStages) - 1);
}

lmoe_status lmoe_profile_begin_stages(lmoe_layer* h, int max_forwards, unsigned stage_mask) {
  if (!h || max_forwards < 1 || (stage_mask & ((1u << kStages) - 1)) == 0)
    return LMOE_ERR_INVALID_ARG;
  DevGuard g(h->device);
  LMOE_CUDA(h, cudaDeviceSynchronize());
  destroy_events(h);
  const size_t n = (size_t)max_forwards * kMarks;
  h->events.resize(n, nullptr);
  h->prof_side.assign((size_t)max_forwards, 0);
  for (size_t i = 0; i < n; ++i) {
    cudaError_t e = cudaEventCreate(&h->events[i]);
    if (e != cudaSuccess) {
      h->events.resize(i);
      destroy_events(h);
      return cuda_fail(h, e, "cudaEventCreate");
    }
  }
  h->prof_cap = max_forwards;
  h->prof_count = 0;
  h->prof_mask = stage_mask & ((1u << kStages) - 1);
  h->profiling = true;
  return LMOE_OK;
}

lmoe_status lmoe_profile_end(lmoe_layer* h, float* ms, int capacity, int* n_forwards, int* n_stages) {
  if (!h || !n_forwards || !n_stages || (capacity > 0 && !ms)) return LMOE_ERR_INVALID_ARG;
  DevGuard g(h->device);
  *n_forwards = 0;
  *n_stages = kStages;
  if (!h->profiling) return LMOE_ERR_NOT_READY;
  LMOE_CUDA(h, cudaDeviceSynchronize());
  int written = 0;
  for (int f = 0; f < h->prof_count; ++f) {
    if ((f + 1) * kStages > capacity) break;
    cudaEvent_t* ev = &h->events[(size_t)f * kMarks];
    for (int s = 0; s < kStages; ++s) {
      if (!((h->prof_mask >> s) & 1u)) {
        ms[f * kStages + s] = -1.f;  // not recorded
        continue;
      }
      // with the side stream, the down-projection and shared FC1 stages are
      // timed there (they overlap the router and routing stages)
      int a = s, b = s + 1;
      if (h->prof_side[f] && (s == 3 || s == 4)) {
        a = kSideMark0 + (s - 3);
        b = a + 1;
      }
      float t = 0.f;
      LMOE_CUDA(h, cudaEventElapsedTime(&t, ev[a], ev[b]));
      ms[f * kStages + s] = t;
    }
    written = f + 1;
  }
  *n_forwards = written;
  destroy_events(h);
  return LMOE_OK;
}

// ---- expert parallelism ------------------------------------------------------

lmoe_status lmoe_ep_local_plan(const int* recv_counts, int world, int n_local, int* offsets,
                               int* perm) {
  if (!recv_counts || !offsets || world < 1 || n_local < 1) return LMOE_ERR_INVALID_ARG;
  std::vector<int> counts(n_local), src(world + 1), roff((size_t)world * n_local),
      goff((size_t)world * n_local);
  const long Rr = ep_host_tables(recv_counts, world, n_local, counts.data(), offsets, src.data(),
                                 roff.data(), goff.data());
  if (Rr < 0 || Rr > INT32_MAX) return LMOE_ERR_INVALID_ARG;
  if (Rr > 0 && !perm) return LMOE_ERR_INVALID_ARG;
  for (int s = 0; s < world; ++s)
    for (int e = 0; e < n_local; ++e) {
      const int c = recv_counts[(size_t)s * n_local + e];
      for (int i = 0; i < c; ++i) perm[goff[(size_t)e * world + s] + i] = roff[(size_t)s * n_local + e] + i;
    }
  return LMOE_OK;
}

lmoe_status lmoe_ep_reserve(lmoe_layer* h, int max_recv_rows) {
  if (!h || max_recv_rows < 1) return LMOE_ERR_INVALID_ARG;
  if (h->max_T == 0) return LMOE_ERR_NOT_READY;
  if (max_recv_rows <= h->ep_max_rows) return LMOE_OK;
  DevGuard g(h->device);
  LMOE_CUDA(h, cudaDeviceSynchronize());
  free_ep(h);
  const size_t N = h->N, Rr = max_recv_rows, es = h->es;
  const size_t tab = 4 * (N + 1) + 7 * (N + 1);
#define ALLOC(ptr, bytes) LMOE_CUDA(h, cudaMalloc((void**)&(ptr), std::max<size_t>(bytes, 16)))
  ALLOC(h->ep_tab, tab * sizeof(int));
  LMOE_CUDA(h, cudaMallocHost((void**)&h->ep_tab_host, 4 * (N + 1) * sizeof(int)));
  LMOE_CUDA(h, cudaEventCreateWithFlags(&h->ep_uploaded, cudaEventDisableTiming));
  ALLOC(h->ep_perm, Rr * sizeof(int));
  ALLOC(h->ep_inv, Rr * sizeof(int));
  ALLOC(h->ep_gates, Rr * sizeof(float));
  ALLOC(h->ep_h, Rr * h->m * es);
  ALLOC(h->ep_ys, Rr * h->l * es);
#undef ALLOC
  LMOE_CUDA(h, cudaMemset(h->ep_tab, 0, tab * sizeof(int)));
  h->ep_max_rows = max_recv_rows;
  return LMOE_OK;
}

lmoe_status lmoe_ep_dispatch(lmoe_layer* h, const void* x, int T, void* send_rows,
                             float* send_gates, int* expert_counts, lmoe_stream_t stream) {
  if (!h) return LMOE_ERR_INVALID_ARG;
  if (!layer_ready(h) || h->max_T == 0) return LMOE_ERR_NOT_READY;
  if (h->flags & (LMOE_EXPERTS_FP8 | LMOE_EXPERTS_FP4)) return LMOE_ERR_UNSUPPORTED;
  if (T < 1 || T > h->max_T || !x || !send_rows || !send_gates || !expert_counts)
    return LMOE_ERR_INVALID_ARG;
  DevGuard g(h->device);
  cudaStream_t st = (cudaStream_t)stream;
  const bool prof = h->profiling;  // profiling covers lmoe_forward only
  h->profiling = false;
  h->launches = 0;
  const lmoe_status r = run_front(h, x, T, st);
  h->profiling = prof;
  LMOE_TRY(r);
  const bool skip = (h->flags & LMOE_SKIP_PROJ) != 0;
  const int cols = skip ? h->d : h->l;
  const void* A = skip ? x : h->z;
  const long R = (long)T * h->k;
  const int vec = (cols % 8 == 0 && aligned16(A) && aligned16(send_rows)) ? 1 : 0;
  const unsigned blocks = (unsigned)std::max<long>(1, std::min<long>((R + 7) / 8, 8L * h->num_sms));
  if (h->dtype == LMOE_BF16) {
    LMOE_LAUNCH(h, gather_rows_kernel, dim3(blocks), dim3(256), 0, st,
                static_cast<const uint16_t*>(A), (long)cols, (const int*)h->row_tok, R, cols,
                static_cast<uint16_t*>(send_rows), vec);
  } else {  // fp32 rows: two 16-bit halves per element
    LMOE_LAUNCH(h, gather_rows_kernel, dim3(blocks), dim3(256), 0, st,
                static_cast<const uint16_t*>(A), 2L * cols, (const int*)h->row_tok, R, 2 * cols,
                static_cast<uint16_t*>(send_rows), vec);
  }
  LMOE_CUDA(h, cudaMemcpyAsync(send_gates, h->row_w, R * sizeof(float), cudaMemcpyDeviceToDevice,
                               st));
  LMOE_CUDA(h, cudaMemcpyAsync(expert_counts, h->counts, (size_t)h->N * sizeof(int),
                               cudaMemcpyDeviceToDevice, st));
  h->ep_T = T;
  h->pdl_hold = true;  // the next launch follows memcpys: full stream order
  return LMOE_OK;
}

lmoe_status lmoe_ep_experts(lmoe_layer* h, const void* recv_rows, const float* recv_gates,
                            const int* recv_counts, int rank, int world, void* out_rows,
                            lmoe_stream_t stream) {
  if (!h) return LMOE_ERR_INVALID_ARG;
  if (!layer_ready(h)) return LMOE_ERR_NOT_READY;
  if (h->ep_max_rows == 0) return LMOE_ERR_NOT_READY;
  if (h->flags & (LMOE_EXPERTS_FP8 | LMOE_EXPERTS_FP4)) return LMOE_ERR_UNSUPPORTED;
  if (!recv_counts || world < 1 || rank < 0 || rank >= world || h->N % world != 0)
    return LMOE_ERR_INVALID_ARG;
  const int n = h->N / world;
  DevGuard g(h->device);
  cudaStream_t st = (cudaStream_t)stream;
  // host tables into the pinned staging buffer (after its previous upload)
  LMOE_CUDA(h, cudaEventSynchronize(h->ep_uploaded));
  const size_t N1 = (size_t)h->N + 1;
  int* hc = h->ep_tab_host;  // counts [n] | src_start [world+1] | roff [world n] | goff [n world]
  std::vector<int> offsets(n + 1);
  const long Rr = ep_host_tables(recv_counts, world, n, hc, offsets.data(), hc + N1, hc + 2 * N1,
                                 hc + 3 * N1);
  if (Rr < 0) return LMOE_ERR_INVALID_ARG;
  if (Rr > h->ep_max_rows) return LMOE_ERR_UNSUPPORTED;
  if (Rr > 0 && (!recv_rows || !recv_gates || !out_rows)) return LMOE_ERR_INVALID_ARG;
  h->launches = 0;
  if (Rr == 0) return LMOE_OK;
  int* dt = h->ep_tab;
  LMOE_CUDA(h, cudaMemcpyAsync(dt, hc, 4 * N1 * sizeof(int), cudaMemcpyHostToDevice, st));
  LMOE_CUDA(h, cudaEventRecord(h->ep_uploaded, st));
  int* d_offsets = dt + 4 * N1;
  int* pref = dt + 5 * N1;  // tp128, tp256, tp64, big256, small128, small256
  h->pdl_hold = true;  // after a memcpy: full stream order
  LMOE_LAUNCH(h, ep_scan_kernel, dim3(1), dim3(256), 0, st, (const int*)dt, n, d_offsets, pref,
              pref + N1, pref + 2 * N1, pref + 3 * N1, pref + 4 * N1, pref + 5 * N1);
  const unsigned pblocks =
      (unsigned)std::max<long>(1, std::min<long>((Rr + 255) / 256, 8L * h->num_sms));
  LMOE_LAUNCH(h, ep_perm_kernel, dim3(pblocks), dim3(256), 0, st, Rr, world, n,
              (const int*)(dt + N1), (const int*)(dt + 2 * N1), (const int*)(dt + 3 * N1),
              recv_gates, h->ep_perm, h->ep_inv, h->ep_gates);
  Grouping& eg = h->ep_grp;
  eg.G = n;
  eg.e0 = rank * n;
  eg.offsets = d_offsets;
  eg.tp128 = pref;
  eg.tp256 = pref + N1;
  eg.tp64 = pref + 2 * N1;
  eg.big256 = pref + 3 * N1;
  eg.small128 = pref + 4 * N1;
  eg.small256 = pref + 5 * N1;
  const bool skip = (h->flags & LMOE_SKIP_PROJ) != 0;
  const int cols = skip ? h->d : h->l;
  const bool prof = h->profiling;
  h->profiling = false;
  const lmoe_status r = run_expert_gemms(h, eg, recv_rows, cols, Rr, h->ep_perm, Rr, h->ep_h,
                                         h->ep_ys, h->ep_gates, st);
  h->profiling = prof;
  LMOE_TRY(r);
  // the outputs back in received order
  const int l = h->l;
  const int vec = (l % 8 == 0 && aligned16(out_rows)) ? 1 : 0;
  const unsigned blocks = (unsigned)std::max<long>(1, std::min<long>((Rr + 7) / 8, 8L * h->num_sms));
  const int ecols = h->dtype == LMOE_BF16 ? l : 2 * l;
  LMOE_LAUNCH(h, gather_rows_kernel, dim3(blocks), dim3(256), 0, st,
              static_cast<const uint16_t*>(h->ep_ys), (long)ecols, (const int*)h->ep_inv, Rr, ecols,
              static_cast<uint16_t*>(out_rows), vec);
  return LMOE_OK;
}

lmoe_status lmoe_ep_combine(lmoe_layer* h, const void* x, const void* back_rows, void* out, int T,
                            lmoe_stream_t stream) {
  if (!h) return LMOE_ERR_INVALID_ARG;
  if (h->ep_T < 0 || T != h->ep_T) return LMOE_ERR_NOT_READY;
  if (!x || !back_rows || !out || x == out) return LMOE_ERR_INVALID_ARG;
  DevGuard g(h->device);
  const bool prof = h->profiling;
  h->profiling = false;
  h->launches = 0;
  h->pdl_hold = true;  // the rows arrived by copies the library does not see
  const lmoe_status r = run_back(h, x, back_rows, out, T, (cudaStream_t)stream);
  h->profiling = prof;
  h->ep_T = -1;
  h->last_T = T;
  return r;
}

int lmoe_last_launch_count(const lmoe_layer* h) { return h ? h->launches : 0; }
int lmoe_last_expert_path(const lmoe_layer* h) { return h ? h->expert_path : -1; }

void lmoe_destroy(lmoe_layer* h) {
  if (!h) return;
  {
    DevGuard g(h->device);
    cudaDeviceSynchronize();
    destroy_events(h);
    free_workspace(h);
    free_ep(h);
    free_weights(h);
  }
  delete h;
}

}  // extern "C"
