// Host side of the C ABI declared in include/fp8pd.h: argument validation
// (nothing is launched unless every check passes), split planning, the
// per-device split workspace, options, run info and optional kernel timing.

#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstring>
#include <mutex>
#include <vector>

#include "../../include/fp8pd.h"
#include "fp8pd_internal.h"

// L2 promotion of the pool tensor maps' tile loads (a build setting).
#ifndef FP8PD_L2_PROMOTION
#define FP8PD_L2_PROMOTION CU_TENSOR_MAP_L2_PROMOTION_L2_256B
#endif

using fp8pd::AppendParams;
using fp8pd::DecodeParams;

namespace {

constexpr int kMaxDevices = 64;

thread_local int32_t t_last_cuda_error = 0;
thread_local fp8pd_run_info t_run_info = {};
std::atomic<int64_t> g_calls{0}, g_appends{0}, g_launches{0};
std::atomic<int64_t> g_opt_num_splits{0}, g_opt_schedule{0}, g_opt_k_decode{1}, g_opt_v_decode{1},
    g_opt_wait_polls{1 << 17}, g_opt_test_stall{0}, g_opt_compute{0}, g_opt_kernel{0};

struct Workspace {
  void* ptr = nullptr;
  size_t bytes = 0;
};
std::mutex g_ws_mutex;
Workspace g_ws[kMaxDevices];

struct EventPair {
  cudaEvent_t a = nullptr, b = nullptr;
  int kind = 0;  // 0 = attention kernel, 1 = append kernel
};
std::mutex g_timing_mutex;
std::atomic<int> g_timing_on{0};
std::vector<EventPair> g_timing_pool;  // events of the current device(s)
size_t g_timing_used = 0;

int fail_cuda(cudaError_t e) {
  t_last_cuda_error = static_cast<int32_t>(e);
  return FP8PD_ERR_CUDA;
}

bool is_capturing(cudaStream_t s) {
  cudaStreamCaptureStatus st = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(s, &st) != cudaSuccess) {
    cudaGetLastError();
    return false;
  }
  return st != cudaStreamCaptureStatusNone;
}

// ---- descriptor checks -------------------------------------------------------
int check(const fp8pd_tensor* t, int32_t dtype, int32_t ndim) {
  if (!t || !t->data) return FP8PD_ERR_NULL;
  if (t->dtype != dtype) return FP8PD_ERR_DTYPE;
  if (t->ndim != ndim) return FP8PD_ERR_SHAPE;
  for (int i = 0; i < ndim; ++i)
    if (t->shape[i] < 0) return FP8PD_ERR_SHAPE;
  return FP8PD_OK;
}

bool fits_i32(int64_t v) { return v >= 0 && v <= INT32_MAX; }

// Scale descriptor -> (page, slot, head, group) strides in elements; *tok =
// 1 for the per-token form [num_pages, ps, Hkv] (one scale per stored token
// and KV head), 0 for [Hkv] (slot and page strides 0) and [num_pages, Hkv]
// (slot stride 0). [num_pages, ps, Hkv, groups] adds sub-row groups (*groups
// = the last extent, a power of two up to 16 dividing d; 1 otherwise);
// `max_groups` caps it (1: no sub-row groups).
int scale_strides(const fp8pd_tensor* s, int64_t num_pages, int64_t ps, int64_t hkv, int64_t d,
                  int max_groups, int64_t* sp, int64_t* st, int64_t* sh, int64_t* sg, int* tok,
                  int* groups, int* mx = nullptr) {
  if (!s || !s->data) return FP8PD_ERR_NULL;
  *st = 0;
  *sg = 0;
  *tok = 0;
  *groups = 1;
  if (mx) *mx = 0;
  if (s->dtype == FP8PD_DTYPE_U8) {
    // MXFP8: E8M0 block scales [num_pages, ps, Hkv, D / 32], one byte per 32 entries
    if (!mx) return FP8PD_ERR_DTYPE;
    if (s->ndim != 4) return FP8PD_ERR_SHAPE;
    if (d % 32) return FP8PD_ERR_UNSUPPORTED;
    if (s->shape[0] != num_pages || s->shape[1] != ps || s->shape[2] != hkv || s->shape[3] != d / 32)
      return FP8PD_ERR_SHAPE;
    *sp = s->stride[0];
    *st = s->stride[1];
    *sh = s->stride[2];
    *sg = s->stride[3];
    *tok = 1;
    *groups = static_cast<int>(d / 32);
    *mx = 1;
    return FP8PD_OK;
  }
  if (s->dtype != FP8PD_DTYPE_F32) return FP8PD_ERR_DTYPE;
  if (s->ndim == 1) {
    if (s->shape[0] != hkv) return FP8PD_ERR_SHAPE;
    *sp = 0;
    *sh = s->stride[0];
    return FP8PD_OK;
  }
  if (s->ndim == 2) {
    if (s->shape[0] != num_pages || s->shape[1] != hkv) return FP8PD_ERR_SHAPE;
    *sp = s->stride[0];
    *sh = s->stride[1];
    return FP8PD_OK;
  }
  if (s->ndim == 3 || s->ndim == 4) {
    if (s->shape[0] != num_pages || s->shape[1] != ps || s->shape[2] != hkv) return FP8PD_ERR_SHAPE;
    *sp = s->stride[0];
    *st = s->stride[1];
    *sh = s->stride[2];
    *tok = 1;
    if (s->ndim == 4) {
      const int64_t g = s->shape[3];
      if (g < 1 || g > 16 || (g & (g - 1)) || d % g) return FP8PD_ERR_UNSUPPORTED;
      if (g > max_groups) return FP8PD_ERR_UNSUPPORTED;
      *sg = s->stride[3];
      *groups = static_cast<int>(g);
    }
    return FP8PD_OK;
  }
  return FP8PD_ERR_SHAPE;
}

// Pool view [num_pages, ps, Hkv, D] of uint8 codes.
int check_pool(const fp8pd_tensor* t, bool aligned) {
  int r = check(t, FP8PD_DTYPE_U8, 4);
  if (r) return r;
  if (t->stride[3] != 1) return FP8PD_ERR_ALIGN;
  if (aligned) {
    if (reinterpret_cast<uintptr_t>(t->data) % 16) return FP8PD_ERR_ALIGN;
    for (int i = 0; i < 3; ++i)
      if (t->stride[i] % 16 || t->stride[i] < 0) return FP8PD_ERR_ALIGN;
  }
  return FP8PD_OK;
}

bool same_pool_shape(const fp8pd_tensor* a, const fp8pd_tensor* b) {
  for (int i = 0; i < 4; ++i)
    if (a->shape[i] != b->shape[i]) return false;
  return true;
}

struct Plan {
  int num_splits = 1;
  int chunk_pages = 1;
  int head_groups = 1;
  int grid_blocks = 0;
  int combine = 0;
  int num_groups = 1;
  size_t counters_bytes = 0;  // ticket counters (counter area of the workspace)
  size_t ml_bytes = 0;        // split (max, sum) pairs
  size_t o_bytes = 0;         // split numerators
  size_t grp_ml_bytes = 0;    // merged groups of splits
  size_t grp_o_bytes = 0;
  size_t workspace = 0;
  int schedule = 1;            // 1 = uniform splits, 3 = proportional splits
  int nbx = 0;                 // proportional: blocks per KV head x head group
};

int current_device(int* dev) {
  cudaError_t e = cudaGetDevice(dev);
  if (e != cudaSuccess) return fail_cuda(e);
  if (*dev < 0 || *dev >= kMaxDevices) return FP8PD_ERR_TOO_LARGE;
  return FP8PD_OK;
}

// Splits per (sequence, KV head, head group). Split s covers pages
// [s * chunk, (s+1) * chunk) of a sequence's attended range, so every block
// has the same amount of work whatever the sequence lengths (blocks past the
// end of a short sequence finish at once). The count aims at just under two
// waves of the device, with >= 512 keys per split, never more than 8,192 keys
// per split (the kernel's per-warp tile list) nor more than kMaxSplits splits.
size_t align256(size_t v) { return (v + 255) & ~static_cast<size_t>(255); }

int device_sms() {
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) {
    int v = 0;
    if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess && v > 0) sms = v;
  }
  cudaGetLastError();
  return sms;
}

// Proportional splits: the split kernel on a grid of nbx blocks per KV head x
// head group, shared among the sequences in the kernel in proportion to their
// tiles (at least one block per sequence with keys, and no split above 8,192
// keys). nbx is one full wave of blocks, or two when the sequences would
// take more than half a wave with one block each (then rounding would leave
// many blocks a whole sequence, so a second wave of halves balances better).
// Needs at most 1,024 sequences; the planner's own choice also needs at least
// 4 tiles per block slot when every sequence has its table's full length.
// Whether the tensor-memory kernel runs a call: head dim 64 or 128, page or
// head scales (no per-token, sub-row or MX scales), f32 compute with the
// hardware-cvt decodes, no timeout test hook, and FP8PD_OPT_KERNEL not 1.
constexpr bool kUmmaByDefault = false;
bool use_umma(int D, bool tok, bool mx, int k_groups) {
  const int64_t k = g_opt_kernel.load();
  if (k == 1 || (D != 64 && D != 128) || tok || mx || k_groups > 1) return false;
  if (g_opt_compute.load() != 0 || g_opt_k_decode.load() != 1 || g_opt_v_decode.load() != 1 ||
      g_opt_test_stall.load() != 0)
    return false;
  return k == 2 || kUmmaByDefault;
}

// Warps per tile stream of the split kernel, each on its part of the head
// dim: FP8PD_DSPLIT_D512 at D = 512 with page or head scales, f32 compute
// with the hardware-cvt decodes and no fused append (at D = 512 a block of
// four whole-width streams fills the SM's shared memory with four warps);
// otherwise 1.
int use_dsplit(int D, bool tok, bool mx, int k_groups, bool append, bool umma) {
  static_assert(FP8PD_DSPLIT_D512 == 1 || FP8PD_DSPLIT_D512 == 2 || FP8PD_DSPLIT_D512 == 4,
                "FP8PD_DSPLIT_D512: 1, 2 or 4");
  if (D != 512 || umma || tok || mx || k_groups > 1 || append) return 1;
  if (g_opt_compute.load() != 0 || g_opt_k_decode.load() != 1 || g_opt_v_decode.load() != 1)
    return 1;
  return FP8PD_DSPLIT_D512;
}

// Thread blocks one SM holds for the kernel that will run.
int blocks_per_sm(int D, bool umma, int dsplit = 1) {
  return umma ? fp8pd::decode_umma_blocks_per_sm(D) : fp8pd::decode_blocks_per_sm(D, dsplit);
}

bool plan_proportional(int B, int Hq, int Hkv, int D, int ps, int max_pages, int window,
                       Plan* plan, bool umma) {
  if (g_opt_num_splits.load() > 0 || B > fp8pd::kPropMaxBatch) return false;
  const int G = Hq / Hkv;
  const int hg = (G + fp8pd::kHeadsPerGroup - 1) / fp8pd::kHeadsPerGroup;
  const int64_t HX = static_cast<int64_t>(Hkv) * hg;
  const int64_t keys = static_cast<int64_t>(max_pages) * ps;
  const int64_t seq_tiles = window > 0 ? std::min<int64_t>(keys, window) / fp8pd::kTileTokens + 2
                                       : (keys + fp8pd::kTileTokens - 1) / fp8pd::kTileTokens;
  const int64_t m_max = (seq_tiles + fp8pd::kMaxSplitTiles - 1) / fp8pd::kMaxSplitTiles;
  if (m_max > fp8pd::kMaxSplits) return false;
  const int64_t slots = static_cast<int64_t>(device_sms()) * blocks_per_sm(D, umma);
  if (g_opt_schedule.load() == 0 && B * HX * seq_tiles < 4 * slots) return false;  // little work
#ifdef FP8PD_PROP_WAVES
  const int64_t waves = FP8PD_PROP_WAVES;  // tuning builds
#else
  const int64_t waves = (static_cast<int64_t>(B) * HX * 2 > slots) ? 2 : 1;
#endif
  int64_t nbx = (waves * slots + HX - 1) / HX;
  // By default only in one wave: with a second wave every later block pays
  // the split search again and the blocks without a split still take slots,
  // and uniform splits measured faster there (equal-length batches of 64
  // sequences, and 8 sequences of 131k keys).
  if (g_opt_schedule.load() == 0 && (waves > 1 || B * m_max > nbx)) return false;
  nbx = std::max<int64_t>(nbx, B * m_max);  // room for every sequence's minimum splits
  nbx = std::min<int64_t>(nbx, std::min<int64_t>(65535, static_cast<int64_t>(B) * fp8pd::kMaxSplits));
  if (nbx < B * m_max) return false;
  plan->schedule = 3;
  plan->head_groups = hg;
  plan->nbx = static_cast<int>(nbx);
  plan->num_splits = 0;
  plan->chunk_pages = 0;
  plan->num_groups = 0;
  plan->grid_blocks = static_cast<int>(std::min<int64_t>(INT32_MAX, HX * nbx));
  plan->combine = 1;
  const int64_t groups = nbx / fp8pd::kMergeFan + B + 1;  // >= sum over sequences of ceil(S_b / 8)
  const size_t rows = static_cast<size_t>(nbx * HX) * fp8pd::kHeadsPerGroup;
  const size_t grows = static_cast<size_t>(groups * HX) * fp8pd::kHeadsPerGroup;
  plan->counters_bytes = align256(static_cast<size_t>((B + groups) * HX) * sizeof(int));
  plan->ml_bytes = align256(rows * 2 * sizeof(float));
  plan->o_bytes = align256(rows * D * sizeof(float));
  plan->grp_ml_bytes = align256(grows * 2 * sizeof(float));
  plan->grp_o_bytes = align256(grows * D * sizeof(float));
  plan->workspace = plan->counters_bytes + plan->ml_bytes + plan->o_bytes + plan->grp_ml_bytes +
                    plan->grp_o_bytes;
  return true;
}

int make_plan(int B, int Hq, int Hkv, int D, int ps, int max_pages, int window, Plan* plan,
              bool umma = false) {
  // Proportional splits balance sequences of uneven length within one launch;
  // with a short window every sequence has about the same few tiles, and the
  // uniform splits below cost less.
  const int64_t sched = g_opt_schedule.load();
  if ((sched == 3 || (sched == 0 && (window == 0 || window >= 2048))) &&
      plan_proportional(B, Hq, Hkv, D, ps, max_pages, window, plan, umma))
    return FP8PD_OK;
  plan->schedule = 1;
  const int G = Hq / Hkv;
  plan->head_groups = (G + fp8pd::kHeadsPerGroup - 1) / fp8pd::kHeadsPerGroup;
  const int64_t units = static_cast<int64_t>(B) * Hkv * plan->head_groups;
  int64_t pages = max_pages;
  if (window > 0) pages = std::min<int64_t>(pages, (window + ps - 1) / ps + 1);
  pages = std::max<int64_t>(pages, 1);
  const int64_t max_chunk = std::max<int64_t>(1, fp8pd::kMaxSplitTokens / ps);
  const int64_t s_min = (pages + max_chunk - 1) / max_chunk;
  if (s_min > fp8pd::kMaxSplits) return FP8PD_ERR_TOO_LARGE;  // > 2 Mi keys in one sequence
  const int64_t min_chunk = std::max(1, 512 / ps);
  const int64_t s_max = std::min<int64_t>(
      fp8pd::kMaxSplits, std::max<int64_t>(s_min, (pages + min_chunk - 1) / min_chunk));
  int64_t S = 1;
  const int64_t forced = g_opt_num_splits.load();
  if (forced > 0) {
    S = std::min<int64_t>(forced, std::min<int64_t>(pages, fp8pd::kMaxSplits));
  } else if (units > 0) {
    // Just under two waves of blocks: equal-sized splits fill whole waves
    // for uniform lengths (a partial extra wave would cost a whole split),
    // and the second wave lets the scheduler even out ragged lengths.
    const int sms = device_sms();
    const int64_t slots = static_cast<int64_t>(sms) * blocks_per_sm(D, umma);
    S = std::min<int64_t>(s_max, (2 * slots) / units);
    S = std::max<int64_t>(S, 1);
    // A second wave that the splits cannot fill costs a whole split time with
    // part of the device idle: when one wave of at least two splits per unit
    // fills at least half the slots, take it (a sliding layer of 128 units:
    // 2 splits per unit in one wave instead of 3 in 1.3 waves). With a single
    // split per unit the blocks are too coarse to even out over the SMs
    // (gpt-oss full: 1 split per unit measured slower than 2).
    const int64_t one = std::min<int64_t>(s_max, slots / units);
    if (units * S > slots && one >= std::max<int64_t>(2, s_min) && 2 * units * one >= slots) S = one;
  }
  S = std::max<int64_t>(S, s_min);
  const int64_t chunk = (pages + S - 1) / S;
  S = (pages + chunk - 1) / chunk;
  plan->num_splits = static_cast<int>(S);
  plan->chunk_pages = static_cast<int>(chunk);
  plan->grid_blocks = static_cast<int>(std::min<int64_t>(INT32_MAX, units * S));
  plan->combine = S > 1 ? 1 : 0;
  const int64_t NG = (S + 7) / 8;
  plan->num_groups = static_cast<int>(NG);
  const size_t rows = static_cast<size_t>(B) * Hq;
  plan->counters_bytes = S > 1 ? align256(static_cast<size_t>(units) * (1 + NG) * sizeof(int)) : 0;
  plan->ml_bytes = S > 1 ? align256(rows * S * 2 * sizeof(float)) : 0;
  plan->o_bytes = S > 1 ? align256(rows * S * D * sizeof(float)) : 0;
  plan->grp_ml_bytes = NG > 1 ? align256(rows * NG * 2 * sizeof(float)) : 0;
  plan->grp_o_bytes = NG > 1 ? align256(rows * NG * D * sizeof(float)) : 0;
  plan->workspace = plan->counters_bytes + plan->ml_bytes + plan->o_bytes + plan->grp_ml_bytes +
                    plan->grp_o_bytes;
  return FP8PD_OK;
}

// ---- TMA tensor maps over pool views ---------------------------------------
// A pool view [num_pages, ps, Hkv, D] (byte strides sp, st, sh, 1) is described
// to the TMA as 5 dims, innermost first: head-dim bytes within a 128-byte
// block (min(D, 128)), slot (stride st), 128-byte block (stride 128, D / 128
// of them), KV head (stride sh), page (stride sp). One box = one 16-token tile
// of one KV head, laid out in shared memory as [block][slot][bytes] with the
// 128-byte swizzle (64-byte for D = 64).
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static std::once_flag once;
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &ptr, 12000, cudaEnableDefault,
                                         &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    cudaGetLastError();
  });
  return fn;
}

struct MapKey {
  const void* base;
  int64_t shape[4];
  int64_t stride[4];
  int dsplit;
  bool operator==(const MapKey& o) const {
    return base == o.base && std::memcmp(shape, o.shape, sizeof(shape)) == 0 &&
           std::memcmp(stride, o.stride, sizeof(stride)) == 0 && dsplit == o.dsplit;
  }
};
struct MapEntry {
  MapKey key;
  CUtensorMap map;
};
std::mutex g_map_mutex;
std::vector<MapEntry> g_maps;  // small most-recently-used cache

// The box is one 16-token tile of one KV head: whole rows, or with dsplit = 2
// or 4 the first half or quarter of each row (the kernel moves the start to
// its own part).
int make_pool_map(const fp8pd_tensor* pool, CUtensorMap* out, int dsplit = 1) {
  if (dsplit != 2 && dsplit != 4) dsplit = 1;
  MapKey key{pool->data, {}, {}, dsplit};
  for (int i = 0; i < 4; ++i) {
    key.shape[i] = pool->shape[i];
    key.stride[i] = pool->stride[i];
  }
  {
    std::lock_guard<std::mutex> lock(g_map_mutex);
    for (size_t i = 0; i < g_maps.size(); ++i)
      if (g_maps[i].key == key) {
        *out = g_maps[i].map;
        if (i) std::swap(g_maps[i], g_maps[0]);
        return FP8PD_OK;
      }
  }
  PFN_cuTensorMapEncodeTiled_v12000 enc = encode_fn();
  if (!enc) return fail_cuda(cudaErrorNotSupported);
  const int64_t P = pool->shape[0], ps = pool->shape[1], Hkv = pool->shape[2], D = pool->shape[3];
  const cuuint64_t x = D < 128 ? D : 128;
  const cuuint64_t nblk = D < 128 ? 1 : D / 128;
  const cuuint64_t dims[5] = {x, static_cast<cuuint64_t>(ps), nblk, static_cast<cuuint64_t>(Hkv),
                              static_cast<cuuint64_t>(P)};
  const cuuint64_t strides[4] = {static_cast<cuuint64_t>(pool->stride[1]), 128,
                                 static_cast<cuuint64_t>(pool->stride[2]),
                                 static_cast<cuuint64_t>(pool->stride[0])};
  if (nblk % dsplit != 0) return FP8PD_ERR_SHAPE;
  const cuuint32_t box[5] = {static_cast<cuuint32_t>(x), static_cast<cuuint32_t>(fp8pd::kTileTokens),
                             static_cast<cuuint32_t>(nblk / dsplit), 1, 1};
  const cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  CUtensorMap map;
  const CUresult r = enc(&map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 5, pool->data, dims, strides, box, estr,
                         CU_TENSOR_MAP_INTERLEAVE_NONE,
                         D == 64 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B,
                         FP8PD_L2_PROMOTION, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail_cuda(cudaErrorInvalidValue);
  {
    std::lock_guard<std::mutex> lock(g_map_mutex);
    g_maps.insert(g_maps.begin(), MapEntry{key, map});
    if (g_maps.size() > 32) g_maps.pop_back();
  }
  *out = map;
  return FP8PD_OK;
}

struct DecodeArgs {
  int B, Hq, Hkv, D, ps, num_pages, max_pages;
};

int validate_decode(const fp8pd_tensor* q, const fp8pd_tensor* k_pages, const fp8pd_tensor* v_pages,
                    const fp8pd_tensor* k_scale, const fp8pd_tensor* v_scale,
                    const fp8pd_tensor* block_table, const fp8pd_tensor* seq_lens, int32_t window,
                    const fp8pd_tensor* sinks, float sm_scale, const fp8pd_tensor* out,
                    DecodeParams* p, DecodeArgs* a) {
  int r;
  if ((r = check(q, FP8PD_DTYPE_BF16, 3))) return r;
  if ((r = check_pool(k_pages, true))) return r;
  if ((r = check_pool(v_pages, true))) return r;
  if (!same_pool_shape(k_pages, v_pages)) return FP8PD_ERR_SHAPE;
  if ((r = check(block_table, FP8PD_DTYPE_I32, 2))) return r;
  if ((r = check(seq_lens, FP8PD_DTYPE_I32, 1))) return r;
  if ((r = check(out, FP8PD_DTYPE_F32, 3))) return r;
  const int64_t B = q->shape[0], Hq = q->shape[1], D = q->shape[2];
  const int64_t P = k_pages->shape[0], ps = k_pages->shape[1], Hkv = k_pages->shape[2];
  if (k_pages->shape[3] != D) return FP8PD_ERR_SHAPE;
  if (block_table->shape[0] != B || seq_lens->shape[0] != B) return FP8PD_ERR_SHAPE;
  if (out->shape[0] != B || out->shape[1] != Hq || out->shape[2] != D) return FP8PD_ERR_SHAPE;
  if (!(D == 64 || D == 128 || D == 256 || D == 512)) return FP8PD_ERR_UNSUPPORTED;
  if (ps < 16 || ps > 256 || ps % 16) return FP8PD_ERR_UNSUPPORTED;
  if (Hkv < 1 || Hq < Hkv || Hq % Hkv) return FP8PD_ERR_UNSUPPORTED;
  if (out->stride[2] != 1 || reinterpret_cast<uintptr_t>(out->data) % 16 || out->stride[0] % 4 ||
      out->stride[1] % 4)
    return FP8PD_ERR_ALIGN;
  if (window < 0) return FP8PD_ERR_ARG;
  if (!(std::isfinite(sm_scale) && sm_scale > 0.f)) return FP8PD_ERR_ARG;
  // Sub-row K groups: each covers whole 16-entry blocks of the QK contraction
  // (D / groups >= 16); V takes one scale per token at most.
  int64_t ks_sp, ks_st, ks_sh, ks_sg, vs_sp, vs_st, vs_sh, vs_sg;
  int k_tok, v_tok, k_groups, v_groups, k_mx, v_mx;
  if ((r = scale_strides(k_scale, P, ps, Hkv, D, static_cast<int>(D / 16), &ks_sp, &ks_st, &ks_sh,
                         &ks_sg, &k_tok, &k_groups, &k_mx)))
    return r;
  if ((r = scale_strides(v_scale, P, ps, Hkv, D, 1, &vs_sp, &vs_st, &vs_sh, &vs_sg, &v_tok,
                         &v_groups, &v_mx)))
    return r;
  if (sinks) {
    if ((r = check(sinks, FP8PD_DTYPE_F32, 1))) return r;
    if (sinks->shape[0] != Hq) return FP8PD_ERR_SHAPE;
  }
  const int64_t max_pages = block_table->shape[1];
  if (!fits_i32(B) || B > 65535 || P > fp8pd::kMaxPages || !fits_i32(max_pages) ||
      max_pages * ps > INT32_MAX || Hkv * ((Hq / Hkv + 7) / 8) > 65535 || !fits_i32(Hq))
    return FP8PD_ERR_TOO_LARGE;

  std::memset(p, 0, sizeof(*p));
  p->q = static_cast<const uint16_t*>(q->data);
  p->q_sb = q->stride[0];
  p->q_sh = q->stride[1];
  p->q_sd = q->stride[2];
  p->k = static_cast<const uint8_t*>(k_pages->data);
  p->v = static_cast<const uint8_t*>(v_pages->data);
  p->k_sp = k_pages->stride[0];
  p->k_st = k_pages->stride[1];
  p->k_sh = k_pages->stride[2];
  p->v_sp = v_pages->stride[0];
  p->v_st = v_pages->stride[1];
  p->v_sh = v_pages->stride[2];
  p->ks = static_cast<const float*>(k_scale->data);
  p->vs = static_cast<const float*>(v_scale->data);
  p->ks_sp = ks_sp;
  p->ks_sh = ks_sh;
  p->vs_sp = vs_sp;
  p->vs_sh = vs_sh;
  p->ks_st = ks_st;
  p->vs_st = vs_st;
  p->k_tok = k_tok;
  p->v_tok = v_tok;
  p->ks_sg = ks_sg;
  p->k_groups = k_groups;
  p->k_mx = k_mx;
  p->v_mx = v_mx;
  p->vs_sg = vs_sg;
  p->table = static_cast<const int32_t*>(block_table->data);
  p->tab_sb = block_table->stride[0];
  p->tab_sp = block_table->stride[1];
  p->lens = static_cast<const int32_t*>(seq_lens->data);
  p->lens_s = seq_lens->stride[0];
  p->sinks = sinks ? static_cast<const float*>(sinks->data) : nullptr;
  p->sinks_s = sinks ? sinks->stride[0] : 0;
  p->out = static_cast<float*>(out->data);
  p->o_sb = out->stride[0];
  p->o_sh = out->stride[1];
  p->B = static_cast<int>(B);
  p->Hq = static_cast<int>(Hq);
  p->Hkv = static_cast<int>(Hkv);
  p->G = static_cast<int>(Hq / Hkv);
  p->D = static_cast<int>(D);
  p->ps = static_cast<int>(ps);
  p->num_pages = static_cast<int>(P);
  p->max_pages = static_cast<int>(max_pages);
  p->window = window;
  p->sm_scale_log2 = sm_scale * 1.4426950408889634f;
  p->q_vec = (q->stride[2] == 1 && q->stride[1] % 4 == 0 && q->stride[0] % 4 == 0 &&
              reinterpret_cast<uintptr_t>(q->data) % 8 == 0)
                 ? 1
                 : 0;
  a->B = p->B;
  a->Hq = p->Hq;
  a->Hkv = p->Hkv;
  a->D = p->D;
  a->ps = p->ps;
  a->num_pages = p->num_pages;
  a->max_pages = p->max_pages;
  return FP8PD_OK;
}

// The split workspace of a device has two areas. The counter area holds
// only ticket counters: every call's merging blocks put the counters they
// used back to zero, so it reads zero between calls whatever the shapes of
// earlier calls. The partial area holds the split partials, whose layout
// changes with the call's shape. Keeping the two apart matters: if the
// counters sat at the start of one shared area, a call with few counters
// would write partials over bytes that a later call with more counters
// reads as tickets, and that later call's merges would misfire.
//
// The capacity T of the partial area fixes the counter area at
// align256(T / 32 + 256) bytes. Every call has at most one ticket per 33
// floats of partials: a split call (S >= 2 splits, D >= 64) has at most
// units * S tickets and units * S * 66 floats; a proportional call
// (nbx >= B blocks per KV head x head group) at most (2B + nbx / 8 + 1) * HX
// <= 3 * nbx * HX tickets and nbx * HX * 8 * 66 floats. So every call
// whose plan fits in T bytes (fp8pd_plan's workspace_bytes) also fits in the
// counter area: fp8pd_reserve_workspace(T) covers it.
size_t counter_area(size_t T) { return align256(T / 32 + 256); }

// Returns the counter and partial areas for a call needing `counters` and
// `partials` bytes, growing the workspace (zero-filled) unless the stream is
// capturing.
int get_workspace(size_t counters, size_t partials, cudaStream_t s, void** ctr, void** part) {
  int dev;
  int r = current_device(&dev);
  if (r) return r;
  std::lock_guard<std::mutex> lock(g_ws_mutex);
  Workspace& w = g_ws[dev];
  if (w.bytes < partials || counter_area(w.bytes) < counters) {
    if (is_capturing(s)) return FP8PD_ERR_CAPTURE_WORKSPACE;
    if (w.ptr) {
      cudaError_t e = cudaFree(w.ptr);  // synchronizes the device first
      w.ptr = nullptr;
      w.bytes = 0;
      if (e != cudaSuccess) return fail_cuda(e);
    }
    size_t T = std::max({partials, static_cast<size_t>(1) << 20, w.bytes});
    while (counter_area(T) < counters) T *= 2;
    const size_t total = counter_area(T) + T;
    cudaError_t e = cudaMalloc(&w.ptr, total);
    if (e != cudaSuccess) {
      cudaGetLastError();
      w.ptr = nullptr;
      return FP8PD_ERR_WORKSPACE;
    }
    e = cudaMemset(w.ptr, 0, total);
    if (e != cudaSuccess) {
      cudaFree(w.ptr);
      w.ptr = nullptr;
      return fail_cuda(e);
    }
    w.bytes = T;
  }
  *ctr = w.ptr;
  *part = static_cast<uint8_t*>(w.ptr) + counter_area(w.bytes);
  return FP8PD_OK;
}

EventPair* timing_slot(int kind) {
  if (!g_timing_on.load()) return nullptr;
  std::lock_guard<std::mutex> lock(g_timing_mutex);
  if (g_timing_used == g_timing_pool.size()) {
    EventPair ep;
    if (cudaEventCreate(&ep.a) != cudaSuccess || cudaEventCreate(&ep.b) != cudaSuccess) {
      cudaGetLastError();
      return nullptr;
    }
    g_timing_pool.push_back(ep);
  }
  EventPair* ep = &g_timing_pool[g_timing_used++];
  ep->kind = kind;
  return ep;
}

}  // namespace

extern "C" {

namespace {

// Kernel parameters that come from the plan, and the workspace layout:
// counters in the counter area; (m, l) partials, numerators, then the group
// (m, l) and numerators in the partial area.
void apply_plan(const Plan& plan, DecodeParams* p) {
  p->num_splits = plan.num_splits;
  p->chunk_pages = plan.chunk_pages;
  p->num_groups = plan.num_groups;
  p->head_groups = plan.head_groups;
  p->prop = plan.schedule == 3 ? 1 : 0;
  p->nbx = plan.nbx;
  p->wait_polls = static_cast<int>(g_opt_wait_polls.load());
  p->test_stall = g_opt_test_stall.load() ? 1 : 0;
}

void lay_out(const Plan& plan, void* ctr, void* part, DecodeParams* p) {
  p->counters = static_cast<int*>(ctr);
  uint8_t* base = static_cast<uint8_t*>(part);
  p->part_ml = reinterpret_cast<float*>(base);
  base += plan.ml_bytes;
  p->part_o = reinterpret_cast<float*>(base);
  base += plan.o_bytes;
  p->grp_ml = reinterpret_cast<float*>(base);
  base += plan.grp_ml_bytes;
  p->grp_o = reinterpret_cast<float*>(base);
}

cudaError_t launch_planned(const Plan& plan, const DecodeParams& p, const CUtensorMap& tmk,
                           const CUtensorMap& tmv, cudaStream_t s) {
  (void)plan;
  const int k_mode = g_opt_compute.load() == 1 ? 3 : static_cast<int>(g_opt_k_decode.load());
  return fp8pd::launch_decode(p, tmk, tmv, k_mode, g_opt_v_decode.load() == 1, s);
}

void record_run(const Plan& plan, int D, bool umma, int dsplit) {
  t_run_info.kernel = umma ? 2 : 1;
  t_run_info.dim_split = umma ? 1 : dsplit;
  t_run_info.schedule = plan.schedule;
  t_run_info.num_splits = plan.num_splits;
  t_run_info.head_groups = plan.head_groups;
  t_run_info.grid_blocks = plan.grid_blocks;
  t_run_info.combine = plan.combine;
  t_run_info.head_dim = D;
  t_run_info.compute = static_cast<int32_t>(g_opt_compute.load());
}

}  // namespace

namespace {

// Plans, sizes the workspace, encodes the tensor maps and launches one
// validated decode-attention call.
int run_decode(DecodeParams& p, const DecodeArgs& a, const fp8pd_tensor* k_pages,
               const fp8pd_tensor* v_pages, int32_t window, fp8pd_stream_t stream) {
  // the fp8 compute path takes page and head scales only: refused, never downgraded
  if (g_opt_compute.load() == 1 && (p.k_tok || p.v_tok)) return FP8PD_ERR_UNSUPPORTED;
  Plan plan;
  const bool um = use_umma(a.D, p.k_tok || p.v_tok, p.k_mx || p.v_mx, p.k_groups);
  int r = make_plan(a.B, a.Hq, a.Hkv, a.D, a.ps, a.max_pages, window, &plan, um);
  if (r) return r;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  apply_plan(plan, &p);
  p.umma = um ? 1 : 0;
  p.dsplit = use_dsplit(a.D, p.k_tok || p.v_tok, p.k_mx || p.v_mx, p.k_groups, p.append != 0, um);
  if (plan.combine) {
    void *ctr = nullptr, *part = nullptr;
    r = get_workspace(plan.counters_bytes, plan.workspace - plan.counters_bytes, s, &ctr, &part);
    if (r) return r;
    lay_out(plan, ctr, part, &p);
  }
  CUtensorMap tmk, tmv;
  if ((r = make_pool_map(k_pages, &tmk, p.dsplit))) return r;
  if ((r = make_pool_map(v_pages, &tmv, p.dsplit))) return r;
  EventPair* ev = timing_slot(0);
  if (ev) cudaEventRecord(ev->a, s);
  cudaError_t e = launch_planned(plan, p, tmk, tmv, s);
  if (e != cudaSuccess) return fail_cuda(e);
  ++g_launches;
  if (ev) cudaEventRecord(ev->b, s);
  ++g_calls;
  record_run(plan, a.D, p.umma != 0, p.dsplit);
  return FP8PD_OK;
}

}  // namespace

int fp8_paged_decode_attention(const fp8pd_tensor* q, const fp8pd_tensor* k_pages,
                               const fp8pd_tensor* v_pages, const fp8pd_tensor* k_scale,
                               const fp8pd_tensor* v_scale, const fp8pd_tensor* block_table,
                               const fp8pd_tensor* seq_lens, int32_t window,
                               const fp8pd_tensor* sinks, float sm_scale, fp8pd_tensor* out,
                               fp8pd_stream_t stream) {
  DecodeParams p;
  DecodeArgs a;
  int r = validate_decode(q, k_pages, v_pages, k_scale, v_scale, block_table, seq_lens, window,
                          sinks, sm_scale, out, &p, &a);
  if (r) return r;
  if (a.B == 0 || a.Hq == 0) return FP8PD_OK;
  return run_decode(p, a, k_pages, v_pages, window, stream);
}

namespace {
bool contiguous(const fp8pd_tensor* t) {
  int64_t st = 1;
  for (int i = t->ndim - 1; i >= 0; --i) {
    if (t->shape[i] > 1 && t->stride[i] != st) return false;
    st *= t->shape[i];
  }
  return true;
}
}  // namespace

int fp8_paged_decode_attention_partial(const fp8pd_tensor* q, const fp8pd_tensor* k_pages,
                                       const fp8pd_tensor* v_pages, const fp8pd_tensor* k_scale,
                                       const fp8pd_tensor* v_scale,
                                       const fp8pd_tensor* block_table,
                                       const fp8pd_tensor* seq_lens,
                                       const fp8pd_tensor* key_ranges, int32_t window,
                                       float sm_scale, fp8pd_tensor* part_o,
                                       fp8pd_tensor* part_ml, fp8pd_stream_t stream) {
  DecodeParams p;
  DecodeArgs a;
  int r = validate_decode(q, k_pages, v_pages, k_scale, v_scale, block_table, seq_lens, window,
                          nullptr, sm_scale, part_o, &p, &a);
  if (r) return r;
  if (!contiguous(part_o)) return FP8PD_ERR_ALIGN;
  if ((r = check(part_ml, FP8PD_DTYPE_F32, 3))) return r;
  if (part_ml->shape[0] != a.B || part_ml->shape[1] != a.Hq || part_ml->shape[2] != 2)
    return FP8PD_ERR_SHAPE;
  if (!contiguous(part_ml) || reinterpret_cast<uintptr_t>(part_ml->data) % 8) return FP8PD_ERR_ALIGN;
  if (key_ranges) {
    if ((r = check(key_ranges, FP8PD_DTYPE_I32, 2))) return r;
    if (key_ranges->shape[0] != a.B || key_ranges->shape[1] != 2) return FP8PD_ERR_SHAPE;
    p.kr = static_cast<const int32_t*>(key_ranges->data);
    p.kr_sb = key_ranges->stride[0];
    p.kr_s1 = key_ranges->stride[1];
  }
  p.pout_o = static_cast<float*>(part_o->data);
  p.pout_ml = static_cast<float*>(part_ml->data);
  if (a.B == 0 || a.Hq == 0) return FP8PD_OK;
  return run_decode(p, a, k_pages, v_pages, window, stream);
}

int fp8pd_combine_partials(const fp8pd_tensor* part_o, const fp8pd_tensor* part_ml,
                           const fp8pd_tensor* sinks, fp8pd_tensor* out, fp8pd_stream_t stream) {
  int r;
  if ((r = check(part_o, FP8PD_DTYPE_F32, 4))) return r;
  if ((r = check(part_ml, FP8PD_DTYPE_F32, 4))) return r;
  if ((r = check(out, FP8PD_DTYPE_F32, 3))) return r;
  const int64_t R = part_o->shape[0], B = part_o->shape[1], Hq = part_o->shape[2],
                D = part_o->shape[3];
  if (part_ml->shape[0] != R || part_ml->shape[1] != B || part_ml->shape[2] != Hq ||
      part_ml->shape[3] != 2)
    return FP8PD_ERR_SHAPE;
  if (out->shape[0] != B || out->shape[1] != Hq || out->shape[2] != D) return FP8PD_ERR_SHAPE;
  if (R < 1 || R > 1024) return FP8PD_ERR_TOO_LARGE;
  if (D % 4) return FP8PD_ERR_UNSUPPORTED;
  if (!contiguous(part_o) || !contiguous(part_ml) ||
      reinterpret_cast<uintptr_t>(part_o->data) % 16 || reinterpret_cast<uintptr_t>(part_ml->data) % 8)
    return FP8PD_ERR_ALIGN;
  if (out->stride[2] != 1 || reinterpret_cast<uintptr_t>(out->data) % 16 || out->stride[0] % 4 ||
      out->stride[1] % 4)
    return FP8PD_ERR_ALIGN;
  if (sinks) {
    if ((r = check(sinks, FP8PD_DTYPE_F32, 1))) return r;
    if (sinks->shape[0] != Hq) return FP8PD_ERR_SHAPE;
  }
  if (!fits_i32(B) || !fits_i32(Hq) || !fits_i32(D) || B * Hq > INT32_MAX) return FP8PD_ERR_TOO_LARGE;
  if (B == 0 || Hq == 0 || D == 0) return FP8PD_OK;
  const cudaError_t e = fp8pd::launch_combine(
      static_cast<const float*>(part_o->data), static_cast<const float*>(part_ml->data),
      static_cast<int>(R), static_cast<int>(B), static_cast<int>(Hq), static_cast<int>(D),
      sinks ? static_cast<const float*>(sinks->data) : nullptr, sinks ? sinks->stride[0] : 0,
      static_cast<float*>(out->data), out->stride[0], out->stride[1],
      reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return fail_cuda(e);
  ++g_launches;
  return FP8PD_OK;
}

int fp8_paged_decode_append_attention(const fp8pd_tensor* q, const fp8pd_tensor* k_new,
                                      const fp8pd_tensor* v_new, fp8pd_tensor* k_pages,
                                      fp8pd_tensor* v_pages, const fp8pd_tensor* k_scale,
                                      const fp8pd_tensor* v_scale, const fp8pd_tensor* block_table,
                                      const fp8pd_tensor* positions, int32_t window,
                                      const fp8pd_tensor* sinks, float sm_scale, fp8pd_tensor* out,
                                      fp8pd_stream_t stream) {
  DecodeParams p;
  DecodeArgs a;
  int r = validate_decode(q, k_pages, v_pages, k_scale, v_scale, block_table, positions, window,
                          sinks, sm_scale, out, &p, &a);
  if (r) return r;
  if ((r = check(k_new, FP8PD_DTYPE_BF16, 3))) return r;
  if ((r = check(v_new, FP8PD_DTYPE_BF16, 3))) return r;
  for (int i = 0; i < 3; ++i)
    if (v_new->shape[i] != k_new->shape[i]) return FP8PD_ERR_SHAPE;
  if (k_new->shape[0] != a.B || k_new->shape[1] != a.Hkv || k_new->shape[2] != a.D)
    return FP8PD_ERR_SHAPE;
  if (a.B == 0 || a.Hq == 0) return FP8PD_OK;
  p.append = 1;
  p.kn = static_cast<const uint16_t*>(k_new->data);
  p.vn = static_cast<const uint16_t*>(v_new->data);
  p.kn_sb = k_new->stride[0];
  p.kn_sh = k_new->stride[1];
  p.kn_sd = k_new->stride[2];
  p.vn_sb = v_new->stride[0];
  p.vn_sh = v_new->stride[1];
  p.vn_sd = v_new->stride[2];
  p.kw = static_cast<uint8_t*>(k_pages->data);
  p.vw = static_cast<uint8_t*>(v_pages->data);
  p.ksw = static_cast<float*>(k_scale->data);
  p.vsw = static_cast<float*>(v_scale->data);
  r = run_decode(p, a, k_pages, v_pages, window, stream);
  if (r == FP8PD_OK) ++g_appends;
  return r;
}

int fp8pd_plan(const fp8pd_tensor* q, const fp8pd_tensor* k_pages, const fp8pd_tensor* block_table,
               int32_t window, fp8pd_plan_info* info) {
  int r;
  if (!info) return FP8PD_ERR_NULL;
  if ((r = check(q, FP8PD_DTYPE_BF16, 3))) return r;
  if ((r = check_pool(k_pages, true))) return r;
  if ((r = check(block_table, FP8PD_DTYPE_I32, 2))) return r;
  const int64_t B = q->shape[0], Hq = q->shape[1], D = q->shape[2];
  const int64_t ps = k_pages->shape[1], Hkv = k_pages->shape[2];
  if (!(D == 64 || D == 128 || D == 256 || D == 512) || k_pages->shape[3] != D)
    return FP8PD_ERR_UNSUPPORTED;
  if (ps < 16 || ps > 256 || ps % 16 || Hkv < 1 || Hq % Hkv) return FP8PD_ERR_UNSUPPORTED;
  if (window < 0) return FP8PD_ERR_ARG;
  if (!fits_i32(B) || !fits_i32(block_table->shape[1])) return FP8PD_ERR_TOO_LARGE;
  Plan plan;
  const bool um = use_umma(static_cast<int>(D), false, false, 1);  // page or head scales
  r = make_plan(static_cast<int>(B), static_cast<int>(Hq), static_cast<int>(Hkv), static_cast<int>(D),
                static_cast<int>(ps), static_cast<int>(block_table->shape[1]), window, &plan, um);
  if (r) return r;
  info->num_splits = plan.num_splits;
  info->head_groups = plan.head_groups;
  info->grid_blocks = plan.grid_blocks;
  info->combine = plan.combine;
  info->workspace_bytes = plan.workspace;
  info->schedule = plan.schedule;
  // the tensor-memory kernel: 8 compute warps and the QK and PV issuing warps
  const int ds = use_dsplit(static_cast<int>(D), false, false, 1, false, um);
  info->warps = plan.grid_blocks * (um ? 10 : fp8pd::decode_warps_per_block(static_cast<int>(D), ds));
  return FP8PD_OK;
}

int fp8_kv_append(const fp8pd_tensor* k_new, const fp8pd_tensor* v_new, fp8pd_tensor* k_pages,
                  fp8pd_tensor* v_pages, const fp8pd_scales* scales,
                  const fp8pd_tensor* block_table, const fp8pd_tensor* positions,
                  fp8pd_stream_t stream) {
  int r;
  if (!scales) return FP8PD_ERR_NULL;
  if ((r = check(k_new, FP8PD_DTYPE_BF16, 3))) return r;
  if ((r = check(v_new, FP8PD_DTYPE_BF16, 3))) return r;
  if ((r = check_pool(k_pages, false))) return r;
  if ((r = check_pool(v_pages, false))) return r;
  if (!same_pool_shape(k_pages, v_pages)) return FP8PD_ERR_SHAPE;
  if ((r = check(block_table, FP8PD_DTYPE_I32, 2))) return r;
  if ((r = check(positions, FP8PD_DTYPE_I32, 1))) return r;
  const int64_t B = k_new->shape[0], Hkv = k_new->shape[1], D = k_new->shape[2];
  const int64_t P = k_pages->shape[0], ps = k_pages->shape[1];
  for (int i = 0; i < 3; ++i)
    if (v_new->shape[i] != k_new->shape[i]) return FP8PD_ERR_SHAPE;
  if (k_pages->shape[2] != Hkv || k_pages->shape[3] != D) return FP8PD_ERR_SHAPE;
  if (block_table->shape[0] != B || positions->shape[0] != B) return FP8PD_ERR_SHAPE;
  if (ps < 1) return FP8PD_ERR_UNSUPPORTED;
  int64_t ks_sp, ks_st, ks_sh, ks_sg, vs_sp, vs_st, vs_sh, vs_sg;
  int k_tok, v_tok, k_groups, v_groups, k_mx, v_mx;
  if ((r = scale_strides(&scales->k_scale, P, ps, Hkv, D, 16, &ks_sp, &ks_st, &ks_sh, &ks_sg,
                         &k_tok, &k_groups, &k_mx)))
    return r;
  if ((r = scale_strides(&scales->v_scale, P, ps, Hkv, D, 1, &vs_sp, &vs_st, &vs_sh, &vs_sg,
                         &v_tok, &v_groups, &v_mx)))
    return r;
  const int64_t max_pages = block_table->shape[1];
  if (!fits_i32(B) || !fits_i32(P) || !fits_i32(Hkv) || !fits_i32(D) || !fits_i32(max_pages) ||
      max_pages * ps > INT32_MAX || B * Hkv * ((D + 1) / 2) > (int64_t(1) << 40))
    return FP8PD_ERR_TOO_LARGE;
  if (B == 0 || Hkv == 0 || D == 0) return FP8PD_OK;
  AppendParams p;
  std::memset(&p, 0, sizeof(p));
  p.kn = static_cast<const uint16_t*>(k_new->data);
  p.vn = static_cast<const uint16_t*>(v_new->data);
  p.kn_sb = k_new->stride[0];
  p.kn_sh = k_new->stride[1];
  p.kn_sd = k_new->stride[2];
  p.vn_sb = v_new->stride[0];
  p.vn_sh = v_new->stride[1];
  p.vn_sd = v_new->stride[2];
  p.k = static_cast<uint8_t*>(k_pages->data);
  p.v = static_cast<uint8_t*>(v_pages->data);
  p.k_sp = k_pages->stride[0];
  p.k_st = k_pages->stride[1];
  p.k_sh = k_pages->stride[2];
  p.v_sp = v_pages->stride[0];
  p.v_st = v_pages->stride[1];
  p.v_sh = v_pages->stride[2];
  p.ks = static_cast<const float*>(scales->k_scale.data);
  p.vs = static_cast<const float*>(scales->v_scale.data);
  p.ks_sp = ks_sp;
  p.ks_sh = ks_sh;
  p.vs_sp = vs_sp;
  p.vs_sh = vs_sh;
  p.ks_st = ks_st;
  p.vs_st = vs_st;
  p.k_tok = k_tok;
  p.v_tok = v_tok;
  p.ks_sg = ks_sg;
  p.k_groups = k_groups;
  p.k_mx = k_mx;
  p.v_mx = v_mx;
  p.vs_sg = vs_sg;
  p.ksw = static_cast<float*>(scales->k_scale.data);
  p.vsw = static_cast<float*>(scales->v_scale.data);
  p.table = static_cast<const int32_t*>(block_table->data);
  p.tab_sb = block_table->stride[0];
  p.tab_sp = block_table->stride[1];
  p.pos = static_cast<const int32_t*>(positions->data);
  p.pos_s = positions->stride[0];
  p.B = static_cast<int>(B);
  p.Hkv = static_cast<int>(Hkv);
  p.D = static_cast<int>(D);
  p.ps = static_cast<int>(ps);
  p.num_pages = static_cast<int>(P);
  p.max_pages = static_cast<int>(max_pages);
  EventPair* ev = timing_slot(1);
  if (ev) cudaEventRecord(ev->a, reinterpret_cast<cudaStream_t>(stream));
  cudaError_t e = fp8pd::launch_append(p, reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return fail_cuda(e);
  if (ev) cudaEventRecord(ev->b, reinterpret_cast<cudaStream_t>(stream));
  ++g_appends;
  ++g_launches;
  return FP8PD_OK;
}

int fp8pd_e4m3_encode(const fp8pd_tensor* x, fp8pd_tensor* codes, fp8pd_stream_t stream) {
  int r;
  if ((r = check(x, FP8PD_DTYPE_F32, 1))) return r;
  if ((r = check(codes, FP8PD_DTYPE_U8, 1))) return r;
  if (codes->shape[0] != x->shape[0]) return FP8PD_ERR_SHAPE;
  if (x->stride[0] < 0 || codes->stride[0] < 0) return FP8PD_ERR_SHAPE;
  const int64_t n = x->shape[0];
  if (n == 0) return FP8PD_OK;
  const cudaError_t e = fp8pd::launch_encode(
      static_cast<const float*>(x->data), x->stride[0], static_cast<uint8_t*>(codes->data),
      codes->stride[0], n, reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return fail_cuda(e);
  ++g_launches;
  return FP8PD_OK;
}

int fp8pd_reserve_workspace(uint64_t bytes) {
  void *ctr = nullptr, *part = nullptr;
  return get_workspace(0, static_cast<size_t>(bytes), nullptr, &ctr, &part);
}

int fp8pd_check_errors(fp8pd_stream_t stream, uint32_t* flags) {
  uint32_t v = 0;
  cudaError_t e = fp8pd::read_and_clear_error_word(&v, reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return fail_cuda(e);
  if (flags) *flags = v;
  return FP8PD_OK;
}

int fp8pd_set_option(int32_t option, int64_t value) {
  switch (option) {
    case FP8PD_OPT_NUM_SPLITS:
      if (value < 0 || value > 65535) return FP8PD_ERR_ARG;
      g_opt_num_splits = value;
      return FP8PD_OK;
    case FP8PD_OPT_SCHEDULE:
      if (value != 0 && value != 1 && value != 3) return FP8PD_ERR_ARG;
      g_opt_schedule = value;
      return FP8PD_OK;
    case FP8PD_OPT_K_DECODE:
      if (value < 0 || value > 2) return FP8PD_ERR_ARG;
      g_opt_k_decode = value;
      return FP8PD_OK;
    case FP8PD_OPT_V_DECODE:
      if (value < 0 || value > 1) return FP8PD_ERR_ARG;
      g_opt_v_decode = value;
      return FP8PD_OK;
    case FP8PD_OPT_WAIT_POLLS:
      if (value < 1 || value > (1 << 20)) return FP8PD_ERR_ARG;
      g_opt_wait_polls = value;
      return FP8PD_OK;
    case FP8PD_OPT_TEST_STALL:
      if (value < 0 || value > 1) return FP8PD_ERR_ARG;
      g_opt_test_stall = value;
      return FP8PD_OK;
    case FP8PD_OPT_COMPUTE:
      if (value < 0 || value > 1) return FP8PD_ERR_ARG;
      g_opt_compute = value;
      return FP8PD_OK;
    case FP8PD_OPT_KERNEL:
      if (value < 0 || value > 2) return FP8PD_ERR_ARG;
      g_opt_kernel = value;
      return FP8PD_OK;
    default:
      return FP8PD_ERR_ARG;
  }
}

int64_t fp8pd_get_option(int32_t option) {
  switch (option) {
    case FP8PD_OPT_NUM_SPLITS: return g_opt_num_splits.load();
    case FP8PD_OPT_SCHEDULE: return g_opt_schedule.load();
    case FP8PD_OPT_K_DECODE: return g_opt_k_decode.load();
    case FP8PD_OPT_V_DECODE: return g_opt_v_decode.load();
    case FP8PD_OPT_WAIT_POLLS: return g_opt_wait_polls.load();
    case FP8PD_OPT_TEST_STALL: return g_opt_test_stall.load();
    case FP8PD_OPT_COMPUTE: return g_opt_compute.load();
    case FP8PD_OPT_KERNEL: return g_opt_kernel.load();
    default: return -1;
  }
}

int fp8pd_last_run_info(fp8pd_run_info* info) {
  if (!info) return FP8PD_ERR_NULL;
  *info = t_run_info;
  info->calls = g_calls.load();
  info->appends = g_appends.load();
  info->kernel_launches = g_launches.load();
  return FP8PD_OK;
}

int fp8pd_timing_enable(int32_t on) {
  g_timing_on = on ? 1 : 0;
  return FP8PD_OK;
}

int fp8pd_timing_collect(double* attention_ms, int32_t* attention_launches, double* append_ms,
                         int32_t* append_launches) {
  std::lock_guard<std::mutex> lock(g_timing_mutex);
  double t[2] = {0.0, 0.0};
  int32_t n[2] = {0, 0};
  for (size_t i = 0; i < g_timing_used; ++i) {
    EventPair& ep = g_timing_pool[i];
    cudaError_t e = cudaEventSynchronize(ep.b);
    if (e != cudaSuccess) return fail_cuda(e);
    float ms = 0.f;
    e = cudaEventElapsedTime(&ms, ep.a, ep.b);
    if (e != cudaSuccess) return fail_cuda(e);
    t[ep.kind] += ms;
    n[ep.kind] += 1;
  }
  g_timing_used = 0;
  if (attention_ms) *attention_ms = t[0];
  if (attention_launches) *attention_launches = n[0];
  if (append_ms) *append_ms = t[1];
  if (append_launches) *append_launches = n[1];
  return FP8PD_OK;
}

const char* fp8pd_status_string(int32_t status) {
  switch (status) {
    case FP8PD_OK: return "ok";
    case FP8PD_ERR_NULL: return "a required descriptor or pointer is NULL";
    case FP8PD_ERR_DTYPE: return "wrong element type";
    case FP8PD_ERR_SHAPE: return "inconsistent or unsupported shape";
    case FP8PD_ERR_ALIGN: return "misaligned pointer or stride (16-byte pool rule, contiguous inner dim)";
    case FP8PD_ERR_UNSUPPORTED: return "unsupported configuration (head dim, page size, head ratio)";
    case FP8PD_ERR_ARG: return "bad scalar argument";
    case FP8PD_ERR_WORKSPACE: return "split workspace allocation failed";
    case FP8PD_ERR_CAPTURE_WORKSPACE: return "split workspace too small during stream capture";
    case FP8PD_ERR_CUDA: return "CUDA runtime error";
    case FP8PD_ERR_TOO_LARGE: return "size exceeds a documented limit";
    default: return "unknown status";
  }
}

int32_t fp8pd_last_cuda_error(void) { return t_last_cuda_error; }

int32_t fp8pd_version(void) { return FP8PD_VERSION; }

}  // extern "C"

// ---------------------------------------------------------------------------
// Decode attention that allocates nothing.
//
// Some callers cannot allocate device memory at the point where they run
// attention: an allocator-free runtime, a custom memory manager that owns all
// of the device's memory, or code that must never call cudaMalloc because it
// would synchronize the device. fp8_paged_decode_attention keeps its split
// scratch in a workspace it allocates on first need; this entry point uses a
// fixed array inside the library's own device image instead, so no call
// allocates. Every GPU that loads the library holds the array until exit.
// ---------------------------------------------------------------------------
namespace {

constexpr size_t kNoAllocScratchBytes = size_t(8) << 20;  // 8 MiB
static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];
std::mutex g_noalloc_mutex;
void* g_noalloc_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device. Host code only
// sees a stand-in for the array's name, so the address is looked up once per
// device, with that device current, and cached.
int noalloc_scratch(void** out) {
  int dev;
  int r = current_device(&dev);
  if (r) return r;
  std::lock_guard<std::mutex> lock(g_noalloc_mutex);
  if (!g_noalloc_ptr[dev]) {
    void* ptr = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&ptr, g_noalloc_scratch);
    if (e != cudaSuccess) return fail_cuda(e);
    g_noalloc_ptr[dev] = ptr;
  }
  *out = g_noalloc_ptr[dev];
  return FP8PD_OK;
}

}  // namespace

extern "C" int fp8_paged_decode_attention_noalloc(
    const fp8pd_tensor* q, const fp8pd_tensor* k_pages, const fp8pd_tensor* v_pages,
    const fp8pd_tensor* k_scale, const fp8pd_tensor* v_scale, const fp8pd_tensor* block_table,
    const fp8pd_tensor* seq_lens, int32_t window, const fp8pd_tensor* sinks, float sm_scale,
    fp8pd_tensor* out, fp8pd_stream_t stream) {
  DecodeParams p;
  DecodeArgs a;
  int r = validate_decode(q, k_pages, v_pages, k_scale, v_scale, block_table, seq_lens, window,
                          sinks, sm_scale, out, &p, &a);
  if (r) return r;
  if (a.B == 0 || a.Hq == 0) return FP8PD_OK;
  if (g_opt_compute.load() == 1 && (p.k_tok || p.v_tok)) return FP8PD_ERR_UNSUPPORTED;
  Plan plan;
  const bool um = use_umma(a.D, p.k_tok || p.v_tok, p.k_mx || p.v_mx, p.k_groups);
  r = make_plan(a.B, a.Hq, a.Hkv, a.D, a.ps, a.max_pages, window, &plan, um);
  if (r) return r;
  if (plan.workspace > kNoAllocScratchBytes) return FP8PD_ERR_TOO_LARGE;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  apply_plan(plan, &p);
  p.umma = um ? 1 : 0;
  p.dsplit = use_dsplit(a.D, p.k_tok || p.v_tok, p.k_mx || p.v_mx, p.k_groups, p.append != 0, um);
  if (plan.combine) {
    void* ws = nullptr;
    r = noalloc_scratch(&ws);
    if (r) return r;
    uint8_t* base = static_cast<uint8_t*>(ws);
    // The ticket counters must read zero when the kernel starts; the array
    // keeps whatever the previous call left, so clear them on the stream.
    cudaError_t e = cudaMemsetAsync(base, 0, plan.counters_bytes, s);
    if (e != cudaSuccess) return fail_cuda(e);
    lay_out(plan, base, base + plan.counters_bytes, &p);
  }
  CUtensorMap tmk, tmv;
  if ((r = make_pool_map(k_pages, &tmk, p.dsplit))) return r;
  if ((r = make_pool_map(v_pages, &tmv, p.dsplit))) return r;
  const cudaError_t e = launch_planned(plan, p, tmk, tmv, s);
  if (e != cudaSuccess) return fail_cuda(e);
  ++g_launches;
  ++g_calls;
  record_run(plan, a.D, p.umma != 0, p.dsplit);
  return FP8PD_OK;
}
