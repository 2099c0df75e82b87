// Kernels of the FP8 (E4M3) paged split-KV decode attention library, sm_100a.
//
// Method (the "FP8 paged attention for MoE serving" solution page, sections
// "Why it happens" and "Expected result"): flash-decode over a paged E4M3
// KV cache with a grid over (sequence, KV head, split), E4M3 decoded in
// registers (exactly, by the hardware cvt or by bit assembly), scales read
// at their natural shape (per KV head, per page, per stored token, K also in
// sub-row groups: "Supported scope"), the query heads of one KV head packed so each K/V
// byte is read once, online softmax with a sliding window and sink logits,
// and a log-sum-exp combine of the splits. With a fused append (the
// "Lecture 8 -- Inference Path" page, "In-kernel KV cache update") the block
// holding a sequence's new position quantizes the new token, stores it and
// attends it.
//
// Design on B200:
// * One thread block = one (sequence b, KV head h, group of <= 8 query
//   heads, split of the key range). Its tile streams (4 warps; at D = 512 6
//   pairs, each warp on half the head dim) take 16-token tiles round robin;
//   each warp copies its tiles with TMA (one cp.async.bulk.tensor per K or V
//   tile, one lane, no multicast) into a private ring on mbarriers (no
//   block-wide barrier in the main loop); a stream keeps its own online-
//   softmax state (at head dim 64, two tiles per softmax step). The streams
//   are merged once at the end; when the keys are split over several blocks the
//   last block of a (sequence, KV head, head group) to finish merges the
//   splits (a ticket counter, never a wait), so one launch does the call.
// * QK and PV are tensor-core contractions (mma.sync m16n8k16, f16 inputs,
//   f32 accumulate): rows = 16 tokens (QK) or 16 head-dim entries (PV),
//   columns = the 8 packed query heads. E4M3 -> f16 is exact, so K and V
//   enter the MMA without rounding; q enters exactly as f16 after a
//   power-of-two rescale; P enters as an f16 hi + lo pair (two MMAs), which
//   keeps it to about 22 significant bits.
// * Operands leave shared memory through ldmatrix (K as stored, V
//   transposed: a pair of E4M3 bytes is one 16-bit matrix element), which
//   with the TMA's 128-byte swizzle reads every 8-row column without bank
//   conflicts and needs one address per lane per 32 columns.

#include <cuda.h>
#include <cuda_fp16.h>
#include <math_constants.h>

#include <atomic>

#include "../../include/fp8pd.h"
#include "fp8pd_internal.h"

namespace fp8pd {

__device__ uint32_t g_error_word;

__device__ __forceinline__ void raise_flag(uint32_t f) { atomicOr(&g_error_word, f); }

cudaError_t read_and_clear_error_word(uint32_t* value, cudaStream_t s) {
  uint32_t v = 0;
  cudaError_t e = cudaMemcpyFromSymbolAsync(&v, g_error_word, sizeof(v), 0,
                                            cudaMemcpyDeviceToHost, s);
  if (e != cudaSuccess) return e;
  e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return e;
  const uint32_t zero = 0;
  e = cudaMemcpyToSymbolAsync(g_error_word, &zero, sizeof(zero), 0, cudaMemcpyHostToDevice, s);
  if (e != cudaSuccess) return e;
  e = cudaStreamSynchronize(s);
  if (value) *value = v;
  return e;
}

// ---------------------------------------------------------------------------
// E4M3 -> f16 by bit assembly.
// An E4M3 byte c = s|eeee|mmm written as (s << 15) | ((c & 0x7F) << 7) is the
// f16 with exponent field eeee and mantissa mmm0000000. f16's exponent bias
// (15) is E4M3's (7) plus 8, so that f16 equals value(c) * 2^-8 exactly, for
// subnormal codes too (f16 subnormal m * 2^-17 = m * 2^-9 * 2^-8). The NaN
// codes 0x7F / 0xFF become +-480 * 2^-8, finite, so a masked garbage byte can
// never poison an accumulator.
// ---------------------------------------------------------------------------

// Bytes 1 and 3 of x -> (lo, hi) halves of an f16x2.
__device__ __forceinline__ uint32_t e4m3x2_b13_to_f16x2(uint32_t x) {
  return ((x >> 1) & 0x3F803F80u) | (x & 0x80008000u);
}
// Bytes 0 and 2 of x -> (lo, hi) halves of an f16x2.
__device__ __forceinline__ uint32_t e4m3x2_b02_to_f16x2(uint32_t x) {
  return e4m3x2_b13_to_f16x2(x << 8);
}

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t r;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(sel));
  return r;
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint32_t lds32(uint32_t a) {
  uint32_t v;
  asm volatile("ld.shared.u32 %0, [%1];\n" : "=r"(v) : "r"(a));
  return v;
}

// D[16x8] += A[16x16] * B[16x8], f16 inputs, f32 accumulate.
__device__ __forceinline__ void mma16816(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};\n"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// D[16x8] += A[16x32] * B[32x8], E4M3 inputs, f32 accumulate. A fragment:
// a0 / a2 = row g, k = 4t .. 4t+3 / 16+4t .. 16+4t+3; a1 / a3 the same for
// row g+8; B fragment: b0 / b1 = column g, k = 4t .. / 16+4t .. (g = lane /
// 4, t = lane % 4, byte i of a register = element k + i).
__device__ __forceinline__ void mma16832_e4m3(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                              uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.f32.e4m3.e4m3.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};\n"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t pack_f16x2(float lo, float hi) {
  const __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&h);
}

__device__ __forceinline__ float bf16_bits_to_float(uint16_t b) {
  return __uint_as_float(static_cast<uint32_t>(b) << 16);
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// Hardware E4M3 -> f16 conversion of bytes (0,1) or (2,3) of a word
// (cvt.rn.f16x2.e4m3x2; exact). Used by the K path when selected.
__device__ __forceinline__ uint32_t e4m3x2_lo16_to_f16x2(uint32_t w) {
  uint32_t r;
  asm("{\n.reg .b16 lo, hi;\nmov.b32 {lo, hi}, %1;\ncvt.rn.f16x2.e4m3x2 %0, lo;\n}\n"
      : "=r"(r) : "r"(w));
  return r;
}
__device__ __forceinline__ uint32_t e4m3x2_hi16_to_f16x2(uint32_t w) {
  uint32_t r;
  asm("{\n.reg .b16 lo, hi;\nmov.b32 {lo, hi}, %1;\ncvt.rn.f16x2.e4m3x2 %0, hi;\n}\n"
      : "=r"(r) : "r"(w));
  return r;
}

// E4M3 codes of two f32 values: round to nearest even, saturating to +-448.
__device__ __forceinline__ uint16_t e4m3x2_rn_sat(float lo, float hi) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return r;  // low byte = lo, high byte = hi
}

// MXFP8 (OCP microscaling): an E8M0 scale code c is 2^(c - 127), exact in
// f32 (c = 0 is the subnormal 2^-127; c = 255 is NaN).
__device__ __forceinline__ float e8m0_to_f32(uint32_t c) {
  if (c == 0u) return __uint_as_float(0x00400000u);
  if (c == 255u) return __uint_as_float(0x7fc00000u);
  return __uint_as_float(c << 23);
}
// The E8M0 code of an MX block whose largest magnitude is m (NaN entries
// already skipped): floor(log2 m) - 8 + 127, so that m / scale lies in
// [2^8, 2^9), clamped to [0, 254]; an all-zero block takes 127 (scale 1).
__device__ __forceinline__ uint32_t mx_code(float m) {
  if (!(m > 0.f)) return 127u;
  if (isinf(m)) return 254u;
  int e;
  frexpf(m, &e);  // m in [2^(e-1), 2^e)
  return static_cast<uint32_t>(min(254, max(0, e - 1 - 8 + 127)));
}

__device__ __forceinline__ float4 ldcg4(const float* p) {
  float4 v;
  asm volatile("ld.global.cg.v4.f32 {%0,%1,%2,%3}, [%4];\n"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
               : "l"(p));
  return v;
}
__device__ __forceinline__ float2 ldcg2(const float* p) {
  float2 v;
  asm volatile("ld.global.cg.v2.f32 {%0,%1}, [%2];\n" : "=f"(v.x), "=f"(v.y) : "l"(p));
  return v;
}

// ---------------------------------------------------------------------------
// Asynchronous tile copies (TMA) and their mbarriers.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;\n" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;\n" ::"r"(bar), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];\n" ::"r"(bar) : "memory");
}
// Waits for phase `parity` of the barrier. Each poll lets the warp sleep in
// the barrier for up to 20 us (the suspend-time hint) instead of spinning;
// after `polls` polls (by default 2^17, about 2.6 s) it gives up and returns
// false, so a lost copy can never hang the GPU.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, int polls) {
#pragma unroll 1
  for (int it = 0; it < polls; ++it) {
    uint32_t ok;
    asm volatile(
        "{\n.reg .pred p;\nmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, 20000;\n"
        "selp.u32 %0, 1, 0, p;\n}\n"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    if (ok) return true;
  }
  return false;
}
__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
}
__device__ __forceinline__ void fence_proxy_async() {
  asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");
}
// 5-D tiled TMA load (no multicast) into this block's shared memory. With
// FP8PD_EVICT_FIRST (a build setting) the load carries an L2 evict-first
// policy: K/V bytes are read once per step.
__device__ __forceinline__ void tma_load_5d(uint32_t dst, const CUtensorMap* map, uint32_t bar, int c0,
                                            int c1, int c2, int c3, int c4) {
#ifdef FP8PD_EVICT_FIRST
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
  asm volatile(
      "cp.async.bulk.tensor.5d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint "
      "[%0], [%1, {%2, %3, %4, %5, %6}], [%7], %8;\n" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(c4), "r"(bar),
      "l"(pol)
      : "memory");
#else
  asm volatile(
      "cp.async.bulk.tensor.5d.shared::cluster.global.tile.mbarrier::complete_tx::bytes "
      "[%0], [%1, {%2, %3, %4, %5, %6}], [%7];\n" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(c4), "r"(bar)
      : "memory");
#endif
}
// 4-byte asynchronous copy global -> shared (no register round trip); the
// issuing thread waits for all of its copies with cp_async_wait_all.
__device__ __forceinline__ void cp_async4(void* smem_dst, const void* gmem_src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;\n" ::"r"(smem_u32(smem_dst)),
               "l"(gmem_src)
               : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() {
  asm volatile("cp.async.wait_all;\n" ::: "memory");
}
__device__ __forceinline__ void prefetch_tensormap(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];\n" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// Four 8x8 matrices of 16-bit elements (here: pairs of E4M3 bytes); lane l
// supplies the address of row l % 8 of matrix l / 8.
__device__ __forceinline__ uint4 ldsm_x4(uint32_t addr) {
  uint4 r;
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "r"(addr));
  return r;
}
__device__ __forceinline__ uint4 ldsm_x4_trans(uint32_t addr) {
  uint4 r;
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "r"(addr));
  return r;
}

__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Transposes an 8x8 matrix of 16-bit elements held one row pair per lane
// (lane = 4 * row + col / 2), the layout of an MMA accumulator fragment.
__device__ __forceinline__ uint32_t movmatrix_trans(uint32_t a) {
  uint32_t d;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;\n" : "=r"(d) : "r"(a));
  return d;
}

__device__ __forceinline__ float2 unpack_f16x2(uint32_t h) {
  return __half22float2(*reinterpret_cast<const __half2*>(&h));
}


// Pipeline depth (ring stages per warp) and blocks per SM the register budget
// targets; compile-time settings, overridable for tuning builds.
#ifndef FP8PD_NS_D64
#define FP8PD_NS_D64 4
#endif
#ifndef FP8PD_NS_D128
#define FP8PD_NS_D128 3
#endif
#ifndef FP8PD_PAIR_D64
#define FP8PD_PAIR_D64 1
#endif
#ifndef FP8PD_NS_D256
#define FP8PD_NS_D256 3
#endif
#ifndef FP8PD_NS_D512
#define FP8PD_NS_D512 3
#endif
#ifndef FP8PD_MIN_BLOCKS_D64
#define FP8PD_MIN_BLOCKS_D64 5
#endif
#ifndef FP8PD_MIN_BLOCKS_D128
#define FP8PD_MIN_BLOCKS_D128 4
#endif
#ifndef FP8PD_MIN_BLOCKS_D256
#define FP8PD_MIN_BLOCKS_D256 2
#endif
// Warps per block (each streams its own tiles through its own ring).
#ifndef FP8PD_NW_D64
#define FP8PD_NW_D64 4
#endif
#ifndef FP8PD_NW_D128
#define FP8PD_NW_D128 4
#endif
#ifndef FP8PD_NW_D256
#define FP8PD_NW_D256 4
#endif
#ifndef FP8PD_NW_D512
#define FP8PD_NW_D512 4
#endif
// Tile streams and ring stages of the D = 512 head-dim split (its warps are
// streams x split; the rings hold the same 192 KiB as the whole-width shape).
#ifndef FP8PD_NW_D512_SPLIT
#define FP8PD_NW_D512_SPLIT 6
#endif
#ifndef FP8PD_NS_D512_SPLIT
#define FP8PD_NS_D512_SPLIT 2
#endif

// ---------------------------------------------------------------------------
// Shared-memory tile layout. The TMA writes one 16-token tile of one KV head
// as [D/128 column blocks][16 rows][128 bytes] (D >= 128, 128-byte swizzle:
// 16-byte chunk c of row r sits at chunk c ^ (r % 8)) or [16 rows][64 bytes]
// (D = 64, 64-byte swizzle: chunk c of row r at c ^ ((r / 2) % 4)). Every
// ldmatrix then reads 8 rows of one 16-byte column with no bank conflict.
// tile_off(r, b) = byte offset of row r, byte column b (b a multiple of 16).
// ---------------------------------------------------------------------------
template <int D>
__device__ __forceinline__ uint32_t tile_off(int r, int b) {
  if constexpr (D == 64) {
    return r * 64 + ((((b >> 4) ^ ((r >> 1) & 3))) << 4);
  } else {
    return (b >> 7) * 2048 + r * 128 + (((((b & 127) >> 4) ^ (r & 7))) << 4);
  }
}

// DS (head-dim split): each tile stream of a block is shared by DS warps,
// warp h of the stream copying and contracting head-dim entries
// [h * D / DS, (h + 1) * D / DS) of every tile (its own ring of part-width
// tiles), the partial scores summed through shared memory once per tile.
// DS = 2 and 4 are built for D = 512 only, where a block of four whole-width
// streams fills the SM's shared memory with four warps.
template <int D, int DS = 1>
struct Cfg {
  static_assert(DS == 1 || (D == 512 && (DS == 2 || DS == 4)),
                "head-dim split: D = 512, two or four warps per stream");
  static constexpr int DW = D / DS;                                    // head-dim entries per warp
  static constexpr int NLW = (D == 64) ? FP8PD_NW_D64 : (D == 128) ? FP8PD_NW_D128 : (D == 256) ? FP8PD_NW_D256 : (DS > 1) ? FP8PD_NW_D512_SPLIT : FP8PD_NW_D512;  // tile streams per block
  static constexpr int NW = NLW * DS;                                  // warps per block
  static constexpr int NT = NW * 32;                                  // threads per block
  static constexpr int NS = (D == 64) ? FP8PD_NS_D64 : (D == 128) ? FP8PD_NS_D128 : (D == 256) ? FP8PD_NS_D256 : (DS > 1) ? FP8PD_NS_D512_SPLIT : FP8PD_NS_D512;  // ring stages per warp
  static constexpr bool PAIR = (D == 64) && FP8PD_PAIR_D64;           // two tiles per softmax step
  static constexpr int TILE = kTileTokens * DW;                       // bytes of a warp's K or V tile
  static constexpr int STAGE = 2 * TILE;
  static constexpr int WARP_BYTES = NS * STAGE;
  static constexpr int PIPE_BYTES = NW * WARP_BYTES;                  // multiple of 1024
  static constexpr bool Q_IN_SMEM = (D > 256);                        // q fragments in smem
  static constexpr int QFRAG_BYTES = Q_IN_SMEM ? (D / 16) * 32 * 8 : 0;
  // per stream, two buffers of the DS warps' score parts (float4 per lane) and their flags
  static constexpr int XCH_BYTES = DS > 1 ? NLW * 2 * DS * (32 * 16 + 16) : 0;
  static constexpr int LIST_BYTES = NLW * kMaxWarpTiles * 12;         // tile entry, k / v scale
  static constexpr int BAR_BYTES = NW * NS * 8;
  static constexpr int MISC_FLOATS = NW * 8 * 2 + 4;
  static constexpr int SMEM = 1024 /* alignment slack */ + PIPE_BYTES + QFRAG_BYTES + XCH_BYTES +
                              LIST_BYTES + BAR_BYTES + MISC_FLOATS * 4;
  static constexpr int MIN_BLOCKS = (D == 512) ? 1 : (D == 256) ? FP8PD_MIN_BLOCKS_D256 : (D == 128) ? FP8PD_MIN_BLOCKS_D128 : FP8PD_MIN_BLOCKS_D64;
  static_assert(PIPE_BYTES % 1024 == 0, "tiles must stay 1024-byte aligned for the swizzle");
  static_assert(DW % 128 == 0 || DS == 1, "a warp's part of a row is whole 128-byte blocks");
  static_assert(NLW * 8 * D * 4 <= PIPE_BYTES, "merge scratch must fit in the ring");
  static_assert(NLW * kMaxWarpTiles >= kMaxSplitTiles, "a split's tiles fit the streams' lists");
  static_assert(8 * 32 * 4 <= PIPE_BYTES, "merge weights must fit in the ring");
  static_assert(SMEM <= 232448, "shared memory per block");
};

// Merges K partial rows (max m, sum l, numerator O, all in log2 units) of one
// (sequence, head group): for head n they are rows row0 + n * head_rows + s,
// s < K, of (ml, o). With `final`, the sink enters the denominator once and
// numerator / denominator goes to `out`; otherwise the merged (m, l, O) goes to
// row dst_row0 + n * dst_head_rows of (dst_ml, dst_o). Called by the whole block.
template <int D, int NW>
__device__ void merge_partials(const float* ml, const float* o, int64_t row0, int64_t head_rows,
                               int K, int nheads, bool final, const DecodeParams& p, int b,
                               int head0, float* dst_ml, float* dst_o, int64_t dst_row0,
                               int64_t dst_head_rows, float* wts) {
  constexpr float kLog2e = 1.4426950408889634f;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  for (int n = warp; n < nheads; n += NW) {
    const int head = head0 + n;
    const float* pml = ml + (row0 + n * head_rows) * 2;
    const float2 me = lane < K ? ldcg2(pml + 2 * lane) : make_float2(-CUDART_INF_F, 0.f);
    const float M = warp_max(me.x);
    const float sl = (final && p.sinks) ? p.sinks[(int64_t)head * p.sinks_s] * kLog2e : -CUDART_INF_F;
    const float M2 = fmaxf(M, sl);
    const float w = (M2 == -CUDART_INF_F || me.x == -CUDART_INF_F) ? 0.f : fast_exp2(me.x - M2);
    float l = w * me.y;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) l += __shfl_xor_sync(0xffffffffu, l, off);
    if (final) {
      const float den = l + ((p.sinks && M2 != -CUDART_INF_F) ? fast_exp2(sl - M2) : 0.f);
      const float inv = den > 0.f ? 1.f / den : 0.f;
      if (lane < K) wts[n * 32 + lane] = w * inv;
    } else {
      if (lane < K) wts[n * 32 + lane] = w;
      if (lane == 0)
        *reinterpret_cast<float2*>(dst_ml + (dst_row0 + n * dst_head_rows) * 2) = make_float2(M, l);
    }
  }
  __syncthreads();
  // two output entries per thread and pass, so that both entries' loads of
  // a group of partials are in flight together
  const int items = nheads * (D / 4);
  for (int it0 = tid; it0 < items; it0 += 2 * NW * 32) {
    int n[2], d[2];
    const float* po[2];
    const float* wn[2];
    bool ok[2];
    float4 acc[2];
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int it = it0 + u * NW * 32;
      ok[u] = it < items;
      const int itc = ok[u] ? it : it0;
      n[u] = itc / (D / 4);
      d[u] = (itc - n[u] * (D / 4)) * 4;
      po[u] = o + (row0 + n[u] * head_rows) * D + d[u];
      wn[u] = wts + n[u] * 32;
      acc[u] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll 8
    for (int s = 0; s < K; ++s) {
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const float ws = wn[u][s];
        const float4 v = ldcg4(po[u] + (int64_t)s * D);
        acc[u].x += ws * v.x;
        acc[u].y += ws * v.y;
        acc[u].z += ws * v.z;
        acc[u].w += ws * v.w;
      }
    }
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      if (!ok[u]) continue;
      if (final)
        *reinterpret_cast<float4*>(p.out + (int64_t)b * p.o_sb + (int64_t)(head0 + n[u]) * p.o_sh +
                                   d[u]) = acc[u];
      else
        *reinterpret_cast<float4*>(dst_o + (dst_row0 + n[u] * dst_head_rows) * D + d[u]) = acc[u];
    }
  }
}

// Byte offset inside a tile of 32-byte block kc for one lane's ldmatrix
// row: blocks 4.. of a 128-byte line group repeat the offsets of blocks 0..3
// one 2048-byte column block further (D >= 128).
template <int D>
__device__ __forceinline__ uint32_t blk_off(const uint32_t (&off)[4], int kc) {
  if constexpr (D == 64) return off[kc];
  else return off[kc & 3] + (kc >> 2) * 2048;
}

// Per-lane ldmatrix row offsets inside a tile. K (no transpose): matrix
// i = lane / 8 is rows (lane % 8) + 8 * (i % 2) at byte column 16 * (i / 2)
// of each 32-byte block; V (transposed): rows (lane % 8) + 8 * (i / 2) at
// byte column 16 * (i % 2). The swizzle makes the offset of 32-byte block kc
// depend on kc % 4 (D >= 128) or kc (D = 64), so four offsets per operand.
template <int D>
__device__ __forceinline__ void ldsm_offsets(int lane, uint32_t (&koff)[4], uint32_t (&voff)[4]) {
  const int i = lane >> 3;
  const int rk = (lane & 7) + 8 * (i & 1), hk = i >> 1;
  const int rv = (lane & 7) + 8 * (i >> 1), hv = i & 1;
#pragma unroll
  for (int kc = 0; kc < 4; ++kc) {
    koff[kc] = tile_off<D>(rk, 32 * kc + 16 * hk);
    voff[kc] = tile_off<D>(rv, 32 * kc + 16 * hv);
  }
}

// One warp's online-softmax state for up to 8 query heads: O^T[d][head] as
// PV accumulator fragments (sum of P * v_scale / vref), the running maxima
// (log2 units) and this lane's share of the running sums of heads 2q and
// 2q+1, and the running V reference scale vref (the largest |v_scale| seen).
template <int D>
struct Acc {
  float O[D / 32][2][4];
  float m0, m1, l0, l1, vref, inv_vref;
  float x0, x1;  // lazy maxima: this lane's largest scores of heads 2qd / 2qd+1 so far
  __device__ __forceinline__ void reset() {
#pragma unroll
    for (int jb = 0; jb < D / 32; ++jb)
#pragma unroll
      for (int h = 0; h < 2; ++h)
#pragma unroll
        for (int c = 0; c < 4; ++c) O[jb][h][c] = 0.f;
    m0 = m1 = x0 = x1 = -CUDART_INF_F;
    l0 = l1 = 0.f;
    vref = inv_vref = 0.f;
  }
};

// S = K q'^T of one 16-token tile in shared memory (K at sk, the swizzled
// layout of tile_off) on the tensor cores, then the masked scores in log2
// units of this lane: tokens grp / grp + 8 of the tile, heads 2qd / 2qd+1,
// returned as (x, y, z, w) = (grp, 2qd), (grp, 2qd+1), (grp+8, 2qd),
// (grp+8, 2qd+1). Tokens outside [t0, t1), or the whole tile when its page
// is out of range, are -inf. kfa / kfb = score factors of tokens grp /
// grp + 8 (equal unless the scales are per token); `full`:
// every token is attended (warp-uniform). qfr(kb) gives the q' B-fragment
// of k16 block kb. KM selects the contraction: 0 / 1 = E4M3 decoded to f16 by
// bit assembly / the hardware cvt, then f16 MMAs (m16n8k16); 2 = the E4M3
// bytes themselves in E4M3 MMAs (m16n8k32), q' as two E4M3 terms (qfr(kb) =
// (hi, lo) of the k16 block's four entries per lane), no conversion of K.
template <int D, int KM, class QFrag>
__device__ __forceinline__ float4 tile_scores(const QFrag& qfr, uint32_t sk,
                                              const uint32_t (&koff)[4], float kfa, float kfb,
                                              int tok0, int t0, int t1, bool page_ok, bool full,
                                              int grp, float2 hf = make_float2(1.f, 1.f)) {
  // two independent accumulator chains
  float Sa[4] = {0.f, 0.f, 0.f, 0.f}, Sb[4] = {0.f, 0.f, 0.f, 0.f};
  if constexpr (KM == 3) {
    // fp8 compute: q' as one E4M3 term (qfr(kb).x), per-head factors hf of
    // this lane's heads 2qd / 2qd + 1; the two k32 blocks' chains alternate
#pragma unroll
    for (int kc = 0; kc < D / 32; ++kc) {
      const uint4 kw = ldsm_x4(sk + blk_off<D>(koff, kc));
      const uint2 f0 = qfr(2 * kc), f1 = qfr(2 * kc + 1);
      if (kc & 1) mma16832_e4m3(Sb, kw.x, kw.y, kw.z, kw.w, f0.x, f1.x);
      else mma16832_e4m3(Sa, kw.x, kw.y, kw.z, kw.w, f0.x, f1.x);
    }
  } else if constexpr (KM == 2) {
    // the ldmatrix of a 32-byte block is the MMA's A fragment as is: rows g /
    // g+8, bytes 4t.. (x / y) and 16+4t.. (z / w)
#pragma unroll
    for (int kc = 0; kc < D / 32; ++kc) {
      const uint4 kw = ldsm_x4(sk + blk_off<D>(koff, kc));
      const uint2 f0 = qfr(2 * kc), f1 = qfr(2 * kc + 1);
      mma16832_e4m3(Sa, kw.x, kw.y, kw.z, kw.w, f0.x, f1.x);
      mma16832_e4m3(Sb, kw.x, kw.y, kw.z, kw.w, f0.y, f1.y);
    }
  } else {
#pragma unroll
  for (int kc = 0; kc < D / 32; ++kc) {
    // rows g / g+8, bytes 32kc + 4q.. (regs 0 / 1) and 32kc + 16 + 4q.. (2 / 3)
    const uint4 kw = ldsm_x4(sk + blk_off<D>(koff, kc));
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      const int kb = 2 * kc + half;
      const uint32_t wa = half ? kw.z : kw.x, wb = half ? kw.w : kw.y;
      uint32_t b0, b1;
      {
        const uint2 f = qfr(kb);
        b0 = f.x;
        b1 = f.y;
      }
      uint32_t a0, a1, a2, a3;
      if constexpr (KM == 1) {
        a0 = e4m3x2_lo16_to_f16x2(wa);
        a1 = e4m3x2_lo16_to_f16x2(wb);
        a2 = e4m3x2_hi16_to_f16x2(wa);
        a3 = e4m3x2_hi16_to_f16x2(wb);
      } else {
        a0 = e4m3x2_b02_to_f16x2(wa);
        a1 = e4m3x2_b02_to_f16x2(wb);
        a2 = e4m3x2_b13_to_f16x2(wa);
        a3 = e4m3x2_b13_to_f16x2(wb);
      }
      if (half)
        mma16816(Sb, a0, a1, a2, a3, b0, b1);
      else
        mma16816(Sa, a0, a1, a2, a3, b0, b1);
    }
  }
  }
  // A masked row may hold stale or NaN-decoded bytes: select, never multiply.
  const int ta = tok0 + grp, tb = ta + 8;
  const bool va = full || (page_ok && ta >= t0 && ta < t1);
  const bool vb = full || (page_ok && tb >= t0 && tb < t1);
  if constexpr (KM == 3) {
    return make_float4(va ? (Sa[0] + Sb[0]) * (kfa * hf.x) : -CUDART_INF_F,
                       va ? (Sa[1] + Sb[1]) * (kfa * hf.y) : -CUDART_INF_F,
                       vb ? (Sa[2] + Sb[2]) * (kfb * hf.x) : -CUDART_INF_F,
                       vb ? (Sa[3] + Sb[3]) * (kfb * hf.y) : -CUDART_INF_F);
  }
  return make_float4(va ? (Sa[0] + Sb[0]) * kfa : -CUDART_INF_F,
                     va ? (Sa[1] + Sb[1]) * kfa : -CUDART_INF_F,
                     vb ? (Sa[2] + Sb[2]) * kfb : -CUDART_INF_F,
                     vb ? (Sa[3] + Sb[3]) * kfb : -CUDART_INF_F);
}

// tile_scores with sub-row K group scales: the MMAs of each run of D / G
// head-dim entries (2^bpg_log2 k16 blocks) accumulate on their own, then
// are scaled by the group's K scale of this lane's token rows grp / grp + 8
// (ga[g] / gb[g], shared memory) and summed. kf = the score factor without
// the K scale. Masking as tile_scores.
template <int D, int KM, class QFrag>
__device__ __forceinline__ float4 tile_scores_groups(const QFrag& qfr, uint32_t sk,
                                                     const uint32_t (&koff)[4], const float* ga,
                                                     const float* gb, int bpg_log2, float kf,
                                                     int tok0, int t0, int t1, bool page_ok,
                                                     bool full, int grp) {
  float S[4] = {0.f, 0.f, 0.f, 0.f}, Sg[4] = {0.f, 0.f, 0.f, 0.f};
  const int bpg_mask = (1 << bpg_log2) - 1;
#pragma unroll
  for (int kc = 0; kc < D / 32; ++kc) {
    const uint4 kw = ldsm_x4(sk + blk_off<D>(koff, kc));
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      const int kb = 2 * kc + half;
      const uint32_t wa = half ? kw.z : kw.x, wb = half ? kw.w : kw.y;
      const uint2 f = qfr(kb);
      uint32_t a0, a1, a2, a3;
      static_assert(KM != 2, "sub-row K groups use a 16-bit decode of K");
      if constexpr (KM == 1) {
        a0 = e4m3x2_lo16_to_f16x2(wa);
        a1 = e4m3x2_lo16_to_f16x2(wb);
        a2 = e4m3x2_hi16_to_f16x2(wa);
        a3 = e4m3x2_hi16_to_f16x2(wb);
      } else {
        a0 = e4m3x2_b02_to_f16x2(wa);
        a1 = e4m3x2_b02_to_f16x2(wb);
        a2 = e4m3x2_b13_to_f16x2(wa);
        a3 = e4m3x2_b13_to_f16x2(wb);
      }
      mma16816(Sg, a0, a1, a2, a3, f.x, f.y);
      if ((kb & bpg_mask) == bpg_mask) {  // the group's last k16 block
        const int g = kb >> bpg_log2;
        const float sa = ga[g], sb = gb[g];
        S[0] = fmaf(Sg[0], sa, S[0]);
        S[1] = fmaf(Sg[1], sa, S[1]);
        S[2] = fmaf(Sg[2], sb, S[2]);
        S[3] = fmaf(Sg[3], sb, S[3]);
        Sg[0] = Sg[1] = Sg[2] = Sg[3] = 0.f;
      }
    }
  }
  const int ta = tok0 + grp, tb = ta + 8;
  const bool va = full || (page_ok && ta >= t0 && ta < t1);
  const bool vb = full || (page_ok && tb >= t0 && tb < t1);
  return make_float4(va ? S[0] * kf : -CUDART_INF_F, va ? S[1] * kf : -CUDART_INF_F,
                     vb ? S[2] * kf : -CUDART_INF_F, vb ? S[3] * kf : -CUDART_INF_F);
}

// Online-softmax update for new scores whose per-head maxima over this
// lane's tokens are (tm0, tm1) and whose largest |V scale| is vabs: the
// running maxima and the V reference scale grow, and l and O are rescaled,
// only when one of them changes (warp-uniform test).
// LAZY: the reference maxima m0 / m1 move only when some score exceeds them
// by more than kLazyLog2 (or the V scale grows), so most tiles skip the
// cross-lane maximum; P = 2^(s - m) then stays below 2^kLazyLog2, which the
// f16 hi + lo operands hold exactly as before. Each lane keeps its own true
// maxima (x0 / x1); lazy_finish moves l and O onto them once at the end.
constexpr float kLazyLog2 = 8.f;

template <int D, bool LAZY = false>
__device__ __forceinline__ void softmax_rescale(Acc<D>& a, float tm0, float tm1, float vabs) {
  if constexpr (LAZY) {
    a.x0 = fmaxf(a.x0, tm0);
    a.x1 = fmaxf(a.x1, tm1);
    if (!(vabs > a.vref) &&
        !__any_sync(0xffffffffu, (tm0 > a.m0 + kLazyLog2) || (tm1 > a.m1 + kLazyLog2)))
      return;
  }
#pragma unroll
  for (int o = 4; o < 32; o <<= 1) {
    tm0 = fmaxf(tm0, __shfl_xor_sync(0xffffffffu, tm0, o));
    tm1 = fmaxf(tm1, __shfl_xor_sync(0xffffffffu, tm1, o));
  }
  const float mn0 = fmaxf(a.m0, tm0), mn1 = fmaxf(a.m1, tm1);
  const bool grow_v = vabs > a.vref;  // warp-uniform
  if (grow_v || __any_sync(0xffffffffu, (mn0 > a.m0) || (mn1 > a.m1))) {
    const float c0 = (mn0 > a.m0) ? fast_exp2(a.m0 - mn0) : 1.f;  // exp2(-inf) = 0 for a first max
    const float c1 = (mn1 > a.m1) ? fast_exp2(a.m1 - mn1) : 1.f;
    const float fv = grow_v ? a.vref / vabs : 1.f;
    a.l0 *= c0;
    a.l1 *= c1;
    const float o0 = c0 * fv, o1 = c1 * fv;
#pragma unroll
    for (int jb = 0; jb < D / 32; ++jb)
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        a.O[jb][h][0] *= o0;
        a.O[jb][h][1] *= o1;
        a.O[jb][h][2] *= o0;
        a.O[jb][h][3] *= o1;
      }
    a.m0 = mn0;
    a.m1 = mn1;
    if (grow_v) {
      a.vref = vabs;
      a.inv_vref = 1.f / vabs;
    }
  }
}

// End of a lazy stream: the exact per-head maxima of this warp's scores
// (reduced over the 8 lanes of a head pair) replace the reference maxima, l
// and O scaled to match, so a partial's m is the maximum score as documented.
template <int D>
__device__ __forceinline__ void lazy_finish(Acc<D>& a) {
  float x0 = a.x0, x1 = a.x1;
#pragma unroll
  for (int o = 4; o < 32; o <<= 1) {
    x0 = fmaxf(x0, __shfl_xor_sync(0xffffffffu, x0, o));
    x1 = fmaxf(x1, __shfl_xor_sync(0xffffffffu, x1, o));
  }
  const float c0 = (x0 > a.m0) ? fast_exp2(a.m0 - x0) : 1.f;
  const float c1 = (x1 > a.m1) ? fast_exp2(a.m1 - x1) : 1.f;
  a.l0 *= c0;
  a.l1 *= c1;
#pragma unroll
  for (int jb = 0; jb < D / 32; ++jb)
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      a.O[jb][h][0] *= c0;
      a.O[jb][h][1] *= c1;
      a.O[jb][h][2] *= c0;
      a.O[jb][h][3] *= c1;
    }
  a.m0 = fmaxf(a.m0, x0);
  a.m1 = fmaxf(a.m1, x1);
}

// P of one tile: exp2 of the scores against the running maxima, added to
// the running sums; then P * v_scale / vref as an f16 hi + lo pair, whose PV
// B fragments are the transposes of the score fragment's 8x8 blocks
// (movmatrix): bh / bl[0] for tokens 2qd.., bh / bl[1] for 2qd+8...
// vsa / vsb: V scales of tokens grp / grp + 8.
template <int D>
__device__ __forceinline__ void tile_probs(Acc<D>& a, float4 sc, float vsa, float vsb,
                                           uint32_t (&bh)[2], uint32_t (&bl)[2]) {
  const float mb0 = (a.m0 == -CUDART_INF_F) ? 0.f : a.m0;
  const float mb1 = (a.m1 == -CUDART_INF_F) ? 0.f : a.m1;
  const float p00 = fast_exp2(sc.x - mb0), p01 = fast_exp2(sc.y - mb1);
  const float p10 = fast_exp2(sc.z - mb0), p11 = fast_exp2(sc.w - mb1);
  a.l0 += p00 + p10;
  a.l1 += p01 + p11;
  const float vra = vsa * a.inv_vref, vrb = vsb * a.inv_vref;
  const float w00 = p00 * vra, w01 = p01 * vra, w10 = p10 * vrb, w11 = p11 * vrb;
  const uint32_t ha = pack_f16x2(w00, w01), hb = pack_f16x2(w10, w11);
  const float2 fa = unpack_f16x2(ha), fb = unpack_f16x2(hb);
  const uint32_t la = pack_f16x2(w00 - fa.x, w01 - fa.y), lb = pack_f16x2(w10 - fb.x, w11 - fb.y);
  bh[0] = movmatrix_trans(ha);
  bh[1] = movmatrix_trans(hb);
  bl[0] = movmatrix_trans(la);
  bl[1] = movmatrix_trans(lb);
}

// O^T[d][head] += V^T P of one tile (V at sv). ldmatrix.trans of the
// 32-byte block jb gives lane (g, q) the bytes (d, d+1), d = 32jb + 2g, of
// tokens 2q and 2q+1 (reg 0), the same for d + 16 (reg 1), and for tokens
// 2q+8, 2q+9 (regs 2, 3). M tile (jb, 0) rows g / g+8 are d / d+1; M tile
// (jb, 1) adds 16.
// f16 bits of 2^d for an MX block exponent difference d <= 0 (subnormal from
// -15 down to -24, 0 below).
__device__ __forceinline__ uint32_t f16_pow2(int d) {
  if (d >= -14) return static_cast<uint32_t>(d + 15) << 10;
  if (d >= -24) return 1u << (d + 24);
  return 0u;
}

// With vmx (MXFP8 V): vmw = this lane's words of its token's E8M0 codes
// (lanes 16 + r: token r of the tile, byte g = block g), E = the tile's
// largest code: each decoded V pair of tokens (2qd, 2qd+1) and (2qd+8,
// 2qd+9) in 32-entry block jb is multiplied by 2^(code - E), exactly (the
// tile's 2^(E - 127) goes through P as its V scale).
template <int D, bool VCVT>
__device__ __forceinline__ void tile_pv(Acc<D>& a, uint32_t sv, const uint32_t (&voff)[4],
                                        const uint32_t (&bh)[2], const uint32_t (&bl)[2], int tok0,
                                        int t0, int t1, bool page_ok, bool full, int qd,
                                        bool vmx = false, const uint32_t* vmw = nullptr,
                                        int E = 0) {
  uint32_t wa0 = 0u, wa1 = 0u, wb0 = 0u, wb1 = 0u;
  // Byte permutes of the transposed words into token pairs per column
  // (0x3120). With the hardware cvt a masked row must be zeroed (a NaN byte
  // times P = 0 would still be NaN): its bytes (0-1: token 2q, 2-3: token
  // 2q+1 of the word) are taken from the zero word instead (selector 4).
  uint32_t sel_lo = 0x3120u, sel_hi = 0x3120u;
  if (VCVT && !full) {
    const int r = tok0 + 2 * qd;
    auto in = [&](int t) { return page_ok && t >= t0 && t < t1; };
    auto sel = [](bool a, bool b) -> uint32_t {
      return (a ? 0x0u : 0x4u) | ((b ? 0x2u : 0x4u) << 4) | ((a ? 0x1u : 0x4u) << 8) |
             ((b ? 0x3u : 0x4u) << 12);
    };
    sel_lo = sel(in(r), in(r + 1));
    sel_hi = sel(in(r + 8), in(r + 9));
  }
#pragma unroll
  for (int jb = 0; jb < D / 32; ++jb) {
    const uint4 vw = ldsm_x4_trans(sv + blk_off<D>(voff, jb));
    uint32_t a0, a1, a2, a3, e0, e1, e2, e3;
    if constexpr (VCVT) {
      // [t.d, t'.d, t.d+1, t'.d+1]: each 16-bit half is one column's token pair
      const uint32_t z0 = prmt(vw.x, 0, sel_lo), z1 = prmt(vw.y, 0, sel_lo);
      const uint32_t z2 = prmt(vw.z, 0, sel_hi), z3 = prmt(vw.w, 0, sel_hi);
      a0 = e4m3x2_lo16_to_f16x2(z0);
      a1 = e4m3x2_hi16_to_f16x2(z0);
      a2 = e4m3x2_lo16_to_f16x2(z2);
      a3 = e4m3x2_hi16_to_f16x2(z2);
      e0 = e4m3x2_lo16_to_f16x2(z1);
      e1 = e4m3x2_hi16_to_f16x2(z1);
      e2 = e4m3x2_lo16_to_f16x2(z3);
      e3 = e4m3x2_hi16_to_f16x2(z3);
    } else {
      // [t.d, t.d+1, t'.d, t'.d+1]: bytes (0,2) and (1,3) are token pairs
      a0 = e4m3x2_b02_to_f16x2(vw.x);
      a1 = e4m3x2_b13_to_f16x2(vw.x);
      a2 = e4m3x2_b02_to_f16x2(vw.z);
      a3 = e4m3x2_b13_to_f16x2(vw.z);
      e0 = e4m3x2_b02_to_f16x2(vw.y);
      e1 = e4m3x2_b13_to_f16x2(vw.y);
      e2 = e4m3x2_b02_to_f16x2(vw.w);
      e3 = e4m3x2_b13_to_f16x2(vw.w);
    }
    if (vmx) {
      if ((jb & 3) == 0) {
        const uint32_t w = vmw[jb >> 2];
        wa0 = __shfl_sync(0xffffffffu, w, 16 + 2 * qd);
        wa1 = __shfl_sync(0xffffffffu, w, 17 + 2 * qd);
        wb0 = __shfl_sync(0xffffffffu, w, 24 + 2 * qd);
        wb1 = __shfl_sync(0xffffffffu, w, 25 + 2 * qd);
      }
      const int sh = 8 * (jb & 3);
      const uint32_t fa = f16_pow2(static_cast<int>((wa0 >> sh) & 0xFFu) - E) |
                          (f16_pow2(static_cast<int>((wa1 >> sh) & 0xFFu) - E) << 16);
      const uint32_t fb = f16_pow2(static_cast<int>((wb0 >> sh) & 0xFFu) - E) |
                          (f16_pow2(static_cast<int>((wb1 >> sh) & 0xFFu) - E) << 16);
      auto mul = [](uint32_t x, uint32_t f) -> uint32_t {
        const __half2 r = __hmul2(*reinterpret_cast<const __half2*>(&x),
                                  *reinterpret_cast<const __half2*>(&f));
        return *reinterpret_cast<const uint32_t*>(&r);
      };
      a0 = mul(a0, fa);
      a1 = mul(a1, fa);
      e0 = mul(e0, fa);
      e1 = mul(e1, fa);
      a2 = mul(a2, fb);
      a3 = mul(a3, fb);
      e2 = mul(e2, fb);
      e3 = mul(e3, fb);
    }
    mma16816(a.O[jb][0], a0, a1, a2, a3, bh[0], bh[1]);
    mma16816(a.O[jb][0], a0, a1, a2, a3, bl[0], bl[1]);
    mma16816(a.O[jb][1], e0, e1, e2, e3, bh[0], bh[1]);
    mma16816(a.O[jb][1], e0, e1, e2, e3, bl[0], bl[1]);
  }
}

// ---------------------------------------------------------------------------
// The fp8 compute path (opt-in; the solution page's compute="fp8"): P is
// rounded once to E4M3 and multiplies V's E4M3 bytes in E4M3 MMAs
// (m16n8k32), so neither K nor V is decoded. The MMA's 32 k-entries are 32
// tokens: this lane's k = 4t .. 4t+3 are tokens 2t, 2t+1, 2t+8, 2t+9 of the
// first tile and k = 16 + 4t .. those of the second (zero for a single tile).
// ---------------------------------------------------------------------------

// f16x2 -> E4M3x2 of values already on the E4M3 grid (exact).
__device__ __forceinline__ uint32_t f16x2_to_e4m3x2(uint32_t h) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f16x2 %0, %1;" : "=h"(r) : "r"(h));
  return r;
}

// P of one tile for the fp8 path: exp2 of the scores against the running
// maxima, added to the running sums (unrounded), then P * v_scale / vref *
// 2^8 rounded once to E4M3 (from f32), moved to the PV B layout through
// movmatrix as exact f16 values: returns this lane's bytes [p(2t), p(2t+1),
// p(2t+8), p(2t+9)] of head g = lane / 4.
template <int D>
__device__ __forceinline__ uint32_t tile_probs8(Acc<D>& a, float4 sc, float vsa, float vsb) {
  const float mb0 = (a.m0 == -CUDART_INF_F) ? 0.f : a.m0;
  const float mb1 = (a.m1 == -CUDART_INF_F) ? 0.f : a.m1;
  const float p00 = fast_exp2(sc.x - mb0), p01 = fast_exp2(sc.y - mb1);
  const float p10 = fast_exp2(sc.z - mb0), p11 = fast_exp2(sc.w - mb1);
  a.l0 += p00 + p10;
  a.l1 += p01 + p11;
  const float vra = vsa * a.inv_vref * 256.f, vrb = vsb * a.inv_vref * 256.f;
  const uint32_t ea = e4m3x2_rn_sat(p00 * vra, p01 * vra);  // token g, heads 2t, 2t+1
  const uint32_t eb = e4m3x2_rn_sat(p10 * vrb, p11 * vrb);  // token g + 8
  const uint32_t ha = movmatrix_trans(e4m3x2_lo16_to_f16x2(ea));  // head g, tokens 2t, 2t+1
  const uint32_t hb = movmatrix_trans(e4m3x2_lo16_to_f16x2(eb));  // head g, tokens 2t+8, 2t+9
  return f16x2_to_e4m3x2(ha) | (f16x2_to_e4m3x2(hb) << 16);
}

// This lane's token bytes of a transposed V block for the fp8 path: from the
// ldmatrix.trans words (bytes [t.d, t.d+1, t'.d, t'.d+1] of tokens 2t, 2t+1
// in lo and 2t+8, 2t+9 in hi), the bytes of head-dim entry d (even = false)
// or d + 1 (true) of tokens 2t, 2t+1, 2t+8, 2t+9.
__device__ __forceinline__ uint32_t v_tokens4(uint32_t lo, uint32_t hi, bool odd) {
  return prmt(lo, hi, odd ? 0x7531u : 0x6420u);
}

// Byte mask of this lane's tokens 2t, 2t+1, 2t+8, 2t+9 of a tile (0 for a
// masked token: its V bytes may be NaN codes, and NaN * 0 is NaN).
__device__ __forceinline__ uint32_t tok_mask4(int tok0, int t0, int t1, bool page_ok, bool full,
                                              int qd) {
  if (full) return ~0u;
  const int r = tok0 + 2 * qd;
  auto in = [&](int t) { return page_ok && t >= t0 && t < t1; };
  return (in(r) ? 0xFFu : 0u) | (in(r + 1) ? 0xFF00u : 0u) | (in(r + 8) ? 0xFF0000u : 0u) |
         (in(r + 9) ? 0xFF000000u : 0u);
}

// O^T[d][head] += V^T P for one or two tiles (V at sv[u], P bytes pb[u]) in
// E4M3 MMAs; the accumulator rows are those of tile_pv (d / d+1 of 32-byte
// block jb, and d + 16 / d + 17), so the epilogue is shared.
template <int D, int NT>
__device__ __forceinline__ void tile_pv8(Acc<D>& a, const uint32_t (&sv)[2], const uint32_t (&voff)[4],
                                         const uint32_t (&pb)[2], const uint32_t (&vm)[2]) {
#pragma unroll
  for (int jb = 0; jb < D / 32; ++jb) {
    uint32_t e[2][4];
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      if (u < NT) {
        const uint4 vw = ldsm_x4_trans(sv[u] + blk_off<D>(voff, jb));
        e[u][0] = v_tokens4(vw.x, vw.z, false) & vm[u];  // entry d
        e[u][1] = v_tokens4(vw.x, vw.z, true) & vm[u];   // d + 1
        e[u][2] = v_tokens4(vw.y, vw.w, false) & vm[u];  // d + 16
        e[u][3] = v_tokens4(vw.y, vw.w, true) & vm[u];   // d + 17
      } else {
        e[u][0] = e[u][1] = e[u][2] = e[u][3] = 0u;
      }
    }
    const uint32_t b1 = NT > 1 ? pb[1] : 0u;
    mma16832_e4m3(a.O[jb][0], e[0][0], e[0][1], e[1][0], e[1][1], pb[0], b1);
    mma16832_e4m3(a.O[jb][1], e[0][2], e[0][3], e[1][2], e[1][3], pb[0], b1);
  }
}

// Attends one 16-token tile already in shared memory (K at sk, V at sv) for
// one warp: S = K q'^T, masking, the online-softmax update, and O += V^T P
// with P as an f16 hi + lo pair. kfa / kfb = score factors (log2 units) and
// vsa / vsb = V scales of this lane's tokens grp / grp + 8, vabs = the
// largest |V scale| of the tile's attended tokens; tok0 = first token of the
// tile.
template <int D, int KM, bool VCVT, class QFrag>
__device__ __forceinline__ void attend_tile(Acc<D>& a, const QFrag& qfr, uint32_t sk, uint32_t sv,
                                            const uint32_t (&koff)[4], const uint32_t (&voff)[4],
                                            float kfa, float kfb, float vsa, float vsb, float vabs,
                                            int tok0, int t0, int t1, bool page_ok, bool full,
                                            int grp, int qd, float2 hf = make_float2(1.f, 1.f)) {
  const float4 sc =
      tile_scores<D, KM>(qfr, sk, koff, kfa, kfb, tok0, t0, t1, page_ok, full, grp, hf);
  softmax_rescale<D, KM != 3>(a, fmaxf(sc.x, sc.z), fmaxf(sc.y, sc.w), vabs);
  if constexpr (KM == 3) {
    const uint32_t pb[2] = {tile_probs8<D>(a, sc, vsa, vsb), 0u};
    const uint32_t svv[2] = {sv, sv};
    const uint32_t vm[2] = {tok_mask4(tok0, t0, t1, page_ok, full, qd), 0u};
    tile_pv8<D, 1>(a, svv, voff, pb, vm);
  } else {
    uint32_t bh[2], bl[2];
    tile_probs<D>(a, sc, vsa, vsb, bh, bl);
    tile_pv<D, VCVT>(a, sv, voff, bh, bl, tok0, t0, t1, page_ok, full, qd);
  }
}

// Two tiles (u = 0, 1) at once: both score blocks, one softmax update (one
// set of maximum shuffles and one rescale test for 32 keys), then both PV
// blocks; `between` runs after the first tile's PV (its stage is free then).
template <int D, int KM, bool VCVT, class QFrag, class Between>
__device__ __forceinline__ void attend_pair(Acc<D>& a, const QFrag& qfr, const uint32_t (&sk)[2],
                                            const uint32_t (&koff)[4], const uint32_t (&voff)[4],
                                            const float (&kfac)[2], const float (&vs)[2],
                                            const int (&tok0)[2], int t0, int t1,
                                            const bool (&page_ok)[2], const bool (&full)[2],
                                            int grp, int qd, const Between& between,
                                            float2 hf = make_float2(1.f, 1.f)) {
  constexpr int TILE = kTileTokens * D;
  const float4 s0 = tile_scores<D, KM>(qfr, sk[0], koff, kfac[0], kfac[0], tok0[0], t0, t1,
                                         page_ok[0], full[0], grp, hf);
  const float4 s1 = tile_scores<D, KM>(qfr, sk[1], koff, kfac[1], kfac[1], tok0[1], t0, t1,
                                         page_ok[1], full[1], grp, hf);
  softmax_rescale<D, KM != 3>(a, fmaxf(fmaxf(s0.x, s0.z), fmaxf(s1.x, s1.z)),
                     fmaxf(fmaxf(s0.y, s0.w), fmaxf(s1.y, s1.w)), fmaxf(fabsf(vs[0]), fabsf(vs[1])));
  if constexpr (KM == 3) {
    // one k32 MMA per 32-byte block covers both tiles' tokens
    const uint32_t pb[2] = {tile_probs8<D>(a, s0, vs[0], vs[0]), tile_probs8<D>(a, s1, vs[1], vs[1])};
    const uint32_t svv[2] = {sk[0] + TILE, sk[1] + TILE};
    const uint32_t vm[2] = {tok_mask4(tok0[0], t0, t1, page_ok[0], full[0], qd),
                            tok_mask4(tok0[1], t0, t1, page_ok[1], full[1], qd)};
    tile_pv8<D, 2>(a, svv, voff, pb, vm);
    between();
    return;
  }
  uint32_t bh0[2], bl0[2], bh1[2], bl1[2];
  tile_probs<D>(a, s0, vs[0], vs[0], bh0, bl0);
  tile_probs<D>(a, s1, vs[1], vs[1], bh1, bl1);
  tile_pv<D, VCVT>(a, sk[0] + TILE, voff, bh0, bl0, tok0[0], t0, t1, page_ok[0], full[0], qd);
  between();
  tile_pv<D, VCVT>(a, sk[1] + TILE, voff, bh1, bl1, tok0[1], t0, t1, page_ok[1], full[1], qd);
}

// Keys sequence b attends over: its length, or with a fused append its
// position + 1. An out-of-range value sets `flag` (when `report`) and gives 0.
__device__ __forceinline__ int attended_keys(const DecodeParams& p, int b, bool report) {
  const int v = __ldg(p.lens + (int64_t)b * p.lens_s);
  const int lim = p.max_pages * p.ps;
  if (p.append) {
    if (v >= 0 && v < lim) return v + 1;
    if (report) raise_flag(FP8PD_FLAG_POS_OOB);
    return 0;
  }
  if (v >= 0 && v <= lim) return v;
  if (report) raise_flag(FP8PD_FLAG_SEQLEN_OOB);
  return 0;
}

// The keys [lo, hi) sequence b attends, of its L: the window's range, cut to
// the sequence's key range [begin, end) when the call has one (a context-
// parallel slice).
__device__ __forceinline__ void key_range(const DecodeParams& p, int b, int L, int& lo, int& hi) {
  lo = p.window > 0 ? max(0, L - p.window) : 0;
  hi = L;
  if (p.kr) {
    lo = max(lo, __ldg(p.kr + (int64_t)b * p.kr_sb));
    hi = min(hi, __ldg(p.kr + (int64_t)b * p.kr_sb + p.kr_s1));
    hi = max(hi, lo);
  }
}

// Unnormalized result of one (sequence, query head) in partial-output mode
// (the context-parallel slices): O = sum_t 2^(s2_t - m) v_t, m = max_t s2_t
// (log2 units: the scaled score times log2 e), l = sum_t 2^(s2_t - m); no sink.
__device__ __forceinline__ void store_partial(const DecodeParams& p, int b, int head, int d,
                                              float4 o, float m, float l) {
  const int64_t row = (int64_t)b * p.Hq + head;
  *reinterpret_cast<float4*>(p.pout_o + row * p.D + d) = o;
  if (d == 0) *reinterpret_cast<float2*>(p.pout_ml + row * 2) = make_float2(m, l);
}


// Two E4M3 terms of four values x (|x| < 256): hi = E4M3(x) (round to
// nearest even), lo = E4M3(x - hi), one value per byte. A bf16 value whose
// magnitude is at least 2^-2 splits exactly (its 8 significant bits are hi's
// 4 and at most 4 more, above E4M3's smallest subnormal 2^-9); smaller ones
// keep an error below 2^-10.
__device__ __forceinline__ void e4m3_split4(float x0, float x1, float x2, float x3, uint32_t& hi,
                                            uint32_t& lo) {
  hi = (uint32_t)e4m3x2_rn_sat(x0, x1) | ((uint32_t)e4m3x2_rn_sat(x2, x3) << 16);
  const float2 h01 = unpack_f16x2(e4m3x2_lo16_to_f16x2(hi));  // exact
  const float2 h23 = unpack_f16x2(e4m3x2_hi16_to_f16x2(hi));
  lo = (uint32_t)e4m3x2_rn_sat(x0 - h01.x, x1 - h01.y) |
       ((uint32_t)e4m3x2_rn_sat(x2 - h23.x, x3 - h23.y) << 16);
}

// Per-token-per-head scale of one head's D values spread over a warp (PER
// per lane): max |x| / 448 in IEEE f32, NaN entries skipped (fmaxf), 1 for an
// all-zero row.
template <int PER>
__device__ __forceinline__ float warp_token_scale(const float (&x)[PER]) {
  float m = 0.f;
#pragma unroll
  for (int i = 0; i < PER; ++i) m = fmaxf(m, fabsf(x[i]));
  m = warp_max(m);
  return m == 0.f ? 1.f : __fdiv_rn(m, 448.f);
}

// Fused append, one warp: quantizes the new token of (sequence b, KV head
// kvh) (IEEE f32 division, then E4M3 round to nearest even with saturation,
// as fp8_kv_append), writes its codes into row r of the K and V tiles in
// shared memory (the TMA's swizzled layout, see tile_off) and, when `store`,
// into the pools at (page, slot). Lane l owns head-dim bytes
// [l D/32, (l+1) D/32). ks / vs: the page's scales; with per-token scales
// (TOK and p.k_tok / p.v_tok) they are replaced by the new token's own,
// which `store` also writes to the scale array (with sub-row K groups, ks is
// the scale of this lane's group: its 32 / k_groups lanes hold one group).
template <int D, bool TOK>
__device__ __forceinline__ void append_new_token(const DecodeParams& p, int b, int kvh, bool store,
                                              int page, int slot, int r, uint32_t sk, uint32_t sv,
                                              float& ks, float& vs, uint32_t* vcode = nullptr) {
  constexpr int PER = D / 32;  // 2, 4, 8 or 16 bytes per lane
  const int lane = threadIdx.x & 31;
  const int d0 = lane * PER;
  const uint16_t* kn = p.kn + (int64_t)b * p.kn_sb + (int64_t)kvh * p.kn_sh;
  const uint16_t* vn = p.vn + (int64_t)b * p.vn_sb + (int64_t)kvh * p.vn_sh;
  float xk[PER], xv[PER];
#pragma unroll
  for (int i = 0; i < PER; ++i) {
    xk[i] = bf16_bits_to_float(kn[(int64_t)(d0 + i) * p.kn_sd]);
    xv[i] = bf16_bits_to_float(vn[(int64_t)(d0 + i) * p.vn_sd]);
  }
  if constexpr (TOK) {
    if (p.k_tok && p.k_groups > 1) {
      // sub-row groups: the 32 / k_groups lanes of a group agree on its
      // maximum; ks becomes this lane's group scale
      const int lpg = 32 / p.k_groups;
      float m = 0.f;
#pragma unroll
      for (int i = 0; i < PER; ++i) m = fmaxf(m, fabsf(xk[i]));
      for (int o = 1; o < lpg; o <<= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
      const int64_t so = (int64_t)page * p.ks_sp + (int64_t)slot * p.ks_st + (int64_t)kvh * p.ks_sh +
                         (int64_t)(lane / lpg) * p.ks_sg;
      if (p.k_mx) {  // MXFP8: the block's E8M0 code (k_groups = D / 32)
        const uint32_t c = mx_code(m);
        ks = e8m0_to_f32(c);
        if (store && (lane & (lpg - 1)) == 0) reinterpret_cast<uint8_t*>(p.ksw)[so] = c;
      } else {
        ks = m == 0.f ? 1.f : __fdiv_rn(m, 448.f);
        if (store && (lane & (lpg - 1)) == 0) p.ksw[so] = ks;
      }
    } else if (p.k_tok) {
      ks = warp_token_scale<PER>(xk);
      if (store && lane == 0)
        p.ksw[(int64_t)page * p.ks_sp + (int64_t)slot * p.ks_st + (int64_t)kvh * p.ks_sh] = ks;
    }
    if (p.v_mx) {
      // MXFP8 V: the 1024 / D lanes of a 32-entry block agree on its code
      constexpr int LPB = 1024 / D;
      float m = 0.f;
#pragma unroll
      for (int i = 0; i < PER; ++i) m = fmaxf(m, fabsf(xv[i]));
#pragma unroll
      for (int o = 1; o < LPB; o <<= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
      const uint32_t c = mx_code(m);
      vs = e8m0_to_f32(c);
      if (vcode) *vcode = c;
      if (store && (lane & (LPB - 1)) == 0)
        reinterpret_cast<uint8_t*>(p.vsw)[(int64_t)page * p.vs_sp + (int64_t)slot * p.vs_st +
                                          (int64_t)kvh * p.vs_sh + (int64_t)(lane / LPB) * p.vs_sg] = c;
    } else if (p.v_tok) {
      vs = warp_token_scale<PER>(xv);
      if (store && lane == 0)
        p.vsw[(int64_t)page * p.vs_sp + (int64_t)slot * p.vs_st + (int64_t)kvh * p.vs_sh] = vs;
    }
  }
  uint32_t kw[(PER + 3) / 4], vw[(PER + 3) / 4];
#pragma unroll
  for (int i = 0; i < (PER + 3) / 4; ++i) kw[i] = vw[i] = 0u;
#pragma unroll
  for (int i = 0; i < PER; i += 2) {
    const uint32_t kc = e4m3x2_rn_sat(__fdiv_rn(xk[i], ks), __fdiv_rn(xk[i + 1], ks));
    const uint32_t vc = e4m3x2_rn_sat(__fdiv_rn(xv[i], vs), __fdiv_rn(xv[i + 1], vs));
    kw[i / 4] |= kc << (8 * (i % 4));
    vw[i / 4] |= vc << (8 * (i % 4));
  }
  // PER divides 16, so the lane's bytes sit inside one 16-byte chunk of the row
  const uint32_t off = tile_off<D>(r, d0 & ~15) + (d0 & 15);
  uint8_t* gk = p.kw + (int64_t)page * p.k_sp + (int64_t)slot * p.k_st + (int64_t)kvh * p.k_sh + d0;
  uint8_t* gv = p.vw + (int64_t)page * p.v_sp + (int64_t)slot * p.v_st + (int64_t)kvh * p.v_sh + d0;
  if constexpr (PER == 2) {
    asm volatile("st.shared.u16 [%0], %1;" ::"r"(sk + off), "h"((uint16_t)kw[0]) : "memory");
    asm volatile("st.shared.u16 [%0], %1;" ::"r"(sv + off), "h"((uint16_t)vw[0]) : "memory");
    if (store) {
      *reinterpret_cast<uint16_t*>(gk) = (uint16_t)kw[0];
      *reinterpret_cast<uint16_t*>(gv) = (uint16_t)vw[0];
    }
  } else if constexpr (PER == 4) {
    asm volatile("st.shared.u32 [%0], %1;" ::"r"(sk + off), "r"(kw[0]) : "memory");
    asm volatile("st.shared.u32 [%0], %1;" ::"r"(sv + off), "r"(vw[0]) : "memory");
    if (store) {
      *reinterpret_cast<uint32_t*>(gk) = kw[0];
      *reinterpret_cast<uint32_t*>(gv) = vw[0];
    }
  } else if constexpr (PER == 8) {
    asm volatile("st.shared.v2.u32 [%0], {%1, %2};" ::"r"(sk + off), "r"(kw[0]), "r"(kw[1]) : "memory");
    asm volatile("st.shared.v2.u32 [%0], {%1, %2};" ::"r"(sv + off), "r"(vw[0]), "r"(vw[1]) : "memory");
    if (store) {
      *reinterpret_cast<uint2*>(gk) = make_uint2(kw[0], kw[1]);
      *reinterpret_cast<uint2*>(gv) = make_uint2(vw[0], vw[1]);
    }
  } else {
    asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(sk + off), "r"(kw[0]), "r"(kw[1]),
                 "r"(kw[2]), "r"(kw[3]) : "memory");
    asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(sv + off), "r"(vw[0]), "r"(vw[1]),
                 "r"(vw[2]), "r"(vw[3]) : "memory");
    if (store) {
      *reinterpret_cast<uint4*>(gk) = make_uint4(kw[0], kw[1], kw[2], kw[3]);
      *reinterpret_cast<uint4*>(gv) = make_uint4(vw[0], vw[1], vw[2], vw[3]);
    }
  }
}

// Proportional splits. From the lengths, every sequence's tiles nt_b; the
// smallest split size C (tiles) with sum_b ceil(nt_b / C) <= nbx, found by
// bisection between ceil(total / nbx) and min(max nt_b, kMaxSplitTiles) (the
// planner makes nbx at least sum_b ceil(nt_b / kMaxSplitTiles), so that
// bound holds), which minimises the largest split; S_b = ceil(nt_b / C). The
// splits and the merge groups ceil(S_b / 8) go into prefix sums in
// `scratch` (the ring buffer, unused until the first copy). Block blockIdx.y
// = k takes split k - sp_b of the sequence b whose splits hold k; its tiles
// are [split * nt_b / S_b, (split + 1) * nt_b / S_b) of the attended range.
// Every block also writes the zero outputs of sequences k, k + nbx, ...
// that have no keys. Called by the whole block; ends with a barrier, after
// which the scratch is free. Returns false for a block beyond all splits.
template <int NW>
__device__ bool prop_assign(const DecodeParams& p, int* scratch, int* red, int head0, int nheads,
                            int& b, int& split, int& S, int& j0, int& j1, int& sp_b, int& gp_b) {
  constexpr int NT = NW * 32;
  constexpr unsigned FULL = 0xffffffffu;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int B = p.B;
  int* s_nt = scratch;       // [B] tiles of each sequence
  int* s_sp = s_nt + B;      // [B + 1] splits of the sequences before b
  int* s_gp = s_sp + B + 1;  // [B + 1] merge groups of the sequences before b
  int tsum = 0, tmax = 0, tcnt = 0;
  for (int bb = tid; bb < B; bb += NT) {
    const int L = attended_keys(p, bb, blockIdx.x == 0 && blockIdx.y == 0);
    int lo, hi;
    key_range(p, bb, L, lo, hi);
    const int nt = hi > lo ? (hi - 1) / kTileTokens - lo / kTileTokens + 1 : 0;
    s_nt[bb] = nt;
    tsum += nt;
    tmax = max(tmax, nt);
    tcnt += nt > 0;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    tsum += __shfl_xor_sync(FULL, tsum, o);
    tmax = max(tmax, __shfl_xor_sync(FULL, tmax, o));
    tcnt += __shfl_xor_sync(FULL, tcnt, o);
  }
  if (lane == 0) {
    red[warp] = tsum;
    red[NW + warp] = tmax;
    red[2 * NW + 1 + warp] = tcnt;
  }
  __syncthreads();
  if (warp == 0) {
    int total = 0, nmax = 0, nne = 0;
#pragma unroll
    for (int w = 0; w < NW; ++w) {
      total += red[w];
      nmax = max(nmax, red[NW + w]);
      nne += red[2 * NW + 1 + w];
    }
    // bisection for the split size C: count(C) = sum_b ceil(nt_b / C). Every
    // upper bound used satisfies count <= nbx: nmax (count = sequences with
    // keys), kMaxSplitTiles (the planner's guarantee) and, with more blocks
    // than such sequences, ceil(total / (nbx - nne)) (count <= total / C + nne).
    int lo = max(1, max((total + p.nbx - 1) / max(p.nbx, 1), (nmax + kMaxSplits - 1) / kMaxSplits));
    int hi = min(nmax, kMaxSplitTiles);
    if (p.nbx > nne) hi = min(hi, (total + (p.nbx - nne) - 1) / (p.nbx - nne));
    hi = max(lo, hi);
    if (B <= 64) {
      // Few sequences: each lane counts one candidate over all sequences (no
      // cross-lane reduction per step), candidates lo + step * lane with lane
      // 31 at hi (feasible); the smallest feasible one narrows the bracket
      // about 31-fold per round. ceil(nt
      // / c) comes from a float product: for nt < 2^22 (a sequence has at
      // most 2^17 tiles here) it is within 0.5 of nt / c, so its floor is at
      // most two below the ceiling and two exact corrections give it.
      while (lo < hi) {
        const int step = (hi - lo + 30) / 31;
        const int c = min(hi, lo + step * lane);
        const float rc = 1.f / static_cast<float>(c);
        int cnt = 0;
        for (int bb = 0; bb < B; ++bb) {
          const int nt = s_nt[bb];
          int q = static_cast<int>(static_cast<float>(nt) * rc);
          q += (q * c < nt);
          q += (q * c < nt);
          cnt += q;
        }
        const unsigned ok = __ballot_sync(FULL, cnt <= p.nbx);  // never 0: lane 31 is at hi
        const int first = __ffs(ok) - 1;
        const int c_first = min(hi, lo + step * first);
        if (first == 0) hi = lo;
        else {
          lo = min(hi, lo + step * (first - 1)) + 1;
          hi = c_first;
        }
      }
    } else {
      while (lo < hi) {
        const int mid = (lo + hi) >> 1;
        int cnt = 0;
        for (int bb = lane; bb < B; bb += 32) cnt += (s_nt[bb] + mid - 1) / mid;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) cnt += __shfl_xor_sync(FULL, cnt, o);
        if (cnt <= p.nbx) hi = mid;
        else lo = mid + 1;
      }
    }
    __syncwarp();
    if (lane == 0) red[2 * NW] = lo;
  }
  __syncthreads();
  const int C = red[2 * NW];
  auto splits_of = [&](int nt) -> int { return (nt + C - 1) / C; };
  // exclusive prefix sums, a contiguous run of sequences per thread
  const int per = (B + NT - 1) / NT;
  const int b0 = min(B, tid * per), b1 = min(B, b0 + per);
  int ssum = 0, gsum = 0;
  for (int bb = b0; bb < b1; ++bb) {
    const int s = splits_of(s_nt[bb]);
    ssum += s;
    gsum += (s + kMergeFan - 1) / kMergeFan;
  }
  int si = ssum, gi = gsum;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int vs = __shfl_up_sync(FULL, si, o), vg = __shfl_up_sync(FULL, gi, o);
    if (lane >= o) {
      si += vs;
      gi += vg;
    }
  }
  __syncthreads();  // everyone has read the block sums
  if (lane == 31) {
    red[warp] = si;
    red[NW + warp] = gi;
  }
  __syncthreads();
  int soff = si - ssum, goff = gi - gsum;
  for (int w = 0; w < warp; ++w) {
    soff += red[w];
    goff += red[NW + w];
  }
  for (int bb = b0; bb < b1; ++bb) {
    s_sp[bb] = soff;
    s_gp[bb] = goff;
    const int s = splits_of(s_nt[bb]);
    soff += s;
    goff += (s + kMergeFan - 1) / kMergeFan;
  }
  if (tid == NT - 1) {
    s_sp[B] = soff;
    s_gp[B] = goff;
  }
  __syncthreads();
  const int k = blockIdx.y;
  for (int bb = k; bb < B; bb += p.nbx) {
    if (s_nt[bb] != 0) continue;
    for (int e = tid; e < nheads * p.D; e += NT) {
      if (p.pout_o) {
        const int64_t row = (int64_t)bb * p.Hq + head0 + e / p.D;
        p.pout_o[row * p.D + (e % p.D)] = 0.f;
        if (e % p.D == 0) *reinterpret_cast<float2*>(p.pout_ml + row * 2) =
            make_float2(-CUDART_INF_F, 0.f);
      } else {
        p.out[(int64_t)bb * p.o_sb + (int64_t)(head0 + e / p.D) * p.o_sh + (e % p.D)] = 0.f;
      }
    }
  }
  const bool has = k < s_sp[B];
  if (has) {
    int lo = 0, hi = B;  // the last sequence b with s_sp[b] <= k
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (s_sp[mid] <= k) lo = mid;
      else hi = mid;
    }
    b = lo;
    sp_b = s_sp[b];
    gp_b = s_gp[b];
    split = k - sp_b;
    S = s_sp[b + 1] - sp_b;
    const int nt = s_nt[b];
    j0 = static_cast<int>((int64_t)split * nt / S);
    j1 = static_cast<int>((int64_t)(split + 1) * nt / S);
  }
  __syncthreads();  // the scratch is free again
  return has;
}

// One thread block: (split, KV head x head group, sequence). KM selects the
// QK contraction: 0 = K decoded to f16 by bit assembly (value * 2^-8), 1 = by
// the hardware cvt.rn.f16x2.e4m3x2 (the value itself), both into f16 MMAs;
// 2 = K's E4M3 bytes straight into E4M3 MMAs with q as two E4M3 terms. VCVT
// selects the E4M3 -> f16 decode of V (false = bit assembly, true = cvt). The
// q fragments follow the K byte pairing. tmk / tmv: 5-D tensor maps over the K / V pool
// views, dims (head-dim bytes within a 128-byte block, slot, 128-byte block,
// KV head, page), box (min(D,128), 16, max(1, D/128), 1, 1). TOK: the scales
// are read per token (one per stored token and KV head) instead of per page.
template <int D, int KM, bool VCVT, int SC, int DS = 1>
__global__ void __launch_bounds__(Cfg<D, DS>::NT, Cfg<D, DS>::MIN_BLOCKS)
    decode_tma_kernel(const DecodeParams p, const __grid_constant__ CUtensorMap tmk,
                      const __grid_constant__ CUtensorMap tmv) {
  using C = Cfg<D, DS>;
  static_assert(DS == 1 || (KM == 1 && VCVT && SC == 0 && C::Q_IN_SMEM),
                "head-dim split: page or head scales, cvt decodes, q fragments in smem");
  constexpr int DW = C::DW;  // head-dim entries this warp copies and contracts
  constexpr bool TOK = SC >= 1;  // scales read per stored token
  constexpr bool VMX = SC == 2;  // V in MXFP8 (E8M0 block scales)
  constexpr int KB = D / 16;  // k16 blocks of the QK contraction
  extern __shared__ uint8_t smem_raw[];
  // 1024-byte aligned base for the swizzled tiles
  uint8_t* smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
  uint8_t* pipe = smem;
  uint2* qfrag_s = reinterpret_cast<uint2*>(smem + C::PIPE_BYTES);
  float4* s_xch = reinterpret_cast<float4*>(smem + C::PIPE_BYTES + C::QFRAG_BYTES);
  int32_t* s_ent = reinterpret_cast<int32_t*>(smem + C::PIPE_BYTES + C::QFRAG_BYTES + C::XCH_BYTES);
  float* s_ks = reinterpret_cast<float*>(s_ent + C::NLW * kMaxWarpTiles);
  float* s_vs = s_ks + C::NLW * kMaxWarpTiles;
  uint64_t* s_bar = reinterpret_cast<uint64_t*>(s_vs + C::NLW * kMaxWarpTiles);
  float* misc = reinterpret_cast<float*>(s_bar + C::NW * C::NS);

  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31, grp = lane >> 2, qd = lane & 3;
  // tile stream lw of the block; this warp's part of its head dim: `half`
  const int lw = warp / DS, half = warp - lw * DS;
  // The DS warps of a stream meet at named barrier 1 + lw (64 threads).
  auto stream_sync = [&]() {
    if constexpr (DS > 1) asm volatile("bar.sync %0, %1;" ::"r"(1 + lw), "r"(DS * 32) : "memory");
    else __syncwarp();
  };
  const int kvh = blockIdx.x / p.head_groups;
  const int hg = blockIdx.x - kvh * p.head_groups;
  const int head0 = kvh * p.G + hg * 8;
  const int nheads = min(8, p.G - hg * 8);

  // Which split of which sequence this block takes. Uniform splits: grid
  // (KV head x head group, sequence, split), every sequence cut into S equal
  // page ranges; all first splits dispatch before any second split, so the
  // longest blocks start first. Proportional splits: grid (KV head x head
  // group, nbx); sequence b gets S_b of the nbx blocks, S_b proportional to
  // its tiles, and its tiles are cut into S_b near-equal ranges.
  int b, split, S;
  int prop_j0 = 0, prop_j1 = 0;  // proportional: tiles [j0, j1) of the attended range
  int sp_b = 0, gp_b = 0;        // proportional: splits and merge groups of sequences < b
  if (p.prop) {
    if (!prop_assign<C::NW>(p, reinterpret_cast<int*>(pipe), reinterpret_cast<int*>(misc), head0,
                            nheads, b, split, S, prop_j0, prop_j1, sp_b, gp_b))
      return;  // a block beyond the splits of all sequences
  } else {
    b = blockIdx.y;
    split = blockIdx.z;
    S = p.num_splits;
  }

  // q of this lane's query head (grp): entries 16kb + 4q + {0..3} of every
  // k16 block kb, loaded before anything else so that their latency overlaps
  // the rest of the setup (one 8-byte load per block when q is contiguous).
  const bool q_head_ok = grp < nheads;
  const uint16_t* qrow = p.q + (int64_t)b * p.q_sb + (int64_t)(head0 + (q_head_ok ? grp : 0)) * p.q_sh;
  constexpr int QR = C::Q_IN_SMEM ? 1 : KB;
  uint2 qraw[QR];
  if constexpr (!C::Q_IN_SMEM) {
#pragma unroll
    for (int kb = 0; kb < KB; ++kb) {
      const int d = 16 * kb + 4 * qd;
      uint2 v = make_uint2(0u, 0u);
      if (q_head_ok) {
        if (p.q_vec) {
          v = __ldg(reinterpret_cast<const uint2*>(qrow + d));
        } else {
          const uint32_t e0 = __ldg(qrow + (int64_t)(d + 0) * p.q_sd);
          const uint32_t e1 = __ldg(qrow + (int64_t)(d + 1) * p.q_sd);
          const uint32_t e2 = __ldg(qrow + (int64_t)(d + 2) * p.q_sd);
          const uint32_t e3 = __ldg(qrow + (int64_t)(d + 3) * p.q_sd);
          v = make_uint2(e0 | (e1 << 16), e2 | (e3 << 16));
        }
      }
      qraw[kb] = v;
    }
  }

  const uint32_t wbar = smem_u32(s_bar + warp * C::NS);
  if (lane == 0) {
    prefetch_tensormap(&tmk);
    prefetch_tensormap(&tmv);
#pragma unroll
    for (int s = 0; s < C::NS; ++s) mbar_init(wbar + 8 * s, 1);
    fence_barrier_init();
    fence_proxy_async();
  }

  const int32_t* trow = p.table + (int64_t)b * p.tab_sb;
  const uint32_t wpipe = smem_u32(pipe + warp * C::WARP_BYTES);
  // Lane 0 copies the tile with entry e (see below) into ring stage `stage`:
  // one TMA for K, one for V, both completing on the stage's barrier. A tile
  // whose page is out of range is not copied; its barrier phase still
  // completes.
  // Test hook of the bounded waits (p.test_stall): warp 0 of the launch's
  // first block posts the bytes of its first copy on the stage's barrier but
  // issues no copy, so that wait, and only that one, runs out.
  bool stall = p.test_stall && warp == 0 && blockIdx.x == 0 && blockIdx.y == 0 && blockIdx.z == 0;
  auto issue = [&](int e, int stage) {
    if (lane != 0) return;
    const uint32_t bar = wbar + 8 * stage;
    if (e < 0) {
      mbar_arrive(bar);
      return;
    }
    const int page = e >> 4, slot0 = (e & 15) * kTileTokens;
    const uint32_t sk = wpipe + stage * C::STAGE;
    fence_proxy_async();  // this warp's earlier reads of the stage come first
    mbar_arrive_expect_tx(bar, 2 * C::TILE);
    if (stall) {
      stall = false;
      return;
    }
    tma_load_5d(sk, &tmk, bar, 0, slot0, half * (DW / 128), kvh, page);
    tma_load_5d(sk + C::TILE, &tmv, bar, 0, slot0, half * (DW / 128), kvh, page);
  };
  // Without a window a split starts at page split * chunk whatever the
  // sequence length, so the first tiles of each warp are copied before the
  // length is known. Copies past the end of a short sequence are drained
  // before the block exits; a page id outside the pool is never copied.
  // (Proportional splits know their range by now: they build the tile list
  // first and copy from it, which saves a second block-table round trip.)
  const bool spec = p.window == 0 && !p.prop && !p.kr;
  if (spec) {
    const int tf = p.prop ? prop_j0 : split * p.chunk_pages * (p.ps / kTileTokens);
    int e = -1;
    if (lane < C::NS - 1) {
      const int tok = (tf + lw + C::NLW * lane) * kTileTokens;
      const int lp = tok / p.ps;
      if (lp < p.max_pages) {
        const int page = __ldg(trow + (int64_t)lp * p.tab_sp);
        if ((unsigned)page < (unsigned)p.num_pages) e = (page << 4) | ((tok - lp * p.ps) / kTileTokens);
      }
    }
#pragma unroll
    for (int s = 0; s < C::NS - 1; ++s) issue(__shfl_sync(0xffffffffu, e, s), s);
  }

  // ---- the keys this block attends: [t0, t1) ------------------------------
  // Split s of a sequence covers pages [first + s * chunk, first + (s+1) * chunk)
  // of its attended range: equal-sized work per block whatever the length,
  // and the blocks past the end of a short sequence have nothing to do.
  const int L = attended_keys(p, b, tid == 0 && split == 0 && blockIdx.x == 0);
  int lo, hi;  // the attended keys of the sequence
  key_range(p, b, L, lo, hi);
  int t0, t1;
  if (p.prop) {
    t0 = max(lo, (lo / kTileTokens + prop_j0) * kTileTokens);
    t1 = min(hi, (lo / kTileTokens + prop_j1) * kTileTokens);
  } else {
    const int first_page = lo / p.ps;
    const int n_pages = (hi > lo) ? (hi - 1) / p.ps - first_page + 1 : 0;
    const int pg0 = first_page + split * p.chunk_pages;
    const int pg1 = min(first_page + n_pages, pg0 + p.chunk_pages);
    t0 = max(lo, pg0 * p.ps);
    t1 = min(hi, pg1 * p.ps);
  }
  const int tile_first = t0 / kTileTokens;
  const int n_tiles = (t1 > t0) ? (t1 + kTileTokens - 1) / kTileTokens - tile_first : 0;
  int my_tiles = (n_tiles > lw) ? (n_tiles - lw + C::NLW - 1) / C::NLW : 0;
  if (my_tiles > kMaxWarpTiles) {  // the planner never does this; refuse rather than overflow
    if (lane == 0) raise_flag(FP8PD_FLAG_INTERNAL);
    my_tiles = 0;
  }

  // ---- warp-local setup: tile list, first copies, scales, q fragments -------
  // Tile j of stream w starts at token 16 * (tile_first + w + 4j). Its entry is
  // (page << 4) | (tile index inside the page), or -1 for a block-table entry
  // outside the pool; the page's k and v scales sit beside it. The page ids
  // come first so the first tile copies are in flight while the scales and
  // the q fragments load.
  int32_t* went = s_ent + lw * kMaxWarpTiles;
  float* wks = s_ks + lw * kMaxWarpTiles;
  float* wvs = s_vs + lw * kMaxWarpTiles;
#pragma unroll 2
  for (int j = lane; half == 0 && j < my_tiles; j += 32) {
    const int tok = (tile_first + lw + C::NLW * j) * kTileTokens;
    const int lp = tok / p.ps;
    const int page = __ldg(trow + (int64_t)lp * p.tab_sp);
    int e = -1;
    if ((unsigned)page < (unsigned)p.num_pages) {
      e = (page << 4) | ((tok - lp * p.ps) / kTileTokens);
    } else if (hg == 0) {
      raise_flag(FP8PD_FLAG_PAGE_OOB);
    }
    went[j] = e;
  }
  stream_sync();

  if (!spec) {
#pragma unroll 1
    for (int s = 0; s < C::NS - 1; ++s)
      if (s < my_tiles) issue(went[s], s);
  }

  // The scales go straight to shared memory (asynchronous copies); each lane
  // waits for its own copies after the first tile has arrived, so their
  // latency overlaps that of the first tile copies.
  const float* ksbase = p.ks + (int64_t)kvh * p.ks_sh;
  const float* vsbase = p.vs + (int64_t)kvh * p.vs_sh;
  if constexpr (!TOK) {
#pragma unroll 2
    for (int j = lane; half == 0 && j < my_tiles; j += 32) {
      const int e = went[j];
      if (e >= 0) {
        cp_async4(wks + j, ksbase + (int64_t)(e >> 4) * p.ks_sp);
        cp_async4(wvs + j, vsbase + (int64_t)(e >> 4) * p.vs_sp);
      } else {
        wks[j] = 0.f;
        wvs[j] = 0.f;
      }
    }
  }
  // Lane (g, q) holds query head g of the group; the k16 block kb covers
  // head-dim entries 16kb + 4q + {0..3} of lane quad q. Hardware-cvt K pairs
  // bytes (0,1) and (2,3): k = 2q -> +0, 2q+1 -> +1, 2q+8 -> +2, 2q+9 -> +3;
  // bit-assembly K pairs (0,2) and (1,3): k = 2q -> +0, 2q+1 -> +2, 2q+8 -> +1,
  // 2q+9 -> +3.
  auto max4 = [](uint2 v) -> float {
    return fmaxf(fmaxf(fabsf(__uint_as_float(v.x << 16)), fabsf(__uint_as_float(v.x & 0xFFFF0000u))),
                 fmaxf(fabsf(__uint_as_float(v.y << 16)), fabsf(__uint_as_float(v.y & 0xFFFF0000u))));
  };
  float qmax = 0.f;
  if constexpr (C::Q_IN_SMEM) {
    // this warp's k16 blocks (kb = warp mod NW): one 8-byte load of raw bf16
    // pairs per lane and block, all in flight together, parked in the
    // fragment slots they become; the block then agrees on max|q|
#pragma unroll
    for (int i = 0; i < (KB + C::NW - 1) / C::NW; ++i) {
      const int kb = warp + C::NW * i;
      if (kb >= KB) break;
      const int d = 16 * kb + 4 * qd;
      uint2 v = make_uint2(0u, 0u);
      if (q_head_ok) {
        if (p.q_vec) {
          v = __ldg(reinterpret_cast<const uint2*>(qrow + d));
        } else {
          const uint32_t e0 = __ldg(qrow + (int64_t)(d + 0) * p.q_sd);
          const uint32_t e1 = __ldg(qrow + (int64_t)(d + 1) * p.q_sd);
          const uint32_t e2 = __ldg(qrow + (int64_t)(d + 2) * p.q_sd);
          const uint32_t e3 = __ldg(qrow + (int64_t)(d + 3) * p.q_sd);
          v = make_uint2(e0 | (e1 << 16), e2 | (e3 << 16));
        }
      }
      qfrag_s[kb * 32 + lane] = v;
      qmax = fmaxf(qmax, max4(v));
    }
    if constexpr (KM == 3) {
      // fp8 compute: one maximum per query head (this lane's head g lives in
      // lanes 4g .. 4g+3 of every warp)
      qmax = fmaxf(qmax, __shfl_xor_sync(0xffffffffu, qmax, 1));
      qmax = fmaxf(qmax, __shfl_xor_sync(0xffffffffu, qmax, 2));
      if (qd == 0) misc[warp * 8 + grp] = qmax;  // free until the warps merge
      __syncthreads();
#pragma unroll
      for (int w = 0; w < C::NW; ++w) qmax = fmaxf(qmax, misc[w * 8 + grp]);
    } else {
      qmax = warp_max(qmax);
      if (lane == 0) misc[warp] = qmax;  // free until the warps merge
      __syncthreads();
#pragma unroll
      for (int w = 0; w < C::NW; ++w) qmax = fmaxf(qmax, misc[w]);
    }
  } else {
#pragma unroll
    for (int kb = 0; kb < KB; ++kb) qmax = fmaxf(qmax, max4(qraw[kb]));
    if constexpr (KM == 3) {
      qmax = fmaxf(qmax, __shfl_xor_sync(0xffffffffu, qmax, 1));
      qmax = fmaxf(qmax, __shfl_xor_sync(0xffffffffu, qmax, 2));
    } else {
      qmax = warp_max(qmax);
    }
  }
  // q' = q * 2^(15 - e) puts max|q'| in [2^14, 2^15): exact in f16 for every
  // element above max|q| * 2^-28 (bf16 has 8 significant bits). For the E4M3
  // contraction q' = q * 2^(8 - e) puts it in [2^7, 2^8), below E4M3's 448,
  // and every element above max|q| * 2^-10 splits exactly into two terms.
  int qe = 0;
  if (qmax > 0.f && isfinite(qmax)) frexpf(qmax, &qe);
  qe = max(qe, -111);
  const float qmul = ldexpf(1.f, (KM >= 2 ? 8 : 15) - qe);
  // kfac = sm_scale * log2(e) / qmul * k_scale(page), times 2^8 when K is
  // decoded by bit assembly (which yields value * 2^-8); the hardware cvt
  // and the E4M3 MMA take the value itself. The fp8 compute path scales each
  // query head by its own power of two: its factors hf (of this lane's score
  // heads 2qd and 2qd + 1) stay out of score_base.
  const float score_base = p.sm_scale_log2 * (KM == 0 ? 256.f : 1.f) / (KM == 3 ? 1.f : qmul);
  float2 hf = make_float2(1.f, 1.f);
  if constexpr (KM == 3) {
    const float inv = 1.f / qmul;  // a power of two: exact
    hf = make_float2(__shfl_sync(0xffffffffu, inv, 8 * qd), __shfl_sync(0xffffffffu, inv, 8 * qd + 4));
  }
  uint32_t qf[C::Q_IN_SMEM ? 1 : KB][2];
#pragma unroll
  for (int kb = 0; kb < KB; ++kb) {
    float x0, x1, x2, x3;
    if constexpr (C::Q_IN_SMEM) {
      if ((kb % C::NW) != warp) continue;  // this warp's blocks, converted in place
      const uint2 v = qfrag_s[kb * 32 + lane];
      x0 = __uint_as_float(v.x << 16);
      x1 = __uint_as_float(v.x & 0xFFFF0000u);
      x2 = __uint_as_float(v.y << 16);
      x3 = __uint_as_float(v.y & 0xFFFF0000u);
    } else {
      const uint2 v = qraw[kb];
      x0 = __uint_as_float(v.x << 16);
      x1 = __uint_as_float(v.x & 0xFFFF0000u);
      x2 = __uint_as_float(v.y << 16);
      x3 = __uint_as_float(v.y & 0xFFFF0000u);
    }
    uint32_t r0, r1;
    if constexpr (KM == 3) {
      // one E4M3 rounding of q (the fp8 compute path)
      r0 = (uint32_t)e4m3x2_rn_sat(x0 * qmul, x1 * qmul) |
           ((uint32_t)e4m3x2_rn_sat(x2 * qmul, x3 * qmul) << 16);
      r1 = 0u;
    } else if constexpr (KM == 2) {
      e4m3_split4(x0 * qmul, x1 * qmul, x2 * qmul, x3 * qmul, r0, r1);  // (hi, lo)
    } else if constexpr (KM == 1) {
      r0 = pack_f16x2(x0 * qmul, x1 * qmul);
      r1 = pack_f16x2(x2 * qmul, x3 * qmul);
    } else {
      r0 = pack_f16x2(x0 * qmul, x2 * qmul);
      r1 = pack_f16x2(x1 * qmul, x3 * qmul);
    }
    if constexpr (C::Q_IN_SMEM) {
      qfrag_s[kb * 32 + lane] = make_uint2(r0, r1);
    } else {
      qf[kb][0] = r0;
      qf[kb][1] = r1;
    }
  }
  // With a head-dim split the stream's first warp copied the scales: its
  // copies complete before the block barrier, which shows them to the other.
  if constexpr (DS > 1) cp_async_wait_all();
  if constexpr (C::Q_IN_SMEM) __syncthreads();
  __syncwarp();

  // ---- per-warp pipeline over 16-token tiles --------------------------------
  uint32_t koff[4], voff[4];
  ldsm_offsets<DW>(lane, koff, voff);
  // q' fragment of k16 block kb of this warp's part of the head dim
  auto qfr = [&](int kb) -> uint2 {
    if constexpr (C::Q_IN_SMEM) return qfrag_s[(kb + half * (DW / 16)) * 32 + lane];
    else return make_uint2(qf[kb][0], qf[kb][1]);
  };
  Acc<DW> acc;
  acc.reset();
  bool ok_all = true;

  // Per-token scales (TOK): lane l < 16 holds the K scale of token l of a
  // tile and lane 16 + l its V scale, 0 for a token outside [t0, t1); the
  // next tile's are loaded while this one is attended.
  auto tok_scale = [&](int j) -> float {
    const int e = went[j];
    const int r = lane & 15;
    const int t = (tile_first + lw + C::NLW * j) * kTileTokens + r;
    if (e < 0 || t < t0 || t >= t1 || (lane < 16 && p.k_groups > 1)) return 0.f;
    if (VMX && lane >= 16) return 1.f;  // attended; the tile's MX scale comes later
    const int64_t slot = (e & 15) * kTileTokens + r;
    return lane < 16 ? __ldg(ksbase + (int64_t)(e >> 4) * p.ks_sp + slot * p.ks_st)
                     : __ldg(vsbase + (int64_t)(e >> 4) * p.vs_sp + slot * p.vs_st);
  };
  float tsc_next = 0.f;
  // MXFP8 V (VMX): lane 16 + r holds the D / 32 E8M0 codes of token r of a
  // tile in VW words (byte g = block g; 0 for a token outside the keys), the
  // next tile's loaded while this one is attended.
  constexpr int VW = VMX ? (D / 32 + 3) / 4 : 1;
  const uint8_t* vs8 = reinterpret_cast<const uint8_t*>(p.vs) + (int64_t)kvh * p.vs_sh;
  uint32_t vmw[VW], vmw_next[VW];
#pragma unroll
  for (int k = 0; k < VW; ++k) vmw[k] = vmw_next[k] = 0u;
  auto vmx_load = [&](int j, uint32_t (&w)[VW]) {
#pragma unroll
    for (int k = 0; k < VW; ++k) w[k] = 0u;
    if (!VMX || lane < 16) return;
    const int e = went[j];
    const int r = lane - 16;
    const int t = (tile_first + lw + C::NLW * j) * kTileTokens + r;
    if (e < 0 || t < t0 || t >= t1) return;
    const uint8_t* src = vs8 + (int64_t)(e >> 4) * p.vs_sp +
                         (int64_t)((e & 15) * kTileTokens + r) * p.vs_st;
#pragma unroll
    for (int g = 0; g < D / 32; ++g)
      w[g >> 2] |= static_cast<uint32_t>(__ldg(src + (int64_t)g * p.vs_sg)) << (8 * (g & 3));
  };
  // Sub-row K groups (TOK, k_groups = G > 1, G <= D / 16): the tile's
  // 16 x G K scales, entry i = 16-token row r = i / G, group g = i % G; lane l
  // loads entries l + 32 m (m < G / 2 <= GKN) of the next tile into gk_next and, when the tile
  // comes up, stores them in shared memory (rows 0-7 in this warp's wks,
  // rows 8-15 in its wvs, G floats per row; both are free with TOK).
  const int kg = TOK ? p.k_groups : 1;
  const int kg_log2 = 31 - __clz(kg);
  const int kb_log2 = 31 - __clz(max(1, KB / kg));  // k16 blocks per group (log2)
  constexpr int GKN = (D / 32 < 8) ? D / 32 : 8;
  float gk_next[GKN];
  auto group_scales = [&](int j, float (&o)[GKN]) {
    const int e = went[j];
#pragma unroll
    for (int m = 0; m < GKN; ++m) {
      const int i = lane + 32 * m;
      float v = 0.f;
      if (e >= 0 && i < 16 * kg) {
        const int r = i >> kg_log2, g = i & (kg - 1);
        const int64_t off = (int64_t)(e >> 4) * p.ks_sp +
                            (int64_t)((e & 15) * kTileTokens + r) * p.ks_st + (int64_t)g * p.ks_sg;
        v = p.k_mx ? e8m0_to_f32(__ldg(reinterpret_cast<const uint8_t*>(p.ks) +
                                       (int64_t)kvh * p.ks_sh + off))
                   : __ldg(ksbase + off);
      }
      o[m] = v;
    }
  };
  auto group_row = [&](int r) -> float* { return (r < 8 ? wks : wvs) + (r & 7) * kg; };
  if constexpr (TOK) {
    if (my_tiles > 0) {
      tsc_next = tok_scale(0);
      if (kg > 1) group_scales(0, gk_next);
      if constexpr (VMX) vmx_load(0, vmw_next);
    }
  }

  int stage = 0;
  uint32_t phase = 0;
  int tok0 = (tile_first + lw) * kTileTokens;
  // two tiles per softmax step: the ring must hold both next to the one being
  // refilled, so the step needs at least three stages
  constexpr bool PAIRS = (C::PAIR || KM == 3) && C::NS >= 3 && DS == 1;
  if constexpr (PAIRS && !TOK) {
    // Two tiles per step while two are left (one softmax update per 32 keys;
    // the copy into the first tile's stage is issued once its PV is done).
#pragma unroll 1
    for (int j = 0; j + 1 < my_tiles; j += 2, tok0 += 2 * C::NLW * kTileTokens) {
      const int st1 = (stage + 1 == C::NS) ? 0 : stage + 1;
      const uint32_t ph1 = (stage + 1 == C::NS) ? (phase ^ 1u) : phase;
      if (!mbar_wait(wbar + 8 * stage, phase, p.wait_polls) || !mbar_wait(wbar + 8 * st1, ph1, p.wait_polls)) {
        if (lane == 0) raise_flag(FP8PD_FLAG_TIMEOUT);
        ok_all = false;
        break;
      }
      if (j == 0) cp_async_wait_all();  // this lane's scale copies
      __syncwarp();
      {
        const int nj = j + C::NS - 1;
        if (nj < my_tiles) issue(went[nj], stage == 0 ? C::NS - 1 : stage - 1);
      }
      const int st0 = stage;
      uint32_t sk[2];
      float kfac[2], vsc[2];
      int tk[2];
      bool pok[2], full[2];
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const int jj = j + u;
        tk[u] = tok0 + u * C::NLW * kTileTokens;
        pok[u] = went[jj] >= 0;
        full[u] = pok[u] && tk[u] >= t0 && tk[u] + kTileTokens <= t1;
        sk[u] = wpipe + (u ? st1 : st0) * C::STAGE;
        kfac[u] = score_base * wks[jj];
        vsc[u] = wvs[jj];
        if (p.append && pok[u] && L - 1 >= tk[u] && L - 1 < tk[u] + kTileTokens) {
          // the new token: quantized here, stored by head group 0, attended by all
          const int r = L - 1 - tk[u];
          float ks = wks[jj];
          append_new_token<D, false>(p, b, kvh, hg == 0, went[jj] >> 4,
                                     (went[jj] & 15) * kTileTokens + r, r, sk[u],
                                     sk[u] + C::TILE, ks, vsc[u]);
          __syncwarp();
        }
      }
      stage = st1;
      if (++stage == C::NS) {
        stage = 0;
        phase = ph1 ^ 1u;
      } else {
        phase = ph1;
      }
      attend_pair<D, KM, VCVT>(acc, qfr, sk, koff, voff, kfac, vsc, tk, t0, t1, pok, full, grp,
                                 qd, [&]() {
                                   const int nj = j + C::NS;
                                   if (nj < my_tiles) issue(went[nj], st0);
                                 }, hf);
    }
  }
  if constexpr (DS > 1) {
    // Head-dim split: each warp of the stream waits for its own part-width
    // tile, contracts its part of S, and the parts (and whether each copy
    // arrived) meet in shared memory, so all the stream's warps run the same
    // softmax on the same scores and leave the loop together; then each
    // accumulates its own head-dim part of O. The copy into the previous
    // stage is issued once all have decided to go on.
    int* s_xok = reinterpret_cast<int*>(s_xch + C::NLW * 2 * DS * 32);
#pragma unroll 1
    for (int j = 0; ok_all && j < my_tiles; ++j, tok0 += C::NLW * kTileTokens) {
      const bool got = mbar_wait(wbar + 8 * stage, phase, p.wait_polls);
      if (!got && lane == 0) raise_flag(FP8PD_FLAG_TIMEOUT);
      const bool page_ok = went[j] >= 0;
      const bool full = page_ok && tok0 >= t0 && tok0 + kTileTokens <= t1;  // warp-uniform
      const uint32_t sk = wpipe + stage * C::STAGE;
      const uint32_t sv = sk + C::TILE;
      const float kfac = score_base * wks[j];
      const float vs = wvs[j];
      // (a tile that never arrived is read all the same; its scores are dropped)
      float4 sc = tile_scores<DW, 1>(qfr, sk, koff, kfac, kfac, tok0, t0, t1, page_ok, full, grp);
      const int xb = (lw * 2 + (j & 1)) * DS;  // this tile's buffer of the stream
      s_xch[(xb + half) * 32 + lane] = sc;
      if (lane == 0) s_xok[xb + half] = got ? 1 : 0;
      stream_sync();
      bool all_got = true;
#pragma unroll
      for (int h = 0; h < DS; ++h) all_got = all_got && s_xok[xb + h] != 0;
      if (!all_got) {
        ok_all = false;
        break;
      }
      // the parts summed in the same order by every warp of the stream, so
      // all of them hold the same scores (masked entries are -inf in every part)
      {
        float4 t = (half == 0) ? sc : s_xch[xb * 32 + lane];
#pragma unroll
        for (int h = 1; h < DS; ++h) {
          const float4 o = (h == half) ? sc : s_xch[(xb + h) * 32 + lane];
          t = make_float4(t.x + o.x, t.y + o.y, t.z + o.z, t.w + o.w);
        }
        sc = t;
      }
      {
        const int nj = j + C::NS - 1;
        if (nj < my_tiles) issue(went[nj], stage == 0 ? C::NS - 1 : stage - 1);
      }
      if (++stage == C::NS) {
        stage = 0;
        phase ^= 1;
      }
      softmax_rescale<DW, true>(acc, fmaxf(sc.x, sc.z), fmaxf(sc.y, sc.w), fabsf(vs));
      uint32_t bh[2], bl[2];
      tile_probs<DW>(acc, sc, vs, vs, bh, bl);
      tile_pv<DW, VCVT>(acc, sv, voff, bh, bl, tok0, t0, t1, page_ok, full, qd);
    }
  } else {
#pragma unroll 1
  for (int j = (PAIRS && !TOK) ? (my_tiles & ~1) : 0; ok_all && j < my_tiles;
       ++j, tok0 += C::NLW * kTileTokens) {
    if (!mbar_wait(wbar + 8 * stage, phase, p.wait_polls)) {
      if (lane == 0) raise_flag(FP8PD_FLAG_TIMEOUT);
      ok_all = false;
      break;
    }
    if (j == 0) cp_async_wait_all();  // this lane's scale copies
    __syncwarp();
    {
      const int nj = j + C::NS - 1;
      if (nj < my_tiles) issue(went[nj], stage == 0 ? C::NS - 1 : stage - 1);
    }
    const bool page_ok = went[j] >= 0;
    const bool full = page_ok && tok0 >= t0 && tok0 + kTileTokens <= t1;  // warp-uniform
    const uint32_t sk = wpipe + stage * C::STAGE;
    const uint32_t sv = sk + C::TILE;
    if (++stage == C::NS) {
      stage = 0;
      phase ^= 1;
    }
    // the new token: quantized here, stored by head group 0, attended by all
    const bool has_new = p.append && page_ok && L - 1 >= tok0 && L - 1 < tok0 + kTileTokens;
    if constexpr (TOK) {
      float tsc = tsc_next;
      if (j + 1 < my_tiles) tsc_next = tok_scale(j + 1);
      if constexpr (VMX) {
#pragma unroll
        for (int k = 0; k < VW; ++k) vmw[k] = vmw_next[k];
        if (j + 1 < my_tiles) vmx_load(j + 1, vmw_next);
      }
      if (kg > 1) {
        float gk[GKN];
#pragma unroll
        for (int m = 0; m < GKN; ++m) gk[m] = gk_next[m];
        if (j + 1 < my_tiles) group_scales(j + 1, gk_next);
        __syncwarp();  // the previous tile's reads of the rows are done
#pragma unroll
        for (int m = 0; m < GKN; ++m) {
          const int i = lane + 32 * m;
          if (i < 16 * kg) group_row(i >> kg_log2)[i & (kg - 1)] = gk[m];
        }
        __syncwarp();
      }
      if (has_new) {
        const int r = L - 1 - tok0;
        float ks = __shfl_sync(0xffffffffu, tsc, r), vs = __shfl_sync(0xffffffffu, tsc, 16 + r);
        uint32_t vcode = 0u;
        append_new_token<D, true>(p, b, kvh, hg == 0, went[j] >> 4,
                                  (went[j] & 15) * kTileTokens + r, r, sk, sv, ks, vs, &vcode);
        if (kg > 1) {
          const int lpg = 32 / kg;  // lanes of one K group in the append
          if ((lane & (lpg - 1)) == 0) group_row(r)[lane / lpg] = ks;
        } else if (lane == r) {
          tsc = ks;
        }
        if (lane == 16 + r) tsc = vs;
        if constexpr (VMX) {
          // the new token's block codes into the words of lane 16 + r
#pragma unroll
          for (int g = 0; g < D / 32; ++g) {
            const uint32_t c = __shfl_sync(0xffffffffu, vcode, g * (1024 / D));
            if (lane == 16 + r) {
              if ((g & 3) == 0) vmw[g >> 2] = 0u;
              vmw[g >> 2] |= c << (8 * (g & 3));
            }
          }
        }
        __syncwarp();
      }
      int vE = 0;  // MXFP8 V: the tile's largest block code of an attended token
      if constexpr (VMX) {
        int mine = -1;
        if (lane >= 16 && tsc != 0.f) {
#pragma unroll
          for (int g = 0; g < D / 32; ++g)
            mine = max(mine, static_cast<int>((vmw[g >> 2] >> (8 * (g & 3))) & 0xFFu));
        }
        vE = __reduce_max_sync(0xffffffffu, mine);
        const float vtile = vE >= 0 ? e8m0_to_f32(static_cast<uint32_t>(vE)) : 0.f;
        if (lane >= 16) tsc = tsc != 0.f ? vtile : 0.f;
      }
      const float vsa = __shfl_sync(0xffffffffu, tsc, 16 + grp);
      const float vsb = __shfl_sync(0xffffffffu, tsc, 24 + grp);
      const float vabs = warp_max(lane >= 16 ? fabsf(tsc) : 0.f);
      float4 sc;
      if (kg > 1) {
        sc = tile_scores_groups<D, (KM == 0 ? 0 : 1)>(
            qfr, sk, koff, group_row(grp), group_row(grp + 8), kb_log2, score_base, tok0, t0, t1,
            page_ok, full, grp);
      } else {
        const float kfa = score_base * __shfl_sync(0xffffffffu, tsc, grp);
        const float kfb = score_base * __shfl_sync(0xffffffffu, tsc, grp + 8);
        sc = tile_scores<D, (KM == 0 ? 0 : 1)>(qfr, sk, koff, kfa, kfb, tok0, t0, t1, page_ok,
                                               full, grp);
      }
      softmax_rescale<D, true>(acc, fmaxf(sc.x, sc.z), fmaxf(sc.y, sc.w), vabs);
      uint32_t bh[2], bl[2];
      tile_probs<D>(acc, sc, vsa, vsb, bh, bl);
      tile_pv<D, VCVT>(acc, sv, voff, bh, bl, tok0, t0, t1, page_ok, full, qd, VMX, vmw, vE);
    } else {
      const float kfac = score_base * wks[j];
      float ks = wks[j], vs = wvs[j];
      if (has_new) {
        const int r = L - 1 - tok0;
        append_new_token<D, false>(p, b, kvh, hg == 0, went[j] >> 4,
                                   (went[j] & 15) * kTileTokens + r, r, sk, sv, ks, vs);
        __syncwarp();
      }
      attend_tile<D, KM, VCVT>(acc, qfr, sk, sv, koff, voff, kfac, kfac, vs, vs, fabsf(vs), tok0,
                                 t0, t1, page_ok, full, grp, qd, hf);
    }
  }
  }
  if constexpr (KM != 3) lazy_finish<DW>(acc);
  if (!ok_all) {
    // A copy never completed: leave this warp's result out (its flag is set)
    // and wait, again bounded, for whatever this warp still has in flight.
    cp_async_wait_all();
    for (int s = 0; s < C::NS; ++s) mbar_wait(wbar + 8 * s, phase ^ (s < stage ? 1u : 0u), p.wait_polls);
    acc.m0 = acc.m1 = -CUDART_INF_F;
    acc.l0 = acc.l1 = 0.f;
  }

  // speculative copies past this warp's last tile (first use of their stage)
  if (spec)
    for (int j = my_tiles; j < C::NS - 1; ++j) mbar_wait(wbar + 8 * j, 0, p.wait_polls);

  // ---- merge the warps ------------------------------------------------------
#pragma unroll
  for (int o = 4; o < 32; o <<= 1) {
    acc.l0 += __shfl_xor_sync(0xffffffffu, acc.l0, o);
    acc.l1 += __shfl_xor_sync(0xffffffffu, acc.l1, o);
  }
  __syncthreads();  // every warp is done with its ring
  float* Os = reinterpret_cast<float*>(pipe);  // [NLW][8][D], already times fold
  float* ml = misc;                            // [NLW][8][2]
  // f16 offset of the decoded V (bit assembly only), times the V reference scale
  const float fold = !ok_all ? 0.f : KM == 3 ? acc.vref * (1.f / 256.f)
                                              : (VCVT ? 1.f : 256.f) * acc.vref;
#pragma unroll
  for (int jb = 0; jb < DW / 32; ++jb) {
    const int d = half * DW + 32 * jb + 2 * grp;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      *reinterpret_cast<float2*>(Os + (lw * 8 + 2 * qd) * D + d + 16 * h) =
          make_float2(acc.O[jb][h][0] * fold, acc.O[jb][h][2] * fold);
      *reinterpret_cast<float2*>(Os + (lw * 8 + 2 * qd + 1) * D + d + 16 * h) =
          make_float2(acc.O[jb][h][1] * fold, acc.O[jb][h][3] * fold);
    }
  }
  if (grp == 0 && half == 0) {  // (m, l) are the same in every warp of a stream
    ml[(lw * 8 + 2 * qd) * 2 + 0] = acc.m0;
    ml[(lw * 8 + 2 * qd) * 2 + 1] = acc.l0;
    ml[(lw * 8 + 2 * qd + 1) * 2 + 0] = acc.m1;
    ml[(lw * 8 + 2 * qd + 1) * 2 + 1] = acc.l1;
  }
  __syncthreads();

  constexpr float kLog2e = 1.4426950408889634f;
  // Partial rows of this (sequence, KV head x head group): head n's rows are
  // prow0 + n * S + s; its merge-group rows grow0 + n * NG + g; its tickets
  // ucnt[0 .. NG] (NG = ceil(S / 8)). Proportional splits pack the units of
  // sequence b after those of the sequences before it.
  const int NG = (S + kMergeFan - 1) / kMergeFan;
  const int HX = gridDim.x;
  int64_t prow0, grow0, cnt0;
  if (p.prop) {
    prow0 = ((int64_t)sp_b * HX + (int64_t)blockIdx.x * S) * kHeadsPerGroup;
    grow0 = ((int64_t)gp_b * HX + (int64_t)blockIdx.x * NG) * kHeadsPerGroup;
    cnt0 = (int64_t)(b + gp_b) * HX + (int64_t)blockIdx.x * (1 + NG);
  } else {
    prow0 = ((int64_t)b * p.Hq + head0) * S;
    grow0 = ((int64_t)b * p.Hq + head0) * NG;
    cnt0 = ((int64_t)b * HX + blockIdx.x) * (1 + NG);
  }
  for (int it = tid; it < 8 * (D / 4); it += C::NT) {
    const int n = it / (D / 4);
    const int d = (it - n * (D / 4)) * 4;
    if (n >= nheads) continue;
    float M = -CUDART_INF_F;
#pragma unroll
    for (int w = 0; w < C::NLW; ++w) M = fmaxf(M, ml[(w * 8 + n) * 2]);
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    float l = 0.f;
    if (M != -CUDART_INF_F) {
#pragma unroll
      for (int w = 0; w < C::NLW; ++w) {
        const float mw = ml[(w * 8 + n) * 2];
        const float f = (mw == -CUDART_INF_F) ? 0.f : fast_exp2(mw - M);
        const float4 o = *reinterpret_cast<const float4*>(Os + (w * 8 + n) * D + d);
        acc.x += f * o.x;
        acc.y += f * o.y;
        acc.z += f * o.z;
        acc.w += f * o.w;
        l += f * ml[(w * 8 + n) * 2 + 1];
      }
    }
    const int head = head0 + n;
    if (S == 1 && p.pout_o) {
      store_partial(p, b, head, d, acc, M, l);
    } else if (S == 1) {
      const float sl = p.sinks ? p.sinks[(int64_t)head * p.sinks_s] * kLog2e : -CUDART_INF_F;
      const float M2 = fmaxf(M, sl);
      float4 r = make_float4(0.f, 0.f, 0.f, 0.f);
      if (M2 != -CUDART_INF_F) {
        const float a = (M == -CUDART_INF_F) ? 0.f : fast_exp2(M - M2);
        const float den = l * a + (p.sinks ? fast_exp2(sl - M2) : 0.f);
        if (den > 0.f) {
          const float f = a / den;
          r = make_float4(acc.x * f, acc.y * f, acc.z * f, acc.w * f);
        }
      }
      *reinterpret_cast<float4*>(p.out + (int64_t)b * p.o_sb + (int64_t)head * p.o_sh + d) = r;
    } else {
      const int64_t row = prow0 + (int64_t)n * S + split;
      *reinterpret_cast<float4*>(p.part_o + row * D + d) = acc;
      if (d == 0) *reinterpret_cast<float2*>(p.part_ml + row * 2) = make_float2(M, l);
    }
  }
  if (S == 1) return;

  // ---- two-level merge by the last blocks to finish --------------------------
  // Splits form groups of kMergeFan. Every block publishes its partial, then
  // takes a ticket of its group; the block drawing the group's last ticket
  // merges the group (or, with a single group, produces the output). With
  // several groups, each group merger then takes a ticket of the (sequence,
  // KV head, head group) and the last one merges the group partials, adding
  // the sink once. Mergers reset their counters; no block ever waits. One
  // thread fences after the barrier: the barrier orders the block's partial
  // writes before its fence, and the fence orders them before the ticket.
  __syncthreads();
  int* flag = reinterpret_cast<int*>(misc + C::NW * 8 * 2);
  int* ucnt = p.counters + cnt0;
  const int g = split / kMergeFan;
  const int gsize = min(kMergeFan, S - g * kMergeFan);
  if (tid == 0) {
    __threadfence();
    *flag = (atomicAdd(ucnt + 1 + g, 1) == gsize - 1);
  }
  __syncthreads();
  if (!*flag) return;
  __threadfence();
  float* wts = reinterpret_cast<float*>(pipe);  // [8][32] merge weights
  // partial-output mode: the final merges write (O, m, l) rows, no sink
  const bool fin = p.pout_o == nullptr;
  float* fml = fin ? nullptr : p.pout_ml;
  float* fo = fin ? nullptr : p.pout_o;
  const int64_t frow = (int64_t)b * p.Hq + head0;
  if (NG == 1) {
    merge_partials<D, C::NW>(p.part_ml, p.part_o, prow0, S, S, nheads, fin, p, b, head0,
                             fml, fo, frow, 1, wts);
    if (tid == 0) ucnt[1] = 0;
    return;
  }
  merge_partials<D, C::NW>(p.part_ml, p.part_o, prow0 + g * kMergeFan, S, gsize, nheads, false,
                           p, b, head0, p.grp_ml, p.grp_o, grow0 + g, NG, wts);
  if (tid == 0) ucnt[1 + g] = 0;
  __syncthreads();
  if (tid == 0) {
    __threadfence();
    *flag = (atomicAdd(ucnt, 1) == NG - 1);
  }
  __syncthreads();
  if (!*flag) return;
  __threadfence();
  merge_partials<D, C::NW>(p.grp_ml, p.grp_o, grow0, NG, NG, nheads, fin, p, b, head0,
                           fml, fo, frow, 1, wts);
  if (tid == 0) ucnt[0] = 0;
}

// ---------------------------------------------------------------------------
// Tensor-memory split kernel (tcgen05). The same splits, plans, masking,
// fused append and split merge as the kernel above, with the attention of
// each 128-token chunk on the 5th-generation tensor cores:
//   S = K q'^T   kind::f8f6f4, M = 128 tokens, N = 16 (8 query heads x the two
//                E4M3 terms of q'), K's E4M3 bytes straight from the TMA tile;
//   O^T += V^T P kind::f16, M = D, N = 16 (8 heads x the f16 hi + lo terms of
//                P), V decoded once to f16 in shared memory.
// Both accumulators live in tensor memory. Two warpgroups of four warps take
// alternate chunks (group g the chunks c = g mod 2), each with its own S, P,
// f16 V buffer, O accumulator and online-softmax state, merged at the end.
// Warp w of a group owns tokens 32w .. 32w+31 of its chunks (its TMEM lane
// quarter): it reads S, runs the softmax (one token per thread, the 8 heads in
// registers), writes P and the decoded V rows, and copies its own two tiles of
// each chunk (lanes 0-3: K and V of tiles 2w, 2w+1, on its own barrier),
// refilling them once it has decoded their V rows. Warp 8 issues the MMAs and
// their commits from one lane. Every wait is bounded.
// ---------------------------------------------------------------------------

#ifndef FP8PD_UNS_D64
#define FP8PD_UNS_D64 10
#endif
#ifndef FP8PD_UNS_D128
#define FP8PD_UNS_D128 4
#endif

template <int D>
struct UCfg {
  static_assert(D == 64 || D == 128, "tensor-memory kernel: D = 64 or 128");
  static constexpr int NS = (D == 64) ? FP8PD_UNS_D64 : FP8PD_UNS_D128;  // K/V ring stages
  static_assert(NS % 2 == 0 && NS >= 2, "a stage keeps its warpgroup: an even ring");
  static constexpr int NWG = 2;                      // warpgroups (alternate chunks)
  static constexpr int NCW = 4 * NWG;                // compute warps
  static constexpr int NT = (NCW + 2) * 32;          // + the QK and PV MMA warps
  static constexpr int CHUNK = 128;                  // tokens per chunk (MMA M of QK)
  static constexpr int KV = CHUNK * D;               // K (or V) bytes of a chunk
  static constexpr int STAGE = 2 * KV;
  static constexpr int RING = NS * STAGE;
  static constexpr int VF16 = CHUNK * D * 2;         // V of a chunk as f16 (one per group)
  static constexpr int PBUF = CHUNK * 32;            // P of a chunk: 16 f16 per token (one per group)
  static constexpr int QT = 16 * D;                  // q' as 16 rows of E4M3 (8 heads x 2 terms)
  static constexpr int LIST = kMaxSplitTiles * 12;   // per tile: entry, k scale, v scale
  static constexpr int NBAR = 5 * NS + 5;            // full[NS][4], sbar[2], pready[NS], pvbar[2], patched
  static constexpr int MISC = 256;                   // floats
  static constexpr int SMEM = 1024 + RING + NWG * (VF16 + PBUF) + QT + LIST + NBAR * 8 + MISC * 4;
  static constexpr int MIN_BLOCKS = 1;
  static constexpr uint32_t TMEM_COLS = 64;          // S[g] at 16 g, O[g] at 32 + 16 g
  static constexpr uint32_t SWZ = (D == 128) ? 2u : 4u;  // descriptor layout: 128-byte / 64-byte swizzle
  static_assert(RING % 1024 == 0 && VF16 % 1024 == 0 && PBUF % 1024 == 0 && QT % 1024 == 0,
                "1024-byte aligned operand buffers");
  static_assert(NWG * (8 * D + 16) * 4 <= 16384 && 16384 + 8 * 32 * 4 <= RING,
                "epilogue scratch and merge weights fit in the ring");
};

// byte offsets (all >> 4), version 1, layout type (swizzle) in bits 61-63.
__device__ __forceinline__ uint64_t umma_sdesc(uint32_t addr, uint32_t lbo, uint32_t sbo,
                                               uint32_t layout) {
  return static_cast<uint64_t>((addr >> 4) & 0x3FFFu) |
         (static_cast<uint64_t>((lbo >> 4) & 0x3FFFu) << 16) |
         (static_cast<uint64_t>((sbo >> 4) & 0x3FFFu) << 32) | (static_cast<uint64_t>(1) << 46) |
         (static_cast<uint64_t>(layout) << 61);
}

__device__ __forceinline__ void umma_f8f6f4(uint32_t tmem_d, uint64_t da, uint64_t db,
                                            uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n.reg .pred p;\nsetp.ne.b32 p, %4, 0;\n"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, {%5, %5, %5, %5}, p;\n}\n" ::"r"(
          tmem_d),
      "l"(da), "l"(db), "r"(idesc), "r"(accumulate), "r"(0u)
      : "memory");
}
__device__ __forceinline__ void umma_f16(uint32_t tmem_d, uint64_t da, uint64_t db, uint32_t idesc,
                                         uint32_t accumulate) {
  asm volatile(
      "{\n.reg .pred p;\nsetp.ne.b32 p, %4, 0;\n"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, {%5, %5, %5, %5}, p;\n}\n" ::"r"(
          tmem_d),
      "l"(da), "l"(db), "r"(idesc), "r"(accumulate), "r"(0u)
      : "memory");
}
// Arrives on the barrier once every MMA this thread issued so far has completed.
__device__ __forceinline__ void umma_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n" ::"r"(
                   bar)
               : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;\n" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;\n" ::: "memory");
}
// 16 consecutive 32-bit columns of this thread's TMEM lane.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, "
      "%12, %13, %14, %15}, [%16];\n"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;\n" ::: "memory");
}
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
      "%11, %12, %13, %14, %15, %16};\n" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
  asm volatile("tcgen05.wait::st.sync.aligned;\n" ::: "memory");
}
// Waits for phase `parity` of the barrier with short polls (no suspend hint:
// a hand-off between warps is seen within the hardware's own short limit),
// giving up after polls * 20 us of global time (the same bound as mbar_wait).
__device__ __forceinline__ bool mbar_wait_poll(uint32_t bar, uint32_t parity, int polls) {
  uint64_t t0;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t0));
  const uint64_t limit = static_cast<uint64_t>(polls) * 20000u;
#pragma unroll 1
  for (;;) {
    uint32_t ok;
    asm volatile(
        "{\n.reg .pred p;\nmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
        "selp.u32 %0, 1, 0, p;\n}\n"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    if (ok) return true;
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    if (t - t0 > limit) return false;
  }
}

__device__ __forceinline__ void named_sync(int id, int threads) {
  asm volatile("bar.sync %0, %1;\n" ::"r"(id), "r"(threads) : "memory");
}


template <int D>
__global__ void __launch_bounds__(UCfg<D>::NT, UCfg<D>::MIN_BLOCKS)
    decode_umma_kernel(const DecodeParams p, const __grid_constant__ CUtensorMap tmk,
                       const __grid_constant__ CUtensorMap tmv) {
  using C = UCfg<D>;
  constexpr float kLog2e = 1.4426950408889634f;
  constexpr unsigned FULL = 0xffffffffu;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
  const uint32_t s_ring = smem_u32(smem);
  const uint32_t s_vf = s_ring + C::RING;            // [group] f16 V
  const uint32_t s_p = s_vf + C::NWG * C::VF16;      // [group] P
  const uint32_t s_q = s_p + C::NWG * C::PBUF;
  int32_t* l_ent = reinterpret_cast<int32_t*>(smem + C::RING + C::NWG * (C::VF16 + C::PBUF) + C::QT);
  float* l_ks = reinterpret_cast<float*>(l_ent + kMaxSplitTiles);
  float* l_vs = l_ks + kMaxSplitTiles;
  uint64_t* bars = reinterpret_cast<uint64_t*>(l_vs + kMaxSplitTiles);
  float* misc = reinterpret_cast<float*>(bars + C::NBAR);
  const uint32_t b_full = smem_u32(bars), b_s = b_full + 32 * C::NS, b_pr = b_s + 16,
                 b_pv = b_pr + 8 * C::NS, b_patch = b_pv + 16;
  // misc: [0] TMEM base, [1] abort, [2..4) vote words (per group), [8..72)
  // per-warp head maxima, [72..80) per-warp |v scale| maxima, [80..144) per-warp
  // l sums, [144..160) q maximum exchange
  uint32_t* m_tmem = reinterpret_cast<uint32_t*>(misc);
  volatile int* m_abort = reinterpret_cast<volatile int*>(misc + 1);
  volatile uint32_t* m_vote = reinterpret_cast<volatile uint32_t*>(misc + 2);
  float* m_hmax = misc + 8;
  float* m_vmax = misc + 72;
  float* m_lsum = misc + 80;
  float* m_qmax = misc + 144;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int kvh = blockIdx.x / p.head_groups;
  const int hg = blockIdx.x - kvh * p.head_groups;
  const int head0 = kvh * p.G + hg * 8;
  const int nheads = min(8, p.G - hg * 8);

  int b, split, S;
  int prop_j0 = 0, prop_j1 = 0, sp_b = 0, gp_b = 0;
  if (p.prop) {
    if (!prop_assign<C::NCW + 2>(p, reinterpret_cast<int*>(smem), reinterpret_cast<int*>(misc),
                                 head0, nheads, b, split, S, prop_j0, prop_j1, sp_b, gp_b))
      return;
  } else {
    b = blockIdx.y;
    split = blockIdx.z;
    S = p.num_splits;
  }
  const int L = attended_keys(p, b, tid == 0 && split == 0 && blockIdx.x == 0);
  int lo, hi;
  key_range(p, b, L, lo, hi);
  int t0, t1;
  if (p.prop) {
    t0 = max(lo, (lo / kTileTokens + prop_j0) * kTileTokens);
    t1 = min(hi, (lo / kTileTokens + prop_j1) * kTileTokens);
  } else {
    const int first_page = lo / p.ps;
    const int n_pages = (hi > lo) ? (hi - 1) / p.ps - first_page + 1 : 0;
    const int pg0 = first_page + split * p.chunk_pages;
    const int pg1 = min(first_page + n_pages, pg0 + p.chunk_pages);
    t0 = max(lo, pg0 * p.ps);
    t1 = min(hi, pg1 * p.ps);
  }
  const int tile_first = t0 / kTileTokens;
  int n_tiles = (t1 > t0) ? (t1 + kTileTokens - 1) / kTileTokens - tile_first : 0;
  if (n_tiles > kMaxSplitTiles) {
    if (tid == 0) raise_flag(FP8PD_FLAG_INTERNAL);
    n_tiles = 0;
  }
  const int nch = (n_tiles + 7) / 8;

  // ---- tile list (entry = page << 4 | tile in page, -1 = outside the pool), scales
  const int32_t* trow = p.table + (int64_t)b * p.tab_sb;
  const float* ksbase = p.ks + (int64_t)kvh * p.ks_sh;
  const float* vsbase = p.vs + (int64_t)kvh * p.vs_sh;
  for (int j = tid; j < n_tiles; j += C::NT) {
    const int tok = (tile_first + j) * kTileTokens;
    const int lp = tok / p.ps;
    const int page = __ldg(trow + (int64_t)lp * p.tab_sp);
    int e = -1;
    float ks = 0.f, vs = 0.f;
    if ((unsigned)page < (unsigned)p.num_pages) {
      e = (page << 4) | ((tok - lp * p.ps) / kTileTokens);
      ks = __ldg(ksbase + (int64_t)page * p.ks_sp);
      vs = __ldg(vsbase + (int64_t)page * p.vs_sp);
    } else if (hg == 0) {
      raise_flag(FP8PD_FLAG_PAGE_OOB);
    }
    l_ent[j] = e;
    l_ks[j] = ks;
    l_vs[j] = vs;
  }
  if (tid == 0) {
    for (int i = 0; i < 4 * C::NS; ++i) mbar_init(b_full + 8 * i, 1);
    for (int s = 0; s < C::NS; ++s) mbar_init(b_pr + 8 * s, 4 * 32);
    for (int i = 0; i < 2; ++i) {
      mbar_init(b_s + 8 * i, 1);
      mbar_init(b_pv + 8 * i, 1);
    }
    mbar_init(b_patch, 1);
    *m_abort = 0;
    m_vote[0] = m_vote[1] = 0u;
    fence_barrier_init();
  }
  if (warp == C::NCW) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;\n" ::"r"(
                     smem_u32(m_tmem)),
                 "r"(C::TMEM_COLS)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;\n" ::: "memory");
  }
  // the new token (fused append): its tile and chunk in this block's range
  int j_new = -1;
  if (p.append && L - 1 >= t0 && L - 1 < t1) j_new = (L - 1) / kTileTokens - tile_first;
  const int c_new = j_new >= 0 ? j_new / 8 : -1;

  // ---- q' = q * 2^(8 - e) (max |q'| in [2^7, 2^8)) as two E4M3 terms, rows
  // n (hi of head n) and 8 + n (lo), K-major with the tiles' swizzle
  constexpr int QITEMS = 8 * (D / 16);
  float qv[16];
  int q_n = -1, q_c = 0;
  float qm = 0.f;
  if (tid < QITEMS) {
    q_n = tid / (D / 16);
    q_c = tid - q_n * (D / 16);
    const bool ok = q_n < nheads;
    const uint16_t* qrow = p.q + (int64_t)b * p.q_sb + (int64_t)(head0 + (ok ? q_n : 0)) * p.q_sh;
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      qv[i] = ok ? bf16_bits_to_float(__ldg(qrow + (int64_t)(16 * q_c + i) * p.q_sd)) : 0.f;
      qm = fmaxf(qm, fabsf(qv[i]));
    }
  }
  qm = warp_max(qm);
  if (lane == 0) m_qmax[warp] = qm;
  __syncthreads();
  qm = 0.f;
#pragma unroll
  for (int w = 0; w < C::NCW + 2; ++w) qm = fmaxf(qm, m_qmax[w]);
  int qe = 0;
  if (qm > 0.f && isfinite(qm)) frexpf(qm, &qe);
  qe = max(qe, -111);
  const float qmul = ldexpf(1.f, 8 - qe);
  const float score_base = p.sm_scale_log2 / qmul;
  if (tid < QITEMS) {
    uint32_t h4[4], l4[4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
      e4m3_split4(qv[4 * i] * qmul, qv[4 * i + 1] * qmul, qv[4 * i + 2] * qmul,
                  qv[4 * i + 3] * qmul, h4[i], l4[i]);
    const uint32_t ah = s_q + tile_off<D>(q_n, 16 * q_c), al = s_q + tile_off<D>(8 + q_n, 16 * q_c);
    asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(ah), "r"(h4[0]), "r"(h4[1]),
                 "r"(h4[2]), "r"(h4[3]) : "memory");
    asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(al), "r"(l4[0]), "r"(l4[1]),
                 "r"(l4[2]), "r"(l4[3]) : "memory");
  }
  fence_proxy_async();  // q' (and later P, V) reach the tensor core through the async proxy
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *m_tmem;
  // S of group g at columns 16 g, O of group g at 32 + 16 g
  constexpr uint32_t IDESC_QK = (1u << 4) | (2u << 17) | (8u << 24);  // f32 += e4m3 x e4m3, M 128, N 16
  constexpr uint32_t IDESC_PV = (1u << 4) | (1u << 15) | (1u << 16) | (2u << 17) |
                                (static_cast<uint32_t>(D >> 4) << 24);  // f32 += f16 x f16, MN-major
  const int polls = p.wait_polls;
  bool failed = false;
  // A wait that gives up marks the warp failed (warp-uniform); the warp then
  // skips its later waits but still walks every chunk and named barrier, so no
  // other warp blocks on it, and the block's result is zero.
  auto wait = [&](uint32_t bar, uint32_t parity) -> bool {
    if (failed) return false;
    const bool ok = __all_sync(FULL, mbar_wait_poll(bar, parity, polls) && !*m_abort);
    if (!ok) {
      failed = true;
      if (lane == 0) {
        raise_flag(FP8PD_FLAG_TIMEOUT);
        *m_abort = 1;
      }
    }
    return ok;
  };
  // warp q of group c % 2 copies tiles 2q, 2q+1 of chunk c (K and V); they land
  // on full(c % NS, q). The group releases stage c % NS on pready(c % NS).
  auto full_bar = [&](int c, int q) { return b_full + 8 * ((c % C::NS) * 4 + q); };
  auto pready_bar = [&](int c) { return b_pr + 8 * (c % C::NS); };

  if (warp == C::NCW) {
    // ======================= QK warp (one lane issues) =======================
    for (int c = 0; c < nch && !failed; ++c) {
      const int s = c % C::NS;
      bool ok = true;
      for (int q = 0; q < 4 && ok; ++q) ok = wait(full_bar(c, q), (c / C::NS) & 1);
      if (!ok) break;
      if (c == c_new && !wait(b_patch, 0)) break;
      if (c >= 2 && !wait(pready_bar(c - 2), ((c - 2) / C::NS) & 1)) break;  // S[c & 1] read
      tc_fence_after();
      if (lane == 0) {
        const uint32_t ka = s_ring + s * C::STAGE;
#pragma unroll
        for (int kc = 0; kc < D / 32; ++kc) {
          const uint64_t da = umma_sdesc(ka + 32 * kc, 16, 8 * D, C::SWZ);
          const uint64_t db = umma_sdesc(s_q + 32 * kc, 16, 8 * D, C::SWZ);
          umma_f8f6f4(tmem + 16 * (c & 1), da, db, IDESC_QK, kc > 0 ? 1u : 0u);
        }
        umma_commit(b_s + 8 * (c & 1));
      }
      __syncwarp();
    }
  } else if (warp == C::NCW + 1) {
    // ======================= PV warp (one lane issues) =======================
    int pv_done = 0;  // chunks whose PV MMAs were issued
    for (int c = 0; c < nch && !failed; ++c) {
      if (!wait(pready_bar(c), (c / C::NS) & 1)) break;
      tc_fence_after();
      if (lane == 0) {
        const uint32_t vb = s_vf + (c & 1) * C::VF16, pb = s_p + (c & 1) * C::PBUF;
        for (int kk = 0; kk < C::CHUNK / 16; ++kk) {
          const uint64_t da = umma_sdesc(vb + kk * 2048, 16384, 1024, 2);
          const uint64_t db = umma_sdesc(pb + kk * 512, 4096, 256, 6);
          umma_f16(tmem + 32 + 16 * (c & 1), da, db, IDESC_PV, (c > 1 || kk > 0) ? 1u : 0u);
        }
        umma_commit(b_pv + 8 * (c & 1));
      }
      __syncwarp();
      pv_done = c + 1;
    }
    // drain: every committed MMA has finished before the block moves on
    for (int c = max(0, pv_done - 2); c < pv_done; ++c)
      mbar_wait(b_pv + 8 * (c & 1), (c >> 1) & 1, polls);
  } else {
    // ======================= compute warpgroups =======================
    const int g = warp >> 2, wq = warp & 3;
    const int t = tid & 127;  // token row of the group's chunks, and TMEM lane
    const uint32_t lane_base = static_cast<uint32_t>(32 * wq) << 16;
    const uint32_t t_s = tmem + lane_base + 16 * g, t_o = tmem + lane_base + 32 + 16 * g;
    const uint32_t vbuf = s_vf + g * C::VF16, pbuf = s_p + g * C::PBUF;
    float m[8], l[8], x[8];
#pragma unroll
    for (int h = 0; h < 8; ++h) {
      m[h] = -CUDART_INF_F;
      l[h] = 0.f;
      x[h] = -CUDART_INF_F;
    }
    float vref = 0.f, inv_vref = 0.f;
    const int kt = t >> 4, r = t & 15;  // tile of the chunk, row of the tile
    int issued = -1;  // the last chunk this warp issued copies for
    auto issue_part = [&](int c) {
      const int s = c % C::NS;
      const int k = 2 * wq + ((lane >> 1) & 1);
      const int j = 8 * c + k;
      const int e = (lane < 4 && j < n_tiles) ? l_ent[j] : -1;
      const int tiles = __popc(__ballot_sync(FULL, e >= 0 && (lane & 1) == 0));
      const uint32_t bar = full_bar(c, wq);
      if (lane == 0) {
        fence_proxy_async();  // this warp's reads of the stage come first
        if (tiles) mbar_arrive_expect_tx(bar, static_cast<uint32_t>(tiles) * 2u * kTileTokens * D);
        else mbar_arrive(bar);  // nothing to copy: the phase completes empty
      }
      __syncwarp();
      if (e >= 0) {
        const uint32_t dst = s_ring + s * C::STAGE + ((lane & 1) ? C::KV : 0) + k * kTileTokens * D;
        tma_load_5d(dst, (lane & 1) ? &tmv : &tmk, bar, 0, (e & 15) * kTileTokens, 0, kvh, e >> 4);
      }
      issued = c;
    };
    if (lane == 0 && warp == 0) {
      prefetch_tensormap(&tmk);
      prefetch_tensormap(&tmv);
    }
    for (int c = g; c < min(C::NS, nch); c += 2) issue_part(c);
    int last = -1;  // this group's last chunk
    for (int c = g; c < nch; c += 2) {
      last = c;
      const int s = c % C::NS;
      const uint32_t sk = s_ring + s * C::STAGE, sv = sk + C::KV;
      const int j = 8 * c + kt;
      const int e = j < n_tiles ? l_ent[j] : -1;
      const int tok = (tile_first + j) * kTileTokens + r;
      const bool valid = e >= 0 && tok >= t0 && tok < t1;
      const float ks = e >= 0 ? l_ks[j] : 0.f, vs = e >= 0 ? l_vs[j] : 0.f;
      if (c == c_new && wq == (j_new % 8) >> 1) {
        // the new token: quantized with its page's scales, stored by head
        // group 0, patched into the chunk before the QK MMA reads it
        if (wait(full_bar(c, wq), (c / C::NS) & 1)) {
          const int en = l_ent[j_new];
          if (en >= 0) {
            float kss = l_ks[j_new], vss = l_vs[j_new];
            const int rn = (L - 1) - (tile_first + j_new) * kTileTokens;
            append_new_token<D, false>(p, b, kvh, hg == 0, en >> 4, (en & 15) * kTileTokens + rn,
                                       rn, sk + (j_new % 8) * kTileTokens * D,
                                       sv + (j_new % 8) * kTileTokens * D, kss, vss);
          }
          fence_proxy_async();
          __syncwarp();
          if (lane == 0) mbar_arrive(b_patch);
        }
      }
      // this warp's tiles of the chunk have landed; the group's P and f16 V
      // buffers are free once the PV of its previous chunk has run
      wait(full_bar(c, wq), (c / C::NS) & 1);
      if (c >= 2) wait(b_pv + 8 * g, ((c - 2) >> 1) & 1);
      {
        // V row t decoded to f16, MN-major with the 128-byte swizzle: head-dim
        // entries 64a .. 64a+63 of token t in the 128-byte row t % 8 of k-group
        // t / 8 of atom a; 16-byte chunk q of that row at q ^ (t % 8)
        const uint32_t vrow = sv + kt * kTileTokens * D;
#pragma unroll
        for (int cb = 0; cb < D / 16; ++cb) {
          uint4 w = make_uint4(0u, 0u, 0u, 0u);
          if (valid) {
            const uint32_t a = vrow + tile_off<D>(r, 16 * cb);
            asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                         : "=r"(w.x), "=r"(w.y), "=r"(w.z), "=r"(w.w) : "r"(a));
          }
          const uint32_t f[8] = {e4m3x2_lo16_to_f16x2(w.x), e4m3x2_hi16_to_f16x2(w.x),
                                 e4m3x2_lo16_to_f16x2(w.y), e4m3x2_hi16_to_f16x2(w.y),
                                 e4m3x2_lo16_to_f16x2(w.z), e4m3x2_hi16_to_f16x2(w.z),
                                 e4m3x2_lo16_to_f16x2(w.w), e4m3x2_hi16_to_f16x2(w.w)};
#pragma unroll
          for (int u = 0; u < 2; ++u) {
            const int d0 = 16 * cb + 8 * u;
            const int atom = d0 >> 6, q = (d0 & 63) >> 3;
            const uint32_t dst = vbuf + atom * 16384 + (t >> 3) * 1024 + (t & 7) * 128 +
                                 ((q ^ (t & 7)) << 4);
            asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(dst), "r"(f[4 * u]),
                         "r"(f[4 * u + 1]), "r"(f[4 * u + 2]), "r"(f[4 * u + 3]) : "memory");
          }
        }
      }
      // QK of the chunk has run: its K is consumed and this warp's V rows are
      // decoded, so the warp refills its tiles of the stage right away
      wait(b_s + 8 * g, (c >> 1) & 1);
      tc_fence_after();
      fence_proxy_async();
      __syncwarp();
      if (c + C::NS < nch && !failed) issue_part(c + C::NS);
      uint32_t sr[16];
      tmem_ld16(t_s, sr);
      tc_fence_before();
      const float kf = score_base * ks;
      float sc[8];
      bool trig = valid && fabsf(vs) > vref;
#pragma unroll
      for (int h = 0; h < 8; ++h) {
        sc[h] = (valid && h < nheads)
                    ? (__uint_as_float(sr[h]) + __uint_as_float(sr[8 + h])) * kf
                    : -CUDART_INF_F;
        x[h] = fmaxf(x[h], sc[h]);
        trig = trig || (sc[h] > m[h] + kLazyLog2);
      }
      // group-wide vote on a rescale (the chunk's P share one reference per head)
      const unsigned vote = __ballot_sync(FULL, trig);
      if (lane == 0 && vote) atomicOr(const_cast<uint32_t*>(m_vote + g), 1u << wq);
      named_sync(1 + g, 128);
      const uint32_t any = m_vote[g];
      if (any) {
        float wm[8];
#pragma unroll
        for (int h = 0; h < 8; ++h) wm[h] = warp_max(sc[h]);
        const float wv = warp_max(valid ? fabsf(vs) : 0.f);
        if (lane == 0) {
#pragma unroll
          for (int h = 0; h < 8; ++h) m_hmax[warp * 8 + h] = wm[h];
          m_vmax[warp] = wv;
        }
        named_sync(1 + g, 128);
        if (t == 0) m_vote[g] = 0u;  // read by every warp of the group before this barrier
        float cf[8];
        float nv = vref;
#pragma unroll
        for (int w = 0; w < 4; ++w) nv = fmaxf(nv, m_vmax[4 * g + w]);
        const float fv = (nv > vref && vref > 0.f) ? vref / nv : 1.f;
#pragma unroll
        for (int h = 0; h < 8; ++h) {
          float nm = m[h];
#pragma unroll
          for (int w = 0; w < 4; ++w) nm = fmaxf(nm, m_hmax[(4 * g + w) * 8 + h]);
          cf[h] = (nm > m[h]) ? fast_exp2(m[h] - nm) : 1.f;
          l[h] *= cf[h];
          m[h] = nm;
        }
        if (nv > vref) {
          vref = nv;
          inv_vref = 1.f / nv;
        }
        if (c >= 2 && !failed) {
          // O holds this group's chunks < c: its last PV has run; rescale O in place
          tc_fence_after();
          uint32_t o[16];
          tmem_ld16(t_o, o);
#pragma unroll
          for (int h = 0; h < 8; ++h) {
            o[h] = __float_as_uint(__uint_as_float(o[h]) * cf[h] * fv);
            o[8 + h] = __float_as_uint(__uint_as_float(o[8 + h]) * cf[h] * fv);
          }
          tmem_st16(t_o, o);
          tc_fence_before();
        }
        named_sync(1 + g, 128);  // everyone has read the maxima before they are reused
      }
      // P = 2^(s - m) * v_scale / vref as f16 hi + lo, columns h (hi) and 8 + h (lo)
      uint32_t ph[4], pl[4];
      const float vr = vs * inv_vref;
#pragma unroll
      for (int h = 0; h < 8; h += 2) {
        const float mb0 = (m[h] == -CUDART_INF_F) ? 0.f : m[h];
        const float mb1 = (m[h + 1] == -CUDART_INF_F) ? 0.f : m[h + 1];
        const float p0 = fast_exp2(sc[h] - mb0), p1 = fast_exp2(sc[h + 1] - mb1);
        l[h] += p0;
        l[h + 1] += p1;
        const float w0 = p0 * vr, w1 = p1 * vr;
        const uint32_t hh = pack_f16x2(w0, w1);
        const float2 fh = unpack_f16x2(hh);
        ph[h >> 1] = hh;
        pl[h >> 1] = pack_f16x2(w0 - fh.x, w1 - fh.y);
      }
      {
        // P row t: 32 bytes, 32-byte swizzle (chunk ^= bit 2 of t)
        const uint32_t pr = pbuf + t * 32, sw = (t >> 2) & 1;
        asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(pr + (sw << 4)), "r"(ph[0]),
                     "r"(ph[1]), "r"(ph[2]), "r"(ph[3]) : "memory");
        asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(pr + ((sw ^ 1) << 4)),
                     "r"(pl[0]), "r"(pl[1]), "r"(pl[2]), "r"(pl[3]) : "memory");
      }
      fence_proxy_async();
      mbar_arrive(pready_bar(c));
    }
    // copies of this warp still in flight (only after a failed wait) land first
    for (int c = issued; c >= 0 && c > issued - C::NS; c -= 2)
      mbar_wait(full_bar(c, wq), (c / C::NS) & 1, polls);
    // ---- this group's (m, l, O) moved onto the exact maxima, l over its tokens
    if (last >= 0) wait(b_pv + 8 * g, (last >> 1) & 1);
    tc_fence_after();
    // the epilogue scratch overlays ring stage 0: both groups are past their
    // last chunk (and its copies and MMAs) before either writes it
    named_sync(3, C::NCW * 32);
    float* Os = reinterpret_cast<float*>(smem);  // [group][8][D] (the ring is idle now)
    float* ml = Os + C::NWG * 8 * D;             // [group][8][2]
#pragma unroll
    for (int h = 0; h < 8; ++h) {
      const float xm = warp_max(x[h]);
      if (lane == 0) m_hmax[warp * 8 + h] = xm;
      float ls = l[h];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) ls += __shfl_xor_sync(FULL, ls, o);
      if (lane == 0) m_lsum[warp * 8 + h] = ls;
    }
    named_sync(1 + g, 128);
    float fx[8];
#pragma unroll
    for (int h = 0; h < 8; ++h) {
      float xm = -CUDART_INF_F, ls = 0.f;
#pragma unroll
      for (int w = 0; w < 4; ++w) {
        xm = fmaxf(xm, m_hmax[(4 * g + w) * 8 + h]);
        ls += m_lsum[(4 * g + w) * 8 + h];
      }
      // l and O are relative to the reference m; move them onto the maximum
      fx[h] = (xm > m[h] && m[h] != -CUDART_INF_F) ? fast_exp2(m[h] - xm) : 1.f;
      if (failed || last < 0) {
        xm = -CUDART_INF_F;
        ls = 0.f;
      }
      if (t == 0) {
        ml[(g * 8 + h) * 2] = xm;
        ml[(g * 8 + h) * 2 + 1] = ls * fx[h];
      }
    }
    // O rows: D = 128, lane = head-dim entry; D = 64 (M = 64), entry 16q + i
    // sits in lane i < 16 of the warp's quarter
    const int d = (D == 128) ? t : (lane < 16 ? 16 * wq + lane : -1);
    uint32_t o[16];
    const bool have = last >= 0 && !failed;
    if (have) tmem_ld16(t_o, o);
    tc_fence_before();
    if (d >= 0) {
#pragma unroll
      for (int h = 0; h < 8; ++h)
        Os[(g * 8 + h) * D + d] =
            have ? (__uint_as_float(o[h]) + __uint_as_float(o[8 + h])) * vref * fx[h] : 0.f;
    }
  }
  __syncthreads();
  if (warp == C::NCW) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;\n" ::"r"(tmem),
                 "r"(C::TMEM_COLS)
                 : "memory");
  }

  // ---- the two groups' results merged, then published and the splits merged
  // (as the kernel above)
  float* Os = reinterpret_cast<float*>(smem);
  const float* ml = Os + C::NWG * 8 * D;
  const int NG = (S + kMergeFan - 1) / kMergeFan;
  const int HX = gridDim.x;
  int64_t prow0, grow0, cnt0;
  if (p.prop) {
    prow0 = ((int64_t)sp_b * HX + (int64_t)blockIdx.x * S) * kHeadsPerGroup;
    grow0 = ((int64_t)gp_b * HX + (int64_t)blockIdx.x * NG) * kHeadsPerGroup;
    cnt0 = (int64_t)(b + gp_b) * HX + (int64_t)blockIdx.x * (1 + NG);
  } else {
    prow0 = ((int64_t)b * p.Hq + head0) * S;
    grow0 = ((int64_t)b * p.Hq + head0) * NG;
    cnt0 = ((int64_t)b * HX + blockIdx.x) * (1 + NG);
  }
  for (int it = tid; it < 8 * (D / 4); it += C::NT) {
    const int n = it / (D / 4);
    const int dd = (it - n * (D / 4)) * 4;
    if (n >= nheads) continue;
    const float m0 = ml[(0 * 8 + n) * 2], l0 = ml[(0 * 8 + n) * 2 + 1];
    const float m1 = ml[(1 * 8 + n) * 2], l1 = ml[(1 * 8 + n) * 2 + 1];
    const float M = fmaxf(m0, m1);
    const float w0 = (m0 == -CUDART_INF_F) ? 0.f : fast_exp2(m0 - M);
    const float w1 = (m1 == -CUDART_INF_F) ? 0.f : fast_exp2(m1 - M);
    const float l = w0 * l0 + w1 * l1;
    const float4 a0 = *reinterpret_cast<const float4*>(Os + (0 * 8 + n) * D + dd);
    const float4 a1 = *reinterpret_cast<const float4*>(Os + (1 * 8 + n) * D + dd);
    const float4 acc = make_float4(w0 * a0.x + w1 * a1.x, w0 * a0.y + w1 * a1.y,
                                   w0 * a0.z + w1 * a1.z, w0 * a0.w + w1 * a1.w);
    const int head = head0 + n;
    if (S == 1 && p.pout_o) {
      store_partial(p, b, head, dd, acc, M, l);
    } else if (S == 1) {
      const float sl = p.sinks ? p.sinks[(int64_t)head * p.sinks_s] * kLog2e : -CUDART_INF_F;
      const float M2 = fmaxf(M, sl);
      float4 res = make_float4(0.f, 0.f, 0.f, 0.f);
      if (M2 != -CUDART_INF_F) {
        const float a = (M == -CUDART_INF_F) ? 0.f : fast_exp2(M - M2);
        const float den = l * a + (p.sinks ? fast_exp2(sl - M2) : 0.f);
        if (den > 0.f) {
          const float f = a / den;
          res = make_float4(acc.x * f, acc.y * f, acc.z * f, acc.w * f);
        }
      }
      *reinterpret_cast<float4*>(p.out + (int64_t)b * p.o_sb + (int64_t)head * p.o_sh + dd) = res;
    } else {
      const int64_t row = prow0 + (int64_t)n * S + split;
      *reinterpret_cast<float4*>(p.part_o + row * D + dd) = acc;
      if (dd == 0) *reinterpret_cast<float2*>(p.part_ml + row * 2) = make_float2(M, l);
    }
  }
  if (S == 1) return;
  __syncthreads();
  int* flag = reinterpret_cast<int*>(misc + 1);
  int* ucnt = p.counters + cnt0;
  const int gi = split / kMergeFan;
  const int gsize = min(kMergeFan, S - gi * kMergeFan);
  if (tid == 0) {
    __threadfence();
    *flag = (atomicAdd(ucnt + 1 + gi, 1) == gsize - 1);
  }
  __syncthreads();
  if (!*flag) return;
  __threadfence();
  float* wts = reinterpret_cast<float*>(smem + 16384);  // [8][32] merge weights
  const bool fin = p.pout_o == nullptr;
  float* fml = fin ? nullptr : p.pout_ml;
  float* fo = fin ? nullptr : p.pout_o;
  const int64_t frow = (int64_t)b * p.Hq + head0;
  if (NG == 1) {
    merge_partials<D, C::NCW + 2>(p.part_ml, p.part_o, prow0, S, S, nheads, fin, p, b, head0, fml,
                                  fo, frow, 1, wts);
    if (tid == 0) ucnt[1] = 0;
    return;
  }
  merge_partials<D, C::NCW + 2>(p.part_ml, p.part_o, prow0 + gi * kMergeFan, S, gsize, nheads,
                                false, p, b, head0, p.grp_ml, p.grp_o, grow0 + gi, NG, wts);
  if (tid == 0) ucnt[1 + gi] = 0;
  __syncthreads();
  if (tid == 0) {
    __threadfence();
    *flag = (atomicAdd(ucnt, 1) == NG - 1);
  }
  __syncthreads();
  if (!*flag) return;
  __threadfence();
  merge_partials<D, C::NCW + 2>(p.grp_ml, p.grp_o, grow0, NG, NG, nheads, fin, p, b, head0, fml,
                                fo, frow, 1, wts);
  if (tid == 0) ucnt[0] = 0;
}

// ---------------------------------------------------------------------------
// Quantize-append: one thread per (sequence, KV head, pair of head-dim
// entries), for K and V. code = E4M3_RNE_SAT(float32(x) / scale): IEEE float32
// division (__fdiv_rn), then cvt.rn.satfinite.e4m3x2.f32, which rounds to
// nearest even and saturates to +-448 (NaN stays NaN).
// ---------------------------------------------------------------------------

// Per-token-per-head scale of one bf16 row of n values (stride sd): max |x| /
// 448 in IEEE f32, NaN entries skipped (fmaxf), 1 for an all-zero row.
__device__ float row_amax(const uint16_t* x, int64_t sd, int n) {
  float m = 0.f;
  for (int i = 0; i < n; ++i) m = fmaxf(m, fabsf(bf16_bits_to_float(x[(int64_t)i * sd])));
  return m;
}
__device__ float row_token_scale(const uint16_t* x, int64_t sd, int n) {
  const float m = row_amax(x, sd, n);
  return m == 0.f ? 1.f : __fdiv_rn(m, 448.f);
}

__global__ void __launch_bounds__(256) append_kernel(const AppendParams p) {
  const int npair = (p.D + 1) / 2;
  const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const int64_t total = (int64_t)p.B * p.Hkv * npair;
  if (idx >= total) return;
  const int b = static_cast<int>(idx / ((int64_t)p.Hkv * npair));
  const int rem = static_cast<int>(idx - (int64_t)b * p.Hkv * npair);
  const int h = rem / npair;
  const int d = (rem - h * npair) * 2;
  const int pos = p.pos[(int64_t)b * p.pos_s];
  if (pos < 0 || pos >= p.max_pages * p.ps) {
    if (h == 0 && d == 0) raise_flag(FP8PD_FLAG_POS_OOB);
    return;
  }
  const int lp = pos / p.ps;
  const int page = p.table[(int64_t)b * p.tab_sb + (int64_t)lp * p.tab_sp];
  if ((unsigned)page >= (unsigned)p.num_pages) {
    if (h == 0 && d == 0) raise_flag(FP8PD_FLAG_PAGE_OOB);
    return;
  }
  const int slot = pos - lp * p.ps;
  const bool two = d + 1 < p.D;
  const uint16_t* knr = p.kn + (int64_t)b * p.kn_sb + (int64_t)h * p.kn_sh;
  const uint16_t* vnr = p.vn + (int64_t)b * p.vn_sb + (int64_t)h * p.vn_sh;
  const int64_t kso = (int64_t)page * p.ks_sp + (int64_t)slot * p.ks_st + (int64_t)h * p.ks_sh;
  const int64_t vso = (int64_t)page * p.vs_sp + (int64_t)slot * p.vs_st + (int64_t)h * p.vs_sh;
  // A per-token scale is the new token's own: every thread of the row
  // derives it from the row's D values, the row's first thread stores it.
  float ks = 0.f, ks1 = 0.f;  // K scales of entries d and d + 1
  if (p.k_mx) {
    // MXFP8: the 32-entry block of d and d + 1 (d is even): its E8M0 code,
    // stored by the thread holding the block's first entry
    const int blk = d / 32;
    const uint32_t c = mx_code(row_amax(knr + (int64_t)blk * 32 * p.kn_sd, p.kn_sd, 32));
    ks = ks1 = e8m0_to_f32(c);
    if (d == blk * 32) reinterpret_cast<uint8_t*>(p.ksw)[kso + (int64_t)blk * p.ks_sg] = c;
  } else if (p.k_tok && p.k_groups > 1) {
    // sub-row groups of gs entries: each entry's group scale; the thread
    // holding a group's first entry stores it
    const int gs = p.D / p.k_groups;
    const int g0 = d / gs, g1 = two ? (d + 1) / gs : g0;
    ks = row_token_scale(knr + (int64_t)g0 * gs * p.kn_sd, p.kn_sd, gs);
    ks1 = g1 == g0 ? ks : row_token_scale(knr + (int64_t)g1 * gs * p.kn_sd, p.kn_sd, gs);
    if (d == g0 * gs) p.ksw[kso + (int64_t)g0 * p.ks_sg] = ks;
    if (g1 != g0 && d + 1 == g1 * gs) p.ksw[kso + (int64_t)g1 * p.ks_sg] = ks1;
  } else {
    ks = ks1 = p.k_tok ? row_token_scale(knr, p.kn_sd, p.D) : p.ks[kso];
    if (d == 0 && p.k_tok) p.ksw[kso] = ks;
  }
  float vs;
  if (p.v_mx) {
    const int blk = d / 32;
    const uint32_t c = mx_code(row_amax(vnr + (int64_t)blk * 32 * p.vn_sd, p.vn_sd, 32));
    vs = e8m0_to_f32(c);
    if (d == blk * 32) reinterpret_cast<uint8_t*>(p.vsw)[vso + (int64_t)blk * p.vs_sg] = c;
  } else {
    vs = p.v_tok ? row_token_scale(vnr, p.vn_sd, p.D) : p.vs[vso];
    if (d == 0 && p.v_tok) p.vsw[vso] = vs;
  }
  const uint16_t* kn = knr + (int64_t)d * p.kn_sd;
  const uint16_t* vn = vnr + (int64_t)d * p.vn_sd;
  const float k0 = __fdiv_rn(bf16_bits_to_float(kn[0]), ks);
  const float k1 = two ? __fdiv_rn(bf16_bits_to_float(kn[p.kn_sd]), ks1) : 0.f;
  const float v0 = __fdiv_rn(bf16_bits_to_float(vn[0]), vs);
  const float v1 = two ? __fdiv_rn(bf16_bits_to_float(vn[p.vn_sd]), vs) : 0.f;
  const uint16_t kc = e4m3x2_rn_sat(k0, k1);
  const uint16_t vc = e4m3x2_rn_sat(v0, v1);
  uint8_t* kd = p.k + (int64_t)page * p.k_sp + (int64_t)slot * p.k_st + (int64_t)h * p.k_sh + d;
  uint8_t* vd = p.v + (int64_t)page * p.v_sp + (int64_t)slot * p.v_st + (int64_t)h * p.v_sh + d;
  kd[0] = static_cast<uint8_t>(kc & 0xFF);
  vd[0] = static_cast<uint8_t>(vc & 0xFF);
  if (two) {
    kd[1] = static_cast<uint8_t>(kc >> 8);
    vd[1] = static_cast<uint8_t>(vc >> 8);
  }
}

// ---------------------------------------------------------------------------
// Launchers
// ---------------------------------------------------------------------------
template <int D, int KM, bool VCVT, int SC, int DS = 1>
static cudaError_t launch_decode_d(const DecodeParams& p, const CUtensorMap& tmk,
                                   const CUtensorMap& tmv, cudaStream_t s) {
  // The shared-memory opt-in is a per-device function attribute: set it once
  // per device (an idempotent call, so a race only repeats it).
  static std::atomic<uint64_t> configured{0};
  const int smem = Cfg<D, DS>::SMEM;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const uint64_t bit = (dev >= 0 && dev < 64) ? (uint64_t(1) << dev) : 0;
  if (!bit || !(configured.load() & bit)) {
    e = cudaFuncSetAttribute(decode_tma_kernel<D, KM, VCVT, SC, DS>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    configured.fetch_or(bit);
  }
  const dim3 grid = p.prop ? dim3(p.Hkv * p.head_groups, p.nbx, 1)
                           : dim3(p.Hkv * p.head_groups, p.B, p.num_splits);
  decode_tma_kernel<D, KM, VCVT, SC, DS><<<grid, Cfg<D, DS>::NT, smem, s>>>(p, tmk, tmv);
  return cudaGetLastError();
}

// K mode 2 (E4M3 MMAs) is built with the cvt decode of V and without
// per-token scales; other combinations take mode 1 for K. Mode 3 is the fp8
// compute path (V is not decoded), page and head scales only. SC: 0 = page
// or head scales, 1 = per-token scales (K sub-row groups, MXFP8 K), 2 = MXFP8
// V (built with the cvt decodes only).
template <int D, int SC>
static cudaError_t launch_decode_kv(const DecodeParams& p, const CUtensorMap& tmk,
                                    const CUtensorMap& tmv, int k_mode, bool v_cvt,
                                    cudaStream_t s) {
  if constexpr (SC == 2) {
    if (k_mode == 3) return cudaErrorInvalidValue;  // refused by the host first
    return launch_decode_d<D, 1, true, 2>(p, tmk, tmv, s);
  } else {
    if constexpr (SC == 0) {
      if constexpr (D == 512 && FP8PD_DSPLIT_D512 > 1) {
        // the head-dim split (the host chose it and built part-width tensor maps)
        if (p.dsplit > 1) {
          if (p.dsplit != FP8PD_DSPLIT_D512 || k_mode != 1 || !v_cvt) return cudaErrorInvalidValue;
          return launch_decode_d<D, 1, true, 0, FP8PD_DSPLIT_D512>(p, tmk, tmv, s);
        }
      }
      if (k_mode == 3) return launch_decode_d<D, 3, true, 0>(p, tmk, tmv, s);
      if (k_mode == 2 && v_cvt) return launch_decode_d<D, 2, true, 0>(p, tmk, tmv, s);
    } else {
      if (k_mode == 3) return cudaErrorInvalidValue;  // refused by the host first
    }
    if (k_mode >= 1)
      return v_cvt ? launch_decode_d<D, 1, true, SC>(p, tmk, tmv, s)
                   : launch_decode_d<D, 1, false, SC>(p, tmk, tmv, s);
    return v_cvt ? launch_decode_d<D, 0, true, SC>(p, tmk, tmv, s)
                 : launch_decode_d<D, 0, false, SC>(p, tmk, tmv, s);
  }
}

template <int D>
static cudaError_t launch_decode_umma(const DecodeParams& p, const CUtensorMap& tmk,
                                      const CUtensorMap& tmv, cudaStream_t s) {
  static std::atomic<uint64_t> configured{0};
  const int smem = UCfg<D>::SMEM;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const uint64_t bit = (dev >= 0 && dev < 64) ? (uint64_t(1) << dev) : 0;
  if (!bit || !(configured.load() & bit)) {
    e = cudaFuncSetAttribute(decode_umma_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             smem);
    if (e != cudaSuccess) return e;
    configured.fetch_or(bit);
  }
  const dim3 grid = p.prop ? dim3(p.Hkv * p.head_groups, p.nbx, 1)
                           : dim3(p.Hkv * p.head_groups, p.B, p.num_splits);
  decode_umma_kernel<D><<<grid, UCfg<D>::NT, smem, s>>>(p, tmk, tmv);
  return cudaGetLastError();
}

template <int D>
static cudaError_t launch_decode_dt(const DecodeParams& p, const CUtensorMap& tmk,
                                    const CUtensorMap& tmv, int k_mode, bool v_cvt,
                                    cudaStream_t s) {
  if constexpr (D == 64 || D == 128) {
    if (p.umma) return launch_decode_umma<D>(p, tmk, tmv, s);
  }
  if (p.v_mx) return launch_decode_kv<D, 2>(p, tmk, tmv, k_mode, v_cvt, s);
  if (p.k_tok || p.v_tok) return launch_decode_kv<D, 1>(p, tmk, tmv, k_mode, v_cvt, s);
  return launch_decode_kv<D, 0>(p, tmk, tmv, k_mode, v_cvt, s);
}

cudaError_t launch_decode(const DecodeParams& p, const CUtensorMap& tmk, const CUtensorMap& tmv,
                          int k_mode, bool v_cvt, cudaStream_t s) {
  switch (p.D) {
    case 64: return launch_decode_dt<64>(p, tmk, tmv, k_mode, v_cvt, s);
    case 128: return launch_decode_dt<128>(p, tmk, tmv, k_mode, v_cvt, s);
    case 256: return launch_decode_dt<256>(p, tmk, tmv, k_mode, v_cvt, s);
    case 512: return launch_decode_dt<512>(p, tmk, tmv, k_mode, v_cvt, s);
    default: return cudaErrorInvalidValue;
  }
}

template <int D, int DS = 1>
static int blocks_per_sm_d() {
  static std::atomic<int> cached{-1};
  int c = cached.load();
  if (c >= 0) return c;
  int n = 0;
  if (cudaFuncSetAttribute(decode_tma_kernel<D, 1, true, 0, DS>,
                           cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg<D, DS>::SMEM) != cudaSuccess ||
      cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, decode_tma_kernel<D, 1, true, 0, DS>,
                                                    Cfg<D, DS>::NT, Cfg<D, DS>::SMEM) != cudaSuccess) {
    cudaGetLastError();
    return Cfg<D, DS>::MIN_BLOCKS;  // no device: do not cache the guess
  }
  c = n > 0 ? n : 1;
  cached.store(c);
  return c;
}

template <int D>
static int umma_blocks_per_sm_d() {
  static std::atomic<int> cached{-1};
  int c = cached.load();
  if (c >= 0) return c;
  int n = 0;
  if (cudaFuncSetAttribute(decode_umma_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           UCfg<D>::SMEM) != cudaSuccess ||
      cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, decode_umma_kernel<D>, UCfg<D>::NT,
                                                    UCfg<D>::SMEM) != cudaSuccess) {
    cudaGetLastError();
    return UCfg<D>::MIN_BLOCKS;  // no device: do not cache the guess
  }
  c = n > 0 ? n : 1;
  cached.store(c);
  return c;
}

int decode_umma_blocks_per_sm(int D) {
  switch (D) {
    case 64: return umma_blocks_per_sm_d<64>();
    case 128: return umma_blocks_per_sm_d<128>();
    default: return 0;
  }
}

int decode_blocks_per_sm(int D, int dsplit) {
  switch (D) {
    case 64: return blocks_per_sm_d<64>();
    case 128: return blocks_per_sm_d<128>();
    case 256: return blocks_per_sm_d<256>();
    case 512: return dsplit > 1 ? blocks_per_sm_d<512, FP8PD_DSPLIT_D512>() : blocks_per_sm_d<512>();
    default: return 1;
  }
}

int decode_warps_per_block(int D, int dsplit) {
  switch (D) {
    case 64: return Cfg<64>::NW;
    case 128: return Cfg<128>::NW;
    case 256: return Cfg<256>::NW;
    case 512: return dsplit > 1 ? Cfg<512, FP8PD_DSPLIT_D512>::NW : Cfg<512>::NW;
    default: return 4;
  }
}

int decode_smem_bytes(int D, int dsplit) {
  switch (D) {
    case 64: return Cfg<64>::SMEM;
    case 128: return Cfg<128>::SMEM;
    case 256: return Cfg<256>::SMEM;
    case 512: return dsplit > 1 ? Cfg<512, FP8PD_DSPLIT_D512>::SMEM : Cfg<512>::SMEM;
    default: return 0;
  }
}

// Merge of R context-parallel partials of each (sequence, query head): with
// m_r, l_r, O_r the rank's maximum (log2 units), sum and numerator,
// M = max(max_r m_r, sink * log2 e), den = sum_r l_r 2^(m_r - M) + 2^(sink
// log2 e - M), out = sum_r O_r 2^(m_r - M) / den (0 when den is 0). One block
// of 128 threads per (sequence, query head); R <= kCombineMaxRanks.
constexpr int kCombineMaxRanks = 1024;
__global__ void __launch_bounds__(128)
    combine_kernel(const float* po, const float* pml, int R, int BH, int Hq, int D,
                   const float* sinks, int64_t sinks_s, float* out, int64_t o_sb, int64_t o_sh) {
  constexpr float kLog2e = 1.4426950408889634f;
  __shared__ float w[kCombineMaxRanks];
  __shared__ float red[2];
  const int row = blockIdx.x, b = row / Hq, h = row - b * Hq;
  const int tid = threadIdx.x, lane = tid & 31;
  if (tid < 32) {
    float M = -CUDART_INF_F;
    for (int r = lane; r < R; r += 32) M = fmaxf(M, pml[((int64_t)r * BH + row) * 2]);
    M = warp_max(M);
    const float sl = sinks ? sinks[(int64_t)h * sinks_s] * kLog2e : -CUDART_INF_F;
    const float M2 = fmaxf(M, sl);
    float den = 0.f;
    for (int r = lane; r < R; r += 32) {
      const float2 ml = *reinterpret_cast<const float2*>(pml + ((int64_t)r * BH + row) * 2);
      const float wr = (M2 == -CUDART_INF_F || ml.x == -CUDART_INF_F) ? 0.f : fast_exp2(ml.x - M2);
      w[r] = wr;
      den += wr * ml.y;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) den += __shfl_xor_sync(0xffffffffu, den, o);
    if (lane == 0) {
      if (sinks && M2 != -CUDART_INF_F) den += fast_exp2(sl - M2);
      red[0] = den > 0.f ? 1.f / den : 0.f;
    }
  }
  __syncthreads();
  const float inv = red[0];
  for (int d = tid * 4; d < D; d += 128 * 4) {
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int r = 0; r < R; ++r) {
      const float wr = w[r];
      if (wr == 0.f) continue;  // an empty or masked rank: its numerator may be anything
      const float4 v = *reinterpret_cast<const float4*>(po + ((int64_t)r * BH + row) * D + d);
      acc.x += wr * v.x;
      acc.y += wr * v.y;
      acc.z += wr * v.z;
      acc.w += wr * v.w;
    }
    *reinterpret_cast<float4*>(out + (int64_t)b * o_sb + (int64_t)h * o_sh + d) =
        make_float4(acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv);
  }
}

cudaError_t launch_combine(const float* po, const float* pml, int R, int B, int Hq, int D,
                           const float* sinks, int64_t sinks_s, float* out, int64_t o_sb,
                           int64_t o_sh, cudaStream_t s) {
  if (R < 1 || R > kCombineMaxRanks || D % 4) return cudaErrorInvalidValue;
  const int BH = B * Hq;
  if (BH == 0) return cudaSuccess;
  combine_kernel<<<BH, 128, 0, s>>>(po, pml, R, BH, Hq, D, sinks, sinks_s, out, o_sb, o_sh);
  return cudaGetLastError();
}

// E4M3 codes of n float32 values with the append's rounding
// (cvt.rn.satfinite: nearest, ties to even, +-448 for larger magnitudes and
// infinities, NaN to the NaN code with its sign); strides in elements.
__global__ void __launch_bounds__(256)
    encode_kernel(const float* x, int64_t xs, uint8_t* c, int64_t cs, int64_t n) {
  const int64_t step = (int64_t)gridDim.x * blockDim.x;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += step)
    c[i * cs] = static_cast<uint8_t>(e4m3x2_rn_sat(x[i * xs], 0.f) & 0xFFu);
}

cudaError_t launch_encode(const float* x, int64_t xs, uint8_t* c, int64_t cs, int64_t n,
                          cudaStream_t s) {
  if (n <= 0) return cudaSuccess;
  const int threads = 256;
  const int64_t want = (n + threads - 1) / threads;
  const int64_t cap = 148 * 32;  // a grid-stride loop past 32 blocks per SM
  encode_kernel<<<static_cast<unsigned>(want < cap ? want : cap), threads, 0, s>>>(x, xs, c, cs,
                                                                                   n);
  return cudaGetLastError();
}

cudaError_t launch_append(const AppendParams& p, cudaStream_t s) {
  const int64_t total = (int64_t)p.B * p.Hkv * ((p.D + 1) / 2);
  if (total == 0) return cudaSuccess;
  const int threads = 256;
  const int64_t blocks = (total + threads - 1) / threads;
  append_kernel<<<static_cast<unsigned>(blocks), threads, 0, s>>>(p);
  return cudaGetLastError();
}

}  // namespace fp8pd
