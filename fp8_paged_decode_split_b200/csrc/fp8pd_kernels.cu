// Kernels of the FP8 (E4M3) paged split-KV decode attention library, sm_100a.
//
// Method (the "FP8 paged attention for MoE serving" solution page, sections
// "Why it happens" and "Expected result"): flash-decode over a paged E4M3
// KV cache with a grid over (sequence, KV head, split), E4M3 decoded in
// registers by bit assembly, scales read at their natural shape, the query
// heads of one KV head packed so each K/V byte is read once, online softmax
// with a sliding window and sink logits, and a log-sum-exp combine of the
// splits.
//
// Design on B200:
// * One thread block = one (sequence b, KV head h, group of <= 8 query
//   heads, split of the key range). Its 4 warps take 16-token tiles of the
//   split round robin; each warp streams its tiles HBM -> shared memory with
//   16-byte cp.async into a private multi-stage ring (no block-wide barrier
//   in the main loop) and keeps its own online-softmax state. The warps are
//   merged once at the end; when the keys are split over several blocks the
//   last block of a (sequence, KV head, head group) to finish merges the
//   splits (a ticket counter, never a wait), so one launch does the call.
// * QK and PV are tensor-core contractions (mma.sync m16n8k16, f16 inputs,
//   f32 accumulate): rows = 16 tokens (QK) or 16 head-dim entries (PV),
//   columns = the 8 packed query heads. E4M3 -> f16 is exact, so K and V
//   enter the MMA without rounding; q enters exactly as f16 after a
//   power-of-two rescale; P enters as an f16 hi + lo pair (two MMAs), which
//   keeps it to about 22 significant bits.
// * The MMA k index may map to any head-dim (QK) or token (PV) order as
//   long as both operands agree; the orders below are chosen so that every
//   operand word comes from one 32-bit shared-memory word or one byte
//   permute, and the shared-memory layouts are XOR-swizzled so that those
//   loads are free of bank conflicts.

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

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;\n" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;\n" ::"n"(N) : "memory");
}

__device__ __forceinline__ uint4 lds128(uint32_t a) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(a));
  return v;
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

// ---------------------------------------------------------------------------
// Tile layouts in shared memory: a 16-token K (or V) tile of one KV head is
// 16 rows of D bytes, stored in 16-byte chunks with an XOR swizzle on the
// chunk index inside each 128-byte line.
//  K: lane (g, q) of a warp reads 16 bytes at (row g, chunk 4j + q); rows g
//     and g+1 share a read phase, so odd rows flip chunk bit 2.
//  V: lane (g, q) reads 4 bytes at (row 2q + e, byte 32j + 4g); the four
//     rows 2q + e of one read must land in different 32-byte groups, so
//     chunk bits 1..2 are flipped by row bits 1..2.
// D = 64 packs two rows per 128-byte line; its K rows already split the line
// and its V swizzle works on the line index.
// ---------------------------------------------------------------------------
template <int D>
__device__ __forceinline__ uint32_t k_off(int row, int chunk) {
  if constexpr (D == 64) {
    return row * 64 + chunk * 16;
  } else {
    return row * D + ((chunk ^ ((row & 1) << 2)) << 4);
  }
}
template <int D>
__device__ __forceinline__ uint32_t v_off(int row, int chunk) {
  if constexpr (D == 64) {
    const int line = row >> 1;
    const int cil = ((row & 1) << 2) | chunk;
    return line * 128 + ((cil ^ ((line & 3) << 1)) << 4);
  } else {
    return row * D + ((chunk ^ (row & 6)) << 4);
  }
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

__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ void cp_async4(uint32_t dst, const void* src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;\n" ::"r"(dst), "l"(src) : "memory");
}

template <int D>
struct Cfg {
  static constexpr int NW = 4;                                        // warps per block
  static constexpr int NS = (D == 64) ? 6 : (D == 128) ? 3 : 2;       // ring stages per warp
  static constexpr int TILE = kTileTokens * D;                        // bytes of a K or V tile
  static constexpr int STAGE = 2 * TILE + 16;                         // K, V, then k / v scale
  static constexpr int WARP_BYTES = NS * STAGE;
  static constexpr int PIPE_BYTES = (NW * WARP_BYTES + 127) / 128 * 128;
  static constexpr bool Q_IN_SMEM = (D > 256);                        // q fragments in smem
  static constexpr int QFRAG_BYTES = Q_IN_SMEM ? (D / 16) * 32 * 8 : 0;
  static constexpr int PROW = 24;                                     // halves per P row
  static constexpr int PBUF_BYTES = NW * 2 * 8 * PROW * 2;
  static constexpr int PID_BYTES = NW * kMaxWarpTiles * 4;            // each warp's page ids
  static constexpr int MISC_FLOATS = NW * 8 * 2 + 4;
  static constexpr int SMEM =
      PIPE_BYTES + QFRAG_BYTES + PBUF_BYTES + PID_BYTES + MISC_FLOATS * 4;
  static constexpr int MIN_BLOCKS = (D == 512) ? 1 : (D == 256) ? 2 : 4;
  static_assert(NW * 8 * D * 4 <= PIPE_BYTES, "merge scratch must fit in the ring");
  static_assert(8 * kMaxSplits * 4 <= PIPE_BYTES, "combine weights must fit in the ring");
};

// One thread block: (split, KV head x head group, sequence). KCVT selects the
// K decode: false = bit assembly (byte pairs (0,2)/(1,3)), true = hardware
// cvt (byte pairs (0,1)/(2,3)); the q fragments follow the same pairing.
template <int D, bool KCVT>
__global__ void __launch_bounds__(128, Cfg<D>::MIN_BLOCKS)
    decode_mma_kernel(const DecodeParams p) {
  using C = Cfg<D>;
  constexpr int KB = D / 16;  // k16 blocks of the QK contraction
  extern __shared__ __align__(128) uint8_t smem[];
  uint8_t* pipe = smem;
  uint2* qfrag_s = reinterpret_cast<uint2*>(smem + C::PIPE_BYTES);
  __half* pbuf = reinterpret_cast<__half*>(smem + C::PIPE_BYTES + C::QFRAG_BYTES);
  int32_t* s_pid = reinterpret_cast<int32_t*>(smem + C::PIPE_BYTES + C::QFRAG_BYTES + C::PBUF_BYTES);
  float* misc = reinterpret_cast<float*>(s_pid + C::NW * kMaxWarpTiles);

  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31, grp = lane >> 2, qd = lane & 3;
  const int split = blockIdx.x, b = blockIdx.z;
  const int kvh = blockIdx.y / p.head_groups;
  const int hg = blockIdx.y - kvh * p.head_groups;
  const int head0 = kvh * p.G + hg * 8;
  const int nheads = min(8, p.G - hg * 8);

  // ---- the keys this block attends: [t0, t1) ------------------------------
  // Split s of a sequence covers pages [first + s * chunk, first + (s+1) * chunk)
  // of its attended range: equal-sized work per block whatever the length,
  // and the blocks past the end of a short sequence have nothing to do.
  int L = __ldg(p.lens + (int64_t)b * p.lens_s);
  if (L < 0 || L > p.max_pages * p.ps) {
    if (tid == 0 && split == 0 && blockIdx.y == 0) raise_flag(FP8PD_FLAG_SEQLEN_OOB);
    L = 0;
  }
  const int lo = p.window > 0 ? max(0, L - p.window) : 0;
  const int first_page = lo / p.ps;
  const int n_pages = (L > lo) ? (L - 1) / p.ps - first_page + 1 : 0;
  const int pg0 = first_page + split * p.chunk_pages;
  const int pg1 = min(first_page + n_pages, pg0 + p.chunk_pages);
  const int t0 = max(lo, pg0 * p.ps);
  const int t1 = min(L, pg1 * p.ps);
  const int tile_first = t0 / kTileTokens;
  const int n_tiles = (t1 > t0) ? (t1 + kTileTokens - 1) / kTileTokens - tile_first : 0;
  int my_tiles = (n_tiles > warp) ? (n_tiles - warp + C::NW - 1) / C::NW : 0;
  if (my_tiles > kMaxWarpTiles) {  // the planner never does this; refuse rather than overflow
    if (lane == 0) raise_flag(FP8PD_FLAG_INTERNAL);
    my_tiles = 0;
  }
  const int32_t* trow = p.table + (int64_t)b * p.tab_sb;

  // ---- warp-local setup: this warp's page ids, q fragments ------------------
  int32_t* wpid = s_pid + warp * kMaxWarpTiles;
  for (int j = lane; j < my_tiles; j += 32) {
    const int lp = (tile_first + warp + C::NW * j) * kTileTokens / p.ps;
    int page = __ldg(trow + (int64_t)lp * p.tab_sp);
    if ((unsigned)page >= (unsigned)p.num_pages) {
      if (hg == 0) raise_flag(FP8PD_FLAG_PAGE_OOB);
      page = -1;
    }
    wpid[j] = page;
  }
  // Lane (g, q) holds query head g of the group at head-dim entries
  // 64jj + 16q + {0..15}; the k16 block (jj, i) covers entries
  // 64jj + 16q + 4i + {0..3}. Bit-assembly K pairs bytes (0,2) and (1,3):
  // k = 2q -> +0, 2q+1 -> +2, 2q+8 -> +1, 2q+9 -> +3; hardware-cvt K pairs
  // (0,1) and (2,3).
  const bool q_head_ok = grp < nheads;
  const uint16_t* qrow = p.q + (int64_t)b * p.q_sb + (int64_t)(head0 + (q_head_ok ? grp : 0)) * p.q_sh;
  float qmax = 0.f;
  if (q_head_ok) {
#pragma unroll 4
    for (int e = 0; e < D / 4; ++e) {
      const int d = 64 * (e >> 4) + 16 * qd + (e & 15);
      qmax = fmaxf(qmax, fabsf(bf16_bits_to_float(__ldg(qrow + (int64_t)d * p.q_sd))));
    }
  }
  qmax = warp_max(qmax);
  // q' = q * 2^(15 - e) puts max|q'| in [2^14, 2^15): exact in f16 for every
  // element above max|q| * 2^-28 (bf16 has 8 significant bits).
  int qe = 0;
  if (qmax > 0.f && isfinite(qmax)) frexpf(qmax, &qe);
  qe = max(qe, -111);
  const float qmul = ldexpf(1.f, 15 - qe);
  // kfac = sm_scale * log2(e) / qmul * k_scale(page), times 2^8 when K is
  // decoded by bit assembly (which yields value * 2^-8); the hardware cvt
  // yields the value itself.
  const float score_base = p.sm_scale_log2 * (KCVT ? 1.f : 256.f) / qmul;
  auto qval = [&](int d) -> float {
    return q_head_ok ? bf16_bits_to_float(__ldg(qrow + (int64_t)d * p.q_sd)) * qmul : 0.f;
  };
  uint32_t qf[C::Q_IN_SMEM ? 1 : KB][2];
#pragma unroll
  for (int kb = 0; kb < KB; ++kb) {
    if constexpr (C::Q_IN_SMEM) {
      if ((kb & 3) != warp) continue;  // the four warps share the work
    }
    const int d = 64 * (kb >> 2) + 16 * qd + 4 * (kb & 3);
    uint32_t r0, r1;
    if constexpr (KCVT) {
      r0 = pack_f16x2(qval(d + 0), qval(d + 1));
      r1 = pack_f16x2(qval(d + 2), qval(d + 3));
    } else {
      r0 = pack_f16x2(qval(d + 0), qval(d + 2));
      r1 = pack_f16x2(qval(d + 1), qval(d + 3));
    }
    if constexpr (C::Q_IN_SMEM) {
      qfrag_s[kb * 32 + lane] = make_uint2(r0, r1);
    } else {
      qf[kb][0] = r0;
      qf[kb][1] = r1;
    }
  }
  if constexpr (C::Q_IN_SMEM) __syncthreads();
  __syncwarp();

  // ---- per-warp pipeline over 16-token tiles --------------------------------
  const uint32_t wpipe = smem_u32(pipe + warp * C::WARP_BYTES);
  __half* p_hi = pbuf + warp * (2 * 8 * C::PROW);
  __half* p_lo = p_hi + 8 * C::PROW;
  const uint8_t* kbase = p.k + (int64_t)kvh * p.k_sh;
  const uint8_t* vbase = p.v + (int64_t)kvh * p.v_sh;
  const float* ksbase = p.ks + (int64_t)kvh * p.ks_sh;
  const float* vsbase = p.vs + (int64_t)kvh * p.vs_sh;

  // Copies tile j of this warp into ring stage `stage`: K and V rows (16-byte
  // cp.async per lane), then the page's k and v scales (4 bytes each).
  auto issue = [&](int j, int stage) {
    const int page = wpid[j];
    if (page < 0) return;
    const int tok0 = (tile_first + warp + C::NW * j) * kTileTokens;
    const int slot0 = tok0 - (tok0 / p.ps) * p.ps;
    const uint8_t* gk = kbase + (int64_t)page * p.k_sp + (int64_t)slot0 * p.k_st;
    const uint8_t* gv = vbase + (int64_t)page * p.v_sp + (int64_t)slot0 * p.v_st;
    const uint32_t sk = wpipe + stage * C::STAGE;
    const uint32_t sv = sk + C::TILE;
    constexpr int CPR = D / 16;
#pragma unroll
    for (int it = 0; it < (kTileTokens * CPR) / 32; ++it) {
      const int idx = it * 32 + lane;
      const int r = idx / CPR, c = idx - r * CPR;
      cp_async16(sk + k_off<D>(r, c), gk + (int64_t)r * p.k_st + c * 16);
      cp_async16(sv + v_off<D>(r, c), gv + (int64_t)r * p.v_st + c * 16);
    }
    if (lane == 0) cp_async4(sv + C::TILE, ksbase + (int64_t)page * p.ks_sp);
    if (lane == 1) cp_async4(sv + C::TILE + 4, vsbase + (int64_t)page * p.vs_sp);
  };

  float O[D / 32][2][4];
#pragma unroll
  for (int jb = 0; jb < D / 32; ++jb)
#pragma unroll
    for (int h = 0; h < 2; ++h)
#pragma unroll
      for (int c = 0; c < 4; ++c) O[jb][h][c] = 0.f;
  float m0 = -CUDART_INF_F, m1 = -CUDART_INF_F;  // running max, heads 2qd / 2qd+1 (log2 units)
  float l0 = 0.f, l1 = 0.f;                      // this lane's share of the running sums
  // Running V reference scale: the largest |v_scale| seen so far. O holds
  // sum P * v_scale / vref, so every f16 P operand stays <= 1 in magnitude.
  float vref = 0.f;

#pragma unroll 1
  for (int s = 0; s < C::NS - 1; ++s) {
    if (s < my_tiles) issue(s, s);
    cp_async_commit();
  }

#pragma unroll 1
  for (int j = 0; j < my_tiles; ++j) {
    cp_async_wait<C::NS - 2>();
    __syncwarp();
    {
      const int nj = j + C::NS - 1;
      if (nj < my_tiles) issue(nj, nj % C::NS);
      cp_async_commit();
    }
    const int tok0 = (tile_first + warp + C::NW * j) * kTileTokens;
    const bool page_ok = wpid[j] >= 0;
    const uint32_t sk = wpipe + (j % C::NS) * C::STAGE;
    const uint32_t sv = sk + C::TILE;
    float kfac = 0.f, vs = 0.f;
    if (page_ok) {
      kfac = score_base * __uint_as_float(lds32(sv + C::TILE));
      vs = __uint_as_float(lds32(sv + C::TILE + 4));
    }

    // -- S[token][head] = K q'^T (two independent accumulator chains) --------
    float Sa[4] = {0.f, 0.f, 0.f, 0.f}, Sb[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int jj = 0; jj < D / 64; ++jj) {
      const uint4 ka = lds128(sk + k_off<D>(grp, 4 * jj + qd));
      const uint4 kb = lds128(sk + k_off<D>(grp + 8, 4 * jj + qd));
      const uint32_t wa[4] = {ka.x, ka.y, ka.z, ka.w};
      const uint32_t wb[4] = {kb.x, kb.y, kb.z, kb.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        uint32_t b0, b1;
        if constexpr (C::Q_IN_SMEM) {
          const uint2 f = qfrag_s[(jj * 4 + i) * 32 + lane];
          b0 = f.x;
          b1 = f.y;
        } else {
          b0 = qf[jj * 4 + i][0];
          b1 = qf[jj * 4 + i][1];
        }
        uint32_t a0, a1, a2, a3;
        if constexpr (KCVT) {
          a0 = e4m3x2_lo16_to_f16x2(wa[i]);
          a1 = e4m3x2_lo16_to_f16x2(wb[i]);
          a2 = e4m3x2_hi16_to_f16x2(wa[i]);
          a3 = e4m3x2_hi16_to_f16x2(wb[i]);
        } else {
          a0 = e4m3x2_b02_to_f16x2(wa[i]);
          a1 = e4m3x2_b02_to_f16x2(wb[i]);
          a2 = e4m3x2_b13_to_f16x2(wa[i]);
          a3 = e4m3x2_b13_to_f16x2(wb[i]);
        }
        if (i & 1)
          mma16816(Sb, a0, a1, a2, a3, b0, b1);
        else
          mma16816(Sa, a0, a1, a2, a3, b0, b1);
      }
    }

    // -- masked scores (log2 units), online softmax ------------------------
    const int ta = tok0 + grp, tb = ta + 8;
    const bool va = page_ok && ta >= t0 && ta < t1;
    const bool vb = page_ok && tb >= t0 && tb < t1;
    // a masked row may hold stale or NaN-decoded bytes: select, never multiply
    const float s00 = va ? (Sa[0] + Sb[0]) * kfac : -CUDART_INF_F;  // token grp,   head 2qd
    const float s01 = va ? (Sa[1] + Sb[1]) * kfac : -CUDART_INF_F;  // token grp,   head 2qd+1
    const float s10 = vb ? (Sa[2] + Sb[2]) * kfac : -CUDART_INF_F;  // token grp+8, head 2qd
    const float s11 = vb ? (Sa[3] + Sb[3]) * kfac : -CUDART_INF_F;  // token grp+8, head 2qd+1
    float tm0 = fmaxf(s00, s10), tm1 = fmaxf(s01, s11);
#pragma unroll
    for (int o = 4; o < 32; o <<= 1) {
      tm0 = fmaxf(tm0, __shfl_xor_sync(0xffffffffu, tm0, o));
      tm1 = fmaxf(tm1, __shfl_xor_sync(0xffffffffu, tm1, o));
    }
    const float mn0 = fmaxf(m0, tm0), mn1 = fmaxf(m1, tm1);
    const float vabs = fabsf(vs);
    const bool grow_v = vabs > vref;  // warp-uniform: one scale per tile
    if (grow_v || __any_sync(0xffffffffu, (mn0 > m0) || (mn1 > m1))) {
      const float c0 = (mn0 > m0) ? fast_exp2(m0 - mn0) : 1.f;  // exp2(-inf) = 0 for a first max
      const float c1 = (mn1 > m1) ? fast_exp2(m1 - mn1) : 1.f;
      const float fv = grow_v ? vref / vabs : 1.f;
      l0 *= c0;
      l1 *= c1;
      const float o0 = c0 * fv, o1 = c1 * fv;
#pragma unroll
      for (int jb = 0; jb < D / 32; ++jb)
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          O[jb][h][0] *= o0;
          O[jb][h][1] *= o1;
          O[jb][h][2] *= o0;
          O[jb][h][3] *= o1;
        }
      m0 = mn0;
      m1 = mn1;
      if (grow_v) vref = vabs;
    }
    const float mb0 = (m0 == -CUDART_INF_F) ? 0.f : m0;
    const float mb1 = (m1 == -CUDART_INF_F) ? 0.f : m1;
    const float p00 = fast_exp2(s00 - mb0), p01 = fast_exp2(s01 - mb1);
    const float p10 = fast_exp2(s10 - mb0), p11 = fast_exp2(s11 - mb1);
    l0 += p00 + p10;
    l1 += p01 + p11;

    // -- P * v_scale / vref as f16 hi + lo, transposed through shared memory
    {
      const float vsr = (vref > 0.f) ? vs / vref : 0.f;
      const float w00 = p00 * vsr, w01 = p01 * vsr, w10 = p10 * vsr, w11 = p11 * vsr;
      const __half h00 = __float2half_rn(w00), h01 = __float2half_rn(w01);
      const __half h10 = __float2half_rn(w10), h11 = __float2half_rn(w11);
      const int r0 = (2 * qd) * C::PROW, r1 = r0 + C::PROW;
      p_hi[r0 + grp] = h00;
      p_hi[r0 + grp + 8] = h10;
      p_hi[r1 + grp] = h01;
      p_hi[r1 + grp + 8] = h11;
      p_lo[r0 + grp] = __float2half_rn(w00 - __half2float(h00));
      p_lo[r0 + grp + 8] = __float2half_rn(w10 - __half2float(h10));
      p_lo[r1 + grp] = __float2half_rn(w01 - __half2float(h01));
      p_lo[r1 + grp + 8] = __float2half_rn(w11 - __half2float(h11));
    }
    __syncwarp();
    const uint32_t* phw = reinterpret_cast<const uint32_t*>(p_hi + grp * C::PROW);
    const uint32_t* plw = reinterpret_cast<const uint32_t*>(p_lo + grp * C::PROW);
    const uint32_t bh0 = phw[qd], bh1 = phw[qd + 4];  // tokens (2qd, 2qd+1), (2qd+8, 2qd+9)
    const uint32_t bl0 = plw[qd], bl1 = plw[qd + 4];

    // -- O^T[d][head] += V^T P ---------------------------------------------
    // Block jb covers d in [32jb, 32jb+32). Lane (g, q) reads bytes 4g..4g+3
    // of the block from tokens 2q, 2q+1, 2q+8, 2q+9; M tile (jb, h) row g is
    // d = 32jb + 4g + 2h, row g+8 is d + 1.
#pragma unroll
    for (int jb = 0; jb < D / 32; ++jb) {
      const int c = 2 * jb + (grp >> 2);
      const uint32_t cb = (grp & 3) * 4;
      const uint32_t w0 = lds32(sv + v_off<D>(2 * qd, c) + cb);
      const uint32_t w1 = lds32(sv + v_off<D>(2 * qd + 1, c) + cb);
      const uint32_t w2 = lds32(sv + v_off<D>(2 * qd + 8, c) + cb);
      const uint32_t w3 = lds32(sv + v_off<D>(2 * qd + 9, c) + cb);
      const uint32_t za = prmt(w0, w1, 0x5410), zb = prmt(w0, w1, 0x7632);
      const uint32_t zc = prmt(w2, w3, 0x5410), zd = prmt(w2, w3, 0x7632);
      const uint32_t a0 = e4m3x2_b02_to_f16x2(za), a1 = e4m3x2_b13_to_f16x2(za);
      const uint32_t a2 = e4m3x2_b02_to_f16x2(zc), a3 = e4m3x2_b13_to_f16x2(zc);
      mma16816(O[jb][0], a0, a1, a2, a3, bh0, bh1);
      mma16816(O[jb][0], a0, a1, a2, a3, bl0, bl1);
      const uint32_t e0 = e4m3x2_b02_to_f16x2(zb), e1 = e4m3x2_b13_to_f16x2(zb);
      const uint32_t e2 = e4m3x2_b02_to_f16x2(zd), e3 = e4m3x2_b13_to_f16x2(zd);
      mma16816(O[jb][1], e0, e1, e2, e3, bh0, bh1);
      mma16816(O[jb][1], e0, e1, e2, e3, bl0, bl1);
    }
  }
  cp_async_wait<0>();

  // ---- merge the warps ------------------------------------------------------
#pragma unroll
  for (int o = 4; o < 32; o <<= 1) {
    l0 += __shfl_xor_sync(0xffffffffu, l0, o);
    l1 += __shfl_xor_sync(0xffffffffu, l1, o);
  }
  __syncthreads();  // every warp is done with its ring
  float* Os = reinterpret_cast<float*>(pipe);  // [NW][8][D], already times 2^8 * vref
  float* ml = misc;                            // [NW][8][2]
  const float fold = 256.f * vref;             // f16 offset of the decoded V, V reference scale
#pragma unroll
  for (int jb = 0; jb < D / 32; ++jb) {
    const int d = 32 * jb + 4 * grp;
    *reinterpret_cast<float4*>(Os + (warp * 8 + 2 * qd) * D + d) = make_float4(
        O[jb][0][0] * fold, O[jb][0][2] * fold, O[jb][1][0] * fold, O[jb][1][2] * fold);
    *reinterpret_cast<float4*>(Os + (warp * 8 + 2 * qd + 1) * D + d) = make_float4(
        O[jb][0][1] * fold, O[jb][0][3] * fold, O[jb][1][1] * fold, O[jb][1][3] * fold);
  }
  if (grp == 0) {
    ml[(warp * 8 + 2 * qd) * 2 + 0] = m0;
    ml[(warp * 8 + 2 * qd) * 2 + 1] = l0;
    ml[(warp * 8 + 2 * qd + 1) * 2 + 0] = m1;
    ml[(warp * 8 + 2 * qd + 1) * 2 + 1] = l1;
  }
  __syncthreads();

  constexpr float kLog2e = 1.4426950408889634f;
  const int S = p.num_splits;
  for (int it = tid; it < 8 * (D / 4); it += 128) {
    const int n = it / (D / 4);
    const int d = (it - n * (D / 4)) * 4;
    if (n >= nheads) continue;
    float M = -CUDART_INF_F;
#pragma unroll
    for (int w = 0; w < C::NW; ++w) M = fmaxf(M, ml[(w * 8 + n) * 2]);
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    float l = 0.f;
    if (M != -CUDART_INF_F) {
#pragma unroll
      for (int w = 0; w < C::NW; ++w) {
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
    if (S == 1) {
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
      const int64_t row = ((int64_t)b * p.Hq + head) * S + split;
      *reinterpret_cast<float4*>(p.part_o + row * D + d) = acc;
      if (d == 0) *reinterpret_cast<float2*>(p.part_ml + row * 2) = make_float2(M, l);
    }
  }
  if (S == 1) return;

  // ---- the last block of this (sequence, KV head, head group) combines ------
  // Every block publishes its partials, then takes a ticket; the block that
  // draws the last ticket merges all S partials (log-sum-exp, sink added once)
  // and resets the counter for the next call. No block ever waits for another.
  __threadfence();
  __syncthreads();
  int* last_flag = reinterpret_cast<int*>(misc + C::NW * 8 * 2);
  const int64_t unit = (int64_t)b * gridDim.y + blockIdx.y;
  if (tid == 0) {
    const int prev = atomicAdd(p.counters + unit, 1);
    *last_flag = (prev == S - 1);
  }
  __syncthreads();
  if (!*last_flag) return;
  __threadfence();

  float* wts = reinterpret_cast<float*>(pipe);  // [8][kMaxSplits] split weight / den
  for (int n = warp; n < nheads; n += C::NW) {
    const int head = head0 + n;
    const float* pml = p.part_ml + ((int64_t)b * p.Hq + head) * S * 2;
    float M = -CUDART_INF_F;
    for (int s = lane; s < S; s += 32) M = fmaxf(M, ldcg2(pml + 2 * s).x);
    M = warp_max(M);
    const float sl = p.sinks ? p.sinks[(int64_t)head * p.sinks_s] * kLog2e : -CUDART_INF_F;
    const float M2 = fmaxf(M, sl);
    float den = 0.f;
    if (M2 != -CUDART_INF_F) {
      for (int s = lane; s < S; s += 32) {
        const float2 ml2 = ldcg2(pml + 2 * s);
        if (ml2.x != -CUDART_INF_F) den += ml2.y * fast_exp2(ml2.x - M2);
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) den += __shfl_xor_sync(0xffffffffu, den, o);
      if (p.sinks) den += fast_exp2(sl - M2);
    }
    const float inv = (M2 != -CUDART_INF_F && den > 0.f) ? 1.f / den : 0.f;
    for (int s = lane; s < S; s += 32) {
      const float ms = ldcg2(pml + 2 * s).x;
      wts[n * kMaxSplits + s] = (inv == 0.f || ms == -CUDART_INF_F) ? 0.f : fast_exp2(ms - M2) * inv;
    }
  }
  __syncthreads();
  // Every split wrote its row (zeros for an empty one), so the weighted sum
  // needs no branch and its loads can all be in flight at once.
  for (int it = tid; it < nheads * (D / 4); it += 128) {
    const int n = it / (D / 4);
    const int d = (it - n * (D / 4)) * 4;
    const int head = head0 + n;
    const float* po = p.part_o + ((int64_t)b * p.Hq + head) * S * D + d;
    const float* wn = wts + n * kMaxSplits;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 8
    for (int s = 0; s < S; ++s) {
      const float w = wn[s];
      const float4 o = ldcg4(po + (int64_t)s * D);
      acc.x += w * o.x;
      acc.y += w * o.y;
      acc.z += w * o.z;
      acc.w += w * o.w;
    }
    *reinterpret_cast<float4*>(p.out + (int64_t)b * p.o_sb + (int64_t)head * p.o_sh + d) = acc;
  }
  if (tid == 0) p.counters[unit] = 0;
}

// ---------------------------------------------------------------------------
// Quantize-append: one thread per (sequence, KV head, pair of head-dim
// entries), for K and V. code = E4M3_RNE_SAT(float32(x) / scale): IEEE float32
// division (__fdiv_rn), then cvt.rn.satfinite.e4m3x2.f32, which rounds to
// nearest even and saturates to +-448 (NaN stays NaN).
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint16_t e4m3x2_from_f32(float lo, float hi) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return r;  // low byte = lo, high byte = hi
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
  const float ks = p.ks[(int64_t)page * p.ks_sp + (int64_t)h * p.ks_sh];
  const float vs = p.vs[(int64_t)page * p.vs_sp + (int64_t)h * p.vs_sh];
  const uint16_t* kn = p.kn + (int64_t)b * p.kn_sb + (int64_t)h * p.kn_sh + (int64_t)d * p.kn_sd;
  const uint16_t* vn = p.vn + (int64_t)b * p.vn_sb + (int64_t)h * p.vn_sh + (int64_t)d * p.vn_sd;
  const float k0 = __fdiv_rn(bf16_bits_to_float(kn[0]), ks);
  const float k1 = two ? __fdiv_rn(bf16_bits_to_float(kn[p.kn_sd]), ks) : 0.f;
  const float v0 = __fdiv_rn(bf16_bits_to_float(vn[0]), vs);
  const float v1 = two ? __fdiv_rn(bf16_bits_to_float(vn[p.vn_sd]), vs) : 0.f;
  const uint16_t kc = e4m3x2_from_f32(k0, k1);
  const uint16_t vc = e4m3x2_from_f32(v0, v1);
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
template <int D, bool KCVT>
static cudaError_t launch_decode_mma_d(const DecodeParams& p, cudaStream_t s) {
  // The shared-memory opt-in is a per-device function attribute: set it once
  // per device (an idempotent call, so a race only repeats it).
  static std::atomic<uint64_t> configured{0};
  const int smem = Cfg<D>::SMEM;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const uint64_t bit = (dev >= 0 && dev < 64) ? (uint64_t(1) << dev) : 0;
  if (!bit || !(configured.load() & bit)) {
    e = cudaFuncSetAttribute(decode_mma_kernel<D, KCVT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             smem);
    if (e != cudaSuccess) return e;
    configured.fetch_or(bit);
  }
  const dim3 grid(p.num_splits, p.Hkv * p.head_groups, p.B);
  decode_mma_kernel<D, KCVT><<<grid, 128, smem, s>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_decode_mma(const DecodeParams& p, int D, bool k_cvt, cudaStream_t s) {
  switch (D) {
    case 64: return k_cvt ? launch_decode_mma_d<64, true>(p, s) : launch_decode_mma_d<64, false>(p, s);
    case 128: return k_cvt ? launch_decode_mma_d<128, true>(p, s) : launch_decode_mma_d<128, false>(p, s);
    case 256: return k_cvt ? launch_decode_mma_d<256, true>(p, s) : launch_decode_mma_d<256, false>(p, s);
    case 512: return k_cvt ? launch_decode_mma_d<512, true>(p, s) : launch_decode_mma_d<512, false>(p, s);
    default: return cudaErrorInvalidValue;
  }
}

int decode_mma_smem_bytes(int D) {
  switch (D) {
    case 64: return Cfg<64>::SMEM;
    case 128: return Cfg<128>::SMEM;
    case 256: return Cfg<256>::SMEM;
    case 512: return Cfg<512>::SMEM;
    default: return 0;
  }
}

template <int D>
static int blocks_per_sm_d() {
  static std::atomic<int> cached{-1};
  int c = cached.load();
  if (c >= 0) return c;
  int n = 0;
  if (cudaFuncSetAttribute(decode_mma_kernel<D, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           Cfg<D>::SMEM) != cudaSuccess ||
      cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, decode_mma_kernel<D, false>, 128,
                                                    Cfg<D>::SMEM) != cudaSuccess) {
    cudaGetLastError();
    return Cfg<D>::MIN_BLOCKS;  // no device: do not cache the guess
  }
  c = n > 0 ? n : 1;
  cached.store(c);
  return c;
}

int decode_mma_blocks_per_sm(int D) {
  switch (D) {
    case 64: return blocks_per_sm_d<64>();
    case 128: return blocks_per_sm_d<128>();
    case 256: return blocks_per_sm_d<256>();
    case 512: return blocks_per_sm_d<512>();
    default: return 1;
  }
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
