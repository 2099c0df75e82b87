// Internal declarations shared by the host API and the kernels of the FP8
// paged decode attention library (not part of the public ABI).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace fp8pd {

// Everything the split kernel needs, resolved from the public descriptors.
// Strides of the pools are in bytes; of scales, tables, q and out in elements.
struct DecodeParams {
  const uint16_t* q;          // bf16 bits [B, Hq, D]
  int64_t q_sb, q_sh, q_sd;
  const uint8_t* k;           // pool views [num_pages, ps, Hkv, D]
  const uint8_t* v;
  int64_t k_sp, k_st, k_sh;
  int64_t v_sp, v_st, v_sh;
  const float* ks;            // scale(page, slot, h) = ks[page * ks_sp + slot * ks_st + h * ks_sh]
  const float* vs;
  int64_t ks_sp, ks_sh, vs_sp, vs_sh;
  int64_t ks_st, vs_st;       // 0 unless the scales are per token
  int k_tok, v_tok;           // 1: per-token-per-head scales [num_pages, ps, Hkv]
  int64_t ks_sg;              // K sub-row groups [num_pages, ps, Hkv, k_groups]: group stride
  int k_groups;               // 1, or 2..16 (D / k_groups >= 16): K entry d uses group d / (D / k_groups)
  // MXFP8: K / V scales are E8M0 bytes [num_pages, ps, Hkv, D / 32] (ks / vs
  // then point at uint8, strides in bytes); K takes k_groups = D / 32, V one
  // code per 32-entry block (vs_sg its stride).
  int k_mx, v_mx;
  int64_t vs_sg;
  const int32_t* table;       // [B, max_pages]
  int64_t tab_sb, tab_sp;
  const int32_t* lens;        // [B]
  int64_t lens_s;
  const float* sinks;         // [Hq] or nullptr
  int64_t sinks_s;
  float* out;                 // [B, Hq, D], d contiguous
  int64_t o_sb, o_sh;
  float* part_o;              // [B * Hq * S, D] split numerators (S > 1)
  float* part_ml;             // [B * Hq * S, 2] split (max, sum) in log2 units
  int* counters;              // [B * Hkv * head_groups][1 + num_groups] tickets, zero between calls
  float* grp_o;               // [B * Hq * num_groups, D] merged groups of splits
  float* grp_ml;              // [B * Hq * num_groups, 2]
  int B, Hq, Hkv, G, D, ps, num_pages, max_pages, window, num_splits, head_groups;
  int chunk_pages;            // pages per split (the last split of a sequence may have fewer)
  int num_groups;             // ceil(num_splits / 8): groups of the two-level split merge
  int q_vec;                  // 1: q rows are contiguous and 8-byte aligned (vector loads)
  float sm_scale_log2;        // sm_scale * log2(e)
  // Proportional splits (split kernel with prop = 1): grid (HX, nbx); each
  // sequence b gets S_b of the nbx blocks of every KV head x head group, at
  // least ceil(tiles / kMaxSplitTiles), the rest in proportion to its tiles.
  int prop;
  int nbx;
  // Bounded waits: polls of a tile barrier before a wait gives up (sets
  // FLAG_TIMEOUT); test_stall: the first block's warp 0 never issues its
  // first copy (the timeout path's test hook).
  int wait_polls;
  int test_stall;
  // Context-parallel slices: kr (int32 [B, 2], or nullptr) cuts each
  // sequence's attended keys to [kr[b][0], kr[b][1]); with pout_o set, each
  // (sequence, query head) is written unnormalized to pout_o [B * Hq, D] and
  // (m, l) to pout_ml [B * Hq, 2] (m in log2 units, no sink) instead of out.
  const int32_t* kr;
  int64_t kr_sb, kr_s1;
  float* pout_o;
  float* pout_ml;
  // Fused append (split kernel only): `lens` holds positions; sequence b
  // attends over positions[b] + 1 keys, the last of them the new token
  // (kn, vn: bf16 [B, Hkv, D]), which the block holding it quantizes, stores
  // through kw / vw (the pools, writable) and attends.
  int append;
  const uint16_t* kn;
  const uint16_t* vn;
  int64_t kn_sb, kn_sh, kn_sd, vn_sb, vn_sh, vn_sd;
  uint8_t* kw;
  uint8_t* vw;
  float* ksw;                 // the scales, writable: a per-token scale of the new token is stored
  float* vsw;
  // 1: the tensor-memory kernel (D = 64 / 128, page or head scales, f32
  // compute) runs this call
  int umma;
  // Warps sharing each tile stream of the split kernel, each on its part of
  // the head dim: 1, or 2 / 4 at D = 512 (page or head scales, f32 compute
  // with the cvt decodes, no fused append), where the tensor maps copy half
  // or quarter rows.
  int dsplit;
};

struct AppendParams {
  const uint16_t* kn;         // bf16 bits [B, Hkv, D]
  const uint16_t* vn;
  int64_t kn_sb, kn_sh, kn_sd, vn_sb, vn_sh, vn_sd;
  uint8_t* k;
  uint8_t* v;
  int64_t k_sp, k_st, k_sh, v_sp, v_st, v_sh;
  const float* ks;
  const float* vs;
  int64_t ks_sp, ks_sh, vs_sp, vs_sh;
  int64_t ks_st, vs_st;       // slot strides (per-token scales), else 0
  int k_tok, v_tok;           // 1: the scale is the new token's own max|x| / 448, written here
  int64_t ks_sg;              // K sub-row groups: group stride; k_groups groups of D / k_groups
  int k_groups;
  int k_mx, v_mx;             // MXFP8 block scales (E8M0 bytes, one per 32 entries), written here
  int64_t vs_sg;
  float* ksw;
  float* vsw;
  const int32_t* table;
  int64_t tab_sb, tab_sp;
  const int32_t* pos;
  int64_t pos_s;
  int B, Hkv, D, ps, num_pages, max_pages;
};

// Launchers (defined with the kernels). Return a cudaError_t of the launch.
// tmk / tmv: tensor maps over the K / V pool views (see make_pool_map).
// k_mode: 0 / 1 = K decoded to f16 (bit assembly / hardware cvt) for f16
// MMAs, 2 = E4M3 MMAs on K's bytes, 3 = the fp8 compute path (q and P
// rounded once to E4M3, E4M3 MMAs on K's and V's bytes); v_cvt: V decoded by
// the hardware cvt.
cudaError_t launch_decode(const DecodeParams& p, const CUtensorMap& tmk, const CUtensorMap& tmv,
                          int k_mode, bool v_cvt, cudaStream_t s);
cudaError_t launch_append(const AppendParams& p, cudaStream_t s);
// Merge of R partial results (O, m, l) per (sequence, query head) into out,
// adding the sink once: po [R][BH][D], pml [R][BH][2] contiguous, BH = B * Hq.
cudaError_t launch_combine(const float* po, const float* pml, int R, int B, int Hq, int D,
                           const float* sinks, int64_t sinks_s, float* out, int64_t o_sb,
                           int64_t o_sh, cudaStream_t s);
// E4M3 codes (the append's rounding) of n float32 values; strides in elements.
cudaError_t launch_encode(const float* x, int64_t xs, uint8_t* c, int64_t cs, int64_t n,
                          cudaStream_t s);

// Warps per tile stream of the split kernel at D = 512 (1, 2 or 4) where a
// call allows the head-dim split; a compile-time setting for tuning builds.
// Two measured fastest: four repeat the softmax in every warp of a stream.
#ifndef FP8PD_DSPLIT_D512
#define FP8PD_DSPLIT_D512 2
#endif

// Thread blocks of the split kernel one SM holds for head dim D (dsplit: the
// warps sharing each tile stream, 1, 2 or 4).
int decode_blocks_per_sm(int D, int dsplit = 1);
// Thread blocks of the tensor-memory kernel one SM holds (D = 64 / 128; else 0).
int decode_umma_blocks_per_sm(int D);
// Warps per block of the split kernel for head dim D.
int decode_warps_per_block(int D, int dsplit = 1);
// Dynamic shared memory of the split kernel for head dim D.
int decode_smem_bytes(int D, int dsplit = 1);

// Device error word (one per device): read and cleared by the host API.
cudaError_t read_and_clear_error_word(uint32_t* value, cudaStream_t s);

constexpr int kHeadsPerGroup = 8;   // query heads one thread block serves (MMA N)
constexpr int kTileTokens = 16;     // tokens per MMA row tile
constexpr int kMaxWarpTiles = 128;  // 16-token tiles one warp takes in a split (list in smem)
constexpr int kMaxSplitTokens = kMaxWarpTiles * 4 * kTileTokens;  // 8,192 keys per split
constexpr int kMaxSplitTiles = kMaxSplitTokens / kTileTokens;      // 512 tiles per split
constexpr int kPropMaxBatch = 1024;  // sequences the proportional planner handles in the kernel
constexpr int kMergeFan = 8;         // splits per group of the two-level split merge
constexpr int kMaxSplits = 256;     // splits per (sequence, KV head, head group)
constexpr int kMaxPages = (1 << 27) - 1;  // pool pages (tile lists pack page << 4)

}  // namespace fp8pd
