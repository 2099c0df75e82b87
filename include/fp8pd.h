/*
 * fp8pd.h -- C ABI of the FP8 (E4M3) paged split-KV decode attention library
 * for NVIDIA B200 (sm_100a).
 *
 * Two operations, both from the "FP8 paged attention for MoE serving"
 * solution page (cerinamroth.com, "How do I run paged decode attention over
 * an FP8 KV cache ... with sliding windows, attention sinks and a custom
 * scale?"):
 *
 *   fp8_paged_decode_attention  one decode query per sequence attending over
 *                               a paged E4M3 KV cache, with grouped-query
 *                               heads, an optional sliding window, optional
 *                               per-head sink logits and a caller softmax
 *                               scale (sections "Expected result" and
 *                               "Supported scope").
 *   fp8_kv_append               quantize one new token per sequence to E4M3
 *                               and store it in its page (section "Supported
 *                               scope", the one-launch T=1 append; the
 *                               "Lecture 8 -- Inference Path" page, "In-kernel
 *                               KV cache update").
 *   fp8_paged_decode_append_attention
 *                               both in one launch: the append, then the
 *                               attention over the cache that now holds the
 *                               new token (the same Lecture 8 section: the
 *                               cache is updated inside the attention kernel,
 *                               before the query reads it).
 *
 * K and V scales come per KV head, per (page, KV head) or per (stored token,
 * KV head), K also in sub-row groups (the solution page's "Supported scope":
 * quantize_kv_fp8's per-token-per-head scales and k_groups). Helpers: an
 * allocation-free attention entry point, planning, workspace, options, the
 * device error word, timing, and fp8pd_e4m3_encode (the append's rounding on
 * a float32 array).
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * - Every buffer is caller-owned device memory described by fp8pd_tensor
 *   (pointer, dtype, shape, strides in ELEMENTS). The library never frees or
 *   keeps a caller pointer past the call.
 * - Calls are asynchronous on `stream` (a cudaStream_t; NULL = the legacy
 *   default stream) and return a status: 0 = success, negative = the call
 *   was refused and NOTHING was launched (validation happens on the host
 *   before any launch). FP8PD_ERR_CUDA means a CUDA call failed; the CUDA
 *   error is available from fp8pd_last_cuda_error().
 * - Problems only visible on the device never trap: the kernel skips the
 *   offending work and sets a bit in the device error word, read and
 *   cleared by fp8pd_check_errors(). A sequence length outside
 *   [0, max_pages * page_size] makes that sequence's output 0; a 16-token
 *   tile whose block-table entry is outside [0, num_pages) is left out of
 *   the softmax; an append position outside the block table, or whose page
 *   is outside the pool, is not written.
 * - The library is thread-safe; per-device state (split workspace) is
 *   guarded by a mutex. The split workspace is reused by every call on the
 *   device, so calls that overlap on the GPU (different streams, no
 *   ordering) must not both need it; calls on one stream are ordered.
 */
#ifndef FP8PD_H_
#define FP8PD_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define FP8PD_VERSION 1

/* A CUDA stream handle (identical to cudaStream_t / CUstream). */
typedef struct CUstream_st* fp8pd_stream_t;

/* Element types. */
enum {
  FP8PD_DTYPE_U8 = 1,   /* uint8: E4M3 codes (pools) */
  FP8PD_DTYPE_I32 = 2,  /* int32: block tables, lengths, positions */
  FP8PD_DTYPE_F32 = 3,  /* float32: scales, sinks, output */
  FP8PD_DTYPE_BF16 = 4  /* bfloat16: q, new K/V */
};

/* A strided view of device memory. `data` points at element [0,..,0];
 * element (i0,..,i{n-1}) lives at data + sum_k i_k * stride[k] elements.
 * Unused trailing entries of shape/stride are ignored. */
typedef struct fp8pd_tensor {
  void* data;
  int32_t dtype;
  int32_t ndim;
  int64_t shape[4];
  int64_t stride[4];
} fp8pd_tensor;

/* K and V scales for fp8_kv_append. Each is float32 of shape [Hkv] (one
 * scale per KV head), [num_pages, Hkv] (one per physical page and KV head,
 * indexed by the page id found in the block table) -- both read only -- or
 * [num_pages, ps, Hkv] (one per stored token and KV head, the cache-write
 * quantizer's per-token-per-head form named in the solution page's
 * "Supported scope"), which the append writes; K also
 * [num_pages, ps, Hkv, G] (sub-row groups, written per group). */
typedef struct fp8pd_scales {
  fp8pd_tensor k_scale;
  fp8pd_tensor v_scale;
} fp8pd_scales;

/* Status codes. */
enum {
  FP8PD_OK = 0,
  FP8PD_ERR_NULL = -1,              /* a required descriptor or pointer is NULL */
  FP8PD_ERR_DTYPE = -2,             /* wrong element type */
  FP8PD_ERR_SHAPE = -3,             /* inconsistent or unsupported shape */
  FP8PD_ERR_ALIGN = -4,             /* pool base / strides not multiples of 16 bytes, or
                                       inner dimension not contiguous */
  FP8PD_ERR_UNSUPPORTED = -5,       /* head_dim not in {64,128,256,512}, page size not a
                                       multiple of 16, Hq not a multiple of Hkv, ... */
  FP8PD_ERR_ARG = -6,               /* bad scalar: window < 0, sm_scale not finite and > 0,
                                       unknown option */
  FP8PD_ERR_WORKSPACE = -7,         /* the split workspace could not be allocated */
  FP8PD_ERR_CAPTURE_WORKSPACE = -8, /* the stream is capturing and the split workspace is
                                       smaller than the call needs (reserve it first) */
  FP8PD_ERR_CUDA = -9,              /* a CUDA runtime call failed */
  FP8PD_ERR_TOO_LARGE = -10         /* a size exceeds a documented limit (e.g. more than
                                       2,097,152 attended keys in one sequence) */
};

/* Bits of the device error word. */
enum {
  FP8PD_FLAG_PAGE_OOB = 1u,    /* block-table entry outside [0, num_pages): tile skipped */
  FP8PD_FLAG_SEQLEN_OOB = 2u,  /* seq_lens[b] < 0 or > max_pages * page_size: sequence skipped */
  FP8PD_FLAG_POS_OOB = 4u,     /* append position < 0 or >= max_pages * page_size: not written */
  FP8PD_FLAG_INTERNAL = 8u,    /* a split covered more keys than the kernel holds (a planner
                                  bug): that split is left out */
  FP8PD_FLAG_TIMEOUT = 16u     /* a tile copy did not complete within the kernel's bounded wait:
                                  that warp's keys are left out */
};

/*
 * fp8_paged_decode_attention -- decode attention over a paged E4M3 KV cache.
 *
 * Defines (for each sequence b and query head hq, h = hq / (Hq / Hkv)):
 *   keys t in [lo, L), L = seq_lens[b], lo = window > 0 ? max(0, L - window) : 0
 *   K(t, d) = e4m3(k_pages[page(t), t % ps, h, d]) * k_scale(page(t), t % ps, h)
 *   V(t, d) likewise, page(t) = block_table[b, t / ps]
 *   s_t = sm_scale * sum_d q[b, hq, d] * K(t, d)
 *   M = max(max_t s_t, sink[hq]);  den = sum_t exp(s_t - M) + exp(sink[hq] - M)
 *   out[b, hq, :] = sum_t exp(s_t - M) * V(t, :) / den     (0 if there is nothing to attend)
 * The window keeps the last `window` keys; a sink is a logit in the scaled
 * space that enters the denominator only (the solution page's "Expected
 * result": `window=W` keeps the last W keys, sinks are [H_q] fp32 with no
 * value, `sm_scale` replaces D**-0.5). Query head hq reads KV head
 * hq / (Hq/Hkv) ("Smallest correct example", q.view(H_KV, H_Q // H_KV, D)).
 * E4M3 codes 0x7F / 0xFF (NaN) decode as +-480: finite inputs never
 * produce them.
 *
 * Arguments (shapes; all device memory):
 *   q            bf16 [B, Hq, D], any strides.
 *   k_pages,     uint8 [num_pages, ps, Hkv, D] E4M3 codes; stride[3] must be 1;
 *   v_pages      base pointer and strides 0..2 must be multiples of 16 bytes
 *                (a page stride wider than one layer's page is allowed: several
 *                layers may share one pool -- the solution page's per-layer row
 *                strides; the 16-byte rule follows DeepGEMM PR #459's paged
 *                accessor). D in {64, 128, 256, 512}; ps a multiple of 16, <= 256;
 *                num_pages < 2^27.
 *   k_scale,     float32 [Hkv] (per KV head), [num_pages, Hkv] (per page and KV
 *   v_scale      head) or [num_pages, ps, Hkv] (per stored token and KV head),
 *                any strides (0 = broadcast); k_scale(page, slot, h) ignores
 *                the missing axes. K and V may use different forms. K may
 *                also be [num_pages, ps, Hkv, G] (the solution page's k_groups
 *                sub-row key scales): head-dim entry d of a key uses scale
 *                [page, slot, h, d / (D / G)]; G in {1, 2, 4, 8, 16} with
 *                D / G >= 16, else FP8PD_ERR_UNSUPPORTED. V takes G = 1 only.
 *   block_table  int32 [B, max_pages]: physical page of each logical page.
 *                Entries past the attended range are never read.
 *   seq_lens     int32 [B]: number of keys visible to the query (positions 0..L-1).
 *   window       >= 0; 0 = full attention.
 *   sinks        float32 [Hq] or NULL.
 *   sm_scale     finite, > 0.
 *   out          float32 [B, Hq, D]; stride[2] must be 1, rows 16-byte aligned.
 *   stream       CUDA stream.
 * Launches one kernel, with one of two schedules. Uniform splits (1): the
 * split kernel gives each (sequence, KV head, head group) the same number of
 * blocks, each an equal share of its table's pages. Proportional splits (3):
 * the split kernel on one wave of blocks per KV head x head group, shared
 * among the sequences in proportion to their tiles (the kernel reads the
 * lengths). In both, the last block of each (sequence, KV head, head group)
 * to finish merges its splits. The planner takes proportional splits for
 * full attention and windows of at least 2,048 keys when there is enough
 * work and their grid fits one wave of the device, uniform splits otherwise.
 * The partial results and the ticket counters live
 * in a library-owned per-device workspace: it grows on demand outside stream
 * capture; under capture a call that would need to grow it fails with
 * FP8PD_ERR_CAPTURE_WORKSPACE (call fp8pd_reserve_workspace, or run the call
 * once eagerly, before capturing).
 */
int fp8_paged_decode_attention(const fp8pd_tensor* q, const fp8pd_tensor* k_pages,
                               const fp8pd_tensor* v_pages, const fp8pd_tensor* k_scale,
                               const fp8pd_tensor* v_scale, const fp8pd_tensor* block_table,
                               const fp8pd_tensor* seq_lens, int32_t window,
                               const fp8pd_tensor* sinks, float sm_scale, fp8pd_tensor* out,
                               fp8pd_stream_t stream);

/*
 * fp8_kv_append -- quantize one new token per sequence and store it.
 *
 * For each b and KV head h, with p = positions[b], page = block_table[b, p / ps]:
 *   k_pages[page, p % ps, h, d] = E4M3_RNE_SAT( float(k_new[b, h, d]) / ks )
 * and the same for V. The division is IEEE float32 round-to-nearest; the
 * rounding to E4M3 is round-to-nearest-even, saturating to +-448 (a NaN
 * input gives the NaN code). A per-head or per-page scale is read only:
 * ks = k_scale(page, h). A per-token scale ([num_pages, ps, Hkv]) is the new
 * token's own, ks = max_d |k_new[b, h, d]| / 448 in IEEE float32 (NaN entries
 * skipped, 1 for an all-zero row), and is written to k_scale[page, p % ps, h].
 * With sub-row groups ([num_pages, ps, Hkv, G], G a power of two up to 16
 * dividing D) each run of D / G entries takes and writes its own scale.
 * Nothing else in the pools or scales is written. The new token is then visible to an attention call with
 * seq_lens[b] = p + 1 (the "Lecture 8" page's kv-cache update before the
 * decode attention).
 *
 * Arguments:
 *   k_new, v_new  bf16 [B, Hkv, D], any strides.
 *   k_pages,      uint8 [num_pages, ps, Hkv, D], as for the attention
 *   v_pages       (stride[3] must be 1; no alignment rule).
 *   scales        k_scale / v_scale as for the attention.
 *   block_table   int32 [B, max_pages]; stride[0] may be 0 (every b uses one row,
 *                 e.g. to write many tokens of one sequence in one call).
 *   positions     int32 [B].
 * One kernel launch; no workspace. Two entries that name the same slot race.
 */
int fp8_kv_append(const fp8pd_tensor* k_new, const fp8pd_tensor* v_new, fp8pd_tensor* k_pages,
                  fp8pd_tensor* v_pages, const fp8pd_scales* scales,
                  const fp8pd_tensor* block_table, const fp8pd_tensor* positions,
                  fp8pd_stream_t stream);


/*
 * fp8_paged_decode_append_attention -- fp8_kv_append followed by
 * fp8_paged_decode_attention, in one kernel launch.
 *
 * For each sequence b, with pos = positions[b]: the new token (k_new[b],
 * v_new[b], bf16 [B, Hkv, D]) is quantized exactly as fp8_kv_append does
 * (E4M3 code = round-to-nearest-even(float32 x / scale), saturated to +-448,
 * with the scale of the page that holds position pos, or with a per-token
 * form the token's own max|x| / 448, which is written too), written at position
 * pos of the pools, and the query then attends over the pos + 1 keys
 * 0 .. pos, the new one included -- the result of fp8_kv_append(..., positions)
 * followed by fp8_paged_decode_attention(..., seq_lens = positions + 1),
 * codes bit-identical and attention within float32 rounding. The block of
 * the launch that holds position pos quantizes the token, stores it (once
 * per KV head) and uses the codes it computed, so no block depends on
 * another's write. The Lecture 8 page ("In-kernel KV cache update") states
 * the order: the cache is updated, then read.
 *
 * Arguments: as fp8_paged_decode_attention, plus k_new / v_new (bf16
 * [B, Hkv, D], any strides) and positions (int32 [B]) in place of seq_lens;
 * the pools are written. A position outside [0, max_pages * page_size) sets
 * FP8PD_FLAG_POS_OOB and that sequence's output is 0, nothing is written; a
 * block-table entry outside the pool sets FP8PD_FLAG_PAGE_OOB. Runs the split
 * kernel (uniform or proportional splits). Workspace rules as fp8_paged_decode_attention.
 */
int fp8_paged_decode_append_attention(const fp8pd_tensor* q, const fp8pd_tensor* k_new,
                                      const fp8pd_tensor* v_new, fp8pd_tensor* k_pages,
                                      fp8pd_tensor* v_pages, const fp8pd_tensor* k_scale,
                                      const fp8pd_tensor* v_scale, const fp8pd_tensor* block_table,
                                      const fp8pd_tensor* positions, int32_t window,
                                      const fp8pd_tensor* sinks, float sm_scale, fp8pd_tensor* out,
                                      fp8pd_stream_t stream);
/*
 * fp8_paged_decode_attention_partial -- decode attention over a slice of each
 * sequence's keys, left unnormalized, for context-parallel split-KV: each GPU
 * holds part of a long sequence's pages, attends its slice, and the slices'
 * results are merged by fp8pd_combine_partials (the log-sum-exp combine of
 * splits; the solution page's "Why it happens": a grid over (sequence, KV
 * head, split), splitting a long sequence's keys being what keeps every SM --
 * here every GPU -- busy).
 *
 * For each b and query head hq, with the keys [lo, hi) = the window's range
 * of the L = seq_lens[b] keys (as fp8_paged_decode_attention) cut to
 * [key_ranges[b, 0], key_ranges[b, 1]) (the whole range when key_ranges is
 * NULL), and s2_t = sm_scale * log2(e) * q . K(t):
 *   part_ml[b, hq, 0] = m = max_t s2_t             (-inf with no keys)
 *   part_ml[b, hq, 1] = l = sum_t 2^(s2_t - m)     (0 with no keys)
 *   part_o[b, hq, :]  =     sum_t 2^(s2_t - m) V(t) (0 with no keys)
 * There is no sink term: fp8pd_combine_partials adds it once. Only the pages
 * holding attended keys are read, so a rank's block table may mark every
 * other entry unused (-1).
 *
 * Arguments: as fp8_paged_decode_attention without sinks, plus
 *   key_ranges  int32 [B, 2] (begin, end) or NULL, any strides;
 *   part_o      float32 [B, Hq, D], contiguous, 16-byte aligned;
 *   part_ml     float32 [B, Hq, 2], contiguous, 8-byte aligned.
 * Same planning, workspace and error rules as fp8_paged_decode_attention
 * (FP8PD_OPT_COMPUTE applies).
 */
int fp8_paged_decode_attention_partial(const fp8pd_tensor* q, const fp8pd_tensor* k_pages,
                                       const fp8pd_tensor* v_pages, const fp8pd_tensor* k_scale,
                                       const fp8pd_tensor* v_scale,
                                       const fp8pd_tensor* block_table,
                                       const fp8pd_tensor* seq_lens,
                                       const fp8pd_tensor* key_ranges, int32_t window,
                                       float sm_scale, fp8pd_tensor* part_o,
                                       fp8pd_tensor* part_ml, fp8pd_stream_t stream);

/*
 * fp8pd_combine_partials -- merges R partial results per (sequence, query
 * head), as fp8_paged_decode_attention_partial writes them, into the
 * attention output, adding the sink once (the log-sum-exp combine of splits;
 * the solution page's "Expected result" for the sink: one logit per query
 * head in the denominator, no value):
 *   M = max(max_r m_r, sink * log2 e)
 *   den = sum_r l_r 2^(m_r - M) + 2^(sink * log2 e - M)
 *   out = sum_r O_r 2^(m_r - M) / den              (0 when den is 0)
 * A rank with no keys (m = -inf) contributes nothing, whatever its O holds.
 *   part_o   float32 [R, B, Hq, D], contiguous, 16-byte aligned, D % 4 == 0;
 *   part_ml  float32 [R, B, Hq, 2], contiguous, 8-byte aligned; 1 <= R <= 1024;
 *   sinks    float32 [Hq] or NULL;
 *   out      float32 [B, Hq, D]; stride[2] must be 1, rows 16-byte aligned.
 * One kernel launch; no workspace.
 */
int fp8pd_combine_partials(const fp8pd_tensor* part_o, const fp8pd_tensor* part_ml,
                           const fp8pd_tensor* sinks, fp8pd_tensor* out, fp8pd_stream_t stream);

/*
 * fp8_paged_decode_attention_noalloc -- the same operation, allocating nothing.
 *
 * This entry point has no counterpart in the method's description; it is for
 * callers that cannot allocate device memory where they run attention (an
 * allocator-free runtime, a memory manager that owns all of the device's
 * memory, or code that must not call cudaMalloc because it synchronizes the
 * device). Arguments, results and errors are those of
 * fp8_paged_decode_attention. The split scratch is a fixed 8 MiB array inside
 * the library's device image (every GPU that loads the library holds it until
 * the process exits) instead of the allocated workspace; a call whose plan
 * needs more returns FP8PD_ERR_TOO_LARGE and launches nothing. No call
 * allocates or frees memory: the first call on a device looks up the array's
 * device address once (cudaGetSymbolAddress), so make that first call before
 * any stream capture. Each call clears the array's ticket counters with an
 * asynchronous memset on `stream`. All calls on a device share the array, and
 * the array keeps the last call's contents: calls that overlap on the GPU
 * (different streams without ordering) race and give wrong results.
 */
int fp8_paged_decode_attention_noalloc(const fp8pd_tensor* q, const fp8pd_tensor* k_pages,
                                       const fp8pd_tensor* v_pages, const fp8pd_tensor* k_scale,
                                       const fp8pd_tensor* v_scale,
                                       const fp8pd_tensor* block_table,
                                       const fp8pd_tensor* seq_lens, int32_t window,
                                       const fp8pd_tensor* sinks, float sm_scale,
                                       fp8pd_tensor* out, fp8pd_stream_t stream);

/* What a call with these arguments would launch, without launching it. */
typedef struct fp8pd_plan_info {
  int32_t num_splits;        /* uniform splits: blocks per (sequence, KV head, head group);
                                proportional splits: 0 */
  int32_t head_groups;       /* ceil(G / 8) query-head groups per KV head */
  int32_t grid_blocks;       /* thread blocks of the launch */
  int32_t combine;           /* 1 if partial results are merged (workspace used) */
  uint64_t workspace_bytes;  /* split workspace the call needs (0 if none) */
  int32_t schedule;          /* 1 = uniform splits, 3 = proportional splits */
  int32_t warps;             /* warps of the launch */
} fp8pd_plan_info;

/* Plans a decode-attention call (same argument rules; nothing launched). */
int fp8pd_plan(const fp8pd_tensor* q, const fp8pd_tensor* k_pages,
               const fp8pd_tensor* block_table, int32_t window, fp8pd_plan_info* info);

/*
 * fp8pd_e4m3_encode -- E4M3 codes of float32 values, with the rounding the
 * append applies to its quotients: round to nearest, ties to an even
 * mantissa, magnitudes above 448 and infinities saturated to +-448, NaN to
 * the NaN code with its sign, -0 to 0x80 (the E4M3 RNE with saturation named
 * by the solution page's "Supported scope" for the cache's quantizer).
 *   x      float32 [n] in device memory, any stride >= 0.
 *   codes  uint8 [n] in device memory, any stride >= 0 (written).
 * One kernel launch; n = 0 launches nothing (the data pointers must still be
 * non-NULL, as for every descriptor).
 */
int fp8pd_e4m3_encode(const fp8pd_tensor* x, fp8pd_tensor* codes, fp8pd_stream_t stream);

/* Grows the current device's split workspace to at least `bytes` (never
 * shrinks). Must not be called while a stream of the device is capturing. */
int fp8pd_reserve_workspace(uint64_t bytes);

/* Waits for `stream`, returns the current device's error word in *flags (may
 * be NULL) and clears it. */
int fp8pd_check_errors(fp8pd_stream_t stream, uint32_t* flags);

/* Options (process-wide). */
enum {
  FP8PD_OPT_NUM_SPLITS = 1,  /* 0 = planner chooses (default); n > 0 asks for n splits (raised
                                so that no split covers more than 8,192 keys, capped at 256
                                splits and at the number of pages) */
  FP8PD_OPT_SCHEDULE = 2,    /* 0 = planner chooses (default); 1 = uniform splits;
                                3 = proportional splits where they apply (B <= 1024, no
                                forced split count), else uniform splits; any other value
                                is refused with FP8PD_ERR_ARG */
  FP8PD_OPT_K_DECODE = 3,    /* the QK contraction: 0 = K decoded to f16 by bit assembly,
                                1 = by the hardware cvt.rn.f16x2.e4m3x2 (both into f16 MMAs),
                                2 = K's E4M3 bytes into E4M3 MMAs, q as two exact E4M3 terms
                                (no decode of K); mode 2 applies with the cvt decode of V and
                                page or head scales, mode 1 runs otherwise. Default 1. */
  FP8PD_OPT_V_DECODE = 4,    /* the same for V (default 1) */
  FP8PD_OPT_WAIT_POLLS = 6,  /* polls of a tile copy's barrier before the wait gives up and sets
                                FP8PD_FLAG_TIMEOUT; each poll sleeps at most 20 us. Default
                                131,072 (about 2.6 s); 1 .. 1,048,576 */
  FP8PD_OPT_TEST_STALL = 7,  /* test hook of the timeout path, 0 (default) or 1: warp 0 of the
                                first block of each attention launch never issues its first tile
                                copy, so that one wait runs out; the keys of that warp are left
                                out and FP8PD_FLAG_TIMEOUT is set. No copy is in flight on the
                                stalled stage, so the launch ends normally. */
  FP8PD_OPT_COMPUTE = 8,     /* numerical path of the attention: 0 (default) = f32 compute (K and
                                V decoded exactly, q exact in f16, P as an f16 hi + lo pair; max
                                |err| <= 1e-3 * max(1, |ref|)); 1 = fp8 compute (the solution
                                page's compute="fp8": q rounded once to E4M3 per query head after
                                a power-of-two scale, each weight exp(s - running max) * v_scale /
                                max v_scale * 2^8 rounded once to E4M3, K and V bytes into E4M3
                                MMAs; the page holds it to 1.5e-1). Per-token scales are refused
                                on the fp8 path with FP8PD_ERR_UNSUPPORTED, never downgraded. */
  FP8PD_OPT_KERNEL = 9       /* the attention kernel: 0 = the planner's choice (default), 1 = the
                                split kernel (mma.sync tiles of 16 tokens per warp), 2 = the
                                tensor-memory kernel (tcgen05 MMAs on 128-token chunks,
                                accumulators in TMEM) where it applies -- head dim 64 or 128,
                                page or head scales, f32 compute, FP8PD_OPT_K_DECODE and
                                FP8PD_OPT_V_DECODE at 1, no timeout test hook -- else the split
                                kernel. Both give the same results within the f32 tolerance. */
};
int fp8pd_set_option(int32_t option, int64_t value);
int64_t fp8pd_get_option(int32_t option);

/* What the last attention call on this host thread launched. */
typedef struct fp8pd_run_info {
  int32_t schedule;          /* 1 = uniform splits, 3 = proportional splits */
  int32_t num_splits;
  int32_t head_groups;
  int32_t grid_blocks;
  int32_t combine;
  int32_t head_dim;
  int64_t calls;             /* attention calls made by this process */
  int64_t appends;           /* append calls made by this process */
  int64_t kernel_launches;   /* kernels this library launched in this process */
  int32_t compute;           /* FP8PD_OPT_COMPUTE of the last attention call (0 f32, 1 fp8) */
  int32_t kernel;            /* kernel of the last attention call: 1 split, 2 tensor-memory */
  int32_t dim_split;         /* warps sharing each tile stream of the split kernel, each on its
                                part of the head dim: 1, or (a build setting, 2 or 4) at
                                head_dim 512 with page or head scales, f32 compute, the cvt
                                decodes and no fused append */
} fp8pd_run_info;
int fp8pd_last_run_info(fp8pd_run_info* info);

/* Device timing of the library's own kernels (for benchmarks): while
 * enabled, each attention call records CUDA events around its kernel, and
 * each append call around its kernel, on the call's stream (eager calls only;
 * do not enable while a stream is capturing). fp8pd_timing_collect waits for
 * those events, returns the summed milliseconds and launch counts since the
 * last collect, and resets them. Enabling allocates events lazily. */
int fp8pd_timing_enable(int32_t on);
int fp8pd_timing_collect(double* attention_ms, int32_t* attention_launches, double* append_ms,
                         int32_t* append_launches);

/* Human-readable status text (static storage). */
const char* fp8pd_status_string(int32_t status);
/* cudaError_t of the last failed CUDA call on this host thread (0 if none). */
int32_t fp8pd_last_cuda_error(void);
int32_t fp8pd_version(void);

#ifdef __cplusplus
}
#endif
#endif /* FP8PD_H_ */
