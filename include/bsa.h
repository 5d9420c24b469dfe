/*
 * bsa.h - C ABI of the dynamic block-sparse attention library for long-context
 * decode and prefill on NVIDIA B200 (sm_100a). Shared library: libbsa.so.
 *
 * The method (cited by page title and section of the gist.science summaries):
 *   1. Score. Every 64-token KV block gets a score from a low-dimensional index
 *      (r = 16 index keys and queries, RTPurbo "Full Attention Strikes Back",
 *      Methodology §2): per token t, u_t = idx_scale * sum_h w_h ReLU(q_idx[h] . k_idx[t])
 *      over the query heads h of the kv group (SpotAttention, Methodology §1);
 *      the block score is the max of u over the block's tokens (prefill: over the
 *      query block x key block tile).
 *   2. Select. Keep the sink blocks and the local (recency) blocks; among the
 *      remaining candidate blocks keep the shortest prefix, in order of score
 *      (ties to the lower block id), whose softmax mass over the candidates
 *      reaches p, capped at k_max and floored at k_min (SpotAttention,
 *      Methodology §3; RTPurbo, Methodology §3). Prefill also keeps the current
 *      (diagonal) block (HGA, Central mechanism §2).
 *   3. Attend. Exact softmax attention over the token-level K/V of the kept
 *      blocks only (HGA, Central mechanism §4), causal within the diagonal block
 *      in prefill.
 *
 * Conventions for every entry point:
 *   - Every pointer argument except `stream` is a DEVICE pointer unless stated.
 *     The caller owns all memory; the library never allocates, frees or
 *     synchronizes, and keeps no global state apart from per-device launch
 *     parameters read once (SM count) and the TMA encode entry point.
 *   - All work is enqueued on `stream` (a cudaStream_t passed as void*; NULL =
 *     the legacy default stream). Calls return after the launch, not after the
 *     work; they are re-entrant on distinct output and workspace buffers.
 *   - Host-checkable errors (shapes, null pointers, alignment) return a status
 *     and launch nothing. Data errors found on the device (page id out of range,
 *     kept id out of range, non-finite score, a bounded wait that gave up) are
 *     OR-ed as BSA_DEV_* bits into *dev_status (int32, may be NULL); kernels
 *     never trap. A launch failure returns BSA_ERR_CUDA.
 *   - Supported shapes: block = 64, r = 16, d in {64, 128}, Hq % Hkv == 0,
 *     G = Hq / Hkv in {1, 2, 4, 8, 16}, k_min <= k_max <= 8192, contexts up to
 *     32768 blocks (2^21 tokens). bf16 tensors must be 16-byte aligned.
 */
#ifndef BSA_H
#define BSA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  BSA_OK = 0,
  BSA_ERR_INVALID_ARG = 1, /* bad argument; nothing launched */
  BSA_ERR_UNSUPPORTED = 2, /* valid but outside the supported shapes; nothing launched */
  BSA_ERR_WORKSPACE = 3,   /* workspace NULL or smaller than bsa_workspace_size() */
  BSA_ERR_CUDA = 4         /* a CUDA call or kernel launch failed */
} bsa_status_t;

/* Bits OR-ed into *dev_status by the kernels. */
#define BSA_DEV_BAD_PAGE 0x1   /* page id outside [0, num_pages) or block beyond extent: skipped */
#define BSA_DEV_BAD_KEPT 0x2   /* kept block id outside [0, nb): skipped */
#define BSA_DEV_NONFINITE 0x4  /* a computed block score was +-inf or NaN (a block that
                                  failed validation is written as -inf and reported as
                                  BSA_DEV_BAD_PAGE only) */
#define BSA_DEV_TIMEOUT 0x8    /* a bounded wait inside a kernel gave up; outputs invalid */
#define BSA_DEV_FP16_RANGE 0x10 /* a value outside the fp16 range: a prefill V value, or an
                                   index query scored against an FP4 index-key cache */

typedef enum { BSA_PHASE_DECODE = 0, BSA_PHASE_PREFILL = 1 } bsa_phase_t;

typedef enum { BSA_OP_SCORE = 0, BSA_OP_SELECT = 1, BSA_OP_DECODE = 2, BSA_OP_PREFILL = 3,
               BSA_OP_PBS_PERMUTE = 4 } bsa_op_t;

/* Addressing of one bf16 cache tensor (K, V or index keys), contiguous or paged.
 * Token t of sequence b, kv head g starts at element
 *     b*seq_stride + phys*block_stride + g*head_stride + (t % 64)*width
 * from `base`, where phys = page_table[b*page_table_stride + t/64] when
 * page_table != NULL and phys = t/64 otherwise, and width = d (K, V) or r
 * (index keys). The 64 rows of one block of one head are contiguous.
 * Contiguous [B, Hkv, T, w]: seq_stride = Hkv*T*w, block_stride = 64*w,
 * head_stride = T*w. Paged pool [P, Hkv, 64, w]: seq_stride = 0,
 * block_stride = Hkv*64*w, head_stride = 64*w, num_pages = P.
 * `extent` = number of elements addressable from base; every block read is
 * checked against it (and page ids against num_pages). */
typedef struct {
  const void* base;
  int64_t seq_stride;
  int64_t block_stride;
  int64_t head_stride;
  const int32_t* page_table; /* [B, page_table_stride] or NULL */
  int32_t page_table_stride;
  int32_t num_pages;         /* used when page_table != NULL */
  int64_t extent;
} bsa_cache_t;

/* Problem description shared by all entry points. */
typedef struct {
  int32_t phase;            /* bsa_phase_t */
  int32_t B, Hq, Hkv, d, r, block;
  int32_t T;                /* decode: capacity, every seq_lens[b] <= T; prefill: sequence length */
  const int32_t* seq_lens;  /* decode: device [B] tokens per sequence (>= 0), or NULL = T */
  int32_t n_sink;           /* sink blocks kept [0, n_sink) */
  int32_t n_local;          /* local blocks kept: decode [nb-n_local, nb), prefill [i-n_local, i) */
  int32_t k_max;            /* cap on dynamically selected blocks */
  int32_t k_min;            /* floor on dynamically selected blocks (<= k_max) */
  float p;                  /* top-p threshold; <= 0: none, >= 1: all (then capped) */
  float idx_scale;          /* index score scale; 0 = 1/sqrt(r) */
  float attn_scale;         /* softmax scale; 0 = 1/sqrt(d) */
  const float* head_w;      /* device [Hq] non-negative index-head weights, or NULL = 1/G */
  const float* head_p;      /* device [Hkv] top-p per kv head, or NULL = p for every head.
                               A head with p <= 0 and k_min = 0 is a local head (RTPurbo,
                               Methodology §1: local heads keep sinks + a sliding window,
                               retrieval heads select dynamically): it keeps only its
                               reserved blocks, and the scorers skip it (its block_scores
                               are left unwritten). */
  int32_t idx_heads;        /* index heads per kv group: 0 = one per query head (G; q_idx
                               has Hq rows and head_w Hq entries), 1 = one per group (SparDA,
                               Main innovations §2: a compact indexer; q_idx has Hkv rows,
                               head_w Hkv entries or NULL = 1). Other values: unsupported. */
  int32_t segment;          /* prefill only: 0, or the segment length (tokens, a multiple of
                               64, at most 8192) of a key order permuted inside segments by
                               bsa_pbs_permute (PBS-Attn, Methodology §2-§4). Selection then
                               keeps the query block's whole segment (instead of its diagonal
                               block), the sinks and the n_local blocks before the segment,
                               and chooses among the blocks of earlier segments. */
  const int32_t* key_pos;   /* prefill with segment > 0: device [B, Hkv, T] original position
                               of the key at each permuted position (bsa_pbs_permute's output);
                               bsa_prefill masks the keys of the query's own segment by it */
  int32_t group_size;       /* decode only: 0, or 16, 32 or 64 for two-level routing (HGA,
                               "Hierarchical Global Attention", Central mechanism §2): the
                               dynamically selected blocks are refined to their best groups
                               of group_size tokens. A group's score is the max of its tokens'
                               index scores; the k_groups best groups of the dynamic blocks
                               (score descending, lower group id on ties) are kept; sink and
                               local blocks stay whole. k_max * 64 / group_size <= 8192. */
  int32_t k_groups;         /* cap on the kept groups (group_size > 0) */
  float* group_scores;      /* group_size > 0: device [B, Hkv, nb * 64 / group_size] fp32
                               (16-byte aligned),
                               written by bsa_score_blocks (groups past a sequence: -inf) */
  int32_t* kept_groups;     /* group_size > 0: device [B, Hkv, max_kept] int32, written by
                               bsa_select_top_p: bit k of entry e set when group k of kept
                               block e is attended (all bits for sink and local blocks, 0 for
                               unused slots); read by bsa_decode */
} bsa_problem_t;

/* Length of one kept list: decode n_sink + n_local + k_max; prefill
 * 1 + n_sink + n_local + k_max, or segment/64 + n_sink + n_local + k_max with a
 * permuted key order (segment > 0). Unused slots of a list hold -1. */
int32_t bsa_max_kept(const bsa_problem_t* prob);

/* Workspace bytes `op` needs for `prob` (0 when none). Host only. */
bsa_status_t bsa_workspace_size(const bsa_problem_t* prob, int32_t op, size_t* bytes);

/* Step 1, block scores (SpotAttention, Methodology §1; RTPurbo, Methodology §2).
 * decode:  q_idx [B, Hq, r] bf16 (Hkv rows when idx_heads = 1)
 *          -> block_scores [B, Hkv, nb] fp32, nb = ceil(T/64);
 *          entries j >= ceil(seq_lens[b]/64) are set to -inf.
 * prefill: q_idx [B, Hq, T, r] bf16 (Hkv rows when idx_heads = 1)
 *          -> block_scores [B, Hkv, nqb, nqb] fp32,
 *          nqb = ceil(T/64); entry [i, j] written for j < i only.
 * k_idx addresses index keys (width r). */
bsa_status_t bsa_score_blocks(const bsa_problem_t* prob, const void* q_idx, bsa_cache_t k_idx,
                              float* block_scores, int32_t* dev_status, void* stream);

/* Step 2, selection (SpotAttention, Methodology §3; RTPurbo, Methodology §3 and
 * §5 - histogram thresholding without a sort over all blocks).
 * decode:  rows (b, g): kept [B, Hkv, max_kept] ascending block ids, -1 padded;
 *          kept_count [B, Hkv].
 * prefill: rows (b, g, i): kept [B, Hkv, nqb, max_kept], kept_count [B, Hkv, nqb];
 *          candidates are key blocks j < i outside the reserved set. */
bsa_status_t bsa_select_top_p(const bsa_problem_t* prob, const float* block_scores,
                              int32_t* kept, int32_t* kept_count, int32_t* dev_status,
                              void* stream);

/* Step 3, decode attention over the kept blocks (HGA, Central mechanism §4):
 * split-K flash-decode with an LSE merge.
 * q [B, Hq, d] bf16; k, v caches (width d); kept/kept_count from step 2.
 * Outputs: o [B, Hq, d] bf16, lse [B, Hq] fp32 (natural log; -inf and o = 0 when
 * a row has no visible token), o_f32 [B, Hq, d] fp32 or NULL. Workspace: see
 * bsa_workspace_size(BSA_OP_DECODE). */
bsa_status_t bsa_decode(const bsa_problem_t* prob, const void* q, bsa_cache_t k, bsa_cache_t v,
                        const int32_t* kept, const int32_t* kept_count, void* o, float* lse,
                        float* o_f32, void* workspace, size_t workspace_bytes,
                        int32_t* dev_status, void* stream);

/* Step 3, block-sparse causal prefill attention (HGA, Central mechanism §4).
 * q [B, Hq, T, d] bf16; k, v caches (width d) holding the T prompt tokens;
 * kept/kept_count from step 2 (prefill). Outputs: o [B, Hq, T, d] bf16,
 * lse [B, Hq, T] fp32, o_f32 [B, Hq, T, d] fp32 or NULL. V values must lie in
 * the fp16 range (|v| <= 65504): P.V runs on fp16 tensor-core operands. */
bsa_status_t bsa_prefill(const bsa_problem_t* prob, const void* q, bsa_cache_t k, bsa_cache_t v,
                         const int32_t* kept, const int32_t* kept_count, void* o, float* lse,
                         float* o_f32, void* workspace, size_t workspace_bytes,
                         int32_t* dev_status, void* stream);

/* Segment permutation of the keys for block-sparse prefill (PBS-Attn, "Sparser
 * Block-Sparse Attention via Token Permutation", Methodology §2-§3).
 * For every (sequence b, kv head g) of a prefill problem with prob->segment = S > 0:
 *   1. importance of key t = the mean, over the query rows of the last query block
 *      (positions [64 * (nqb - 1), T)) of the group's query heads, of the causal
 *      softmax probability that row gives t (scale attn_scale, keys t' <= the row's
 *      position); computed in float32 in a fixed order;
 *   2. inside each segment [s * S, min((s + 1) * S, T)) the keys are ordered by
 *      importance descending, equal importance by lower position;
 *   3. key_pos[b, g, p] = original position of the key at permuted position p, and
 *      the permuted copies k_perm, v_perm [B, Hkv, T, d] and kidx_perm [B, Hkv, T, r]
 *      (bf16, contiguous) hold row key_pos[b, g, p] of k, v and k_idx at row p.
 * Queries are not permuted, so no output permutation has to be undone. The permuted
 * caches then go to bsa_score_blocks, bsa_select_top_p and bsa_prefill with the same
 * problem (segment and key_pos set). q is [B, Hq, T, d] bf16; k, v (width d) and
 * k_idx (width r) are caches as elsewhere. Workspace: bsa_workspace_size with
 * BSA_OP_PBS_PERMUTE. Runs four kernels on `stream`. */
bsa_status_t bsa_pbs_permute(const bsa_problem_t* prob, const void* q, bsa_cache_t k,
                             bsa_cache_t v, bsa_cache_t k_idx, void* k_perm, void* v_perm,
                             void* kidx_perm, int32_t* key_pos, void* workspace,
                             size_t workspace_bytes, int32_t* dev_status, void* stream);

/* ------------------------------------------------------------------------
 * 4-bit index-key cache (SpotAttention, Methodology §4: the selector's K cache
 * may be stored as microscaled INT4 or FP4, about 3.5x smaller than bf16; the
 * backbone's K/V cache is untouched).
 *
 * Format. Each token's r = 16 index-key elements are 16 4-bit codes plus one
 * E4M3 (FP8) scale byte: 9 bytes instead of 32. A code is sign-magnitude: bit 3
 * = sign, bits 0-2 = magnitude index m. FP4: magnitude = E2M1 value of m
 * (0, 0.5, 1, 1.5, 2, 3, 4, 6); INT4: magnitude = m (0..7). One fp32 scale g
 * covers the whole cache. Element c of a token is
 *     k[c] = +-magnitude(m_c) * e4m3(scale) * g.
 * Storage is one 576-byte record per (sequence, kv head, 64-token block): 64
 * tokens x 8 bytes of codes (byte c holds element 2c in its low nibble and
 * element 2c+1 in its high nibble), then the 64 scale bytes. Tokens t >= T_b of
 * a partial last block hold zero codes and a zero scale.
 *
 * Addressing counts RECORDS: the record of block j of sequence b, kv head g is
 *     records + 576 * (b*seq_stride + phys*block_stride + g*head_stride)
 * with phys = page_table[b*page_table_stride + j] when page_table != NULL and
 * phys = j otherwise. Contiguous [B, Hkv, nb]: seq_stride = Hkv*nb,
 * block_stride = 1, head_stride = nb. Paged [P, Hkv]: seq_stride = 0,
 * block_stride = Hkv, head_stride = 1, num_pages = P. `extent` = records
 * addressable from `records`. `records` must be 16-byte aligned.
 * ---------------------------------------------------------------------- */
#define BSA_QIDX_RECORD_BYTES 576

typedef enum { BSA_IDX_FP4 = 1, BSA_IDX_INT4 = 2 } bsa_idx_format_t;

typedef struct {
  void* records;             /* device, 576-byte records as above */
  float* gscale;             /* device, one float: the cache scale g */
  int64_t seq_stride;
  int64_t block_stride;
  int64_t head_stride;
  const int32_t* page_table; /* [B, page_table_stride] or NULL */
  int32_t page_table_stride;
  int32_t num_pages;         /* used when page_table != NULL */
  int64_t extent;            /* records */
  int32_t format;            /* bsa_idx_format_t */
} bsa_qcache_t;

/* Quantise the bf16 index keys k_idx (width r = 16) of every token t < seq_lens[b]
 * (decode problems) into `out`, writing every record of blocks [0, ceil(T_b/64))
 * and *out.gscale. qmax = 6 (FP4) or 7 (INT4). Every step is float32 with
 * round-to-nearest-even:
 *   1. A = max |k| over all those tokens; g = A / (qmax * 448), or 1 when A = 0;
 *   2. per token: a = max_c |k[c]|, s = (a / qmax) / g; scale = the E4M3 value
 *      nearest to s (ties to the even mantissa), 448 when s >= 448;
 *   3. S = e4m3(scale); if S = 0 every magnitude is 0; else t = S * g and per
 *      element m_c = the magnitude nearest to |k[c] / t| (ties to the even index),
 *      at most 7; the sign bit is the sign bit of k[c].
 * Runs three kernels on `stream` and uses *out.gscale as scratch in between. */
bsa_status_t bsa_quantize_index_keys(const bsa_problem_t* prob, bsa_cache_t k_idx,
                                     bsa_qcache_t out, int32_t* dev_status, void* stream);

/* Step 1 (decode) on a 4-bit index-key cache: as bsa_score_blocks, with the index
 * keys of `k_idx` dequantised exactly (codes and scales are exact in bf16; the
 * E4M3 scale and g multiply the head sum, ReLU being positively homogeneous).
 * Prefill problems return BSA_ERR_UNSUPPORTED. */
bsa_status_t bsa_score_blocks_q(const bsa_problem_t* prob, const void* q_idx, bsa_qcache_t k_idx,
                                float* block_scores, int32_t* dev_status, void* stream);

/* Size of the fixed device scratch array used by bsa_decode_noalloc (8 MiB). */
#define BSA_NOALLOC_SCRATCH_BYTES (8u << 20)

/* Decode attention without a caller-provided workspace, for callers that cannot
 * allocate device memory (a host framework that owns every allocation, a plugin
 * with a memory budget fixed at start-up, a path where cudaMalloc would stall the
 * device). It has no counterpart on the pages: it is bsa_decode with its split-K
 * scratch placed in a file-scope device array of BSA_NOALLOC_SCRATCH_BYTES that
 * every device loading this library reserves until the process exits.
 * Arguments and outputs are those of bsa_decode minus the workspace. Returns
 * BSA_ERR_WORKSPACE, launching nothing, when the problem needs more scratch than
 * BSA_NOALLOC_SCRATCH_BYTES (bsa_workspace_size(BSA_OP_DECODE) tells how much).
 * Every call outside stream capture looks up the array's address on the current
 * device (cudaGetSymbolAddress), so a reset and re-created context is followed; a
 * call on a capturing stream reuses the address of the last uncaptured call on
 * that device and returns BSA_ERR_UNSUPPORTED when there was none, so make one
 * call before capturing. All calls on a device share the array: calls whose work
 * overlaps on the GPU race and must be serialised by the caller. Allocates and
 * frees nothing. */
bsa_status_t bsa_decode_noalloc(const bsa_problem_t* prob, const void* q, bsa_cache_t k,
                                bsa_cache_t v, const int32_t* kept, const int32_t* kept_count,
                                void* o, float* lse, float* o_f32, int32_t* dev_status,
                                void* stream);

/* Static description of a status code. */
const char* bsa_status_string(bsa_status_t status);

/* Last CUDA error string seen by this thread's most recent BSA_ERR_CUDA (or ""). */
const char* bsa_last_cuda_error(void);

#ifdef __cplusplus
}
#endif

#endif /* BSA_H */
