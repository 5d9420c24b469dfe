// Internal launch interface between the C ABI (bsa_api.cu) and the kernels.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/bsa.h"

namespace bsa {

// Device-side copy of a bsa_cache_t (strides in elements).
struct CacheView {
  const void* base;
  int64_t seq_stride, block_stride, head_stride;
  const int32_t* page_table;
  int32_t pt_stride, num_pages;
  int64_t extent;
};

struct ScoreDecodeArgs {
  const void* q_idx;          // [B, Hq, 16] bf16
  CacheView kidx;             // width 16
  const int32_t* seq_lens;    // [B] or null
  const float* head_w;        // [Hq] or null
  const float* head_p;        // [Hkv] or null; heads with p <= 0 (k_min = 0) are skipped
  int k_min;
  float* scores;              // [B*Hkv, nb_max]
  int32_t* status;
  int B, Hq, Hkv, G, T, nb_max, chunks_per_row;
  int64_t total_items;
  float idx_scale;
  int kfmt;                   // 0: bf16 keys; 1: FP4 / 2: INT4 records (kidx counts records)
  const float* gscale;        // 4-bit formats: the cache scale g (device)
  int group_size;             // 0, or 16 / 32 / 64: also write group maxima
  float* group_scores;        // [B*Hkv, nb_max * 64 / group_size]
};

// 4-bit index-key cache: 576-byte records of 64 tokens (codes, then scales).
constexpr int kQRecord = 576;

struct QuantArgs {
  CacheView src;              // bf16 index keys, width 16
  CacheView dst;              // records; strides and extent count records
  float* gscale;              // one float: amax scratch, then g
  const int32_t* seq_lens;    // [B] or null
  int32_t* status;
  int B, Hkv, T, nb, fmt;     // fmt 1 = FP4, 2 = INT4
};

struct ScorePrefillArgs {
  const void* q_idx;          // [B, Hq, T, 16] bf16
  CacheView kidx;             // width 16
  const float* head_w;
  const float* head_p;        // [Hkv] or null; heads with p <= 0 (k_min = 0) are skipped
  int k_min;
  float* scores;              // [B*Hkv, nqb, nqb]
  int32_t* status;
  int B, Hq, Hkv, G, T, nqb;
  float idx_scale;
};

struct SelectArgs {
  const float* scores;
  int32_t* kept;
  int32_t* kept_count;
  const int32_t* seq_lens;
  int32_t* status;
  int phase, B, Hkv, T, nb_max, nqb, max_kept;
  int seg_blocks;             // prefill: blocks per segment (1: the diagonal block alone)
  int n_sink, n_local, k_max, k_min;
  float p;
  const float* head_p;        // [Hkv] or null: per-head p
};

// Level-2 routing of decode rows: the best groups of the dynamically kept blocks.
struct GroupSelectArgs {
  const float* group_scores;  // [B*Hkv, nb_max * gpb]
  const int32_t* kept;        // [B*Hkv, max_kept]
  const int32_t* kept_count;  // [B*Hkv]
  const int32_t* seq_lens;
  int32_t* kept_groups;       // [B*Hkv, max_kept] bitmasks
  int32_t* status;
  int B, Hkv, T, nb_max, max_kept, n_sink, n_local, group_size, k_groups;
  int max_cand;               // k_max * 64 / group_size: candidate groups of a row, at most
};

struct DecodeArgs {
  const void* q;              // [B, Hq, d] bf16
  CacheView k, v;
  const int32_t* kept;        // [B*Hkv, max_kept]
  const int32_t* kept_count;  // [B*Hkv]
  const int32_t* seq_lens;
  void* o;                    // [B, Hq, d] bf16
  float* lse;                 // [B, Hq]
  float* o_f32;               // [B, Hq, d] or null
  float* part_o;              // [units, G, d]
  float* part_ml;             // [units, G, 2]
  const int32_t* kept_groups; // [B*Hkv, max_kept] group bitmasks, or null (whole blocks)
  int group_size;
  int32_t* status;
  int B, Hq, Hkv, G, d, T, max_kept, splits, split_len;
  float scale_log2;           // attn_scale * log2(e)
};

struct PrefillArgs {
  const void* q;              // [B, Hq, T, d] bf16
  CacheView k, v;
  const void* v16;            // [B*Hkv, Tpad, d] fp16 (workspace copy of V)
  const int32_t* kept;        // [B*Hkv*nqb, max_kept]
  const int32_t* kept_count;  // [B*Hkv*nqb]
  void* o;                    // [B, Hq, T, d] bf16
  float* lse;                 // [B, Hq, T]
  float* o_f32;               // or null
  int32_t* status;
  int B, Hq, Hkv, G, d, T, nqb, Tpad, max_kept;
  float scale_log2;
  int seg_blocks;             // blocks per segment of a permuted key order (1: none)
  const int32_t* key_pos;     // [B*Hkv, T] original key positions of a permuted order, or null
};

// Segment permutation of the keys (PBS-Attn): importance, sort, gather.
struct PbsArgs {
  const void* q;              // [B, Hq, T, d] bf16
  CacheView k, v, kidx;       // widths d, d, 16
  void* k_perm;               // [B*Hkv, T, d] bf16
  void* v_perm;               // [B*Hkv, T, d] bf16
  void* kidx_perm;            // [B*Hkv, T, 16] bf16
  int32_t* key_pos;           // [B*Hkv, T]
  float* ml;                  // [B*Hkv, G*64, nchunk, 2] per-chunk (max, sum), log2 units
  float* lse2;                // [B*Hkv, G*64] log-sum-exp of each last-block row, log2 units
  float* imp;                 // [B*Hkv, T] importance
  int32_t* status;
  int B, Hq, Hkv, G, d, T, nqb, nchunk, segment;
  float scale_log2;
};

// Launch with programmatic stream serialization: the kernel's CTAs may start while
// the previous kernel of the stream drains; the kernel orders itself after it with
// grid_dependency_wait(). Hides launch latency between the steps of the path.
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem,
                              cudaStream_t s, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...);
}

// Each launcher returns the cudaError_t of its launch.
cudaError_t launch_score_decode(const ScoreDecodeArgs& a, int num_sms, cudaStream_t s);
cudaError_t launch_quantize_index(const QuantArgs& a, int num_sms, cudaStream_t s);
cudaError_t launch_score_prefill(const ScorePrefillArgs& a, int num_sms, cudaStream_t s);
cudaError_t launch_select(const SelectArgs& a, cudaStream_t s);
cudaError_t launch_select_groups(const GroupSelectArgs& a, cudaStream_t s);
// Tensor maps of the K and V caches for decode: 64-row boxes (whole blocks) and
// 16-row boxes (kept 16-token quarters under two-level routing).
struct DecodeMaps {
  CUtensorMap k, v, k16, v16;
};
cudaError_t launch_decode(const DecodeArgs& a, const DecodeMaps& m, int num_units, int num_sms,
                          cudaStream_t s);
cudaError_t launch_v_to_f16(const PrefillArgs& a, cudaStream_t s);
cudaError_t launch_prefill_tc(const PrefillArgs& a, const CUtensorMap& tq, const CUtensorMap& tk,
                              const CUtensorMap& tv16, int* unit_counter, int num_sms,
                              cudaStream_t s);

cudaError_t launch_pbs_permute(const PbsArgs& a, int num_sms, cudaStream_t s);
// Key chunks (CTAs per (b, g)) of the importance passes.
int pbs_chunks(int T);

// Blocks per work item of the decode scorer (items are (row, chunk) pairs).
int score_decode_chunk_blocks();

// Records a CUDA error for bsa_last_cuda_error() and returns BSA_ERR_CUDA.
bsa_status_t record_cuda_error(cudaError_t e);

// Decode split-K geometry chosen on the host from the worst-case kept count.
void decode_split_plan(int rows, int max_kept, int num_sms, int* splits, int* split_len);

}  // namespace bsa
