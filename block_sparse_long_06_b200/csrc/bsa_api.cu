// C ABI of libbsa.so: argument validation, workspace sizing, TMA descriptor
// creation and kernel launches. No allocation, no synchronisation.
#include <cudaTypedefs.h>

#include <cmath>
#include <cstdio>
#include <cstring>
#include <mutex>

#include "bsa_internal.h"

namespace {

thread_local char g_last_cuda_error[256] = "";

bsa_status_t cuda_fail(cudaError_t e) {
  std::snprintf(g_last_cuda_error, sizeof(g_last_cuda_error), "%s: %s", cudaGetErrorName(e),
                cudaGetErrorString(e));
  return BSA_ERR_CUDA;
}

// SM count of the current device, read once per device.
int num_sms_current(int* out_dev = nullptr) {
  static int cache[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) dev = 0;
  if (out_dev) *out_dev = dev;
  if (dev < 0 || dev >= 64) {
    int n = 148;
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    return n;
  }
  if (cache[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
      n = 148;
    cache[dev] = n;
  }
  return cache[dev];
}

PFN_cuTensorMapEncodeTiled_v12000 get_encode() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// 2-D map over rows of `width` 16-bit elements, 64-wide boxes of `box_rows` rows,
// 128-byte swizzle.
bool make_map(CUtensorMap* m, const void* base, int64_t rows, int width, bool fp16,
              int box_rows = 64) {
  auto enc = get_encode();
  if (!enc) return false;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(width), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(width) * 2};
  cuuint32_t box[2] = {64, static_cast<cuuint32_t>(box_rows)};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(m, fp16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
                   const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool is_pow2_group(int G) { return G == 1 || G == 2 || G == 4 || G == 8 || G == 16; }

int nblocks(int T) { return (T + 63) / 64; }

// Shape checks shared by every entry point.
bsa_status_t check_problem(const bsa_problem_t* p) {
  if (p == nullptr) return BSA_ERR_INVALID_ARG;
  if (p->phase != BSA_PHASE_DECODE && p->phase != BSA_PHASE_PREFILL) return BSA_ERR_INVALID_ARG;
  if (p->B <= 0 || p->Hq <= 0 || p->Hkv <= 0 || p->T < 0) return BSA_ERR_INVALID_ARG;
  if (p->Hq % p->Hkv != 0) return BSA_ERR_INVALID_ARG;
  if (p->n_sink < 0 || p->n_local < 0 || p->k_max < 0 || p->k_min < 0) return BSA_ERR_INVALID_ARG;
  if (p->k_min > p->k_max) return BSA_ERR_INVALID_ARG;
  if (!std::isfinite(p->p) || !std::isfinite(p->idx_scale) || !std::isfinite(p->attn_scale))
    return BSA_ERR_INVALID_ARG;
  if (p->idx_scale < 0.f || p->attn_scale < 0.f) return BSA_ERR_INVALID_ARG;
  if (p->block != 64 || p->r != 16) return BSA_ERR_UNSUPPORTED;
  if (p->d != 64 && p->d != 128) return BSA_ERR_UNSUPPORTED;
  if (!is_pow2_group(p->Hq / p->Hkv)) return BSA_ERR_UNSUPPORTED;
  if (p->k_max > 8192) return BSA_ERR_UNSUPPORTED;
  if (nblocks(p->T) > 32768) return BSA_ERR_UNSUPPORTED;
  if (p->phase == BSA_PHASE_PREFILL && p->seq_lens != nullptr) return BSA_ERR_UNSUPPORTED;
  if (p->phase == BSA_PHASE_PREFILL && p->T <= 0) return BSA_ERR_INVALID_ARG;
  if (p->idx_heads != 0 && p->idx_heads != 1 && p->idx_heads != p->Hq / p->Hkv)
    return BSA_ERR_UNSUPPORTED;
  if (p->segment != 0) {
    if (p->phase != BSA_PHASE_PREFILL || p->segment < 0 || p->segment % 64 != 0)
      return BSA_ERR_INVALID_ARG;
    if (p->segment > 8192) return BSA_ERR_UNSUPPORTED;
  }
  if (p->group_size != 0) {
    if (p->phase != BSA_PHASE_DECODE || p->k_groups < 0) return BSA_ERR_INVALID_ARG;
    if (p->group_size != 16 && p->group_size != 32 && p->group_size != 64)
      return BSA_ERR_UNSUPPORTED;
    if (static_cast<int64_t>(p->k_max) * (64 / p->group_size) > 8192) return BSA_ERR_UNSUPPORTED;
  }
  return BSA_OK;
}

// Blocks per segment of a permuted key order (1 when the keys keep their order).
int seg_blocks_of(const bsa_problem_t* p) { return p->segment > 0 ? p->segment / 64 : 1; }

// Index heads per kv group: one per query head (the default) or one per group
// (SparDA, Main innovations §2: a compact indexer with one head per GQA group).
int idx_group(const bsa_problem_t* p) { return p->idx_heads == 1 ? 1 : p->Hq / p->Hkv; }

float idx_scale_of(const bsa_problem_t* p) {
  return p->idx_scale > 0.f ? p->idx_scale : 1.0f / std::sqrt(static_cast<float>(p->r));
}
float attn_scale_of(const bsa_problem_t* p) {
  return p->attn_scale > 0.f ? p->attn_scale : 1.0f / std::sqrt(static_cast<float>(p->d));
}

// Cache checks: non-null 16-byte aligned base, strides that keep every row 16-byte
// aligned and (for K/V, read through TMA) whole rows of `width`.
bsa_status_t check_cache(const bsa_cache_t& c, const bsa_problem_t* p, int width, bool rows_tma) {
  if (c.base == nullptr || !aligned16(c.base) || c.extent <= 0) return BSA_ERR_INVALID_ARG;
  const int64_t unit = rows_tma ? width : 8;
  if (c.seq_stride < 0 || c.block_stride <= 0 || c.head_stride < 0) return BSA_ERR_INVALID_ARG;
  if (c.seq_stride % unit || c.block_stride % unit || c.head_stride % unit)
    return BSA_ERR_INVALID_ARG;
  if (c.page_table != nullptr) {
    if (c.num_pages <= 0 || c.page_table_stride < nblocks(p->T)) return BSA_ERR_INVALID_ARG;
  }
  if (rows_tma && c.extent / width > 0x7fffffffLL) return BSA_ERR_UNSUPPORTED;
  return BSA_OK;
}

bsa::CacheView view(const bsa_cache_t& c) {
  bsa::CacheView v;
  v.base = c.base;
  v.seq_stride = c.seq_stride;
  v.block_stride = c.block_stride;
  v.head_stride = c.head_stride;
  v.page_table = c.page_table;
  v.pt_stride = c.page_table_stride;
  v.num_pages = c.num_pages;
  v.extent = c.extent;
  return v;
}

struct DecodePlan {
  int splits, split_len, units;
  size_t part_o_bytes, part_ml_bytes;
};

DecodePlan decode_plan(const bsa_problem_t* p, int num_sms) {
  DecodePlan pl;
  const int rows = p->B * p->Hkv;
  const int mk = bsa_max_kept(p);
  bsa::decode_split_plan(rows, mk, num_sms, &pl.splits, &pl.split_len);
  pl.units = rows * pl.splits;
  const int G = p->Hq / p->Hkv;
  pl.part_o_bytes = static_cast<size_t>(pl.units) * G * p->d * sizeof(float);
  pl.part_ml_bytes = static_cast<size_t>(pl.units) * G * 2 * sizeof(float);
  return pl;
}

size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

// 4-bit index-key cache checks: 16-byte aligned records, record strides >= 0,
// a valid format and a scale pointer.
bsa_status_t check_qcache(const bsa_qcache_t& c, const bsa_problem_t* p) {
  if (c.records == nullptr || !aligned16(c.records) || c.gscale == nullptr || c.extent <= 0)
    return BSA_ERR_INVALID_ARG;
  if (c.format != BSA_IDX_FP4 && c.format != BSA_IDX_INT4) return BSA_ERR_INVALID_ARG;
  if (c.seq_stride < 0 || c.block_stride <= 0 || c.head_stride < 0) return BSA_ERR_INVALID_ARG;
  if (c.page_table != nullptr) {
    if (c.num_pages <= 0 || c.page_table_stride < nblocks(p->T)) return BSA_ERR_INVALID_ARG;
  }
  return BSA_OK;
}

bsa::CacheView qview(const bsa_qcache_t& c) {
  bsa::CacheView v;
  v.base = c.records;
  v.seq_stride = c.seq_stride;
  v.block_stride = c.block_stride;
  v.head_stride = c.head_stride;
  v.page_table = c.page_table;
  v.pt_stride = c.page_table_stride;
  v.num_pages = c.num_pages;
  v.extent = c.extent;
  return v;
}

// Workspace of bsa_pbs_permute: per-chunk row statistics, row log-sum-exps, importance.
struct PbsWorkspace {
  size_t ml, lse2, imp, total;
};
PbsWorkspace pbs_workspace(const bsa_problem_t* p) {
  const size_t bh = static_cast<size_t>(p->B) * p->Hkv;
  const size_t rows = bh * (p->Hq / p->Hkv) * 64;
  PbsWorkspace w;
  w.ml = 0;
  w.lse2 = align256(rows * bsa::pbs_chunks(p->T) * 2 * sizeof(float));
  w.imp = w.lse2 + align256(rows * sizeof(float));
  w.total = w.imp + align256(bh * static_cast<size_t>(p->T) * sizeof(float));
  return w;
}

}  // namespace

namespace bsa {
bsa_status_t record_cuda_error(cudaError_t e) { return cuda_fail(e); }
}  // namespace bsa

extern "C" {

int32_t bsa_max_kept(const bsa_problem_t* p) {
  if (p == nullptr) return 0;
  const int32_t base = p->n_sink + p->n_local + p->k_max;
  if (p->phase != BSA_PHASE_PREFILL) return base;
  return base + (p->segment > 0 ? p->segment / 64 : 1);
}

bsa_status_t bsa_workspace_size(const bsa_problem_t* p, int32_t op, size_t* bytes) {
  if (bytes == nullptr) return BSA_ERR_INVALID_ARG;
  *bytes = 0;
  bsa_status_t st = check_problem(p);
  if (st != BSA_OK) return st;
  switch (op) {
    case BSA_OP_SCORE:
    case BSA_OP_SELECT:
      return BSA_OK;
    case BSA_OP_DECODE: {
      if (p->phase != BSA_PHASE_DECODE) return BSA_ERR_INVALID_ARG;
      const DecodePlan pl = decode_plan(p, num_sms_current());
      *bytes = align256(pl.part_o_bytes) + align256(pl.part_ml_bytes);
      return BSA_OK;
    }
    case BSA_OP_PREFILL: {
      if (p->phase != BSA_PHASE_PREFILL) return BSA_ERR_INVALID_ARG;
      const int64_t Tpad = static_cast<int64_t>(nblocks(p->T)) * 64;
      *bytes = align256(static_cast<size_t>(p->B) * p->Hkv * Tpad * p->d * 2) + 256;
      return BSA_OK;
    }
    case BSA_OP_PBS_PERMUTE: {
      if (p->phase != BSA_PHASE_PREFILL || p->segment <= 0) return BSA_ERR_INVALID_ARG;
      *bytes = pbs_workspace(p).total;
      return BSA_OK;
    }
    default:
      return BSA_ERR_INVALID_ARG;
  }
}

bsa_status_t bsa_score_blocks(const bsa_problem_t* p, const void* q_idx, bsa_cache_t k_idx,
                              float* block_scores, int32_t* dev_status, void* stream) {
  bsa_status_t st = check_problem(p);
  if (st != BSA_OK) return st;
  if (q_idx == nullptr || block_scores == nullptr || !aligned16(q_idx)) return BSA_ERR_INVALID_ARG;
  if (p->group_size > 0 && (p->group_scores == nullptr || !aligned16(p->group_scores)))
    return BSA_ERR_INVALID_ARG;
  if ((st = check_cache(k_idx, p, p->r, false)) != BSA_OK) return st;
  const int num_sms = num_sms_current();
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e;
  if (p->phase == BSA_PHASE_DECODE) {
    bsa::ScoreDecodeArgs a{};
    a.q_idx = q_idx;
    a.kidx = view(k_idx);
    a.seq_lens = p->seq_lens;
    a.head_w = p->head_w;
    a.head_p = p->head_p;
    a.k_min = p->k_min;
    a.scores = block_scores;
    a.status = dev_status;
    a.B = p->B;
    a.G = idx_group(p);
    a.Hq = p->Hkv * a.G;   // index heads: q_idx rows and head weights
    a.Hkv = p->Hkv;
    a.T = p->T;
    a.nb_max = nblocks(p->T);
    const int cb = bsa::score_decode_chunk_blocks();
    a.chunks_per_row = (a.nb_max + cb - 1) / cb;
    a.total_items = static_cast<int64_t>(p->B) * p->Hkv * a.chunks_per_row;
    a.idx_scale = idx_scale_of(p);
    a.group_size = p->group_size;
    a.group_scores = p->group_scores;
    e = bsa::launch_score_decode(a, num_sms, s);
  } else {
    bsa::ScorePrefillArgs a{};
    a.q_idx = q_idx;
    a.kidx = view(k_idx);
    a.head_w = p->head_w;
    a.head_p = p->head_p;
    a.k_min = p->k_min;
    a.scores = block_scores;
    a.status = dev_status;
    a.B = p->B;
    a.G = idx_group(p);
    a.Hq = p->Hkv * a.G;   // index heads: q_idx rows and head weights
    a.Hkv = p->Hkv;
    a.T = p->T;
    a.nqb = nblocks(p->T);
    a.idx_scale = idx_scale_of(p);
    e = bsa::launch_score_prefill(a, num_sms, s);
  }
  return e == cudaSuccess ? BSA_OK : cuda_fail(e);
}

bsa_status_t bsa_quantize_index_keys(const bsa_problem_t* p, bsa_cache_t k_idx, bsa_qcache_t out,
                                     int32_t* dev_status, void* stream) {
  bsa_status_t st = check_problem(p);
  if (st != BSA_OK) return st;
  if (p->phase != BSA_PHASE_DECODE) return BSA_ERR_UNSUPPORTED;
  if ((st = check_cache(k_idx, p, p->r, false)) != BSA_OK) return st;
  if ((st = check_qcache(out, p)) != BSA_OK) return st;
  bsa::QuantArgs a{};
  a.src = view(k_idx);
  a.dst = qview(out);
  a.gscale = out.gscale;
  a.seq_lens = p->seq_lens;
  a.status = dev_status;
  a.B = p->B;
  a.Hkv = p->Hkv;
  a.T = p->T;
  a.nb = nblocks(p->T);
  a.fmt = out.format;
  const cudaError_t e = bsa::launch_quantize_index(a, num_sms_current(), static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? BSA_OK : cuda_fail(e);
}

bsa_status_t bsa_score_blocks_q(const bsa_problem_t* p, const void* q_idx, bsa_qcache_t k_idx,
                                float* block_scores, int32_t* dev_status, void* stream) {
  bsa_status_t st = check_problem(p);
  if (st != BSA_OK) return st;
  if (p->phase != BSA_PHASE_DECODE) return BSA_ERR_UNSUPPORTED;
  if (q_idx == nullptr || block_scores == nullptr || !aligned16(q_idx)) return BSA_ERR_INVALID_ARG;
  if (p->group_size > 0 && (p->group_scores == nullptr || !aligned16(p->group_scores)))
    return BSA_ERR_INVALID_ARG;
  if ((st = check_qcache(k_idx, p)) != BSA_OK) return st;
  bsa::ScoreDecodeArgs a{};
  a.q_idx = q_idx;
  a.kidx = qview(k_idx);
  a.seq_lens = p->seq_lens;
  a.head_w = p->head_w;
    a.head_p = p->head_p;
    a.k_min = p->k_min;
  a.scores = block_scores;
  a.status = dev_status;
  a.B = p->B;
  a.G = idx_group(p);
  a.Hq = p->Hkv * a.G;   // index heads: q_idx rows and head weights
  a.Hkv = p->Hkv;
  a.T = p->T;
  a.nb_max = nblocks(p->T);
  const int cb = bsa::score_decode_chunk_blocks();
  a.chunks_per_row = (a.nb_max + cb - 1) / cb;
  a.total_items = static_cast<int64_t>(p->B) * p->Hkv * a.chunks_per_row;
  a.idx_scale = idx_scale_of(p);
  a.kfmt = k_idx.format;
  a.gscale = k_idx.gscale;
  a.group_size = p->group_size;
  a.group_scores = p->group_scores;
  const cudaError_t e = bsa::launch_score_decode(a, num_sms_current(), static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? BSA_OK : cuda_fail(e);
}

bsa_status_t bsa_select_top_p(const bsa_problem_t* p, const float* block_scores, int32_t* kept,
                              int32_t* kept_count, int32_t* dev_status, void* stream) {
  bsa_status_t st = check_problem(p);
  if (st != BSA_OK) return st;
  if (block_scores == nullptr || kept == nullptr || kept_count == nullptr)
    return BSA_ERR_INVALID_ARG;
  if (p->group_size > 0 && (p->group_scores == nullptr || p->kept_groups == nullptr))
    return BSA_ERR_INVALID_ARG;
  bsa::SelectArgs a{};
  a.scores = block_scores;
  a.kept = kept;
  a.kept_count = kept_count;
  a.seq_lens = p->phase == BSA_PHASE_DECODE ? p->seq_lens : nullptr;
  a.status = dev_status;
  a.phase = p->phase;
  a.B = p->B;
  a.Hkv = p->Hkv;
  a.T = p->T;
  a.nb_max = nblocks(p->T);
  a.nqb = nblocks(p->T);
  a.max_kept = bsa_max_kept(p);
  a.n_sink = p->n_sink;
  a.n_local = p->n_local;
  a.k_max = p->k_max;
  a.k_min = p->k_min;
  a.p = p->p;
  a.head_p = p->head_p;
  a.seg_blocks = seg_blocks_of(p);
  cudaError_t e = bsa::launch_select(a, static_cast<cudaStream_t>(stream));
  if (e == cudaSuccess && p->group_size > 0) {
    // level 2: the best token groups of the kept blocks
    bsa::GroupSelectArgs ga{};
    ga.group_scores = p->group_scores;
    ga.kept = kept;
    ga.kept_count = kept_count;
    ga.seq_lens = p->seq_lens;
    ga.kept_groups = p->kept_groups;
    ga.status = dev_status;
    ga.B = p->B;
    ga.Hkv = p->Hkv;
    ga.T = p->T;
    ga.nb_max = nblocks(p->T);
    ga.max_kept = a.max_kept;
    ga.n_sink = p->n_sink;
    ga.n_local = p->n_local;
    ga.group_size = p->group_size;
    ga.k_groups = p->k_groups;
    ga.max_cand = p->k_max * (64 / p->group_size);
    e = bsa::launch_select_groups(ga, static_cast<cudaStream_t>(stream));
  }
  return e == cudaSuccess ? BSA_OK : cuda_fail(e);
}

bsa_status_t bsa_decode(const bsa_problem_t* p, const void* q, bsa_cache_t k, bsa_cache_t v,
                        const int32_t* kept, const int32_t* kept_count, void* o, float* lse,
                        float* o_f32, void* workspace, size_t workspace_bytes,
                        int32_t* dev_status, void* stream) {
  bsa_status_t st = check_problem(p);
  if (st != BSA_OK) return st;
  if (p->phase != BSA_PHASE_DECODE) return BSA_ERR_INVALID_ARG;
  if (q == nullptr || kept == nullptr || kept_count == nullptr || o == nullptr || lse == nullptr)
    return BSA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(o)) return BSA_ERR_INVALID_ARG;
  if ((st = check_cache(k, p, p->d, true)) != BSA_OK) return st;
  if ((st = check_cache(v, p, p->d, true)) != BSA_OK) return st;
  const int num_sms = num_sms_current();
  const DecodePlan pl = decode_plan(p, num_sms);
  const size_t need = align256(pl.part_o_bytes) + align256(pl.part_ml_bytes);
  if (workspace == nullptr || workspace_bytes < need || (reinterpret_cast<uintptr_t>(workspace) & 255))
    return BSA_ERR_WORKSPACE;
  if (p->group_size > 0 && p->kept_groups == nullptr) return BSA_ERR_INVALID_ARG;
  bsa::DecodeMaps maps;
  if (!make_map(&maps.k, k.base, k.extent / p->d, p->d, false) ||
      !make_map(&maps.v, v.base, v.extent / p->d, p->d, false))
    return cuda_fail(cudaErrorInvalidValue);
  if (p->group_size > 0) {
    if (!make_map(&maps.k16, k.base, k.extent / p->d, p->d, false, 16) ||
        !make_map(&maps.v16, v.base, v.extent / p->d, p->d, false, 16))
      return cuda_fail(cudaErrorInvalidValue);
  } else {
    // not read: every kept block is copied whole
    maps.k16 = maps.k;
    maps.v16 = maps.v;
  }
  bsa::DecodeArgs a{};
  a.q = q;
  a.k = view(k);
  a.v = view(v);
  a.kept = kept;
  a.kept_count = kept_count;
  a.seq_lens = p->seq_lens;
  a.o = o;
  a.lse = lse;
  a.o_f32 = o_f32;
  a.part_o = static_cast<float*>(workspace);
  a.part_ml = reinterpret_cast<float*>(static_cast<char*>(workspace) + align256(pl.part_o_bytes));
  a.status = dev_status;
  a.B = p->B;
  a.Hq = p->Hq;
  a.Hkv = p->Hkv;
  a.G = p->Hq / p->Hkv;
  a.d = p->d;
  a.T = p->T;
  a.max_kept = bsa_max_kept(p);
  a.splits = pl.splits;
  a.split_len = pl.split_len;
  a.scale_log2 = attn_scale_of(p) * 1.4426950408889634f;
  a.kept_groups = p->group_size > 0 ? p->kept_groups : nullptr;
  a.group_size = p->group_size;
  cudaError_t e = bsa::launch_decode(a, maps, pl.units, num_sms, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? BSA_OK : cuda_fail(e);
}

bsa_status_t bsa_prefill(const bsa_problem_t* p, const void* q, bsa_cache_t k, bsa_cache_t v,
                         const int32_t* kept, const int32_t* kept_count, void* o, float* lse,
                         float* o_f32, void* workspace, size_t workspace_bytes,
                         int32_t* dev_status, void* stream) {
  bsa_status_t st = check_problem(p);
  if (st != BSA_OK) return st;
  if (p->phase != BSA_PHASE_PREFILL) return BSA_ERR_INVALID_ARG;
  if (q == nullptr || kept == nullptr || kept_count == nullptr || o == nullptr || lse == nullptr)
    return BSA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(o) || (o_f32 && !aligned16(o_f32))) return BSA_ERR_INVALID_ARG;
  if (p->segment > 0 && p->key_pos == nullptr) return BSA_ERR_INVALID_ARG;
  if ((st = check_cache(k, p, p->d, true)) != BSA_OK) return st;
  if ((st = check_cache(v, p, p->d, false)) != BSA_OK) return st;
  const int nqb = nblocks(p->T);
  const int64_t Tpad = static_cast<int64_t>(nqb) * 64;
  const size_t v16_bytes = align256(static_cast<size_t>(p->B) * p->Hkv * Tpad * p->d * 2);
  const size_t need = v16_bytes + 256;
  if (workspace == nullptr || workspace_bytes < need || (reinterpret_cast<uintptr_t>(workspace) & 255))
    return BSA_ERR_WORKSPACE;
  const int64_t qrows = static_cast<int64_t>(p->B) * p->Hq * p->T;
  const int64_t vrows = static_cast<int64_t>(p->B) * p->Hkv * Tpad;
  if (qrows > 0x7fffffffLL || vrows > 0x7fffffffLL) return BSA_ERR_UNSUPPORTED;
  CUtensorMap tq, tk, tv;
  if (!make_map(&tq, q, qrows, p->d, false) || !make_map(&tk, k.base, k.extent / p->d, p->d, false) ||
      !make_map(&tv, workspace, vrows, p->d, true))
    return cuda_fail(cudaErrorInvalidValue);
  bsa::PrefillArgs a{};
  a.q = q;
  a.k = view(k);
  a.v = view(v);
  a.v16 = workspace;
  a.kept = kept;
  a.kept_count = kept_count;
  a.o = o;
  a.lse = lse;
  a.o_f32 = o_f32;
  a.status = dev_status;
  a.B = p->B;
  a.Hq = p->Hq;
  a.Hkv = p->Hkv;
  a.G = p->Hq / p->Hkv;
  a.d = p->d;
  a.T = p->T;
  a.nqb = nqb;
  a.Tpad = static_cast<int>(Tpad);
  a.max_kept = bsa_max_kept(p);
  a.scale_log2 = attn_scale_of(p) * 1.4426950408889634f;
  a.seg_blocks = seg_blocks_of(p);
  a.key_pos = p->segment > 0 ? p->key_pos : nullptr;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e = bsa::launch_v_to_f16(a, s);
  if (e != cudaSuccess) return cuda_fail(e);
  int* unit_counter = reinterpret_cast<int*>(static_cast<char*>(workspace) + v16_bytes);
  e = bsa::launch_prefill_tc(a, tq, tk, tv, unit_counter, num_sms_current(), s);
  return e == cudaSuccess ? BSA_OK : cuda_fail(e);
}

bsa_status_t bsa_pbs_permute(const bsa_problem_t* p, const void* q, bsa_cache_t k, bsa_cache_t v,
                             bsa_cache_t k_idx, void* k_perm, void* v_perm, void* kidx_perm,
                             int32_t* key_pos, void* workspace, size_t workspace_bytes,
                             int32_t* dev_status, void* stream) {
  bsa_status_t st = check_problem(p);
  if (st != BSA_OK) return st;
  if (p->phase != BSA_PHASE_PREFILL || p->segment <= 0) return BSA_ERR_INVALID_ARG;
  if (q == nullptr || k_perm == nullptr || v_perm == nullptr || kidx_perm == nullptr ||
      key_pos == nullptr)
    return BSA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k_perm) || !aligned16(v_perm) || !aligned16(kidx_perm) ||
      !aligned16(key_pos))
    return BSA_ERR_INVALID_ARG;
  if ((st = check_cache(k, p, p->d, false)) != BSA_OK) return st;
  if ((st = check_cache(v, p, p->d, false)) != BSA_OK) return st;
  if ((st = check_cache(k_idx, p, p->r, false)) != BSA_OK) return st;
  const PbsWorkspace ws = pbs_workspace(p);
  if (workspace == nullptr || workspace_bytes < ws.total ||
      (reinterpret_cast<uintptr_t>(workspace) & 255))
    return BSA_ERR_WORKSPACE;
  bsa::PbsArgs a{};
  a.q = q;
  a.k = view(k);
  a.v = view(v);
  a.kidx = view(k_idx);
  a.k_perm = k_perm;
  a.v_perm = v_perm;
  a.kidx_perm = kidx_perm;
  a.key_pos = key_pos;
  char* w = static_cast<char*>(workspace);
  a.ml = reinterpret_cast<float*>(w + ws.ml);
  a.lse2 = reinterpret_cast<float*>(w + ws.lse2);
  a.imp = reinterpret_cast<float*>(w + ws.imp);
  a.status = dev_status;
  a.B = p->B;
  a.Hq = p->Hq;
  a.Hkv = p->Hkv;
  a.G = p->Hq / p->Hkv;
  a.d = p->d;
  a.T = p->T;
  a.nqb = nblocks(p->T);
  a.nchunk = bsa::pbs_chunks(p->T);
  a.segment = p->segment;
  a.scale_log2 = attn_scale_of(p) * 1.4426950408889634f;
  const cudaError_t e =
      bsa::launch_pbs_permute(a, num_sms_current(), static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? BSA_OK : cuda_fail(e);
}

const char* bsa_status_string(bsa_status_t s) {
  switch (s) {
    case BSA_OK: return "ok";
    case BSA_ERR_INVALID_ARG: return "invalid argument";
    case BSA_ERR_UNSUPPORTED: return "unsupported shape or parameter";
    case BSA_ERR_WORKSPACE: return "workspace missing or too small";
    case BSA_ERR_CUDA: return "CUDA error";
    default: return "unknown status";
  }
}

const char* bsa_last_cuda_error(void) { return g_last_cuda_error; }

}  // extern "C"
