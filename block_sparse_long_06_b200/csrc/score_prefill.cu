// Prefill block scorer.
//
// For every (sequence b, kv head g, query block i) and key block j < i:
//   S[b,g,i,j] = idx_scale * max_{tq in block i, tq < T; tk in block j}
//                sum_{h in group g} w_h ReLU(q_idx[b,h,tq] . k_idx[b,g,tk])
// (SpotAttention, Methodology §1: weighted-ReLU selector score, run as one
//  matrix product; the O(T^2) cost of this step is the point SparDA,
//  "Problem statement", makes about block selection.)
//
// Design: one CTA (4 warps) per query-block row; warp w owns query tokens
// [16w, 16w+16). Its index-query fragments stay in registers for the whole row:
// mma.m16n8k16 with rows = (head pair, 8 query tokens), columns = 8 key tokens,
// K = r = 16 (same dim relabelling as the decode scorer, so each lane loads one
// 8-byte run per token). A lane then holds every head's dot product for its
// (tq, tk) pairs, so ReLU, weights and the head sum need no shuffles; the 64x64
// tile max is a per-lane running max plus one warp reduction, and the four
// warps' maxima are combined through shared memory in batches of key blocks.
#include "bsa_common.cuh"
#include "bsa_internal.h"

namespace bsa {
namespace {

constexpr int kWarps = 4;

BSA_DEVFN float max3f(float x, float y, float z) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(x), "f"(y), "f"(z));
  return r;
}
constexpr int kBatch = 32;  // key blocks per shared-memory combine

template <int HP>  // head pairs = ceil(G / 2)
__global__ void __launch_bounds__(kWarps * 32) score_prefill_kernel(const ScorePrefillArgs a) {
  __shared__ float pm[kWarps][kBatch];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int gid = lane >> 2, tig = lane & 3;
  const int BH = a.B * a.Hkv;
  const int i = a.nqb - 1 - static_cast<int>(blockIdx.x) / BH;  // heavy rows first
  const int bg = static_cast<int>(blockIdx.x) % BH;
  const int b = bg / a.Hkv, g = bg % a.Hkv;
  if (i <= 0) return;
  if (a.head_p != nullptr && a.k_min == 0 && !(a.head_p[g] > 0.f)) return;   // local head

  // query fragments: tq group tg (8 tokens), head pair hp
  uint32_t aq[2][HP][4];
  float w[HP][2];
  float2 w0p[HP], w1p[HP];   // first head's weight, half the second head's, duplicated for FFMA2
  const char* qbase = static_cast<const char*>(a.q_idx);
  const float dflt = 1.0f / static_cast<float>(a.G);
#pragma unroll
  for (int hp = 0; hp < HP; ++hp) {
    const int h0 = 2 * hp, h1 = 2 * hp + 1;
    w[hp][0] = h0 < a.G ? (a.head_w ? a.head_w[g * a.G + h0] : dflt) : 0.f;
    w[hp][1] = h1 < a.G ? (a.head_w ? a.head_w[g * a.G + h1] : dflt) : 0.f;
#pragma unroll
    for (int tg = 0; tg < 2; ++tg) {
      const int tq = i * kBlock + 16 * warp + 8 * tg + gid;
      const bool tv = tq < a.T;
      uint2 x0 = make_uint2(0u, 0u), x1 = make_uint2(0u, 0u);
      if (tv && h0 < a.G)
        x0 = *reinterpret_cast<const uint2*>(
            qbase + (((static_cast<int64_t>(b) * a.Hq + g * a.G + h0) * a.T + tq) * kR + 4 * tig) * 2);
      if (tv && h1 < a.G)
        x1 = *reinterpret_cast<const uint2*>(
            qbase + (((static_cast<int64_t>(b) * a.Hq + g * a.G + h1) * a.T + tq) * kR + 4 * tig) * 2);
      aq[tg][hp][0] = x0.x;
      aq[tg][hp][1] = x1.x;
      aq[tg][hp][2] = x0.y;
      aq[tg][hp][3] = x1.y;
    }
  }
#pragma unroll
  for (int hp = 0; hp < HP; ++hp) {
    w0p[hp] = make_float2(w[hp][0], w[hp][0]);
    w1p[hp] = make_float2(0.5f * w[hp][1], 0.5f * w[hp][1]);
  }
  // query tokens of this lane that exist (a ragged last query block)
  const bool q0v = i * kBlock + 16 * warp + gid < a.T;
  const bool q1v = i * kBlock + 16 * warp + 8 + gid < a.T;

  const char* kbase = static_cast<const char*>(a.kidx.base);
  float* out = a.scores + (static_cast<int64_t>(bg) * a.nqb + i) * a.nqb;

  for (int j0 = 0; j0 < i; j0 += kBatch) {
    const int jn = min(kBatch, i - j0);
    for (int jj = 0; jj < jn; ++jj) {
      const int j = j0 + jj;
      int64_t phys = j;
      bool ok = true;
      if (a.kidx.page_table != nullptr) {
        phys = a.kidx.page_table[static_cast<int64_t>(b) * a.kidx.pt_stride + j];
        ok = phys >= 0 && phys < a.kidx.num_pages;
      }
      const int64_t off = static_cast<int64_t>(b) * a.kidx.seq_stride + phys * a.kidx.block_stride +
                          static_cast<int64_t>(g) * a.kidx.head_stride;
      ok = ok && off >= 0 && off + kBlock * kR <= a.kidx.extent;
      float mx = 0.f;
      if (ok) {
        const char* kb = kbase + off * 2;
#pragma unroll
        for (int nt = 0; nt < 8; ++nt) {
          const uint2 kv = *reinterpret_cast<const uint2*>(kb + (nt * 8 + gid) * 32 + tig * 8);
#pragma unroll
          for (int tg = 0; tg < 2; ++tg) {
            // u = (key 2*tig, key 2*tig + 1): two-wide FMAs, head by head in order.
            // The ReLU of the pair's first head runs on the ALU pipe (max with 0), the
            // second head's on the FMA pipe: c + |c| is exactly 2c for c > 0 and +0
            // otherwise, so (w/2) * (c + |c|) + u rounds exactly as w * ReLU(c) + u.
            // Splitting the two keeps both pipes busy.
            float2 u = make_float2(0.f, 0.f);
#pragma unroll
            for (int hp = 0; hp < HP; ++hp) {
              float c[4] = {0.f, 0.f, 0.f, 0.f};
              mma_bf16(c, aq[tg][hp], kv.x, kv.y);
              u = __ffma2_rn(w0p[hp], make_float2(fmaxf(c[0], 0.f), fmaxf(c[1], 0.f)), u);
              u = __ffma2_rn(w1p[hp], make_float2(c[2] + fabsf(c[2]), c[3] + fabsf(c[3])), u);
            }
            const bool qv = tg == 0 ? q0v : q1v;
            if (qv) mx = max3f(mx, u.x, u.y);
          }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      } else {
        mx = -INFINITY;
        if (lane == 0 && warp == 0) report(a.status, BSA_DEV_BAD_PAGE);
      }
      if (lane == 0) pm[warp][jj] = mx;
    }
    __syncthreads();
    if (threadIdx.x < jn) {
      float m = pm[0][threadIdx.x];
#pragma unroll
      for (int ww = 1; ww < kWarps; ++ww) m = fmaxf(m, pm[ww][threadIdx.x]);
      // a computed score is >= 0; -inf marks a block that failed validation (its
      // BSA_DEV_BAD_PAGE is already reported)
      const float sc = a.idx_scale * m;
      out[j0 + threadIdx.x] = sc;
      if (m != -INFINITY && !isfinite(sc)) report(a.status, BSA_DEV_NONFINITE);
    }
    __syncthreads();
  }
}

// One index head per group (G = 1: SparDA's compact indexer, or Hq = Hkv). With a
// single weight w >= 0, max over pairs of w ReLU(q.k) = w ReLU(max over pairs of q.k)
// exactly (rounding of w * x is monotone in x), so the per-pair epilogue is one max.
// MMA rows are 16 query tokens (tokens gid and gid + 8 of the warp's 16).
__global__ void __launch_bounds__(kWarps * 32) score_prefill_g1_kernel(const ScorePrefillArgs a) {
  __shared__ float pm[kWarps][kBatch];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int gid = lane >> 2, tig = lane & 3;
  const int BH = a.B * a.Hkv;
  const int i = a.nqb - 1 - static_cast<int>(blockIdx.x) / BH;  // heavy rows first
  const int bg = static_cast<int>(blockIdx.x) % BH;
  const int b = bg / a.Hkv, g = bg % a.Hkv;
  if (i <= 0) return;
  if (a.head_p != nullptr && a.k_min == 0 && !(a.head_p[g] > 0.f)) return;   // local head
  const float w = a.head_w ? a.head_w[g] : 1.0f;
  const char* qbase = static_cast<const char*>(a.q_idx);
  uint32_t aq[4] = {0u, 0u, 0u, 0u};
  const int tq0 = i * kBlock + 16 * warp + gid, tq1 = tq0 + 8;
  const bool q0v = tq0 < a.T, q1v = tq1 < a.T;
  if (q0v) {
    const uint2 x = *reinterpret_cast<const uint2*>(
        qbase + (((static_cast<int64_t>(b) * a.Hq + g) * a.T + tq0) * kR + 4 * tig) * 2);
    aq[0] = x.x;
    aq[2] = x.y;
  }
  if (q1v) {
    const uint2 x = *reinterpret_cast<const uint2*>(
        qbase + (((static_cast<int64_t>(b) * a.Hq + g) * a.T + tq1) * kR + 4 * tig) * 2);
    aq[1] = x.x;
    aq[3] = x.y;
  }
  const char* kbase = static_cast<const char*>(a.kidx.base);
  float* out = a.scores + (static_cast<int64_t>(bg) * a.nqb + i) * a.nqb;
  for (int j0 = 0; j0 < i; j0 += kBatch) {
    const int jn = min(kBatch, i - j0);
    for (int jj = 0; jj < jn; ++jj) {
      const int j = j0 + jj;
      int64_t phys = j;
      bool ok = true;
      if (a.kidx.page_table != nullptr) {
        phys = a.kidx.page_table[static_cast<int64_t>(b) * a.kidx.pt_stride + j];
        ok = phys >= 0 && phys < a.kidx.num_pages;
      }
      const int64_t off = static_cast<int64_t>(b) * a.kidx.seq_stride + phys * a.kidx.block_stride +
                          static_cast<int64_t>(g) * a.kidx.head_stride;
      ok = ok && off >= 0 && off + kBlock * kR <= a.kidx.extent;
      float m0 = -INFINITY, m1 = -INFINITY;
      if (ok) {
        const char* kb = kbase + off * 2;
#pragma unroll
        for (int nt = 0; nt < 8; ++nt) {
          const uint2 kv = *reinterpret_cast<const uint2*>(kb + (nt * 8 + gid) * 32 + tig * 8);
          float c[4] = {0.f, 0.f, 0.f, 0.f};
          mma_bf16(c, aq, kv.x, kv.y);
          m0 = max3f(m0, c[0], c[1]);
          m1 = max3f(m1, c[2], c[3]);
        }
        float mx = fmaxf(q0v ? m0 : -INFINITY, q1v ? m1 : -INFINITY);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        if (lane == 0) pm[warp][jj] = mx;
      } else {
        if (lane == 0) {
          pm[warp][jj] = NAN;   // marks a failed block
          if (warp == 0) report(a.status, BSA_DEV_BAD_PAGE);
        }
      }
    }
    __syncthreads();
    if (threadIdx.x < jn) {
      float m = pm[0][threadIdx.x];
      bool bad = m != m;
#pragma unroll
      for (int ww = 1; ww < kWarps; ++ww) {
        const float v = pm[ww][threadIdx.x];
        bad = bad || v != v;
        m = fmaxf(m, v);
      }
      const float sc = bad ? -INFINITY : a.idx_scale * (w * fmaxf(m, 0.f));
      out[j0 + threadIdx.x] = sc;
      if (!bad && !isfinite(sc)) report(a.status, BSA_DEV_NONFINITE);
    }
    __syncthreads();
  }
}

}  // namespace

cudaError_t launch_score_prefill(const ScorePrefillArgs& a, int num_sms, cudaStream_t s) {
  (void)num_sms;
  const int rows = a.B * a.Hkv * a.nqb;
  if (rows <= 0) return cudaSuccess;
  const int HP = (a.G + 1) / 2;
  if (a.G == 1) {
    score_prefill_g1_kernel<<<rows, kWarps * 32, 0, s>>>(a);
    return cudaGetLastError();
  }
  switch (HP) {
    case 1: score_prefill_kernel<1><<<rows, kWarps * 32, 0, s>>>(a); break;
    case 2: score_prefill_kernel<2><<<rows, kWarps * 32, 0, s>>>(a); break;
    case 4: score_prefill_kernel<4><<<rows, kWarps * 32, 0, s>>>(a); break;
    case 8: score_prefill_kernel<8><<<rows, kWarps * 32, 0, s>>>(a); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

}  // namespace bsa
