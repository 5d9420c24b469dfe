// Decode block scorer.
//
// For every (sequence b, kv head g) row and 64-token block j:
//   S[b,g,j] = idx_scale * max_{t in block j, t < T_b} sum_{h in group g} w_h ReLU(q_idx[b,h] . k_idx[b,g,t])
// (SpotAttention, Methodology §1: weighted-ReLU score over the index heads;
//  RTPurbo, Methodology §2: r = 16 index keys; block aggregate = max).
//
// Design (HBM-bound stream of 32 bytes per token):
//  * warp-private rings of 1-D bulk copies (cp.async.bulk + mbarrier): each stage
//    holds kStageBlocks blocks of 64 tokens x 16 bf16 = 2 KB; a warp owns a
//    contiguous range of (row, chunk) items, so its reads are sequential;
//  * the 16-dim dot products run on the tensor cores: mma.m16n8k16 with the
//    tokens as M (16 per tile), the group's heads as N (8 per tile, zero padded),
//    K = r = 16. The K dimension is relabelled so that each lane's fragment is one
//    8-byte run of a token (lane t holds dims 4t..4t+3), which makes the shared
//    memory reads conflict-free 64-bit loads; the query fragment uses the same
//    relabelling, so every dot product is unchanged;
//  * epilogue in fp32: ReLU, head weights, head sum with two shuffles (each lane
//    pair exchanges the half it does not keep), running max, then a 4-shuffle
//    warp max per block.
#include "bsa_common.cuh"
#include "bsa_internal.h"

namespace bsa {
namespace {

constexpr int kWarps = 4;          // warps per CTA
constexpr int kStages = 4;         // ring depth per warp
constexpr int kStageBlocks = 2;    // 64-token blocks per stage
constexpr int kBlockBytes = kBlock * kR * 2;                 // 2048
constexpr int kStageBytes = kStageBlocks * kBlockBytes;      // 4096
constexpr int kCtasPerSm = 3;

struct ItemGeom {
  int row, b, g, j0, nb_row, Tb;
};

BSA_DEVFN ItemGeom item_geom(const ScoreDecodeArgs& a, int64_t item) {
  ItemGeom it;
  it.row = static_cast<int>(item / a.chunks_per_row);
  const int chunk = static_cast<int>(item % a.chunks_per_row);
  it.b = it.row / a.Hkv;
  it.g = it.row % a.Hkv;
  it.j0 = chunk * kStageBlocks;
  int Tb = a.seq_lens ? a.seq_lens[it.b] : a.T;
  Tb = Tb < 0 ? 0 : (Tb > a.T ? a.T : Tb);
  it.Tb = Tb;
  it.nb_row = (Tb + kBlock - 1) / kBlock;
  return it;
}

// Element offset of block `blk` of (b, g); false when the page id or extent check
// fails for the `rows` tokens of the block that exist.
BSA_DEVFN bool block_offset(const CacheView& c, int b, int g, int blk, int rows, int64_t& off) {
  int64_t phys = blk;
  if (c.page_table != nullptr) {
    phys = c.page_table[static_cast<int64_t>(b) * c.pt_stride + blk];
    if (phys < 0 || phys >= c.num_pages) return false;
  }
  off = static_cast<int64_t>(b) * c.seq_stride + phys * c.block_stride +
        static_cast<int64_t>(g) * c.head_stride;
  return off >= 0 && off + static_cast<int64_t>(rows) * kR <= c.extent;
}

BSA_DEVFN int rows_of(const ItemGeom& it, int j) {
  const int r = it.Tb - j * kBlock;
  return r < kBlock ? r : kBlock;
}

template <int NT>
__global__ void __launch_bounds__(kWarps * 32) score_decode_kernel(const ScoreDecodeArgs a) {
  extern __shared__ __align__(128) unsigned char smem[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int gid = lane >> 2, tig = lane & 3;
  unsigned char* ring = smem + warp * (kStages * kStageBytes);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kWarps * kStages * kStageBytes) + warp * kStages;

  if (lane == 0) {
    for (int s = 0; s < kStages; ++s) mbar_init(&bars[s], 1);
    fence_mbar_init();
  }
  __syncwarp();

  const int64_t nwarps = static_cast<int64_t>(gridDim.x) * kWarps;
  const int64_t gw = static_cast<int64_t>(blockIdx.x) * kWarps + warp;
  const int64_t per = (a.total_items + nwarps - 1) / nwarps;
  const int64_t it_begin = gw * per;
  const int64_t it_end = min(a.total_items, it_begin + per);
  const int64_t n_items = it_end > it_begin ? it_end - it_begin : 0;
  const char* kbase = static_cast<const char*>(a.kidx.base);

  // lane 0 issues the copies of one item into one stage
  auto issue = [&](int64_t item, int s) {
    if (lane != 0) return;
    const ItemGeom it = item_geom(a, item);
    uint32_t bytes = 0;
    int64_t offs[kStageBlocks];
    uint32_t nbytes[kStageBlocks];
#pragma unroll
    for (int q = 0; q < kStageBlocks; ++q) {
      const int j = it.j0 + q;
      nbytes[q] = 0;
      if (j < it.nb_row) {
        const int rows = rows_of(it, j);   // a partial last block copies only its tokens
        if (block_offset(a.kidx, it.b, it.g, j, rows, offs[q])) nbytes[q] = rows * kR * 2;
      }
      bytes += nbytes[q];
    }
    mbar_arrive_expect_tx(&bars[s], bytes);
#pragma unroll
    for (int q = 0; q < kStageBlocks; ++q)
      if (nbytes[q])
        bulk_g2s(ring + s * kStageBytes + q * kBlockBytes, kbase + offs[q] * 2, nbytes[q],
                 &bars[s]);
  };

  const int pre = static_cast<int>(n_items < kStages ? n_items : kStages);
  for (int s = 0; s < pre; ++s) issue(it_begin + s, s);

  int cur_row = -1;
  uint32_t bq[NT][2];
  float w0[NT], w1[NT];
  bool timed_out = false;

  for (int64_t k = 0; k < n_items; ++k) {
    const int s = static_cast<int>(k % kStages);
    const uint32_t parity = static_cast<uint32_t>((k / kStages) & 1);
    const ItemGeom it = item_geom(a, it_begin + k);
    if (it.row != cur_row) {
      cur_row = it.row;
      // query fragment: lane (gid, tig) holds head 8*nt + gid, dims 4*tig .. 4*tig+3
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        const int hl = nt * 8 + gid;
        bq[nt][0] = bq[nt][1] = 0u;
        if (hl < a.G) {
          const uint2 v = *reinterpret_cast<const uint2*>(
              static_cast<const char*>(a.q_idx) +
              ((static_cast<int64_t>(it.b) * a.Hq + it.g * a.G + hl) * kR + 4 * tig) * 2);
          bq[nt][0] = v.x;
          bq[nt][1] = v.y;
        }
        const int h0 = nt * 8 + 2 * tig, h1 = h0 + 1;
        const float dflt = 1.0f / static_cast<float>(a.G);
        w0[nt] = h0 < a.G ? (a.head_w ? a.head_w[it.g * a.G + h0] : dflt) : 0.f;
        w1[nt] = h1 < a.G ? (a.head_w ? a.head_w[it.g * a.G + h1] : dflt) : 0.f;
      }
    }
    if (!mbar_wait(&bars[s], parity)) {
      timed_out = true;
      break;
    }
    const unsigned char* st = ring + s * kStageBytes;
    float* out = a.scores + static_cast<int64_t>(it.row) * a.nb_max;
#pragma unroll
    for (int q = 0; q < kStageBlocks; ++q) {
      const int j = it.j0 + q;
      if (j >= a.nb_max) break;
      if (j >= it.nb_row) {
        if (lane == 0) out[j] = -INFINITY;
        continue;
      }
      int64_t off_unused;
      if (!block_offset(a.kidx, it.b, it.g, j, rows_of(it, j), off_unused)) {
        if (lane == 0) {
          out[j] = -INFINITY;
          report(a.status, BSA_DEV_BAD_PAGE);
        }
        continue;
      }
      const unsigned char* blk = st + q * kBlockBytes;
      const int valid = it.Tb - j * kBlock;  // tokens of this block that exist (>= 1)
      float mx = 0.f;
#pragma unroll
      for (int mt = 0; mt < 4; ++mt) {
        const int r0 = mt * 16 + gid, r1 = r0 + 8;
        const uint2 x0 = *reinterpret_cast<const uint2*>(blk + r0 * 32 + tig * 8);
        const uint2 x1 = *reinterpret_cast<const uint2*>(blk + r1 * 32 + tig * 8);
        const uint32_t af[4] = {x0.x, x1.x, x0.y, x1.y};
        float vr0 = 0.f, vr1 = 0.f;
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          float c[4] = {0.f, 0.f, 0.f, 0.f};
          mma_bf16(c, af, bq[nt][0], bq[nt][1]);
          vr0 = fmaf(w0[nt], fmaxf(c[0], 0.f), vr0);
          vr0 = fmaf(w1[nt], fmaxf(c[1], 0.f), vr0);
          vr1 = fmaf(w0[nt], fmaxf(c[2], 0.f), vr1);
          vr1 = fmaf(w1[nt], fmaxf(c[3], 0.f), vr1);
        }
        // head sum over the 4 lanes of a row group: even lanes keep token r0,
        // odd lanes token r1
        const bool odd = tig & 1;
        const float send = odd ? vr0 : vr1;
        float keep = odd ? vr1 : vr0;
        keep += __shfl_xor_sync(0xffffffffu, send, 1);
        keep += __shfl_xor_sync(0xffffffffu, keep, 2);
        const int tok = odd ? r1 : r0;
        if (tok < valid) mx = fmaxf(mx, keep);
      }
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
      if (lane == 0) {
        const float sc = a.idx_scale * mx;
        out[j] = sc;
        if (!isfinite(sc)) report(a.status, BSA_DEV_NONFINITE);
      }
    }
    __syncwarp();
    if (k + kStages < n_items) {
      fence_proxy_async_smem();
      issue(it_begin + k + kStages, s);
    }
  }

  if (timed_out) {
    if (lane == 0) report(a.status, BSA_DEV_TIMEOUT);
    // let copies still in flight land before the CTA exits (bounded)
    for (int64_t k = 0; k < n_items && k < kStages; ++k) {
      const int64_t kk = n_items - 1 - k;
      mbar_wait(&bars[kk % kStages], static_cast<uint32_t>((kk / kStages) & 1), 100000000ull);
    }
  }
}

}  // namespace

cudaError_t launch_score_decode(const ScoreDecodeArgs& a, int num_sms, cudaStream_t s) {
  if (a.total_items <= 0) return cudaSuccess;
  const size_t smem = kWarps * kStages * kStageBytes + kWarps * kStages * sizeof(uint64_t);
  int64_t warps_needed = a.total_items;
  int64_t ctas = (warps_needed + kWarps - 1) / kWarps;
  const int64_t cap = static_cast<int64_t>(num_sms) * kCtasPerSm;
  if (ctas > cap) ctas = cap;
  auto kern = (a.G > 8) ? score_decode_kernel<2> : score_decode_kernel<1>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  kern<<<static_cast<unsigned>(ctas), kWarps * 32, smem, s>>>(a);
  return cudaGetLastError();
}

}  // namespace bsa
