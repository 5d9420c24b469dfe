// Decode block scorer.
//
// For every (sequence b, kv head g) row and 64-token block j:
//   S[b,g,j] = idx_scale * max_{t in block j, t < T_b} sum_{h in group g} w_h ReLU(q_idx[b,h] . k_idx[b,g,t])
// (SpotAttention, Methodology §1: weighted-ReLU score over the index heads;
//  RTPurbo, Methodology §2: r = 16 index keys; block aggregate = max).
//
// Design (HBM-bound stream of 32 bytes per token):
//  * persistent CTAs, each owning a contiguous range of items; an item is a chunk
//    of kChunk consecutive blocks of one row (16 KB of index keys). One producer
//    lane computes the item's geometry once, publishes it in shared memory and
//    streams the chunk into a ring of stages with 1-D bulk copies (one copy per
//    chunk when the blocks are contiguous, one per block otherwise), completion
//    counted on per-stage "full" mbarriers;
//  * consumer warp w scores block w of every chunk. The 16-dim dot products run
//    on mma.m16n8k16 with tokens as M (16 per tile), the group's heads as N (8 per
//    tile, zero padded) and K = r = 16. The K dimension is relabelled so that each
//    lane's fragment is one 8-byte run of a token (lane t holds dims 4t..4t+3):
//    shared-memory reads are conflict-free 64-bit loads, and the query fragment
//    uses the same relabelling, so every dot product is unchanged;
//  * epilogue in fp32: ReLU, head weights, head sum with two shuffles (each lane
//    pair exchanges the half it does not keep), running max, a 4-shuffle warp max
//    per block, then the stage is released through its "empty" mbarrier.
//  * 4-bit index keys (SpotAttention, Methodology §4; format in include/bsa.h):
//    the same kernel streams 576-byte block records (9 B per token), with four
//    CTAs per SM. FP4 codes are E2M1 values (sign bit 3, exponent and mantissa in
//    bits 0-2), so one hardware conversion turns a byte of two codes into an f16
//    pair, exactly; the MMA then runs on f16 operands, with the index query
//    converted to f16 once per row (exact for |q| in [2^-14, 65504]; a larger one
//    is reported as BSA_DEV_FP16_RANGE). INT4 codes are turned into bf16 with two
//    byte-permute table lookups plus the sign bits. Either way the MMA runs on the
//    unscaled codes and the token's ReLU head sum is multiplied by its E4M3 scale
//    (ReLU is positively homogeneous, and the scales are > 0); the cache scale g
//    multiplies the block score.
//  * with group_size > 0 (two-level routing) the same token scores also give the
//    max of every group of 16, 32 or 64 tokens, written beside the block scores.
#include "bsa_common.cuh"
#include "bsa_internal.h"

namespace bsa {
namespace {

constexpr int kConsumers = 8;                              // consumer warps = blocks per chunk
constexpr int kChunk = kConsumers;                         // blocks per item / stage
constexpr int kThreads = (kConsumers + 1) * 32;

struct StageInfo {
  int row;        // b * Hkv + g
  int j0;         // first block of the chunk
  int Tb;         // tokens of sequence b; -1: a local head, nothing to score
  uint32_t ok;    // bit q: block j0 + q was copied
};

// A local head (p <= 0 with no K_min floor) keeps its reserved blocks only: no scores.
BSA_DEVFN bool local_head(const ScoreDecodeArgs& a, int g) {
  return a.head_p != nullptr && a.k_min == 0 && !(a.head_p[g] > 0.f);
}

// KF: key format, 0 = bf16 rows (32 B per token), 1 = FP4 / 2 = INT4 records.
template <int KF>
struct ScoreSmem {
  static constexpr int kBlockBytes = KF == 0 ? kBlock * kR * 2 : kQRecord;   // 2048 or 576
  static constexpr int kStages = KF == 0 ? 6 : 8;
  // 4-bit keys cost more instructions per byte: more resident CTAs hide the latency
  static constexpr int kCtasPerSm = KF == 0 ? 2 : 4;
  static constexpr int kStageBytes = kChunk * kBlockBytes;
  static constexpr int kRing = kStages * kStageBytes;
  static constexpr int kInfo = kStages * static_cast<int>(sizeof(StageInfo));
  static constexpr int kTotal = kRing + kInfo + 2 * kStages * 8 + 128;
};

// Record index of block `blk` of (b, g) in a 4-bit cache, false when invalid.
BSA_DEVFN bool block_record(const CacheView& c, int b, int g, int blk, int64_t& rec) {
  int64_t phys = blk;
  if (c.page_table != nullptr) {
    phys = c.page_table[static_cast<int64_t>(b) * c.pt_stride + blk];
    if (phys < 0 || phys >= c.num_pages) return false;
  }
  rec = static_cast<int64_t>(b) * c.seq_stride + phys * c.block_stride +
        static_cast<int64_t>(g) * c.head_stride;
  return rec >= 0 && rec + 1 <= c.extent;
}

// Four 4-bit codes (elements 4t..4t+3 of a token, low nibble first) -> four bf16
// values (two bf16x2 words). Byte-permute tables give the low and high byte of
// the bf16 of each magnitude index; the sign bits are ORed in.
template <int KF>
BSA_DEVFN uint2 dequant4(uint32_t c16) {
  // magnitudes: FP4 (E2M1) 0, .5, 1, 1.5, 2, 3, 4, 6; INT4 0..7
  constexpr uint32_t kLoX = KF == 1 ? 0xC0800000u : 0x40008000u;
  constexpr uint32_t kLoY = KF == 1 ? 0xC0804000u : 0xE0C0A080u;
  constexpr uint32_t kHiX = KF == 1 ? 0x3F3F3F00u : 0x40403F00u;
  constexpr uint32_t kHiY = 0x40404040u;
  const uint32_t sel = c16 & 0x7777u;
  const uint32_t lo = __byte_perm(kLoX, kLoY, sel), hi = __byte_perm(kHiX, kHiY, sel);
  // sign bits 3, 7 (11, 15) of the codes -> bits 15, 31 of the words: one multiply
  // places both copies (x * (2^12 + 2^24) puts bit 3 at 15 and bit 7 at 31).
  const uint32_t s0 = (c16 & 0x88u) * 0x01001000u, s1 = (c16 & 0x8800u) * 0x00010010u;
  const uint32_t w0 = __byte_perm(lo, hi, 0x5140u) | (s0 & 0x80008000u);
  const uint32_t w1 = __byte_perm(lo, hi, 0x7362u) | (s1 & 0x80008000u);
  return make_uint2(w0, w1);
}

BSA_DEVFN uint32_t lds_u16(uint32_t addr) {
  uint16_t v;
  asm volatile("ld.shared.u16 %0, [%1];" : "=h"(v) : "r"(addr));
  return v;
}
BSA_DEVFN uint32_t lds_u8(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.shared.u8 %0, [%1];" : "=r"(v) : "r"(addr));
  return v;
}

// Two FP4 (E2M1) codes in the low byte of x -> f16x2, the low nibble in the low half;
// every E2M1 value is exact in f16.
BSA_DEVFN uint32_t e2m1x2_to_f16x2(uint32_t x) {
  uint32_t d;
  asm("{\n .reg .b8 t;\n mov.b32 {t, _, _, _}, %1;\n cvt.rn.f16x2.e2m1x2 %0, t;\n}"
      : "=r"(d) : "r"(x));
  return d;
}

// bf16x2 -> f16x2 (exact for magnitudes in [2^-14, 65504]); sets `big` when a value
// is beyond the f16 range.
BSA_DEVFN uint32_t bf16x2_to_f16x2(uint32_t x, bool& big) {
  const float2 f = unpack_bf16(x);
  big = big || fabsf(f.x) > 65504.f || fabsf(f.y) > 65504.f;
  return pack_f16(f.x, f.y);
}

BSA_DEVFN int clamp_len(const ScoreDecodeArgs& a, int b) {
  int Tb = a.seq_lens ? a.seq_lens[b] : a.T;
  return Tb < 0 ? 0 : (Tb > a.T ? a.T : Tb);
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

// GRP: also write the maxima of the token groups (two-level routing).
template <int NT, int KF, bool GRP>
__global__ void __launch_bounds__(kThreads) score_decode_kernel(const ScoreDecodeArgs a) {
  using SM = ScoreSmem<KF>;
  constexpr int kStages = SM::kStages, kStageBytes = SM::kStageBytes, kBlockBytes = SM::kBlockBytes;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~static_cast<uintptr_t>(127));
  unsigned char* ring = smem;
  StageInfo* info = reinterpret_cast<StageInfo*>(smem + SM::kRing);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + SM::kRing + SM::kInfo);
  uint64_t* empty = full + kStages;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  __shared__ float scale_lut[128];   // E4M3 code -> value (4-bit keys)
  if (KF != 0 && threadIdx.x < 128) scale_lut[threadIdx.x] = e4m3_value(threadIdx.x);
  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kConsumers);
    }
    fence_mbar_init();
  }
  __syncthreads();
  grid_dependency_wait();   // the previous step may still read the score buffer

  const int64_t per = (a.total_items + gridDim.x - 1) / gridDim.x;
  const int64_t it0 = static_cast<int64_t>(blockIdx.x) * per;
  const int64_t it1 = min(a.total_items, it0 + per);
  const int n_items = it1 > it0 ? static_cast<int>(it1 - it0) : 0;

  if (warp == kConsumers) {
    // ---------------------------------------------------------------- producer
    if (lane == 0) {
      const char* kbase = static_cast<const char*>(a.kidx.base);
      const bool contiguous =
          a.kidx.page_table == nullptr && a.kidx.block_stride == (KF == 0 ? kBlock * kR : 1);
      // walk the item range incrementally: (row, j0) without a division per item
      int row = static_cast<int>(it0 / a.chunks_per_row);
      int j0 = static_cast<int>(it0 - static_cast<int64_t>(row) * a.chunks_per_row) * kChunk;
      int b = row / a.Hkv, g = row - b * a.Hkv;
      int Tb = clamp_len(a, b);
      for (int k = 0; k < n_items; ++k) {
        const int s = k % kStages;
        if (!mbar_wait(&empty[s], ((k / kStages) & 1) ^ 1)) {
          report(a.status, BSA_DEV_TIMEOUT);
          break;
        }
        const int nb_row = (Tb + kBlock - 1) / kBlock;
        if (local_head(a, g)) {
          info[s] = StageInfo{row, j0, -1, 0u};
          mbar_arrive(&full[s]);
        } else {
          const int nblk = max(0, min(kChunk, nb_row - j0));      // blocks of the chunk that exist
          unsigned char* dst = ring + s * kStageBytes;
          uint32_t ok = 0, bytes = 0;
          if (KF != 0 && contiguous && nblk > 0) {
            // adjacent whole records: one range check, one copy
            int64_t rec;
            if (block_record(a.kidx, b, g, j0, rec) && rec + nblk <= a.kidx.extent) {
              ok = (1u << nblk) - 1u;
              bytes = nblk * kBlockBytes;
            }
            info[s] = StageInfo{row, j0, Tb, ok};
            mbar_arrive_expect_tx(&full[s], bytes);
            if (ok) bulk_g2s(dst, kbase + rec * kBlockBytes, bytes, &full[s]);
          } else if (KF != 0) {
            int64_t recs[kChunk];
            for (int q = 0; q < nblk; ++q)
              if (block_record(a.kidx, b, g, j0 + q, recs[q])) {
                ok |= 1u << q;
                bytes += kBlockBytes;
              }
            info[s] = StageInfo{row, j0, Tb, ok};
            mbar_arrive_expect_tx(&full[s], bytes);
            for (int q = 0; q < nblk; ++q)
              if (ok & (1u << q))
                bulk_g2s(dst + q * kBlockBytes, kbase + recs[q] * kBlockBytes, kBlockBytes, &full[s]);
          } else if (contiguous && nblk > 0) {
            // the chunk's blocks are adjacent: one range check, one copy
            const int rows = min(nblk * kBlock, Tb - j0 * kBlock);
            int64_t off;
            if (block_offset(a.kidx, b, g, j0, rows, off)) {
              ok = (1u << nblk) - 1u;
              bytes = rows * kR * 2;
            }
            info[s] = StageInfo{row, j0, Tb, ok};
            mbar_arrive_expect_tx(&full[s], bytes);
            if (ok) bulk_g2s(dst, kbase + off * 2, bytes, &full[s]);
          } else {
            int64_t offs[kChunk];
            int rows_q[kChunk];
            for (int q = 0; q < nblk; ++q) {
              rows_q[q] = min(kBlock, Tb - (j0 + q) * kBlock);
              if (block_offset(a.kidx, b, g, j0 + q, rows_q[q], offs[q])) {
                ok |= 1u << q;
                bytes += rows_q[q] * kR * 2;
              }
            }
            info[s] = StageInfo{row, j0, Tb, ok};
            mbar_arrive_expect_tx(&full[s], bytes);
            for (int q = 0; q < nblk; ++q)
              if (ok & (1u << q))
                bulk_g2s(dst + q * kBlockBytes, kbase + offs[q] * 2, rows_q[q] * kR * 2, &full[s]);
          }
        }
        // next item
        j0 += kChunk;
        if (j0 >= a.chunks_per_row * kChunk) {
          j0 = 0;
          ++row;
          if (++g == a.Hkv) {
            g = 0;
            ++b;
            if (b < a.B) Tb = clamp_len(a, b);
          }
        }
      }
      // let the consumers release what was issued before the CTA can exit (bounded)
      for (int k = max(0, n_items - kStages); k < n_items; ++k)
        mbar_wait(&empty[k % kStages], (k / kStages) & 1, 200000000ull);
    }
    return;
  }

  // ------------------------------------------------------------------ consumers
  const int gid = lane >> 2, tig = lane & 3;
  const float kscale = KF == 0 ? 1.0f : *a.gscale;   // cache scale g of 4-bit keys
  int cur_row = -1;
  uint32_t bq[NT][2];
  float w0[NT], w1[NT];
  for (int k = 0; k < n_items; ++k) {
    const int s = k % kStages;
    if (!mbar_wait(&full[s], (k / kStages) & 1)) {
      if (lane == 0) report(a.status, BSA_DEV_TIMEOUT);
      break;
    }
    const StageInfo in = info[s];
    const int j = in.j0 + warp;
    if (in.Tb < 0) {   // local head: release the stage, write nothing
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[s]);
      continue;
    }
    if (in.row != cur_row) {
      cur_row = in.row;
      const int b = in.row / a.Hkv, g = in.row - b * a.Hkv;
      const float dflt = 1.0f / static_cast<float>(a.G);
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        const int hl = nt * 8 + gid;
        bq[nt][0] = bq[nt][1] = 0u;
        if (hl < a.G) {
          const uint2 v = *reinterpret_cast<const uint2*>(
              static_cast<const char*>(a.q_idx) +
              ((static_cast<int64_t>(b) * a.Hq + g * a.G + hl) * kR + 4 * tig) * 2);
          bq[nt][0] = v.x;
          bq[nt][1] = v.y;
          if constexpr (KF == 1) {   // f16 MMA operands for FP4 keys
            bool big = false;
            bq[nt][0] = bf16x2_to_f16x2(v.x, big);
            bq[nt][1] = bf16x2_to_f16x2(v.y, big);
            if (big && tig == 0 && warp == 0) report(a.status, BSA_DEV_FP16_RANGE);
          }
        }
        const int h0 = nt * 8 + 2 * tig, h1 = h0 + 1;
        // half weights: (w/2) * (c + |c|) = w * ReLU(c) exactly (c + |c| is 2c or +0)
        w0[nt] = 0.5f * (h0 < a.G ? (a.head_w ? a.head_w[g * a.G + h0] : dflt) : 0.f);
        w1[nt] = 0.5f * (h1 < a.G ? (a.head_w ? a.head_w[g * a.G + h1] : dflt) : 0.f);
      }
    }
    if (j < a.nb_max) {
      float* out = a.scores + static_cast<int64_t>(in.row) * a.nb_max + j;
      const int valid = in.Tb - j * kBlock;  // tokens of this block that exist
      const int gpb = GRP ? kBlock / a.group_size : 0;
      float* gout = gpb ? a.group_scores + (static_cast<int64_t>(in.row) * a.nb_max + j) * gpb : nullptr;
      if (valid <= 0 || !(in.ok & (1u << warp))) {
        if (lane == 0) {
          *out = -INFINITY;
          if (valid > 0) report(a.status, BSA_DEV_BAD_PAGE);
        }
        if (lane < gpb) gout[lane] = -INFINITY;
      } else {
        const unsigned char* blk = ring + s * kStageBytes + warp * kBlockBytes;
        const uint32_t blk_s = smem_u32(blk);
        const bool whole = valid >= kBlock;   // every token of the block exists
        float mx = 0.f;
        // two-level routing: the max of each 16-token group (tile mt) as the bits of a
        // non-negative float (the scores are >= 0, so integer order is float order),
        // -1 when the group holds no token of the sequence
        int gbits[4] = {-1, -1, -1, -1};
        const bool odd = tig & 1;
#pragma unroll
        for (int mt = 0; mt < 4; ++mt) {
          const int r0 = mt * 16 + gid, r1 = r0 + 8;
          uint2 x0, x1;
          if constexpr (KF == 0) {
            x0 = *reinterpret_cast<const uint2*>(blk + r0 * 32 + tig * 8);
            x1 = *reinterpret_cast<const uint2*>(blk + r1 * 32 + tig * 8);
          } else if constexpr (KF == 1) {
            const uint32_t c0 = lds_u16(blk_s + r0 * 8 + tig * 2);
            const uint32_t c1 = lds_u16(blk_s + r1 * 8 + tig * 2);
            x0 = make_uint2(e2m1x2_to_f16x2(c0), e2m1x2_to_f16x2(c0 >> 8));
            x1 = make_uint2(e2m1x2_to_f16x2(c1), e2m1x2_to_f16x2(c1 >> 8));
          } else {
            x0 = dequant4<KF>(*reinterpret_cast<const uint16_t*>(blk + r0 * 8 + tig * 2));
            x1 = dequant4<KF>(*reinterpret_cast<const uint16_t*>(blk + r1 * 8 + tig * 2));
          }
          const uint32_t af[4] = {x0.x, x1.x, x0.y, x1.y};
          float vr0 = 0.f, vr1 = 0.f;
#pragma unroll
          for (int nt = 0; nt < NT; ++nt) {
            float c[4] = {0.f, 0.f, 0.f, 0.f};
            if constexpr (KF == 1) mma_f16(c, af, bq[nt][0], bq[nt][1]);
            else mma_bf16(c, af, bq[nt][0], bq[nt][1]);
            // ReLU on the FMA pipe (the ALU pipe is the busier one)
            vr0 = fmaf(w0[nt], c[0] + fabsf(c[0]), vr0);
            vr0 = fmaf(w1[nt], c[1] + fabsf(c[1]), vr0);
            vr1 = fmaf(w0[nt], c[2] + fabsf(c[2]), vr1);
            vr1 = fmaf(w1[nt], c[3] + fabsf(c[3]), vr1);
          }
          // head sum over the 4 lanes of a row group: even lanes keep token r0,
          // odd lanes token r1
          const float send = odd ? vr0 : vr1;
          float keep = odd ? vr1 : vr0;
          keep += __shfl_xor_sync(0xffffffffu, send, 1);
          // lanes 2 and 3 of a row group hold heads 4-7 of each 8-head tile: with at most
          // four heads those are zero-weight padding and the second exchange adds nothing
          if (NT > 1 || a.G > 4) keep += __shfl_xor_sync(0xffffffffu, keep, 2);
          const int tok = odd ? r1 : r0;
          if constexpr (KF != 0)   // token scale
            keep *= scale_lut[lds_u8(blk_s + kBlock * 8 + tok) & 0x7Fu];
          if (whole || tok < valid) mx = fmaxf(mx, keep);
          if constexpr (GRP) gbits[mt] = __reduce_max_sync(0xffffffffu, tok < valid ? __float_as_int(keep) : -1);
        }
        if (GRP && lane == 0) {
          // group summaries (HGA, Central mechanism §2), here the max of the group's
          // token scores: 16-token groups are the tiles, larger ones their maxima
          const float sc = a.idx_scale * kscale;
          auto val = [sc](int bits) { return bits < 0 ? -INFINITY : sc * __int_as_float(bits); };
          if (gpb == 4) {
            *reinterpret_cast<float4*>(gout) =
                make_float4(val(gbits[0]), val(gbits[1]), val(gbits[2]), val(gbits[3]));
          } else if (gpb == 2) {
            *reinterpret_cast<float2*>(gout) =
                make_float2(val(max(gbits[0], gbits[1])), val(max(gbits[2], gbits[3])));
          } else {
            *gout = val(max(max(gbits[0], gbits[1]), max(gbits[2], gbits[3])));
          }
        }
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
        if (lane == 0) {
          const float sc = a.idx_scale * (kscale * mx);
          *out = sc;
          if (!isfinite(sc)) report(a.status, BSA_DEV_NONFINITE);
        }
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[s]);
  }
}

template <int KF>
cudaError_t launch_fmt(const ScoreDecodeArgs& a, int num_sms, cudaStream_t s) {
  const int smem = ScoreSmem<KF>::kTotal;
  int64_t ctas = static_cast<int64_t>(num_sms) * ScoreSmem<KF>::kCtasPerSm;
  if (ctas > a.total_items) ctas = a.total_items;
  const bool grp = a.group_size > 0;
  auto kern = a.G > 8 ? (grp ? score_decode_kernel<2, KF, true> : score_decode_kernel<2, KF, false>)
                      : (grp ? score_decode_kernel<1, KF, true> : score_decode_kernel<1, KF, false>);
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  return launch_pdl(kern, dim3(static_cast<unsigned>(ctas)), dim3(kThreads), smem, s, a);
}

}  // namespace

cudaError_t launch_score_decode(const ScoreDecodeArgs& a, int num_sms, cudaStream_t s) {
  if (a.total_items <= 0) return cudaSuccess;
  switch (a.kfmt) {
    case 0: return launch_fmt<0>(a, num_sms, s);
    case 1: return launch_fmt<1>(a, num_sms, s);
    case 2: return launch_fmt<2>(a, num_sms, s);
    default: return cudaErrorInvalidValue;
  }
}

int score_decode_chunk_blocks() { return kChunk; }

}  // namespace bsa
