// Split-K sparse flash-decode over the kept blocks, then an LSE merge.
//
// For each query head h of kv group g of sequence b: exact softmax attention over
// the tokens t < T_b of the kept 64-token blocks (HGA, Central mechanism §4 and
// Key contributions §2: exact token-level attention over the routed set).
//
// Design (HBM-bound: 2 * 64 * d * 2 bytes of K/V per kept block per (b, g)):
//  * work unit = (row (b, g), split s) = a slice of split_len consecutive entries
//    of the row's kept list; persistent CTAs (one per SM) stride over the units;
//  * one producer warp streams each kept block's K and V tiles into a ring of
//    shared-memory stages with TMA (2-D tensor maps, 128-byte swizzle, one box =
//    64 tokens x 64 dims), completion on per-stage "full" mbarriers; four
//    consumer warps release stages through "empty" mbarriers;
//  * consumer warp w owns tokens [16w, 16w+16) of every block: S^T = K_w Q^T on
//    mma.m16n8k16 (tokens as M, the group's heads as N), online softmax in fp32
//    (log2 domain), then O^T += V_w^T P^T (V^T via ldmatrix.trans, P^T moved into
//    the B-fragment layout with movmatrix). P is split into bf16 hi + lo parts, so
//    the P.V products keep ~16 mantissa bits;
//  * at the end of a unit the four warps' (m, l, O) are merged in shared memory
//    and written as one partial; the merge kernel combines the splits of a row
//    with their log-sum-exp weights and writes o (bf16), o_f32 and lse.
//  * a stage holds four 16-token slots, consumer warp w attends slot w; the
//    producer publishes each slot's first token (or -1) and whether the stage is
//    the last of its unit. Without group masks a stage is one kept block.
//  * two-level routing (HGA, Central mechanism §2): each kept entry carries a
//    bitmask of its kept token groups, and the producer packs the 16-token
//    quarters of the kept groups of consecutive entries densely into the slots
//    (16-row boxes at the slots' swizzled offsets), so a stage carries four
//    quarters of useful work whatever the groups kept.
#include "bsa_common.cuh"
#include "bsa_internal.h"

namespace bsa {
namespace {

constexpr int kConsumerWarps = 4;
// Producer warps: one streams whole kept blocks; under two-level routing all of them
// walk the same quarter sequence and each fills the stages s with s % kProducers equal
// to its index, so the per-copy issue work is spread over several warps.
constexpr int kProducers = 4;
constexpr int kThreads = (kConsumerWarps + kProducers) * 32;

template <int D>
struct DecodeCfg {
  static constexpr int kBoxes = D / 64;                       // 64-dim boxes per tile
  static constexpr int kTileBytes = kBlock * D * 2;           // one K or V tile
  static constexpr int kStageBytes = 2 * kTileBytes;          // K + V
  static constexpr int kStages = D == 128 ? 5 : 8;
  static constexpr int kKsteps = D / 16;
};

template <int D, int NT>
struct DecodeSmem {
  static constexpr int kRing = DecodeCfg<D>::kStages * DecodeCfg<D>::kStageBytes;
  static constexpr int kComb = kConsumerWarps * (NT * 8) * D * 4;   // partial O per warp
  static constexpr int kStats = kConsumerWarps * (NT * 8) * 2 * 4;  // m, l per warp
  static constexpr int kBars = 2 * DecodeCfg<D>::kStages * 8;
  static constexpr int kInfoW = 5;   // per stage: first token of slots 0..3, last-of-unit flag
  static constexpr int kInfo = DecodeCfg<D>::kStages * kInfoW * 4;
  static constexpr int kTotal = kRing + kComb + kStats + kBars + kInfo + 1024;  // + alignment
};

BSA_DEVFN void consumer_sync() { asm volatile("bar.sync 1, %0;" ::"n"(kConsumerWarps * 32)); }
// Barrier over the consumer warps that also ANDs a flag across them, so a
// decision to stop is taken by all of them together.
BSA_DEVFN bool consumer_sync_and(bool v) {
  uint32_t out;
  asm volatile(
      "{\n .reg .pred pi, po;\n setp.ne.u32 pi, %1, 0;\n bar.red.and.pred po, 1, %2, pi;\n"
      " selp.u32 %0, 1, 0, po;\n}\n"
      : "=r"(out)
      : "r"(static_cast<uint32_t>(v)), "n"(kConsumerWarps * 32));
  return out != 0;
}

BSA_DEVFN int seq_len(const DecodeArgs& a, int b) {
  int Tb = a.seq_lens ? a.seq_lens[b] : a.T;
  return Tb < 0 ? 0 : (Tb > a.T ? a.T : Tb);
}

// Row (in rows of width d) of the first token of block `blk` of (b, g); -1 if the
// page id is invalid or the `rows` existing tokens of the block leave the extent.
// (TMA fills rows of a box beyond the tensor with zeros; those tokens are masked.)
BSA_DEVFN int64_t tile_row(const CacheView& c, int b, int g, int blk, int rows, int d) {
  int64_t phys = blk;
  if (c.page_table != nullptr) {
    phys = c.page_table[static_cast<int64_t>(b) * c.pt_stride + blk];
    if (phys < 0 || phys >= c.num_pages) return -1;
  }
  const int64_t off = static_cast<int64_t>(b) * c.seq_stride + phys * c.block_stride +
                      static_cast<int64_t>(g) * c.head_stride;
  if (off < 0 || off + static_cast<int64_t>(rows) * d > c.extent) return -1;
  return off / d;
}

template <int D, int NT>
__global__ void __launch_bounds__(kThreads, 1)
    decode_attn_kernel(const DecodeArgs a, const __grid_constant__ CUtensorMap tmk,
                       const __grid_constant__ CUtensorMap tmv,
                       const __grid_constant__ CUtensorMap tmk16,
                       const __grid_constant__ CUtensorMap tmv16, const int num_units) {
  using Cfg = DecodeCfg<D>;
  using Sm = DecodeSmem<D, NT>;
  constexpr int S = Cfg::kStages;
  // A producer waits for a ring slot's release by parity, which tells apart only the
  // phase it waits for and the one before. Its previous own stage (kProducers back)
  // guaranteed the release of the stage kProducers + S back, so the slot is at most one
  // phase behind only while kProducers <= S.
  static_assert(kProducers <= S, "more producers than ring stages");
  constexpr int NH = NT * 8;  // padded heads
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  unsigned char* ring = smem;
  float* comb = reinterpret_cast<float*>(smem + Sm::kRing);
  float* stats = reinterpret_cast<float*>(smem + Sm::kRing + Sm::kComb);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + Sm::kRing + Sm::kComb + Sm::kStats);
  uint64_t* empty = full + S;
  int* sinfo = reinterpret_cast<int*>(empty + S);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kConsumerWarps);
    }
    fence_mbar_init();
  }
  __syncthreads();
  grid_dependency_wait();   // kept lists come from the selection kernel

  if (warp >= kConsumerWarps) {
    // ------------------------------------------------------------- producers
    const int pi = warp - kConsumerWarps;
    // The warp resolves 32 kept entries at a time (block id, then the K and V rows
    // through the page table), one per lane, so the dependent global loads overlap;
    // lane 0 then issues the TMA copies of those blocks back to back.
    if (lane == 0) {
      prefetch_tensormap(&tmk);
      prefetch_tensormap(&tmv);
      if (a.kept_groups != nullptr) {
        prefetch_tensormap(&tmk16);
        prefetch_tensormap(&tmv16);
      }
    }
    constexpr int kW = Sm::kInfoW;
    const bool packed = a.kept_groups != nullptr;
    if (!packed && pi != 0) return;   // whole blocks: one producer
    // the producer that fills stage number k
    auto owner = [packed](uint32_t k) { return packed ? static_cast<int>(k % kProducers) : 0; };
    uint32_t it = 0;   // stages issued (by all producers; every producer counts them all)
    bool ok_all = true;
    for (int unit = blockIdx.x; unit < num_units && ok_all; unit += gridDim.x) {
      const int row = unit / a.splits, sp = unit % a.splits;
      const int b = row / a.Hkv, g = row % a.Hkv;
      const int cnt = min(a.kept_count[row], a.max_kept);
      const int e0 = sp * a.split_len, e1 = min(cnt, e0 + a.split_len);
      const int Tb = seq_len(a, b);
      const int nb = (Tb + kBlock - 1) / kBlock;
      bool open = false;   // packed: a stage is being filled (lane 0)
      int fill = 0;        // packed: its slots in use
      for (int base = e0; base < e1 && ok_all; base += 32) {
        const int e = base + lane;
        int blk = -1, qm = 15;   // qm: 16-token quarters to copy and attend
        int64_t rk = -1, rv = -1;
        if (e < e1) {
          blk = a.kept[static_cast<int64_t>(row) * a.max_kept + e];
          if (blk >= 0 && blk < nb) {
            const int rows = min(kBlock, Tb - blk * kBlock);
            rk = tile_row(a.k, b, g, blk, rows, D);
            rv = tile_row(a.v, b, g, blk, rows, D);
            if (rk < 0 || rv < 0) report(a.status, BSA_DEV_BAD_PAGE);
            if (packed) {
              const uint32_t gm = static_cast<uint32_t>(
                  a.kept_groups[static_cast<int64_t>(row) * a.max_kept + e]);
              qm = 0;
#pragma unroll
              for (int q = 0; q < 4; ++q) qm |= static_cast<int>((gm >> (q * 16 / a.group_size)) & 1u) << q;
              qm &= (1 << ((rows + 15) / 16)) - 1;   // quarters that hold tokens
            }
          } else {
            report(a.status, BSA_DEV_BAD_KEPT);
          }
        }
        const int n_here = min(32, e1 - base);
        for (int q = 0; q < n_here; ++q) {
          const int blk_q = __shfl_sync(0xffffffffu, blk, q);
          const int64_t rk_q = __shfl_sync(0xffffffffu, rk, q);
          const int64_t rv_q = __shfl_sync(0xffffffffu, rv, q);
          const int qm_q = __shfl_sync(0xffffffffu, qm, q);
          if (lane == 0) {
            const bool ok = rk_q >= 0 && rv_q >= 0;
            if (!packed) {
              // one kept block per stage
              const int s = it % S;
              if (!mbar_wait(&empty[s], ((it / S) & 1) ^ 1)) {
                report(a.status, BSA_DEV_TIMEOUT);
                ok_all = false;
              } else {
#pragma unroll
                for (int w = 0; w < 4; ++w) sinfo[s * kW + w] = ok ? blk_q * kBlock + 16 * w : -1;
                sinfo[s * kW + 4] = base + q == e1 - 1;
                unsigned char* st = ring + s * Cfg::kStageBytes;
                if (ok) {
                  mbar_arrive_expect_tx(&full[s], Cfg::kStageBytes);
#pragma unroll
                  for (int x = 0; x < Cfg::kBoxes; ++x) {
                    tma_load_2d(st + x * 8192, &tmk, x * 64, static_cast<int32_t>(rk_q), &full[s]);
                    tma_load_2d(st + Cfg::kTileBytes + x * 8192, &tmv, x * 64,
                                static_cast<int32_t>(rv_q), &full[s]);
                  }
                } else {
                  mbar_arrive(&full[s]);
                }
                ++it;
              }
            } else {
              // the entry's kept quarters go to the next free slots, one 16-row copy
              // each (issuing whole runs through run-length-dependent branches measured
              // slower); a full stage is handed over once it is known not to be the
              // unit's last. Every producer walks the same sequence; only the owner of a
              // stage waits for it, fills it and hands it over.
              for (int q4 = 0; q4 < 4 && ok && ok_all; ++q4) {
                if (!((qm_q >> q4) & 1)) continue;
                if (open && fill == 4) {
                  if (owner(it - 1) == pi) {
                    const int s = (it - 1) % S;
                    sinfo[s * kW + 4] = 0;
                    mbar_arrive(&full[s]);
                  }
                  open = false;
                }
                if (!open) {
                  if (owner(it) == pi && !mbar_wait(&empty[it % S], ((it / S) & 1) ^ 1)) {
                    report(a.status, BSA_DEV_TIMEOUT);
                    ok_all = false;
                    break;
                  }
                  ++it;
                  open = true;
                  fill = 0;
                }
                if (owner(it - 1) == pi) {
                  const int s = (it - 1) % S;
                  sinfo[s * kW + fill] = blk_q * kBlock + 16 * q4;
                  unsigned char* st = ring + s * Cfg::kStageBytes + fill * 2048;
                  mbar_expect_tx(&full[s], Cfg::kStageBytes / 4);
#pragma unroll
                  for (int x = 0; x < Cfg::kBoxes; ++x) {
                    tma_load_2d(st + x * 8192, &tmk16, x * 64, static_cast<int32_t>(rk_q + 16 * q4),
                                &full[s]);
                    tma_load_2d(st + Cfg::kTileBytes + x * 8192, &tmv16, x * 64,
                                static_cast<int32_t>(rv_q + 16 * q4), &full[s]);
                  }
                }
                ++fill;
              }
            }
          }
          ok_all = __shfl_sync(0xffffffffu, ok_all ? 1 : 0, 0) != 0;
          if (!ok_all) break;
        }
      }
      // packed: close the unit's last stage (an empty one when no quarter was kept)
      if (packed && e1 > e0 && ok_all && lane == 0) {
        if (!open) {
          if (owner(it) == pi && !mbar_wait(&empty[it % S], ((it / S) & 1) ^ 1)) {
            report(a.status, BSA_DEV_TIMEOUT);
            ok_all = false;
          } else {
            ++it;
            open = true;
            fill = 0;
          }
        }
        if (open && owner(it - 1) == pi) {
          const int s = (it - 1) % S;
          for (int w = fill; w < 4; ++w) sinfo[s * kW + w] = -1;
          sinfo[s * kW + 4] = 1;
          mbar_arrive(&full[s]);
        }
        open = false;
      }
      ok_all = __shfl_sync(0xffffffffu, ok_all ? 1 : 0, 0) != 0;
    }
    // drain: wait until the consumers released every stage this warp filled (bounded)
    if (lane == 0) {
      for (uint32_t k = 0; k < S && k < it; ++k) {
        const uint32_t j = it - 1 - k;
        if (owner(j) == pi) mbar_wait(&empty[j % S], (j / S) & 1, 200000000ull);
      }
    }
    return;
  }

  // --------------------------------------------------------------- consumers
  const int gid = lane >> 2, tig = lane & 3;
  const int rr = lane & 7, mi = lane >> 3;
  uint32_t it = 0;
  bool alive = true;
  for (int unit = blockIdx.x; unit < num_units; unit += gridDim.x) {
    const int row = unit / a.splits, sp = unit % a.splits;
    const int b = row / a.Hkv, g = row % a.Hkv;
    const int cnt = min(a.kept_count[row], a.max_kept);
    const int e0 = sp * a.split_len, e1 = min(cnt, e0 + a.split_len);
    const int Tb = seq_len(a, b);

    // Q^T fragments: head (8*nt + gid) of the group, dims 16ks + 2tig (+1), +8
    uint32_t bq[NT][Cfg::kKsteps][2];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const int hl = nt * 8 + gid;
      const bool hv = hl < a.G;
      const uint32_t* qrow = reinterpret_cast<const uint32_t*>(
          static_cast<const char*>(a.q) +
          ((static_cast<int64_t>(b) * a.Hq + g * a.G + (hv ? hl : 0)) * D) * 2);
#pragma unroll
      for (int ks = 0; ks < Cfg::kKsteps; ++ks) {
        bq[nt][ks][0] = hv ? qrow[(ks * 16 + 2 * tig) / 2] : 0u;
        bq[nt][ks][1] = hv ? qrow[(ks * 16 + 8 + 2 * tig) / 2] : 0u;
      }
    }
    float m[NT][2], l[NT][2];
    float acc[NT][Cfg::kKsteps][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      m[nt][0] = m[nt][1] = -INFINITY;
      l[nt][0] = l[nt][1] = 0.f;
#pragma unroll
      for (int mt = 0; mt < Cfg::kKsteps; ++mt)
        acc[nt][mt][0] = acc[nt][mt][1] = acc[nt][mt][2] = acc[nt][mt][3] = 0.f;
    }

    // stages of this unit until the one marked last (none for an empty unit)
    for (bool last = e1 <= e0; !last && alive; ++it) {
      const int s = it % S;
      if (!mbar_wait(&full[s], (it / S) & 1)) {
        if (lane == 0) report(a.status, BSA_DEV_TIMEOUT);
        alive = false;
        break;
      }
      last = sinfo[s * Sm::kInfoW + 4] != 0;
      const int tok0 = sinfo[s * Sm::kInfoW + warp];   // first token of this warp's slot
      if (tok0 >= 0) {
        const uint32_t kb = smem_u32(ring + s * Cfg::kStageBytes);
        const uint32_t vb = kb + Cfg::kTileBytes;
        const int valid = Tb - tok0;  // tokens of this warp's slot that exist
        // ---- S^T = K_w Q^T
        float sc[NT][4];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) sc[nt][0] = sc[nt][1] = sc[nt][2] = sc[nt][3] = 0.f;
#pragma unroll
        for (int ks = 0; ks < Cfg::kKsteps; ++ks) {
          const int trow = 16 * warp + rr + 8 * (mi & 1);
          const int chunk = 2 * ks + (mi >> 1);
          uint32_t af[4];
          ldsm_x4(af, kb + (chunk >> 3) * 8192 + swz128(trow, chunk & 7));
#pragma unroll
          for (int nt = 0; nt < NT; ++nt) mma_bf16(sc[nt], af, bq[nt][ks][0], bq[nt][ks][1]);
        }
        // ---- online softmax (log2 domain) per head column
        const bool v0 = gid < valid, v1 = gid + 8 < valid;
        uint32_t phi[NT][2], plo[NT][2];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          float p[4];
#pragma unroll
          for (int c = 0; c < 2; ++c) {
            const float s0 = v0 ? sc[nt][c] * a.scale_log2 : -INFINITY;
            const float s1 = v1 ? sc[nt][2 + c] * a.scale_log2 : -INFINITY;
            float mx = fmaxf(s0, s1);
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
            const float mnew = fmaxf(m[nt][c], mx);
            const float base = mnew == -INFINITY ? 0.f : mnew;
            const float corr = ex2(m[nt][c] - base);
            m[nt][c] = mnew;
            p[c] = ex2(s0 - base);
            p[2 + c] = ex2(s1 - base);
            l[nt][c] = l[nt][c] * corr + p[c] + p[2 + c];
#pragma unroll
            for (int mt = 0; mt < Cfg::kKsteps; ++mt) {
              acc[nt][mt][c] *= corr;
              acc[nt][mt][2 + c] *= corr;
            }
          }
          // P^T B-fragments (hi and lo bf16 parts)
          const uint32_t h0 = pack_bf16(p[0], p[1]);
          const uint32_t h1 = pack_bf16(p[2], p[3]);
          const float2 f0 = unpack_bf16(h0), f1 = unpack_bf16(h1);
          const uint32_t l0 = pack_bf16(p[0] - f0.x, p[1] - f0.y);
          const uint32_t l1 = pack_bf16(p[2] - f1.x, p[3] - f1.y);
          phi[nt][0] = movmatrix_t(h0);
          phi[nt][1] = movmatrix_t(h1);
          plo[nt][0] = movmatrix_t(l0);
          plo[nt][1] = movmatrix_t(l1);
        }
        // ---- O^T += V_w^T P^T
        const bool partial = valid < 16;
#pragma unroll
        for (int mt = 0; mt < Cfg::kKsteps; ++mt) {
          const int trow = 16 * warp + rr + 8 * (mi >> 1);
          const int chunk = 2 * mt + (mi & 1);
          uint32_t af[4];
          ldsm_x4_t(af, vb + (chunk >> 3) * 8192 + swz128(trow, chunk & 7));
          if (partial) {
            // zero V of tokens that do not exist (their P is 0; avoid 0 * NaN)
            const int t0 = 2 * tig, t1 = 2 * tig + 8;
            const uint32_t m0 = (t0 < valid ? 0x0000ffffu : 0u) | (t0 + 1 < valid ? 0xffff0000u : 0u);
            const uint32_t m1 = (t1 < valid ? 0x0000ffffu : 0u) | (t1 + 1 < valid ? 0xffff0000u : 0u);
            af[0] &= m0;
            af[1] &= m0;
            af[2] &= m1;
            af[3] &= m1;
          }
#pragma unroll
          for (int nt = 0; nt < NT; ++nt) {
            mma_bf16(acc[nt][mt], af, phi[nt][0], phi[nt][1]);
            mma_bf16(acc[nt][mt], af, plo[nt][0], plo[nt][1]);
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[s]);
    }

    // ---- merge the four warps' partials of this unit
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        float lv = l[nt][c];
        lv += __shfl_xor_sync(0xffffffffu, lv, 4);
        lv += __shfl_xor_sync(0xffffffffu, lv, 8);
        lv += __shfl_xor_sync(0xffffffffu, lv, 16);
        const int h = nt * 8 + 2 * tig + c;
        if (gid == 0) {
          stats[(warp * NH + h) * 2 + 0] = m[nt][c];
          stats[(warp * NH + h) * 2 + 1] = lv;
        }
#pragma unroll
        for (int mt = 0; mt < Cfg::kKsteps; ++mt) {
          comb[(warp * NH + h) * D + 16 * mt + gid] = acc[nt][mt][c];
          comb[(warp * NH + h) * D + 16 * mt + gid + 8] = acc[nt][mt][2 + c];
        }
      }
    }
    consumer_sync();
    const int tid = threadIdx.x;
    for (int x = tid; x < a.G * D; x += kConsumerWarps * 32) {
      const int h = x / D, dd = x % D;
      float M = -INFINITY;
#pragma unroll
      for (int w = 0; w < kConsumerWarps; ++w) M = fmaxf(M, stats[(w * NH + h) * 2]);
      const float base = M == -INFINITY ? 0.f : M;
      float o = 0.f, L = 0.f;
#pragma unroll
      for (int w = 0; w < kConsumerWarps; ++w) {
        const float f = ex2(stats[(w * NH + h) * 2] - base);
        o += comb[(w * NH + h) * D + dd] * f;
        L += stats[(w * NH + h) * 2 + 1] * f;
      }
      const int64_t pidx = static_cast<int64_t>(unit) * a.G + h;
      a.part_o[pidx * D + dd] = o;
      if (dd == 0) {
        a.part_ml[pidx * 2 + 0] = M;
        a.part_ml[pidx * 2 + 1] = L;
      }
    }
    if (!consumer_sync_and(alive)) break;
  }
}

// One warp per (b, h): combine the splits of its row. The lanes read 32 splits'
// (m, l) at once; the partial outputs of a chunk are then read with independent
// loads (unrolled), added in split order.
template <int D>
__global__ void __launch_bounds__(256) lse_merge_kernel(const DecodeArgs a) {
  grid_dependency_wait();   // partials come from the attention kernel
  const int wid = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (wid >= a.B * a.Hq) return;
  const int b = wid / a.Hq, h = wid % a.Hq;
  const int g = h / a.G, hl = h % a.G;
  const int row = b * a.Hkv + g;
  constexpr int PER = D / 32;
  const int64_t p0 = static_cast<int64_t>(row) * a.splits * a.G + hl;   // split s: p0 + s * G
  float M = -INFINITY;
  for (int s = lane; s < a.splits; s += 32) M = fmaxf(M, a.part_ml[(p0 + static_cast<int64_t>(s) * a.G) * 2]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
  const float base = M == -INFINITY ? 0.f : M;
  float o[PER];
#pragma unroll
  for (int q = 0; q < PER; ++q) o[q] = 0.f;
  float L = 0.f;
  for (int c = 0; c < a.splits; c += 32) {
    const int s = c + lane;
    float f = 0.f;
    if (s < a.splits) {
      const int64_t pidx = p0 + static_cast<int64_t>(s) * a.G;
      f = ex2(a.part_ml[pidx * 2] - base);
      L += a.part_ml[pidx * 2 + 1] * f;
    }
    const int nn = min(32, a.splits - c);
#pragma unroll 4
    for (int j = 0; j < nn; ++j) {
      const float fj = __shfl_sync(0xffffffffu, f, j);
      const float* po = a.part_o + (p0 + static_cast<int64_t>(c + j) * a.G) * D;
#pragma unroll
      for (int q = 0; q < PER; ++q) o[q] += po[lane + 32 * q] * fj;
    }
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) L += __shfl_xor_sync(0xffffffffu, L, off);
  const float inv = L > 0.f ? 1.0f / L : 0.f;
  const int64_t obase = (static_cast<int64_t>(b) * a.Hq + h) * D;
  __nv_bfloat16* ob = static_cast<__nv_bfloat16*>(a.o);
#pragma unroll
  for (int q = 0; q < PER; ++q) {
    const float v = o[q] * inv;
    ob[obase + lane + 32 * q] = __float2bfloat16_rn(v);
    if (a.o_f32) a.o_f32[obase + lane + 32 * q] = v;
  }
  if (lane == 0) {
    // natural-log LSE from the log2-domain running max and sum
    a.lse[static_cast<int64_t>(b) * a.Hq + h] =
        L > 0.f ? (M + log2f(L)) * 0.69314718055994530942f : -INFINITY;
  }
}

template <int D, int NT>
cudaError_t launch_dn(const DecodeArgs& a, const CUtensorMap& tk, const CUtensorMap& tv,
                      const CUtensorMap& tk16, const CUtensorMap& tv16, int num_units, int num_sms,
                      cudaStream_t s) {
  const int smem = DecodeSmem<D, NT>::kTotal;
  auto kern = decode_attn_kernel<D, NT>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  const int grid = num_units < num_sms ? num_units : num_sms;
  if (grid > 0) {
    e = launch_pdl(kern, dim3(grid), dim3(kThreads), smem, s, a, tk, tv, tk16, tv16, num_units);
    if (e != cudaSuccess) return e;
  }
  const int warps = a.B * a.Hq;
  return launch_pdl(lse_merge_kernel<D>, dim3((warps * 32 + 255) / 256), dim3(256), 0, s, a);
}

}  // namespace

void decode_split_plan(int rows, int max_kept, int num_sms, int* splits, int* split_len) {
  // minimise (units per CTA, rounded up) * (blocks per unit + per-unit overhead)
  const double overhead = 2.0;
  int best_len = max_kept > 0 ? max_kept : 1;
  double best = 1e300;
  for (int len = 1; len <= (max_kept > 0 ? max_kept : 1); ++len) {
    const int sp = (max_kept + len - 1) / len;
    const long units = static_cast<long>(rows) * (sp > 0 ? sp : 1);
    const long waves = (units + num_sms - 1) / num_sms;
    const double cost = static_cast<double>(waves) * (len + overhead);
    if (cost < best - 1e-9) {
      best = cost;
      best_len = len;
    }
  }
  *split_len = best_len;
  *splits = max_kept > 0 ? (max_kept + best_len - 1) / best_len : 1;
}

cudaError_t launch_decode(const DecodeArgs& a, const DecodeMaps& m, int num_units, int num_sms,
                          cudaStream_t s) {
  const int NT = a.G > 8 ? 2 : 1;
  if (a.d == 128) {
    return NT == 1 ? launch_dn<128, 1>(a, m.k, m.v, m.k16, m.v16, num_units, num_sms, s)
                   : launch_dn<128, 2>(a, m.k, m.v, m.k16, m.v16, num_units, num_sms, s);
  }
  return NT == 1 ? launch_dn<64, 1>(a, m.k, m.v, m.k16, m.v16, num_units, num_sms, s)
                 : launch_dn<64, 2>(a, m.k, m.v, m.k16, m.v16, num_units, num_sms, s);
}

}  // namespace bsa
