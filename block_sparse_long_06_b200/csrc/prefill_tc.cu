// Block-sparse causal prefill attention on the 5th-generation tensor cores
// (tcgen05.mma with accumulators in tensor memory).
//
// For each query token tq of query block i and head h of kv group g: exact
// softmax over the tokens tk <= tq of the kept key blocks of row (b, g, i) (HGA,
// Central mechanism §4: exact token-level attention over the routed set; the
// diagonal block is always kept and is causally masked).
//
// Design:
//  * unit = (b, g, query block i, quad of heads): up to 4 heads x 64 queries,
//    as two 128-row Q tiles (two heads each). Persistent CTAs (one per SM) take
//    units from a global counter in (b, g)-major, heavy-first order, so the K/V
//    of one kv head is shared through L2 by all SMs at a time;
//  * kept key blocks are processed in pairs: a pair is a 128-key tile, so every
//    MMA has N = 128 (a lone last block uses N = 64);
//  * warp 0 (one lane) loads Q once per unit and the K (bf16) and V (fp16) tiles of
//    each pair with TMA (128-byte swizzle) into a 2-stage ring;
//  * warp 1 (one lane) issues the MMAs: S_t = Q_t K^T (bf16, M = 128, N = 128,
//    K = d) into tensor memory, and after the softmax O_t += P_t V (fp16, P read
//    from tensor memory, V from shared memory, N = d);
//  * warps 4-7 and 8-11 are the softmax warpgroups of tile 0 and tile 1 (one
//    thread per row, i.e. per tensor-memory lane). They read S, apply the causal
//    mask and the online softmax in fp32 (log2 domain), and write P as fp16 over
//    the S columns. The running max is only moved (and O rescaled in tensor
//    memory) when it grows by more than 2^8, so P stays <= 256 and the rescale is
//    rare; the final normalisation uses the same max, so the result is exact.
//    While one warpgroup works on its softmax the tensor core runs the other
//    tile's MMAs;
//  * epilogue: O / l from tensor memory straight to global memory (bf16, and fp32
//    when requested), LSE in natural log.
// Tensor memory: 512 columns: S/P of tile 0 at 0, of tile 1 at 128; O of tile 0
// at 256, of tile 1 at 384. Every wait is bounded; on a timeout the kernel sets
// BSA_DEV_TIMEOUT, drains, frees its tensor memory and returns.
#include "bsa_common.cuh"
#include "bsa_internal.h"
#include "tcgen05.cuh"

namespace bsa {
namespace {

constexpr int kThreads = 384;
constexpr int kWarpLoad = 0, kWarpMma = 1, kWarpSm0 = 4;
constexpr uint32_t kTmemCols = 512;

template <int D>
struct Cfg {
  static constexpr int kHalves = D / 64;            // 64-dim slabs of 128 rows x 128 B
  static constexpr int kSlab = 128 * 128;
  static constexpr int kTile = kHalves * kSlab;     // 128 rows x D (one Q tile / K pair / V pair)
  static constexpr int kStages = D == 128 ? 2 : 4;
  static constexpr int kStage = 2 * kTile;          // K pair + V pair
  static constexpr int kKsteps = D / 16;
  static constexpr int kOffKV = 2 * kTile;
  static constexpr int kOffBar = kOffKV + kStages * kStage;
  static constexpr int kSmem = kOffBar + 512 + 1024;
};

struct UnitInfo {
  int u;  // unit id or -1 (no more work)
};

struct Bars {
  uint64_t info_full[2], info_empty[2];
  uint64_t q_full, q_empty;
  uint64_t kv_full[4], kv_empty[4];
  uint64_t s_full[2], p_ready[2], o_done[2], o_free[2];
  uint64_t mma_done;
  UnitInfo info[2];
  uint32_t tmem_base;
  int abort_flag;
};

struct Geo {
  int b, g, i, hq, cnt, ntiles;
  int64_t krow;
};

BSA_DEVFN Geo unit_geo(const PrefillArgs& a, int u) {
  Geo G;
  const int hq_n = a.G >= 4 ? a.G / 4 : 1;
  const int per_bg = a.nqb * hq_n;
  const int bg = u / per_bg;
  const int rem = u - bg * per_bg;
  G.i = a.nqb - 1 - rem / hq_n;
  G.hq = rem % hq_n;
  G.b = bg / a.Hkv;
  G.g = bg % a.Hkv;
  G.krow = static_cast<int64_t>(bg) * a.nqb + G.i;
  G.cnt = min(a.kept_count[G.krow], a.max_kept);
  G.ntiles = a.G >= 4 ? 2 : 1;
  return G;
}

// Row of the first token of block `blk` (rows of width d) or -1 when invalid.
BSA_DEVFN int64_t krow_of(const CacheView& c, const PrefillArgs& a, int b, int g, int blk, int i) {
  if (blk < 0 || blk > i) return -1;
  int64_t phys = blk;
  if (c.page_table != nullptr) {
    phys = c.page_table[static_cast<int64_t>(b) * c.pt_stride + blk];
    if (phys < 0 || phys >= c.num_pages) return -1;
  }
  const int rows = min(kBlock, a.T - blk * kBlock);
  const int64_t off = static_cast<int64_t>(b) * c.seq_stride + phys * c.block_stride +
                      static_cast<int64_t>(g) * c.head_stride;
  if (off < 0 || off + static_cast<int64_t>(rows) * a.d > c.extent) return -1;
  return off / a.d;
}

// Head (within the group) of row r of tile t of head quad hq.
BSA_DEVFN int row_head(const PrefillArgs& a, int hq, int t, int r) {
  const int hl = 4 * hq + 2 * t + (r >> 6);
  return hl < a.G ? hl : a.G - 1;
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    prefill_tc_kernel(const PrefillArgs a, const __grid_constant__ CUtensorMap tmq,
                      const __grid_constant__ CUtensorMap tmk,
                      const __grid_constant__ CUtensorMap tmv, int* unit_counter,
                      const int num_units) {
  using C = Cfg<D>;
  constexpr int S = C::kStages;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  Bars* bars = reinterpret_cast<Bars*>(smem + C::kOffBar);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int x = 0; x < 2; ++x) {
      mbar_init(&bars->info_full[x], 1);
      mbar_init(&bars->info_empty[x], 1 + 8);   // MMA lane + one lane per softmax warp
      mbar_init(&bars->s_full[x], 1);
      mbar_init(&bars->p_ready[x], 4);          // one lane per warp of the warpgroup
      mbar_init(&bars->o_done[x], 1);
      mbar_init(&bars->o_free[x], 4);
    }
    for (int s = 0; s < S; ++s) {
      mbar_init(&bars->kv_full[s], 1);
      mbar_init(&bars->kv_empty[s], 1);
    }
    mbar_init(&bars->q_full, 1);
    mbar_init(&bars->q_empty, 1);
    mbar_init(&bars->mma_done, 1);
    bars->abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kWarpMma) {
    tc::tmem_alloc(&bars->tmem_base, kTmemCols);
    tc::tmem_relinquish();
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = bars->tmem_base;

  if (warp == kWarpLoad) {
    // ------------------------------------------------------------------ loader
    if (lane == 0) {
      prefetch_tensormap(&tmq);
      prefetch_tensormap(&tmk);
      prefetch_tensormap(&tmv);
      uint32_t un = 0, kc = 0;
      bool ok = true;
      while (ok) {
        int u = atomicAdd(unit_counter, 1);
        if (u >= num_units) u = -1;
        const int slot = un & 1;
        if (!mbar_wait(&bars->info_empty[slot], ((un >> 1) & 1) ^ 1)) { ok = false; break; }
        bars->info[slot].u = u;
        mbar_arrive(&bars->info_full[slot]);
        if (u < 0 || *reinterpret_cast<volatile int*>(&bars->abort_flag)) break;
        const Geo G = unit_geo(a, u);
        const int32_t* klist = a.kept + G.krow * a.max_kept;
        // Q tiles (two heads per tile, one 64-row box per head and 64-dim slab)
        if (!mbar_wait(&bars->q_empty, (un & 1) ^ 1)) { ok = false; break; }
        mbar_arrive_expect_tx(&bars->q_full, G.ntiles * 2 * C::kHalves * 8192);
        for (int t = 0; t < G.ntiles; ++t)
          for (int hh = 0; hh < 2; ++hh) {
            const int h = G.g * a.G + row_head(a, G.hq, t, hh * 64);
            const int32_t qr = static_cast<int32_t>((static_cast<int64_t>(G.b) * a.Hq + h) * a.T +
                                                    G.i * kBlock);
            for (int x = 0; x < C::kHalves; ++x)
              tma_load_2d(smem + t * C::kTile + x * C::kSlab + hh * 8192, &tmq, x * 64, qr,
                          &bars->q_full);
          }
        // K / V pairs
        const int npairs = (G.cnt + 1) / 2;
        for (int pp = 0; pp < npairs; ++pp, ++kc) {
          const int s = kc % S;
          if (!mbar_wait(&bars->kv_empty[s], ((kc / S) & 1) ^ 1)) { ok = false; break; }
          const int nb = (2 * pp + 1 < G.cnt) ? 2 : 1;
          unsigned char* st = smem + C::kOffKV + s * C::kStage;
          mbar_arrive_expect_tx(&bars->kv_full[s], nb * C::kHalves * 8192 * 2);
          for (int q = 0; q < nb; ++q) {
            int blk = klist[2 * pp + q];
            int64_t rk = krow_of(a.k, a, G.b, G.g, blk, G.i);
            if (rk < 0) {
              // masked by the softmax; load the (always valid) diagonal block instead
              report(a.status, blk < 0 || blk > G.i ? BSA_DEV_BAD_KEPT : BSA_DEV_BAD_PAGE);
              blk = G.i;
              rk = krow_of(a.k, a, G.b, G.g, blk, G.i);
              if (rk < 0) rk = 0;
            }
            const int32_t rv = static_cast<int32_t>(
                (static_cast<int64_t>(G.b) * a.Hkv + G.g) * a.Tpad + blk * kBlock);
            for (int x = 0; x < C::kHalves; ++x) {
              tma_load_2d(st + x * C::kSlab + q * 8192, &tmk, x * 64, static_cast<int32_t>(rk),
                          &bars->kv_full[s]);
              tma_load_2d(st + C::kTile + x * C::kSlab + q * 8192, &tmv, x * 64, rv,
                          &bars->kv_full[s]);
            }
          }
        }
        if (!ok) break;
        ++un;
      }
      if (!ok) {
        bars->abort_flag = 1;
        report(a.status, BSA_DEV_TIMEOUT);
      }
      // copies in flight must land before the CTA exits (bounded)
      for (uint32_t k = (kc > S ? kc - S : 0); k < kc; ++k)
        mbar_wait(&bars->kv_full[k % S], (k / S) & 1, 100000000ull);
    }
  } else if (warp == kWarpMma) {
    // --------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      const uint32_t idS128 = tc::idesc_f16(128, 128, 1, false);
      const uint32_t idS64 = tc::idesc_f16(128, 64, 1, false);
      const uint32_t idPV = tc::idesc_f16(128, D, 0, true);
      const uint32_t sbase = smem_u32(smem);
      uint32_t un = 0, kc = 0;
      bool ok = true;
      while (ok) {
        const int slot = un & 1;
        if (!mbar_wait(&bars->info_full[slot], (un >> 1) & 1)) { ok = false; break; }
        const int u = bars->info[slot].u;
        mbar_arrive(&bars->info_empty[slot]);
        if (u < 0 || *reinterpret_cast<volatile int*>(&bars->abort_flag)) break;
        const Geo G = unit_geo(a, u);
        const int npairs = (G.cnt + 1) / 2;
        if (!mbar_wait(&bars->q_full, un & 1)) { ok = false; break; }
        for (int pp = 0; pp < npairs && ok; ++pp, ++kc) {
          const int s = kc % S;
          if (!mbar_wait(&bars->kv_full[s], (kc / S) & 1)) { ok = false; break; }
          const int nk = (2 * pp + 1 < G.cnt) ? 128 : 64;
          const uint32_t kbase = sbase + C::kOffKV + s * C::kStage;
          const uint32_t vbase = kbase + C::kTile;
          for (int t = 0; t < G.ntiles; ++t) {
            if (kc > 0 && !mbar_wait(&bars->o_done[t], (kc - 1) & 1)) { ok = false; break; }
            tc::fence_after_sync();
            const uint32_t qbase = sbase + t * C::kTile;
            for (int ks = 0; ks < C::kKsteps; ++ks) {
              const uint32_t off = (ks >> 2) * C::kSlab + (ks & 3) * 32;
              tc::mma_ss(tmem + 128 * t, tc::smem_desc_sw128(qbase + off, 16, 1024),
                         tc::smem_desc_sw128(kbase + off, 16, 1024), nk == 128 ? idS128 : idS64,
                         ks > 0);
            }
            tc::commit(&bars->s_full[t]);
          }
          if (!ok) break;
          if (pp == npairs - 1) tc::commit(&bars->q_empty);
          for (int t = 0; t < G.ntiles; ++t) {
            if (pp == 0 && un > 0 && !mbar_wait(&bars->o_free[t], (un - 1) & 1)) { ok = false; break; }
            if (!mbar_wait(&bars->p_ready[t], kc & 1)) { ok = false; break; }
            tc::fence_after_sync();
            for (int kk = 0; kk < nk / 16; ++kk)
              tc::mma_ts(tmem + 256 + 128 * t, tmem + 128 * t + kk * 8,
                         tc::smem_desc_sw128(vbase + kk * 2048, C::kSlab, 1024), idPV,
                         pp > 0 || kk > 0);
            tc::commit(&bars->o_done[t]);
          }
          if (!ok) break;
          tc::commit(&bars->kv_empty[s]);
        }
        if (!ok) break;
        ++un;
      }
      if (!ok) {
        bars->abort_flag = 1;
        report(a.status, BSA_DEV_TIMEOUT);
      }
      // every MMA issued so far must finish before tensor memory is freed (bounded)
      tc::commit(&bars->mma_done);
      mbar_wait(&bars->mma_done, 0, 200000000ull);
    }
  } else if (warp >= kWarpSm0) {
    // ----------------------------------------------------------- softmax warps
    const int t = (warp - kWarpSm0) >> 2;            // tile of this warpgroup
    const int q4 = warp & 3;                         // tensor-memory lane quarter
    const int r = q4 * 32 + lane;                    // row of the tile
    const uint32_t lane_addr = static_cast<uint32_t>(q4 * 32) << 16;
    const uint32_t s_col = tmem + lane_addr + 128 * t;
    const uint32_t o_col = tmem + lane_addr + 256 + 128 * t;
    uint32_t un = 0, kc = 0;
    while (true) {
      const int slot = un & 1;
      if (!__all_sync(0xffffffffu, mbar_wait(&bars->info_full[slot], (un >> 1) & 1))) {
        if (lane == 0) {
          bars->abort_flag = 1;
          report(a.status, BSA_DEV_TIMEOUT);
        }
        break;
      }
      const int u = bars->info[slot].u;
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->info_empty[slot]);
      if (u < 0) break;
      const Geo G = unit_geo(a, u);
      ++un;
      if (t >= G.ntiles) continue;
      const int32_t* klist = a.kept + G.krow * a.max_kept;
      const int npairs = (G.cnt + 1) / 2;
      const int tq = G.i * kBlock + (r & 63);
      float m = -INFINITY, l = 0.f;
      bool ok = true;
      for (int pp = 0; pp < npairs; ++pp, ++kc) {
        if (!__all_sync(0xffffffffu, mbar_wait(&bars->s_full[t], kc & 1))) { ok = false; break; }
        tc::fence_after_sync();
        const int nb = (2 * pp + 1 < G.cnt) ? 2 : 1;     // key blocks in this pair
        // per block (= 64-column half): 0 fully visible, 1 causal diagonal, 2 masked
        int mode[2];
        int blk[2];
#pragma unroll
        for (int q = 0; q < 2; ++q) {
          blk[q] = q < nb ? klist[2 * pp + q] : -1;
          const bool valid = q < nb && krow_of(a.k, a, G.b, G.g, blk[q], G.i) >= 0;
          mode[q] = !valid ? 2 : (blk[q] == G.i ? 1 : 0);
        }
        // pass 1: row max of the scaled, masked scores (log2 domain)
        float mx = -INFINITY;
#pragma unroll
        for (int q = 0; q < 2; ++q) {
          if (q < nb && mode[q] != 2) {
            uint32_t r0[32], r1[32];
            tc::ld32(s_col + 64 * q, r0);
            tc::ld32(s_col + 64 * q + 32, r1);
            tc::wait_ld();
            const int lim = mode[q] == 1 ? (tq - blk[q] * kBlock) : 63;  // last visible column
#pragma unroll
            for (int x = 0; x < 32; ++x) {
              if (x <= lim) mx = fmaxf(mx, __uint_as_float(r0[x]));
              if (x + 32 <= lim) mx = fmaxf(mx, __uint_as_float(r1[x]));
            }
          }
        }
        mx *= a.scale_log2;
        if (mx > m + 8.0f) {
          // move the running max: rescale l and the O row already accumulated
          const float f = ex2(m - mx);
          l *= f;
          if (pp > 0) {
#pragma unroll 1
            for (int c = 0; c < D / 32; ++c) {
              uint32_t ov[32];
              tc::ld32(o_col + c * 32, ov);
              tc::wait_ld();
#pragma unroll
              for (int x = 0; x < 32; ++x) ov[x] = __float_as_uint(__uint_as_float(ov[x]) * f);
              tc::st32(o_col + c * 32, ov);
            }
            tc::wait_st();
          }
          m = mx;
        }
        const float base = m == -INFINITY ? 0.f : m;
        // pass 2: P = 2^(s*scale - m) as fp16, written over the S columns already read
#pragma unroll
        for (int q = 0; q < 2; ++q) {
          if (q < nb) {
            uint32_t r0[32], r1[32];
            tc::ld32(s_col + 64 * q, r0);
            tc::ld32(s_col + 64 * q + 32, r1);
            tc::wait_ld();
            const int lim = mode[q] == 2 ? -1 : (mode[q] == 1 ? (tq - blk[q] * kBlock) : 63);
            uint32_t pk0[16], pk1[16];
#pragma unroll
            for (int x = 0; x < 16; ++x) {
              const float a0 = (2 * x <= lim) ? ex2(fmaf(__uint_as_float(r0[2 * x]), a.scale_log2, -base)) : 0.f;
              const float a1 = (2 * x + 1 <= lim) ? ex2(fmaf(__uint_as_float(r0[2 * x + 1]), a.scale_log2, -base)) : 0.f;
              const float b0 = (2 * x + 32 <= lim) ? ex2(fmaf(__uint_as_float(r1[2 * x]), a.scale_log2, -base)) : 0.f;
              const float b1 = (2 * x + 33 <= lim) ? ex2(fmaf(__uint_as_float(r1[2 * x + 1]), a.scale_log2, -base)) : 0.f;
              l += (a0 + a1) + (b0 + b1);
              pk0[x] = pack_f16(a0, a1);
              pk1[x] = pack_f16(b0, b1);
            }
            tc::st16(s_col + 32 * q, pk0);
            tc::st16(s_col + 32 * q + 16, pk1);
          }
        }
        tc::wait_st();
        tc::fence_before_sync();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->p_ready[t]);
      }
      if (!ok || *reinterpret_cast<volatile int*>(&bars->abort_flag)) {
        if (lane == 0) {
          bars->abort_flag = 1;
          report(a.status, BSA_DEV_TIMEOUT);
        }
        break;
      }
      // ---- epilogue: O / l
      if (!__all_sync(0xffffffffu, mbar_wait(&bars->o_done[t], (kc - 1) & 1))) {
        if (lane == 0) {
          bars->abort_flag = 1;
          report(a.status, BSA_DEV_TIMEOUT);
        }
        break;
      }
      tc::fence_after_sync();
      const int hl = row_head(a, G.hq, t, r);
      const bool write = tq < a.T && (4 * G.hq + 2 * t + (r >> 6)) < a.G;
      const int64_t ro = ((static_cast<int64_t>(G.b) * a.Hq + G.g * a.G + hl) * a.T + tq) * D;
      const float inv = l > 0.f ? 1.0f / l : 0.f;
#pragma unroll 1
      for (int c = 0; c < D / 32; ++c) {
        uint32_t ov[32];
        tc::ld32(o_col + c * 32, ov);
        tc::wait_ld();
        if (write) {
          uint32_t pk[16];
#pragma unroll
          for (int x = 0; x < 16; ++x)
            pk[x] = pack_bf16(__uint_as_float(ov[2 * x]) * inv, __uint_as_float(ov[2 * x + 1]) * inv);
          uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(a.o) + ro + c * 32);
#pragma unroll
          for (int x = 0; x < 4; ++x)
            dst[x] = make_uint4(pk[4 * x], pk[4 * x + 1], pk[4 * x + 2], pk[4 * x + 3]);
          if (a.o_f32) {
            float4* df = reinterpret_cast<float4*>(a.o_f32 + ro + c * 32);
#pragma unroll
            for (int x = 0; x < 8; ++x)
              df[x] = make_float4(__uint_as_float(ov[4 * x]) * inv, __uint_as_float(ov[4 * x + 1]) * inv,
                                  __uint_as_float(ov[4 * x + 2]) * inv,
                                  __uint_as_float(ov[4 * x + 3]) * inv);
          }
        }
      }
      if (write)
        a.lse[(static_cast<int64_t>(G.b) * a.Hq + G.g * a.G + hl) * a.T + tq] =
            l > 0.f ? (m + log2f(l)) * 0.69314718055994530942f : -INFINITY;
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->o_free[t]);
    }
  }

  tc::fence_before_sync();
  __syncthreads();
  if (warp == kWarpMma) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace

cudaError_t launch_prefill_tc(const PrefillArgs& a, const CUtensorMap& tq, const CUtensorMap& tk,
                              const CUtensorMap& tv16, int* unit_counter, int num_sms,
                              cudaStream_t s) {
  const int hq_n = a.G >= 4 ? a.G / 4 : 1;
  const int num_units = a.B * a.Hkv * a.nqb * hq_n;
  if (num_units <= 0) return cudaSuccess;
  cudaError_t e = cudaMemsetAsync(unit_counter, 0, sizeof(int), s);
  if (e != cudaSuccess) return e;
  const int grid = num_units < num_sms ? num_units : num_sms;
  if (a.d == 128) {
    e = cudaFuncSetAttribute(prefill_tc_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             Cfg<128>::kSmem);
    if (e != cudaSuccess) return e;
    prefill_tc_kernel<128><<<grid, kThreads, Cfg<128>::kSmem, s>>>(a, tq, tk, tv16, unit_counter,
                                                                    num_units);
  } else {
    e = cudaFuncSetAttribute(prefill_tc_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             Cfg<64>::kSmem);
    if (e != cudaSuccess) return e;
    prefill_tc_kernel<64><<<grid, kThreads, Cfg<64>::kSmem, s>>>(a, tq, tk, tv16, unit_counter,
                                                                  num_units);
  }
  return cudaGetLastError();
}

}  // namespace bsa
