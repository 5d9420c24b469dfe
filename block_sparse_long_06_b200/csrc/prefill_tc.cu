// Block-sparse causal prefill attention on the 5th-generation tensor cores
// (tcgen05.mma with accumulators in tensor memory).
//
// For each query token tq of query block i and head h of kv group g: exact
// softmax over the tokens tk <= tq of the kept key blocks of row (b, g, i) (HGA,
// Central mechanism §4: exact token-level attention over the routed set; the
// diagonal block is always kept and is causally masked).
//
// Design:
//  * unit = (b, g, query block i, quad of heads): up to 4 heads x 64 queries, as
//    two 128-row Q tiles (two heads each). Persistent CTAs (one per SM) take units
//    from a global counter in (b, g)-major, heavy-first order, so all SMs share the
//    K/V of one kv head through L2 at a time;
//  * a step is one kept key block (64 keys) for both tiles. Warp 0 (one lane)
//    loads Q once per unit and, per step, the K block (bf16) and the V block (fp16)
//    into one stage of a K/V ring (TMA, 128-byte swizzle);
//  * three MMA-issuing threads (warps 1-2: scores of tile 0/1, warp 3: P.V of both
//    tiles): a single thread can issue a tcgen05.mma only every ~50 cycles and a
//    commit costs about as much, so one issuer would leave the tensor core idle.
//    S_t(j) = Q_t K_j^T (bf16, M = 128, N = 64, K = d) goes to the tile's S buffer in
//    tensor memory; O_t += P_t(j) V_j (fp16, P read from tensor memory, N = d).
//    P has tensor-memory buffers of its own (two per tile), so the S buffer of a
//    tile is free as soon as its softmax warps have loaded S into registers: the
//    score MMAs of step j+1 run while the softmax of step j computes, and the P.V
//    is off that loop (a P buffer is reused two steps later). A K/V stage is
//    released by the P.V of every tile;
//  * warps 4-11 and 12-19 are the softmax warps of tile 0 and tile 1, 16 rows each
//    (tensor-memory lane quarter = warp % 4). They read the step's block id from
//    the kept list and validate it themselves, so the only per-step wait is for S.
//    A thread holds 2 rows x 16 columns of S, masks the causal diagonal block (and
//    blocks that failed validation), takes the row max (three-input max, then 2
//    shuffles), computes P with packed two-wide fp32 arithmetic and writes it as
//    fp16 to the P buffer. 3/8 of the exponentials run as a cubic polynomial on
//    the FMA pipes (exp2_poly below) instead of the MUFU unit. The running max only
//    moves (and O is rescaled in tensor memory, after the previous P.V has
//    completed) when it grows by more than 8 (log2), so P <= 256 fits fp16 and the
//    rescale is rare; the final normalisation uses the same max, so it is exact;
//  * epilogue: O / l from tensor memory straight to global memory (bf16, and fp32
//    when requested), LSE in natural log.
// Tensor memory: 512 columns: O of tile t at 128 t, S of tile t at 256 + 64 t, P
// buffer b of tile t at 384 + 64 t + 32 b. Every wait is bounded; on a timeout the kernel sets
// BSA_DEV_TIMEOUT, drains, frees its tensor memory and returns.
#include "bsa_common.cuh"
#include "bsa_internal.h"
#include "tcgen05.cuh"

namespace bsa {
namespace {

constexpr int kThreads = 640;
// warp roles: loader, score-MMA issuers of tiles 0/1, the P.V issuer of both tiles, and
// the 16 softmax warps 4-19 (a softmax warp's tensor-memory lane quarter is warp % 4).
// 20 warps = 5 per SM sub-partition, which leaves 96 registers a thread.
constexpr int kWarpLoad = 0, kWarpS0 = 1, kWarpPV = 3, kWarpSm0 = 4;
constexpr int kIssuers = 3;
constexpr uint32_t kTmemCols = 512;
constexpr int kMaxStages = 8;
constexpr int kPolyGroups = 3;  // of every 8 column groups of a row: exponentials by polynomial

template <int D>
struct Cfg {
  static constexpr int kHalves = D / 64;          // 64-dim slabs (rows of 128 B)
  static constexpr int kSlab = 128 * 128;         // one slab of a 128-row Q tile
  static constexpr int kTile = kHalves * kSlab;   // 128 rows x D
  static constexpr int kBlk = kHalves * 8192;     // one key block: 64 rows x D
  static constexpr int kStage = 2 * kBlk;         // K block, then V block
  static constexpr int kStages = D == 128 ? 5 : 8;
  static constexpr int kKsteps = D / 16;
  static constexpr int kOffKV = 2 * kTile;
  static constexpr int kOffBar = kOffKV + kStages * kStage;
};

struct UnitInfo {
  int u, b, g, i, hq, cnt;
};

struct Bars {
  uint64_t info_full[2], info_empty[2];
  uint64_t q_full, q_empty;
  uint64_t kv_full[kMaxStages], kv_empty[kMaxStages];
  uint64_t s_full[2], s_free[2];                        // [tile]
  uint64_t p_ready[2][2], pv_done[2][2];                 // [tile][P buffer]
  uint64_t o_free[2];
  uint64_t mma_done[kIssuers];
  UnitInfo info[2];
  uint32_t tmem_base;
  int abort_flag;
};

template <int D>
constexpr int smem_bytes() {
  return Cfg<D>::kOffBar + static_cast<int>(sizeof(Bars)) + 1024;
}
static_assert(smem_bytes<128>() <= 232448, "shared memory");

BSA_DEVFN bool aborted(Bars* b) { return *reinterpret_cast<volatile int*>(&b->abort_flag) != 0; }
BSA_DEVFN void set_abort(Bars* b, int32_t* status) {
  *reinterpret_cast<volatile int*>(&b->abort_flag) = 1;
  report(status, BSA_DEV_TIMEOUT);
}

BSA_DEVFN UnitInfo unit_of(const PrefillArgs& a, int u) {
  UnitInfo U;
  U.u = u;
  const int hq_n = a.G >= 4 ? a.G / 4 : 1;
  const int per_bg = a.nqb * hq_n;
  const int bg = u / per_bg;
  const int rem = u - bg * per_bg;
  U.i = a.nqb - 1 - rem / hq_n;
  U.hq = rem % hq_n;
  U.b = bg / a.Hkv;
  U.g = bg % a.Hkv;
  U.cnt = min(a.kept_count[static_cast<int64_t>(bg) * a.nqb + U.i], a.max_kept);
  return U;
}

// First block of query block i's segment, and the end of the segment (with seg_blocks
// = 1: i and i + 1).
BSA_DEVFN int seg_begin(const PrefillArgs& a, int i) { return (i / a.seg_blocks) * a.seg_blocks; }
BSA_DEVFN int seg_end(const PrefillArgs& a, int i) {
  return min(seg_begin(a, i) + a.seg_blocks, a.nqb);
}

// Element offset of the first token of block `blk` in cache `c`, or -1 when the block
// is not a valid kept block of query block i (out of range, bad page, past the extent).
BSA_DEVFN int64_t block_off(const CacheView& c, const PrefillArgs& a, int b, int g, int blk,
                            int i) {
  if (blk < 0 || blk >= seg_end(a, i)) return -1;
  int64_t phys = blk;
  if (c.page_table != nullptr) {
    phys = c.page_table[static_cast<int64_t>(b) * c.pt_stride + blk];
    if (phys < 0 || phys >= c.num_pages) return -1;
  }
  const int rows = min(kBlock, a.T - blk * kBlock);
  const int64_t off = static_cast<int64_t>(b) * c.seq_stride + phys * c.block_stride +
                      static_cast<int64_t>(g) * c.head_stride;
  if (off < 0 || off + static_cast<int64_t>(rows) * a.d > c.extent) return -1;
  return off;
}

// Row of the first token of block `blk` (rows of width d) or -1 when invalid.
BSA_DEVFN int64_t krow_of(const CacheView& c, const PrefillArgs& a, int b, int g, int blk, int i) {
  const int64_t off = block_off(c, a, b, g, blk, i);
  return off < 0 ? -1 : off / a.d;
}

// Head (within the group) of row r of tile t of head quad hq (clamped for G < 4).
BSA_DEVFN int row_head(const PrefillArgs& a, int hq, int t, int r) {
  const int hl = 4 * hq + 2 * t + (r >> 6);
  return hl < a.G ? hl : a.G - 1;
}

// Lane 0 waits on the barrier and the warp follows; the result is warp-uniform.
// (Polling from every lane only adds shared-memory traffic.)
BSA_DEVFN bool warp_wait(uint64_t* bar, uint32_t parity) {
  bool ok = true;
  if ((threadIdx.x & 31) == 0) ok = mbar_wait(bar, parity);
  return __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
}

BSA_DEVFN float max3(float x, float y, float z) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(x), "f"(y), "f"(z));
  return r;
}

// 2^x on the FMA pipes, for x <= 8 (two lanes at once). Split x = n + f with n the
// nearest integer (adding 1.5 * 2^23 rounds x into the low mantissa bits) and f in
// [-1/2, 1/2]; 2^f is a cubic fitted for minimal relative error on [-1/2, 1/2] by
// a Remez exchange (max relative error 7.5e-5, below the 2^-11 rounding of the fp16
// P it feeds); n is added to the exponent field. x is clamped at -126 (2^-126 is 0
// once P is rounded to fp16). The fit is reproduced by exp2_poly_fit.py.
BSA_DEVFN float2 exp2_poly(float2 x) {
  constexpr float kC0 = 0.9999280571937561f, kC1 = 0.6932609677314758f;
  constexpr float kC2 = 0.2426111251115799f, kC3 = 0.0551716685295105f;
  constexpr float kShift = 12582912.0f;  // 1.5 * 2^23
  x.x = fmaxf(x.x, -126.0f);
  x.y = fmaxf(x.y, -126.0f);
  const float2 r = __fadd2_rn(x, make_float2(kShift, kShift));
  const float2 nn = __ffma2_rn(r, make_float2(-1.0f, -1.0f), make_float2(kShift, kShift));  // -n
  const float2 f = __fadd2_rn(x, nn);
  float2 p = __ffma2_rn(make_float2(kC3, kC3), f, make_float2(kC2, kC2));
  p = __ffma2_rn(p, f, make_float2(kC1, kC1));
  p = __ffma2_rn(p, f, make_float2(kC0, kC0));
  return make_float2(__uint_as_float(__float_as_uint(p.x) + (__float_as_uint(r.x) << 23)),
                     __uint_as_float(__float_as_uint(p.y) + (__float_as_uint(r.y) << 23)));
}



// Mask mode of a kept block: 0 visible, 1 the causal diagonal, 2 failed validation
// (the loader then loads the diagonal block in its place), 3 a block of the query's
// own segment of a permuted key order (a key is visible when its original position,
// key_pos, is at most the query's; PBS-Attn, Methodology §2).
BSA_DEVFN int mode_of(const PrefillArgs& a, const UnitInfo& U, int blk) {
  if (block_off(a.k, a, U.b, U.g, blk, U.i) < 0) return 2;
  if (a.key_pos != nullptr) return blk >= seg_begin(a, U.i) ? 3 : 0;
  return blk == U.i ? 1 : 0;
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    prefill_tc_kernel(const PrefillArgs a, const __grid_constant__ CUtensorMap tmq,
                      const __grid_constant__ CUtensorMap tmk,
                      const __grid_constant__ CUtensorMap tmv, int* unit_counter,
                      const int num_units) {
  using C = Cfg<D>;
  constexpr int NS = C::kStages;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  Bars* bars = reinterpret_cast<Bars*>(smem + C::kOffBar);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int ntiles = a.G >= 4 ? 2 : 1;

  if (threadIdx.x == 0) {
    for (int x = 0; x < 2; ++x) {
      mbar_init(&bars->info_full[x], 1);
      mbar_init(&bars->info_empty[x], kIssuers + 16);   // every issuer and softmax warp
      mbar_init(&bars->s_full[x], 1);
      mbar_init(&bars->s_free[x], 8);             // the 8 softmax warps of a tile
      for (int y = 0; y < 2; ++y) {
        mbar_init(&bars->p_ready[x][y], 8);
        mbar_init(&bars->pv_done[x][y], 1);
      }
      mbar_init(&bars->o_free[x], 8);
    }
    for (int x = 0; x < kIssuers; ++x) mbar_init(&bars->mma_done[x], 1);
    for (int s = 0; s < NS; ++s) {
      mbar_init(&bars->kv_full[s], 1);
      mbar_init(&bars->kv_empty[s], 1);           // after the P.V of every tile
    }
    mbar_init(&bars->q_full, 1);
    mbar_init(&bars->q_empty, ntiles);            // the last score MMAs of every tile
    bars->abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kWarpS0) {
    tc::tmem_alloc(&bars->tmem_base, kTmemCols);
    tc::tmem_relinquish();
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = bars->tmem_base;

  if (warp == kWarpLoad) {
    // -------------------------------------------------------------- Q / K / V
    // Lane 0 takes units and loads Q; the warp resolves 32 steps' key blocks at a time
    // (one per lane: kept-list entry, validation, cache row), then lane 0 issues the
    // K and V copies of those steps back to back.
    if (lane == 0) {
      prefetch_tensormap(&tmq);
      prefetch_tensormap(&tmk);
      prefetch_tensormap(&tmv);
    }
    uint32_t un = 0, kc = 0;
    bool ok = true;
    while (ok) {
      const int slot = un & 1;
      int u = -1;
      if (lane == 0) {
        u = atomicAdd(unit_counter, 1);
        if (u >= num_units) u = -1;
        if (!mbar_wait_sleep(&bars->info_empty[slot], ((un >> 1) & 1) ^ 1)) {
          ok = false;
        } else {
          UnitInfo U0 = {u, 0, 0, 0, 0, 0};
          if (u >= 0) U0 = unit_of(a, u);
          bars->info[slot] = U0;
          mbar_arrive(&bars->info_full[slot]);
        }
      }
      ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
      u = __shfl_sync(0xffffffffu, u, 0);
      if (!ok || u < 0 || aborted(bars)) break;
      __syncwarp();
      const UnitInfo U = bars->info[slot];
      const int32_t* klist =
          a.kept + (static_cast<int64_t>(U.b * a.Hkv + U.g) * a.nqb + U.i) * a.max_kept;
      if (lane == 0) {
        if (!mbar_wait_sleep(&bars->q_empty, (un & 1) ^ 1)) {
          ok = false;
        } else {
          mbar_arrive_expect_tx(&bars->q_full, ntiles * 2 * C::kHalves * 8192);
          for (int t = 0; t < ntiles; ++t)
            for (int hh = 0; hh < 2; ++hh) {
              const int h = U.g * a.G + row_head(a, U.hq, t, hh * 64);
              const int32_t qr = static_cast<int32_t>(
                  (static_cast<int64_t>(U.b) * a.Hq + h) * a.T + U.i * kBlock);
              for (int x = 0; x < C::kHalves; ++x)
                tma_load_2d(smem + t * C::kTile + x * C::kSlab + hh * 8192, &tmq, x * 64, qr,
                            &bars->q_full);
            }
        }
      }
      ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
      if (!ok) break;
      const int n = U.cnt > 0 ? U.cnt : 1;
      const int32_t vrow0 = static_cast<int32_t>((static_cast<int64_t>(U.b) * a.Hkv + U.g) * a.Tpad);
      for (int base = 0; base < n && ok; base += 32) {
        const int jj = base + lane;
        int blk = U.i;
        int64_t rk = -1;
        if (jj < U.cnt) {
          blk = klist[jj];
          rk = krow_of(a.k, a, U.b, U.g, blk, U.i);
          if (rk < 0)
            report(a.status, blk < 0 || blk > U.i ? BSA_DEV_BAD_KEPT : BSA_DEV_BAD_PAGE);
        }
        if (rk < 0) {
          blk = U.i;   // load the always-valid diagonal block; its columns are masked
          rk = krow_of(a.k, a, U.b, U.g, blk, U.i);
          if (rk < 0) rk = 0;
        }
        const int n_here = min(32, n - base);
        for (int q = 0; q < n_here; ++q, ++kc) {
          const int blk_q = __shfl_sync(0xffffffffu, blk, q);
          const int64_t rk_q = __shfl_sync(0xffffffffu, rk, q);
          if (lane == 0) {
            const int s = kc % NS;
            if (!mbar_wait_sleep(&bars->kv_empty[s], ((kc / NS) & 1) ^ 1)) {
              ok = false;
            } else {
              mbar_arrive_expect_tx(&bars->kv_full[s], C::kStage);
              unsigned char* st = smem + C::kOffKV + s * C::kStage;
              for (int x = 0; x < C::kHalves; ++x)
                tma_load_2d(st + x * 8192, &tmk, x * 64, static_cast<int32_t>(rk_q),
                            &bars->kv_full[s]);
              for (int x = 0; x < C::kHalves; ++x)
                tma_load_2d(st + C::kBlk + x * 8192, &tmv, x * 64, vrow0 + blk_q * kBlock,
                            &bars->kv_full[s]);
            }
          }
          ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
          if (!ok) break;
        }
      }
      if (!ok) break;
      ++un;
    }
    if (lane == 0) {
      if (!ok) set_abort(bars, a.status);
      // copies in flight must land before the CTA exits (bounded)
      for (uint32_t k = (kc > NS ? kc - NS : 0); k < kc; ++k)
        mbar_wait_sleep(&bars->kv_full[k % NS], (k / NS) & 1, 100000000ull);
      if (un > 0) mbar_wait_sleep(&bars->q_full, (un - 1) & 1, 100000000ull);
    }
  } else if (warp == kWarpS0 || warp == kWarpS0 + 1) {
    // ------------------------------------------ score-MMA issuer of tile t
    // S_t(j) = Q_t K_j^T into the S buffer of tile t, once the softmax warps have
    // loaded S_t(j-1) from it.
    const int t = warp - kWarpS0;
    if (lane == 0) {
      const uint32_t idS = tc::idesc_f16(128, 64, 1, false);
      const uint32_t sbase = smem_u32(smem);
      const uint64_t dq = tc::smem_desc_sw128(sbase + t * C::kTile, 16, 1024);
      const uint32_t s_tm = tmem + 256 + 64 * t;
      uint32_t un = 0, kc = 0;
      bool ok = true;
      while (ok) {
        const int slot = un & 1;
        if (!mbar_wait_sleep(&bars->info_full[slot], (un >> 1) & 1)) { ok = false; break; }
        const UnitInfo U = bars->info[slot];
        mbar_arrive(&bars->info_empty[slot]);
        if (U.u < 0 || aborted(bars)) break;
        if (t >= ntiles) { ++un; continue; }
        const int n = U.cnt > 0 ? U.cnt : 1;
        if (!mbar_wait_sleep(&bars->q_full, un & 1)) { ok = false; break; }
        for (int jj = 0; jj < n; ++jj) {
          const uint32_t j = kc + jj;
          const int s = j % NS;
          if (j >= 1 && !mbar_wait_sleep(&bars->s_free[t], (j - 1) & 1)) { ok = false; break; }
          if (!mbar_wait_sleep(&bars->kv_full[s], (j / NS) & 1)) { ok = false; break; }
          tc::fence_after_sync();
          const uint64_t dk = tc::smem_desc_sw128(sbase + C::kOffKV + s * C::kStage, 16, 1024);
#pragma unroll
          for (int ks = 0; ks < C::kKsteps; ++ks)
            tc::mma_ss(s_tm, dq + (((ks >> 2) * C::kSlab + (ks & 3) * 32) >> 4),
                       dk + (((ks >> 2) * 8192 + (ks & 3) * 32) >> 4), idS, ks > 0);
          tc::commit(&bars->s_full[t]);
        }
        if (!ok) break;
        tc::commit(&bars->q_empty);   // Q of this tile is free once these MMAs complete
        kc += n;
        ++un;
      }
      if (!ok) set_abort(bars, a.status);
      // every MMA this thread issued must finish before tensor memory is freed (bounded)
      tc::commit(&bars->mma_done[t]);
      mbar_wait_sleep(&bars->mma_done[t], 0, 200000000ull);
    }
  } else if (warp == kWarpPV) {
    // ------------------------------------------- P.V issuer of both tiles
    // O_t += P_t(j) V_j once the softmax has written P_t(j); the first step of a unit
    // overwrites O once the epilogue of the previous unit has read it. The commit on
    // kv_empty releases the K/V stage (its S MMAs completed before P was written).
    if (lane == 0) {
      const uint32_t idPV = tc::idesc_f16(128, D, 0, true);
      const uint32_t sbase = smem_u32(smem);
      uint32_t un = 0, kc = 0;
      bool ok = true;
      while (ok) {
        const int slot = un & 1;
        if (!mbar_wait_sleep(&bars->info_full[slot], (un >> 1) & 1)) { ok = false; break; }
        const UnitInfo U = bars->info[slot];
        mbar_arrive(&bars->info_empty[slot]);
        if (U.u < 0 || aborted(bars)) break;
        const int n = U.cnt > 0 ? U.cnt : 1;
        for (int jj = 0; jj < n && ok; ++jj) {
          const uint32_t j = kc + jj;
          const int s = j % NS;
          const uint64_t dv =
              tc::smem_desc_sw128(sbase + C::kOffKV + s * C::kStage + C::kBlk, 8192, 1024);
          for (int t = 0; t < ntiles; ++t) {
            if (jj == 0 && un > 0 && !mbar_wait_sleep(&bars->o_free[t], (un - 1) & 1)) { ok = false; break; }
            if (!mbar_wait_sleep(&bars->p_ready[t][j & 1], (j >> 1) & 1)) { ok = false; break; }
            tc::fence_after_sync();
            const uint32_t o_tm = tmem + 128 * t, p_tm = tmem + 384 + 64 * t + 32 * (j & 1);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              tc::mma_ts(o_tm, p_tm + kk * 8, dv + ((kk * 2048) >> 4), idPV, jj > 0 || kk > 0);
            tc::commit(&bars->pv_done[t][j & 1]);
          }
          if (ok) tc::commit(&bars->kv_empty[s]);
        }
        if (!ok) break;
        kc += n;
        ++un;
      }
      if (!ok) set_abort(bars, a.status);
      tc::commit(&bars->mma_done[2]);
      mbar_wait_sleep(&bars->mma_done[2], 0, 200000000ull);
    }
  } else if (warp >= kWarpSm0 && warp < kWarpSm0 + 16) {
    // ----------------------------------------------------------- softmax warps
    // 8 warps per tile: warp w owns the 16 rows [32*(w%4) + 16*h, +16) of its tile
    // (w % 4 is the tensor-memory lane quarter it may access, h its half of it).
    // Thread (t0 = lane % 4, t1 = lane / 4) holds rows t1 and t1 + 8 of those 16 and,
    // of each 8-column group k, columns 8k + 2*t0 and 8k + 2*t0 + 1 (the .16x256b
    // layout); its packed fp16 P pair of those columns lands in P column 4k + t0
    // (.16x128b), which is where the P.V MMA reads keys 8k + 2*t0, +1 of the row.
    const int t = (warp - kWarpSm0) >> 3;
    const int hseg = ((warp - kWarpSm0) >> 2) & 1;
    const int q4 = warp & 3;
    const int t0 = lane & 3, t1 = lane >> 2;
    const int rbase = q4 * 32 + hseg * 16;
    const int ra = rbase + t1, rb = ra + 8;
    const uint32_t lane_addr = static_cast<uint32_t>(rbase) << 16;
    const uint32_t s_col = tmem + lane_addr + 256 + 64 * t;
    const uint32_t p_col0 = tmem + lane_addr + 384 + 64 * t;
    const uint32_t o_col = tmem + lane_addr + 128 * t;
    const float sc = a.scale_log2;
    const float2 sc2 = make_float2(sc, sc);
    uint32_t un = 0, kc = 0;
    while (true) {
      const int slot = un & 1;
      if (!warp_wait(&bars->info_full[slot], (un >> 1) & 1)) {
        if (lane == 0) set_abort(bars, a.status);
        break;
      }
      const UnitInfo U = bars->info[slot];
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->info_empty[slot]);
      ++un;
      if (U.u < 0) break;
      if (t >= ntiles) continue;
      const int n = U.cnt > 0 ? U.cnt : 1;
      const int32_t* klist =
          a.kept + (static_cast<int64_t>(U.b * a.Hkv + U.g) * a.nqb + U.i) * a.max_kept;
      const int tqa = U.i * kBlock + (ra & 63), tqb = U.i * kBlock + (rb & 63);
      float ma = -INFINITY, mb = -INFINITY;
      float2 la = make_float2(0.f, 0.f), lb = make_float2(0.f, 0.f);
      // block ids and mask modes of 32 steps at a time, one step per lane (fetched and
      // validated in parallel, off the per-step path), then read by shuffle
      int blk_v = U.i, mode_v = 2;
      bool ok = true;
      for (int jj = 0; jj < n; ++jj, ++kc) {
        if ((jj & 31) == 0) {
          const int js = jj + lane;
          blk_v = js < U.cnt ? klist[js] : U.i;
          mode_v = js < U.cnt ? mode_of(a, U, blk_v) : 2;
        }
        const int blk = __shfl_sync(0xffffffffu, blk_v, jj & 31);
        const int mode = __shfl_sync(0xffffffffu, mode_v, jj & 31);
        const int buf = kc & 1;
        // original positions of this thread's 16 keys (columns 8k + 2 t0, +1) of a block
        // of the own segment; positions past T do not exist
        int2 kp[8];
        if (mode == 3) {
          const int32_t* kpos = a.key_pos + (static_cast<int64_t>(U.b) * a.Hkv + U.g) * a.T;
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            const int p = blk * kBlock + k * 8 + 2 * t0;
            kp[k].x = p < a.T ? kpos[p] : 0x7fffffff;
            kp[k].y = p + 1 < a.T ? kpos[p + 1] : 0x7fffffff;
          }
        }
        if (!warp_wait(&bars->s_full[t], kc & 1)) { ok = false; break; }
        tc::fence_after_sync();
        uint32_t sr[32];
        tc::ld16x256_x8(s_col, sr);
        tc::wait_ld();
        // S is in registers: the score MMAs of the next step may overwrite it
        tc::fence_before_sync();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->s_free[t]);
        // masks: the causal diagonal block, blocks that failed validation, and the keys
        // of the own segment that come after the query
        if (mode == 3) {
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            if (kp[k].x > tqa) sr[4 * k] = 0xff800000u;
            if (kp[k].y > tqa) sr[4 * k + 1] = 0xff800000u;
            if (kp[k].x > tqb) sr[4 * k + 2] = 0xff800000u;
            if (kp[k].y > tqb) sr[4 * k + 3] = 0xff800000u;
          }
        } else if (mode != 0) {
          const int dblk = mode == 2 ? 0 : blk;
          const int lima = mode == 2 ? -1 : tqa - dblk * kBlock;
          const int limb = mode == 2 ? -1 : tqb - dblk * kBlock;
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            const int c = k * 8 + 2 * t0;   // column within the block
            if (c > lima) sr[4 * k] = 0xff800000u;
            if (c + 1 > lima) sr[4 * k + 1] = 0xff800000u;
            if (c > limb) sr[4 * k + 2] = 0xff800000u;
            if (c + 1 > limb) sr[4 * k + 3] = 0xff800000u;
          }
        }
        // row maxima (each row spans the 4 threads with the same t1): two chains per row
        float xa = -INFINITY, xa2 = -INFINITY, xb = -INFINITY, xb2 = -INFINITY;
#pragma unroll
        for (int k = 0; k < 8; k += 2) {
          xa = max3(xa, __uint_as_float(sr[4 * k]), __uint_as_float(sr[4 * k + 1]));
          xa2 = max3(xa2, __uint_as_float(sr[4 * k + 4]), __uint_as_float(sr[4 * k + 5]));
          xb = max3(xb, __uint_as_float(sr[4 * k + 2]), __uint_as_float(sr[4 * k + 3]));
          xb2 = max3(xb2, __uint_as_float(sr[4 * k + 6]), __uint_as_float(sr[4 * k + 7]));
        }
        xa = fmaxf(xa, xa2);
        xb = fmaxf(xb, xb2);
        xa = fmaxf(xa, __shfl_xor_sync(0xffffffffu, xa, 1));
        xb = fmaxf(xb, __shfl_xor_sync(0xffffffffu, xb, 1));
        xa = fmaxf(xa, __shfl_xor_sync(0xffffffffu, xa, 2));
        xb = fmaxf(xb, __shfl_xor_sync(0xffffffffu, xb, 2));
        xa *= sc;
        xb *= sc;
        const bool upa = xa > ma + 8.0f, upb = xb > mb + 8.0f;
        // move the running max of the rows that need it (O is rescaled below, after P)
        const bool any_up = __any_sync(0xffffffffu, upa || upb);
        const float fa = upa ? ex2(ma - xa) : 1.0f;
        const float fb = upb ? ex2(mb - xb) : 1.0f;
        if (upa) {
          la.x *= fa;
          la.y *= fa;
          ma = xa;
        }
        if (upb) {
          lb.x *= fb;
          lb.y *= fb;
          mb = xb;
        }
        const float na = ma == -INFINITY ? 0.f : -ma, nbb = mb == -INFINITY ? 0.f : -mb;
        const float2 na2 = make_float2(na, na), nb2 = make_float2(nbb, nbb);
        // P = 2^(s * scale - m) in fp16, packed in place (word 2k: row a, 2k+1: row b)
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const float2 va = __ffma2_rn(make_float2(__uint_as_float(sr[4 * k]), __uint_as_float(sr[4 * k + 1])), sc2, na2);
          const float2 vb = __ffma2_rn(make_float2(__uint_as_float(sr[4 * k + 2]), __uint_as_float(sr[4 * k + 3])), sc2, nb2);
          float2 pa, pb;
          if (k >= 8 - kPolyGroups) {
            pa = exp2_poly(va);
            pb = exp2_poly(vb);
          } else {
            pa = make_float2(ex2(va.x), ex2(va.y));
            pb = make_float2(ex2(vb.x), ex2(vb.y));
          }
          la = __fadd2_rn(la, pa);
          lb = __fadd2_rn(lb, pb);
          sr[2 * k] = pack_f16(pa.x, pa.y);
          sr[2 * k + 1] = pack_f16(pb.x, pb.y);
        }
        // P buffer kc % 2 was last read by the P.V of step kc - 2
        if (kc >= 2) {
          const uint32_t jp = kc - 2;
          if (!warp_wait(&bars->pv_done[t][jp & 1], (jp >> 1) & 1)) { ok = false; break; }
          tc::fence_after_sync();
        }
        tc::st16x128_x8(p_col0 + 32 * buf, *reinterpret_cast<const uint32_t(*)[16]>(&sr[0]));
        if (any_up && jj > 0) {
          // rescale the O rows accumulated so far (warp-wide: tcgen05.ld/st are
          // collective), once the P.V of the previous step has completed
          const uint32_t jp = kc - 1;
          if (!warp_wait(&bars->pv_done[t][jp & 1], (jp >> 1) & 1)) { ok = false; break; }
          tc::fence_after_sync();
#pragma unroll 1
          for (int half = 0; half < D / 64; ++half) {
            uint32_t ov[32];
            tc::ld16x256_x8(o_col + 64 * half, ov);
            tc::wait_ld();
#pragma unroll
            for (int k = 0; k < 8; ++k) {
              ov[4 * k] = __float_as_uint(__uint_as_float(ov[4 * k]) * fa);
              ov[4 * k + 1] = __float_as_uint(__uint_as_float(ov[4 * k + 1]) * fa);
              ov[4 * k + 2] = __float_as_uint(__uint_as_float(ov[4 * k + 2]) * fb);
              ov[4 * k + 3] = __float_as_uint(__uint_as_float(ov[4 * k + 3]) * fb);
            }
            tc::st16x256_x8(o_col + 64 * half, ov);
          }
        }
        tc::wait_st();
        tc::fence_before_sync();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->p_ready[t][buf]);
      }
      if (!ok || aborted(bars)) {
        if (lane == 0) set_abort(bars, a.status);
        break;
      }
      // ---- epilogue: O / l, once the unit's last P.V has completed
      const uint32_t jl = kc - 1;
      if (!warp_wait(&bars->pv_done[t][jl & 1], (jl >> 1) & 1)) {
        if (lane == 0) set_abort(bars, a.status);
        break;
      }
      tc::fence_after_sync();
      float La = la.x + la.y, Lb = lb.x + lb.y;
      La += __shfl_xor_sync(0xffffffffu, La, 1);
      La += __shfl_xor_sync(0xffffffffu, La, 2);
      Lb += __shfl_xor_sync(0xffffffffu, Lb, 1);
      Lb += __shfl_xor_sync(0xffffffffu, Lb, 2);
      const float inva = La > 0.f ? 1.0f / La : 0.f, invb = Lb > 0.f ? 1.0f / Lb : 0.f;
      const bool wa = tqa < a.T && (4 * U.hq + 2 * t + (ra >> 6)) < a.G;
      const bool wb = tqb < a.T && (4 * U.hq + 2 * t + (rb >> 6)) < a.G;
      const int64_t hra =
          (static_cast<int64_t>(U.b) * a.Hq + U.g * a.G + row_head(a, U.hq, t, ra)) * a.T + tqa;
      const int64_t hrb =
          (static_cast<int64_t>(U.b) * a.Hq + U.g * a.G + row_head(a, U.hq, t, rb)) * a.T + tqb;
#pragma unroll 1
      for (int half = 0; half < D / 64; ++half) {
        uint32_t ov[32];
        tc::ld16x256_x8(o_col + 64 * half, ov);
        tc::wait_ld();
#pragma unroll
        for (int rr = 0; rr < 2; ++rr) {
          if (rr ? wb : wa) {
            const int64_t hrow = rr ? hrb : hra;
            const float inv = rr ? invb : inva;
            __nv_bfloat16* ob = static_cast<__nv_bfloat16*>(a.o) + hrow * D + 64 * half;
#pragma unroll
            for (int k = 0; k < 8; ++k) {
              const float v0 = __uint_as_float(ov[4 * k + 2 * rr]) * inv;
              const float v1 = __uint_as_float(ov[4 * k + 2 * rr + 1]) * inv;
              *reinterpret_cast<__nv_bfloat162*>(ob + 8 * k + 2 * t0) = __floats2bfloat162_rn(v0, v1);
              if (a.o_f32)
                *reinterpret_cast<float2*>(a.o_f32 + hrow * D + 64 * half + 8 * k + 2 * t0) =
                    make_float2(v0, v1);
            }
          }
        }
      }
      if (t0 == 0) {
        if (wa) a.lse[hra] = La > 0.f ? (ma + log2f(La)) * 0.69314718055994530942f : -INFINITY;
        if (wb) a.lse[hrb] = Lb > 0.f ? (mb + log2f(Lb)) * 0.69314718055994530942f : -INFINITY;
      }
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->o_free[t]);   // O of this tile may be overwritten now
    }
  }

  tc::fence_before_sync();
  __syncthreads();
  if (warp == kWarpS0) {
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
    constexpr int smem = smem_bytes<128>();
    e = cudaFuncSetAttribute(prefill_tc_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             smem);
    if (e != cudaSuccess) return e;
    prefill_tc_kernel<128><<<grid, kThreads, smem, s>>>(a, tq, tk, tv16, unit_counter, num_units);
  } else {
    constexpr int smem = smem_bytes<64>();
    e = cudaFuncSetAttribute(prefill_tc_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             smem);
    if (e != cudaSuccess) return e;
    prefill_tc_kernel<64><<<grid, kThreads, smem, s>>>(a, tq, tk, tv16, unit_counter, num_units);
  }
  return cudaGetLastError();
}

}  // namespace bsa
