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
//  * kept key blocks are processed in pairs: a pair is a 128-key tile, so every
//    MMA has N = 128 (a lone last block uses N = 64);
//  * warp 0 (one lane) loads Q once per unit and the K tiles (bf16) of each pair
//    into a K ring, and publishes each pair's block ids and mask modes in a small
//    shared-memory ring; warp 2 (one lane) loads the V tiles (fp16) into a V ring.
//    All loads are TMA with 128-byte swizzle;
//  * warp 1 (one lane) issues the MMAs. S_t = Q_t K^T (bf16, M = 128, K = d) goes to
//    tensor memory; O_t += P_t V (fp16, P read from tensor memory, N = d). Per pair
//    k the order is S_0(k), P_1(k-1).V, S_1(k), P_0(k).V, so each tile's softmax
//    runs while the tensor core works for the other tile. S_t(k) overwrites P_t(k-1)
//    and therefore waits for the P.V of tile t on pair k-1;
//  * warps 4-7 and 8-11 are the softmax warpgroups of tile 0 and tile 1 (a thread
//    per row = tensor-memory lane). A thread loads its S row once (128 fp32), masks
//    the causal diagonal block, takes the row max with three-input max, computes P
//    with packed two-wide fp32 arithmetic and writes it as fp16 over the S columns
//    it has consumed. 3/8 of the exponentials run as a cubic polynomial on the FMA
//    pipes (exp2_poly below) instead of the MUFU unit, the co-bottleneck of
//    attention at d = 128. The running max only moves (and O is rescaled in tensor
//    memory) when it grows by more than 8 (log2), so P <= 256 fits fp16 and the
//    rescale is rare; the final normalisation uses the same max, so it is exact;
//  * epilogue: O / l from tensor memory straight to global memory (bf16, and fp32
//    when requested), LSE in natural log.
// Tensor memory: 512 columns: S/P of tile 0 at 0, of tile 1 at 128; O of tile 0 at
// 256, of tile 1 at 384. Every wait is bounded; on a timeout the kernel sets
// BSA_DEV_TIMEOUT, drains, frees its tensor memory and returns.
#include "bsa_common.cuh"
#include "bsa_internal.h"
#include "tcgen05.cuh"

namespace bsa {
namespace {

constexpr int kThreads = 384;
constexpr int kWarpLoadK = 0, kWarpMma = 1, kWarpLoadV = 2, kWarpSm0 = 4;
constexpr uint32_t kTmemCols = 512;
constexpr int kPI = 8;          // depth of the pair-info ring
constexpr int kPolyPairs = 6;   // per 16 packed pairs of a 32-column chunk: computed by polynomial

template <int D>
struct Cfg {
  static constexpr int kHalves = D / 64;          // 64-dim slabs of 128 rows x 128 B
  static constexpr int kSlab = 128 * 128;
  static constexpr int kTile = kHalves * kSlab;   // 128 rows x D
  static constexpr int kSK = D == 128 ? 3 : 4;    // K stages
  static constexpr int kSV = D == 128 ? 2 : 4;    // V stages
  static constexpr int kKsteps = D / 16;
  static constexpr int kOffK = 2 * kTile;
  static constexpr int kOffV = kOffK + kSK * kTile;
  static constexpr int kOffBar = kOffV + kSV * kTile;
};

struct UnitInfo {
  int u, b, g, i, hq, cnt;
};

struct Bars {
  uint64_t info_full[2], info_empty[2];
  uint64_t q_full, q_empty;
  uint64_t k_full[4], k_empty[4], v_full[4], v_empty[4];
  uint64_t pi_full[kPI], pi_empty[kPI];
  uint64_t s_full[2], p_ready[2], o_done[2], o_free[2];
  uint64_t mma_done;
  UnitInfo info[2];
  int4 pinfo[kPI];   // blk0, blk1, nb, mode0 | mode1 << 8   (mode: 0 visible, 1 diagonal, 2 masked)
  uint32_t tmem_base;
  int abort_flag;
};

template <int D>
constexpr int smem_bytes() {
  return Cfg<D>::kOffBar + static_cast<int>(sizeof(Bars)) + 1024;
}

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

// Masks the 64 scores of one key block held in two 32-column chunks: columns past
// `lim` (the last visible key offset; -1 hides the whole block) become -inf.
BSA_DEVFN void mask_block(uint32_t (&c0)[32], uint32_t (&c1)[32], int lim) {
  const uint32_t ninf = 0xff800000u;
#pragma unroll
  for (int x = 0; x < 32; ++x) {
    if (x > lim) c0[x] = ninf;
    if (x + 32 > lim) c1[x] = ninf;
  }
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

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    prefill_tc_kernel(const PrefillArgs a, const __grid_constant__ CUtensorMap tmq,
                      const __grid_constant__ CUtensorMap tmk,
                      const __grid_constant__ CUtensorMap tmv, int* unit_counter,
                      const int num_units) {
  using C = Cfg<D>;
  constexpr int SK = C::kSK, SV = C::kSV;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  Bars* bars = reinterpret_cast<Bars*>(smem + C::kOffBar);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int ntiles = a.G >= 4 ? 2 : 1;

  if (threadIdx.x == 0) {
    for (int x = 0; x < 2; ++x) {
      mbar_init(&bars->info_full[x], 1);
      mbar_init(&bars->info_empty[x], 1 + 1 + 8);   // MMA lane, V loader, every softmax warp
      mbar_init(&bars->s_full[x], 1);
      mbar_init(&bars->p_ready[x], 4);
      mbar_init(&bars->o_done[x], 1);
      mbar_init(&bars->o_free[x], 4);
    }
    for (int s = 0; s < 4; ++s) {
      mbar_init(&bars->k_full[s], 1);
      mbar_init(&bars->k_empty[s], 1);
      mbar_init(&bars->v_full[s], 1);
      mbar_init(&bars->v_empty[s], 1);
    }
    for (int s = 0; s < kPI; ++s) {
      mbar_init(&bars->pi_full[s], 1);
      mbar_init(&bars->pi_empty[s], 1 + 1 + 4 * ntiles);  // MMA lane, V loader, active softmax warps
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

  if (warp == kWarpLoadK) {
    // ---------------------------------------------------------- Q / K / pair info
    if (lane == 0) {
      prefetch_tensormap(&tmq);
      prefetch_tensormap(&tmk);
      uint32_t un = 0, kc = 0;
      bool ok = true;
      while (ok) {
        int u = atomicAdd(unit_counter, 1);
        if (u >= num_units) u = -1;
        const int slot = un & 1;
        if (!mbar_wait(&bars->info_empty[slot], ((un >> 1) & 1) ^ 1)) { ok = false; break; }
        UnitInfo U = {u, 0, 0, 0, 0, 0};
        if (u >= 0) U = unit_of(a, u);
        bars->info[slot] = U;
        mbar_arrive(&bars->info_full[slot]);
        if (u < 0 || aborted(bars)) break;
        const int32_t* klist =
            a.kept + (static_cast<int64_t>(U.b * a.Hkv + U.g) * a.nqb + U.i) * a.max_kept;
        if (!mbar_wait(&bars->q_empty, (un & 1) ^ 1)) { ok = false; break; }
        mbar_arrive_expect_tx(&bars->q_full, ntiles * 2 * C::kHalves * 8192);
        for (int t = 0; t < ntiles; ++t)
          for (int hh = 0; hh < 2; ++hh) {
            const int h = U.g * a.G + row_head(a, U.hq, t, hh * 64);
            const int32_t qr = static_cast<int32_t>((static_cast<int64_t>(U.b) * a.Hq + h) * a.T +
                                                    U.i * kBlock);
            for (int x = 0; x < C::kHalves; ++x)
              tma_load_2d(smem + t * C::kTile + x * C::kSlab + hh * 8192, &tmq, x * 64, qr,
                          &bars->q_full);
          }
        const int npairs = (U.cnt + 1) / 2;
        for (int pp = 0; pp < npairs; ++pp, ++kc) {
          const int nb = (2 * pp + 1 < U.cnt) ? 2 : 1;
          int blk[2] = {-1, -1}, mode[2] = {2, 2};
          int64_t rk[2] = {0, 0};
          for (int q = 0; q < nb; ++q) {
            blk[q] = klist[2 * pp + q];
            rk[q] = krow_of(a.k, a, U.b, U.g, blk[q], U.i);
            if (rk[q] < 0) {
              report(a.status, blk[q] < 0 || blk[q] > U.i ? BSA_DEV_BAD_KEPT : BSA_DEV_BAD_PAGE);
              blk[q] = U.i;   // load the always-valid diagonal block; its columns are masked
              rk[q] = krow_of(a.k, a, U.b, U.g, blk[q], U.i);
              if (rk[q] < 0) rk[q] = 0;
              mode[q] = 2;
            } else {
              mode[q] = blk[q] == U.i ? 1 : 0;
            }
          }
          const int pi = kc % kPI;
          if (!mbar_wait(&bars->pi_empty[pi], ((kc / kPI) & 1) ^ 1)) { ok = false; break; }
          bars->pinfo[pi] = make_int4(blk[0], blk[1], nb, mode[0] | (mode[1] << 8));
          mbar_arrive(&bars->pi_full[pi]);
          const int s = kc % SK;
          if (!mbar_wait(&bars->k_empty[s], ((kc / SK) & 1) ^ 1)) { ok = false; break; }
          mbar_arrive_expect_tx(&bars->k_full[s], nb * C::kHalves * 8192);
          unsigned char* kst = smem + C::kOffK + s * C::kTile;
          for (int q = 0; q < nb; ++q)
            for (int x = 0; x < C::kHalves; ++x)
              tma_load_2d(kst + x * C::kSlab + q * 8192, &tmk, x * 64, static_cast<int32_t>(rk[q]),
                          &bars->k_full[s]);
        }
        if (!ok) break;
        ++un;
      }
      if (!ok) set_abort(bars, a.status);
      // copies in flight must land before the CTA exits (bounded)
      for (uint32_t k = (kc > SK ? kc - SK : 0); k < kc; ++k)
        mbar_wait(&bars->k_full[k % SK], (k / SK) & 1, 100000000ull);
      if (un > 0) mbar_wait(&bars->q_full, (un - 1) & 1, 100000000ull);
    }
  } else if (warp == kWarpLoadV) {
    // ------------------------------------------------------------------ V loader
    if (lane == 0) {
      prefetch_tensormap(&tmv);
      uint32_t un = 0, kc = 0;
      bool ok = true;
      while (ok) {
        const int slot = un & 1;
        if (!mbar_wait(&bars->info_full[slot], (un >> 1) & 1)) { ok = false; break; }
        const UnitInfo U = bars->info[slot];
        mbar_arrive(&bars->info_empty[slot]);
        if (U.u < 0 || aborted(bars)) break;
        const int npairs = (U.cnt + 1) / 2;
        for (int pp = 0; pp < npairs; ++pp, ++kc) {
          const int pi = kc % kPI;
          // the pair's validated block ids come from the K loader
          if (!mbar_wait(&bars->pi_full[pi], (kc / kPI) & 1)) { ok = false; break; }
          const int4 P = bars->pinfo[pi];
          mbar_arrive(&bars->pi_empty[pi]);
          const int s = kc % SV;
          if (!mbar_wait(&bars->v_empty[s], ((kc / SV) & 1) ^ 1)) { ok = false; break; }
          mbar_arrive_expect_tx(&bars->v_full[s], P.z * C::kHalves * 8192);
          unsigned char* vst = smem + C::kOffV + s * C::kTile;
          for (int q = 0; q < P.z; ++q) {
            const int blk = q == 0 ? P.x : P.y;
            const int32_t rv = static_cast<int32_t>(
                (static_cast<int64_t>(U.b) * a.Hkv + U.g) * a.Tpad + blk * kBlock);
            for (int x = 0; x < C::kHalves; ++x)
              tma_load_2d(vst + x * C::kSlab + q * 8192, &tmv, x * 64, rv, &bars->v_full[s]);
          }
        }
        if (!ok) break;
        ++un;
      }
      if (!ok) set_abort(bars, a.status);
      for (uint32_t k = (kc > SV ? kc - SV : 0); k < kc; ++k)
        mbar_wait(&bars->v_full[k % SV], (k / SV) & 1, 100000000ull);
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
        const UnitInfo U = bars->info[slot];
        mbar_arrive(&bars->info_empty[slot]);
        if (U.u < 0 || aborted(bars)) break;
        const int npairs = (U.cnt + 1) / 2;
        if (!mbar_wait(&bars->q_full, un & 1)) { ok = false; break; }
        // Issue order per pair k (two tiles): S_0(k), P_1(k-1).V, S_1(k), P_0(k).V, so the
        // softmax of one tile overlaps MMAs of the other. S_t(k) overwrites P_t(k-1): it
        // waits for the P.V of tile t on pair k-1 (o_done). The P.V of tile 1 on a unit's
        // last pair is issued when the unit ends.
        int nk_prev = 0;
        uint32_t sv_prev = 0;
        for (int pp = 0; pp < npairs && ok; ++pp, ++kc) {
          const int pi = kc % kPI;
          if (!mbar_wait(&bars->pi_full[pi], (kc / kPI) & 1)) { ok = false; break; }
          const int nk = bars->pinfo[pi].z * 64;
          mbar_arrive(&bars->pi_empty[pi]);
          const int sk = kc % SK, sv = kc % SV;
          if (!mbar_wait(&bars->k_full[sk], (kc / SK) & 1)) { ok = false; break; }
          const uint32_t kbase = sbase + C::kOffK + sk * C::kTile;
          // ---- S_0(k)
          if (kc > 0 && !mbar_wait(&bars->o_done[0], (kc - 1) & 1)) { ok = false; break; }
          tc::fence_after_sync();
#pragma unroll
          for (int ks = 0; ks < C::kKsteps; ++ks) {
            const uint32_t off = (ks >> 2) * C::kSlab + (ks & 3) * 32;
            tc::mma_ss(tmem, tc::smem_desc_sw128(sbase + off, 16, 1024),
                       tc::smem_desc_sw128(kbase + off, 16, 1024), nk == 128 ? idS128 : idS64, ks > 0);
          }
          tc::commit(&bars->s_full[0]);
          if (ntiles == 2) {
            // ---- P_1(k-1).V  (same unit)
            if (pp > 0) {
              if (pp == 1 && un > 0 && !mbar_wait(&bars->o_free[1], (un - 1) & 1)) { ok = false; break; }
              if (!mbar_wait(&bars->p_ready[1], (kc - 1) & 1)) { ok = false; break; }
              tc::fence_after_sync();
              for (int kk = 0; kk < nk_prev / 16; ++kk)
                tc::mma_ts(tmem + 384, tmem + 128 + kk * 8,
                           tc::smem_desc_sw128(sv_prev + kk * 2048, C::kSlab, 1024), idPV,
                           pp > 1 || kk > 0);
              tc::commit(&bars->o_done[1]);
              tc::commit(&bars->v_empty[(kc - 1) % SV]);
            }
            // ---- S_1(k)
            if (kc > 0 && !mbar_wait(&bars->o_done[1], (kc - 1) & 1)) { ok = false; break; }
            tc::fence_after_sync();
#pragma unroll
            for (int ks = 0; ks < C::kKsteps; ++ks) {
              const uint32_t off = (ks >> 2) * C::kSlab + (ks & 3) * 32;
              tc::mma_ss(tmem + 128, tc::smem_desc_sw128(sbase + C::kTile + off, 16, 1024),
                         tc::smem_desc_sw128(kbase + off, 16, 1024), nk == 128 ? idS128 : idS64,
                         ks > 0);
            }
            tc::commit(&bars->s_full[1]);
          }
          tc::commit(&bars->k_empty[sk]);
          if (pp == npairs - 1) tc::commit(&bars->q_empty);
          // ---- P_0(k).V
          if (!mbar_wait(&bars->v_full[sv], (kc / SV) & 1)) { ok = false; break; }
          const uint32_t vbase = sbase + C::kOffV + sv * C::kTile;
          if (pp == 0 && un > 0 && !mbar_wait(&bars->o_free[0], (un - 1) & 1)) { ok = false; break; }
          if (!mbar_wait(&bars->p_ready[0], kc & 1)) { ok = false; break; }
          tc::fence_after_sync();
          for (int kk = 0; kk < nk / 16; ++kk)
            tc::mma_ts(tmem + 256, tmem + kk * 8, tc::smem_desc_sw128(vbase + kk * 2048, C::kSlab, 1024),
                       idPV, pp > 0 || kk > 0);
          tc::commit(&bars->o_done[0]);
          if (ntiles == 1) tc::commit(&bars->v_empty[sv]);
          nk_prev = nk;
          sv_prev = vbase;
        }
        if (!ok) break;
        if (ntiles == 2) {
          // ---- P_1(last).V
          if (npairs == 1 && un > 0 && !mbar_wait(&bars->o_free[1], (un - 1) & 1)) { ok = false; break; }
          if (!mbar_wait(&bars->p_ready[1], (kc - 1) & 1)) { ok = false; break; }
          tc::fence_after_sync();
          for (int kk = 0; kk < nk_prev / 16; ++kk)
            tc::mma_ts(tmem + 384, tmem + 128 + kk * 8,
                       tc::smem_desc_sw128(sv_prev + kk * 2048, C::kSlab, 1024), idPV,
                       npairs > 1 || kk > 0);
          tc::commit(&bars->o_done[1]);
          tc::commit(&bars->v_empty[(kc - 1) % SV]);
        }
        if (!ok) break;
        ++un;
      }
      if (!ok) set_abort(bars, a.status);
      // every MMA issued so far must finish before tensor memory is freed (bounded)
      tc::commit(&bars->mma_done);
      mbar_wait(&bars->mma_done, 0, 200000000ull);
    }
  } else if (warp >= kWarpSm0) {
    // ----------------------------------------------------------- softmax warps
    const int t = (warp - kWarpSm0) >> 2;
    const int q4 = warp & 3;
    const int r = q4 * 32 + lane;
    const uint32_t lane_addr = static_cast<uint32_t>(q4 * 32) << 16;
    const uint32_t s_col = tmem + lane_addr + 128 * t;
    const uint32_t o_col = tmem + lane_addr + 256 + 128 * t;
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
      const int npairs = (U.cnt + 1) / 2;
      const int tq = U.i * kBlock + (r & 63);
      float m = -INFINITY;
      float2 l2 = make_float2(0.f, 0.f);
      bool ok = true;
      for (int pp = 0; pp < npairs; ++pp, ++kc) {
        const int pi = kc % kPI;
        if (!warp_wait(&bars->pi_full[pi], (kc / kPI) & 1)) { ok = false; break; }
        const int4 P = bars->pinfo[pi];
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->pi_empty[pi]);
        if (!warp_wait(&bars->s_full[t], kc & 1)) { ok = false; break; }
        tc::fence_after_sync();
        const int nb = P.z;
        const int mode0 = P.w & 0xff, mode1 = (P.w >> 8) & 0xff;
        // S row of this thread: chunks of 32 columns (block q = chunks 2q, 2q+1)
        uint32_t r[4][32];
        tc::ld32(s_col, r[0]);
        tc::ld32(s_col + 32, r[1]);
        if (nb == 2) {
          tc::ld32(s_col + 64, r[2]);
          tc::ld32(s_col + 96, r[3]);
        }
        tc::wait_ld();
        // masks: the causal diagonal block, and blocks that failed validation
        if (mode0 != 0) mask_block(r[0], r[1], mode0 == 2 ? -1 : tq - P.x * kBlock);
        if (nb == 2 && mode1 != 0) mask_block(r[2], r[3], mode1 == 2 ? -1 : tq - P.y * kBlock);
        float mx = -INFINITY;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          if (c < 2 * nb) {
#pragma unroll
            for (int x = 0; x < 32; x += 2)
              mx = max3(mx, __uint_as_float(r[c][x]), __uint_as_float(r[c][x + 1]));
          }
        }
        mx *= sc;
        if (mx > m + 8.0f) {
          // move the running max: rescale l and the O row accumulated so far
          const float f = ex2(m - mx);
          l2.x *= f;
          l2.y *= f;
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
        const float nbase = m == -INFINITY ? 0.f : -m;
        const float2 nb2 = make_float2(nbase, nbase);
        // P = 2^(s * scale - m) in fp16, packed in place over the consumed S values
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          if (c < 2 * nb) {
#pragma unroll
            for (int x = 0; x < 16; ++x) {
              const float2 s2 = make_float2(__uint_as_float(r[c][2 * x]), __uint_as_float(r[c][2 * x + 1]));
              const float2 xv = __ffma2_rn(s2, sc2, nb2);
              float2 p;
              if (x >= 16 - kPolyPairs) {
                p = exp2_poly(xv);
              } else {
                p.x = ex2(xv.x);
                p.y = ex2(xv.y);
              }
              l2 = __fadd2_rn(l2, p);
              r[c][x] = pack_f16(p.x, p.y);
            }
            tc::st16(s_col + 16 * c, *reinterpret_cast<const uint32_t(*)[16]>(&r[c][0]));
          }
        }
        tc::wait_st();
        tc::fence_before_sync();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->p_ready[t]);
      }
      if (!ok || aborted(bars)) {
        if (lane == 0) set_abort(bars, a.status);
        break;
      }
      // ---- epilogue: O / l
      if (!warp_wait(&bars->o_done[t], (kc - 1) & 1)) {
        if (lane == 0) set_abort(bars, a.status);
        break;
      }
      tc::fence_after_sync();
      const float l = l2.x + l2.y;
      const int hl = row_head(a, U.hq, t, r);
      const bool write = tq < a.T && (4 * U.hq + 2 * t + (r >> 6)) < a.G;
      const int64_t hrow = (static_cast<int64_t>(U.b) * a.Hq + U.g * a.G + hl) * a.T + tq;
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
          uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(a.o) + hrow * D + c * 32);
#pragma unroll
          for (int x = 0; x < 4; ++x)
            dst[x] = make_uint4(pk[4 * x], pk[4 * x + 1], pk[4 * x + 2], pk[4 * x + 3]);
          if (a.o_f32) {
            float4* df = reinterpret_cast<float4*>(a.o_f32 + hrow * D + c * 32);
#pragma unroll
            for (int x = 0; x < 8; ++x)
              df[x] = make_float4(__uint_as_float(ov[4 * x]) * inv, __uint_as_float(ov[4 * x + 1]) * inv,
                                  __uint_as_float(ov[4 * x + 2]) * inv,
                                  __uint_as_float(ov[4 * x + 3]) * inv);
          }
        }
      }
      if (write) a.lse[hrow] = l > 0.f ? (m + log2f(l)) * 0.69314718055994530942f : -INFINITY;
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
