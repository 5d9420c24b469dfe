// Block-sparse causal prefill attention, warp-level tensor-core version.
//
// For each query token tq of block i and head h of group g: exact softmax over
// the tokens tk <= tq of the kept key blocks of row (b, g, i) (HGA, Central
// mechanism §4: exact token-level attention over the routed set; the diagonal
// block is always kept and is causally masked).
//
// Design:
//  * V is first converted to fp16 into the workspace (one pass, zero padded to a
//    multiple of 64 tokens), so P.V runs with fp16 P (11 mantissa bits), which
//    keeps the output error well inside the tolerance, while Q.K^T stays bf16;
//  * unit = (b, g, i, head pair): 2 heads x 64 query tokens = 128 rows, 8
//    consumer warps of 16 rows, 1 producer warp. The producer loads the unit's Q
//    tile once and streams the kept blocks' K (bf16) and V (fp16) tiles through
//    a TMA ring (128-byte swizzle); consumers run QK^T and PV on mma.m16n8k16
//    with the online softmax in registers (P feeds the next MMA directly);
//  * the diagonal block applies tk <= tq; rows tq >= T are not written.
#include "bsa_common.cuh"
#include "bsa_internal.h"

namespace bsa {
namespace {

constexpr int kCWarps = 8;
constexpr int kPThreads = (kCWarps + 1) * 32;

template <int D>
struct PCfg {
  static constexpr int kBoxes = D / 64;
  static constexpr int kTileBytes = kBlock * D * 2;
  static constexpr int kStageBytes = 2 * kTileBytes;
  static constexpr int kQBytes = 2 * kBlock * D * 2;  // two heads
  static constexpr int kStages = D == 128 ? 4 : 6;
  static constexpr int kKsteps = D / 16;
  static constexpr int kSmem = kQBytes + kStages * kStageBytes + (2 * kStages + 2) * 8 +
                               kStages * 4 + 1024;
};

BSA_DEVFN int64_t prow(const CacheView& c, int b, int g, int blk, int rows, int d) {
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

template <int D>
__global__ void __launch_bounds__(kPThreads, 1)
    prefill_attn_kernel(const PrefillArgs a, const __grid_constant__ CUtensorMap tmq,
                        const __grid_constant__ CUtensorMap tmk,
                        const __grid_constant__ CUtensorMap tmv) {
  using Cfg = PCfg<D>;
  constexpr int S = Cfg::kStages;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  unsigned char* qs = smem;
  unsigned char* ring = smem + Cfg::kQBytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(ring + S * Cfg::kStageBytes);
  uint64_t* empty = full + S;
  uint64_t* qfull = empty + S;
  int* sinfo = reinterpret_cast<int*>(qfull + 2);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int npair = (a.G + 1) / 2;
  const int BHP = a.B * a.Hkv * npair;
  const int i = a.nqb - 1 - static_cast<int>(blockIdx.x) / BHP;  // heavy rows first
  const int rem = static_cast<int>(blockIdx.x) % BHP;
  const int bg = rem / npair, hp = rem % npair;
  const int b = bg / a.Hkv, g = bg % a.Hkv;
  const int64_t krow = static_cast<int64_t>(bg) * a.nqb + i;
  const int cnt = min(a.kept_count[krow], a.max_kept);
  const int32_t* klist = a.kept + krow * a.max_kept;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kCWarps);
    }
    mbar_init(qfull, 1);
    fence_mbar_init();
  }
  __syncthreads();

  if (warp == kCWarps) {
    if (lane == 0) {
      prefetch_tensormap(&tmq);
      prefetch_tensormap(&tmk);
      prefetch_tensormap(&tmv);
      // Q: two heads x 64 rows x D
      mbar_arrive_expect_tx(qfull, Cfg::kQBytes);
      for (int hh = 0; hh < 2; ++hh) {
        const int h = g * a.G + min(2 * hp + hh, a.G - 1);
        const int32_t qr = static_cast<int32_t>((static_cast<int64_t>(b) * a.Hq + h) * a.T + i * kBlock);
        for (int x = 0; x < Cfg::kBoxes; ++x)
          tma_load_2d(qs + hh * (kBlock * D * 2) + x * 8192, &tmq, x * 64, qr, qfull);
      }
      for (int e = 0; e < cnt; ++e) {
        const int s = e % S;
        if (!mbar_wait(&empty[s], ((e / S) & 1) ^ 1)) {
          report(a.status, BSA_DEV_TIMEOUT);
          break;
        }
        const int blk = klist[e];
        int64_t rk = -1;
        if (blk >= 0 && blk <= i) {
          rk = prow(a.k, b, g, blk, min(kBlock, a.T - blk * kBlock), D);
          if (rk < 0) report(a.status, BSA_DEV_BAD_PAGE);
        } else {
          report(a.status, BSA_DEV_BAD_KEPT);
        }
        sinfo[s] = rk >= 0 ? blk : -1;
        unsigned char* st = ring + s * Cfg::kStageBytes;
        if (rk >= 0) {
          const int32_t rv = static_cast<int32_t>(static_cast<int64_t>(bg) * a.Tpad + blk * kBlock);
          mbar_arrive_expect_tx(&full[s], Cfg::kStageBytes);
          for (int x = 0; x < Cfg::kBoxes; ++x) {
            tma_load_2d(st + x * 8192, &tmk, x * 64, static_cast<int32_t>(rk), &full[s]);
            tma_load_2d(st + Cfg::kTileBytes + x * 8192, &tmv, x * 64, rv, &full[s]);
          }
        } else {
          mbar_arrive(&full[s]);
        }
      }
      const int it = cnt;
      for (int k = 0; k < S && k < it; ++k) {
        const int j = it - 1 - k;
        mbar_wait(&empty[j % S], (j / S) & 1, 200000000ull);
      }
      mbar_wait(qfull, 0, 200000000ull);
    }
    return;
  }

  // ------------------------------------------------------------------ consumers
  const int gid = lane >> 2, tig = lane & 3;
  const int rr = lane & 7, mi = lane >> 3;
  const int hh = warp >> 2;                 // head within the pair
  const int hl = 2 * hp + hh;               // head within the group
  const bool head_ok = hl < a.G;
  const int r0 = 16 * (warp & 3);           // first query row of this warp in the block
  const int tq0 = i * kBlock + r0 + gid, tq1 = tq0 + 8;
  bool alive = mbar_wait(qfull, 0);
  if (!alive && lane == 0) report(a.status, BSA_DEV_TIMEOUT);

  // Q A-fragments for all k-steps
  uint32_t aq[Cfg::kKsteps][4];
  {
    const uint32_t qb = smem_u32(qs + hh * (kBlock * D * 2));
#pragma unroll
    for (int ks = 0; ks < Cfg::kKsteps; ++ks) {
      const int row = r0 + rr + 8 * (mi & 1);
      const int chunk = 2 * ks + (mi >> 1);
      ldsm_x4(aq[ks], qb + (chunk >> 3) * 8192 + swz128(row, chunk & 7));
    }
  }
  float acc[D / 8][4];
#pragma unroll
  for (int n = 0; n < D / 8; ++n) acc[n][0] = acc[n][1] = acc[n][2] = acc[n][3] = 0.f;
  float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;

  for (int e = 0; e < cnt && alive; ++e) {
    const int s = e % S;
    if (!mbar_wait(&full[s], (e / S) & 1)) {
      if (lane == 0) report(a.status, BSA_DEV_TIMEOUT);
      alive = false;
      break;
    }
    const int blk = sinfo[s];
    if (blk >= 0) {
      const uint32_t kb = smem_u32(ring + s * Cfg::kStageBytes);
      const uint32_t vb = kb + Cfg::kTileBytes;
      // S = Q K^T : 16 rows x 64 keys (8 n-tiles)
      float sc[8][4];
#pragma unroll
      for (int n = 0; n < 8; ++n) sc[n][0] = sc[n][1] = sc[n][2] = sc[n][3] = 0.f;
#pragma unroll
      for (int ks = 0; ks < Cfg::kKsteps; ++ks) {
#pragma unroll
        for (int np = 0; np < 4; ++np) {
          // matrices: (tok 0-7, dims lo), (tok 0-7, dims hi), (tok 8-15, lo), (tok 8-15, hi)
          const int trow = 16 * np + rr + 8 * (mi >> 1);
          const int chunk = 2 * ks + (mi & 1);
          uint32_t bk[4];
          ldsm_x4(bk, kb + (chunk >> 3) * 8192 + swz128(trow, chunk & 7));
          mma_bf16(sc[2 * np], aq[ks], bk[0], bk[1]);
          mma_bf16(sc[2 * np + 1], aq[ks], bk[2], bk[3]);
        }
      }
      const bool diag = blk == i;
      float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
      for (int n = 0; n < 8; ++n) {
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          const int tk = blk * kBlock + 8 * n + 2 * tig + c;
          float s0 = sc[n][c] * a.scale_log2, s1 = sc[n][2 + c] * a.scale_log2;
          if (diag) {
            if (tk > tq0) s0 = -INFINITY;
            if (tk > tq1) s1 = -INFINITY;
          }
          sc[n][c] = s0;
          sc[n][2 + c] = s1;
          mx0 = fmaxf(mx0, s0);
          mx1 = fmaxf(mx1, s1);
        }
      }
      mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
      mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
      mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
      mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
      const float mn0 = fmaxf(m0, mx0), mn1 = fmaxf(m1, mx1);
      const float b0 = mn0 == -INFINITY ? 0.f : mn0, b1 = mn1 == -INFINITY ? 0.f : mn1;
      const float c0 = ex2(m0 - b0), c1 = ex2(m1 - b1);
      m0 = mn0;
      m1 = mn1;
      l0 *= c0;
      l1 *= c1;
#pragma unroll
      for (int n = 0; n < D / 8; ++n) {
        acc[n][0] *= c0;
        acc[n][1] *= c0;
        acc[n][2] *= c1;
        acc[n][3] *= c1;
      }
      uint32_t pa[4][4];  // P as A-fragments, 4 k-steps of 16 keys
#pragma unroll
      for (int n = 0; n < 8; ++n) {
        const float p0 = ex2(sc[n][0] - b0), p1 = ex2(sc[n][1] - b0);
        const float p2 = ex2(sc[n][2] - b1), p3 = ex2(sc[n][3] - b1);
        l0 += p0 + p1;
        l1 += p2 + p3;
        const int kk = n >> 1, hi = n & 1;
        pa[kk][0 + 2 * hi] = pack_f16(p0, p1);
        pa[kk][1 + 2 * hi] = pack_f16(p2, p3);
      }
      // O += P V : V^T fragments via ldmatrix.trans (fp16 tile)
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
#pragma unroll
        for (int dp = 0; dp < D / 16; ++dp) {
          // matrices: (tok 0-7, dims 16dp..+7), (tok 8-15, same), (tok 0-7, +8..), (tok 8-15, +8..)
          const int trow = 16 * kk + rr + 8 * (mi & 1);
          const int chunk = 2 * dp + (mi >> 1);
          uint32_t bv[4];
          ldsm_x4_t(bv, vb + (chunk >> 3) * 8192 + swz128(trow, chunk & 7));
          mma_f16(acc[2 * dp], pa[kk], bv[0], bv[1]);
          mma_f16(acc[2 * dp + 1], pa[kk], bv[2], bv[3]);
        }
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[s]);
  }

  // ---- epilogue: normalise and store rows that exist
  l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
  l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
  if (!head_ok || !alive) return;
  const int h = g * a.G + hl;
  const float inv0 = l0 > 0.f ? 1.0f / l0 : 0.f, inv1 = l1 > 0.f ? 1.0f / l1 : 0.f;
  __nv_bfloat16* ob = static_cast<__nv_bfloat16*>(a.o);
  const int64_t hb = (static_cast<int64_t>(b) * a.Hq + h) * a.T;
#pragma unroll
  for (int rsel = 0; rsel < 2; ++rsel) {
    const int tq = rsel ? tq1 : tq0;
    if (tq >= a.T) continue;
    const float inv = rsel ? inv1 : inv0;
    const int64_t ro = (hb + tq) * D;
#pragma unroll
    for (int n = 0; n < D / 8; ++n) {
      const int dim = 8 * n + 2 * tig;
      const float v0 = acc[n][2 * rsel] * inv, v1 = acc[n][2 * rsel + 1] * inv;
      *reinterpret_cast<__nv_bfloat162*>(ob + ro + dim) = __floats2bfloat162_rn(v0, v1);
      if (a.o_f32) *reinterpret_cast<float2*>(a.o_f32 + ro + dim) = make_float2(v0, v1);
    }
    if (tig == 0) {
      const float mm = rsel ? m1 : m0, ll = rsel ? l1 : l0;
      a.lse[hb + tq] = ll > 0.f ? (mm + log2f(ll)) * 0.69314718055994530942f : -INFINITY;
    }
  }
}

// V (bf16, cache layout) -> fp16 [B*Hkv, Tpad, D], zero for t >= T.
__global__ void v_to_f16_kernel(const PrefillArgs a) {
  const int64_t nvec = static_cast<int64_t>(a.B) * a.Hkv * a.Tpad * (a.d / 8);
  const char* vbase = static_cast<const char*>(a.v.base);
  uint4* out = static_cast<uint4*>(const_cast<void*>(a.v16));
  bool bad = false;
  for (int64_t x = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; x < nvec;
       x += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t vecs_per_row = a.d / 8;
    const int64_t rowi = x / vecs_per_row;
    const int c8 = static_cast<int>(x % vecs_per_row);
    const int t = static_cast<int>(rowi % a.Tpad);
    const int bg = static_cast<int>(rowi / a.Tpad);
    const int b = bg / a.Hkv, g = bg % a.Hkv;
    uint4 res = make_uint4(0u, 0u, 0u, 0u);
    if (t < a.T) {
      const int blk = t / kBlock;
      int64_t phys = blk;
      bool ok = true;
      if (a.v.page_table != nullptr) {
        phys = a.v.page_table[static_cast<int64_t>(b) * a.v.pt_stride + blk];
        ok = phys >= 0 && phys < a.v.num_pages;
      }
      const int64_t off = static_cast<int64_t>(b) * a.v.seq_stride + phys * a.v.block_stride +
                          static_cast<int64_t>(g) * a.v.head_stride +
                          static_cast<int64_t>(t % kBlock) * a.d + c8 * 8;
      ok = ok && off >= 0 && off + 8 <= a.v.extent;
      if (ok) {
        const uint4 raw = *reinterpret_cast<const uint4*>(vbase + off * 2);
        const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
        uint32_t o4[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const float2 f = unpack_bf16(w[q]);
          if (fabsf(f.x) > 65504.f || fabsf(f.y) > 65504.f) bad = true;
          o4[q] = pack_f16(f.x, f.y);
        }
        res = make_uint4(o4[0], o4[1], o4[2], o4[3]);
      } else {
        bad = true;
      }
    }
    out[x] = res;
  }
  if (bad) report(a.status, BSA_DEV_FP16_RANGE);
}

}  // namespace

cudaError_t launch_v_to_f16(const PrefillArgs& a, cudaStream_t s) {
  const int64_t nvec = static_cast<int64_t>(a.B) * a.Hkv * a.Tpad * (a.d / 8);
  if (nvec <= 0) return cudaSuccess;
  int64_t blocks = (nvec + 255) / 256;
  if (blocks > 148 * 16) blocks = 148 * 16;
  v_to_f16_kernel<<<static_cast<unsigned>(blocks), 256, 0, s>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_prefill(const PrefillArgs& a, const CUtensorMap& tq, const CUtensorMap& tk,
                           const CUtensorMap& tv16, int num_sms, cudaStream_t s) {
  (void)num_sms;
  const int npair = (a.G + 1) / 2;
  const int64_t units = static_cast<int64_t>(a.B) * a.Hkv * a.nqb * npair;
  if (units <= 0) return cudaSuccess;
  cudaError_t e;
  if (a.d == 128) {
    e = cudaFuncSetAttribute(prefill_attn_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             PCfg<128>::kSmem);
    if (e != cudaSuccess) return e;
    prefill_attn_kernel<128><<<static_cast<unsigned>(units), kPThreads, PCfg<128>::kSmem, s>>>(
        a, tq, tk, tv16);
  } else {
    e = cudaFuncSetAttribute(prefill_attn_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             PCfg<64>::kSmem);
    if (e != cudaSuccess) return e;
    prefill_attn_kernel<64><<<static_cast<unsigned>(units), kPThreads, PCfg<64>::kSmem, s>>>(
        a, tq, tk, tv16);
  }
  return cudaGetLastError();
}

}  // namespace bsa
