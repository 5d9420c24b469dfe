// Segment permutation of the keys for block-sparse prefill (PBS-Attn, "Sparser
// Block-Sparse Attention via Token Permutation", Methodology §2-§3).
//
// Per (sequence b, kv head g):
//  1. importance of key t = mean over the query rows of the last query block (the
//     group's heads x the block's positions) of the causal softmax probability of t.
//     Pass 1 streams the keys in chunks and keeps, per row, a running max and sum of
//     2^(s - max) (s = q.k * scale in log2 units) with the 16-dim dot products on
//     mma.m16n8k16 (keys as M, query rows as N, as in the decode kernel); a combine
//     kernel turns the chunks' (max, sum) into each row's log-sum-exp. Pass 2
//     recomputes the scores and adds 2^(s - lse) over the rows for every key, in a
//     fixed order (warp, then head), so the importance is deterministic;
//  2. a bitonic sort of each segment's (importance descending, position ascending)
//     keys in shared memory gives key_pos;
//  3. a gather writes the permuted K, V and index keys.
#include "bsa_common.cuh"
#include "bsa_internal.h"

namespace bsa {
namespace {

constexpr int kPW = 4;                 // warps per CTA of the importance passes
constexpr int kChunk = 1024;           // keys per CTA
constexpr int kSortThreads = 1024;

// Row (in rows of width d) of the first token of block `blk` of (b, g); -1 if invalid.
BSA_DEVFN int64_t pbs_block_row(const CacheView& c, int b, int g, int blk, int rows, int d) {
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

// PASS 1: per (row, chunk) running (max, sum) in log2 units. PASS 2: importance sums.
template <int D, int PASS>
__global__ void __launch_bounds__(kPW * 32) pbs_rows_kernel(const PbsArgs a) {
  constexpr int kSlabs = D / 64;
  constexpr int kKsteps = D / 16;
  __shared__ __align__(1024) unsigned char ktile[kSlabs * 8192];
  __shared__ float colsum[kPW][64];
  __shared__ float acc[kChunk];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int gid = lane >> 2, tig = lane & 3, rr = lane & 7, mi = lane >> 3;
  const int bg = blockIdx.y, b = bg / a.Hkv, g = bg % a.Hkv;
  const int chunk = blockIdx.x;
  const int k0 = chunk * kChunk;
  const int ntiles = min(kChunk, a.T - k0 + kBlock - 1) / kBlock;   // blocks of this chunk
  const int qpos0 = (a.nqb - 1) * kBlock;                           // last query block
  const int nq = a.T - qpos0;
  const char* kbase = static_cast<const char*>(a.k.base);

  if (PASS == 2)
    for (int x = threadIdx.x; x < kChunk; x += kPW * 32) acc[x] = 0.f;

  for (int h = 0; h < a.G; ++h) {
    const int64_t qrow0 = (static_cast<int64_t>(b) * a.Hq + g * a.G + h) * a.T + qpos0;
    // query fragments (B operand): rows 16 * warp + 8 nt + gid of this head
    uint32_t bq[2][kKsteps][2];
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
      const int r = 16 * warp + 8 * nt + gid;
      const uint32_t* qr = reinterpret_cast<const uint32_t*>(
          static_cast<const char*>(a.q) + (qrow0 + (r < nq ? r : 0)) * D * 2);
#pragma unroll
      for (int ks = 0; ks < kKsteps; ++ks) {
        bq[nt][ks][0] = r < nq ? qr[(ks * 16 + 2 * tig) / 2] : 0u;
        bq[nt][ks][1] = r < nq ? qr[(ks * 16 + 8 + 2 * tig) / 2] : 0u;
      }
    }
    // this thread's 4 query rows: (nt, c) -> 16 * warp + 8 nt + 2 tig + c
    float m[2][2], l[2][2], lse[2][2];
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        m[nt][c] = -INFINITY;
        l[nt][c] = 0.f;
        const int r = 16 * warp + 8 * nt + 2 * tig + c;
        lse[nt][c] = PASS == 2 && r < nq ? a.lse2[static_cast<int64_t>(bg) * a.G * kBlock + h * kBlock + r]
                                         : -INFINITY;
      }
    for (int t = 0; t < ntiles; ++t) {
      const int blk = k0 / kBlock + t;
      const int rows = min(kBlock, a.T - blk * kBlock);
      const int64_t kr = pbs_block_row(a.k, b, g, blk, rows, D);
      if (kr < 0 && threadIdx.x == 0) report(a.status, BSA_DEV_BAD_PAGE);
      __syncthreads();   // the previous tile's fragments are read
      for (int x = threadIdx.x; x < kBlock * D / 8; x += kPW * 32) {
        const int row = x / (D / 8), ch = x % (D / 8);
        uint4 v = make_uint4(0u, 0u, 0u, 0u);
        if (kr >= 0 && row < rows)
          v = *reinterpret_cast<const uint4*>(kbase + ((kr + row) * D + ch * 8) * 2);
        *reinterpret_cast<uint4*>(ktile + (ch >> 3) * 8192 + swz128(row, ch & 7)) = v;
      }
      __syncthreads();
      // S^T = K Q^T: keys 16 mt + gid (+8), query rows 8 nt + 2 tig (+1)
      float sc[4][2][4];
#pragma unroll
      for (int mt = 0; mt < 4; ++mt)
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) sc[mt][nt][0] = sc[mt][nt][1] = sc[mt][nt][2] = sc[mt][nt][3] = 0.f;
      const uint32_t kb = smem_u32(ktile);
#pragma unroll
      for (int ks = 0; ks < kKsteps; ++ks) {
        const int chunk8 = 2 * ks + (mi >> 1);
#pragma unroll
        for (int mt = 0; mt < 4; ++mt) {
          uint32_t af[4];
          ldsm_x4(af, kb + (chunk8 >> 3) * 8192 + swz128(16 * mt + rr + 8 * (mi & 1), chunk8 & 7));
#pragma unroll
          for (int nt = 0; nt < 2; ++nt) mma_bf16(sc[mt][nt], af, bq[nt][ks][0], bq[nt][ks][1]);
        }
      }
      // visibility: key exists (block valid, t < T) and is causal for the row
      const int key0 = blk * kBlock;
      if (PASS == 1) {
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
          for (int c = 0; c < 2; ++c) {
            const int r = 16 * warp + 8 * nt + 2 * tig + c;
            float x[8];
            float mx = -INFINITY;
#pragma unroll
            for (int mt = 0; mt < 4; ++mt)
#pragma unroll
              for (int hi = 0; hi < 2; ++hi) {
                const int kk = 16 * mt + gid + 8 * hi;
                const bool vis = kr >= 0 && kk < rows && key0 + kk <= qpos0 + r && r < nq;
                x[2 * mt + hi] = vis ? sc[mt][nt][2 * hi + c] * a.scale_log2 : -INFINITY;
                mx = fmaxf(mx, x[2 * mt + hi]);
              }
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
            const float mnew = fmaxf(m[nt][c], mx);
            const float base = mnew == -INFINITY ? 0.f : mnew;
            float sum = 0.f;
#pragma unroll
            for (int q = 0; q < 8; ++q) sum += exp2f(x[q] - base);
            sum += __shfl_xor_sync(0xffffffffu, sum, 4);
            sum += __shfl_xor_sync(0xffffffffu, sum, 8);
            sum += __shfl_xor_sync(0xffffffffu, sum, 16);
            l[nt][c] = l[nt][c] * exp2f(m[nt][c] - base) + sum;
            m[nt][c] = mnew;
          }
      } else {
        // probabilities summed over this warp's 16 rows, per key
        float ks_[8];
#pragma unroll
        for (int q = 0; q < 8; ++q) ks_[q] = 0.f;
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
          for (int c = 0; c < 2; ++c) {
            const int r = 16 * warp + 8 * nt + 2 * tig + c;
#pragma unroll
            for (int mt = 0; mt < 4; ++mt)
#pragma unroll
              for (int hi = 0; hi < 2; ++hi) {
                const int kk = 16 * mt + gid + 8 * hi;
                const bool vis = kr >= 0 && kk < rows && key0 + kk <= qpos0 + r && r < nq;
                ks_[2 * mt + hi] += vis ? exp2f(sc[mt][nt][2 * hi + c] * a.scale_log2 - lse[nt][c]) : 0.f;
              }
          }
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          ks_[q] += __shfl_xor_sync(0xffffffffu, ks_[q], 1);
          ks_[q] += __shfl_xor_sync(0xffffffffu, ks_[q], 2);
        }
        if (tig == 0) {
#pragma unroll
          for (int mt = 0; mt < 4; ++mt)
#pragma unroll
            for (int hi = 0; hi < 2; ++hi) colsum[warp][16 * mt + gid + 8 * hi] = ks_[2 * mt + hi];
        }
        __syncthreads();
        if (threadIdx.x < kBlock) {
          float s = 0.f;
#pragma unroll
          for (int w = 0; w < kPW; ++w) s += colsum[w][threadIdx.x];
          acc[t * kBlock + threadIdx.x] += s;
        }
      }
    }
    if (PASS == 1 && gid == 0) {
#pragma unroll
      for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          const int r = 16 * warp + 8 * nt + 2 * tig + c;
          const int64_t idx = ((static_cast<int64_t>(bg) * a.G * kBlock + h * kBlock + r) *
                               a.nchunk + chunk) * 2;
          a.ml[idx] = m[nt][c];
          a.ml[idx + 1] = l[nt][c];
        }
    }
  }
  if (PASS == 2) {
    __syncthreads();
    const float inv = 1.0f / static_cast<float>(a.G * nq);
    for (int x = threadIdx.x; x < ntiles * kBlock; x += kPW * 32)
      if (k0 + x < a.T) a.imp[static_cast<int64_t>(bg) * a.T + k0 + x] = acc[x] * inv;
  }
}

// Log-sum-exp (log2 units) of each row from its chunks' (max, sum), in chunk order.
__global__ void pbs_combine_kernel(const PbsArgs a) {
  const int64_t row = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int64_t nrows = static_cast<int64_t>(a.B) * a.Hkv * a.G * kBlock;
  if (row >= nrows) return;
  const float* ml = a.ml + row * a.nchunk * 2;
  float M = -INFINITY;
  for (int c = 0; c < a.nchunk; ++c) M = fmaxf(M, ml[2 * c]);
  float L = 0.f;
  if (M > -INFINITY)
    for (int c = 0; c < a.nchunk; ++c) L += ml[2 * c + 1] * exp2f(ml[2 * c] - M);
  a.lse2[row] = L > 0.f ? M + log2f(L) : INFINITY;   // +inf: an empty row adds nothing
}

// Sort of one segment: keys (importance descending, position ascending).
__global__ void __launch_bounds__(kSortThreads) pbs_sort_kernel(const PbsArgs a, int sort_n) {
  extern __shared__ unsigned long long sk[];
  const int bg = blockIdx.y;
  const int s0 = blockIdx.x * a.segment;
  const int n = min(a.segment, a.T - s0);
  const float* imp = a.imp + static_cast<int64_t>(bg) * a.T + s0;
  for (int x = threadIdx.x; x < sort_n; x += kSortThreads) {
    unsigned long long key = ~0ull;
    if (x < n) {
      // importance >= 0: its bits order like the value; complemented for descending
      const uint32_t bits = __float_as_uint(fmaxf(imp[x], 0.f));
      key = (static_cast<unsigned long long>(~bits) << 32) | static_cast<uint32_t>(x);
    }
    sk[x] = key;
  }
  __syncthreads();
  for (int kk = 2; kk <= sort_n; kk <<= 1) {
    for (int j = kk >> 1; j > 0; j >>= 1) {
      for (int x = threadIdx.x; x < sort_n; x += kSortThreads) {
        const int y = x ^ j;
        if (y > x) {
          const unsigned long long u = sk[x], v = sk[y];
          const bool asc = (x & kk) == 0;
          if ((u > v) == asc) {
            sk[x] = v;
            sk[y] = u;
          }
        }
      }
      __syncthreads();
    }
  }
  int32_t* out = a.key_pos + static_cast<int64_t>(bg) * a.T + s0;
  for (int x = threadIdx.x; x < n; x += kSortThreads)
    out[x] = s0 + static_cast<int32_t>(sk[x] & 0xffffffffu);
}

// Row p of the permuted K, V (width d) and index keys (width 16) = row key_pos[p].
__global__ void pbs_gather_kernel(const PbsArgs a) {
  const int vk = a.d / 8, vi = kR / 8;   // 16-byte vectors per K/V row, per index-key row
  const int per = 2 * vk + vi;
  const int64_t total = static_cast<int64_t>(a.B) * a.Hkv * a.T * per;
  for (int64_t x = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; x < total;
       x += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t rowp = x / per;                   // (bg, p)
    const int part = static_cast<int>(x % per);
    const int bg = static_cast<int>(rowp / a.T), p = static_cast<int>(rowp % a.T);
    const int b = bg / a.Hkv, g = bg % a.Hkv;
    const int t = a.key_pos[rowp];
    const int blk = t / kBlock, rows = min(kBlock, a.T - blk * kBlock);
    const CacheView& c = part < vk ? a.k : (part < 2 * vk ? a.v : a.kidx);
    const int w = part < 2 * vk ? a.d : kR;
    const int v = part < vk ? part : (part < 2 * vk ? part - vk : part - 2 * vk);
    const int64_t r0 = (t >= 0 && t < a.T) ? pbs_block_row(c, b, g, blk, rows, w) : -1;
    uint4 val = make_uint4(0u, 0u, 0u, 0u);
    if (r0 >= 0)
      val = *reinterpret_cast<const uint4*>(static_cast<const char*>(c.base) +
                                            ((r0 + t % kBlock) * w + v * 8) * 2);
    else if (v == 0)
      report(a.status, BSA_DEV_BAD_PAGE);
    char* dst = static_cast<char*>(part < vk ? a.k_perm : (part < 2 * vk ? a.v_perm : a.kidx_perm));
    *reinterpret_cast<uint4*>(dst + (rowp * w + v * 8) * 2) = val;
  }
}

template <int D>
cudaError_t launch_d(const PbsArgs& a, int num_sms, cudaStream_t s) {
  const dim3 grid(a.nchunk, a.B * a.Hkv);
  pbs_rows_kernel<D, 1><<<grid, kPW * 32, 0, s>>>(a);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const int64_t nrows = static_cast<int64_t>(a.B) * a.Hkv * a.G * kBlock;
  pbs_combine_kernel<<<static_cast<unsigned>((nrows + 255) / 256), 256, 0, s>>>(a);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  pbs_rows_kernel<D, 2><<<grid, kPW * 32, 0, s>>>(a);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  int sort_n = 1;
  while (sort_n < a.segment) sort_n <<= 1;
  const int smem = sort_n * 8;
  if ((e = cudaFuncSetAttribute(pbs_sort_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                smem)) != cudaSuccess)
    return e;
  const dim3 sgrid((a.T + a.segment - 1) / a.segment, a.B * a.Hkv);
  pbs_sort_kernel<<<sgrid, kSortThreads, smem, s>>>(a, sort_n);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  pbs_gather_kernel<<<num_sms * 8, 256, 0, s>>>(a);
  return cudaGetLastError();
}

}  // namespace

int pbs_chunks(int T) { return (T + kChunk - 1) / kChunk; }

cudaError_t launch_pbs_permute(const PbsArgs& a, int num_sms, cudaStream_t s) {
  if (a.B * a.Hkv <= 0 || a.T <= 0) return cudaSuccess;
  return a.d == 128 ? launch_d<128>(a, num_sms, s) : launch_d<64>(a, num_sms, s);
}

}  // namespace bsa
