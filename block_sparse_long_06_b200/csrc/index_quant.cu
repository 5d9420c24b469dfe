// Quantiser of the 4-bit index-key cache (SpotAttention, Methodology §4: the
// selector's K cache may be stored as microscaled INT4 or FP4).
//
// Format (include/bsa.h): per token 16 sign-magnitude 4-bit codes and one E4M3
// scale; per cache one fp32 scale g; per (sequence, kv head, 64-token block) one
// 576-byte record (64 x 8 code bytes, then 64 scale bytes).
//
// Every rounding decision is a float32 operation with round-to-nearest-even,
// written with the _rn intrinsics so that compiler flags cannot change it:
//   g = A / (qmax * 448);  s = (a / qmax) / g;  t = e4m3(s) * g;  x = k / t.
// E4M3 and the 4-bit magnitudes are rounded with integer arithmetic on those
// float32 values (nearest, ties to even, saturating), not with conversion
// instructions, so the rule is the one stated above on every device.
//
// Three kernels: the cache maximum A (atomicMax on the float bits, all values
// being >= 0), the records, and the final write of g over the maximum.
#include "bsa_common.cuh"
#include "bsa_internal.h"

namespace bsa {
namespace {

constexpr int kThreadsQ = 256;

BSA_DEVFN int seq_len(const QuantArgs& a, int b) {
  int Tb = a.seq_lens ? a.seq_lens[b] : a.T;
  return Tb < 0 ? 0 : (Tb > a.T ? a.T : Tb);
}

// Element offset of block `blk` of (b, g) in a bf16 cache of width 16, or -1.
BSA_DEVFN int64_t src_block(const CacheView& c, int b, int g, int blk, int rows) {
  int64_t phys = blk;
  if (c.page_table != nullptr) {
    phys = c.page_table[static_cast<int64_t>(b) * c.pt_stride + blk];
    if (phys < 0 || phys >= c.num_pages) return -1;
  }
  const int64_t off = static_cast<int64_t>(b) * c.seq_stride + phys * c.block_stride +
                      static_cast<int64_t>(g) * c.head_stride;
  if (off < 0 || off + static_cast<int64_t>(rows) * kR > c.extent) return -1;
  return off;
}

// Record index of block `blk` of (b, g), or -1.
BSA_DEVFN int64_t dst_record(const CacheView& c, int b, int g, int blk) {
  int64_t phys = blk;
  if (c.page_table != nullptr) {
    phys = c.page_table[static_cast<int64_t>(b) * c.pt_stride + blk];
    if (phys < 0 || phys >= c.num_pages) return -1;
  }
  const int64_t rec = static_cast<int64_t>(b) * c.seq_stride + phys * c.block_stride +
                      static_cast<int64_t>(g) * c.head_stride;
  return (rec < 0 || rec + 1 > c.extent) ? -1 : rec;
}

BSA_DEVFN void load_token(const CacheView& c, int64_t off, int row, float (&k)[kR], uint32_t& signs) {
  const uint4* p = reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(c.base) + off +
                                                  static_cast<int64_t>(row) * kR);
  const uint4 v0 = p[0], v1 = p[1];
  const uint32_t w[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
  signs = 0;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    k[2 * i] = __uint_as_float(w[i] << 16);
    k[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    signs |= ((w[i] >> 15) & 1u) << (2 * i);
    signs |= (w[i] >> 31) << (2 * i + 1);
  }
}

// E4M3 code of the value nearest to s >= 0 (ties to the even mantissa), 0x7E = 448
// for s >= 448 (saturating).
BSA_DEVFN uint32_t e4m3_code(float s) {
  if (!(s < 448.0f)) return 0x7Eu;
  if (s < 0.015625f) {                         // below 2^-6: steps of 2^-9
    return static_cast<uint32_t>(__float2int_rn(__fmul_rn(s, 512.0f)));   // 0..8; 8 = 2^-6
  }
  const uint32_t bits = __float_as_uint(s);
  int e = static_cast<int>(bits >> 23) - 127;  // -6 .. 8
  uint32_t m = (bits >> 20) & 7u;
  const uint32_t rem = bits & 0xfffffu;
  if (rem > 0x80000u || (rem == 0x80000u && (m & 1u))) ++m;
  if (m == 8u) {
    m = 0u;
    ++e;
  }
  const uint32_t code = (static_cast<uint32_t>(e + 7) << 3) | m;
  return code > 0x7Eu ? 0x7Eu : code;
}

// Magnitude index of |x| on the FP4 (E2M1) or INT4 grid: nearest, ties to even.
BSA_DEVFN uint32_t magnitude_index(float ax, int fmt) {
  if (fmt == 1) {
    return (ax > 0.25f) + (ax >= 0.75f) + (ax > 1.25f) + (ax >= 1.75f) + (ax > 2.5f) +
           (ax >= 3.5f) + (ax > 5.0f);
  }
  const int q = __float2int_rn(ax);
  return static_cast<uint32_t>(q > 7 ? 7 : q);
}

BSA_DEVFN float gscale_from_max(float amax, int fmt) {
  return amax > 0.f ? __fdiv_rn(amax, fmt == 1 ? 2688.0f : 3136.0f) : 1.0f;   // qmax * 448
}

// One thread per visible token: the cache maximum of |k|.
__global__ void __launch_bounds__(kThreadsQ) amax_kernel(const QuantArgs a) {
  const int64_t rows_total = static_cast<int64_t>(a.B) * a.Hkv * a.nb * kBlock;
  float mx = 0.f;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < rows_total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int t = static_cast<int>(i % (static_cast<int64_t>(a.nb) * kBlock));
    const int64_t bg = i / (static_cast<int64_t>(a.nb) * kBlock);
    const int b = static_cast<int>(bg / a.Hkv), g = static_cast<int>(bg % a.Hkv);
    if (t >= seq_len(a, b)) continue;
    const int blk = t / kBlock;
    const int64_t off = src_block(a.src, b, g, blk, min(kBlock, seq_len(a, b) - blk * kBlock));
    if (off < 0) {
      report(a.status, BSA_DEV_BAD_PAGE);
      continue;
    }
    float k[kR];
    uint32_t sg;
    load_token(a.src, off, t % kBlock, k, sg);
#pragma unroll
    for (int c = 0; c < kR; ++c) mx = fmaxf(mx, fabsf(k[c]));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  if ((threadIdx.x & 31) == 0 && mx > 0.f)
    atomicMax(reinterpret_cast<unsigned int*>(a.gscale), __float_as_uint(mx));
}

// One thread per token slot of every record of a visible block.
__global__ void __launch_bounds__(kThreadsQ) quantize_kernel(const QuantArgs a) {
  const int64_t rows_total = static_cast<int64_t>(a.B) * a.Hkv * a.nb * kBlock;
  const float gs = gscale_from_max(*a.gscale, a.fmt);
  const float qmax = a.fmt == 1 ? 6.0f : 7.0f;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < rows_total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int t = static_cast<int>(i % (static_cast<int64_t>(a.nb) * kBlock));
    const int64_t bg = i / (static_cast<int64_t>(a.nb) * kBlock);
    const int b = static_cast<int>(bg / a.Hkv), h = static_cast<int>(bg % a.Hkv);
    const int Tb = seq_len(a, b);
    const int blk = t / kBlock, row = t % kBlock;
    if (blk * kBlock >= Tb) continue;           // block not visible: no record written
    const int64_t rec = dst_record(a.dst, b, h, blk);
    if (rec < 0) {
      report(a.status, BSA_DEV_BAD_PAGE);
      continue;
    }
    unsigned char* r = static_cast<unsigned char*>(const_cast<void*>(a.dst.base)) + rec * kQRecord;
    uint2 packed = make_uint2(0u, 0u);
    uint32_t scode = 0u;
    if (t < Tb) {
      const int64_t off = src_block(a.src, b, h, blk, min(kBlock, Tb - blk * kBlock));
      if (off < 0) {
        report(a.status, BSA_DEV_BAD_PAGE);
      } else {
        float k[kR];
        uint32_t signs;
        load_token(a.src, off, row, k, signs);
        float amax = 0.f;
#pragma unroll
        for (int c = 0; c < kR; ++c) amax = fmaxf(amax, fabsf(k[c]));
        scode = e4m3_code(__fdiv_rn(__fdiv_rn(amax, qmax), gs));
        const float S = e4m3_value(scode);
        uint32_t codes[2] = {0u, 0u};
        if (S > 0.f) {
          const float tq = __fmul_rn(S, gs);
#pragma unroll
          for (int c = 0; c < kR; ++c) {
            const uint32_t m = magnitude_index(fabsf(__fdiv_rn(k[c], tq)), a.fmt);
            codes[c >> 3] |= m << (4 * (c & 7));
          }
        }
#pragma unroll
        for (int c = 0; c < kR; ++c) codes[c >> 3] |= ((signs >> c) & 1u) << (4 * (c & 7) + 3);
        packed = make_uint2(codes[0], codes[1]);
      }
    }
    *reinterpret_cast<uint2*>(r + row * 8) = packed;
    r[kBlock * 8 + row] = static_cast<unsigned char>(scode);
  }
}

__global__ void finalize_kernel(const QuantArgs a) {
  *a.gscale = gscale_from_max(*a.gscale, a.fmt);
}

}  // namespace

cudaError_t launch_quantize_index(const QuantArgs& a, int num_sms, cudaStream_t s) {
  cudaError_t e = cudaMemsetAsync(a.gscale, 0, sizeof(float), s);
  if (e != cudaSuccess) return e;
  const int64_t rows = static_cast<int64_t>(a.B) * a.Hkv * a.nb * kBlock;
  if (rows > 0) {
    int64_t grid = (rows + kThreadsQ - 1) / kThreadsQ;
    const int64_t cap = static_cast<int64_t>(num_sms) * 8;
    if (grid > cap) grid = cap;
    amax_kernel<<<static_cast<unsigned>(grid), kThreadsQ, 0, s>>>(a);
    quantize_kernel<<<static_cast<unsigned>(grid), kThreadsQ, 0, s>>>(a);
  }
  finalize_kernel<<<1, 1, 0, s>>>(a);
  return cudaGetLastError();
}

}  // namespace bsa
