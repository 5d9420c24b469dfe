// V conversion for the prefill attention kernel (prefill_tc.cu).
//
// P.V runs on the tensor cores with fp16 P (11 mantissa bits keep the output
// error well inside the tolerance) and an MMA takes both operands in one type,
// so V is converted once from the bf16 cache into an fp16 copy in the workspace,
// laid out [B*Hkv, Tpad, d] (Tpad = T rounded up to 64, zero padded). Values
// outside the fp16 range are reported (BSA_DEV_FP16_RANGE); rows of a page id
// outside the pool or past the cache extent are left zero and reported
// (BSA_DEV_BAD_PAGE), as the attention kernel masks their keys.
#include "bsa_common.cuh"
#include "bsa_internal.h"

namespace bsa {
namespace {

// V (bf16, cache layout) -> fp16 [B*Hkv, Tpad, D], zero for t >= T.
__global__ void v_to_f16_kernel(const PrefillArgs a) {
  const int64_t nvec = static_cast<int64_t>(a.B) * a.Hkv * a.Tpad * (a.d / 8);
  const char* vbase = static_cast<const char*>(a.v.base);
  uint4* out = static_cast<uint4*>(const_cast<void*>(a.v16));
  bool range_bad = false, page_bad = false;
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
          if (fabsf(f.x) > 65504.f || fabsf(f.y) > 65504.f) range_bad = true;
          o4[q] = pack_f16(f.x, f.y);
        }
        res = make_uint4(o4[0], o4[1], o4[2], o4[3]);
      } else {
        page_bad = true;
      }
    }
    out[x] = res;
  }
  if (range_bad) report(a.status, BSA_DEV_FP16_RANGE);
  if (page_bad) report(a.status, BSA_DEV_BAD_PAGE);
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

}  // namespace bsa
