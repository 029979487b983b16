// lr_repack.cu — copy a bf16 row-major matrix whose rows start at arbitrary
// 2-byte-aligned addresses (e.g. A [K, r] with odd r) into a workspace whose
// row pitch is a multiple of 8 elements (16 bytes), so that the tensor
// memory accelerator (TMA) can tile it.
//
// TMA requires 16-byte-aligned row strides; a factor with r mod 8 != 0 has
// none.  The GAC paper (§3.2, Table 3) shows what libraries do instead:
// fall back to 2- or 1-element loads.  Here the misaligned matrix is read
// once, at full width, with 16-byte loads and written once, aligned; the
// GEMM then runs its normal TMA path.  Cost: one extra read of the matrix
// from HBM and one write that stays in L2 until the GEMM has read it.
#include <algorithm>

#include "lr_internal.h"
#include "lr_load.cuh"

namespace lr {

namespace {

constexpr int kRepackThreads = 256;
constexpr int kRepackU = 4;  // destination chunks in flight per thread

// One thread per 16-byte destination chunk (row k, elements 8j .. 8j+7):
// the chunk's source bytes span at most two aligned 16-byte granules of the
// source, both of which hold an element of the matrix (the first holds the
// chunk's first element; the second is read only if it starts before the end
// of the source buffer), so no load leaves the buffer's pages.  Elements
// past the row's end are written as zero.
__global__ void __launch_bounds__(kRepackThreads) repack_chunks_kernel(
    const __nv_bfloat16* __restrict__ src, int64_t lds, uintptr_t hi,
    __nv_bfloat16* __restrict__ dst, int64_t ldd, uint32_t cols, uint32_t cpr, uint32_t total) {
  griddep_launch_dependents();
  const uint32_t stride = gridDim.x * kRepackThreads;
  for (uint32_t q0 = blockIdx.x * kRepackThreads + threadIdx.x; q0 < total;
       q0 += kRepackU * stride) {
    uint4 lo[kRepackU], hi2[kRepackU];
    uint32_t shift[kRepackU];
#pragma unroll
    for (int u = 0; u < kRepackU; ++u) {
      const uint32_t q = q0 + u * stride;
      if (q < total) {
        const uint32_t k = q / cpr, j = q - k * cpr;
        const uintptr_t p = reinterpret_cast<uintptr_t>(src + static_cast<int64_t>(k) * lds + 8 * j);
        const uintptr_t a = p & ~static_cast<uintptr_t>(15);
        shift[u] = static_cast<uint32_t>(p & 15u);
        lo[u] = ld_nc_v4(a);
        hi2[u] = (shift[u] != 0u && a + 16 < hi) ? ld_nc_v4(a + 16) : make_uint4(0, 0, 0, 0);
      }
    }
#pragma unroll
    for (int u = 0; u < kRepackU; ++u) {
      const uint32_t q = q0 + u * stride;
      if (q < total) {
        const uint32_t k = q / cpr, j = q - k * cpr;
        uint4 v = window16(lo[u], hi2[u], shift[u]);
        const int valid = static_cast<int>(cols) - static_cast<int>(8 * j);
        if (valid < 8) v = mask_tail8(v, valid);
        *reinterpret_cast<uint4*>(dst + static_cast<int64_t>(k) * ldd + 8 * j) = v;
      }
    }
  }
  // A later repack of the same call may start early (programmatic dependent
  // launch); finishing only after this one's predecessor keeps completion in
  // stream order.
  griddep_wait();
}

}  // namespace

cudaError_t launch_repack(const __nv_bfloat16* src, int64_t lds, size_t src_bytes,
                          __nv_bfloat16* dst, int64_t ldd, int64_t rows, int64_t cols,
                          int num_sms, cudaStream_t stream, bool dependent) {
  if (rows <= 0 || cols <= 0) return cudaSuccess;
  const int64_t cpr = (cols + 7) / 8;
  const int64_t total = rows * cpr;
  if (total > 0xFFFFFFFFll - static_cast<int64_t>(num_sms) * 8 * kRepackThreads * kRepackU)
    return cudaErrorInvalidValue;
  const uintptr_t hi = reinterpret_cast<uintptr_t>(src) + src_bytes;
  const int64_t per_cta = static_cast<int64_t>(kRepackThreads) * kRepackU;
  const int blocks = static_cast<int>(
      std::max<int64_t>(1, std::min<int64_t>((total + per_cta - 1) / per_cta,
                                             static_cast<int64_t>(num_sms) * 8)));
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(blocks);
  cfg.blockDim = dim3(kRepackThreads);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = dependent ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, repack_chunks_kernel, src, lds, hi, dst, ldd,
                            static_cast<uint32_t>(cols), static_cast<uint32_t>(cpr),
                            static_cast<uint32_t>(total));
}

}  // namespace lr
