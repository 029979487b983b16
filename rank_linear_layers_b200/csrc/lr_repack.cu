// lr_repack.cu — copy a bf16 row-major matrix whose rows start at arbitrary
// 2-byte-aligned addresses (e.g. A [K, r] with odd r) into a workspace whose
// row pitch is a multiple of 8 elements (16 bytes), so that the tensor
// memory accelerator (TMA) can tile it.
//
// TMA requires 16-byte-aligned row strides; a factor with r mod 8 != 0 has
// none.  The GAC paper (§3.2, Table 3) shows what libraries do instead:
// fall back to 2- or 1-element loads.  Here the misaligned matrix is read
// once, at full width, with 16-byte loads (realigned in registers,
// lr_load.cuh) and written once, aligned; the GEMM then runs its normal TMA
// path.  Cost: one extra read and write of the matrix, bandwidth-bound.
#include <algorithm>

#include "lr_internal.h"
#include "lr_load.cuh"

namespace lr {

namespace {

constexpr int kRepackWarps = 8;
constexpr int kRepackU = 4;  // row segments in flight per warp

// Task t = (row, 256-column segment).  Each warp takes kRepackU tasks at a
// time (grid-stride), loads them all, then realigns and stores them.
__global__ void __launch_bounds__(kRepackWarps * 32) repack_rows_kernel(
    const __nv_bfloat16* __restrict__ src, int64_t lds, uintptr_t lo, uintptr_t hi,
    __nv_bfloat16* __restrict__ dst, int64_t ldd, int64_t rows, int64_t cols) {
  const int lane = threadIdx.x & 31;
  const int64_t segs = (cols + 255) / 256;
  const int64_t tasks = rows * segs;
  const int64_t warp_global = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
  for (int64_t t0 = warp_global * kRepackU; t0 < tasks; t0 += nwarps * kRepackU) {
    uint4 cur[kRepackU], ext[kRepackU];
#pragma unroll
    for (int u = 0; u < kRepackU; ++u) {
      const int64_t t = t0 + u;
      const int64_t row = t / segs, c0 = (t % segs) * 256;
      const int nv = (t < tasks) ? static_cast<int>(std::min<int64_t>(256, cols - c0)) : 0;
      seg16_issue(src + row * lds + c0, lane, 32, nv, lo, hi, cur[u], ext[u]);
    }
#pragma unroll
    for (int u = 0; u < kRepackU; ++u) {
      const int64_t t = t0 + u;
      if (t >= tasks) break;
      const int64_t row = t / segs, c0 = (t % segs) * 256;
      const int nv = static_cast<int>(std::min<int64_t>(256, cols - c0));
      const uint4 v = seg16_finish(cur[u], ext[u], seg_shift(src + row * lds + c0), lane, 32, nv);
      const int c = 8 * lane;
      if (c < nv) {
        // dst rows are 16-byte aligned and c0 + c is a multiple of 8: the
        // chunk is aligned; elements past nv are zero, and the pitch covers
        // them (ldd >= cols rounded up to 8).
        *reinterpret_cast<uint4*>(dst + row * ldd + c0 + c) = v;
      }
    }
  }
}

}  // namespace

cudaError_t launch_repack(const __nv_bfloat16* src, int64_t lds, size_t src_bytes,
                          __nv_bfloat16* dst, int64_t ldd, int64_t rows, int64_t cols,
                          int num_sms, cudaStream_t stream) {
  if (rows <= 0 || cols <= 0) return cudaSuccess;
  const uintptr_t lo = reinterpret_cast<uintptr_t>(src);
  const int64_t tasks = rows * ((cols + 255) / 256);
  const int64_t warps_needed = (tasks + kRepackU - 1) / kRepackU;
  const int64_t blocks_needed = (warps_needed + kRepackWarps - 1) / kRepackWarps;
  const int blocks = static_cast<int>(std::max<int64_t>(1, std::min<int64_t>(blocks_needed, num_sms * 8)));
  repack_rows_kernel<<<blocks, kRepackWarps * 32, 0, stream>>>(src, lds, lo, lo + src_bytes, dst,
                                                               ldd, rows, cols);
  return cudaGetLastError();
}

}  // namespace lr
