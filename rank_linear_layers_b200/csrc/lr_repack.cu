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
constexpr int kRepackU = 8;  // row segments in flight per warp
constexpr int kRepackCtasPerSm = 2;

// The matrix is cut into 256-column segments of each row.  The grid's warps
// are split into `segs` equal groups; the warps of group j copy segment j of
// rows g, g + G, g + 2G, ... (G warps per group, g the warp's index in it),
// through a rolling pipeline of kRepackU register slots: finishing row i
// issues row i + kRepackU in its slot.  Only the start needs a division.
__global__ void __launch_bounds__(kRepackWarps * 32) repack_rows_kernel(
    const __nv_bfloat16* __restrict__ src, int64_t lds, uintptr_t lo, uintptr_t hi,
    __nv_bfloat16* __restrict__ dst, int64_t ldd, int64_t rows, int64_t cols) {
  griddep_launch_dependents();
  const int lane = threadIdx.x & 31;
  const int segs = static_cast<int>((cols + 255) / 256);
  const int w = static_cast<int>((static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5);
  const int W = static_cast<int>((static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5);
  const int G = W / segs;  // warps per segment (the launch makes it >= 1)
  if (w >= G * segs) return;
  const int seg = w % segs, g = w / segs;
  const int64_t c0 = static_cast<int64_t>(seg) * 256;
  const int nv = static_cast<int>(std::min<int64_t>(256, cols - c0));
  const int64_t mine = (rows > g) ? (rows - g + G - 1) / G : 0;  // rows of this warp
  const __nv_bfloat16* s0 = src + static_cast<int64_t>(g) * lds + c0;
  const int64_t sstep = static_cast<int64_t>(G) * lds;
  __nv_bfloat16* d0 = dst + static_cast<int64_t>(g) * ldd + c0;
  const int64_t dstep = static_cast<int64_t>(G) * ldd;

  uint4 cur[kRepackU], ext[kRepackU];
#pragma unroll
  for (int u = 0; u < kRepackU; ++u)
    seg16_issue(s0 + u * sstep, lane, 32, u < mine ? nv : 0, lo, hi, cur[u], ext[u]);
  for (int64_t i0 = 0; i0 < mine; i0 += kRepackU) {
#pragma unroll
    for (int u = 0; u < kRepackU; ++u) {
      const int64_t i = i0 + u;
      if (i >= mine) break;
      const __nv_bfloat16* sp = s0 + i * sstep;
      const uint4 v = seg16_finish(cur[u], ext[u], seg_shift(sp), lane, 32, nv);
      // Refill the slot with row i + U before storing this one.
      seg16_issue(sp + kRepackU * sstep, lane, 32, i + kRepackU < mine ? nv : 0, lo, hi, cur[u],
                  ext[u]);
      const int c = 8 * lane;
      if (c < nv) {
        // dst rows are 16-byte aligned and c0 + c is a multiple of 8: the
        // chunk is aligned; elements past nv are zero, and the pitch covers
        // them (ldd >= cols rounded up to 8).
        *reinterpret_cast<uint4*>(d0 + i * dstep + c) = v;
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
  // Enough warps that every segment gets at least one and the SMs fill.
  const int64_t segs = (cols + 255) / 256;
  const int64_t warps_wanted = std::max<int64_t>(segs, std::min<int64_t>(
      segs * rows, static_cast<int64_t>(num_sms) * kRepackCtasPerSm * kRepackWarps));
  const int blocks = static_cast<int>(std::max<int64_t>(1, (warps_wanted + kRepackWarps - 1) / kRepackWarps));
  repack_rows_kernel<<<blocks, kRepackWarps * 32, 0, stream>>>(src, lds, lo, lo + src_bytes, dst,
                                                               ldd, rows, cols);
  return cudaGetLastError();
}

}  // namespace lr
