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
    __nv_bfloat16* __restrict__ dst, int64_t ldd, uint32_t cols, uint32_t cpr, uint32_t total,
    int read_early) {
  griddep_launch_dependents();
  if (!read_early) griddep_wait();  // the previous launch may write the source
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

// Contiguous sources (row pitch == cols): each CTA copies a contiguous
// range of rows.  Batches of whole rows are brought into shared memory by
// 1-D bulk copies (double-buffered: batch i + 1 in flight while batch i is
// realigned); warp w realigns rows w, w + 8, ... of the batch, lane l the
// 16-byte chunks l, l + 32, ... of a row, with one shift per row (no
// division, no divergence).  Bulk copies start and end on 16-byte granules
// that hold bytes of the source, so they stay inside its pages.  Waits are
// bounded; on a timeout the kernel records it and stops.
constexpr int kBulkThreads = 256;
constexpr uint32_t kBulkBuf = 48 * 1024;

__global__ void __launch_bounds__(kBulkThreads) repack_rows_bulk_kernel(
    const __nv_bfloat16* __restrict__ src, uintptr_t src_end, __nv_bfloat16* __restrict__ dst,
    int64_t ldd, int rows, int cols, int rows_per_cta, int batch_rows, int read_early,
    WaitCtl wait) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ uint64_t bars[2];
  uint8_t* buf = smem_raw;  // 2 × kBulkBuf, 16-byte aligned
  griddep_launch_dependents();
  const int r_begin = blockIdx.x * rows_per_cta;
  const int r_end = min(rows, r_begin + rows_per_cta);
  if (r_begin >= r_end) {
    griddep_wait();  // complete only after the previous launch (stream order)
    return;
  }
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int cpr = (cols + 7) / 8;
  const uintptr_t base = reinterpret_cast<uintptr_t>(src);
  const uintptr_t end16 = (src_end + 15) & ~static_cast<uintptr_t>(15);
  if (threadIdx.x == 0) {
    mbar_init(&bars[0], 1u);
    mbar_init(&bars[1], 1u);
    fence_mbar_init();
  }
  __syncthreads();
  // Source span of rows [r0, r1): [a0, a0 + bytes).
  auto span = [&](int r0, int r1, uint32_t* bytes) {
    const uintptr_t p0 = base + 2 * static_cast<uint64_t>(r0) * cols;
    const uintptr_t p1 = base + 2 * static_cast<uint64_t>(r1) * cols;
    const uintptr_t a0 = p0 & ~static_cast<uintptr_t>(15);
    const uintptr_t a1 = min((p1 + 15) & ~static_cast<uintptr_t>(15), end16);
    *bytes = static_cast<uint32_t>(a1 - a0);
    return a0;
  };
  auto issue = [&](int b) {
    const int r0 = r_begin + b * batch_rows, r1 = min(r_end, r0 + batch_rows);
    uint32_t bytes;
    const uintptr_t a0 = span(r0, r1, &bytes);
    mbar_arrive_expect_tx(&bars[b & 1], bytes);
    for (uint32_t off = 0; off < bytes; off += 16384)
      bulk_load(buf + (b & 1) * kBulkBuf + off, a0 + off, min(16384u, bytes - off), &bars[b & 1]);
  };
  const int nb = (r_end - r_begin + batch_rows - 1) / batch_rows;
  // Unless the host knows the previous launch does not write the source,
  // read it only after that launch has finished.
  if (!read_early) griddep_wait();
  if (threadIdx.x == 0) issue(0);
  uint32_t phase[2] = {0u, 0u};
  bool ok = true;
  for (int b = 0; b < nb && ok; ++b) {
    if (threadIdx.x == 0 && b + 1 < nb) issue(b + 1);
    // Every thread takes the same branch (a block-wide vote), so no thread
    // is left at a barrier the others skip.
    if (!__syncthreads_and(mbar_wait(&bars[b & 1], phase[b & 1], wait, 8u) ? 1 : 0)) {
      ok = false;
      break;
    }
    phase[b & 1] ^= 1u;
    const int r0 = r_begin + b * batch_rows, r1 = min(r_end, r0 + batch_rows);
    uint32_t bytes;
    const uintptr_t a0 = span(r0, r1, &bytes);
    const uint8_t* bb = buf + (b & 1) * kBulkBuf;
    for (int r = r0 + warp; r < r1; r += kBulkThreads / 32) {
      const uint32_t o_row = static_cast<uint32_t>(base + 2 * static_cast<uint64_t>(r) * cols - a0);
      const uint32_t sh = o_row & 15u;
      __nv_bfloat16* drow = dst + static_cast<int64_t>(r) * ldd;
      for (int c = lane; c < cpr; c += 32) {
        const uint32_t g = (o_row & ~15u) + 16u * c;
        const uint4 lo = *reinterpret_cast<const uint4*>(bb + g);
        const uint4 hi = (sh != 0u && g + 16 < bytes) ? *reinterpret_cast<const uint4*>(bb + g + 16)
                                                       : make_uint4(0u, 0u, 0u, 0u);
        uint4 v = window16(lo, hi, sh);
        const int valid = cols - 8 * c;
        if (valid < 8) v = mask_tail8(v, valid);
        *reinterpret_cast<uint4*>(drow + 8 * c) = v;
      }
    }
    // All reads of this buffer are done before it is refilled.
    fence_proxy_async_smem();
    __syncthreads();
  }
  if (!ok && threadIdx.x == 0) {
    // Let copies still in flight land before the CTA leaves.
    for (int i = 0; i < 2; ++i) {
      const unsigned long long t0 = global_ns();
      while (!mbar_try_wait(&bars[i], phase[i]) && global_ns() - t0 < 1000000ull) {
      }
    }
  }
  // Complete only after the previous launch on the stream, so that a launch
  // that waits for this one also waits for that one.
  griddep_wait();
}

}  // namespace

cudaError_t launch_repack(const __nv_bfloat16* src, int64_t lds, size_t src_bytes,
                          __nv_bfloat16* dst, int64_t ldd, int64_t rows, int64_t cols,
                          int num_sms, cudaStream_t stream, bool dependent, WaitCtl wait,
                          bool read_early) {
  if (rows <= 0 || cols <= 0) return cudaSuccess;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  const uintptr_t hi = reinterpret_cast<uintptr_t>(src) + src_bytes;
  if (lds == cols && cols * 2 + 64 <= static_cast<int64_t>(kBulkBuf) && rows < (int64_t(1) << 31)) {
    // Two CTAs per SM, contiguous row ranges, batches that fill a buffer.
    const int64_t ctas = std::min<int64_t>(rows, static_cast<int64_t>(num_sms) * 2);
    const int rows_per_cta = static_cast<int>((rows + ctas - 1) / ctas);
    const int batch_rows = static_cast<int>(std::max<int64_t>(1, (kBulkBuf - 32) / (cols * 2)));
    const int grid = static_cast<int>((rows + rows_per_cta - 1) / rows_per_cta);
    const size_t smem = 2 * kBulkBuf;
    cudaError_t e = ensure_max_smem(reinterpret_cast<const void*>(repack_rows_bulk_kernel),
                                    static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(kBulkThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cfg.attrs = attr;
    cfg.numAttrs = dependent ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, repack_rows_bulk_kernel, src, hi, dst, ldd,
                              static_cast<int>(rows), static_cast<int>(cols), rows_per_cta,
                              batch_rows, (dependent && read_early) ? 1 : 0, wait);
  }
  const int64_t cpr = (cols + 7) / 8;
  const int64_t total = rows * cpr;
  if (total > 0xFFFFFFFFll - static_cast<int64_t>(num_sms) * 8 * kRepackThreads * kRepackU)
    return cudaErrorInvalidValue;
  const int64_t per_cta = static_cast<int64_t>(kRepackThreads) * kRepackU;
  const int blocks = static_cast<int>(
      std::max<int64_t>(1, std::min<int64_t>((total + per_cta - 1) / per_cta,
                                             static_cast<int64_t>(num_sms) * 8)));
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(blocks);
  cfg.blockDim = dim3(kRepackThreads);
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = dependent ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, repack_chunks_kernel, src, lds, hi, dst, ldd,
                            static_cast<uint32_t>(cols), static_cast<uint32_t>(cpr),
                            static_cast<uint32_t>(total), (dependent && read_early) ? 1 : 0);
}

}  // namespace lr
