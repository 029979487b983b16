// lr_tiny.cu — the whole layer Y = (X·A)·B (+bias) in ONE CTA, for layers
// small enough that the launch itself is the cost (M <= 16 tokens and
// factors that fit in shared memory, such as a 16×256 · 256×107 · 107×256
// layer: 1.75 MFLOP, 126 KB).
//
// The decode path streams A and B over all SMs in two launches with split-K
// reductions; at this size each of those launches is a few microseconds of
// fixed cost (launch, cross-CTA partial sums, the last-CTA hand-off) around
// nanoseconds of work.  Here one CTA copies X, A and B into shared memory
// with asynchronous 16-byte copies (the aligned 16-byte chunks that cover
// each tensor, so any base alignment and any row pitch work), computes
// T = X·A in fp32 (kept in shared memory, never rounded), then Y = T·B +
// bias, and stores Y.  A thread takes one output column for all 16 token
// rows (X and T are held transposed, so one 16-byte load feeds four FMAs)
// over one of up to four contiguous k ranges; the ranges' partial sums are
// added in order.  Every product is an fp32 FMA (packed two rows at a time)
// of the exact inputs.
#include <algorithm>

#include "lr_internal.h"

namespace lr {

namespace {

constexpr int kTinyThreads = 512;

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}

__device__ __forceinline__ void cp_async_wait_all() {
  asm volatile("cp.async.wait_all;" ::: "memory");
}

// Copy the aligned 16-byte chunks covering [p, p + bytes) to dst; returns
// the byte offset of p inside the copy.
__device__ __forceinline__ uint32_t stage_raw(uint8_t* dst, const void* p, size_t bytes) {
  const uintptr_t lo = reinterpret_cast<uintptr_t>(p) & ~static_cast<uintptr_t>(15);
  const uintptr_t hi = (reinterpret_cast<uintptr_t>(p) + bytes + 15) & ~static_cast<uintptr_t>(15);
  const uint32_t d = smem_u32(dst);
  for (uintptr_t a = lo + 16u * threadIdx.x; a < hi; a += 16u * kTinyThreads)
    cp_async16(d + static_cast<uint32_t>(a - lo), reinterpret_cast<const void*>(a));
  return static_cast<uint32_t>(reinterpret_cast<uintptr_t>(p) - lo);
}

__device__ __forceinline__ float bf(const uint8_t* base, uint32_t off, int64_t idx) {
  return __bfloat162float(
      *reinterpret_cast<const __nv_bfloat16*>(base + off + static_cast<uint32_t>(idx) * 2u));
}

// Splits of the reduction dimension so that the threads have work: a thread
// takes one output column and one of `split` contiguous k ranges.
__host__ __device__ inline int tiny_split(int cols) {
  const int s = kTinyThreads / (cols > 0 ? cols : 1);
  return s < 1 ? 1 : (s > 4 ? 4 : s);
}

// Shared memory layout (16-byte aligned parts): Xt [K][16] fp32 (X transposed,
// rows past M zero), Tt [r][16] fp32 (T transposed), partial sums
// [split][16][cols] fp32, then the raw 16-byte chunks covering A and B.
struct TinyLayout {
  size_t xt, tt, part, araw, braw, total;
};

__host__ __device__ inline TinyLayout tiny_layout(int64_t K, int64_t r, int64_t N) {
  TinyLayout L;
  L.xt = 0;
  L.tt = L.xt + tiny_align16(static_cast<size_t>(K) * 16 * 4);
  L.part = L.tt + tiny_align16(static_cast<size_t>(r) * 16 * 4);
  const size_t pt = static_cast<size_t>(tiny_split(static_cast<int>(r))) * 16 * r * 4;
  const size_t py = static_cast<size_t>(tiny_split(static_cast<int>(N))) * 16 * N * 4;
  L.araw = L.part + tiny_align16(pt > py ? pt : py);
  L.braw = L.araw + tiny_align16(static_cast<size_t>(K) * r * 2 + 32);
  L.total = L.braw + tiny_align16(static_cast<size_t>(r) * N * 2 + 32);
  return L;
}

// out[m][c] for m < 16, c < cols: sum over k < depth of vt[k][m] · W[k][c]
// (W raw bf16 at wbase + woff, row pitch ldw), k split in `split` ranges whose
// partial sums are added in range order; result to outt[c][m] (transposed)
// or handed to `store`.
template <typename Store>
__device__ __forceinline__ void tiny_product(const float* vt, const uint8_t* wbase, uint32_t woff,
                                             int64_t ldw, int depth, int cols, float* part,
                                             Store store) {
  const int split = tiny_split(cols);
  for (int task = threadIdx.x; task < cols * split; task += kTinyThreads) {
    const int c = task % cols, sp = task / cols;
    const int k0 = depth * sp / split, k1 = depth * (sp + 1) / split;
    float2 acc[8];  // rows (2i, 2i + 1), packed fp32x2 FMA
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] = make_float2(0.f, 0.f);
    for (int k = k0; k < k1; ++k) {
      const float w = bf(wbase, woff, static_cast<int64_t>(k) * ldw + c);
      const float2 w2 = make_float2(w, w);
      const float4* v = reinterpret_cast<const float4*>(vt + k * 16);
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const float4 x = v[q];
        acc[2 * q] = __ffma2_rn(make_float2(x.x, x.y), w2, acc[2 * q]);
        acc[2 * q + 1] = __ffma2_rn(make_float2(x.z, x.w), w2, acc[2 * q + 1]);
      }
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      part[(sp * 16 + 2 * i) * cols + c] = acc[i].x;
      part[(sp * 16 + 2 * i + 1) * cols + c] = acc[i].y;
    }
  }
  __syncthreads();
  for (int i = threadIdx.x; i < 16 * cols; i += kTinyThreads) {
    const int m = i / cols, c = i - m * cols;
    float v = 0.f;
    for (int sp = 0; sp < split; ++sp) v += part[(sp * 16 + m) * cols + c];
    store(m, c, v);
  }
  __syncthreads();
}

__global__ void __launch_bounds__(kTinyThreads, 1) tiny_layer_kernel(TinyArgs a) {
  extern __shared__ __align__(16) uint8_t smem[];
  griddep_wait();
  griddep_launch_dependents();
  const int M = a.M, K = a.K, r = a.r, N = a.N;
  const TinyLayout L = tiny_layout(K, r, N);
  float* xt = reinterpret_cast<float*>(smem + L.xt);
  float* tt = reinterpret_cast<float*>(smem + L.tt);
  float* part = reinterpret_cast<float*>(smem + L.part);
  uint8_t* as = smem + L.araw;
  uint8_t* bs = smem + L.braw;
  const uint32_t ao = stage_raw(as, a.A, static_cast<size_t>(K) * r * 2);
  const uint32_t bo = stage_raw(bs, a.B, static_cast<size_t>(r) * N * 2);
  // X transposed to fp32 while A and B arrive (rows past M read as zero).
  const __nv_bfloat16* X = static_cast<const __nv_bfloat16*>(a.X);
  for (int i = threadIdx.x; i < 16 * K; i += kTinyThreads) {
    const int k = i / 16, m = i - k * 16;
    xt[i] = m < M ? __bfloat162float(X[static_cast<int64_t>(m) * K + k]) : 0.f;
  }
  cp_async_wait_all();
  __syncthreads();
  // T = X·A, kept in fp32 (transposed for the second product).
  tiny_product(xt, as, ao, r, K, r, part, [&](int m, int c, float v) { tt[c * 16 + m] = v; });
  // Y = T·B + bias.
  tiny_product(tt, bs, bo, N, r, N, part, [&](int m, int c, float v) {
    if (m >= M) return;
    if (a.bias) v += __bfloat162float(a.bias[c]);
    const int64_t o = static_cast<int64_t>(m) * a.ldy + c;
    if (a.y_f32)
      static_cast<float*>(a.Y)[o] = v;
    else
      static_cast<__nv_bfloat16*>(a.Y)[o] = __float2bfloat16_rn(v);
  });
}

}  // namespace

size_t tiny_smem_bytes(int64_t M, int64_t K, int64_t r, int64_t N) {
  (void)M;
  return tiny_layout(K, r, N).total;
}

bool tiny_fits(int64_t M, int64_t K, int64_t r, int64_t N) {
  // One CTA's shared memory, and little enough arithmetic that one SM
  // finishes it in a few microseconds (about 8 M multiply-adds at 16 rows).
  return M >= 1 && M <= 16 && K >= 1 && r >= 1 && N >= 1 && K <= 4096 && r <= 4096 &&
         N <= 4096 && tiny_smem_bytes(M, K, r, N) <= kTinyMaxSmem &&
         16 * r * (K + N) <= (int64_t(1) << 23);
}

cudaError_t launch_tiny(const TinyArgs& a, cudaStream_t stream) {
  const size_t smem = tiny_smem_bytes(a.M, a.K, a.r, a.N);
  cudaError_t e = ensure_max_smem(reinterpret_cast<const void*>(tiny_layer_kernel),
                                  static_cast<int>(kTinyMaxSmem));
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(1);
  cfg.blockDim = dim3(kTinyThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, tiny_layer_kernel, a);
}

}  // namespace lr
