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
// bias, and stores Y.  Both products run on mma.sync m16n8k16 (the 16 token
// rows are the MMA's M; bf16 in, fp32 accumulate), each warp taking
// (8-column tile, k range) tasks whose partial sums are added in k-range
// order.  T enters the second product as two bf16 parts, hi = bf16(T) and
// lo = bf16(T - hi), so it keeps about 16 bits, as the decode path does.
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

__device__ __forceinline__ void mma16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                         uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
      "{%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Splits of a product's k steps over warps, so that every warp has work.
__host__ __device__ inline int tiny_ksplit(int n_tiles, int k_steps) {
  int s = (16 + n_tiles - 1) / n_tiles;
  if (s > k_steps) s = k_steps;
  if (s > 4) s = 4;
  return s < 1 ? 1 : s;
}

// Shared memory layout (16-byte aligned parts): X as bf16 [16][kp] (kp = K
// rounded up to 16, zero past K and M), T's bf16 hi and lo parts [16][rp]
// (rp = r rounded up to 16, zero past r), T fp32 [16][r], partial sums
// [splits][16][cols], then the raw 16-byte chunks covering A and B.
struct TinyLayout {
  size_t xs, th, tl, t, part, araw, braw, total;
  int kp, rp;
};

__host__ __device__ inline TinyLayout tiny_layout(int64_t K, int64_t r, int64_t N) {
  TinyLayout L;
  L.kp = static_cast<int>((K + 15) / 16 * 16);
  L.rp = static_cast<int>((r + 15) / 16 * 16);
  L.xs = 0;
  L.th = L.xs + tiny_align16(static_cast<size_t>(16) * L.kp * 2);
  L.tl = L.th + tiny_align16(static_cast<size_t>(16) * L.rp * 2);
  L.t = L.tl + tiny_align16(static_cast<size_t>(16) * L.rp * 2);
  L.part = L.t + tiny_align16(static_cast<size_t>(16) * r * 4);
  const int nt1 = static_cast<int>((r + 7) / 8), nt2 = static_cast<int>((N + 7) / 8);
  const size_t p1 = static_cast<size_t>(tiny_ksplit(nt1, L.kp / 16)) * 16 * nt1 * 8 * 4;
  const size_t p2 = static_cast<size_t>(tiny_ksplit(nt2, L.rp / 16)) * 16 * nt2 * 8 * 4;
  L.araw = L.part + tiny_align16(p1 > p2 ? p1 : p2);
  L.braw = L.araw + tiny_align16(static_cast<size_t>(K) * r * 2 + 32);
  L.total = L.braw + tiny_align16(static_cast<size_t>(r) * N * 2 + 32);
  return L;
}

// out[16][cols] = V[16][depth] · W[depth][cols] on mma.m16n8k16: V from
// bf16 rows (vh, and vl as a second part when non-null) of pitch vp
// (zero-padded to a multiple of 16), W from raw bf16 (wbase + woff, row
// pitch ldw; entries past depth or cols read as zero).  Warps take
// (n tile, k range) tasks; the k ranges' partial sums are added in order and
// handed to store(m, c, value), warp m taking row m.  The shared-memory
// offsets fit in 32 bits (at most 200 KB); a lane's column is checked once
// per task and the rows once per k step.
template <typename Store>
__device__ __forceinline__ void tiny_mma_product(const uint16_t* vh, const uint16_t* vl, int vp,
                                                 const uint8_t* wbase, uint32_t woff, int64_t ldw,
                                                 int depth, int cols, float* part, Store store) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;
  const int nt = (cols + 7) / 8, ks = (depth + 15) / 16;
  const int split = tiny_ksplit(nt, ks);
  const uint32_t row_bytes = static_cast<uint32_t>(ldw) * 2u;
  for (int task = warp; task < nt * split; task += kTinyThreads / 32) {
    const int n_tile = task % nt, sp = task / nt;
    const int k0 = ks * sp / split, k1 = ks * (sp + 1) / split;
    const int n = n_tile * 8 + g;
    const bool n_in = n < cols;
    // This lane's column of W, and its A-fragment rows of V.
    const uint8_t* wcol = wbase + woff + 2u * static_cast<uint32_t>(n_in ? n : 0);
    const uint32_t* vh0 = reinterpret_cast<const uint32_t*>(vh + g * vp) + t;
    const uint32_t* vh8 = reinterpret_cast<const uint32_t*>(vh + (g + 8) * vp) + t;
    const uint32_t* vl0 = vl ? reinterpret_cast<const uint32_t*>(vl + g * vp) + t : nullptr;
    const uint32_t* vl8 = vl ? reinterpret_cast<const uint32_t*>(vl + (g + 8) * vp) + t : nullptr;
    float d[4] = {0.f, 0.f, 0.f, 0.f};
    for (int kstep = k0; kstep < k1; ++kstep) {
      const int kb = kstep * 16;
      const int ka = kb + 2 * t;
      auto w = [&](int k) -> uint32_t {
        return (n_in && k < depth)
                   ? *reinterpret_cast<const unsigned short*>(wcol + static_cast<uint32_t>(k) * row_bytes)
                   : 0u;
      };
      uint32_t b0, b1;
      if (n_in && kb + 16 <= depth) {
        const uint8_t* p = wcol + static_cast<uint32_t>(ka) * row_bytes;
        b0 = *reinterpret_cast<const unsigned short*>(p) |
             (static_cast<uint32_t>(*reinterpret_cast<const unsigned short*>(p + row_bytes)) << 16);
        const uint8_t* q = p + 8u * row_bytes;
        b1 = *reinterpret_cast<const unsigned short*>(q) |
             (static_cast<uint32_t>(*reinterpret_cast<const unsigned short*>(q + row_bytes)) << 16);
      } else {
        b0 = w(ka) | (w(ka + 1) << 16);
        b1 = w(ka + 8) | (w(ka + 9) << 16);
      }
      const int kw = kb / 2;  // 32-bit words into a V row
      uint32_t av[4] = {vh0[kw], vh8[kw], vh0[kw + 4], vh8[kw + 4]};
      mma16816(d, av, b0, b1);
      if (vl) {
        uint32_t al[4] = {vl0[kw], vl8[kw], vl0[kw + 4], vl8[kw + 4]};
        mma16816(d, al, b0, b1);
      }
    }
    // C fragment: rows g, g + 8; columns 2t, 2t + 1 of the n tile.
    float* pp = part + static_cast<int64_t>(sp) * 16 * nt * 8;
    const int c = n_tile * 8 + 2 * t;
    pp[g * nt * 8 + c] = d[0];
    pp[g * nt * 8 + c + 1] = d[1];
    pp[(g + 8) * nt * 8 + c] = d[2];
    pp[(g + 8) * nt * 8 + c + 1] = d[3];
  }
  __syncthreads();
  // Warp m adds up and stores row m (16 warps, 16 rows).
  static_assert(kTinyThreads / 32 == 16, "one warp per token row");
  const int m = warp;
  for (int c = lane; c < cols; c += 32) {
    float v = 0.f;
    for (int sp = 0; sp < split; ++sp) v += part[(sp * 16 + m) * nt * 8 + c];
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
  uint16_t* xs = reinterpret_cast<uint16_t*>(smem + L.xs);
  uint16_t* th = reinterpret_cast<uint16_t*>(smem + L.th);
  uint16_t* tl = reinterpret_cast<uint16_t*>(smem + L.tl);
  float* tf = reinterpret_cast<float*>(smem + L.t);
  float* part = reinterpret_cast<float*>(smem + L.part);
  uint8_t* as = smem + L.araw;
  uint8_t* bs = smem + L.braw;
  const uint32_t ao = stage_raw(as, a.A, static_cast<size_t>(K) * r * 2);
  const uint32_t bo = stage_raw(bs, a.B, static_cast<size_t>(r) * N * 2);
  // X into aligned bf16 rows while A and B arrive (zero past M and K);
  // warp m takes row m.
  const unsigned short* X = static_cast<const unsigned short*>(a.X);
  const int wm = threadIdx.x >> 5, wl = threadIdx.x & 31;
  for (int k = wl; k < L.kp; k += 32)
    xs[wm * L.kp + k] = (wm < M && k < K) ? X[static_cast<int64_t>(wm) * K + k]
                                           : static_cast<unsigned short>(0);
  cp_async_wait_all();
  __syncthreads();
  // T = X·A in fp32; then its bf16 hi and lo parts (zero past r) for the
  // second product, so that T keeps about 16 bits.
  tiny_mma_product(xs, nullptr, L.kp, as, ao, r, K, r, part,
                   [&](int m, int c, float v) { tf[m * r + c] = v; });
  for (int c = wl; c < L.rp; c += 32) {
    const float v = c < r ? tf[wm * r + c] : 0.f;
    const __nv_bfloat16 hi = __float2bfloat16_rn(v);
    const __nv_bfloat16 lo = __float2bfloat16_rn(v - __bfloat162float(hi));
    th[wm * L.rp + c] = __bfloat16_as_ushort(hi);
    tl[wm * L.rp + c] = __bfloat16_as_ushort(lo);
  }
  __syncthreads();
  // Y = T·B + bias.
  tiny_mma_product(th, tl, L.rp, bs, bo, N, r, N, part, [&](int m, int c, float v) {
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
