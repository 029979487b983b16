// lr_decode.cu — the decode (M <= 16) path of Y = (X·A)·B (+bias).
//
// Decode multiplies a few token rows by each factor, so it is bound by the
// bytes of A and B streamed from HBM (LowRankArena review, "Why theoretical
// FLOPs saved does not equal faster inference": decode is memory-bandwidth
// bound; GAC paper §3.2: GEMV is memory-bound).  Both contractions are the
// same "skinny" product out = V·W with W a row-major weight:
//   phase 1: V = X [M, K] (bf16),  W = A [K, r]  -> T (fp32, kept in fp32)
//   phase 2: V = T [M, r] (fp32),  W = B [r, N]  -> Y (bf16, + bias)
//
// Each CTA owns a block of output columns and a range of W's rows; partial
// sums over the row range are combined with fp32 atomics, and the last CTA of
// a column block (counter) writes the final values and resets the workspace.
//
// Misaligned rows without realignment.  With a row pitch of ldw elements, the
// position of row k's first wanted element inside its 16-byte chunk is
// (base + k·ldw + n0) mod 8, which depends only on k mod 8.  Each warp reads
// only rows of one residue class mod 8, so its shift s is constant: lane t
// loads the aligned 16-byte chunk t of the row's window and accumulates into
// the columns that chunk holds, 8t - s .. 8t - s + 7 (a column grid shifted
// by s).  No shuffles, no realignment, 4 registers per row in flight; the
// cross-warp reduction maps every warp's shifted columns back to real ones.
// A column block is 248 (or 120) columns so that a 256 (128) element window
// covers it for every shift.
//
//  * M <= 4 : CUDA cores, packed fp32x2 FMA (FFMA2).  A GEMV-shaped product
//             gains nothing from tensor cores.
//  * M <= 16: mma.sync m16n8k16 (bf16 in, fp32 accumulate): at 16 tokens the
//             FMA rate the CUDA cores would need to keep up with HBM exceeds
//             what they issue.  The warp's 16 rows of a k-step are 16 rows of
//             one residue class (any 16 rows can form an MMA's K dimension as
//             long as the A fragment uses the same ones); their aligned
//             chunks go through shared memory and ldmatrix.trans into the B
//             fragment.  In phase 2 the fp32 T is split into bf16 hi + lo
//             parts and both are multiplied, so T keeps about 16 bits.
#include <algorithm>

#include "lr_internal.h"
#include "lr_load.cuh"

namespace lr {

namespace {

constexpr int kRes = 8;          // residue classes of rows mod 8
constexpr int kFmaWarps = 8;     // one warp per residue class
constexpr int kFmaCB = 248;      // columns per CTA (window: 32 chunks)
constexpr int kFmaU = 16;        // rows in flight per warp
constexpr int kMmaWarps = 16;    // residue class × two column halves
constexpr int kMmaCB = 120;      // columns per CTA (window: 16 chunks)
constexpr int kMmaStepRows = 16 * kRes;  // rows covered by one k-step of all residues
constexpr int kMmaRowBytes = 8 * 16 + 16;  // 8 chunks per warp row, padded for ldmatrix
constexpr int kMmaBufBytes = 16 * kMmaRowBytes;
constexpr int kMmaInflight = 3;  // k-steps whose loads are in flight per warp
// V is staged through the transpose buffers in blocks of kMmaRawK values of
// k (rows padded to kMmaRawLd floats: at most 2-way bank conflicts when the
// fragments are read back).
constexpr int kMmaRawK = 512;
constexpr int kMmaRawLd = kMmaRawK + 2;
static_assert(kMmaRawK % kMmaStepRows == 0, "raw blocks hold whole k-steps");
static_assert(16 * kMmaRawLd * 4 <= kMmaWarps * kMmaBufBytes, "raw block fits the buffers");
static_assert((16 * kMmaRawK) % (kMmaWarps * 32) == 0, "whole loads per thread");


constexpr int kSkinnyMaxSmem = 200 * 1024;

// Load the aligned 16-byte chunk at address c (within the tensor [lo, hi))
// if `need`; `fast` says the whole row window is inside the tensor.
__device__ __forceinline__ uint4 window_chunk(uintptr_t c, bool need, bool fast, uintptr_t lo,
                                              uintptr_t hi) {
  if (!need) return make_uint4(0u, 0u, 0u, 0u);
  return fast ? ld_nc_v4(c) : chunk16(c, lo, hi);
}

// Add the CTA's partial sums part[m][c] (c < nvalid) to acc with float4
// atomics; the last CTA of the column block writes the result and leaves acc
// and its counter at zero.
template <int MT, int CB>
__device__ __forceinline__ void reduce_and_finalise(const SkinnyArgs& a, const float* part,
                                                    int64_t n0, int nvalid) {
  __shared__ unsigned int s_is_last;
  __syncthreads();
  constexpr int Q = MT * CB / 4;
  for (int q = threadIdx.x; q < Q; q += blockDim.x) {
    const int m = (4 * q) / CB, c = (4 * q) % CB;
    if (m >= a.M || c >= nvalid) continue;
    const float* src = part + m * CB + c;
    float4 v = make_float4(src[0], c + 1 < nvalid ? src[1] : 0.f, c + 2 < nvalid ? src[2] : 0.f,
                           c + 3 < nvalid ? src[3] : 0.f);
    atomicAdd(reinterpret_cast<float4*>(a.acc + static_cast<int64_t>(m) * a.ld_acc + n0 + c), v);
  }
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) {
    const unsigned int prev = atomicAdd(a.counters + blockIdx.x, 1u);
    s_is_last = (prev == static_cast<unsigned int>(a.splits - 1)) ? 1u : 0u;
  }
  __syncthreads();
  if (!s_is_last) return;
  __threadfence();
  for (int i = threadIdx.x; i < a.M * CB; i += blockDim.x) {
    const int m = i / CB, c = i % CB;
    if (c >= nvalid) continue;
    float* src = a.acc + static_cast<int64_t>(m) * a.ld_acc + n0 + c;
    const float v = __ldcg(src);
    __stcg(src, 0.f);
    const float b = a.bias ? __bfloat162float(a.bias[n0 + c]) : 0.f;
    if (a.out_f32)
      a.out_f32[static_cast<int64_t>(m) * a.ld_out_f32 + n0 + c] = v + b;
    else
      a.out_bf16[static_cast<int64_t>(m) * a.ld_out + n0 + c] = __float2bfloat16_rn(v + b);
  }
  if (threadIdx.x == 0) a.counters[blockIdx.x] = 0u;
}

__device__ __forceinline__ float load_v(const SkinnyArgs& a, int m, int64_t k) {
  const int64_t idx = static_cast<int64_t>(m) * a.ldv + k;
  return a.v_f32 ? __ldcg(static_cast<const float*>(a.V) + idx)
                 : __bfloat162float(static_cast<const __nv_bfloat16*>(a.V)[idx]);
}

// ---------------------------------------------------------------- FMA path
// sv2[kk][m] = (v, v): V[m, k0 + kk] duplicated, the broadcast operand of FFMA2.
template <int MT>
__global__ void __launch_bounds__(kFmaWarps * 32, 2) skinny_fma_kernel(SkinnyArgs a) {
  constexpr int CB = kFmaCB;
  constexpr int U = kFmaU;
  extern __shared__ __align__(16) float smem[];
  float2* sv2 = reinterpret_cast<float2*>(smem);             // [k_chunk][MT]
  float* part = smem + 2 * a.k_chunk * MT;                   // [MT][CB]
  griddep_launch_dependents();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t n0 = static_cast<int64_t>(blockIdx.x) * CB;
  const int64_t k0 = static_cast<int64_t>(blockIdx.y) * a.k_chunk;
  const int kc = static_cast<int>(std::max<int64_t>(0, std::min<int64_t>(a.Kd - k0, a.k_chunk)));
  const int nvalid = static_cast<int>(std::min<int64_t>(CB, a.Nd - n0));

  // This warp's rows: k0 + warp + 8j.  Their shift s is the same for all j.
  const int nrows = (kc > warp) ? (kc - warp + kRes - 1) / kRes : 0;
  const uintptr_t row0 = reinterpret_cast<uintptr_t>(a.W + (k0 + warp) * a.ldw + n0);
  const int s = static_cast<int>((row0 >> 1) & 7u);
  const uintptr_t win0 = row0 & ~static_cast<uintptr_t>(15);
  const uintptr_t step = static_cast<uintptr_t>(kRes * a.ldw * 2);  // bytes between this warp's rows
  const int c0 = 8 * lane - s;                                       // first column of lane's chunk
  const bool need = (c0 < nvalid) && (c0 + 8 > 0);
  // Rows whose whole window lies inside W load without bounds checks.
  const bool all_fast = win0 >= a.w_lo &&
                        win0 + static_cast<uintptr_t>(nrows > 0 ? nrows - 1 : 0) * step + 512 <= a.w_hi;

  auto load_row = [&](int j) -> uint4 {
    const uintptr_t c = win0 + static_cast<uintptr_t>(j) * step + 16u * lane;
    if (!need || j >= nrows) return make_uint4(0u, 0u, 0u, 0u);
    return all_fast ? ld_nc_v4(c) : chunk16(c, a.w_lo, a.w_hi);
  };

  // V's slice into shared memory (duplicated pairs) and zeroed partial sums.
  auto stage_v = [&]() {
    for (int m = 0; m < MT; ++m)
      for (int kk = threadIdx.x; kk < a.k_chunk; kk += blockDim.x) {
        const float v = (m < a.M && kk < kc) ? load_v(a, m, k0 + kk) : 0.f;
        sv2[kk * MT + m] = make_float2(v, v);
      }
    for (int i = threadIdx.x; i < MT * CB; i += blockDim.x) part[i] = 0.f;
    __syncthreads();
  };

  // Rolling pipeline: U rows in flight; consuming row j issues row j + U
  // into the same register slot.  When V is written by the previous launch,
  // the first U rows of W (which do not depend on V) are in flight before
  // waiting for it; otherwise V is staged first, so that its few loads do not
  // queue behind the CTA's (and the whole grid's) loads of W.
  uint4 cur[U];
  if (!a.after_previous) stage_v();
#pragma unroll
  for (int u = 0; u < U; ++u) cur[u] = load_row(u);
  if (a.after_previous) {
    griddep_wait();
    stage_v();
  }

  float2 acc[MT][4];
#pragma unroll
  for (int m = 0; m < MT; ++m)
#pragma unroll
    for (int i = 0; i < 4; ++i) acc[m][i] = make_float2(0.f, 0.f);

  for (int j0 = 0; j0 < nrows; j0 += U) {
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int j = j0 + u;
      if (j < nrows) {
        const float2* vrow = sv2 + (warp + kRes * j) * MT;
        const uint32_t ww[4] = {cur[u].x, cur[u].y, cur[u].z, cur[u].w};
        cur[u] = load_row(j + U);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float2 wp = make_float2(bf16lo_to_f32(ww[i]), bf16hi_to_f32(ww[i]));
#pragma unroll
          for (int m = 0; m < MT; ++m) acc[m][i] = __ffma2_rn(wp, vrow[m], acc[m][i]);
        }
      }
    }
  }

  // Shifted columns back to real ones: lane's element e is column c0 + e.
#pragma unroll
  for (int m = 0; m < MT; ++m)
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int c = c0 + 2 * i;
      if (c >= 0 && c < CB) atomicAdd(part + m * CB + c, acc[m][i].x);
      if (c + 1 >= 0 && c + 1 < CB) atomicAdd(part + m * CB + c + 1, acc[m][i].y);
    }
  reduce_and_finalise<MT, CB>(a, part, n0, nvalid);
}

// ---------------------------------------------------------------- MMA path
__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                               uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
      "{%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void ldsm_x4_trans(uint32_t addr, uint32_t& r0, uint32_t& r1,
                                              uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

// Warp (residue res, half h): k-step j covers rows k0 + res + 8·(16j + i),
// i = 0..15, and chunks 8h .. 8h+7 of each row's 16-chunk window.  Lane l
// loads row i = 4q + l/8 (q = 0..3), chunk 8h + l%8.
struct MmaWarp {
  uintptr_t win0;   // window of row k0 + res
  uintptr_t step;   // bytes between rows of one residue (8 rows)
  uintptr_t lo, hi;
  int nrows;        // rows of this residue in the CTA's range
  bool need;        // this lane's chunk holds wanted columns
  int lane;
  int chunk;        // window chunk this lane loads: 8·half + lane % 8
};

__device__ __forceinline__ void mma_issue(const MmaWarp& w, int j, uint4 (&cur)[4]) {
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const int row = 16 * j + 4 * q + (w.lane >> 3);
    const uintptr_t win = w.win0 + static_cast<uintptr_t>(row) * w.step;
    const bool fast = win >= w.lo && win + 256 <= w.hi;
    cur[q] = window_chunk(win + 16u * w.chunk, w.need && row < w.nrows, fast, w.lo, w.hi);
  }
}

// A fragments staged in the order the warps read them: sfrag[j][res][lane]
// holds the 4 bf16x2 words of the hi part and (phase 2) the 4 of the lo part
// for residue res, k-step j.
template <bool V_F32>
__device__ __forceinline__ void mma_consume(const MmaWarp& w, int j, const uint4 (&cur)[4],
                                            uint8_t* tbuf, const uint4* sfrag, int res,
                                            float (&d)[8][4]) {
  const int lane = w.lane;
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const int i = 4 * q + (lane >> 3);
    *reinterpret_cast<uint4*>(tbuf + i * kMmaRowBytes + (lane & 7) * 16) = cur[q];
  }
  __syncwarp();
  const uint4* fr = sfrag + ((j * kRes + res) * 32 + lane) * 2;
  const uint4 h4 = fr[0];
  const uint32_t ahi[4] = {h4.x, h4.y, h4.z, h4.w};
  uint32_t alo[4] = {0u, 0u, 0u, 0u};
  if (V_F32) {
    const uint4 l4 = fr[1];
    alo[0] = l4.x;
    alo[1] = l4.y;
    alo[2] = l4.z;
    alo[3] = l4.w;
  }
  const uint32_t tb = smem_u32(tbuf);
  const int lm_row = (lane & 7) + ((lane >> 3) & 1) * 8;
  const int lm_col = (lane >> 4) * 8;
#pragma unroll
  for (int nb = 0; nb < 4; ++nb) {
    uint32_t b0, b1, b2, b3;
    ldsm_x4_trans(tb + lm_row * kMmaRowBytes + (nb * 16 + lm_col) * 2, b0, b1, b2, b3);
    mma_bf16_16816(d[2 * nb], ahi, b0, b1);
    mma_bf16_16816(d[2 * nb + 1], ahi, b2, b3);
    if (V_F32) {
      mma_bf16_16816(d[2 * nb], alo, b0, b1);
      mma_bf16_16816(d[2 * nb + 1], alo, b2, b3);
    }
  }
  __syncwarp();
}

template <bool V_F32>
__global__ void __launch_bounds__(kMmaWarps * 32, 1) skinny_mma_kernel(SkinnyArgs a) {
  constexpr int CB = kMmaCB;
  extern __shared__ __align__(16) float smem[];
  uint4* sfrag = reinterpret_cast<uint4*>(smem);                      // [k_chunk/128][8][32][2]
  griddep_launch_dependents();
  float* part = smem + a.k_chunk * 16;                                // [16][CB]
  uint8_t* bufs = reinterpret_cast<uint8_t*>(part + 16 * CB);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int res = warp & (kRes - 1), half = warp >> 3;
  uint8_t* tbuf = bufs + warp * kMmaBufBytes;
  const int64_t n0 = static_cast<int64_t>(blockIdx.x) * CB;
  const int64_t k0 = static_cast<int64_t>(blockIdx.y) * a.k_chunk;
  const int kc = static_cast<int>(std::max<int64_t>(0, std::min<int64_t>(a.Kd - k0, a.k_chunk)));
  const int nvalid = static_cast<int>(std::min<int64_t>(CB, a.Nd - n0));

  MmaWarp w;
  const uintptr_t row0 = reinterpret_cast<uintptr_t>(a.W + (k0 + res) * a.ldw + n0);
  const int s = static_cast<int>((row0 >> 1) & 7u);
  w.win0 = row0 & ~static_cast<uintptr_t>(15);
  w.step = static_cast<uintptr_t>(kRes * a.ldw * 2);
  w.lo = a.w_lo;
  w.hi = a.w_hi;
  w.nrows = (kc > res) ? (kc - res + kRes - 1) / kRes : 0;
  w.lane = lane;
  w.chunk = 8 * half + (lane & 7);
  const int c0 = 8 * w.chunk - s;  // first column of the lane's load chunk
  w.need = (c0 < nvalid) && (c0 + 8 > 0);
  const int nsteps = (w.nrows + 15) / 16;

  float d[8][4];
#pragma unroll
  for (int t = 0; t < 8; ++t)
#pragma unroll
    for (int i = 0; i < 4; ++i) d[t][i] = 0.f;

  // V's slice is staged as the warps read it: sfrag[j][res][lane] holds
  // fragment element e of lane f (g = f/4, tq = f%4) for residue res and
  // k-step j: token g or g+8, local row res + 8·(16j + i) with
  // i in {2tq, 2tq+1, 2tq+8, 2tq+9} (the mma.m16n8k16 A layout), as a bf16
  // hi part and a bf16 lo part (the rounding error of hi; zero for bf16 V).
  auto put_frag = [&](int gi, const float (&v)[8]) {
    uint4 hi, lo;
    hi.x = pack_bf16x2(v[0], v[1]);
    hi.y = pack_bf16x2(v[2], v[3]);
    hi.z = pack_bf16x2(v[4], v[5]);
    hi.w = pack_bf16x2(v[6], v[7]);
    lo.x = pack_bf16x2(v[0] - bf16lo_to_f32(hi.x), v[1] - bf16hi_to_f32(hi.x));
    lo.y = pack_bf16x2(v[2] - bf16lo_to_f32(hi.y), v[3] - bf16hi_to_f32(hi.y));
    lo.z = pack_bf16x2(v[4] - bf16lo_to_f32(hi.z), v[5] - bf16hi_to_f32(hi.z));
    lo.w = pack_bf16x2(v[6] - bf16lo_to_f32(hi.w), v[7] - bf16hi_to_f32(hi.w));
    sfrag[2 * gi] = hi;
    sfrag[2 * gi + 1] = lo;
  };
  // Order of one fragment's elements: (g, i0) (g, i1) (g+8, i0) (g+8, i1)
  // (g, i8) (g, i9) (g+8, i8) (g+8, i9).
  // Direct: each element loaded from V in fragment order (bf16 V: the
  // scattered loads mostly hit L1).
  auto stage_direct = [&]() {
    const int nfrag = (a.k_chunk / kMmaStepRows) * kRes * 32;
    for (int idx = threadIdx.x; idx < nfrag; idx += blockDim.x) {
      const int f = idx & 31, rs = (idx >> 5) & (kRes - 1), j = idx >> 8;
      const int g = f >> 2, tq = f & 3;
      const int ii[4] = {2 * tq, 2 * tq + 1, 2 * tq + 8, 2 * tq + 9};
      float v[8];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int kk = rs + kRes * (16 * j + ii[q]);
        const bool in = kk < kc;
        const int slot = (q < 2) ? q : 4 + (q - 2);
        v[slot] = (in && g < a.M) ? load_v(a, g, k0 + kk) : 0.f;
        v[slot + 2] = (in && g + 8 < a.M) ? load_v(a, g + 8, k0 + kk) : 0.f;
      }
      put_frag(idx, v);
    }
  };
  // Blocked (fp32 V, read from L2 one 32-byte sector per element when loaded
  // in fragment order): through the still idle transpose buffers in blocks
  // of kMmaRawK values of k, coalesced loads into raw[16][kMmaRawLd] (zero
  // outside M and kc), then the fragments of the block's k-steps from there.
  auto stage_blocked = [&]() {
    constexpr int kThreads = kMmaWarps * 32;
    constexpr int kPer = 16 * kMmaRawK / kThreads;
    float* raw = reinterpret_cast<float*>(bufs);
    for (int kb = 0; kb < a.k_chunk; kb += kMmaRawK) {
      float t[kPer];
#pragma unroll
      for (int u = 0; u < kPer; ++u) {
        const int idx = threadIdx.x + u * kThreads;
        const int m = idx / kMmaRawK, kk = kb + idx % kMmaRawK;
        t[u] = (m < a.M && kk < kc) ? load_v(a, m, k0 + kk) : 0.f;
      }
#pragma unroll
      for (int u = 0; u < kPer; ++u) {
        const int idx = threadIdx.x + u * kThreads;
        raw[(idx / kMmaRawK) * kMmaRawLd + idx % kMmaRawK] = t[u];
      }
      __syncthreads();
      const int j0 = kb / kMmaStepRows;
      const int span = (a.k_chunk - kb < kMmaRawK) ? a.k_chunk - kb : kMmaRawK;
      const int nfrag = (span / kMmaStepRows) * kRes * 32;
      for (int idx = threadIdx.x; idx < nfrag; idx += kThreads) {
        const int f = idx & 31, rs = (idx >> 5) & (kRes - 1), jl = idx >> 8;
        const int g = f >> 2, tq = f & 3;
        const int ii[4] = {2 * tq, 2 * tq + 1, 2 * tq + 8, 2 * tq + 9};
        float v[8];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int kl = rs + kRes * (16 * jl + ii[q]);
          const int slot = (q < 2) ? q : 4 + (q - 2);
          v[slot] = raw[g * kMmaRawLd + kl];
          v[slot + 2] = raw[(g + 8) * kMmaRawLd + kl];
        }
        put_frag(j0 * kRes * 32 + idx, v);
      }
      __syncthreads();  // raw is refilled by the next block
    }
  };
  auto stage_v = [&]() {
    if (V_F32) stage_blocked();
    else stage_direct();
    for (int i = threadIdx.x; i < 16 * CB; i += blockDim.x) part[i] = 0.f;
    __syncthreads();
  };
  // When V is written by the previous launch, the first k-steps' rows of W
  // (which do not depend on V) are issued before waiting for it; otherwise V
  // is staged first, so that its loads do not queue behind W's.
  uint4 c_a[4], c_b[4], c_c[4];
  if (!a.after_previous) stage_v();
  mma_issue(w, 0, c_a);
  mma_issue(w, 1, c_b);
  mma_issue(w, 2, c_c);
  if (a.after_previous) {
    griddep_wait();
    stage_v();
  }

  for (int j = 0; j < nsteps; j += kMmaInflight) {
    mma_consume<V_F32>(w, j, c_a, tbuf, sfrag, res, d);
    mma_issue(w, j + 3, c_a);
    if (j + 1 < nsteps) mma_consume<V_F32>(w, j + 1, c_b, tbuf, sfrag, res, d);
    mma_issue(w, j + 4, c_b);
    if (j + 2 < nsteps) mma_consume<V_F32>(w, j + 2, c_c, tbuf, sfrag, res, d);
    mma_issue(w, j + 5, c_c);
  }

  // d[t] holds tokens g, g+8 of n8-tile t: chunk 8·half + t, columns
  // 8·(8·half + t) - s + 2tq, +1 (the shifted grid) -> real columns.
  const int g = lane >> 2, tq = lane & 3;
#pragma unroll
  for (int t = 0; t < 8; ++t) {
    const int c = 8 * (8 * half + t) - s + 2 * tq;
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      if (c + e >= 0 && c + e < CB) {
        atomicAdd(part + g * CB + c + e, d[t][e]);
        atomicAdd(part + (g + 8) * CB + c + e, d[t][2 + e]);
      }
    }
  }
  reduce_and_finalise<16, CB>(a, part, n0, nvalid);
}

}  // namespace

SkinnyPlan plan_skinny(int M, int64_t Kd, int64_t Nd, int num_sms) {
  SkinnyPlan p{};
  int capacity, gran;
  int64_t cap;
  if (M <= 4) {
    p.kind = SkinnyKind::kFma;
    p.mt = M <= 1 ? 1 : (M <= 2 ? 2 : 4);
    p.cols = kFmaCB;
    p.threads = kFmaWarps * 32;
    capacity = std::max(1, num_sms * 2);
    gran = kRes;
    cap = (8192 / p.mt) / gran * gran;  // V slice: k_chunk × MT × 8 bytes <= 64 KB
  } else {
    p.kind = SkinnyKind::kMma;
    p.mt = 16;
    p.cols = kMmaCB;
    p.threads = kMmaWarps * 32;
    capacity = std::max(1, num_sms);
    gran = kMmaStepRows;
    cap = 2048;  // V slice: k_chunk × 64 bytes <= 128 KB
  }
  p.col_blocks = static_cast<int>((Nd + p.cols - 1) / p.cols);
  // Split W's rows so that the grid fills the resident CTA slots in whole
  // waves: the cost of a split count is (waves × rows per CTA), scaled up
  // when the grid leaves slots empty, plus a small charge per split for the
  // partial-sum atomics.
  // Fixed cost of a CTA (staging V, zeroing, the atomics and the last-CTA
  // write), in rows of W.
  const int64_t overhead = (p.kind == SkinnyKind::kFma) ? 160 : 256;
  const int64_t max_splits = std::max<int64_t>(1, std::min<int64_t>(512, (Kd + gran - 1) / gran));
  double best = 1e300;
  p.k_chunk = static_cast<int>(cap);
  p.splits = static_cast<int>((Kd + p.k_chunk - 1) / p.k_chunk);
  for (int64_t sp = 1; sp <= max_splits; ++sp) {
    int64_t chunk = (Kd + sp - 1) / sp;
    chunk = std::min<int64_t>(cap, (chunk + gran - 1) / gran * gran);
    const int64_t splits = (Kd + chunk - 1) / chunk;
    const int64_t items = splits * p.col_blocks;
    const int64_t waves = (items + capacity - 1) / capacity;
    const double fill = static_cast<double>(std::min<int64_t>(items, capacity)) / capacity;
    const double cost = static_cast<double>(waves * (chunk + overhead)) / fill;
    if (cost < best) {
      best = cost;
      p.k_chunk = static_cast<int>(chunk);
      p.splits = static_cast<int>(splits);
    }
  }
  if (p.splits < 1) p.splits = 1;
  if (p.kind == SkinnyKind::kFma) {
    p.smem = static_cast<size_t>(p.k_chunk) * p.mt * sizeof(float2) +
             static_cast<size_t>(p.mt) * kFmaCB * sizeof(float);
  } else {
    p.smem = static_cast<size_t>(p.k_chunk) * 16 * sizeof(float) +
             static_cast<size_t>(16) * kMmaCB * sizeof(float) +
             static_cast<size_t>(kMmaWarps) * kMmaBufBytes;
  }
  return p;
}

cudaError_t launch_skinny(const SkinnyPlan& p, const SkinnyArgs& args, cudaStream_t stream,
                          bool dependent) {
  SkinnyArgs a = args;
  a.k_chunk = p.k_chunk;
  a.splits = p.splits;
  a.after_previous = dependent ? 1 : 0;
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(p.col_blocks, p.splits);
  cfg.blockDim = dim3(p.threads);
  cfg.dynamicSmemBytes = p.smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = dependent ? 1 : 0;
  cudaError_t e = cudaSuccess;
  auto go = [&](auto kern) {
    // Allow the largest dynamic shared memory any plan asks for.
    e = ensure_max_smem(reinterpret_cast<const void*>(kern), kSkinnyMaxSmem);
    if (e != cudaSuccess) return;
    e = cudaLaunchKernelEx(&cfg, kern, a);
  };
  if (p.kind == SkinnyKind::kFma) {
    if (p.mt == 1) go(skinny_fma_kernel<1>);
    else if (p.mt == 2) go(skinny_fma_kernel<2>);
    else go(skinny_fma_kernel<4>);
  } else {
    if (a.v_f32) go(skinny_mma_kernel<true>);
    else go(skinny_mma_kernel<false>);
  }
  return e;
}

}  // namespace lr
