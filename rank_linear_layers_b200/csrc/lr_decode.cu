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
// Each CTA owns a block of output columns and a range of W's rows.  Rows are
// read whole-segment at a time (coalesced 16-byte loads, realigned when the
// row stride r·2 bytes is not a multiple of 16).  Partial sums over the row
// range are combined with fp32 atomics; the last CTA of a column block
// (counter) writes the final values and resets the workspace.
//
//  * M <= 4 : CUDA cores, packed fp32x2 FMA (FFMA2).  A GEMV-shaped product
//             gains nothing from tensor cores.
//  * M <= 16: 16 tokens × 8 columns × 16 rows per mma.sync (bf16 in, fp32
//             accumulate).  At 16 tokens the FMA rate the CUDA cores would
//             need to keep up with HBM exceeds what they issue.  W's rows go
//             through shared memory and ldmatrix.trans into the B fragment.
//             In phase 2 the fp32 T is split into bf16 hi + lo parts and
//             both are multiplied, so T keeps about 16 significant bits.
#include <algorithm>

#include "lr_internal.h"
#include "lr_load.cuh"

namespace lr {

namespace {

constexpr int kWarps = 8;

// Stage V[:, k0:k0+kc] as fp32 [kc_pad][MT] in shared memory (zero padded).
template <int MT>
__device__ __forceinline__ void stage_v_kmajor(float* sv, const SkinnyArgs& a, int64_t k0, int kc,
                                               int kc_pad) {
  for (int i = threadIdx.x; i < MT * kc_pad; i += blockDim.x) {
    const int m = i / kc_pad, kk = i % kc_pad;
    float v = 0.f;
    if (m < a.M && kk < kc) {
      const int64_t idx = static_cast<int64_t>(m) * a.ldv + k0 + kk;
      v = a.v_f32 ? __ldg(static_cast<const float*>(a.V) + idx)
                  : __bfloat162float(static_cast<const __nv_bfloat16*>(a.V)[idx]);
    }
    sv[kk * MT + m] = v;
  }
}

// Sum the per-warp partials [kWarps][MT][COLS] and add them to acc with
// float4 atomics; then let the last CTA of the column block finalise.
template <int MT, int COLS>
__device__ __forceinline__ void reduce_and_finalise(const SkinnyArgs& a, float* part, int64_t n0,
                                                    int nvalid) {
  __shared__ unsigned int s_is_last;
  __syncthreads();
  constexpr int Q = MT * COLS / 4;  // float4 quads per CTA tile
  for (int q = threadIdx.x; q < Q; q += blockDim.x) {
    const int m = (q * 4) / COLS, c = (q * 4) % COLS;
    float4 s = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int w = 0; w < kWarps; ++w) {
      const float4 v = *reinterpret_cast<const float4*>(part + (w * MT + m) * COLS + c);
      s.x += v.x;
      s.y += v.y;
      s.z += v.z;
      s.w += v.w;
    }
    if (m < a.M && c < nvalid) {
      float* dst = a.acc + static_cast<int64_t>(m) * a.ld_acc + n0 + c;
      atomicAdd(reinterpret_cast<float4*>(dst), s);
    }
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
  for (int i = threadIdx.x; i < a.M * COLS; i += blockDim.x) {
    const int m = i / COLS, c = i % COLS;
    if (c >= nvalid) continue;
    float* src = a.acc + static_cast<int64_t>(m) * a.ld_acc + n0 + c;
    const float v = __ldcg(src);
    __stcg(src, 0.f);
    if (a.out_f32) {
      a.out_f32[static_cast<int64_t>(m) * a.ld_out_f32 + n0 + c] = v;
    } else {
      const float b = a.bias ? __bfloat162float(a.bias[n0 + c]) : 0.f;
      a.out_bf16[static_cast<int64_t>(m) * a.ld_out + n0 + c] = __float2bfloat16_rn(v + b);
    }
  }
  if (threadIdx.x == 0) a.counters[blockIdx.x] = 0u;
}

// ---------------------------------------------------------------- FMA path
// One warp reads one 256-column row segment (32 lanes × 8 columns); the 8
// warps take rows round robin, each with U rows in flight.
constexpr int kFmaU = 8;

template <int MT>
__global__ void __launch_bounds__(kWarps * 32, 2) skinny_fma_kernel(SkinnyArgs a) {
  constexpr int CW = 8;
  constexpr int COLS = 32 * CW;
  constexpr int U = kFmaU;
  extern __shared__ __align__(16) float smem[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t n0 = static_cast<int64_t>(blockIdx.x) * COLS;
  const int64_t k0 = static_cast<int64_t>(blockIdx.y) * a.k_chunk;
  const int kc = static_cast<int>(std::max<int64_t>(0, std::min<int64_t>(a.Kd - k0, a.k_chunk)));
  const int nvalid = static_cast<int>(std::min<int64_t>(COLS, a.Nd - n0));

  float* sv = smem;  // [k_chunk][MT]
  stage_v_kmajor<MT>(sv, a, k0, kc, a.k_chunk);
  __syncthreads();

  // acc[m/2][c] holds (token m, token m+1) for column c (FFMA2 pairs over m).
  constexpr int MP = (MT + 1) / 2;
  float2 acc[MP][CW];
#pragma unroll
  for (int i = 0; i < MP; ++i)
#pragma unroll
    for (int c = 0; c < CW; ++c) acc[i][c] = make_float2(0.f, 0.f);

  const __nv_bfloat16* wbase = a.W + n0;
  for (int kk = warp; kk < kc; kk += kWarps * U) {
    uint4 cur[U], ext[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int k = kk + u * kWarps;
      const int nv = (k < kc) ? nvalid : 0;
      seg16_issue(wbase + (k0 + k) * a.ldw, lane, 32, nv, a.w_lo, a.w_hi, cur[u], ext[u]);
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int k = kk + u * kWarps;
      if (k >= kc) break;
      const __nv_bfloat16* rowp = wbase + (k0 + k) * a.ldw;
      const uint4 w = seg16_finish(cur[u], ext[u], seg_shift(rowp), lane, 32, nvalid);
      const float* vrow = sv + k * MT;
      float wf[CW];
      const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        wf[2 * i] = bf16lo_to_f32(ww[i]);
        wf[2 * i + 1] = bf16hi_to_f32(ww[i]);
      }
      if (MT == 1) {
        // One token: plain FMA, acc[0][c].x only.
        const float v = vrow[0];
#pragma unroll
        for (int c = 0; c < CW; ++c) acc[0][c].x = fmaf(v, wf[c], acc[0][c].x);
      } else {
#pragma unroll
        for (int p = 0; p < MP; ++p) {
          const float2 vv = *reinterpret_cast<const float2*>(vrow + 2 * p);
#pragma unroll
          for (int c = 0; c < CW; ++c)
            acc[p][c] = __ffma2_rn(vv, make_float2(wf[c], wf[c]), acc[p][c]);
        }
      }
    }
  }

  // Per-warp partials to shared memory: part[warp][m][col].
  __syncthreads();
  float* part = smem;
#pragma unroll
  for (int p = 0; p < MP; ++p) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int m = 2 * p + h;
      if (m >= MT) break;
      float* dst = part + (warp * MT + m) * COLS + lane * CW;
      float v[CW];
#pragma unroll
      for (int c = 0; c < CW; ++c) v[c] = h ? acc[p][c].y : acc[p][c].x;
      *reinterpret_cast<float4*>(dst) = make_float4(v[0], v[1], v[2], v[3]);
      *reinterpret_cast<float4*>(dst + 4) = make_float4(v[4], v[5], v[6], v[7]);
    }
  }
  reduce_and_finalise<MT, COLS>(a, part, n0, nvalid);
}

// ---------------------------------------------------------------- MMA path
// The CTA owns 64 columns.  A warp step covers 16 rows of W: four load
// instructions of four rows each (8 lanes × 16 B per row), realigned, stored
// to the warp's shared buffer, then read back with ldmatrix.trans as the B
// fragments of 8 mma.m16n8k16 (16 in phase 2).  Two steps are in flight per
// warp (the next step's loads are issued before this step's MMAs).
constexpr int kMmaCols = 64;
constexpr int kMmaRowBytes = kMmaCols * 2 + 16;  // padded: conflict-free ldmatrix
constexpr int kMmaBufBytes = 16 * kMmaRowBytes;
constexpr int kMmaStep = 16 * kWarps;            // rows between a warp's steps

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

struct MmaCtx {
  const __nv_bfloat16* wbase;  // W + n0
  int64_t k0, ldw;
  int kc, nvalid;
  uintptr_t lo, hi;
  int rg, g8;  // row within a load instruction (0..3), lane within the row (0..7)
};

__device__ __forceinline__ void mma_issue(const MmaCtx& c, int ks, uint4 (&cur)[4],
                                          uint4 (&ext)[4]) {
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int k = ks + 4 * i + c.rg;
    const int nv = (k < c.kc) ? c.nvalid : 0;
    seg16_issue(c.wbase + (c.k0 + k) * c.ldw, c.g8, 8, nv, c.lo, c.hi, cur[i], ext[i]);
  }
}

template <bool V_F32>
__device__ __forceinline__ void mma_step(const MmaCtx& c, int ks, const uint4 (&cur)[4],
                                         const uint4 (&ext)[4], uint8_t* tbuf, const float* sv,
                                         float (&d)[8][4], int lane) {
  constexpr int MT = 16;
  // 1. Realign the 16 rows into the warp buffer.
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int row = 4 * i + c.rg;
    const int k = ks + row;
    const int nv = (k < c.kc) ? c.nvalid : 0;
    const uint4 w = seg16_finish(cur[i], ext[i], seg_shift(c.wbase + (c.k0 + k) * c.ldw), c.g8, 8, nv);
    *reinterpret_cast<uint4*>(tbuf + row * kMmaRowBytes + c.g8 * 16) = w;
  }
  __syncwarp();
  // 2. A fragment (tokens × 16 rows of W) from the staged V.
  const int g = lane >> 2, tq = lane & 3;
  uint32_t ahi[4], alo[4];
  {
    const float* v0 = sv + (ks + 2 * tq) * MT;
    const float* v1 = v0 + MT;
    const float* v8 = v0 + 8 * MT;
    const float* v9 = v8 + MT;
    const float f[8] = {v0[g], v1[g], v0[g + 8], v1[g + 8], v8[g], v9[g], v8[g + 8], v9[g + 8]};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint32_t h = pack_bf16x2(f[2 * i], f[2 * i + 1]);
      ahi[i] = h;
      if (V_F32) {
        alo[i] = pack_bf16x2(f[2 * i] - bf16lo_to_f32(h), f[2 * i + 1] - bf16hi_to_f32(h));
      }
    }
  }
  // 3. B fragments via ldmatrix.trans; matrix j = lane/8 covers rows
  // (j&1)*8 .. +7 and columns (j>>1)*8 .. +7 of a 16×16 block.
  const uint32_t tb = smem_u32(tbuf);
  const int lm_row = (lane & 7) + ((lane >> 3) & 1) * 8;
  const int lm_col = (lane >> 4) * 8;
#pragma unroll
  for (int nb = 0; nb < kMmaCols / 16; ++nb) {
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
__global__ void __launch_bounds__(kWarps * 32, 2) skinny_mma_kernel(SkinnyArgs a) {
  constexpr int MT = 16;
  constexpr int COLS = kMmaCols;
  extern __shared__ __align__(16) float smem[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t n0 = static_cast<int64_t>(blockIdx.x) * COLS;
  const int64_t k0 = static_cast<int64_t>(blockIdx.y) * a.k_chunk;
  const int kc = static_cast<int>(std::max<int64_t>(0, std::min<int64_t>(a.Kd - k0, a.k_chunk)));
  const int nvalid = static_cast<int>(std::min<int64_t>(COLS, a.Nd - n0));

  float* sv = smem;  // [k_chunk][16] fp32
  uint8_t* tbuf = reinterpret_cast<uint8_t*>(smem + a.k_chunk * MT) + warp * kMmaBufBytes;
  stage_v_kmajor<MT>(sv, a, k0, kc, a.k_chunk);
  __syncthreads();

  float d[8][4];
#pragma unroll
  for (int t = 0; t < 8; ++t)
#pragma unroll
    for (int i = 0; i < 4; ++i) d[t][i] = 0.f;

  MmaCtx c{a.W + n0, k0, a.ldw, kc, nvalid, a.w_lo, a.w_hi, lane >> 3, lane & 7};
  uint4 ca[4], ea[4], cb[4], eb[4];
  int ks = warp * 16;
  mma_issue(c, ks, ca, ea);
  mma_issue(c, ks + kMmaStep, cb, eb);
  for (; ks < kc; ks += 2 * kMmaStep) {
    mma_step<V_F32>(c, ks, ca, ea, tbuf, sv, d, lane);
    mma_issue(c, ks + 2 * kMmaStep, ca, ea);
    if (ks + kMmaStep < kc) mma_step<V_F32>(c, ks + kMmaStep, cb, eb, tbuf, sv, d, lane);
    mma_issue(c, ks + 3 * kMmaStep, cb, eb);
  }

  // Per-warp partials: d[t] holds rows g, g+8 and columns 8t + 2tq, +1.
  __syncthreads();
  float* part = smem;  // [kWarps][16][COLS]
  const int g = lane >> 2, tq = lane & 3;
#pragma unroll
  for (int t = 0; t < 8; ++t) {
    const int col = 8 * t + 2 * tq;
    *reinterpret_cast<float2*>(part + (warp * MT + g) * COLS + col) = make_float2(d[t][0], d[t][1]);
    *reinterpret_cast<float2*>(part + (warp * MT + g + 8) * COLS + col) =
        make_float2(d[t][2], d[t][3]);
  }
  reduce_and_finalise<MT, COLS>(a, part, n0, nvalid);
}

int round_up(int x, int m) { return (x + m - 1) / m * m; }

constexpr int kSkinnyMaxSmem = 112 * 1024;

}  // namespace

SkinnyPlan plan_skinny(int M, int64_t Kd, int64_t Nd, int num_sms) {
  SkinnyPlan p{};
  p.threads = kWarps * 32;
  if (M <= 4) {
    p.kind = SkinnyKind::kFma;
    p.mt = M <= 1 ? 1 : (M <= 2 ? 2 : 4);
    p.cols = 256;
  } else {
    p.kind = SkinnyKind::kMma;
    p.mt = 16;
    p.cols = kMmaCols;
  }
  p.col_blocks = static_cast<int>((Nd + p.cols - 1) / p.cols);
  // Split W's rows so that the grid fills the resident CTA slots in whole
  // waves: the cost of a split count is (waves × rows per CTA), scaled up
  // when the grid leaves slots empty, plus a small charge per split for the
  // partial-sum atomics.
  const int capacity = std::max(1, num_sms * 2);
  const int gran = (p.kind == SkinnyKind::kFma) ? kWarps : 16;
  const int64_t cap = (p.kind == SkinnyKind::kFma) ? (24576 / p.mt) / gran * gran : 1024;
  const int64_t max_splits = std::max<int64_t>(1, std::min<int64_t>(512, (Kd + gran - 1) / gran));
  double best = 1e300;
  p.k_chunk = static_cast<int>(std::min<int64_t>(cap, round_up(static_cast<int>(std::min<int64_t>(Kd, 1 << 30)), gran)));
  p.splits = static_cast<int>((Kd + p.k_chunk - 1) / p.k_chunk);
  for (int64_t sp = 1; sp <= max_splits; ++sp) {
    int64_t chunk = (Kd + sp - 1) / sp;
    chunk = std::min<int64_t>(cap, (chunk + gran - 1) / gran * gran);
    const int64_t splits = (Kd + chunk - 1) / chunk;
    const int64_t items = splits * p.col_blocks;
    const int64_t waves = (items + capacity - 1) / capacity;
    const double fill = static_cast<double>(std::min<int64_t>(items, capacity)) / capacity;
    const double cost = static_cast<double>(waves * chunk) / fill + 0.5 * static_cast<double>(splits);
    if (cost < best) {
      best = cost;
      p.k_chunk = static_cast<int>(chunk);
      p.splits = static_cast<int>(splits);
    }
  }
  if (p.splits < 1) p.splits = 1;
  const size_t stage = static_cast<size_t>(p.k_chunk) * p.mt * sizeof(float);
  const size_t part = static_cast<size_t>(kWarps) * p.mt * p.cols * sizeof(float);
  if (p.kind == SkinnyKind::kFma) {
    p.smem = std::max(stage, part);
  } else {
    p.smem = std::max(stage + static_cast<size_t>(kWarps) * kMmaBufBytes, part);
  }
  return p;
}

cudaError_t launch_skinny(const SkinnyPlan& p, const SkinnyArgs& args, cudaStream_t stream) {
  dim3 grid(p.col_blocks, p.splits);
  dim3 block(p.threads);
  SkinnyArgs a = args;
  a.k_chunk = p.k_chunk;
  a.splits = p.splits;
  cudaError_t e = cudaSuccess;
  auto go = [&](auto kern) {
    // Allow the largest dynamic shared memory any plan asks for.
    e = ensure_max_smem(reinterpret_cast<const void*>(kern), kSkinnyMaxSmem);
    if (e != cudaSuccess) return;
    kern<<<grid, block, p.smem, stream>>>(a);
    e = cudaGetLastError();
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
