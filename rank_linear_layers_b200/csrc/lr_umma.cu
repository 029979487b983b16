// lr_umma.cu — tcgen05 (5th-generation tensor core) GEMM engine for the
// prefill path of Y = (X·A)·B (+bias).
//
//   GEMM1:  T [M, r] = X [M, K] · A [K, r]        (T written once, bf16)
//   GEMM2:  Y [M, N] = T [M, r] · B [r, N] + bias
//
// Both are C = Aop · Bop with Aop row-major (K contiguous: "K-major") and
// Bop row-major (N contiguous: "MN-major"); the tensor core reads both
// layouts from shared memory directly, so no operand is transposed.
//
// umma_chain_kernel runs a list of such GEMMs in one persistent launch (one
// CTA per SM, warp-specialised, 320 threads):
//   warps 0-7  epilogue: TMEM -> registers -> +bias -> bf16 (or fp32) -> global
//   warp 8     one elected thread issues tcgen05.mma (128 × bn × 16 per issue)
//   warp 9     one thread issues the TMA tile loads (128-byte swizzle)
// A 4-stage shared-memory ring (mbarrier full/empty pairs) feeds the MMA;
// two TMEM accumulators (2 × 256 fp32 columns) let the epilogue of one tile
// overlap the main loop of the next.  Each problem has its own tile width
// bn (a multiple of 16 up to 256), chosen on the host so that the launch's
// tiles spread evenly over the SMs.  GEMM2's tiles of a 128-row block wait
// (bounded) for GEMM1's tiles of that block, so the two contractions share
// one launch and GEMM2 starts row block by row block.  Operands must have
// 16-byte-aligned bases and row pitches (TMA's rule); the host realigns any
// that do not (lr_repack.cu) before launching.
//
// Ragged edges cost no padding on the host: TMA zero-fills out-of-bounds
// rows and columns, the last K block issues only the 16-deep MMA steps it
// needs, and the epilogue predicates rows and columns.  This is the point of
// the GAC paper's §3 analysis (misaligned K or N fall to slower library
// kernels and partially filled tensor-core tiles): here a misaligned r
// changes neither the tile shape nor the MMA rate.
#include <algorithm>

#include "lr_internal.h"

namespace lr {

namespace {

constexpr int BM = kGemmBM;
constexpr int BK = kGemmBK;
constexpr int STAGES = kGemmStages;
constexpr int MAX_BN = 256;
constexpr int A_STAGE = BM * BK * 2;      // 16 KB
constexpr int B_STAGE = BK * MAX_BN * 2;  // 32 KB
constexpr int STAGE = A_STAGE + B_STAGE;
constexpr int B_ATOM = BK * 128;          // one 64-column MN-major atom column: 8 KB
// CTA-pair kernel roles.
constexpr int EPI_WARPS = 4;
constexpr int MMA_WARP = 4;
constexpr int TMA_WARP = 5;
// Chain kernel roles: two epilogue warps per 32-lane quarter of TMEM (warp w
// reads lanes 32·(w mod 4) and takes every other 32-column chunk), then the
// MMA warp and the TMA warp.
constexpr int C_EPI_WARPS = kChainEpiWarps;
constexpr int C_MMA_WARP = C_EPI_WARPS;
constexpr int C_TMA_WARP = C_EPI_WARPS + 1;
constexpr int kChainThreads = (C_EPI_WARPS + 2) * 32;
constexpr uint32_t TMEM_COLS = 2 * MAX_BN;
// Epilogue transpose buffers: per epilogue warp two 32-row × 32-column bf16
// boxes (64-byte rows), used alternately.
constexpr int EPI_BOX = 32 * 64;
constexpr int EPI_STAGE_BYTES = kChainEpiWarps * 2 * EPI_BOX;  // 32 KB

constexpr unsigned kWhereProducer = 1, kWhereMma = 3, kWhereMmaAcc = 4, kWhereEpilogue = 5,
                   kWhereDependency = 6;

__device__ __forceinline__ bool mbar_wait_drain(uint64_t* bar, uint32_t parity,
                                                unsigned long long limit_ns) {
  const unsigned long long t0 = global_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (global_ns() - t0 > limit_ns) return false;
  }
  return true;
}

// Store 32 accumulator columns [col0, col0 + 32) of one output row, columns
// at or past `cend` skipped (the CTA-pair kernel's epilogue).
__device__ __forceinline__ void store_chunk(__nv_bfloat16* c, int64_t ldc,
                                            const __nv_bfloat16* bias, int row, int col0, int cend,
                                            const uint32_t (&v)[32], bool vec_ok) {
  float f[32];
#pragma unroll
  for (int i = 0; i < 32; ++i) f[i] = __uint_as_float(v[i]);
  if (bias) {
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      const int col = col0 + i;
      if (col < cend) f[i] += __bfloat162float(bias[col]);
    }
  }
  __nv_bfloat16* dst = c + static_cast<int64_t>(row) * ldc + col0;
  if (vec_ok && col0 + 32 <= cend) {
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      uint4 w;
      w.x = pack_bf16x2(f[8 * q + 0], f[8 * q + 1]);
      w.y = pack_bf16x2(f[8 * q + 2], f[8 * q + 3]);
      w.z = pack_bf16x2(f[8 * q + 4], f[8 * q + 5]);
      w.w = pack_bf16x2(f[8 * q + 6], f[8 * q + 7]);
      *reinterpret_cast<uint4*>(dst + 8 * q) = w;
    }
  } else {
#pragma unroll
    for (int i = 0; i < 32; ++i)
      if (col0 + i < cend) dst[i] = __float2bfloat16_rn(f[i]);
  }
}

// The chain kernel's epilogue for one 32-row × 32-column chunk held one row
// per lane (v = fp32 columns col0 .. col0 + 31 of row row0 + lane): round to
// bf16 (+bias) and transpose through a 2 KB shared buffer (64-byte rows,
// 16-byte chunks swizzled by row so that both the row-wise writes and the
// column-wise reads touch each bank once per 128 bytes), then store with
// each instruction covering 8 rows × 64 contiguous bytes instead of 32 rows
// × 16 bytes.  Generic loads and stores only: no proxy fence, so nothing
// waits for the SM's in-flight TMA or tensor-core traffic.
__device__ __forceinline__ void emit_chunk(uint8_t* buf, const uint32_t (&v)[32],
                                           __nv_bfloat16* c, int64_t ldc,
                                           const __nv_bfloat16* bias, int row0, int Mr, int col0,
                                           int cend, bool vec_ok, int lane) {
  uint32_t w[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    float lo = __uint_as_float(v[2 * i]), hi = __uint_as_float(v[2 * i + 1]);
    if (bias) {
      const int cl = col0 + 2 * i;
      if (cl < cend) lo += __bfloat162float(bias[cl]);
      if (cl + 1 < cend) hi += __bfloat162float(bias[cl + 1]);
    }
    w[i] = pack_bf16x2(lo, hi);
  }
  const int sw = (lane >> 1) & 3;
#pragma unroll
  for (int q = 0; q < 4; ++q)
    *reinterpret_cast<uint4*>(buf + lane * 64 + ((q ^ sw) << 4)) =
        make_uint4(w[4 * q], w[4 * q + 1], w[4 * q + 2], w[4 * q + 3]);
  __syncwarp();
  const int q = lane & 3;
  const int col = col0 + 8 * q;
#pragma unroll
  for (int s = 0; s < 4; ++s) {
    const int r = 8 * s + (lane >> 2);
    const uint4 u = *reinterpret_cast<const uint4*>(buf + r * 64 + ((q ^ ((r >> 1) & 3)) << 4));
    const int row = row0 + r;
    if (row >= Mr || col >= cend) continue;
    __nv_bfloat16* dst = c + static_cast<int64_t>(row) * ldc + col;
    if (vec_ok && col + 8 <= cend) {
      *reinterpret_cast<uint4*>(dst) = u;
    } else {
      const uint32_t e[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
      for (int i = 0; i < 8; ++i)
        if (col + i < cend)
          dst[i] = __ushort_as_bfloat16(static_cast<unsigned short>(e[i >> 1] >> (16 * (i & 1))));
    }
  }
  __syncwarp();
}

// Split K: add one 32-row × 32-column fp32 chunk (one row per lane, as read
// from TMEM) into the workspace, transposed through the warp's 4 KB buffer
// (128-byte rows, 16-byte chunks swizzled by row) so that each vector
// reduction covers 4 rows × 128 contiguous bytes.
__device__ __forceinline__ void split_add_chunk(uint8_t* buf, const uint32_t (&v)[32], float* ws,
                                                int64_t ld, int row0, int col0, int lane) {
#pragma unroll
  for (int q = 0; q < 8; ++q)
    *reinterpret_cast<uint4*>(buf + lane * 128 + ((q ^ (lane & 7)) << 4)) =
        make_uint4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
  __syncwarp();
  const int c = lane & 7;
#pragma unroll
  for (int s = 0; s < 8; ++s) {
    const int r = 4 * s + (lane >> 3);
    const uint4 u = *reinterpret_cast<const uint4*>(buf + r * 128 + ((c ^ (r & 7)) << 4));
    float4* dst = reinterpret_cast<float4*>(ws + static_cast<int64_t>(row0 + r) * ld + col0 + 4 * c);
    atomicAdd(dst, make_float4(__uint_as_float(u.x), __uint_as_float(u.y), __uint_as_float(u.z),
                               __uint_as_float(u.w)));
  }
  __syncwarp();
}

// fp32 output: one 32-row × 32-column chunk (one row per lane) plus bias,
// unrounded, transposed through the warp's 4 KB buffer (128-byte rows,
// 16-byte chunks swizzled by row) so that each store covers 4 rows × 128
// contiguous bytes.
__device__ __forceinline__ void emit_chunk_f32(uint8_t* buf, const uint32_t (&v)[32], float* c,
                                               int64_t ldc, const __nv_bfloat16* bias, int row0,
                                               int Mr, int col0, int cend, bool vec_ok, int lane) {
  float f[32];
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    f[i] = __uint_as_float(v[i]);
    if (bias && col0 + i < cend) f[i] += __bfloat162float(bias[col0 + i]);
  }
#pragma unroll
  for (int q = 0; q < 8; ++q)
    *reinterpret_cast<float4*>(buf + lane * 128 + ((q ^ (lane & 7)) << 4)) =
        make_float4(f[4 * q], f[4 * q + 1], f[4 * q + 2], f[4 * q + 3]);
  __syncwarp();
  const int cq = lane & 7;
  const int col = col0 + 4 * cq;
#pragma unroll
  for (int s = 0; s < 8; ++s) {
    const int r = 4 * s + (lane >> 3);
    const float4 u = *reinterpret_cast<const float4*>(buf + r * 128 + ((cq ^ (r & 7)) << 4));
    const int row = row0 + r;
    if (row >= Mr || col >= cend) continue;
    float* dst = c + static_cast<int64_t>(row) * ldc + col;
    if (vec_ok && col + 4 <= cend) {
      *reinterpret_cast<float4*>(dst) = u;
    } else {
      const float e[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
      for (int i = 0; i < 4; ++i)
        if (col + i < cend) dst[i] = e[i];
    }
  }
  __syncwarp();
}

// Store one accumulator chunk in the problem's output form: bf16 (+bias),
// fp32 (+bias), or the two bf16 parts hi = bf16(v), lo = bf16(v - hi) (no
// bias).  Uses the warp's whole 4 KB buffer.
__device__ __forceinline__ void emit_out(const ChainProblem& P, uint8_t* bufs,
                                         const uint32_t (&v)[32], int row0, int col0, int cend,
                                         int lane) {
  if (P.c32) {
    const bool vec32 = ((reinterpret_cast<uintptr_t>(P.c32) & 15u) == 0) && ((P.ldc & 3) == 0);
    emit_chunk_f32(bufs, v, P.c32, P.ldc, P.bias, row0, P.Mr, col0, cend, vec32, lane);
    return;
  }
  const bool vec_ok = ((reinterpret_cast<uintptr_t>(P.c) & 15u) == 0) && ((P.ldc & 7) == 0);
  emit_chunk(bufs, v, P.c, P.ldc, P.bias, row0, P.Mr, col0, cend, vec_ok, lane);
  if (P.c_lo) {
    uint32_t lo[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      const float f = __uint_as_float(v[i]);
      lo[i] = __float_as_uint(f - __bfloat162float(__float2bfloat16_rn(f)));
    }
    const bool vec_lo = ((reinterpret_cast<uintptr_t>(P.c_lo) & 15u) == 0) && ((P.ldc & 7) == 0);
    emit_chunk(bufs + EPI_BOX, lo, P.c_lo, P.ldc, nullptr, row0, P.Mr, col0, cend, vec_lo, lane);
  }
}

constexpr int kGemmThreads = 6 * 32;

__device__ __forceinline__ int find_problem(const ChainArgs& g, int tile) {
  int i = 0;
  while (i + 1 < g.n_prob && tile >= g.p[i + 1].tile_begin) ++i;
  return i;
}

// Wait until row block m_blk of counter group `grp` has `count` arrivals.
// Bounded; on a timeout it records the error.
__device__ bool wait_rows_ready(const ChainArgs& g, int grp, int m_blk, int count) {
  const unsigned int* ctr = g.counters + static_cast<int64_t>(grp) * g.ctr_stride + m_blk;
  unsigned long long t0 = 0;
  for (uint32_t it = 0;; ++it) {
    if (ld_acquire_u32(ctr) >= static_cast<unsigned int>(count)) break;
    if (it == 0) t0 = global_ns();
    __nanosleep(64);
    if ((it & 15u) == 15u) {
      if (aborted(g.wait)) return false;
      if (global_ns() - t0 > g.wait.timeout_ns) {
        record_timeout(g.wait, kWhereDependency);
        return false;
      }
    }
  }
  // Order the acquire before this thread's TMA (async-proxy) reads.
  fence_proxy_async_global();
  return true;
}

// kTwo: some problem reads operand a in two parts; without it the two-part
// code is compiled out of the copy and MMA loops.
template <bool kTwo>
__global__ void __launch_bounds__(kChainThreads, 1)
    umma_chain_kernel(const __grid_constant__ ChainMaps maps, const __grid_constant__ ChainArgs g) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* base = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  uint8_t* epi_stage = base + STAGES * STAGE;  // 1024-aligned
  uint64_t* full = reinterpret_cast<uint64_t*>(epi_stage + EPI_STAGE_BYTES);
  uint64_t* empty = full + STAGES;
  uint64_t* tfull = empty + STAGES;
  uint64_t* tempty = tfull + 2;
  uint64_t* fin = tempty + 2;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(fin + 1);
  auto stage_a = [&](int s) { return base + s * STAGE; };
  auto stage_b = [&](int s) { return base + s * STAGE + A_STAGE; };

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  griddep_launch_dependents();

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1u);
      mbar_init(&empty[s], 1u);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&tfull[i], 1u);
      mbar_init(&tempty[i], C_EPI_WARPS);
    }
    mbar_init(fin, 1u);
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(tmem_holder, TMEM_COLS);
    tmem_relinquish();
  }
  if (warp == C_TMA_WARP && lane == 0 && blockIdx.x < g.total_tiles) {
    const ChainProblem& P = g.p[find_problem(g, blockIdx.x)];
    tma_prefetch_desc(&maps.m[P.map_a]);
    tma_prefetch_desc(&maps.m[P.map_b]);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;

  // Producer bookkeeping for a clean exit after a timeout.
  int issued_phase[STAGES];
#pragma unroll
  for (int s = 0; s < STAGES; ++s) issued_phase[s] = -1;
  bool ok = true;

  if (warp == C_TMA_WARP) {
    if (lane == 0) {
      int s = 0;
      uint32_t ph = 0;
      bool first = true;
      for (int tile = blockIdx.x; tile < g.total_tiles && ok; tile += gridDim.x) {
        const ChainProblem& P = g.p[find_problem(g, tile)];
        const int local = tile - P.tile_begin;
        const int otile = local / P.splits, kbase = (local - otile * P.splits) * P.kb_per_split;
        const int m_blk = otile / P.tiles_n, n_blk = otile - m_blk * P.tiles_n;
        const int num_kb = min((P.Kc + BK - 1) / BK - kbase, P.kb_per_split);
        const int nbox = (P.bn + 63) / 64;
        const bool two = kTwo && P.map_a_lo >= 0;  // bn <= 128: the low part goes after the b tile
        const uint32_t bytes = (two ? 2 : 1) * A_STAGE + nbox * B_ATOM;
        const CUtensorMap* ma = &maps.m[P.map_a];
        const CUtensorMap* ma_lo = two ? &maps.m[P.map_a_lo] : nullptr;
        const CUtensorMap* mb = &maps.m[P.map_b];
        auto load_a = [&](int st, int kb) {
          const int x = P.a_col0 + (kbase + kb) * BK, y = m_blk * BM;
          tma_load_2d(stage_a(st), ma, &full[st], x, y);
          if (two) tma_load_2d(stage_b(st) + 2 * B_ATOM, ma_lo, &full[st], x, y);
        };
        auto load_b = [&](int st, int kb) {
          for (int c = 0; c < nbox; ++c)
            tma_load_2d(stage_b(st) + c * B_ATOM, mb, &full[st], P.b_col0 + n_blk * P.bn + c * 64,
                        (kbase + kb) * BK);
        };
        const bool gated_a = P.dep_a || P.wait_group >= 0;
        const bool gated_b = P.dep_b;
        int kb0 = 0;
        if (first) {
          first = false;
          if (g.pdl) {
            // Fill the first (free) stages with operands nothing earlier
            // writes, wait for the previous launch, then add the rest.
            const int pre = num_kb < STAGES ? num_kb : STAGES;
            const int skip = g.withhold_first_stage ? 1 : 0;
            for (int kb = skip; kb < pre; ++kb) {
              mbar_arrive_expect_tx(&full[kb], bytes);
              if (!gated_a) load_a(kb, kb);
              if (!gated_b) load_b(kb, kb);
              issued_phase[kb] = 0;
            }
            griddep_wait();
            if (P.wait_group >= 0 && !wait_rows_ready(g, P.wait_group, m_blk, P.wait_count)) {
              ok = false;
              break;
            }
            for (int kb = skip; kb < pre; ++kb) {
              if (gated_a) load_a(kb, kb);
              if (gated_b) load_b(kb, kb);
            }
            kb0 = pre;
            s = pre % STAGES;
            ph = (pre == STAGES) ? 1u : 0u;
          }
        }
        if (kb0 == 0 && P.wait_group >= 0) {
          // Operand b does not depend on the rows being waited for: put it
          // into the first stages, then wait, then add operand a.
          const int pre = num_kb < STAGES ? num_kb : STAGES;
          const int s0 = s;
          for (int kb = 0; kb < pre && ok; ++kb) {
            if (!mbar_wait(&empty[s], ph ^ 1u, g.wait, kWhereProducer)) {
              ok = false;
              break;
            }
            mbar_arrive_expect_tx(&full[s], bytes);
            load_b(s, kb);
            issued_phase[s] = static_cast<int>(ph);
            if (++s == STAGES) {
              s = 0;
              ph ^= 1u;
            }
          }
          if (!ok || !wait_rows_ready(g, P.wait_group, m_blk, P.wait_count)) {
            ok = false;
            break;
          }
          for (int kb = 0; kb < pre; ++kb) load_a((s0 + kb) % STAGES, kb);
          kb0 = pre;
        }
        for (int kb = kb0; kb < num_kb; ++kb) {
          if (!mbar_wait(&empty[s], ph ^ 1u, g.wait, kWhereProducer)) {
            ok = false;
            break;
          }
          if (!(g.withhold_first_stage && kb == 0 && tile == static_cast<int>(blockIdx.x))) {
            mbar_arrive_expect_tx(&full[s], bytes);
            load_a(s, kb);
            load_b(s, kb);
            issued_phase[s] = static_cast<int>(ph);
          }
          if (++s == STAGES) {
            s = 0;
            ph ^= 1u;
          }
        }
      }
    }
  } else if (warp == C_MMA_WARP) {
    int s = 0;
    uint32_t ph = 0;
    int it = 0;
    for (int tile = blockIdx.x; tile < g.total_tiles && ok; tile += gridDim.x, ++it) {
      const ChainProblem& P = g.p[find_problem(g, tile)];
      const int local = tile - P.tile_begin;
      const int kbase = (local - (local / P.splits) * P.splits) * P.kb_per_split;
      const int num_kb = min((P.Kc + BK - 1) / BK - kbase, P.kb_per_split);
      const uint32_t idesc = idesc_bf16_f32(BM, P.bn, false, true);
      const bool two = kTwo && P.map_a_lo >= 0;
      const int acc = it & 1;
      const uint32_t aph = static_cast<uint32_t>(it >> 1) & 1u;
      if (!mbar_wait(&tempty[acc], aph ^ 1u, g.wait, kWhereMmaAcc)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * MAX_BN);
      for (int kb = 0; kb < num_kb; ++kb) {
        if (!mbar_wait(&full[s], ph, g.wait, kWhereMma)) {
          ok = false;
          break;
        }
        tc_fence_after();
        if (lane == 0) {
          const int krem = P.Kc - (kbase + kb) * BK;
          const int nk = krem >= BK ? BK / 16 : (krem + 15) / 16;
          const uint32_t a0 = smem_u32(stage_a(s));
          const uint32_t b0 = smem_u32(stage_b(s));
          for (int kk = 0; kk < nk; ++kk) {
            const uint64_t ad = sdesc_sw128(a0 + kk * 32, 16, 1024);
            const uint64_t bd = sdesc_sw128(b0 + kk * 2048, B_ATOM, 1024);
            umma_bf16(d_tmem, ad, bd, idesc, (kb | kk) != 0 ? 1u : 0u);
            if (two) {
              const uint64_t ad_lo = sdesc_sw128(b0 + 2 * B_ATOM + kk * 32, 16, 1024);
              umma_bf16(d_tmem, ad_lo, bd, idesc, 1u);
            }
          }
          umma_commit(&empty[s]);
        }
        __syncwarp();
        if (++s == STAGES) {
          s = 0;
          ph ^= 1u;
        }
      }
      if (!ok) break;
      if (lane == 0) umma_commit(&tfull[acc]);
      __syncwarp();
    }
  } else if (warp < C_EPI_WARPS) {
    // Under programmatic dependent launch, write nothing before the previous
    // launch on the stream has finished (it may still read these buffers).
    griddep_wait();
    if (blockIdx.x == 0)  // the next launch's counter bank (the previous launch used it)
      for (int i = threadIdx.x; i < g.n_counters; i += C_EPI_WARPS * 32) g.counters_next[i] = 0u;
    int it = 0;
    for (int tile = blockIdx.x; tile < g.total_tiles && ok; tile += gridDim.x, ++it) {
      const ChainProblem& P = g.p[find_problem(g, tile)];
      const int local = tile - P.tile_begin;
      const int otile = local / P.splits;
      const int m_blk = otile / P.tiles_n, n_blk = otile - m_blk * P.tiles_n;
      const int acc = it & 1;
      const uint32_t aph = static_cast<uint32_t>(it >> 1) & 1u;
      if (!mbar_wait(&tfull[acc], aph, g.wait, kWhereEpilogue)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const bool vec_ok =
          ((reinterpret_cast<uintptr_t>(P.c) & 15u) == 0) && ((P.ldc & 7) == 0);
      const int quarter = warp & 3, half = warp >> 2;
      const int row0 = m_blk * BM + quarter * 32;
      const int n0 = n_blk * P.bn;
      const int cend = min(P.Nc, n0 + P.bn);
      const uint32_t t_row = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) +
                             static_cast<uint32_t>(acc * MAX_BN);
      uint8_t* bufs = epi_stage + warp * (2 * EPI_BOX);
      // This warp's chunks are half, half + 2, ...  They alternate between
      // two register sets (the TMEM load of the next chunk is in flight
      // while one is rounded and stored) and two shared buffers.
      const int nch = (min(P.bn, cend - n0) + 31) / 32;
      uint32_t va[32], vb[32];
      bool last = true;  // this warp's region of the output tile is final
      if (P.splits == 1 && (P.c32 || P.c_lo)) {
#pragma unroll 1
        for (int c = half; c < nch; c += 2) {
          tmem_ld_32x32b_x32(t_row + static_cast<uint32_t>(c * 32), va);
          tmem_ld_wait(va);
          emit_out(P, bufs, va, row0, n0 + c * 32, cend, lane);
        }
      } else if (P.splits == 1) {
        if (half < nch) tmem_ld_32x32b_x32(t_row + static_cast<uint32_t>(half * 32), va);
#pragma unroll 1
        for (int c = half; c < nch; c += 4) {
          tmem_ld_wait(va);
          if (c + 2 < nch) tmem_ld_32x32b_x32(t_row + static_cast<uint32_t>((c + 2) * 32), vb);
          emit_chunk(bufs, va, P.c, P.ldc, P.bias, row0, P.Mr, n0 + c * 32, cend, vec_ok, lane);
          if (c + 2 < nch) {
            tmem_ld_wait(vb);
            if (c + 4 < nch) tmem_ld_32x32b_x32(t_row + static_cast<uint32_t>((c + 4) * 32), va);
            emit_chunk(bufs + EPI_BOX, vb, P.c, P.ldc, P.bias, row0, P.Mr, n0 + (c + 2) * 32,
                       cend, vec_ok, lane);
          }
        }
      } else {
        // Split K: add this split's partial sums into the workspace; the
        // last split of this warp's region rounds, stores and re-zeroes it.
#pragma unroll 1
        for (int c = half; c < nch; c += 2) {
          tmem_ld_32x32b_x32(t_row + static_cast<uint32_t>(c * 32), va);
          tmem_ld_wait(va);
          split_add_chunk(bufs, va, P.ws, P.ws_ld, row0, n0 + c * 32, lane);
        }
        __threadfence();
        __syncwarp();
        unsigned int before = 0;
        if (lane == 0)
          before = atomicAdd(g.counters + static_cast<int64_t>(P.split_group) * g.ctr_stride +
                                 static_cast<int64_t>(otile) * C_EPI_WARPS + warp,
                             1u);
        before = __shfl_sync(0xffffffffu, before, 0);
        last = (before == static_cast<unsigned int>(P.splits - 1));
        if (last) {
          __threadfence();
#pragma unroll 1
          for (int c = half; c < nch; c += 2) {
            float4* src = reinterpret_cast<float4*>(
                P.ws + static_cast<int64_t>(row0 + lane) * P.ws_ld + n0 + c * 32);
#pragma unroll
            for (int q = 0; q < 8; ++q) {
              const float4 f = __ldcg(src + q);
              va[4 * q] = __float_as_uint(f.x);
              va[4 * q + 1] = __float_as_uint(f.y);
              va[4 * q + 2] = __float_as_uint(f.z);
              va[4 * q + 3] = __float_as_uint(f.w);
              __stcg(src + q, make_float4(0.f, 0.f, 0.f, 0.f));
            }
            emit_out(P, bufs, va, row0, n0 + c * 32, cend, lane);
          }
        }
      }
      tc_fence_before();
      if (P.signal_group >= 0 && last) {
        // This warp's rows of the tile are written: make them visible to the
        // TMA loads of other CTAs, then count the arrival.
        fence_proxy_async_global();
        __syncwarp();
        if (lane == 0) {
          fence_proxy_async_global();
          __threadfence();
          atomicAdd(g.counters + static_cast<int64_t>(P.signal_group) * g.ctr_stride + m_blk, 1u);
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty[acc]);
    }
  }

  // Teardown.  Every wait above is bounded, so every thread gets here.
  if (warp == C_MMA_WARP && lane == 0) {
    // All MMAs this thread issued are complete once fin flips.
    umma_commit(fin);
    mbar_wait_drain(fin, 0u, 2000000000ull);
  }
  if (warp == C_TMA_WARP && lane == 0 && !ok) {
    // After a timeout: let any TMA load still in flight land before exit.
    for (int s = 0; s < STAGES; ++s)
      if (issued_phase[s] >= 0)
        mbar_wait_drain(&full[s], static_cast<uint32_t>(issued_phase[s]), 1000000ull);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

// ---------------------------------------------------------------- CTA pairs
// The same GEMM on pairs of SMs (a cluster of two CTAs, tcgen05 cta_group::2):
// a pair computes a 256×256 tile; CTA r of the pair loads rows
// [128r, 128r+128) of the A tile and columns [128r, 128r+128) of the B tile,
// and its TMEM receives rows [128r, 128r+128) × all 256 columns of the
// result.  Per SM a k block moves 32 KB (16 KB of A, 16 KB of B) instead of
// 48 KB for the same tensor-core time, so shared-memory traffic drops by a
// third and six stages fit.  The even CTA issues the MMAs; its commits
// arrive on the barriers of both CTAs; the odd CTA's TMA loads complete on
// the even CTA's full barrier; both epilogues release the accumulator on the
// even CTA's barrier.
constexpr int P_BM = 256;           // pair tile rows (128 per CTA)
constexpr int P_BN = 256;           // pair tile columns (128 loaded per CTA)
constexpr int P_STAGES = 6;
constexpr int P_A_STAGE = 128 * BK * 2;  // 16 KB
constexpr int P_B_STAGE = 128 * BK * 2;  // 16 KB (this CTA's half of B)
constexpr int P_STAGE = P_A_STAGE + P_B_STAGE;
constexpr int P_EPI_ARRIVALS = 2 * EPI_WARPS;

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kGemmThreads, 1)
    umma_gemm_pair_kernel(const __grid_constant__ CUtensorMap map_a,
                          const __grid_constant__ CUtensorMap map_b, const GemmArgs g) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* base = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  uint64_t* full = reinterpret_cast<uint64_t*>(base + P_STAGES * P_STAGE);
  uint64_t* empty = full + P_STAGES;
  uint64_t* tfull = empty + P_STAGES;
  uint64_t* tempty = tfull + 2;
  uint64_t* fin = tempty + 2;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(fin + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = (rank == 0);

  if (threadIdx.x == 0) {
    for (int s = 0; s < P_STAGES; ++s) {
      mbar_init(&full[s], 1u);   // the even CTA's expect_tx; both CTAs' bytes
      mbar_init(&empty[s], 1u);  // one multicast commit per stage
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&tfull[i], 1u);
      mbar_init(&tempty[i], P_EPI_ARRIVALS);
    }
    mbar_init(fin, 1u);
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc_pair(tmem_holder, TMEM_COLS);
    tmem_relinquish_pair();
  }
  if (warp == TMA_WARP && lane == 0) {
    tma_prefetch_desc(&map_a);
    tma_prefetch_desc(&map_b);
  }
  tc_fence_before();
  cluster_sync_all();  // barriers of both CTAs initialised before any remote use
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;

  const int tiles_m = (g.Mr + P_BM - 1) / P_BM;
  const int tiles_n = (g.Nc + P_BN - 1) / P_BN;
  const int num_tiles = tiles_m * tiles_n;
  const int cluster = blockIdx.x >> 1, clusters = gridDim.x >> 1;
  const int num_kb = (g.Kc + BK - 1) / BK;
  int issued_phase[P_STAGES];
#pragma unroll
  for (int s = 0; s < P_STAGES; ++s) issued_phase[s] = -1;
  bool ok = true;

  if (warp == TMA_WARP) {
    if (lane == 0) {
      int s = 0;
      uint32_t ph = 0;
      for (int tile = cluster; tile < num_tiles && ok; tile += clusters) {
        const int m_blk = tile % tiles_m, n_blk = tile / tiles_m;
        const int row0 = m_blk * P_BM + static_cast<int>(rank) * 128;
        const int col0 = n_blk * P_BN + static_cast<int>(rank) * 128;
        for (int kb = 0; kb < num_kb; ++kb) {
          if (!mbar_wait(&empty[s], ph ^ 1u, g.wait, kWhereProducer)) {
            ok = false;
            break;
          }
          if (leader) mbar_arrive_expect_tx(&full[s], 2 * P_STAGE);
          uint8_t* a_dst = base + s * P_STAGE;
          uint8_t* b_dst = a_dst + P_A_STAGE;
          tma_load_2d_pair(a_dst, &map_a, &full[s], kb * BK, row0);
          tma_load_2d_pair(b_dst, &map_b, &full[s], col0, kb * BK);
          tma_load_2d_pair(b_dst + B_ATOM, &map_b, &full[s], col0 + 64, kb * BK);
          issued_phase[s] = static_cast<int>(ph);
          if (++s == P_STAGES) {
            s = 0;
            ph ^= 1u;
          }
        }
      }
    }
  } else if (warp == MMA_WARP) {
    if (leader) {
      const uint32_t idesc = idesc_bf16_f32(P_BM, P_BN, false, true);
      int s = 0;
      uint32_t ph = 0;
      int it = 0;
      for (int tile = cluster; tile < num_tiles && ok; tile += clusters, ++it) {
        const int acc = it & 1;
        const uint32_t aph = static_cast<uint32_t>(it >> 1) & 1u;
        if (!mbar_wait(&tempty[acc], aph ^ 1u, g.wait, kWhereMmaAcc)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * P_BN);
        for (int kb = 0; kb < num_kb; ++kb) {
          if (!mbar_wait(&full[s], ph, g.wait, kWhereMma)) {
            ok = false;
            break;
          }
          tc_fence_after();
          if (lane == 0) {
            const int krem = g.Kc - kb * BK;
            const int nk = krem >= BK ? BK / 16 : (krem + 15) / 16;
            const uint32_t a0 = smem_u32(base + s * P_STAGE);
            const uint32_t b0 = a0 + P_A_STAGE;
            for (int kk = 0; kk < nk; ++kk) {
              const uint64_t ad = sdesc_sw128(a0 + kk * 32, 16, 1024);
              const uint64_t bd = sdesc_sw128(b0 + kk * 2048, B_ATOM, 1024);
              umma_bf16_pair(d_tmem, ad, bd, idesc, (kb | kk) != 0 ? 1u : 0u);
            }
            umma_commit_pair(&empty[s], 0x3);
          }
          __syncwarp();
          if (++s == P_STAGES) {
            s = 0;
            ph ^= 1u;
          }
        }
        if (!ok) break;
        if (lane == 0) umma_commit_pair(&tfull[acc], 0x3);
        __syncwarp();
      }
    }
  } else if (warp < EPI_WARPS) {
    const bool vec_ok = ((reinterpret_cast<uintptr_t>(g.c) & 15u) == 0) && ((g.ldc & 7) == 0);
    const uint32_t leader_tempty0 = mapa_shared(smem_u32(&tempty[0]), 0);
    int it = 0;
    for (int tile = cluster; tile < num_tiles && ok; tile += clusters, ++it) {
      const int m_blk = tile % tiles_m, n_blk = tile / tiles_m;
      const int acc = it & 1;
      const uint32_t aph = static_cast<uint32_t>(it >> 1) & 1u;
      if (!mbar_wait(&tfull[acc], aph, g.wait, kWhereEpilogue)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const int row = m_blk * P_BM + static_cast<int>(rank) * 128 + warp * 32 + lane;
      const uint32_t t_row = tmem_base + (static_cast<uint32_t>(warp * 32) << 16) +
                             static_cast<uint32_t>(acc * P_BN);
#pragma unroll 1
      for (int c = 0; c < P_BN / 32; ++c) {
        const int col0 = n_blk * P_BN + c * 32;
        if (col0 >= g.Nc) break;
        uint32_t v[32];
        tmem_ld_32x32b_x32(t_row + static_cast<uint32_t>(c * 32), v);
        tmem_ld_wait();
        if (row < g.Mr) store_chunk(g.c, g.ldc, g.bias, row, col0, g.Nc, v, vec_ok);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(leader_tempty0 + static_cast<uint32_t>(acc * 8));
    }
  }

  // Teardown.  Every wait above is bounded, so every thread gets here.
  if (leader && warp == MMA_WARP && lane == 0) {
    umma_commit_pair(fin, 0x1);
    mbar_wait_drain(fin, 0u, 2000000000ull);
  }
  if (leader && warp == TMA_WARP && lane == 0 && !ok) {
    // After a timeout: the pair's TMA loads complete on these barriers.
    for (int s = 0; s < P_STAGES; ++s)
      if (issued_phase[s] >= 0)
        mbar_wait_drain(&full[s], static_cast<uint32_t>(issued_phase[s]), 1000000ull);
  }
  tc_fence_before();
  cluster_sync_all();  // no CTA leaves while its peer may still touch its memory
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, TMEM_COLS);
  }
}

__global__ void fill_bias_kernel(__nv_bfloat16* Y, float* Y32, int64_t ldy, int64_t M, int64_t N,
                                 const __nv_bfloat16* bias) {
  const int64_t total = M * N;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t m = i / N, n = i % N;
    if (Y32)
      Y32[m * ldy + n] = bias ? __bfloat162float(bias[n]) : 0.f;
    else
      Y[m * ldy + n] = bias ? bias[n] : __float2bfloat16_rn(0.f);
  }
}

}  // namespace

size_t chain_smem_bytes() {
  return 1024 + static_cast<size_t>(STAGES) * STAGE + EPI_STAGE_BYTES +
         (2 * STAGES + 5) * sizeof(uint64_t) + 16;
}

size_t gemm_pair_smem_bytes() {
  return 1024 + static_cast<size_t>(P_STAGES) * P_STAGE + (2 * P_STAGES + 5) * sizeof(uint64_t) +
         16;
}

cudaError_t launch_gemm_pair(const GemmArgs& g, const GemmMaps& maps, int num_sms,
                             cudaStream_t stream) {
  const size_t smem = gemm_pair_smem_bytes();
  cudaError_t e = ensure_max_smem(reinterpret_cast<const void*>(umma_gemm_pair_kernel),
                                  static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  const int tiles = ((g.Mr + P_BM - 1) / P_BM) * ((g.Nc + P_BN - 1) / P_BN);
  const int clusters = std::max(1, std::min(tiles, num_sms / 2));
  umma_gemm_pair_kernel<<<2 * clusters, kGemmThreads, smem, stream>>>(maps.a, maps.b, g);
  return cudaGetLastError();
}

cudaError_t launch_chain(const ChainMaps& maps, const ChainArgs& g, int grid, bool two,
                         cudaStream_t stream) {
  const size_t smem = chain_smem_bytes();
  const void* kern = two ? reinterpret_cast<const void*>(umma_chain_kernel<true>)
                         : reinterpret_cast<const void*>(umma_chain_kernel<false>);
  cudaError_t e = ensure_max_smem(kern, static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(std::max(1, grid));
  cfg.blockDim = dim3(kChainThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = g.pdl ? 1 : 0;
  if (two) return cudaLaunchKernelEx(&cfg, umma_chain_kernel<true>, maps, g);
  return cudaLaunchKernelEx(&cfg, umma_chain_kernel<false>, maps, g);
}

cudaError_t launch_fill_bias(void* Y, bool y_f32, int64_t ldy, int64_t M, int64_t N,
                             const __nv_bfloat16* bias, cudaStream_t stream) {
  const int64_t total = M * N;
  const int threads = 256;
  const int blocks = static_cast<int>(std::min<int64_t>((total + threads - 1) / threads, 4096));
  fill_bias_kernel<<<std::max(blocks, 1), threads, 0, stream>>>(
      y_f32 ? nullptr : static_cast<__nv_bfloat16*>(Y), y_f32 ? static_cast<float*>(Y) : nullptr,
      ldy, M, N, bias);
  return cudaGetLastError();
}

}  // namespace lr
