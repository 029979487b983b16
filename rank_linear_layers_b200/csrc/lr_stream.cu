// lr_stream.cu — the streamed decode kernel: both skinny products of a
// decode call (phase 0: T = X·A, phase 1: Y = T·B + bias), or of a whole
// group of them, in one persistent launch.
//
// Decode is bound by the bytes of A and B read from HBM (LowRankArena
// review, "Why theoretical FLOPs saved does not equal faster inference";
// GAC paper §3.2, GEMV is memory-bound).  What keeps HBM busy is a long,
// deep stream per SM: one CTA per SM whose 16 warps each keep 8 row windows
// of W (512 bytes each) in flight with plain 16-byte loads — 64 KB per SM —
// and pass them through a double-buffered shared-memory stage into the
// tensor cores.  (Copy engines were measured here first: one bulk copy or
// one warp of cp.async per 512-byte row window issue at about 10 GB/s per
// SM, a third of what the loads reach.)  Every CTA takes a slice of phase 0
// and a slice of phase 1; its phase-1 rows are loaded while phase 0 is still
// being summed elsewhere, and a block of T is read as soon as the last CTA
// adding to that block has written it (a flag per block).
//
// The product.  A stage holds 128 rows k of one column block of W.  With
// M <= 8 tokens the per-stage work is out^T[n, m] += W^T[n, k] · V^T[k, m]:
// an mma.sync m16n8k16 takes 16 columns × 16 rows of W (ldmatrix.trans from
// the stage) as its A operand and V^T (16 rows × 8 tokens) as B, so no token
// slot is wasted.  A phase-1 V (fp32 T) is split into bf16 hi + lo and both
// are multiplied, so T keeps about 16 bits.
//
// Misaligned rows.  Loads move whole 16-byte granules, so row k's window
// starts at the granule holding its first wanted element, s_k = (address /
// 2) mod 8 elements before it.  s_k depends only on k mod 8, so the stage is
// worked residue class by residue class (rows kb + res + 8i, i = 0..15):
// they share one shift, and the MMA tiles cover the columns on a grid
// shifted by s; the partial sums are put back on the real columns when they
// are added up.  No data is realigned.  A residue's rows sit in consecutive
// slots of 33 granules, so an ldmatrix's 8 rows fall in 8 different bank
// groups.
//
// Partial sums of a (block, row range) piece are added to an fp32 workspace
// with vector atomics; each block counts the rows added so far, and the CTA
// whose rows complete it writes the result and leaves workspace and counter
// at zero for the next launch.
#include <algorithm>

#include "lr_internal.h"
#include "lr_load.cuh"

namespace lr {

namespace {

constexpr int kWarps = 16;     // residue class (8) × half (2)
constexpr int kThreads = kWarps * 32;
constexpr int kRows = 128;     // rows of W per stage, 16 per residue class
constexpr int kPitch = 33 * 16;  // a row slot: 32 granules of window + 1 of padding
constexpr int kStageBytes = kRows * kPitch;
constexpr int kPartCols = 256;
constexpr unsigned kWhereStreamReady = 22;

constexpr int kBufs = 2;        // stage buffers, alternating
constexpr int kVBytes = 64 * 1024;  // V rows held in shared memory (fp32)

template <int MT>
constexpr size_t stream_smem() {
  return static_cast<size_t>(kBufs) * kStageBytes + kVBytes +
         2 * kStreamMaxSegs * sizeof(StreamSeg) + 16;
}
// At the end of a piece the buffer just multiplied holds each residue
// class's partial sums, [8 residues][MT tokens][kPartCols columns] fp32.
static_assert(8 * 8 * kPartCols * 4 <= kStageBytes, "partial sums fit a stage buffer");

// The two warps that load a residue class's 16 rows of a stage.
__device__ __forceinline__ void residue_sync(int res) {
  asm volatile("bar.sync %0, 64;" ::"r"(res + 1) : "memory");
}

__device__ __forceinline__ void red_add_v4(float* p, float a, float b, float c, float d) {
  asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(p), "f"(a), "f"(b), "f"(c),
               "f"(d)
               : "memory");
}

__device__ __forceinline__ void st_release_u32(unsigned int* p, unsigned int v) {
  asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

__device__ __forceinline__ void ldsm_x4_trans(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}

__device__ __forceinline__ void mma_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                          uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
      "{%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint4 v) {
  asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(v.x), "r"(v.y), "r"(v.z),
               "r"(v.w)
               : "memory");
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  const __nv_bfloat162 p = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&p);
}

__device__ __forceinline__ int row_shift(const StreamJob& J, int64_t k, int64_t n0) {
  return static_cast<int>(((reinterpret_cast<uintptr_t>(J.W) >> 1) + k * J.ldw + n0) & 7);
}

// Wait (bounded) until *flag is set.  One lane waits; the warp follows it.
__device__ __forceinline__ bool wait_flag(const StreamArgs& a, const unsigned int* flag, int lane) {
  bool ok = true;
  if (lane == 0 && ld_acquire_u32(flag) == 0u) {
    const unsigned long long t_start = global_ns();
    for (uint32_t it = 1;; ++it) {
      if (ld_acquire_u32(flag) != 0u) break;
      if ((it & 63u) == 0u) {
        if (aborted(a.wait)) {
          ok = false;
          break;
        }
        if (global_ns() - t_start > a.wait.timeout_ns) {
          record_timeout(a.wait, kWhereStreamReady);
          ok = false;
          break;
        }
      }
    }
  }
  __syncwarp();
  return __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
}

// Wait (bounded) until the blocks of phase-0 job S holding columns
// [c0, c1] are finished.  One lane waits; the warp follows it.
__device__ __forceinline__ bool wait_ready(const StreamArgs& a, const StreamJob& S, int64_t c0,
                                           int64_t c1, int lane) {
  bool ok = true;
  if (lane == 0) {
    for (int64_t b = c0 / S.cb; b <= c1 / S.cb && ok; ++b) {
      const unsigned int* flag = S.ready + b;
      if (ld_acquire_u32(flag) != 0u) continue;
      const unsigned long long t_start = global_ns();
      for (uint32_t it = 1;; ++it) {
        if (ld_acquire_u32(flag) != 0u) break;
        if ((it & 63u) == 0u) {
          if (aborted(a.wait)) {
            ok = false;
            break;
          }
          if (global_ns() - t_start > a.wait.timeout_ns) {
            record_timeout(a.wait, kWhereStreamReady);
            ok = false;
            break;
          }
        }
      }
    }
  }
  __syncwarp();
  return __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
}

// The B operands (V^T) of one k step, from the V rows held in shared memory
// (vs[m][k - vbase]): rows k_i = kb + res + 8i of the piece (0 past its
// end), tokens g = lane / 4; lane (g, t) holds i = 2t, 2t+1 in b0 and 2t+8,
// 2t+9 in b1.  A phase-1 V (fp32 T) gives hi and lo parts.
__device__ __forceinline__ void load_b(const float* vs, int vrows, int64_t vbase, int M, bool two,
                                       int64_t kb, int res, int64_t k1, int lane, uint32_t (&bh)[2],
                                       uint32_t (&bl)[2]) {
  const int g = lane >> 2, t = lane & 3;
  const int ii[4] = {2 * t, 2 * t + 1, 2 * t + 8, 2 * t + 9};
  float f[4];
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const int64_t k = kb + res + 8 * ii[q];
    f[q] = (g < M && k < k1) ? vs[g * vrows + static_cast<int>(k - vbase)] : 0.f;
  }
  if (two) {
    float h[4], l[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      h[q] = __bfloat162float(__float2bfloat16_rn(f[q]));
      l[q] = f[q] - h[q];
    }
    bh[0] = pack_bf16(h[0], h[1]);
    bh[1] = pack_bf16(h[2], h[3]);
    bl[0] = pack_bf16(l[0], l[1]);
    bl[1] = pack_bf16(l[2], l[3]);
  } else {
    // A phase-0 V is bf16: exact in fp32 and back.
    bh[0] = pack_bf16(f[0], f[1]);
    bh[1] = pack_bf16(f[2], f[3]);
    bl[0] = bl[1] = 0u;
  }
}

// Rows [vbase, vend) of the piece's V into shared memory (fp32), by the
// whole CTA.  A phase-1 V is read once the blocks of T holding those rows
// are finished.  Returns false if that wait ran out (recorded in the status
// word).
__device__ __forceinline__ bool fill_v(const StreamArgs& a, const StreamJob& J, float* vs,
                                       int vrows, int64_t vbase, int64_t vend) {
  bool ok = true;
  __syncthreads();  // every warp is done with the previous rows
  if (J.phase == 1 && threadIdx.x < 32)
    ok = wait_ready(a, a.job[J.src], vbase, vend - 1, threadIdx.x & 31);
  __syncthreads();
  const int n = static_cast<int>(vend - vbase);
  for (int i = threadIdx.x; i < a.M * n; i += kThreads) {
    const int m = i / n, kk = i - m * n;
    const int64_t k = vbase + kk;
    float v;
    if (J.phase == 1)
      v = __ldcg(static_cast<const float*>(J.V) + m * J.ldv + k);
    else
      v = __bfloat162float(static_cast<const __nv_bfloat16*>(J.V)[m * J.ldv + k]);
    vs[m * vrows + kk] = v;
  }
  __syncthreads();
  return ok;
}

// Row k's window of the block at column n0 (wb <= 248 columns): lane l's
// granule l (zero past the window; bounded loads where a granule reaches
// outside W's rows, which only the first and the last row of W can do).
__device__ __forceinline__ uint4 load_granule(const StreamJob& J, int64_t k, int64_t n0, int wb,
                                              int lane) {
  const uintptr_t a0 = reinterpret_cast<uintptr_t>(J.W + k * J.ldw + n0);
  const uintptr_t ws = a0 & ~static_cast<uintptr_t>(15);
  const uintptr_t we = (a0 + 2u * static_cast<uintptr_t>(wb) + 15u) & ~static_cast<uintptr_t>(15);
  const uintptr_t src = ws + 16u * static_cast<uintptr_t>(lane);
  if (src >= we) return make_uint4(0u, 0u, 0u, 0u);
  if (src >= J.w_lo && src + 16 <= J.w_hi) return ld_nc_v4(src);
  return chunk16(src, J.w_lo, J.w_hi);
}

// Warp (res, h)'s rows of the stage at row kb of piece sg: rows
// kb + res + 8i, i = 8h .. 8h+7 (zero past the piece).
__device__ __forceinline__ void load_stage(const StreamArgs& a, const StreamSeg& sg, int64_t kb,
                                           int res, int half, int lane, uint4 (&cur)[8]) {
  const StreamJob& J = a.job[sg.job];
  const int64_t n0 = static_cast<int64_t>(sg.b) * J.cb;
  const int wb = static_cast<int>(min(static_cast<int64_t>(J.cb), J.N - n0));
#pragma unroll
  for (int q = 0; q < 8; ++q) {
    const int64_t k = kb + res + 8 * (8 * half + q);
    cur[q] = k < sg.k1 ? load_granule(J, k, n0, wb, lane) : make_uint4(0u, 0u, 0u, 0u);
  }
}

template <int MT>
__global__ void __launch_bounds__(kThreads, 1) stream_kernel(const __grid_constant__ StreamArgs a) {
  constexpr int G = MT / 8;  // token groups of 8 (MMA n)
  static_assert(G == 1, "M <= 8");
  extern __shared__ __align__(128) uint8_t smem[];
  uint8_t* stages = smem;                                                // [2][128 slots][528 B]
  float* vs = reinterpret_cast<float*>(smem + kBufs * kStageBytes);     // [M][vrows]
  StreamSeg* segs = reinterpret_cast<StreamSeg*>(smem + kBufs * kStageBytes + kVBytes);
  int* s_nseg = reinterpret_cast<int*>(segs + 2 * kStreamMaxSegs);  // [2]
  unsigned int* s_last = reinterpret_cast<unsigned int*>(s_nseg + 2);
  const int vrows = kVBytes / 4 / a.M;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  griddep_launch_dependents();
  int nseg = 0;
  if (a.pieces) {
    const int p0 = a.piece_off[blockIdx.x];
    nseg = min(a.piece_off[blockIdx.x + 1] - p0, 2 * kStreamMaxSegs);
    for (int i = threadIdx.x; i < nseg; i += kThreads) segs[i] = a.pieces[p0 + i];
    __syncthreads();
  } else {
    // No table: one thread per (job, block) finds its row range; phase-0
    // pieces are listed before phase-1 pieces (their order within a phase
    // does not matter).  The stage buffers hold the two lists meanwhile.
    StreamSeg* lists = reinterpret_cast<StreamSeg*>(stages);  // [2][kStreamMaxSegs]
    if (threadIdx.x < 2) s_nseg[threadIdx.x] = 0;
    __syncthreads();
    for (int j = 0, first = 0; j < a.n_jobs; ++j) {
      const int nb = (a.job[j].N + a.job[j].cb - 1) / a.job[j].cb;
      for (int b = static_cast<int>(threadIdx.x) - first; b < nb; b += kThreads) {
        if (b < 0) continue;
        const StreamSeg p = stream_piece(a, j, b, blockIdx.x, gridDim.x);
        if (p.k0 < p.k1) {
          const int ph = a.job[j].phase;
          const int at = atomicAdd(&s_nseg[ph], 1);
          if (at < kStreamMaxSegs) lists[ph * kStreamMaxSegs + at] = p;  // the host checked the count
        }
      }
      first = (first + nb) % kThreads;
    }
    __syncthreads();
    const int n0s = min(s_nseg[0], kStreamMaxSegs), n1s = min(s_nseg[1], kStreamMaxSegs);
    for (int i = threadIdx.x; i < n0s + n1s; i += kThreads)
      segs[i] = i < n0s ? lists[i] : lists[kStreamMaxSegs + i - n0s];
    __syncthreads();
    nseg = n0s + n1s;
  }
  griddep_wait();

  // Warp (res, h) loads rows kb + res + 8i, i = 8h .. 8h+7, of each stage
  // and multiplies the 16 rows of its residue class by the window's
  // 16-column tiles 8h .. 8h+7.  The rows of the next stage (of the next
  // piece after a piece's last stage) are in flight while a stage is
  // multiplied.  (cp.async into a third buffer, two stages ahead, was
  // measured slower: 2.9 against 2.4 µs per 64 KB stage.)
  const int res = warp & 7, half = warp >> 3;
  const int g = lane >> 2, t = lane & 3;
  // ldmatrix row address of this lane within a stage: slot res·16 + (l mod
  // 8) + 8·(l / 16), granule (l / 8) mod 2 of the tile.
  const uint32_t lrow = static_cast<uint32_t>((res * 16 + (lane & 7) + ((lane >> 4) << 3)) * kPitch +
                                              (((lane >> 3) & 1) << 4));
  // This warp's stores: slot res·16 + 8h + q, granule `lane`.
  const uint32_t srow = static_cast<uint32_t>((res * 16 + 8 * half) * kPitch + 16 * lane);
  const uint32_t base = smem_u32(stages);
  int stage = 0;
  uint4 cur[8];
  if (nseg > 0) load_stage(a, segs[0], segs[0].k0, res, half, lane, cur);
  for (int si = 0; si < nseg; ++si) {
    const StreamSeg sg = segs[si];
    const StreamJob& J = a.job[sg.job];
    const int64_t n0 = static_cast<int64_t>(sg.b) * J.cb;
    const int wb = static_cast<int>(min(static_cast<int64_t>(J.cb), J.N - n0));
    const int s = row_shift(J, sg.k0 + res, n0);  // the same for rows sg.k0 + res + 8i
    const int nt = (s + wb + 15) / 16;            // 16-column tiles of the window
    const bool two = J.phase == 1;
    float d[8][4];
#pragma unroll
    for (int tt = 0; tt < 8; ++tt)
#pragma unroll
      for (int e = 0; e < 4; ++e) d[tt][e] = 0.f;
    // V for up to vrows rows sits in shared memory (a global load under
    // full HBM traffic takes microseconds: none is waited for inside a
    // stage).  A wait for T that runs out is recorded in the status word;
    // the launch then finishes with whatever T holds.
    int64_t vbase = sg.k0, vend = min(static_cast<int64_t>(sg.k1), static_cast<int64_t>(sg.k0) + vrows);
    (void)fill_v(a, J, vs, vrows, vbase, vend);
    for (int64_t kb = sg.k0; kb < sg.k1; kb += kRows, ++stage) {
      if (kb + kRows > vend && vend < sg.k1) {
        vbase = kb;
        vend = min(static_cast<int64_t>(sg.k1), kb + vrows);
        (void)fill_v(a, J, vs, vrows, vbase, vend);
      }
      const uint32_t sb = base + static_cast<uint32_t>((stage % kBufs) * kStageBytes);
#pragma unroll
      for (int q = 0; q < 8; ++q) st_shared_v4(sb + srow + static_cast<uint32_t>(q * kPitch), cur[q]);
      residue_sync(res);
      const int64_t kn = kb + kRows;
      if (kn < sg.k1)
        load_stage(a, sg, kn, res, half, lane, cur);
      else if (si + 1 < nseg)
        load_stage(a, segs[si + 1], segs[si + 1].k0, res, half, lane, cur);
      uint32_t bh[2], bl[2];
      load_b(vs, vrows, vbase, a.M, two, kb, res, sg.k1, lane, bh, bl);
#pragma unroll
      for (int tt = 0; tt < 8; ++tt) {
        const int tile = half * 8 + tt;
        if (tile < nt) {
          uint32_t af[4];
          ldsm_x4_trans(sb + lrow + static_cast<uint32_t>(tile) * 32u, af);
          mma_16816(d[tt], af, bh[0], bh[1]);
          if (two) mma_16816(d[tt], af, bl[0], bl[1]);
        }
      }
    }
    float* part = reinterpret_cast<float*>(stages + ((stage - 1) % kBufs) * kStageBytes);

    // The piece's partial sums onto the real columns: lane (g, t) holds
    // window columns 16·tile + g (+8) for tokens 2t, 2t+1; the real column
    // is the window column - s.  Each residue class writes its own area of
    // the buffer just multiplied (the next stage's rows go to the other
    // buffer); the areas are then added up column by column and the sums
    // added to the workspace.
    __syncthreads();  // every warp is done with that buffer
#pragma unroll
    for (int tt = 0; tt < 8; ++tt) {
      const int tile = half * 8 + tt;
      if (tile < nt) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int c = 16 * tile + g + 8 * (e >> 1) - s;
          const int m = 2 * t + (e & 1);
          if (c >= 0 && c < kPartCols) part[(res * 8 + m) * kPartCols + c] = d[tt][e];
        }
      }
    }
    __syncthreads();
    const int wb4 = (wb + 3) / 4;
    for (int q = threadIdx.x; q < a.M * wb4; q += kThreads) {
      const int m = q / wb4, c4 = 4 * (q - m * wb4);
      float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int r = 0; r < 8; ++r) {
        const float4 u = *reinterpret_cast<const float4*>(part + (r * 8 + m) * kPartCols + c4);
        v.x += u.x;
        v.y += u.y;
        v.z += u.z;
        v.w += u.w;
      }
      // Columns past the block (never written in the areas) add nothing.
      if (c4 + 1 >= wb) v.y = 0.f;
      if (c4 + 2 >= wb) v.z = 0.f;
      if (c4 + 3 >= wb) v.w = 0.f;
      red_add_v4(J.acc + m * J.ld_acc + n0 + c4, v.x, v.y, v.z, v.w);
    }
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) {
      const unsigned int add = static_cast<unsigned int>(sg.k1 - sg.k0);
      const unsigned int prev = atomicAdd(J.cnt + sg.b, add);
      *s_last = (prev + add == static_cast<unsigned int>(J.K)) ? 1u : 0u;
    }
    __syncthreads();
    if (*s_last) {
      // This piece completed the block: write it, re-zero the workspace.
      // A gated block first waits (bounded) for the gate's same block.
      __threadfence();
      if (J.gate_y) {
        if (threadIdx.x < 32) (void)wait_flag(a, J.gate_fin + sg.b, threadIdx.x & 31);
        __syncthreads();
      }
      for (int i = threadIdx.x; i < a.M * wb; i += kThreads) {
        const int m = i / wb, c = i - m * wb;
        float* src = J.acc + m * J.ld_acc + n0 + c;
        float v = __ldcg(src);
        __stcg(src, 0.f);
        if (J.bias) v += __bfloat162float(J.bias[n0 + c]);
        if (J.gate_y) {
          const int64_t gi = m * J.gate_ld + n0 + c;
          const float gv = J.gate_f32 ? __ldcg(static_cast<const float*>(J.gate_y) + gi)
                                      : __bfloat162float(__ushort_as_bfloat16(__ldcg(
                                            static_cast<const unsigned short*>(J.gate_y) + gi)));
          v *= gv / (1.f + expf(-gv));
        }
        if (J.out_f32)
          J.out_f32[m * J.ld_out + n0 + c] = v;
        else
          J.out_bf16[m * J.ld_out + n0 + c] = __float2bfloat16_rn(v);
      }
      __threadfence();
      __syncthreads();
      if (threadIdx.x == 0) {
        J.cnt[sg.b] = 0u;
        if (J.phase == 0) {
          st_release_u32(J.ready + sg.b, 1u);
        } else {
          if (J.fin) st_release_u32(J.fin + sg.b, 1u);
          if (atomicAdd(a.done, 1u) + 1u == static_cast<unsigned int>(a.n_final)) {
            // Every phase-1 block is finished, so every read of a flag is
            // done: clear them for the next launch.
            for (int j = 0; j < a.n_jobs; ++j) {
              const StreamJob& Q = a.job[j];
              const int nb = (Q.N + Q.cb - 1) / Q.cb;
              unsigned int* f = Q.phase == 0 ? Q.ready : Q.fin;
              if (f)
                for (int b = 0; b < nb; ++b) f[b] = 0u;
            }
            *a.done = 0u;
          }
        }
      }
    }
  }
}

template <int MT>
cudaError_t launch_mt(const StreamArgs& a, int grid, cudaStream_t stream, bool dependent) {
  static_assert(stream_smem<MT>() <= 227 * 1024, "shared memory");
  cudaError_t e = ensure_max_smem(reinterpret_cast<const void*>(stream_kernel<MT>),
                                  static_cast<int>(stream_smem<MT>()));
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = stream_smem<MT>();
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = dependent ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, stream_kernel<MT>, a);
}

}  // namespace

namespace {
__global__ void silu_mul_kernel(const void* G, int64_t ld_g, int g_f32, const float* P, void* Y,
                                int64_t ld_y, int y_f32, int64_t M, int64_t N) {
  const int64_t total = M * N;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t m = i / N, n = i - m * N;
    const float g = g_f32 ? static_cast<const float*>(G)[m * ld_g + n]
                          : __bfloat162float(static_cast<const __nv_bfloat16*>(G)[m * ld_g + n]);
    const float v = P[i] * (g / (1.f + expf(-g)));
    if (y_f32)
      static_cast<float*>(Y)[m * ld_y + n] = v;
    else
      static_cast<__nv_bfloat16*>(Y)[m * ld_y + n] = __float2bfloat16_rn(v);
  }
}
}  // namespace

cudaError_t launch_silu_mul(const void* G, int64_t ld_g, bool g_f32, const float* P, void* Y,
                            int64_t ld_y, bool y_f32, int64_t M, int64_t N, cudaStream_t stream) {
  const int64_t total = M * N;
  if (total == 0) return cudaSuccess;
  const int64_t blocks = std::min<int64_t>((total + 255) / 256, 148 * 8);
  silu_mul_kernel<<<static_cast<unsigned>(blocks), 256, 0, stream>>>(G, ld_g, g_f32 ? 1 : 0, P, Y,
                                                                     ld_y, y_f32 ? 1 : 0, M, N);
  return cudaGetLastError();
}

cudaError_t launch_stream(const StreamArgs& a, int grid, cudaStream_t stream, bool dependent) {
  if (a.M > 8) return cudaErrorInvalidValue;
  return launch_mt<8>(a, grid, stream, dependent);
}

}  // namespace lr
