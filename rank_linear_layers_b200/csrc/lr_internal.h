// lr_internal.h — declarations shared by the host library and the kernels.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "lr_ptx.cuh"

namespace lr {

// Record a CUDA error for lr_last_cuda_error(), and count kernel launches
// for lr_kernel_launch_count(), from entry points outside lr_api.cu.
void note_cuda_error(int e);
void note_launches(int n);
// Record that an entry point outside lr_api.cu wrote [y, y + bytes) on
// `stream` (the prefill path checks its inputs against recent outputs).
void note_output(cudaStream_t stream, const void* y, size_t bytes);

// Read and clear the status word of lr_linear_decode_static on the current
// device (0 if that entry point was never used there).  Allocates nothing.
cudaError_t static_status_take(unsigned int* code);

// Raise a kernel's dynamic shared-memory limit to `bytes` once per device.
cudaError_t ensure_max_smem(const void* kernel, int bytes);

// The time limit of device-side bounded waits (lr_set_wait_limit_ns).
unsigned long long wait_limit_ns();

// ------------------------------------------------------- streamed decode
// out[m, n] = sum_k V[m, k] · W[k, n] (m < M <= 8) for several "jobs" in
// one persistent launch (one CTA per SM).  A job's W is cut into column
// blocks of cb <= 248 columns; every CTA takes one contiguous slice of each
// phase's (block, row) units, weighted by block width, and streams its rows
// of W through shared memory into the tensor cores.  Phase-0 jobs read a bf16 V; a phase-1 job reads
// as V the fp32 result of phase-0 job `src`, block by block as each block of
// it is finished (a flag per block), so its W stream starts before phase 0
// ends.  The CTA that finishes the last phase-1 block clears the flags: the
// workspace is zero again when the launch ends, and the launch can be
// replayed from a CUDA graph.
constexpr int kStreamMaxJobs = 14;
constexpr int kStreamMaxSegs = 64;  // (job, block, row range) pieces per CTA

struct StreamSeg {
  int job, b, k0, k1;      // rows [k0, k1) of block b of job `job`
};

struct StreamJob {
  const __nv_bfloat16* W;  // [K, ldw] bf16
  int64_t ldw;
  uintptr_t w_lo, w_hi;    // byte extent of W's rows
  int K, N;                // rows and columns of W
  int cb;                  // columns per block: a multiple of 8, at most 248
  int phase;               // 0 or 1
  const void* V;           // [M, ldv]: bf16 (phase 0) or fp32 (phase 1)
  int64_t ldv;
  int src;                 // phase 1: the job whose result V is
  float* acc;              // [M, ld_acc] fp32 partial sums, zero at rest
  int64_t ld_acc;
  unsigned int* cnt;       // [blocks] rows added so far, zero at rest
  unsigned int* ready;     // [blocks] 1 once the block is finished (phase 0), zero at rest
  float* out_f32;          // fp32 result [M, ld_out], or null
  __nv_bfloat16* out_bf16; // bf16 result [M, ld_out], or null
  int64_t ld_out;
  const __nv_bfloat16* bias;  // [N] added to the result, or null
  int64_t unit0;           // first unit of the job within its phase (unit = one element of W)
  // Phase 1, gated output: the result is silu(G) · (sum + bias), G the gate
  // job's stored output (same N and blocks), read once gate_fin[b] is set.
  const void* gate_y;      // null: no gate
  int64_t gate_ld;
  int gate_f32;
  const unsigned int* gate_fin;
  unsigned int* fin;       // phase 1: [blocks] 1 once the block is written (gates), or null
};

struct StreamArgs {
  StreamJob job[kStreamMaxJobs];
  int n_jobs;
  int M;
  unsigned int* done;      // phase-1 blocks finished so far, zero at rest
  int n_final;             // phase-1 blocks in all
  // Each CTA's pieces (stream_segments), computed once per set of job
  // shapes: CTA g's are pieces[piece_off[g] .. piece_off[g + 1]).  Null:
  // the CTAs compute their own.
  const StreamSeg* pieces;
  const int* piece_off;
  int w_early;             // W may be read before the previous launch on the stream ends
  int64_t units[2];        // units of each phase
  WaitCtl wait;
};



// floor(x / w) for 0 <= x < 2^53, w > 0.  On the device through a double
// division and an exact correction (a 64-bit integer division is a long
// software routine there).
__host__ __device__ inline int64_t stream_div(int64_t x, int64_t w) {
#ifdef __CUDA_ARCH__
  int64_t q = static_cast<int64_t>(static_cast<double>(x) / static_cast<double>(w));
  while (q > 0 && q * w > x) --q;
  while ((q + 1) * w <= x) ++q;
  return q;
#else
  return x / w;
#endif
}

__host__ __device__ inline int64_t stream_cdiv_clamp(int64_t x, int64_t w, int64_t hi) {
  if (x <= 0) return 0;
  const int64_t q = stream_div(x + w - 1, w);
  return q < hi ? q : hi;
}

// The pieces CTA g of G streams, phase 0 first: in each phase the units
// [U·g/G, U·(g+1)/G) of the phase's jobs laid end to end, a job's units in
// block order and, within a block, row by row (a row of block b is width(b)
// units).  A row belongs to the CTA whose range holds its first unit.
// Writes at most `cap` pieces; returns how many there are.
__host__ __device__ inline int stream_segments(const StreamArgs& a, int g, int G, StreamSeg* out,
                                               int cap) {
  int n = 0;
  for (int ph = 0; ph < 2; ++ph) {
    const int64_t U = a.units[ph];
    if (U <= 0) continue;
    const int64_t lo = U * g / G, hi = U * (g + 1) / G;
    for (int j = 0; j < a.n_jobs; ++j) {
      const StreamJob& J = a.job[j];
      if (J.phase != ph) continue;
      const int64_t K = J.K, N = J.N, cb = J.cb;
      if (J.unit0 >= hi || J.unit0 + K * N <= lo) continue;
      const int64_t nb = (N + cb - 1) / cb;
      for (int64_t b = 0; b < nb; ++b) {
        const int64_t wb = (N - b * cb) < cb ? (N - b * cb) : cb;
        const int64_t base = J.unit0 + b * K * cb;
        const int64_t k0 = stream_cdiv_clamp(lo - base, wb, K);
        const int64_t k1 = stream_cdiv_clamp(hi - base, wb, K);
        if (k0 < k1) {
          if (n < cap) out[n] = StreamSeg{j, static_cast<int>(b), static_cast<int>(k0),
                                          static_cast<int>(k1)};
          ++n;
        }
      }
    }
  }
  return n;
}

// The piece of block b of job j that CTA g of G takes (k0 == k1: none); the
// same rule as stream_segments, for one block.
__host__ __device__ inline StreamSeg stream_piece(const StreamArgs& a, int j, int64_t b, int g,
                                                  int G) {
  const StreamJob& J = a.job[j];
  const int64_t U = a.units[J.phase];
  const int64_t lo = stream_div(U * g, G), hi = stream_div(U * (g + 1), G);
  const int64_t K = J.K, N = J.N, cb = J.cb;
  const int64_t wb = (N - b * cb) < cb ? (N - b * cb) : cb;
  const int64_t base = J.unit0 + b * K * cb;
  const int64_t k0 = stream_cdiv_clamp(lo - base, wb, K);
  const int64_t k1 = stream_cdiv_clamp(hi - base, wb, K);
  return StreamSeg{j, static_cast<int>(b), static_cast<int>(k0), static_cast<int>(k1)};
}

// Column block width for an output of n columns: the fewest blocks of at
// most 248 columns, of equal width rounded up to a multiple of 8 (a row's
// window of up to 248 + 7 columns is 32 granules of 16 bytes).
inline int stream_block_cols(int64_t n) {
  const int64_t nb = (n + 247) / 248;
  return static_cast<int>(((n + nb - 1) / nb + 7) / 8 * 8);
}

cudaError_t launch_stream(const StreamArgs& a, int grid, cudaStream_t stream, bool dependent);
// Y[m, n] = silu(G[m, n]) · P[m, n] for m < M, n < N (G bf16 or fp32 at
// stride ld_g, P fp32 at stride N, Y bf16 or fp32 at stride ld_y).
cudaError_t launch_silu_mul(const void* G, int64_t ld_g, bool g_f32, const float* P, void* Y,
                            int64_t ld_y, bool y_f32, int64_t M, int64_t N, cudaStream_t stream);

// ------------------------------------------------------------------ decode
// out[m, n] = sum_k V[m, k] · W[k, n] for m < M (M <= 16), W a bf16 [Kd, Nd]
// row-major matrix with row stride ldw.  Split over column blocks (grid.x)
// and row ranges of W (grid.y); partial sums go to acc with fp32 atomics and
// the last CTA of each column block writes the result and re-zeroes acc and
// its counter, so the workspace is zero again when the launch ends.
struct SkinnyArgs {
  int M;
  int64_t Kd, Nd;
  const void* V;   // [M, ldv], bf16 (v_f32 == 0) or fp32
  int64_t ldv;
  int v_f32;
  const __nv_bfloat16* W;
  int64_t ldw;
  uintptr_t w_lo, w_hi;  // byte extent of W's buffer
  float* acc;            // [M, ld_acc] fp32, zero at rest
  int64_t ld_acc;
  unsigned int* counters;  // one per column block, zero at rest
  int k_chunk;             // rows of W per CTA
  int splits;              // == gridDim.y
  float* out_f32;          // if non-null: fp32 result (+bias) [M, ld_out_f32]
  int64_t ld_out_f32;
  __nv_bfloat16* out_bf16;  // else bf16 result (+bias) [M, ld_out]
  int64_t ld_out;
  const __nv_bfloat16* bias;
  WaitCtl wait;             // bounded waits on the copy pipeline
  int after_previous;       // V is written by the previous launch (PDL wait)
};

enum class SkinnyKind { kFma, kMma };

struct SkinnyPlan {
  SkinnyKind kind;
  int mt;         // token tile (1, 2, 4 or 16)
  int cols;       // columns per CTA
  int threads;    // threads per CTA
  int k_chunk;
  int splits;
  int col_blocks;
  size_t smem;    // dynamic shared memory bytes
};

SkinnyPlan plan_skinny(int M, int64_t Kd, int64_t Nd, int num_sms);
// With `dependent`, the launch may start while the previous launch on the
// stream still runs (programmatic dependent launch); the kernel loads its
// first rows of W and then waits for that launch before reading V.
cudaError_t launch_skinny(const SkinnyPlan& plan, const SkinnyArgs& args, cudaStream_t stream,
                          bool dependent = false);

// ------------------------------------------------------------------ tiny layers
// The whole layer in one CTA (lr_tiny.cu) when it fits its shared memory:
// M <= 16 and small factors.
struct TinyArgs {
  int M, K, r, N;
  const void* X;
  const void* A;
  const void* B;
  const __nv_bfloat16* bias;
  void* Y;
  int64_t ldy;
  int y_f32;
};
constexpr size_t kTinyMaxSmem = 200 * 1024;
__host__ __device__ inline size_t tiny_align16(size_t x) { return (x + 15) / 16 * 16; }
size_t tiny_smem_bytes(int64_t M, int64_t K, int64_t r, int64_t N);
bool tiny_fits(int64_t M, int64_t K, int64_t r, int64_t N);
cudaError_t launch_tiny(const TinyArgs& a, cudaStream_t stream);

// ------------------------------------------------------------------ prefill
// C[Mr, Nc] = Aop[Mr, Kc] · Bop[Kc, Nc] (+ bias), bf16 in, fp32 accumulate,
// bf16 out.  Aop is row-major (K contiguous), Bop is row-major (N
// contiguous); both are read through TMA tensor maps, so their base
// addresses and row pitches must be 16-byte aligned.  C may have any
// 2-byte-aligned base and pitch.
struct GemmArgs {
  int Mr, Nc, Kc;
  __nv_bfloat16* c;
  int64_t ldc;
  const __nv_bfloat16* bias;
  int tiles_m, tiles_n;
  WaitCtl wait;
  // Programmatic dependent launch: when `pdl`, the kernel may start while the
  // previous launch on the stream runs; operands flagged dep_a / dep_b are
  // written by earlier launches of the same call and are loaded only after
  // griddepcontrol.wait, the others are loaded before it.
  int pdl, dep_a, dep_b;
  // Testing only: the producer withholds stage 0 of its first tile, so the
  // MMA's bounded wait on it runs out (failure-detection test).
  int withhold_first_stage;
};

struct GemmMaps {
  CUtensorMap a;  // Aop: dims {Kc, Mr}, box {64, 128}
  CUtensorMap b;  // Bop: dims {Nc, Kc}, box {64, 64}
};

constexpr int kGemmBM = 128;
constexpr int kGemmBK = 64;
constexpr int kGemmStages = 4;

// The same GEMM on CTA pairs (2-SM MMA, 256×256 tiles).  The A map's box
// must be {64, 128} and the B map's {64, 64}.
size_t gemm_pair_smem_bytes();
cudaError_t launch_gemm_pair(const GemmArgs& args, const GemmMaps& maps, int num_sms,
                             cudaStream_t stream);

// ------------------------------------------------------------------ chain
// Several GEMMs C_p = Aop_p · Bop_p (+bias_p) in one persistent launch.  The
// launch's tiles are the problems' tiles in order (within a problem, the
// column tiles of one 128-row block are consecutive); CTA i takes tiles
// i, i + grid, i + 2·grid, ...  A problem may signal a counter group: each
// of its tiles, once stored, adds one arrival per epilogue warp
// (kChainEpiWarps) to the counter of its row block.  A later problem may wait on a group: before
// loading operand a (the earlier problem's output) for a row block it waits
// until that row block has `wait_count` arrivals.  Launches alternate
// between two banks of counters; each launch zeroes the bank the next launch
// will use (after the previous launch on the stream has finished), so the
// counters need no reset from the host, even after an aborted launch.
// Every dependency points to a lower tile index, which a running CTA owns,
// so the waits always end (and are bounded regardless).
constexpr int kChainMaxProbs = 12;
constexpr int kChainEpiWarps = 8;  // arrivals per finished tile
constexpr int kChainMaxMaps = 24;

struct ChainProblem {
  int Mr, Nc, Kc;
  int bn;            // tile columns: a multiple of 32 in [32, 256]
  int tiles_m, tiles_n;
  int tile_begin;    // index of the problem's first tile in the launch
  int map_a, map_b;  // indices into ChainMaps
  int a_col0;        // column of operand a where this problem's K range starts
  int b_col0;        // column of operand b where this problem's N range starts
  __nv_bfloat16* c;
  int64_t ldc;
  const __nv_bfloat16* bias;
  // fp32 output: when c32 is set the result (+bias) is stored unrounded as
  // fp32 at c32 [Mr, ldc] and c is unused.
  float* c32;
  // Two-part output (GEMM1 writing T): when c_lo is set, c receives
  // hi = bf16(v) and c_lo [Mr, ldc] receives lo = bf16(v - hi), so that
  // hi + lo carries v to about 16 significant bits.
  __nv_bfloat16* c_lo;
  // Two-part operand a (GEMM2 reading T): when map_a_lo >= 0, every k step
  // is multiplied twice into the same accumulator, once with operand a from
  // map_a and once from map_a_lo (same coordinates).  Both parts and the
  // operand-b tile share one pipeline stage, so bn is at most 128.
  int map_a_lo;
  int wait_group;    // -1, or the counter group that gates operand a
  int wait_count;    // arrivals that complete one row block of that group
  int signal_group;  // -1, or the counter group this problem arrives on
  int dep_a, dep_b;  // operand written by the previous launch on the stream
  // Split K: each output tile is `splits` tiles of the launch, each over
  // kb_per_split k blocks; partial sums are added (fp32 vector reductions)
  // into ws [tiles_m·128, ws_ld], zero at rest, and the last split to
  // finish a warp's region (arrival counter in group split_group, one per
  // tile and epilogue warp) rounds, stores and re-zeroes it.
  int splits, kb_per_split, split_group;
  float* ws;
  int64_t ws_ld;
};

struct ChainArgs {
  int n_prob;
  int total_tiles;
  ChainProblem p[kChainMaxProbs];
  unsigned int* counters;       // this launch's bank: [group][ctr_stride], zero on entry
  unsigned int* counters_next;  // the other bank, zeroed by this launch
  int ctr_stride;
  int n_counters;               // entries per bank
  WaitCtl wait;
  // The launch may start while the previous launch on the stream runs
  // (programmatic dependent launch): operands flagged dep_a / dep_b are
  // loaded only after griddepcontrol.wait, and every thread that writes
  // global memory waits first too.
  int pdl;
  // Testing only: the producer withholds stage 0 of its first tile, so the
  // MMA's bounded wait on it runs out (failure-detection test).
  int withhold_first_stage;
};

struct ChainMaps {
  CUtensorMap m[kChainMaxMaps];  // operand a: box {64, 128}; operand b: box {64, 64}
};

size_t chain_smem_bytes();
// `two`: some problem of the launch reads operand a in two parts (map_a_lo).
cudaError_t launch_chain(const ChainMaps& maps, const ChainArgs& args, int grid, bool two,
                         cudaStream_t stream);

// Copy a [rows, cols] bf16 matrix with any 2-byte-aligned base and pitch lds
// into dst (16-byte-aligned base, pitch ldd >= cols rounded up to 8; the
// columns from cols up to the next multiple of 8 are written as zero).
// src_bytes is the byte extent of the source from its first element.  With
// `dependent`, the launch may start while the previous launch on the stream
// (which must not touch dst) still runs, and completes after it.  Contiguous
// sources go through shared memory with bulk copies (bounded waits: `wait`).
// With `read_early` (contiguous sources only) the copy may read the source
// before the previous launch has finished: only for a source that launch
// does not write.  Either way the launch completes after the previous one.
cudaError_t launch_repack(const __nv_bfloat16* src, int64_t lds, size_t src_bytes,
                          __nv_bfloat16* dst, int64_t ldd, int64_t rows, int64_t cols,
                          int num_sms, cudaStream_t stream, bool dependent, WaitCtl wait,
                          bool read_early = false);

// Y[m, n] = bias[n] (or 0) for an empty contraction (K == 0 or r == 0); Y is
// bf16, or fp32 when y_f32.
cudaError_t launch_fill_bias(void* Y, bool y_f32, int64_t ldy, int64_t M, int64_t N,
                             const __nv_bfloat16* bias, cudaStream_t stream);

}  // namespace lr
