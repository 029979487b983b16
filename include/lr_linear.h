/*
 * lr_linear.h — C ABI of the B200 (sm_100a) low-rank linear layer library.
 *
 * The layer:   Y = (X · A) · B  (+ bias)
 *
 *   X    [M, K]  activations (M tokens)
 *   A    [K, r]  first factor      } W [K, N] ≈ A · B, the factorisation that
 *   B    [r, N]  second factor     } SVD-style compression puts in place of a
 *   bias [N]     optional          } dense Y = X · W
 *   Y    [M, N]  output
 *
 * Sources: "Why Smaller Is Slower? Dimensional Misalignment in Compressed
 * LLMs" (GAC), §1 Introduction and Figure 1 — low-rank factorisation replaces
 * W by A·B and makes the reduced rank r the inner dimension of two smaller
 * GEMMs; LowRankArena review, "What SVD-based LLM compression actually does" —
 * a truncated SVD stored as two factors, k(m+n) parameters, forward pass as
 * two multiplies.  r is often not a multiple of 8 (e.g. 107, 1741); every
 * entry point accepts any r >= 0.
 *
 * Conventions for every entry point:
 *   - All tensors are bf16 (IEEE bfloat16 bit patterns), row-major and
 *     contiguous unless a leading dimension is given.  Accumulation is fp32;
 *     Y is rounded once to bf16 (nearest-even) after the bias is added, or
 *     stored unrounded in fp32 by lr_linear_f32 (and by group entries with
 *     y_f32 set).
 *   - Device pointers point to memory of the current CUDA device.  Any
 *     2-byte-aligned pointer is accepted; 16-byte-aligned pointers with row
 *     strides that are multiples of 8 elements take the TMA fast path.
 *   - `stream` is a cudaStream_t (NULL = the legacy default stream).  Calls
 *     are asynchronous: Y is valid once the stream has been synchronised.
 *   - The caller owns every tensor.  The library owns a workspace per
 *     (device, stream) for the intermediate T = X·A and split-K partial sums,
 *     grown on demand with cudaMalloc (which synchronises the device); it is
 *     kept until lr_release_workspaces() or process exit.
 *   - Errors: invalid arguments return LR_ERR_INVALID_ARG before anything is
 *     launched; a failed CUDA call returns LR_ERR_CUDA (see lr_last_cuda_error).
 *     Device-side bounded waits that run out set a device status word, which
 *     lr_last_device_status() reports; no kernel traps or asserts.
 *   - Calls on one stream are ordered; calls that share a stream must not run
 *     concurrently from several host threads.
 */
#ifndef LR_LINEAR_H
#define LR_LINEAR_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  LR_OK = 0,
  LR_ERR_INVALID_ARG = 1,  /* bad size, null or overlapping pointer            */
  LR_ERR_UNSUPPORTED = 2,  /* no sm_100 device, or a size beyond int32 tiles  */
  LR_ERR_CUDA = 3,         /* a CUDA runtime/driver call failed                */
  LR_ERR_TIMEOUT = 4,      /* a device-side bounded wait ran out               */
  LR_ERR_NO_MEMORY = 5,    /* workspace allocation failed                      */
  LR_ERR_INFEASIBLE = 6    /* lr_gac_select: no selection fits the budget      */
} lr_status;

/*
 * lr_linear — Y = (X·A)·B + bias on the device.
 *
 * X [M,K], A [K,r], B [r,N], bias [N] (may be NULL), Y [M,N]: device
 * pointers, bf16, row-major contiguous.  Y must not overlap X, A, B or bias.
 * Sizes: 0 <= M, K, r, N < 2^31.  M == 0 or N == 0: nothing is launched.
 * K == 0 or r == 0: the sum is empty and Y = bias (or 0).
 *
 * Path: a layer small enough for one SM (M <= 16; K, r, N <= 4096; X, A, B
 * and the intermediates within 200 KB of shared memory; contiguous operands;
 * automatic path only) runs in one CTA and one launch.  Otherwise M <= 16
 * takes the decode kernels (bandwidth-bound streaming of A then B, T kept in
 * fp32; two launches, the second streaming B while the first finishes).
 * Larger M takes the tcgen05 prefill path: one launch
 * computes T = X·A (written once as bf16) and Y = T·B, GEMM2's tiles
 * waiting for GEMM1's rows inside the launch.  Neither path pads r on the
 * host.  Prefill operands whose rows do not start on 32-byte boundaries
 * (for instance A with r not a multiple of 16) are first copied to a
 * 128-byte row pitch by the library.  That copy, and the loads of the
 * operands that need none, may begin before the previous kernel on `stream`
 * has finished (programmatic dependent launch) when, by the library's own
 * record, its last launch was a prefill launch with a CTA on every SM,
 * nothing else of the library was launched since, and none of its last
 * four outputs on the stream overlaps X, A or B.  The library sees only its
 * own launches: a kernel of the caller's, enqueued on `stream` between two
 * calls, is waited for in full unless it lets its dependents start early
 * (griddepcontrol.launch_dependents); a caller whose such kernels write X,
 * A or B of the next call turns the early copy off (lr_set_early_copy).
 * Results are deterministic except that split K (small prefill GEMMs, see
 * lr_set_split_k) adds fp32 partial sums in a run-dependent order.
 *
 * Precision of T on the prefill path: the tensor cores take bf16 operands,
 * so GEMM2 reads T either rounded once to bf16 or as two bf16 parts
 * hi = bf16(T), lo = bf16(T − hi) multiplied into the same fp32 accumulator
 * (about 16 significant bits of T; twice GEMM2's tensor work).  The automatic
 * choice takes the two parts whenever the extra tensor work (2·M·r·N FLOPs)
 * costs at most a third of the call's ideal time, max(2·M·r·(K+N) FLOPs at
 * 1.6 PFLOP/s, (MK+Kr+rN+MN)·2 bytes at 6.4 TB/s, 5 µs): small calls, and
 * bandwidth-bound ones such as small r at large M, K, N.
 * lr_set_t_precision overrides it.  The decode path keeps T in fp32.
 */
lr_status lr_linear(const void* X, const void* A, const void* B, const void* bias, void* Y,
                    int64_t M, int64_t K, int64_t r, int64_t N, void* stream);

/*
 * lr_linear_f32 — lr_linear with Y [M,N] written as fp32 (IEEE binary32):
 * the fp32 accumulator plus bias, without the final rounding to bf16 (Y
 * 4-byte aligned).  Same kernels, paths and T precision as lr_linear; the
 * bf16 result of lr_linear is this value rounded to nearest-even whenever
 * both calls add their partial sums in the same order (no split K).  The
 * accuracy the methods' pages state (bf16 inputs, fp32 accumulation) is a
 * property of this value: rounding Y to bf16 adds up to 2^-8·|Y| per
 * element on top of it.  Not available on the CTA-pair path (path 4:
 * LR_ERR_UNSUPPORTED).
 */
lr_status lr_linear_f32(const void* X, const void* A, const void* B, const void* bias, void* Y,
                        int64_t M, int64_t K, int64_t r, int64_t N, void* stream);

/*
 * lr_linear_strided — lr_linear on row-major operands with any row pitches
 * (elements): X [M,K] pitch ldx >= K, A [K,r] pitch lda >= r, B [r,N] pitch
 * ldb >= N, Y [M,N] pitch ldy >= N; Y is bf16 (y_f32 = 0) or fp32
 * (y_f32 != 0, as lr_linear_f32).  Same paths and results as lr_linear.
 *
 * A prefill operand whose base is 32-byte aligned and whose pitch is a
 * multiple of 16 elements is read in place; any other is first copied to an
 * aligned pitch on every call (for a factor with r = 1741, 14 MB per call).
 * A caller that keeps its factors in buffers of pitch lr_factor_pitch(cols)
 * (cudaMalloc bases are 256-byte aligned) pays that copy once, when it
 * stores them, instead of on every call: the "prepared weight" form of a
 * static factor.  Not this library's allocation: the caller owns those
 * buffers.
 */
lr_status lr_linear_strided(const void* X, int64_t ldx, const void* A, int64_t lda, const void* B,
                            int64_t ldb, const void* bias, void* Y, int64_t ldy, int64_t M,
                            int64_t K, int64_t r, int64_t N, int32_t y_f32, void* stream);

/*
 * lr_factor_pitch — the row pitch (elements) at which a stored factor with
 * `cols` columns is read in place by the prefill path: cols rounded up to a
 * multiple of 64 (128-byte rows).  -1 for cols < 0.
 */
int64_t lr_factor_pitch(int64_t cols);

/*
 * One projection of a group (a decoder layer's q/k/v/o/gate/up/down).
 * X [M,K] (entries may share one X pointer), A [K,r], B [r,N], bias [N] or
 * NULL, Y with row stride ld_y >= N (so two projections can write the two
 * halves of one packed [M, N1+N2] buffer, e.g. gate and up).  y_f32 = 0: Y
 * is bf16; nonzero: Y is fp32 as in lr_linear_f32 (4-byte aligned).
 */
typedef struct {
  const void* X;
  int64_t K;
  const void* A;
  const void* B;
  const void* bias;
  void* Y;
  int64_t ld_y;
  int64_t r;
  int64_t N;
  int32_t y_f32;
  /* 0: none.  j + 1: projection j of the same group is this one's gate, and
   * this projection's Y receives silu(G) * P instead of P, where P is its
   * own product (X·A·B + bias, fp32) and G the gate's Y as stored (bf16 or
   * fp32); silu(g) = g / (1 + e^-g).  The gated MLP's SiLU(gate) ⊙ up on the
   * way to the down projection.  The gate must have the same N and no gate
   * of its own. */
  int32_t silu_gate;
} lr_proj;

/*
 * lr_linear_group — every projection of `projs` (n_proj >= 0) on the same M,
 * in one call, on `stream`.  Each projection's result equals lr_linear on its
 * own arguments (bit for bit when split K is off; otherwise up to the order
 * of fp32 partial sums).  The Y ranges (rows × [0, N) at stride ld_y) of
 * different projections must not overlap each other or any input.
 * At M > 16 the group is one prefill launch when it fits the launch's tables
 * (at most 12 GEMMs: one per set of projections sharing X, plus one per
 * projection): projections with the same X pointer and K are one GEMM1 over
 * their A factors copied side by side.  At M <= 8 a group of at most 7
 * projections, each with K, r, N > 0, is one persistent launch: every SM
 * streams a slice of every projection's A, then of every B (rows of W
 * through shared memory into mma.sync; T in fp32, multiplied as bf16
 * hi + lo), each B block starting as soon as the blocks of T it needs are
 * summed; results equal lr_linear's up to fp32 rounding (another kernel).
 * Otherwise the projections run one by one.  FlashSVD v1.5's abstract describes the packed
 * execution of a layer's projections this mirrors (catalogue record of
 * arXiv 2605.08314).
 * silu_gate: at M <= 8 the product silu(G) * P is formed where the
 * streamed launch writes the up projection's blocks (each block waits,
 * bounded, for the same block of the gate); on the other paths P goes to a
 * library-owned fp32 buffer and one elementwise launch forms it.  Either
 * way P is not rounded before the product; the result is rounded once.
 * A projection with silu_gate, or one that is a gate, must not share Y
 * memory with the inputs of any projection (checked like every Y).
 */
lr_status lr_linear_group(const lr_proj* projs, int n_proj, int64_t M, void* stream);

/*
 * lr_linear_host — the same layer on HOST buffers: copies X, A, B and bias
 * to library-owned device buffers, runs lr_linear, copies Y back and
 * synchronises `stream`.  Pinned host memory gives asynchronous copies;
 * pageable memory works too.  Returns when Y (host) is written.
 */
lr_status lr_linear_host(const void* X, const void* A, const void* B, const void* bias, void* Y,
                         int64_t M, int64_t K, int64_t r, int64_t N, void* stream);

/*
 * lr_dense — Y = X·W + bias, W [K,N], with the same kernels (the dense layer
 * the factorisation replaces; the comparison the GAC paper's title asks
 * about: is the smaller layer still slower?).
 */
lr_status lr_dense(const void* X, const void* W, const void* bias, void* Y, int64_t M, int64_t K,
                   int64_t N, void* stream);

/*
 * lr_linear_decode_static — the decode path of lr_linear (M <= 16) for callers
 * that cannot let a library allocate device memory: a serving loop with a
 * hard latency budget (cudaMalloc/cudaFree synchronise the whole device), or
 * a host application whose own pool allocator owns all device memory.  The
 * paper has no counterpart to this entry point; it exists for such callers.
 *
 * Arguments and result are those of lr_linear (device pointers, bf16,
 * row-major; asynchronous on `stream`).  The caller still provides X, A, B,
 * bias and Y.  All scratch (partial sums, counters, T = X·A in fp32, about
 * 1.6 MB) is one fixed array compiled into the library, which every GPU that
 * loads the library holds until the process exits.  Never calls cudaMalloc,
 * cudaFree or any allocating library routine.
 *
 * Limits: M <= 16, r <= 4096, N <= 16384 (K < 2^31).  Larger sizes return
 * LR_ERR_UNSUPPORTED without launching anything.
 *
 * The first call on a device looks up the array's device address
 * (cudaGetSymbolAddress, with that device current); make that first call
 * before any stream capture.  Every call clears the parts of the array that
 * must start at zero.  All calls on a device share the array: calls whose
 * kernels overlap on the GPU (on different streams or host threads) race and
 * give wrong results; order them on one stream.
 */
lr_status lr_linear_decode_static(const void* X, const void* A, const void* B, const void* bias,
                                  void* Y, int64_t M, int64_t K, int64_t r, int64_t N,
                                  void* stream);

/*
 * lr_last_device_status — synchronises `stream`, then reports and clears the
 * device status word of the current device: LR_ERR_TIMEOUT if a bounded
 * device-side wait ran out since the last call, else LR_OK.  After a timeout
 * the kernels of later calls stop early until this is called.
 */
lr_status lr_last_device_status(void* stream);

/* Human-readable name of a status code (static string). */
const char* lr_status_string(lr_status s);

/* The last CUDA error code (cudaError_t as int) seen by this thread. */
int lr_last_cuda_error(void);

/*
 * lr_set_path — testing and benchmarking control of the dispatch:
 *   0 = automatic (M <= 16 decode, else prefill), 1 = force decode (M <= 16
 *   only; larger M returns LR_ERR_INVALID_ARG), 2 = force prefill, 3 = force
 *   prefill on single-SM tiles (the default prefill kernel), 4 = force prefill
 *   on CTA pairs (2-SM MMA, 256×256 tiles, GEMM1 and GEMM2 as two launches;
 *   M <= 128 still uses single SMs), 5 = force decode on the two-launch
 *   kernels, groups included (M <= 16 only), 6 = force decode, and for
 *   M <= 8 on the streamed one-launch kernel that decode-size groups use
 *   (M <= 16 only; see lr_linear_group).
 * lr_set_wait_limit_ns — time limit of every device-side bounded wait
 *   (default 2e9 ns); 0 restores the default.
 * lr_set_tile_n — column width of the prefill kernel's single-SM tiles:
 *   0 (the default) lets the library choose per GEMM (a schedule model picks
 *   the width that spreads the launch's tiles most evenly over the SMs);
 *   32..256 in steps of 32 forces that width for every GEMM (for tests and
 *   tuning).  Other values return LR_ERR_INVALID_ARG.
 * lr_set_split_k — on = 1 (the default): a prefill GEMM with fewer tiles
 *   than half the SMs and at least 16 k blocks of 64 (GEMM1 at small ranks)
 *   splits its K loop over several CTAs, which add fp32 partial sums into a
 *   workspace; the last one rounds and stores.  on = 0 turns it off (for
 *   tests and tuning).  Other values return LR_ERR_INVALID_ARG.
 * lr_set_early_copy — on = 1 (the default): a prefill call's realignment
 *   copy may overlap the library's previous prefill launch on the stream
 *   (conditions under lr_linear).  on = 0: every call's first copy waits
 *   for all earlier work on the stream, so a caller's kernel that starts
 *   its dependents early can safely write the next call's operands.  Other
 *   values return LR_ERR_INVALID_ARG.
 * lr_set_t_precision — how a prefill GEMM2 reads T: 0 = automatic (the
 *   default, see lr_linear), 1 = T rounded once to bf16, 2 = T as two bf16
 *   parts hi + lo.  Other values return LR_ERR_INVALID_ARG.
 * All six are process-wide and take effect on the next call.
 */
lr_status lr_set_path(int path);
lr_status lr_set_wait_limit_ns(int64_t ns);
lr_status lr_set_tile_n(int bn);
lr_status lr_set_split_k(int on);
lr_status lr_set_early_copy(int on);
lr_status lr_set_t_precision(int mode);

/*
 * lr_set_withhold_first_stage — testing failure detection only.  With on = 1,
 * the prefill kernels' copy thread never fills the first pipeline stage of
 * its first tile, so the tensor-core thread's bounded wait on it runs out:
 * the kernel records LR_ERR_TIMEOUT in the device status word, waits for its
 * own copies and MMAs, frees its tensor memory and returns (Y is then not
 * written).  Nothing faults or hangs.  on = 0 (the default) turns it off.
 */
lr_status lr_set_withhold_first_stage(int on);

/*
 * lr_gac_select — re-select the dimensions of n_items compressed weights
 * under a parameter budget, as GAC does ("Why Smaller Is Slower?
 * Dimensional Misalignment in Compressed LLMs", §4.3 Step 3: Constrained
 * Optimization, and its budget-quantization paragraph).  Host memory and
 * host code only; no GPU is needed.
 *
 * Weight i has n_cand[i] candidates (1..255; the aligned dimensions its
 * dimension sweep, §4.2, kept), candidate j storing cost[off_i + j]
 * parameters (off_i = n_cand[0] + … + n_cand[i-1]; 0 <= cost < 2^53), an
 * importance score[i] (finite) and base[i] = |W_i*| (0 <= base < 2^53), the
 * parameters at its unconstrained dimension.  The call picks one candidate
 * per weight to maximise  Σ_i score[i]·(cost_i,choice[i] − base[i])  subject
 * to  Σ_i ⌈cost_i,choice[i] / unit⌉ <= ⌊budget / unit⌋  (unit >= 1: the
 * quantum u of the budget, e.g. 8·(smallest cost of one dimension step)),
 * by the recurrence D[i][b] = max_j D[i−1][b − ⌈w_ij/u⌉] + v_ij with
 * D[0][b] = 0.  Rounding costs up and the budget down keeps the selection's
 * true parameter count within `budget`.  Among equally good candidates of a
 * weight at a given remaining budget the lowest index is taken, so the
 * result is deterministic.
 *
 * choice[n_items] receives the chosen candidate indices; *objective (may be
 * NULL) the maximised sum, accumulated over the weights in order.
 * Errors: LR_ERR_INVALID_ARG for null pointers, n_items < 1, counts, costs
 * or scores out of range, budget < 0 or unit < 1; LR_ERR_INFEASIBLE when
 * even the cheapest candidates exceed the quantized budget; LR_ERR_UNSUPPORTED
 * when the table (n_items × (⌊budget/unit⌋ + 1) bytes) would exceed 1 GiB;
 * LR_ERR_NO_MEMORY if host allocation fails.  choice is written only on
 * LR_OK.
 */
lr_status lr_gac_select(int n_items, const int* n_cand, const int64_t* cost, const double* score,
                        const int64_t* base, int64_t budget, int64_t unit, int* choice,
                        double* objective);

/* Counts the kernels launched by this library in this process. */
int64_t lr_kernel_launch_count(void);

/* Frees every workspace, staging buffer and decode piece table
 * (synchronises each stream the library used). */
lr_status lr_release_workspaces(void);

#ifdef __cplusplus
}
#endif

#endif /* LR_LINEAR_H */
