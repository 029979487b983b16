// lr_api.cu — the C ABI of include/lr_linear.h: argument validation, path
// selection, workspaces, TMA descriptors and status reporting.  Every step
// of the layer itself runs in the kernels of lr_decode.cu and lr_umma.cu.
#include <algorithm>
#include <atomic>
#include <cstdlib>
#include <cstring>
#include <map>
#include <mutex>
#include <set>
#include <tuple>
#include <vector>

#include <cudaTypedefs.h>

#include "../../include/lr_linear.h"
#include "lr_internal.h"

namespace lr {
namespace {

thread_local int g_last_cuda_error = 0;
std::atomic<int> g_path{0};
std::atomic<long long> g_wait_ns{0};
std::atomic<long long> g_launches{0};
std::atomic<int> g_withhold{0};
std::atomic<int> g_tile_n{0};
std::atomic<int> g_split_k{1};
std::atomic<int> g_early_copy{1};
std::atomic<int> g_t_precision{0};
constexpr long long kDefaultWaitNs = 2000000000LL;

struct DeviceInfo {
  int sms = 0;
  int major = 0;
  DevStatus* status = nullptr;
};

std::mutex g_mu;
std::map<int, DeviceInfo> g_dev;

struct Workspace {
  char* ptr = nullptr;
  size_t cap = 0;
  size_t zero_bytes = 0;  // prefix that is all-zero between calls
  // Row-block counters of the chain kernel: two banks of n_ctrs, used by
  // alternate launches.
  unsigned int* ctrs = nullptr;
  size_t n_ctrs = 0;
  unsigned int launches = 0;
  // Split-K partial sums of the chain kernel (fp32, zero at rest).
  float* split_ws = nullptr;
  size_t split_cap = 0;
  // The prefill path's realigned operands, in two areas used by alternate
  // calls (a call's repack may overlap the previous call's chain launch).
  char* rp_area[2] = {nullptr, nullptr};
  size_t rp_cap = 0;
  // fp32 products of gated group projections (paths that do not fuse the
  // gate's product).
  float* act = nullptr;
  size_t act_cap = 0;
};
std::map<std::pair<int, cudaStream_t>, Workspace> g_ws;

// What the library last launched on a stream: whether it was a prefill
// chain launch (whose output Y is known), and the parity that alternates the
// prefill path's two realignment areas between calls.
struct StreamState {
  bool last_chain = false;
  uintptr_t y_lo[4] = {0, 0, 0, 0}, y_hi[4] = {0, 0, 0, 0};  // last outputs written
  unsigned int n_out = 0;
  unsigned int parity = 0;
  long long launches_after = -1;  // library launch count right after that launch
  bool full_grid = false;         // that launch had a CTA on every SM
};
std::map<std::pair<int, cudaStream_t>, StreamState> g_streams;

void note_call(cudaStream_t stream, bool chain, const void* y, size_t ybytes,
               bool full_grid = false) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return;
  std::lock_guard<std::mutex> lk(g_mu);
  StreamState& st = g_streams[{dev, stream}];
  st.last_chain = chain;
  st.launches_after = chain ? g_launches.load() : -1;
  st.full_grid = chain && full_grid;
  const unsigned int i = (st.n_out++) & 3u;
  st.y_lo[i] = reinterpret_cast<uintptr_t>(y);
  st.y_hi[i] = st.y_lo[i] + ybytes;
}

struct Staging {
  char* ptr = nullptr;
  size_t cap = 0;
};
std::map<std::pair<int, cudaStream_t>, Staging> g_stage;

PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

struct MapKey {
  const void* ptr;
  uint64_t inner, outer, stride;
  uint32_t box_inner, box_outer;
  bool operator<(const MapKey& o) const {
    return std::tie(ptr, inner, outer, stride, box_inner, box_outer) <
           std::tie(o.ptr, o.inner, o.outer, o.stride, o.box_inner, o.box_outer);
  }
};
std::map<MapKey, CUtensorMap> g_maps;

lr_status cuda_fail(cudaError_t e) {
  g_last_cuda_error = static_cast<int>(e);
  if (e == cudaErrorMemoryAllocation) return LR_ERR_NO_MEMORY;
  return LR_ERR_CUDA;
}

#define LR_CUDA(call)                          \
  do {                                         \
    cudaError_t e_ = (call);                   \
    if (e_ != cudaSuccess) return cuda_fail(e_); \
  } while (0)

lr_status device_info(DeviceInfo** out, int* dev_out) {
  int dev = 0;
  LR_CUDA(cudaGetDevice(&dev));
  std::lock_guard<std::mutex> lk(g_mu);
  auto it = g_dev.find(dev);
  if (it == g_dev.end()) {
    DeviceInfo d;
    LR_CUDA(cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev));
    LR_CUDA(cudaDeviceGetAttribute(&d.major, cudaDevAttrComputeCapabilityMajor, dev));
    if (d.major != 10) return LR_ERR_UNSUPPORTED;
    LR_CUDA(cudaMalloc(&d.status, sizeof(DevStatus)));
    LR_CUDA(cudaMemset(d.status, 0, sizeof(DevStatus)));
    it = g_dev.emplace(dev, d).first;
  }
  *out = &it->second;
  *dev_out = dev;
  return LR_OK;
}

lr_status get_encoder() {
  std::lock_guard<std::mutex> lk(g_mu);
  if (g_encode) return LR_OK;
  void* fn = nullptr;
  cudaDriverEntryPointQueryResult q;
  LR_CUDA(cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q));
  if (q != cudaDriverEntryPointSuccess || fn == nullptr) return LR_ERR_UNSUPPORTED;
  g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  return LR_OK;
}

// 2-D bf16 tensor map, 128-byte swizzle, out-of-bounds elements read as zero.
lr_status tensor_map(CUtensorMap* out, const void* ptr, uint64_t inner, uint64_t outer,
                     uint64_t row_stride_elems, uint32_t box_inner, uint32_t box_outer) {
  lr_status st = get_encoder();
  if (st != LR_OK) return st;
  MapKey key{ptr, inner, outer, row_stride_elems, box_inner, box_outer};
  {
    std::lock_guard<std::mutex> lk(g_mu);
    auto it = g_maps.find(key);
    if (it != g_maps.end()) {
      *out = it->second;
      return LR_OK;
    }
  }
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {row_stride_elems * 2};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = g_encode(out, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims,
                        strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    g_last_cuda_error = static_cast<int>(r);
    return LR_ERR_CUDA;
  }
  std::lock_guard<std::mutex> lk(g_mu);
  if (g_maps.size() > 4096) g_maps.clear();
  g_maps.emplace(key, *out);
  return LR_OK;
}

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// A workspace whose first `zero_need` bytes are zero on entry (and must be
// left zero by the kernels) followed by `scratch_need` bytes of scratch.
lr_status workspace(cudaStream_t stream, size_t zero_need, size_t scratch_need, char** zero,
                    char** scratch) {
  int dev = 0;
  LR_CUDA(cudaGetDevice(&dev));
  std::lock_guard<std::mutex> lk(g_mu);
  Workspace& w = g_ws[{dev, stream}];
  zero_need = align_up(zero_need, 256);
  const size_t z = std::max(zero_need, w.zero_bytes);
  const size_t need = z + align_up(scratch_need, 256);
  if (need > w.cap) {
    if (w.ptr) {
      LR_CUDA(cudaStreamSynchronize(stream));
      LR_CUDA(cudaFree(w.ptr));
      w.ptr = nullptr;
      w.cap = 0;
    }
    const size_t cap = align_up(need + need / 4, 1 << 20);
    LR_CUDA(cudaMalloc(&w.ptr, cap));
    w.cap = cap;
    LR_CUDA(cudaMemsetAsync(w.ptr, 0, z, stream));
    w.zero_bytes = z;
  } else if (z > w.zero_bytes) {
    LR_CUDA(cudaMemsetAsync(w.ptr + w.zero_bytes, 0, z - w.zero_bytes, stream));
    w.zero_bytes = z;
  }
  *zero = w.ptr;
  *scratch = w.ptr + w.zero_bytes;
  return LR_OK;
}

bool ranges_overlap(const void* a, size_t abytes, const void* b, size_t bbytes) {
  if (!a || !b || abytes == 0 || bbytes == 0) return false;
  const uintptr_t a0 = reinterpret_cast<uintptr_t>(a), b0 = reinterpret_cast<uintptr_t>(b);
  return a0 < b0 + bbytes && b0 < a0 + abytes;
}

size_t span_bytes(int64_t rows, int64_t cols, int64_t ld) {
  if (rows <= 0 || cols <= 0) return 0;
  return static_cast<size_t>((rows - 1) * ld + cols) * 2;
}

constexpr int64_t kMaxDim = (int64_t(1) << 31) - 1;

bool aligned2(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 1u) == 0; }

WaitCtl wait_ctl(DeviceInfo* d) { return WaitCtl{d->status, wait_limit_ns()}; }

// Row pitches (elements) of X, A and B; contiguous unless a caller says so.
struct Pitch {
  int64_t x, a, b;
};

lr_status validate(const void* X, const void* A, const void* B, const void* bias, const void* Y,
                   int64_t M, int64_t K, int64_t r, int64_t N, int64_t ldy, bool y_f32 = false,
                   Pitch ld = Pitch{-1, -1, -1}) {
  if (M < 0 || K < 0 || r < 0 || N < 0) return LR_ERR_INVALID_ARG;
  if (M > kMaxDim || K > kMaxDim || r > kMaxDim || N > kMaxDim) return LR_ERR_UNSUPPORTED;
  if (ld.x < 0) ld = Pitch{K, r, N};
  if (ldy < N || ld.x < K || ld.a < r || ld.b < N) return LR_ERR_INVALID_ARG;
  if (ldy > kMaxDim || ld.x > kMaxDim || ld.a > kMaxDim || ld.b > kMaxDim) return LR_ERR_UNSUPPORTED;
  if (M > 0 && N > 0 && !Y) return LR_ERR_INVALID_ARG;
  if (M > 0 && K > 0 && r > 0 && N > 0 && (!X || !A || !B)) return LR_ERR_INVALID_ARG;
  for (const void* p : {X, A, B, bias, Y})
    if (p && !aligned2(p)) return LR_ERR_INVALID_ARG;
  if (y_f32 && Y && (reinterpret_cast<uintptr_t>(Y) & 3u) != 0) return LR_ERR_INVALID_ARG;
  const size_t ybytes = span_bytes(M, N, ldy) * (y_f32 ? 2 : 1);
  if (ranges_overlap(Y, ybytes, X, span_bytes(M, K, ld.x)) ||
      ranges_overlap(Y, ybytes, A, span_bytes(K, r, ld.a)) ||
      ranges_overlap(Y, ybytes, B, span_bytes(r, N, ld.b)) ||
      ranges_overlap(Y, ybytes, bias, span_bytes(1, N, N)))
    return LR_ERR_INVALID_ARG;
  return LR_OK;
}

lr_status launched(cudaError_t e, int n = 1) {
  if (e != cudaSuccess) return cuda_fail(e);
  g_launches += n;
  return LR_OK;
}

// out = V · W (+bias) for M <= 16 tokens through one skinny launch.
lr_status skinny(DeviceInfo* d, cudaStream_t stream, int M, const void* V, int64_t ldv, bool v_f32,
                 const void* W, int64_t Kd, int64_t Nd, float* acc, unsigned int* counters,
                 float* out_f32, int64_t ld_out_f32, void* out_bf16, int64_t ld_out,
                 const void* bias, bool dependent = false, int64_t ldw = -1) {
  if (ldw < 0) ldw = Nd;
  const SkinnyPlan plan = plan_skinny(M, Kd, Nd, d->sms);
  SkinnyArgs a{};
  a.M = M;
  a.Kd = Kd;
  a.Nd = Nd;
  a.V = V;
  a.ldv = ldv;
  a.v_f32 = v_f32 ? 1 : 0;
  a.W = static_cast<const __nv_bfloat16*>(W);
  a.ldw = ldw;
  a.w_lo = reinterpret_cast<uintptr_t>(W);
  a.w_hi = a.w_lo + static_cast<uintptr_t>(span_bytes(Kd, Nd, ldw));
  a.acc = acc;
  a.ld_acc = static_cast<int64_t>(align_up(static_cast<size_t>(Nd), 4));
  a.counters = counters;
  a.out_f32 = out_f32;
  a.ld_out_f32 = ld_out_f32;
  a.out_bf16 = static_cast<__nv_bfloat16*>(out_bf16);
  a.ld_out = ld_out;
  a.bias = static_cast<const __nv_bfloat16*>(bias);
  a.wait = wait_ctl(d);
  return launched(launch_skinny(plan, a, stream, dependent));
}

size_t acc_bytes(int M, int64_t n) { return align_up(static_cast<size_t>(M) * align_up(n, 4) * 4, 256); }
size_t ctr_bytes(int M, int64_t Kd, int64_t n, int sms) {
  const SkinnyPlan p = plan_skinny(M, Kd, n, sms);
  return align_up(static_cast<size_t>(p.col_blocks) * 4, 256);
}

int64_t ceil_div(int64_t a, int64_t b);

// One decode-size pair of jobs (T = X·A, then Y = T·B + bias) of the
// streamed kernel, appended to `a`; its workspace areas are carved from
// `zero` (zero at rest) and `scratch`, and its flags from `flags`.
struct StreamPair {
  const void *X, *A, *B, *bias;
  void* Y;
  int64_t K, r, N, ldy;
  bool y_f32;
  Pitch ld;
  int gate = -1;  // index (in the same array) of the pair gating this one's output
};

size_t stream_pair_zero(int M, const StreamPair& p) {
  const int64_t n0 = ceil_div(p.r, stream_block_cols(p.r)), n1 = ceil_div(p.N, stream_block_cols(p.N));
  return align_up(static_cast<size_t>(M) * align_up(static_cast<size_t>(p.r), 8) * 4, 256) +
         align_up(static_cast<size_t>(M) * align_up(static_cast<size_t>(p.N), 8) * 4, 256) +
         align_up(static_cast<size_t>(2 * n0 + 2 * n1) * 4, 256);
}
size_t stream_pair_scratch(int M, const StreamPair& p) {
  return align_up(static_cast<size_t>(M) * align_up(static_cast<size_t>(p.r), 8) * 4, 256);
}
void stream_add_pair(StreamArgs& a, const StreamPair& p, char** zero, char** scratch) {
  const int M = a.M;
  const int64_t ldt = static_cast<int64_t>(align_up(static_cast<size_t>(p.r), 8));
  const int64_t ldn = static_cast<int64_t>(align_up(static_cast<size_t>(p.N), 8));
  float* acc0 = reinterpret_cast<float*>(*zero);
  *zero += align_up(static_cast<size_t>(M) * ldt * 4, 256);
  float* acc1 = reinterpret_cast<float*>(*zero);
  *zero += align_up(static_cast<size_t>(M) * ldn * 4, 256);
  const int cb0 = stream_block_cols(p.r), cb1 = stream_block_cols(p.N);
  const int64_t nb0 = ceil_div(p.r, cb0), nb1 = ceil_div(p.N, cb1);
  unsigned int* cnt = reinterpret_cast<unsigned int*>(*zero);
  unsigned int* ready = cnt + nb0 + nb1;
  unsigned int* fin = ready + nb0;
  *zero += align_up(static_cast<size_t>(2 * nb0 + 2 * nb1) * 4, 256);
  float* T = reinterpret_cast<float*>(*scratch);
  *scratch += align_up(static_cast<size_t>(M) * ldt * 4, 256);

  StreamJob& j0 = a.job[a.n_jobs];
  j0 = StreamJob{};
  j0.W = static_cast<const __nv_bfloat16*>(p.A);
  j0.ldw = p.ld.a;
  j0.w_lo = reinterpret_cast<uintptr_t>(p.A);
  j0.w_hi = j0.w_lo + span_bytes(p.K, p.r, p.ld.a);
  j0.K = static_cast<int>(p.K);
  j0.N = static_cast<int>(p.r);
  j0.cb = cb0;
  j0.phase = 0;
  j0.V = p.X;
  j0.ldv = p.ld.x;
  j0.src = -1;
  j0.acc = acc0;
  j0.ld_acc = ldt;
  j0.cnt = cnt;
  j0.ready = ready;
  j0.out_f32 = T;
  j0.ld_out = ldt;
  j0.unit0 = a.units[0];
  a.units[0] += p.K * p.r;
  const int src = a.n_jobs++;

  StreamJob& j1 = a.job[a.n_jobs++];
  j1 = StreamJob{};
  j1.W = static_cast<const __nv_bfloat16*>(p.B);
  j1.ldw = p.ld.b;
  j1.w_lo = reinterpret_cast<uintptr_t>(p.B);
  j1.w_hi = j1.w_lo + span_bytes(p.r, p.N, p.ld.b);
  j1.K = static_cast<int>(p.r);
  j1.N = static_cast<int>(p.N);
  j1.cb = cb1;
  j1.phase = 1;
  j1.V = T;
  j1.ldv = ldt;
  j1.src = src;
  j1.acc = acc1;
  j1.ld_acc = ldn;
  j1.cnt = cnt + nb0;
  j1.ready = nullptr;
  if (p.y_f32)
    j1.out_f32 = static_cast<float*>(p.Y);
  else
    j1.out_bf16 = static_cast<__nv_bfloat16*>(p.Y);
  j1.ld_out = p.ldy;
  j1.bias = static_cast<const __nv_bfloat16*>(p.bias);
  j1.unit0 = a.units[1];
  j1.fin = fin;
  a.units[1] += p.r * p.N;
  a.n_final += static_cast<int>(nb1);
}

// Every CTA's pieces for a set of job shapes, computed once on the host and
// kept on the device (a few KB per set of shapes; the kernel reads its own
// instead of computing them, which took its threads microseconds).  Kept
// until lr_release_workspaces; a decode loop uses a handful of shapes.
struct PieceTable {
  StreamSeg* pieces = nullptr;
  int* off = nullptr;
};
std::mutex g_piece_mu;
std::map<std::vector<int64_t>, PieceTable> g_piece_tables;
constexpr size_t kMaxPieceTables = 1024;

// Attach the piece table of `a` (grid CTAs) to it: LR_OK, or
// LR_ERR_UNSUPPORTED when a CTA's pieces exceed the kernel's list.
lr_status stream_pieces(StreamArgs& a, int grid) {
  int dev = 0;
  LR_CUDA(cudaGetDevice(&dev));
  std::vector<int64_t> key{dev, grid, a.n_jobs};
  for (int j = 0; j < a.n_jobs; ++j)
    key.insert(key.end(), {a.job[j].phase, a.job[j].K, a.job[j].N, a.job[j].cb});
  std::lock_guard<std::mutex> lk(g_piece_mu);
  auto it = g_piece_tables.find(key);
  if (it == g_piece_tables.end()) {
    std::vector<StreamSeg> all;
    std::vector<int> off(static_cast<size_t>(grid) + 1, 0);
    StreamSeg tmp[2 * kStreamMaxSegs];
    for (int g = 0; g < grid; ++g) {
      const int n = stream_segments(a, g, grid, tmp, 2 * kStreamMaxSegs);
      if (n > 2 * kStreamMaxSegs) return LR_ERR_UNSUPPORTED;
      all.insert(all.end(), tmp, tmp + n);
      off[g + 1] = static_cast<int>(all.size());
    }
    if (g_piece_tables.size() >= kMaxPieceTables) {
      // Too many shapes to keep: the CTAs compute their pieces themselves.
      if (!std::all_of(off.begin() + 1, off.end(), [&, prev = 0](int o) mutable {
            const bool ok = o - prev <= kStreamMaxSegs;
            prev = o;
            return ok;
          }))
        return LR_ERR_UNSUPPORTED;
      a.pieces = nullptr;
      a.piece_off = nullptr;
      return LR_OK;
    }
    PieceTable t;
    LR_CUDA(cudaMalloc(&t.pieces, std::max<size_t>(all.size(), 1) * sizeof(StreamSeg)));
    LR_CUDA(cudaMalloc(&t.off, off.size() * sizeof(int)));
    LR_CUDA(cudaMemcpy(t.pieces, all.data(), all.size() * sizeof(StreamSeg), cudaMemcpyHostToDevice));
    LR_CUDA(cudaMemcpy(t.off, off.data(), off.size() * sizeof(int), cudaMemcpyHostToDevice));
    it = g_piece_tables.emplace(key, t).first;
  }
  a.pieces = it->second.pieces;
  a.piece_off = it->second.off;
  return LR_OK;
}

// Decode-size pairs on the streamed kernel (M <= 8): one launch.
lr_status run_stream(DeviceInfo* d, cudaStream_t stream, int M, const StreamPair* pairs, int n) {
  size_t zneed = 256, sneed = 0;
  for (int i = 0; i < n; ++i) {
    zneed += stream_pair_zero(M, pairs[i]);
    sneed += stream_pair_scratch(M, pairs[i]);
  }
  char *zero = nullptr, *scratch = nullptr;
  lr_status st = workspace(stream, zneed, sneed, &zero, &scratch);
  if (st != LR_OK) return st;
  StreamArgs a{};
  a.M = M;
  a.done = reinterpret_cast<unsigned int*>(zero);
  zero += 256;
  // Gates first: a CTA's phase-1 pieces run in job order, so a gated block
  // never waits for a gate block that the same CTA has yet to stream.
  std::vector<int> order, job1(static_cast<size_t>(n), -1);
  for (int i = 0; i < n; ++i)
    if (pairs[i].gate < 0) order.push_back(i);
  for (int i = 0; i < n; ++i)
    if (pairs[i].gate >= 0) order.push_back(i);
  for (int i : order) {
    stream_add_pair(a, pairs[i], &zero, &scratch);
    job1[static_cast<size_t>(i)] = a.n_jobs - 1;
  }
  for (int i = 0; i < n; ++i) {
    const int g = pairs[i].gate;
    if (g < 0) continue;
    StreamJob& J = a.job[job1[static_cast<size_t>(i)]];
    const StreamJob& Gj = a.job[job1[static_cast<size_t>(g)]];
    J.gate_y = pairs[g].Y;
    J.gate_ld = pairs[g].ldy;
    J.gate_f32 = pairs[g].y_f32 ? 1 : 0;
    J.gate_fin = Gj.fin;
  }
  a.w_early = 1;
  a.wait = wait_ctl(d);
  st = stream_pieces(a, d->sms);
  if (st != LR_OK) return st;
  return launched(launch_stream(a, d->sms, stream, false));
}

// A single decode call takes the two-launch skinny kernels, or with path 6
// (M <= 8) the streamed one-launch kernel.  (Measured on B200 at the
// Llama-3-8B MLP shapes, M = 1: 32 µs two-launch, 59 µs streamed; the
// streamed kernel pays ~5 µs at each piece boundary and waits for the
// slowest CTA's phase 0.  It is the decode group's kernel, where one launch
// replaces fourteen.)
bool use_stream(int64_t M) { return g_path.load() == 6 && M <= 8; }

lr_status run_decode(DeviceInfo* d, cudaStream_t stream, const void* X, const void* A,
                     const void* B, const void* bias, void* Y, int64_t M, int64_t K, int64_t r,
                     int64_t N, int64_t ldy, bool y_f32, Pitch ld) {
  const int m = static_cast<int>(M);
  if (use_stream(M)) {
    const StreamPair p{X, A, B, bias, Y, K, r, N, ldy, y_f32, ld};
    lr_status st = run_stream(d, stream, m, &p, 1);
    if (st != LR_ERR_UNSUPPORTED) return st;
  }
  const size_t acc1 = acc_bytes(m, r), acc2 = acc_bytes(m, N);
  const size_t c1 = ctr_bytes(m, K, r, d->sms), c2 = ctr_bytes(m, r, N, d->sms);
  const int64_t ldt = static_cast<int64_t>(align_up(static_cast<size_t>(r), 4));
  char *zero = nullptr, *scratch = nullptr;
  lr_status st = workspace(stream, acc1 + acc2 + c1 + c2, static_cast<size_t>(M) * ldt * 4, &zero,
                           &scratch);
  if (st != LR_OK) return st;
  float* a1 = reinterpret_cast<float*>(zero);
  float* a2 = reinterpret_cast<float*>(zero + acc1);
  unsigned int* k1 = reinterpret_cast<unsigned int*>(zero + acc1 + acc2);
  unsigned int* k2 = reinterpret_cast<unsigned int*>(zero + acc1 + acc2 + c1);
  float* T = reinterpret_cast<float*>(scratch);
  // Phase 1: T = X·A (fp32).  Phase 2: Y = T·B + bias.
  st = skinny(d, stream, m, X, ld.x, false, A, K, r, a1, k1, T, ldt, nullptr, 0, nullptr, false,
              ld.a);
  if (st != LR_OK) return st;
  // Phase 2 starts streaming B while phase 1 finishes (programmatic
  // dependent launch); it reads T only after phase 1 has completed.
  if (y_f32)
    return skinny(d, stream, m, T, ldt, true, B, r, N, a2, k2, static_cast<float*>(Y), ldy,
                  nullptr, 0, bias, true, ld.b);
  return skinny(d, stream, m, T, ldt, true, B, r, N, a2, k2, nullptr, 0, Y, ldy, bias, true, ld.b);
}

// Row pitch (elements) of the buffers the library lays out itself (T and
// realigned copies): 128-byte rows.  Rows that are 16- but not 32-byte
// aligned make every 128-byte TMA box row touch five 32-byte sectors instead
// of four (measured: r = 1025..1032 and 1089..1096 at M = K = N = 4096 ran
// 12-20% slower than their 32-byte-aligned neighbours).
constexpr int64_t kPitchElems = 64;

// An operand is read in place when its rows start on 32-byte boundaries
// (TMA itself needs 16); rows that are only 16-byte aligned are realigned
// like misaligned ones, which costs one copy (overlapped with the previous
// launch in back-to-back calls) and saves a fifth of the L2 sectors of every
// tile load (measured: M = K = N = 4096 at r = 1000, 1032, 1064, 1096 ran
// 4-8% faster).
bool tma_ok(const void* p, int64_t ld) {
  return (reinterpret_cast<uintptr_t>(p) % 32 == 0) && (ld % 16 == 0);
}

// Counter banks for one chain launch on `stream`: the launch's bank (zero)
// and the other one (which the launch zeroes for the next).
lr_status chain_counters(cudaStream_t stream, size_t n, unsigned int** bank,
                         unsigned int** next, int* per_bank) {
  int dev = 0;
  LR_CUDA(cudaGetDevice(&dev));
  std::lock_guard<std::mutex> lk(g_mu);
  Workspace& w = g_ws[{dev, stream}];
  if (n > w.n_ctrs) {
    if (w.ctrs) {
      LR_CUDA(cudaStreamSynchronize(stream));
      LR_CUDA(cudaFree(w.ctrs));
      w.ctrs = nullptr;
      w.n_ctrs = 0;
    }
    const size_t cap = align_up(std::max<size_t>(n, 1024), 1024);
    LR_CUDA(cudaMalloc(&w.ctrs, 2 * cap * sizeof(unsigned int)));
    LR_CUDA(cudaMemsetAsync(w.ctrs, 0, 2 * cap * sizeof(unsigned int), stream));
    w.n_ctrs = cap;
  }
  const unsigned int b = (w.launches++) & 1u;
  *bank = w.ctrs + b * w.n_ctrs;
  *next = w.ctrs + (1u - b) * w.n_ctrs;
  *per_bank = static_cast<int>(w.n_ctrs);
  return LR_OK;
}

// fp32 split-K workspace of `bytes` on `stream`, zero at rest.
lr_status chain_split_ws(cudaStream_t stream, size_t bytes, float** out) {
  int dev = 0;
  LR_CUDA(cudaGetDevice(&dev));
  std::lock_guard<std::mutex> lk(g_mu);
  Workspace& w = g_ws[{dev, stream}];
  if (bytes > w.split_cap) {
    if (w.split_ws) {
      LR_CUDA(cudaStreamSynchronize(stream));
      LR_CUDA(cudaFree(w.split_ws));
      w.split_ws = nullptr;
      w.split_cap = 0;
    }
    const size_t cap = align_up(bytes + bytes / 4, 1 << 20);
    LR_CUDA(cudaMalloc(&w.split_ws, cap));
    LR_CUDA(cudaMemsetAsync(w.split_ws, 0, cap, stream));
    w.split_cap = cap;
  }
  *out = w.split_ws;
  return LR_OK;
}

// The realignment area of this prefill call on `stream` (`bytes` each, the
// two areas alternating between calls), and whether the call's first repack
// may read its sources while the previous launch on the stream still runs:
// only if that launch is the library's own prefill chain launch with a CTA
// on every SM (so that when all of its CTAs have started — which is when the
// copy may start — every CTA of the launch before it, which may still read
// the other area, has left), and none of the last four outputs the library
// wrote on the stream overlaps `srcs`, and the early copy is on
// (lr_set_early_copy).
lr_status repack_area(cudaStream_t stream, size_t bytes,
                      std::initializer_list<std::pair<const void*, size_t>> srcs, char** area,
                      bool* early) {
  int dev = 0;
  LR_CUDA(cudaGetDevice(&dev));
  std::lock_guard<std::mutex> lk(g_mu);
  Workspace& w = g_ws[{dev, stream}];
  StreamState& ss = g_streams[{dev, stream}];
  if (bytes > w.rp_cap) {
    LR_CUDA(cudaStreamSynchronize(stream));
    for (char*& a : w.rp_area) {
      if (a) LR_CUDA(cudaFree(a));
      a = nullptr;
    }
    w.rp_cap = 0;
    const size_t cap = align_up(bytes + bytes / 4, 1 << 20);
    for (char*& a : w.rp_area) LR_CUDA(cudaMalloc(&a, cap));
    w.rp_cap = cap;
  }
  *area = w.rp_area[ss.parity & 1u];
  ss.parity ^= 1u;
  // ... and nothing else the library counts was launched since (any stream).
  bool ok = g_early_copy.load() != 0 && ss.last_chain && ss.full_grid &&
            ss.launches_after == g_launches.load();
  for (const auto& sr : srcs) {
    const uintptr_t lo = reinterpret_cast<uintptr_t>(sr.first), hi = lo + sr.second;
    for (int i = 0; i < 4; ++i)
      if (sr.second && lo < ss.y_hi[i] && ss.y_lo[i] < hi) ok = false;
  }
  *early = ok;
  return LR_OK;
}

// One launch of the chain kernel under construction.
struct ChainBuild {
  ChainMaps maps{};
  ChainArgs args{};
  int n_maps = 0;
};

// Tensor map for operand a (K-major, box 64 × 128 rows) or operand b
// (MN-major, box 64 columns × 64 rows) of the chain kernel.
lr_status chain_map(ChainBuild& cb, const void* p, int64_t inner, int64_t outer, int64_t ld,
                    bool operand_a, int* idx) {
  if (cb.n_maps >= kChainMaxMaps) return LR_ERR_UNSUPPORTED;
  lr_status st = tensor_map(&cb.maps.m[cb.n_maps], p, static_cast<uint64_t>(inner),
                            static_cast<uint64_t>(outer), static_cast<uint64_t>(ld), 64,
                            operand_a ? kGemmBM : kGemmBK);
  if (st != LR_OK) return st;
  *idx = cb.n_maps++;
  return LR_OK;
}

lr_status chain_problem(ChainBuild& cb, int map_a, int a_col0, int map_b, int64_t Mr, int64_t Nc,
                        int64_t Kc, void* c, int64_t ldc, const void* bias, int wait_group,
                        int signal_group, bool dep_a, bool dep_b, int b_col0 = 0) {
  if (cb.args.n_prob >= kChainMaxProbs) return LR_ERR_UNSUPPORTED;
  ChainProblem& P = cb.args.p[cb.args.n_prob++];
  P = ChainProblem{};
  P.Mr = static_cast<int>(Mr);
  P.Nc = static_cast<int>(Nc);
  P.Kc = static_cast<int>(Kc);
  P.map_a = map_a;
  P.map_b = map_b;
  P.map_a_lo = -1;
  P.a_col0 = a_col0;
  P.c = static_cast<__nv_bfloat16*>(c);
  P.ldc = ldc;
  P.bias = static_cast<const __nv_bfloat16*>(bias);
  P.wait_group = wait_group;
  P.signal_group = signal_group;
  P.dep_a = dep_a ? 1 : 0;
  P.dep_b = dep_b ? 1 : 0;
  P.b_col0 = b_col0;
  return LR_OK;
}

// ---- tile-width planning
// Estimated time of one 64-deep k block of a 128 × bn tile.  Measured on
// B200 (dense 4096³ at each width): 0.38 µs at bn = 64 rising to 0.44 µs at
// bn = 256 — the copy pipeline, not the tensor core, sets the pace, so
// narrow tiles buy little time per tile.
double kblock_us(int bn) { return 0.37 + 0.07 * bn / 256.0; }
double epilogue_us(int bn) { return 0.6 + 1.0 * bn / 256.0; }

int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

// K splits of a GEMM with `tiles` output tiles and `nkb` k blocks: a GEMM
// with too few tiles to fill half the SMs and a long K loop (GEMM1 at small
// ranks) splits K, up to one split per 8 k blocks, as many as fill the SMs.
// Returns the k blocks per split; *splits receives the split count.
int split_plan(int64_t tiles, int nkb, int sms, int* splits) {
  int s = 1;
  if (g_split_k.load() && tiles * 2 <= sms && nkb >= 16)
    s = static_cast<int>(std::max<int64_t>(1, std::min<int64_t>({nkb / 8, sms / tiles, 16})));
  const int per = static_cast<int>(ceil_div(nkb, s));
  *splits = static_cast<int>(ceil_div(nkb, per));
  return per;
}

// Simulate the static round-robin schedule of the chain kernel.
// A k block of a problem whose operand a has two parts issues twice the
// tensor-core work of its tile width.  The splits of a split tile are
// consecutive items; each adds fp32 partial sums to the workspace (costed
// as two epilogues of its width) and the tile is done one epilogue after
// its last split.
double kblock_cost(const ChainProblem& P, int bn) {
  return kblock_us(P.map_a_lo >= 0 ? 2 * bn : bn);
}

double simulate_chain(const ChainArgs& a, const std::vector<int>& bn, int sms) {
  int64_t total = 0;
  std::vector<int> splits(static_cast<size_t>(a.n_prob)), per(static_cast<size_t>(a.n_prob));
  for (int i = 0; i < a.n_prob; ++i) {
    const int64_t tiles = ceil_div(a.p[i].Mr, kGemmBM) * ceil_div(a.p[i].Nc, bn[i]);
    per[i] = split_plan(tiles, static_cast<int>(ceil_div(a.p[i].Kc, kGemmBK)), sms, &splits[i]);
    total += tiles * splits[i];
  }
  const int64_t G = std::max<int64_t>(1, std::min<int64_t>(total, sms));
  std::vector<double> t(static_cast<size_t>(G), 0.0);
  std::map<int, std::vector<double>> ready;
  int64_t idx = 0;
  double tail = 0.0;
  for (int i = 0; i < a.n_prob; ++i) {
    const ChainProblem& P = a.p[i];
    const int64_t tm = ceil_div(P.Mr, kGemmBM), tn = ceil_div(P.Nc, bn[i]);
    const int nkb = static_cast<int>(ceil_div(P.Kc, kGemmBK));
    const double epi = epilogue_us(bn[i]);
    std::vector<double>* sig = nullptr;
    const std::vector<double>* wait = nullptr;
    if (P.signal_group >= 0) {
      sig = &ready[P.signal_group];
      sig->assign(static_cast<size_t>(tm), 0.0);
    }
    if (P.wait_group >= 0) {
      auto it = ready.find(P.wait_group);
      if (it != ready.end()) wait = &it->second;
    }
    for (int64_t l = 0; l < tm * tn; ++l) {
      const int64_t m = l / tn;
      double done = 0.0;
      for (int s = 0; s < splits[i]; ++s, ++idx) {
        double& tc = t[static_cast<size_t>(idx % G)];
        double start = tc;
        if (wait && m < static_cast<int64_t>(wait->size())) start = std::max(start, (*wait)[m]);
        const int kb = std::min(per[i], nkb - s * per[i]);
        tc = start + kb * kblock_cost(P, bn[i]) + 0.15 + (splits[i] > 1 ? 2.0 * epi : 0.0);
        done = std::max(done, tc);
      }
      if (sig) (*sig)[m] = std::max((*sig)[m], done + epi);
    }
    tail = epi;
  }
  return *std::max_element(t.begin(), t.end()) + tail;
}

std::mutex g_plan_mu;
std::map<std::vector<int64_t>, std::vector<int>> g_plans;

// Choose each problem's tile width.  Candidates are the multiples of 32 up
// to min(256, N rounded up to 32); two problems are searched jointly, more
// by coordinate descent from the widest tiles.
std::vector<int> plan_chain(const ChainArgs& a, int sms) {
  const int forced = g_tile_n.load();
  std::vector<int64_t> key{sms, forced, g_split_k.load()};
  for (int i = 0; i < a.n_prob; ++i) {
    const ChainProblem& P = a.p[i];
    key.insert(key.end(), {P.Mr, P.Nc, P.Kc, P.wait_group, P.signal_group, P.map_a_lo >= 0});
  }
  {
    std::lock_guard<std::mutex> lk(g_plan_mu);
    auto it = g_plans.find(key);
    if (it != g_plans.end()) return it->second;
  }
  // Two-part operand a: both parts and the b tile share a stage (bn <= 128).
  auto cap = [&](int i) { return a.p[i].map_a_lo >= 0 ? 128 : 256; };
  std::vector<int> bn(static_cast<size_t>(a.n_prob), 256);
  if (forced > 0) {
    for (int i = 0; i < a.n_prob; ++i) bn[i] = std::min(forced, cap(i));
  } else {
    std::vector<std::vector<int>> cand(static_cast<size_t>(a.n_prob));
    for (int i = 0; i < a.n_prob; ++i) {
      const int top = static_cast<int>(std::min<int64_t>(cap(i), ceil_div(a.p[i].Nc, 32) * 32));
      for (int b = top; b >= 32; b -= 32) cand[i].push_back(b);
      bn[i] = top;
    }
    double best = simulate_chain(a, bn, sms);
    if (a.n_prob == 2) {
      for (int b0 : cand[0])
        for (int b1 : cand[1]) {
          std::vector<int> tryb{b0, b1};
          const double t = simulate_chain(a, tryb, sms);
          if (t < best * 0.999) {
            best = t;
            bn = tryb;
          }
        }
    } else {
      for (int pass = 0; pass < 2; ++pass)
        for (int i = 0; i < a.n_prob; ++i)
          for (int b : cand[i]) {
            std::vector<int> tryb = bn;
            tryb[i] = b;
            const double t = simulate_chain(a, tryb, sms);
            if (t < best * 0.999) {
              best = t;
              bn = tryb;
            }
          }
    }
  }
  std::lock_guard<std::mutex> lk(g_plan_mu);
  if (g_plans.size() > 4096) g_plans.clear();
  g_plans.emplace(key, bn);
  return bn;
}

// Plan, number the tiles and launch.  The launch may start while the
// previous kernel on the stream still runs (programmatic dependent launch);
// the problems' dep_a / dep_b say which operands that kernel may write.
lr_status run_chain(DeviceInfo* d, cudaStream_t stream, ChainBuild& cb) {
  ChainArgs& a = cb.args;
  if (a.n_prob == 0) return LR_OK;
  const std::vector<int> bn = plan_chain(a, d->sms);
  int64_t total = 0;
  int groups = 0, stride = 1;
  for (int i = 0; i < a.n_prob; ++i) {
    ChainProblem& P = a.p[i];
    if (P.signal_group >= 0) groups = std::max(groups, P.signal_group + 1);
  }
  // K splits: split_plan.
  int64_t split_floats = 0;
  for (int i = 0; i < a.n_prob; ++i) {
    ChainProblem& P = a.p[i];
    P.bn = bn[i];
    P.tiles_m = static_cast<int>(ceil_div(P.Mr, kGemmBM));
    P.tiles_n = static_cast<int>(ceil_div(P.Nc, P.bn));
    const int64_t tiles = static_cast<int64_t>(P.tiles_m) * P.tiles_n;
    P.kb_per_split =
        split_plan(tiles, static_cast<int>(ceil_div(P.Kc, kGemmBK)), d->sms, &P.splits);
    P.split_group = -1;
    if (P.splits > 1) {
      P.split_group = groups++;
      stride = static_cast<int>(std::max<int64_t>(stride, tiles * kChainEpiWarps));
      P.ws_ld = static_cast<int64_t>(P.tiles_n) * P.bn;
      split_floats += static_cast<int64_t>(P.tiles_m) * kGemmBM * P.ws_ld;
    }
    P.tile_begin = static_cast<int>(total);
    total += tiles * P.splits;
    if (total > kMaxDim) return LR_ERR_UNSUPPORTED;
    if (P.signal_group >= 0) stride = std::max(stride, P.tiles_m);
  }
  if (split_floats > 0) {
    float* ws = nullptr;
    lr_status st = chain_split_ws(stream, static_cast<size_t>(split_floats) * 4, &ws);
    if (st != LR_OK) return st;
    for (int i = 0; i < a.n_prob; ++i) {
      ChainProblem& P = a.p[i];
      if (P.splits > 1) {
        P.ws = ws;
        ws += static_cast<int64_t>(P.tiles_m) * kGemmBM * P.ws_ld;
      }
    }
  }
  for (int i = 0; i < a.n_prob; ++i) {
    ChainProblem& P = a.p[i];
    if (P.wait_group < 0) continue;
    P.wait_count = 0;
    for (int j = 0; j < i; ++j)
      if (a.p[j].signal_group == P.wait_group) P.wait_count += kChainEpiWarps * a.p[j].tiles_n;
  }
  a.total_tiles = static_cast<int>(total);
  if (total == 0) return LR_OK;
  a.ctr_stride = stride;
  lr_status st = chain_counters(stream, static_cast<size_t>(std::max(groups, 1)) * stride,
                                &a.counters, &a.counters_next, &a.n_counters);
  if (st != LR_OK) return st;
  a.wait = wait_ctl(d);
  a.pdl = 1;
  a.withhold_first_stage = g_withhold.load();
  const int grid = static_cast<int>(std::min<int64_t>(total, d->sms));
  bool two = false;
  for (int i = 0; i < a.n_prob; ++i) two = two || a.p[i].map_a_lo >= 0;
  return launched(launch_chain(cb.maps, a, grid, two, stream));
}

// One GEMM on CTA pairs (path 4): C = a · b (+bias).
lr_status gemm_pair(DeviceInfo* d, cudaStream_t stream, const void* a, int64_t lda, const void* b,
                    int64_t ldb, void* c, int64_t ldc, const void* bias, int64_t Mr, int64_t Nc,
                    int64_t Kc) {
  GemmArgs g{};
  g.Mr = static_cast<int>(Mr);
  g.Nc = static_cast<int>(Nc);
  g.Kc = static_cast<int>(Kc);
  g.c = static_cast<__nv_bfloat16*>(c);
  g.ldc = ldc;
  g.bias = static_cast<const __nv_bfloat16*>(bias);
  g.wait = wait_ctl(d);
  GemmMaps maps{};
  lr_status st = tensor_map(&maps.a, a, Kc, Mr, lda, kGemmBK, kGemmBM);
  if (st != LR_OK) return st;
  st = tensor_map(&maps.b, b, Nc, Kc, ldb, 64, kGemmBK);
  if (st != LR_OK) return st;
  return launched(launch_gemm_pair(g, maps, d->sms, stream));
}

// A TMA-able view of a [rows, cols] operand: itself, or a realigned copy in
// `scratch` (advanced past the copy).
struct Operand {
  const void* p;
  int64_t ld;
};

size_t repack_bytes(const void* p, int64_t ld, int64_t rows, int64_t cols) {
  if (tma_ok(p, ld) || rows == 0 || cols == 0) return 0;
  return align_up(static_cast<size_t>(rows) * align_up(static_cast<size_t>(cols), kPitchElems) * 2,
                  256);
}

// `*repacks` counts the repack launches of the call so far: all but the first
// may start early (programmatic dependent launch).
// With `early`, the call's first repack may overlap the previous launch and
// read its source before that launch ends (the caller has checked that the
// previous launch does not write it).
lr_status tma_operand(DeviceInfo* d, cudaStream_t stream, const void* p, int64_t ld, int64_t rows,
                      int64_t cols, char** scratch, Operand* out, int* repacks,
                      bool early = false) {
  if (tma_ok(p, ld)) {
    *out = Operand{p, ld};
    return LR_OK;
  }
  const int64_t ldd = static_cast<int64_t>(align_up(static_cast<size_t>(cols), kPitchElems));
  __nv_bfloat16* dst = reinterpret_cast<__nv_bfloat16*>(*scratch);
  *scratch += repack_bytes(p, ld, rows, cols);
  lr_status st = launched(launch_repack(static_cast<const __nv_bfloat16*>(p), ld,
                                        span_bytes(rows, cols, ld), dst, ldd, rows, cols, d->sms,
                                        stream, *repacks > 0 || early, wait_ctl(d),
                                        *repacks > 0 || early));
  if (st != LR_OK) return st;
  ++*repacks;
  *out = Operand{dst, ldd};
  return LR_OK;
}

// Whether a prefill GEMM2 Y = T·B takes T as two bf16 parts, hi = bf16(T) and
// lo = bf16(T - hi) (about 16 significant bits, two tensor-core products per
// k step), instead of T rounded once to bf16.  Rounding T adds an error of
// relative size about 2^-9/sqrt(3) to every output (on top of the output's
// own rounding when Y is bf16), whatever the shape; the two parts remove it
// and add GEMM2's tensor work once more.  Automatic choice
// (lr_set_t_precision(0)): two parts whenever that extra work costs at most
// a third of the call's ideal time, max(FLOPs / tensor peak, bytes / HBM
// bandwidth, 5 µs of launch latency), with B200's dense bf16 peak
// (1.6 PFLOP/s) and HBM bandwidth (6.4 TB/s) as measured with cuBLAS and a
// device copy.
bool t_in_two_parts(int64_t M, int64_t K, int64_t r, int64_t N) {
  const int mode = g_t_precision.load();
  if (mode == 1) return false;
  if (mode == 2) return true;
  const double peak = 1.6e15, bw = 6.4e12;
  const double m = static_cast<double>(M), k = static_cast<double>(K),
               rr = static_cast<double>(r), n = static_cast<double>(N);
  const double extra = 2.0 * m * rr * n / peak;
  const double ideal = std::max({2.0 * m * rr * (k + n) / peak,
                                 2.0 * (m * k + k * rr + rr * n + m * n) / bw, 5e-6});
  return 3.0 * extra <= ideal;
}

lr_status run_prefill(DeviceInfo* d, cudaStream_t stream, const void* X, const void* A,
                      const void* B, const void* bias, void* Y, int64_t M, int64_t K, int64_t r,
                      int64_t N, int64_t ldy, bool y_f32, Pitch ld) {
  const int64_t ldt = static_cast<int64_t>(align_up(static_cast<size_t>(r), kPitchElems));
  const size_t tbytes = align_up(static_cast<size_t>(M) * ldt * 2, 256);
  const size_t rp = repack_bytes(X, ld.x, M, K) + repack_bytes(A, ld.a, K, r) +
                    repack_bytes(B, ld.b, r, N);
  const bool pairs = g_path.load() == 4;
  if (pairs && y_f32) return LR_ERR_UNSUPPORTED;
  const bool two = !pairs && t_in_two_parts(M, K, r, N);
  char *zero = nullptr, *scratch = nullptr;
  lr_status st = workspace(stream, 0, tbytes * (two ? 2 : 1) + (pairs ? rp : 0), &zero, &scratch);
  if (st != LR_OK) return st;
  void* T = scratch;
  scratch += tbytes;
  __nv_bfloat16* T_lo = nullptr;
  if (two) {
    T_lo = reinterpret_cast<__nv_bfloat16*>(scratch);
    scratch += tbytes;
  }
  // Misaligned operands are realigned into an area of their own; the
  // call's first repack may overlap the previous launch (see repack_area).
  bool early = false;
  if (rp > 0 && !pairs) {
    st = repack_area(stream, rp,
                     {{X, span_bytes(M, K, ld.x)}, {A, span_bytes(K, r, ld.a)},
                      {B, span_bytes(r, N, ld.b)}},
                     &scratch, &early);
    if (st != LR_OK) return st;
  }
  Operand x, a, b;
  int repacks = 0;
  if ((st = tma_operand(d, stream, X, ld.x, M, K, &scratch, &x, &repacks, early)) != LR_OK) return st;
  if ((st = tma_operand(d, stream, A, ld.a, K, r, &scratch, &a, &repacks, early)) != LR_OK) return st;
  if ((st = tma_operand(d, stream, B, ld.b, r, N, &scratch, &b, &repacks, early)) != LR_OK) return st;
  if (pairs) {
    // CTA-pair tiles: the two GEMMs as two launches.
    note_call(stream, false, Y, span_bytes(M, N, ldy));
    st = gemm_pair(d, stream, x.p, x.ld, a.p, a.ld, T, ldt, nullptr, M, r, K);
    if (st != LR_OK) return st;
    return gemm_pair(d, stream, T, ldt, b.p, b.ld, Y, ldy, bias, M, N, r);
  }
  // One launch: GEMM1 T = X·A signals counter group 0 per 128-row block;
  // GEMM2 Y = T·B + bias waits on it row block by row block.  The launch
  // may overlap the kernel before it: after this call's repacks only the
  // repacked operands depend on that kernel (the repacks finish after the
  // launch before them); with no repack, it is the caller's previous kernel,
  // which may have written any input.
  const bool after_repack = repacks > 0;
  auto dep = [&](const void* used, const void* given) { return !after_repack || used != given; };
  ChainBuild cb;
  int mx, ma, mt, mb, mt_lo = -1;
  if ((st = chain_map(cb, x.p, K, M, x.ld, true, &mx)) != LR_OK) return st;
  if ((st = chain_map(cb, a.p, r, K, a.ld, false, &ma)) != LR_OK) return st;
  if ((st = chain_map(cb, T, r, M, ldt, true, &mt)) != LR_OK) return st;
  if (two && (st = chain_map(cb, T_lo, r, M, ldt, true, &mt_lo)) != LR_OK) return st;
  if ((st = chain_map(cb, b.p, N, r, b.ld, false, &mb)) != LR_OK) return st;
  // GEMM1's columns: when whole 256-column tiles already take more than one
  // wave and the last tile would be at most half full, the tail columns are
  // a problem of their own (narrow tiles that split K over the idle SMs)
  // instead of a second wave of full-depth tiles.
  const int64_t main_cols = r / 256 * 256, tail = r - main_cols;
  if (main_cols > 0 && tail > 0 && tail <= 128 &&
      ceil_div(M, kGemmBM) * ceil_div(r, 256) > d->sms && g_tile_n.load() == 0) {
    st = chain_problem(cb, mx, 0, ma, M, main_cols, K, T, ldt, nullptr, -1, 0, dep(x.p, X),
                       dep(a.p, A));
    if (st != LR_OK) return st;
    cb.args.p[cb.args.n_prob - 1].c_lo = T_lo;
    st = chain_problem(cb, mx, 0, ma, M, tail, K, static_cast<__nv_bfloat16*>(T) + main_cols, ldt,
                       nullptr, -1, 0, dep(x.p, X), dep(a.p, A), static_cast<int>(main_cols));
    if (st != LR_OK) return st;
    cb.args.p[cb.args.n_prob - 1].c_lo = two ? T_lo + main_cols : nullptr;
  } else {
    st = chain_problem(cb, mx, 0, ma, M, r, K, T, ldt, nullptr, -1, 0, dep(x.p, X), dep(a.p, A));
    if (st != LR_OK) return st;
    cb.args.p[cb.args.n_prob - 1].c_lo = T_lo;
  }
  st = chain_problem(cb, mt, 0, mb, M, N, r, Y, ldy, bias, 0, -1, false, dep(b.p, B));
  if (st != LR_OK) return st;
  cb.args.p[cb.args.n_prob - 1].map_a_lo = mt_lo;
  if (y_f32) cb.args.p[cb.args.n_prob - 1].c32 = static_cast<float*>(Y);
  st = run_chain(d, stream, cb);
  note_call(stream, st == LR_OK, Y, span_bytes(M, N, ldy) * (y_f32 ? 2 : 1),
            cb.args.total_tiles >= d->sms);
  return st;
}

lr_status run_linear(const void* X, const void* A, const void* B, const void* bias, void* Y,
                     int64_t M, int64_t K, int64_t r, int64_t N, int64_t ldy, cudaStream_t stream,
                     bool y_f32 = false, Pitch ld = Pitch{-1, -1, -1}) {
  if (ld.x < 0) ld = Pitch{K, r, N};
  lr_status st = validate(X, A, B, bias, Y, M, K, r, N, ldy, y_f32, ld);
  if (st != LR_OK) return st;
  const int path = g_path.load();
  if ((path == 1 || path == 5 || path == 6) && M > 16) return LR_ERR_INVALID_ARG;
  if (M == 0 || N == 0) return LR_OK;
  DeviceInfo* d = nullptr;
  int dev = 0;
  st = device_info(&d, &dev);
  if (st != LR_OK) return st;
  const size_t ybytes = span_bytes(M, N, ldy) * (y_f32 ? 2 : 1);
  if (K == 0 || r == 0) {
    note_call(stream, false, Y, ybytes);
    return launched(launch_fill_bias(Y, y_f32, ldy, M, N, static_cast<const __nv_bfloat16*>(bias),
                                     stream));
  }
  const bool contiguous = ld.x == K && ld.a == r && ld.b == N;
  if (path == 0 && contiguous && tiny_fits(M, K, r, N)) {
    note_call(stream, false, Y, ybytes);
    TinyArgs t{};
    t.M = static_cast<int>(M);
    t.K = static_cast<int>(K);
    t.r = static_cast<int>(r);
    t.N = static_cast<int>(N);
    t.X = X;
    t.A = A;
    t.B = B;
    t.bias = static_cast<const __nv_bfloat16*>(bias);
    t.Y = Y;
    t.ldy = ldy;
    t.y_f32 = y_f32 ? 1 : 0;
    return launched(launch_tiny(t, stream));
  }
  const bool decode = (path == 1) || (path == 5) || (path == 6) || (path == 0 && M <= 16);
  if (decode) {
    note_call(stream, false, Y, ybytes);
    return run_decode(d, stream, X, A, B, bias, Y, M, K, r, N, ldy, y_f32, ld);
  }
  return run_prefill(d, stream, X, A, B, bias, Y, M, K, r, N, ldy, y_f32, ld);
}


// The projections of a group at prefill sizes, in one chain launch.
// Projections that share X (same pointer and K) form a set: their A factors
// are copied side by side into one [K, Σ r_i] factor (each r_i rounded up to
// 8 columns, so every slice starts on a 16-byte boundary) and the set runs
// one GEMM1 T_set = X·A_set; projection i then runs GEMM2 Y_i = T_set[:,
// off_i : off_i + r_i]·B_i (+bias_i), waiting for T_set's row blocks.  Its
// K loop may read T_set columns past r_i (the next slice) but B_i's rows
// past r_i read as zero, so those products are zero.  X is read once per set
// and the whole layer is one launch.  Returns LR_ERR_UNSUPPORTED (before any
// launch) when the group does not fit one launch's tables.
lr_status run_group_prefill(DeviceInfo* d, cudaStream_t stream, const lr_proj* projs, int n,
                            int64_t M) {
  for (int i = 0; i < n; ++i)
    note_call(stream, false, projs[i].Y,
              span_bytes(M, projs[i].N, projs[i].ld_y) * (projs[i].y_f32 ? 2 : 1));
  struct Set {
    const void* X;
    int64_t K;
    std::vector<int> members;
    int64_t width = 0;  // columns of T_set (sum of slices)
    int64_t pitch = 0;  // row pitch of T_set and A_set: width in 128-byte rows
    bool concat = false;  // A copied into a concatenated factor
    bool two = false;     // T_set also written as a low part (some member reads two parts)
  };
  std::vector<Set> sets;
  std::vector<int64_t> off(static_cast<size_t>(n), 0);
  std::vector<int> set_of(static_cast<size_t>(n), -1);
  int gemm2 = 0;
  for (int i = 0; i < n; ++i) {
    const lr_proj& p = projs[i];
    if (p.N == 0 || p.K == 0 || p.r == 0) continue;
    int si = -1;
    for (size_t k = 0; k < sets.size(); ++k)
      if (sets[k].X == p.X && sets[k].K == p.K) si = static_cast<int>(k);
    if (si < 0) {
      sets.push_back(Set{p.X, p.K, {}, 0, 0, false, false});
      si = static_cast<int>(sets.size()) - 1;
    }
    Set& st = sets[static_cast<size_t>(si)];
    off[static_cast<size_t>(i)] = st.width;
    st.width += static_cast<int64_t>(align_up(static_cast<size_t>(p.r), 8));
    st.members.push_back(i);
    if (t_in_two_parts(M, p.K, p.r, p.N)) st.two = true;
    set_of[static_cast<size_t>(i)] = si;
    ++gemm2;
  }
  int n_two = 0;
  for (Set& st : sets) {
    st.pitch = static_cast<int64_t>(align_up(static_cast<size_t>(st.width), kPitchElems));
    n_two += st.two ? 1 : 0;
  }
  if (static_cast<int>(sets.size()) + gemm2 > kChainMaxProbs ||
      3 * static_cast<int>(sets.size()) + n_two + gemm2 > kChainMaxMaps)
    return LR_ERR_UNSUPPORTED;
  // Workspace: T per set, concatenated factors, realigned X and B copies.
  size_t need = 0;
  for (Set& st : sets) {
    const lr_proj& p0 = projs[st.members[0]];
    st.concat = st.members.size() > 1 || !tma_ok(p0.A, p0.r);
    need += align_up(static_cast<size_t>(M) * st.pitch * 2, 256) * (st.two ? 2 : 1);
    if (st.concat) need += align_up(static_cast<size_t>(st.K) * st.pitch * 2, 256);
    need += repack_bytes(st.X, st.K, M, st.K);
  }
  for (int i = 0; i < n; ++i)
    if (set_of[static_cast<size_t>(i)] >= 0) need += repack_bytes(projs[i].B, projs[i].N, projs[i].r, projs[i].N);
  char *zero = nullptr, *scratch = nullptr;
  lr_status stt = workspace(stream, 0, need, &zero, &scratch);
  if (stt != LR_OK) return stt;
  // Empty contractions: Y = bias.
  for (int i = 0; i < n; ++i) {
    const lr_proj& p = projs[i];
    if (M > 0 && p.N > 0 && (p.K == 0 || p.r == 0)) {
      stt = launched(launch_fill_bias(p.Y, p.y_f32 != 0, p.ld_y, M, p.N,
                                      static_cast<const __nv_bfloat16*>(p.bias), stream));
      if (stt != LR_OK) return stt;
    }
  }
  // Copies (repack kernels), then the chain launch.
  int repacks = 0;
  struct SetOps {
    void* T;
    __nv_bfloat16* T_lo;
    Operand x, a;
  };
  std::vector<SetOps> ops(sets.size());
  for (size_t k = 0; k < sets.size(); ++k) {
    Set& st = sets[k];
    ops[k].T = scratch;
    scratch += align_up(static_cast<size_t>(M) * st.pitch * 2, 256);
    ops[k].T_lo = nullptr;
    if (st.two) {
      ops[k].T_lo = reinterpret_cast<__nv_bfloat16*>(scratch);
      scratch += align_up(static_cast<size_t>(M) * st.pitch * 2, 256);
    }
    stt = tma_operand(d, stream, st.X, st.K, M, st.K, &scratch, &ops[k].x, &repacks);
    if (stt != LR_OK) return stt;
    if (st.concat) {
      __nv_bfloat16* cat = reinterpret_cast<__nv_bfloat16*>(scratch);
      scratch += align_up(static_cast<size_t>(st.K) * st.pitch * 2, 256);
      for (int i : st.members) {
        const lr_proj& p = projs[i];
        stt = launched(launch_repack(static_cast<const __nv_bfloat16*>(p.A), p.r,
                                     span_bytes(p.K, p.r, p.r), cat + off[static_cast<size_t>(i)],
                                     st.pitch, p.K, p.r, d->sms, stream, repacks > 0,
                                     wait_ctl(d)));
        if (stt != LR_OK) return stt;
        ++repacks;
      }
      ops[k].a = Operand{cat, st.pitch};
    } else {
      const lr_proj& p = projs[st.members[0]];
      ops[k].a = Operand{p.A, p.r};
    }
  }
  std::vector<Operand> bops(static_cast<size_t>(n));
  for (int i = 0; i < n; ++i) {
    if (set_of[static_cast<size_t>(i)] < 0) continue;
    const lr_proj& p = projs[i];
    stt = tma_operand(d, stream, p.B, p.N, p.r, p.N, &scratch, &bops[static_cast<size_t>(i)], &repacks);
    if (stt != LR_OK) return stt;
  }
  const bool after_repack = repacks > 0;
  auto dep = [&](const void* used, const void* given) { return !after_repack || used != given; };
  ChainBuild cb;
  std::vector<int> tmap(sets.size()), tmap_lo(sets.size(), -1);
  for (size_t k = 0; k < sets.size(); ++k) {
    const Set& st = sets[k];
    const lr_proj& p0 = projs[st.members[0]];
    const int64_t nc = st.concat ? st.width : p0.r;  // T columns GEMM1 writes
    int mx, ma, mt;
    if ((stt = chain_map(cb, ops[k].x.p, st.K, M, ops[k].x.ld, true, &mx)) != LR_OK) return stt;
    if ((stt = chain_map(cb, ops[k].a.p, nc, st.K, ops[k].a.ld, false, &ma)) != LR_OK) return stt;
    // T's columns past nc are never written: the map ends there (they read as
    // zero); a concatenated T's slice pads are written as zero by GEMM1.
    if ((stt = chain_map(cb, ops[k].T, nc, M, st.pitch, true, &mt)) != LR_OK) return stt;
    tmap[k] = mt;
    if (st.two &&
        (stt = chain_map(cb, ops[k].T_lo, nc, M, st.pitch, true, &tmap_lo[k])) != LR_OK)
      return stt;
    stt = chain_problem(cb, mx, 0, ma, M, nc, st.K, ops[k].T, st.pitch, nullptr, -1,
                        static_cast<int>(k), dep(ops[k].x.p, st.X), dep(ops[k].a.p, p0.A));
    if (stt != LR_OK) return stt;
    cb.args.p[cb.args.n_prob - 1].c_lo = ops[k].T_lo;
  }
  for (size_t k = 0; k < sets.size(); ++k) {
    for (int i : sets[k].members) {
      const lr_proj& p = projs[i];
      const Operand& b = bops[static_cast<size_t>(i)];
      int mb;
      if ((stt = chain_map(cb, b.p, p.N, p.r, b.ld, false, &mb)) != LR_OK) return stt;
      stt = chain_problem(cb, tmap[k], static_cast<int>(off[static_cast<size_t>(i)]), mb, M, p.N,
                          p.r, p.Y, p.ld_y, p.bias, static_cast<int>(k), -1, false, dep(b.p, p.B));
      if (stt != LR_OK) return stt;
      ChainProblem& P = cb.args.p[cb.args.n_prob - 1];
      if (t_in_two_parts(M, p.K, p.r, p.N)) P.map_a_lo = tmap_lo[k];
      if (p.y_f32) P.c32 = static_cast<float*>(p.Y);
    }
  }
  return run_chain(d, stream, cb);
}

// Two projections' outputs may interleave (gate and up writing the two halves
// of one packed buffer) but must not share an element.  Conservative: equal
// row strides and no row that spills into the next are required when the byte
// ranges overlap at all.
bool y_disjoint(const lr_proj& p, const lr_proj& q, int64_t M) {
  if (!p.Y || !q.Y || M == 0 || p.N == 0 || q.N == 0) return true;
  const int64_t es = p.y_f32 ? 4 : 2;
  if (!ranges_overlap(p.Y, span_bytes(M, p.N, p.ld_y) * (es / 2), q.Y,
                      span_bytes(M, q.N, q.ld_y) * (q.y_f32 ? 2 : 1)))
    return true;
  if (p.ld_y != q.ld_y || (p.y_f32 != 0) != (q.y_f32 != 0)) return false;
  const intptr_t d = reinterpret_cast<intptr_t>(q.Y) - reinterpret_cast<intptr_t>(p.Y);
  if (d % es != 0) return false;
  const int64_t off = d / es, ld = p.ld_y;
  int64_t a = off / ld, b = off % ld;
  if (b < 0) {
    b += ld;
    a -= 1;
  }
  if (b + q.N > ld) return false;
  const bool rows = (a < 0 ? -a : a) < M;
  const bool cols = b < p.N;
  return !(rows && cols);
}

}  // namespace

void note_cuda_error(int e) { g_last_cuda_error = e; }

unsigned long long wait_limit_ns() {
  const long long ns = g_wait_ns.load();
  return static_cast<unsigned long long>(ns > 0 ? ns : kDefaultWaitNs);
}

void note_launches(int n) { g_launches += n; }

void note_output(cudaStream_t stream, const void* y, size_t bytes) {
  note_call(stream, false, y, bytes);
}

cudaError_t ensure_max_smem(const void* kernel, int bytes) {
  static std::mutex mu;
  static std::set<std::tuple<const void*, int, int>> done;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lk(mu);
  if (done.count({kernel, dev, bytes})) return cudaSuccess;
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess) done.insert({kernel, dev, bytes});
  return e;
}

}  // namespace lr

using namespace lr;

extern "C" {

lr_status lr_linear(const void* X, const void* A, const void* B, const void* bias, void* Y,
                    int64_t M, int64_t K, int64_t r, int64_t N, void* stream) {
  return run_linear(X, A, B, bias, Y, M, K, r, N, N, static_cast<cudaStream_t>(stream));
}

lr_status lr_linear_f32(const void* X, const void* A, const void* B, const void* bias, void* Y,
                        int64_t M, int64_t K, int64_t r, int64_t N, void* stream) {
  return run_linear(X, A, B, bias, Y, M, K, r, N, N, static_cast<cudaStream_t>(stream), true);
}

lr_status lr_linear_strided(const void* X, int64_t ldx, const void* A, int64_t lda, const void* B,
                            int64_t ldb, const void* bias, void* Y, int64_t ldy, int64_t M,
                            int64_t K, int64_t r, int64_t N, int32_t y_f32, void* stream) {
  return run_linear(X, A, B, bias, Y, M, K, r, N, ldy, static_cast<cudaStream_t>(stream),
                    y_f32 != 0, Pitch{ldx, lda, ldb});
}

int64_t lr_factor_pitch(int64_t cols) {
  if (cols < 0) return -1;
  return (cols + kPitchElems - 1) / kPitchElems * kPitchElems;
}

// The area for the fp32 products of a group's gated projections on
// `stream` (`bytes`, grown on demand).
lr_status act_area(cudaStream_t stream, size_t bytes, float** out) {
  int dev = 0;
  LR_CUDA(cudaGetDevice(&dev));
  std::lock_guard<std::mutex> lk(g_mu);
  Workspace& w = g_ws[{dev, stream}];
  if (bytes > w.act_cap) {
    if (w.act) {
      LR_CUDA(cudaStreamSynchronize(stream));
      LR_CUDA(cudaFree(w.act));
      w.act = nullptr;
      w.act_cap = 0;
    }
    const size_t cap = align_up(bytes + bytes / 4, 1 << 20);
    LR_CUDA(cudaMalloc(&w.act, cap));
    w.act_cap = cap;
  }
  *out = w.act;
  return LR_OK;
}

lr_status lr_linear_group(const lr_proj* projs, int n_proj, int64_t M, void* stream) {
  if (n_proj < 0 || (n_proj > 0 && !projs) || M < 0) return LR_ERR_INVALID_ARG;
  bool gated = false;
  for (int i = 0; i < n_proj; ++i) {
    const int g = projs[i].silu_gate - 1;
    if (g == -1) continue;
    if (g < 0 || g >= n_proj || g == i || projs[g].silu_gate != 0 || projs[g].N != projs[i].N)
      return LR_ERR_INVALID_ARG;
    gated = true;
  }
  // Validate everything before the first launch, including Y overlaps.
  for (int i = 0; i < n_proj; ++i) {
    const lr_proj& p = projs[i];
    lr_status st = validate(p.X, p.A, p.B, p.bias, p.Y, M, p.K, p.r, p.N, p.ld_y, p.y_f32 != 0);
    if (st != LR_OK) return st;
    const size_t yi = span_bytes(M, p.N, p.ld_y) * (p.y_f32 ? 2 : 1);
    for (int j = 0; j < n_proj; ++j) {
      const lr_proj& q = projs[j];
      if (j != i) {
        if (!y_disjoint(p, q, M)) return LR_ERR_INVALID_ARG;
        if (ranges_overlap(p.Y, yi, q.X, span_bytes(M, q.K, q.K)) ||
            ranges_overlap(p.Y, yi, q.A, span_bytes(q.K, q.r, q.r)) ||
            ranges_overlap(p.Y, yi, q.B, span_bytes(q.r, q.N, q.N)) ||
            ranges_overlap(p.Y, yi, q.bias, span_bytes(1, q.N, q.N)))
          return LR_ERR_INVALID_ARG;
      }
    }
  }
  const int path = g_path.load();
  const bool streamed = M > 0 && M <= 8 && (path == 0 || path == 6) && n_proj > 0 &&
                        n_proj <= kStreamMaxJobs / 2;
  bool all_work = true;
  for (int i = 0; i < n_proj; ++i)
    all_work = all_work && projs[i].K > 0 && projs[i].r > 0 && projs[i].N > 0;
  // Decode sizes (M <= 8): the whole group in one streamed launch, when
  // every projection has work (K, r, N > 0) and the group fits the launch's
  // table (at most kStreamMaxJobs / 2 projections); gated outputs are formed
  // there.
  if (streamed) {
    if (all_work) {
      DeviceInfo* d = nullptr;
      int dev = 0;
      lr_status st = device_info(&d, &dev);
      if (st != LR_OK) return st;
      StreamPair pairs[kStreamMaxJobs / 2];
      for (int i = 0; i < n_proj; ++i) {
        const lr_proj& p = projs[i];
        pairs[i] = StreamPair{p.X, p.A, p.B, p.bias, p.Y, p.K, p.r, p.N, p.ld_y, p.y_f32 != 0,
                              Pitch{p.K, p.r, p.N}, p.silu_gate - 1};
        note_call(static_cast<cudaStream_t>(stream), false, p.Y,
                  span_bytes(M, p.N, p.ld_y) * (p.y_f32 ? 2 : 1));
      }
      st = run_stream(d, static_cast<cudaStream_t>(stream), static_cast<int>(M), pairs, n_proj);
      if (st != LR_ERR_UNSUPPORTED) return st;
    }
  }
  if (gated) {
    // Gated outputs without the fused path: the gated projections' products
    // go to an fp32 area, the group runs as usual, then one elementwise
    // launch per gated projection forms silu(G) · P.
    if (M == 0) return LR_OK;
    size_t need = 0;
    for (int i = 0; i < n_proj; ++i)
      if (projs[i].silu_gate) need += align_up(static_cast<size_t>(M * projs[i].N) * 4, 256);
    float* area = nullptr;
    lr_status st = act_area(static_cast<cudaStream_t>(stream), need, &area);
    if (st != LR_OK) return st;
    std::vector<lr_proj> q(projs, projs + n_proj);
    std::vector<float*> prod(static_cast<size_t>(n_proj), nullptr);
    for (int i = 0; i < n_proj; ++i) {
      if (!projs[i].silu_gate) continue;
      prod[i] = area;
      area += align_up(static_cast<size_t>(M * projs[i].N) * 4, 256) / 4;
      q[i].Y = prod[i];
      q[i].ld_y = projs[i].N;
      q[i].y_f32 = 1;
      q[i].silu_gate = 0;
    }
    st = lr_linear_group(q.data(), n_proj, M, stream);
    if (st != LR_OK) return st;
    for (int i = 0; i < n_proj; ++i) {
      if (!projs[i].silu_gate) continue;
      const lr_proj& g = projs[projs[i].silu_gate - 1];
      st = launched(launch_silu_mul(g.Y, g.ld_y, g.y_f32 != 0, prod[i], projs[i].Y,
                                    projs[i].ld_y, projs[i].y_f32 != 0, M, projs[i].N,
                                    static_cast<cudaStream_t>(stream)));
      if (st != LR_OK) return st;
    }
    return LR_OK;
  }
  // Prefill sizes: the whole group in one chain launch (see run_group_prefill).
  if (M > 16 && path != 1 && path != 4 && path != 5 && path != 6 && n_proj > 0) {
    DeviceInfo* d = nullptr;
    int dev = 0;
    lr_status st = device_info(&d, &dev);
    if (st != LR_OK) return st;
    st = run_group_prefill(d, static_cast<cudaStream_t>(stream), projs, n_proj, M);
    if (st != LR_ERR_UNSUPPORTED) return st;
  }
  for (int i = 0; i < n_proj; ++i) {
    const lr_proj& p = projs[i];
    lr_status st = run_linear(p.X, p.A, p.B, p.bias, p.Y, M, p.K, p.r, p.N, p.ld_y,
                              static_cast<cudaStream_t>(stream), p.y_f32 != 0);
    if (st != LR_OK) return st;
  }
  return LR_OK;
}

lr_status lr_linear_host(const void* X, const void* A, const void* B, const void* bias, void* Y,
                         int64_t M, int64_t K, int64_t r, int64_t N, void* stream_) {
  if (M < 0 || K < 0 || r < 0 || N < 0) return LR_ERR_INVALID_ARG;
  if (M > kMaxDim || K > kMaxDim || r > kMaxDim || N > kMaxDim) return LR_ERR_UNSUPPORTED;
  if (M > 0 && N > 0 && !Y) return LR_ERR_INVALID_ARG;
  if (M > 0 && K > 0 && r > 0 && N > 0 && (!X || !A || !B)) return LR_ERR_INVALID_ARG;
  if (M == 0 || N == 0) return LR_OK;
  cudaStream_t stream = static_cast<cudaStream_t>(stream_);
  const size_t bx = align_up(static_cast<size_t>(M * K) * 2, 256);
  const size_t ba = align_up(static_cast<size_t>(K * r) * 2, 256);
  const size_t bb = align_up(static_cast<size_t>(r * N) * 2, 256);
  const size_t bz = align_up(static_cast<size_t>(N) * 2, 256);
  const size_t by = align_up(static_cast<size_t>(M * N) * 2, 256);
  const size_t need = bx + ba + bb + bz + by;
  char* base = nullptr;
  {
    int dev = 0;
    LR_CUDA(cudaGetDevice(&dev));
    std::lock_guard<std::mutex> lk(g_mu);
    Staging& s = g_stage[{dev, stream}];
    if (need > s.cap) {
      if (s.ptr) {
        LR_CUDA(cudaStreamSynchronize(stream));
        LR_CUDA(cudaFree(s.ptr));
        s.ptr = nullptr;
        s.cap = 0;
      }
      LR_CUDA(cudaMalloc(&s.ptr, need));
      s.cap = need;
    }
    base = s.ptr;
  }
  char* dX = base;
  char* dA = dX + bx;
  char* dB = dA + ba;
  char* dz = dB + bb;
  char* dY = dz + bz;
  if (M * K) LR_CUDA(cudaMemcpyAsync(dX, X, M * K * 2, cudaMemcpyHostToDevice, stream));
  if (K * r) LR_CUDA(cudaMemcpyAsync(dA, A, K * r * 2, cudaMemcpyHostToDevice, stream));
  if (r * N) LR_CUDA(cudaMemcpyAsync(dB, B, r * N * 2, cudaMemcpyHostToDevice, stream));
  if (bias) LR_CUDA(cudaMemcpyAsync(dz, bias, N * 2, cudaMemcpyHostToDevice, stream));
  lr_status st = run_linear(dX, dA, dB, bias ? dz : nullptr, dY, M, K, r, N, N, stream);
  if (st != LR_OK) return st;
  LR_CUDA(cudaMemcpyAsync(Y, dY, M * N * 2, cudaMemcpyDeviceToHost, stream));
  LR_CUDA(cudaStreamSynchronize(stream));
  return LR_OK;
}

lr_status lr_dense(const void* X, const void* W, const void* bias, void* Y, int64_t M, int64_t K,
                   int64_t N, void* stream_) {
  // W [K, N] plays the role of A with r = N (no second factor).
  lr_status st = validate(X, W, W, bias, Y, M, K, N, N, N);
  if (st != LR_OK) return st;
  if (M == 0 || N == 0) return LR_OK;
  cudaStream_t stream = static_cast<cudaStream_t>(stream_);
  note_call(stream, false, Y, span_bytes(M, N, N));
  DeviceInfo* d = nullptr;
  int dev = 0;
  st = device_info(&d, &dev);
  if (st != LR_OK) return st;
  if (K == 0)
    return launched(launch_fill_bias(Y, false, N, M, N, static_cast<const __nv_bfloat16*>(bias),
                                     stream));
  const int path = g_path.load();
  const bool decode = (path == 1) || (path == 5) || (path == 6) || (path == 0 && M <= 16);
  if (decode) {
    if (M > 16) return LR_ERR_INVALID_ARG;
    const int m = static_cast<int>(M);
    const size_t acc = acc_bytes(m, N), c = ctr_bytes(m, K, N, d->sms);
    char *zero = nullptr, *scratch = nullptr;
    st = workspace(stream, acc + c, 0, &zero, &scratch);
    if (st != LR_OK) return st;
    return skinny(d, stream, m, X, K, false, W, K, N, reinterpret_cast<float*>(zero),
                  reinterpret_cast<unsigned int*>(zero + acc), nullptr, 0, Y, N, bias);
  }
  {
    const size_t need = repack_bytes(X, K, M, K) + repack_bytes(W, N, K, N);
    char *zero = nullptr, *scratch = nullptr;
    st = workspace(stream, 0, need, &zero, &scratch);
    if (st != LR_OK) return st;
    Operand x, w;
    int repacks = 0;
    if ((st = tma_operand(d, stream, X, K, M, K, &scratch, &x, &repacks)) != LR_OK) return st;
    if ((st = tma_operand(d, stream, W, N, K, N, &scratch, &w, &repacks)) != LR_OK) return st;
    if (path == 4) return gemm_pair(d, stream, x.p, x.ld, w.p, w.ld, Y, N, bias, M, N, K);
    ChainBuild cb;
    int mx, mw;
    if ((st = chain_map(cb, x.p, K, M, x.ld, true, &mx)) != LR_OK) return st;
    if ((st = chain_map(cb, w.p, N, K, w.ld, false, &mw)) != LR_OK) return st;
    const bool after_repack = repacks > 0;
    st = chain_problem(cb, mx, 0, mw, M, N, K, Y, N, bias, -1, -1, !after_repack || x.p != X,
                       !after_repack || w.p != W);
    if (st != LR_OK) return st;
    return run_chain(d, stream, cb);
  }
}

lr_status lr_last_device_status(void* stream) {
  cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e);
  DeviceInfo* d = nullptr;
  int dev = 0;
  lr_status st = device_info(&d, &dev);
  if (st != LR_OK) return st;
  DevStatus h{};
  LR_CUDA(cudaMemcpy(&h, d->status, sizeof h, cudaMemcpyDeviceToHost));
  // The allocation-free entry point keeps its own status word.
  unsigned int static_code = 0;
  LR_CUDA(static_status_take(&static_code));
  h.code |= static_code;
  if (h.code == 0 && h.abort == 0) return LR_OK;
  LR_CUDA(cudaMemset(d->status, 0, sizeof(DevStatus)));
  {
    // A launch that gave up may have left partial sums behind: zero what
    // this stream's workspace must hold zero between calls.
    std::lock_guard<std::mutex> lk(g_mu);
    auto it = g_ws.find({dev, static_cast<cudaStream_t>(stream)});
    if (it != g_ws.end()) {
      if (it->second.ptr && it->second.zero_bytes)
        LR_CUDA(cudaMemset(it->second.ptr, 0, it->second.zero_bytes));
      if (it->second.split_ws) LR_CUDA(cudaMemset(it->second.split_ws, 0, it->second.split_cap));
    }
  }
  return (h.code & LR_DEV_TIMEOUT) ? LR_ERR_TIMEOUT : LR_ERR_CUDA;
}

const char* lr_status_string(lr_status s) {
  switch (s) {
    case LR_OK: return "LR_OK";
    case LR_ERR_INVALID_ARG: return "LR_ERR_INVALID_ARG";
    case LR_ERR_UNSUPPORTED: return "LR_ERR_UNSUPPORTED";
    case LR_ERR_CUDA: return "LR_ERR_CUDA";
    case LR_ERR_TIMEOUT: return "LR_ERR_TIMEOUT";
    case LR_ERR_NO_MEMORY: return "LR_ERR_NO_MEMORY";
    case LR_ERR_INFEASIBLE: return "LR_ERR_INFEASIBLE";
  }
  return "LR_ERR_UNKNOWN";
}

int lr_last_cuda_error(void) { return g_last_cuda_error; }

lr_status lr_set_path(int path) {
  if (path < 0 || path > 6) return LR_ERR_INVALID_ARG;
  g_path.store(path);
  return LR_OK;
}

lr_status lr_set_wait_limit_ns(int64_t ns) {
  if (ns < 0) return LR_ERR_INVALID_ARG;
  g_wait_ns.store(ns);
  return LR_OK;
}

int64_t lr_kernel_launch_count(void) { return g_launches.load(); }

lr_status lr_set_split_k(int on) {
  if (on < 0 || on > 1) return LR_ERR_INVALID_ARG;
  g_split_k.store(on);
  return LR_OK;
}

lr_status lr_set_early_copy(int on) {
  if (on != 0 && on != 1) return LR_ERR_INVALID_ARG;
  g_early_copy.store(on);
  return LR_OK;
}

lr_status lr_set_t_precision(int mode) {
  if (mode < 0 || mode > 2) return LR_ERR_INVALID_ARG;
  g_t_precision.store(mode);
  return LR_OK;
}

lr_status lr_set_tile_n(int bn) {
  if (bn < 0 || bn > 256 || bn % 32 != 0) return LR_ERR_INVALID_ARG;
  g_tile_n.store(bn);
  return LR_OK;
}

lr_status lr_set_withhold_first_stage(int on) {
  if (on != 0 && on != 1) return LR_ERR_INVALID_ARG;
  g_withhold.store(on);
  return LR_OK;
}

lr_status lr_release_workspaces(void) {
  std::lock_guard<std::mutex> lk(g_mu);
  int cur = 0;
  cudaGetDevice(&cur);
  for (auto& kv : g_ws) {
    if (!kv.second.ptr && !kv.second.ctrs && !kv.second.split_ws && !kv.second.rp_area[0] &&
        !kv.second.act)
      continue;
    cudaSetDevice(kv.first.first);
    cudaStreamSynchronize(kv.first.second);
    if (kv.second.ptr) cudaFree(kv.second.ptr);
    if (kv.second.ctrs) cudaFree(kv.second.ctrs);
    if (kv.second.split_ws) cudaFree(kv.second.split_ws);
    if (kv.second.act) cudaFree(kv.second.act);
    for (char* a : kv.second.rp_area)
      if (a) cudaFree(a);
  }
  g_ws.clear();
  {
    // Every stream that ran the streamed kernel has a workspace, synchronised
    // above: no launch still reads a piece table.
    std::lock_guard<std::mutex> plk(g_piece_mu);
    for (auto& kv : g_piece_tables) {
      cudaSetDevice(static_cast<int>(kv.first[0]));
      cudaFree(kv.second.pieces);
      cudaFree(kv.second.off);
    }
    g_piece_tables.clear();
  }
  g_streams.clear();
  for (auto& kv : g_stage) {
    if (!kv.second.ptr) continue;
    cudaSetDevice(kv.first.first);
    cudaStreamSynchronize(kv.first.second);
    cudaFree(kv.second.ptr);
  }
  g_stage.clear();
  g_maps.clear();
  cudaSetDevice(cur);
  return LR_OK;
}

}  // extern "C"
