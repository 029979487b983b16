// lr_static.cu — lr_linear_decode_static: the decode path (M <= 16) of the
// layer with every byte of scratch taken from a fixed array compiled into
// this library, so the call never allocates device memory.
//
// Who needs it: callers that cannot let a library call cudaMalloc.  A serving
// loop with a hard latency budget cannot afford it (cudaMalloc and cudaFree
// synchronise the whole device, stalling every stream); a host application
// that hands all device memory to its own pool allocator forbids outside
// allocations so that its memory budget holds.  lr_linear grows a workspace
// with cudaMalloc on first use; this entry point does not.
//
// The scratch array below is file-scope `static __device__` memory: every
// GPU that loads this library holds kStaticBytes of it until the process
// exits.  All calls on a device share it, so calls whose kernels overlap on
// the GPU (different streams, or different host threads) race on it.
#include <mutex>

#include "../../include/lr_linear.h"
#include "lr_internal.h"

namespace lr {
namespace {

// Limits of the static scratch (documented in include/lr_linear.h).
constexpr int64_t kStaticMaxM = 16;
constexpr int64_t kStaticMaxR = 4096;
constexpr int64_t kStaticMaxN = 16384;
constexpr int64_t kStaticMaxCounters = 4096;  // column blocks per phase

constexpr size_t kAcc1Bytes = kStaticMaxM * kStaticMaxR * 4;   // phase-1 partial sums
constexpr size_t kAcc2Bytes = kStaticMaxM * kStaticMaxN * 4;   // phase-2 partial sums
constexpr size_t kCtrBytes = 2 * kStaticMaxCounters * 4;        // last-CTA counters
constexpr size_t kTBytes = kStaticMaxM * kStaticMaxR * 4;      // T = X·A in fp32
constexpr size_t kStatusBytes = 256;                            // device status word
constexpr size_t kStaticBytes = kAcc1Bytes + kAcc2Bytes + kCtrBytes + kTBytes + kStatusBytes;

static __device__ __align__(256) unsigned char g_static_scratch[kStaticBytes];

constexpr int kMaxDevices = 64;
std::mutex g_static_mu;
char* g_static_ptr[kMaxDevices];  // device address of g_static_scratch, per device
int g_static_sms[kMaxDevices];

lr_status fail(cudaError_t e) {
  note_cuda_error(static_cast<int>(e));
  return LR_ERR_CUDA;
}

// Once per device, with that device current: the device address of the
// scratch array (in host code its name is only a host-side stand-in) and the
// SM count.  Neither call allocates.
lr_status static_setup(char** ptr, int* sms) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fail(e);
  if (dev < 0 || dev >= kMaxDevices) return LR_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lk(g_static_mu);
  if (!g_static_ptr[dev]) {
    int major = 0, n = 0;
    e = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
    if (e != cudaSuccess) return fail(e);
    if (major != 10) return LR_ERR_UNSUPPORTED;
    e = cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return fail(e);
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_static_scratch);
    if (e != cudaSuccess || p == nullptr) return fail(e == cudaSuccess ? cudaErrorInvalidSymbol : e);
    g_static_ptr[dev] = static_cast<char*>(p);
    g_static_sms[dev] = n;
  }
  *ptr = g_static_ptr[dev];
  *sms = g_static_sms[dev];
  return LR_OK;
}

int64_t round4(int64_t x) { return (x + 3) / 4 * 4; }

bool overlaps(const void* a, int64_t abytes, const void* b, int64_t bbytes) {
  if (!a || !b || abytes <= 0 || bbytes <= 0) return false;
  const uintptr_t a0 = reinterpret_cast<uintptr_t>(a), b0 = reinterpret_cast<uintptr_t>(b);
  return a0 < b0 + static_cast<uintptr_t>(bbytes) && b0 < a0 + static_cast<uintptr_t>(abytes);
}

}  // namespace

cudaError_t static_status_take(unsigned int* code) {
  *code = 0;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  char* base = nullptr;
  {
    std::lock_guard<std::mutex> lk(g_static_mu);
    if (dev < 0 || dev >= kMaxDevices || !g_static_ptr[dev]) return cudaSuccess;
    base = g_static_ptr[dev];
  }
  DevStatus* st = reinterpret_cast<DevStatus*>(base + kStaticBytes - kStatusBytes);
  DevStatus h{};
  e = cudaMemcpy(&h, st, sizeof h, cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return e;
  if (h.code || h.abort) e = cudaMemset(st, 0, sizeof(DevStatus));
  *code = h.code;
  return e;
}

}  // namespace lr

using namespace lr;

extern "C" lr_status lr_linear_decode_static(const void* X, const void* A, const void* B,
                                             const void* bias, void* Y, int64_t M, int64_t K,
                                             int64_t r, int64_t N, void* stream_) {
  if (M < 0 || K < 0 || r < 0 || N < 0) return LR_ERR_INVALID_ARG;
  if (M > kStaticMaxM || r > kStaticMaxR || N > kStaticMaxN || K > (int64_t(1) << 31) - 1)
    return LR_ERR_UNSUPPORTED;  // beyond what the static scratch holds
  if (M == 0 || N == 0) return LR_OK;
  if (!Y || (K > 0 && r > 0 && (!X || !A || !B))) return LR_ERR_INVALID_ARG;
  for (const void* p : {X, A, B, bias, static_cast<const void*>(Y)})
    if (p && (reinterpret_cast<uintptr_t>(p) & 1u)) return LR_ERR_INVALID_ARG;
  const int64_t ybytes = M * N * 2;
  if (overlaps(Y, ybytes, X, M * K * 2) || overlaps(Y, ybytes, A, K * r * 2) ||
      overlaps(Y, ybytes, B, r * N * 2) || overlaps(Y, ybytes, bias, N * 2))
    return LR_ERR_INVALID_ARG;
  cudaStream_t stream = static_cast<cudaStream_t>(stream_);
  char* scratch = nullptr;
  int sms = 0;
  lr_status st = static_setup(&scratch, &sms);
  if (st != LR_OK) return st;
  if (K == 0 || r == 0) {
    cudaError_t e = launch_fill_bias(Y, false, N, M, N,
                                     static_cast<const __nv_bfloat16*>(bias), stream);
    if (e != cudaSuccess) return fail(e);
    note_launches(1);
    return LR_OK;
  }
  const int m = static_cast<int>(M);
  const SkinnyPlan p1 = plan_skinny(m, K, r, sms);
  const SkinnyPlan p2 = plan_skinny(m, r, N, sms);
  if (p1.col_blocks > kStaticMaxCounters || p2.col_blocks > kStaticMaxCounters)
    return LR_ERR_UNSUPPORTED;
  float* acc1 = reinterpret_cast<float*>(scratch);
  float* acc2 = reinterpret_cast<float*>(scratch + kAcc1Bytes);
  unsigned int* ctr1 = reinterpret_cast<unsigned int*>(scratch + kAcc1Bytes + kAcc2Bytes);
  unsigned int* ctr2 = ctr1 + kStaticMaxCounters;
  float* T = reinterpret_cast<float*>(scratch + kAcc1Bytes + kAcc2Bytes + kCtrBytes);
  const int64_t ldt = round4(r), ldn = round4(N);
  // The array keeps the previous call's contents: clear the partial sums and
  // counters the kernels expect to start at zero.
  cudaError_t e = cudaMemsetAsync(acc1, 0, static_cast<size_t>(M * ldt * 4), stream);
  if (e == cudaSuccess) e = cudaMemsetAsync(acc2, 0, static_cast<size_t>(M * ldn * 4), stream);
  if (e == cudaSuccess) e = cudaMemsetAsync(ctr1, 0, kCtrBytes, stream);
  if (e != cudaSuccess) return fail(e);

  SkinnyArgs a{};
  a.M = m;
  // Bounded waits would report to a status word kept in the same array, with
  // the library's wait limit (lr_set_wait_limit_ns).  The decode kernels have
  // none today (their one wait, for the previous launch's grid, is resolved
  // by the hardware), so the word stays zero; lr_last_device_status reads it
  // all the same.
  a.wait = WaitCtl{reinterpret_cast<DevStatus*>(scratch + kStaticBytes - kStatusBytes),
                   wait_limit_ns()};
  // Phase 1: T = X·A (fp32).
  a.Kd = K;
  a.Nd = r;
  a.V = X;
  a.ldv = K;
  a.v_f32 = 0;
  a.W = static_cast<const __nv_bfloat16*>(A);
  a.ldw = r;
  a.w_lo = reinterpret_cast<uintptr_t>(A);
  a.w_hi = a.w_lo + static_cast<uintptr_t>(K * r * 2);
  a.acc = acc1;
  a.ld_acc = ldt;
  a.counters = ctr1;
  a.out_f32 = T;
  a.ld_out_f32 = ldt;
  e = launch_skinny(p1, a, stream);
  if (e != cudaSuccess) return fail(e);
  note_launches(1);
  // Phase 2: Y = T·B + bias.
  a.Kd = r;
  a.Nd = N;
  a.V = T;
  a.ldv = ldt;
  a.v_f32 = 1;
  a.W = static_cast<const __nv_bfloat16*>(B);
  a.ldw = N;
  a.w_lo = reinterpret_cast<uintptr_t>(B);
  a.w_hi = a.w_lo + static_cast<uintptr_t>(r * N * 2);
  a.acc = acc2;
  a.ld_acc = ldn;
  a.counters = ctr2;
  a.out_f32 = nullptr;
  a.ld_out_f32 = 0;
  a.out_bf16 = static_cast<__nv_bfloat16*>(Y);
  a.ld_out = N;
  a.bias = static_cast<const __nv_bfloat16*>(bias);
  e = launch_skinny(p2, a, stream, true);
  if (e != cudaSuccess) return fail(e);
  note_launches(1);
  return LR_OK;
}
