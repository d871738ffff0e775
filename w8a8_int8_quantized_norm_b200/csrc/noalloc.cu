// noalloc.cu -- an entry point of the INT8 GEMM that never allocates.
//
// sq_w8a8_gemm_dequant asks its caller for a split-K workspace.  Some callers
// cannot provide one on demand: a plugin inside an inference engine whose
// enqueue path may not allocate (the engine owns the device memory, and
// cudaMalloc / cudaFree can synchronise the whole device), or a serving loop
// whose memory has been reserved up front by a framework's caching allocator.
// sq_w8a8_gemm_dequant_noalloc serves them: its split-K partial sums live in a
// fixed array of device memory that belongs to the library itself.
//
// The array is a file-scope __device__ variable, so every GPU that loads the
// library holds SQ_NOALLOC_SCRATCH_BYTES of it until the process exits.  Host
// code cannot use the array's name as a device address; the address is looked
// up with cudaGetSymbolAddress, with the device current, on the first call
// made on a device, and looked up again when that device's context is a new
// one (after cudaDeviceReset the module is loaded again and the array may
// move).
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>

#include "../../include/sq.h"
#include "sq_launch.h"

// The library's own split-K scratch: one copy per device, for the life of the
// process.  Nothing needs to start at zero (every partial sum a call reads was
// written earlier in the same call).
static __device__ __align__(256) unsigned char g_noalloc_scratch[SQ_NOALLOC_SCRATCH_BYTES];

namespace sq {
namespace {

constexpr int kMaxDevices = 64;

typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long*);

// Unique id of the current context (0 if the driver cannot tell): a context
// created after a device reset has a new one.
unsigned long long current_context_id() {
  static CtxGetCurrentFn get_current = nullptr;
  static CtxGetIdFn get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<CtxGetCurrentFn>(p);
    p = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<CtxGetIdFn>(p);
  });
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (!get_current || !get_id || get_current(&ctx) != CUDA_SUCCESS || !ctx ||
      get_id(ctx, &id) != CUDA_SUCCESS)
    return 0;
  return id;
}

// Device address of the scratch array for the current device: looked up on
// the first call on the device and again whenever its context has changed;
// nullptr if the lookup failed.
void* scratch_address() {
  static void* addr[kMaxDevices] = {};
  static unsigned long long ctx_of[kMaxDevices] = {};
  static std::mutex mu;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  const unsigned long long ctx = current_context_id();
  std::lock_guard<std::mutex> lock(mu);
  if (!addr[dev] || ctx != ctx_of[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess) return nullptr;
    addr[dev] = p;
    ctx_of[dev] = ctx;
  }
  return addr[dev];
}

}  // namespace
}  // namespace sq

extern "C" sq_status sq_w8a8_gemm_dequant_noalloc(const int8_t* Xq, const int8_t* Wq,
                                                  const float* x_scale, const float* w_scale,
                                                  int64_t M, int64_t N, int64_t K,
                                                  sq_epilogue epi, void* out, int64_t ldo,
                                                  int path_hint, int split_k, void* stream) {
  using namespace sq;
  if (M < 0 || N < 0 || K <= 0 || split_k < 0 || path_hint < 0 || path_hint > 3)
    return SQ_ERR_INVALID_ARG;
  if (M == 0 || N == 0) {
    return sq_w8a8_gemm_dequant(Xq, Wq, x_scale, w_scale, M, N, K, epi, out, ldo, nullptr, 0,
                                path_hint, split_k, stream);
  }
  const int sms = num_sms_current_device();
  GemmPlan plan = plan_gemm(M, N, K, path_hint, split_k, sms);
  if (plan.workspace_bytes > SQ_NOALLOC_SCRATCH_BYTES && split_k == 0 && plan.streamk) {
    // the automatic decode plan's stream-K slots do not fit: whole tiles, no scratch
    split_k = 1;
    plan = plan_gemm(M, N, K, path_hint, split_k, sms);
  }
  if (plan.workspace_bytes > SQ_NOALLOC_SCRATCH_BYTES) return SQ_ERR_WORKSPACE;
  // every non-empty call sets the address up (cached), whether or not its own
  // plan needs scratch, so that the first call on a device does it
  void* scratch = scratch_address();
  if (!scratch) return SQ_ERR_CUDA;
  if (plan.workspace_bytes == 0) scratch = nullptr;
  // the allocating entry point does the remaining checks and the launches;
  // the library's own array stands in for the caller's workspace
  return sq_w8a8_gemm_dequant(Xq, Wq, x_scale, w_scale, M, N, K, epi, out, ldo, scratch,
                              scratch ? SQ_NOALLOC_SCRATCH_BYTES : 0, path_hint, split_k, stream);
}
