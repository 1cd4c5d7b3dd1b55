// ep_load_matrix_static: the load matrix L[r][e] of one layer for callers that
// cannot allocate device memory.
//
// Some callers cannot call cudaMalloc on this path: serving engines that
// reserve (nearly) all device memory up front and hand out nothing more,
// embedded C callers without an allocator of their own, and hot loops where an
// allocation would synchronise the device.  For them this entry point keeps its
// only scratch — the per-sub-chunk expert counts — in a file-scope device
// array of fixed size, so a call allocates nothing; the caller still passes
// the inputs and outputs.
//
// The array is module state: every GPU that loads this library holds it (4 MiB)
// until the process exits.  Every call on a device shares it and it keeps the
// last call's contents; each call overwrites every entry it later reads, so
// nothing in it has to start at zero.  Calls whose executions overlap on the
// GPU (two streams, or two host threads) race on the array: serialise them.
//
// Host code cannot use the array's name as a device address, so the address is
// looked up with cudaGetSymbolAddress once per device and cached together with
// the unique id of the CUDA context it belongs to.  After a device reset the
// module is loaded again in a new context, possibly at another address; the
// next call sees the new context id and looks the address up again.
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>

#include "ep_internal.cuh"

namespace {

constexpr int kWarps = 8;
constexpr int kMaxDevices = 64;
constexpr unsigned kFull = 0xffffffffu;

// Scratch of the static variant: [R][ceil(T/128)][E] int32 sub-chunk counts.
static __device__ __align__(256) int32_t g_load_scratch[EP_LOAD_STATIC_MAX_SCRATCH];

std::mutex g_setup_mu;

struct CachedAddress {
  int32_t* addr = nullptr;
  unsigned long long ctx_id = 0;  // unique id of the context the address belongs to
};
CachedAddress g_scratch_addr[kMaxDevices];

// Driver entry points, fetched through the runtime (no link against libcuda).
using CtxGetCurrentFn = CUresult (*)(CUcontext*);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long*);
CtxGetCurrentFn g_ctx_get_current = nullptr;
CtxGetIdFn g_ctx_get_id = nullptr;
bool g_driver_fns_tried = false;

// Unique id of the current context (0 if it cannot be read; ids are never 0).
unsigned long long current_context_id() {
  if (!g_driver_fns_tried) {
    g_driver_fns_tried = true;
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_ctx_get_current = reinterpret_cast<CtxGetCurrentFn>(f);
    f = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_ctx_get_id = reinterpret_cast<CtxGetIdFn>(f);
  }
  if (!g_ctx_get_current || !g_ctx_get_id) return 0;
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (g_ctx_get_current(&ctx) != CUDA_SUCCESS || !ctx) return 0;
  if (g_ctx_get_id(ctx, &id) != CUDA_SUCCESS) return 0;
  return id;
}

// Device address of g_load_scratch on the current device, looked up once per
// device and context (host code may not use the array's name as an address).
cudaError_t scratch_address(int32_t** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_setup_mu);
  CachedAddress& c = g_scratch_addr[dev];
  const unsigned long long id = c.addr ? current_context_id() : 0;
  if (!c.addr || id == 0 || id != c.ctx_id) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_load_scratch);  // makes the device's context current
    if (e != cudaSuccess) return e;
    c.addr = static_cast<int32_t*>(p);
    c.ctx_id = current_context_id();
  }
  *out = c.addr;
  return cudaSuccess;
}

// Variant of the plan's histogram kernel: one warp per sub-chunk of 128 tokens
// of one source rank; lanes with equal ids are grouped with match.any and the
// group leader adds the group size to the warp's shared histogram, which is
// then written to the sub-chunk's row of the static scratch.
__global__ void __launch_bounds__(kWarps * 32)
k_hist_static(const int32_t* __restrict__ ids, int R, int E, int K, int T, int nsub,
              int32_t* __restrict__ scratch, int32_t* __restrict__ status) {
  extern __shared__ int32_t sm_hist[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int gw = blockIdx.x * kWarps + warp;
  if (gw >= R * nsub) return;
  int32_t* hist = sm_hist + warp * E;
  for (int e = lane; e < E; e += 32) hist[e] = 0;
  __syncwarp();
  const int r = gw / nsub, sub = gw - r * nsub;
  const int t0 = sub * ep::kSubT, t1 = min(T, t0 + ep::kSubT);
  const int32_t* src = ids + (int64_t)r * T * K;
  const int a1 = t1 * K;
  int bad = 0;
  for (int a = t0 * K; a < a1; a += 32) {
    const int idx = a + lane;
    int v = idx < a1 ? __ldg(src + idx) : -1;
    if (idx < a1 && (v < 0 || v >= E)) { bad = 1; v = -1; }
    const unsigned peers = __match_any_sync(kFull, v);
    if (v >= 0 && lane == __ffs(peers) - 1) hist[v] += __popc(peers);
    __syncwarp();
  }
  int32_t* row = scratch + (int64_t)gw * E;
  for (int e = lane; e < E; e += 32) row[e] = hist[e];
  if (status && __any_sync(kFull, bad) && lane == 0) atomicOr(status, EP_DEV_BAD_ID);
}

// L[r][e] = sum over the rank's sub-chunks of the scratch counts.
__global__ void __launch_bounds__(256)
k_load_static(int R, int E, int nsub, const int32_t* __restrict__ scratch, int32_t* __restrict__ load) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= R * E) return;
  const int r = i / E, e = i - r * E;
  const int32_t* p = scratch + (int64_t)r * nsub * E + e;
  int acc = 0;
  for (int sub = 0; sub < nsub; ++sub) acc += p[(int64_t)sub * E];
  load[i] = acc;
}

}  // namespace

extern "C" ep_status_t ep_load_matrix_static(int32_t R, int32_t E, int32_t K, int32_t T,
                                             const int32_t* d_topk_ids, int32_t* d_load,
                                             int32_t* d_status, void* stream) {
  if (R < 1 || E < 1 || K < 1 || T < 0) return EP_ERR_INVALID_ARGUMENT;
  if (E > ep::kMaxE || K > ep::kMaxK || (int64_t)R * T * K >= (int64_t)INT32_MAX ||
      (int64_t)R * E >= (int64_t)INT32_MAX)
    return EP_ERR_UNSUPPORTED;
  const int nsub = (T + ep::kSubT - 1) / ep::kSubT;
  if ((int64_t)R * nsub * E > (int64_t)EP_LOAD_STATIC_MAX_SCRATCH) return EP_ERR_UNSUPPORTED;
  if (!d_load || (T > 0 && !d_topk_ids)) return EP_ERR_INVALID_ARGUMENT;
  int32_t* scratch = nullptr;
  if (scratch_address(&scratch) != cudaSuccess) return EP_ERR_CUDA;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (d_status && cudaMemsetAsync(d_status, 0, sizeof(int32_t), st) != cudaSuccess)
    return EP_ERR_CUDA;
  // each launch's own return code: an error left pending by unrelated earlier
  // work is neither reported here nor cleared
  const int nwarps = R * nsub;
  if (nwarps > 0) {
    void* args[] = {&d_topk_ids, &R, &E, &K, &T, const_cast<int*>(&nsub), &scratch, &d_status};
    if (cudaLaunchKernel(reinterpret_cast<const void*>(k_hist_static),
                         dim3((unsigned)((nwarps + kWarps - 1) / kWarps)), dim3(kWarps * 32), args,
                         sizeof(int32_t) * kWarps * E, st) != cudaSuccess)
      return EP_ERR_CUDA;
  }
  const int32_t* cscratch = scratch;
  void* args2[] = {&R, &E, const_cast<int*>(&nsub), &cscratch, &d_load};
  if (cudaLaunchKernel(reinterpret_cast<const void*>(k_load_static),
                       dim3((unsigned)(((int64_t)R * E + 255) / 256)), dim3(256), args2, 0, st) !=
      cudaSuccess)
    return EP_ERR_CUDA;
  return EP_OK;
}
