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
int32_t* g_scratch_addr[kMaxDevices] = {};

// Device address of g_load_scratch on the current device, looked up once per
// device (host code may not use the array's name as an address).
cudaError_t scratch_address(int32_t** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_setup_mu);
  if (!g_scratch_addr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_load_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_addr[dev] = static_cast<int32_t*>(p);
  }
  *out = g_scratch_addr[dev];
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
  if (E > ep::kMaxE || K > ep::kMaxK || (int64_t)R * T * K >= (int64_t)INT32_MAX)
    return EP_ERR_UNSUPPORTED;
  const int nsub = (T + ep::kSubT - 1) / ep::kSubT;
  if ((int64_t)R * nsub * E > (int64_t)EP_LOAD_STATIC_MAX_SCRATCH) return EP_ERR_UNSUPPORTED;
  if (!d_load || (T > 0 && !d_topk_ids)) return EP_ERR_INVALID_ARGUMENT;
  int32_t* scratch = nullptr;
  if (scratch_address(&scratch) != cudaSuccess) return EP_ERR_CUDA;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (d_status && cudaMemsetAsync(d_status, 0, sizeof(int32_t), st) != cudaSuccess)
    return EP_ERR_CUDA;
  const int nwarps = R * nsub;
  if (nwarps > 0)
    k_hist_static<<<(nwarps + kWarps - 1) / kWarps, kWarps * 32, sizeof(int32_t) * kWarps * E, st>>>(
        d_topk_ids, R, E, K, T, nsub, scratch, d_status);
  k_load_static<<<(R * E + 255) / 256, 256, 0, st>>>(R, E, nsub, scratch, d_load);
  return cudaGetLastError() == cudaSuccess ? EP_OK : EP_ERR_CUDA;
}
