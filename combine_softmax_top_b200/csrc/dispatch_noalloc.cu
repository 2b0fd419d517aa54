// moe_dispatch_noalloc: the one-pass dispatch for callers that cannot give the
// library a workspace.
//
// Some callers may not allocate device memory at the point where they
// dispatch: an inference engine that reserves all device memory in its own
// pool at start-up and forbids cudaMalloc on the serving path (an allocation
// there would fail or throw the pool's accounting off), or a latency-bound
// decode loop where a cudaMalloc would stall the device. This entry point
// needs nothing from them beyond the inputs and outputs of moe_dispatch: the
// counters, sentinels and tile ring the dispatch kernel keeps between its CTAs
// live in a fixed array in device memory that the library owns, below.
//
// The array is a file-scope __device__ variable of kNoAllocScratchBytes, so
// every GPU that loads the library holds it until the process exits. Host
// code cannot use its name as a device address, so the first call on each
// device looks the address up with cudaGetSymbolAddress (with that device
// current) and keeps it; that first call must therefore happen before any
// stream capture. All calls share the array: each call first clears the part
// the kernel needs zeroed, and calls that overlap on the GPU (other streams,
// other threads) race on it.
#include <mutex>

#include "moe_internal.cuh"

namespace moe {
namespace {

constexpr size_t kNoAllocScratchBytes = 4u << 20;   // 4 MiB
constexpr int kMaxDevices = 64;

static __device__ __align__(256) uint8_t g_dispatch_scratch[kNoAllocScratchBytes];

std::mutex g_mu;
void* g_scratch_addr[kMaxDevices];   // device address of g_dispatch_scratch, per device

// Device address of the scratch array on the current device (looked up once).
cudaError_t scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_scratch_addr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_dispatch_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return cudaSuccess;
}

// Zero the header, both counter sets, the sentinels and the ring; epoch 1.
__global__ void clear_scratch_kernel(uint32_t* words, size_t n) {
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x)
    words[i] = (i == 0) ? 1u : 0u;   // word 0 is Header::epoch_next
}

}  // namespace
}  // namespace moe

using namespace moe;

extern "C" moe_status moe_dispatch_noalloc(const moe_shape* shape, const void* x, const int32_t* topk_idx,
                                           const moe_dispatch_bufs* bufs, moe_stream_t stream) {
  moe_status st = check_shape(shape);
  if (st != MOE_OK) return st;
  // compact windows need the counting pass's words in a workspace
  if (shape->flags & MOE_FLAG_COMPACT) return MOE_ERR_UNSUPPORTED;
  if (shape->T > 0 && (!x || !topk_idx)) return MOE_ERR_INVALID_ARG;
  if (!aligned16(x)) return MOE_ERR_INVALID_ARG;
  Ctx c;
  c.s = effective_shape(*shape);
  c.routed_E = shape->E;
  c.routed_k = shape->topk;
  c.shared = (shape->flags & MOE_FLAG_SHARED_EXPERT) ? 1 : 0;
  st = check_bufs(&c.s, bufs, false);
  if (st != MOE_OK) return st;
  c.L = make_layout(c.s);
  // counters, sentinels and ring only: the scale atoms for the tensor-core
  // FFN are not written on this path
  if (c.L.off_xsf > kNoAllocScratchBytes) return MOE_ERR_INVALID_ARG;   // too big for the fixed scratch
  void* scratch = nullptr;
  if (scratch_address(&scratch) != cudaSuccess) return MOE_ERR_CUDA;
  c.ws = ws_view(scratch, c.L);
  c.stream = (cudaStream_t)stream;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&c.num_sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return MOE_ERR_CUDA;
  const size_t words = c.L.off_xsf / 4;
  clear_scratch_kernel<<<(unsigned)std::min<size_t>((words + 255) / 256, 256), 256, 0, c.stream>>>(
      (uint32_t*)scratch, words);
  if (cudaGetLastError() != cudaSuccess) return MOE_ERR_CUDA;
  return launch_dispatch(c, x, topk_idx, *bufs, /*write_sf=*/false) == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}
