// noalloc.cu -- w4a16_gemv_noalloc: the decode GEMV for callers that cannot allocate device memory.
//
// Some callers have no way to hand this library a workspace: a plug-in whose host framework owns every
// device allocation and exposes no allocator to it, or a serving loop with a device-memory budget
// fixed at start-up that must not allocate per request.  For them the GEMV's split-K scratch lives in
// a file-scope __device__ array of kNoAllocScratchBytes (512 KiB), which every GPU that loads this library holds
// until the process exits.
//
// The host code below never passes the array's name to a kernel (in host code it is only a stand-in);
// it looks up the array's device address once per device with cudaGetSymbolAddress and passes that.
// The first call on each device performs this lookup, so make that first call before any stream
// capture.  Every call shares the one array and keeps the last call's contents, so each call whose
// plan uses the scratch clears the counters that must start at zero (cudaMemsetAsync, no allocation).  Calls on one device that
// overlap on the GPU (for example, issued on two streams) race on the array; the caller must order
// them.  Each device has its own copy of the array.
#include "common.cuh"
#include "internal.h"

namespace awq {

constexpr size_t kNoAllocScratchBytes = size_t(512) << 10;  // 512 KiB per device

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

static void* noalloc_scratch_address() {
  static void* cached[64] = {nullptr};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  if (cached[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess) return nullptr;
    cached[dev] = p;
  }
  return cached[dev];
}

}  // namespace awq

extern "C" awq_status w4a16_gemv_noalloc(const uint16_t* d_x, const uint32_t* d_qweight, const uint16_t* d_scales,
                                         const uint32_t* d_qzeros, uint16_t* d_y, int M, int N, int K, int g,
                                         awq_stream_t stream) {
  using namespace awq;
  awq_status st = check_linear(d_x, d_qweight, d_scales, d_qzeros, d_y, M, N, K, g);
  if (st != AWQ_OK) return st;
  const size_t need = gemv_workspace_bytes(M, N, K, g);
  if (need > kNoAllocScratchBytes) return AWQ_ERR_WORKSPACE;
  void* scratch = noalloc_scratch_address();
  if (scratch == nullptr) return AWQ_ERR_CUDA;
  unsigned* status = device_status_ptr();
  if (status == nullptr) return AWQ_ERR_CUDA;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  // Only a split plan touches the scratch; a plan without split row blocks needs no clearing (and a
  // memset between two GEMVs would keep the second from overlapping the first).
  if (need > 0 && cudaMemsetAsync(scratch, 0, kWorkspaceCounterBytes, s) != cudaSuccess) return AWQ_ERR_CUDA;
  LinearArgs a;
  a.x = d_x;
  a.qw = d_qweight;
  a.scales = d_scales;
  a.qzeros = d_qzeros;
  a.y = d_y;
  a.M = M;
  a.N = N;
  a.K = K;
  a.g = g;
  a.ws = scratch;
  a.ws_bytes = kNoAllocScratchBytes;
  a.status = status;
  a.st = s;
  return gemv_launch(a);
}
