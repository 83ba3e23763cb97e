// internal.h -- declarations shared by the library's translation units (not installed).
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "../../include/awq_w4a16.h"

namespace awq {

// The first kWorkspaceCounterBytes of every workspace hold per-tile counters (zero between calls);
// split-K partials follow.  A fixed size keeps the counters in place whatever shape used the
// workspace before.
constexpr size_t kWorkspaceCounterBytes = 64 * 1024;

int num_sms();  // SM count of the current device (cached per device)

// Host-side argument checks shared by the linear-layer entry points (AWQ_OK when valid).
awq_status check_linear(const uint16_t* x, const uint32_t* qw, const uint16_t* sc, const uint32_t* qz,
                        const uint16_t* y, int M, int N, int K, int g);

// Launch with programmatic stream serialization, so the kernel may start while the previous kernel
// on the stream drains; the kernels order their dependent accesses with griddepcontrol.wait.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                       Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

// kernels (each launcher returns AWQ_OK or an error; arguments are validated by the caller)
awq_status prep_act_scale_launch(const uint16_t* xcal, int R, int K, uint16_t* s, cudaStream_t st);
awq_status prep_inv_scale_launch(const uint16_t* x, const uint16_t* s, int M, int K, uint16_t* xp,
                                 cudaStream_t st);
// Pack N rows of K channels at group size g.  W2 == NULL: row n of the packed weight is W[n].  W2 != NULL
// (gate|up, N = 2 * NI, NI % 16 == 0): row 32j + i of the packed weight is W[16j + i] for i < 16 and
// W2[16j + i - 16] for i >= 16.
awq_status pack_launch(const uint16_t* W, const uint16_t* W2, const uint16_t* s, int N, int K, int g, uint32_t* qw,
                       uint16_t* scales, uint32_t* qz, cudaStream_t st, int w_bit = 4, int storage_bits = 4);

// One linear-layer call as the kernels see it.
struct LinearArgs {
  const uint16_t* x = nullptr;
  const uint32_t* qw = nullptr;
  const uint16_t* scales = nullptr;
  const uint32_t* qzeros = nullptr;
  uint16_t* y = nullptr;
  int M = 0, N = 0, K = 0, g = 128;
  int epi = 0;  // 0: y [M][N]; 1: gate|up packed by pack_launch with W2, y [M][N/2] = silu(gate) * up
  int bits = 4;  // code layout: 4 (the 4-bit layout) or 3 (the packed 3-bit layout; GEMV only, no epi / inv_s)
  void* ws = nullptr;
  size_t ws_bytes = 0;
  unsigned* status = nullptr;
  cudaStream_t st = nullptr;
  const void* pf = nullptr;        // GEMV only: optional L2 prefetch of another buffer (16-B aligned, size % 16 == 0)
  size_t pf_bytes = 0;
  const uint16_t* inv_s = nullptr;  // GEMV only: x holds raw activations, the kernel uses x' = fp16(x / s) (the
                                    // same bits as awq_apply_inv_scale); AWQ_ERR_UNSUPPORTED when x does not
                                    // fit in shared memory
};
size_t gemv_workspace_bytes(int M, int N, int K, int g);
awq_status gemv_launch(const LinearArgs& a);
size_t gemm_workspace_bytes(int M, int N, int K, int g);
awq_status gemm_launch(const LinearArgs& a);
unsigned* device_status_ptr();  // address of the device status word on the current device
// GPTQ (gptq.cu): workspace bytes and the launch sequence (arguments validated by the caller).
size_t gptq_workspace_bytes(int N, int K);
awq_status gptq_launch(const uint16_t* W, const uint16_t* xcal, int N, int K, int R, int g, double damp,
                       uint32_t* qw, uint16_t* scales, uint32_t* qz, void* ws, size_t ws_bytes, unsigned* status,
                       cudaStream_t st);
// AWQ scale search (search.cu): workspace bytes and the launch sequence (arguments validated by the caller).
size_t search_workspace_bytes(int N, int K, int R, int g);
awq_status search_launch(const uint16_t* W, const uint16_t* xcal, int N, int K, int R, int g, int n_grid,
                         double* losses, uint16_t* s_out, int* best_out, void* ws, size_t ws_bytes,
                         unsigned* status, cudaStream_t st);

}  // namespace awq
