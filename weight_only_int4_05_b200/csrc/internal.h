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
awq_status pack_launch(const uint16_t* W, const uint16_t* s, int N, int K, uint32_t* qw, uint16_t* scales,
                       uint32_t* qz, cudaStream_t st);
size_t gemv_workspace_bytes(int M, int N, int K);
// pf / pf_bytes: optional L2 prefetch of another buffer while the GEMV runs (16-byte aligned, size a
// multiple of 16; NULL / 0 for none).
// inv_s: optional AWQ scale; when given, x holds raw activations and the kernel uses x' = fp16(x / s) (the
// same bits as awq_apply_inv_scale), staged in shared memory (AWQ_ERR_UNSUPPORTED when it does not fit).
awq_status gemv_launch(const uint16_t* x, const uint32_t* qw, const uint16_t* scales, const uint32_t* qzeros,
                       uint16_t* y, int M, int N, int K, void* ws, size_t ws_bytes, unsigned* dev_status,
                       cudaStream_t st, const void* pf = nullptr, size_t pf_bytes = 0,
                       const uint16_t* inv_s = nullptr);
unsigned* device_status_ptr();  // address of the device status word on the current device
size_t gemm_workspace_bytes(int M, int N, int K);
awq_status gemm_launch(const uint16_t* x, const uint32_t* qw, const uint16_t* scales, const uint32_t* qzeros,
                       uint16_t* y, int M, int N, int K, void* ws, size_t ws_bytes, unsigned* dev_status,
                       cudaStream_t st);

}  // namespace awq
