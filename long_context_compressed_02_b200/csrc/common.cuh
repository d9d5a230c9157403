// Host-side helpers shared by the C-ABI translation units: last-error text,
// argument checks, and the per-unit device error words.
#pragma once
#include <cstdarg>
#include <cstdint>
#include <cstdio>
#include <utility>
#include <cuda_runtime.h>
#include "../../include/csa.h"

namespace csa {

csa_status_t fail(csa_status_t s, const char* fmt, ...);
void clear_error();

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

inline csa_status_t check_launch(const char* what) {
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return fail(CSA_ERR_CUDA, "%s: launch failed: %s", what, cudaGetErrorString(e));
  return CSA_OK;
}

// Programmatic dependent launch: a kernel launched this way may start while
// the previous kernel on the stream finishes; it must call pdl_wait() before
// touching anything that kernel (or an earlier one) writes, and does so first
// thing, which also keeps the chain of completions transitive.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
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
  return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

inline int num_sms() {
  int dev = 0, n = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n > 0 ? n : 148;
}

// Each translation unit that launches kernels owns a device error word and
// exposes a reader that returns and clears it (synchronous).
uint32_t read_clear_err_indexer();
uint32_t read_clear_err_attention();
uint32_t read_clear_err_proj();
uint32_t read_clear_err_compress();
uint32_t read_clear_err_selftest();

}  // namespace csa

#define CSA_REQUIRE(cond, ...)                                 \
  do {                                                         \
    if (!(cond)) return ::csa::fail(CSA_ERR_INVALID_ARG, __VA_ARGS__); \
  } while (0)
