// Status reporting shared by all entry points of libcsa.so, and the self-test
// of the bounded on-chip waits.
#include <string>
#include "common.cuh"
#include "tc.cuh"

namespace csa {

static thread_local std::string g_last_error;

csa_status_t fail(csa_status_t s, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return s;
}

void clear_error() { g_last_error.clear(); }

static __device__ uint32_t g_err_selftest;

uint32_t read_clear_err_selftest() {
  uint32_t v = 0, z = 0;
  cudaMemcpyFromSymbol(&v, g_err_selftest, sizeof(v));
  cudaMemcpyToSymbol(g_err_selftest, &z, sizeof(z));
  return v;
}

// One thread waits on an mbarrier phase that nothing completes, through the
// same bounded wait the kernels use, with the given limit; the expiry is
// recorded in the device error word and the kernel returns.
__global__ void selftest_wait_kernel(uint64_t limit_ns) {
  __shared__ uint64_t bar;
  mbar_init(&bar, 1);
  fence_mbar_init();
  mbar_wait(&bar, 0, &g_err_selftest, limit_ns);
}

}  // namespace csa

extern "C" int csa_abi_version(void) { return 1; }

extern "C" const char* csa_status_string(csa_status_t s) {
  switch (s) {
    case CSA_OK: return "CSA_OK";
    case CSA_ERR_INVALID_ARG: return "CSA_ERR_INVALID_ARG";
    case CSA_ERR_UNSUPPORTED: return "CSA_ERR_UNSUPPORTED";
    case CSA_ERR_WORKSPACE: return "CSA_ERR_WORKSPACE";
    case CSA_ERR_CUDA: return "CSA_ERR_CUDA";
    case CSA_ERR_TIMEOUT: return "CSA_ERR_TIMEOUT";
    case CSA_ERR_DEVICE: return "CSA_ERR_DEVICE";
  }
  return "CSA_UNKNOWN_STATUS";
}

extern "C" const char* csa_last_error(void) { return csa::g_last_error.c_str(); }

extern "C" const char* csa_get_last_error_string(void) { return csa_last_error(); }

extern "C" size_t csa_workspace_size(int n_seq, int T, int64_t cap, int k, int H, int D, int n_split) {
  const size_t a = csa_index_topk_workspace(n_seq, T, cap, k);
  const size_t b = n_split > 1 ? csa_fused_attention_workspace(n_seq, T, H, D, n_split) : 0;
  return a > b ? a : b;
}

extern "C" csa_status_t csa_check_device_error(cudaStream_t stream) {
  cudaError_t e = cudaStreamSynchronize(stream);
  if (e != cudaSuccess)
    return csa::fail(CSA_ERR_CUDA, "csa_check_device_error: stream sync failed: %s", cudaGetErrorString(e));
  uint32_t w = csa::read_clear_err_indexer() | csa::read_clear_err_attention() | csa::read_clear_err_proj() |
               csa::read_clear_err_compress() | csa::read_clear_err_selftest();
  if (w & 1u) return csa::fail(CSA_ERR_TIMEOUT, "a bounded on-chip wait expired (device error word 0x%x)", w);
  if (w) return csa::fail(CSA_ERR_DEVICE, "a kernel recorded an out-of-range gather index (device error word 0x%x)", w);
  return CSA_OK;
}

extern "C" csa_status_t csa_selftest_wait_timeout(uint64_t limit_ns, cudaStream_t stream) {
  csa::clear_error();
  CSA_REQUIRE(limit_ns >= 1000 && limit_ns <= 100000000ull, "csa_selftest_wait_timeout: limit_ns must be in [1 us, 100 ms]");
  csa::selftest_wait_kernel<<<1, 1, 0, stream>>>(limit_ns);
  return csa::check_launch("csa_selftest_wait_timeout");
}
