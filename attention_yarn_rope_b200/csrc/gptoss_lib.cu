// gptoss_lib.cu -- the C ABI of libgptoss_attn (declared in include/gptoss.h).
// One translation unit: the status and wait-limit entry points are here; the
// RoPE / prefill, decode and backward entry points are in fwd_host.cuh,
// decode_host.cuh and bwd_host.cuh, included at the end, and the kernels in
// the headers those include.
// Every entry point validates on the host, encodes its TMA descriptors and
// launches asynchronously on the caller's stream; nothing is allocated.

#include <cuda_runtime.h>

#include "gptoss.h"
#include "host_util.cuh"
#include "sm100_ptx.cuh"

using namespace gptoss;

namespace {

// One mbarrier that nothing ever arrives at: the kernel's bounded wait must
// give up and record GPTOSS_ERR_TIMEOUT.  Exercises the device failure path.
__global__ void wait_timeout_probe_kernel(uint64_t limit_ns, int* result) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
  }
  __syncthreads();
  const bool ok = mbar_wait(&bar, 0, limit_ns);
  if (threadIdx.x == 0) *result = ok ? 1 : 0;
}

}  // namespace

extern "C" {

const char* gptoss_status_string(gptoss_status s) {
  switch (s) {
    case GPTOSS_OK: return "GPTOSS_OK";
    case GPTOSS_ERR_INVALID_ARG: return "GPTOSS_ERR_INVALID_ARG";
    case GPTOSS_ERR_UNSUPPORTED: return "GPTOSS_ERR_UNSUPPORTED";
    case GPTOSS_ERR_CUDA: return "GPTOSS_ERR_CUDA";
    case GPTOSS_ERR_TIMEOUT: return "GPTOSS_ERR_TIMEOUT";
  }
  return "GPTOSS_ERR_UNKNOWN";
}

gptoss_status gptoss_set_wait_limit(uint32_t microseconds) {
  wait_limit_ns() = microseconds == 0 ? 2000000000ull : static_cast<uint64_t>(microseconds) * 1000ull;
  return GPTOSS_OK;
}

gptoss_status gptoss_read_device_status(int32_t* status_out, int32_t reset, struct CUstream_st* stream) {
  if (status_out == nullptr) return GPTOSS_ERR_INVALID_ARG;
  cudaStream_t st = as_stream(stream);
  int v = 0;
  if (cudaMemcpyFromSymbolAsync(&v, g_device_status, sizeof(int), 0, cudaMemcpyDeviceToHost, st) != cudaSuccess)
    return GPTOSS_ERR_CUDA;
  if (reset) {
    static const int zero = 0;
    if (cudaMemcpyToSymbolAsync(g_device_status, &zero, sizeof(int), 0, cudaMemcpyHostToDevice, st) != cudaSuccess)
      return GPTOSS_ERR_CUDA;
  }
  if (cudaStreamSynchronize(st) != cudaSuccess) return GPTOSS_ERR_CUDA;
  *status_out = v;
  return GPTOSS_OK;
}

gptoss_status gptoss_selftest_wait_timeout(uint32_t limit_us, int32_t* result_dev, struct CUstream_st* stream) {
  if (result_dev == nullptr || limit_us == 0 || limit_us > 1000000) return GPTOSS_ERR_INVALID_ARG;
  wait_timeout_probe_kernel<<<1, 32, 0, as_stream(stream)>>>(static_cast<uint64_t>(limit_us) * 1000ull,
                                                             reinterpret_cast<int*>(result_dev));
  return check_launch();
}

}  // extern "C"

// the RoPE and prefill entry points (self-attention and the block form)
#include "fwd_host.cuh"
// the log-sum-exp merge of key-block results
#include "attn_merge.cuh"
// the q / k / v projections with RoPE in the GEMM epilogue
#include "qkv_rope.cuh"
// the decode entry points (split-KV decode, paged cache, append, no-alloc)
#include "decode_host.cuh"
// the backward entry points
#include "bwd_host.cuh"
