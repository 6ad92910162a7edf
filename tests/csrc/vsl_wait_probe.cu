// vsl_wait_probe.cu - test-only entry point of libvsl_test.so (the library's
// objects plus this file; never part of libvsl.so).
//
// vsl_test_wait_probe launches one warp that initialises an mbarrier expecting
// one arrival and waits on its first phase with the library's bounded wait and
// a caller-chosen limit.  With arrive == 0 nothing ever arrives: no copy is in
// flight and no other thread touches the barrier, so the wait runs out after
// `limit_cycles` SM clock cycles, the kernel ORs kErrWaitProbe into the
// library's device error word and returns.  With arrive != 0 the waiting thread
// arrives first and the wait completes at once.  The host then reads (and
// clears) the word with vsl_device_error, as after a product kernel's wait.
#include <cuda_runtime.h>

#include <cstdint>

#include "../../vocab_sharded_logits_b200/csrc/vsl_internal.h"
#include "../../vocab_sharded_logits_b200/csrc/vsl_ptx.cuh"

namespace {

__global__ void wait_probe_kernel(uint32_t* err, long long limit, int arrive) {
  __shared__ __align__(8) unsigned long long bar;
  if (threadIdx.x == 0) {
    vsl::mbar_init(vsl::smem_u32(&bar), 1);
    vsl::fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    if (arrive) {
      asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(vsl::smem_u32(&bar)) : "memory");
    }
    if (!vsl::mbar_wait_bounded_for(vsl::smem_u32(&bar), 0, limit)) atomicOr(err, vsl::kErrWaitProbe);
  }
}

}  // namespace

extern "C" __attribute__((visibility("default"))) vsl_status vsl_test_wait_probe(long long limit_cycles, int arrive,
                                                                                 void* stream) {
  if (limit_cycles <= 0 || limit_cycles > 4000000000LL) return VSL_ERR_INVALID_ARG;
  uint32_t* err = vsl::device_error_word();
  if (err == nullptr) return VSL_ERR_CUDA;
  wait_probe_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(err, limit_cycles, arrive);
  return cudaGetLastError() == cudaSuccess ? VSL_OK : VSL_ERR_CUDA;
}

extern "C" __attribute__((visibility("default"))) uint32_t vsl_test_probe_site(void) { return vsl::kErrWaitProbe; }
