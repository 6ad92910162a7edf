// vsl_test_probes.cu - test-only entry points of libvsl_test.so (the library's
// objects plus this file; never part of libvsl.so).
//
// vsl_test_div_mismatches compares the sampler's fast quotient x = fl(l / T)
// (scale_x_fast, vsl_math.cuh) bit for bit with CUDA's IEEE round-to-nearest
// division __fdiv_rn over every float32 bit pattern l in [lo, hi] that lies in
// the fast path's domain (zero, or 2^-60 <= |l| <= 2^100; a zero quotient of
// either sign counts as zero) for each T given.
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
#include "../../vocab_sharded_logits_b200/csrc/vsl_math.cuh"
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

// One T per grid row; threads stride over the bit patterns.  Mismatches are
// counted; the smallest (T index, bits) pair is kept as (T index << 32 | bits).
__global__ void div_check_kernel(const float* Ts, uint32_t lo, uint32_t hi, unsigned long long* count,
                                 unsigned long long* first) {
  const float T = Ts[blockIdx.y];
  const unsigned long long span = static_cast<unsigned long long>(hi) - lo + 1ull;
  const unsigned long long stride = static_cast<unsigned long long>(gridDim.x) * blockDim.x;
  unsigned long long bad = 0;
  for (unsigned long long k = static_cast<unsigned long long>(blockIdx.x) * blockDim.x + threadIdx.x; k < span;
       k += stride) {
    const uint32_t bits = lo + static_cast<uint32_t>(k);
    const float l = __uint_as_float(bits);
    const float al = fabsf(l);
    if (!(al <= 0x1p100f) || (al != 0.0f && al < 0x1p-60f)) continue;  // outside the fast path's domain
    const float a = vsl::scale_x_fast(l, T, __frcp_rn(T));
    const float b = __fdiv_rn(l, T);
    if (__float_as_uint(a) != __float_as_uint(b) && !(a == 0.0f && b == 0.0f)) {
      ++bad;
      atomicMin(first, (static_cast<unsigned long long>(blockIdx.y) << 32) | bits);
    }
  }
  if (bad) atomicAdd(count, bad);
}

}  // namespace

extern "C" __attribute__((visibility("default"))) vsl_status vsl_test_div_mismatches(
    const float* Ts_host, int nT, uint32_t lo, uint32_t hi, unsigned long long* count_out,
    unsigned long long* first_out) {
  if (Ts_host == nullptr || nT <= 0 || nT > 65535 || hi < lo || count_out == nullptr || first_out == nullptr)
    return VSL_ERR_INVALID_ARG;
  float* Ts = nullptr;
  unsigned long long* res = nullptr;
  if (cudaMalloc(&Ts, sizeof(float) * nT) != cudaSuccess) return VSL_ERR_CUDA;
  if (cudaMalloc(&res, 2 * sizeof(unsigned long long)) != cudaSuccess) {
    cudaFree(Ts);
    return VSL_ERR_CUDA;
  }
  const unsigned long long init[2] = {0ull, ~0ull};
  cudaError_t e = cudaMemcpy(Ts, Ts_host, sizeof(float) * nT, cudaMemcpyHostToDevice);
  if (e == cudaSuccess) e = cudaMemcpy(res, init, sizeof(init), cudaMemcpyHostToDevice);
  if (e == cudaSuccess) {
    div_check_kernel<<<dim3(1184, nT), 256>>>(Ts, lo, hi, res, res + 1);
    e = cudaGetLastError();
  }
  unsigned long long out[2] = {0ull, 0ull};
  if (e == cudaSuccess) e = cudaMemcpy(out, res, sizeof(out), cudaMemcpyDeviceToHost);
  cudaFree(Ts);
  cudaFree(res);
  if (e != cudaSuccess) return VSL_ERR_CUDA;
  *count_out = out[0];
  *first_out = out[1];
  return VSL_OK;
}

extern "C" __attribute__((visibility("default"))) vsl_status vsl_test_wait_probe(long long limit_cycles, int arrive,
                                                                                 void* stream) {
  if (limit_cycles <= 0 || limit_cycles > 4000000000LL) return VSL_ERR_INVALID_ARG;
  uint32_t* err = vsl::device_error_word();
  if (err == nullptr) return VSL_ERR_CUDA;
  wait_probe_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(err, limit_cycles, arrive);
  return cudaGetLastError() == cudaSuccess ? VSL_OK : VSL_ERR_CUDA;
}

extern "C" __attribute__((visibility("default"))) uint32_t vsl_test_probe_site(void) { return vsl::kErrWaitProbe; }
