// vsl_verify.cu - speculative verification of deterministic drafts over the
// rows one vsl_sample call drew.
//
// "Qwen4Exp batch-sharded sampling: inside vLLM PR #61018" (orcarouter.ai
// blog): the sampler's batch x (speculative tokens + 1) x vocab rows (section
// "batch-sharded sampling in one paragraph", which also leaves sharded draft
// logits for later) and the acceptance length its measurements report
// (section "the 1.5 % estimate").  Request q's row j holds the target's draw
// t_j for position j; its drafts d_0 .. d_{spec-1} are point masses.  Draft j
// is accepted while t_j == d_j (t_j >= 0); the request emits the accepted
// drafts, then t_a (the correction, or the bonus token after spec
// acceptances), then -1.  With the draw keyed by (seed, request, position,
// token) this is the rejection rule for a point-mass draft: d_j is accepted
// with probability p(d_j), and a rejected position emits a token distributed
// as p without d_j.
//
// One thread per request: a few compares per row, bound by launch latency.
#include <cuda_runtime.h>

#include <cstdint>

#include "vsl_internal.h"

namespace vsl {

namespace {

__global__ void verify_kernel(const int32_t* __restrict__ t, const float* __restrict__ tlp,
                              const int32_t* __restrict__ d, int requests, int spec, int32_t* __restrict__ out,
                              float* __restrict__ olp, int32_t* __restrict__ accepted) {
  const int q = blockIdx.x * blockDim.x + threadIdx.x;
  if (q >= requests) return;
  const size_t rb = static_cast<size_t>(q) * (spec + 1);
  const size_t db = static_cast<size_t>(q) * spec;
  int a = 0;
  while (a < spec) {
    const int32_t tv = t[rb + a];
    if (tv < 0 || tv != d[db + a]) break;
    out[rb + a] = tv;
    if (olp != nullptr) olp[rb + a] = tlp[rb + a];
    ++a;
  }
  out[rb + a] = t[rb + a];
  if (olp != nullptr) olp[rb + a] = tlp[rb + a];
  for (int j = a + 1; j <= spec; ++j) {
    out[rb + j] = -1;
    if (olp != nullptr) olp[rb + j] = __int_as_float(0x7FC00000);
  }
  accepted[q] = a;
}

}  // namespace

cudaError_t launch_verify(const int32_t* token_ids, const float* token_logprob, const int32_t* draft_ids,
                          int requests, int spec, int32_t* out_ids, float* out_logprob, int32_t* accepted,
                          cudaStream_t stream) {
  constexpr int kBlock = 128;
  const int grid = (requests + kBlock - 1) / kBlock;
  verify_kernel<<<grid, kBlock, 0, stream>>>(token_ids, token_logprob, draft_ids, requests, spec, out_ids,
                                            out_logprob, accepted);
  return cudaGetLastError();
}

}  // namespace vsl
