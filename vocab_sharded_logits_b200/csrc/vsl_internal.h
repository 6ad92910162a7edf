// vsl_internal.h - declarations shared by the libvsl translation units (host side).
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>

#include "../../include/vsl.h"

namespace vsl {

// Device address of the library's error word on the current device.
uint32_t* device_error_word();

// Launch the vocab-slice projection.  Arguments already validated.
cudaError_t launch_logits_local(const void* hidden, const void* const* w_slices,
                                float* const* logits, int R, int H, int S, int V_s,
                                cudaStream_t stream);

// Launch the sampler.  Arguments already validated.
cudaError_t launch_sample(const float* const* logits, int R, int S, int V_s,
                          const vsl_row_params* params, uint64_t seed, int n_logprobs,
                          int32_t* token_ids, float* token_logprob, int32_t* topn_ids,
                          float* topn_logprob, uint32_t* row_flags, cudaStream_t stream);

// Sampler launch geometry for a vocabulary of V tokens: CTAs per row (cluster
// size) and elements per CTA.  Returns false if V cannot be handled.
bool sample_geometry(long long V, int* cluster, int* part);
int sample_launches(int R, long long V);
bool sample_plan(int R, long long V, int sms, int maxc, vsl_sample_plan* out);

}  // namespace vsl
