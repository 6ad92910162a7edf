// vsl_internal.h - declarations shared by the libvsl translation units (host side).
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>

#include "../../include/vsl.h"

namespace vsl {

// Device address of the library's error word on the current device.
uint32_t* device_error_word();

// Launch the vocab-slice projection (stats: optional tile statistics, or
// nullptr).  Arguments already validated.
cudaError_t launch_logits_local(const void* hidden, const void* const* w_slices,
                                float* const* logits, int R, int H, int S, int V_s,
                                float* stats, cudaStream_t stream);

// Launch the tile statistics of logits in memory.  Arguments already validated.
cudaError_t launch_tile_stats(const float* const* logits, int R, int S, int V_s, float* stats,
                              cudaStream_t stream);

// Launch the sampler.  Arguments already validated.
cudaError_t launch_sample(const float* const* logits, int R, int S, int V_s,
                          const vsl_row_params* params, uint64_t seed, int n_logprobs,
                          int32_t* token_ids, float* token_logprob, int32_t* topn_ids,
                          float* topn_logprob, uint32_t* row_flags, float* kept_theta,
                          const float* tile_stats, cudaStream_t stream);

// Launch the processed-logprobs pass (after the sampler, same stream).
cudaError_t launch_processed(const float* const* logits, int R, int S, int V_s, const vsl_row_params* params,
                             int n_logprobs, const int32_t* token_ids, const int32_t* topn_ids,
                             const uint32_t* row_flags, const float* kept_theta, float* p_token,
                             int32_t* p_topn_ids, float* p_topn, cudaStream_t stream);

// Launch the speculative verification.  Arguments already validated.
cudaError_t launch_verify(const int32_t* token_ids, const float* token_logprob, const int32_t* draft_ids,
                          int requests, int spec, int32_t* out_ids, float* out_logprob, int32_t* accepted,
                          cudaStream_t stream);

// Sampler launch geometry for a vocabulary of V tokens on a device that
// schedules clusters of at most maxc CTAs: CTAs per row (cluster size) and
// elements per CTA.  Returns false if V cannot be handled.
bool sample_geometry_for(long long V, int maxc, int* cluster, int* part);
// Largest vocabulary the sampler handles on any device (host only).
long long sample_max_vocab();
// Largest cluster the current device schedules for the cluster kernel (the
// device's launch state is prepared on first use).
cudaError_t sample_max_cluster(int* maxc);
int sample_launches(int R, long long V);
bool sample_plan(int R, long long V, int sms, int maxc, vsl_sample_plan* out);

}  // namespace vsl
