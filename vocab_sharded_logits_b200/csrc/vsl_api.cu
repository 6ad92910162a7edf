// vsl_api.cu - the extern "C" entry points of libvsl: host-side argument
// validation, then a launch of the projection or the sampler kernel.
#include <cuda_runtime.h>

#include <cstdint>

#include "vsl_internal.h"

namespace vsl {

// Device error word: kernels OR a site bit into it when a bounded wait gives up.
__device__ uint32_t g_device_error = 0;

uint32_t* device_error_word() {
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_device_error) != cudaSuccess) return nullptr;
  return static_cast<uint32_t*>(p);
}

namespace {
bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned32(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 31u) == 0; }
}  // namespace

}  // namespace vsl

extern "C" {

const char* vsl_version(void) { return "libvsl 0.1 (sm_100a)"; }

const char* vsl_status_string(vsl_status status) {
  switch (status) {
    case VSL_OK: return "ok";
    case VSL_ERR_INVALID_ARG: return "invalid argument";
    case VSL_ERR_ALIGNMENT: return "pointer or row pitch not 16-byte aligned";
    case VSL_ERR_UNSUPPORTED: return "size beyond the library's limits";
    case VSL_ERR_WORKSPACE_TOO_SMALL: return "workspace too small";
    case VSL_ERR_CUDA: return "CUDA call failed";
    case VSL_ERR_DEVICE_TIMEOUT: return "a kernel gave up a bounded wait";
  }
  return "unknown status";
}

size_t vsl_tile_stats_floats(int32_t R, int32_t S, int32_t V_s) {
  if (R <= 0 || S <= 0 || V_s <= 0) return 0;
  return static_cast<size_t>(R) * static_cast<size_t>(S) * ((static_cast<size_t>(V_s) + 127) / 128) * 8;
}

vsl_status vsl_tile_stats(const float* const* logits_slices, int32_t R, int32_t S, int32_t V_s, float* tile_stats,
                          void* stream) {
  if (logits_slices == nullptr || tile_stats == nullptr) return VSL_ERR_INVALID_ARG;
  if (R <= 0 || S <= 0 || V_s <= 0) return VSL_ERR_INVALID_ARG;
  if (S > VSL_MAX_SLICES) return VSL_ERR_UNSUPPORTED;
  if (V_s % 4 != 0 || !vsl::aligned32(tile_stats)) return VSL_ERR_ALIGNMENT;
  for (int s = 0; s < S; ++s) {
    if (logits_slices[s] == nullptr) return VSL_ERR_INVALID_ARG;
    if (!vsl::aligned16(logits_slices[s])) return VSL_ERR_ALIGNMENT;
  }
  const cudaError_t e = vsl::launch_tile_stats(logits_slices, R, S, V_s, tile_stats, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? VSL_OK : VSL_ERR_CUDA;
}

vsl_status vsl_logits_local(const void* hidden_bf16, const void* const* w_slices_bf16, float* const* logits_slices,
                            int32_t R, int32_t H, int32_t S, int32_t V_s, void* stream) {
  return vsl_logits_local_ex(hidden_bf16, w_slices_bf16, logits_slices, R, H, S, V_s, nullptr, stream);
}

vsl_status vsl_logits_local_ex(const void* hidden_bf16, const void* const* w_slices_bf16, float* const* logits_slices,
                               int32_t R, int32_t H, int32_t S, int32_t V_s, float* tile_stats, void* stream) {
  if (hidden_bf16 == nullptr || w_slices_bf16 == nullptr || logits_slices == nullptr) return VSL_ERR_INVALID_ARG;
  if (R <= 0 || H <= 0 || S <= 0 || V_s <= 0) return VSL_ERR_INVALID_ARG;
  if (S > VSL_MAX_SLICES) return VSL_ERR_UNSUPPORTED;
  if (H % 8 != 0 || V_s % 4 != 0) return VSL_ERR_ALIGNMENT;
  if (!vsl::aligned16(hidden_bf16)) return VSL_ERR_ALIGNMENT;
  for (int s = 0; s < S; ++s) {
    if (w_slices_bf16[s] == nullptr || logits_slices[s] == nullptr) return VSL_ERR_INVALID_ARG;
    if (!vsl::aligned16(w_slices_bf16[s]) || !vsl::aligned16(logits_slices[s])) return VSL_ERR_ALIGNMENT;
  }
  if (tile_stats != nullptr && !vsl::aligned32(tile_stats)) return VSL_ERR_ALIGNMENT;
  const cudaError_t e = vsl::launch_logits_local(hidden_bf16, w_slices_bf16, logits_slices, R, H, S, V_s, tile_stats,
                                                 static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? VSL_OK : VSL_ERR_CUDA;
}

size_t vsl_sample_workspace_bytes(int32_t R, int32_t S, int32_t V_s, int32_t n_logprobs) {
  (void)R;
  (void)S;
  (void)V_s;
  (void)n_logprobs;
  return 0;  // every intermediate lives in shared memory
}

int32_t vsl_sample_launches(int32_t R, int32_t S, int32_t V_s) {
  if (R <= 0 || S <= 0 || S > VSL_MAX_SLICES || V_s <= 0 || V_s % 4 != 0) return -1;
  return vsl::sample_launches(R, static_cast<long long>(S) * V_s);
}

vsl_status vsl_sample_plan_for(int32_t R, int32_t S, int32_t V_s, int32_t sms, int32_t max_cluster,
                               vsl_sample_plan* out) {
  if (out == nullptr || R <= 0 || S <= 0 || V_s <= 0 || sms <= 0 || max_cluster <= 0) return VSL_ERR_INVALID_ARG;
  if (S > VSL_MAX_SLICES) return VSL_ERR_UNSUPPORTED;
  if (V_s % 4 != 0) return VSL_ERR_ALIGNMENT;
  const long long V = static_cast<long long>(S) * V_s;
  if (V > 0x7FFFFFFFLL || !vsl::sample_plan(R, V, sms, max_cluster, out)) return VSL_ERR_UNSUPPORTED;
  return VSL_OK;
}

vsl_status vsl_sample_ex(const float* const* logits_slices, int32_t R, int32_t S, int32_t V_s,
                         const vsl_row_params* params_dev, uint64_t seed, int32_t n_logprobs, int32_t* token_ids,
                         float* token_logprob, int32_t* topn_ids, float* topn_logprob, uint32_t* row_flags,
                         void* workspace, size_t workspace_bytes, const vsl_sample_extras* extras, void* stream) {
  (void)workspace;
  if (logits_slices == nullptr || params_dev == nullptr || token_ids == nullptr || token_logprob == nullptr ||
      row_flags == nullptr)
    return VSL_ERR_INVALID_ARG;
  if (R <= 0 || S <= 0 || V_s <= 0 || n_logprobs < 0) return VSL_ERR_INVALID_ARG;
  if (S > VSL_MAX_SLICES || n_logprobs > VSL_MAX_LOGPROBS) return VSL_ERR_UNSUPPORTED;
  const long long V = static_cast<long long>(S) * V_s;
  if (n_logprobs > V) return VSL_ERR_INVALID_ARG;
  if (n_logprobs > 0 && (topn_ids == nullptr || topn_logprob == nullptr)) return VSL_ERR_INVALID_ARG;
  if (V_s % 4 != 0) return VSL_ERR_ALIGNMENT;
  for (int s = 0; s < S; ++s) {
    if (logits_slices[s] == nullptr) return VSL_ERR_INVALID_ARG;
    if (!vsl::aligned16(logits_slices[s])) return VSL_ERR_ALIGNMENT;
  }
  float* kept_theta = extras != nullptr ? extras->kept_theta : nullptr;
  if (kept_theta != nullptr && (reinterpret_cast<uintptr_t>(kept_theta) & 7u) != 0) return VSL_ERR_ALIGNMENT;
  float* p_token = extras != nullptr ? extras->processed_logprob : nullptr;
  int32_t* p_topn_ids = extras != nullptr ? extras->processed_topn_ids : nullptr;
  float* p_topn = extras != nullptr ? extras->processed_topn_logprob : nullptr;
  if (p_token == nullptr && (p_topn_ids != nullptr || p_topn != nullptr)) return VSL_ERR_INVALID_ARG;
  if (p_token != nullptr && kept_theta == nullptr) return VSL_ERR_INVALID_ARG;
  if (p_token != nullptr && n_logprobs > 0 && (p_topn_ids == nullptr || p_topn == nullptr)) return VSL_ERR_INVALID_ARG;
  const float* tile_stats = extras != nullptr ? extras->tile_stats : nullptr;
  if (tile_stats != nullptr && !vsl::aligned32(tile_stats)) return VSL_ERR_ALIGNMENT;
  if (V > vsl::sample_max_vocab()) return VSL_ERR_UNSUPPORTED;
  int maxc = 0, c = 0, part = 0;
  if (vsl::sample_max_cluster(&maxc) != cudaSuccess) return VSL_ERR_CUDA;
  if (!vsl::sample_geometry_for(V, maxc, &c, &part)) return VSL_ERR_UNSUPPORTED;
  if (workspace_bytes < vsl_sample_workspace_bytes(R, S, V_s, n_logprobs)) return VSL_ERR_WORKSPACE_TOO_SMALL;
  cudaError_t e = vsl::launch_sample(logits_slices, R, S, V_s, params_dev, seed, n_logprobs, token_ids,
                                     token_logprob, topn_ids, topn_logprob, row_flags, kept_theta, tile_stats,
                                     static_cast<cudaStream_t>(stream));
  if (e == cudaSuccess && p_token != nullptr)
    e = vsl::launch_processed(logits_slices, R, S, V_s, params_dev, n_logprobs, token_ids, topn_ids, row_flags,
                              kept_theta, p_token, p_topn_ids, p_topn, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? VSL_OK : VSL_ERR_CUDA;
}

vsl_status vsl_sample(const float* const* logits_slices, int32_t R, int32_t S, int32_t V_s,
                      const vsl_row_params* params_dev, uint64_t seed, int32_t n_logprobs, int32_t* token_ids,
                      float* token_logprob, int32_t* topn_ids, float* topn_logprob, uint32_t* row_flags,
                      void* workspace, size_t workspace_bytes, void* stream) {
  return vsl_sample_ex(logits_slices, R, S, V_s, params_dev, seed, n_logprobs, token_ids, token_logprob, topn_ids,
                       topn_logprob, row_flags, workspace, workspace_bytes, nullptr, stream);
}

vsl_status vsl_verify_drafts(const int32_t* token_ids, const float* token_logprob, const int32_t* draft_ids,
                             int32_t requests, int32_t spec, int32_t* out_ids, float* out_logprob,
                             int32_t* accepted, void* stream) {
  if (token_ids == nullptr || out_ids == nullptr || accepted == nullptr) return VSL_ERR_INVALID_ARG;
  if (requests <= 0 || spec < 0 || spec > VSL_MAX_SPEC) return VSL_ERR_INVALID_ARG;
  if (spec > 0 && draft_ids == nullptr) return VSL_ERR_INVALID_ARG;
  if ((out_logprob == nullptr) != (token_logprob == nullptr)) return VSL_ERR_INVALID_ARG;
  if (static_cast<long long>(requests) * (spec + 1) > 0x7FFFFFFFLL) return VSL_ERR_UNSUPPORTED;
  const cudaError_t e = vsl::launch_verify(token_ids, token_logprob, draft_ids, requests, spec, out_ids,
                                           out_logprob, accepted, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? VSL_OK : VSL_ERR_CUDA;
}

vsl_status vsl_device_error(uint32_t* code_out) {
  if (cudaDeviceSynchronize() != cudaSuccess) return VSL_ERR_CUDA;
  uint32_t v = 0;
  if (cudaMemcpyFromSymbol(&v, vsl::g_device_error, sizeof(v)) != cudaSuccess) return VSL_ERR_CUDA;
  const uint32_t zero = 0;
  if (cudaMemcpyToSymbol(vsl::g_device_error, &zero, sizeof(zero)) != cudaSuccess) return VSL_ERR_CUDA;
  if (code_out) *code_out = v;
  return v ? VSL_ERR_DEVICE_TIMEOUT : VSL_OK;
}

}  // extern "C"
