// vsl_processed.cu - the processed logprobs of sampled rows: log-probabilities
// of the distribution each token was drawn from (after temperature, top-k and
// top-p), an optional output of vsl_sample_ex.
//
// "Qwen4Exp batch-sharded sampling: inside vLLM PR #61018" (orcarouter.ai
// blog), section "batch-sharded sampling in one paragraph": logprobs requested
// through a non-negative max_logprobs, next to the sampler's top-k / top-p.
// For a sampling row the draw's kept set is K = { finite x : x >= theta },
// theta = max(theta_k, theta_p) (the thresholds vsl_sample wrote), and
// log q_i = (x_i - m) - log sum_{j in K} exp(x_j - m), m = max_K x; a greedy
// row draws its token with certainty (log q = 0); a flagged row gets NaN.
// The top-n lists the n largest x of K, lower id first on equal x, then
// (-1, -inf) once K is exhausted.
//
// One CTA per row, one pass over the row: x = fl(l / T) for every logit, an
// online float64 (max, sum of exp) over the kept x, and the top-n candidates.
// The n-th largest x, x_n, is fl(l_n / T) of the n-th raw top-n logit (x is
// non-decreasing in l); every kept x > max(theta, x_n) is a candidate (fewer
// than n), and of the x equal to it the lowest ids: the row is scanned in id
// order, one block-wide chunk at a time, until enough of them are listed.
#include <cuda_runtime.h>

#include <cstdint>

#include "vsl_internal.h"
#include "vsl_math.cuh"

namespace vsl {

namespace {

constexpr int kPThreads = 256;
constexpr int kPWarps = kPThreads / 32;
constexpr int kPCand = 2048;  // strictly larger (< n) + the ties of up to two chunks

struct ProcArgs {
  const float* slices[VSL_MAX_SLICES];
  const vsl_row_params* params;
  const int32_t* token_ids;
  const int32_t* topn_ids;
  const uint32_t* row_flags;
  const float* kept_theta;
  float* p_token;
  int32_t* p_topn_ids;
  float* p_topn;
  int R, S, V_s, n;
};

__device__ __forceinline__ uint32_t key_of(float v) {
  uint32_t b = __float_as_uint(v);
  b = (b == 0x80000000u) ? 0u : b;
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}
__device__ __forceinline__ float logit_at(const ProcArgs& a, int row, int id) {
  const int s = id / a.V_s;
  return a.slices[s][static_cast<size_t>(row) * a.V_s + (id - s * a.V_s)];
}
// exp(d) for d <= 0 in float64 (CUDA's exp; the sums here feed a logprob
// compared within 1e-4, so no exactness argument rests on them).
__device__ __forceinline__ double e64(double d) { return exp(d); }

__global__ void __launch_bounds__(kPThreads) processed_kernel(const __grid_constant__ ProcArgs a) {
  __shared__ uint64_t cand[kPCand];  // (~x key) << 32 | id: ascending = x desc, id asc
  __shared__ uint32_t ncand, nties;
  __shared__ double red_m[kPWarps], red_s[kPWarps];
  __shared__ float sh_cut;
  const int row = blockIdx.x;
  const int n = a.n;
  const size_t o = static_cast<size_t>(row) * n;
  const float nan = __int_as_float(0x7FC00000);
  if (a.row_flags[row] != 0u) {
    if (threadIdx.x == 0) a.p_token[row] = nan;
    for (int j = threadIdx.x; j < n; j += kPThreads) {
      a.p_topn_ids[o + j] = -1;
      a.p_topn[o + j] = nan;
    }
    return;
  }
  const float T = a.params[row].temperature;
  if (T == 0.0f) {  // greedy: the token with certainty
    if (threadIdx.x == 0) a.p_token[row] = 0.0f;
    for (int j = threadIdx.x; j < n; j += kPThreads) {
      a.p_topn_ids[o + j] = j == 0 ? a.token_ids[row] : -1;
      a.p_topn[o + j] = j == 0 ? 0.0f : -INFINITY;
    }
    return;
  }
  const float theta = fmaxf(a.kept_theta[2 * static_cast<size_t>(row)], a.kept_theta[2 * static_cast<size_t>(row) + 1]);
  if (threadIdx.x == 0) {
    // the cut of the candidates: max(theta, x_n), x_n the n-th largest x
    float cut = theta;
    if (n > 0) cut = fmaxf(cut, scale_x(logit_at(a, row, a.topn_ids[o + n - 1]), T));
    sh_cut = cut;
    ncand = 0;
    nties = 0;
  }
  __syncthreads();
  const float cut = sh_cut;
  const uint32_t need_ties = static_cast<uint32_t>(n);  // enough ties: the top-n never needs more
  double m = -INFINITY, s = 0.0;
  bool ties_open = n > 0;
  for (int sl = 0; sl < a.S; ++sl) {
    const float4* p4 = reinterpret_cast<const float4*>(a.slices[sl] + static_cast<size_t>(row) * a.V_s);
    const int n4 = a.V_s >> 2;
    // block-wide chunks of kPThreads float4, in id order
    for (int base = 0; base < n4; base += kPThreads) {
      const int q = base + static_cast<int>(threadIdx.x);
      if (q < n4) {
        const float4 v4 = p4[q];
        const float v[4] = {v4.x, v4.y, v4.z, v4.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const uint32_t k = key_of(v[i]);
          if (!(k > 0x007FFFFFu && k < 0xFF800000u)) continue;  // -inf (NaN / +inf rows are flagged)
          const float x = scale_x(v[i], T);
          if (!(x >= theta)) continue;
          if (x > m) {
            s = (m == -INFINITY) ? 0.0 : s * e64(m - static_cast<double>(x));
            m = x;
          }
          s += e64(static_cast<double>(x) - m);
          const int id = sl * a.V_s + 4 * q + i;
          const bool take = n > 0 && (x > cut || (x == cut && ties_open));
          if (take) {
            const uint32_t c = atomicAdd(&ncand, 1u);
            if (x == cut) atomicAdd(&nties, 1u);
            if (c < static_cast<uint32_t>(kPCand))
              cand[c] = (static_cast<uint64_t>(~key_of(x)) << 32) | static_cast<uint32_t>(id);
          }
        }
      }
      if (ties_open) {
        // close the ties once a chunk has listed enough (later ones have larger
        // ids); every thread reads the count before any adds the next chunk's
        __syncthreads();
        const bool open = nties < need_ties;
        __syncthreads();
        ties_open = open;
      }
    }
  }
  // block merge of the online (m, s): fixed shuffle tree, warps in order
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    const double om = __shfl_xor_sync(0xFFFFFFFFu, m, off);
    const double os = __shfl_xor_sync(0xFFFFFFFFu, s, off);
    const double nm = fmax(m, om);
    if (nm > -INFINITY) s = (m > -INFINITY ? s * e64(m - nm) : 0.0) + (om > -INFINITY ? os * e64(om - nm) : 0.0);
    m = nm;
  }
  if ((threadIdx.x & 31) == 0) {
    red_m[threadIdx.x >> 5] = m;
    red_s[threadIdx.x >> 5] = s;
  }
  __syncthreads();
  double M = -INFINITY, Z = 0.0;
  for (int w = 0; w < kPWarps; ++w) M = fmax(M, red_m[w]);
  for (int w = 0; w < kPWarps; ++w)
    if (red_m[w] > -INFINITY) Z += red_s[w] * e64(red_m[w] - M);
  const double lz = M + log(Z);  // log sum_K exp(x)
  if (threadIdx.x == 0) {
    const int tok = a.token_ids[row];
    a.p_token[row] = tok >= 0 ? static_cast<float>(static_cast<double>(scale_x(logit_at(a, row, tok), T)) - lz) : nan;
  }
  if (n == 0) return;
  // the n smallest sort keys of the candidates (x desc, id asc), by rank
  __syncthreads();
  const int count = min(static_cast<int>(ncand), kPCand);
  for (int j = threadIdx.x; j < count; j += kPThreads) {
    const uint64_t e = cand[j];
    int rank = 0;
    for (int i = 0; i < count; ++i) rank += cand[i] < e ? 1 : 0;
    if (rank < n) {
      const uint32_t k = ~static_cast<uint32_t>(e >> 32);  // the key of x, inverted back to its bits
      const uint32_t b = (k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k;
      a.p_topn_ids[o + rank] = static_cast<int32_t>(e & 0xFFFFFFFFu);
      a.p_topn[o + rank] = static_cast<float>(static_cast<double>(__uint_as_float(b)) - lz);
    }
  }
  for (int j = count + threadIdx.x; j < n; j += kPThreads) {
    a.p_topn_ids[o + j] = -1;
    a.p_topn[o + j] = -INFINITY;
  }
}

}  // namespace

cudaError_t launch_processed(const float* const* logits, int R, int S, int V_s, const vsl_row_params* params,
                             int n_logprobs, const int32_t* token_ids, const int32_t* topn_ids,
                             const uint32_t* row_flags, const float* kept_theta, float* p_token,
                             int32_t* p_topn_ids, float* p_topn, cudaStream_t stream) {
  ProcArgs a{};
  for (int s = 0; s < S; ++s) a.slices[s] = logits[s];
  a.params = params;
  a.token_ids = token_ids;
  a.topn_ids = topn_ids;
  a.row_flags = row_flags;
  a.kept_theta = kept_theta;
  a.p_token = p_token;
  a.p_topn_ids = p_topn_ids;
  a.p_topn = p_topn;
  a.R = R;
  a.S = S;
  a.V_s = V_s;
  a.n = n_logprobs;
  processed_kernel<<<R, kPThreads, 0, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace vsl
