// vsl_tiles.cu - tile statistics of logits that already sit in memory (the
// projection writes the same records from its epilogue, vsl_gemm.cu).
//
// "Qwen4Exp batch-sharded sampling: inside vLLM PR #61018" (orcarouter.ai
// blog), section "batch-sharded sampling in one paragraph": the sampler's
// top-k / top-p and logprobs need, per row, the softmax statistics and the
// top candidates of the whole vocabulary.  Per block of 128 ids of a slice the
// record holds the four 32-id quarter maxima, the sum of exp(l - c) (c the
// block's largest logit when finite, else 0), the smallest finite logit and
// the smallest nonzero |l|;
// a sampler that has them reads only the quarters that can hold its top
// candidates.
//
// One warp per (row, block): each lane loads one float4 (ids 4 lane .. 4 lane
// + 3 of the block, quarter lane / 8), the quarter and block maxima and the
// smallest finite value are reduced on order-preserving keys (integer max /
// min, exact), then the sum of exp2((l - c) log2 e) across the warp.  Bound
// by the read of the logits.
#include <cuda_runtime.h>

#include <cstdint>

#include "vsl_internal.h"

namespace vsl {

namespace {

constexpr int kTileWarps = 8;
constexpr uint32_t kNegInfKey = 0x007FFFFFu;  // key(-inf)
constexpr uint32_t kPosInfKey = 0xFF800000u;  // key(+inf)

struct TileArgs {
  const float* slices[VSL_MAX_SLICES];
  float* stats;
  int R, S, V_s, B;
  int per_row;  // CTAs per row
};

__device__ __forceinline__ uint32_t order_key(float v) {
  uint32_t b = __float_as_uint(v);
  b = (b == 0x80000000u) ? 0u : b;
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}
__device__ __forceinline__ float key_float(uint32_t k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k);
}
__device__ __forceinline__ float exp2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__global__ void __launch_bounds__(kTileWarps * 32) tile_stats_kernel(const __grid_constant__ TileArgs a) {
  const int lane = threadIdx.x & 31;
  const int row = static_cast<int>(blockIdx.x) / a.per_row;
  const int i = (static_cast<int>(blockIdx.x) - row * a.per_row) * kTileWarps + (threadIdx.x >> 5);  // block of the row
  if (i >= a.S * a.B) return;
  const int s = i / a.B;
  const int j0 = (i - s * a.B) * 128 + 4 * lane;
  const bool valid = j0 < a.V_s;  // V_s % 4 == 0: a float4 is all in or all out
  float v[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
  if (valid) {
    const float4 x = __ldg(reinterpret_cast<const float4*>(a.slices[s] + static_cast<size_t>(row) * a.V_s + j0));
    v[0] = x.x;
    v[1] = x.y;
    v[2] = x.z;
    v[3] = x.w;
  }
  uint32_t kq = 0, kf = 0xFFFFFFFFu, am = 0xFFFFFFFFu;
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const uint32_t k = order_key(v[u]);
    kq = max(kq, k);
    kf = min(kf, k - (kNegInfKey + 1u));  // -inf and negative NaN wrap above every finite key
    const uint32_t ab = __float_as_uint(v[u]) & 0x7FFFFFFFu;  // |l|: nonzero and not NaN
    am = min(am, (ab != 0u && ab <= 0x7F800000u) ? ab : 0xFFFFFFFFu);
  }
#pragma unroll
  for (int o = 1; o < 8; o <<= 1) kq = max(kq, __shfl_xor_sync(0xFFFFFFFFu, kq, o));  // the quarter's 8 lanes
  uint32_t kb = kq;
#pragma unroll
  for (int o = 8; o < 32; o <<= 1) kb = max(kb, __shfl_xor_sync(0xFFFFFFFFu, kb, o));
  kf = __reduce_min_sync(0xFFFFFFFFu, kf);
  am = __reduce_min_sync(0xFFFFFFFFu, am);
  const float c = (kb > kNegInfKey && kb < kPosInfKey) ? key_float(kb) : 0.0f;
  constexpr float kLog2e = 1.4426950408889634f;
  float e = 0.0f;
#pragma unroll
  for (int u = 0; u < 4; ++u) e += exp2_approx((v[u] - c) * kLog2e);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) e += __shfl_xor_sync(0xFFFFFFFFu, e, o);
  const float q0 = key_float(__shfl_sync(0xFFFFFFFFu, kq, 0));
  const float q1 = key_float(__shfl_sync(0xFFFFFFFFu, kq, 8));
  const float q2 = key_float(__shfl_sync(0xFFFFFFFFu, kq, 16));
  const float q3 = key_float(__shfl_sync(0xFFFFFFFFu, kq, 24));
  if (lane == 0) {
    float4* rec = reinterpret_cast<float4*>(a.stats + (static_cast<size_t>(row) * a.S * a.B + i) * 8);
    const float bmin = kf == 0xFFFFFFFFu ? INFINITY : key_float(kf + kNegInfKey + 1u);
    rec[0] = make_float4(q0, q1, q2, q3);
    rec[1] = make_float4(e, bmin, am == 0xFFFFFFFFu ? INFINITY : __uint_as_float(am), 0.0f);
  }
}

}  // namespace

cudaError_t launch_tile_stats(const float* const* logits, int R, int S, int V_s, float* stats, cudaStream_t stream) {
  TileArgs a{};
  for (int s = 0; s < S; ++s) a.slices[s] = logits[s];
  a.stats = stats;
  a.R = R;
  a.S = S;
  a.V_s = V_s;
  a.B = (V_s + 127) / 128;
  a.per_row = (S * a.B + kTileWarps - 1) / kTileWarps;
  const long long grid = static_cast<long long>(R) * a.per_row;
  if (grid > 0x7FFFFFFFLL) return cudaErrorInvalidConfiguration;
  tile_stats_kernel<<<static_cast<unsigned>(grid), kTileWarps * 32, 0, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace vsl
