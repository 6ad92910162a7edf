// vsl_sample.cu - per-row sampler over vocab-sliced fp32 logits on sm_100a.
//
// For every row (a request's spec+1 rows are independent rows): temperature,
// top-k, top-p, a Philox4x32-keyed Gumbel-max draw and the top-n raw
// logprobs, over the concatenation of the row's S vocab slices
// ("Qwen4Exp batch-sharded sampling: inside vLLM PR #61018", orcarouter.ai
// blog, section "batch-sharded sampling in one paragraph": the sampler's
// top-k / top-p per request over batch x (spec+1) x vocab logits, logprobs
// under a non-negative max_logprobs).
//
// Execution model: one thread-block cluster of C CTAs per row.  CTA c copies
// its contiguous part of the row (global ids [c*part, (c+1)*part)) from HBM
// into shared memory with 1-D bulk copies, once; every later pass re-reads
// shared memory, so each logit crosses HBM exactly once.  CTA rank 0 (the
// leader) merges the CTAs' partial results through distributed shared memory
// and plans the next pass ("op"); the cluster runs ops until the row is done:
//
//   pass 1 (always)  max / min keys, online sum exp(l - M), and a 4096-bin
//                    histogram of order-preserving keys of the raw logits
//   COLLECT_RAW      candidates with key >= lo go to the leader's list: the
//                    top-n, the argmax, and (when it fits) all top-k
//                    survivors, resolved exactly by a sort in shared memory
//   MASS_HIST        (top-k off / too large) float64 masses exp(x - m) of the
//                    survivors, histogrammed on keys of x, and their sum Z
//   COLLECT_X        survivors with x-key in [lo, hi] to the leader's list
//   NARROW_COUNT/MASS  256-bin refinement of a key range (counts or masses)
//   NEXT_MAX         the next largest (key, lowest id) after a given pair
//   GUMBEL           Philox + Gumbel scores over every kept logit, per-CTA best
//
// Exactness: x = fl(l / T) uses IEEE division; top-k / top-p thresholds are
// found by exact integer selection on keys and float64 masses; the draw's
// float32 scores are re-compared in float64 whenever two candidates are
// closer than the float32 error bound, so the result is the float64 argmax.
#include <cuda_runtime.h>

#include <cfloat>
#include <cmath>
#include <cstdint>

#include "vsl_internal.h"
#include "vsl_ptx.cuh"

namespace vsl {

constexpr int kThreads = 512;
constexpr int kWarps = kThreads / 32;
constexpr int kHistBins = 4096;      // level-1 bins: key >> 20
constexpr int kListCap = 4096;       // leader candidate list capacity
constexpr int kSubBins = 256;        // narrowing bins
constexpr int kMaxCluster = 16;
constexpr int kMaxPart = 32768;      // floats per CTA (128 KB)
constexpr int kPreferredPart = 20480;  // floats per CTA (80 KB) when the cluster allows it

constexpr uint32_t kKeyNegInf = 0x007FFFFFu;  // key(-inf)
constexpr uint32_t kKeyPosInf = 0xFF800000u;  // key(+inf)

// Philox4x32-10 constants (Salmon et al., SC'11, Table 2, and the Weyl key increments).
constexpr uint32_t kPhiloxM0 = 0xD2511F53u, kPhiloxM1 = 0xCD9E8D57u;
constexpr uint32_t kPhiloxW0 = 0x9E3779B9u, kPhiloxW1 = 0xBB67AE85u;

enum Op : uint32_t {
  OP_END = 0,
  OP_COLLECT_RAW,
  OP_COLLECT_X,
  OP_MASS_HIST,
  OP_NARROW_COUNT,
  OP_NARROW_MASS,
  OP_NEXT_MAX,
  OP_GUMBEL,
};

struct SampleArgs {
  const float* slices[VSL_MAX_SLICES];
  const vsl_row_params* params;
  int32_t* token_ids;
  float* token_logprob;
  int32_t* topn_ids;
  float* topn_logprob;
  uint32_t* row_flags;
  uint32_t* err;
  unsigned long long seed;
  int R, S, V_s, V, C, part, n_logprobs;
};

// Per-CTA results the leader reads through distributed shared memory.
struct CtaStats {
  uint32_t kmax, kmin, kminf, bad;
  float m, s;           // online softmax partial: max finite logit, sum exp(l - m)
  double z;             // MASS_HIST: sum of survivor masses
  double best_sd;       // GUMBEL: float64 score of this CTA's best
  int32_t best_id;
  float best_l;
  uint32_t nm_key;      // NEXT_MAX result
  int32_t nm_id;
};

struct Plan {
  uint32_t op;
  uint32_t lo, hi, shift;  // key range and narrowing bin shift
  uint32_t raw_lo;         // raw-key prefilter: elements below cannot be survivors / kept
  float theta;             // survivor (MASS, NARROW_MASS, COLLECT_X) or kept (GUMBEL) threshold on x
  float m;                 // max x (masses are exp(x - m))
  uint32_t nm_key;         // NEXT_MAX: previous (key, id)
  int32_t nm_id;
};

enum Phase : uint32_t {
  PH_START = 0,
  PH_AFTER_COLLECT_RAW,
  PH_TOPN_NEXT_MAX,
  PH_TOPK_NARROW,
  PH_AFTER_MASS,
  PH_MASS_NARROW,
  PH_AFTER_COLLECT_X,
  PH_AFTER_GUMBEL,
  PH_DONE,
};

// Leader-only working state.
struct LeaderState {
  uint32_t phase, flags;
  uint32_t kmax, kminf;
  float M, lse, T, top_p;
  int32_t top_k;
  uint32_t req, pos;
  int r_n, r_k;
  bool greedy, k_listed, topn_done;
  uint32_t collect_lo;
  float theta_k, theta_p, m;
  uint32_t surv_raw_lo;     // raw prefilter for survivors of top-k
  double Z;
  // narrowing state
  uint32_t nlo, nhi, nshift;
  uint32_t nrank;
  double cum_above;
  int topn_count;
  uint32_t prev_key;
  int32_t prev_id;
  // result
  int32_t token;
  float token_l;
  // scratch for block-wide searches
  int found_bin;
  uint32_t found_cum;
  double found_mass;
  int sstar, send;
  int last_bin;
  double last_before;
  uint32_t last_cumc;
  bool x_from_top;          // the x-key list starts at the top of the row
};

struct __align__(16) SharedHeader {
  CtaStats stats;
  Plan plan;
  LeaderState L;
  uint32_t list_count;
  uint32_t pad;
  unsigned long long mbar;
  double red_d[kWarps];
  uint32_t red_u[kWarps * 4];
  float red_f[kWarps * 2];
  int32_t red_i[kWarps];
  double scan_d[kWarps];
  uint32_t scan_u[kWarps];
};

// Scratch union (48 KB).
constexpr size_t kScratchBytes = kHistBins * 8 + kHistBins * 4;
constexpr size_t kListBytes = kListCap * 8;

// ------------------------------------------------------------------ small helpers
// Order-preserving key of a float, computed on its bits with integer operations
// only (no float arithmetic, so NaN payloads cannot change the result): -0 and
// +0 share one key, larger keys are larger values, -inf < finite < +inf.
__device__ __forceinline__ uint32_t fkey_bits(uint32_t b) {
  b = (b == 0x80000000u) ? 0u : b;
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}
__device__ __forceinline__ uint32_t fkey(float v) { return fkey_bits(__float_as_uint(v)); }
// NaN of either sign, or +inf (-inf is a legal logit).
__device__ __forceinline__ bool nan_or_pos_inf(uint32_t b) {
  return (b & 0x7FFFFFFFu) > 0x7F800000u || b == 0x7F800000u;
}
__device__ __forceinline__ float key_value(uint32_t k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k);
}
__device__ __forceinline__ bool key_finite(uint32_t k) { return k > kKeyNegInf && k < kKeyPosInf; }
__device__ __forceinline__ float scale_x(float l, float T) { return __fdiv_rn(l, T); }

__device__ __forceinline__ float fast_exp2(float t) {
  float r;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(t));
  return r;
}

__device__ __forceinline__ uint4 philox4x32_10(uint4 c, uint32_t k0, uint32_t k1) {
#pragma unroll
  for (int r = 0; r < 10; ++r) {
    if (r > 0) {
      k0 += kPhiloxW0;
      k1 += kPhiloxW1;
    }
    const uint32_t hi0 = __umulhi(kPhiloxM0, c.x), lo0 = kPhiloxM0 * c.x;
    const uint32_t hi1 = __umulhi(kPhiloxM1, c.z), lo1 = kPhiloxM1 * c.z;
    c = make_uint4(hi1 ^ c.y ^ k0, lo1, hi0 ^ c.w ^ k1, lo0);
  }
  return c;
}
__device__ __forceinline__ uint32_t word_of(const uint4& w, int i) {
  return i == 0 ? w.x : i == 1 ? w.y : i == 2 ? w.z : w.w;
}
// Gumbel noise -log(-log u), u = ((w >> 9) + 0.5) * 2^-23, in float32.  -log u
// is taken as -log1p(-(1 - u)) above one half so that it keeps full relative
// precision near u = 1 (1 - u is exact).
__device__ __forceinline__ float gumbel32(uint32_t w) {
  const uint32_t b = w >> 9;
  const float u = (static_cast<float>(b) + 0.5f) * 0x1p-23f;
  const float v = (static_cast<float>(0x7FFFFFu - b) + 0.5f) * 0x1p-23f;  // 1 - u, exact
  const float nl = (u < 0.5f) ? -logf(u) : -log1pf(-v);
  return -logf(nl);
}
__device__ __forceinline__ double gumbel64(uint32_t w) {
  const double u = (static_cast<double>(w >> 9) + 0.5) * 0x1p-23;
  return -log(-log(u));
}
// Bound on |float32 score - exact score| for score s (logf / log1pf are within
// 1 ulp; |g| < 17), with a 3x safety factor.
__device__ __forceinline__ float score_tol(float s) { return 8e-6f + 3e-7f * fabsf(s); }

// Running best of the draw, exact in float64 whenever float32 cannot decide.
struct Best {
  float s, x, l;
  double sd;
  uint32_t w;
  int32_t id;
  bool valid, have_sd;
  __device__ void init() {
    valid = false;
    have_sd = false;
    s = -INFINITY;
    id = 0x7FFFFFFF;
    sd = -INFINITY;
  }
  __device__ double exact() {
    if (!have_sd) {
      sd = static_cast<double>(x) + gumbel64(w);
      have_sd = true;
    }
    return sd;
  }
  __device__ void offer(float cx, float cl, uint32_t cw, int32_t cid) {
    const float cs = cx + gumbel32(cw);
    if (!valid) {
      s = cs; x = cx; l = cl; w = cw; id = cid; valid = true; have_sd = false;
      return;
    }
    const float tol = score_tol(cs) + score_tol(s);
    if (cs > s + tol) {
      s = cs; x = cx; l = cl; w = cw; id = cid; have_sd = false;
    } else if (cs >= s - tol) {
      const double csd = static_cast<double>(cx) + gumbel64(cw);
      const double bsd = exact();
      if (csd > bsd || (csd == bsd && cid < id)) {
        s = cs; x = cx; l = cl; w = cw; id = cid; sd = csd; have_sd = true;
      }
    }
  }
};

// ------------------------------------------------------------------ block reductions
template <typename T, typename F>
__device__ __forceinline__ T warp_reduce(T v, F f) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = f(v, __shfl_xor_sync(0xFFFFFFFFu, v, o));
  return v;
}

__device__ __forceinline__ double block_sum_d(double v, SharedHeader* H) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  v = warp_reduce(v, [](double a, double b) { return a + b; });
  __syncthreads();
  if (lane == 0) H->red_d[warp] = v;
  __syncthreads();
  double t = 0.0;
  for (int i = 0; i < kWarps; ++i) t += H->red_d[i];  // fixed order: deterministic
  return t;
}

__device__ __forceinline__ int block_max_i(int v, SharedHeader* H) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  v = warp_reduce(v, [](int a, int b) { return a > b ? a : b; });
  __syncthreads();
  if (lane == 0) H->red_i[warp] = v;
  __syncthreads();
  int t = H->red_i[0];
  for (int i = 1; i < kWarps; ++i) t = max(t, H->red_i[i]);
  return t;
}
__device__ __forceinline__ int block_min_i(int v, SharedHeader* H) {
  return -block_max_i(-v, H);
}

// Inclusive prefix sum over threads (thread order), u32; also returns the block total.
__device__ __forceinline__ uint32_t block_scan_u(uint32_t v, uint32_t* total, SharedHeader* H) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xFFFFFFFFu, x, o);
    if (lane >= o) x += y;
  }
  __syncthreads();
  if (lane == 31) H->scan_u[warp] = x;
  __syncthreads();
  uint32_t off = 0, tot = 0;
  for (int i = 0; i < kWarps; ++i) {
    if (i < warp) off += H->scan_u[i];
    tot += H->scan_u[i];
  }
  *total = tot;
  return x + off;
}
__device__ __forceinline__ double block_scan_d(double v, double* total, SharedHeader* H) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  double x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const double y = __shfl_up_sync(0xFFFFFFFFu, x, o);
    if (lane >= o) x += y;
  }
  __syncthreads();
  if (lane == 31) H->scan_d[warp] = x;
  __syncthreads();
  double off = 0.0, tot = 0.0;
  for (int i = 0; i < kWarps; ++i) {
    if (i < warp) off += H->scan_d[i];
    tot += H->scan_d[i];
  }
  *total = tot;
  return x + off;
}

// Block argmax of (sd desc, id asc); every thread gets the winner's (sd, id, l).
__device__ void block_best(double& sd, int32_t& id, float& l, SharedHeader* H) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const double osd = __shfl_xor_sync(0xFFFFFFFFu, sd, o);
    const int32_t oid = __shfl_xor_sync(0xFFFFFFFFu, id, o);
    const float ol = __shfl_xor_sync(0xFFFFFFFFu, l, o);
    if (osd > sd || (osd == sd && oid < id)) {
      sd = osd;
      id = oid;
      l = ol;
    }
  }
  __syncthreads();
  if (lane == 0) {
    H->red_d[warp] = sd;
    H->red_i[warp] = id;
    H->red_f[warp] = l;
  }
  __syncthreads();
  sd = H->red_d[0];
  id = H->red_i[0];
  l = H->red_f[0];
  for (int i = 1; i < kWarps; ++i) {
    if (H->red_d[i] > sd || (H->red_d[i] == sd && H->red_i[i] < id)) {
      sd = H->red_d[i];
      id = H->red_i[i];
      l = H->red_f[i];
    }
  }
}

// Ascending bitonic sort of n (power of two) u64 keys in shared memory.
__device__ void bitonic_sort(uint64_t* a, int n) {
  for (int k = 2; k <= n; k <<= 1) {
    for (int j = k >> 1; j > 0; j >>= 1) {
      for (int i = threadIdx.x; i < n; i += kThreads) {
        const int p = i ^ j;
        if (p > i) {
          const uint64_t x = a[i], y = a[p];
          const bool up = (i & k) == 0;
          if ((x > y) == up) {
            a[i] = y;
            a[p] = x;
          }
        }
      }
      __syncthreads();
    }
  }
}

// ------------------------------------------------------------------ the kernel
struct Ctx {
  const SampleArgs* a;
  SharedHeader* H;
  const float4* part4;
  uint8_t* scratch;
  uint64_t* list;
  int row, n4;
  long long g0;          // global id of the first element of this CTA's part
  uint32_t rank, C;
  float T;
  uint32_t req, pos;
};

// Raw-key lower bound for l such that fl(l / T) >= theta is possible.
__device__ uint32_t raw_prefilter(float theta, float T) {
  if (theta == -INFINITY) return kKeyNegInf + 1;
  const float t2 = nextafterf(nextafterf(theta, -INFINITY), -INFINITY);
  const double lo = static_cast<double>(t2) * static_cast<double>(T);
  const float lo32 = __double2float_rd(lo);
  if (!(lo32 > -INFINITY)) return kKeyNegInf + 1;
  return fkey(lo32);
}

// Warp-aggregated append of sort keys to the leader's list.
__device__ __forceinline__ void list_append(const Ctx& cx, bool pred, uint64_t key) {
  const uint32_t mask = __ballot_sync(0xFFFFFFFFu, pred);
  if (mask == 0) return;
  const int lane = threadIdx.x & 31;
  uint32_t base = 0;
  if (lane == __ffs(mask) - 1)
    base = atom_add_dsmem_u32(mapa(smem_u32(&cx.H->list_count), 0), __popc(mask));
  base = __shfl_sync(0xFFFFFFFFu, base, __ffs(mask) - 1);
  if (pred) {
    const uint32_t idx = base + __popc(mask & ((1u << lane) - 1u));
    if (idx < static_cast<uint32_t>(kListCap))
      st_dsmem_u64(mapa(smem_u32(cx.list + idx), 0), key);
  }
}

// ---- pass 1: stats + level-1 raw histogram
__device__ void pass_stats(const Ctx& cx) {
  uint32_t* hist = reinterpret_cast<uint32_t*>(cx.scratch);
  uint32_t kmax = 0, kmin = 0xFFFFFFFFu, kminf = 0xFFFFFFFFu, bad = 0;
  float m = -INFINITY, s = 0.0f;
  constexpr float kLog2e = 1.4426950408889634f;
  for (int q = threadIdx.x; q < cx.n4; q += kThreads) {
    const float4 v4 = cx.part4[q];
    const float v[4] = {v4.x, v4.y, v4.z, v4.w};
    float mx = -INFINITY;
    bool fin[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint32_t raw = __float_as_uint(v[i]);
      bad |= nan_or_pos_inf(raw) ? 1u : 0u;
      const uint32_t k = fkey_bits(raw);
      kmax = max(kmax, k);
      kmin = min(kmin, k);
      fin[i] = key_finite(k) && !nan_or_pos_inf(raw);
      if (fin[i]) {
        kminf = min(kminf, k);
        mx = fmaxf(mx, v[i]);
      }
      atomicAdd(&hist[k >> 20], 1u);
    }
    if (mx > m) {
      s = (m == -INFINITY) ? 0.0f : s * fast_exp2((m - mx) * kLog2e);
      m = mx;
    }
#pragma unroll
    for (int i = 0; i < 4; ++i)
      if (fin[i]) s += fast_exp2((v[i] - m) * kLog2e);
  }
  // block reduce
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    kmax = max(kmax, __shfl_xor_sync(0xFFFFFFFFu, kmax, o));
    kmin = min(kmin, __shfl_xor_sync(0xFFFFFFFFu, kmin, o));
    kminf = min(kminf, __shfl_xor_sync(0xFFFFFFFFu, kminf, o));
    bad |= __shfl_xor_sync(0xFFFFFFFFu, bad, o);
    const float om = __shfl_xor_sync(0xFFFFFFFFu, m, o);
    const float os = __shfl_xor_sync(0xFFFFFFFFu, s, o);
    const float nm = fmaxf(m, om);
    if (nm > -INFINITY) s = (m > -INFINITY ? s * fast_exp2((m - nm) * kLog2e) : 0.0f) +
                            (om > -INFINITY ? os * fast_exp2((om - nm) * kLog2e) : 0.0f);
    m = nm;
  }
  SharedHeader* H = cx.H;
  if (lane == 0) {
    H->red_u[warp * 4 + 0] = kmax;
    H->red_u[warp * 4 + 1] = kmin;
    H->red_u[warp * 4 + 2] = kminf;
    H->red_u[warp * 4 + 3] = bad;
    H->red_f[warp * 2 + 0] = m;
    H->red_f[warp * 2 + 1] = s;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    uint32_t a = 0, b = 0xFFFFFFFFu, c = 0xFFFFFFFFu, d = 0;
    float M = -INFINITY;
    for (int i = 0; i < kWarps; ++i) {
      d |= H->red_u[i * 4 + 3];
      a = max(a, H->red_u[i * 4 + 0]);
      b = min(b, H->red_u[i * 4 + 1]);
      c = min(c, H->red_u[i * 4 + 2]);
      M = fmaxf(M, H->red_f[i * 2]);
    }
    float S = 0.0f;
    if (M > -INFINITY)
      for (int i = 0; i < kWarps; ++i)
        if (H->red_f[i * 2] > -INFINITY) S += H->red_f[i * 2 + 1] * fast_exp2((H->red_f[i * 2] - M) * kLog2e);
    H->stats.kmax = a;
    H->stats.kmin = b;
    H->stats.kminf = c;
    H->stats.bad = d;
    H->stats.m = M;
    H->stats.s = S;
  }
}

// ---- COLLECT_RAW: raw keys in [lo, hi] -> leader list (sort key: ~key, id)
__device__ void op_collect_raw(const Ctx& cx, const Plan& p) {
  const int nq = (cx.n4 + kThreads - 1) / kThreads * kThreads;
  for (int q = threadIdx.x; q < nq; q += kThreads) {
    const bool valid = q < cx.n4;
    const float4 v4 = valid ? cx.part4[q] : make_float4(0.f, 0.f, 0.f, 0.f);
    const float v[4] = {v4.x, v4.y, v4.z, v4.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint32_t k = fkey(v[i]);
      const bool pred = valid && k >= p.lo && k <= p.hi;
      const uint32_t gid = static_cast<uint32_t>(cx.g0 + 4 * q + i);
      list_append(cx, pred, (static_cast<uint64_t>(~k) << 32) | gid);
    }
  }
}

// ---- COLLECT_X: survivors with x-key in [lo, hi] -> leader list (sort key: ~xkey, id)
__device__ void op_collect_x(const Ctx& cx, const Plan& p) {
  const int nq = (cx.n4 + kThreads - 1) / kThreads * kThreads;
  for (int q = threadIdx.x; q < nq; q += kThreads) {
    const bool valid = q < cx.n4;
    const float4 v4 = valid ? cx.part4[q] : make_float4(0.f, 0.f, 0.f, 0.f);
    const float v[4] = {v4.x, v4.y, v4.z, v4.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      bool pred = false;
      uint32_t xk = 0;
      const uint32_t k = fkey(v[i]);
      if (valid && key_finite(k) && k >= p.raw_lo) {
        const float x = scale_x(v[i], cx.T);
        xk = fkey(x);
        pred = x >= p.theta && xk >= p.lo && xk <= p.hi;
      }
      const uint32_t gid = static_cast<uint32_t>(cx.g0 + 4 * q + i);
      list_append(cx, pred, (static_cast<uint64_t>(~xk) << 32) | gid);
    }
  }
}

// ---- MASS_HIST: float64 masses of survivors on 4096 x-key bins, and their sum
__device__ void op_mass_hist(const Ctx& cx, const Plan& p) {
  double* mass = reinterpret_cast<double*>(cx.scratch);
  uint32_t* cnt = reinterpret_cast<uint32_t*>(cx.scratch + kHistBins * 8);
  for (int i = threadIdx.x; i < kHistBins; i += kThreads) {
    mass[i] = 0.0;
    cnt[i] = 0;
  }
  __syncthreads();
  const double m = p.m;
  double z = 0.0;
  for (int q = threadIdx.x; q < cx.n4; q += kThreads) {
    const float4 v4 = cx.part4[q];
    const float v[4] = {v4.x, v4.y, v4.z, v4.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint32_t k = fkey(v[i]);
      if (key_finite(k) && k >= p.raw_lo) {
        const float x = scale_x(v[i], cx.T);
        if (x >= p.theta) {
          const double e = exp(static_cast<double>(x) - m);
          const uint32_t b = fkey(x) >> 20;
          atomicAdd(&mass[b], e);
          atomicAdd(&cnt[b], 1u);
          z += e;
        }
      }
    }
  }
  const double zt = block_sum_d(z, cx.H);
  if (threadIdx.x == 0) cx.H->stats.z = zt;
}

// ---- NARROW_COUNT: counts of raw keys in [lo, hi] on 256 bins from the top
__device__ void op_narrow_count(const Ctx& cx, const Plan& p) {
  uint32_t* cnt = reinterpret_cast<uint32_t*>(cx.scratch);
  for (int i = threadIdx.x; i < kSubBins; i += kThreads) cnt[i] = 0;
  __syncthreads();
  for (int q = threadIdx.x; q < cx.n4; q += kThreads) {
    const float4 v4 = cx.part4[q];
    const float v[4] = {v4.x, v4.y, v4.z, v4.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint32_t k = fkey(v[i]);
      if (k >= p.lo && k <= p.hi) atomicAdd(&cnt[(p.hi - k) >> p.shift], 1u);
    }
  }
}

// ---- NARROW_MASS: masses and counts of survivor x-keys in [lo, hi] on 256 bins from the top
__device__ void op_narrow_mass(const Ctx& cx, const Plan& p) {
  double* mass = reinterpret_cast<double*>(cx.scratch);
  uint32_t* cnt = reinterpret_cast<uint32_t*>(cx.scratch + kHistBins * 8);
  for (int i = threadIdx.x; i < kSubBins; i += kThreads) {
    mass[i] = 0.0;
    cnt[i] = 0;
  }
  __syncthreads();
  const double m = p.m;
  for (int q = threadIdx.x; q < cx.n4; q += kThreads) {
    const float4 v4 = cx.part4[q];
    const float v[4] = {v4.x, v4.y, v4.z, v4.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint32_t k = fkey(v[i]);
      if (key_finite(k) && k >= p.raw_lo) {
        const float x = scale_x(v[i], cx.T);
        const uint32_t xk = fkey(x);
        if (x >= p.theta && xk >= p.lo && xk <= p.hi) {
          const uint32_t b = (p.hi - xk) >> p.shift;
          atomicAdd(&mass[b], exp(static_cast<double>(x) - m));
          atomicAdd(&cnt[b], 1u);
        }
      }
    }
  }
}

// ---- NEXT_MAX: largest (key, lowest id) strictly after (nm_key, nm_id) in (key desc, id asc) order
__device__ void op_next_max(const Ctx& cx, const Plan& p) {
  uint32_t bk = 0;
  int32_t bid = 0x7FFFFFFF;
  bool have = false;
  for (int q = threadIdx.x; q < cx.n4; q += kThreads) {
    const float4 v4 = cx.part4[q];
    const float v[4] = {v4.x, v4.y, v4.z, v4.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint32_t k = fkey(v[i]);
      const int32_t id = static_cast<int32_t>(cx.g0 + 4 * q + i);
      const bool after = k < p.nm_key || (k == p.nm_key && id > p.nm_id);
      if (after && (!have || k > bk || (k == bk && id < bid))) {
        bk = k;
        bid = id;
        have = true;
      }
    }
  }
  // block reduce (key desc, id asc); "none" is (0, INT_MAX)
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const uint32_t ok = __shfl_xor_sync(0xFFFFFFFFu, bk, o);
    const int32_t oid = __shfl_xor_sync(0xFFFFFFFFu, bid, o);
    if (ok > bk || (ok == bk && oid < bid)) {
      bk = ok;
      bid = oid;
    }
  }
  SharedHeader* H = cx.H;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (lane == 0) {
    H->red_u[warp] = bk;
    H->red_i[warp] = bid;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    uint32_t k = H->red_u[0];
    int32_t id = H->red_i[0];
    for (int i = 1; i < kWarps; ++i)
      if (H->red_u[i] > k || (H->red_u[i] == k && H->red_i[i] < id)) {
        k = H->red_u[i];
        id = H->red_i[i];
      }
    H->stats.nm_key = k;
    H->stats.nm_id = id;
  }
}

// ---- GUMBEL: argmax of x + g over kept elements (x >= theta), float64-exact
__device__ void op_gumbel(const Ctx& cx, const Plan& p) {
  Best b;
  b.init();
  const uint32_t k0 = static_cast<uint32_t>(cx.a->seed), k1 = static_cast<uint32_t>(cx.a->seed >> 32);
  constexpr float kGMax = 16.7f;  // > -log(-log(1 - 2^-24)) = 16.63: the largest noise value
  for (int q = threadIdx.x; q < cx.n4; q += kThreads) {
    const float4 v4 = cx.part4[q];
    const float v[4] = {v4.x, v4.y, v4.z, v4.w};
    float x[4];
    bool kept[4];
    bool any = false;
    float xmax = -INFINITY;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint32_t k = fkey(v[i]);
      kept[i] = false;
      x[i] = -INFINITY;
      if (key_finite(k) && k >= p.raw_lo) {
        x[i] = scale_x(v[i], cx.T);
        kept[i] = x[i] >= p.theta;
        if (kept[i]) xmax = fmaxf(xmax, x[i]);
        any |= kept[i];
      }
    }
    // no kept element of this group can beat the current best, whatever its noise
    if (!any || (b.valid && xmax + kGMax < b.s - score_tol(b.s))) continue;
    const long long gid0 = cx.g0 + 4LL * q;
    const uint4 w = philox4x32_10(make_uint4(static_cast<uint32_t>(gid0 >> 2), cx.pos, cx.req, 0u), k0, k1);
#pragma unroll
    for (int i = 0; i < 4; ++i)
      if (kept[i]) b.offer(x[i], v[i], word_of(w, i), static_cast<int32_t>(gid0 + i));
  }
  double sd = b.valid ? b.exact() : -INFINITY;
  int32_t id = b.valid ? b.id : 0x7FFFFFFF;
  float l = b.valid ? b.l : 0.0f;
  block_best(sd, id, l, cx.H);
  if (threadIdx.x == 0) {
    cx.H->stats.best_sd = sd;
    cx.H->stats.best_id = id;
    cx.H->stats.best_l = l;
  }
}

// ------------------------------------------------------------------ leader logic
__device__ __forceinline__ void write_plan_all(const Ctx& cx, const Plan& p) {
  // thread t < C copies the plan into CTA t (word by word)
  if (threadIdx.x < cx.C) {
    const uint32_t* src = reinterpret_cast<const uint32_t*>(&p);
    const uint32_t dst = mapa(smem_u32(&cx.H->plan), threadIdx.x);
#pragma unroll
    for (int i = 0; i < static_cast<int>(sizeof(Plan) / 4); ++i) st_dsmem_u32(dst + 4 * i, src[i]);
  }
}

__device__ __forceinline__ uint32_t remote_u32(const Ctx& cx, const void* local, uint32_t rank) {
  return ld_dsmem_u32(mapa(smem_u32(local), rank));
}

// Scan the C CTAs' histograms (u32 counts, bin b at cnt[b]) from bin `top`
// downward; find the bin where the running count reaches `rank`.  Sets
// L.found_bin (or -1) and L.found_cum (count strictly above that bin).
__device__ void find_rank_bin(const Ctx& cx, const uint32_t* cnt_local, int top, int nbins_desc,
                              bool desc_from_top, uint32_t rank, LeaderState& L) {
  // nbins_desc bins, visited in order j = 0.. : bin index = desc_from_top ? top - j : j
  uint32_t cum = 0;
  if (threadIdx.x == 0) L.found_bin = -1;
  __syncthreads();
  for (int base = 0; base < nbins_desc; base += kThreads) {
    const int j = base + threadIdx.x;
    uint32_t c = 0;
    if (j < nbins_desc) {
      const int b = desc_from_top ? top - j : j;
      for (uint32_t r = 0; r < cx.C; ++r) c += remote_u32(cx, cnt_local + b, r);
    }
    uint32_t tot;
    const uint32_t incl = block_scan_u(c, &tot, cx.H);
    if (j < nbins_desc && c > 0 && cum + incl >= rank && cum + incl - c < rank) {
      L.found_bin = desc_from_top ? top - j : j;
      L.found_cum = cum + incl - c;
    }
    cum += tot;
    __syncthreads();
    if (L.found_bin >= 0) break;
  }
  __syncthreads();
}

__device__ void finalize_row(const Ctx& cx, LeaderState& L) {
  if (threadIdx.x == 0) {
    const SampleArgs& a = *cx.a;
    a.token_ids[cx.row] = L.token;
    a.token_logprob[cx.row] = L.token_l - L.lse;
    a.row_flags[cx.row] = 0;
  }
}

// Exact top-p on the leader's sorted list of survivors (entries 0..ns-1, x
// descending), with `cum_above` mass strictly above the list.  Returns via L:
// sstar (last kept group start) and send (kept prefix length).
__device__ void list_top_p(const Ctx& cx, LeaderState& L, int ns, double Z, double cum_above, bool x_keys) {
  const uint64_t* list = cx.list;
  const double m = L.m;
  constexpr int kPer = kListCap / kThreads;  // entries per thread (contiguous)
  double e[kPer];
  double tsum = 0.0;
  const int j0 = threadIdx.x * kPer;
#pragma unroll
  for (int i = 0; i < kPer; ++i) {
    const int j = j0 + i;
    e[i] = 0.0;
    if (j < ns) {
      const uint32_t key = ~static_cast<uint32_t>(list[j] >> 32);
      const float x = x_keys ? key_value(key) : scale_x(key_value(key), L.T);
      e[i] = exp(static_cast<double>(x) - m);
    }
    tsum += e[i];
  }
  double total;
  const double incl = block_scan_d(tsum, &total, cx.H);
  if (Z <= 0.0) Z = total;  // survivors all listed: Z is their sum
  const double pz = static_cast<double>(L.top_p);
  double run = incl - tsum;  // exclusive prefix of this thread's first entry
  int sstar = -1;
#pragma unroll
  for (int i = 0; i < kPer; ++i) {
    const int j = j0 + i;
    if (j < ns) {
      const uint32_t kj = ~static_cast<uint32_t>(list[j] >> 32);
      bool start = j == 0;
      if (!start) {
        const uint32_t kp = ~static_cast<uint32_t>(list[j - 1] >> 32);
        start = x_keys ? kp != kj : scale_x(key_value(kp), L.T) != scale_x(key_value(kj), L.T);
      }
      if (start && (cum_above + run) / Z < pz) sstar = j;
    }
    run += e[i];
  }
  sstar = block_max_i(sstar, cx.H);
  if (sstar < 0) sstar = 0;
  // end of the kept group: the next group start after sstar
  const uint32_t ks = ~static_cast<uint32_t>(list[sstar] >> 32);
  const float xs = x_keys ? key_value(ks) : scale_x(key_value(ks), L.T);
  int send = ns;
  for (int j = threadIdx.x; j < ns; j += kThreads) {
    if (j > sstar) {
      const uint32_t kj = ~static_cast<uint32_t>(list[j] >> 32);
      const float xj = x_keys ? key_value(kj) : scale_x(key_value(kj), L.T);
      if (xj != xs) send = min(send, j);
    }
  }
  send = block_min_i(send, cx.H);
  if (threadIdx.x == 0) {
    L.sstar = sstar;
    L.send = send;
    L.theta_p = xs;
  }
  __syncthreads();
}

// Gumbel draw over list entries [0, n) (keys raw or x); result into L.token / L.token_l.
__device__ void list_gumbel(const Ctx& cx, LeaderState& L, int n, bool x_keys) {
  Best b;
  b.init();
  const uint32_t k0 = static_cast<uint32_t>(cx.a->seed), k1 = static_cast<uint32_t>(cx.a->seed >> 32);
  for (int j = threadIdx.x; j < n; j += kThreads) {
    const uint64_t e = cx.list[j];
    const uint32_t key = ~static_cast<uint32_t>(e >> 32);
    const int32_t id = static_cast<int32_t>(e & 0xFFFFFFFFu);
    float x, l;
    if (x_keys) {
      x = key_value(key);
      l = -INFINITY;  // raw logit looked up below
    } else {
      l = key_value(key);
      x = scale_x(l, L.T);
    }
    const uint4 w = philox4x32_10(make_uint4(static_cast<uint32_t>(id) >> 2, cx.pos, cx.req, 0u), k0, k1);
    b.offer(x, l, word_of(w, id & 3), id);
  }
  double sd = b.valid ? b.exact() : -INFINITY;
  int32_t id = b.valid ? b.id : 0x7FFFFFFF;
  float l = b.valid ? b.l : 0.0f;
  block_best(sd, id, l, cx.H);
  if (threadIdx.x == 0) {
    const bool ok = id >= 0 && id < cx.a->V;  // a kept set is never empty; guard anyway
    L.token = ok ? id : -1;
    if (x_keys && ok) {
      const int s = id / cx.a->V_s, j = id - s * cx.a->V_s;
      l = cx.a->slices[s][static_cast<size_t>(cx.row) * cx.a->V_s + j];
    }
    L.token_l = ok ? l : __int_as_float(0x7FC00000);
  }
  __syncthreads();
}

__device__ void write_topn_from_list(const Ctx& cx, const LeaderState& L) {
  const SampleArgs& a = *cx.a;
  for (int j = threadIdx.x; j < a.n_logprobs; j += kThreads) {
    const uint64_t e = cx.list[j];
    const float l = key_value(~static_cast<uint32_t>(e >> 32));
    a.topn_ids[static_cast<size_t>(cx.row) * a.n_logprobs + j] = static_cast<int32_t>(e & 0xFFFFFFFFu);
    a.topn_logprob[static_cast<size_t>(cx.row) * a.n_logprobs + j] = l - L.lse;
  }
}

__device__ __forceinline__ int pow2_ceil(int n) {
  int p = 2;
  while (p < n) p <<= 1;
  return p;
}

// Sorts the list's first `count` entries (pads to a power of two).
__device__ void sort_list(const Ctx& cx, int count) {
  const int n = pow2_ceil(count);
  for (int j = count + threadIdx.x; j < n; j += kThreads) cx.list[j] = ~0ull;
  __syncthreads();
  bitonic_sort(cx.list, n);
}

// Plans the narrowing of the top-k rank search inside [lo, hi].
__device__ Plan narrow_count_plan(LeaderState& L) {
  Plan p{};
  p.op = OP_NARROW_COUNT;
  p.lo = L.nlo;
  p.hi = L.nhi;
  const uint32_t width = L.nhi - L.nlo;
  const int bits = width == 0 ? 0 : 32 - __clz(width);
  p.shift = bits > 8 ? bits - 8 : 0;
  __syncthreads();
  if (threadIdx.x == 0) L.nshift = p.shift;
  __syncthreads();
  return p;
}
__device__ Plan narrow_mass_plan(LeaderState& L) {
  Plan p{};
  p.op = OP_NARROW_MASS;
  p.lo = L.nlo;
  p.hi = L.nhi;
  const uint32_t width = L.nhi - L.nlo;
  const int bits = width == 0 ? 0 : 32 - __clz(width);
  p.shift = bits > 8 ? bits - 8 : 0;
  __syncthreads();
  if (threadIdx.x == 0) L.nshift = p.shift;
  __syncthreads();
  p.theta = L.theta_k;
  p.raw_lo = L.surv_raw_lo;
  p.m = L.m;
  return p;
}

// After the top-n / argmax is known: start the sampling part of the row.
// Returns the next plan (or OP_END after finishing the row).
__device__ Plan plan_sampling(const Ctx& cx, LeaderState& L);

__device__ Plan plan_after_theta_k(const Ctx& cx, LeaderState& L) {
  // survivors: finite with x >= theta_k (theta_k = -inf when top-k is off)
  const uint32_t surv_raw_lo = raw_prefilter(L.theta_k, L.T);
  __syncthreads();
  if (threadIdx.x == 0) L.surv_raw_lo = surv_raw_lo;
  __syncthreads();
  Plan p{};
  if (L.top_p < 1.0f) {
    p.op = OP_MASS_HIST;
    p.theta = L.theta_k;
    p.raw_lo = L.surv_raw_lo;
    p.m = L.m;
    if (threadIdx.x == 0) L.phase = PH_AFTER_MASS;
  } else {
    p.op = OP_GUMBEL;
    p.theta = L.theta_k;
    p.raw_lo = L.surv_raw_lo;
    if (threadIdx.x == 0) L.phase = PH_AFTER_GUMBEL;
  }
  return p;
}

__device__ Plan plan_sampling(const Ctx& cx, LeaderState& L) {
  Plan p{};
  if (L.greedy) {
    finalize_row(cx, L);
    p.op = OP_END;
    return p;
  }
  if (L.r_k == 0) {
    __syncthreads();
    if (threadIdx.x == 0) L.theta_k = -INFINITY;
    __syncthreads();
    return plan_after_theta_k(cx, L);
  }
  // top-k rank search by narrowing inside the level-1 bin found at the start
  return narrow_count_plan(L);
}

__device__ Plan leader_step(const Ctx& cx) {
  LeaderState& L = cx.H->L;
  const SampleArgs& a = *cx.a;
  Plan p{};
  p.op = OP_END;
  switch (L.phase) {
    case PH_START: {
      if (threadIdx.x == 0) {
        uint32_t kmax = 0, kmin = 0xFFFFFFFFu, kminf = 0xFFFFFFFFu, bad = 0;
        float M = -INFINITY;
        for (uint32_t r = 0; r < cx.C; ++r) {
          bad |= remote_u32(cx, &cx.H->stats.bad, r);
          kmax = max(kmax, remote_u32(cx, &cx.H->stats.kmax, r));
          kmin = min(kmin, remote_u32(cx, &cx.H->stats.kmin, r));
          kminf = min(kminf, remote_u32(cx, &cx.H->stats.kminf, r));
          M = fmaxf(M, __uint_as_float(remote_u32(cx, &cx.H->stats.m, r)));
        }
        float S = 0.0f;
        for (uint32_t r = 0; r < cx.C; ++r) {
          const float mr = __uint_as_float(remote_u32(cx, &cx.H->stats.m, r));
          const float sr = __uint_as_float(remote_u32(cx, &cx.H->stats.s, r));
          if (mr > -INFINITY) S += sr * fast_exp2((mr - M) * 1.4426950408889634f);
        }
        const vsl_row_params prm = a.params[cx.row];
        uint32_t flags = 0;
        if (bad) flags |= VSL_ROW_NONFINITE;
        else if (kmax == kKeyNegInf) flags |= VSL_ROW_ALL_NEG_INF;
        if (!(prm.temperature >= 0.0f && prm.temperature < INFINITY)) flags |= VSL_ROW_BAD_TEMPERATURE;
        if (!(prm.top_p > 0.0f)) flags |= VSL_ROW_BAD_TOP_P;
        if (prm.top_k < 0) flags |= VSL_ROW_BAD_TOP_K;
        if (flags == 0 && prm.temperature > 0.0f) {
          const float xmax = __fdiv_rn(key_value(kmax), prm.temperature);
          const float xmin = __fdiv_rn(key_value(kminf), prm.temperature);
          if (isinf(xmax) || isinf(xmin)) flags |= VSL_ROW_SCALE_OVERFLOW;
        }
        L.flags = flags;
        L.kmax = kmax;
        L.kminf = kminf;
        L.M = M;
        L.lse = M + logf(S);
        L.T = prm.temperature;
        L.top_p = prm.top_p;
        L.top_k = prm.top_k;
        L.req = prm.request_id;
        L.pos = prm.position;
        L.greedy = prm.temperature == 0.0f;
        L.r_n = a.n_logprobs > 0 ? a.n_logprobs : 1;
        L.r_k = (!L.greedy && prm.top_k > 0 && prm.top_k < a.V) ? prm.top_k : 0;
        L.m = L.greedy ? 0.0f : scale_x(M, prm.temperature);
        L.theta_k = -INFINITY;
        L.theta_p = -INFINITY;
        L.topn_done = false;
        L.token = -1;
      }
      __syncthreads();
      if (L.flags) {
        if (threadIdx.x == 0) {
          a.token_ids[cx.row] = -1;
          a.token_logprob[cx.row] = __int_as_float(0x7FC00000);
          a.row_flags[cx.row] = L.flags;
        }
        for (int j = threadIdx.x; j < a.n_logprobs; j += kThreads) {
          a.topn_ids[static_cast<size_t>(cx.row) * a.n_logprobs + j] = -1;
          a.topn_logprob[static_cast<size_t>(cx.row) * a.n_logprobs + j] = __int_as_float(0x7FC00000);
        }
        break;
      }
      // level-1 search: bins of the raw histogram from the max key downward
      const uint32_t* hist = reinterpret_cast<const uint32_t*>(cx.scratch);
      const int top = static_cast<int>(L.kmax >> 20);
      find_rank_bin(cx, hist, top, top + 1, true, static_cast<uint32_t>(L.r_n), L);
      const int bn = L.found_bin;
      const uint32_t cnt_n_incl = L.found_cum + (bn >= 0 ? [&] {
        uint32_t c = 0;
        for (uint32_t r = 0; r < cx.C; ++r) c += remote_u32(cx, hist + bn, r);
        return c;
      }() : 0u);
      int bk = -1;
      uint32_t cnt_k_incl = 0, cum_k = 0;
      if (L.r_k > 0) {
        find_rank_bin(cx, hist, top, top + 1, true, static_cast<uint32_t>(L.r_k), L);
        bk = L.found_bin;
        cum_k = L.found_cum;
        uint32_t c = 0, cbelow = 0;
        for (uint32_t r = 0; r < cx.C; ++r) {
          c += remote_u32(cx, hist + bk, r);
          if (bk > 0) cbelow += remote_u32(cx, hist + bk - 1, r);
        }
        cnt_k_incl = cum_k + c + cbelow;
      }
      __syncthreads();
      if (threadIdx.x == 0) {
        uint32_t lo = static_cast<uint32_t>(bn) << 20;
        uint32_t need = cnt_n_incl;
        L.k_listed = false;
        if (L.r_k > 0 && cnt_k_incl <= static_cast<uint32_t>(kListCap)) {
          const uint32_t lo_k = bk > 0 ? static_cast<uint32_t>(bk - 1) << 20 : 0u;
          lo = min(lo, lo_k);
          need = max(need, cnt_k_incl);
          L.k_listed = true;
        }
        // narrowing state for a top-k search outside the list
        L.nlo = static_cast<uint32_t>(max(bk, 0)) << 20;
        L.nhi = L.nlo | 0xFFFFFu;
        L.nrank = static_cast<uint32_t>(L.r_k) - cum_k;
        if (need <= static_cast<uint32_t>(kListCap)) {
          L.collect_lo = lo;
          cx.H->list_count = 0;
          L.phase = PH_AFTER_COLLECT_RAW;
        } else {
          // top-n not listable (dense or tied top bins): extract it one by one
          L.topn_count = 0;
          L.prev_key = 0xFFFFFFFFu;
          L.prev_id = -1;
          L.k_listed = false;
          L.phase = PH_TOPN_NEXT_MAX;
        }
      }
      __syncthreads();
      if (L.phase == PH_AFTER_COLLECT_RAW) {
        p.op = OP_COLLECT_RAW;
        p.lo = L.collect_lo;
        p.hi = 0xFFFFFFFFu;
      } else {
        p.op = OP_NEXT_MAX;
        p.nm_key = 0xFFFFFFFFu;
        p.nm_id = -1;
      }
      break;
    }

    case PH_TOPN_NEXT_MAX: {
      // result of one NEXT_MAX round: merge the CTAs' candidates
      if (threadIdx.x == 0) {
        uint32_t bk = 0;
        int32_t bid = 0x7FFFFFFF;
        for (uint32_t r = 0; r < cx.C; ++r) {
          const uint32_t k = remote_u32(cx, &cx.H->stats.nm_key, r);
          const int32_t id = static_cast<int32_t>(remote_u32(cx, &cx.H->stats.nm_id, r));
          if (k > bk || (k == bk && id < bid)) {
            bk = k;
            bid = id;
          }
        }
        const int j = L.topn_count;
        if (j < a.n_logprobs) {
          a.topn_ids[static_cast<size_t>(cx.row) * a.n_logprobs + j] = bid;
          a.topn_logprob[static_cast<size_t>(cx.row) * a.n_logprobs + j] = key_value(bk) - L.lse;
        }
        if (j == 0 && L.greedy) {
          L.token = bid;
          L.token_l = key_value(bk);
        }
        L.topn_count = j + 1;
        L.prev_key = bk;
        L.prev_id = bid;
      }
      __syncthreads();
      if (L.topn_count < L.r_n) {
        p.op = OP_NEXT_MAX;
        p.nm_key = L.prev_key;
        p.nm_id = L.prev_id;
        break;
      }
      if (threadIdx.x == 0) {
        L.topn_done = true;
        if (L.r_k > 0) L.phase = PH_TOPK_NARROW;
      }
      __syncthreads();
      p = plan_sampling(cx, L);
      break;
    }

    case PH_AFTER_COLLECT_RAW: {
      const int count = min(static_cast<int>(cx.H->list_count), kListCap);
      sort_list(cx, count);
      write_topn_from_list(cx, L);
      if (L.greedy) {
        if (threadIdx.x == 0) {
          L.token = static_cast<int32_t>(cx.list[0] & 0xFFFFFFFFu);
          L.token_l = key_value(~static_cast<uint32_t>(cx.list[0] >> 32));
        }
        __syncthreads();
        finalize_row(cx, L);
        break;
      }
      if (L.r_k > 0 && L.k_listed) {
        // theta_k from the list; all survivors are listed iff the largest
        // unlisted logit scales strictly below theta_k
        const uint32_t kk = ~static_cast<uint32_t>(cx.list[L.r_k - 1] >> 32);
        const float theta_k = scale_x(key_value(kk), L.T);
        bool all_listed = true;
        if (L.collect_lo > kKeyNegInf + 1) {
          const float l_nc = key_value(L.collect_lo - 1);
          all_listed = scale_x(l_nc, L.T) < theta_k;
        }
        if (threadIdx.x == 0) L.theta_k = theta_k;
        __syncthreads();
        if (all_listed) {
          // survivors: the list prefix with x >= theta_k
          int ns = 0;
          for (int j = threadIdx.x; j < count; j += kThreads) {
            const float x = scale_x(key_value(~static_cast<uint32_t>(cx.list[j] >> 32)), L.T);
            if (x >= theta_k && x > -INFINITY) ns = max(ns, j + 1);
          }
          ns = block_max_i(ns, cx.H);
          int nk = ns;
          if (L.top_p < 1.0f) {
            list_top_p(cx, L, ns, 0.0, 0.0, false);
            nk = L.send;
          }
          list_gumbel(cx, L, nk, false);
          finalize_row(cx, L);
          break;
        }
        p = plan_after_theta_k(cx, L);
        break;
      }
      if (L.r_k > 0) {
        if (threadIdx.x == 0) L.phase = PH_TOPK_NARROW;
        __syncthreads();
        p = narrow_count_plan(L);
        break;
      }
      if (threadIdx.x == 0) L.theta_k = -INFINITY;
      __syncthreads();
      p = plan_after_theta_k(cx, L);
      break;
    }

    case PH_TOPK_NARROW: {
      // merge the 256 narrowing bins; find the rank's sub-bin
      const uint32_t* cnt = reinterpret_cast<const uint32_t*>(cx.scratch);
      const int nb = static_cast<int>(((L.nhi - L.nlo) >> L.nshift) + 1);
      find_rank_bin(cx, cnt, 0, nb, false, L.nrank, L);
      if (threadIdx.x == 0) {
        const int j = max(L.found_bin, 0);
        const uint32_t hi = L.nhi - (static_cast<uint32_t>(j) << L.nshift);
        const uint32_t lo_c = (static_cast<uint32_t>(j + 1) << L.nshift) - 1;
        const uint32_t lo = (L.nhi - L.nlo) > lo_c ? L.nhi - lo_c : L.nlo;
        L.nrank -= L.found_cum;
        L.nlo = lo;
        L.nhi = hi;
      }
      __syncthreads();
      if (L.nlo != L.nhi) {
        p = narrow_count_plan(L);
        break;
      }
      if (threadIdx.x == 0) L.theta_k = scale_x(key_value(L.nlo), L.T);
      __syncthreads();
      p = plan_after_theta_k(cx, L);
      break;
    }

    case PH_AFTER_MASS: {
      // Z from the CTAs' deterministic sums; find the cut bin on the x-key histogram
      if (threadIdx.x == 0) {
        double Z = 0.0;
        for (uint32_t r = 0; r < cx.C; ++r) Z += ld_dsmem_f64(mapa(smem_u32(&cx.H->stats.z), r));
        L.Z = Z;
        L.found_bin = -1;
        L.last_bin = -1;
      }
      __syncthreads();
      const double* mass = reinterpret_cast<const double*>(cx.scratch);
      const uint32_t* cnt = reinterpret_cast<const uint32_t*>(cx.scratch + kHistBins * 8);
      const int top = static_cast<int>(fkey(L.m) >> 20);
      const double pz = static_cast<double>(L.top_p) * L.Z;
      double cum = 0.0;
      uint32_t cumc = 0;
      for (int base = 0; base <= top; base += kThreads) {
        const int j = base + threadIdx.x;
        double mj = 0.0;
        uint32_t cj = 0;
        if (j <= top) {
          for (uint32_t r = 0; r < cx.C; ++r) {
            mj += ld_dsmem_f64(mapa(smem_u32(mass + (top - j)), r));
            cj += remote_u32(cx, cnt + (top - j), r);
          }
        }
        double mt;
        uint32_t ct;
        const double mincl = block_scan_d(mj, &mt, cx.H);
        const uint32_t cincl = block_scan_u(cj, &ct, cx.H);
        const double before = cum + mincl - mj;
        if (cj > 0 && before < pz && cum + mincl >= pz) {
          L.found_bin = top - j;
          L.found_mass = before;
          L.found_cum = cumc + cincl;  // elements from the top through this bin
        }
        const int ln = block_max_i(cj > 0 ? j : -1, cx.H);
        if (ln >= 0 && threadIdx.x == ln - base) {
          L.last_bin = top - ln;
          L.last_before = before;
          L.last_cumc = cumc + cincl;
        }
        cum += mt;
        cumc += ct;
        __syncthreads();
        if (L.found_bin >= 0) break;
      }
      __syncthreads();
      if (threadIdx.x == 0) {
        if (L.found_bin < 0) {
          // rounding left pZ beyond the last bin: the cut is in the last non-empty bin
          L.found_bin = L.last_bin;
          L.found_mass = L.last_before;
          L.found_cum = L.last_cumc;
        }
        L.nlo = static_cast<uint32_t>(L.found_bin) << 20;
        L.nhi = L.nlo | 0xFFFFFu;
        L.cum_above = L.found_mass;
        L.x_from_top = L.found_cum <= static_cast<uint32_t>(kListCap);
        if (L.x_from_top) {
          // everything from the top through the cut bin fits: list it and finish exactly
          L.cum_above = 0.0;
          cx.H->list_count = 0;
          L.phase = PH_AFTER_COLLECT_X;
        } else {
          L.phase = PH_MASS_NARROW;
        }
      }
      __syncthreads();
      if (L.x_from_top) {
        p.op = OP_COLLECT_X;
        p.lo = L.nlo;
        p.hi = 0xFFFFFFFFu;
        p.theta = L.theta_k;
        p.raw_lo = L.surv_raw_lo;
        p.m = L.m;
        break;
      }
      p = narrow_mass_plan(L);
      break;
    }

    case PH_MASS_NARROW: {
      const double* mass = reinterpret_cast<const double*>(cx.scratch);
      const uint32_t* cnt = reinterpret_cast<const uint32_t*>(cx.scratch + kHistBins * 8);
      const int nb = static_cast<int>(((L.nhi - L.nlo) >> L.nshift) + 1);
      const double pz = static_cast<double>(L.top_p) * L.Z;
      if (threadIdx.x == 0) L.found_bin = -1;
      __syncthreads();
      const int j = threadIdx.x;
      double mj = 0.0;
      uint32_t cj = 0;
      if (j < nb) {
        for (uint32_t r = 0; r < cx.C; ++r) {
          mj += ld_dsmem_f64(mapa(smem_u32(mass + j), r));
          cj += remote_u32(cx, cnt + j, r);
        }
      }
      double mt;
      const double mincl = block_scan_d(mj, &mt, cx.H);
      const double before = L.cum_above + mincl - mj;
      // last non-empty sub-bin whose mass above is < pZ
      int cand = (j < nb && cj > 0 && before < pz) ? j : -1;
      cand = block_max_i(cand, cx.H);
      if (cand < 0) cand = 0;
      if (threadIdx.x == cand) {
        L.found_bin = cand;
        L.found_mass = before;
        L.found_cum = cj;
      }
      __syncthreads();
      if (threadIdx.x == 0) {
        const uint32_t jj = static_cast<uint32_t>(L.found_bin);
        const uint32_t hi = L.nhi - (jj << L.nshift);
        const uint32_t lo_c = ((jj + 1) << L.nshift) - 1;
        const uint32_t lo = (L.nhi - L.nlo) > lo_c ? L.nhi - lo_c : L.nlo;
        L.nlo = lo;
        L.nhi = hi;
        L.cum_above = L.found_mass;
      }
      __syncthreads();
      if (L.nlo == L.nhi) {
        // one x value: every survivor with it has the same mass above (< pZ): kept
        Plan g{};
        g.op = OP_GUMBEL;
        g.theta = fmaxf(L.theta_k, key_value(L.nlo));
        g.raw_lo = raw_prefilter(g.theta, L.T);
        if (threadIdx.x == 0) L.phase = PH_AFTER_GUMBEL;
        __syncthreads();
        p = g;
        break;
      }
      if (L.found_cum <= static_cast<uint32_t>(kListCap)) {
        if (threadIdx.x == 0) {
          cx.H->list_count = 0;
          L.phase = PH_AFTER_COLLECT_X;
        }
        __syncthreads();
        p.op = OP_COLLECT_X;
        p.lo = L.nlo;
        p.hi = L.nhi;
        p.theta = L.theta_k;
        p.raw_lo = L.surv_raw_lo;
        p.m = L.m;
        break;
      }
      p = narrow_mass_plan(L);
      break;
    }

    case PH_AFTER_COLLECT_X: {
      const int count = min(static_cast<int>(cx.H->list_count), kListCap);
      sort_list(cx, count);
      list_top_p(cx, L, count, L.Z, L.cum_above, true);
      if (L.x_from_top) {
        // the list holds every survivor above the cut: draw from it directly
        list_gumbel(cx, L, L.send, true);
        finalize_row(cx, L);
        break;
      }
      Plan g{};
      g.op = OP_GUMBEL;
      g.theta = fmaxf(L.theta_k, L.theta_p);
      g.raw_lo = raw_prefilter(g.theta, L.T);
      if (threadIdx.x == 0) L.phase = PH_AFTER_GUMBEL;
      __syncthreads();
      p = g;
      break;
    }

    case PH_AFTER_GUMBEL: {
      if (threadIdx.x == 0) {
        double bsd = -INFINITY;
        int32_t bid = 0x7FFFFFFF;
        float bl = 0.0f;
        for (uint32_t r = 0; r < cx.C; ++r) {
          const double sd = ld_dsmem_f64(mapa(smem_u32(&cx.H->stats.best_sd), r));
          const int32_t id = static_cast<int32_t>(remote_u32(cx, &cx.H->stats.best_id, r));
          const float l = __uint_as_float(remote_u32(cx, &cx.H->stats.best_l, r));
          if (sd > bsd || (sd == bsd && id < bid)) {
            bsd = sd;
            bid = id;
            bl = l;
          }
        }
        const bool ok = bid >= 0 && bid < a.V;
        L.token = ok ? bid : -1;
        L.token_l = ok ? bl : __int_as_float(0x7FC00000);
      }
      __syncthreads();
      finalize_row(cx, L);
      break;
    }
    default:
      break;
  }
  return p;
}

__global__ void __launch_bounds__(kThreads, 1) sample_kernel(const __grid_constant__ SampleArgs a) {
  extern __shared__ __align__(128) uint8_t smem_raw[];
  SharedHeader* H = reinterpret_cast<SharedHeader*>(smem_raw);
  uint8_t* scratch = smem_raw + ((sizeof(SharedHeader) + 127) & ~size_t(127));
  uint64_t* list = reinterpret_cast<uint64_t*>(scratch + kScratchBytes);
  float* part = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(list) + kListBytes);

  Ctx cx;
  cx.a = &a;
  cx.H = H;
  cx.scratch = scratch;
  cx.list = list;
  cx.C = static_cast<uint32_t>(a.C);
  cx.rank = cluster_ctarank();
  cx.row = static_cast<int>(blockIdx.x / a.C);
  cx.g0 = static_cast<long long>(cx.rank) * a.part;
  const long long g1 = min(cx.g0 + a.part, static_cast<long long>(a.V));
  const int n = g1 > cx.g0 ? static_cast<int>(g1 - cx.g0) : 0;
  cx.n4 = n >> 2;
  cx.part4 = reinterpret_cast<const float4*>(part);

  // ---- load this CTA's part of the row (1-D bulk copies, one per slice segment)
  const uint32_t bar = smem_u32(&H->mbar);
  if (threadIdx.x == 0) {
    mbar_init(bar, 1);
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    mbar_arrive_expect_tx(bar, static_cast<uint32_t>(n) * 4u);
    const uint64_t pol = policy_evict_first();
    long long g = cx.g0;
    while (g < g1) {
      const int s = static_cast<int>(g / a.V_s);
      const long long s_end = min(static_cast<long long>(s + 1) * a.V_s, g1);
      const float* src = a.slices[s] + static_cast<size_t>(cx.row) * a.V_s + (g - static_cast<long long>(s) * a.V_s);
      long long off = g;
      while (off < s_end) {
        const long long chunk = min(s_end - off, 8192LL);  // 32 KB per copy
        bulk_load(smem_u32(part + (off - cx.g0)), src + (off - g), static_cast<uint32_t>(chunk * 4), bar, pol);
        off += chunk;
      }
      g = s_end;
    }
  }
  {
    uint32_t* hist = reinterpret_cast<uint32_t*>(scratch);
    for (int i = threadIdx.x; i < kHistBins; i += kThreads) hist[i] = 0;
    if (threadIdx.x == 0) {
      H->L.phase = PH_START;
      H->list_count = 0;
    }
  }
  __syncthreads();
  if (!mbar_wait_bounded(bar, 0)) {
    // the copy never landed (a bug): report and leave the row unwritten
    if (threadIdx.x == 0) atomicOr(a.err, kErrSampleLoad);
  }

  // ---- row params needed by every CTA
  {
    const vsl_row_params prm = a.params[cx.row];
    cx.T = prm.temperature;
    cx.req = prm.request_id;
    cx.pos = prm.position;
  }

  pass_stats(cx);
  cluster_sync();

  for (int iter = 0; iter < 64; ++iter) {
    Plan next{};
    if (cx.rank == 0) {
      next = leader_step(cx);
      __syncthreads();
      write_plan_all(cx, next);
    }
    cluster_sync();
    const Plan p = H->plan;
    if (p.op == OP_END) break;
    switch (p.op) {
      case OP_COLLECT_RAW: op_collect_raw(cx, p); break;
      case OP_COLLECT_X: op_collect_x(cx, p); break;
      case OP_MASS_HIST: op_mass_hist(cx, p); break;
      case OP_NARROW_COUNT: op_narrow_count(cx, p); break;
      case OP_NARROW_MASS: op_narrow_mass(cx, p); break;
      case OP_NEXT_MAX: op_next_max(cx, p); break;
      case OP_GUMBEL: op_gumbel(cx, p); break;
      default: break;
    }
    __syncthreads();
    cluster_sync();
  }
}

// ------------------------------------------------------------------ host side
size_t sample_smem_bytes(int part) {
  return ((sizeof(SharedHeader) + 127) & ~size_t(127)) + kScratchBytes + kListBytes +
         static_cast<size_t>(part) * 4;
}

static int g_max_cluster = -1;  // largest cluster size the device schedules for this kernel

bool sample_geometry(long long V, int* cluster, int* part) {
  if (V <= 0 || V > static_cast<long long>(kMaxCluster) * kMaxPart) return false;
  int c = 1;
  while (c < kMaxCluster && (V + c - 1) / c > kPreferredPart) c <<= 1;
  const int maxc = g_max_cluster > 0 ? g_max_cluster : 8;
  while (c > maxc) c >>= 1;
  long long p = (V + c - 1) / c;
  p = (p + 3) / 4 * 4;
  if (p > kMaxPart) return false;
  *cluster = c;
  *part = static_cast<int>(p);
  return true;
}

static cudaError_t prepare_sample_kernel() {
  static bool done = false;
  if (done) return cudaSuccess;
  cudaError_t e = cudaFuncSetAttribute(sample_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(sample_smem_bytes(kMaxPart)));
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(sample_kernel, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
  if (e != cudaSuccess) return e;
  // largest schedulable cluster at the preferred part size
  g_max_cluster = 8;
  for (int c = kMaxCluster; c >= 8; c >>= 1) {
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(c, 1, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = sample_smem_bytes(kPreferredPart);
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = c;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, sample_kernel, &cfg) == cudaSuccess && n > 0) {
      g_max_cluster = c;
      break;
    }
    cudaGetLastError();
  }
  done = true;
  return cudaSuccess;
}

cudaError_t launch_sample(const float* const* logits, int R, int S, int V_s, const vsl_row_params* params,
                          uint64_t seed, int n_logprobs, int32_t* token_ids, float* token_logprob,
                          int32_t* topn_ids, float* topn_logprob, uint32_t* row_flags, cudaStream_t stream) {
  cudaError_t e = prepare_sample_kernel();
  if (e != cudaSuccess) return e;
  SampleArgs a{};
  for (int s = 0; s < S; ++s) a.slices[s] = logits[s];
  a.params = params;
  a.token_ids = token_ids;
  a.token_logprob = token_logprob;
  a.topn_ids = topn_ids;
  a.topn_logprob = topn_logprob;
  a.row_flags = row_flags;
  a.err = device_error_word();
  if (a.err == nullptr) return cudaErrorUnknown;
  a.seed = seed;
  a.R = R;
  a.S = S;
  a.V_s = V_s;
  a.V = S * V_s;
  a.n_logprobs = n_logprobs;
  int c = 0, part = 0;
  if (!sample_geometry(a.V, &c, &part)) return cudaErrorInvalidValue;
  a.C = c;
  a.part = part;
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(static_cast<unsigned>(R) * c, 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = sample_smem_bytes(part);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = c;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, sample_kernel, a);
}

}  // namespace vsl
