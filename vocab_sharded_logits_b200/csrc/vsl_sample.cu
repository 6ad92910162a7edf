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
// Execution model: one thread-block cluster of C CTAs per row, several
// clusters resident at once.  CTA c copies its contiguous part of the row
// (global ids [c*part, (c+1)*part)) from HBM into shared memory with chunked
// 1-D bulk copies, once, and starts its first pass on the chunks that have
// landed; every later pass re-reads shared memory, so each logit crosses HBM
// exactly once.  CTA rank 0 (the leader) merges partial results through
// distributed shared memory and plans the next pass ("op"):
//
//   pass 1 (always)  max key, NaN and +inf, online sum exp(l - M) and a
//                    4096-bin histogram of order-preserving keys of raw logits
//   COLLECT_RAW      keys >= lo go to the leader's list: the top-n and, when
//                    every top-k survivor fits, all of them; the leader then
//                    resolves top-n, top-k, top-p and the draw on the sorted
//                    list alone while the other CTAs leave
//   NEXT_MAX         the next (key desc, id asc) element: top-n under ties
//   NARROW_COUNT     256-bin refinement of the top-k rank inside a key range
//   MASS             x = fl(l / T) written in place, and the float64 masses
//                    exp(x - m) of the survivors summed exactly in 76-bit
//                    fixed point on 240 bins of equal width in x below m,
//                    whose edges are exact key boundaries
//   NARROW_MASS      256-bin refinement of the top-p cut inside an x-key range
//   GUMBEL           Philox + Gumbel scores over every kept x, per-CTA best
//   XHIST            (top-k off, top_p < 1) x = fl(l / T) in place, 2,048 fine
//                    bins of x below m with counts and in-bin offset sums; the
//                    CTAs bound every bin's mass and agree on the window of
//                    bins that may hold the cut without a leader round
//   EXACT            float64 masses above and below the window, the window's
//                    members listed, the draw over the certainly kept x; the
//                    leader places the cut inside the sorted window
//
// Launches (host side, end of file): a batch of more rows than SMs runs the
// streaming kernel (vsl_stream.cuh) first, then this kernel on the rows it
// marked, on a fixed number of clusters that walk those rows; a smaller batch
// runs this kernel beside the streaming kernel on the rows the parameters give
// it, then the same marked-row pass.
//
// Exactness: x uses IEEE division; the top-k threshold is an exact integer
// rank selection on keys; the top-p cut compares exact sums of float64 masses
// (fixed point, independent of summation order); the draw's float32 scores are
// re-compared in float64 whenever float32 cannot separate two candidates.
#include <cuda_runtime.h>

#include <algorithm>
#include <cfloat>
#include <cmath>
#include <cstdint>
#include <mutex>

#include "vsl_internal.h"
#include "vsl_math.cuh"
#include "vsl_ptx.cuh"

namespace vsl {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kHistBins = 4096;        // pass-1 bins: raw key >> 20 (1/8 octave)
constexpr int kMassBins = 240;         // mass bins: equal steps of x below the max
constexpr int kSubBins = 256;          // narrowing bins
constexpr int kListCap = 2048;         // leader candidate list capacity
constexpr int kMaxCluster = 16;
constexpr int kMaxPart = 32768;        // floats per CTA (128 KB)
constexpr int kPreferredPart = 20480;  // floats per CTA (80 KB) when the cluster size allows it
constexpr int kLoadChunks = 4;
constexpr int kLocalTopK = 64;         // top-k up to this is resolved from per-CTA candidate lists
constexpr int32_t kDeferred = -2;      // token id of a row the streaming kernel leaves to the cluster kernel
constexpr int kStreamMaxK = 1024;      // largest top-k resolved from streamed candidates
// sample_kernel row selection: rows whose token id reads kDeferred (after the
// streaming kernel), or every row the streaming kernel does not take (run
// alongside it).  stream_kernel: kStreamMarks makes it mark those rows
// kDeferred; kStreamKoff makes it also take top-k-off rows (one CTA per row).
constexpr int kSelectDeferred = 0, kSelectOthers = 1, kStreamMarks = 1, kStreamKoff = 2;
constexpr int kStreamChunk = 2048;     // streaming kernel: floats per ring stage (8 KB)
constexpr int kStreamStages = 8;       // streaming kernel: ring depth (56 KB in flight per CTA)
constexpr int kXBins = 2048;           // fine bins of x below m (top-p window search)
constexpr float kXQuant = 4096.0f;     // in-bin offset quantum: 1 / 4096 of a bin
constexpr float kXRange = 40.0f;       // x more than 40 below m (mass < 5e-18 each) share the last bin

constexpr uint32_t kKeyNegInf = 0x007FFFFFu;  // key(-inf)
constexpr uint32_t kKeyPosInf = 0xFF800000u;  // key(+inf)

// Philox4x32-10 constants (Salmon et al., SC'11, Table 2, and the Weyl key increments).
constexpr uint32_t kPhiloxM0 = 0xD2511F53u, kPhiloxM1 = 0xCD9E8D57u;
constexpr uint32_t kPhiloxW0 = 0x9E3779B9u, kPhiloxW1 = 0xBB67AE85u;

enum Op : uint32_t {
  OP_END = 0,
  OP_COLLECT_RAW,
  OP_NEXT_MAX,
  OP_NARROW_COUNT,
  OP_MASS,
  OP_NARROW_MASS,
  OP_COLLECT_X,
  OP_GUMBEL,
  OP_XHIST,
  OP_EXACT,
};

enum Tail : uint32_t { TAIL_NONE = 0, TAIL_LIST_GREEDY, TAIL_LIST_SAMPLE, TAIL_STREAM_DONE };

struct SampleArgs {
  const float* slices[VSL_MAX_SLICES];
  const vsl_row_params* params;
  int32_t* token_ids;
  float* token_logprob;
  int32_t* topn_ids;
  float* topn_logprob;
  uint32_t* row_flags;
  float* kept_theta;  // optional [R][2]: theta_k, theta_p of each row (nullptr: not written)
  const float* tile_stats;  // streaming kernel: optional records [R][S * tile_blocks][8] (nullptr: none)
  int tile_blocks;          // blocks of 128 ids per slice
  uint32_t* err;
  unsigned long long seed;
  int R, S, V_s, V, C, part, n_logprobs;
  int select;  // rows a kernel takes: see kSelectDeferred, kSelectOthers, kStreamMarks
};

// Per-CTA results the leader reads through distributed shared memory.
struct CtaStats {
  uint32_t kmax, kminf, bad, pad;
  float m, s;           // online softmax partial: max finite logit, sum exp(l - m)
  uint32_t nm_key;      // NEXT_MAX result
  int32_t nm_id;
};

// GUMBEL result pushed by each CTA into the leader's slot [rank].
struct BestSlot {
  double sd;
  int32_t id;
  float l;
};

struct Plan {
  uint32_t op;
  uint32_t lo, hi, shift;  // key range and narrowing bin shift
  float theta;             // survivor (MASS, NARROW_MASS) or kept (GUMBEL) threshold on x
  float m;                 // max x (masses are exp(x - m))
  uint32_t nm_key;         // NEXT_MAX: previous (key, id)
  int32_t nm_id;
  uint32_t part_is_x;      // shared memory holds x = fl(l / T) instead of l
  uint32_t last;           // the cluster's last op for this row
  float step;              // MASS: width in x of one bin
  uint32_t pad;
};

enum Phase : uint32_t {
  PH_START = 0,
  PH_TOPN_NEXT_MAX,
  PH_AFTER_TOPN_COLLECT,
  PH_TOPK_NARROW,
  PH_AFTER_MASS,
  PH_MASS_NARROW,
  PH_AFTER_COLLECT_X,
  PH_AFTER_GUMBEL,
  PH_AFTER_XHIST,
  PH_AFTER_EXACT,
};

// Exact fixed-point mass: e * 2^60 held as four 16-bit limbs; a sum keeps each
// limb's total separately in 64 bits (value = sum_k v[k] * 2^(16k - 60)).
struct Fx4 {
  unsigned long long v[4];
};

// Leader-only working state.
struct LeaderState {
  uint32_t phase, flags;
  uint32_t kmax, kminf;
  float M, lse, T, top_p;
  int32_t top_k;
  uint32_t req, pos;
  int r_n, r_k;
  int greedy, topn_listed, topn_done, part_is_x, mode;
  uint32_t collect_lo;
  float theta_k, theta_p, m;
  // narrowing state
  uint32_t nlo, nhi, nshift, nrank;
  Fx4 cum;                             // exact mass strictly above the range (fixed point)
  Fx4 z;                               // exact total mass (fixed point)
  int topn_count;
  uint32_t prev_key;
  int32_t prev_id;
  int32_t token;
  float token_l;
  // scratch for block-wide searches
  int found_bin;
  uint32_t found_cum;
  uint32_t found_cnt;
  Fx4 found_above;
};

struct __align__(16) SharedHeader {
  CtaStats stats;
  CtaStats all[kMaxCluster];   // leader only: every CTA's stats, pushed before a cluster barrier
  Plan plan;
  LeaderState L;
  BestSlot best[kMaxCluster];
  double ex_above[kMaxCluster];    // leader only: EXACT sums pushed by every CTA
  double ex_below[kMaxCluster];
  float ex_xmin[kMaxCluster];      // leader only: EXACT's smallest x above the window, per CTA
  double win_lo[kMaxCluster];      // every CTA: each slice's lower / upper mass bound
  double win_hi[kMaxCluster];
  int32_t win_jlo[kMaxCluster];    // every CTA: each slice's window edges and count
  int32_t win_jhi[kMaxCluster];
  uint32_t win_cnt[kMaxCluster];
  uint32_t need_all[kMaxCluster];  // every CTA: each CTA's first-pass candidate count
  uint32_t ok_all[kMaxCluster];    // every CTA: each CTA's list is usable for top-k
  uint32_t listed;                 // the first-pass list holds the top-n (and top-k) union
  uint32_t list_aux;               // staging count of a local collection / leader small-buffer counter
  uint32_t list_base;              // reserved offset in the leader's list
  uint32_t list_count;
  uint32_t gbound;                 // CTA-wide draw bound (key of a published float32 score)
  unsigned long long mbar[kLoadChunks];
  unsigned long long ring_bar[kStreamStages];  // streaming kernel: one per ring stage
  double red_d[kWarps];
  uint32_t red_u[kWarps * 4];
  float red_f[kWarps * 2];
  int32_t red_i[kWarps];
  double scan_d[kWarps];
  uint32_t scan_u[kWarps];
  unsigned long long scan_fx[kWarps][4];
  double exp_tab[256];
  int32_t drows[kThreads];        // deferred-row pass: the rows of one block of marks
  uint32_t row_amin;               // streaming kernel: smallest bit pattern of a nonzero |l| (top-k-off rows)
  uint32_t kcut_above, kcut_window;  // streaming kernel: raw-key thresholds of the top-p window
  double row_z;                    // streaming kernel: the float64 mass of every finite x of the row
};

constexpr size_t kScratchBytes = kHistBins * 4;  // 16 KB: raw histogram, later mass / narrowing bins
constexpr size_t kListBytes = kListCap * 8;

// ------------------------------------------------------------------ small helpers
// Rows the streaming kernel resolves: valid parameters, and greedy or a top-k
// its candidate list holds, or (koff) top-k off.
__device__ __forceinline__ bool stream_row(const vsl_row_params& p, int V, bool koff = false) {
  if (!(p.top_p > 0.0f) || p.top_k < 0) return false;
  if (p.temperature == 0.0f) return true;
  if (!(p.temperature > 0.0f && p.temperature < INFINITY)) return false;
  if (p.top_k > 0 && p.top_k < V) return p.top_k <= kStreamMaxK;
  return koff;
}

// Order-preserving key of a float, computed on its bits with integer operations
// only (no float arithmetic, so NaN payloads cannot change the result): -0 and
// +0 share one key, larger keys are larger values, -inf < finite < +inf.
__device__ __forceinline__ uint32_t fkey_bits(uint32_t b) {
  b = (b == 0x80000000u) ? 0u : b;
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}
__device__ __forceinline__ uint32_t fkey(float v) { return fkey_bits(__float_as_uint(v)); }
__device__ __forceinline__ float key_value(uint32_t k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k);
}
// NaN of either sign, or +inf (-inf is a legal logit).
__device__ __forceinline__ bool nan_or_pos_inf(uint32_t b) {
  return (b & 0x7FFFFFFFu) > 0x7F800000u || b == 0x7F800000u;
}
__device__ __forceinline__ bool key_finite(uint32_t k) { return k > kKeyNegInf && k < kKeyPosInf; }

__device__ __forceinline__ float fast_exp2(float t) {
  float r;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(t));
  return r;
}

// Mass-bin edges: bin j holds the x-keys in (edge[j + 1], edge[j]], with
// edge[j] = key(fl(m - j * step)) (non-increasing in j) and the last bin
// open below.  Computed the same way by every CTA, so the bins agree exactly.
__device__ __forceinline__ uint32_t mass_edge(float m, float step, int j) {
  return fkey(__fsub_rn(m, __fmul_rn(static_cast<float>(j), step)));
}
__device__ __forceinline__ int mass_bin(const uint32_t* edge, float m, float inv_step, float x, uint32_t k) {
  int j = static_cast<int>(fminf(fmaxf(__fmul_rn(__fsub_rn(m, x), inv_step), 0.0f), static_cast<float>(kMassBins - 1)));
  while (j > 0 && k > edge[j]) --j;
  while (j < kMassBins - 1 && k <= edge[j + 1]) ++j;
  return j;
}

// Fine bin of a finite x <= m: t = fl(fl(m - x) * inv_w) clamped to the last
// bin, rounded to the nearest integer j.  Every CTA evaluates the same float32
// operations, so a value falls in the same bin everywhere, and the bin is
// non-increasing in x (each rounding step is monotone).  With the two
// roundings of relative size 2^-24 before the last one, bin j holds x with
// tau = (m - x) * inv_w in [(j - 0.5)(1 - 2^-22), (j + 0.5)(1 + 2^-22)] (the
// last bin: open above).  `q` is the offset t - j + 0.5 in [0, 1] rounded to
// a multiple of 1 / kXQuant (error <= 2^-13 with the float32 steps).
__device__ __forceinline__ int xbin(float x, float m, float inv_w) {
  const float t = fminf(__fmul_rn(__fsub_rn(m, x), inv_w), static_cast<float>(kXBins - 1));
  return __float_as_int(__fadd_rn(t, 0x1p23f)) - 0x4B000000;
}
__device__ __forceinline__ int xbin_q(float x, float m, float inv_w, uint32_t& q) {
  const float t = fminf(__fmul_rn(__fsub_rn(m, x), inv_w), static_cast<float>(kXBins - 1));
  const float r = __fadd_rn(t, 0x1p23f);
  const float o = __fadd_rn(__fsub_rn(t, __fsub_rn(r, 0x1p23f)), 0.5f);  // t - j exact (Sterbenz)
  q = __float_as_uint(__fmaf_rn(o, kXQuant, 0x1p23f)) - 0x4B000000u;
  return __float_as_int(r) - 0x4B000000;
}
// Bins per unit of x: the finite x range [x_min, m], at most kXRange wide, on kXBins bins.
__device__ __forceinline__ float xbin_scale(float m, float x_min) {
  float r = fminf(__fsub_rn(m, x_min), kXRange);
  if (!(r > 0.0f)) r = 1.0f;
  return __fdiv_rn(static_cast<float>(kXBins - 1), r);
}

// exp(d) for d <= 0 in float64, table-driven (P. T. P. Tang, "Table-driven
// implementation of the exponential function in IEEE floating-point
// arithmetic", ACM TOMS 15(2), 1989), with a 256-entry table: d = (256 h + j)
// ln2/256 + r with |r| <= ln2/512, exp(d) = 2^h * 2^(j/256) * p(r), p the cubic
// Taylor polynomial of exp (relative truncation < 1.5e-13; the one-constant
// reduction adds < 3e-14).  n = 256 h + j is rounded by adding 1.5 * 2^52, so
// no integer <-> float64 conversion is issued.  tab[j] = 2^(j/256).  d is
// clamped at -700 (the result there, < 1e-304, is below what any sum of < 2^20
// masses resolves), so no branch is taken.
__device__ __forceinline__ double exp_neg64(double d, const double* tab) {
  d = fmax(d, -700.0);  // exp(-700) < 1e-304: no sum of < 2^20 masses resolves it
  constexpr double kInvLn2x256 = 369.3299304675746;      // 256 / ln 2
  constexpr double kLn2d256 = 0.0027076061740622863;     // ln 2 / 256
  constexpr double kShifter = 6755399441055744.0;        // 1.5 * 2^52
  const double t = fma(d, kInvLn2x256, kShifter);
  const int n = __double2loint(t);
  const double nd = t - kShifter;
  const double r = fma(-nd, kLn2d256, d);
  double p = fma(r, 1.0 / 6.0, 0.5);
  p = fma(p, r, 1.0);
  p = fma(p, r, 1.0);
  const double v = tab[n & 255] * p;
  return __hiloint2double(__double2hiint(v) + ((n >> 8) << 20), __double2loint(v));
}

// e in (0, 1] as the integer round(e * 2^60) (error <= 2^-61): exact sums of up
// to 2^20 masses differ from the float64 sum by < 2^-41.  Each CTA adds the
// four 16-bit limbs in u32 bins: a CTA holds at most 2^15 logits, so a limb
// total stays below 2^31; the cluster-wide totals are kept per limb in 64 bits.
__device__ __forceinline__ unsigned long long mass_q(double e) { return __double2ull_rn(e * 0x1p60); }
__device__ __forceinline__ double fx_to_double(const Fx4& f) {
  return static_cast<double>(f.v[0]) * 0x1p-60 + static_cast<double>(f.v[1]) * 0x1p-44 +
         static_cast<double>(f.v[2]) * 0x1p-28 + static_cast<double>(f.v[3]) * 0x1p-12;
}
__device__ __forceinline__ Fx4 fx_zero() {
  Fx4 f;
#pragma unroll
  for (int k = 0; k < 4; ++k) f.v[k] = 0;
  return f;
}
__device__ __forceinline__ Fx4 fx_add(const Fx4& a, const Fx4& b) {
  Fx4 f;
#pragma unroll
  for (int k = 0; k < 4; ++k) f.v[k] = a.v[k] + b.v[k];
  return f;
}
__device__ __forceinline__ Fx4 fx_sub(const Fx4& a, const Fx4& b) {
  Fx4 f;
#pragma unroll
  for (int k = 0; k < 4; ++k) f.v[k] = a.v[k] - b.v[k];
  return f;
}
__device__ __forceinline__ Fx4 fx_of(double e) {
  const unsigned long long q = mass_q(e);
  Fx4 f;
#pragma unroll
  for (int k = 0; k < 4; ++k) f.v[k] = (q >> (16 * k)) & 0xFFFFull;
  return f;
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
__device__ __noinline__ float gumbel32(uint32_t w) {
  const uint32_t b = w >> 9;
  const float u = (static_cast<float>(b) + 0.5f) * 0x1p-23f;
  const float v = (static_cast<float>(0x7FFFFFu - b) + 0.5f) * 0x1p-23f;  // 1 - u, exact
  const float nl = (u < 0.5f) ? -logf(u) : -log1pf(-v);
  return -logf(nl);
}
__device__ __noinline__ double gumbel64(uint32_t w) {
  const double u = (static_cast<double>(w >> 9) + 0.5) * 0x1p-23;
  return -log(-log(u));
}
// 1 - u for the word, exact in float32: (0x7FFFFF - (w >> 9) + 0.5) * 2^-23,
// as (1 + (0x7FFFFF - (w >> 9)) * 2^-23) - (1 - 2^-24) from the bits (no
// int -> float conversion; the subtraction is exact).
__device__ __forceinline__ float one_minus_u(uint32_t w) {
  return __fsub_rn(__uint_as_float(0x3F800000u | (~w >> 9)), 0x1.fffffep-1f);
}
// Bound on |float32 score - exact score| for score s (logf / log1pf are within
// 1 ulp; |g| < 17), with a 3x safety factor.
__device__ __forceinline__ float score_tol(float s) { return 8e-6f + 3e-7f * fabsf(s); }

// Running best of the draw, exact in float64 whenever float32 cannot decide.
// `shared_key`, when set, is a CTA-wide word holding the order-preserving key
// of the best float32 score any thread has published: a candidate that cannot
// beat it is rejected as early as one that cannot beat the thread's own best,
// so the slow path stays rare for the warp as a whole, not only per thread.
struct Best {
  float s, x, l;
  double sd;
  uint32_t w;
  int32_t id;
  bool valid, have_sd;
  uint32_t* shared_key;
  __device__ void init(uint32_t* shared = nullptr) {
    valid = false;
    have_sd = false;
    s = -INFINITY;
    id = 0x7FFFFFFF;
    sd = -INFINITY;
    x = 0.f;
    l = 0.f;
    w = 0;
    shared_key = shared;
  }
  // The best score known to this thread: its own or the CTA's published one.
  __device__ __forceinline__ float bound_score() const {
    float b = valid ? s : -INFINITY;
    if (shared_key) b = fmaxf(b, key_value(*reinterpret_cast<volatile uint32_t*>(shared_key)));
    return b;
  }
  __device__ double exact() {
    if (!have_sd) {
      sd = static_cast<double>(x) + gumbel64(w);
      have_sd = true;
    }
    return sd;
  }
  __device__ __forceinline__ void take(float cs, float cx, float cl, uint32_t cw, int32_t cid) {
    s = cs; x = cx; l = cl; w = cw; id = cid; valid = true; have_sd = false;
    if (shared_key) atomicMax(shared_key, fkey(cs));
  }
  // log2(e) times a value below the exact score of the best known score s
  // (kNoBound when there is none): the rejection test's reference.
  static constexpr float kNoBound = -3.0e38f;
  __device__ __forceinline__ float bound_l2e() const {
    const float sb = bound_score();
    return sb > -INFINITY ? (sb - score_tol(sb) - 3e-5f) * 1.4426950408889634f : kNoBound;
  }
  // Cheap test that candidate (x, word) cannot beat the bound: beating a score
  // needs -log u < exp(x - bound), and -log u >= 1 - u.
  static __device__ __forceinline__ bool rejects(float bl2e, float cx, uint32_t cw) {
    const float q = fast_exp2(fmaf(cx, 1.4426950408889634f, -bl2e));
    return one_minus_u(cw) > q * 1.0001f + 1e-30f;
  }
  // Offers candidate (x, raw l, Philox word, id).
  __device__ __forceinline__ void offer(float cx, float cl, uint32_t cw, int32_t cid) {
    const float bl = bound_l2e();
    if (bl != kNoBound && rejects(bl, cx, cw)) return;
    offer_passed(cx, cl, cw, cid);
  }
  // The exact comparison for a candidate that passed the cheap test.
  __device__ __forceinline__ void offer_passed(float cx, float cl, uint32_t cw, int32_t cid) {
    const float cs = cx + gumbel32(cw);
    if (!valid) {
      take(cs, cx, cl, cw, cid);
      return;
    }
    const float tol = score_tol(cs) + score_tol(s);
    if (cs > s + tol) {
      take(cs, cx, cl, cw, cid);
    } else if (cs >= s - tol) {
      const double csd = static_cast<double>(cx) + gumbel64(cw);
      const double bsd = exact();
      if (csd > bsd || (csd == bsd && cid < id)) {
        take(cs, cx, cl, cw, cid);
        sd = csd;
        have_sd = true;
      }
    }
  }
};

// Per-warp queue of kept tokens in shared memory (kDrawQueue entries per
// warp, each a 32-bit payload and the token id).  A pass that finds kept
// tokens scattered among many dropped ones queues them, and the warp works
// on 32 queued tokens at a time, one per lane, so the per-token work (the
// Philox words, the quotient, the exp) runs at full width instead of once per
// warp step whenever any lane has a kept token.  Every lane of the warp
// calls push and drain together (the count n is warp-uniform).
// A queue may also carry each token's Philox word (kWords: the pass computed
// it once per float4 group, for rows where most groups hold a kept token).
constexpr int kDrawQueue = 160;  // a drain leaves < 32 entries; at most 128 are pushed before the next
constexpr size_t kDrawQueueBytes = static_cast<size_t>(kWarps) * kDrawQueue * 12;
template <bool kWords>
struct DrawQueue {
  uint64_t* q;   // this warp's entries: payload << 32 | id
  uint32_t* wq;  // (kWords) their Philox words
  uint32_t n;
  __device__ __forceinline__ void init(void* base) {
    q = reinterpret_cast<uint64_t*>(base) + (threadIdx.x >> 5) * kDrawQueue;
    wq = reinterpret_cast<uint32_t*>(reinterpret_cast<uint64_t*>(base) + kWarps * kDrawQueue) +
         (threadIdx.x >> 5) * kDrawQueue;
    n = 0;
  }
  __device__ __forceinline__ void push(bool pred, uint64_t e, uint32_t word = 0u) {
    const uint32_t m = __ballot_sync(0xFFFFFFFFu, pred);
    if (pred) {
      const uint32_t i = n + __popc(m & ((1u << (threadIdx.x & 31)) - 1u));
      q[i] = e;
      if (kWords) wq[i] = word;
    }
    n += __popc(m);
  }
  // Takes queued tokens 32 at a time while a full batch is queued (all:
  // until the queue is empty), each through one(payload, Philox word, id).
  template <typename F>
  __device__ __forceinline__ void drain(bool all, uint32_t pos, uint32_t req, uint32_t k0, uint32_t k1, F&& one) {
    while (n >= 32u || (all && n > 0u)) {
      __syncwarp();
      const uint32_t lane = threadIdx.x & 31;
      const uint32_t take = min(n, 32u);
      const uint32_t base = n - take;
      const bool act = lane < take;
      const uint64_t e = act ? q[base + lane] : 0ull;
      const uint32_t wd = (kWords && act) ? wq[base + lane] : 0u;
      __syncwarp();
      n = base;
      if (act) {
        const uint32_t id = static_cast<uint32_t>(e);
        uint32_t word = wd;
        if (!kWords) word = word_of(philox4x32_10(make_uint4(id >> 2, pos, req, 0u), k0, k1), static_cast<int>(id & 3u));
        one(static_cast<uint32_t>(e >> 32), word, static_cast<int32_t>(id));
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
__device__ __forceinline__ int block_min_i(int v, SharedHeader* H) { return -block_max_i(-v, H); }

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
// Inclusive prefix sum of fixed-point values over threads: exact.
__device__ __forceinline__ void block_scan_fx(Fx4& x, SharedHeader* H) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const unsigned long long y = __shfl_up_sync(0xFFFFFFFFu, x.v[k], o);
      if (lane >= o) x.v[k] += y;
    }
  }
  __syncthreads();
  if (lane == 31)
#pragma unroll
    for (int k = 0; k < 4; ++k) H->scan_fx[warp][k] = x.v[k];
  __syncthreads();
  for (int i = 0; i < warp; ++i)
#pragma unroll
    for (int k = 0; k < 4; ++k) x.v[k] += H->scan_fx[i][k];
  __syncthreads();
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

// Ascending bitonic sort of n u64 keys in shared memory, n a power of two,
// 2 <= n <= 8 * kThreads.  Thread t holds elements [t E, t E + E) in registers
// (E = max(1, n / kThreads); threads past n hold ~0 and only swap among
// themselves): a step of stride j < E swaps registers of one thread, j < 32 E
// goes through warp shuffles, and only the larger strides go through shared
// memory, so 2048 keys take 6 barrier-separated steps instead of 66.
template <int E>
__device__ __forceinline__ void sort_step_regs(uint64_t (&v)[E], int base, int k, int j) {
#pragma unroll
  for (int i = 0; i < E; ++i) {
#pragma unroll
    for (int jj = 1; jj < E; jj <<= 1) {
      if (jj == j && (i & jj) == 0) {
        const bool up = ((base + i) & k) == 0;
        const uint64_t x = v[i], y = v[i + jj];
        const bool sw = (x > y) == up;
        v[i] = sw ? y : x;
        v[i + jj] = sw ? x : y;
      }
    }
  }
}
template <int E>
__device__ void bitonic_sort_e(uint64_t* a, int n) {
  uint64_t v[E];
  const int base = static_cast<int>(threadIdx.x) * E;
#pragma unroll
  for (int i = 0; i < E; ++i) v[i] = base + i < n ? a[base + i] : ~0ull;
  for (int k = 2; k <= n; k <<= 1) {
    for (int j = k >> 1; j > 0; j >>= 1) {
      if (j < E) {
        sort_step_regs<E>(v, base, k, j);
      } else if (j < 32 * E) {
        const int lj = j / E;  // the partner is lane ^ lj, same register
#pragma unroll
        for (int i = 0; i < E; ++i) {
          const uint64_t y = __shfl_xor_sync(0xFFFFFFFFu, v[i], lj);
          const int e = base + i;
          const bool keep_min = ((e & j) == 0) == ((e & k) == 0);
          v[i] = keep_min ? min(v[i], y) : max(v[i], y);
        }
      } else {
        __syncthreads();
#pragma unroll
        for (int i = 0; i < E; ++i)
          if (base + i < n) a[base + i] = v[i];
        __syncthreads();
#pragma unroll
        for (int i = 0; i < E; ++i) {
          const int e = base + i;
          if (e < n) {
            const uint64_t y = a[e ^ j];
            const bool keep_min = ((e & j) == 0) == ((e & k) == 0);
            v[i] = keep_min ? min(v[i], y) : max(v[i], y);
          }
        }
      }
    }
  }
  __syncthreads();
#pragma unroll
  for (int i = 0; i < E; ++i)
    if (base + i < n) a[base + i] = v[i];
  __syncthreads();
}
__device__ void bitonic_sort(uint64_t* a, int n) {
  if (n <= kThreads) bitonic_sort_e<1>(a, n);
  else if (n <= 2 * kThreads) bitonic_sort_e<2>(a, n);
  else if (n <= 4 * kThreads) bitonic_sort_e<4>(a, n);
  else bitonic_sort_e<8>(a, n);
}

// ------------------------------------------------------------------ per-CTA context
struct Ctx {
  const SampleArgs* a;
  SharedHeader* H;
  float4* part4;
  uint8_t* scratch;
  uint64_t* list;
  int row, n4;
  long long g0;          // global id of the first element of this CTA's part
  uint32_t rank, C;
  float T, top_p;
  int top_k;
  uint32_t req, pos;
};

// Sum over the cluster's CTAs of one shared variable (loads issued together).
template <typename T>
__device__ __forceinline__ T cluster_sum(const Ctx& cx, const T* local) {
  T v[kMaxCluster];
#pragma unroll
  for (int r = 0; r < kMaxCluster; ++r) v[r] = r < static_cast<int>(cx.C) ? *cluster_ptr(local, r) : T(0);
  T t = 0;
#pragma unroll
  for (int r = 0; r < kMaxCluster; ++r) t += v[r];
  return t;
}

// Raw-key lower bound for l such that fl(l / T) >= theta is possible.
__device__ uint32_t raw_prefilter(float theta, float T) {
  if (theta == -INFINITY) return kKeyNegInf + 1;
  const float t2 = nextafterf(nextafterf(theta, -INFINITY), -INFINITY);
  const double lo = static_cast<double>(t2) * static_cast<double>(T);
  const float lo32 = __double2float_rd(lo);
  if (!(lo32 > -INFINITY)) return kKeyNegInf + 1;
  return fkey(lo32);
}

// Warp-aggregated append of sort keys to a list in this CTA's own shared memory.
__device__ __forceinline__ void local_append(uint32_t* counter, uint64_t* list, bool pred, uint64_t key) {
  const uint32_t mask = __ballot_sync(0xFFFFFFFFu, pred);
  if (mask == 0) return;
  const int lane = threadIdx.x & 31;
  const int first = __ffs(mask) - 1;
  uint32_t base = 0;
  if (lane == first) base = atomicAdd(counter, static_cast<uint32_t>(__popc(mask)));
  base = __shfl_sync(0xFFFFFFFFu, base, first);
  if (pred) {
    const uint32_t idx = base + __popc(mask & ((1u << lane) - 1u));
    if (idx < static_cast<uint32_t>(kListCap)) list[idx] = key;
  }
}

// After a local collection into this CTA's list (count in list_aux): a
// non-leader reserves its exact count in the leader's list with one remote
// atomic and copies its entries there.  The leader collects in place.
__device__ void publish_local_list(const Ctx& cx) {
  SharedHeader* H = cx.H;
  if (cx.rank == 0) return;
  __syncthreads();
  const uint32_t cnt = min(H->list_aux, static_cast<uint32_t>(kListCap));
  if (threadIdx.x == 0) H->list_base = atom_add_dsmem_u32(mapa(smem_u32(&H->list_count), 0), cnt);
  __syncthreads();
  const uint32_t base = H->list_base;
  uint64_t* dst = cluster_ptr(cx.list, 0);
  for (uint32_t i = threadIdx.x; i < cnt; i += kThreads)
    if (base + i < static_cast<uint32_t>(kListCap)) dst[base + i] = cx.list[i];
}
// Counter and list a collection appends to: the leader's own, or a staging one.
__device__ __forceinline__ uint32_t* collect_counter(const Ctx& cx) {
  return cx.rank == 0 ? &cx.H->list_count : &cx.H->list_aux;
}

// ---- pass 1: stats + raw-key histogram, chunk by chunk as the bulk copies land
__device__ void pass_stats(const Ctx& cx, const int* chunk_q, uint32_t parity) {
  uint32_t* hist = reinterpret_cast<uint32_t*>(cx.scratch);
  uint32_t kmax = 0, kminf = 0xFFFFFFFFu, bad = 0;
  float m = -INFINITY, s = 0.0f;
  bool load_ok = true;
  constexpr float kLog2e = 1.4426950408889634f;
  for (int c = 0; c < kLoadChunks; ++c) {
    if (load_ok && !mbar_wait_bounded(smem_u32(&cx.H->mbar[c]), parity)) {
      if (threadIdx.x == 0) atomicOr(cx.a->err, kErrSampleLoad);
      load_ok = false;
    }
    for (int q = chunk_q[c] + threadIdx.x; q < chunk_q[c + 1]; q += kThreads) {
      const float4 v4 = cx.part4[q];
      const float v[4] = {v4.x, v4.y, v4.z, v4.w};
      float mx = -INFINITY;
      bool fin[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const uint32_t raw = __float_as_uint(v[i]);
        const bool nb = nan_or_pos_inf(raw);
        bad |= nb ? 1u : 0u;
        const uint32_t k = fkey_bits(raw);
        kmax = max(kmax, k);
        fin[i] = key_finite(k) && !nb;
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
  }
  // block reduce
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    kmax = max(kmax, __shfl_xor_sync(0xFFFFFFFFu, kmax, o));
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
    H->red_u[warp * 4 + 2] = kminf;
    H->red_u[warp * 4 + 3] = bad | (load_ok ? 0u : 1u);
    H->red_f[warp * 2 + 0] = m;
    H->red_f[warp * 2 + 1] = s;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    uint32_t a = 0, c = 0xFFFFFFFFu, d = 0;
    float M = -INFINITY;
    for (int i = 0; i < kWarps; ++i) {
      d |= H->red_u[i * 4 + 3];
      a = max(a, H->red_u[i * 4 + 0]);
      c = min(c, H->red_u[i * 4 + 2]);
      M = fmaxf(M, H->red_f[i * 2]);
    }
    float S = 0.0f;
    if (M > -INFINITY)
      for (int i = 0; i < kWarps; ++i)
        if (H->red_f[i * 2] > -INFINITY) S += H->red_f[i * 2 + 1] * fast_exp2((H->red_f[i * 2] - M) * kLog2e);
    H->stats.kmax = a;
    H->stats.kminf = c;
    H->stats.bad = d;
    H->stats.m = M;
    H->stats.s = S;
  }
  __syncthreads();  // every thread reads the CTA's stats next (local_pick)
}

// ---- COLLECT_RAW: raw keys >= lo -> leader list (sort key: ~key, id)
__device__ void op_collect_raw(const Ctx& cx, const Plan& p) {
  uint32_t* counter = collect_counter(cx);
  if (cx.rank != 0) {
    if (threadIdx.x == 0) cx.H->list_aux = 0;
    __syncthreads();
  }
  const int nq = (cx.n4 + kThreads - 1) / kThreads * kThreads;
  for (int q = threadIdx.x; q < nq; q += kThreads) {
    const bool valid = q < cx.n4;
    const float4 v4 = valid ? cx.part4[q] : make_float4(0.f, 0.f, 0.f, 0.f);
    const float v[4] = {v4.x, v4.y, v4.z, v4.w};
    uint32_t k[4];
    bool any = false;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      k[i] = fkey(v[i]);
      any |= valid && k[i] >= p.lo;
    }
    if (!__any_sync(0xFFFFFFFFu, any)) continue;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const bool pred = valid && k[i] >= p.lo;
      const uint32_t gid = static_cast<uint32_t>(cx.g0 + 4 * q + i);
      local_append(counter, cx.list, pred, (static_cast<uint64_t>(~k[i]) << 32) | gid);
    }
  }
  publish_local_list(cx);
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
    CtaStats* dst = cluster_ptr(&H->all[cx.rank], 0);
    dst->nm_key = k;
    dst->nm_id = id;
  }
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

// Fixed-point mass bins in the scratch area: limb[4][256], cnt[256], edge[256]
// (u32 only: the only shared-memory atomics that are native on this part).
struct MassBins {
  uint32_t* limb;   // limb[k * 256 + bin]
  uint32_t* cnt;
  uint32_t* edge;
};
__device__ __forceinline__ MassBins mass_bins(uint8_t* scratch) {
  MassBins b;
  b.limb = reinterpret_cast<uint32_t*>(scratch);
  b.cnt = b.limb + 4 * kSubBins;
  b.edge = b.cnt + kSubBins;
  return b;
}
__device__ __forceinline__ void clear_mass_bins(const MassBins& b) {
  for (int i = threadIdx.x; i < 5 * kSubBins; i += kThreads) b.limb[i] = 0;  // limbs and counts
  __syncthreads();
}
__device__ __forceinline__ void add_mass(const MassBins& b, uint32_t bin, double e) {
  const unsigned long long q = mass_q(e);
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const uint32_t limb = static_cast<uint32_t>((q >> (16 * k)) & 0xFFFFull);
    if (limb) atomicAdd(&b.limb[k * kSubBins + bin], limb);
  }
  atomicAdd(&b.cnt[bin], 1u);
}
// Sum over the cluster's CTAs of a u32 shared variable, widened to 64 bits.
__device__ __forceinline__ unsigned long long cluster_sum_wide(const Ctx& cx, const uint32_t* local) {
  unsigned long long v[kMaxCluster];
#pragma unroll
  for (int r = 0; r < kMaxCluster; ++r) v[r] = r < static_cast<int>(cx.C) ? *cluster_ptr(local, r) : 0ull;
  unsigned long long t = 0;
#pragma unroll
  for (int r = 0; r < kMaxCluster; ++r) t += v[r];
  return t;
}
// Cluster-wide fixed-point mass of bin j.
__device__ __forceinline__ Fx4 bin_mass(const Ctx& cx, const MassBins& b, int j) {
  Fx4 f;
#pragma unroll
  for (int k = 0; k < 4; ++k) f.v[k] = cluster_sum_wide(cx, b.limb + k * kSubBins + j);
  return f;
}

// ---- MASS: x = fl(l / T) written in place (unless the part holds x already); survivors' masses on bins of
// equal width in x below m (exact key edges), exact fixed point.
__device__ void op_mass(const Ctx& cx, const Plan& p) {
  const MassBins b = mass_bins(cx.scratch);
  for (int j = threadIdx.x; j <= kMassBins; j += kThreads) b.edge[j] = mass_edge(p.m, p.step, j);
  clear_mass_bins(b);
  const double m = p.m;
  const float inv_step = 1.0f / p.step;
  const double* tab = cx.H->exp_tab;
  for (int q = threadIdx.x; q < cx.n4; q += kThreads) {
    float4 v4 = cx.part4[q];
    float v[4] = {v4.x, v4.y, v4.z, v4.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float x = p.part_is_x ? v[i] : key_finite(fkey(v[i])) ? scale_x(v[i], cx.T) : -INFINITY;
      v[i] = x;
      if (x >= p.theta && x > -INFINITY)
        add_mass(b, mass_bin(b.edge, p.m, inv_step, x, fkey(x)), exp_neg64(static_cast<double>(x) - m, tab));
    }
    if (!p.part_is_x) cx.part4[q] = make_float4(v[0], v[1], v[2], v[3]);
  }
}

// ---- NARROW_MASS: survivors' masses of x-keys in [lo, hi] on 256 bins from the top
__device__ void op_narrow_mass(const Ctx& cx, const Plan& p) {
  const MassBins b = mass_bins(cx.scratch);
  clear_mass_bins(b);
  const double m = p.m;
  const double* tab = cx.H->exp_tab;
  for (int q = threadIdx.x; q < cx.n4; q += kThreads) {
    const float4 v4 = cx.part4[q];
    const float v[4] = {v4.x, v4.y, v4.z, v4.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint32_t xk = fkey(v[i]);
      if (xk >= p.lo && xk <= p.hi && v[i] >= p.theta && v[i] > -INFINITY)
        add_mass(b, (p.hi - xk) >> p.shift, exp_neg64(static_cast<double>(v[i]) - m, tab));
    }
  }
}

// Pushes this CTA's best draw candidate into the leader's slot [rank].
__device__ __forceinline__ void push_best(const Ctx& cx, Best& b) {
  double sd = b.valid ? b.exact() : -INFINITY;
  int32_t id = b.valid ? b.id : 0x7FFFFFFF;
  float l = b.valid ? b.l : 0.0f;
  block_best(sd, id, l, cx.H);
  if (threadIdx.x == 0) {
    const uint32_t slot = mapa(smem_u32(&cx.H->best[cx.rank]), 0);
    st_dsmem_u64(slot, static_cast<uint64_t>(__double_as_longlong(sd)));
    st_dsmem_u32(slot + 8, static_cast<uint32_t>(id));
    st_dsmem_u32(slot + 12, __float_as_uint(l));
  }
}

// ---- COLLECT_X: survivors (x >= theta, x in shared memory) with x-key in
// [lo, hi] -> leader list (sort key: ~xkey, id).  Every survivor above the
// range is kept whatever the cut inside it, so the same pass draws over them:
// the CTA's best is pushed to the leader, which adds the range's kept entries.
__device__ void op_collect_x(const Ctx& cx, const Plan& p) {
  uint32_t* counter = collect_counter(cx);
  if (cx.rank != 0) {
    if (threadIdx.x == 0) cx.H->list_aux = 0;
    __syncthreads();
  }
  if (threadIdx.x == 0) cx.H->gbound = kKeyNegInf;
  __syncthreads();
  Best b;
  b.init(&cx.H->gbound);
  const uint32_t k0 = static_cast<uint32_t>(cx.a->seed), k1 = static_cast<uint32_t>(cx.a->seed >> 32);
  constexpr float kGMax = 16.7f;  // > the largest noise value, -log(-log(1 - 2^-24)) = 16.63
  const int nq = (cx.n4 + kThreads - 1) / kThreads * kThreads;
  for (int q = threadIdx.x; q < nq; q += kThreads) {
    const bool valid = q < cx.n4;
    const float4 v4 = valid ? cx.part4[q] : make_float4(-INFINITY, -INFINITY, -INFINITY, -INFINITY);
    const float v[4] = {v4.x, v4.y, v4.z, v4.w};
    uint32_t k[4];
    bool pred[4], above[4];
    bool any = false, any_above = false;
    float xmax = -INFINITY;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      k[i] = fkey(v[i]);
      const bool surv = valid && v[i] >= p.theta && v[i] > -INFINITY;
      pred[i] = surv && k[i] >= p.lo && k[i] <= p.hi;
      above[i] = surv && k[i] > p.hi;
      any |= pred[i];
      any_above |= above[i];
      if (above[i]) xmax = fmaxf(xmax, v[i]);
    }
    if (__any_sync(0xFFFFFFFFu, any)) {
#pragma unroll
      for (int i = 0; i < 4; ++i)
        local_append(counter, cx.list, pred[i],
                     (static_cast<uint64_t>(~k[i]) << 32) | static_cast<uint32_t>(cx.g0 + 4 * q + i));
    }
    if (!any_above) continue;
    {
      const float sb = b.bound_score();
      if (sb > -INFINITY && xmax + kGMax < sb - score_tol(sb)) continue;
    }
    const long long gid0 = cx.g0 + 4LL * q;
    const uint4 w = philox4x32_10(make_uint4(static_cast<uint32_t>(gid0 >> 2), cx.pos, cx.req, 0u), k0, k1);
    const float bl = b.bound_l2e();
#pragma unroll
    for (int i = 0; i < 4; ++i)
      if (above[i] && (bl == Best::kNoBound || !Best::rejects(bl, v[i], word_of(w, i))))
        b.offer_passed(v[i], 0.0f, word_of(w, i), static_cast<int32_t>(gid0 + i));
  }
  publish_local_list(cx);
  push_best(cx, b);
}

// ---- GUMBEL: argmax of x + g over kept elements (x >= theta), float64-exact;
// the CTA's best is pushed into the leader's slot [rank].  On raw logits the
// tests run first on xa = l * (1 / T), within |xa| * 2^-21 of x = fl(l / T), and
// the division is done only for the rare element that passes them.
__device__ void op_gumbel(const Ctx& cx, const Plan& p) {
  if (threadIdx.x == 0) cx.H->gbound = kKeyNegInf;
  __syncthreads();
  Best b;
  b.init(&cx.H->gbound);
  const uint32_t k0 = static_cast<uint32_t>(cx.a->seed), k1 = static_cast<uint32_t>(cx.a->seed >> 32);
  constexpr float kGMax = 16.7f;  // > -log(-log(1 - 2^-24)) = 16.63: the largest noise value
  const float invT = __frcp_rn(cx.T);
  const bool approx = !p.part_is_x && invT < INFINITY;
  for (int q = threadIdx.x; q < cx.n4; q += kThreads) {
    const float4 v4 = cx.part4[q];
    const float v[4] = {v4.x, v4.y, v4.z, v4.w};
    float xu[4];  // upper bound of x (exact on an x part)
    bool maybe[4];
    bool any = false;
    float xmax = -INFINITY;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      if (p.part_is_x) {
        xu[i] = v[i];
      } else if (approx) {
        const float xa = key_finite(fkey(v[i])) ? v[i] * invT : -INFINITY;
        xu[i] = xa + fabsf(xa) * 5e-7f + 1e-37f;
      } else {
        xu[i] = key_finite(fkey(v[i])) ? scale_x(v[i], cx.T) : -INFINITY;
      }
      maybe[i] = xu[i] >= p.theta && xu[i] > -INFINITY;
      if (maybe[i]) xmax = fmaxf(xmax, xu[i]);
      any |= maybe[i];
    }
    // no kept element of this group can beat the current best, whatever its noise
    if (!any) continue;
    const float sb = b.bound_score();
    if (sb > -INFINITY && xmax + kGMax < sb - score_tol(sb)) continue;
    const long long gid0 = cx.g0 + 4LL * q;
    const uint4 w = philox4x32_10(make_uint4(static_cast<uint32_t>(gid0 >> 2), cx.pos, cx.req, 0u), k0, k1);
    const float bl = b.bound_l2e();
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      if (!maybe[i]) continue;
      const uint32_t wi = word_of(w, i);
      if (bl != Best::kNoBound && Best::rejects(bl, xu[i], wi)) continue;
      const float x = p.part_is_x ? v[i] : scale_x(v[i], cx.T);
      if (x >= p.theta) b.offer_passed(x, p.part_is_x ? 0.0f : v[i], wi, static_cast<int32_t>(gid0 + i));
    }
  }
  push_best(cx, b);
}

// ---- XHIST: x = fl(l / T) written in place, and per fine bin below m (p.m,
// bins per unit p.step) the count of the finite x and the sum of their
// quantised in-bin offsets; then CTA r replaces its own bins [r, r + 1) *
// kXBins / C with their sums over the cluster (only CTA r reads that slice of
// any CTA, so the slice can be overwritten in place).
__device__ void op_xhist(const Ctx& cx, const Plan& p, uint32_t collect_lo = 0xFFFFFFFFu) {
  uint32_t* cnt = reinterpret_cast<uint32_t*>(cx.scratch);
  uint32_t* qs = cnt + kXBins;
  for (int i = threadIdx.x; i < 2 * kXBins; i += kThreads) cnt[i] = 0;
  // collect_lo: the raw keys at or above it are this CTA's first-pass candidates,
  // listed here (the conversion below reads every logit anyway)
  const bool collect = collect_lo != 0xFFFFFFFFu;
  uint32_t* counter = collect_counter(cx);
  if (collect && cx.rank != 0 && threadIdx.x == 0) cx.H->list_aux = 0;
  __syncthreads();
  // x = fl(l / T): the fused quotient where it is exact (T in [2^-20, 2^20] and
  // l zero or 2^-60 <= |l| <= 2^100, checked per logit), else the IEEE division
  // out of line (a rare, divergent branch)
  const float yT = __frcp_rn(cx.T);
  const bool t_ok = cx.T >= 0x1p-20f && cx.T <= 0x1p20f;
  const int nq = (cx.n4 + kThreads - 1) / kThreads * kThreads;  // whole warps: the appends are warp-wide
  for (int q = threadIdx.x; q < nq; q += kThreads) {
    const bool valid = q < cx.n4;
    const float4 v4 = valid ? cx.part4[q] : make_float4(-INFINITY, -INFINITY, -INFINITY, -INFINITY);
    float v[4] = {v4.x, v4.y, v4.z, v4.w};
    if (collect) {
      uint32_t k[4];
      bool any = false;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        k[i] = fkey(v[i]);
        any |= valid && k[i] >= collect_lo;
      }
      if (__any_sync(0xFFFFFFFFu, any)) {
#pragma unroll
        for (int i = 0; i < 4; ++i)
          local_append(counter, cx.list, valid && k[i] >= collect_lo,
                       (static_cast<uint64_t>(~k[i]) << 32) | static_cast<uint32_t>(cx.g0 + 4 * q + i));
      }
    }
    if (!valid) continue;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const bool fin = key_finite(fkey(v[i]));
      const float al = fabsf(v[i]);
      float x = -INFINITY;
      if (fin) {
        if (t_ok && (al == 0.0f || (al >= 0x1p-60f && al <= 0x1p100f))) x = scale_x_fast(v[i], cx.T, yT);
        else x = div_ieee(v[i], cx.T);
      }
      v[i] = x;
      if (fin) {
        uint32_t qo;
        const int j = xbin_q(x, p.m, p.step, qo);
        atomicAdd(&cnt[j], 1u);
        atomicAdd(&qs[j], qo);
      }
    }
    cx.part4[q] = make_float4(v[0], v[1], v[2], v[3]);
  }
  if (collect) publish_local_list(cx);
  __syncthreads();
  cluster_sync();  // every CTA's counts are complete
  const int per = kXBins / static_cast<int>(cx.C);
  const int j0 = static_cast<int>(cx.rank) * per;
  for (int j = j0 + threadIdx.x; j < j0 + per; j += kThreads) {
    const uint32_t tc = cluster_sum(cx, cnt + j);
    const uint32_t tq = cluster_sum(cx, qs + j);
    cnt[j] = tc;
    qs[j] = tq;
  }
}

// Deterministic block sum of a double (fixed shuffle tree, warps in order);
// thread 0 gets the total.
__device__ __forceinline__ double block_sum_d0(double v, SharedHeader* H) {
  v = warp_reduce(v, [](double a, double b) { return a + b; });
  __syncthreads();
  if ((threadIdx.x & 31) == 0) H->red_d[threadIdx.x >> 5] = v;
  __syncthreads();
  double t = 0.0;
  if (threadIdx.x == 0)
    for (int i = 0; i < kWarps; ++i) t += H->red_d[i];
  return t;
}

// Block minimum of a float; thread 0 gets it.
__device__ __forceinline__ float block_min_f0(float v, SharedHeader* H) {
  v = warp_reduce(v, [](float a, float b) { return fminf(a, b); });
  __syncthreads();
  if ((threadIdx.x & 31) == 0) H->red_f[threadIdx.x >> 5] = v;
  __syncthreads();
  float t = INFINITY;
  if (threadIdx.x == 0)
    for (int i = 0; i < kWarps; ++i) t = fminf(t, H->red_f[i]);
  return t;
}

// ---- EXACT: with the window of fine bins [lo, hi] that may hold the top-p
// cut, every finite x above the window is kept for certain (its float64 mass
// summed, the draw run over it here), every x below it is dropped (mass
// summed), and the window's members go to the leader's list (sort key ~xkey, id).
__device__ void op_exact(const Ctx& cx, const Plan& p) {
  uint32_t* counter = collect_counter(cx);
  if (cx.rank != 0) {
    if (threadIdx.x == 0) cx.H->list_aux = 0;
    __syncthreads();
  }
  if (threadIdx.x == 0) cx.H->gbound = kKeyNegInf;
  __syncthreads();
  Best b;
  b.init(&cx.H->gbound);
  const uint32_t k0 = static_cast<uint32_t>(cx.a->seed), k1 = static_cast<uint32_t>(cx.a->seed >> 32);
  constexpr float kGMax = 16.7f;
  const double m = p.m;
  const double* tab = cx.H->exp_tab;
  const int jlo = static_cast<int>(p.lo), jhi = static_cast<int>(p.hi);
  double above = 0.0, below = 0.0;
  float xmin_ab = INFINITY;  // smallest x above the window (theta_p when the window keeps nothing)
  // two float4 groups per iteration (q and q + kThreads): their float64 exps
  // and Philox words are independent chains the warp issues interleaved
  const int nq = (cx.n4 + kThreads - 1) / kThreads * kThreads;
  for (int q0 = threadIdx.x; q0 < nq; q0 += 2 * kThreads) {
    float v[2][4];
    bool win[2][4], ab[2][4];
    bool any_win[2] = {false, false}, any_ab[2] = {false, false};
    float xmax[2] = {-INFINITY, -INFINITY};
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int q = q0 + u * kThreads;
      const float4 v4 = q < cx.n4 ? cx.part4[q] : make_float4(-INFINITY, -INFINITY, -INFINITY, -INFINITY);
      v[u][0] = v4.x;
      v[u][1] = v4.y;
      v[u][2] = v4.z;
      v[u][3] = v4.w;
    }
#pragma unroll
    for (int u = 0; u < 2; ++u)
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const bool fin = v[u][i] > -INFINITY;
        const int j = fin ? xbin(v[u][i], p.m, p.step) : kXBins;
        win[u][i] = fin && j >= jlo && j <= jhi;
        ab[u][i] = fin && j < jlo;
        // exp(-inf - m) is the clamped, negligible value: no branch around the chain
        const double e = exp_neg64(static_cast<double>(v[u][i]) - m, tab);
        const double ee = (fin && !win[u][i]) ? e : 0.0;
        above += ab[u][i] ? ee : 0.0;
        below += ab[u][i] ? 0.0 : ee;
        any_win[u] |= win[u][i];
        any_ab[u] |= ab[u][i];
        if (ab[u][i]) {
          xmax[u] = fmaxf(xmax[u], v[u][i]);
          xmin_ab = fminf(xmin_ab, v[u][i]);
        }
      }
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int q = q0 + u * kThreads;
      if (__any_sync(0xFFFFFFFFu, any_win[u])) {
#pragma unroll
        for (int i = 0; i < 4; ++i)
          local_append(counter, cx.list, win[u][i],
                       (static_cast<uint64_t>(~fkey(v[u][i])) << 32) | static_cast<uint32_t>(cx.g0 + 4 * q + i));
      }
    }
    // a group no kept element of which can beat the current best, whatever its noise, is skipped
    bool need[2];
    {
      const float sb = b.bound_score();
#pragma unroll
      for (int u = 0; u < 2; ++u) need[u] = any_ab[u] && !(sb > -INFINITY && xmax[u] + kGMax < sb - score_tol(sb));
    }
    if (!(need[0] || need[1])) continue;
    uint4 w[2];
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const long long gid0 = cx.g0 + 4LL * (q0 + u * kThreads);
      w[u] = philox4x32_10(make_uint4(static_cast<uint32_t>(gid0 >> 2), cx.pos, cx.req, 0u), k0, k1);
    }
    const float bl = b.bound_l2e();  // a bound a little behind the best is still a valid one
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      if (!need[u]) continue;
      const long long gid0 = cx.g0 + 4LL * (q0 + u * kThreads);
#pragma unroll
      for (int i = 0; i < 4; ++i)
        if (ab[u][i] && (bl == Best::kNoBound || !Best::rejects(bl, v[u][i], word_of(w[u], i))))
          b.offer_passed(v[u][i], 0.0f, word_of(w[u], i), static_cast<int32_t>(gid0 + i));
    }
  }
  const double ta = block_sum_d0(above, cx.H);
  const double tb = block_sum_d0(below, cx.H);
  const float tx = block_min_f0(xmin_ab, cx.H);
  if (threadIdx.x == 0) {
    *cluster_ptr(&cx.H->ex_above[cx.rank], 0) = ta;
    *cluster_ptr(&cx.H->ex_below[cx.rank], 0) = tb;
    *cluster_ptr(&cx.H->ex_xmin[cx.rank], 0) = tx;
  }
  publish_local_list(cx);
  push_best(cx, b);
}

// ---- per-CTA candidate threshold from this CTA's own histogram: the bin where
// the running count from its max reaches `rank`.  Every element of the row's
// top `rank` is in its CTA's local top `rank`, so the union of the per-CTA
// collections holds the row's top `rank` (ties included: bins hold equal keys).
struct LocalPick {
  uint32_t lo, need, ok;
};
__device__ LocalPick local_pick(const Ctx& cx, uint32_t rank, bool check_T) {
  const uint32_t* hist = reinterpret_cast<const uint32_t*>(cx.scratch);
  SharedHeader* H = cx.H;
  const int top = static_cast<int>(H->stats.kmax >> 20);
  uint32_t cum = 0;
  if (threadIdx.x == 0) H->L.found_bin = -1;  // scratch use in every CTA
  __syncthreads();
  for (int base = 0; base <= top; base += kThreads) {
    const int j = base + threadIdx.x;
    const uint32_t c = j <= top ? hist[top - j] : 0u;
    uint32_t tot;
    const uint32_t incl = block_scan_u(c, &tot, H);
    if (c > 0 && cum + incl >= rank && cum + incl - c < rank) {
      H->L.found_bin = top - j;
      H->L.found_cum = cum + incl;
    }
    cum += tot;
    __syncthreads();
    if (H->L.found_bin >= 0) break;
  }
  LocalPick lp;
  if (H->L.found_bin < 0) {  // fewer than `rank` elements here: take them all
    lp.lo = 0;
    lp.need = cum;
  } else {
    lp.lo = static_cast<uint32_t>(H->L.found_bin) << 20;
    lp.need = H->L.found_cum;
  }
  __syncthreads();
  // top-k survivors: no element below the bin may scale to the bin's lowest x
  lp.ok = 1;
  if (check_T && lp.lo > kKeyNegInf + 1)
    lp.ok = scale_x(key_value(lp.lo - 1), cx.T) < scale_x(key_value(lp.lo), cx.T) ? 1u : 0u;
  return lp;
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

// Scan the C CTAs' u32 histograms (bin b at cnt[b]); visit bins j = 0.. as
// bin(j) = desc ? top - j : j; find the bin where the running count reaches
// `rank`.  Sets L.found_bin (or -1), L.found_cum (count strictly before it)
// and L.found_cnt (its count).
__device__ void find_rank_bin(const Ctx& cx, const uint32_t* cnt_local, int top, int nbins, bool desc,
                              uint32_t rank, LeaderState& L) {
  uint32_t cum = 0;
  if (threadIdx.x == 0) L.found_bin = -1;
  __syncthreads();
  for (int base = 0; base < nbins; base += kThreads) {
    const int j = base + threadIdx.x;
    uint32_t c = 0;
    if (j < nbins) {
      const int b = desc ? top - j : j;
      c = cluster_sum(cx, cnt_local + b);
    }
    uint32_t tot;
    const uint32_t incl = block_scan_u(c, &tot, cx.H);
    if (j < nbins && c > 0 && cum + incl >= rank && cum + incl - c < rank) {
      L.found_bin = desc ? top - j : j;
      L.found_cum = cum + incl - c;
      L.found_cnt = c;
    }
    cum += tot;
    __syncthreads();
    if (L.found_bin >= 0) break;
  }
  __syncthreads();
}

// Mass bins merged over the cluster; finds the last non-empty bin whose exact
// mass strictly above (cum + bins before it) is < top_p * Z.  Sets
// L.found_bin, L.found_above (mass above it) and L.found_cnt (its count).
__device__ void find_mass_bin(const Ctx& cx, int nbins, LeaderState& L) {
  const MassBins b = mass_bins(cx.scratch);
  const int j = threadIdx.x;
  Fx4 own = fx_zero();
  uint32_t c = 0;
  if (j < nbins) {
    own = bin_mass(cx, b, j);
    c = static_cast<uint32_t>(cluster_sum_wide(cx, b.cnt + j));
  }
  Fx4 incl = own;
  block_scan_fx(incl, cx.H);
  const Fx4 above = fx_add(L.cum, fx_sub(incl, own));  // exact mass strictly above bin j
  const double pz = static_cast<double>(L.top_p) * fx_to_double(L.z);
  const bool cand = j < nbins && c > 0 && fx_to_double(above) < pz;
  const int best = block_max_i(cand ? j : -1, cx.H);
  if (threadIdx.x == 0) L.found_bin = -1;
  __syncthreads();
  if (best >= 0 && j == best) {
    L.found_bin = j;
    L.found_above = above;
    L.found_cnt = c;
  }
  __syncthreads();
}

// The kept-set thresholds of a row (optional output): theta_k and theta_p on
// x = fl(l / T); -inf for a rule that is off, NaN for a greedy or flagged row.
// The draw's kept set is every finite x >= max(theta_k, theta_p).
__device__ __forceinline__ void write_kept_theta(const SampleArgs& a, int row, float theta_k, float theta_p) {
  if (a.kept_theta != nullptr) {
    a.kept_theta[2 * static_cast<size_t>(row)] = theta_k;
    a.kept_theta[2 * static_cast<size_t>(row) + 1] = theta_p;
  }
}

__device__ void write_outputs(const Ctx& cx, LeaderState& L) {
  if (threadIdx.x == 0) {
    const SampleArgs& a = *cx.a;
    a.token_ids[cx.row] = L.token;
    a.token_logprob[cx.row] = L.token_l - L.lse;
    a.row_flags[cx.row] = 0;
    const float nan = __int_as_float(0x7FC00000);
    write_kept_theta(a, cx.row, L.greedy ? nan : L.theta_k, L.greedy ? nan : L.theta_p);
  }
}

__device__ __forceinline__ int pow2_ceil(int n) {
  int p = 2;
  while (p < n) p <<= 1;
  return p;
}

// ---- leader list toolkit.  The list holds sort keys (~key << 32 | id), where
// key is an order-preserving key (of l, or of x for x-lists).  Selections are
// histogram narrowings over the list with native u32 shared atomics; only the
// handful of top-n entries is ever sorted.
__device__ __forceinline__ uint32_t entry_key(uint64_t e) { return ~static_cast<uint32_t>(e >> 32); }
__device__ __forceinline__ int32_t entry_id(uint64_t e) { return static_cast<int32_t>(e & 0xFFFFFFFFu); }

// x of a raw-list entry (or of an x-list entry).
__device__ __forceinline__ float entry_x(uint64_t e, bool x_keys, float T) {
  const float v = key_value(entry_key(e));
  return x_keys ? v : scale_x(v, T);
}

// Key range [lo, hi] of the entries (all of them).
__device__ void list_key_range(const Ctx& cx, int count, uint32_t& lo, uint32_t& hi) {
  uint32_t mn = 0xFFFFFFFFu, mx = 0;
  for (int j = threadIdx.x; j < count; j += kThreads) {
    const uint32_t k = entry_key(cx.list[j]);
    mn = min(mn, k);
    mx = max(mx, k);
  }
  mn = warp_reduce(mn, [](uint32_t a, uint32_t b) { return a < b ? a : b; });
  mx = warp_reduce(mx, [](uint32_t a, uint32_t b) { return a > b ? a : b; });
  SharedHeader* H = cx.H;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  __syncthreads();
  if (lane == 0) {
    H->red_u[warp * 2] = mn;
    H->red_u[warp * 2 + 1] = mx;
  }
  __syncthreads();
  lo = 0xFFFFFFFFu;
  hi = 0;
  for (int i = 0; i < kWarps; ++i) {
    lo = min(lo, H->red_u[i * 2]);
    hi = max(hi, H->red_u[i * 2 + 1]);
  }
  __syncthreads();
}

// The r-th largest key among the list entries (1 <= r <= count), by 256-bin
// rank narrowing on the key.  With a limit on the narrowing rounds, the lower
// end of the key range still holding the r-th key (a key <= the r-th).
__device__ uint32_t list_rank_key(const Ctx& cx, int count, uint32_t r, int max_rounds = 64) {
  uint32_t lo, hi;
  list_key_range(cx, count, lo, hi);
  uint32_t* cnt = reinterpret_cast<uint32_t*>(cx.scratch);
  SharedHeader* H = cx.H;
  for (int round = 0; lo != hi && round < max_rounds; ++round) {
    const uint32_t width = hi - lo;
    const int bits = 32 - __clz(width);
    const int shift = bits > 8 ? bits - 8 : 0;
    for (int i = threadIdx.x; i < kSubBins; i += kThreads) cnt[i] = 0;
    __syncthreads();
    for (int j = threadIdx.x; j < count; j += kThreads) {
      const uint32_t k = entry_key(cx.list[j]);
      if (k >= lo && k <= hi) atomicAdd(&cnt[(hi - k) >> shift], 1u);
    }
    __syncthreads();
    const uint32_t c = cnt[threadIdx.x];
    uint32_t tot;
    const uint32_t incl = block_scan_u(c, &tot, H);
    if (threadIdx.x == 0) H->L.found_bin = 0;
    __syncthreads();
    if (c > 0 && incl >= r && incl - c < r) {
      H->L.found_bin = threadIdx.x;
      H->L.found_cum = incl - c;
    }
    __syncthreads();
    const int jb = H->L.found_bin;
    const uint32_t before = H->L.found_cum;
    __syncthreads();
    const uint32_t nhi = hi - (static_cast<uint32_t>(jb) << shift);
    const uint32_t span = (static_cast<uint32_t>(jb + 1) << shift) - 1u;
    lo = (hi - lo) > span ? hi - span : lo;
    hi = nhi;
    r -= before;
  }
  return lo;
}

// Writes the top-n (key desc, id asc) of a raw list that holds the row's top n.
constexpr int kRankAllMax = 64;  // see sort_entries
__device__ void sort_entries(const uint64_t* in, int count, uint64_t* out);

// scratch_free: the caller no longer needs cx.scratch, so a list of more than
// kRankAllMax entries is sorted there by the bitonic network instead of being
// ranked entry against entry.
__device__ void list_topn(const Ctx& cx, const LeaderState& L, int count, bool scratch_free = false) {
  const SampleArgs& a = *cx.a;
  const int n = a.n_logprobs;
  if (n <= 0) return;
  if (scratch_free && count > kRankAllMax && count <= 2 * kThreads) {
    uint64_t* buf = reinterpret_cast<uint64_t*>(cx.scratch);
    sort_entries(cx.list, count, buf);
    for (int j = threadIdx.x; j < min(n, count); j += kThreads) {
      const uint64_t e = buf[j];
      a.topn_ids[static_cast<size_t>(cx.row) * n + j] = entry_id(e);
      a.topn_logprob[static_cast<size_t>(cx.row) * n + j] = key_value(entry_key(e)) - L.lse;
    }
    __syncthreads();
    return;
  }
  if (count <= 2 * kThreads) {
    // sort keys are distinct: an entry of rank r < n (entries smaller than it) is the (r+1)-th
    const int t = static_cast<int>(threadIdx.x);
    const uint64_t e0 = t < count ? cx.list[t] : ~0ull;
    const uint64_t e1 = t + kThreads < count ? cx.list[t + kThreads] : ~0ull;
    int r0 = 0, r1 = 0;
#pragma unroll 8
    for (int j = 0; j < count; ++j) {
      const uint64_t y = cx.list[j];
      r0 += y < e0 ? 1 : 0;
      r1 += y < e1 ? 1 : 0;
    }
    const size_t o = static_cast<size_t>(cx.row) * n;
    if (t < count && r0 < n) {
      a.topn_ids[o + r0] = entry_id(e0);
      a.topn_logprob[o + r0] = key_value(entry_key(e0)) - L.lse;
    }
    if (t + kThreads < count && r1 < n) {
      a.topn_ids[o + r1] = entry_id(e1);
      a.topn_logprob[o + r1] = key_value(entry_key(e1)) - L.lse;
    }
    __syncthreads();
    return;
  }
  const uint32_t kn = list_rank_key(cx, count, static_cast<uint32_t>(n));
  // gather every entry with key >= the n-th key into a small buffer, sort it
  uint64_t* buf = reinterpret_cast<uint64_t*>(cx.scratch);
  uint32_t* nbuf = &cx.H->list_aux;
  if (threadIdx.x == 0) *nbuf = 0;
  __syncthreads();
  for (int j = threadIdx.x; j < count; j += kThreads) {
    const uint64_t e = cx.list[j];
    if (entry_key(e) >= kn) {
      const uint32_t i = atomicAdd(nbuf, 1u);
      if (i < static_cast<uint32_t>(kListCap)) buf[i] = e;
    }
  }
  __syncthreads();
  const int m = min(static_cast<int>(*nbuf), kListCap);
  const int np2 = pow2_ceil(m);
  for (int j = m + threadIdx.x; j < np2; j += kThreads) buf[j] = ~0ull;
  __syncthreads();
  bitonic_sort(buf, np2);
  for (int j = threadIdx.x; j < n; j += kThreads) {
    const uint64_t e = buf[j];
    a.topn_ids[static_cast<size_t>(cx.row) * n + j] = entry_id(e);
    a.topn_logprob[static_cast<size_t>(cx.row) * n + j] = key_value(entry_key(e)) - L.lse;
  }
  __syncthreads();
}

// The list entry with the largest key (lowest id among equal keys).
__device__ uint64_t list_max_entry(const Ctx& cx, int count) {
  uint64_t best = ~0ull;  // sort keys: smaller = larger key, then lower id
  for (int j = threadIdx.x; j < count; j += kThreads) best = min(best, cx.list[j]);
  best = warp_reduce(best, [](uint64_t a, uint64_t b) { return a < b ? a : b; });
  SharedHeader* H = cx.H;
  __syncthreads();
  if ((threadIdx.x & 31) == 0) reinterpret_cast<uint64_t*>(H->red_d)[threadIdx.x >> 5] = best;
  __syncthreads();
  uint64_t t = ~0ull;
  for (int i = 0; i < kWarps; ++i) t = min(t, reinterpret_cast<uint64_t*>(H->red_d)[i]);
  __syncthreads();
  return t;
}

// Exact top-p cut over the list's survivors (x >= theta_s, x finite; x-key in
// [lo, hi]), given the exact mass strictly above the list (`above`) and the
// total Z: the smallest x value whose mass of strictly larger values is
// < top_p * Z.  256-bin narrowing on x-keys with fixed-point masses.
__device__ float list_mass_cut(const Ctx& cx, LeaderState& L, int count, bool x_keys, float theta_s, Fx4 above,
                               const Fx4& Z) {
  const MassBins b = mass_bins(cx.scratch);
  const double m = static_cast<double>(L.m);
  const double pz = static_cast<double>(L.top_p) * fx_to_double(Z);
  // x-key range of the survivors
  uint32_t mn = 0xFFFFFFFFu, mx = 0;
  for (int j = threadIdx.x; j < count; j += kThreads) {
    const float x = entry_x(cx.list[j], x_keys, L.T);
    if (x >= theta_s && x > -INFINITY) {
      const uint32_t k = fkey(x);
      mn = min(mn, k);
      mx = max(mx, k);
    }
  }
  mn = warp_reduce(mn, [](uint32_t a, uint32_t c) { return a < c ? a : c; });
  mx = warp_reduce(mx, [](uint32_t a, uint32_t c) { return a > c ? a : c; });
  SharedHeader* H = cx.H;
  __syncthreads();
  if ((threadIdx.x & 31) == 0) {
    H->red_u[(threadIdx.x >> 5) * 2] = mn;
    H->red_u[(threadIdx.x >> 5) * 2 + 1] = mx;
  }
  __syncthreads();
  uint32_t lo = 0xFFFFFFFFu, hi = 0;
  for (int i = 0; i < kWarps; ++i) {
    lo = min(lo, H->red_u[i * 2]);
    hi = max(hi, H->red_u[i * 2 + 1]);
  }
  __syncthreads();
  if (lo > hi) return key_value(0xFFFFFFFFu);  // no survivor (cannot happen: the max survives)
  while (lo != hi) {
    const uint32_t width = hi - lo;
    const int bits = 32 - __clz(width);
    const int shift = bits > 8 ? bits - 8 : 0;
    clear_mass_bins(b);
    for (int j = threadIdx.x; j < count; j += kThreads) {
      const float x = entry_x(cx.list[j], x_keys, L.T);
      const uint32_t k = fkey(x);
      if (x >= theta_s && x > -INFINITY && k >= lo && k <= hi)
        add_mass(b, (hi - k) >> shift, exp_neg64(static_cast<double>(x) - m, H->exp_tab));
    }
    __syncthreads();
    const int j = threadIdx.x;
    Fx4 own = fx_zero();
#pragma unroll
    for (int k = 0; k < 4; ++k) own.v[k] = b.limb[k * kSubBins + j];
    const uint32_t c = b.cnt[j];
    Fx4 incl = own;
    block_scan_fx(incl, H);
    const Fx4 before = fx_add(above, fx_sub(incl, own));
    const bool cand = c > 0 && fx_to_double(before) < pz;
    const int jb = max(block_max_i(cand ? j : -1, H), 0);
    if (j == jb) H->L.found_above = before;
    __syncthreads();
    above = H->L.found_above;
    __syncthreads();
    const uint32_t nhi = hi - (static_cast<uint32_t>(jb) << shift);
    const uint32_t span = (static_cast<uint32_t>(jb + 1) << shift) - 1u;
    lo = (hi - lo) > span ? hi - span : lo;
    hi = nhi;
  }
  return key_value(lo);
}

// Exact fixed-point total mass of the raw list's survivors (x >= theta_s).
__device__ Fx4 list_mass_total(const Ctx& cx, const LeaderState& L, int count, float theta_s) {
  Fx4 t = fx_zero();
  const double m = static_cast<double>(L.m);
  for (int j = threadIdx.x; j < count; j += kThreads) {
    const float x = entry_x(cx.list[j], false, L.T);
    if (x >= theta_s && x > -INFINITY) t = fx_add(t, fx_of(exp_neg64(static_cast<double>(x) - m, cx.H->exp_tab)));
  }
  Fx4 incl = t;
  block_scan_fx(incl, cx.H);  // the last thread holds the total
  SharedHeader* H = cx.H;
  if (threadIdx.x == kThreads - 1) H->L.found_above = incl;
  __syncthreads();
  const Fx4 z = H->L.found_above;
  __syncthreads();
  return z;
}

// Best draw candidate (float64 score, id, raw l or 0 for x-lists) over list
// entries with x >= theta (x finite); every thread gets the result.
__device__ void list_best(const Ctx& cx, const LeaderState& L, int count, bool x_keys, float theta, double& sd,
                          int32_t& id, float& l) {
  if (threadIdx.x == 0) cx.H->gbound = kKeyNegInf;
  __syncthreads();
  Best b;
  b.init(&cx.H->gbound);
  const uint32_t k0 = static_cast<uint32_t>(cx.a->seed), k1 = static_cast<uint32_t>(cx.a->seed >> 32);
  for (int j = threadIdx.x; j < count; j += kThreads) {
    const uint64_t e = cx.list[j];
    const float x = entry_x(e, x_keys, L.T);
    if (!(x >= theta && x > -INFINITY)) continue;
    const int32_t id = entry_id(e);
    const uint4 w = philox4x32_10(make_uint4(static_cast<uint32_t>(id) >> 2, cx.pos, cx.req, 0u), k0, k1);
    b.offer(x, x_keys ? 0.0f : key_value(entry_key(e)), word_of(w, id & 3), id);
  }
  sd = b.valid ? b.exact() : -INFINITY;
  id = b.valid ? b.id : 0x7FFFFFFF;
  l = b.valid ? b.l : 0.0f;
  block_best(sd, id, l, cx.H);
}

// The draw over list entries with x >= theta (x finite), into L.token.
__device__ void list_gumbel(const Ctx& cx, LeaderState& L, int count, bool x_keys, float theta) {
  double sd;
  int32_t id;
  float l;
  list_best(cx, L, count, x_keys, theta, sd, id, l);
  if (threadIdx.x == 0) {
    const bool ok = id >= 0 && id < cx.a->V;
    L.token = ok ? id : -1;
    L.token_l = ok ? l : __int_as_float(0x7FC00000);
  }
  __syncthreads();
}

// Sorts `count` distinct sort keys (~key << 32 | id) ascending from `in` into
// `out` (count <= kListCap; `out` distinct from `in`).  Up to 2 * kThreads
// entries every thread ranks its entries against all of them in one pass of
// broadcast reads and stores each at its rank; a longer list is copied and
// sorted by the bitonic network.
// Lists of at most kRankAllMax entries are sorted by ranking every entry
// against all (one pass, broadcast reads); longer ones by the bitonic network
// (register steps, warp shuffles, shared memory only for the largest strides):
// at 240 entries the ranking took ~9k cycles, the network far fewer barriers'
// worth.  The output buffer holds up to the next power of two of count.
__device__ void sort_entries(const uint64_t* in, int count, uint64_t* out) {
  if (count <= kRankAllMax) {
    const int t = static_cast<int>(threadIdx.x);
    const uint64_t e0 = t < count ? in[t] : ~0ull;
    const uint64_t e1 = t + kThreads < count ? in[t + kThreads] : ~0ull;
    int r0 = 0, r1 = 0;
#pragma unroll 8
    for (int j = 0; j < count; ++j) {
      const uint64_t y = in[j];
      r0 += y < e0 ? 1 : 0;
      r1 += y < e1 ? 1 : 0;
    }
    if (t < count) out[r0] = e0;
    if (t + kThreads < count) out[r1] = e1;
    __syncthreads();
    return;
  }
  const int np2 = pow2_ceil(count);
  for (int j = threadIdx.x; j < np2; j += kThreads) out[j] = j < count ? in[j] : ~0ull;
  __syncthreads();
  bitonic_sort(out, np2);
}

// Resolves a list row from its list sorted by (raw key desc, id asc) in `buf`
// (every top-n entry and every top-k survivor present): the top-n is the
// prefix; greedy takes the first entry; a sampling row keeps x >= theta_k (a
// prefix: x = fl(l / T) is monotone in l), cuts top-p on float64 masses summed
// in that order, and draws over the kept prefix.  Fills L.token / L.token_l.
__device__ void list_resolve_sorted(const Ctx& cx, LeaderState& L, const uint64_t* buf, int count, bool sample) {
  const SampleArgs& a = *cx.a;
  SharedHeader* H = cx.H;
  const int n = a.n_logprobs;
  for (int j = threadIdx.x; j < n; j += kThreads) {
    const uint64_t e = buf[min(j, count - 1)];
    a.topn_ids[static_cast<size_t>(cx.row) * n + j] = entry_id(e);
    a.topn_logprob[static_cast<size_t>(cx.row) * n + j] = key_value(entry_key(e)) - L.lse;
  }
  if (!sample) {
    if (threadIdx.x == 0) {
      L.token = entry_id(buf[0]);
      L.token_l = key_value(entry_key(buf[0]));
    }
    __syncthreads();
    return;
  }
  const float T = L.T;
  const float theta_k = L.r_k > 0 ? scale_x(key_value(entry_key(buf[min(L.r_k, count) - 1])), T) : -INFINITY;
  // survivors: the prefix of entries with x >= theta_k (and x finite)
  int s_own = 0;
  for (int j = threadIdx.x; j < count; j += kThreads) {
    const float x = scale_x(key_value(entry_key(buf[j])), T);
    if (x >= theta_k && x > -INFINITY) s_own = max(s_own, j + 1);
  }
  const int s = block_max_i(s_own, H);
  float theta = theta_k;
  if (L.top_p < 1.0f && s > 0) {
    const double m = static_cast<double>(scale_x(key_value(entry_key(buf[0])), T));
    const int cs = (s + kThreads - 1) / kThreads;
    const int i0 = min(static_cast<int>(threadIdx.x) * cs, s), i1 = min(i0 + cs, s);
    double sum = 0.0;
    for (int i = i0; i < i1; ++i)
      sum += exp_neg64(static_cast<double>(scale_x(key_value(entry_key(buf[i])), T)) - m, H->exp_tab);
    double Z;
    const double incl = block_scan_d(sum, &Z, H);
    const double pz = static_cast<double>(L.top_p) * Z;
    double run = incl - sum;  // mass of the entries before i0
    int cand = -1;
    float prev = i0 > 0 ? scale_x(key_value(entry_key(buf[i0 - 1])), T) : INFINITY;
    for (int i = i0; i < i1; ++i) {
      const float x = scale_x(key_value(entry_key(buf[i])), T);
      if (x != prev && run < pz) cand = i;  // first of its x value, mass of larger x below top_p * Z
      run += exp_neg64(static_cast<double>(x) - m, H->exp_tab);
      prev = x;
    }
    const int cut = block_max_i(cand, H);
    if (cut >= 0) {
      const float theta_p = scale_x(key_value(entry_key(buf[cut])), T);
      theta = fmaxf(theta, theta_p);
      if (threadIdx.x == 0) L.theta_p = theta_p;
    }
  }
  if (threadIdx.x == 0) L.theta_k = theta_k;
  // the draw over the kept prefix
  Ctx sub = cx;
  sub.list = const_cast<uint64_t*>(buf);
  list_gumbel(sub, L, s, false, theta);
}

// Sorts the leader's list into the scratch area and resolves the row (list tails).
__device__ void list_resolve(const Ctx& cx, LeaderState& L, int count, bool sample) {
  uint64_t* buf = reinterpret_cast<uint64_t*>(cx.scratch);
  sort_entries(cx.list, count, buf);
  list_resolve_sorted(cx, L, buf, count, sample);
}

__device__ Plan narrow_plan(LeaderState& L, uint32_t op) {
  Plan p{};
  p.op = op;
  p.lo = L.nlo;
  p.hi = L.nhi;
  const uint32_t width = L.nhi - L.nlo;
  const int bits = width == 0 ? 0 : 32 - __clz(width);
  p.shift = bits > 8 ? bits - 8 : 0;
  p.theta = L.theta_k;
  p.m = L.m;
  p.part_is_x = L.part_is_x;
  __syncthreads();
  if (threadIdx.x == 0) L.nshift = p.shift;
  __syncthreads();
  return p;
}

// Narrows [nlo, nhi] to its sub-bin j (bins of 2^nshift keys from the top).
__device__ __forceinline__ void narrow_range(LeaderState& L, int j) {
  const uint32_t hi = L.nhi - (static_cast<uint32_t>(j) << L.nshift);
  const uint32_t span = (static_cast<uint32_t>(j + 1) << L.nshift) - 1u;
  const uint32_t lo = (L.nhi - L.nlo) > span ? L.nhi - span : L.nlo;
  L.nlo = lo;
  L.nhi = hi;
}

// MASS plan: survivors x >= theta_k; bins span [x_low, m], x_low the smallest
// survivor x (at most 96 below m).
__device__ __forceinline__ Plan mass_plan(float m, float theta_k, uint32_t kminf, float T) {
  Plan p{};
  p.op = OP_MASS;
  p.theta = theta_k;
  p.m = m;
  const float x_low = fmaxf(theta_k, scale_x(key_value(kminf), T));
  float width = fminf(__fsub_rn(m, x_low), 96.0f);
  if (!(width > 0.0f)) width = 1.0f;
  p.step = width / static_cast<float>(kMassBins);
  return p;
}

// Survivors known (theta_k): masses for top-p, or the draw directly.
__device__ Plan plan_after_theta_k(const Ctx& cx, LeaderState& L) {
  Plan p{};
  __syncthreads();
  if (L.top_p < 1.0f) {
    p = mass_plan(L.m, L.theta_k, L.kminf, L.T);
    if (threadIdx.x == 0) {
      L.phase = PH_AFTER_MASS;
      L.part_is_x = 1;
    }
  } else {
    p.op = OP_GUMBEL;
    p.theta = L.theta_k;
    p.part_is_x = L.part_is_x;
    p.last = 1;
    if (threadIdx.x == 0) L.phase = PH_AFTER_GUMBEL;
  }
  __syncthreads();
  return p;
}

// After the top-n is known (listed or extracted): the sampling part of a streamed row.
__device__ Plan plan_stream_sampling(const Ctx& cx, LeaderState& L) {
  __syncthreads();
  if (L.r_k == 0) {
    if (threadIdx.x == 0) L.theta_k = -INFINITY;
    return plan_after_theta_k(cx, L);
  }
  if (threadIdx.x == 0) L.phase = PH_TOPK_NARROW;
  return narrow_plan(L, OP_NARROW_COUNT);
}

__device__ Plan gumbel_plan(LeaderState& L) {
  __syncthreads();  // theta_p was just written by thread 0
  Plan p{};
  p.op = OP_GUMBEL;
  p.theta = fmaxf(L.theta_k, L.theta_p);
  p.part_is_x = 1;
  p.last = 1;
  __syncthreads();
  if (threadIdx.x == 0) L.phase = PH_AFTER_GUMBEL;
  __syncthreads();
  return p;
}

// The top-p cut lies in the x-key range [nlo, nhi] (found_cnt survivors, exact
// mass L.cum above it): one x value decides it, a range that fits the list is
// resolved on the leader, a larger one is narrowed further.
__device__ Plan plan_cut_range(LeaderState& L, SharedHeader* H) {
  if (L.nlo == L.nhi) {
    // one x value: every survivor holding it has the same mass above (< pZ)
    if (threadIdx.x == 0) L.theta_p = key_value(L.nlo);
    return gumbel_plan(L);
  }
  if (L.found_cnt <= static_cast<uint32_t>(kListCap)) {
    Plan p{};
    p.op = OP_COLLECT_X;
    p.lo = L.nlo;
    p.hi = L.nhi;
    p.theta = L.theta_k;
    p.part_is_x = 1;
    p.last = 1;
    __syncthreads();
    if (threadIdx.x == 0) {
      L.phase = PH_AFTER_COLLECT_X;
      H->list_count = 0;
    }
    return p;
  }
  return narrow_plan(L, OP_NARROW_MASS);
}

// Resolves theta_p from the x-key list of every survivor in the cut range,
// with the exact mass above the range (L.cum) and the total (L.z).
__device__ void list_cut(const Ctx& cx, LeaderState& L, int count) {
  const float theta_p = list_mass_cut(cx, L, count, true, -INFINITY, L.cum, L.z);
  if (threadIdx.x == 0) L.theta_p = theta_p;
  __syncthreads();
}

// Mass bounds of fine bin j from its count n and offset sum qsum: with g(tau)
// = exp(-tau w), w = 1 / inv_w, and every tau of the bin in [ta, tb], the
// bin's mass lies between n g(mean tau) (Jensen: g is convex) and the chord of
// g over [ta, tb] at the mean (above g on the interval).  The mean of t is
// j - 0.5 + qsum / (n kXQuant) within 2^-12 (float32 here: its error is far
// below that slack), tau within a factor 1 +- 2^-22 of t.  The last bin, open
// above, is bounded by [0, n g(ta)].  ga = g(ta), gb = g(tb) are passed in.
__device__ __forceinline__ void bin_bounds(int j, uint32_t n, uint32_t qsum, double w, double ga, double gb,
                                           const double* tab, double& lo, double& hi) {
  lo = hi = 0.0;
  if (n == 0) return;
  constexpr double eps = 0x1p-22;
  if (j == kXBins - 1) {
    hi = n * ga;
    return;
  }
  const double ta = fmax(0.0, (j - 0.5) * (1.0 - eps));
  const double tb = (j + 0.5) * (1.0 + eps);
  const float mo = __fdiv_rn(static_cast<float>(qsum), static_cast<float>(n) * kXQuant);
  const double mt_hi = fmin(tb, (j - 0.5 + fmin(1.0, static_cast<double>(mo) + 0x1p-12)) * (1.0 + eps));
  const double mt_lo = fmax(ta, (j - 0.5 + fmax(0.0, static_cast<double>(mo) - 0x1p-12)) * (1.0 - eps));
  lo = n * exp_neg64(-mt_hi * w, tab);
  hi = n * (ga + (gb - ga) * ((mt_lo - ta) / (tb - ta)));
}

// Window of the top-p cut from the fine bins (cluster totals in the list area:
// counts, then offset sums).  With P_lo(j), P_hi(j) bounds of the mass above
// bin j and Z_lo, Z_hi of the total, a non-empty bin is kept for certain when
// P_hi(j + 1) < top_p Z_lo and dropped for certain when P_lo(j) >= top_p Z_hi
// (each side with a relative slack of 1e-11 for float64 rounding); the window
// is the non-empty bins between.  A window that fits the list is resolved by
// EXACT, a larger one by the fixed-point mass bins.
__device__ Plan window_plan(const Ctx& cx, LeaderState& L) {
  constexpr int per = kXBins / kThreads;
  SharedHeader* H = cx.H;
  // this thread's bins [j0, j0 + per) lie in one CTA's slice: read the totals there
  const uint32_t owner = (static_cast<uint32_t>(threadIdx.x) * per) / (kXBins / cx.C);
  const uint32_t* cnt = cluster_ptr(reinterpret_cast<const uint32_t*>(cx.scratch), owner);
  const uint32_t* qs = cnt + kXBins;
  const float inv_w = xbin_scale(L.m, scale_x(key_value(L.kminf), L.T));
  const double w = 1.0 / static_cast<double>(inv_w);
  const int j0 = static_cast<int>(threadIdx.x) * per;
  uint32_t c[per];
  double blo[per], bhi[per];
  double slo = 0.0, shi = 0.0;
  {
    // g at the bin ends: geometric in j (ratios qa, qb), started exactly for this thread's run
    constexpr double eps = 0x1p-22;
    const double wa = (1.0 - eps) * w, wb = (1.0 + eps) * w;
    const double qa = exp_neg64(-wa, H->exp_tab), qb = exp_neg64(-wb, H->exp_tab);
    double ga = exp_neg64(-fmax(0.0, (j0 - 0.5) * (1.0 - eps)) * w, H->exp_tab);
    double gb = exp_neg64(-(j0 + 0.5) * (1.0 + eps) * w, H->exp_tab);
#pragma unroll
    for (int k = 0; k < per; ++k) {
      c[k] = cnt[j0 + k];
      bin_bounds(j0 + k, c[k], qs[j0 + k], w, ga, gb, H->exp_tab, blo[k], bhi[k]);
      slo += blo[k];
      shi += bhi[k];
      ga = j0 + k == 0 ? exp_neg64(-0.5 * wa, H->exp_tab) : ga * qa;
      gb *= qb;
    }
    // the recurrences' rounding (< 1e-15 relative) is covered by the 1e-11 slack below
  }
  double zlo, zhi;
  const double plo0 = block_scan_d(slo, &zlo, H) - slo;
  const double phi0 = block_scan_d(shi, &zhi, H) - shi;
  const double tp = static_cast<double>(L.top_p);
  const double keep_lim = tp * zlo * (1.0 - 1e-11);
  const double drop_lim = tp * zhi * (1.0 + 1e-11);
  int jlo = kXBins, jhi = -1;
  {
    double plo = plo0, phi = phi0;
#pragma unroll
    for (int k = 0; k < per; ++k) {
      const int j = j0 + k;
      const double nphi = phi + bhi[k];
      if (c[k] > 0) {
        if (!(nphi * (1.0 + 1e-11) < keep_lim)) jlo = min(jlo, j);
        if (!(plo * (1.0 - 1e-11) >= drop_lim)) jhi = max(jhi, j);
      }
      plo += blo[k];
      phi = nphi;
    }
  }
  jlo = block_min_i(jlo, H);
  jhi = block_max_i(jhi, H);
  uint32_t in_win = 0;
#pragma unroll
  for (int k = 0; k < per; ++k) in_win += (j0 + k >= jlo && j0 + k <= jhi) ? c[k] : 0u;
  uint32_t total;
  block_scan_u(in_win, &total, H);
  // the window's entries go after the first-pass list, which still holds the top-n
  const uint32_t first = min(H->list_count, static_cast<uint32_t>(kListCap));
  Plan p{};
  if (total <= static_cast<uint32_t>(kListCap) - first) {
    p.op = OP_EXACT;
    p.lo = static_cast<uint32_t>(jlo);
    p.hi = static_cast<uint32_t>(jhi);
    p.m = L.m;
    p.step = inv_w;
    p.theta = -INFINITY;
    p.part_is_x = 1;
    p.last = 1;
    __syncthreads();
    if (threadIdx.x == 0) {
      L.phase = PH_AFTER_EXACT;
      L.topn_count = static_cast<int>(first);
    }
  } else {
    list_topn(cx, L, static_cast<int>(first));  // before the list area is reused
    p = mass_plan(L.m, -INFINITY, L.kminf, L.T);
    p.part_is_x = 1;
    __syncthreads();
    if (threadIdx.x == 0) L.phase = PH_AFTER_MASS;
  }
  __syncthreads();
  return p;
}

// The top-p window computed by the whole cluster right after XHIST (each CTA
// holds the cluster totals of its slice of the fine bins): every CTA bounds
// its own bins, the slices' mass bounds are exchanged (prefix offsets and Z in
// rank order, the same in every CTA), then each slice's window edges and
// count.  Returns false when the window does not fit the list (the leader
// then plans the fixed-point fallback); else `e` is the EXACT plan.
__device__ bool window_distributed(const Ctx& cx, const Plan& px, Plan& e) {
  SharedHeader* H = cx.H;
  const uint32_t* cnt = reinterpret_cast<const uint32_t*>(cx.scratch);
  const uint32_t* qs = cnt + kXBins;
  const int S = kXBins / static_cast<int>(cx.C);
  const int q = max(1, S / kThreads);
  const int t = static_cast<int>(threadIdx.x);
  const bool act = t * q < S;
  const int b0 = static_cast<int>(cx.rank) * S + t * q;
  const double w = 1.0 / static_cast<double>(px.step);
  constexpr double eps = 0x1p-22;
  constexpr int kMaxQ = kXBins / kThreads;
  uint32_t c[kMaxQ];
  double blo[kMaxQ], bhi[kMaxQ];
  double slo = 0.0, shi = 0.0;
#pragma unroll
  for (int k = 0; k < kMaxQ; ++k) {
    c[k] = 0;
    blo[k] = bhi[k] = 0.0;
    if (k < q && act) {
      const int j = b0 + k;
      c[k] = cnt[j];
      const double ga = exp_neg64(-fmax(0.0, (j - 0.5) * (1.0 - eps)) * w, H->exp_tab);
      const double gb = exp_neg64(-(j + 0.5) * (1.0 + eps) * w, H->exp_tab);
      bin_bounds(j, c[k], qs[j], w, ga, gb, H->exp_tab, blo[k], bhi[k]);
      slo += blo[k];
      shi += bhi[k];
    }
  }
  double tlo, thi;
  const double ilo = block_scan_d(slo, &tlo, H) - slo;
  const double ihi = block_scan_d(shi, &thi, H) - shi;
  if (threadIdx.x < cx.C) {
    cluster_ptr(H->win_lo, threadIdx.x)[cx.rank] = tlo;
    cluster_ptr(H->win_hi, threadIdx.x)[cx.rank] = thi;
  }
  __syncthreads();
  cluster_sync();
  double zlo = 0.0, zhi = 0.0, olo = 0.0, ohi = 0.0;
  for (uint32_t r = 0; r < cx.C; ++r) {
    if (r < cx.rank) {
      olo += H->win_lo[r];
      ohi += H->win_hi[r];
    }
    zlo += H->win_lo[r];
    zhi += H->win_hi[r];
  }
  const double tp = static_cast<double>(cx.top_p);
  const double keep_lim = tp * zlo * (1.0 - 1e-11);
  const double drop_lim = tp * zhi * (1.0 + 1e-11);
  int jlo = kXBins, jhi = -1;
  uint32_t nwin = 0;
  double plo = olo + ilo, phi = ohi + ihi;
#pragma unroll
  for (int k = 0; k < kMaxQ; ++k) {
    if (k < q && act && c[k] > 0) {
      const int j = b0 + k;
      const double nphi = phi + bhi[k];
      const bool keep = nphi * (1.0 + 1e-11) < keep_lim;  // kept for certain
      const bool drop = plo * (1.0 - 1e-11) >= drop_lim;  // dropped for certain
      if (!keep) jlo = min(jlo, j);
      if (!drop) jhi = max(jhi, j);
      if (!keep && !drop) nwin += c[k];
    }
    plo += blo[k];
    phi += bhi[k];
  }
  jlo = block_min_i(jlo, H);
  jhi = block_max_i(jhi, H);
  uint32_t nt;
  block_scan_u(nwin, &nt, H);
  if (threadIdx.x < cx.C) {
    cluster_ptr(H->win_jlo, threadIdx.x)[cx.rank] = jlo;
    cluster_ptr(H->win_jhi, threadIdx.x)[cx.rank] = jhi;
    cluster_ptr(H->win_cnt, threadIdx.x)[cx.rank] = nt;
  }
  __syncthreads();
  cluster_sync();
  int glo = kXBins, ghi = -1;
  uint32_t gn = 0;
  for (uint32_t r = 0; r < cx.C; ++r) {
    glo = min(glo, H->win_jlo[r]);
    ghi = max(ghi, H->win_jhi[r]);
    gn += H->win_cnt[r];
  }
  const uint32_t first = min(*cluster_ptr(&H->list_count, 0), static_cast<uint32_t>(kListCap));
  if (gn > static_cast<uint32_t>(kListCap) - first) return false;
  e = Plan{};
  e.op = OP_EXACT;
  e.lo = static_cast<uint32_t>(glo);
  e.hi = static_cast<uint32_t>(ghi);
  e.m = px.m;
  e.step = px.step;
  e.theta = -INFINITY;
  e.part_is_x = 1;
  e.last = 1;
  return true;
}

// The row's token from the leader's best (sd, id) and every CTA's pushed best;
// its raw logit is read back from the slices.
__device__ void finish_draw(const Ctx& cx, LeaderState& L, double sd, int32_t id) {
  const SampleArgs& a = *cx.a;
  if (threadIdx.x == 0) {
    for (uint32_t r = 0; r < cx.C; ++r) {
      const BestSlot& s = cx.H->best[r];
      if (s.sd > sd || (s.sd == sd && s.id < id)) {
        sd = s.sd;
        id = s.id;
      }
    }
    const bool ok = id >= 0 && id < a.V;
    L.token = ok ? id : -1;
    float tl = __int_as_float(0x7FC00000);
    if (ok) {
      const int sl = id / a.V_s, jj = id - sl * a.V_s;
      tl = a.slices[sl][static_cast<size_t>(cx.row) * a.V_s + jj];
    }
    L.token_l = tl;
  }
  __syncthreads();
}

// After EXACT: Z = A + W + B from the pushed sums and the window's exact
// masses; the window sorted by (x desc, id asc) gives the cut as the smallest
// x whose mass of strictly larger values is < top_p Z; the draw adds the
// window's kept entries to the CTAs' bests.
__device__ void exact_tail(const Ctx& cx, LeaderState& L, double z_total = -1.0) {
  SharedHeader* H = cx.H;
  const int first = L.topn_count;  // the first-pass list [0, first), then the window
  const int count = min(static_cast<int>(H->list_count), kListCap) - first;
  Ctx win = cx;
  win.list = cx.list + first;
  double A = 0.0, B = 0.0;
  for (uint32_t r = 0; r < cx.C; ++r) {
    A += H->ex_above[r];
    B += H->ex_below[r];
  }
  float theta_p = INFINITY;  // no window entry is kept unless the cut is found in it
  if (count > 0) {
    uint64_t* buf = reinterpret_cast<uint64_t*>(cx.scratch);  // the window sorted by (x desc, id asc)
    sort_entries(win.list, count, buf);
    const double m = static_cast<double>(L.m);
    const int cs = (count + kThreads - 1) / kThreads;
    const int i0 = min(static_cast<int>(threadIdx.x) * cs, count), i1 = min(i0 + cs, count);
    double sum = 0.0;
    for (int i = i0; i < i1; ++i) sum += exp_neg64(static_cast<double>(key_value(entry_key(buf[i]))) - m, H->exp_tab);
    double W;
    const double incl = block_scan_d(sum, &W, H);
    // Z = A + W + B, or the total mass when the caller summed it over the whole row
    const double pz = static_cast<double>(L.top_p) * (z_total >= 0.0 ? z_total : A + W + B);
    double run = A + (incl - sum);
    int cand = -1;
    for (int i = i0; i < i1; ++i) {
      const uint32_t k = entry_key(buf[i]);
      const bool start = i == 0 || entry_key(buf[i - 1]) != k;
      if (start && run < pz) cand = i;
      run += exp_neg64(static_cast<double>(key_value(k)) - m, H->exp_tab);
    }
    const int best = block_max_i(cand, H);
    if (best >= 0) theta_p = key_value(entry_key(buf[best]));
  }
  if (threadIdx.x == 0) {
    // the kept set's smallest x: the window's cut, else (the window keeps
    // nothing) the smallest x above the window
    float t = theta_p;
    if (!(t < INFINITY))
      for (uint32_t r = 0; r < cx.C; ++r) t = fminf(t, H->ex_xmin[r]);
    L.theta_p = t;
  }
  double sd;
  int32_t id;
  float l;
  list_best(win, L, count, true, theta_p, sd, id, l);
  finish_draw(cx, L, sd, id);
  list_topn(cx, L, first, true);  // the sorted window in the scratch is no longer read
}

// Leader: merges the statistics every CTA pushed, validates data and parameters,
// and fills the row state.  A flagged row gets its outputs here; returns true
// for it.  When the first pass's list is complete (`listed`), the top-n is
// written from it now.
__device__ bool leader_merge(const Ctx& cx, LeaderState& L, bool topn_now = true) {
  const SampleArgs& a = *cx.a;
      if (threadIdx.x == 0) {
        uint32_t kmax = 0, kminf = 0xFFFFFFFFu, bad = 0;
        float M = -INFINITY;
        for (uint32_t r = 0; r < cx.C; ++r) {
          const CtaStats& st = cx.H->all[r];
          bad |= st.bad;
          kmax = max(kmax, st.kmax);
          kminf = min(kminf, st.kminf);
          M = fmaxf(M, st.m);
        }
        float S = 0.0f;
        for (uint32_t r = 0; r < cx.C; ++r) {
          const CtaStats& st = cx.H->all[r];
          if (st.m > -INFINITY) S += st.s * fast_exp2((st.m - M) * 1.4426950408889634f);
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
        L.part_is_x = 0;
        L.token = -1;
        L.cum = fx_zero();
        L.topn_done = 0;
      }
      __syncthreads();
      if (L.flags) {
        if (threadIdx.x == 0) {
          a.token_ids[cx.row] = -1;
          a.token_logprob[cx.row] = __int_as_float(0x7FC00000);
          a.row_flags[cx.row] = L.flags;
          write_kept_theta(a, cx.row, __int_as_float(0x7FC00000), __int_as_float(0x7FC00000));
        }
        for (int j = threadIdx.x; j < a.n_logprobs; j += kThreads) {
          a.topn_ids[static_cast<size_t>(cx.row) * a.n_logprobs + j] = -1;
          a.topn_logprob[static_cast<size_t>(cx.row) * a.n_logprobs + j] = __int_as_float(0x7FC00000);
        }
        return true;
      }
  if (cx.H->listed && topn_now) {
    // the first pass's union of per-CTA candidates holds the exact top-n
    const int count = min(static_cast<int>(cx.H->list_count), kListCap);
    list_topn(cx, L, count);
    const uint64_t top = list_max_entry(cx, count);
    if (threadIdx.x == 0) {
      L.topn_done = 1;
      L.token = entry_id(top);  // the argmax (greedy rows)
      L.token_l = key_value(entry_key(top));
    }
    __syncthreads();
  }
  return false;
}

__device__ Plan leader_step(const Ctx& cx, uint32_t& tail) {
  LeaderState& L = cx.H->L;
  const SampleArgs& a = *cx.a;
  Plan p{};
  p.op = OP_END;
  tail = TAIL_NONE;
  switch (L.phase) {
    case PH_START: {
      if (leader_merge(cx, L)) break;  // flagged row: outputs written
      if (L.topn_done && L.greedy) {
        write_outputs(cx, L);
        break;
      }
      // raw-histogram bins from the max key downward
      const uint32_t* hist = reinterpret_cast<const uint32_t*>(cx.scratch);
      const int top = static_cast<int>(L.kmax >> 20);
      int bn = 0;
      uint32_t need_n = 0;
      if (!L.topn_done) {
        find_rank_bin(cx, hist, top, top + 1, true, static_cast<uint32_t>(L.r_n), L);
        bn = max(L.found_bin, 0);
        need_n = L.found_cum + L.found_cnt;
      }
      int bk = 0;
      uint32_t need_k = 0, cum_k = 0;
      if (L.r_k > 0) {
        find_rank_bin(cx, hist, top, top + 1, true, static_cast<uint32_t>(L.r_k), L);
        bk = max(L.found_bin, 0);
        cum_k = L.found_cum;
        need_k = L.found_cum + L.found_cnt;
      }
      if (threadIdx.x == 0) {
        const uint32_t lo_n = L.topn_done ? 0xFFFFFFFFu : static_cast<uint32_t>(bn) << 20;
        L.topn_listed = L.topn_done || need_n <= static_cast<uint32_t>(kListCap);
        uint32_t lo = lo_n;
        int mode = 0;  // 0 = stream, 1 = list greedy, 2 = list sample
        if (L.greedy) {
          mode = L.topn_listed ? 1 : 0;
        } else if (L.r_k > 0 && L.topn_listed && need_k <= static_cast<uint32_t>(kListCap)) {
          // every survivor is listed when no value below the k-th key's bin can
          // scale to that bin's lowest x: adjacent keys at the boundary stay apart
          const uint32_t lo_k = static_cast<uint32_t>(bk) << 20;
          bool ok = lo_k <= kKeyNegInf + 1;
          if (!ok) ok = scale_x(key_value(lo_k - 1), L.T) < scale_x(key_value(lo_k), L.T);
          if (ok) {
            mode = 2;
            lo = min(lo_n, lo_k);
          }
        }
        // narrowing state for a top-k search outside the list
        L.nlo = static_cast<uint32_t>(bk) << 20;
        L.nhi = L.nlo | 0xFFFFFu;
        L.nrank = static_cast<uint32_t>(L.r_k) - cum_k;
        L.mode = mode;
        L.collect_lo = lo;
        cx.H->list_count = 0;
        if (mode == 0 && !L.topn_done) {
          if (L.topn_listed) {
            L.phase = PH_AFTER_TOPN_COLLECT;
          } else {
            L.topn_count = 0;
            L.prev_key = 0xFFFFFFFFu;
            L.prev_id = -1;
            L.phase = PH_TOPN_NEXT_MAX;
          }
        }
      }
      __syncthreads();
      if (L.mode == 0 && L.topn_done) {
        p = plan_stream_sampling(cx, L);
      } else if (L.mode != 0 || L.topn_listed) {
        p.op = OP_COLLECT_RAW;
        p.lo = L.collect_lo;
        if (L.mode == 1) tail = TAIL_LIST_GREEDY;
        if (L.mode == 2) tail = TAIL_LIST_SAMPLE;
        p.last = L.mode != 0;
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
          const uint32_t k = cx.H->all[r].nm_key;
          const int32_t id = cx.H->all[r].nm_id;
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
      if (L.greedy) {
        write_outputs(cx, L);
        break;
      }
      p = plan_stream_sampling(cx, L);
      break;
    }

    case PH_AFTER_TOPN_COLLECT: {
      // write the top-n now: the list is reused for the top-p cut later
      list_topn(cx, L, min(static_cast<int>(cx.H->list_count), kListCap));
      if (threadIdx.x == 0) L.topn_done = 1;
      p = plan_stream_sampling(cx, L);
      break;
    }

    case PH_TOPK_NARROW: {
      const uint32_t* cnt = reinterpret_cast<const uint32_t*>(cx.scratch);
      const int nb = static_cast<int>(((L.nhi - L.nlo) >> L.nshift) + 1);
      find_rank_bin(cx, cnt, 0, nb, false, L.nrank, L);
      if (threadIdx.x == 0) {
        narrow_range(L, max(L.found_bin, 0));
        L.nrank -= L.found_cum;
      }
      __syncthreads();
      if (L.nlo != L.nhi) {
        p = narrow_plan(L, OP_NARROW_COUNT);
        break;
      }
      if (threadIdx.x == 0) L.theta_k = scale_x(key_value(L.nlo), L.T);
      p = plan_after_theta_k(cx, L);
      break;
    }

    case PH_AFTER_MASS: {
      // exact total mass, then the bin holding the cut
      {
        const MassBins b = mass_bins(cx.scratch);
        const int j = threadIdx.x;
        Fx4 f = j < kMassBins ? bin_mass(cx, b, j) : fx_zero();
        block_scan_fx(f, cx.H);
        if (j == kThreads - 1) L.z = f;
        __syncthreads();
      }
      find_mass_bin(cx, kMassBins, L);
      if (threadIdx.x == 0) {
        const int bin = max(L.found_bin, 0);
        // bin j holds x-keys in (edge[j + 1], edge[j]]; the last bin is open below
        const uint32_t* edge = mass_bins(cx.scratch).edge;
        L.nhi = edge[bin];
        L.nlo = bin == kMassBins - 1 ? 0u : edge[bin + 1] + 1u;
        L.cum = L.found_above;
        L.phase = PH_MASS_NARROW;
      }
      __syncthreads();
      p = plan_cut_range(L, cx.H);
      break;
    }

    case PH_MASS_NARROW: {
      const int nb = static_cast<int>(((L.nhi - L.nlo) >> L.nshift) + 1);
      find_mass_bin(cx, nb, L);
      if (threadIdx.x == 0) {
        narrow_range(L, max(L.found_bin, 0));
        L.cum = L.found_above;
      }
      __syncthreads();
      p = plan_cut_range(L, cx.H);
      break;
    }

    case PH_AFTER_COLLECT_X: {
      // exact cut inside the range, then the draw: the range's kept entries
      // here, every survivor above the range in the CTAs' pushed bests
      const int count = min(static_cast<int>(cx.H->list_count), kListCap);
      list_cut(cx, L, count);
      double sd;
      int32_t id;
      float l;
      list_best(cx, L, count, true, L.theta_p, sd, id, l);
      if (threadIdx.x == 0) {
        for (uint32_t r = 0; r < cx.C; ++r) {
          const BestSlot& s = cx.H->best[r];
          if (s.sd > sd || (s.sd == sd && s.id < id)) {
            sd = s.sd;
            id = s.id;
          }
        }
        const bool ok = id >= 0 && id < a.V;
        L.token = ok ? id : -1;
        float tl = __int_as_float(0x7FC00000);
        if (ok) {
          const int sl = id / a.V_s, jj = id - sl * a.V_s;
          tl = a.slices[sl][static_cast<size_t>(cx.row) * a.V_s + jj];
        }
        L.token_l = tl;
      }
      __syncthreads();
      tail = TAIL_STREAM_DONE;
      break;
    }

    case PH_AFTER_XHIST: {
      p = window_plan(cx, L);
      break;
    }

    case PH_AFTER_EXACT: {
      exact_tail(cx, L);
      tail = TAIL_STREAM_DONE;
      break;
    }

    case PH_AFTER_GUMBEL: {
      if (threadIdx.x == 0) {
        double bsd = -INFINITY;
        int32_t bid = 0x7FFFFFFF;
        float bl = 0.0f;
        for (uint32_t r = 0; r < cx.C; ++r) {
          const BestSlot& s = cx.H->best[r];
          if (s.sd > bsd || (s.sd == bsd && s.id < bid)) {
            bsd = s.sd;
            bid = s.id;
            bl = s.l;
          }
        }
        const bool ok = bid >= 0 && bid < a.V;
        L.token = ok ? bid : -1;
        if (ok && L.part_is_x) {
          const int s = bid / a.V_s, jj = bid - s * a.V_s;
          bl = a.slices[s][static_cast<size_t>(cx.row) * a.V_s + jj];
        }
        L.token_l = ok ? bl : __int_as_float(0x7FC00000);
      }
      __syncthreads();
      tail = TAIL_STREAM_DONE;
      break;
    }
    default:
      break;
  }
  return p;
}

// Leader work after the row's last cluster-wide step (the other CTAs have left).
__device__ void leader_tail(const Ctx& cx, uint32_t tail) {
  LeaderState& L = cx.H->L;
  if (tail == TAIL_NONE) return;
  const int count = min(static_cast<int>(cx.H->list_count), kListCap);
  if (tail == TAIL_STREAM_DONE) {
    write_outputs(cx, L);
    return;
  }
  // the list holds the top-n and every top-k survivor: resolve from it sorted
  list_resolve(cx, L, count, tail == TAIL_LIST_SAMPLE);
  write_outputs(cx, L);
}

// One row on the cluster (every CTA of it calls this with the same row).
// Returns when this CTA's share of the row is done: a non-leader may return
// while the leader still finishes the row from its own shared memory.  The
// load barriers are initialised once per CTA; `parity` is the phase this
// row's loads complete (the CTA's rows so far, mod 2).
__device__ __noinline__ void sample_row(const SampleArgs& a, int row, uint32_t parity) {
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
  cx.row = row;
  cx.g0 = static_cast<long long>(cx.rank) * a.part;
  const long long g1 = min(cx.g0 + a.part, static_cast<long long>(a.V));
  const int n = g1 > cx.g0 ? static_cast<int>(g1 - cx.g0) : 0;
  cx.n4 = n >> 2;
  cx.part4 = reinterpret_cast<float4*>(part);

  // ---- chunked load of this CTA's part (1-D bulk copies), one mbarrier per chunk
  int chunk_q[kLoadChunks + 1];
  for (int c = 0; c <= kLoadChunks; ++c) chunk_q[c] = static_cast<int>((static_cast<long long>(cx.n4) * c) / kLoadChunks);
  // a previous row's writes to the part (x in place) are ordered before the copies overwrite it
  fence_proxy_async_smem();
  __syncthreads();
  if (threadIdx.x == 0) {
    const uint64_t pol = policy_evict_first();
    for (int c = 0; c < kLoadChunks; ++c) {
      const long long e0 = cx.g0 + 4LL * chunk_q[c], e1 = cx.g0 + 4LL * chunk_q[c + 1];
      const uint32_t bar = smem_u32(&H->mbar[c]);
      mbar_arrive_expect_tx(bar, static_cast<uint32_t>((e1 - e0) * 4));
      long long g = e0;
      while (g < e1) {
        const int s = static_cast<int>(g / a.V_s);
        const long long s_end = min(static_cast<long long>(s + 1) * a.V_s, e1);
        const float* src = a.slices[s] + static_cast<size_t>(cx.row) * a.V_s + (g - static_cast<long long>(s) * a.V_s);
        bulk_load(smem_u32(part + (g - cx.g0)), src, static_cast<uint32_t>((s_end - g) * 4), bar, pol);
        g = s_end;
      }
    }
  }
  {
    uint32_t* hist = reinterpret_cast<uint32_t*>(scratch);
    for (int i = threadIdx.x; i < kHistBins; i += kThreads) hist[i] = 0;
    for (int j = threadIdx.x; j < 256; j += kThreads) H->exp_tab[j] = exp2(static_cast<double>(j) / 256.0);
    if (threadIdx.x == 0) {
      H->L.phase = PH_START;
      H->list_count = 0;
    }
    const vsl_row_params prm = a.params[cx.row];
    cx.T = prm.temperature;
    cx.top_k = prm.top_k;
    cx.top_p = prm.top_p;
    cx.req = prm.request_id;
    cx.pos = prm.position;
  }
  __syncthreads();

  cluster_arrive();  // this CTA's shared memory is initialised
  pass_stats(cx, chunk_q, parity);

  // ---- first-pass candidates from this CTA's own threshold, straight into the leader's list
  const bool greedy = cx.T == 0.0f;
  const bool k_on = cx.T > 0.0f && cx.top_k > 0 && cx.top_k < a.V;
  const bool eligible = greedy || (k_on && cx.top_k <= kLocalTopK);
  uint32_t rank = a.n_logprobs > 0 ? static_cast<uint32_t>(a.n_logprobs) : 1u;
  if (eligible && k_on) rank = max(rank, static_cast<uint32_t>(cx.top_k));
  const LocalPick lp = local_pick(cx, rank, eligible && k_on);
  cluster_wait();    // every CTA's shared memory is initialised: remote access is safe
  if (threadIdx.x < cx.C) {
    cluster_ptr(H->need_all, threadIdx.x)[cx.rank] = lp.need;
    cluster_ptr(H->ok_all, threadIdx.x)[cx.rank] = lp.ok;
    *cluster_ptr(&H->all[cx.rank], threadIdx.x) = H->stats;  // every CTA sees every CTA's stats
  }
  __syncthreads();
  cluster_sync();
  uint32_t total = 0, all_ok = 1;
  for (uint32_t r = 0; r < cx.C; ++r) {
    total += H->need_all[r];
    all_ok &= H->ok_all[r];
  }
  const bool listed = total <= static_cast<uint32_t>(kListCap);
  // the merged statistics decide the row's path
  uint32_t kmax = 0, kminf = 0xFFFFFFFFu, bad = 0;
  float M = -INFINITY;
  for (uint32_t r = 0; r < cx.C; ++r) {
    const CtaStats& st = H->all[r];
    bad |= st.bad;
    kmax = max(kmax, st.kmax);
    kminf = min(kminf, st.kminf);
    M = fmaxf(M, st.m);
  }
  const bool valid_row = !bad && kmax != kKeyNegInf && cx.T > 0.0f && cx.T < INFINITY && cx.top_p > 0.0f &&
                         cx.top_k >= 0 && !isinf(scale_x(key_value(kmax), cx.T)) &&
                         !isinf(scale_x(key_value(kminf), cx.T));
  // a top-k-off top-p row lists its first-pass candidates during XHIST, which
  // reads every logit anyway; every other row lists them now
  const bool xhist_direct = valid_row && !k_on && listed && cx.top_p < 1.0f;
  if (!xhist_direct) {
    Plan pc{};
    pc.lo = lp.lo;
    op_collect_raw(cx, pc);
    __syncthreads();
    cluster_sync();  // every CTA's candidates are in the leader's list
  }
  if (eligible && listed && all_ok) {
    // the list holds the top-n and every top-k survivor: the leader finishes alone
    if (cx.rank == 0) {
      if (threadIdx.x == 0) H->listed = 0;
      __syncthreads();
      LeaderState& L = H->L;
      if (!leader_merge(cx, L)) leader_tail(cx, greedy ? TAIL_LIST_GREEDY : TAIL_LIST_SAMPLE);
    }
    return;
  }
  if (threadIdx.x == 0) H->listed = listed ? 1u : 0u;
  __syncthreads();

  uint32_t tail = TAIL_NONE;
  // ---- streamed rows with top-k off and the top-n listed: every CTA derives the
  // same first op from the merged statistics and starts it without a plan round
  {
    if (valid_row && !k_on && listed) {
      const float m = scale_x(M, cx.T);
      Plan p{};
      if (cx.top_p < 1.0f) {
        p.op = OP_XHIST;
        p.m = m;
        p.step = xbin_scale(m, scale_x(key_value(kminf), cx.T));
      } else {
        p.op = OP_GUMBEL;
        p.theta = -INFINITY;
      }
      if (cx.rank == 0) {
        LeaderState& L = H->L;
        // the top-n from the first-pass list: now, or (XHIST path) at the end, off the critical path
        leader_merge(cx, L, p.op != OP_XHIST);
        if (threadIdx.x == 0) {
          L.phase = p.op == OP_XHIST ? PH_AFTER_XHIST : PH_AFTER_GUMBEL;
          L.part_is_x = p.op == OP_XHIST ? 1 : 0;
        }
        __syncthreads();
      }
      if (p.op == OP_XHIST) op_xhist(cx, p, lp.lo);
      else op_gumbel(cx, p);
      __syncthreads();
      cluster_sync();
      Plan ex;
      if (p.op == OP_XHIST && window_distributed(cx, p, ex)) {
        // every CTA knows the window: EXACT without a plan round
        if (cx.rank == 0 && threadIdx.x == 0) {
          H->L.phase = PH_AFTER_EXACT;
          H->L.topn_count = static_cast<int>(min(H->list_count, static_cast<uint32_t>(kListCap)));
        }
        op_exact(cx, ex);
        __syncthreads();
        cluster_sync();
        if (cx.rank == 0) {
          leader_step(cx, tail);
          leader_tail(cx, tail);
        }
        return;
      }
      if (p.op == OP_GUMBEL) {
        // what remains is the leader's alone: the CTAs' bests are in its slots
        if (cx.rank == 0) {
          leader_step(cx, tail);
          leader_tail(cx, tail);
        }
        return;
      }
    }
  }
  for (int iter = 0; iter < 64; ++iter) {
    if (cx.rank == 0) {
      const Plan next = leader_step(cx, tail);
      __syncthreads();
      write_plan_all(cx, next);
    }
    cluster_sync();
    const Plan p = H->plan;
    if (p.op == OP_END) break;
    switch (p.op) {
      case OP_COLLECT_RAW: op_collect_raw(cx, p); break;
      case OP_NEXT_MAX: op_next_max(cx, p); break;
      case OP_NARROW_COUNT: op_narrow_count(cx, p); break;
      case OP_MASS: op_mass(cx, p); break;
      case OP_NARROW_MASS: op_narrow_mass(cx, p); break;
      case OP_COLLECT_X: op_collect_x(cx, p); break;
      case OP_GUMBEL: op_gumbel(cx, p); break;
      case OP_EXACT: op_exact(cx, p); break;
      default: break;
    }
    __syncthreads();
    cluster_sync();
    if (p.last) break;  // what remains of the row is the leader's alone
  }
  if (cx.rank == 0) {
    // a last op after which only the leader's own memory is read: its step runs here
    const uint32_t ph = H->L.phase;
    if (tail == TAIL_NONE && (ph == PH_AFTER_EXACT || ph == PH_AFTER_GUMBEL || ph == PH_AFTER_COLLECT_X))
      leader_step(cx, tail);
    leader_tail(cx, tail);
  }
}

// Alongside the streaming kernel (kSelectOthers): cluster g samples row g
// unless the streaming kernel takes it; grid R * C.  After it
// (kSelectDeferred): G clusters, cluster g samples the rows g, g + G, ...
// that the streaming kernel marked kDeferred, one after another (the cluster
// meets at the end of each row), so a launch costs G clusters whatever R is.
// Only cluster g reads or writes the marks of its rows, and every CTA of it
// reads a block of marks before the first cluster barrier of the block's
// first row, ahead of the leader's writes.
__global__ void __launch_bounds__(kThreads, 2) sample_kernel(const __grid_constant__ SampleArgs a) {
  extern __shared__ __align__(128) uint8_t smem_raw[];
  SharedHeader* H = reinterpret_cast<SharedHeader*>(smem_raw);
  const int g = static_cast<int>(blockIdx.x / a.C);
  const bool others = a.select == kSelectOthers;
  if (threadIdx.x == 0) {
    for (int c = 0; c < kLoadChunks; ++c) mbar_init(smem_u32(&H->mbar[c]), 1);
    fence_mbar_init();
  }
  __syncthreads();
  uint32_t rows_done = 0;
  const long long G = others ? 1 : gridDim.x / a.C;
  const long long end = others ? g + 1 : a.R;
  for (long long base = g; base < end; base += G * kThreads) {
    uint32_t total = 0;
    if (others) {
      total = stream_row(a.params[g], a.V) ? 0u : 1u;
      if (threadIdx.x == 0) H->drows[0] = g;
    } else {
      const long long r = base + G * threadIdx.x;
      const uint32_t d = (r < a.R && a.token_ids[r] == kDeferred) ? 1u : 0u;
      const uint32_t idx = block_scan_u(d, &total, H) - d;
      if (d) H->drows[idx] = static_cast<int32_t>(r);
    }
    __syncthreads();
    for (uint32_t i = 0; i < total; ++i) {
      sample_row(a, H->drows[i], rows_done++ & 1u);
      if (others) return;  // one row: the CTA leaves when its share is done
      __syncthreads();
      cluster_sync();  // the leader has finished the row: the next one may write into its memory
    }
  }
}

}  // namespace vsl

#include "vsl_stream.cuh"

namespace vsl {

// ------------------------------------------------------------------ host side
size_t sample_smem_bytes(int part) {
  return ((sizeof(SharedHeader) + 127) & ~size_t(127)) + kScratchBytes + kListBytes +
         static_cast<size_t>(part) * 4;
}

// Per-device launch state: the kernels' attributes are set, and the largest
// schedulable cluster and the SM count are read, once per device (with that
// device current); the side stream and its two events are created on the
// first side-by-side call on the device.
struct DeviceState {
  std::once_flag once;
  cudaError_t status = cudaSuccess;
  int max_cluster = 8;  // largest cluster size the device schedules for the cluster kernel
  int sms = 0;
  std::mutex mu;        // orders the fork / join event pairs of concurrent calls
  cudaStream_t side = nullptr;
  cudaEvent_t fork = nullptr, join = nullptr;
};
constexpr int kMaxDevices = 64;
static DeviceState g_devices[kMaxDevices];

// The same for a device that schedules clusters of at most maxc CTAs.
bool sample_geometry_for(long long V, int maxc, int* cluster, int* part) {
  if (V <= 0 || V > static_cast<long long>(kMaxCluster) * kMaxPart || maxc < 1) return false;
  int c = 1;
  while (c < kMaxCluster && (V + c - 1) / c > kPreferredPart) c <<= 1;
  while (c > maxc) c >>= 1;
  long long p = (V + c - 1) / c;
  p = (p + 3) / 4 * 4;
  if (p > kMaxPart) return false;
  *cluster = c;
  *part = static_cast<int>(p);
  return true;
}

static cudaError_t prepare_device(DeviceState& d, int dev) {
  cudaError_t e = cudaFuncSetAttribute(sample_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(sample_smem_bytes(kMaxPart)));
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(sample_kernel, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(stream_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(stream_smem_bytes()));
  if (e != cudaSuccess) return e;
  e = cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return e;
  // largest schedulable cluster at the preferred part size
  d.max_cluster = 8;
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
    int nclusters = 0;
    if (cudaOccupancyMaxActiveClusters(&nclusters, sample_kernel, &cfg) == cudaSuccess && nclusters > 0) {
      d.max_cluster = c;
      break;
    }
    cudaGetLastError();
  }
  return cudaSuccess;
}

// The current device's state, prepared on first use.
static cudaError_t current_device_state(DeviceState** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  DeviceState& d = g_devices[dev];
  std::call_once(d.once, [&] { d.status = prepare_device(d, dev); });
  if (d.status != cudaSuccess) return d.status;
  *out = &d;
  return cudaSuccess;
}

long long sample_max_vocab() { return static_cast<long long>(kMaxCluster) * kMaxPart; }

cudaError_t sample_max_cluster(int* maxc) {
  DeviceState* d = nullptr;
  const cudaError_t e = current_device_state(&d);
  if (e == cudaSuccess) *maxc = d->max_cluster;
  return e;
}

// Streaming kernel geometry: the most CTAs per row (at most 8, a portable
// cluster) for which R * C still runs in one wave of two CTAs per SM (a
// second wave would start only once the first has streamed its parts), and
// the part of each (a multiple of 4 floats: every part starts 16-byte aligned).
static void stream_geometry(int R, long long V, int sms, int* cluster, int* part) {
  int c = 1;
  while (c < 8 && static_cast<long long>(R) * c * 2 <= 2LL * sms) c <<= 1;
  long long p = (V + c - 1) / c;
  p = (p + 3) / 4 * 4;
  *cluster = c;
  *part = static_cast<int>(p);
}

// `urgent`: the launch gets the device's greatest scheduling priority, so
// its CTAs are placed before those of a kernel launched beside it.
static cudaError_t launch_with_cluster(const void* fn, const SampleArgs& a, int grid, size_t smem, cudaStream_t stream,
                                       bool urgent = false) {
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(static_cast<unsigned>(grid), 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = static_cast<unsigned>(a.C);
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (urgent) {
    int least = 0, greatest = 0;
    const cudaError_t e = cudaDeviceGetStreamPriorityRange(&least, &greatest);
    if (e != cudaSuccess) return e;
    attr[1].id = cudaLaunchAttributePriority;
    attr[1].val.priority = greatest;
    cfg.numAttrs = 2;
  }
  void* args[] = {const_cast<SampleArgs*>(&a)};
  return cudaLaunchKernelExC(&cfg, fn, args);
}

// Clusters of the deferred-row pass: as many as run at once (two CTAs per
// SM), at most one per row.
static int deferred_clusters(int R, int cluster, int sms) {
  return std::max(1, std::min(R, 2 * sms / cluster));
}

// A batch whose streaming kernel spreads each row over more than one CTA (R
// at most the SM count) is latency bound: the sampler's kernels then run side
// by side (three launches), the cluster kernel taking the top-k-off rows the
// streaming kernel leaves at that geometry.
static bool small_batch(int R, long long V, int sms) {
  int sc = 0, sp = 0;
  stream_geometry(R, V, sms, &sc, &sp);
  return sc > 1;
}

// The launches of one call for R rows of V tokens on a device with `sms` SMs
// that schedules clusters of at most `maxc` CTAs: the choices launch_sample
// makes, as plain data.  Returns false if V cannot be handled.
bool sample_plan(int R, long long V, int sms, int maxc, vsl_sample_plan* out) {
  int c = 0, part = 0;
  if (R <= 0 || sms <= 0 || !sample_geometry_for(V, maxc, &c, &part)) return false;
  int sc = 0, sp = 0;
  stream_geometry(R, V, sms, &sc, &sp);
  const bool side = small_batch(R, V, sms);
  out->launches = side ? 3 : 2;
  out->side_by_side = side ? 1 : 0;
  out->stream_cluster = sc;
  out->stream_part = sp;
  out->stream_grid = R * sc;
  out->cluster = c;
  out->part = part;
  out->others_grid = side ? R * c : 0;
  out->deferred_grid = deferred_clusters(R, c, sms) * c;
  return true;
}

int sample_launches(int R, long long V) {
  DeviceState* d = nullptr;
  if (current_device_state(&d) != cudaSuccess) return -1;
  vsl_sample_plan p{};
  if (!sample_plan(R, V, d->sms, d->max_cluster, &p)) return -1;
  return p.launches;
}

cudaError_t launch_sample(const float* const* logits, int R, int S, int V_s, const vsl_row_params* params,
                          uint64_t seed, int n_logprobs, int32_t* token_ids, float* token_logprob,
                          int32_t* topn_ids, float* topn_logprob, uint32_t* row_flags, float* kept_theta,
                          const float* tile_stats, cudaStream_t stream) {
  DeviceState* d = nullptr;
  cudaError_t e = current_device_state(&d);
  if (e != cudaSuccess) return e;
  SampleArgs a{};
  for (int s = 0; s < S; ++s) a.slices[s] = logits[s];
  a.params = params;
  a.token_ids = token_ids;
  a.token_logprob = token_logprob;
  a.topn_ids = topn_ids;
  a.topn_logprob = topn_logprob;
  a.row_flags = row_flags;
  a.kept_theta = kept_theta;
  a.err = device_error_word();
  if (a.err == nullptr) return cudaErrorUnknown;
  a.seed = seed;
  a.R = R;
  a.S = S;
  a.V_s = V_s;
  a.V = S * V_s;
  a.n_logprobs = n_logprobs;
  int c = 0, part = 0;
  if (!sample_geometry_for(a.V, d->max_cluster, &c, &part)) return cudaErrorInvalidValue;
  const int sms = d->sms;
  SampleArgs sa = a;
  stream_geometry(R, a.V, sms, &sa.C, &sa.part);
  const int tile_blocks = (V_s + 127) / 128;
  if (tile_stats != nullptr && static_cast<long long>(S) * tile_blocks <= kStreamCap) {
    // tile mode: each greedy / top-k row reads its records and a few quarters on one CTA
    sa.tile_stats = tile_stats;
    sa.tile_blocks = tile_blocks;
    sa.C = 1;
    sa.part = a.V;
  }
  a.C = c;
  a.part = part;
  const void* fs = reinterpret_cast<const void*>(stream_kernel);
  const void* fc = reinterpret_cast<const void*>(sample_kernel);
  if (!small_batch(R, a.V, sms)) {
    // a large batch: the streaming kernel first (it marks the rows it leaves),
    // then the cluster kernel on the marked rows
    sa.select = kStreamMarks | (sa.C == 1 ? kStreamKoff : 0);
    a.select = kSelectDeferred;
    if ((e = launch_with_cluster(fs, sa, R * sa.C, stream_smem_bytes(), stream)) != cudaSuccess) return e;
    return launch_with_cluster(fc, a, deferred_clusters(R, c, sms) * c, sample_smem_bytes(part), stream);
  }
  // a small batch is latency-bound: the two kernels take disjoint rows (decided
  // by the parameters alone) and run side by side, the streaming kernel on a
  // side stream forked from and joined back to the caller's; then the cluster
  // kernel samples the rows the streaming kernel could not hold (marked
  // kDeferred).  The cluster kernel's rows take the longest, so it is launched
  // first and with the greatest priority: its CTAs get the SMs first.
  std::lock_guard<std::mutex> lock(d->mu);
  if (d->side == nullptr) {
    if ((e = cudaStreamCreateWithFlags(&d->side, cudaStreamNonBlocking)) != cudaSuccess) return e;
    if ((e = cudaEventCreateWithFlags(&d->fork, cudaEventDisableTiming)) != cudaSuccess) return e;
    if ((e = cudaEventCreateWithFlags(&d->join, cudaEventDisableTiming)) != cudaSuccess) return e;
  }
  sa.select = 0;  // the streaming kernel leaves the other rows untouched
  a.select = kSelectOthers;
  if ((e = cudaEventRecord(d->fork, stream)) != cudaSuccess) return e;
  if ((e = cudaStreamWaitEvent(d->side, d->fork, 0)) != cudaSuccess) return e;
  // once forked, the side stream is always joined back (also when a launch
  // fails), so a capture in progress stays well-formed and reports the error
  e = launch_with_cluster(fc, a, R * c, sample_smem_bytes(part), stream, true);
  if (e == cudaSuccess) e = launch_with_cluster(fs, sa, R * sa.C, stream_smem_bytes(), d->side);
  cudaError_t ej = cudaEventRecord(d->join, d->side);
  if (ej == cudaSuccess) ej = cudaStreamWaitEvent(stream, d->join, 0);
  if (e != cudaSuccess) return e;
  if (ej != cudaSuccess) return ej;
  a.select = kSelectDeferred;
  return launch_with_cluster(fc, a, deferred_clusters(R, c, sms) * c, sample_smem_bytes(part), stream);
}

}  // namespace vsl
