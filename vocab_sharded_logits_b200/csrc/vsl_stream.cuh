// vsl_stream.cuh - streaming sampler for rows resolved from a candidate list
// (greedy rows, sampling rows with 0 < top_k <= kStreamMaxK, and, in a large
// batch with one CTA per row, top-k-off rows), included by vsl_sample.cu
// after the cluster kernel it shares the list toolkit with.
//
// A top-k row needs one pass over its logits: the statistics of the softmax
// (max, sum of exp, NaN / +inf, smallest finite value) and every logit that
// can be among the top max(n, k), ties included.  Its part of the row streams
// from HBM through a ring of shared-memory stages fed by 1-D bulk copies, so
// the row is never held on chip: while a stage is scanned the next ones are
// in flight.  Candidates above a running threshold go to a list; when the
// list fills up it is compacted and the threshold raised.  The cluster's
// leader then resolves the row from the merged list with the same toolkit as
// the cluster kernel.  A top-k-off row streams its row up to twice more (the
// fine bins of x, then the masses, window and draw: stream_koff).  A row this
// kernel does not take (or whose candidates do not fit) gets the token id
// kDeferred, and the cluster kernel's pass over marked rows, launched after
// this kernel on the caller's stream, samples exactly those rows.
#pragma once

#include <type_traits>

namespace vsl {

constexpr int kStreamCap = 4096;      // candidate list capacity while streaming
constexpr int kStreamRound = 4;       // chunks per block barrier once the threshold is set

constexpr size_t kStreamListBytes = static_cast<size_t>(kStreamCap) * 8;
constexpr size_t kStreamRingBytes = static_cast<size_t>(kStreamStages) * kStreamChunk * 4;

// Layout: header | 1 KB of narrowing bins | list | ring.  After the stream the
// ring's first kScratchBytes serve as the leader's scratch (every copy into
// the ring has landed by then).
constexpr size_t kStreamBinsBytes = 1024;
static_assert(kStreamRingBytes >= kScratchBytes, "the ring doubles as the leader's scratch");
static_assert(kDrawQueueBytes <= kListCap * 8, "the third pass's draw queue lives in the list's first half");
__host__ __device__ __forceinline__ size_t stream_smem_bytes() {
  return ((sizeof(SharedHeader) + 127) & ~size_t(127)) + kStreamBinsBytes + kStreamListBytes + kStreamRingBytes;
}

// Lowest raw key a compaction may keep when the rank-`r` value found is `v`:
// for a sampling row every l that can scale to the same x as v (the
// temperature maps up to a few adjacent floats to one x) stays listed.
__device__ __forceinline__ uint32_t stream_floor(uint32_t key, float T) {
  if (!(T > 0.0f) || !key_finite(key)) return key;
  return min(key, raw_prefilter(scale_x(key_value(key), T), T));
}

// Keeps the list entries whose key is >= a new threshold at or below the
// list's r-th largest key (after `rounds` 256-bin narrowings, or exact when
// that leaves less than a chunk of room; lowered by stream_floor), when that
// raises `thr`.  In place: every thread holds its entries in registers before
// any is written back.  Every thread returns the threshold in force and sets
// `left` to the list's count after it (no thread re-reads the shared counter,
// which the next chunk's appends may already be moving).  Called by the whole
// block at a point no thread appends.
__device__ uint32_t stream_compact(const Ctx& cx, uint32_t r, uint32_t thr, int rounds, uint32_t& left) {
  SharedHeader* H = cx.H;
  left = H->list_count;
  const int count = min(static_cast<int>(left), kStreamCap);
  if (count <= static_cast<int>(r)) return thr;
  constexpr int per = kStreamCap / kThreads;
  uint64_t e[per];
#pragma unroll
  for (int i = 0; i < per; ++i) {
    const int idx = static_cast<int>(threadIdx.x) + i * kThreads;
    e[i] = idx < count ? cx.list[idx] : 0ull;
  }
  uint32_t cut;
  if (count <= 2 * kThreads) {
    // a short list: the r-th largest key directly, every entry ranked against all (sort keys are distinct)
    const int t = static_cast<int>(threadIdx.x);
    const uint64_t e0 = t < count ? cx.list[t] : ~0ull, e1 = t + kThreads < count ? cx.list[t + kThreads] : ~0ull;
    int r0 = 0, r1 = 0;
#pragma unroll 8
    for (int j = 0; j < count; ++j) {
      const uint64_t y = cx.list[j];
      r0 += y < e0 ? 1 : 0;
      r1 += y < e1 ? 1 : 0;
    }
    if (t < count && r0 == static_cast<int>(r) - 1) H->L.found_cum = entry_key(e0);
    if (t + kThreads < count && r1 == static_cast<int>(r) - 1) H->L.found_cum = entry_key(e1);
    __syncthreads();
    cut = stream_floor(H->L.found_cum, cx.T);
    rounds = 64;  // exact
  } else {
    cut = stream_floor(list_rank_key(cx, count, r, rounds), cx.T);
  }
  uint32_t kept = 0, total = 0;
  for (int pass = 0; pass < 2; ++pass) {
    kept = 0;
#pragma unroll
    for (int i = 0; i < per; ++i) {
      const int idx = static_cast<int>(threadIdx.x) + i * kThreads;
      kept += (idx < count && entry_key(e[i]) >= cut) ? 1u : 0u;
    }
    block_scan_u(kept, &total, H);
    if (pass == 1 || rounds >= 64 || total <= static_cast<uint32_t>(kStreamCap - kStreamChunk)) break;
    cut = stream_floor(list_rank_key(cx, count, r), cx.T);
  }
  if (cut <= thr) return thr;
  left = total;
  uint32_t off = block_scan_u(kept, &total, H) - kept;
  __syncthreads();
#pragma unroll
  for (int i = 0; i < per; ++i) {
    const int idx = static_cast<int>(threadIdx.x) + i * kThreads;
    if (idx < count && entry_key(e[i]) >= cut) cx.list[off++] = e[i];
  }
  if (threadIdx.x == 0) H->list_count = total;
  __syncthreads();
  return cut;
}

// Issues the bulk copies of chunk `c` of this CTA's part [g0, g0 + n) into
// ring stage c % kStreamStages (thread 0; chunks in increasing order, so the
// slice `s` holding the chunk's start only moves forward).  A chunk may span
// two slices.
__device__ __forceinline__ void stream_issue(const SampleArgs& a, int row, int g0, int n, int c, int& s,
                                             float* ring, unsigned long long* bars, uint64_t pol,
                                             int stage_base = 0) {
  const int stage = (stage_base + c) % kStreamStages;
  const int e0 = g0 + c * kStreamChunk;
  const int e1 = g0 + min((c + 1) * kStreamChunk, n);
  const uint32_t bar = smem_u32(&bars[stage]);
  mbar_arrive_expect_tx(bar, static_cast<uint32_t>(e1 - e0) * 4u);
  float* dst = ring + static_cast<size_t>(stage) * kStreamChunk;
  int g = e0;
  while (g < e1) {
    while (g >= (s + 1) * a.V_s) ++s;
    const int s_end = min((s + 1) * a.V_s, e1);
    const float* src = a.slices[s] + static_cast<size_t>(row) * a.V_s + (g - s * a.V_s);
    bulk_load(smem_u32(dst + (g - e0)), src, static_cast<uint32_t>(s_end - g) * 4u, bar, pol);
    g = s_end;
  }
}

// Statistics a thread keeps over the logits it scans.  The sum of exp runs
// against the thread's largest finite value m (each term exp2((v - m) log2 e),
// so no product overflows whatever the logits' size).  m starts at a finite
// stand-in, so a thread that has seen only -inf adds exp(-inf) = 0; a sum that
// is still 0 has no maximum yet (the stand-in may lie above a row's values):
// it is never rescaled, and the merges ignore its m.  NaN of either sign
// makes the sum NaN; +inf shows in kmax.
struct ScanStats {
  uint32_t kmax;   // largest key
  uint32_t kmf;    // smallest (key - key(-inf) - 1) mod 2^32: the smallest key above key(-inf)
  uint32_t amin;   // (kAmin scans) smallest bit pattern of a nonzero |l|
  float m, s;
};
constexpr float kScanNoMax = -1e30f;

// Scans one ring stage (nq float4 of it) with first id `gid`: statistics and
// candidates (key >= thr) appended to the list (`seen`: this warp's list end).
// A thread takes kPer float4; a warp with any candidate reserves the slots of
// all of them with one atomic.
template <bool kFull, bool kAmin>
__device__ __forceinline__ void stream_scan(const float4* st4, int nq, uint32_t thr, uint32_t gid, ScanStats& st,
                                            uint32_t& seen, uint32_t* counter, uint64_t* list) {
  constexpr float kLog2e = 1.4426950408889634f;
  constexpr int kPer = kStreamChunk / 4 / kThreads;
  const int lane = threadIdx.x & 31;
  uint32_t k[kPer][4];
  bool any = false;
#pragma unroll
  for (int it = 0; it < kPer; ++it) {
    const int q = static_cast<int>(threadIdx.x) + it * kThreads;
    const bool valid = kFull || q < nq;
    const float4 v4 = valid ? st4[q] : make_float4(-INFINITY, -INFINITY, -INFINITY, -INFINITY);
    const float v[4] = {v4.x, v4.y, v4.z, v4.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      // order-preserving key of v + 0 (-0 becomes +0); padding keys are 0 (never listed)
      const uint32_t b = __float_as_uint(__fadd_rn(v[i], 0.0f));
      k[it][i] = valid ? b ^ (static_cast<uint32_t>(static_cast<int32_t>(b) >> 31) | 0x80000000u) : 0u;
      st.kmf = min(st.kmf, valid ? k[it][i] - (kKeyNegInf + 1u) : 0xFFFFFFFFu);
      if (kAmin) {
        const uint32_t ab = __float_as_uint(v[i]) & 0x7FFFFFFFu;
        st.amin = min(st.amin, (valid && ab != 0u) ? ab : 0xFFFFFFFFu);
      }
    }
    const uint32_t kq = max(max(k[it][0], k[it][1]), max(k[it][2], k[it][3]));
    if (kq > st.kmax) {
      st.kmax = kq;
      if (kq > kKeyNegInf) {  // a new largest value: rescale the sum to it
        const float mn = key_value(kq);
        st.s = st.s == 0.0f ? 0.0f : st.s * fast_exp2((st.m - mn) * kLog2e);
        st.m = mn;
      }
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) st.s += fast_exp2((v[i] - st.m) * kLog2e);
    any |= kq >= thr && valid;
  }
  if (!__any_sync(0xFFFFFFFFu, any)) return;
  uint32_t mask[kPer][4];
  uint32_t total = 0;
#pragma unroll
  for (int it = 0; it < kPer; ++it)
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      mask[it][i] = __ballot_sync(0xFFFFFFFFu, k[it][i] >= thr && k[it][i] != 0u);
      total += __popc(mask[it][i]);
    }
  uint32_t base = 0;
  if (lane == 0) base = atomicAdd(counter, total);
  base = __shfl_sync(0xFFFFFFFFu, base, 0);
  seen = max(seen, base + total);
  const uint32_t below = (1u << lane) - 1u;
#pragma unroll
  for (int it = 0; it < kPer; ++it)
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint32_t idx = base + __popc(mask[it][i] & below);
      if (((mask[it][i] >> lane) & 1u) && idx < static_cast<uint32_t>(kStreamCap)) {
        const int q = static_cast<int>(threadIdx.x) + it * kThreads;
        list[idx] = (static_cast<uint64_t>(~k[it][i]) << 32) | (gid + 4u * static_cast<uint32_t>(q) + i);
      }
      base += __popc(mask[it][i]);
    }
}

// Tile mode (a greedy or top-k row on one CTA, with the tile statistics of its
// logits): the row's statistics come from its records, the cut from the block
// maxima, and only the 32-id quarters whose largest raw value reaches the cut
// are read.  The R-th largest block maximum t0 is at most the row's R-th
// largest logit (R blocks hold a value >= t0), and x = fl(l / T) is
// non-decreasing in l, so every top-R logit and every value that scales to the
// same x as the R-th lies in a quarter whose maximum is >= the cut
// stream_floor(t0).  Lists every logit >= the cut and returns the cut;
// `qkeys` (the idle ring, 4 * S * B keys) holds the quarter maxima.  A list
// that overflows shows in the list count (the row is deferred).
struct TileScan {
  ScanStats st;
  uint32_t cut;
};
__device__ __forceinline__ TileScan stream_tiles(const Ctx& cx, const SampleArgs& a, uint32_t R, uint32_t* qkeys) {
  constexpr float kLog2e = 1.4426950408889634f;
  ScanStats st{0u, 0xFFFFFFFFu, 0xFFFFFFFFu, kScanNoMax, 0.0f};
  SharedHeader* H = cx.H;
  const int B = a.tile_blocks;
  const int SB = a.S * B;
  const float4* rec = reinterpret_cast<const float4*>(a.tile_stats) + static_cast<size_t>(cx.row) * SB * 2;
  // records: statistics, the block maxima as list entries, the quarter maxima
  // (four records per thread loaded before any is used: their latencies overlap)
  constexpr int kRecBatch = 4;
  for (int base = threadIdx.x; base < SB; base += kRecBatch * kThreads) {
    float4 qmb[kRecBatch], smb[kRecBatch];
#pragma unroll
    for (int u = 0; u < kRecBatch; ++u) {
      const int i = base + u * kThreads;
      if (i < SB) {
        qmb[u] = __ldg(rec + 2 * i);
        smb[u] = __ldg(rec + 2 * i + 1);
      }
    }
#pragma unroll
    for (int u = 0; u < kRecBatch; ++u) {
      const int i = base + u * kThreads;
      if (i >= SB) break;
      const float4 qm = qmb[u];
      const float4 sm = smb[u];
      const uint4 k = make_uint4(fkey(qm.x), fkey(qm.y), fkey(qm.z), fkey(qm.w));
      reinterpret_cast<uint4*>(qkeys)[i] = k;
      const uint32_t kb = max(max(k.x, k.y), max(k.z, k.w));
      cx.list[i] = (static_cast<uint64_t>(~kb) << 32) | static_cast<uint32_t>(i);
      const uint32_t kmin = fkey(sm.y);
      st.kmf = min(st.kmf, key_finite(kmin) ? kmin - (kKeyNegInf + 1u) : 0xFFFFFFFFu);
      st.amin = min(st.amin, __float_as_uint(sm.z) & 0x7FFFFFFFu);  // smallest nonzero |l| (+inf: none)
      // the block's sum runs against its maximum c (0 when that is not finite)
      if (kb > st.kmax) {
        st.kmax = kb;
        if (key_finite(kb)) {
          const float mn = key_value(kb);
          st.s = st.s == 0.0f ? 0.0f : st.s * fast_exp2((st.m - mn) * kLog2e);
          st.m = mn;
        }
      }
      if (key_finite(kb)) st.s += sm.x * fast_exp2((key_value(kb) - st.m) * kLog2e);
      else if (sm.x != 0.0f) st.s += sm.x;  // NaN or +inf: the row is flagged
    }
  }
  if (threadIdx.x == 0) H->list_count = static_cast<uint32_t>(SB);
  __syncthreads();
  uint32_t left;
  // two 256-bin narrowings: a cut at most ~2^-14 of the block maxima's key range
  // below t0 is still a valid cut and adds next to no quarter (0: every quarter
  // when SB <= R)
  const uint32_t cut = stream_compact(cx, R, 0u, 2, left);
  __syncthreads();
  if (threadIdx.x == 0) H->list_count = 0;
  __syncthreads();
  // each warp compacts the indices of its quarters that reach the cut in place
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int NQ = 4 * SB;
  const int per = ((NQ + kWarps - 1) / kWarps + 31) & ~31;
  const int q0 = min(warp * per, NQ), q1 = min(q0 + per, NQ);
  uint32_t nsel = 0;
  for (int j = q0; j < q1; j += 32) {
    const bool pick = j + lane < q1 && qkeys[j + lane] >= cut;
    const uint32_t m = __ballot_sync(0xFFFFFFFFu, pick);
    if (pick) qkeys[q0 + nsel + __popc(m & ((1u << lane) - 1u))] = static_cast<uint32_t>(j + lane);
    nsel += __popc(m);
    __syncwarp();
  }
  // gather: 8 lanes per quarter (one float4 each), 4 quarters per load, kGather
  // loads in flight per lane
  constexpr int kGather = 8;
  const uint32_t below = (1u << lane) - 1u;
  for (uint32_t u = 0; u < nsel; u += 4u * kGather) {
    float4 v[kGather];
    uint32_t gid[kGather];
#pragma unroll
    for (int w = 0; w < kGather; ++w) {
      const uint32_t qi = u + 4u * w + (lane >> 3);
      gid[w] = 0xFFFFFFFFu;
      v[w] = make_float4(0.f, 0.f, 0.f, 0.f);
      if (qi < nsel) {
        const uint32_t j = qkeys[q0 + qi];
        const int blk = static_cast<int>(j >> 2);
        const int sl = blk / B;
        const int col = (blk - sl * B) * 128 + static_cast<int>(j & 3u) * 32 + 4 * (lane & 7);
        if (col < a.V_s) {
          gid[w] = static_cast<uint32_t>(sl * a.V_s + col);
          v[w] = ldg_stream4(a.slices[sl] + static_cast<size_t>(cx.row) * a.V_s + col);
        }
      }
    }
#pragma unroll
    for (int w = 0; w < kGather; ++w) {
      const float e[4] = {v[w].x, v[w].y, v[w].z, v[w].w};
      uint32_t mask[4], total = 0;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        mask[i] = __ballot_sync(0xFFFFFFFFu, gid[w] != 0xFFFFFFFFu && fkey(e[i]) >= cut);
        total += __popc(mask[i]);
      }
      if (total == 0) continue;
      uint32_t base = 0;
      if (lane == 0) base = atomicAdd(&H->list_count, total);
      base = __shfl_sync(0xFFFFFFFFu, base, 0);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const uint32_t idx = base + __popc(mask[i] & below);
        if (((mask[i] >> lane) & 1u) && idx < static_cast<uint32_t>(kStreamCap))
          cx.list[idx] = (static_cast<uint64_t>(~fkey(e[i])) << 32) | (gid[w] + i);
        base += __popc(mask[i]);
      }
    }
  }
  __syncthreads();
  return TileScan{st, cut};
}

// One more streaming pass over this CTA's part [g0, g0 + n), continuing the
// ring where the previous pass left it (`cg`: chunks streamed so far, which
// fixes each stage's mbarrier phase).  `body(st4, nq, gid)` scans one stage
// (nq float4 from global id gid); every thread calls it for every chunk, so
// it may use warp- and block-collective operations.  Returns false if a load
// did not land within the bounded wait.
template <typename F>
__device__ bool stream_pass(const SampleArgs& a, int row, int g0, int n, float* ring, unsigned long long* bars,
                            int& cg, F&& body) {
  const int nch = (n + kStreamChunk - 1) / kStreamChunk;
  const uint64_t pol = policy_evict_first();
  int s_issue = 0;
  bool ok = true;
  // every stage of the previous pass is consumed, and the leader's writes to
  // the ring (its scratch) are ordered before the copies overwrite it
  fence_proxy_async_smem();
  __syncthreads();
  if (threadIdx.x == 0)
    for (int c = 0; c < min(nch, kStreamStages - 1); ++c)
      stream_issue(a, row, g0, n, c, s_issue, ring, bars, pol, cg % kStreamStages);
  for (int c = 0; c < nch; ++c) {
    const int g = cg + c;
    const int stage = g % kStreamStages;
    if (threadIdx.x == 0 && c + kStreamStages - 1 < nch)
      stream_issue(a, row, g0, n, c + kStreamStages - 1, s_issue, ring, bars, pol, cg % kStreamStages);
    if (ok && !mbar_wait_bounded(smem_u32(&bars[stage]), static_cast<uint32_t>(g / kStreamStages) & 1u)) {
      if (threadIdx.x == 0) atomicOr(a.err, kErrSampleLoad);
      ok = false;
    }
    body(reinterpret_cast<const float4*>(ring + static_cast<size_t>(stage) * kStreamChunk),
         min(kStreamChunk, n - c * kStreamChunk) >> 2, static_cast<uint32_t>(g0 + c * kStreamChunk));
    __syncthreads();  // the stage is consumed
  }
  cg += nch;
  return ok;
}

// A top-k-off row on one CTA (the whole row, top-n already written from
// pass 1).  top_p < 1: pass 2 bins x = fl(l / T) on the fine bins (count and
// offset sums in the list area's first half), the CTA finds the window, pass 3
// sums the float64 masses above and below it, lists its members (the list
// area's second half) and draws over the certainly kept tokens, then the
// exact cut and the draw over the window's kept members.  top_p >= 1: one
// draw pass over every finite token.  Fills L.token / L.token_l; returns false
// when the window does not fit the list (the cluster kernel takes the row).
__device__ bool stream_koff(const Ctx& cx, LeaderState& L, const SampleArgs& a, float* ring, int n, int& cg) {
  SharedHeader* H = cx.H;
  const int g0 = static_cast<int>(cx.g0);
  const float T = L.T;
  const int t = static_cast<int>(threadIdx.x);
  const uint32_t k0 = static_cast<uint32_t>(a.seed), k1 = static_cast<uint32_t>(a.seed >> 32);
  constexpr float kGMax = 16.7f;  // > -log(-log(1 - 2^-24)) = 16.63: the largest noise value
  if (t == 0) H->gbound = kKeyNegInf;
  if (!(L.top_p < 1.0f)) {
    // pure sampling: argmax of x + g over every finite token
    __syncthreads();
    Best b;
    b.init(&H->gbound);
    const float invT = __frcp_rn(T);
    const bool approx = invT < INFINITY;
    stream_pass(a, cx.row, g0, n, ring, H->ring_bar, cg, [&](const float4* st4, int nq, uint32_t gid) {
#pragma unroll
      for (int it = 0; it < kStreamChunk / 4 / kThreads; ++it) {
        const int q = t + it * kThreads;
        if (q >= nq) continue;
        const float4 v4 = st4[q];
        const float v[4] = {v4.x, v4.y, v4.z, v4.w};
        float xu[4];
        bool any = false;
        float xmax = -INFINITY;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const bool fin = key_finite(fkey(v[i]));
          const float xa = approx ? v[i] * invT : scale_x(v[i], T);
          xu[i] = fin ? (approx ? xa + fabsf(xa) * 5e-7f + 1e-37f : xa) : -INFINITY;
          any |= fin;
          xmax = fmaxf(xmax, xu[i]);
        }
        if (!any) continue;
        const float sb = b.bound_score();
        if (sb > -INFINITY && xmax + kGMax < sb - score_tol(sb)) continue;
        const uint32_t gq = gid + 4u * static_cast<uint32_t>(q);
        const uint4 w = philox4x32_10(make_uint4(gq >> 2, cx.pos, cx.req, 0u), k0, k1);
        const float bl = b.bound_l2e();
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          if (!(xu[i] > -INFINITY)) continue;
          const uint32_t wi = word_of(w, i);
          if (bl != Best::kNoBound && Best::rejects(bl, xu[i], wi)) continue;
          b.offer_passed(scale_x(v[i], T), v[i], wi, static_cast<int32_t>(gq + i));
        }
      }
    });
    push_best(cx, b);
    __syncthreads();
    finish_draw(cx, L, -INFINITY, 0x7FFFFFFF);
    return true;
  }
  // passes 2 and 3 divide every logit by T: with scale_x_fast when the row's
  // temperature and the range of its nonzero |l| allow it (decided once per
  // row: each pass is instantiated for both quotients)
  const float y = __frcp_rn(T);
  const bool fast = fast_division_ok(T, fmaxf(fabsf(key_value(L.kmax)), fabsf(key_value(L.kminf))),
                                     H->row_amin == 0xFFFFFFFFu ? INFINITY : __uint_as_float(H->row_amin));
  // ---- pass 2: fine bins of x below m (the list area's first 16 KB)
  uint32_t* cnt = reinterpret_cast<uint32_t*>(cx.list);
  uint32_t* qs = cnt + kXBins;
  for (int i = t; i < 2 * kXBins; i += kThreads) cnt[i] = 0;
  const float m = L.m;
  const float inv_w = xbin_scale(m, scale_x(key_value(L.kminf), T));
  const double md = static_cast<double>(m);
  const double* tab = H->exp_tab;
  double zsum = 0.0;  // the float64 mass of every finite x: Z for the cut
  auto pass2 = [&](auto fast_tag) {
    constexpr bool kF = decltype(fast_tag)::value;
    stream_pass(a, cx.row, g0, n, ring, H->ring_bar, cg, [&](const float4* st4, int nq, uint32_t) {
#pragma unroll
      for (int it = 0; it < kStreamChunk / 4 / kThreads; ++it) {
        const int q = t + it * kThreads;
        if (q >= nq) continue;
        const float4 v4 = st4[q];
        const float v[4] = {v4.x, v4.y, v4.z, v4.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          if (!key_finite(fkey(v[i]))) continue;
          uint32_t qo;
          const float x = kF ? scale_x_fast(v[i], T, y) : scale_x(v[i], T);
          const int j = xbin_q(x, m, inv_w, qo);
          atomicAdd(&cnt[j], 1u);
          atomicAdd(&qs[j], qo);
          zsum += exp_neg64(static_cast<double>(x) - md, tab);
        }
      }
    });
  };
  if (fast) pass2(std::true_type{});
  else pass2(std::false_type{});
  const double zt = block_sum_d0(zsum, H);
  if (t == 0) H->row_z = zt;
  // ---- the window (a cluster of one CTA)
  Ctx wc = cx;
  wc.scratch = reinterpret_cast<uint8_t*>(cnt);
  wc.list = cx.list + kListCap;
  if (t == 0) H->list_count = 0;
  __syncthreads();
  Plan px{};
  px.m = m;
  px.step = inv_w;
  Plan e;
  if (!window_distributed(wc, px, e)) return false;
  // ---- the raw-key thresholds of the window: x = fl(l / T) and its bin are
  // monotone in l, so bin j < jlo (kept for certain) holds exactly for the
  // keys >= ka and jlo <= j <= jhi (the window) for kw <= key < ka; each is
  // found by a binary search over the row's finite keys with the same quotient
  const int jlo = static_cast<int>(e.lo), jhi = static_cast<int>(e.hi);
  auto thresholds = [&](auto fast_tag) {
    constexpr bool kF = decltype(fast_tag)::value;
    auto first_key = [&](auto pred) {  // the smallest key in [kminf, kmax] with pred(bin), else kmax + 1
      uint32_t lo = L.kminf, hi = L.kmax + 1u;
      while (lo < hi) {
        const uint32_t mid = lo + (hi - lo) / 2u;
        const float l = key_value(mid);
        if (pred(xbin(kF ? scale_x_fast(l, T, y) : scale_x(l, T), m, inv_w))) hi = mid;
        else lo = mid + 1u;
      }
      return lo;
    };
    const uint32_t ka = first_key([&](int jb) { return jb < jlo; });
    const uint32_t kw = min(first_key([&](int jb) { return jb <= jhi; }), ka);
    H->kcut_above = ka;
    H->kcut_window = kw;
  };
  if (t == 0) {
    if (fast) thresholds(std::true_type{});
    else thresholds(std::false_type{});
    H->gbound = kKeyNegInf;
  }
  __syncthreads();
  const uint32_t ka = H->kcut_above;
  const uint32_t kw = H->kcut_window;
  const double z_total = H->row_z;
  // tokens kept for certain (the fine bins above the window): when more than
  // a quarter of the row is kept, nearly every float4 group holds one, and
  // one Philox call per group (its four words, queued with the tokens) costs
  // less than one per queued token
  uint32_t kept_here = 0, kept_total = 0;
  for (int j = t; j < jlo; j += kThreads) kept_here += cnt[j];
  block_scan_u(kept_here, &kept_total, H);
  const bool dense = 4ull * kept_total > static_cast<unsigned long long>(n);
  // ---- pass 3: every key compared with the thresholds; the window's members
  // listed (sort key ~x key, id); every token kept for certain queued (with
  // its Philox word on a densely kept row), and the warp drains the queue 32
  // tokens at a time: its x, its float64 mass (the mass above the window, A)
  // and the draw
  Best b;
  b.init(&H->gbound);
  double above = 0.0;
  float xmin_ab = INFINITY;  // smallest x above the window
  // the fine bins' area is free once the window is found, until the window is sorted
  auto pass3 = [&](auto fast_tag, auto words_tag) {
    constexpr bool kF = decltype(fast_tag)::value;
    constexpr bool kW = decltype(words_tag)::value;
    DrawQueue<kW> dq;
    dq.init(cnt);
    auto one = [&](uint32_t lbits, uint32_t wd, int32_t id) {
      const float x = kF ? scale_x_fast(__uint_as_float(lbits), T, y) : scale_x(__uint_as_float(lbits), T);
      above += exp_neg64(static_cast<double>(x) - md, tab);
      xmin_ab = fminf(xmin_ab, x);
      const float bl = b.bound_l2e();
      if (bl == Best::kNoBound || !Best::rejects(bl, x, wd)) b.offer_passed(x, 0.0f, wd, id);
    };
    stream_pass(a, cx.row, g0, n, ring, H->ring_bar, cg, [&](const float4* st4, int nq, uint32_t gid) {
#pragma unroll
      for (int it = 0; it < kStreamChunk / 4 / kThreads; ++it) {
        const int q = t + it * kThreads;
        const bool valid = q < nq;
        const float4 v4 = valid ? st4[q] : make_float4(-INFINITY, -INFINITY, -INFINITY, -INFINITY);
        const float l[4] = {v4.x, v4.y, v4.z, v4.w};
        bool win[4], ab[4];
        bool any_win = false, any_ab = false;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const uint32_t k = fkey(l[i]);  // -inf and padding lie below kw: the row's keys are finite above it
          ab[i] = valid && k >= ka;
          win[i] = valid && k >= kw && k < ka;
          any_win |= win[i];
          any_ab |= ab[i];
        }
        const uint32_t gq = gid + 4u * static_cast<uint32_t>(q);
        if (__any_sync(0xFFFFFFFFu, any_win)) {
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const float x = win[i] ? (kF ? scale_x_fast(l[i], T, y) : scale_x(l[i], T)) : 0.0f;
            local_append(&H->list_count, wc.list, win[i], (static_cast<uint64_t>(~fkey(x)) << 32) | (gq + i));
          }
        }
        uint4 w = make_uint4(0u, 0u, 0u, 0u);
        if (kW && any_ab) w = philox4x32_10(make_uint4(gq >> 2, cx.pos, cx.req, 0u), k0, k1);
#pragma unroll
        for (int i = 0; i < 4; ++i)
          dq.push(ab[i], (static_cast<uint64_t>(__float_as_uint(l[i])) << 32) | (gq + i), word_of(w, i));
        dq.drain(false, cx.pos, cx.req, k0, k1, one);  // at most 31 + 128 queued
      }
    });
    dq.drain(true, cx.pos, cx.req, k0, k1, one);
  };
  if (dense) {
    if (fast) pass3(std::true_type{}, std::true_type{});
    else pass3(std::false_type{}, std::true_type{});
  } else {
    if (fast) pass3(std::true_type{}, std::false_type{});
    else pass3(std::false_type{}, std::false_type{});
  }
  const double ta = block_sum_d0(above, H);
  const float tx = block_min_f0(xmin_ab, H);
  if (t == 0) {
    H->ex_above[0] = ta;
    H->ex_below[0] = 0.0;  // unused: the cut takes the total mass
    H->ex_xmin[0] = tx;
    L.topn_count = 0;  // the window list starts at wc.list[0]
  }
  push_best(wc, b);
  __syncthreads();
  exact_tail(wc, L, z_total);
  return true;
}

// One CTA per (row, part) of a cluster of C CTAs per row; grid R * C.
__global__ void __launch_bounds__(kThreads, 2) stream_kernel(const __grid_constant__ SampleArgs a) {
  extern __shared__ __align__(128) uint8_t smem_raw[];
  SharedHeader* H = reinterpret_cast<SharedHeader*>(smem_raw);
  uint8_t* bins = smem_raw + ((sizeof(SharedHeader) + 127) & ~size_t(127));
  uint64_t* list = reinterpret_cast<uint64_t*>(bins + kStreamBinsBytes);
  float* ring = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(list) + kStreamListBytes);

  Ctx cx;
  cx.a = &a;
  cx.H = H;
  cx.scratch = bins;  // the compactions' 256 narrowing bins while streaming
  cx.list = list;
  cx.C = static_cast<uint32_t>(a.C);
  cx.rank = cluster_ctarank();
  cx.row = static_cast<int>(blockIdx.x / a.C);
  const vsl_row_params prm = a.params[cx.row];
  const bool take_koff = (a.select & kStreamKoff) != 0 && a.C == 1;
  if (!stream_row(prm, a.V, take_koff)) {
    if (a.select == kStreamMarks && cx.rank == 0 && threadIdx.x == 0) a.token_ids[cx.row] = kDeferred;
    return;  // the whole cluster leaves: the row is the cluster kernel's
  }
  cx.T = prm.temperature;
  cx.top_k = prm.top_k;
  cx.top_p = prm.top_p;
  cx.req = prm.request_id;
  cx.pos = prm.position;
  cx.g0 = static_cast<long long>(cx.rank) * a.part;
  const long long g1 = min(cx.g0 + a.part, static_cast<long long>(a.V));
  const int n = g1 > cx.g0 ? static_cast<int>(g1 - cx.g0) : 0;
  cx.n4 = n >> 2;
  cx.part4 = nullptr;
  const int nch = (n + kStreamChunk - 1) / kStreamChunk;
  const bool greedy = prm.temperature == 0.0f;
  const bool k_on = !greedy && prm.top_k > 0 && prm.top_k < a.V;
  uint32_t R = a.n_logprobs > 0 ? static_cast<uint32_t>(a.n_logprobs) : 1u;
  if (k_on) R = max(R, static_cast<uint32_t>(prm.top_k));
  // tile mode: every row this kernel takes on one CTA (a top-k-off row of a
  // large batch then replaces its first pass with the records and the top-n quarters)
  const bool tiles = a.tile_stats != nullptr && a.C == 1 && (greedy || k_on || take_koff);

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStreamStages; ++s) mbar_init(smem_u32(&H->ring_bar[s]), 1);
    fence_mbar_init();
    H->list_count = 0;
  }
  for (int j = threadIdx.x; j < 256; j += kThreads) H->exp_tab[j] = exp2(static_cast<double>(j) / 256.0);
  __syncthreads();
  // thread 0 keeps kStreamStages - 1 chunks in flight ahead of the one scanned
  const uint64_t pol = policy_evict_first();
  const int g0 = static_cast<int>(cx.g0);
  int s_issue = 0;
  if (threadIdx.x == 0 && !tiles)
    for (int c = 0; c < min(nch, kStreamStages - 1); ++c) stream_issue(a, cx.row, g0, n, c, s_issue, ring, H->ring_bar, pol);

  constexpr float kLog2e = 1.4426950408889634f;
  uint32_t thr = 0;  // every key (-inf included) is a candidate until the first compaction
  ScanStats st{0u, 0xFFFFFFFFu, 0xFFFFFFFFu, kScanNoMax, 0.0f};
  // a top-k-off row on one CTA also finds its smallest nonzero |l| (the
  // domain check of the later passes' division)
  const bool amin_scan = take_koff && !greedy && !k_on;
  bool load_ok = true;
  bool dropped = false;  // some candidate was not listed: the row goes to the cluster kernel
  uint32_t seen = 0;     // this warp's list end after its appends of the current chunk
  // compact when less than a chunk of room is left, and, once the threshold
  // is set, whenever the list has grown past 4R + 64: the threshold then
  // follows the R-th largest key seen so far and far fewer logits are listed
  uint32_t grow_limit = static_cast<uint32_t>(kStreamCap - kStreamChunk);
  const uint32_t small_limit = min(grow_limit, 4u * R + 64u);
  const int lane = threadIdx.x & 31;
  // Rounds of one chunk until the first compaction has set the threshold, then
  // of kStreamRound: one block barrier per round, so a warp that lists
  // candidates holds the others up once per round, not once per chunk.  The
  // list then keeps room for one chunk of candidates, not a round's: a round
  // that lists more (a flood of ties at the threshold) overflows it, and the
  // row is deferred.
  int next_issue = min(nch, kStreamStages - 1);  // thread 0: chunks issued so far
  int step = 1;
  if (tiles) {
    const TileScan ts = stream_tiles(cx, a, R, reinterpret_cast<uint32_t*>(ring));
    st = ts.st;
    thr = ts.cut;
  }
  for (int c = 0; c < (tiles ? 0 : nch);) {
    const int cur = step;  // this round's chunks (a compaction below may widen the next rounds)
    // refill every stage whose chunk all threads have scanned (the last barrier has passed)
    if (threadIdx.x == 0)
      for (; next_issue < min(nch, c + kStreamStages); ++next_issue)
        stream_issue(a, cx.row, g0, n, next_issue, s_issue, ring, H->ring_bar, pol);
    for (int u = 0; u < cur && c + u < nch; ++u) {
      const int cc = c + u;
      const int stage = cc % kStreamStages;
      if (load_ok && !mbar_wait_bounded(smem_u32(&H->ring_bar[stage]), static_cast<uint32_t>(cc / kStreamStages) & 1u)) {
        if (threadIdx.x == 0) atomicOr(a.err, kErrSampleLoad);
        load_ok = false;
      }
      const float4* st4 = reinterpret_cast<const float4*>(ring + static_cast<size_t>(stage) * kStreamChunk);
      const int nq = min(kStreamChunk, n - cc * kStreamChunk) >> 2;
      const uint32_t gid = static_cast<uint32_t>(g0 + cc * kStreamChunk);
      if (amin_scan) {
        if (nq == kStreamChunk / 4) stream_scan<true, true>(st4, nq, thr, gid, st, seen, &H->list_count, list);
        else stream_scan<false, true>(st4, nq, thr, gid, st, seen, &H->list_count, list);
      } else {
        if (nq == kStreamChunk / 4) stream_scan<true, false>(st4, nq, thr, gid, st, seen, &H->list_count, list);
        else stream_scan<false, false>(st4, nq, thr, gid, st, seen, &H->list_count, list);
      }
    }
    // the round's stages are consumed and the appends are visible; the barrier
    // also tells every thread whether the list has less than a chunk of room left
    const bool full = __syncthreads_or(seen > grow_limit) != 0;
    seen = 0;
    if (full && !dropped) {
      uint32_t left;
      dropped = H->list_count > static_cast<uint32_t>(kStreamCap);
      thr = stream_compact(cx, R, thr, 2, left);
      // no room for another chunk (ties at the threshold): the row is deferred, stop listing
      if (left > static_cast<uint32_t>(kStreamCap - kStreamChunk)) dropped = true;
      if (dropped) thr = 0xFFFFFFFFu;
      grow_limit = min(static_cast<uint32_t>(kStreamCap - kStreamChunk), max(small_limit, left + 64u));
      step = kStreamRound;
    }
    c += cur;
  }

  int cg = tiles ? 0 : nch;  // chunks streamed so far (the ring's position)
  // ---- CTA statistics (the cluster kernel's CtaStats layout)
  // (m, s) pairs merge by rescaling to the larger m; empty sums add 0
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    st.kmax = max(st.kmax, __shfl_xor_sync(0xFFFFFFFFu, st.kmax, o));
    st.kmf = min(st.kmf, __shfl_xor_sync(0xFFFFFFFFu, st.kmf, o));
    st.amin = min(st.amin, __shfl_xor_sync(0xFFFFFFFFu, st.amin, o));
    const float om = __shfl_xor_sync(0xFFFFFFFFu, st.m, o);
    const float os = __shfl_xor_sync(0xFFFFFFFFu, st.s, o);
    // a lane with an empty sum has no maximum to keep
    const float nm = fmaxf(st.s != 0.0f ? st.m : -INFINITY, os != 0.0f ? om : -INFINITY);
    st.s = (st.s == 0.0f ? 0.0f : st.s * fast_exp2((st.m - nm) * kLog2e)) +
           (os == 0.0f ? 0.0f : os * fast_exp2((om - nm) * kLog2e));
    st.m = nm > -INFINITY ? nm : kScanNoMax;
  }
  const int warp = threadIdx.x >> 5;
  if (lane == 0) {
    H->red_u[warp * 4 + 0] = st.kmax;
    H->red_u[warp * 4 + 1] = st.amin;
    H->red_u[warp * 4 + 2] = st.kmf;
    H->red_u[warp * 4 + 3] = load_ok ? 0u : 1u;
    H->red_f[warp * 2 + 0] = st.m;
    H->red_f[warp * 2 + 1] = st.s;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    uint32_t ka = 0, kf = 0xFFFFFFFFu, bad = 0, am = 0xFFFFFFFFu;
    float M = -INFINITY;  // over the warps whose sum is not empty
    for (int i = 0; i < kWarps; ++i) {
      ka = max(ka, H->red_u[i * 4 + 0]);
      am = min(am, H->red_u[i * 4 + 1]);
      kf = min(kf, H->red_u[i * 4 + 2]);
      bad |= H->red_u[i * 4 + 3];
      if (H->red_f[i * 2 + 1] != 0.0f) M = fmaxf(M, H->red_f[i * 2]);
    }
    float S = 0.0f;
    for (int i = 0; i < kWarps; ++i)
      if (H->red_f[i * 2 + 1] != 0.0f) S += H->red_f[i * 2 + 1] * fast_exp2((H->red_f[i * 2] - M) * kLog2e);
    // NaN of either sign turns the sum NaN; +inf (and a NaN's key) lies at or above key(+inf)
    bad |= (ka >= kKeyPosInf || isnan(S)) ? 1u : 0u;
    H->row_amin = am;
    H->stats.kmax = ka;
    H->stats.kminf = kf == 0xFFFFFFFFu ? kf : kf + (kKeyNegInf + 1u);  // smallest finite key
    H->stats.bad = bad;
    const bool none = !(M > -INFINITY);
    H->stats.m = none ? -INFINITY : M;
    H->stats.s = none ? 0.0f : S;
  }
  // exact local top R: the union of the parts' lists then holds the row's top R
  dropped |= H->list_count > static_cast<uint32_t>(kStreamCap);
  uint32_t own = 0;
  if (!dropped) thr = stream_compact(cx, R, thr, 64, own);
  own = dropped ? 0u : min(own, static_cast<uint32_t>(kStreamCap));
  const uint32_t overflow = dropped ? 1u : 0u;

  cx.scratch = reinterpret_cast<uint8_t*>(ring);  // the stream is over: the ring is scratch
  // ---- merge into the leader: statistics, thresholds, candidates
  if (cx.C > 1) cluster_sync();
  if (cx.rank != 0) {
    if (threadIdx.x == 0) {
      H->list_base = atom_add_dsmem_u32(mapa(smem_u32(&H->list_count), 0), own);
      *cluster_ptr(&H->all[cx.rank], 0) = H->stats;
      cluster_ptr(H->need_all, 0)[cx.rank] = thr;
      cluster_ptr(H->ok_all, 0)[cx.rank] = overflow;
    }
    __syncthreads();
    const uint32_t base = H->list_base;
    uint64_t* dst = cluster_ptr(list, 0);
    for (uint32_t i = threadIdx.x; i < own; i += kThreads)
      if (base + i < static_cast<uint32_t>(kStreamCap)) dst[base + i] = list[i];
    __syncthreads();
    cluster_sync();
    return;
  }
  if (threadIdx.x == 0) {
    H->all[0] = H->stats;
    H->need_all[0] = thr;
    H->ok_all[0] = overflow;
  }
  __syncthreads();
  if (cx.C > 1) cluster_sync();

  // ---- leader: the row from the merged list
  uint32_t defer = H->list_count > static_cast<uint32_t>(kListCap) ? 1u : 0u;
  for (uint32_t r = 0; r < cx.C; ++r) defer |= H->ok_all[r];
  if (defer) {
    if (threadIdx.x == 0) a.token_ids[cx.row] = kDeferred;
    return;
  }
  const int count = static_cast<int>(H->list_count);
  if (threadIdx.x == 0) H->listed = 0;  // leader_merge only merges statistics and flags
  __syncthreads();
  LeaderState& L = H->L;
  if (leader_merge(cx, L)) return;  // flagged row: outputs written
  uint64_t* buf = reinterpret_cast<uint64_t*>(cx.scratch);
  sort_entries(list, count, buf);
  if (!greedy && !k_on) {
    // top-k off (one CTA holds the row): the top-n now, then the passes of stream_koff
    list_resolve_sorted(cx, L, buf, count, false);
    if (!stream_koff(cx, L, a, ring, n, cg)) {
      if (threadIdx.x == 0) a.token_ids[cx.row] = kDeferred;
      return;
    }
    write_outputs(cx, L);
    return;
  }
  if (k_on) {
    // every value that can scale to theta_k must have been a candidate in every part
    const float theta_k = scale_x(key_value(entry_key(buf[min(L.r_k, count) - 1])), L.T);
    const uint32_t lo = raw_prefilter(theta_k, L.T);
    uint32_t miss = 0;
    for (uint32_t r = 0; r < cx.C; ++r) miss |= H->need_all[r] > lo ? 1u : 0u;
    if (miss) {
      if (threadIdx.x == 0) a.token_ids[cx.row] = kDeferred;
      return;
    }
  }
  list_resolve_sorted(cx, L, buf, count, !greedy);
  write_outputs(cx, L);
}

}  // namespace vsl
