// vsl_gemm.cu - vocab-slice lm_head projection on sm_100a tensor cores.
//
// logits_s[r][j] = sum_h hidden[r][h] * W_s[j][h] for every vocab slice s, with
// no gather ("Qwen4Exp batch-sharded sampling: inside vLLM PR #61018",
// orcarouter.ai blog, sections "batch-sharded sampling in one paragraph" and
// "why three lines were the whole job").
//
// Design (each CTA walks the output tiles t = blockIdx.x, blockIdx.x +
// gridDim.x, ...; for batch tiles of 128 and 256 rows, which keep the tensor
// cores busy, the grid is as many CTAs as the SMs hold, so the kernel is
// persistent; for narrower ones, bound by the weight read, one CTA per tile):
//   * The MMA M side is the vocabulary (128 rows of W_s per tile) and the N side
//     is the batch rows (BN in {16, 32, 64, 128, 256}), so a small batch still
//     issues full-height tcgen05.mma instructions ("swap-AB").
//   * Warp 0 (one lane) streams K-slabs of 64 bf16 (one 128-byte swizzle row)
//     of W_s and hidden into a STAGES-deep shared-memory ring with 2-D TMA
//     loads (128B swizzle, zero fill past the edges, no multicast), running
//     ahead across tile boundaries.
//   * Warp 1 (one lane) issues tcgen05.mma.kind::f16 (bf16 x bf16 -> fp32) into
//     one of two 128 x BN fp32 accumulators in tensor memory (tile i uses
//     accumulator i mod 2), releasing each ring slot with tcgen05.commit.
//   * Warps 2..5 read the accumulator of the previous tile with tcgen05.ld
//     (one TMEM lane = one vocab row per thread), 16 batch rows at a time,
//     while the next tile's MMAs run, and hand the accumulator back through an
//     mbarrier once its last columns are in registers.  Each chunk of 16 batch
//     rows x 128 vocab rows is staged in shared memory in the output's layout
//     ([batch row][vocab]) and written with one TMA store (clipped at the
//     slice's edges).
//   * Optionally the epilogue also writes each batch row's tile statistics
//     for the 128 vocab rows of the tile (the block) from the staged chunk:
//     each of the 128 epilogue threads reads 16 consecutive logits of one
//     (batch row, quarter, half) from shared memory (maximum, smallest finite
//     value, smallest nonzero |l|, sum of exp(l - c)), and three shuffle steps
//     among the 8 threads of a batch row give the quarter maxima and the
//     block's sum and minima.
//   * The four epilogue warps meet at two mbarriers per chunk (bounded waits):
//     the chunk is staged, and the buffer is free again (read by the
//     statistics and by the store).
// Every wait is bounded; a wait that gives up sets the device error word and
// the CTA drains its own copies, frees its tensor memory and returns.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <mutex>

#include "vsl_internal.h"
#include "vsl_ptx.cuh"

namespace vsl {

constexpr int kBM = 128;        // vocab rows per tile (MMA M)
constexpr int kBK = 64;         // bf16 elements per K slab = 128 bytes
constexpr int kUmmaK = 16;      // K per tcgen05.mma.kind::f16
constexpr int kGemmThreads = 192;

struct GemmArgs {
  CUtensorMap tmap_w[VSL_MAX_SLICES];
  CUtensorMap tmap_h;
  float* out[VSL_MAX_SLICES];
  int R, H, V_s, S;
  int m_tiles;       // vocab tiles per slice
  int n_tiles;       // batch tiles
  int k_iters;       // K slabs
  int w_evict_first; // W read once (single batch tile): stream it through L2
  float* stats;      // optional tile statistics [R][S * m_tiles][8] (nullptr: none)
  uint32_t* err;
  CUtensorMap tmap_out[VSL_MAX_SLICES];  // fp32 [R][V_s] outputs, box 128 x 16
};

constexpr int kChunk = 16;                                      // batch rows per epilogue chunk
constexpr uint32_t kChunkBytes = kChunk * kBM * 4;              // one staged chunk (8 KB)
// staged chunk buffers: two, except for BN = 64, whose CTAs must fit two per SM
template <int BN>
__host__ __device__ constexpr int chunk_buffers() {
  return BN == 64 ? 1 : 2;
}

__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Shared-memory matrix descriptor for a K-major tile whose rows are 128 bytes,
// stored as TMA writes it with 128-byte swizzle: 8-row groups 1024 bytes apart.
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr & 0x3FFFF) >> 4);      // start address
  d |= static_cast<uint64_t>(1) << 16;                      // leading offset (unused, swizzled)
  d |= static_cast<uint64_t>(1024 >> 4) << 32;              // stride between 8-row groups
  d |= static_cast<uint64_t>(1) << 46;                      // descriptor version (sm_100)
  d |= static_cast<uint64_t>(2) << 61;                      // 128-byte swizzle
  return d;
}

// Instruction descriptor: D fp32, A and B bf16, both K-major, M = 128, N = BN.
template <int BN>
__device__ __forceinline__ uint32_t idesc_bf16_f32() {
  return (1u << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>(BN >> 3) << 17) |
         (static_cast<uint32_t>(kBM >> 4) << 24);
}

template <int BN>
__host__ __device__ constexpr int tmem_cols() {
  return BN < 32 ? 32 : BN;
}

template <int BN, int STAGES>
constexpr size_t gemm_smem_bytes() {
  return 1024 /*alignment slack*/ + static_cast<size_t>(STAGES) * (kBM + BN) * kBK * 2 +
         static_cast<size_t>(chunk_buffers<BN>()) * kChunkBytes + (2 * STAGES + 9) * 8 + 16;
}

// Tile statistics of one staged chunk (16 batch rows x 128 vocab rows,
// [row][vocab], -inf past the slice's end) by the 128 epilogue threads: thread
// e takes batch row e / 8 and the 16 logits of its half (e & 1) of quarter
// (e >> 1) & 3; the 8 threads of a row are consecutive lanes.
__device__ __forceinline__ void chunk_stats(const GemmArgs& a, const float* stage, int e, int lane, int n_first,
                                            int slice, int block) {
  constexpr float kLog2e = 1.4426950408889634f;
  const int row = e >> 3, sub = e & 7;
  const float4* src = reinterpret_cast<const float4*>(stage + row * kBM + sub * 16);
  // the four float4 in an order rotated by sub (fewer bank conflicts among the
  // 8 threads of a phase); the statistics do not depend on the order
  float v[16];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const float4 x = src[(j + sub) & 3];
    v[4 * j] = x.x;
    v[4 * j + 1] = x.y;
    v[4 * j + 2] = x.z;
    v[4 * j + 3] = x.w;
  }
  float mx = v[0], mn = INFINITY, am = INFINITY;
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    mx = fmaxf(mx, v[i]);
    mn = fminf(mn, isfinite(v[i]) ? v[i] : INFINITY);
    am = fminf(am, v[i] != 0.0f ? fabsf(v[i]) : INFINITY);  // fminf drops a NaN
  }
  mx = fmaxf(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, 1));  // the quarter's maximum
  mn = fminf(mn, __shfl_xor_sync(0xFFFFFFFFu, mn, 1));
  float bm = fmaxf(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, 2));
  bm = fmaxf(bm, __shfl_xor_sync(0xFFFFFFFFu, bm, 4));  // the block's maximum
  mn = fminf(mn, __shfl_xor_sync(0xFFFFFFFFu, mn, 2));
  mn = fminf(mn, __shfl_xor_sync(0xFFFFFFFFu, mn, 4));
#pragma unroll
  for (int o = 1; o < 8; o <<= 1) am = fminf(am, __shfl_xor_sync(0xFFFFFFFFu, am, o));
  const float c = isfinite(bm) ? bm : 0.0f;
  float sum = 0.0f;
#pragma unroll
  for (int i = 0; i < 16; ++i) sum += ex2_approx((v[i] - c) * kLog2e);
  sum += __shfl_xor_sync(0xFFFFFFFFu, sum, 1);
  sum += __shfl_xor_sync(0xFFFFFFFFu, sum, 2);
  sum += __shfl_xor_sync(0xFFFFFFFFu, sum, 4);
  const int g = lane & ~7;
  const float q0 = __shfl_sync(0xFFFFFFFFu, mx, g), q1 = __shfl_sync(0xFFFFFFFFu, mx, g + 2);
  const float q2 = __shfl_sync(0xFFFFFFFFu, mx, g + 4), q3 = __shfl_sync(0xFFFFFFFFu, mx, g + 6);
  const int n = n_first + row;
  if (sub == 0 && n < a.R) {
    float4* rec = reinterpret_cast<float4*>(a.stats + ((static_cast<size_t>(n) * a.S + slice) * a.m_tiles + block) * 8);
    rec[0] = make_float4(q0, q1, q2, q3);
    rec[1] = make_float4(sum, mn, am, 0.0f);
  }
}

template <int BN, int STAGES>
__global__ void __launch_bounds__(kGemmThreads, 1) logits_local_kernel(const __grid_constant__ GemmArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  constexpr uint32_t kABytes = kBM * kBK * 2;
  constexpr uint32_t kBBytes = BN * kBK * 2;
  constexpr uint32_t kAccCols = static_cast<uint32_t>(tmem_cols<BN>());
  constexpr int NB = chunk_buffers<BN>();
  uint8_t* sA = smem;
  uint8_t* sB = smem + STAGES * kABytes;
  float* chunk_buf = reinterpret_cast<float*>(smem + STAGES * (kABytes + kBBytes));  // [NB][16][128]
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + STAGES * (kABytes + kBBytes) + NB * kChunkBytes);
  uint64_t* empty = full + STAGES;
  uint64_t* acc_full = empty + STAGES;   // [2]: MMA -> epilogue
  uint64_t* acc_empty = acc_full + 2;    // [2]: epilogue (4 warps) -> MMA
  uint64_t* done = acc_empty + 2;        // every MMA of the CTA has completed
  uint64_t* chunk_full = done + 1;       // [2]: the 4 epilogue warps staged a chunk in buffer b
  uint64_t* chunk_free = chunk_full + 2; // [2]: buffer b was read by the statistics and the store
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(chunk_free + 2);
  volatile uint32_t* abort_flag = tmem_slot + 1;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int total = a.S * a.m_tiles * a.n_tiles;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(smem_u32(&full[s]), 1);
      mbar_init(smem_u32(&empty[s]), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(smem_u32(&acc_full[b]), 1);
      mbar_init(smem_u32(&acc_empty[b]), 4);
    }
    mbar_init(smem_u32(done), 1);
    for (int b = 0; b < 2; ++b) {
      mbar_init(smem_u32(&chunk_full[b]), 4);
      mbar_init(smem_u32(&chunk_free[b]), 4);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), 2 * kAccCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0 && lane == 0) {
    // ---------------- TMA producer: every K slab of every tile of this CTA
    prefetch_tmap(&a.tmap_h);
    const uint64_t pol_w = a.w_evict_first ? policy_evict_first() : policy_evict_last();
    const uint64_t pol_h = policy_evict_last();
    int it = 0;
    for (int t = blockIdx.x; t < total && !*abort_flag; t += gridDim.x) {
      const int mt = t / a.n_tiles;
      const int slice = mt / a.m_tiles;
      const int m0 = (mt % a.m_tiles) * kBM;
      const int n0 = (t % a.n_tiles) * BN;
      for (int k = 0; k < a.k_iters; ++k, ++it) {
        const int s = it % STAGES;
        const uint32_t ph = (it / STAGES) & 1;
        if (it >= STAGES && !mbar_wait_bounded(smem_u32(&empty[s]), ph ^ 1)) {
          atomicOr(a.err, kErrGemmProducer);
          *abort_flag = 1;
        }
        if (*abort_flag) break;
        mbar_arrive_expect_tx(smem_u32(&full[s]), kABytes + kBBytes);
        tma_load_2d(smem_u32(sA + s * kABytes), &a.tmap_w[slice], k * kBK, m0, smem_u32(&full[s]), pol_w);
        tma_load_2d(smem_u32(sB + s * kBBytes), &a.tmap_h, k * kBK, n0, smem_u32(&full[s]), pol_h);
      }
    }
    if (*abort_flag) {
      // drain our own copies: the last load issued to each slot must land
      for (int j = it - 1; j >= 0 && j >= it - STAGES; --j)
        mbar_wait_bounded(smem_u32(&full[j % STAGES]), (j / STAGES) & 1);
    }
  } else if (warp == 1 && lane == 0) {
    // ---------------- MMA issuer: tile i into accumulator i mod 2
    const uint32_t idesc = idesc_bf16_f32<BN>();
    int it = 0, i = 0;
    for (int t = blockIdx.x; t < total && !*abort_flag; t += gridDim.x, ++i) {
      const int b = i & 1;
      // the epilogue has drained this accumulator (tile i - 2)
      if (!mbar_wait_bounded(smem_u32(&acc_empty[b]), ((i >> 1) & 1) ^ 1)) {
        atomicOr(a.err, kErrGemmMma);
        *abort_flag = 1;
        break;
      }
      tc_fence_after();
      const uint32_t acc = tmem + static_cast<uint32_t>(b) * kAccCols;
      for (int k = 0; k < a.k_iters; ++k, ++it) {
        const int s = it % STAGES;
        const uint32_t ph = (it / STAGES) & 1;
        if (!mbar_wait_bounded(smem_u32(&full[s]), ph)) {
          atomicOr(a.err, kErrGemmMma);
          *abort_flag = 1;
        }
        if (*abort_flag) break;
        tc_fence_after();
        const uint64_t da = sw128_desc(smem_u32(sA + s * kABytes));
        const uint64_t db = sw128_desc(smem_u32(sB + s * kBBytes));
#pragma unroll
        for (int kk = 0; kk < kBK / kUmmaK; ++kk) {
          // advancing K by 16 bf16 = 32 bytes moves the start address by 2 (16-byte units)
          umma_f16(acc, da + 2 * kk, db + 2 * kk, idesc, (k | kk) != 0);
        }
        umma_commit(smem_u32(&empty[s]));
      }
      umma_commit(smem_u32(&acc_full[b]));
    }
    // every MMA must be complete before tensor memory is freed below
    umma_commit(smem_u32(done));
    mbar_wait_bounded(smem_u32(done), 0);
  } else if (warp >= 2) {
    // ---------------- epilogue: TMEM -> registers -> staged chunk -> TMA store, one tile behind the MMAs
    const int q = warp & 3;              // TMEM lane quarter this warp may access
    const int e = threadIdx.x - 64;      // 0..127
    const bool leader = threadIdx.x == 64;
    if (leader)
      for (int s = 0; s < a.S; ++s) prefetch_tmap(&a.tmap_out[s]);
    int i = 0;
    uint32_t chunk = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < total && ok; t += gridDim.x, ++i) {
      const int ab = i & 1;
      ok = mbar_wait_bounded(smem_u32(&acc_full[ab]), (i >> 1) & 1);
      if (!ok) {
        if (lane == 0) atomicOr(a.err, kErrGemmEpilogue);
        *abort_flag = 1;
      }
      tc_fence_after();
      // tcgen05.ld is warp-collective: decide for the whole warp
      if (!__all_sync(0xFFFFFFFFu, ok && !*abort_flag)) break;
      const int mt = t / a.n_tiles;
      const int slice = mt / a.m_tiles;
      const int block = mt % a.m_tiles;
      const int m0 = block * kBM;
      const bool m_ok = m0 + q * 32 + lane < a.V_s;  // this thread's vocab row exists
      const int n0 = (t % a.n_tiles) * BN;
      const uint32_t acc = tmem + static_cast<uint32_t>(ab) * kAccCols + (static_cast<uint32_t>(q * 32) << 16);
#pragma unroll 1
      for (int c = 0; c < BN && ok; c += kChunk, ++chunk) {
        uint32_t r[16];
        tmem_ld_x16(acc + c, r);
        tmem_ld_wait();
        if (c + kChunk >= BN) {
          // the accumulator's reads are complete: hand it back to the MMA warp
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(smem_u32(&acc_empty[ab]));
        }
        const uint32_t b = chunk % NB, use = chunk / NB;
        float* stage = chunk_buf + b * (kChunk * kBM);
        // the buffer's previous chunk has been read by the statistics and the store
        if (chunk >= static_cast<uint32_t>(NB) && !mbar_wait_bounded(smem_u32(&chunk_free[b]), (use - 1) & 1u)) {
          ok = false;
          break;
        }
#pragma unroll
        for (int j = 0; j < 16; ++j) stage[j * kBM + q * 32 + lane] = m_ok ? __uint_as_float(r[j]) : -INFINITY;
        fence_proxy_async_smem();  // the TMA store reads what the generic proxy wrote
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&chunk_full[b]));
        if (!mbar_wait_bounded(smem_u32(&chunk_full[b]), use & 1u)) {
          ok = false;
          break;
        }
        if (leader && n0 + c < a.R) {  // a box that starts past the last row writes nothing: not issued
          tma_store_2d(&a.tmap_out[slice], m0, n0 + c, smem_u32(stage));
          bulk_commit_group();
        }
        if (a.stats != nullptr) chunk_stats(a, stage, e, lane, n0 + c, slice, block);
        if (leader) bulk_wait_read_all();
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&chunk_free[b]));
      }
      if (!ok) {
        if (lane == 0) atomicOr(a.err, kErrGemmEpilogue);
        *abort_flag = 1;
      }
    }
    if (leader) bulk_wait_all();
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 2 * kAccCols);
  }
}

// ------------------------------------------------------------------ host side
namespace {

PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;

bool get_encoder() {
  std::call_once(g_encode_once, [] {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &fn, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  });
  return g_encode != nullptr;
}

// 2-D bf16 row-major [rows][cols] map with a box of 64 columns x box_rows rows.
bool encode_bf16_2d(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols, uint32_t box_rows) {
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * 2};
  cuuint32_t box[2] = {static_cast<cuuint32_t>(kBK), box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
                        estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// 2-D fp32 row-major [rows][cols] map with a box of 128 columns x 16 rows (epilogue stores).
bool encode_f32_out(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols) {
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * 4};
  cuuint32_t box[2] = {static_cast<cuuint32_t>(kBM), static_cast<cuuint32_t>(kChunk)};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<void*>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

template <int BN, int STAGES>
cudaError_t launch_bn(GemmArgs& args, const void* hidden, const void* const* w, int S, int H, int R,
                      int V_s, cudaStream_t stream) {
  for (int s = 0; s < S; ++s)
    if (!encode_bf16_2d(&args.tmap_w[s], w[s], V_s, H, kBM)) return cudaErrorInvalidValue;
  for (int s = 0; s < S; ++s)
    if (!encode_f32_out(&args.tmap_out[s], args.out[s], R, V_s)) return cudaErrorInvalidValue;
  if (!encode_bf16_2d(&args.tmap_h, hidden, R, H, BN)) return cudaErrorInvalidValue;
  args.n_tiles = (R + BN - 1) / BN;
  args.w_evict_first = args.n_tiles == 1;
  constexpr size_t smem = gemm_smem_bytes<BN, STAGES>();
  auto kern = logits_local_kernel<BN, STAGES>;
  // per device, with it current: the shared-memory attribute and the number of
  // CTAs that run at once (the persistent grid)
  constexpr int kMaxDevices = 64;
  static std::once_flag once[kMaxDevices];
  static cudaError_t attr_status[kMaxDevices];
  static int slots[kMaxDevices];
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::call_once(once[dev], [&] {
    int sms = 0, per_sm = 0;
    attr_status[dev] = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (attr_status[dev] == cudaSuccess)
      attr_status[dev] = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (attr_status[dev] == cudaSuccess)
      attr_status[dev] = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kGemmThreads, smem);
    slots[dev] = sms * per_sm;
    if (attr_status[dev] == cudaSuccess && slots[dev] <= 0) attr_status[dev] = cudaErrorInvalidConfiguration;
  });
  if (attr_status[dev] != cudaSuccess) return attr_status[dev];
  const long long tiles = static_cast<long long>(S) * args.m_tiles * args.n_tiles;
  if (tiles > 0x7FFFFFFF) return cudaErrorInvalidConfiguration;
  args.S = S;
  // tensor-bound widths (BN >= 128) run persistent, one CTA per slot, so each
  // tile's epilogue overlaps the next tile's MMAs; the narrow widths are bound
  // by the weight read and keep one CTA per tile (the hardware then hands a
  // free slot the next tile, whatever the pace of each SM)
  const int grid = static_cast<int>(BN < 128 || tiles < slots[dev] ? tiles : slots[dev]);
  kern<<<grid, kGemmThreads, smem, stream>>>(args);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_logits_local(const void* hidden, const void* const* w_slices, float* const* logits,
                                int R, int H, int S, int V_s, float* stats, cudaStream_t stream) {
  if (!get_encoder()) return cudaErrorNotSupported;
  GemmArgs args{};
  args.stats = stats;
  for (int s = 0; s < S; ++s) args.out[s] = logits[s];
  args.R = R;
  args.H = H;
  args.V_s = V_s;
  args.m_tiles = (V_s + kBM - 1) / kBM;
  args.k_iters = (H + kBK - 1) / kBK;
  args.err = device_error_word();
  if (args.err == nullptr) return cudaErrorUnknown;
  if (R <= 16) return launch_bn<16, 8>(args, hidden, w_slices, S, H, R, V_s, stream);
  if (R <= 32) return launch_bn<32, 8>(args, hidden, w_slices, S, H, R, V_s, stream);
  if (R <= 64) return launch_bn<64, 4>(args, hidden, w_slices, S, H, R, V_s, stream);
  if (R <= 128) return launch_bn<128, 6>(args, hidden, w_slices, S, H, R, V_s, stream);
  return launch_bn<256, 4>(args, hidden, w_slices, S, H, R, V_s, stream);
}

}  // namespace vsl
