// gemm.cu -- INT8 x INT8 -> INT32 GEMM with the fused dequantising epilogue,
// written for the sm_100a tensor cores (tcgen05 + tensor memory + TMA).
//
// Source pages (by title and section): "SmoothQuant, in depth" --
// "Granularity: O1, O2, O3 and what kernels run today" (an INT32 accumulator,
// both scales applied in the epilogue, out = acc x scale_token[i] x
// scale_channel[j], converted to BF16) and "The problem SmoothQuant solves"
// (both operands 8-bit integers, INT32 accumulation); "SmoothQuant, in depth"
// -- "Serving and operations" (prefill is compute-bound, small-batch decode is
// memory-bound: it streams the INT8 weights once).
//
// One kernel template serves both regimes.  The MMA's M side ("P", 128 rows
// per tile) and N side ("Q", BN rows per tile) are both K-major INT8 tiles:
//   prefill: P = activation rows (tokens), Q = weight rows (channels), BN=256;
//   decode:  P = weight rows, Q = the few token rows (BN = 16..256), so the
//            weight stream fills the 128-row MMA, and stream-K (or an
//            explicit split-K) spreads the weight bytes evenly over all SMs;
//            INT32 partial sums are added exactly by a second kernel.
// Prefill also has a CTA-pair variant (tcgen05 cta_group::2, 256-row tiles).
// Persistent CTAs (one per SM), warp-specialised:
//   warp 0      TMA producer: 128-byte-swizzled K-major tiles into an
//               mbarrier ring of STAGES stages (no cluster multicast);
//   warp 1      allocates tensor memory and issues tcgen05.mma.kind::i8
//               (one thread), committing each stage back to the producer and
//               each finished tile to the epilogue;
//   warps 2-5   epilogue: tcgen05.ld of the INT32 accumulator (double
//               buffered in tensor memory, 2 x BN columns), the two scales,
//               bf16 rounding and the global stores, overlapping the next
//               tile's main loop;
//   warp 6      the issuer's scheduler: it waits on the stage-full and
//               accumulator-free barriers and hands each completed wait to
//               warp 1 through a named barrier, so the issuing thread never
//               touches shared memory between MMAs.
// Every mbarrier wait is bounded; a wait that runs out records
// SQ_ERR_PIPELINE_TIMEOUT in the device error word, and the CTA drains its
// outstanding TMA loads and MMAs, frees its tensor memory and returns.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>

#include "sq_device.cuh"
#include "sq_launch.h"

namespace sq {
namespace {

constexpr int BM = 128;  // MMA M (rows of P per tile)
constexpr int BK = 128;  // K bytes per stage = one 128-byte swizzle atom row
constexpr int UMMA_K = 32;  // K of one kind::i8 MMA
// warp 0 TMA producer, warp 1 MMA issuer, warps 2-5 epilogue, warp 6 the MMA
// issuer's scheduler: it does the issuer's barrier waits and hands each
// completed wait over through named barrier 1.  (A shared-memory access by the
// thread that issues tcgen05.mma -- an mbarrier wait, even on a completed
// phase -- idles the tensor pipe for a few hundred cycles; a named barrier
// does not: measured 128 vs 202 cycles per 256x256x32 pair MMA with a wait
// every four MMAs.)
constexpr int kThreads = 224;
constexpr int kSchedWarp = 6;
// Weight blocks (128 rows x 128 bytes) a decode CTA prefetches into L2 before
// the previous grid has finished: 256 KB per SM, 38 MB over 148 SMs.
constexpr int kPrefetchBlocks = 16;

// Named barrier 1 joins the MMA-issuing warp and its scheduling warp once per
// wait; the OR of the two warps' predicates tells both whether to stop.
__device__ __forceinline__ bool sched_sync(bool stop) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 q, %1, 0;\n\t"
      "bar.red.or.pred p, 1, 64, q;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(r)
      : "r"(stop ? 1u : 0u)
      : "memory");
  return r != 0;
}

template <int BN>
struct Cfg {
  static constexpr int A_BYTES = BM * BK;
  static constexpr int B_BYTES = BN * BK;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  // as many stages as fit 220 KB (at most 12: the narrow decode tiles keep
  // up to 216 KB of weight blocks in flight per SM)
  static constexpr int STAGES_FIT = (220 * 1024) / STAGE_BYTES;
  static constexpr int STAGES = STAGES_FIT > 12 ? 12 : STAGES_FIT;
  static constexpr int TMEM_COLS =
      2 * BN <= 32 ? 32 : 2 * BN <= 64 ? 64 : 2 * BN <= 128 ? 128 : 2 * BN <= 256 ? 256 : 512;
  static constexpr int NUM_BARS = 2 * STAGES + 5;
  static constexpr int SMEM_BYTES = 1024 + STAGES * STAGE_BYTES + 8 * NUM_BARS + 16;
  static constexpr int CHUNK = BN < 32 ? BN : 32;  // accumulator columns per tcgen05.ld
  static_assert(STAGES >= 2, "pipeline too shallow");
  static_assert(BN % 16 == 0 && BN >= 16 && BN <= 256, "invalid MMA N for M = 128");
};

struct Params {
  int P, Q, K;                     // rows on the MMA M side, rows on the N side, reduction
  int p_blocks, q_blocks, k_blocks, splits, group, units;
  const float* p_scale;            // scale per P row
  const float* q_scale;            // scale per Q row
  void* out;
  int64_t ldo;
  int epi;                         // SQ_EPI_*
  int swap;                        // 0: out[p][q]; 1: out[q][p]
  int32_t* partial;                // split-K: raw sums [split][M][N] (M = token extent)
  int64_t wait_polls;              // > 0: poll budget per wait; 0: ~2 s of SM clock cycles
  int* error_word;                 // device error word of this device
  int vec_out;                     // output rows 16-byte aligned: 128-bit stores allowed
  // stream-K (decode tiles): CTA c runs the flattened (tile, k-block)
  // iterations [c * sk_iters / G, (c + 1) * sk_iters / G); a tile whose K
  // range is split between CTAs leaves partial sums in slots 2c (the CTA's
  // first tile) and 2c + 1 (its last), [slot][Q][128], summed afterwards by
  // streamk_fixup_kernel
  int streamk;
  int64_t sk_iters;
  int32_t* sk_partial;
  // prefill bf16 epilogues: running max of |out| per P row (token), as
  // binary32 bits, for a following per-token requantisation (or null)
  float* row_absmax;
};

// Give-up point of a pipeline wait, in SM clock cycles (about 2 s at the
// B200's 1.965 GHz maximum clock, longer at lower clocks).
constexpr long long kWaitBudgetCycles = 4000000000LL;

// Bounded wait on an mbarrier phase; `abort` may be null.  The first probe is
// free of any timer read (the common case: the phase is already complete);
// the budget is kept with the SM-local cycle counter, which is cheap to read
// (the global nanosecond timer costs a few hundred cycles per read).
__device__ bool wait_phase(uint32_t bar, uint32_t parity, int64_t polls, const volatile int* abort) {
  if (mbar_try_wait(bar, parity)) return true;
  if (polls > 0) {
    for (int64_t i = 1; i < polls; ++i) {
      if (mbar_try_wait(bar, parity)) return true;
      if (abort && *abort) return false;
    }
    return false;
  }
  const long long t0 = clock64();
  for (uint32_t i = 0;; ++i) {
    if (mbar_try_wait(bar, parity)) return true;
    if (abort && *abort) return false;
    if ((i & 63u) == 63u && clock64() - t0 > kWaitBudgetCycles) return false;
  }
}

__device__ __forceinline__ void fail(int* word, volatile int* abort) {
  record_device_error(word, SQ_ERR_PIPELINE_TIMEOUT);
  *abort = 1;
}

// Tile number -> (P block, Q block): bands of `group` P blocks sweep all Q
// blocks before the next band starts, so a band's Q operand stays in L2.
__device__ __forceinline__ void tile_coords(const Params& p, int tile, int& pb, int& qb) {
  const int band_tiles = p.group * p.q_blocks;
  const int band = tile / band_tiles;
  const int rem = tile - band * band_tiles;
  const int first = band * p.group;
  const int gsize = min(p.group, p.p_blocks - first);
  pb = first + rem % gsize;
  qb = rem / gsize;
}

__device__ __forceinline__ void decode_unit(const Params& p, int u, int& pb, int& qb, int& kb0,
                                            int& kb1, int& split) {
  split = u % p.splits;
  tile_coords(p, u / p.splits, pb, qb);
  kb0 = static_cast<int>((static_cast<int64_t>(split) * p.k_blocks) / p.splits);
  kb1 = static_cast<int>((static_cast<int64_t>(split + 1) * p.k_blocks) / p.splits);
}

// The work units of one CTA, in order: round-robin tiles (or split-K slices),
// or the CTA's stream-K range cut at tile boundaries.  All three warp roles
// walk the same sequence.
struct Work {
  int u;               // round-robin unit
  int64_t it, it_end;  // stream-K iteration range still to run
  bool first;          // stream-K: the next unit is the CTA's first
};

__device__ __forceinline__ int64_t sk_start(const Params& p, int64_t c) {
  return c * p.sk_iters / gridDim.x;
}

__device__ __forceinline__ void work_init(const Params& p, Work& w) {
  w.u = blockIdx.x;
  w.it = sk_start(p, blockIdx.x);
  w.it_end = sk_start(p, blockIdx.x + 1);
  w.first = true;
}

// Next unit of the CTA, or false.  slot < 0: the unit ends in the output (or
// its split-K slice); slot >= 0: a stream-K partial-sum slot.
__device__ __forceinline__ bool work_next(const Params& p, Work& w, int& pb, int& qb, int& kb0,
                                          int& kb1, int& split, int& slot) {
  if (p.streamk) {
    if (w.it >= w.it_end) return false;
    const int tile = static_cast<int>(w.it / p.k_blocks);
    kb0 = static_cast<int>(w.it - static_cast<int64_t>(tile) * p.k_blocks);
    const int64_t left = w.it_end - w.it;
    kb1 = left < p.k_blocks - kb0 ? kb0 + static_cast<int>(left) : p.k_blocks;
    w.it += kb1 - kb0;
    tile_coords(p, tile, pb, qb);
    split = 0;
    slot = (kb0 == 0 && kb1 == p.k_blocks) ? -1 : 2 * static_cast<int>(blockIdx.x) + (w.first ? 0 : 1);
    w.first = false;
    return true;
  }
  if (w.u >= p.units) return false;
  decode_unit(p, w.u, pb, qb, kb0, kb1, split);
  slot = -1;
  w.u += gridDim.x;
  return true;
}

// Epilogue for one CHUNK of accumulator columns held by this thread (row p of
// the P side, columns q0 .. q0 + CHUNK - 1 of the Q side).
// The accumulator word as a float: INT32 sums convert (rounding above 2^24),
// FP8 GEMMs accumulate in fp32 already.
template <bool kF8>
__device__ __forceinline__ float acc_value(uint32_t r) {
  if constexpr (kF8) return __uint_as_float(r);
  else return __int2float_rn(static_cast<int>(r));
}

// Prefill (tokens on the P side) bf16 epilogue of CHUNK accumulator columns
// of row p (< P), starting at column q0, with the row's token scale xs and
// the columns' channel scales ws.  Returns the chunk's max |bf16 out| when
// prm.row_absmax asks for it (else 0).
template <int CHUNK, bool kF8>
__device__ __forceinline__ float epi_row_bf16(const Params& prm, const uint32_t (&r)[32], int p,
                                              int q0, float xs, const float (&ws)[CHUNK]) {
  const bool relu = prm.epi == SQ_EPI_BF16_RELU;
  float v[CHUNK];
#pragma unroll
  for (int j = 0; j < CHUNK; ++j) {
    float t = __fmul_rn(__fmul_rn(acc_value<kF8>(r[j]), xs), ws[j]);
    if (relu) t = t > 0.0f ? t : 0.0f;  // -0 (a zero scale) becomes +0
    v[j] = t;
  }
  __nv_bfloat16* dst = static_cast<__nv_bfloat16*>(prm.out) + static_cast<int64_t>(p) * prm.ldo + q0;
  // max |bf16 out| of the chunk, as bf16 bits (magnitudes order like ints)
  const bool track = prm.row_absmax != nullptr;
  uint32_t am = 0;
  if (prm.vec_out && q0 + CHUNK <= prm.Q) {
#pragma unroll
    for (int j = 0; j < CHUNK; j += 8) {
      uint32_t w[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const __nv_bfloat162 h = __floats2bfloat162_rn(v[j + 2 * i], v[j + 2 * i + 1]);
        w[i] = *reinterpret_cast<const uint32_t*>(&h);
        if (track) am = max(am, max(w[i] & 0x7fffu, (w[i] >> 16) & 0x7fffu));
      }
      *reinterpret_cast<uint4*>(dst + j) = make_uint4(w[0], w[1], w[2], w[3]);
    }
  } else {
#pragma unroll
    for (int j = 0; j < CHUNK; ++j)
      if (q0 + j < prm.Q) {
        const __nv_bfloat16 h = __float2bfloat16_rn(v[j]);
        dst[j] = h;
        if (track)
          am = max(am, static_cast<uint32_t>(*reinterpret_cast<const uint16_t*>(&h)) & 0x7fffu);
      }
  }
  return __uint_as_float(am << 16);
}

// The channel scales of columns q0 .. q0 + CHUNK - 1 (0 past the matrix).
template <int CHUNK>
__device__ __forceinline__ void load_col_scales(const Params& prm, int q0, float (&ws)[CHUNK]) {
  if (q0 + CHUNK <= prm.Q) {
#pragma unroll
    for (int j = 0; j < CHUNK; j += 4) {
      const float4 t = __ldg(reinterpret_cast<const float4*>(prm.q_scale + q0 + j));
      ws[j] = t.x; ws[j + 1] = t.y; ws[j + 2] = t.z; ws[j + 3] = t.w;
    }
  } else {
#pragma unroll
    for (int j = 0; j < CHUNK; ++j) ws[j] = (q0 + j < prm.Q) ? __ldg(prm.q_scale + q0 + j) : 0.0f;
  }
}

// Returns the chunk's max |bf16 out| when prm.row_absmax asks for it (else 0).
template <int CHUNK, bool kF8 = false>
__device__ __forceinline__ float store_chunk(const Params& prm, const uint32_t (&r)[32], int p,
                                             int q0, int split, int slot) {
  if (p >= prm.P) return 0.0f;
  if (slot >= 0) {  // stream-K partial sums of a decode tile: [slot][Q][128]
    int32_t* dst = prm.sk_partial + static_cast<int64_t>(slot) * prm.Q * BM + (p % BM);
#pragma unroll
    for (int j = 0; j < CHUNK; ++j)
      if (q0 + j < prm.Q) dst[static_cast<int64_t>(q0 + j) * BM] = static_cast<int32_t>(r[j]);
    return 0.0f;
  }
  if (prm.partial) {  // split-K partial sums, [split][M][N] with M = Q (tokens), N = P
#pragma unroll
    for (int j = 0; j < CHUNK; ++j) {
      const int q = q0 + j;
      if (q < prm.Q)
        prm.partial[(static_cast<int64_t>(split) * prm.Q + q) * prm.P + p] =
            static_cast<int32_t>(r[j]);
    }
    return 0.0f;
  }
  if (prm.epi == SQ_EPI_I32_RAW || prm.epi == SQ_EPI_F32_RAW) {  // the accumulator's bits
    int32_t* o = static_cast<int32_t*>(prm.out);
    if (!prm.swap) {
      int32_t* dst = o + static_cast<int64_t>(p) * prm.ldo + q0;
      if (prm.vec_out && q0 + CHUNK <= prm.Q) {
#pragma unroll
        for (int j = 0; j < CHUNK; j += 4)
          *reinterpret_cast<uint4*>(dst + j) = make_uint4(r[j], r[j + 1], r[j + 2], r[j + 3]);
      } else {
#pragma unroll
        for (int j = 0; j < CHUNK; ++j)
          if (q0 + j < prm.Q) dst[j] = static_cast<int32_t>(r[j]);
      }
    } else {
#pragma unroll
      for (int j = 0; j < CHUNK; ++j)
        if (q0 + j < prm.Q) o[static_cast<int64_t>(q0 + j) * prm.ldo + p] = static_cast<int32_t>(r[j]);
    }
    return 0.0f;
  }
  const bool relu = prm.epi == SQ_EPI_BF16_RELU;
  __nv_bfloat16* o = static_cast<__nv_bfloat16*>(prm.out);
  if (!prm.swap) {
    // token scale for this row, channel scale per column
    const float xs = __ldg(prm.p_scale + p);
    float ws[CHUNK];
    load_col_scales<CHUNK>(prm, q0, ws);
    return epi_row_bf16<CHUNK, kF8>(prm, r, p, q0, xs, ws);
  } else {
    // channel scale for this row (weight row p), token scale per column
    const float ws = __ldg(prm.p_scale + p);
#pragma unroll
    for (int j = 0; j < CHUNK; ++j) {
      const int q = q0 + j;
      if (q < prm.Q) {
        const float xs = __ldg(prm.q_scale + q);
        float t = __fmul_rn(__fmul_rn(acc_value<kF8>(r[j]), xs), ws);
        if (relu) t = t > 0.0f ? t : 0.0f;  // -0 (a zero scale) becomes +0
        o[static_cast<int64_t>(q) * prm.ldo + p] = __float2bfloat16_rn(t);
      }
    }
  }
  return 0.0f;
}

template <int BN, bool kF8>
__global__ void __launch_bounds__(kThreads, 1)
    w8a8_gemm_kernel(const __grid_constant__ CUtensorMap mapP,
                     const __grid_constant__ CUtensorMap mapQ, const Params prm) {
  using C = Cfg<BN>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_u32 = smem_u32(smem_raw);
  const uint32_t base = (raw_u32 + 1023u) & ~1023u;
  uint8_t* base_ptr = smem_raw + (base - raw_u32);
  const uint32_t a_base = base;
  const uint32_t b_base = base + C::STAGES * C::A_BYTES;
  const uint32_t bar_base = base + C::STAGES * C::STAGE_BYTES;
  const uint32_t drain_bar = bar_base + 8u * (2 * C::STAGES + 4);
  uint32_t* tmem_slot =
      reinterpret_cast<uint32_t*>(base_ptr + C::STAGES * C::STAGE_BYTES + 8 * C::NUM_BARS);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
#define FULL_BAR(s) (bar_base + 8u * static_cast<uint32_t>(s))
#define EMPTY_BAR(s) (bar_base + 8u * static_cast<uint32_t>(C::STAGES + (s)))
#define TFULL_BAR(a) (bar_base + 8u * static_cast<uint32_t>(2 * C::STAGES + (a)))
#define TEMPTY_BAR(a) (bar_base + 8u * static_cast<uint32_t>(2 * C::STAGES + 2 + (a)))

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(FULL_BAR(s), 1);
      mbar_init(EMPTY_BAR(s), 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(TFULL_BAR(a), 1);
      mbar_init(TEMPTY_BAR(a), 4);
    }
    mbar_init(drain_bar, 1);
    *abort_flag = 0;
    mbar_fence_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&mapP);
    tma_prefetch_desc(&mapQ);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int64_t polls = prm.wait_polls;
  int64_t producer_issued = 0;  // TMA stage loads issued (warp 0)
  // the next kernel (launched as a programmatic dependent: the stream-K
  // fix-up, or the caller's next call) may be scheduled now; it waits for
  // this grid's completion before its own reads.  This grid was launched the
  // same way: everything above touched only its own shared and tensor
  // memory, and nothing below reads or writes global memory before the
  // previous grid has completed
  if (threadIdx.x == 0) asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  if (prm.swap && threadIdx.x == 0) {
    // decode tiles: while the previous grid finishes, pull the first weight
    // blocks of this CTA's range into L2 (a prefetch only: the loads below
    // still come after the wait and see whatever that grid wrote)
    Work wk;
    work_init(prm, wk);
    int pb, qb, kb0, kb1, split, slot, n = 0;
    while (n < kPrefetchBlocks && work_next(prm, wk, pb, qb, kb0, kb1, split, slot))
      for (int kb = kb0; kb < kb1 && n < kPrefetchBlocks; ++kb, ++n)
        tma_prefetch_l2_2d(&mapP, kb * BK, pb * BM);
  }
  asm volatile("griddepcontrol.wait;" ::: "memory");

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    int stage = 0;
    uint32_t phase = 0;
    int64_t issued = 0;
    bool ok = true;
    Work wk;
    work_init(prm, wk);
    int pb, qb, kb0, kb1, split, slot;
    while (ok && work_next(prm, wk, pb, qb, kb0, kb1, split, slot)) {
      for (int kb = kb0; kb < kb1; ++kb) {
        bool w = false;
        if (lane == 0) w = wait_phase(EMPTY_BAR(stage), phase ^ 1u, polls, abort_flag);
        w = __shfl_sync(0xffffffffu, w, 0);
        if (!w) {
          if (lane == 0) fail(prm.error_word, abort_flag);
          ok = false;
          break;
        }
        if (lane == 0) {
          mbar_arrive_expect_tx(FULL_BAR(stage), C::STAGE_BYTES);
          tma_load_2d(a_base + stage * C::A_BYTES, &mapP, FULL_BAR(stage), kb * BK, pb * BM);
          tma_load_2d(b_base + stage * C::B_BYTES, &mapQ, FULL_BAR(stage), kb * BK, qb * BN);
        }
        ++issued;
        if (++stage == C::STAGES) {
          stage = 0;
          phase ^= 1u;
        }
      }
    }
    producer_issued = issued;
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    constexpr uint32_t kIdesc = kF8 ? idesc_f8(BM, BN) : idesc_i8(BM, BN);
    int stage = 0;
    uint32_t phase = 0;
    int acc = 0;
    uint32_t acc_phase = 0;
    bool ok = true;
    Work wk;
    work_init(prm, wk);
    int pb, qb, kb0, kb1, split, slot;
    while (ok && work_next(prm, wk, pb, qb, kb0, kb1, split, slot)) {
      if (sched_sync(false)) {  // the scheduler saw this accumulator free (or gave up)
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * BN);
      for (int kb = kb0; kb < kb1; ++kb) {
        if (sched_sync(false)) {  // the scheduler saw this stage land (or gave up)
          ok = false;
          break;
        }
        tc_fence_after();
        if (lane == 0) {
          const uint32_t sa = a_base + stage * C::A_BYTES;
          const uint32_t sb = b_base + stage * C::B_BYTES;
#pragma unroll
          for (int kk = 0; kk < BK / UMMA_K; ++kk) {
            if constexpr (kF8)
              mma_f8(d_tmem, smem_desc_k_sw128(sa + kk * UMMA_K),
                     smem_desc_k_sw128(sb + kk * UMMA_K), kIdesc, (kb > kb0 || kk > 0) ? 1u : 0u);
            else
              mma_i8(d_tmem, smem_desc_k_sw128(sa + kk * UMMA_K),
                     smem_desc_k_sw128(sb + kk * UMMA_K), kIdesc, (kb > kb0 || kk > 0) ? 1u : 0u);
          }
          mma_commit(EMPTY_BAR(stage));
        }
        __syncwarp();
        if (++stage == C::STAGES) {
          stage = 0;
          phase ^= 1u;
        }
      }
      if (!ok) break;
      if (lane == 0) mma_commit(TFULL_BAR(acc));
      __syncwarp();
      acc ^= 1;
      if (acc == 0) acc_phase ^= 1u;
    }
    if (lane == 0) {
      // every MMA issued by this thread completes before tensor memory is freed
      mma_commit(drain_bar);
      wait_phase(drain_bar, 0, 0, nullptr);
    }
    __syncwarp();
  } else if (warp == kSchedWarp) {
    // ------------------------------------------------------------ MMA scheduler
    // the issuer's waits, in the issuer's order, one named-barrier handoff each
    int stage = 0;
    uint32_t phase = 0;
    int acc = 0;
    uint32_t acc_phase = 0;
    Work wk;
    work_init(prm, wk);
    int pb, qb, kb0, kb1, split, slot;
    bool ok = true;
    while (ok && work_next(prm, wk, pb, qb, kb0, kb1, split, slot)) {
      bool w = false;
      if (lane == 0) w = wait_phase(TEMPTY_BAR(acc), acc_phase ^ 1u, polls, abort_flag);
      w = __shfl_sync(0xffffffffu, w, 0);
      if (!w && lane == 0) fail(prm.error_word, abort_flag);
      if (sched_sync(!w)) {
        ok = false;
        break;
      }
      for (int kb = kb0; kb < kb1; ++kb) {
        w = false;
        if (lane == 0) w = wait_phase(FULL_BAR(stage), phase, polls, abort_flag);
        w = __shfl_sync(0xffffffffu, w, 0);
        if (!w && lane == 0) fail(prm.error_word, abort_flag);
        if (sched_sync(!w)) {
          ok = false;
          break;
        }
        if (++stage == C::STAGES) {
          stage = 0;
          phase ^= 1u;
        }
      }
      acc ^= 1;
      if (acc == 0) acc_phase ^= 1u;
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int quarter = warp & 3;  // tensor-memory lanes this warp may access
    int acc = 0;
    uint32_t acc_phase = 0;
    Work wk;
    work_init(prm, wk);
    int pb, qb, kb0, kb1, split, slot;
    while (work_next(prm, wk, pb, qb, kb0, kb1, split, slot)) {
      bool w = false;
      if (lane == 0) w = wait_phase(TFULL_BAR(acc), acc_phase, polls, abort_flag);
      w = __shfl_sync(0xffffffffu, w, 0);
      if (!w) {
        if (lane == 0) fail(prm.error_word, abort_flag);
        break;
      }
      tc_fence_after();
      const int p = pb * BM + quarter * 32 + lane;
      float rmax = 0.0f;
#pragma unroll 1
      for (int c = 0; c < BN / C::CHUNK; ++c) {
        uint32_t r[32];
        __syncwarp();  // tcgen05.ld is .sync.aligned: the warp must be converged
        const uint32_t taddr = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) +
                               static_cast<uint32_t>(acc * BN + c * C::CHUNK);
        if constexpr (C::CHUNK == 32)
          tmem_ld_32x32b_x32(taddr, r);
        else
          tmem_ld_32x32b_x16(taddr, r);
        tmem_wait_ld();
        rmax = fmaxf(rmax,
                     store_chunk<C::CHUNK, kF8>(prm, r, p, qb * BN + c * C::CHUNK, split, slot));
      }
      if (prm.row_absmax && rmax > 0.0f && p < prm.P)
        atomicMax(reinterpret_cast<unsigned int*>(prm.row_absmax) + p, __float_as_uint(rmax));
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(TEMPTY_BAR(acc));
      acc ^= 1;
      if (acc == 0) acc_phase ^= 1u;
    }
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::TMEM_COLS);
  }
  if (warp == 0 && lane == 0 && *abort_flag) {
    // after an abort some issued TMA loads may not have been consumed: let
    // every one of them land before the CTA releases its shared memory
    for (int s = 0; s < C::STAGES; ++s) {
      const int64_t n = producer_issued / C::STAGES + (s < producer_issued % C::STAGES ? 1 : 0);
      if (n > 0) wait_phase(FULL_BAR(s), static_cast<uint32_t>((n - 1) & 1), 0, nullptr);
    }
  }
#undef FULL_BAR
#undef EMPTY_BAR
#undef TFULL_BAR
#undef TEMPTY_BAR
}

// ---------------------------------------------------------------------------
// 2-SM variant for prefill: a CTA pair computes a 256 x 256 tile with
// tcgen05.mma.cta_group::2.  Each CTA loads its own 128 rows of A and its own
// 128-row half of B (no multicast), so every SM pulls 32 KB of operands per
// 128-deep K step instead of 48 KB.  The leader CTA (rank 0) owns the
// operand-ready barriers (it expects the bytes of both CTAs; the peer's loads
// complete on the leader's barrier) and issues the MMAs; it signals both CTAs'
// stage-free and accumulator-ready barriers with one commit each; both CTAs'
// epilogue warps drain their own 128 accumulator rows and tell the leader.
// ---------------------------------------------------------------------------
// TN: the pair tile's N (Q-side) width, 256, 224 or 192; each CTA loads
// TN / 2 rows of B.  As many stages as fit 227 KB of shared memory (at most 8).
template <int TN>
struct PairCfg {
  static constexpr int ROWS = 128;             // rows of A per CTA
  static constexpr int TILE_M = 2 * ROWS;      // P side of the pair tile
  static constexpr int B_ROWS = TN / 2;        // rows of B per CTA
  static constexpr int A_BYTES = ROWS * BK;
  static constexpr int B_BYTES = B_ROWS * BK;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;  // per CTA
  static constexpr int STAGES_FIT = (227 * 1024 - 1024 - 256) / STAGE_BYTES;
  static constexpr int STAGES = STAGES_FIT < 8 ? STAGES_FIT : 8;
  static constexpr int TMEM_COLS = 512;        // 2 accumulators x TN INT32 columns
  static constexpr int NUM_BARS = 2 * STAGES + 5;
  static constexpr int SMEM_BYTES = 1024 + STAGES * STAGE_BYTES + 8 * NUM_BARS + 16;
  static_assert(TN % 32 == 0 && TN >= 64 && TN <= 256, "pair tile width");
  static_assert(B_BYTES % 1024 == 0, "swizzle atoms need 1024-byte aligned stages");
  static_assert(SMEM_BYTES <= 227 * 1024, "shared memory");
};

__device__ __forceinline__ void mbar_complete_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.complete_tx.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}

// Stage loads issued to stage s after `total` loads round-robin over STAGES.
__device__ __forceinline__ int64_t loads_on_stage(int64_t total, int s, int stages) {
  return total / stages + (s < total % stages ? 1 : 0);
}

template <int TN, bool kF8>
__global__ void __launch_bounds__(kThreads, 1)
    w8a8_gemm_pair_kernel(const __grid_constant__ CUtensorMap mapP,
                          const __grid_constant__ CUtensorMap mapQ, const Params prm) {
  using C = PairCfg<TN>;
  constexpr int ROWS = C::ROWS, TILE_M = C::TILE_M, B_ROWS = C::B_ROWS;
  constexpr int A_BYTES = C::A_BYTES, B_BYTES = C::B_BYTES, STAGE_BYTES = C::STAGE_BYTES;
  constexpr int STAGES = C::STAGES, TMEM_COLS = C::TMEM_COLS, NUM_BARS = C::NUM_BARS;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_u32 = smem_u32(smem_raw);
  const uint32_t base = (raw_u32 + 1023u) & ~1023u;
  uint8_t* base_ptr = smem_raw + (base - raw_u32);
  const uint32_t a_base = base;
  const uint32_t b_base = base + STAGES * A_BYTES;
  const uint32_t bar_base = base + STAGES * STAGE_BYTES;
  const uint32_t drain_bar = bar_base + 8u * (2 * STAGES + 4);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(base_ptr + STAGES * STAGE_BYTES + 8 * NUM_BARS);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  volatile int64_t* peer_issued_slot = reinterpret_cast<volatile int64_t*>(tmem_slot + 2);
#define FULL_BAR(s) (bar_base + 8u * static_cast<uint32_t>(s))
#define EMPTY_BAR(s) (bar_base + 8u * static_cast<uint32_t>(STAGES + (s)))
#define TFULL_BAR(a) (bar_base + 8u * static_cast<uint32_t>(2 * STAGES + (a)))
#define TEMPTY_BAR(a) (bar_base + 8u * static_cast<uint32_t>(2 * STAGES + 2 + (a)))

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int pair_id = static_cast<int>(blockIdx.x >> 1);
  const int num_pairs = static_cast<int>(gridDim.x >> 1);

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(FULL_BAR(s), 1);
      mbar_init(EMPTY_BAR(s), 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(TFULL_BAR(a), 1);
      mbar_init(TEMPTY_BAR(a), 8);  // 4 epilogue warps in each CTA of the pair
    }
    mbar_init(drain_bar, 1);
    *abort_flag = 0;
    *peer_issued_slot = 0;
    mbar_fence_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&mapP);
    tma_prefetch_desc(&mapQ);
  }
  if (warp == 1) {
    tmem_alloc_pair(smem_u32(tmem_slot), TMEM_COLS);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // both CTAs' barriers exist before any cross-CTA signal
  tc_fence_after();
  // programmatic launch: let the next kernel be scheduled, then wait for the
  // previous grid before any global-memory access (above: shared and tensor
  // memory only)
  if (threadIdx.x == 0) asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const uint32_t tmem_base = *tmem_slot;
  const int64_t polls = prm.wait_polls;
  // the partner's abort flag, so a failing CTA stops its partner quickly
  const uint32_t partner_abort = map_to_cta(smem_u32(const_cast<int*>(abort_flag)), rank ^ 1u);
  int64_t producer_issued = 0;

  auto fail_pair = [&]() {
    fail(prm.error_word, abort_flag);
    st_cluster_u32(partner_abort, 1u);
  };

  if (warp == 0) {
    // ------------------------------------------------------------ producer (both CTAs)
    int stage = 0;
    uint32_t phase = 0;
    int64_t issued = 0;
    bool ok = true;
    for (int u = pair_id; u < prm.units && ok; u += num_pairs) {
      int pb, qb, kb0, kb1, split;
      decode_unit(prm, u, pb, qb, kb0, kb1, split);
      for (int kb = kb0; kb < kb1; ++kb) {
        bool w = false;
        if (lane == 0) w = wait_phase(EMPTY_BAR(stage), phase ^ 1u, polls, abort_flag);
        w = __shfl_sync(0xffffffffu, w, 0);
        if (!w) {
          if (lane == 0) fail_pair();
          ok = false;
          break;
        }
        if (lane == 0) {
          const uint32_t fb = leader ? FULL_BAR(stage) : map_to_cta(FULL_BAR(stage), 0);
          if (leader) mbar_arrive_expect_tx(FULL_BAR(stage), 2 * STAGE_BYTES);
          tma_load_2d_pair(a_base + stage * A_BYTES, &mapP, fb, kb * BK,
                           pb * TILE_M + static_cast<int>(rank) * ROWS);
          tma_load_2d_pair(b_base + stage * B_BYTES, &mapQ, fb, kb * BK,
                           qb * TN + static_cast<int>(rank) * B_ROWS);
        }
        ++issued;
        if (++stage == STAGES) {
          stage = 0;
          phase ^= 1u;
        }
      }
    }
    producer_issued = issued;
    if (lane == 0 && !leader)  // the leader needs the peer's count to drain after an abort
      st_cluster_u32(map_to_cta(smem_u32(const_cast<int64_t*>(peer_issued_slot)), 0),
                     static_cast<uint32_t>(issued));
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (leader only)
    if (leader) {
      constexpr uint32_t kIdesc = kF8 ? idesc_f8(TILE_M, TN) : idesc_i8(TILE_M, TN);
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      for (int u = pair_id; u < prm.units && ok; u += num_pairs) {
        int pb, qb, kb0, kb1, split;
        decode_unit(prm, u, pb, qb, kb0, kb1, split);
        if (sched_sync(false)) {  // the scheduler saw this accumulator free (or gave up)
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * TN);
        for (int kb = kb0; kb < kb1; ++kb) {
          if (sched_sync(false)) {  // the scheduler saw both CTAs' stage land (or gave up)
            ok = false;
            break;
          }
          tc_fence_after();
          if (lane == 0) {
            const uint32_t sa = a_base + stage * A_BYTES;
            const uint32_t sb = b_base + stage * B_BYTES;
#pragma unroll
            for (int kk = 0; kk < BK / UMMA_K; ++kk) {
              if constexpr (kF8)
                mma_f8_pair(d_tmem, smem_desc_k_sw128(sa + kk * UMMA_K),
                            smem_desc_k_sw128(sb + kk * UMMA_K), kIdesc,
                            (kb > kb0 || kk > 0) ? 1u : 0u);
              else
                mma_i8_pair(d_tmem, smem_desc_k_sw128(sa + kk * UMMA_K),
                            smem_desc_k_sw128(sb + kk * UMMA_K), kIdesc,
                            (kb > kb0 || kk > 0) ? 1u : 0u);
            }
            // the stage is free in both CTAs once these MMAs have read it
            mma_commit_pair(EMPTY_BAR(stage));
            mma_commit_pair(map_to_cta(EMPTY_BAR(stage), 1));
          }
          __syncwarp();
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        if (lane == 0) {
          mma_commit_pair(TFULL_BAR(acc));
          mma_commit_pair(map_to_cta(TFULL_BAR(acc), 1));
        }
        __syncwarp();
        acc ^= 1;
        if (acc == 0) acc_phase ^= 1u;
      }
      if (lane == 0) {
        mma_commit_pair(drain_bar);
        wait_phase(drain_bar, 0, 0, nullptr);
      }
      __syncwarp();
    }
  } else if (warp == kSchedWarp) {
    // ------------------------------------------------------------ MMA scheduler (leader only)
    if (leader) {
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      for (int u = pair_id; u < prm.units && ok; u += num_pairs) {
        int pb, qb, kb0, kb1, split;
        decode_unit(prm, u, pb, qb, kb0, kb1, split);
        bool w = false;
        if (lane == 0) w = wait_phase(TEMPTY_BAR(acc), acc_phase ^ 1u, polls, abort_flag);
        w = __shfl_sync(0xffffffffu, w, 0);
        if (!w && lane == 0) fail_pair();
        if (sched_sync(!w)) {
          ok = false;
          break;
        }
        for (int kb = kb0; kb < kb1; ++kb) {
          w = false;
          if (lane == 0) w = wait_phase(FULL_BAR(stage), phase, polls, abort_flag);
          w = __shfl_sync(0xffffffffu, w, 0);
          if (!w && lane == 0) fail_pair();
          if (sched_sync(!w)) {
            ok = false;
            break;
          }
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        acc ^= 1;
        if (acc == 0) acc_phase ^= 1u;
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue (both CTAs)
    const int quarter = warp & 3;
    int acc = 0;
    uint32_t acc_phase = 0;
    const uint32_t leader_tempty0 = leader ? TEMPTY_BAR(0) : map_to_cta(TEMPTY_BAR(0), 0);
    const uint32_t leader_tempty1 = leader ? TEMPTY_BAR(1) : map_to_cta(TEMPTY_BAR(1), 0);
    for (int u = pair_id; u < prm.units; u += num_pairs) {
      int pb, qb, kb0, kb1, split;
      decode_unit(prm, u, pb, qb, kb0, kb1, split);
      // the row's token scale, fetched before the accumulator is ready
      const int p_row = pb * TILE_M + static_cast<int>(rank) * ROWS + quarter * 32 + lane;
      const float xs = (prm.epi != SQ_EPI_I32_RAW && prm.epi != SQ_EPI_F32_RAW && p_row < prm.P)
                           ? __ldg(prm.p_scale + p_row) : 0.0f;
      bool w = false;
      if (lane == 0) w = wait_phase(TFULL_BAR(acc), acc_phase, polls, abort_flag);
      w = __shfl_sync(0xffffffffu, w, 0);
      if (!w) {
        if (lane == 0) fail_pair();
        break;
      }
      tc_fence_after();
      const int p = pb * TILE_M + static_cast<int>(rank) * ROWS + quarter * 32 + lane;
      float rmax = 0.0f;
      const uint32_t trow = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) +
                            static_cast<uint32_t>(acc * TN);
      if (prm.epi == SQ_EPI_I32_RAW || prm.epi == SQ_EPI_F32_RAW) {
#pragma unroll 1
        for (int c = 0; c < TN / 32; ++c) {
          uint32_t r[32];
          __syncwarp();
          tmem_ld_32x32b_x32(trow + static_cast<uint32_t>(c * 32), r);
          tmem_wait_ld();
          store_chunk<32, kF8>(prm, r, p, qb * TN + c * 32, 0, -1);
        }
      } else {
        // software-pipelined: chunk c + 1's accumulator load (tensor memory)
        // and channel scales (L2) are in flight while chunk c is converted
        // and stored; the token scale was loaded before the accumulator wait
        uint32_t ra[32], rb[32];
        float wa[32], wb[32];
        const bool row_in = p < prm.P;
        __syncwarp();
        tmem_ld_32x32b_x32(trow, ra);
        load_col_scales<32>(prm, qb * TN, wa);
        tmem_wait_ld();
        constexpr int kChunks = TN / 32;  // odd for TN = 224: the last pair is one chunk
#pragma unroll 1
        for (int c = 0; c < kChunks; c += 2) {
          const bool two = c + 1 < kChunks;
          if (two) {
            __syncwarp();
            tmem_ld_32x32b_x32(trow + static_cast<uint32_t>((c + 1) * 32), rb);
            load_col_scales<32>(prm, qb * TN + (c + 1) * 32, wb);
          }
          if (row_in) rmax = fmaxf(rmax, epi_row_bf16<32, kF8>(prm, ra, p, qb * TN + c * 32, xs, wa));
          if (two) tmem_wait_ld();
          if (c + 2 < kChunks) {
            __syncwarp();
            tmem_ld_32x32b_x32(trow + static_cast<uint32_t>((c + 2) * 32), ra);
            load_col_scales<32>(prm, qb * TN + (c + 2) * 32, wa);
          }
          if (two && row_in)
            rmax = fmaxf(rmax, epi_row_bf16<32, kF8>(prm, rb, p, qb * TN + (c + 1) * 32, xs, wb));
          if (c + 2 < kChunks) tmem_wait_ld();
        }
      }
      if (prm.row_absmax && rmax > 0.0f && p < prm.P)
        atomicMax(reinterpret_cast<unsigned int*>(prm.row_absmax) + p, __float_as_uint(rmax));
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        const uint32_t t = acc ? leader_tempty1 : leader_tempty0;
        if (leader)
          mbar_arrive(t);
        else
          mbar_arrive_cluster(t);
      }
      acc ^= 1;
      if (acc == 0) acc_phase ^= 1u;
    }
  }
  __syncthreads();
  cluster_sync_all();  // no MMA, TMA signal or remote arrive of this tile loop is pending
  if (warp == 0 && lane == 0 && leader && *abort_flag) {
    // after an abort, every stage load either CTA issued lands before either
    // CTA releases its shared memory (the peer's loads complete on the
    // leader's barriers; the two producers are at most one round apart)
    const int64_t peer_issued = *peer_issued_slot;
    for (int s = 0; s < STAGES; ++s) {
      const int64_t nl = loads_on_stage(producer_issued, s, STAGES);
      const int64_t np = loads_on_stage(peer_issued, s, STAGES);
      if (np > nl) mbar_arrive_expect_tx(FULL_BAR(s), STAGE_BYTES);  // the missing leader arrival
      else if (nl > np) mbar_complete_tx(FULL_BAR(s), STAGE_BYTES);  // peer bytes never sent
      const int64_t n = nl > np ? nl : np;
      if (n > 0) wait_phase(FULL_BAR(s), static_cast<uint32_t>((n - 1) & 1), 0, nullptr);
    }
  }
  cluster_sync_all();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, TMEM_COLS);
  }
#undef FULL_BAR
#undef EMPTY_BAR
#undef TFULL_BAR
#undef TEMPTY_BAR
}

// Stream-K fix-up for decode tiles (weight rows on the P side, tokens on the
// Q side, one Q block).  Block (b, y) looks at the start of CTA c = b + 1: if
// that iteration lies inside a tile and no earlier CTA starts inside the same
// tile, the block sums the tile's partial slots (CTA c - 1 up to the last CTA
// starting before the tile ends) for tokens q = y * kFixQ ... and applies the
// epilogue; thread = row of the tile's 128 P rows, so every load and store is
// 128 consecutive words.  INT32 addition is exact, so the result equals the
// unsplit accumulation.  FP8 partials are fp32: they are added in ascending
// CTA order, one rounding per contributor after the first, the same order on
// every run.
constexpr int kFixQ = 8;  // tokens per fix-up block

template <bool kF8>
__global__ void __launch_bounds__(BM) streamk_fixup_kernel(const Params prm, int G) {
  // launched as a programmatic dependent of the main kernel: everything that
  // grid wrote is visible once this returns
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int c = static_cast<int>(blockIdx.x) + 1;
  const int64_t kbt = prm.k_blocks;
  const int64_t b = static_cast<int64_t>(c) * prm.sk_iters / G;
  if (b % kbt == 0) return;
  const int64_t tile = b / kbt;
  const int64_t t0 = tile * kbt, t1 = t0 + kbt;
  if (static_cast<int64_t>(c - 1) * prm.sk_iters / G > t0) return;  // not the first boundary
  int pb, qb;
  tile_coords(prm, static_cast<int>(tile), pb, qb);
  const int pl = static_cast<int>(threadIdx.x);
  const int p = pb * BM + pl;
  if (p >= prm.P) return;
  const int q0 = static_cast<int>(blockIdx.y) * kFixQ;
  const int nq = min(kFixQ, prm.Q - q0);
  int32_t acc[kFixQ];  // INT32 sums, or the fp32 sums' bits
#pragma unroll
  for (int j = 0; j < kFixQ; ++j) acc[j] = 0;
  for (int cc = c - 1; cc < G; ++cc) {
    const int64_t sc = static_cast<int64_t>(cc) * prm.sk_iters / G;
    if (sc >= t1) break;
    const int64_t slot = (sc / kbt == tile) ? 2 * cc : 2 * cc + 1;
    const int32_t* src = prm.sk_partial + (slot * prm.Q + q0) * BM + pl;
    // predicated, not a loop exit: the loads of all kFixQ tokens issue together
#pragma unroll
    for (int j = 0; j < kFixQ; ++j) {
      if (j < nq) {
        const int32_t v = __ldcg(src + j * BM);
        if constexpr (kF8)
          acc[j] = cc == c - 1
                       ? v
                       : __float_as_int(__fadd_rn(__int_as_float(acc[j]), __int_as_float(v)));
        else
          acc[j] += v;
      }
    }
  }
  const float ws =
      (prm.epi == SQ_EPI_I32_RAW || prm.epi == SQ_EPI_F32_RAW) ? 0.0f : __ldg(prm.p_scale + p);
#pragma unroll
  for (int j = 0; j < kFixQ; ++j) {
    if (j >= nq) break;
    const int64_t o = static_cast<int64_t>(q0 + j) * prm.ldo + p;
    if (prm.epi == SQ_EPI_I32_RAW || prm.epi == SQ_EPI_F32_RAW) {
      static_cast<int32_t*>(prm.out)[o] = acc[j];  // the accumulator's bits
    } else {
      const float a = kF8 ? __int_as_float(acc[j]) : __int2float_rn(acc[j]);
      float t = __fmul_rn(__fmul_rn(a, __ldg(prm.q_scale + q0 + j)), ws);
      if (prm.epi == SQ_EPI_BF16_RELU) t = t > 0.0f ? t : 0.0f;
      static_cast<__nv_bfloat16*>(prm.out)[o] = __float2bfloat16_rn(t);
    }
  }
}

// out[m][n] = epilogue(sum_s partial[s][m][n]) (slices of lda * M words,
// rows of stride lda); INT32 addition is exact, so the split does not change
// the result.  With one slice it is the epilogue of a given accumulator.
__global__ void splitk_reduce_kernel(const int32_t* __restrict__ partial, int splits, int64_t M,
                                     int64_t N, int64_t lda, const float* __restrict__ x_scale,
                                     const float* __restrict__ w_scale, int epi, void* out,
                                     int64_t ldo) {
  const int64_t total = M * N, slice = M * lda;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t m = i / N, n = i - m * N;
    int32_t acc = 0;
    for (int s = 0; s < splits; ++s) acc += partial[s * slice + m * lda + n];
    if (epi == SQ_EPI_I32_RAW) {
      static_cast<int32_t*>(out)[m * ldo + n] = acc;
    } else {
      float t = __fmul_rn(__fmul_rn(__int2float_rn(acc), x_scale[m]), w_scale[n]);
      if (epi == SQ_EPI_BF16_RELU) t = t > 0.0f ? t : 0.0f;
      static_cast<__nv_bfloat16*>(out)[m * ldo + n] = __float2bfloat16_rn(t);
    }
  }
}

// --------------------------------------------------------------------------
// host side
// --------------------------------------------------------------------------
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// K-major INT8 matrix [rows, K] (row pitch K bytes), box = box_rows x 128
// bytes, 128-byte swizzle, zero fill outside the matrix.
bool make_map(CUtensorMap* map, const int8_t* ptr, int64_t rows, int64_t K, int box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(rows)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(K)};
  const cuuint32_t box[2] = {static_cast<cuuint32_t>(BK), static_cast<cuuint32_t>(box_rows)};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2,
                        const_cast<void*>(static_cast<const void*>(ptr)), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

template <int BN, bool kF8>
cudaError_t launch_bn(const Params& prm, const CUtensorMap& mp, const CUtensorMap& mq, int grid,
                      cudaStream_t st) {
  using C = Cfg<BN>;
  cudaError_t e = launch_cache().ensure_smem(
      reinterpret_cast<const void*>(w8a8_gemm_kernel<BN, kF8>), C::SMEM_BYTES);
  if (e != cudaSuccess) return e;
  // a programmatic dependent of the previous kernel in the stream: its CTAs
  // set up their barriers and tensor memory while that kernel finishes
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(grid));
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = C::SMEM_BYTES;
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, w8a8_gemm_kernel<BN, kF8>, mp, mq, prm);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

template <int TN, bool kF8>
cudaError_t launch_pair(const Params& prm, const CUtensorMap& mp, const CUtensorMap& mq,
                        int max_pairs, cudaStream_t st) {
  using C = PairCfg<TN>;
  auto kern = w8a8_gemm_pair_kernel<TN, kF8>;
  cudaError_t e = launch_cache().ensure_smem(reinterpret_cast<const void*>(kern), C::SMEM_BYTES);
  if (e != cudaSuccess) return e;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  // a programmatic dependent of the previous kernel in the stream
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = C::SMEM_BYTES;
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  // as many co-resident CTA pairs as the device holds (one per SM pair)
  static int max_clusters[64] = {};  // per instantiation
  const int dev = LaunchCache::device();
  if (dev >= 0 && dev < 64 && max_clusters[dev] == 0) {
    cfg.gridDim = dim3(2 * max_pairs);
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess || n <= 0) n = max_pairs;
    max_clusters[dev] = n;
  }
  int pairs = (dev >= 0 && dev < 64) ? max_clusters[dev] : max_pairs;
  if (pairs > max_pairs) pairs = max_pairs;
  if (pairs > prm.units) pairs = prm.units;
  cfg.gridDim = dim3(2 * pairs);
  e = cudaLaunchKernelEx(&cfg, kern, mp, mq, prm);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

int bn_for_tokens(int64_t M) {
  return M <= 16 ? 16 : M <= 32 ? 32 : M <= 64 ? 64 : M <= 128 ? 128 : 256;
}

}  // namespace

int num_sms_current_device() { return launch_cache().sms(); }

GemmPlan plan_gemm(int64_t M, int64_t N, int64_t K, int path_hint, int split_k, int num_sms) {
  GemmPlan p{};
  const int64_t kblocks = (K + BK - 1) / BK;
  p.swap = (path_hint == 2 || (path_hint == 0 && M <= 128)) ? 1 : 0;
  p.pair = 0;
  if (!p.swap) {
    p.bn = 256;
    p.splits = 1;
    p.pair = path_hint == 3 ? 0 : 1;
    if (p.pair) {
      // pair tile width: rounds of tiles over the SM pairs times the time of
      // a tile's 128-deep K step, which operand delivery sets rather than the
      // MMA (measured 600 and 640 cycles per step at widths 192 and 256, the
      // MMA alone taking 384 and 512): step ~ 480 + 0.625 TN cycles, in
      // units of 1/1.6 cycle 768 + TN
      const int64_t pairs = (num_sms > 0 ? num_sms : 148) / 2;
      const int64_t p_blocks = (M + 255) / 256;
      int64_t best = -1;
      for (int tn : {256, 224, 192}) {
        const int64_t tiles = p_blocks * ((N + tn - 1) / tn);
        const int64_t cost = ((tiles + pairs - 1) / pairs) * (768 + tn);
        if (best < 0 || cost < best) {
          best = cost;
          p.bn = tn;
        }
      }
    }
  } else if (split_k <= 0) {
    // decode tiles, stream-K: every SM streams the same number of k-blocks
    p.bn = bn_for_tokens(M);
    const int64_t tiles = (N + BM - 1) / BM;
    const int64_t iters = tiles * kblocks;
    const int64_t sms = num_sms > 0 ? num_sms : 148;
    const int64_t G = iters < sms ? iters : sms;
    p.splits = 1;
    p.streamk = 1;
    p.grid = static_cast<int>(G);
    p.sk_iters = iters;
    bool split_tiles = false;
    for (int64_t c = 1; c < G && !split_tiles; ++c) split_tiles = (c * iters / G) % kblocks != 0;
    p.workspace_bytes = split_tiles ? static_cast<size_t>(2 * G) * BM * static_cast<size_t>(M) * 4u
                                    : 0u;
    return p;
  } else {
    p.bn = bn_for_tokens(M);
    const int64_t tiles = (N + BM - 1) / BM;
    int splits = split_k;
    if (splits <= 0) {
      // pick the split that best fills the SMs, keeping the INT32 partial
      // traffic (splits * M * N * 4 bytes) under a quarter of the weight bytes
      const int64_t sms = num_sms > 0 ? num_sms : 148;
      int64_t cap = K / (16 * (M > 0 ? M : 1));
      if (cap > 8) cap = 8;
      if (cap > kblocks) cap = kblocks;
      if (cap < 1) cap = 1;
      double best = -1.0;
      splits = 1;
      for (int64_t s = 1; s <= cap; ++s) {
        const int64_t units = tiles * s;
        const int64_t waves = (units + sms - 1) / sms;
        const double eff = static_cast<double>(units) / static_cast<double>(waves * sms);
        if (eff > best + 0.02) {
          best = eff;
          splits = static_cast<int>(s);
        }
      }
    }
    if (splits > kblocks) splits = static_cast<int>(kblocks > 0 ? kblocks : 1);
    p.splits = splits < 1 ? 1 : splits;
  }
  p.workspace_bytes =
      p.splits > 1 ? static_cast<size_t>(p.splits) * static_cast<size_t>(M) * static_cast<size_t>(N) * 4u
                   : 0u;
  return p;
}

cudaError_t launch_gemm(const GemmPlan& plan, const int8_t* Xq, const int8_t* Wq,
                        const float* x_scale, const float* w_scale, int64_t M, int64_t N,
                        int64_t K, int epi, void* out, int64_t ldo, void* workspace, int num_sms,
                        int64_t wait_polls, int* error_word, cudaStream_t st,
                        float* row_absmax, bool fp8) {
  if (M == 0 || N == 0) return cudaSuccess;
  // FP8 accumulators are fp32: stream-K partials are added in a fixed order
  // by the fix-up; no explicit split-K, no INT32 epilogue
  if (fp8 && (plan.splits > 1 || epi == SQ_EPI_I32_RAW)) return cudaErrorInvalidValue;
  if (!fp8 && epi == SQ_EPI_F32_RAW) return cudaErrorInvalidValue;
  Params prm{};
  const int8_t* Pptr = plan.swap ? Wq : Xq;
  const int8_t* Qptr = plan.swap ? Xq : Wq;
  prm.P = static_cast<int>(plan.swap ? N : M);
  prm.Q = static_cast<int>(plan.swap ? M : N);
  prm.K = static_cast<int>(K);
  const int p_tile = plan.pair ? 256 : BM;
  prm.p_blocks = (prm.P + p_tile - 1) / p_tile;
  prm.q_blocks = (prm.Q + plan.bn - 1) / plan.bn;
  prm.k_blocks = static_cast<int>((K + BK - 1) / BK);
  prm.splits = plan.splits;
  prm.group = plan.swap ? 1 : 16;
  prm.units = prm.p_blocks * prm.q_blocks * prm.splits;
  prm.p_scale = plan.swap ? w_scale : x_scale;
  prm.q_scale = plan.swap ? x_scale : w_scale;
  prm.out = out;
  prm.ldo = ldo;
  prm.epi = epi;
  prm.swap = plan.swap;
  prm.partial = plan.splits > 1 ? static_cast<int32_t*>(workspace) : nullptr;
  prm.streamk = plan.streamk;
  prm.sk_iters = plan.sk_iters;
  prm.sk_partial = plan.streamk ? static_cast<int32_t*>(workspace) : nullptr;
  if (row_absmax && (plan.swap || epi == SQ_EPI_I32_RAW || epi == SQ_EPI_F32_RAW))
    return cudaErrorInvalidValue;
  prm.row_absmax = row_absmax;
  prm.wait_polls = wait_polls;
  prm.error_word = error_word;
  {
    const int64_t esz = (epi == SQ_EPI_I32_RAW || epi == SQ_EPI_F32_RAW) ? 4 : 2;
    prm.vec_out = ((reinterpret_cast<uintptr_t>(out) & 15u) == 0 && (ldo * esz) % 16 == 0) ? 1 : 0;
  }

  CUtensorMap mp, mq;
  if (K == 0) return cudaErrorInvalidValue;
  const int sms = num_sms > 0 ? num_sms : 148;
  if (plan.pair) {
    // each CTA of a pair loads 128 rows of A and 128 rows of B
    if (!make_map(&mp, Pptr, prm.P, K, 128) || !make_map(&mq, Qptr, prm.Q, K, plan.bn / 2))
      return cudaErrorInvalidValue;
    switch (plan.bn * 2 + (fp8 ? 1 : 0)) {
      case 512: return launch_pair<256, false>(prm, mp, mq, sms / 2, st);
      case 448: return launch_pair<224, false>(prm, mp, mq, sms / 2, st);
      case 384: return launch_pair<192, false>(prm, mp, mq, sms / 2, st);
      case 513: return launch_pair<256, true>(prm, mp, mq, sms / 2, st);
      case 449: return launch_pair<224, true>(prm, mp, mq, sms / 2, st);
      case 385: return launch_pair<192, true>(prm, mp, mq, sms / 2, st);
      default: return cudaErrorInvalidValue;
    }
  }
  if (!make_map(&mp, Pptr, prm.P, K, BM) || !make_map(&mq, Qptr, prm.Q, K, plan.bn))
    return cudaErrorInvalidValue;
  const int grid = plan.streamk ? plan.grid : (prm.units < sms ? prm.units : sms);
  cudaError_t e;
  if (fp8) {
    switch (plan.bn) {
      case 16: e = launch_bn<16, true>(prm, mp, mq, grid, st); break;
      case 32: e = launch_bn<32, true>(prm, mp, mq, grid, st); break;
      case 64: e = launch_bn<64, true>(prm, mp, mq, grid, st); break;
      case 128: e = launch_bn<128, true>(prm, mp, mq, grid, st); break;
      case 256: e = launch_bn<256, true>(prm, mp, mq, grid, st); break;
      default: return cudaErrorInvalidValue;
    }
  } else {
    switch (plan.bn) {
      case 16: e = launch_bn<16, false>(prm, mp, mq, grid, st); break;
      case 32: e = launch_bn<32, false>(prm, mp, mq, grid, st); break;
      case 64: e = launch_bn<64, false>(prm, mp, mq, grid, st); break;
      case 128: e = launch_bn<128, false>(prm, mp, mq, grid, st); break;
      case 256: e = launch_bn<256, false>(prm, mp, mq, grid, st); break;
      default: return cudaErrorInvalidValue;
    }
  }
  if (e != cudaSuccess) return e;
  if (plan.streamk) {
    if (plan.workspace_bytes == 0 || plan.grid < 2) return cudaSuccess;
    const dim3 fgrid(static_cast<unsigned>(plan.grid - 1),
                     static_cast<unsigned>((prm.Q + kFixQ - 1) / kFixQ));
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = fgrid;
    cfg.blockDim = dim3(BM);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = st;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t fe = fp8 ? cudaLaunchKernelEx(&cfg, streamk_fixup_kernel<true>, prm, plan.grid)
                         : cudaLaunchKernelEx(&cfg, streamk_fixup_kernel<false>, prm, plan.grid);
    if (fe != cudaSuccess) return fe;
    return cudaGetLastError();
  }
  if (plan.splits <= 1) return e;
  const int64_t total = M * N;
  int blocks = static_cast<int>((total + 255) / 256);
  if (blocks > sms * 8) blocks = sms * 8;
  splitk_reduce_kernel<<<blocks, 256, 0, st>>>(static_cast<const int32_t*>(workspace), plan.splits,
                                               M, N, N, x_scale, w_scale, epi, out, ldo);
  return cudaGetLastError();
}

cudaError_t launch_dequant_i32(const int32_t* acc, int64_t M, int64_t N, int64_t lda,
                               const float* x_scale, const float* w_scale, int epi, void* out,
                               int64_t ldo, cudaStream_t st) {
  if (M == 0 || N == 0) return cudaSuccess;
  const int64_t total = M * N;
  int blocks = static_cast<int>((total + 255) / 256);
  const int cap = num_sms_current_device() * 8;
  if (blocks > cap) blocks = cap;
  splitk_reduce_kernel<<<blocks, 256, 0, st>>>(acc, 1, M, N, lda, x_scale, w_scale, epi, out, ldo);
  return cudaGetLastError();
}

}  // namespace sq
