// Grouped SwiGLU expert MLP on MXFP4 weights: block-scaled tcgen05 GEMMs.
//
// "Welcome GPT OSS ..." (summary), section 4: SwiGLU experts;
// "Tricks from OpenAI gpt-oss ..." (summary), sections 6 and 8: E2M1 weights
// with one shared scale per 32 elements, and GEMMs that read those blocks and
// scales directly; aitrends.kr talk summary, "Hardware optimisation": the
// weights stay 4-bit in memory and are raised to higher precision only for
// the arithmetic.
//
// The weights never leave their 4-bit form: the tensor core's block-scaled
// MMA (kind::mxf8f6f4) multiplies E2M1 codes by their E8M0 block scales
// itself.  Its other operand must be an 8-bit float, so every bf16
// activation a is split exactly into two E4M3 pieces under the exponent t of
// its 32-element block (t = floor(log2 max|a|) - 7, so |a| / 2^t < 256):
//     hi = RNE_e4m3(a / 2^t),   lo = 16 (a / 2^t - hi),
//     a  = hi * 2^t + lo * 2^(t-4).
// A bf16 value has 8 significant bits and hi keeps the leading 4, so the
// remainder has at most 4 and lo holds it exactly whenever a / 2^t >= 2^-6,
// i.e. for every element within 2^13 of its block's largest; smaller ones
// lose bits below 2^(t-13), under 2^-20 of the block maximum.  The products
// with the weights are then the exact products of the bf16 activations, as
// in a bf16 GEMM on decoded weights, and only the fp32 accumulation order
// differs from a sequential sum.
//
// MMA shape: M = 128 weight rows, N = 2 NT token piece rows (the hi and lo
// pieces of NT tokens, interleaved: piece row 2t = hi of token t, 2t + 1 =
// lo), K = 32.  The weights take the M side because the block-scaled MMA
// reads both operands from shared memory and M is fixed at 128: the token
// side then costs only its real rows, N x 32 bytes per MMA, and an MMA reads
// 4 KB of codes plus 1-4 KB of pieces.  The epilogue adds accumulator
// columns 2t and 2t + 1.
//   * gate/up: the 128 rows are 64 gate rows and the matching 64 up rows,
//     interleaved by the copy's box order (row 2j = gate j, 2j + 1 = up j), so
//     neighbouring lanes hold the two halves of SwiGLU.  The epilogue rounds
//     h to bf16 into a shared-memory tile [NT][64], then, one warp per
//     (token, 32-feature block), stores h to [S][F] when asked and splits it
//     into the pieces the down GEMM reads.
//   * down: 128 rows of the [D][F] matrix; output y_perm [S][D] bf16.
// Both GEMMs run in one persistent launch (one CTA per SM, two for 16-token
// tiles).  Its work items are (token tile, 128 weight rows) of the gate/up
// GEMM, then those of the down GEMM; the CTAs take them one at a time from a
// counter in the workspace, in index order, so an SM that finishes early
// takes the next item, whichever GEMM it belongs to, and the down GEMM starts
// on SMs the gate/up GEMM no longer fills.  A down item waits (bounded, on a
// per-tile count that each gate/up item raises with release semantics after
// its pieces of h are stored) until every gate/up item of its tile is done.
// Every gate/up item is taken before any down item and never waits on
// another CTA, so every such wait ends, however many CTAs are resident.
// Each CTA's copy ring (up to 12 stages of two 128-K windows each, so one
// barrier round trip covers 256 of K) runs on across items, the weight-scale
// block of an item is single- or double-buffered and the accumulator
// double-buffered, so one item's epilogue overlaps the next item's MMAs.
// Warp roles (14 warps):
//   warp 0      producer: takes the work items and posts each to the other
//               roles through a small queue in shared memory; per item the
//               weight-scale bytes and the token-scale
//               words (bulk copies), per 128-K window the weight codes (TMA,
//               8 KB of packed codes that land as the 16 KB one-byte-per-code
//               layout the MMA reads) and the token pieces (TMA, 2 NT x 128 B)
//   warp 1      tensor-memory owner and MMA issuer: 4 MMAs per window
//   warps 2-5   scale writers: per window they copy the weight scales and the
//               token scales (both from the item's auxiliary block) into the
//               stage slot's scale columns in tensor memory, every lane quarter
//               its own copy, and add their arrival to the stage's barrier, so
//               the MMA thread waits on one barrier per stage
//   warps 6-13  epilogue: two warps per lane quarter, one per half of the
//               tile's tokens
// When K is not a multiple of 128 the last window re-reads [K - 128, K) and
// issues only the MMAs over its new 32-element blocks.
// The token pieces sit in a tile-padded layout (tile t owns piece rows
// [2 t NT, 2 t NT + 2 NT)), so every copy of a tile's rows is aligned and
// whole.  Pieces of padding rows are never written here (their accumulator
// columns depend only on their own rows and scales, and are never read).
// Every wait is bounded (2 s); on expiry the kernel records MOE_ERR_TIMEOUT
// in the status word and unwinds: every role leaves its loop, the scale
// writers complete the stage arrivals they skipped (the producer's copy
// barrier also counts them), the producer waits for every copy it issued to
// land and the MMA thread's last commit for every MMA it issued, and only
// then is tensor memory freed and the CTA gone.
#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>

#include <atomic>

#include "common.cuh"
#include "mlp_plan.cuh"
#include "tc_sm100.cuh"

namespace moe {
namespace {

constexpr int BKS = 128;            // K elements per window (one 128-byte swizzle row of codes)
constexpr int WPS = 2;              // windows per pipeline stage
constexpr int BN = 128;             // weight rows per work item (MMA M)
constexpr int W_SMEM = BN * BKS;    // one byte per code in shared memory
constexpr int W_TX = BN * BKS / 2;  // bytes one window's weight copy reads
constexpr int kEpiWarps = 8;
constexpr int kThreads = 32 * (6 + kEpiWarps);
constexpr int kMaxStages = 12;      // copy ring depth limit (stage slot s also owns scale slot s)
constexpr int kSlotCols = 8 * WPS;  // per stage and window: 4 token-scale + 4 weight-scale columns
// Tensor memory: two accumulators, then the scale slots.  One CTA per SM
// holds all 512 columns (accumulators 128 apart); with two CTAs per SM
// (16-token tiles) each holds 128: accumulators of 2 NT = 32 columns and up
// to 4 stage slots.
__host__ __device__ constexpr int acc_cols_for(bool two) { return two ? 32 : 128; }
__host__ __device__ constexpr int tmem_cols_for(bool two) { return two ? 128 : 512; }
constexpr int kTwoMaxStages = (128 - 2 * 32) / (8 * 2);
constexpr uint64_t kWaitLimitNs = 2000000000ull;
constexpr uint64_t kTestWaitNs = 200000ull;  // the injected wait of test_timeout_cta

// Per work item the producer also loads an auxiliary block: the weight-scale
// bytes of the item's rows [BN][K/32] and the token-scale words of its tile
// [stages][2 NT]; NB = 1 or 2 of them (double-buffered across items).
// The gate/up epilogue also stages h in two tiles [NT][64] bf16.
struct SmemLayout {
  int x_off, w_off, a_off, wsc_bytes, aux_bytes, h_off, bar_off, total;
};

__host__ __device__ inline SmemLayout smem_layout(int NT, int NS, int NB, int K) {
  SmemLayout L;
  L.x_off = 0;
  L.w_off = NS * WPS * 2 * NT * BKS;
  L.a_off = L.w_off + NS * WPS * W_SMEM;
  L.wsc_bytes = ((BN * (K / 32)) + 127) / 128 * 128;
  L.aux_bytes = L.wsc_bytes + ((K + BKS - 1) / BKS) * 2 * NT * 4;
  L.h_off = L.a_off + NB * L.aux_bytes;
  L.bar_off = L.h_off + 2 * NT * (BN / 2) * 2;
  L.total = L.bar_off + 1024;
  return L;
}

// first K element of 128-K window st; the last window of a K that is not a
// multiple of 128 is moved back to end at K
__host__ __device__ __forceinline__ int stage_k0(int st, int K) {
  return st * BKS < K - BKS ? st * BKS : K - BKS;
}

// ------------------------------------------------ exact two-piece E4M3 split

// Block exponent t = floor(log2 amax) - 7 from the biased exponent field;
// zero and subnormal blocks take the floor -123, which keeps both scale
// bytes (t + 127 for hi, t + 123 for lo) >= 0.
__device__ __forceinline__ int split_exponent(float amax) {
  const int ebits = static_cast<int>((__float_as_uint(amax) >> 23) & 0xFFu);
  return max(ebits - 127 - 7, -123);
}

// Four bf16-exact values of one block -> their hi and lo E4M3 bytes.
__device__ __forceinline__ void split4(const float (&v)[4], int t, uint32_t& hi4, uint32_t& lo4) {
  const float inv = __uint_as_float(static_cast<uint32_t>(127 - t) << 23);  // 2^-t
  hi4 = 0;
  lo4 = 0;
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const float u = v[j] * inv;
    const __nv_fp8_storage_t h8 = __nv_cvt_float_to_fp8(u, __NV_SATFINITE, __NV_E4M3);
    const float hf = __half2float(__half(__nv_cvt_fp8_to_halfraw(h8, __NV_E4M3)));
    const __nv_fp8_storage_t l8 =
        __nv_cvt_float_to_fp8((u - hf) * 16.0f, __NV_SATFINITE, __NV_E4M3);
    hi4 |= static_cast<uint32_t>(h8) << (8 * j);
    lo4 |= static_cast<uint32_t>(l8) << (8 * j);
  }
}

// One bf16-exact value -> its hi and lo E4M3 bytes.
__device__ __forceinline__ void split1(float v, int t, uint8_t& hi, uint8_t& lo) {
  const float u = v * __uint_as_float(static_cast<uint32_t>(127 - t) << 23);  // v / 2^t
  const __nv_fp8_storage_t h8 = __nv_cvt_float_to_fp8(u, __NV_SATFINITE, __NV_E4M3);
  const float hf = __half2float(__half(__nv_cvt_fp8_to_halfraw(h8, __NV_E4M3)));
  hi = static_cast<uint8_t>(h8);
  lo = static_cast<uint8_t>(__nv_cvt_float_to_fp8((u - hf) * 16.0f, __NV_SATFINITE, __NV_E4M3));
}

// ------------------------------------------------------------------ waits

__device__ __forceinline__ void abort_cta(volatile int* abort, int32_t* status) {
  *abort = 1;
  record_status(status, MOE_ERR_TIMEOUT);
}

__device__ __forceinline__ bool wait1(uint64_t* bar, uint32_t parity, volatile int* abort,
                                      int32_t* status) {
  if (tc::mbar_wait(bar, parity, abort, kWaitLimitNs)) return true;
  abort_cta(abort, status);
  return false;
}

// A whole warp waits for a phase: lane 0 polls (sleeping sleep_ns between
// polls when non-zero), then every lane takes the completed phase with one
// poll of its own, which gives each of them the acquire ordering.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort,
                                          int32_t* status, uint32_t sleep_ns = 0) {
  bool r = true;
  if ((threadIdx.x & 31) == 0)
    r = sleep_ns ? tc::mbar_wait_sleep(bar, parity, abort, kWaitLimitNs, sleep_ns)
                 : tc::mbar_wait(bar, parity, abort, kWaitLimitNs);
  r = __shfl_sync(0xFFFFFFFFu, r, 0);
  if (r) {
    // the phase has completed and cannot move on before this warp acts on it
    bool mine = tc::mbar_try_wait(bar, parity);
    for (int k = 0; k < 1024 && !mine; ++k) mine = tc::mbar_try_wait(bar, parity);
    r = __all_sync(0xFFFFFFFFu, mine);
  }
  if (!r) abort_cta(abort, status);
  return r;
}

// Arguments of one GEMM of the pair: the gate/up GEMM (kind 0, input the
// pieces of the rows, K = d_model) or the down GEMM (kind 1, input the pieces
// of h, K = d_ff).
struct GemmArgs {
  const uint32_t* sfx_words;  // token-scale words of the input pieces
  const uint8_t* scales;      // weight scale bytes [E][R][K/32]
  int rows_per_expert, K, out_ld;
  uint16_t* out;  // h (gate/up; may be null) or y_perm (down)
};

// Arguments of one launch: both GEMMs in one persistent grid.
struct MlpArgs {
  GemmArgs gu, dn;
  const Tile* tiles;
  const int* n_tiles;
  int NS, NB, Kmax;
  // written by the gate/up items: the pieces of h, [2 * padded rows][F]
  // bytes, and their scale words [tiles][F/128 windows][2 NT]
  uint8_t* pieces_h;
  uint32_t* words_h;
  int* work;  // the next work item to take; zero at launch
  int* done;  // [tiles] gate/up items finished per token tile; zero at launch
  int32_t* status;
  int fail_cta;
};

// The tensor maps of both GEMMs, indexed by kind: weights (per window, the
// moved-back last window, two windows per box) and input pieces (per
// window, two windows per box).
struct MlpMaps {
  CUtensorMap w[2], wt[2], w2[2], x[2], x2[2];
};

constexpr int kQueue = 4;  // work items handed from the producer to the other roles
constexpr int kQueueReaders = 1 + 4 + kEpiWarps;  // MMA thread, scale writers, epilogue warps

// Wait until *p >= want (a count another CTA raises with release semantics),
// then order this thread's later copies (async proxy) after what it saw.
__device__ __forceinline__ bool wait_count(const int* p, int want, volatile int* abort,
                                           int32_t* status) {
  auto seen = [&]() {
    int v;
    asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v >= want;
  };
  bool ok = seen();
  if (!ok) {
    const uint64_t t0 = tc::globaltimer_ns();
    for (uint32_t i = 1;; ++i) {
      __nanosleep(64);
      if ((ok = seen())) break;
      if (*abort) return false;
      if ((i & 15u) == 0 && tc::globaltimer_ns() - t0 > kWaitLimitNs) {
        abort_cta(abort, status);
        return false;
      }
    }
  }
  asm volatile("fence.proxy.async.global;" ::: "memory");
  return true;
}

// One work item: kind 0 = gate/up (token tile t, 64 gate + 64 up rows at
// feature mt * 64), kind 1 = down (tile t, 128 output rows at mt * 128).
// Every gate/up item comes before every down item.
struct Item {
  int kind, t, mt;
};

__device__ __forceinline__ Item item_of(int i, int n_gu, int n_mt_gu, int n_mt_dn) {
  Item r;
  if (i < n_gu) {
    r.kind = 0;
    r.t = i / n_mt_gu;
    r.mt = i % n_mt_gu;
  } else {
    r.kind = 1;
    r.t = (i - n_gu) / n_mt_dn;
    r.mt = (i - n_gu) % n_mt_dn;
  }
  return r;
}

template <int NT, bool TWO>
__global__ void __launch_bounds__(kThreads, TWO ? 2 : 1)
    grouped_mx_mlp(const __grid_constant__ MlpMaps maps, const MlpArgs args) {
  constexpr int XR = 2 * NT;  // token piece rows per window
  constexpr uint32_t X_BYTES = XR * BKS;
  constexpr uint32_t IDESC = tc::idesc_mx(tc::kFmtE2M1, tc::kFmtE4M3, BN, XR);
  constexpr int kAccCols = acc_cols_for(TWO);
  constexpr int kTmemCols = tmem_cols_for(TWO);
  static_assert(XR >= 16 && XR <= kAccCols && (X_BYTES % 1024) == 0, "token tile of 8..64 tokens");
  static_assert(!TWO || NT == 16, "two CTAs per SM only for 16-token tiles");
  const int NS = args.NS, NB = args.NB;
  const Tile* __restrict__ tiles = args.tiles;
  int32_t* status = args.status;
  const int D = args.dn.rows_per_expert, F = args.gu.rows_per_expert / 2;
  const int n_mt_gu = (F + BN / 2 - 1) / (BN / 2), n_mt_dn = (D + BN - 1) / BN;

  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const SmemLayout L = smem_layout(NT, NS, NB, args.Kmax);
  uint8_t* xs = smem + L.x_off;
  uint8_t* wsm = smem + L.w_off;
  uint8_t* aux = smem + L.a_off;
  uint16_t* hstage = reinterpret_cast<uint16_t*>(smem + L.h_off);  // [2][NT][64] bf16
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L.bar_off);
  uint64_t* full = bars;                  // [NS] stage copies landed and scales written
  uint64_t* empty = full + kMaxStages;    // [NS] stage MMAs complete
  uint64_t* sbar = empty + kMaxStages;    // [2] item auxiliary block landed
  uint64_t* sfree = sbar + 2;             // [2] item auxiliary block no longer read
  uint64_t* dfull = sfree + 2;            // [2] accumulator complete
  uint64_t* dempty = dfull + 2;           // [2] accumulator read by the epilogue
  uint64_t* drain = dempty + 2;           // every MMA issued has completed
  uint64_t* never = drain + 1;            // completed by nothing (the injected test wait)
  uint64_t* qfull = never + 1;            // [kQueue] work item posted
  uint64_t* qempty = qfull + kQueue;      // [kQueue] work item read by every role
  int* qitem = reinterpret_cast<int*>(qempty + kQueue);  // [kQueue]; -1 = no more work
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(qitem + kQueue);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
  volatile int* prod_stages = abort_flag + 1;  // stages the producer issued (read on unwind)

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < NS; ++s) {
      tc::mbar_init(&full[s], 5);  // the producer's copies + the four scale writers
      tc::mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < NB; ++b) {
      tc::mbar_init(&sbar[b], 1);
      tc::mbar_init(&sfree[b], 4);
    }
    for (int a = 0; a < 2; ++a) {
      tc::mbar_init(&dfull[a], 1);
      tc::mbar_init(&dempty[a], kEpiWarps);
    }
    for (int q = 0; q < kQueue; ++q) {
      tc::mbar_init(&qfull[q], 1);
      tc::mbar_init(&qempty[q], kQueueReaders);
    }
    tc::mbar_init(drain, 1);
    tc::mbar_init(never, 1);
    *abort_flag = 0;
    *prod_stages = 0;
    tc::fence_mbar_init();
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      tc::tma_prefetch_desc(&maps.w[k]);
      tc::tma_prefetch_desc(&maps.wt[k]);
      tc::tma_prefetch_desc(&maps.w2[k]);
      tc::tma_prefetch_desc(&maps.x[k]);
      tc::tma_prefetch_desc(&maps.x2[k]);
    }
  }
  if (warp == 1) {
    tc::tmem_alloc(tmem_holder, kTmemCols);
    tc::tmem_relinquish();
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  const uint32_t t_sf = tmem + 2 * kAccCols;  // stage slot s: columns t_sf + s * kSlotCols ...
  int my_stages = 0;  // scale writers: stages this warp has arrived on
  const int n_tiles = __ldg(args.n_tiles);
  const int n_gu = n_tiles * n_mt_gu;
  const int n_items = n_gu + n_tiles * n_mt_dn;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    // Takes the work items one at a time from the grid's counter (the next
    // one while the current one's last two stages go out, so the atomic's
    // round trip is hidden), posts each to the other roles, and issues its
    // copies.  A down item first waits until every gate/up item of its tile
    // has written its pieces of h.  Items are taken in index order, so every
    // gate/up item is taken before any down item, and a producer never
    // waits on another CTA while it holds a gate/up item: the wait always
    // ends.
    if (lane == 0) {
      int g = 0, it = 0;
      int s_slot = 0;          // ring slot of stage g
      uint32_t s_phase = 0;    // parity of slot s_slot's current use
      int next = 0;
      bool taken = false;      // next holds an item already taken
      bool dep = false;        // waited for the split kernel before this launch
      for (;;) {
        const int qs = it % kQueue;
        if (it >= kQueue && !wait1(&qempty[qs], ((it / kQueue) - 1) & 1, abort_flag, status)) break;
        const int b = it % NB, use = it / NB;
        // the auxiliary buffer is free once the scale writers are done with its last item
        if (use > 0 && !wait1(&sfree[b], (use - 1) & 1, abort_flag, status)) break;
        const int i = taken ? next : atomicAdd(args.work, 1);
        taken = false;
        qitem[qs] = i < n_items ? i : -1;
        tc::mbar_arrive(&qfull[qs]);
        if (i >= n_items) break;
        const Item I = item_of(i, n_gu, n_mt_gu, n_mt_dn);
        const bool gu = I.kind == 0;
        if (!gu && !wait_count(args.done + I.t, n_mt_gu, abort_flag, status)) break;
        const int K = gu ? args.gu.K : args.dn.K;
        const int rows_per_expert = gu ? args.gu.rows_per_expert : args.dn.rows_per_expert;
        const uint8_t* scales = gu ? args.gu.scales : args.dn.scales;
        const uint32_t* sfx_words = gu ? args.gu.sfx_words : args.dn.sfx_words;
        const int nwin = (K + BKS - 1) / BKS, nstg = (nwin + WPS - 1) / WPS, kscale = K / 32;
        const CUtensorMap* mw = &maps.w[I.kind];
        const CUtensorMap* mwt = &maps.wt[I.kind];
        const CUtensorMap* mw2 = &maps.w2[I.kind];
        const CUtensorMap* mx = &maps.x[I.kind];
        const CUtensorMap* mx2 = &maps.x2[I.kind];
        const Tile tile = tiles[I.t];
        const int64_t erow = static_cast<int64_t>(tile.e) * rows_per_expert;
        uint8_t* sdst = aux + b * L.aux_bytes;
        const uint32_t wbytes = static_cast<uint32_t>(nwin) * XR * 4;
        if (gu) {
          const int f0 = I.mt * (BN / 2);
          const uint32_t bytes = static_cast<uint32_t>(min(BN / 2, F - f0)) * kscale;
          tc::mbar_arrive_expect_tx(&sbar[b], 2 * bytes + wbytes);
          tc::bulk_load(sdst, scales + (erow + f0) * kscale, bytes, &sbar[b]);
          tc::bulk_load(sdst + (BN / 2) * kscale, scales + (erow + F + f0) * kscale, bytes,
                        &sbar[b]);
        } else {
          const int d0 = I.mt * BN;
          const uint32_t bytes = static_cast<uint32_t>(min(BN, rows_per_expert - d0)) * kscale;
          tc::mbar_arrive_expect_tx(&sbar[b], bytes + wbytes);
          tc::bulk_load(sdst, scales + (erow + d0) * kscale, bytes, &sbar[b]);
        }
        // the first gate/up item of this CTA: its token side (pieces and
        // words, written by the split kernel) waits for that kernel, its
        // weights do not
        const bool early = gu && !dep;
        if (!early)
          tc::bulk_load(sdst + L.wsc_bytes, sfx_words + static_cast<int64_t>(I.t) * nwin * XR,
                        wbytes, &sbar[b]);
        ++it;  // items whose auxiliary copies were issued
        const int wrow = gu ? I.mt * (BN / 2) : I.mt * BN;
        const int take_at = nstg >= 2 ? nstg - 2 : 0;
        // stage st into ring slot `slot`: the barrier's byte count and the
        // weight copies, then the token copies
        auto issue_w = [&](int st, int slot) {
          const int w0 = st * WPS;
          const int nv = min(WPS, nwin - w0);
          tc::mbar_arrive_expect_tx(&full[slot], nv * (W_TX + X_BYTES));
          if (nv == 2 && w0 + 1 < K / BKS) {
            // two whole windows: one copy of each operand for the stage (the
            // copy engine's cost is mostly per copy, not per byte)
            uint8_t* wdst = wsm + slot * WPS * W_SMEM;
            if (gu) {
              tc::tma_load_5d(wdst, mw2, &full[slot], 0, 0, wrow, w0, tile.e);
            } else {
              tc::tma_load_4d(wdst, mw2, &full[slot], 0, wrow, w0, tile.e);
            }
          } else {
            for (int v = 0; v < nv; ++v) {
              const int w = w0 + v;
              uint8_t* wdst = wsm + (slot * WPS + v) * W_SMEM;
              if (stage_k0(w, K) == w * BKS) {
                if (gu) {
                  tc::tma_load_5d(wdst, mw, &full[slot], 0, w, 0, wrow, tile.e);
                } else {
                  tc::tma_load_4d(wdst, mw, &full[slot], 0, w, wrow, tile.e);
                }
              } else {
                if (gu) {
                  tc::tma_load_4d(wdst, mwt, &full[slot], 0, 0, wrow, tile.e);
                } else {
                  tc::tma_load_3d(wdst, mwt, &full[slot], 0, wrow, tile.e);
                }
              }
            }
          }
        };
        auto issue_x = [&](int st, int slot) {
          const int w0 = st * WPS;
          const int nv = min(WPS, nwin - w0);
          if (nv == 2 && w0 + 1 < K / BKS) {
            tc::tma_load_3d(xs + slot * WPS * X_BYTES, mx2, &full[slot], 0, I.t * XR, w0);
          } else {
            for (int v = 0; v < nv; ++v)
              tc::tma_load_2d(xs + (slot * WPS + v) * X_BYTES, mx, &full[slot],
                              stage_k0(w0 + v, K), I.t * XR);
          }
        };
        int st0 = 0;
        if (early) {
          // on this CTA's first item the first NS stages need no free slot:
          // their weights go out before the wait
          const int pre = g == 0 ? min(NS, nstg) : 0;
          for (int st = 0; st < pre; ++st) {
            if (st == take_at) {
              next = atomicAdd(args.work, 1);
              taken = true;
            }
            issue_w(st, st);
          }
          wait_for_previous();
          dep = true;
          tc::bulk_load(sdst + L.wsc_bytes, sfx_words + static_cast<int64_t>(I.t) * nwin * XR,
                        wbytes, &sbar[b]);
          for (int st = 0; st < pre; ++st) issue_x(st, st);
          st0 = pre;
          g += pre;
          s_slot = pre % NS;
          s_phase = pre == NS ? 1u : 0u;
        }
        bool ok = true;
        for (int st = st0; st < nstg; ++st, ++g) {
          if (st == take_at) {
            next = atomicAdd(args.work, 1);
            taken = true;
          }
          if (g >= NS && !wait1(&empty[s_slot], s_phase ^ 1u, abort_flag, status)) {
            ok = false;
            break;
          }
          issue_w(st, s_slot);
          issue_x(st, s_slot);
          if (++s_slot == NS) {
            s_slot = 0;
            s_phase ^= 1u;
          }
        }
        if (!ok) break;
      }
      *prod_stages = g;
      // the items whose auxiliary copies were issued: [it - NB, it) at most
      // (their drain comes after the scale writers' catch-up, below)
      my_stages = it;
    }
  } else if (warp == 1) {
    // ----------------------------------------------------------- MMA issuer
    // The loop keeps every index in running counters and every operand
    // address in a descriptor that only gets constants added: one thread
    // issues all MMAs, so its per-stage instruction chain is the MMA rate.
    if (lane == 0) {
      int it = 0;
      int s_slot = 0;
      uint32_t s_phase = 0, d_phase = 0;
      bool ok = true, any = false;
      const uint64_t xdesc0 = tc::smem_desc_sw128(tc::smem_u32(xs));
      const uint64_t wdesc0 = tc::smem_desc_sw128(tc::smem_u32(wsm));
      // testing only: the first wait of this CTA waits on a barrier that
      // nothing completes, with a short limit, and gives up as a timeout would
      if (static_cast<int>(blockIdx.x) == args.fail_cta &&
          !tc::mbar_wait(never, 0, abort_flag, kTestWaitNs)) {
        abort_cta(abort_flag, status);
        ok = false;
      }
      for (; ok; ++it) {
        const int qs = it % kQueue;
        if (!wait1(&qfull[qs], (it / kQueue) & 1, abort_flag, status)) break;
        const int i = qitem[qs];
        tc::mbar_arrive(&qempty[qs]);
        if (i < 0) break;
        const int K = i < n_gu ? args.gu.K : args.dn.K;
        const int nwin = (K + BKS - 1) / BKS, nstg = (nwin + WPS - 1) / WPS;
        const int tail_w = (K % BKS) ? nwin - 1 : nwin;  // the re-read window, if any
        const uint32_t d = tmem + (it & 1) * kAccCols;
        // accumulator it & 1 was last used by item it - 2
        if (it >= 2) {
          if (!wait1(&dempty[it & 1], d_phase, abort_flag, status)) break;
          if (it & 1) d_phase ^= 1u;
        }
        uint64_t xdesc = xdesc0 + static_cast<uint64_t>(s_slot * WPS * (X_BYTES >> 4));
        uint64_t wdesc = wdesc0 + static_cast<uint64_t>(s_slot * WPS * (W_SMEM >> 4));
        uint32_t sfa = t_sf + s_slot * kSlotCols;
        for (int st = 0; st < nstg; ++st) {
          if (!wait1(&full[s_slot], s_phase, abort_flag, status)) {
            ok = false;
            break;
          }
          tc::tc_fence_after();
          // a descriptor addresses shared memory in 16-byte units: +2 per 32
          // bytes; A = weights with their scales in the slot's columns 4-7,
          // B = token pieces with theirs in columns 0-3
#pragma unroll
          for (int v = 0; v < WPS; ++v) {
            const int w = st * WPS + v;
            if (w >= nwin) break;
            const uint64_t xv = xdesc + v * (X_BYTES >> 4), wv = wdesc + v * (W_SMEM >> 4);
            const uint32_t sx = sfa + 8 * v, sw = sx + 4;
            if (w != tail_w) {
              tc::mma_mx_ss(d, wv, xv, IDESC | tc::idesc_sf_ids(0, 0), w > 0 ? 1u : 0u, sw, sx);
              tc::mma_mx_ss(d, wv + 2, xv + 2, IDESC | tc::idesc_sf_ids(1, 1), 1u, sw, sx);
            }
            tc::mma_mx_ss(d, wv + 4, xv + 4, IDESC | tc::idesc_sf_ids(2, 2),
                          (w != tail_w || w > 0) ? 1u : 0u, sw, sx);
            tc::mma_mx_ss(d, wv + 6, xv + 6, IDESC | tc::idesc_sf_ids(3, 3), 1u, sw, sx);
          }
          tc::mma_commit(&empty[s_slot]);
          any = true;
          xdesc += WPS * (X_BYTES >> 4);
          wdesc += WPS * (W_SMEM >> 4);
          sfa += kSlotCols;
          if (++s_slot == NS) {
            s_slot = 0;
            s_phase ^= 1u;
            xdesc = xdesc0;
            wdesc = wdesc0;
            sfa = t_sf;
          }
        }
        if (ok) tc::mma_commit(&dfull[it & 1]);
      }
      // completes once every MMA this thread issued has finished
      if (any)
        tc::mma_commit(drain);
      else
        tc::mbar_arrive(drain);
    }
  } else if (warp < 6) {
    // ------------------------------------------------------- scale writers
    const int q = warp & 3;
    const uint32_t lane_base = static_cast<uint32_t>(q * 32) << 16;
    int g = 0, it = 0;
    int s_slot = 0;        // stage slot (and scale slot) of stage g
    uint32_t s_phase = 0;  // parity of its current use
    for (;; ++it) {
      const int qs = it % kQueue;
      if (!warp_wait(&qfull[qs], (it / kQueue) & 1, abort_flag, status, 64)) break;
      const int i = qitem[qs];
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&qempty[qs]);
      if (i < 0) break;
      const Item I = item_of(i, n_gu, n_mt_gu, n_mt_dn);
      const bool gu = I.kind == 0;
      const int K = gu ? args.gu.K : args.dn.K;
      const int nwin = (K + BKS - 1) / BKS, nstg = (nwin + WPS - 1) / WPS, kscale = K / 32;
      const int mt = I.mt;
      const int b = it % NB;
      if (!warp_wait(&sbar[b], (it / NB) & 1, abort_flag, status, 64)) break;
      const uint8_t* sblock = aux + b * L.aux_bytes;
      const uint32_t* xwords = reinterpret_cast<const uint32_t*>(sblock + L.wsc_bytes);
      // weight-scale column c of lane l holds weight row n = 32c + l
      int srow[4];
      bool live[4];
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const int n = 32 * c + lane;
        if (gu) {
          srow[c] = (n & 1) * (BN / 2) + (n >> 1);
          live[c] = mt * (BN / 2) + (n >> 1) < F;
        } else {
          srow[c] = n;
          live[c] = mt * BN + n < D;
        }
      }
      const uint8_t* wsc[4];
#pragma unroll
      for (int c = 0; c < 4; ++c) wsc[c] = sblock + srow[c] * kscale;
      bool ok = true;
      for (int st = 0; st < nstg; ++st, ++g) {
        // the slot's previous MMAs have completed (so has its previous copy
        // phase, which those MMAs waited for): lane 0 polls, the warp follows
        if (g >= NS) {
          bool r = true;
          if (lane == 0) r = tc::mbar_wait(&empty[s_slot], s_phase ^ 1u, abort_flag, kWaitLimitNs);
          if (!__shfl_sync(0xFFFFFFFFu, r, 0)) {
            abort_cta(abort_flag, status);
            ok = false;
            break;
          }
          tc::tc_fence_after();
        }
#pragma unroll
        for (int v = 0; v < WPS; ++v) {
          const int w = st * WPS + v;
          if (w >= nwin) break;
          const int kb0 = stage_k0(w, K) / 32;
          // token-scale column c of lane l holds piece row 32c + l
          const uint32_t* sx = xwords + w * XR;
          uint32_t wx[4];
#pragma unroll
          for (int c = 0; c < 4; ++c) wx[c] = (32 * c + lane < XR) ? sx[32 * c + lane] : 0x7F7F7F7Fu;
          uint32_t ww[4];
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            if (live[c]) {
              const uint16_t* p = reinterpret_cast<const uint16_t*>(wsc[c] + kb0);
              ww[c] = static_cast<uint32_t>(p[0]) | (static_cast<uint32_t>(p[1]) << 16);
            } else {
              ww[c] = 0x7F7F7F7Fu;
            }
          }
          const uint32_t col = t_sf + s_slot * kSlotCols + 8 * v;
          tc::tmem_st4(lane_base + col, wx);
          tc::tmem_st4(lane_base + col + 4, ww);
        }
        tc::tmem_st_wait();
        tc::tc_fence_before();
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(&full[s_slot]);
        if (++s_slot == NS) {
          s_slot = 0;
          s_phase ^= 1u;
        }
      }
      if (!ok) break;
      // the item's auxiliary block is no longer read
      if (lane == 0) tc::mbar_arrive(&sfree[b]);
    }
    my_stages = g;
  } else {
    // ------------------------------------------------------------ epilogue
    // Lane l of quarter q holds weight row m = 32 q + l of the item; this
    // warp reads the accumulator columns of tokens [half HT, half HT + HT).
    // The eight warps leave the loop only together (after a barrier that all
    // of them reach), so none is left waiting at one of their barriers.
    constexpr int HT = NT / 2;
    const int q = warp & 3;
    const int half = (warp - 6) >> 2;
    const int ew = warp - 6;  // epilogue warp 0..7
    const uint32_t lane_base = static_cast<uint32_t>(q * 32) << 16;
    for (int it = 0;; ++it) {
      const int qs = it % kQueue;
      bool ok = warp_wait(&qfull[qs], (it / kQueue) & 1, abort_flag, status, 256);
      int i = -1;
      if (ok) {
        i = qitem[qs];
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(&qempty[qs]);
      }
      if (!tc::bar_and(1, 32 * kEpiWarps, ok) || i < 0) break;
      const Item I = item_of(i, n_gu, n_mt_gu, n_mt_dn);
      const Tile tile = tiles[I.t];
      const int a = it & 1;
      ok = warp_wait(&dfull[a], (it >> 1) & 1, abort_flag, status, 256);
      float acc[HT];  // token half HT + j of this lane's row: hi + lo piece
      if (ok) {
        tc::tc_fence_after();
        const uint32_t dcol = tmem + a * kAccCols + half * NT + lane_base;
#pragma unroll
        for (int c = 0; c < NT; c += 16) {
          uint32_t r[16];
          tc::tmem_ld16(dcol + c, r);
          tc::tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < 8; ++j)
            acc[c / 2 + j] = __uint_as_float(r[2 * j]) + __uint_as_float(r[2 * j + 1]);
        }
        // this warp has read its part of the accumulator
        tc::tc_fence_before();
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(&dempty[a]);
      }
      if (I.kind == 0) {
        // lanes 2j (gate) and 2j + 1 (up) hold local feature fl = 16 q + j;
        // the gate lane finishes the first HT / 2 tokens, the up lane the rest
        constexpr int QT = HT / 2;
        const bool up = lane & 1;
        const int fl = 16 * q + (lane >> 1);
        uint16_t* hs = hstage + a * NT * (BN / 2);
        if (ok) {
#pragma unroll
          for (int j = 0; j < QT; ++j) {
            const float recv = __shfl_xor_sync(0xFFFFFFFFu, up ? acc[j] : acc[QT + j], 1);
            const float gv = up ? recv : acc[j];
            const float uv = up ? acc[QT + j] : recv;
            const float hh = __fdividef(gv, 1.0f + __expf(-gv)) * uv;
            hs[(half * HT + (up ? QT : 0) + j) * (BN / 2) + fl] = f32_to_bf16_rne(hh);
          }
        }
        if (!tc::bar_and(1, 32 * kEpiWarps, ok)) break;
        // one warp per (token, 32-feature block): store h, split it into the
        // pieces of the down GEMM and write the block's scale bytes
        const int fb0 = I.mt * (BN / 2);
        const int nunits = tile.nrows * 2;
        for (int u = ew; u < nunits; u += kEpiWarps) {
          const int tl = u >> 1, b = u & 1;
          const int f = fb0 + 32 * b + lane;
          const uint16_t hbits = hs[tl * (BN / 2) + 32 * b + lane];
          const float v = bf16_to_f32(hbits);
          if (args.gu.out)
            args.gu.out[static_cast<int64_t>(tile.row0 + tl) * args.gu.out_ld + f] = hbits;
          float amax = fabsf(v);
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, o));
          const int te = split_exponent(amax);
          uint8_t hi, lo;
          split1(v, te, hi, lo);
          const int64_t p = static_cast<int64_t>(I.t) * NT + tl;  // padded row of this token
          args.pieces_h[(2 * p) * F + f] = hi;
          args.pieces_h[(2 * p + 1) * F + f] = lo;
          if (lane == 0) {
            // scale bytes of block blk in the words of the window(s) that
            // cover it: window blk / 4 (byte blk % 4), and, when F is not a
            // multiple of 128, the moved-back last window [F - 128, F)
            const int nwo = (F + BKS - 1) / BKS;
            const int blk = (fb0 + 32 * b) / 32;
            const int tail0 = (F % BKS) ? (F - BKS) / 32 : 0x7FFFFFFF;
            auto put = [&](int w, int byte) {
              uint8_t* wb = reinterpret_cast<uint8_t*>(
                  args.words_h + (static_cast<int64_t>(I.t) * nwo + w) * (2 * NT) + 2 * tl);
              wb[byte] = static_cast<uint8_t>(te + 127);
              wb[4 + byte] = static_cast<uint8_t>(te + 123);
            };
            if (F % BKS == 0 || blk / 4 < nwo - 1) put(blk / 4, blk % 4);
            if (blk >= tail0) put(nwo - 1, blk - tail0);
          }
        }
        // every store of this item is done: release it to the tile's down
        // items (read by copies in other CTAs)
        tc::bar_and(1, 32 * kEpiWarps, true);
        if (ew == 0 && lane == 0) {
          __threadfence();
          asm volatile("fence.proxy.async.global;" ::: "memory");
          asm volatile("red.release.gpu.global.add.s32 [%0], 1;" ::"l"(args.done + I.t) : "memory");
        }
      } else if (ok) {
        const int dd = I.mt * BN + 32 * q + lane;
        if (dd < D) {
          uint16_t* ocol = args.dn.out + static_cast<int64_t>(tile.row0) * args.dn.out_ld + dd;
#pragma unroll
          for (int j = 0; j < HT; ++j) {
            const int tl = half * HT + j;
            if (tl < tile.nrows) ocol[static_cast<int64_t>(tl) * args.dn.out_ld] = f32_to_bf16_rne(acc[j]);
          }
        }
      }
    }
  }

  // ---------------------------------------------------------------- unwind
  tc::tc_fence_before();
  __syncthreads();
  if (*abort_flag) {
    // A stage's copy barrier also counts the four scale writers: a writer
    // that gave up adds the arrivals it skipped for the stages the producer
    // issued, so those phases complete as soon as their copies land.
    if (warp >= 2 && warp < 6 && lane == 0) {
      const int g_p = *prod_stages;
      for (int gg = my_stages; gg < g_p; ++gg) tc::mbar_arrive(&full[gg % NS]);
    }
    __syncthreads();
  }
  if (warp == 0 && lane == 0) {
    // every copy this thread issued has landed before the CTA exits
    const int g = *prod_stages, it = my_stages;
    for (int gg = max(0, g - NS); gg < g; ++gg)
      tc::mbar_drain(&full[gg % NS], (gg / NS) & 1, kWaitLimitNs / 8);
    for (int j = max(0, it - NB); j < it; ++j)
      tc::mbar_drain(&sbar[j % NB], (j / NB) & 1, kWaitLimitNs / 8);
  }
  if (warp == 1) {
    // every MMA has completed (already on the normal path)
    if (lane == 0) tc::mbar_drain(drain, 0, kWaitLimitNs / 8);
    __syncwarp();
    tc::tc_fence_after();
    tc::tmem_dealloc(tmem, kTmemCols);
  }
}

// Exact two-piece E4M3 split of bf16 rows (see the file comment), written in
// the tile-padded layout: piece rows [2 * tiles * NT][K] bytes, row 2p = hi
// and 2p + 1 = lo of padded row p = t NT + i, and, per tile and 128-K window,
// the scale words [2 NT] in the same row order (byte b of a word = E8M0 scale
// of the window's 32-element block b).  One warp per (padded row, window);
// lane l holds elements 4l..4l+3 of the window, a block is 8 lanes.  Padded
// rows get zero pieces.  Row r of the permuted order is src[r], or, with
// `gather`, src[gather[r] / k] (the layer splits straight from x).
__global__ void __launch_bounds__(256) split_rows_kernel(
    const uint16_t* __restrict__ src, const int32_t* __restrict__ gather, int k, int K,
    const Tile* __restrict__ tiles, const int* __restrict__ n_tiles, int NT, int64_t padded_rows,
    uint8_t* __restrict__ pieces, uint32_t* __restrict__ words) {
  // the GEMM launch that follows may start; it waits for this kernel before
  // it reads the pieces or their words
  allow_dependents();
  const int nstg = (K + BKS - 1) / BKS;
  const int st = blockIdx.y;
  const int lane = threadIdx.x & 31;
  const int64_t p = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (p >= padded_rows) return;
  const int ti = static_cast<int>(p / NT), i = static_cast<int>(p % NT);
  if (ti >= __ldg(n_tiles)) return;
  const Tile tl = tiles[ti];
  const int k0 = stage_k0(st, K);
  const int kk = k0 + lane * 4;
  float v[4] = {0.f, 0.f, 0.f, 0.f};
  if (i < tl.nrows) {
    int64_t r = tl.row0 + i;
    if (gather) r = __ldg(gather + r) / k;
    const uint2 raw = *reinterpret_cast<const uint2*>(src + r * K + kk);
    v[0] = bf16_to_f32(static_cast<uint16_t>(raw.x));
    v[1] = bf16_to_f32(static_cast<uint16_t>(raw.x >> 16));
    v[2] = bf16_to_f32(static_cast<uint16_t>(raw.y));
    v[3] = bf16_to_f32(static_cast<uint16_t>(raw.y >> 16));
  }
  float amax = fmaxf(fmaxf(fabsf(v[0]), fabsf(v[1])), fmaxf(fabsf(v[2]), fabsf(v[3])));
  amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, 1));
  amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, 2));
  amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, 4));
  const int t = split_exponent(amax);
  uint32_t hi4, lo4;
  split4(v, t, hi4, lo4);
  // a moved-back last window re-reads [K - 128, 128 st): only its new elements are written
  if (kk >= st * BKS) {
    *reinterpret_cast<uint32_t*>(pieces + (2 * p) * K + kk) = hi4;
    *reinterpret_cast<uint32_t*>(pieces + (2 * p + 1) * K + kk) = lo4;
  }
  uint32_t whi = 0, wlo = 0;
#pragma unroll
  for (int b = 0; b < 4; ++b) {
    const int tb = __shfl_sync(0xFFFFFFFFu, t, 8 * b);
    whi |= static_cast<uint32_t>(tb + 127) << (8 * b);
    wlo |= static_cast<uint32_t>(tb + 123) << (8 * b);
  }
  if (lane == 0) {
    uint32_t* w = words + (static_cast<int64_t>(ti) * nstg + st) * (2 * NT);
    w[2 * i] = whi;
    w[2 * i + 1] = wlo;
  }
}

// ------------------------------------------------------------ host helpers

bool encode(CUtensorMap* map, CUtensorMapDataType type, int rank, const void* base,
            const cuuint64_t* dims, const cuuint64_t* strides, const cuuint32_t* box) {
  EncodeTiledFn fn = encode_tiled_fn();
  if (!fn) return false;
  const cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  return fn(map, type, static_cast<cuuint32_t>(rank), const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Weight codes [E][R][K/2] (two codes per byte, element 2i in the low
// nibble), read in 128-code windows that land one byte per code.  Gate/up
// (R = 2F): the box takes a gate row and its up row for 64 consecutive f,
// interleaved; down: 128 consecutive rows.  `main` walks the windows at
// multiples of 128 codes, `tail` is the single window [K - 128, K).
bool make_weight_maps(CUtensorMap* main, CUtensorMap* tail, CUtensorMap* main2, const uint8_t* q,
                      int E, int R, int K, bool gate_up) {
  const cuuint64_t row = static_cast<cuuint64_t>(K / 2);
  const cuuint64_t mat = static_cast<cuuint64_t>(R) * row;
  const CUtensorMapDataType T = CU_TENSOR_MAP_DATA_TYPE_16U4_ALIGN16B;
  const uint8_t* tail_base = q + (K - BKS) / 2;
  // two consecutive whole windows in one box: the window is the outer box
  // dimension, so each lands as its own [128 rows][128 B] block
  const cuuint64_t nwf = static_cast<cuuint64_t>(K / BKS);
  if (gate_up) {
    const cuuint64_t F2 = static_cast<cuuint64_t>(R / 2);
    const cuuint64_t d2[5] = {BKS, 2, F2, nwf, static_cast<cuuint64_t>(E)};
    const cuuint64_t s2[4] = {F2 * row, row, BKS / 2, mat};
    const cuuint32_t b2[5] = {BKS, 2, BN / 2, 2, 1};
    if (!encode(main2, T, 5, q, d2, s2, b2)) return false;
  } else {
    const cuuint64_t d2[4] = {BKS, static_cast<cuuint64_t>(R), nwf, static_cast<cuuint64_t>(E)};
    const cuuint64_t s2[3] = {row, BKS / 2, mat};
    const cuuint32_t b2[4] = {BKS, BN, 2, 1};
    if (!encode(main2, T, 4, q, d2, s2, b2)) return false;
  }
  if (gate_up) {
    const cuuint64_t F = static_cast<cuuint64_t>(R / 2);
    const cuuint64_t d5[5] = {BKS, static_cast<cuuint64_t>(K / BKS), 2, F,
                              static_cast<cuuint64_t>(E)};
    const cuuint64_t s5[4] = {BKS / 2, F * row, row, mat};
    const cuuint32_t b5[5] = {BKS, 1, 2, BN / 2, 1};
    const cuuint64_t d4[4] = {BKS, 2, F, static_cast<cuuint64_t>(E)};
    const cuuint64_t s4[3] = {F * row, row, mat};
    const cuuint32_t b4[4] = {BKS, 2, BN / 2, 1};
    if (!encode(main, T, 5, q, d5, s5, b5)) return false;
    return K % BKS == 0 ? encode(tail, T, 5, q, d5, s5, b5)
                        : encode(tail, T, 4, tail_base, d4, s4, b4);
  }
  const cuuint64_t d4[4] = {BKS, static_cast<cuuint64_t>(K / BKS), static_cast<cuuint64_t>(R),
                            static_cast<cuuint64_t>(E)};
  const cuuint64_t s4[3] = {BKS / 2, row, mat};
  const cuuint32_t b4[4] = {BKS, 1, BN, 1};
  const cuuint64_t d3[3] = {BKS, static_cast<cuuint64_t>(R), static_cast<cuuint64_t>(E)};
  const cuuint64_t s3[2] = {row, mat};
  const cuuint32_t b3[3] = {BKS, BN, 1};
  if (!encode(main, T, 4, q, d4, s4, b4)) return false;
  return K % BKS == 0 ? encode(tail, T, 4, q, d4, s4, b4)
                      : encode(tail, T, 3, tail_base, d3, s3, b3);
}

// token piece rows [2 * padded rows][K] bytes, box = 128 K x 2 NT rows; the
// second map takes two consecutive whole windows per box
bool make_piece_map(CUtensorMap* map, CUtensorMap* map2, const uint8_t* pieces,
                    int64_t padded_rows, int K, int NT) {
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(2 * padded_rows)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(K)};
  const cuuint32_t box[2] = {BKS, static_cast<cuuint32_t>(2 * NT)};
  if (!encode(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, pieces, dims, strides, box)) return false;
  const cuuint64_t d2[3] = {BKS, static_cast<cuuint64_t>(2 * padded_rows),
                            static_cast<cuuint64_t>(K / BKS)};
  const cuuint64_t s2[2] = {static_cast<cuuint64_t>(K), BKS};
  const cuuint32_t b2[3] = {BKS, static_cast<cuuint32_t>(2 * NT), 2};
  return encode(map2, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, pieces, d2, s2, b2);
}

struct GemmConfig {
  int NT, NS, NB, CPS;
};

constexpr int kMaxSmemPerCta = 227 * 1024;
// two CTAs share an SM's 228 KB, each with 1 KB reserved
constexpr int kTwoSmemPerCta = 112 * 1024;

int smem_bytes(int NT, int NS, int NB, int K) { return smem_layout(NT, NS, NB, K).total + 1024; }

// token-tile width: about twice the mean rows per expert, 16..64.  16-token
// tiles run two CTAs per SM when two stages fit in half the shared memory:
// one thread issuing every copy of an SM's ring was measured to cap the
// stream of the 4-bit weight boxes well below the HBM rate, and two CTAs
// (two issuing threads, two rings) lift it.  Otherwise one CTA per SM with
// the deepest copy ring (up to 12 stages), its weight-scale block
// double-buffered when that costs no stage.
GemmConfig choose_config(const moe_shape& sh) {
  const int64_t S = static_cast<int64_t>(sh.T) * sh.k;
  const int64_t want = 2 * ((S + sh.E - 1) / sh.E);
  int nt = 16;
  while (nt < want && nt < 64) nt *= 2;
  const int K = sh.d_model > sh.d_ff ? sh.d_model : sh.d_ff;
  if (nt == 16) {
    for (int ns = kTwoMaxStages; ns >= 2; --ns) {
      if (smem_bytes(16, ns, 2, K) <= kTwoSmemPerCta) return {16, ns, 2, 2};
      if (smem_bytes(16, ns, 1, K) <= kTwoSmemPerCta) return {16, ns, 1, 2};
    }
  }
  for (;;) {
    for (int ns = kMaxStages; ns >= 2; --ns) {
      if (smem_bytes(nt, ns, 2, K) <= kMaxSmemPerCta) return {nt, ns, 2, 1};
      if (smem_bytes(nt, ns, 1, K) <= kMaxSmemPerCta) return {nt, ns, 1, 1};
    }
    if (nt == 16) return {16, 0, 1, 1};  // does not fit: refused by the plan
    nt /= 2;
  }
}

// The dynamic shared-memory opt-in of a kernel, once per device.
template <typename Kern>
bool allow_smem(Kern kern, std::atomic<uint64_t>& done) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return false;
  }
  const uint64_t bit = dev < 64 ? (uint64_t(1) << dev) : 0;
  if (bit && (done.load() & bit)) return true;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kMaxSmemPerCta) !=
      cudaSuccess) {
    cudaGetLastError();
    return false;
  }
  done.fetch_or(bit);
  return true;
}

template <int NT, bool TWO>
bool prepare_mlp() {
  static std::atomic<uint64_t> done{0};
  return allow_smem(grouped_mx_mlp<NT, TWO>, done);
}

bool prepare_nt(int NT, int CPS) {
  switch (NT) {
    case 16:
      return CPS == 2 ? prepare_mlp<16, true>() : prepare_mlp<16, false>();
    case 32:
      return prepare_mlp<32, false>();
    default:
      return prepare_mlp<64, false>();
  }
}

template <int NT, bool TWO>
moe_status launch_mlp(const MxPlan& P, const MlpMaps& maps, const MlpArgs& a, int max_items,
                      cudaStream_t stream) {
  const int smem = smem_bytes(NT, P.NS, P.NB, a.Kmax);
  const int slots = (TWO ? 2 : 1) * sm_count();
  const int grid = max_items < slots ? max_items : slots;
  // one CTA per SM holds all 512 tensor-memory columns: it asks for enough
  // shared memory that no second CTA shares the SM
  const int smem_launch =
      TWO || smem > kMaxSmemPerCta / 2 + 1024 ? smem : kMaxSmemPerCta / 2 + 1024;
  // launched early: it starts while the split kernel before it finishes
  return launch_ex(grouped_mx_mlp<NT, TWO>, dim3(grid), dim3(kThreads), smem_launch, stream,
                   true, maps, a);
}

moe_status launch_nt(const MxPlan& P, const MlpMaps& maps, const MlpArgs& a, int max_items,
                     cudaStream_t st) {
  switch (P.NT) {
    case 16:
      return P.CPS == 2 ? launch_mlp<16, true>(P, maps, a, max_items, st)
                        : launch_mlp<16, false>(P, maps, a, max_items, st);
    case 32:
      return launch_mlp<32, false>(P, maps, a, max_items, st);
    default:
      return launch_mlp<64, false>(P, maps, a, max_items, st);
  }
}

// Workspace of the block-scaled path: the tile list, then for the input rows
// and for h each its pieces [2 * padded rows][K] and scale words
// [tiles][K/128 windows][2 NT].
struct MxWs {
  size_t n_tiles, tiles, pieces_x, words_x, pieces_h, words_h, sched, total;
  int64_t max_tiles, padded_rows;
};

MxWs mx_ws(const moe_shape& sh) {
  const int NT = choose_config(sh).NT;
  const int64_t S = static_cast<int64_t>(sh.T) * sh.k;
  const int D = sh.d_model, F = sh.d_ff;
  MxWs w;
  w.max_tiles = sh.E + (S + NT - 1) / NT;
  w.padded_rows = w.max_tiles * NT;
  auto words_bytes = [&](int K) {
    return static_cast<size_t>(w.max_tiles * ((K + BKS - 1) / BKS)) * 2 * NT * 4;
  };
  w.n_tiles = 0;
  w.tiles = 256;
  w.pieces_x = align_up(w.tiles + static_cast<size_t>(w.max_tiles) * sizeof(Tile), 256);
  w.words_x = align_up(w.pieces_x + 2 * static_cast<size_t>(w.padded_rows) * D, 256);
  w.pieces_h = align_up(w.words_x + words_bytes(D), 256);
  w.words_h = align_up(w.pieces_h + 2 * static_cast<size_t>(w.padded_rows) * F, 256);
  w.sched = align_up(w.words_h + words_bytes(F), 256);  // work counter, then [max tiles] counts
  w.total = align_up(w.sched + (1 + static_cast<size_t>(w.max_tiles)) * sizeof(int), 256);
  return w;
}

}  // namespace

int mx_tile_width(const moe_shape& sh) { return choose_config(sh).NT; }
size_t mx_workspace(const moe_shape& sh) { return mx_ws(sh).total; }

moe_status mx_plan(MlpPlan* p, void* ws) {
  const moe_shape& sh = p->sh;
  const GemmConfig cfg = choose_config(sh);
  if (cfg.NS < 2) return MOE_ERR_SHAPE;
  const MxWs W = mx_ws(sh);
  char* base = static_cast<char*>(ws);
  MxPlan& P = p->mx;
  P.NT = cfg.NT;
  P.NS = cfg.NS;
  P.NB = cfg.NB;
  P.CPS = cfg.CPS;
  P.max_tiles = W.max_tiles;
  P.padded_rows = W.padded_rows;
  p->n_tiles = reinterpret_cast<int*>(base + W.n_tiles);
  p->tiles = reinterpret_cast<Tile*>(base + W.tiles);
  P.pieces_x = reinterpret_cast<uint8_t*>(base + W.pieces_x);
  P.words_x = reinterpret_cast<uint32_t*>(base + W.words_x);
  P.pieces_h = reinterpret_cast<uint8_t*>(base + W.pieces_h);
  P.words_h = reinterpret_cast<uint32_t*>(base + W.words_h);
  P.work = reinterpret_cast<int*>(base + W.sched);
  P.done = P.work + 1;
  p->sched = P.work;
  p->n_sched = 1 + static_cast<int>(W.max_tiles);
  const int D = sh.d_model, F = sh.d_ff, E = sh.E;
  if (!make_weight_maps(&P.m_gu, &P.m_gu_t, &P.m_gu2, p->wgu_q, E, 2 * F, D, true) ||
      !make_weight_maps(&P.m_dn, &P.m_dn_t, &P.m_dn2, p->wdn_q, E, D, F, false) ||
      !make_piece_map(&P.m_x, &P.m_x2, P.pieces_x, W.padded_rows, D, cfg.NT) ||
      !make_piece_map(&P.m_h, &P.m_h2, P.pieces_h, W.padded_rows, F, cfg.NT))
    return MOE_ERR_CUDA;
  if (!prepare_nt(cfg.NT, cfg.CPS)) return MOE_ERR_CUDA;
  return MOE_OK;
}

moe_status mx_enqueue(const MlpPlan& p, const MlpInput& in, int32_t* status, int fail_cta,
                      cudaStream_t stream) {
  const MxPlan& P = p.mx;
  const moe_shape& sh = p.sh;
  const int NT = P.NT, D = sh.d_model, F = sh.d_ff, E = sh.E;
  moe_status st;
  if (!in.tiles_ready &&
      (st = plan_tiles_launch(in.offsets, E, NT, p.tiles, p.n_tiles, p.sched, p.n_sched, stream)) != MOE_OK)
    return st;
  // the input rows, split into pieces (straight from x inside the layer)
  {
    const bool from_x = in.x != nullptr;
    const int nwin = (D + BKS - 1) / BKS;
    const int64_t blocks = (P.padded_rows + 7) / 8;  // 8 warps per block, one row each
    // after the tile plan, or after the layer's permute
    st = launch(split_rows_kernel, dim3(static_cast<unsigned>(blocks), nwin), dim3(256), 0, stream,
                from_x ? in.x : p.x_perm,
                from_x ? in.sorted_slot : static_cast<const int32_t*>(nullptr), from_x ? in.k : 1,
                D, static_cast<const Tile*>(p.tiles), static_cast<const int*>(p.n_tiles), NT,
                P.padded_rows, P.pieces_x, P.words_x);
    if (st != MOE_OK) return st;
  }
  const int max_tiles = static_cast<int>(P.max_tiles);
  const int mt_gu = (F + BN / 2 - 1) / (BN / 2), mt_dn = (D + BN - 1) / BN;
  MlpMaps maps;
  maps.w[0] = P.m_gu;
  maps.wt[0] = P.m_gu_t;
  maps.w2[0] = P.m_gu2;
  maps.x[0] = P.m_x;
  maps.x2[0] = P.m_x2;
  maps.w[1] = P.m_dn;
  maps.wt[1] = P.m_dn_t;
  maps.w2[1] = P.m_dn2;
  maps.x[1] = P.m_h;
  maps.x2[1] = P.m_h2;
  MlpArgs a{};
  a.tiles = p.tiles;
  a.n_tiles = p.n_tiles;
  a.NS = P.NS;
  a.NB = P.NB;
  a.Kmax = D > F ? D : F;
  // gate/up + SwiGLU: h (when asked) and the pieces of h
  a.gu.sfx_words = P.words_x;
  a.gu.scales = p.wgu_s;
  a.gu.rows_per_expert = 2 * F;
  a.gu.K = D;
  a.gu.out_ld = F;
  a.gu.out = p.h;
  a.pieces_h = P.pieces_h;
  a.words_h = P.words_h;
  // down
  a.dn.sfx_words = P.words_h;
  a.dn.scales = p.wdn_s;
  a.dn.rows_per_expert = D;
  a.dn.K = F;
  a.dn.out_ld = D;
  a.dn.out = p.y_perm;
  a.work = P.work;
  a.done = P.done;
  a.status = status;
  a.fail_cta = fail_cta;
  (void)E;
  return launch_nt(P, maps, a, max_tiles * (mt_gu + mt_dn), stream);
}

}  // namespace moe
