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
// MMA shape: M = 128 token rows (the hi and lo pieces of up to 64 tokens,
// interleaved: row 2t = hi of token t, row 2t + 1 = lo), N = 128 weight rows,
// K = 32.  With the weights on N an MMA covers 128 rows x 32 codes and runs at
// the tensor core's full rate (64 cycles), so a 128-K window of 8 KB of codes
// costs 256 cycles of MMA, under the ~370 cycles the SM's share of HBM
// bandwidth needs to deliver it; narrower MMAs are bound by their issue rate.
// The epilogue adds rows 2t and 2t + 1 (neighbouring lanes).
//   * gate/up: the 128 rows are 64 gate rows and the matching 64 up rows,
//     interleaved by the copy's box order (row 2j = gate j, 2j + 1 = up j), so
//     a lane holds both halves of SwiGLU; output h [S][F] bf16.
//   * down: 128 rows of the [D][F] matrix; output y_perm [S][D] bf16.
// The kernel is persistent: one CTA per SM walks the work items (token tile,
// weight slice) b, b + grid, ...; its copy ring (up to 12 stages of two
// 128-K windows each, so one barrier round trip covers 256 of K) runs on
// across items, the weight-scale block of an item is double-buffered and so
// is the accumulator, so one item's epilogue overlaps the next item's MMAs.
// Warp roles (14 warps):
//   warp 0      producer: per item the weight-scale bytes and the token-scale
//               words (bulk copies), per 128-K window the weight codes (TMA,
//               8 KB of packed codes that land as the 16 KB one-byte-per-code
//               layout the MMA reads) and the token pieces (TMA, 2 NT x 128 B)
//   warp 1      tensor-memory owner and MMA issuer: 4 MMAs per window
//   warps 2-5   scale writers: per window they copy the token scales and the
//               weight scales (both from the item's auxiliary block) into the
//               stage slot's scale columns in tensor memory, every lane quarter
//               its own copy, and add their arrival to the stage's barrier, so
//               the MMA thread waits on one barrier per stage
//   warps 6-13  epilogue: two warps per lane quarter, 64 accumulator columns
//               each; a quarter whose tokens are all padding is skipped
// When K is not a multiple of 128 the last window re-reads [K - 128, K) and
// issues only the MMAs over its new 32-element blocks.
// The token pieces sit in a tile-padded layout (tile t owns piece rows
// [2 t NT, 2 t NT + 2 NT)), so every copy of a tile's rows is aligned and
// whole; the MMA's 128-row view of a stage narrower than 128 rows reads on
// into the following shared memory, and those accumulator rows are ignored.
// Every wait is bounded (2 s); on expiry the kernel records MOE_ERR_TIMEOUT
// in the status word, drains its copies and MMAs and returns.
#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>

#include "common.cuh"
#include "tc_sm100.cuh"

namespace moe {
namespace {

constexpr int BKS = 128;            // K elements per window (one 128-byte swizzle row of codes)
constexpr int WPS = 2;              // windows per pipeline stage
constexpr int BN = 128;             // weight rows per work item (MMA N)
constexpr int MM = 128;             // MMA M: token piece rows
constexpr int W_SMEM = BN * BKS;    // one byte per code in shared memory
constexpr int W_TX = BN * BKS / 2;  // bytes one window's weight copy reads
constexpr int kEpiWarps = 8;
constexpr int kThreads = 32 * (6 + kEpiWarps);
constexpr int kMaxStages = 12;      // copy ring depth limit (stage slot s also owns scale slot s)
constexpr int kSlotCols = 8 * WPS;  // per stage and window: 4 token-scale + 4 weight-scale columns
constexpr int kTmemCols = 512;      // two accumulators of BN columns, then the scale slots
constexpr uint64_t kWaitLimitNs = 2000000000ull;

struct Tile {
  int e, row0, nrows, pad;
};

// Per work item the producer also loads an auxiliary block: the weight-scale
// bytes of the item's rows [BN][K/32] and the token-scale words of its tile
// [stages][2 NT]; NB = 1 or 2 of them (double-buffered across items).
struct SmemLayout {
  int x_off, w_off, a_off, wsc_bytes, aux_bytes, bar_off, total;
};

__host__ __device__ inline SmemLayout smem_layout(int NT, int NS, int NB, int K) {
  SmemLayout L;
  L.x_off = 0;  // token ring first: a window's 128-row MMA view runs on into the weight ring
  L.w_off = NS * WPS * 2 * NT * BKS;
  L.a_off = L.w_off + NS * WPS * W_SMEM;
  L.wsc_bytes = ((BN * (K / 32)) + 127) / 128 * 128;
  L.aux_bytes = L.wsc_bytes + ((K + BKS - 1) / BKS) * 2 * NT * 4;
  L.bar_off = L.a_off + NB * L.aux_bytes;
  L.total = L.bar_off + 1024;
  return L;
}

// first K element of 128-K window st; the last window of a K that is not a
// multiple of 128 is moved back to end at K
__host__ __device__ __forceinline__ int stage_k0(int st, int K) {
  return st * BKS < K - BKS ? st * BKS : K - BKS;
}

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

template <int NT, bool GATE_UP>
__global__ void __launch_bounds__(kThreads, 1)
    grouped_mx_gemm(const __grid_constant__ CUtensorMap map_w,
                    const __grid_constant__ CUtensorMap map_w_tail,
                    const __grid_constant__ CUtensorMap map_x,
                    const uint32_t* __restrict__ sfx_words, const uint8_t* __restrict__ scales,
                    const Tile* __restrict__ tiles, const int* __restrict__ n_tiles_dev,
                    int rows_per_expert, int K, int NS, int NB, int out_ld,
                    uint16_t* __restrict__ out, int32_t* __restrict__ status) {
  constexpr int XR = 2 * NT;  // token piece rows per window
  constexpr uint32_t X_BYTES = XR * BKS;
  constexpr uint32_t IDESC = tc::idesc_mx(tc::kFmtE4M3, tc::kFmtE2M1, MM, BN);
  static_assert(XR <= MM && (X_BYTES % 1024) == 0, "token tile of 8..64 tokens");
  const int n_tiles = __ldg(n_tiles_dev);
  const int F = rows_per_expert / 2;
  const int n_mt = GATE_UP ? (F + BN / 2 - 1) / (BN / 2) : (rows_per_expert + BN - 1) / BN;
  const int n_items = n_tiles * n_mt;
  if (static_cast<int>(blockIdx.x) >= n_items) return;  // whole CTA, before any set-up

  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const SmemLayout L = smem_layout(NT, NS, NB, K);
  uint8_t* xs = smem + L.x_off;
  uint8_t* wsm = smem + L.w_off;
  uint8_t* aux = smem + L.a_off;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L.bar_off);
  uint64_t* full = bars;                  // [NS] stage copies landed and scales written
  uint64_t* empty = full + kMaxStages;    // [NS] stage MMAs complete
  uint64_t* sbar = empty + kMaxStages;    // [2] item auxiliary block landed
  uint64_t* sfree = sbar + 2;             // [2] item auxiliary block no longer read
  uint64_t* dfull = sfree + 2;            // [2] accumulator complete
  uint64_t* dempty = dfull + 2;           // [2] accumulator read by the epilogue
  uint64_t* drain = dempty + 2;           // every MMA issued has completed
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nwin = (K + BKS - 1) / BKS;    // 128-K windows
  const int nstg = (nwin + WPS - 1) / WPS;  // pipeline stages of WPS windows
  const int kscale = K / 32;

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
    tc::mbar_init(drain, 1);
    *abort_flag = 0;
    tc::fence_mbar_init();
    tc::tma_prefetch_desc(&map_w);
    tc::tma_prefetch_desc(&map_w_tail);
    tc::tma_prefetch_desc(&map_x);
  }
  if (warp == 1) {
    tc::tmem_alloc(tmem_holder, kTmemCols);
    tc::tmem_relinquish();
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  const uint32_t t_sf = tmem + 2 * BN;  // stage slot s: columns t_sf + s * kSlotCols ...

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int g = 0, it = 0;
      int s_slot = 0;          // ring slot of stage g
      uint32_t s_phase = 0;    // parity of slot s_slot's current use
      bool ok = true;
      for (int i = blockIdx.x; ok && i < n_items; i += gridDim.x, ++it) {
        const int t = i / n_mt, mt = i % n_mt;
        const Tile tile = tiles[t];
        const int b = it % NB, use = it / NB;
        // the auxiliary buffer is free once the scale writers are done with its last item
        if (use > 0 && !wait1(&sfree[b], (use - 1) & 1, abort_flag, status)) break;
        const int64_t erow = static_cast<int64_t>(tile.e) * rows_per_expert;
        uint8_t* sdst = aux + b * L.aux_bytes;
        const uint32_t wbytes = static_cast<uint32_t>(nwin) * XR * 4;
        if (GATE_UP) {
          const int f0 = mt * (BN / 2);
          const uint32_t bytes = static_cast<uint32_t>(min(BN / 2, F - f0)) * kscale;
          tc::mbar_arrive_expect_tx(&sbar[b], 2 * bytes + wbytes);
          tc::bulk_load(sdst, scales + (erow + f0) * kscale, bytes, &sbar[b]);
          tc::bulk_load(sdst + (BN / 2) * kscale, scales + (erow + F + f0) * kscale, bytes,
                        &sbar[b]);
        } else {
          const int d0 = mt * BN;
          const uint32_t bytes = static_cast<uint32_t>(min(BN, rows_per_expert - d0)) * kscale;
          tc::mbar_arrive_expect_tx(&sbar[b], bytes + wbytes);
          tc::bulk_load(sdst, scales + (erow + d0) * kscale, bytes, &sbar[b]);
        }
        tc::bulk_load(sdst + L.wsc_bytes, sfx_words + static_cast<int64_t>(t) * nwin * XR, wbytes,
                      &sbar[b]);
        const int wrow = GATE_UP ? mt * (BN / 2) : mt * BN;
        for (int st = 0; st < nstg; ++st, ++g) {
          if (g >= NS && !wait1(&empty[s_slot], s_phase ^ 1u, abort_flag, status)) {
            ok = false;
            break;
          }
          const int w0 = st * WPS;
          const int nv = min(WPS, nwin - w0);
          tc::mbar_arrive_expect_tx(&full[s_slot], nv * (W_TX + X_BYTES));
          for (int v = 0; v < nv; ++v) {
            const int w = w0 + v;
            const int k0 = stage_k0(w, K);
            uint8_t* wdst = wsm + (s_slot * WPS + v) * W_SMEM;
            if (k0 == w * BKS) {
              if (GATE_UP)
                tc::tma_load_5d(wdst, &map_w, &full[s_slot], 0, w, 0, wrow, tile.e);
              else
                tc::tma_load_4d(wdst, &map_w, &full[s_slot], 0, w, wrow, tile.e);
            } else {
              if (GATE_UP)
                tc::tma_load_4d(wdst, &map_w_tail, &full[s_slot], 0, 0, wrow, tile.e);
              else
                tc::tma_load_3d(wdst, &map_w_tail, &full[s_slot], 0, wrow, tile.e);
            }
            tc::tma_load_2d(xs + (s_slot * WPS + v) * X_BYTES, &map_x, &full[s_slot], k0, t * XR);
          }
          if (++s_slot == NS) {
            s_slot = 0;
            s_phase ^= 1u;
          }
        }
      }
      // drain: every copy this thread issued has landed before the CTA exits
      for (int gg = max(0, g - NS); gg < g; ++gg)
        tc::mbar_wait(&full[gg % NS], (gg / NS) & 1, abort_flag, kWaitLimitNs / 8);
      for (int j = max(0, it - NB); j < it; ++j)
        tc::mbar_wait(&sbar[j % NB], (j / NB) & 1, abort_flag, kWaitLimitNs / 8);
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
      const int tail_w = (K % BKS) ? nwin - 1 : nwin;  // the re-read window, if any
      for (int i = blockIdx.x; ok && i < n_items; i += gridDim.x, ++it) {
        const uint32_t d = tmem + (it & 1) * BN;
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
          // a descriptor addresses shared memory in 16-byte units: +2 per 32 bytes
#pragma unroll
          for (int v = 0; v < WPS; ++v) {
            const int w = st * WPS + v;
            if (w >= nwin) break;
            const uint64_t xv = xdesc + v * (X_BYTES >> 4), wv = wdesc + v * (W_SMEM >> 4);
            const uint32_t sv = sfa + 8 * v;
            if (w != tail_w) {
              tc::mma_mx_ss(d, xv, wv, IDESC | tc::idesc_sf_ids(0, 0), w > 0 ? 1u : 0u, sv, sv + 4);
              tc::mma_mx_ss(d, xv + 2, wv + 2, IDESC | tc::idesc_sf_ids(1, 1), 1u, sv, sv + 4);
            }
            tc::mma_mx_ss(d, xv + 4, wv + 4, IDESC | tc::idesc_sf_ids(2, 2),
                          (w != tail_w || w > 0) ? 1u : 0u, sv, sv + 4);
            tc::mma_mx_ss(d, xv + 6, wv + 6, IDESC | tc::idesc_sf_ids(3, 3), 1u, sv, sv + 4);
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
    for (int i = blockIdx.x; i < n_items; i += gridDim.x, ++it) {
      const int mt = i % n_mt;
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
        if (GATE_UP) {
          srow[c] = (n & 1) * (BN / 2) + (n >> 1);
          live[c] = mt * (BN / 2) + (n >> 1) < F;
        } else {
          srow[c] = n;
          live[c] = mt * BN + n < rows_per_expert;
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
  } else {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;                // tensor-memory lane quarter
    const int half = (warp - 6) >> 2;      // accumulator columns [64 half, 64 half + 64)
    const uint32_t lane_base = static_cast<uint32_t>(q * 32) << 16;
    const int m = q * 32 + lane;  // accumulator row: token m >> 1, piece m & 1
    const int tl = m >> 1;
    const bool lo = m & 1;
    int it = 0;
    for (int i = blockIdx.x; i < n_items; i += gridDim.x, ++it) {
      const int t = i / n_mt, mt = i % n_mt;
      const Tile tile = tiles[t];
      const int a = it & 1;
      if (!warp_wait(&dfull[a], (it >> 1) & 1, abort_flag, status, 256)) break;
      tc::tc_fence_after();
      if (16 * q < tile.nrows) {  // this quarter holds at least one real token
        const bool live_row = tl < tile.nrows;
        uint16_t* orow = out + static_cast<int64_t>(tile.row0 + tl) * out_ld;
        const uint32_t dcol = tmem + a * BN + 64 * half;
        // 16 accumulator columns starting at item column cc -> outputs
        auto finish16 = [&](const uint32_t(&r)[16], int cc) {
          // the hi lane finishes columns cc..cc+7, the lo lane cc+8..cc+15
          float sum[8];
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const float x = __uint_as_float(r[j]);
            const float y = __uint_as_float(r[8 + j]);
            const float recv = __shfl_xor_sync(0xFFFFFFFFu, lo ? x : y, 1);
            sum[j] = (lo ? y : x) + recv;
          }
          const int c0 = cc + (lo ? 8 : 0);
          if (GATE_UP) {
            // columns 2j (gate) and 2j + 1 (up) of feature mt * 64 + j
            const int f = mt * (BN / 2) + c0 / 2;
            uint32_t hw[2];
#pragma unroll
            for (int j = 0; j < 2; ++j) {
              float hv[2];
#pragma unroll
              for (int p2 = 0; p2 < 2; ++p2) {
                const float gv = sum[4 * j + 2 * p2], uv = sum[4 * j + 2 * p2 + 1];
                hv[p2] = __fdividef(gv, 1.0f + __expf(-gv)) * uv;
              }
              hw[j] = pack_bf16x2(hv[0], hv[1]);
            }
            if (live_row && f < F) *reinterpret_cast<uint2*>(orow + f) = make_uint2(hw[0], hw[1]);
          } else {
            const int dd = mt * BN + c0;
            if (live_row && dd < rows_per_expert)
              *reinterpret_cast<uint4*>(orow + dd) =
                  make_uint4(pack_bf16x2(sum[0], sum[1]), pack_bf16x2(sum[2], sum[3]),
                             pack_bf16x2(sum[4], sum[5]), pack_bf16x2(sum[6], sum[7]));
          }
        };
#pragma unroll 1
        for (int c = 0; c < 64; c += 32) {
          uint32_t ra[16], rb[16];
          tc::tmem_ld16(dcol + lane_base + c, ra);
          tc::tmem_ld16(dcol + lane_base + c + 16, rb);
          tc::tmem_ld_wait();
          finish16(ra, 64 * half + c);
          finish16(rb, 64 * half + c + 16);
        }
      }
      // this warp has read its part of the accumulator
      tc::tc_fence_before();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&dempty[a]);
    }
  }

  tc::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    // every MMA has completed (already on the normal path; bounded on abort)
    tc::mbar_wait(drain, 0, abort_flag, kWaitLimitNs / 8);
    __syncwarp();
    tc::tc_fence_after();
    tc::tmem_dealloc(tmem, kTmemCols);
  }
}

// Tile list: expert e contributes ceil(count_e / NT) tiles of up to NT rows.
__global__ void plan_tiles_kernel(const int32_t* __restrict__ offsets, int E, int NT,
                                  Tile* __restrict__ tiles, int* __restrict__ n_tiles) {
  __shared__ int base[257];
  const int e = threadIdx.x;
  int cnt = 0;
  if (e < E) {
    const int c = offsets[e + 1] - offsets[e];
    cnt = (c + NT - 1) / NT;
  }
  base[e + 1] = cnt;
  if (e == 0) base[0] = 0;
  __syncthreads();
  if (e == 0)
    for (int i = 1; i <= E; ++i) base[i] += base[i - 1];
  __syncthreads();
  if (e < E) {
    const int r0 = offsets[e], c = offsets[e + 1] - offsets[e];
    for (int t = 0; t < cnt; ++t) {
      Tile tl;
      tl.e = e;
      tl.row0 = r0 + t * NT;
      tl.nrows = min(NT, c - t * NT);
      tl.pad = 0;
      tiles[base[e] + t] = tl;
    }
  }
  if (e == 0) *n_tiles = base[E];
}

// Exact two-piece E4M3 split of bf16 rows (see the file comment), written in
// the tile-padded layout: piece rows [2 * tiles * NT][K] bytes, row 2p = hi
// and 2p + 1 = lo of padded row p = t NT + i, and, per tile and 128-K window,
// the scale words [2 NT] in the same row order (byte b of a word = E8M0 scale
// of the window's 32-element block b).  One warp per (padded row, window);
// lane l holds elements 4l..4l+3 of the window, a block is 8 lanes.  Padded
// rows get zero pieces.
__global__ void __launch_bounds__(256) split_rows_kernel(
    const uint16_t* __restrict__ src, int K, const Tile* __restrict__ tiles,
    const int* __restrict__ n_tiles, int NT, int64_t padded_rows, uint8_t* __restrict__ pieces,
    uint32_t* __restrict__ words) {
  const int nstg = (K + BKS - 1) / BKS;
  const int st = blockIdx.y;
  const int lane = threadIdx.x & 31;
  const int64_t p = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (p >= padded_rows) return;
  const int ti = static_cast<int>(p / NT), i = static_cast<int>(p % NT);
  if (ti >= __ldg(n_tiles)) return;
  const Tile tl = tiles[ti];
  const int k0 = stage_k0(st, K);
  const int k = k0 + lane * 4;
  float v[4] = {0.f, 0.f, 0.f, 0.f};
  if (i < tl.nrows) {
    const uint2 raw =
        *reinterpret_cast<const uint2*>(src + static_cast<int64_t>(tl.row0 + i) * K + k);
    v[0] = bf16_to_f32(static_cast<uint16_t>(raw.x));
    v[1] = bf16_to_f32(static_cast<uint16_t>(raw.x >> 16));
    v[2] = bf16_to_f32(static_cast<uint16_t>(raw.y));
    v[3] = bf16_to_f32(static_cast<uint16_t>(raw.y >> 16));
  }
  float amax = fmaxf(fmaxf(fabsf(v[0]), fabsf(v[1])), fmaxf(fabsf(v[2]), fabsf(v[3])));
  amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, 1));
  amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, 2));
  amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, 4));
  // block exponent floor(log2 amax) - 7 from the biased exponent field; zero
  // and subnormal blocks take the floor -123, which keeps both scale bytes >= 0
  const int ebits = static_cast<int>((__float_as_uint(amax) >> 23) & 0xFFu);
  const int t = max(ebits - 127 - 7, -123);
  const float inv = __uint_as_float(static_cast<uint32_t>(127 - t) << 23);  // 2^-t
  uint32_t hi4 = 0, lo4 = 0;
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
  // a moved-back last window re-reads [K - 128, 128 st): only its new elements are written
  if (k >= st * BKS) {
    *reinterpret_cast<uint32_t*>(pieces + (2 * p) * K + k) = hi4;
    *reinterpret_cast<uint32_t*>(pieces + (2 * p + 1) * K + k) = lo4;
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

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) !=
            cudaSuccess ||
        q != cudaDriverEntryPointSuccess) {
      cudaGetLastError();
      return static_cast<EncodeTiledFn>(nullptr);
    }
    return reinterpret_cast<EncodeTiledFn>(p);
  }();
  return fn;
}

bool encode(CUtensorMap* map, CUtensorMapDataType type, int rank, const void* base,
            const cuuint64_t* dims, const cuuint64_t* strides, const cuuint32_t* box) {
  EncodeTiledFn fn = encode_fn();
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
bool make_weight_maps(CUtensorMap* main, CUtensorMap* tail, const uint8_t* q, int E, int R,
                      int K, bool gate_up) {
  const cuuint64_t row = static_cast<cuuint64_t>(K / 2);
  const cuuint64_t mat = static_cast<cuuint64_t>(R) * row;
  const CUtensorMapDataType T = CU_TENSOR_MAP_DATA_TYPE_16U4_ALIGN16B;
  const uint8_t* tail_base = q + (K - BKS) / 2;
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

// token piece rows [2 * padded rows][K] bytes, box = 128 K x 2 NT rows
bool make_piece_map(CUtensorMap* map, const uint8_t* pieces, int64_t padded_rows, int K, int NT) {
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(2 * padded_rows)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(K)};
  const cuuint32_t box[2] = {BKS, static_cast<cuuint32_t>(2 * NT)};
  return encode(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, pieces, dims, strides, box);
}

struct GemmConfig {
  int NT, NS, NB;
};

constexpr int kMaxSmemPerCta = 227 * 1024;

int smem_bytes(int NT, int NS, int NB, int K) { return smem_layout(NT, NS, NB, K).total + 1024; }

// token-tile width: about twice the mean rows per expert, 16..64; then the
// deepest copy ring (up to 12 stages) beside a double-buffered weight-scale
// block, with at least 4 stages; failing that, a single scale block
GemmConfig choose_config(const moe_shape& sh) {
  const int64_t S = static_cast<int64_t>(sh.T) * sh.k;
  const int64_t want = 2 * ((S + sh.E - 1) / sh.E);
  int nt = 16;
  while (nt < want && nt < 64) nt *= 2;
  const int K = sh.d_model > sh.d_ff ? sh.d_model : sh.d_ff;
  for (;;) {
    for (int ns = kMaxStages; ns >= 4; --ns)
      if (smem_bytes(nt, ns, 2, K) <= kMaxSmemPerCta) return {nt, ns, 2};
    for (int ns = kMaxStages; ns >= 2; --ns)
      if (smem_bytes(nt, ns, 1, K) <= kMaxSmemPerCta) return {nt, ns, 1};
    if (nt == 16) return {16, 0, 1};  // does not fit: rejected at launch
    nt /= 2;
  }
}

template <int NT, bool GATE_UP>
moe_status launch_gemm(const GemmConfig& cfg, const CUtensorMap& mw, const CUtensorMap& mwt,
                       const CUtensorMap& mx, const uint32_t* words, const uint8_t* scales,
                       const Tile* tiles, const int* n_tiles, int max_items, int R, int K,
                       int out_ld, uint16_t* out, int32_t* status, cudaStream_t stream) {
  const int smem = smem_bytes(NT, cfg.NS, cfg.NB, K);
  if (cfg.NS < 2 || cfg.NS > kMaxStages || smem > kMaxSmemPerCta) return MOE_ERR_SHAPE;
  auto kern = grouped_mx_gemm<NT, GATE_UP>;
  static bool attr_done = false;
  if (!attr_done) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kMaxSmemPerCta) !=
        cudaSuccess) {
      cudaGetLastError();
      return MOE_ERR_CUDA;
    }
    attr_done = true;
  }
  const int grid = max_items < sm_count() ? max_items : sm_count();
  // each CTA holds all 512 tensor-memory columns: ask for enough shared
  // memory that no second CTA shares the SM
  const int smem_launch = smem > kMaxSmemPerCta / 2 + 1024 ? smem : kMaxSmemPerCta / 2 + 1024;
  kern<<<grid, kThreads, smem_launch, stream>>>(mw, mwt, mx, words, scales, tiles, n_tiles, R, K, cfg.NS,
                                         cfg.NB, out_ld, out, status);
  return launch_status();
}

template <bool GATE_UP>
moe_status launch_nt(const GemmConfig& cfg, const CUtensorMap& mw, const CUtensorMap& mwt,
                     const CUtensorMap& mx, const uint32_t* words, const uint8_t* scales,
                     const Tile* tiles, const int* n_tiles, int max_items, int R, int K, int ld,
                     uint16_t* out, int32_t* status, cudaStream_t st) {
  switch (cfg.NT) {
    case 16:
      return launch_gemm<16, GATE_UP>(cfg, mw, mwt, mx, words, scales, tiles, n_tiles, max_items,
                                      R, K, ld, out, status, st);
    case 32:
      return launch_gemm<32, GATE_UP>(cfg, mw, mwt, mx, words, scales, tiles, n_tiles, max_items,
                                      R, K, ld, out, status, st);
    default:
      return launch_gemm<64, GATE_UP>(cfg, mw, mwt, mx, words, scales, tiles, n_tiles, max_items,
                                      R, K, ld, out, status, st);
  }
}

struct MlpWs {
  size_t n_tiles, tiles, pieces, words, total;
  int64_t max_tiles, padded_rows;
};

MlpWs mlp_ws(const moe_shape& sh) {
  const int NT = choose_config(sh).NT;
  const int64_t S = static_cast<int64_t>(sh.T) * sh.k;
  const int K = sh.d_model > sh.d_ff ? sh.d_model : sh.d_ff;
  const int64_t nstg = (K + BKS - 1) / BKS;
  MlpWs w;
  w.max_tiles = sh.E + (S + NT - 1) / NT;
  w.padded_rows = w.max_tiles * NT;
  w.n_tiles = 0;
  w.tiles = 256;
  w.pieces = align_up(w.tiles + static_cast<size_t>(w.max_tiles) * sizeof(Tile), 256);
  w.words = align_up(w.pieces + 2 * static_cast<size_t>(w.padded_rows) * K, 256);
  w.total = align_up(w.words + static_cast<size_t>(w.max_tiles * nstg) * 2 * NT * 4, 256);
  return w;
}

moe_status split_launch(const uint16_t* src, int K, const Tile* tiles, const int* n_tiles, int NT,
                        const MlpWs& W, uint8_t* pieces, uint32_t* words, cudaStream_t stream) {
  const int nstg = (K + BKS - 1) / BKS;
  const int64_t blocks = (W.padded_rows + 7) / 8;  // 8 warps per block, one row each
  split_rows_kernel<<<dim3(static_cast<unsigned>(blocks), nstg), 256, 0, stream>>>(
      src, K, tiles, n_tiles, NT, W.padded_rows, pieces, words);
  return launch_status();
}

moe_status mx_launch(const uint16_t* x_perm, const int32_t* offsets, const moe_shape& sh,
                     const uint8_t* wgu_q, const uint8_t* wgu_s, const uint8_t* wdn_q,
                     const uint8_t* wdn_s, uint16_t* h, uint16_t* y_perm, void* ws,
                     int32_t* status, cudaStream_t stream) {
  if (sh.T == 0) return MOE_OK;
  const GemmConfig cfg = choose_config(sh);
  if (cfg.NS < 2) return MOE_ERR_SHAPE;
  const int NT = cfg.NT;
  const MlpWs W = mlp_ws(sh);
  char* base = static_cast<char*>(ws);
  int* n_tiles = reinterpret_cast<int*>(base + W.n_tiles);
  Tile* tiles = reinterpret_cast<Tile*>(base + W.tiles);
  uint8_t* pieces = reinterpret_cast<uint8_t*>(base + W.pieces);
  uint32_t* words = reinterpret_cast<uint32_t*>(base + W.words);
  const int max_tiles = static_cast<int>(W.max_tiles);
  const int D = sh.d_model, F = sh.d_ff, E = sh.E;

  CUtensorMap m_gu, m_gu_t, m_dn, m_dn_t, m_x, m_h;
  if (!make_weight_maps(&m_gu, &m_gu_t, wgu_q, E, 2 * F, D, true) ||
      !make_weight_maps(&m_dn, &m_dn_t, wdn_q, E, D, F, false) ||
      !make_piece_map(&m_x, pieces, W.padded_rows, D, NT) ||
      !make_piece_map(&m_h, pieces, W.padded_rows, F, NT))
    return MOE_ERR_CUDA;

  plan_tiles_kernel<<<1, 256, 0, stream>>>(offsets, E, NT, tiles, n_tiles);
  moe_status st = launch_status();
  if (st != MOE_OK) return st;
  if ((st = split_launch(x_perm, D, tiles, n_tiles, NT, W, pieces, words, stream)) != MOE_OK)
    return st;
  const int mt_gu = (F + BN / 2 - 1) / (BN / 2), mt_dn = (D + BN - 1) / BN;
  st = launch_nt<true>(cfg, m_gu, m_gu_t, m_x, words, wgu_s, tiles, n_tiles, max_tiles * mt_gu,
                       2 * F, D, F, h, status, stream);
  if (st != MOE_OK) return st;
  if ((st = split_launch(h, F, tiles, n_tiles, NT, W, pieces, words, stream)) != MOE_OK) return st;
  return launch_nt<false>(cfg, m_dn, m_dn_t, m_h, words, wdn_s, tiles, n_tiles, max_tiles * mt_dn,
                          D, F, D, y_perm, status, stream);
}

// Shapes with few routed rows per expert (decode) stream the weights once per
// small token tile and are bound by HBM: they take the block-scaled path
// above, which moves the codes straight into the tensor core.  Token-heavy
// shapes (prefill) are bound by the tensor core and take the decode-to-bf16
// path, whose 2-CTA-per-SM pipeline with 256-token tiles keeps it busier.
bool native_path(const moe_shape& sh) {
  const int64_t S = static_cast<int64_t>(sh.T) * sh.k;
  return 2 * ((S + sh.E - 1) / sh.E) <= 64;
}

}  // namespace

size_t expert_mlp_bf16_workspace(const moe_shape& sh);
moe_status expert_mlp_bf16_launch(const uint16_t* x_perm, const int32_t* offsets,
                                  const moe_shape& sh, const uint8_t* wgu_q, const uint8_t* wgu_s,
                                  const uint8_t* wdn_q, const uint8_t* wdn_s, uint16_t* h,
                                  uint16_t* y_perm, void* ws, int32_t* status,
                                  cudaStream_t stream);

size_t expert_mlp_workspace(const moe_shape& sh) {
  return native_path(sh) ? mlp_ws(sh).total : expert_mlp_bf16_workspace(sh);
}

moe_status expert_mlp_launch(const uint16_t* x_perm, const int32_t* offsets, const moe_shape& sh,
                             const uint8_t* wgu_q, const uint8_t* wgu_s, const uint8_t* wdn_q,
                             const uint8_t* wdn_s, uint16_t* h, uint16_t* y_perm, void* ws,
                             int32_t* status, cudaStream_t stream) {
  if (native_path(sh))
    return mx_launch(x_perm, offsets, sh, wgu_q, wgu_s, wdn_q, wdn_s, h, y_perm, ws, status,
                     stream);
  return expert_mlp_bf16_launch(x_perm, offsets, sh, wgu_q, wgu_s, wdn_q, wdn_s, h, y_perm, ws,
                                status, stream);
}

}  // namespace moe
