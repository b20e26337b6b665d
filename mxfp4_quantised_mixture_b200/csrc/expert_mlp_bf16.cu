// Grouped SwiGLU expert MLP on MXFP4 weights, decode-to-bf16 variant: the
// path taken for token-heavy (prefill) shapes, where the GEMMs are bound by
// the tensor core rather than by streaming the weights.
//
// "Welcome GPT OSS ..." (summary), section 4: SwiGLU experts;
// "Tricks from OpenAI gpt-oss ..." (summary), sections 6 and 8: E2M1 weights
// with one shared scale per 32 elements, and GEMMs that read those blocks and
// scales directly; aitrends.kr talk summary, "Hardware optimisation": the
// weights stay 4-bit in memory and are raised to higher precision only for
// the arithmetic.
//
// One kernel template runs both GEMMs of the MLP.  A CTA owns one tile:
// 128 weight rows (the MMA's M side) x up to NT routed token rows of one
// expert (the N side) x the whole reduction axis K, in stages of BK = 64.
//   * gate/up: the 128 rows are 64 gate rows and the matching 64 up rows,
//     interleaved in tensor memory (lane 2j = gate j, lane 2j+1 = up j), so
//     the SwiGLU epilogue pairs neighbouring lanes; output h [S][F] bf16.
//   * down: 128 rows of the [D][F] matrix; output y_perm [S][D] bf16.
// Warp roles (4 + 4 * decode groups warps; 3 groups for tiles of up to 64
// rows, which run two CTAs per SM, 4 for wider tiles):
//   warp 0       weight producer: the tile's E8M0 scale bytes (one bulk
//                copy) and per stage the packed codes (TMA, 4 KB) into a
//                ring of 8 or 9 stages released by the decoders
//   warp 1       token producer and tensor-memory owner: per stage NT token
//                rows x 64 bf16 (TMA, 128-byte swizzle) into slot j of a ring
//                whose slot j pairs with A slot j in tensor memory
//   warps 2, 3   MMA issuers (two for tiles of 32 and 128 rows, else one),
//                taking stages round-robin into one fp32 accumulator each in
//                tensor memory (D0, D1); one commit per stage frees both the
//                token slot and the A slot.  One thread issues an M=128,
//                N<=64 MMA only every ~50 cycles and a commit costs a few
//                hundred, so a second issuer helps where the MMAs are short.
//   warpgroups   decoders, taking stages round-robin: each thread owns one
//                weight row (its tensor-memory lane), turns 64 codes per
//                stage into exact bf16 and writes them to the stage's A slot;
//                after the K loop they add D0 + D1 and run the epilogue.
// Decode: code nibble s|m2|m1|m0 is placed as the bf16 bit pattern
// s<<15 | m2<<8 | m1<<7 | m0<<6, which is the E2M1 value times 2^-126 (code 1
// lands on the subnormal 2^-127); two byte-table permutes build the high and
// low bytes and two more interleave them, then one bf16x2 multiply by
// 2^(b-1) applies the block scale 2^(b-127).  Every decoded weight is the
// exact value of the MXFP4 element, so the tensor-core products are exact and
// only the fp32 accumulation order differs from a sequential sum.
// Every wait on a barrier is bounded (2 s); on expiry the kernel records
// MOE_ERR_TIMEOUT in the status word, drains its copies and returns.
#include <cuda.h>

#include <atomic>

#include "common.cuh"
#include "mlp_plan.cuh"
#include "tc_sm100.cuh"

namespace moe {
namespace {

constexpr int BK = 64;                // K elements per pipeline stage
constexpr int BM = 128;               // weight rows per tile (MMA M)
constexpr int W_STAGE = BM * BK / 2;  // packed code bytes per stage
constexpr int kDecWarp0 = 4;
constexpr uint64_t kWaitLimitNs = 2000000000ull;
constexpr uint64_t kTestWaitNs = 200000ull;  // the injected wait of test_timeout_cta

// Per token-tile width: decode groups, MMA issuers, token/A slot pairs and
// weight-ring depth.  Tensor memory holds NMMA accumulators of NT columns
// plus the A slots (32 columns each); narrow tiles run two CTAs per SM (256
// columns each), wide ones one.
// An mbarrier waiter names a phase by its parity alone, so it must never
// wait on a phase two ahead of the barrier's current one (the parity would
// match the phase before, already complete).  Every waiter below therefore
// sees every phase of each barrier it waits on: a weight stage and a slot
// pair always go to the same decode group (ring depths multiples of the
// group count) and a slot pair always to the same MMA issuer.
__host__ __device__ constexpr int groups_for(int NT) { return NT <= 64 ? 3 : 4; }
__host__ __device__ constexpr int threads_for(int NT) { return 32 * (kDecWarp0 + 4 * groups_for(NT)); }
__host__ __device__ constexpr int issuers_for(int NT) { return (NT == 32 || NT == 128) ? 2 : 1; }
__host__ __device__ constexpr int slots_for(int NT) {
  return NT <= 64 ? 6 : (NT == 128 ? 8 : 4);
}
__host__ __device__ constexpr int nsw_for(int NT) { return NT <= 64 ? 9 : 8; }
__host__ __device__ constexpr int tmem_cols_for(int NT) {
  return issuers_for(NT) * NT + slots_for(NT) * 32 <= 256 ? 256 : 512;
}

struct SmemLayout {
  int x_off, w_off, s_off, bar_off, total;
};

__host__ __device__ inline SmemLayout smem_layout(int NT, int K) {
  SmemLayout L;
  L.x_off = 0;
  L.w_off = L.x_off + slots_for(NT) * NT * 128;
  L.s_off = L.w_off + nsw_for(NT) * W_STAGE;
  L.bar_off = L.s_off + ((BM * (K / 32) + 127) / 128) * 128;
  L.total = L.bar_off + 512;
  return L;
}

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
  return d;
}

__device__ __forceinline__ uint32_t mul_bf16x2(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

// 8 codes (one word: element i in bits 4i..4i+3) -> 4 words of bf16 pairs,
// each the element value times 2^-126 (see the file comment)
__device__ __forceinline__ void decode8_raw(uint32_t w, uint32_t* o) {
  constexpr uint32_t kLowBytes = 0xC0804000u;   // m1m0 = 0..3 -> 0x00,0x40,0x80,0xC0
  constexpr uint32_t kHighBytes = 0x81800100u;  // s m2 = 0..3 -> 0x00,0x01,0x80,0x81
  const uint32_t sel_lo = w & 0x33333333u;
  const uint32_t sel_hi = (w >> 2) & 0x33333333u;
  const uint32_t lo_a = prmt(kLowBytes, 0u, sel_lo);
  const uint32_t hi_a = prmt(kHighBytes, 0u, sel_hi);
  const uint32_t lo_b = prmt(kLowBytes, 0u, sel_lo >> 16);
  const uint32_t hi_b = prmt(kHighBytes, 0u, sel_hi >> 16);
  o[0] = prmt(lo_a, hi_a, 0x5140u);
  o[1] = prmt(lo_a, hi_a, 0x7362u);
  o[2] = prmt(lo_b, hi_b, 0x5140u);
  o[3] = prmt(lo_b, hi_b, 0x7362u);
}

// 32 codes (4 words) under scale byte sb -> 16 words of exact bf16 pairs
__device__ __forceinline__ void decode32(const uint4& p, uint32_t sb, uint32_t (&o)[16]) {
  decode8_raw(p.x, o + 0);
  decode8_raw(p.y, o + 4);
  decode8_raw(p.z, o + 8);
  decode8_raw(p.w, o + 12);
  if (sb <= 128u) {
    // 2^(sb-1) has exponent field sb+126 in [126, 254]
    const uint32_t m = (sb + 126u) << 7;
    const uint32_t m2 = m | (m << 16);
#pragma unroll
    for (int i = 0; i < 16; ++i) o[i] = mul_bf16x2(o[i], m2);
  } else {
    // two exact steps: *2^126 gives the plain E2M1 values, then *2^(sb-127)
    const uint32_t c = (126u + 127u) << 7;
    const uint32_t c2 = c | (c << 16);
    const uint32_t m = sb << 7;
    const uint32_t m2 = m | (m << 16);
#pragma unroll
    for (int i = 0; i < 16; ++i) o[i] = mul_bf16x2(mul_bf16x2(o[i], c2), m2);
  }
}

__device__ __forceinline__ void abort_cta(volatile int* abort, int32_t* status) {
  *abort = 1;
  record_status(status, MOE_ERR_TIMEOUT);
}

__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, const volatile int* abort) {
  const bool r = tc::mbar_wait(bar, parity, abort, kWaitLimitNs);
  return __all_sync(0xFFFFFFFFu, r);
}

template <int NT, bool GATE_UP>
__global__ void __launch_bounds__(threads_for(NT), NT <= 64 ? 2 : 1)  // two CTAs per SM for narrow tiles
    grouped_mxfp4_gemm(const __grid_constant__ CUtensorMap map_w,
                       const __grid_constant__ CUtensorMap map_x, const uint8_t* __restrict__ scales,
                       const Tile* __restrict__ tiles, const int* __restrict__ n_tiles,
                       int rows_per_expert, int K, int out_ld, uint16_t* __restrict__ out,
                       int32_t* __restrict__ status, int fail_cta) {
  constexpr int NA = slots_for(NT);
  constexpr int NMMA = issuers_for(NT);
  constexpr int NSW = nsw_for(NT);
  constexpr int DG = groups_for(NT);
  static_assert(NSW % DG == 0 && NA % DG == 0 && NA % NMMA == 0, "slot owners");
  static_assert(NT > 64 || tmem_cols_for(NT) == 256, "two CTAs per SM share tensor memory");
  constexpr int X_STAGE = NT * 128;
  constexpr int TMEM_COLS = tmem_cols_for(NT);
  // a CTA beyond the tile count leaves before any set-up
  if (static_cast<int>(blockIdx.y) >= __ldg(n_tiles)) return;

  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const SmemLayout L = smem_layout(NT, K);
  uint8_t* xs = smem + L.x_off;
  uint8_t* wsm = smem + L.w_off;
  uint8_t* ssm = smem + L.s_off;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L.bar_off);
  uint64_t* wfull = bars;              // [NSW] weight codes landed
  uint64_t* wempty = wfull + NSW;      // [NSW] weight codes read by the decoders
  uint64_t* xfull = wempty + NSW;      // [NA]  token rows landed
  uint64_t* afull = xfull + NA;        // [NA]  A slot written by the decoders
  uint64_t* consumed = afull + NA;     // [NA]  MMA done with token slot + A slot
  uint64_t* sbar = consumed + NA;      // scales landed
  uint64_t* dfull = sbar + 1;          // accumulators complete (one commit per issuer)
  uint64_t* never = dfull + 1;         // completed by nothing (the injected test wait)
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(never + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const Tile tile = tiles[blockIdx.y];
  // the MMAs cover the tile's rows rounded up to 16, not the whole width: a
  // ragged tile (an expert's last, or a cold expert's only) costs the tensor
  // core only its own rows
  const int NV = min(NT, (tile.nrows + 15) & ~15);
  const uint32_t IDESC = tc::idesc_bf16_f32(BM, NV);
  const int mt = blockIdx.x;
  const int KB = K / BK;
  const int kscale = K / 32;

  if (threadIdx.x == 0) {
    for (int s = 0; s < NSW; ++s) {
      tc::mbar_init(&wfull[s], 1);
      tc::mbar_init(&wempty[s], 4);
    }
    for (int j = 0; j < NA; ++j) {
      tc::mbar_init(&xfull[j], 1);
      tc::mbar_init(&afull[j], 4);
      tc::mbar_init(&consumed[j], 1);
    }
    tc::mbar_init(sbar, 1);
    tc::mbar_init(dfull, NMMA);
    tc::mbar_init(never, 1);
    *abort_flag = 0;
    tc::fence_mbar_init();
    tc::tma_prefetch_desc(&map_w);
    tc::tma_prefetch_desc(&map_x);
  }
  if (warp == 1) {
    tc::tmem_alloc(tmem_holder, TMEM_COLS);
    tc::tmem_relinquish();
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  const uint32_t tmem_a = tmem + NMMA * NT;  // A slots follow the accumulators

  if (warp == 0) {
    // -------------------------------------------------- weight producer
    if (lane == 0) {
      const int r0 = GATE_UP ? mt * 64 : mt * BM;
      const int64_t srow = static_cast<int64_t>(tile.e) * rows_per_expert;
      if (GATE_UP) {
        const uint32_t half = 64u * kscale;
        tc::mbar_arrive_expect_tx(sbar, 2 * half);
        const int F = rows_per_expert / 2;
        tc::bulk_load(ssm, scales + (srow + r0) * kscale, half, sbar);
        tc::bulk_load(ssm + half, scales + (srow + F + r0) * kscale, half, sbar);
      } else {
        const uint32_t bytes = static_cast<uint32_t>(min(BM, rows_per_expert - r0)) * kscale;
        tc::mbar_arrive_expect_tx(sbar, bytes);
        tc::bulk_load(ssm, scales + (srow + r0) * kscale, bytes, sbar);
      }
      int issued = 0;
      for (int kb = 0; kb < KB; ++kb) {
        const int s = kb % NSW, n = kb / NSW;
        if (n > 0 && !tc::mbar_wait(&wempty[s], (n - 1) & 1, abort_flag, kWaitLimitNs)) {
          abort_cta(abort_flag, status);
          break;
        }
        tc::mbar_arrive_expect_tx(&wfull[s], W_STAGE);
        uint8_t* wdst = wsm + s * W_STAGE;
        if (GATE_UP) {
          // the gate rows and the matching up rows in one copy (gate block first)
          tc::tma_load_4d(wdst, &map_w, &wfull[s], kb * (BK / 2), r0, 0, tile.e);
        } else {
          tc::tma_load_3d(wdst, &map_w, &wfull[s], kb * (BK / 2), r0, tile.e);
        }
        ++issued;
      }
      // drain: every copy this thread issued has landed before the CTA exits
      for (int kb = max(0, issued - NSW); kb < issued; ++kb)
        tc::mbar_drain(&wfull[kb % NSW], (kb / NSW) & 1, kWaitLimitNs / 8);
      tc::mbar_drain(sbar, 0, kWaitLimitNs / 8);
    }
  } else if (warp == 1) {
    // --------------------------------------------------- token producer
    if (lane == 0) {
      int issued = 0;
      for (int kb = 0; kb < KB; ++kb) {
        const int j = kb % NA, n = kb / NA;
        if (n > 0 && !tc::mbar_wait(&consumed[j], (n - 1) & 1, abort_flag, kWaitLimitNs)) {
          abort_cta(abort_flag, status);
          break;
        }
        tc::mbar_arrive_expect_tx(&xfull[j], X_STAGE);
        tc::tma_load_2d(xs + j * X_STAGE, &map_x, &xfull[j], kb * BK, tile.row0);
        ++issued;
      }
      for (int kb = max(0, issued - NA); kb < issued; ++kb)
        tc::mbar_drain(&xfull[kb % NA], (kb / NA) & 1, kWaitLimitNs / 8);
    }
  } else if (warp < kDecWarp0) {
    // ---------------------------------------------------------- MMA issuers
    const int mi = warp - 2;  // this issuer's stages: kb = mi, mi + NMMA, ...
    if (lane == 0 && mi < NMMA) {
      const uint32_t tmem_d = tmem + mi * NT;
      int done = 0;
      bool ok = true;
      // testing only: the first wait of this CTA's first issuer waits on a
      // barrier that nothing completes, with a short limit, and gives up as a
      // timeout would
      if (mi == 0 && static_cast<int>(blockIdx.y * gridDim.x + blockIdx.x) == fail_cta &&
          !tc::mbar_wait(never, 0, abort_flag, kTestWaitNs)) {
        abort_cta(abort_flag, status);
        ok = false;
      }
      for (int kb = mi; ok && kb < KB; kb += NMMA) {
        const int j = kb % NA;
        const uint32_t par = (kb / NA) & 1;
        if (!tc::mbar_wait(&xfull[j], par, abort_flag, kWaitLimitNs) ||
            !tc::mbar_wait(&afull[j], par, abort_flag, kWaitLimitNs)) {
          abort_cta(abort_flag, status);
          break;
        }
        tc::tc_fence_after();
        const uint64_t bdesc = tc::smem_desc_sw128(tc::smem_u32(xs + j * X_STAGE));
#pragma unroll
        for (int i = 0; i < BK / 16; ++i)
          tc::mma_bf16_ts(tmem_d, tmem_a + j * 32 + i * 8, bdesc + static_cast<uint64_t>(i * 2),
                          IDESC, (done | i) != 0);
        tc::mma_commit(&consumed[j]);
        ++done;
      }
      // completes once every MMA this thread issued has finished (also on
      // abort); an issuer with no stage (K = 64) only arrives
      if (done > 0)
        tc::mma_commit(dfull);
      else
        tc::mbar_arrive(dfull);
    }
  } else {
    // ----------------------------------------------------------- decoders
    const int g = (warp - kDecWarp0) >> 2;  // decode group
    const int q = warp & 3;                 // tensor-memory lane quarter of this warp
    const int m = q * 32 + lane;            // tensor-memory lane = weight row in tile
    int wrow, srow_s, rot;
    if (GATE_UP) {
      wrow = (m & 1) * (W_STAGE / 2) + (m >> 1) * (BK / 2);
      srow_s = (m & 1) * 64 + (m >> 1);
      rot = m & 1;
    } else {
      wrow = m * (BK / 2);
      srow_s = m;
      rot = (m >> 2) & 1;
    }
    const uint32_t lane_base = static_cast<uint32_t>(q * 32) << 16;
    bool ok = warp_wait(sbar, 0, abort_flag);
    if (!ok) abort_cta(abort_flag, status);
    // rows past the end of the expert's matrix (last down tile) read no scales
    const bool row_live = GATE_UP || (mt * BM + m < rows_per_expert);
    const uint8_t* my_scales = ssm + srow_s * kscale;
    for (int kb = g; ok && kb < KB; kb += DG) {
      const int s = kb % NSW, j = kb % NA;
      if (!warp_wait(&wfull[s], (kb / NSW) & 1, abort_flag)) {
        abort_cta(abort_flag, status);
        ok = false;
        break;
      }
      const uint8_t* src = wsm + s * W_STAGE + wrow;
      // read the two 16-byte halves in an order that spreads the 8 lanes of
      // each quarter-warp phase over all 32 banks
      const uint4 first = *reinterpret_cast<const uint4*>(src + 16 * rot);
      const uint4 second = *reinterpret_cast<const uint4*>(src + 16 * (rot ^ 1));
      const uint4 p0 = rot ? second : first;
      const uint4 p1 = rot ? first : second;
      uint32_t s0 = 127u, s1 = 127u;
      if (row_live) {
        s0 = my_scales[2 * kb];
        s1 = my_scales[2 * kb + 1];
      }
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&wempty[s]);
      uint32_t o0[16], o1[16];
      decode32(p0, s0, o0);
      decode32(p1, s1, o1);
      const int use = kb / NA;
      if (use > 0 && !warp_wait(&consumed[j], (use - 1) & 1, abort_flag)) {
        abort_cta(abort_flag, status);
        ok = false;
        break;
      }
      tc::tc_fence_after();
      tc::tmem_st16(tmem_a + lane_base + j * 32, o0);
      tc::tmem_st16(tmem_a + lane_base + j * 32 + 16, o1);
      tc::tmem_st_wait();
      tc::tc_fence_before();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&afull[j]);
    }
    // ---------------------------------------------------------- epilogue
    ok = ok && warp_wait(dfull, 0, abort_flag) && *abort_flag == 0;
    const int used = KB < NMMA ? KB : NMMA;  // accumulators that hold a partial sum
    if (ok) {
      tc::tc_fence_after();
      uint8_t* stg = xs;  // every token slot has been consumed: reuse as staging
      for (int c = g * 16; c < NV; c += 16 * DG) {
        float v[16];
        uint32_t r[16];
        tc::tmem_ld16(tmem + lane_base + c, r);
        tc::tmem_ld_wait();
#pragma unroll
        for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
        if (used > 1) {
          tc::tmem_ld16(tmem + NT + lane_base + c, r);
          tc::tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 16; ++i) v[i] += __uint_as_float(r[i]);  // D0 + D1, fixed order
        }
        if (GATE_UP) {
          // even lane: gate row f, odd lane: up row f (f = m >> 1); the even
          // lane finishes tokens c..c+7, the odd lane tokens c+8..c+15
          const bool up = m & 1;
          uint16_t hv[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const float send = up ? v[i] : v[8 + i];
            const float recv = __shfl_xor_sync(0xFFFFFFFFu, send, 1);
            const float gv = up ? recv : v[i];
            const float uv = up ? v[8 + i] : recv;
            const float silu = gv / (1.0f + expf(-gv));
            hv[i] = f32_to_bf16_rne(silu * uv);
          }
          const int f = m >> 1;
          const int t0 = c + (up ? 8 : 0);
          uint16_t* st16 = reinterpret_cast<uint16_t*>(stg);
#pragma unroll
          for (int i = 0; i < 8; ++i) st16[(t0 + i) * 64 + f] = hv[i];
        } else {
          uint16_t* st16 = reinterpret_cast<uint16_t*>(stg);
#pragma unroll
          for (int i = 0; i < 16; ++i) st16[(c + i) * BM + m] = f32_to_bf16_rne(v[i]);
        }
      }
    }
    // all decoder warps meet before the coalesced stores
    asm volatile("bar.sync 1, %0;" ::"r"(128 * DG));
    if (ok && !*abort_flag) {
      const int tid = threadIdx.x - kDecWarp0 * 32;
      const int nthr = 128 * DG;
      if (GATE_UP) {
        // h rows: 64 features (128 bytes = 8 x 16 B) per token
        const int f0 = mt * 64;
        for (int i = tid; i < tile.nrows * 8; i += nthr) {
          const int t = i >> 3, v = i & 7;
          const uint4 val = reinterpret_cast<const uint4*>(xs + t * 128)[v];
          *reinterpret_cast<uint4*>(out + static_cast<int64_t>(tile.row0 + t) * out_ld + f0 +
                                    v * 8) = val;
        }
      } else {
        const int d0 = mt * BM;
        const int nv = min(BM, rows_per_expert - d0) / 8;  // 16-byte vectors per token row
        for (int i = tid; i < tile.nrows * 16; i += nthr) {
          const int t = i >> 4, v = i & 15;
          if (v >= nv) continue;
          const uint4 val = reinterpret_cast<const uint4*>(xs + t * (BM * 2))[v];
          *reinterpret_cast<uint4*>(out + static_cast<int64_t>(tile.row0 + t) * out_ld + d0 +
                                    v * 8) = val;
        }
      }
    }
  }

  tc::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    // the accumulator barrier completes once every issued MMA has finished
    // (already observed on the normal path)
    tc::mbar_drain(dfull, 0, kWaitLimitNs / 8);
    __syncwarp();
    tc::tc_fence_after();
    tc::tmem_dealloc(tmem, TMEM_COLS);
  }
}


// ------------------------------------------------------------ host helpers

// packed codes [E][R][K/2] bytes.  Down: box = (BK/2 bytes, 128 rows, 1
// expert).  Gate/up (R = 2F): box = (BK/2 bytes, 64 rows, gate and up half,
// 1 expert), landing as 64 gate rows then the matching 64 up rows.
bool make_weight_map(CUtensorMap* map, const uint8_t* q, int E, int R, int K, bool gate_up) {
  EncodeTiledFn fn = encode_tiled_fn();
  if (!fn) return false;
  const cuuint64_t row = static_cast<cuuint64_t>(K / 2);
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  if (gate_up) {
    const cuuint64_t F = static_cast<cuuint64_t>(R / 2);
    const cuuint64_t dims[4] = {row, F, 2, static_cast<cuuint64_t>(E)};
    const cuuint64_t strides[3] = {row, F * row, static_cast<cuuint64_t>(R) * row};
    const cuuint32_t box[4] = {BK / 2, 64, 2, 1};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 4, const_cast<uint8_t*>(q), dims, strides, box,
              estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
  }
  const cuuint64_t dims[3] = {row, static_cast<cuuint64_t>(R), static_cast<cuuint64_t>(E)};
  const cuuint64_t strides[2] = {row, static_cast<cuuint64_t>(R) * row};
  const cuuint32_t box[3] = {BK / 2, static_cast<cuuint32_t>(BM), 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<uint8_t*>(q), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// token rows [rows][K] bf16, box = (BK elements, NT rows), 128-byte swizzle
bool make_token_map(CUtensorMap* map, const uint16_t* x, int64_t rows, int K, int NT) {
  EncodeTiledFn fn = encode_tiled_fn();
  if (!fn) return false;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(rows)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(K) * 2};
  const cuuint32_t box[2] = {BK, static_cast<cuuint32_t>(NT)};
  const cuuint32_t estr[2] = {1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<uint16_t*>(x), dims, strides,
            box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// token-tile width: about twice the mean rows per expert, 32..256
int choose_nt(const moe_shape& sh) {
  const int64_t S = static_cast<int64_t>(sh.T) * sh.k;
  const int64_t want = 2 * ((S + sh.E - 1) / sh.E);
  int nt = 32;
  while (nt < want && nt < 256) nt *= 2;
  // the tile must fit shared memory together with the scale bytes of K
  const int K = sh.d_model > sh.d_ff ? sh.d_model : sh.d_ff;
  while (nt > 32 && smem_layout(nt, K).total + 1024 > 227 * 1024) nt /= 2;
  return nt;
}

// The dynamic shared-memory opt-in of both kernels of a tile width, once per
// device.
template <int NT>
bool prepare_gemm() {
  static std::atomic<uint64_t> done{0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return false;
  }
  const uint64_t bit = dev < 64 ? (uint64_t(1) << dev) : 0;
  if (bit && (done.load() & bit)) return true;
  if (cudaFuncSetAttribute(grouped_mxfp4_gemm<NT, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           227 * 1024) != cudaSuccess ||
      cudaFuncSetAttribute(grouped_mxfp4_gemm<NT, false>,
                           cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024) != cudaSuccess) {
    cudaGetLastError();
    return false;
  }
  done.fetch_or(bit);
  return true;
}

bool prepare_nt(int NT) {
  switch (NT) {
    case 32:
      return prepare_gemm<32>();
    case 64:
      return prepare_gemm<64>();
    case 128:
      return prepare_gemm<128>();
    default:
      return prepare_gemm<256>();
  }
}

template <int NT, bool GATE_UP>
moe_status launch_gemm(const CUtensorMap& mw, const CUtensorMap& mx, const uint8_t* scales,
                       const Tile* tiles, const int* n_tiles, int grid_x, int grid_y, int R, int K,
                       int out_ld, uint16_t* out, int32_t* status, int fail_cta,
                       cudaStream_t stream) {
  const int smem = smem_layout(NT, K).total + 1024;
  return launch(grouped_mxfp4_gemm<NT, GATE_UP>, dim3(grid_x, grid_y), dim3(threads_for(NT)), smem,
                stream, mw, mx, scales, tiles, n_tiles, R, K, out_ld, out, status,
                fail_cta);
}

template <bool GATE_UP>
moe_status launch_nt(int NT, const CUtensorMap& mw, const CUtensorMap& mx, const uint8_t* scales,
                     const Tile* tiles, const int* n_tiles, int gx, int gy, int R, int K, int ld,
                     uint16_t* out, int32_t* status, int fail_cta, cudaStream_t st) {
  switch (NT) {
    case 32:
      return launch_gemm<32, GATE_UP>(mw, mx, scales, tiles, n_tiles, gx, gy, R, K, ld, out,
                                      status, fail_cta, st);
    case 64:
      return launch_gemm<64, GATE_UP>(mw, mx, scales, tiles, n_tiles, gx, gy, R, K, ld, out,
                                      status, fail_cta, st);
    case 128:
      return launch_gemm<128, GATE_UP>(mw, mx, scales, tiles, n_tiles, gx, gy, R, K, ld, out,
                                       status, fail_cta, st);
    default:
      return launch_gemm<256, GATE_UP>(mw, mx, scales, tiles, n_tiles, gx, gy, R, K, ld, out,
                                       status, fail_cta, st);
  }
}

// Workspace of this path: the tile count and the tile list.
struct BfWs {
  size_t n_tiles, tiles, total;
  int64_t max_tiles;
};

BfWs bf_ws(const moe_shape& sh) {
  const int NT = choose_nt(sh);
  const int64_t S = static_cast<int64_t>(sh.T) * sh.k;
  BfWs w;
  w.max_tiles = sh.E + (S + NT - 1) / NT;
  w.n_tiles = 0;
  w.tiles = 256;
  w.total = align_up(w.tiles + static_cast<size_t>(w.max_tiles) * sizeof(Tile), 256);
  return w;
}

}  // namespace

int bf_tile_width(const moe_shape& sh) { return choose_nt(sh); }
size_t bf_workspace(const moe_shape& sh) { return bf_ws(sh).total; }

moe_status bf_plan(MlpPlan* p, void* ws) {
  const moe_shape& sh = p->sh;
  const int NT = choose_nt(sh);
  const int K = sh.d_model > sh.d_ff ? sh.d_model : sh.d_ff;
  if (smem_layout(NT, K).total + 1024 > 227 * 1024) return MOE_ERR_SHAPE;
  const BfWs W = bf_ws(sh);
  char* base = static_cast<char*>(ws);
  BfPlan& P = p->bf;
  P.NT = NT;
  P.max_tiles = W.max_tiles;
  p->n_tiles = reinterpret_cast<int*>(base + W.n_tiles);
  p->tiles = reinterpret_cast<Tile*>(base + W.tiles);
  const int64_t S = static_cast<int64_t>(sh.T) * sh.k;
  const int D = sh.d_model, F = sh.d_ff, E = sh.E;
  if (!make_weight_map(&P.m_gu, p->wgu_q, E, 2 * F, D, true) ||
      !make_token_map(&P.m_x, p->x_perm, S, D, NT) ||
      !make_weight_map(&P.m_dn, p->wdn_q, E, D, F, false) || !make_token_map(&P.m_h, p->h, S, F, NT))
    return MOE_ERR_CUDA;
  if (!prepare_nt(NT)) return MOE_ERR_CUDA;
  return MOE_OK;
}

moe_status bf_enqueue(const MlpPlan& p, const MlpInput& in, int32_t* status, int fail_cta,
                      cudaStream_t stream) {
  const BfPlan& P = p.bf;
  const moe_shape& sh = p.sh;
  const int NT = P.NT, D = sh.d_model, F = sh.d_ff, E = sh.E;
  const int max_tiles = static_cast<int>(P.max_tiles);
  moe_status st;
  if (!in.tiles_ready &&
      (st = plan_tiles_launch(in.offsets, E, NT, p.tiles, p.n_tiles, p.sched, p.n_sched, stream)) != MOE_OK)
    return st;
  st = launch_nt<true>(NT, P.m_gu, P.m_x, p.wgu_s, p.tiles, p.n_tiles, F / 64, max_tiles, 2 * F,
                       D, F, p.h, status, fail_cta, stream);
  if (st != MOE_OK) return st;
  return launch_nt<false>(NT, P.m_dn, P.m_h, p.wdn_s, p.tiles, p.n_tiles, (D + BM - 1) / BM,
                          max_tiles, D, F, D, p.y_perm, status, -1, stream);
}

}  // namespace moe
