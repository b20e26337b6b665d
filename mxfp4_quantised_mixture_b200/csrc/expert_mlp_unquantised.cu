// Grouped SwiGLU expert MLP on unquantised bf16 weights: the comparison
// point for the MXFP4 path.
//
// "Tricks from OpenAI gpt-oss you can use with transformers" (summary),
// section 7: without MXFP4 support the experts are held in bf16, at about
// four times the memory; agentlenshq "Transformers ... GPT-OSS" (ja), "What is
// MXFP4": the same comparison.  "Welcome GPT OSS ..." (summary), section 4:
// SwiGLU experts.
//
// The same grouped GEMMs as the MXFP4 paths with the weight decode taken out:
// the weight tiles arrive by TMA as bf16, already in the layout the tensor
// core reads.  A CTA owns one tile: 128 weight rows (the MMA's M side) x up to
// NT routed token rows of one expert (N) x the whole reduction axis K, in
// stages of 64 (one 128-byte swizzle row of bf16).
//   * gate/up: the 128 rows are 64 gate rows and the matching 64 up rows,
//     interleaved by the copy's box order (row 2j = gate j, 2j + 1 = up j), so
//     the SwiGLU epilogue pairs neighbouring lanes; output h [S][F] bf16.
//   * down: 128 rows of the [D][F] matrix; output y_perm [S][D] bf16.
// Warp roles (6 warps):
//   warp 0      producer: per stage the weight tile (16 KB) and the token
//               rows (NT x 128 B), both by TMA into one ring slot
//   warp 1      tensor-memory owner and MMA issuer: kind::f16 MMAs, M = 128,
//               N = NT, K = 16, both operands from shared memory, fp32
//               accumulator in tensor memory; one commit per stage frees the
//               slot
//   warps 2-5   epilogue: lane quarter q reads accumulator rows 32q..32q+31,
//               applies SwiGLU (gate/up) or rounds (down) and stages the tile
//               in shared memory for coalesced stores
// Narrow tiles run two or three CTAs per SM, so one CTA's set-up and epilogue
// overlap another's weight stream.  Every wait is bounded (2 s); on expiry the
// kernel records MOE_ERR_TIMEOUT, waits for its own copies and MMAs to finish
// and returns.
#include <cuda.h>

#include <atomic>

#include "common.cuh"
#include "mlp_plan.cuh"
#include "tc_sm100.cuh"

namespace moe {
namespace {

constexpr int BK = 64;                 // K elements per stage
constexpr int BM = 128;                // weight rows per tile (MMA M)
constexpr int A_STAGE = BM * BK * 2;   // 16 KB of bf16 weights per stage
constexpr int kThreads = 192;
constexpr uint64_t kWaitLimitNs = 2000000000ull;

// ring depth per tile width: narrow tiles keep 2 CTAs per SM
__host__ __device__ constexpr int stages_for(int NT) {
  return NT == 32 ? 5 : (NT == 64 ? 4 : (NT == 128 ? 6 : 4));
}
__host__ __device__ constexpr int stage_bytes(int NT) { return A_STAGE + NT * BK * 2; }
__host__ __device__ constexpr int smem_total(int NT) {
  // ring, then barriers; +1024 for the manual 1024-byte alignment
  return stages_for(NT) * stage_bytes(NT) + 256 + 1024;
}

__device__ __forceinline__ void abort_cta(volatile int* abort, int32_t* status) {
  *abort = 1;
  record_status(status, MOE_ERR_TIMEOUT);
}

template <int NT, bool GATE_UP>
__global__ void __launch_bounds__(kThreads, 1)
    grouped_bf16w_gemm(const __grid_constant__ CUtensorMap map_w,
                       const __grid_constant__ CUtensorMap map_x, const Tile* __restrict__ tiles,
                       const int* __restrict__ n_tiles, int rows_per_expert, int K, int out_ld,
                       uint16_t* __restrict__ out, int32_t* __restrict__ status) {
  constexpr int NS = stages_for(NT);
  constexpr int STAGE = stage_bytes(NT);
  constexpr int TMEM_COLS = NT < 32 ? 32 : NT;
  if (static_cast<int>(blockIdx.y) >= __ldg(n_tiles)) return;  // whole CTA, before any set-up

  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + NS * STAGE);
  uint64_t* full = bars;        // [NS] stage copies landed
  uint64_t* empty = full + NS;  // [NS] stage MMAs complete
  uint64_t* dfull = empty + NS; // accumulator complete
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(dfull + 1);
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

  if (threadIdx.x == 0) {
    for (int s = 0; s < NS; ++s) {
      tc::mbar_init(&full[s], 1);
      tc::mbar_init(&empty[s], 1);
    }
    tc::mbar_init(dfull, 1);
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

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      const int r0 = GATE_UP ? mt * 64 : mt * BM;
      int issued = 0;
      for (int kb = 0; kb < KB; ++kb) {
        const int s = kb % NS, n = kb / NS;
        if (n > 0 && !tc::mbar_wait(&empty[s], (n - 1) & 1, abort_flag, kWaitLimitNs)) {
          abort_cta(abort_flag, status);
          break;
        }
        uint8_t* dst = smem + s * STAGE;
        tc::mbar_arrive_expect_tx(&full[s], STAGE);
        if (GATE_UP)
          tc::tma_load_5d(dst, &map_w, &full[s], 0, kb, 0, r0, tile.e);
        else
          tc::tma_load_3d(dst, &map_w, &full[s], kb * BK, r0, tile.e);
        tc::tma_load_2d(dst + A_STAGE, &map_x, &full[s], kb * BK, tile.row0);
        ++issued;
      }
      // every copy this thread issued has landed before the CTA exits
      for (int kb = max(0, issued - NS); kb < issued; ++kb)
        tc::mbar_drain(&full[kb % NS], (kb / NS) & 1, kWaitLimitNs / 8);
    }
  } else if (warp == 1) {
    // ----------------------------------------------------------- MMA issuer
    if (lane == 0) {
      int done = 0;
      for (int kb = 0; kb < KB; ++kb) {
        const int s = kb % NS;
        if (!tc::mbar_wait(&full[s], (kb / NS) & 1, abort_flag, kWaitLimitNs)) {
          abort_cta(abort_flag, status);
          break;
        }
        tc::tc_fence_after();
        const uint64_t ad = tc::smem_desc_sw128(tc::smem_u32(smem + s * STAGE));
        const uint64_t bd = tc::smem_desc_sw128(tc::smem_u32(smem + s * STAGE + A_STAGE));
        // a descriptor addresses shared memory in 16-byte units: +2 per 16 bf16
#pragma unroll
        for (int i = 0; i < BK / 16; ++i)
          tc::mma_bf16_ss(tmem, ad + 2 * i, bd + 2 * i, IDESC, (kb | i) != 0);
        tc::mma_commit(&empty[s]);
        ++done;
      }
      // completes once every MMA this thread issued has finished
      if (done > 0)
        tc::mma_commit(dfull);
      else
        tc::mbar_arrive(dfull);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;
    const int m = q * 32 + lane;  // accumulator row = weight row of the tile
    const uint32_t lane_base = static_cast<uint32_t>(q * 32) << 16;
    bool ok = tc::mbar_wait(dfull, 0, abort_flag, kWaitLimitNs);
    ok = __all_sync(0xFFFFFFFFu, ok) && *abort_flag == 0;
    // every stage has been consumed once the accumulator is complete: the
    // ring is reused as the output staging area
    uint16_t* stg = reinterpret_cast<uint16_t*>(smem);
    if (ok) {
      tc::tc_fence_after();
      for (int c = 0; c < NV; c += 16) {
        uint32_t r[16];
        tc::tmem_ld16(tmem + lane_base + c, r);
        tc::tmem_ld_wait();
        if (GATE_UP) {
          // even lane: gate row f, odd lane: up row f (f = m >> 1); the even
          // lane finishes tokens c..c+7, the odd lane tokens c+8..c+15
          const bool up = m & 1;
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const float send = __uint_as_float(up ? r[i] : r[8 + i]);
            const float recv = __shfl_xor_sync(0xFFFFFFFFu, send, 1);
            const float gv = up ? recv : __uint_as_float(r[i]);
            const float uv = up ? __uint_as_float(r[8 + i]) : recv;
            const float silu = gv / (1.0f + expf(-gv));
            stg[(c + (up ? 8 : 0) + i) * 64 + (m >> 1)] = f32_to_bf16_rne(silu * uv);
          }
        } else {
#pragma unroll
          for (int i = 0; i < 16; ++i) stg[(c + i) * BM + m] = f32_to_bf16_rne(__uint_as_float(r[i]));
        }
      }
    }
    // the four epilogue warps meet before the coalesced stores
    asm volatile("bar.sync 1, 128;" ::: "memory");
    if (ok) {
      const int tid = threadIdx.x - 64;
      if (GATE_UP) {
        // h rows: 64 features (8 x 16 B) per token
        const int f0 = mt * 64;
        for (int i = tid; i < tile.nrows * 8; i += 128) {
          const int t = i >> 3, v = i & 7;
          const uint4 val = reinterpret_cast<const uint4*>(stg + t * 64)[v];
          *reinterpret_cast<uint4*>(out + static_cast<int64_t>(tile.row0 + t) * out_ld + f0 +
                                    v * 8) = val;
        }
      } else {
        const int d0 = mt * BM;
        const int nv = min(BM, rows_per_expert - d0) / 8;  // 16-byte vectors per token row
        for (int i = tid; i < tile.nrows * 16; i += 128) {
          const int t = i >> 4, v = i & 15;
          if (v >= nv) continue;
          const uint4 val = reinterpret_cast<const uint4*>(stg + t * BM)[v];
          *reinterpret_cast<uint4*>(out + static_cast<int64_t>(tile.row0 + t) * out_ld + d0 +
                                    v * 8) = val;
        }
      }
    }
  }

  tc::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    // every issued MMA has finished (already observed on the normal path)
    if (lane == 0) tc::mbar_drain(dfull, 0, kWaitLimitNs / 8);
    __syncwarp();
    tc::tc_fence_after();
    tc::tmem_dealloc(tmem, TMEM_COLS);
  }
}

// ------------------------------------------------------------ host helpers

bool encode_bf16(CUtensorMap* map, int rank, const void* base, const cuuint64_t* dims,
                 const cuuint64_t* strides, const cuuint32_t* box) {
  EncodeTiledFn fn = encode_tiled_fn();
  if (!fn) return false;
  const cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, static_cast<cuuint32_t>(rank),
            const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Gate/up weights [E][2F][D] bf16: a 64-element window of gate row f and of
// up row f for 64 consecutive f, interleaved (box order: K window, gate/up,
// rows).  Down weights [E][D][F] bf16: 64 elements of 128 consecutive rows.
bool make_weight_map(CUtensorMap* map, const uint16_t* w, int E, int R, int K, bool gate_up) {
  const cuuint64_t row = static_cast<cuuint64_t>(K) * 2;  // bytes
  const cuuint64_t mat = static_cast<cuuint64_t>(R) * row;
  if (gate_up) {
    const cuuint64_t F = static_cast<cuuint64_t>(R / 2);
    const cuuint64_t dims[5] = {BK, static_cast<cuuint64_t>(K / BK), 2, F,
                                static_cast<cuuint64_t>(E)};
    const cuuint64_t strides[4] = {BK * 2, F * row, row, mat};
    const cuuint32_t box[5] = {BK, 1, 2, 64, 1};
    return encode_bf16(map, 5, w, dims, strides, box);
  }
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(R),
                              static_cast<cuuint64_t>(E)};
  const cuuint64_t strides[2] = {row, mat};
  const cuuint32_t box[3] = {BK, BM, 1};
  return encode_bf16(map, 3, w, dims, strides, box);
}

// token rows [rows][K] bf16, box = (64 elements, NT rows)
bool make_token_map(CUtensorMap* map, const uint16_t* x, int64_t rows, int K, int NT) {
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(rows)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(K) * 2};
  const cuuint32_t box[2] = {BK, static_cast<cuuint32_t>(NT)};
  return encode_bf16(map, 2, x, dims, strides, box);
}

// token-tile width: about twice the mean rows per expert, 32..256
int choose_nt(const moe_shape& sh) {
  const int64_t S = static_cast<int64_t>(sh.T) * sh.k;
  const int64_t want = 2 * ((S + sh.E - 1) / sh.E);
  int nt = 32;
  while (nt < want && nt < 256) nt *= 2;
  return nt;
}

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
  if (cudaFuncSetAttribute(grouped_bf16w_gemm<NT, true>,
                           cudaFuncAttributeMaxDynamicSharedMemorySize, smem_total(NT)) !=
          cudaSuccess ||
      cudaFuncSetAttribute(grouped_bf16w_gemm<NT, false>,
                           cudaFuncAttributeMaxDynamicSharedMemorySize, smem_total(NT)) !=
          cudaSuccess) {
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

template <bool GATE_UP>
void launch_nt(int NT, const CUtensorMap& mw, const CUtensorMap& mx, const Tile* tiles,
               const int* n_tiles, int gx, int gy, int R, int K, int ld, uint16_t* out,
               int32_t* status, cudaStream_t st) {
  const dim3 grid(gx, gy);
  switch (NT) {
    case 32:
      grouped_bf16w_gemm<32, GATE_UP><<<grid, kThreads, smem_total(32), st>>>(
          mw, mx, tiles, n_tiles, R, K, ld, out, status);
      break;
    case 64:
      grouped_bf16w_gemm<64, GATE_UP><<<grid, kThreads, smem_total(64), st>>>(
          mw, mx, tiles, n_tiles, R, K, ld, out, status);
      break;
    case 128:
      grouped_bf16w_gemm<128, GATE_UP><<<grid, kThreads, smem_total(128), st>>>(
          mw, mx, tiles, n_tiles, R, K, ld, out, status);
      break;
    default:
      grouped_bf16w_gemm<256, GATE_UP><<<grid, kThreads, smem_total(256), st>>>(
          mw, mx, tiles, n_tiles, R, K, ld, out, status);
  }
}

struct UqWs {
  size_t n_tiles, tiles, total;
  int64_t max_tiles;
};

UqWs uq_ws(const moe_shape& sh) {
  const int NT = choose_nt(sh);
  const int64_t S = static_cast<int64_t>(sh.T) * sh.k;
  UqWs w;
  w.max_tiles = sh.E + (S + NT - 1) / NT;
  w.n_tiles = 0;
  w.tiles = 256;
  w.total = align_up(w.tiles + static_cast<size_t>(w.max_tiles) * sizeof(Tile), 256);
  return w;
}

}  // namespace

size_t unquantised_workspace(const moe_shape& sh) { return uq_ws(sh).total; }

// Plan (tile width, tensor maps, kernel attributes), then the tile list and
// the two GEMMs; nothing is enqueued when the plan fails.
moe_status unquantised_mlp(const uint16_t* x_perm, const int32_t* offsets, const moe_shape& sh,
                           const uint16_t* w_gu, const uint16_t* w_dn, uint16_t* h,
                           uint16_t* y_perm, void* ws, int32_t* status, cudaStream_t stream) {
  const int NT = choose_nt(sh);
  const UqWs W = uq_ws(sh);
  char* base = static_cast<char*>(ws);
  int* n_tiles = reinterpret_cast<int*>(base + W.n_tiles);
  Tile* tiles = reinterpret_cast<Tile*>(base + W.tiles);
  const int64_t S = static_cast<int64_t>(sh.T) * sh.k;
  const int D = sh.d_model, F = sh.d_ff, E = sh.E;
  CUtensorMap m_gu, m_x, m_dn, m_h;
  if (!make_weight_map(&m_gu, w_gu, E, 2 * F, D, true) || !make_token_map(&m_x, x_perm, S, D, NT) ||
      !make_weight_map(&m_dn, w_dn, E, D, F, false) || !make_token_map(&m_h, h, S, F, NT))
    return MOE_ERR_CUDA;
  if (!prepare_nt(NT)) return MOE_ERR_CUDA;
  if (cudaMemsetAsync(status, 0, 4, stream) != cudaSuccess) {
    cudaGetLastError();
    return MOE_ERR_CUDA;
  }
  moe_status st = plan_tiles_launch(offsets, E, NT, tiles, n_tiles, nullptr, 0, stream);
  if (st != MOE_OK) return st;
  const int max_tiles = static_cast<int>(W.max_tiles);
  launch_nt<true>(NT, m_gu, m_x, tiles, n_tiles, F / 64, max_tiles, 2 * F, D, F, h, status, stream);
  if ((st = launch_status()) != MOE_OK) return st;
  launch_nt<false>(NT, m_dn, m_h, tiles, n_tiles, (D + BM - 1) / BM, max_tiles, D, F, D, y_perm,
                   status, stream);
  return launch_status();
}

}  // namespace moe
