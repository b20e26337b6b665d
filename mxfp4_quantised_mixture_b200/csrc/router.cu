// Router: logits = x . W_router^T fused with token-choice top-k and the
// softmax over the chosen experts.
//
// "Welcome GPT OSS, the new open-source model family from OpenAI" (summary),
// section 4: token-choice MoE with the softmax taken after the top-k;
// aitrends.kr talk summary, "Architecture details": 4 of 32 or 128 experts.
// The router scores every token against every expert; the routing that
// follows is the one moe_route computes from given logits.
//
// Batches of T * E <= 16384 take a small kernel on the CUDA cores, one or
// two CTAs per token (below).  Larger ones: one cluster of up to 8 CTAs per 128
// tokens, each CTA taking a contiguous share of the reduction axis.  The scores are a bf16 GEMM on the tensor core:
// tokens on the MMA's M side (128), the experts on N (E padded to a multiple
// of 16, at most 256), K = D in stages of 64 (one 128-byte swizzle row of
// bf16), both operands by TMA into shared memory, the fp32 accumulator in
// tensor memory.  Each CTA moves its partial scores from tensor memory to its
// shared memory; after a cluster barrier the CTA that owns a token (rank
// token % cluster size) adds the partials over distributed shared memory in
// rank order, a fixed order, so the scores do not depend on scheduling.
// One thread per token row keeps a running top-8 list in
// registers (value descending, index ascending), and applies the softmax
// over the first k in fp32 with the same summation order as moe_route, so
// the routing equals moe_route applied to the returned logits.
// Every wait is bounded (2 s); on expiry the kernel records MOE_ERR_TIMEOUT
// in the status word and returns after draining its copies and MMAs.
#include <cuda.h>
#include <math.h>

#include <atomic>

#include "common.cuh"
#include "tc_sm100.cuh"

namespace moe {
namespace {

constexpr int BKR = 64;                 // K elements per stage (128 bytes of bf16)
constexpr int MT = 128;                 // tokens per CTA (MMA M)
constexpr int A_BYTES = MT * BKR * 2;   // token rows per stage
constexpr int NSR = 4;                  // stages in the ring
constexpr int kThreads = 192;
constexpr int64_t kSmallRouterWork = 16384;  // T * E at or below which the small-batch kernel runs
constexpr uint64_t kWaitLimitNs = 2000000000ull;

__host__ __device__ inline int smem_bytes_router(int npad) {
  return 1024 + NSR * (A_BYTES + npad * BKR * 2) + 256;
}

__device__ __forceinline__ bool better(float va, int ia, float vb, int ib) {
  return va > vb || (va == vb && ia < ib);
}

// Running top-8 list (value descending, index ascending).  Experts arrive in
// index order, so an equal value never displaces an earlier one and ties keep
// the lower index.
__device__ __forceinline__ void insert_top8(float v, int e, float (&tv)[8], int (&ti)[8]) {
  if (better(v, e, tv[7], ti[7])) {
    tv[7] = v;
    ti[7] = e;
#pragma unroll
    for (int j = 7; j > 0; --j) {
      if (better(tv[j], ti[j], tv[j - 1], ti[j - 1])) {
        const float fv = tv[j];
        tv[j] = tv[j - 1];
        tv[j - 1] = fv;
        const int fi = ti[j];
        ti[j] = ti[j - 1];
        ti[j - 1] = fi;
      }
    }
  }
}

// Softmax over the first k of the list, summed in the order of moe_route's
// butterfly over lanes j = 0..7 (zero beyond k), and the stores of token t.
__device__ __forceinline__ void store_topk(const float (&tv)[8], const int (&ti)[8], int k,
                                           int64_t t, int32_t* __restrict__ idx,
                                           float* __restrict__ wts) {
  float ex[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) ex[j] = j < k ? expf(tv[j] - tv[0]) : 0.f;
  const float z = ((ex[0] + ex[4]) + (ex[2] + ex[6])) + ((ex[1] + ex[5]) + (ex[3] + ex[7]));
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    if (j < k) {
      idx[t * k + j] = ti[j];
      wts[t * k + j] = ex[j] / z;
    }
  }
}

// Small batches (a few tokens against the experts): no tensor core.  A token
// takes a cluster of cs = 1 or 2 CTAs (2 while the batch leaves SMs idle), CTA
// r scoring experts [r Eh, (r + 1) Eh), Eh = ceil(E / cs).  The token's row is
// copied into shared memory asynchronously while every lane requests its share
// of the router rows: warp w scores ROWS experts per pass (w, w + warps, ...
// of the CTA's range), lane l takes the 16-byte vectors l, l + 32, ... of a
// row in order, up to 12 of them per row in flight at once, and the warp adds
// its lanes with a butterfly, a fixed order.  Every CTA writes its scores to
// the logits and into the shared memory of the cluster's first CTA, where,
// after a cluster barrier, warp 0 picks the top k by rounds of a warp arg-max
// over the experts not yet taken (value descending, index ascending: the
// order of the running list) and stores the routing.
constexpr int kSmallThreads = 512;
constexpr int kSmallUnroll = 12;

__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(tc::smem_u32(dst)), "l"(src)
               : "memory");
}

template <int ROWS>
__device__ __forceinline__ void load_router_chunk(const uint4* const (&wr)[ROWS], int j0, int nv,
                                                  uint4 (&b)[ROWS][kSmallUnroll]) {
#pragma unroll
  for (int i = 0; i < kSmallUnroll; ++i) {
    const int j = j0 + 32 * i;
#pragma unroll
    for (int r = 0; r < ROWS; ++r) b[r][i] = j < nv ? __ldg(wr[r] + j) : make_uint4(0u, 0u, 0u, 0u);
  }
}

template <int ROWS>
__device__ __forceinline__ void dot_router_chunk(const uint4* xs, int j0, int nv,
                                                 const uint4 (&b)[ROWS][kSmallUnroll],
                                                 float (&acc)[ROWS]) {
#pragma unroll
  for (int i = 0; i < kSmallUnroll; ++i) {
    const int j = j0 + 32 * i;
    if (j < nv) {
      const uint4 a = xs[j];
      const uint32_t av[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
      for (int r = 0; r < ROWS; ++r) {
        const uint32_t bv[4] = {b[r][i].x, b[r][i].y, b[r][i].z, b[r][i].w};
#pragma unroll
        for (int h = 0; h < 4; ++h) {
          acc[r] = fmaf(__uint_as_float(av[h] << 16), __uint_as_float(bv[h] << 16), acc[r]);
          acc[r] = fmaf(__uint_as_float(av[h] & 0xFFFF0000u), __uint_as_float(bv[h] & 0xFFFF0000u),
                        acc[r]);
        }
      }
    }
  }
}

template <int ROWS>
__global__ void __launch_bounds__(kSmallThreads)
    router_small_kernel(const uint16_t* __restrict__ x, const uint16_t* __restrict__ w, int D,
                        int E, int k, int cs, float* __restrict__ logits,
                        int32_t* __restrict__ idx, float* __restrict__ wts) {
  extern __shared__ __align__(16) uint8_t small_smem[];
  uint4* xs = reinterpret_cast<uint4*>(small_smem);          // [D / 8]
  float* sc = reinterpret_cast<float*>(small_smem + D * 2);  // [E], used in rank 0
  const int rank = cs > 1 ? static_cast<int>(tc::cluster_rank()) : 0;
  if (cs > 1) tc::cluster_arrive_relaxed();
  const int64_t t = blockIdx.x / cs;
  const int Eh = (E + cs - 1) / cs;
  const int e_lo = rank * Eh, e_hi = min(E, e_lo + Eh);
  const int nv = D / 8;
  const uint4* xr = reinterpret_cast<const uint4*>(x + t * D);
  for (int j = threadIdx.x; j < nv; j += blockDim.x) cp_async16(xs + j, xr + j);
  asm volatile("cp.async.commit_group;" ::: "memory");
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
  const uint4* wv = reinterpret_cast<const uint4*>(w);
  const uint4* wr[ROWS];
  uint4 b[ROWS][kSmallUnroll];
  int e0 = e_lo + warp;
  // the first chunk of the first pass goes out with the token row
  bool loaded = e0 < e_hi;
  if (loaded) {
#pragma unroll
    for (int r = 0; r < ROWS; ++r) {
      const int e = e0 + r * nw;
      wr[r] = wv + static_cast<int64_t>(e < e_hi ? e : e0) * nv;
    }
    load_router_chunk<ROWS>(wr, lane, nv, b);
  }
  asm volatile("cp.async.wait_all;" ::: "memory");
  __syncthreads();
  if (cs > 1) tc::cluster_wait();  // every CTA of the cluster has started
  for (; e0 < e_hi; e0 += ROWS * nw) {
#pragma unroll
    for (int r = 0; r < ROWS; ++r) {
      const int e = e0 + r * nw;
      wr[r] = wv + static_cast<int64_t>(e < e_hi ? e : e0) * nv;
    }
    float acc[ROWS];
#pragma unroll
    for (int r = 0; r < ROWS; ++r) acc[r] = 0.f;
    for (int j0 = lane; j0 < nv; j0 += 32 * kSmallUnroll) {
      if (!loaded) load_router_chunk<ROWS>(wr, j0, nv, b);
      loaded = false;
      dot_router_chunk<ROWS>(xs, j0, nv, b, acc);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
#pragma unroll
      for (int r = 0; r < ROWS; ++r) acc[r] += __shfl_xor_sync(0xFFFFFFFFu, acc[r], o);
    }
    if (lane == 0) {
#pragma unroll
      for (int r = 0; r < ROWS; ++r) {
        const int e = e0 + r * nw;
        if (e < e_hi) {
          if (logits) logits[t * E + e] = acc[r];
          if (rank == 0)
            sc[e] = acc[r];
          else
            tc::st_cluster_f32(tc::cluster_addr(sc + e, 0), acc[r]);
        }
      }
    }
  }
  if (cs > 1)
    tc::cluster_sync();  // the other CTA's scores are in sc; it may now exit
  else
    __syncthreads();
  if (rank != 0) return;
  if (warp == 0) {
    // the top k in the order of the running list (value descending, index
    // ascending): k rounds of a warp arg-max over the experts not yet taken
    float tv[8];
    int ti[8];
#pragma unroll
    for (int r = 0; r < 8; ++r) {
      tv[r] = -INFINITY;
      ti[r] = 0x7FFFFFFF;
    }
    uint32_t taken = 0;  // bit c: expert 32 c + lane is already in the list (E <= 256)
#pragma unroll
    for (int r = 0; r < 8; ++r) {
      if (r >= k) break;
      float bv = -INFINITY;
      int bi = 0x7FFFFFFF;
      // lane l owns experts l, l + 32, ...
      for (int c = 0; 32 * c + lane < E; ++c) {
        const int e = 32 * c + lane;
        if (!((taken >> c) & 1u) && better(sc[e], e, bv, bi)) {
          bv = sc[e];
          bi = e;
        }
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        const float ov = __shfl_xor_sync(0xFFFFFFFFu, bv, o);
        const int oi = __shfl_xor_sync(0xFFFFFFFFu, bi, o);
        if (better(ov, oi, bv, bi)) {
          bv = ov;
          bi = oi;
        }
      }
      tv[r] = bv;
      ti[r] = bi;
      if (bi != 0x7FFFFFFF && (bi & 31) == lane) taken |= 1u << (bi >> 5);
    }
    if (lane == 0) store_topk(tv, ti, k, t, idx, wts);
  }
}

__global__ void __launch_bounds__(kThreads, 1)
    router_kernel(const __grid_constant__ CUtensorMap map_x, const __grid_constant__ CUtensorMap map_w,
                  int T, int D, int E, int npad, int k, float* __restrict__ logits,
                  int32_t* __restrict__ idx, float* __restrict__ wts, int32_t* __restrict__ status) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const int b_bytes = npad * BKR * 2;
  uint8_t* as = smem;
  uint8_t* bs = smem + NSR * A_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(bs + NSR * b_bytes);
  uint64_t* full = bars;
  uint64_t* empty = full + NSR;
  uint64_t* dfull = empty + NSR;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(dfull + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
  // the partial scores of this CTA, [npad][MT] fp32, over the ring once every
  // stage is consumed (the ring holds 64 KB + 512 npad bytes, the partials
  // 512 npad)
  float* part = reinterpret_cast<float*>(smem);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // this CTA's share of K: stages [st0, st1) of the cluster's cs CTAs
  const int cs = gridDim.y, rank = blockIdx.y;
  const int nstg_all = D / BKR;
  const int st0 = rank * nstg_all / cs, st1 = (rank + 1) * nstg_all / cs;
  const int nstg = st1 - st0;
  const int t0 = blockIdx.x * MT;
  int tcols = 32;
  while (tcols < npad) tcols *= 2;

  if (threadIdx.x == 0) {
    for (int s = 0; s < NSR; ++s) {
      tc::mbar_init(&full[s], 1);
      tc::mbar_init(&empty[s], 1);
    }
    tc::mbar_init(dfull, 1);
    *abort_flag = 0;
    tc::fence_mbar_init();
    tc::tma_prefetch_desc(&map_x);
    tc::tma_prefetch_desc(&map_w);
  }
  if (warp == 1) {
    tc::tmem_alloc(tmem_holder, tcols);
    tc::tmem_relinquish();
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = *tmem_holder;

  if (warp == 0) {
    if (lane == 0) {
      int issued = 0;
      for (int j = 0; j < nstg; ++j) {
        const int s = j % NSR, u = j / NSR;
        if (u > 0 && !tc::mbar_wait(&empty[s], (u - 1) & 1, abort_flag, kWaitLimitNs)) {
          *abort_flag = 1;
          record_status(status, MOE_ERR_TIMEOUT);
          break;
        }
        tc::mbar_arrive_expect_tx(&full[s], A_BYTES + b_bytes);
        tc::tma_load_2d(as + s * A_BYTES, &map_x, &full[s], (st0 + j) * BKR, t0);
        tc::tma_load_2d(bs + s * b_bytes, &map_w, &full[s], (st0 + j) * BKR, 0);
        ++issued;
      }
      for (int j = max(0, issued - NSR); j < issued; ++j)
        tc::mbar_drain(&full[j % NSR], (j / NSR) & 1, kWaitLimitNs / 8);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = tc::idesc_bf16_f32(MT, npad);
      int done = 0;
      for (int j = 0; j < nstg; ++j) {
        const int s = j % NSR;
        if (!tc::mbar_wait(&full[s], (j / NSR) & 1, abort_flag, kWaitLimitNs)) {
          *abort_flag = 1;
          record_status(status, MOE_ERR_TIMEOUT);
          break;
        }
        tc::tc_fence_after();
        const uint64_t ad = tc::smem_desc_sw128(tc::smem_u32(as + s * A_BYTES));
        const uint64_t bd = tc::smem_desc_sw128(tc::smem_u32(bs + s * b_bytes));
        // a descriptor addresses shared memory in 16-byte units: +2 per 16 bf16
#pragma unroll
        for (int kk = 0; kk < BKR / 16; ++kk)
          tc::mma_bf16_ss(tmem, ad + 2 * kk, bd + 2 * kk, idesc, (j | kk) != 0);
        tc::mma_commit(&empty[s]);
        ++done;
      }
      if (done > 0)
        tc::mma_commit(dfull);
      else
        tc::mbar_arrive(dfull);
    }
  } else {
    // this CTA's partial scores: accumulator row m (token t0 + m) -> part[e][m]
    const int q = warp & 3;
    const int m = q * 32 + lane;
    const uint32_t lane_base = static_cast<uint32_t>(q * 32) << 16;
    bool ok = tc::mbar_wait(dfull, 0, abort_flag, kWaitLimitNs);
    ok = __all_sync(0xFFFFFFFFu, ok) && *abort_flag == 0;
    if (ok) {
      tc::tc_fence_after();
      for (int c = 0; c < npad; c += 16) {
        uint32_t r[16];
        tc::tmem_ld16(tmem + lane_base + c, r);
        tc::tmem_ld_wait();
#pragma unroll
        for (int i = 0; i < 16; ++i) part[(c + i) * MT + m] = __uint_as_float(r[i]);
      }
    }
  }

  // every CTA's partials are in its shared memory
  tc::tc_fence_before();
  tc::cluster_sync();

  if (warp >= 2) {
    // token m belongs to the CTA of rank m % cs: it adds the cs partial
    // scores in rank order (fixed, so the scores do not depend on scheduling),
    // keeps a running top-8 list and applies the softmax over the first k
    const int q = warp & 3;
    const int m = q * 32 + lane;
    const int t = t0 + m;
    if (m % cs == rank && t < T && *abort_flag == 0) {
      float tv[8];
      int ti[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        tv[j] = -INFINITY;
        ti[j] = 0x7FFFFFFF;
      }
      // the partials of rank r sit at base[r] + 4 (e MT + m) in the cluster
      // window; the loads of four experts x all ranks are issued before any
      // is added, so their latencies overlap
      uint32_t base[8];
#pragma unroll
      for (int r = 0; r < 8; ++r) base[r] = r < cs ? tc::cluster_addr(part + m, r) : 0u;
      for (int e0 = 0; e0 < E; e0 += 4) {
        float pv[4][8];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
#pragma unroll
          for (int r = 0; r < 8; ++r)
            pv[u][r] = (r < cs && e0 + u < E)
                           ? tc::ld_cluster_f32(base[r] + static_cast<uint32_t>((e0 + u) * MT * 4))
                           : 0.f;
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int e = e0 + u;
          if (e >= E) break;
          float v = pv[u][0];
#pragma unroll
          for (int r = 1; r < 8; ++r)
            if (r < cs) v += pv[u][r];
          if (logits) logits[static_cast<int64_t>(t) * E + e] = v;
          insert_top8(v, e, tv, ti);
        }
      }
      store_topk(tv, ti, k, t, idx, wts);
    }
  }

  // no CTA leaves while another may still read its partials
  tc::cluster_sync();
  if (warp == 1) {
    if (lane == 0) tc::mbar_drain(dfull, 0, kWaitLimitNs / 8);
    __syncwarp();
    tc::tc_fence_after();
    tc::tmem_dealloc(tmem, tcols);
  }
}

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

// bf16 rows [rows][K], box = 64 K x box_rows rows, 128-byte swizzle
bool make_rows_map(CUtensorMap* map, const uint16_t* base, int64_t rows, int K, int box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(rows)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(K) * 2};
  const cuuint32_t box[2] = {BKR, static_cast<cuuint32_t>(box_rows)};
  const cuuint32_t estr[2] = {1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<uint16_t*>(base), dims, strides,
            box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

moe_status router_launch(const uint16_t* x, const uint16_t* w_router, int T, int D, int E, int k,
                         float* logits, int32_t* idx, float* wts, int32_t* status,
                         cudaStream_t stream) {
  if (T == 0) return MOE_OK;
  if (static_cast<int64_t>(T) * E <= kSmallRouterWork) {
    // a few tokens: one or two CTAs per token on the CUDA cores (a tensor-core tile
    // of 128 tokens would be mostly padding, and its reduction over a
    // cluster costs more than the scores)
    // two CTAs per token while the batch leaves half the SMs idle; each then
    // requests only its half of the router matrix
    const int cs = (E >= 2 && 2 * static_cast<int64_t>(T) <= sm_count()) ? 2 : 1;
    const int eh = (E + cs - 1) / cs;
    const bool two_rows = eh > kSmallThreads / 32;
    auto kern = two_rows ? router_small_kernel<2> : router_small_kernel<1>;
    const int smem = D * 2 + E * 4;
    if (smem > 48 * 1024) {
      static std::atomic<uint64_t> small_done{0};
      int dev = 0;
      if (cudaGetDevice(&dev) != cudaSuccess) {
        cudaGetLastError();
        return MOE_ERR_CUDA;
      }
      const uint64_t bit = dev < 64 ? (uint64_t(1) << dev) : 0;
      if (!bit || !(small_done.load() & bit)) {
        for (auto kf : {router_small_kernel<1>, router_small_kernel<2>}) {
          if (cudaFuncSetAttribute(kf, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                   16384 * 2 + 256 * 4) != cudaSuccess) {
            cudaGetLastError();
            return MOE_ERR_CUDA;
          }
        }
        small_done.fetch_or(bit);
      }
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(T) * cs, 1, 1);
    cfg.blockDim = dim3(kSmallThreads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = cs;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = cs > 1 ? 1 : 0;
    if (cudaLaunchKernelEx(&cfg, kern, x, w_router, D, E, k, cs, logits, idx, wts) != cudaSuccess) {
      cudaGetLastError();
      return MOE_ERR_CUDA;
    }
    return launch_status();
  }
  const int npad = (E + 15) / 16 * 16;
  CUtensorMap mx, mw;
  if (!make_rows_map(&mx, x, T, D, MT) || !make_rows_map(&mw, w_router, E, D, npad))
    return MOE_ERR_CUDA;
  // the dynamic shared-memory opt-in, once per device
  static std::atomic<uint64_t> attr_done{0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return MOE_ERR_CUDA;
  }
  const uint64_t bit = dev < 64 ? (uint64_t(1) << dev) : 0;
  if (!bit || !(attr_done.load() & bit)) {
    if (cudaFuncSetAttribute(router_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             smem_bytes_router(256)) != cudaSuccess) {
      cudaGetLastError();
      return MOE_ERR_CUDA;
    }
    attr_done.fetch_or(bit);
  }
  // one cluster of cs CTAs per 128 tokens splits K: about one SM per CTA
  // overall, at most 8 per cluster, at least one 64-K stage each
  const int nblk = (T + MT - 1) / MT;
  int cs = (sm_count() + nblk - 1) / nblk;
  cs = cs < 1 ? 1 : (cs > 8 ? 8 : cs);
  if (cs > D / BKR) cs = D / BKR;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(nblk, cs, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = smem_bytes_router(npad);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 1;
  attr[0].val.clusterDim.y = cs;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, router_kernel, mx, mw, T, D, E, npad, k, logits, idx, wts,
                         status) != cudaSuccess) {
    cudaGetLastError();
    return MOE_ERR_CUDA;
  }
  return launch_status();
}

}  // namespace moe

extern "C" moe_status moe_router_topk(const uint16_t* x, const uint16_t* w_router, int32_t T,
                                      int32_t D, int32_t E, int32_t k, float* logits,
                                      int32_t* topk_idx, float* topk_w, int32_t* d_status,
                                      moe_stream stream) {
  using namespace moe;
  if (T < 0 || T > (1 << 20) || E < 1 || E > 256 || k < 1 || k > 8 || k > E) return MOE_ERR_SHAPE;
  if (D < 64 || D > 16384 || (D % 64) != 0) return MOE_ERR_SHAPE;
  if (T == 0) return MOE_OK;
  if (!x || !w_router || !topk_idx || !topk_w) return MOE_ERR_INVALID_ARG;
  const void* ptrs[] = {x, w_router, topk_idx, topk_w};
  for (const void* p : ptrs)
    if (!aligned16(p)) return MOE_ERR_INVALID_ARG;
  if (logits && !aligned16(logits)) return MOE_ERR_INVALID_ARG;
  if (d_status && (reinterpret_cast<uintptr_t>(d_status) & 3u)) return MOE_ERR_INVALID_ARG;
  moe_status st = check_device();
  if (st != MOE_OK) return st;
  return router_launch(x, w_router, T, D, E, k, logits, topk_idx, topk_w, d_status,
                       static_cast<cudaStream_t>(stream));
}
