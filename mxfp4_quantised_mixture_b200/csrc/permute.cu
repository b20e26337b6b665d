// Group the T*k routed slots by expert (histogram, exclusive scan, stable
// scatter) and gather the activation rows in that order.
//
// "MXFP4-based MoE technical review", section 4: routing over sparse experts
// and its parallelisation.  The order inside an expert is ascending slot
// index, which makes the result unique and the later gather-sum
// deterministic.
//
// One CTA of 1024 threads does the bookkeeping (S <= 8M slots, E <= 256):
//   1. warp w counts its contiguous chunk of slots per expert (shared-memory
//      atomics into its own row of a [32][E] table);
//   2. per expert, a column scan over warps plus the expert's offset gives
//      the first position of each (warp, expert) run;
//   3. warp w walks its chunk again, 32 slots at a time: lanes with the same
//      expert find each other with __match_any_sync, rank themselves by lane
//      order, and the group leader advances the run.  Chunks are contiguous
//      and walked in order, so positions follow ascending slot index.
// Inside the layer the same CTA also writes the grouped GEMMs' tile list
// (expert e gets ceil(count_e / NT) tiles of up to NT rows), which saves the
// GEMMs a launch of their own.
// The row gather (HBM-bound) runs as a separate full-GPU kernel.
#include "common.cuh"
#include "mlp_plan.cuh"

namespace moe {
namespace {

constexpr int kWarps = 32;
constexpr int kThreads = kWarps * 32;
constexpr int kMaxE = 256;

__global__ void __launch_bounds__(kThreads, 1)
    permute_kernel(const int32_t* __restrict__ idx, int64_t S, int E, int32_t* __restrict__ counts,
                   int32_t* __restrict__ offsets, int32_t* __restrict__ sorted_slot,
                   int32_t* __restrict__ slot_pos, int NT, Tile* __restrict__ tiles,
                   int* __restrict__ n_tiles, int* __restrict__ sched, int n_sched) {
  __shared__ int32_t cnt[kWarps][kMaxE];  // per (warp, expert) count, then running position
  __shared__ int32_t off[kMaxE + 1];
  __shared__ int32_t tbase[kMaxE + 1];    // first tile of each expert (tile list only)
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int i = threadIdx.x; i < kWarps * kMaxE; i += kThreads) (&cnt[0][0])[i] = 0;
  // the GEMM launch's counters (see MlpPlan::sched)
  for (int i = threadIdx.x; i < n_sched; i += kThreads) sched[i] = 0;
  __syncthreads();
  const int64_t chunk = (S + kWarps - 1) / kWarps;
  const int64_t lo = S < warp * chunk ? S : warp * chunk;
  const int64_t hi = S < lo + chunk ? S : lo + chunk;
  for (int64_t s = lo + lane; s < hi; s += 32) {
    const int e = __ldg(idx + s);
    if (static_cast<unsigned>(e) < static_cast<unsigned>(E)) atomicAdd(&cnt[warp][e], 1);
  }
  __syncthreads();
  // per-expert totals and exclusive scan over experts (warp 0)
  if (warp == 0) {
    int carry = 0;
    for (int e0 = 0; e0 < E; e0 += 32) {
      const int e = e0 + lane;
      int tot = 0;
      if (e < E)
        for (int w = 0; w < kWarps; ++w) tot += cnt[w][e];
      int incl = tot;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int n = __shfl_up_sync(0xFFFFFFFFu, incl, o);
        if (lane >= o) incl += n;
      }
      if (e < E) {
        off[e] = carry + incl - tot;
        counts[e] = tot;
      }
      carry += __shfl_sync(0xFFFFFFFFu, incl, 31);
    }
    if (lane == 0) off[E] = carry;
  }
  __syncthreads();
  for (int e = threadIdx.x; e <= E; e += kThreads) offsets[e] = off[e];
  if (tiles) {
    // tile list: per-expert tile counts, their exclusive scan (warp 0), then
    // expert e's tiles written by thread e
    if (warp == 0) {
      int carry = 0;
      for (int e0 = 0; e0 < E; e0 += 32) {
        const int e = e0 + lane;
        const int nt = e < E ? (off[e + 1] - off[e] + NT - 1) / NT : 0;
        int incl = nt;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int n = __shfl_up_sync(0xFFFFFFFFu, incl, o);
          if (lane >= o) incl += n;
        }
        if (e < E) tbase[e] = carry + incl - nt;
        carry += __shfl_sync(0xFFFFFFFFu, incl, 31);
      }
      if (lane == 0) *n_tiles = carry;
    }
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += kThreads) {
      const int r0 = off[e], c = off[e + 1] - off[e];
      for (int t = 0; t * NT < c; ++t) {
        Tile tl;
        tl.e = e;
        tl.row0 = r0 + t * NT;
        tl.nrows = min(NT, c - t * NT);
        tl.pad = 0;
        tiles[tbase[e] + t] = tl;
      }
    }
  }
  // column scan: first position of each (warp, expert) run
  for (int e = threadIdx.x; e < E; e += kThreads) {
    int run = off[e];
    for (int w = 0; w < kWarps; ++w) {
      const int c = cnt[w][e];
      cnt[w][e] = run;
      run += c;
    }
  }
  __syncthreads();
  for (int64_t base = lo; base < hi; base += 32) {
    const int64_t s = base + lane;
    const int e = s < hi ? __ldg(idx + s) : -1;
    // an index outside [0, E) is dropped: it gets no position (slot_pos -1)
    const bool valid = static_cast<unsigned>(e) < static_cast<unsigned>(E);
    if (s < hi && !valid) slot_pos[s] = -1;
    const unsigned active = __ballot_sync(0xFFFFFFFFu, valid);
    if (valid) {
      const unsigned peers = __match_any_sync(active, e);
      const int rank = __popc(peers & ((1u << lane) - 1u));
      const int pos = cnt[warp][e] + rank;
      sorted_slot[pos] = static_cast<int32_t>(s);
      slot_pos[s] = pos;
      __syncwarp(active);
      if (rank == 0) cnt[warp][e] += __popc(peers);
    }
    __syncwarp();
  }
}

// x_perm[p] = x[sorted_slot[p] / k]; one warp per row, 16-byte vectors
// (only the offsets[E] positions that hold a routed slot are gathered)
__global__ void __launch_bounds__(256) gather_rows_kernel(const uint4* __restrict__ x,
                                                         const int32_t* __restrict__ sorted_slot,
                                                         const int32_t* __restrict__ n_valid,
                                                         int k, int vec_per_row,
                                                         uint4* __restrict__ x_perm) {
  const int64_t S = *n_valid;
  const int lane = threadIdx.x & 31;
  const int64_t w0 = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t nw = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
  for (int64_t p = w0; p < S; p += nw) {
    const int64_t t = __ldg(sorted_slot + p) / k;
    const uint4* src = x + t * vec_per_row;
    uint4* dst = x_perm + p * vec_per_row;
    for (int v = lane; v < vec_per_row; v += 32) dst[v] = __ldg(src + v);
  }
}

}  // namespace

moe_status permute_launch(const int32_t* idx, const uint16_t* x, const moe_shape& sh,
                          int32_t* counts, int32_t* offsets, int32_t* sorted_slot,
                          int32_t* slot_pos, uint16_t* x_perm, int NT, Tile* tiles,
                          int* n_tiles, int* sched, int n_sched, cudaStream_t stream) {
  const int64_t S = static_cast<int64_t>(sh.T) * sh.k;
  moe_status st = launch(permute_kernel, dim3(1), dim3(kThreads), 0, stream, idx, S,
                         sh.E, counts, offsets, sorted_slot, slot_pos, NT, tiles, n_tiles,
                         sched, n_sched);
  if (st != MOE_OK || S == 0 || x_perm == nullptr) return st;
  const int vec = sh.d_model / 8;
  int64_t want = (S * 32 + 255) / 256;
  int64_t cap = static_cast<int64_t>(sm_count()) * 8;
  const int grid = static_cast<int>(want < cap ? want : cap);
  return launch(gather_rows_kernel, dim3(grid), dim3(256), 0, stream,
                reinterpret_cast<const uint4*>(x), static_cast<const int32_t*>(sorted_slot),
                static_cast<const int32_t*>(offsets + sh.E), sh.k, vec,
                reinterpret_cast<uint4*>(x_perm));
}

}  // namespace moe

extern "C" moe_status moe_permute(const int32_t* topk_idx, const uint16_t* x, moe_shape shape,
                                  int32_t* counts, int32_t* offsets, int32_t* sorted_slot,
                                  int32_t* slot_pos, uint16_t* x_perm, void* ws, size_t ws_bytes,
                                  moe_stream stream) {
  using namespace moe;
  if (!shape_ok(shape)) return MOE_ERR_SHAPE;
  if (!counts || !offsets) return MOE_ERR_INVALID_ARG;
  const bool empty = shape.T == 0;
  if (!empty && (!topk_idx || !x || !sorted_slot || !slot_pos || !x_perm)) return MOE_ERR_INVALID_ARG;
  const void* ptrs[] = {topk_idx, x, counts, offsets, sorted_slot, slot_pos, x_perm};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return MOE_ERR_INVALID_ARG;
  const size_t need = moe_workspace_size(shape, 0);
  if (need > 0 && (ws == nullptr || ws_bytes < need)) return MOE_ERR_WORKSPACE;
  moe_status st = check_device();
  if (st != MOE_OK) return st;
  return permute_launch(topk_idx, x, shape, counts, offsets, sorted_slot, slot_pos, x_perm, 0,
                        nullptr, nullptr, nullptr, 0, static_cast<cudaStream_t>(stream));
}
