// The grouped expert MLP as two steps on the host: a plan, made before
// anything is enqueued (GEMM path and tile width chosen, every tensor map
// encoded, every kernel attribute set, the workspace carved), and the
// enqueue of its kernels.  A call that cannot run is refused while making the
// plan, so it leaves the stream untouched.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "moe_mxfp4.h"

namespace moe {

// Token tile of the grouped GEMMs: rows [row0, row0 + nrows) of the permuted
// order, all routed to expert e (nrows <= the tile width NT).
struct Tile {
  int e, row0, nrows, pad;
};

// Which pair of GEMM kernels runs the expert MLP.
enum MlpPath : int {
  kPathAuto = MOE_MLP_PATH_AUTO,
  kPathBlockScaled = MOE_MLP_PATH_BLOCK_SCALED,  // tcgen05 block-scaled MMA on the E2M1 codes
  kPathBf16Decode = MOE_MLP_PATH_BF16_DECODE,    // codes decoded to bf16 into tensor memory
};

// The path `path` resolves to for this shape (auto: block-scaled when twice
// the mean routed rows per expert is at most 64).
int resolve_path(const moe_shape& sh, int path);

// Token-tile width of the chosen path (the tile plan is made with it).
int mlp_tile_width(const moe_shape& sh, int path);

// Workspace bytes of the chosen path (tile list, split pieces, ...), without
// the status head of the standalone call.
size_t expert_mlp_workspace(const moe_shape& sh, int path);

// Per-path tile width and workspace (csrc/expert_mlp.cu, csrc/expert_mlp_bf16.cu).
int mx_tile_width(const moe_shape& sh);
size_t mx_workspace(const moe_shape& sh);
int bf_tile_width(const moe_shape& sh);
size_t bf_workspace(const moe_shape& sh);

// Block-scaled path (csrc/expert_mlp.cu)
struct MxPlan {
  CUtensorMap m_gu, m_gu_t, m_dn, m_dn_t, m_x, m_h;
  // the same, two 128-K windows per copy (one instruction per stage)
  CUtensorMap m_gu2, m_dn2, m_x2, m_h2;
  int NT, NS, NB;
  int CPS;  // CTAs per SM of the GEMMs (1, or 2 for 16-token tiles)
  int64_t max_tiles, padded_rows;
  uint8_t *pieces_x, *pieces_h;
  uint32_t *words_x, *words_h;
  int* work;  // the GEMM launch's work counter, then its per-tile counts [max_tiles]
  int* done;
};

// Decode-to-bf16 path (csrc/expert_mlp_bf16.cu)
struct BfPlan {
  CUtensorMap m_gu, m_x, m_dn, m_h;
  int NT;
  int64_t max_tiles;
};

struct MlpPlan {
  moe_shape sh;
  int path;  // resolved: kPathBlockScaled or kPathBf16Decode
  const uint16_t* x_perm;
  const uint8_t *wgu_q, *wgu_s, *wdn_q, *wdn_s;
  uint16_t *h, *y_perm;
  Tile* tiles;
  int* n_tiles;
  // counters the GEMM launch needs zeroed beforehand (null when none): the
  // kernel that writes the tile list zeroes them
  int* sched;
  int n_sched;
  MxPlan mx;
  BfPlan bf;
};

// Fill `plan` for one call; nothing is enqueued.  `h` may be null on the
// block-scaled path (the layer never reads h there), not on the other.
moe_status expert_mlp_plan(const moe_shape& sh, int path, const uint16_t* x_perm,
                           const uint8_t* wgu_q, const uint8_t* wgu_s, const uint8_t* wdn_q,
                           const uint8_t* wdn_s, uint16_t* h, uint16_t* y_perm, void* ws,
                           MlpPlan* plan);
moe_status mx_plan(MlpPlan* p, void* ws);
moe_status bf_plan(MlpPlan* p, void* ws);

// How the rows reach the first GEMM.
struct MlpInput {
  const int32_t* offsets;  // [E+1], device
  bool tiles_ready;        // the tile list was already written (by the permute)
  // block-scaled path inside the layer: split the rows straight from x
  // (row r of the permuted order is x[sorted_slot[r] / k]) instead of x_perm
  const uint16_t* x;
  const int32_t* sorted_slot;
  int k;
};

// Enqueue the plan's kernels.  fail_cta >= 0 (testing only) makes that CTA's
// first MMA-side wait give up, to exercise the timeout path.
moe_status expert_mlp_enqueue(const MlpPlan& plan, const MlpInput& in, int32_t* status,
                              int fail_cta, cudaStream_t stream);
moe_status mx_enqueue(const MlpPlan& plan, const MlpInput& in, int32_t* status, int fail_cta,
                      cudaStream_t stream);
moe_status bf_enqueue(const MlpPlan& plan, const MlpInput& in, int32_t* status, int fail_cta,
                      cudaStream_t stream);

// cuTensorMapEncodeTiled through the runtime's driver entry point (so the
// library loads without a driver).  Null when the driver has none.
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn encode_tiled_fn();

// Tile list of the grouped GEMMs on one CTA: expert e contributes
// ceil(count_e / NT) tiles of up to NT rows, experts ascending; the same CTA
// zeroes sched[0, n_sched).
moe_status plan_tiles_launch(const int32_t* offsets, int E, int NT, Tile* tiles, int* n_tiles,
                             int* sched, int n_sched, cudaStream_t stream);

}  // namespace moe
