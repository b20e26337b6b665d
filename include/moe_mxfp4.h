/*
 * moe_mxfp4.h -- C ABI of the MXFP4 Mixture-of-Experts layer library
 * (libmoe_mxfp4.so, built for NVIDIA B200 / sm_100a).
 *
 * The operation is the MoE MLP block of a GPT-OSS-style decoder:
 *   - token-choice routing, each token picking its top-k experts, with the
 *     softmax taken over the k selected logits only ("softmax-after-topk")
 *     ["Welcome GPT OSS, the new open-source model family from OpenAI"
 *      (summary), section 4 "MoE, quantisation and context handling"];
 *   - 4 active experts per token, 32 or 128 experts per layer, independent
 *     experts with no shared expert [aitrends.kr talk summary, chapters
 *     "Architecture details: MoE and attention" and "Q&A"];
 *   - SwiGLU experts whose weights are MXFP4: E2M1 4-bit elements (1 sign,
 *     2 exponent, 1 mantissa bit) with one shared scale per block of 32
 *     elements ["Tricks from OpenAI gpt-oss you can use with transformers"
 *     (summary), section 6 "MXFP4 format and memory savings";
 *     agentlenshq "Transformers ... GPT-OSS" (ja), section "What is MXFP4"];
 *     the format is the OCP Microscaling (MX) one, so the shared scale is an
 *     E8M0 power of two ["MXFP4-based MoE technical review", section 1];
 *   - weights stay 4-bit in memory and are raised to bf16 only inside the
 *     GEMM [aitrends.kr talk summary, chapter "Hardware optimisation"];
 *     GEMM kernels must understand the 32-element blocks and their scales
 *     ["Tricks from OpenAI gpt-oss ...", section 8].
 *
 * Notation: T tokens, E experts, k experts per token, D = d_model,
 * F = d_ff, S = T*k routed slots; slot s = t*k + j, j = rank within the
 * token's top-k (j = 0 is the highest logit).
 *
 * Data layouts (all row-major, all pointers are DEVICE pointers unless a
 * function says otherwise; bf16 values travel as raw uint16_t bit patterns):
 *   x          bf16  [T][D]
 *   logits     fp32  [T][E]
 *   w_gu       MXFP4 [E][2F][D]  rows [0,F) are the gate projection,
 *                                rows [F,2F) the up projection; the 32-blocks
 *                                run along D (the reduction axis).
 *   w_dn       MXFP4 [E][D][F]   32-blocks run along F.
 *   An MXFP4 matrix [R][K] is two arrays:
 *     q  uint8 [R][K/2]   element 2i in the low nibble of byte i, element
 *                         2i+1 in the high nibble; nibble = sign<<3 | e<<1 | m
 *     s  uint8 [R][K/32]  E8M0 scale byte b, scale = 2^(b-127)
 *   value = (-1)^sign * {0,0.5,1,1.5,2,3,4,6}[nibble & 7] * 2^(b-127).
 *
 * Conventions shared by every call:
 *   - Ownership: the caller allocates and owns every buffer, including the
 *     workspace; the library never allocates, never synchronises the device
 *     and never falls back to another implementation.
 *   - Calls are asynchronous and ordered on `stream` (a cudaStream_t passed
 *     as void*; NULL = the legacy default stream).
 *   - Host-side validation (null pointers, shapes, alignment, workspace
 *     size, device architecture) happens before anything is launched; on
 *     failure the call returns the status and launches nothing.
 *   - MOE_ERR_CUDA is returned when a kernel launch reports an error.
 *   - Conditions only the device can see (non-finite quantiser input, a
 *     bounded wait that gave up) are written to a device status word
 *     (`d_status`, or the first 4 bytes of the workspace); the caller reads
 *     it after synchronising.  Kernels never trap or assert.
 *   - Calls on different streams with different workspaces are independent.
 *   - Every device pointer must be 16-byte aligned; the packed weight code
 *     arrays (wgu_q, wdn_q) 32-byte aligned (the tensor-memory copy engine
 *     reads them in the one-byte-per-code layout the tensor core takes).
 */
#ifndef MOE_MXFP4_H
#define MOE_MXFP4_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = 1, /* null pointer, misaligned pointer, bad enum   */
  MOE_ERR_SHAPE = 2,       /* shape outside the supported range           */
  MOE_ERR_WORKSPACE = 3,   /* workspace missing or smaller than required  */
  MOE_ERR_UNSUPPORTED = 4, /* current device is not compute capability 10.0 */
  MOE_ERR_CUDA = 5,        /* a CUDA runtime call or launch failed        */
  MOE_ERR_NONFINITE = 6,   /* device status only: NaN/Inf quantiser input */
  MOE_ERR_TIMEOUT = 7      /* device status only: a bounded wait gave up  */
} moe_status;

/* Shape of one MoE layer call.
 * Supported: 1 <= T <= 1<<20, 1 <= E <= 256, 1 <= k <= min(E, 8),
 * D and F multiples of 64 in [128, 16384], T*k < 2^31.                   */
typedef struct {
  int32_t T;
  int32_t E;
  int32_t k;
  int32_t d_model;
  int32_t d_ff;
} moe_shape;

typedef void* moe_stream; /* cudaStream_t */

/* exported symbols keep default visibility even when the library is built
 * with -fvisibility=hidden */
#if defined(__GNUC__)
#define MOE_API __attribute__((visibility("default")))
#else
#define MOE_API
#endif

/* mxfp4_quantize -- bf16 -> MXFP4 block quantiser.
 * Passage: E2M1 with a 32-element shared scale ("Tricks from OpenAI
 * gpt-oss ...", section 6; agentlenshq (ja), "What is MXFP4"), OCP MX
 * E8M0 scale ("MXFP4-based MoE technical review", section 1).
 * Per 32-element block of each row: amax = max |x|; scale byte
 * b = clamp(bexp(amax) - 2, 0, 254), where bexp is the 8-bit exponent field
 * of amax (so b = floor(log2 amax) - 2 + 127 for normal amax, 0 for a zero
 * or subnormal amax); each element is |x| / 2^(b-127) rounded to nearest,
 * ties to even mantissa, onto {0,0.5,1,1.5,2,3,4,6}, saturating at 6; the
 * sign bit is the sign of x (so -0 and small negatives give code 8).
 *   w_bf16   in   [rows][K] bf16
 *   rows     in   >= 0 (0 is a no-op), rows*K < 2^40
 *   K        in   multiple of 32, >= 32
 *   q_packed out  [rows][K/2]
 *   scales   out  [rows][K/32]
 *   d_status out  nullable; if a block holds NaN or Inf the kernel stores
 *                 MOE_ERR_NONFINITE there (that block's bytes are
 *                 unspecified); it never writes MOE_OK, so clear it first.
 * Errors: MOE_ERR_INVALID_ARG, MOE_ERR_SHAPE, MOE_ERR_UNSUPPORTED,
 * MOE_ERR_CUDA.                                                          */
MOE_API moe_status mxfp4_quantize(const uint16_t* w_bf16, int64_t rows, int64_t K,
                          uint8_t* q_packed, uint8_t* scales,
                          int32_t* d_status, moe_stream stream);

/* mxfp4_quantize_sr_rht -- training-style bf16 -> MXFP4 quantiser.
 * Passage: "MXFP4-based MoE technical review", sections 2 and 4 (stochastic
 * rounding and a random Hadamard transform keep MXFP4 training close to
 * bf16); the format as for mxfp4_quantize.  Per 32-element block of a row:
 *   MOE_QUANT_RHT  y = H (s . x), H the unnormalised 32-point Sylvester
 *                  Hadamard matrix (+1/-1, H[i][j] = (-1)^popcount(i & j)),
 *                  s_j = -1 where bit j of rht_signs[c / 32] is set (c the
 *                  element's column); y is exact (fp64) whenever the block's
 *                  nonzero exponents span under 40 binades.  A product of two
 *                  operands that carry the same transform along K is 32 times
 *                  the plain product.  Without the flag y = x.
 *   scale byte     floor(log2 amax|y|) - 2 + 127; with MOE_QUANT_SR the
 *                  smallest byte with amax / 2^(byte-127) <= 6, i.e. one more
 *                  when the significand of amax is above 1.5 (no element
 *                  clips, so the rounding is unbiased); clamped to [0, 254];
 *                  an all-zero block gets 0.
 *   codes          v = |y| / scale rounded to nearest even onto
 *                  {0,.5,1,1.5,2,3,4,6} (saturating at 6), or, with
 *                  MOE_QUANT_SR, to the upper neighbour when
 *                  u / 65536 < (v - lo) / (hi - lo), u the 16-bit uniform of
 *                  element n = r K + c: Philox4x32-10 (Salmon et al., SC 2011)
 *                  of counter (n / 8 low, n / 8 high, 0, 0) under key (seed
 *                  low, seed high), output word (n % 8) / 2, low half for even
 *                  n.  Sign bit: y < 0 with the transform, else the sign bit
 *                  of x.  flags == 0 gives exactly mxfp4_quantize's bytes.
 *   w_bf16    in   [rows][K] bf16, 16-byte aligned
 *   rows, K   in   as for mxfp4_quantize
 *   flags     in   MOE_QUANT_RHT | MOE_QUANT_SR, any subset
 *   rht_signs in   [K/32] uint32, 4-byte aligned; required with MOE_QUANT_RHT,
 *                  else ignored (may be NULL)
 *   seed      in   Philox key; the same seed and shape give the same bytes
 *   q_packed  out  [rows][K/2]; scales out [rows][K/32]; both 16-byte aligned
 *   d_status  out  nullable; MOE_ERR_NONFINITE if a block holds NaN or Inf
 *                  (its bytes unspecified); never written otherwise.
 * Errors: MOE_ERR_INVALID_ARG (unknown flag bits, missing signs, null or
 * misaligned pointer), MOE_ERR_SHAPE, MOE_ERR_UNSUPPORTED, MOE_ERR_CUDA.  */
#define MOE_QUANT_RHT 1u
#define MOE_QUANT_SR 2u
MOE_API moe_status mxfp4_quantize_sr_rht(const uint16_t* w_bf16, int64_t rows, int64_t K,
                                         uint32_t flags, const uint32_t* rht_signs,
                                         uint64_t seed, uint8_t* q_packed, uint8_t* scales,
                                         int32_t* d_status, moe_stream stream);

/* moe_route -- token-choice top-k with softmax over the chosen k.
 * Passage: "Welcome GPT OSS ..." (summary), section 4 (token-choice MoE,
 * softmax-after-topk); aitrends.kr talk summary (4 active experts).
 * Per token t: the k experts with the largest logits, ordered by
 * (logit descending, expert index ascending) -- equal logits, including
 * -0 and +0, go to the lower index; topk_w[t][j] = softmax over those k
 * logits, computed in fp32.
 *   logits   in   [T][E] fp32, finite
 *   topk_idx out  [T][k] int32
 *   topk_w   out  [T][k] fp32
 * Errors: MOE_ERR_INVALID_ARG, MOE_ERR_SHAPE, MOE_ERR_UNSUPPORTED,
 * MOE_ERR_CUDA.                                                          */
MOE_API moe_status moe_route(const float* logits, int32_t T, int32_t E, int32_t k,
                     int32_t* topk_idx, float* topk_w, moe_stream stream);

/* moe_router_topk -- router scores fused with moe_route.
 * Passage: "Welcome GPT OSS ..." (summary), section 4 (token-choice MoE, a
 * router scoring every token against every expert, softmax-after-topk);
 * aitrends.kr talk summary (4 active experts).
 * logits[t][e] = sum_d x[t][d] * w_router[e][d]: bf16 inputs, exact
 * products, fp32 accumulation in a fixed but unspecified order (on the
 * tensor core when T * E > 16384, else on the CUDA cores, one or two CTAs
 * per token); then topk_idx / topk_w exactly as moe_route computes them from
 * those logits.
 *   x        in   [T][D] bf16, D a multiple of 64 in [64, 16384]
 *   w_router in   [E][D] bf16 (one row per expert), E <= 256
 *   logits   out  nullable; [T][E] fp32 when given
 *   topk_idx out  [T][k] int32; topk_w out [T][k] fp32
 *   d_status out  nullable; MOE_ERR_TIMEOUT if a bounded wait gave up
 *                 (never written otherwise)
 * Errors: MOE_ERR_INVALID_ARG, MOE_ERR_SHAPE, MOE_ERR_UNSUPPORTED,
 * MOE_ERR_CUDA.                                                          */
MOE_API moe_status moe_router_topk(const uint16_t* x, const uint16_t* w_router, int32_t T,
                                   int32_t D, int32_t E, int32_t k, float* logits,
                                   int32_t* topk_idx, float* topk_w, int32_t* d_status,
                                   moe_stream stream);

/* moe_permute -- group the T*k routed slots by expert.
 * Passage: "MXFP4-based MoE technical review", section 4 (routing and its
 * parallelisation as the core difficulty of sparse experts).
 *   topk_idx    in   [T][k] int32, every entry in [0, E)
 *   x           in   [T][D] bf16
 *   counts      out  [E]   slots routed to each expert
 *   offsets     out  [E+1] exclusive prefix sum of counts (offsets[E] = S)
 *   sorted_slot out  [S]   slots grouped by expert (experts ascending),
 *                          ascending slot order inside each expert
 *   slot_pos    out  [S]   inverse: sorted_slot[slot_pos[s]] == s
 *   x_perm      out  [S][D] bf16, x_perm[p] = x[sorted_slot[p] / k]
 *   ws          in   device workspace of moe_workspace_size(shape, 0) bytes
 * Errors: MOE_ERR_INVALID_ARG, MOE_ERR_SHAPE, MOE_ERR_WORKSPACE,
 * MOE_ERR_UNSUPPORTED, MOE_ERR_CUDA.                                     */
MOE_API moe_status moe_permute(const int32_t* topk_idx, const uint16_t* x,
                       moe_shape shape, int32_t* counts, int32_t* offsets,
                       int32_t* sorted_slot, int32_t* slot_pos,
                       uint16_t* x_perm, void* ws, size_t ws_bytes,
                       moe_stream stream);

/* moe_expert_mlp -- grouped SwiGLU expert MLP on MXFP4 weights.
 * Passage: SwiGLU experts ("Welcome GPT OSS ...", section 4); MXFP4-aware
 * GEMMs ("Tricks from OpenAI gpt-oss ...", section 8); weights raised to
 * bf16 only for compute (aitrends.kr, "Hardware optimisation").
 * For every expert e and every permuted row r in [offsets[e], offsets[e+1]):
 *   g = x_perm[r] . Wg_e^T, u = x_perm[r] . Wu_e^T   (fp32 accumulation of
 *                                                    exact bf16 products)
 *   h[r] = bf16_rne(silu(g) * u),   silu(g) = g / (1 + exp(-g))
 *   y_perm[r] = bf16_rne(h[r] . Wd_e^T)
 *   x_perm  in   [S][D] bf16
 *   offsets in   [E+1] as produced by moe_permute
 *   wgu_q/s in   MXFP4 [E][2F][D]; wdn_q/s in MXFP4 [E][D][F]; the code
 *                arrays wgu_q and wdn_q 32-byte aligned
 *   h       out  [S][F] bf16 (caller-owned intermediate)
 *   y_perm  out  [S][D] bf16
 *   ws      in   device workspace of moe_workspace_size(shape, 1) bytes,
 *                16-byte aligned; its first 4 bytes are the device status
 *                word, cleared by the call and set to MOE_ERR_TIMEOUT if a
 *                bounded wait gave up (read it after the stream syncs)
 * Errors: MOE_ERR_INVALID_ARG, MOE_ERR_SHAPE, MOE_ERR_WORKSPACE,
 * MOE_ERR_UNSUPPORTED, MOE_ERR_CUDA; device status MOE_ERR_TIMEOUT.      */
MOE_API moe_status moe_expert_mlp(const uint16_t* x_perm, const int32_t* offsets,
                          moe_shape shape, const uint8_t* wgu_q,
                          const uint8_t* wgu_s, const uint8_t* wdn_q,
                          const uint8_t* wdn_s, uint16_t* h, uint16_t* y_perm,
                          void* ws, size_t ws_bytes, moe_stream stream);

/* moe_expert_mlp_ex -- moe_expert_mlp with the GEMM path chosen by the
 * caller.  Same operation, passages, arguments and errors as
 * moe_expert_mlp; the results of the two paths agree within the layer
 * tolerance (both take exact products of the bf16 rows and the MXFP4
 * weights; only the fp32 accumulation order differs, and the block-scaled
 * path drops bits of an activation more than 2^13 below its 32-block's
 * largest, below 2^-20 of that largest).
 *   path  MOE_MLP_PATH_AUTO: the path moe_expert_mlp takes (block-scaled
 *         when twice the mean routed rows per expert is at most 64);
 *         MOE_MLP_PATH_BLOCK_SCALED: tcgen05 block-scaled MMAs on the E2M1
 *         codes, each bf16 row split exactly into two E4M3 pieces;
 *         MOE_MLP_PATH_BF16_DECODE: the codes decoded to bf16 into tensor
 *         memory, bf16 MMAs.  Any other value: MOE_ERR_INVALID_ARG.
 *   ws    moe_workspace_size(shape, 1, 3 or 4) bytes for AUTO, BLOCK_SCALED
 *         or BF16_DECODE respectively; first 4 bytes = device status word.
 *   test_timeout_cta  testing support, -1 in normal use.  A value c >= 0
 *         makes the first pipeline wait of the MMA issuer in CTA c of the
 *         first GEMM launch (on the block-scaled path, the one launch of
 *         both GEMMs) give up after a short bounded wait on a barrier that
 *         nothing completes, as a real timeout would: the device status
 *         word becomes MOE_ERR_TIMEOUT, every CTA unwinds after draining
 *         its own copies and MMAs (a CTA waiting on work that CTA c took
 *         and left undone gives up after the wait limit, 2 s), and the
 *         outputs are unspecified.  The next call runs normally.          */
#define MOE_MLP_PATH_AUTO 0
#define MOE_MLP_PATH_BLOCK_SCALED 1
#define MOE_MLP_PATH_BF16_DECODE 2
MOE_API moe_status moe_expert_mlp_ex(const uint16_t* x_perm, const int32_t* offsets,
                                     moe_shape shape, const uint8_t* wgu_q,
                                     const uint8_t* wgu_s, const uint8_t* wdn_q,
                                     const uint8_t* wdn_s, uint16_t* h, uint16_t* y_perm,
                                     void* ws, size_t ws_bytes, int32_t path,
                                     int32_t test_timeout_cta, moe_stream stream);

/* moe_expert_mlp_unquantised -- the grouped SwiGLU expert MLP with
 * unquantised bf16 expert weights: the comparison point for the MXFP4 path.
 * Passage: "Tricks from OpenAI gpt-oss you can use with transformers"
 * (summary), section 7, and agentlenshq (ja), "What is MXFP4" (without
 * MXFP4 the experts are held in bf16, about four times the memory);
 * SwiGLU experts ("Welcome GPT OSS ...", section 4).
 * For every expert e and every permuted row r in [offsets[e], offsets[e+1]):
 *   g = x_perm[r] . Wg_e^T, u = x_perm[r] . Wu_e^T   (fp32 accumulation of
 *                                                    exact bf16 products)
 *   h[r] = bf16_rne(silu(g) * u),   y_perm[r] = bf16_rne(h[r] . Wd_e^T)
 *   x_perm  in   [S][D] bf16; offsets in [E+1] as produced by moe_permute
 *   w_gu    in   bf16 [E][2F][D] (rows [0,F) gate, [F,2F) up)
 *   w_dn    in   bf16 [E][D][F]
 *   h       out  [S][F] bf16 (caller-owned intermediate)
 *   y_perm  out  [S][D] bf16
 *   ws      in   moe_workspace_size(shape, 5) bytes; first 4 bytes = device
 *                status word (cleared by the call; MOE_ERR_TIMEOUT if a
 *                bounded wait gave up)
 * Errors: MOE_ERR_INVALID_ARG, MOE_ERR_SHAPE, MOE_ERR_WORKSPACE,
 * MOE_ERR_UNSUPPORTED, MOE_ERR_CUDA; device status MOE_ERR_TIMEOUT.      */
MOE_API moe_status moe_expert_mlp_unquantised(const uint16_t* x_perm, const int32_t* offsets,
                                              moe_shape shape, const uint16_t* w_gu,
                                              const uint16_t* w_dn, uint16_t* h,
                                              uint16_t* y_perm, void* ws, size_t ws_bytes,
                                              moe_stream stream);

/* moe_combine -- routing-weighted, deterministic gather-sum.
 * Passage: "Welcome GPT OSS ..." (summary), section 4 (the softmax weights
 * of the chosen experts mix their outputs).
 * out[t][d] = bf16_rne( sum_{j=0..k-1, ascending} topk_w[t][j] *
 *                       y_perm[slot_pos[t*k+j]][d] ), summed in fp32.
 *   y_perm   in  [S][D] bf16; slot_pos in [S]; topk_w in [T][k] fp32
 *   out      out [T][D] bf16
 * Errors: MOE_ERR_INVALID_ARG, MOE_ERR_SHAPE, MOE_ERR_UNSUPPORTED,
 * MOE_ERR_CUDA.                                                          */
MOE_API moe_status moe_combine(const uint16_t* y_perm, const int32_t* slot_pos,
                       const float* topk_w, moe_shape shape, uint16_t* out,
                       moe_stream stream);

/* moe_layer_forward -- the whole layer: moe_route -> moe_permute ->
 * moe_expert_mlp -> moe_combine, enqueued on one stream, all intermediates
 * in the caller's workspace (moe_workspace_size(shape, 2) bytes).
 *   x in [T][D] bf16; logits in [T][E] fp32; weights as moe_expert_mlp;
 *   out out [T][D] bf16.  The first 4 bytes of ws are the device status
 *   word; the call's first kernel resets it to MOE_OK.  Every check that
 *   can refuse the call (shape, pointers, workspace, device, the GEMM
 *   configuration and its tensor maps) is made before the first launch.
 * Errors: the union of the four calls.                                   */
MOE_API moe_status moe_layer_forward(const uint16_t* x, const float* logits,
                             moe_shape shape, const uint8_t* wgu_q,
                             const uint8_t* wgu_s, const uint8_t* wdn_q,
                             const uint8_t* wdn_s, uint16_t* out, void* ws,
                             size_t ws_bytes, moe_stream stream);

/* moe_layer_forward_static -- moe_layer_forward without a caller-supplied
 * workspace.  The pages have no counterpart: this entry exists for callers
 * that cannot allocate device memory themselves -- code embedded in a host
 * application or framework that owns every device allocation and hands out
 * no allocator, plug-ins that may only use buffers they are given, or paths
 * where a cudaMalloc (which may synchronise the device) is not acceptable.
 * It allocates nothing and calls no allocating routine: the intermediates
 * live in a device array of MOE_STATIC_SCRATCH_BYTES (16 MiB) inside the
 * library, which every GPU that loads the library holds until the process
 * exits.  The first call on a device looks up that array's device address
 * (cudaGetSymbolAddress, with the device current); make that first call
 * before any stream capture.  A lookup that fails (MOE_ERR_CUDA) is not
 * remembered: the next call on that device tries again.
 *   Arguments, layouts and errors are those of moe_layer_forward, minus the
 *   workspace.  A shape with moe_workspace_size(shape, 2) above
 *   MOE_STATIC_SCRATCH_BYTES is rejected with MOE_ERR_WORKSPACE before
 *   anything runs (at d_model = d_ff = 2880, E = 32 and k = 4 that allows
 *   T <= 113).
 *   Every call uses the same array, and the array keeps the previous call's
 *   contents: each call clears the part that must start at zero (the device
 *   status word) and overwrites the rest before reading it.  Calls that can
 *   overlap on the GPU (other streams, other threads) race on the array and
 *   must be serialised by the caller.  The layer's device status word
 *   (MOE_ERR_TIMEOUT if a bounded wait gave up) lives in the array too:
 *   moe_layer_static_status copies it out.                              */
#define MOE_STATIC_SCRATCH_BYTES (16u << 20)
MOE_API moe_status moe_layer_forward_static(const uint16_t* x, const float* logits,
                                            moe_shape shape, const uint8_t* wgu_q,
                                            const uint8_t* wgu_s, const uint8_t* wdn_q,
                                            const uint8_t* wdn_s, uint16_t* out,
                                            moe_stream stream);

/* moe_layer_static_status -- the device status word of the last
 * moe_layer_forward_static call on the current device, copied on `stream`
 * (one 4-byte device-to-device copy, no allocation) into d_status, a
 * caller-owned, 4-byte aligned device int32; read it after the stream
 * syncs.  Like the entry it serves, it has no counterpart in the pages.
 * Errors: MOE_ERR_INVALID_ARG, MOE_ERR_UNSUPPORTED, MOE_ERR_CUDA.        */
MOE_API moe_status moe_layer_static_status(int32_t* d_status, moe_stream stream);

/* moe_workspace_size -- bytes of device workspace a call needs.
 * which: 0 = moe_permute, 1 = moe_expert_mlp, 2 = moe_layer_forward,
 * 3 = moe_expert_mlp_ex with MOE_MLP_PATH_BLOCK_SCALED,
 * 4 = moe_expert_mlp_ex with MOE_MLP_PATH_BF16_DECODE,
 * 5 = moe_expert_mlp_unquantised.
 * Returns 0 for an unsupported shape or an unknown `which`.  Host only.  */
MOE_API size_t moe_workspace_size(moe_shape shape, int which);

/* moe_status_string -- static, human-readable name of a status. */
MOE_API const char* moe_status_string(moe_status status);

#ifdef __cplusplus
}
#endif

#endif /* MOE_MXFP4_H */
