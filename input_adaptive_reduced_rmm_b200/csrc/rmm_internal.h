// rmm_internal.h -- host-side launchers shared between the library's .cu files.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace rmm {

constexpr int kGemvMaxT = 16;          // largest T of the split-K GEMV
constexpr int kGemmBK = 64;            // kept slices per GEMM pipeline stage (idx padded to this)

// ---- score (rmm_score.cu)
// Folds max_t |X[t,h]| into s32[h] (u32 [H], must hold zeros or smaller
// keys on entry); on the GEMM path (Xt != null) also writes X^T [H, ldT].
cudaError_t launch_score(const uint16_t* X, int T, int H, uint32_t* s32, uint16_t* Xt, int ldT,
                         int num_sms, cudaStream_t stream);

// ---- select (rmm_select.cu)
// Scores: max_t |X[t,h]| folded from X [T, H] when X is not null (decode-sized
// T: score and selection in one launch), else read from s32 (u32 [H]; zeroed
// afterwards when clear_input != 0).  Optionally stores the scores to s_out,
// and writes the k best indices ascending to idx[0..k), then
// idx[k..pad_to) = H; idx_copy (if not null) receives the same k indices
// without padding.
cudaError_t launch_select(const uint16_t* X, int T, uint32_t* s32, int clear_input, int H, int k, int32_t* idx,
                          int pad_to, int32_t* idx_copy, uint32_t* s_out, cudaStream_t stream);

// ---- block-granular kept sets (rmm_blocks.cu)
// block 0 (single slices) or 16..256 dividing H with at most 1024 blocks
bool block_size_ok(int H, int block);
// The kb best blocks of `block` slices -- block score = max of its slices'
// scores from s32 (u32 [H]), or, with X [T, H] given (T <= 16), the block's
// mean magnitude -- their kb * block slices ascending to idx (and idx_copy if
// not null), the blocks to blocks_out if not null; s32 is zeroed afterwards.
cudaError_t launch_block_select(uint32_t* s32, const uint16_t* X, int T, int H, int block, int kb, int32_t* idx,
                                int32_t* idx_copy, int32_t* blocks_out, cudaStream_t stream);

// ---- split-K GEMV (rmm_gemv.cu)
constexpr int kMaxGroupGemv = 4;
// Up to 4 decode products sharing X and the kept list, planned by
// gemv_group_plan (fill count, Wt, Y, N first).
struct GemvGroup {
    const uint16_t* Wt[kMaxGroupGemv];
    uint16_t* Y[kMaxGroupGemv];
    int N[kMaxGroupGemv];               // output columns of the member
    int ld[kMaxGroupGemv];              // row stride (elements) of its W^T and Y; N when 0 at planning
    int col_blocks[kMaxGroupGemv];
    int splits[kMaxGroupGemv];          // the same for every member
    int rows_per_split[kMaxGroupGemv];
    int item_start[kMaxGroupGemv + 1];  // prefix sums of col_blocks (grid x of the product)
    int fold_start[kMaxGroupGemv + 1];  // prefix sums of 256-column blocks (grid x of the fold)
    size_t partial_off[kMaxGroupGemv];  // float offsets of each member's split partials
    int cols;                           // outputs per column block
    int count;
    int swiglu;                         // 1: members 0 and 1 are gate and up; Y[0] = bf16(silu(g) * u)
};
int gemv_cols_for(int T);
// Fills the plan; returns the bytes of split partial sums the group needs.
size_t gemv_group_plan(GemvGroup& g, int T, int k, int forced_splits, int num_sms);
// Upper bound of gemv_group_plan's partial bytes over every k <= H (needs g.N, g.count).
size_t gemv_partials_bound(const GemvGroup& g, int T, int H, int forced_splits, int num_sms);
size_t gemv_smem_bytes(int cols, int T);  // dynamic shared memory of one CTA
constexpr size_t kGemvMaxSmemBytes = 200 * 1024;
// The product (and, with more than one split, the fold of the split partials
// in a second launch).  partials: the planned bytes, no initial contents.
// idx null: every slice kept (k == H), read as the identity list.
cudaError_t launch_gemv(const uint16_t* X, int T, int H, const int32_t* idx, int k, const GemvGroup& g,
                        float* partials, int num_sms, cudaStream_t stream);

// ---- tensor-core prefill attention (rmm_attn_tc.cu): query chunks of at
// least kAttnTcMinT tokens, kept sets from the attention select kernel
constexpr int kAttnTcMinT = 16;
bool attn_tc_supported(int T, int k);
// A 3-D tiled map over a bf16 tensor [n2][n1][n0] with row / plane strides ld1 /
// ld2 elements, box 64 x box1 x 1, 128-byte swizzle, zero fill outside
// (defined in rmm_api.cu).
bool tiled_map_3d(const void* base, uint64_t n0, uint64_t n1, uint64_t n2, uint64_t ld1, uint64_t ld2,
                  uint32_t box1, CUtensorMap* out);
cudaError_t launch_exp2_fma(const float* x, float* y, int n, cudaStream_t stream);
cudaError_t launch_attn_tc(const uint16_t* Q, const uint16_t* Kt, const uint16_t* V, int B, int Hq, int Hkv, int T,
                           int L, int ldL, int k, int causal, float scale, int per_query_head, const int32_t* idx,
                           uint16_t* O, int* status, cudaStream_t stream);

// ---- decoder-layer glue (rmm_layer.cu); bf16 in and out, B = 1, d = 128
cudaError_t launch_add_rmsnorm(const uint16_t* X, const uint16_t* R, int T, int H, float eps, const uint16_t* Wn,
                               uint16_t* Hsum, uint16_t* Y, cudaStream_t stream);
cudaError_t launch_swiglu(const uint16_t* G, const uint16_t* U, size_t n, uint16_t* Out, int num_sms,
                          cudaStream_t stream);
cudaError_t launch_qkv_heads(const uint16_t* Yq, const uint16_t* Yk, const uint16_t* Yv, int T, int Hq, int Hkv,
                             uint16_t* Q, uint16_t* Kt, uint16_t* V, int ldL, int L0, cudaStream_t stream);
cudaError_t launch_heads_to_tokens(const uint16_t* O, int Hq, int T, uint16_t* A, int num_sms, cudaStream_t stream);

// ---- tcgen05 GEMM (rmm_gemm.cu)
// Up to kMaxGroup products that share the activations (X^T, T, H and the kept
// list) and differ in the weight: one persistent launch walks the tiles of
// all of them.
constexpr int kMaxGroup = 4;
static_assert(kMaxGroup == kMaxGroupGemv, "one group size for both products");
struct GemmGroup {
    const uint16_t* Wt[kMaxGroup];
    uint16_t* Y[kMaxGroup];
    int N[kMaxGroup];
    int tile_start[kMaxGroup + 1];  // prefix sums of the products' tile counts
    int count;
    // Work units of the CTA-pair kernel (set by launch_gemm_pair): tiles
    // [0, units_full) whole, the remaining tiles each cut into tail_splits
    // K-ranges whose fp32 partials go to `partials` and are folded afterwards.
    int units_full, tail_splits, units;
    float* partials;
};
// Fills tile_start for the given T and tile shape (pair != 0: the 256 x 256
// CTA-pair tile, else 128 x 256); returns the total tile count.
int gemm_group_tiles(GemmGroup& g, int T, int pair);
// CTA-pair (tcgen05 cta_group::2) GEMM, cp.async producer; tiles from gemm_group_tiles(g, T, 1).
// partials: gemm_pair_partial_bytes(num_sms) of scratch for the split last
// wave (null: no split).
// Output tensor maps of the group's products (Y [T, N] bf16, box 32 rows x 64
// columns, 128-byte swizzle): the epilogue stores its tiles with TMA.
struct __align__(64) GemmOutMaps {
    CUtensorMap m[kMaxGroup];
};
// Input tensor maps for kept lists made of whole 64-slice runs (block-granular
// sets): X^T [H, T] and each member's W^T [H, N], box 64 rows x 64 columns,
// 128-byte swizzle.  With them the GEMM loads its stages by TMA tile copies.
struct __align__(64) GemmInMaps {
    CUtensorMap xt;
    CUtensorMap wt[kMaxGroup];
};
// imaps null: the cp.async gather producer (any kept list).
cudaError_t launch_gemm_pair(const uint16_t* Xt, int ldT, const GemmGroup& group, const GemmOutMaps& ymaps,
                             const GemmInMaps* imaps, const int32_t* idx, int k, int T, int H, float* partials,
                             int* status, int debug_timeout, int num_sms, cudaStream_t stream);
size_t gemm_pair_partial_bytes(int num_sms);
// map_xt / map_wt are used only by the TMA tile::gather4 producer
// (tma_gather != 0), which handles a group of one.
cudaError_t launch_gemm(const CUtensorMap& map_xt, const CUtensorMap& map_wt, const uint16_t* Xt,
                        int ldT, const GemmGroup& group, const int32_t* idx, int k, int T, int H,
                        int* status, int debug_timeout, int tma_gather, int num_sms,
                        cudaStream_t stream);
size_t gemm_smem_bytes();

// ---- attention (rmm_attn.cu)
struct AttnPlan {
    int chunk;    // keys per split
    int nsplit;   // splits over L
    int tq;       // query tokens per CTA
    int nsets;    // kept sets per batch (Hkv or Hq)
    int rows;     // query rows per CTA of the split pass (4 or 8)
};
AttnPlan attn_plan(int B, int Hq, int Hkv, int T, int L, int per_query_head, int num_sms);
size_t attn_partials_bytes(const AttnPlan& p, int B, int Hq, int T);
// path: 0 auto (tensor cores for chunks of kAttnTcMinT+ tokens), 1 the
// CUDA-core split pass, 2 tensor cores.  sc: u32 [B * nsets * d] of zeros
// (left at zero); status: the workspace status word.
cudaError_t launch_attn(const uint16_t* Q, const uint16_t* Kt, const uint16_t* V, int B, int Hq,
                        int Hkv, int T, int L, int ldL, int k, int causal, float scale,
                        int per_query_head, uint16_t* O, int32_t* idx, float* partials, uint32_t* sc,
                        int* status, int path, const AttnPlan& plan, cudaStream_t stream);
// True when the split pass selects the kept head dimensions itself (short
// decode chunks: a set's rows number fewer than 64).
bool attn_dims_in_split(int Hq, int Hkv, int T, int per_query_head);
// The kept head dimensions alone (score + select), as launch_attn runs them.
cudaError_t launch_attn_dims(const uint16_t* Q, int B, int Hq, int Hkv, int T, int k, int per_query_head, int nsets,
                             int32_t* idx, uint32_t* sc, cudaStream_t stream);
// The split pass + combine over kept context blocks (kc blocks of 2^bc_shift
// keys per set, blocks [B * nsets * kc]); plan made for kc << bc_shift keys.
cudaError_t launch_attn_split_ctx(const uint16_t* Q, const uint16_t* Kt, const uint16_t* V, int B, int Hq, int Hkv,
                                  int T, int L, int ldL, int k, int causal, float scale, int per_query_head,
                                  uint16_t* O, int32_t* idx, int select_here, const int32_t* blocks, int bc_shift,
                                  int kc, float* partials, const AttnPlan& p, cudaStream_t stream);

// ---- context-block reduction (rmm_ctx.cu)
constexpr int kCtxMaxBlocks = 2048;  // blocks per cache the select kernel sorts
constexpr int kCtxMaxT = 16;         // query tokens per call (decode and short chunks)
bool ctx_block_ok(int bc);
// Block means of blocks [blk_begin, blk_end): means fp32 [B, Hkv, ceil(ldL/bc), d].
cudaError_t launch_ctx_means(const uint16_t* Kt, int B, int Hkv, int L, int ldL, int bc, int blk_begin, int blk_end,
                             float* means, cudaStream_t stream);
// Dims select, block scores, block select, then the split pass over the kept
// blocks.  keys: u32 [B * nsets * nblk]; blocks: int32 [B * nsets * kc].
cudaError_t launch_attn_ctx(const uint16_t* Q, const uint16_t* Kt, const uint16_t* V, const float* means, int B,
                            int Hq, int Hkv, int T, int L, int ldL, int k, int bc, int kc, int causal, float scale,
                            int per_query_head, uint16_t* O, int32_t* idx, uint32_t* sc, uint32_t* keys,
                            int32_t* blocks, float* partials, const AttnPlan& p, cudaStream_t stream);

// ---- glue (rmm_glue.cu)
cudaError_t launch_transpose(const uint16_t* W, uint16_t* Wt, int N, int H, cudaStream_t stream);
// src null: the identity list 0..k-1 (every slice kept); dst_copy (if not
// null) receives the first k entries.
cudaError_t launch_pad_idx(const int32_t* src, int k, int H, int32_t* dst, int pad_to, cudaStream_t stream,
                           int32_t* dst_copy = nullptr);

}  // namespace rmm
