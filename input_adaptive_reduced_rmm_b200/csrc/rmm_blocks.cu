// rmm_blocks.cu -- block-granular kept sets.
//
// The kept set chosen per block of `block` consecutive contraction slices, as
// in the FFN demo of the cf-1.com post on input-adaptive matrix-product
// reduction (§6.1: 64-wide blocks of the down projection's input scored from
// the current activation, top-k of the block scores, sorted; §3.3 / §6.2:
// blocks suit the tensor cores).  Block j covers slices [j*block, (j+1)*block);
// its score is the largest of its slices' scores max_t |X[t,h]| -- a max, so
// the score stays exact and independent of summation order -- and the kb best
// blocks under (score desc, block index asc) are kept.  The kernel emits the
// ascending list of their slices (kb * block entries), which the reduced
// GEMM and GEMV consume like any kept list: each kept block is `block`
// contiguous rows of W^T and of X^T.
//
// One CTA of 1024 threads, thread j = block j (at most 1024 blocks): the block
// max of the score vector (cleared behind the read for the next call), an
// exact rank among the block scores, one block-wide scan for the output
// position, then the block's slices written out.
#include "rmm_common.cuh"
#include "rmm_internal.h"

namespace rmm {

namespace {

constexpr int kThreads = 1024;

// X non-null: mean-magnitude blocks (T <= 16 tokens of X [T, H]); the block
// score is then the bit pattern of a non-negative float, which orders like
// the float.  s32 is cleared either way (the score pass may have filled it).
__global__ void __launch_bounds__(kThreads)
    block_select_kernel(uint32_t* __restrict__ s32, const uint16_t* __restrict__ X, int T, int H, int block, int kb,
                        int32_t* __restrict__ idx, int32_t* __restrict__ idx_copy, int32_t* __restrict__ blocks_out) {
    __shared__ uint32_t bs[kThreads];
    __shared__ int warp_cnt[kThreads / 32];
    pdl_wait();
    pdl_launch_dependents();
    const int j = threadIdx.x, lane = j & 31, warp = j >> 5;
    const int nb = H / block;
    uint32_t m = 0;
    if (j < nb) {
        if (X) {
            // sum over tokens ascending, within a token the block's slices
            // ascending (16-byte loads of 8 slices, added in order)
            float sum = 0.0f;
            for (int t = 0; t < T; ++t) {
                const uint16_t* row = X + (size_t)t * H + (size_t)j * block;
                for (int i = 0; i < block; i += 8) {
                    const uint4 v = ld_nc_v4(row + i);
                    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        sum += __uint_as_float((w[u] << 16) & 0x7FFF0000u);
                        sum += __uint_as_float(w[u] & 0x7FFF0000u);
                    }
                }
            }
            m = __float_as_uint(__fdiv_rn(sum, (float)(T * block)));
            for (int i = 0; i < block; ++i) s32[j * block + i] = 0;
        } else {
            for (int i = 0; i < block; ++i) {
                const int h = j * block + i;
                m = max(m, s32[h] & 0xFFFFu);
                s32[h] = 0;
            }
        }
    }
    bs[j] = m;
    __syncthreads();
    // rank under (score desc, block index asc)
    int rank = 0;
    if (j < nb)
        for (int i = 0; i < nb; ++i) {
            const uint32_t v = bs[i];
            rank += (v > m) || (v == m && i < j);
        }
    const bool keep = j < nb && rank < kb;
    const unsigned ball = __ballot_sync(0xffffffffu, keep);
    if (lane == 0) warp_cnt[warp] = __popc(ball);
    __syncthreads();
    int pos = __popc(ball & ((1u << lane) - 1u));
    for (int w = 0; w < warp; ++w) pos += warp_cnt[w];
    if (keep) {
        if (blocks_out) blocks_out[pos] = j;
        for (int i = 0; i < block; ++i) {
            idx[pos * block + i] = j * block + i;
            if (idx_copy) idx_copy[pos * block + i] = j * block + i;
        }
    }
}

}  // namespace

bool block_size_ok(int H, int block) {
    if (block == 0) return true;
    if (block != 16 && block != 32 && block != 64 && block != 128 && block != 256) return false;
    return H % block == 0 && H / block <= kThreads;
}

cudaError_t launch_block_select(uint32_t* s32, const uint16_t* X, int T, int H, int block, int kb, int32_t* idx,
                                int32_t* idx_copy, int32_t* blocks_out, cudaStream_t stream) {
    if (!block_size_ok(H, block) || block == 0 || kb < 1 || kb > H / block) return cudaErrorInvalidValue;
    return launch_pdl(block_select_kernel, dim3(1), dim3(kThreads), 0, stream, s32, X, T, H, block, kb, idx, idx_copy,
                      blocks_out);
}

}  // namespace rmm
