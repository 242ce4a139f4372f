// rmm_ctx.cu -- context-block reduction of Q K^T (the sequence direction).
//
// Input-adaptive matrix-product reduction for LLM inference (cf-1.com post),
// §3.1: in generation the cached keys are cut into blocks of consecutive
// positions, a cheap score tells which blocks may draw real attention, and
// the full Q K^T (and softmax . V) runs on the kept blocks only; §7: the gain
// grows with the context.  Readings of what the post leaves open:
//   block j       positions [j*bc, min(L, (j+1)*bc)), bc in {32, 64, 128, 256}
//   summary       the block's mean key  mean_j[c] = (sum_l K[l,c]) / n_j, kept
//                 beside the cache (fp32 [B, Hkv, ceil(ldL/bc), d]) and
//                 refreshed for the blocks that change as keys are appended
//   score         for a kept set (a KV head's stacked query rows, or one
//                 query head's rows): the largest dot product of one of its
//                 query rows with mean_j
//   kept blocks   kc = ceil(r_ctx * nblk) best under (score desc, index asc),
//                 ascending; keys of dropped blocks take no part in the
//                 softmax
// Summary and score decide an integer set, so they are computed in single
// precision in one fixed order: float additions over l ascending from 0,
// then one correctly rounded division by n_j; the dot product as an fmaf
// chain over c ascending from 0.
//
// Kernels:
//   ctx_means_kernel   one CTA per (block, KV head), thread c sums row c of
//                      the d-major K^T cache over the block (16-byte loads)
//   ctx_score_kernel   a CTA per (set, 32 blocks): their mean keys and the
//                      set's query rows staged in shared memory, a thread per
//                      (block, row slot) running fmaf chains; the best dot
//                      written as an order-preserving 32-bit key (-0 and +0
//                      share a key)
//   ctx_select_reg_kernel  one CTA per set, a thread per block (up to 1024):
//                      bitonic sort of (key desc, block asc) in registers,
//                      shuffles inside a warp, shared memory across warps;
//                      then the kept blocks listed ascending by one scan
//   ctx_select_kernel  the same sort in shared memory for 1025-2048 blocks
// The attention itself is the split pass of rmm_attn.cu over the kept blocks.
#include <math.h>

#include "rmm_common.cuh"
#include "rmm_internal.h"

namespace rmm {

namespace {

constexpr int D = 128;
constexpr int kSelThreads = 1024;

__global__ void __launch_bounds__(D)
    ctx_means_kernel(const uint16_t* __restrict__ Kt, int L, int ldL, int bc, int blk_begin, int nblk_stride,
                     float* __restrict__ means) {
    pdl_wait();
    pdl_launch_dependents();
    const int j = blk_begin + blockIdx.x;
    const int bg = blockIdx.y;  // b * Hkv + g
    const int c = threadIdx.x;
    const int l0 = j * bc, l1 = min(L, l0 + bc);
    const uint16_t* row = Kt + ((size_t)bg * D + c) * ldL;
    float sum = 0.0f;
    int l = l0;
    for (; l + 8 <= l1; l += 8) {  // l0 is a multiple of 32 and ldL of 8: 16-byte aligned
        const uint4 v = ld_nc_v4(row + l);
        sum += __uint_as_float(v.x << 16);
        sum += __uint_as_float(v.x & 0xFFFF0000u);
        sum += __uint_as_float(v.y << 16);
        sum += __uint_as_float(v.y & 0xFFFF0000u);
        sum += __uint_as_float(v.z << 16);
        sum += __uint_as_float(v.z & 0xFFFF0000u);
        sum += __uint_as_float(v.w << 16);
        sum += __uint_as_float(v.w & 0xFFFF0000u);
    }
    for (; l < l1; ++l) sum += bf16_bits_to_float(row[l]);
    means[((size_t)bg * nblk_stride + j) * D + c] = __fdiv_rn(sum, (float)(l1 - l0));
}

// Order-preserving key of a finite float: larger float, larger key; -0 -> +0.
__device__ __forceinline__ uint32_t float_key(float f) {
    if (f == 0.0f) f = 0.0f;
    const uint32_t b = __float_as_uint(f);
    return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

// CTA = 32 blocks x 4 row slots (128 threads): the 32 blocks' mean keys and
// 16 query rows at a time are staged in shared memory (rows padded to 129
// floats: conflict-free column reads), thread (block, slot) runs the fmaf
// chain of rows slot, slot + 4, ... over the 128 dims in order and keeps the
// best; the 4 slots' bests are folded by shuffles (a max: exact).
constexpr int kScoreBlocks = 32;
__global__ void __launch_bounds__(128)
    ctx_score_kernel(const uint16_t* __restrict__ Q, const float* __restrict__ means, int Hq, int Hkv, int T,
                     int nblk, int nblk_stride, int per_query_head, uint32_t* __restrict__ keys) {
    __shared__ float qs[16][D + 1];
    __shared__ float mt[kScoreBlocks][D + 1];
    const int nsets = per_query_head ? Hq : Hkv;
    const int set = blockIdx.y % nsets;
    const int b = blockIdx.y / nsets;
    const int G = Hq / Hkv;
    const int g = per_query_head ? set / G : set;
    const int q_lo = per_query_head ? set : set * G;
    const int nq = per_query_head ? 1 : G;
    const int R = nq * T;
    const int tid = threadIdx.x;
    const int bl = tid >> 2, slot = tid & 3;
    const int j0 = blockIdx.x * kScoreBlocks;
    const int j = j0 + bl;
    pdl_wait();
    pdl_launch_dependents();
    // the 32 mean keys: 128 threads x 8 float4, coalesced
    const float4* m4 = reinterpret_cast<const float4*>(means + ((size_t)(b * Hkv + g) * nblk_stride + j0) * D);
#pragma unroll
    for (int u = 0; u < 8; ++u) {
        const int e = tid + 128 * u;  // float4 index in the tile: block e / 32, dims 4 * (e % 32) ..
        const int eb = e >> 5, ec = (e & 31) * 4;
        const float4 v = (j0 + eb < nblk) ? __ldg(m4 + e) : make_float4(0.f, 0.f, 0.f, 0.f);
        mt[eb][ec] = v.x;
        mt[eb][ec + 1] = v.y;
        mt[eb][ec + 2] = v.z;
        mt[eb][ec + 3] = v.w;
    }
    float best = -INFINITY;
    for (int r0 = 0; r0 < R; r0 += 16) {
        __syncthreads();
        // 16 rows x 128 dims: two 16-byte pieces per thread, both loads in flight
        uint4 piece[2];
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            const int e = tid + 128 * u, rr = e / 16, r = r0 + rr;
            piece[u] = r < R ? ld_nc_v4(Q + (((size_t)b * Hq + q_lo + r / T) * T + r % T) * D + (e % 16) * 8)
                             : make_uint4(0u, 0u, 0u, 0u);
        }
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            const int e = tid + 128 * u, rr = e / 16, c = (e % 16) * 8;
            const uint32_t w[4] = {piece[u].x, piece[u].y, piece[u].z, piece[u].w};
#pragma unroll
            for (int h = 0; h < 4; ++h) {
                qs[rr][c + 2 * h] = __uint_as_float(w[h] << 16);
                qs[rr][c + 2 * h + 1] = __uint_as_float(w[h] & 0xFFFF0000u);
            }
        }
        __syncthreads();
        const int nr = min(16, R - r0);
        for (int rr = slot; rr < nr; rr += 4) {
            float acc = 0.0f;
#pragma unroll 16
            for (int c = 0; c < D; ++c) acc = fmaf(qs[rr][c], mt[bl][c], acc);
            if (acc > best) best = acc;
        }
    }
    best = fmaxf(best, __shfl_xor_sync(0xffffffffu, best, 1));
    best = fmaxf(best, __shfl_xor_sync(0xffffffffu, best, 2));
    if (slot == 0 && j < nblk) keys[(size_t)blockIdx.y * nblk + j] = float_key(best);
}

// One CTA of P threads per set (P = the power of two >= nblk, at most 1024):
// thread i holds element i of (key desc, block asc) packed in 64 bits; a
// bitonic sort in registers, partners within a warp by shuffle and across
// warps through shared memory (two barriers per such stage); the first kc
// elements are the kept blocks, listed ascending by one block-wide scan.
__global__ void __launch_bounds__(kSelThreads)
    ctx_select_reg_kernel(const uint32_t* __restrict__ keys, int nblk, int kc, int32_t* __restrict__ blocks) {
    __shared__ uint64_t xs[kSelThreads];
    __shared__ uint8_t flag[kSelThreads];
    __shared__ int warp_sum[kSelThreads / 32];
    pdl_wait();
    pdl_launch_dependents();
    const int P = blockDim.x;
    const int i = threadIdx.x, lane = i & 31, warp = i >> 5;
    const uint32_t* key = keys + (size_t)blockIdx.x * nblk;
    uint64_t v = i < nblk ? ((uint64_t)(~key[i]) << 32) | (uint32_t)i : ~0ull;
    flag[i] = 0;
    for (int k2 = 2; k2 <= P; k2 <<= 1)
        for (int jj = k2 >> 1; jj > 0; jj >>= 1) {
            uint64_t o;
            if (jj >= 32) {
                xs[i] = v;
                __syncthreads();
                o = xs[i ^ jj];
                __syncthreads();
            } else {
                o = __shfl_xor_sync(0xffffffffu, v, jj);
            }
            // the lower index of a pair takes the smaller value in an ascending run
            const bool take_min = ((i & k2) == 0) == (i < (i ^ jj));
            v = take_min ? (o < v ? o : v) : (o < v ? v : o);
        }
    __syncthreads();
    if (i < kc) flag[(uint32_t)v] = 1;
    __syncthreads();
    const int cnt = flag[i];
    int incl = cnt;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
    }
    if (lane == 31) warp_sum[warp] = incl;
    __syncthreads();
    int pos = incl - cnt;
    for (int w = 0; w < warp; ++w) pos += warp_sum[w];
    if (cnt) blocks[(size_t)blockIdx.x * kc + pos] = i;
}

// The same selection for 1025-2048 blocks: the sort in shared memory (P
// entries, up to two per thread), a barrier per stage.
__global__ void __launch_bounds__(kSelThreads)
    ctx_select_kernel(const uint32_t* __restrict__ keys, int nblk, int P, int kc, int32_t* __restrict__ blocks) {
    extern __shared__ uint64_t v[];  // P entries
    __shared__ uint8_t flag[2 * kSelThreads];
    __shared__ int warp_sum[kSelThreads / 32];
    pdl_wait();
    pdl_launch_dependents();
    const int tid = threadIdx.x;
    const uint32_t* key = keys + (size_t)blockIdx.x * nblk;
    // ascending order of (~key, block) = (score desc, block asc)
    for (int i = tid; i < P; i += kSelThreads)
        v[i] = i < nblk ? ((uint64_t)(~key[i]) << 32) | (uint32_t)i : ~0ull;
    for (int i = tid; i < 2 * kSelThreads; i += kSelThreads) flag[i] = 0;
    __syncthreads();
    for (int k2 = 2; k2 <= P; k2 <<= 1)
        for (int jj = k2 >> 1; jj > 0; jj >>= 1) {
            for (int i = tid; i < P; i += kSelThreads) {
                const int ixj = i ^ jj;
                if (ixj > i) {
                    const uint64_t a = v[i], c = v[ixj];
                    if ((a > c) == ((i & k2) == 0)) {
                        v[i] = c;
                        v[ixj] = a;
                    }
                }
            }
            __syncthreads();
        }
    for (int i = tid; i < kc; i += kSelThreads) flag[(uint32_t)v[i]] = 1;
    __syncthreads();
    // thread t owns blocks 2t and 2t+1: exclusive scan of the kept counts
    const int cnt = flag[2 * tid] + flag[2 * tid + 1];
    const int lane = tid & 31, warp = tid >> 5;
    int incl = cnt;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
    }
    if (lane == 31) warp_sum[warp] = incl;
    __syncthreads();
    int pos = incl - cnt;
    for (int w = 0; w < warp; ++w) pos += warp_sum[w];
    int32_t* out = blocks + (size_t)blockIdx.x * kc;
    if (flag[2 * tid]) out[pos++] = 2 * tid;
    if (flag[2 * tid + 1]) out[pos] = 2 * tid + 1;
}

}  // namespace

bool ctx_block_ok(int bc) { return bc == 32 || bc == 64 || bc == 128 || bc == 256; }

cudaError_t launch_ctx_means(const uint16_t* Kt, int B, int Hkv, int L, int ldL, int bc, int blk_begin, int blk_end,
                             float* means, cudaStream_t stream) {
    const int nblk_stride = (ldL + bc - 1) / bc;
    return launch_pdl(ctx_means_kernel, dim3(blk_end - blk_begin, B * Hkv), dim3(D), 0, stream, Kt, L, ldL, bc,
                      blk_begin, nblk_stride, means);
}

cudaError_t launch_attn_ctx(const uint16_t* Q, const uint16_t* Kt, const uint16_t* V, const float* means, int B,
                            int Hq, int Hkv, int T, int L, int ldL, int k, int bc, int kc, int causal, float scale,
                            int per_query_head, uint16_t* O, int32_t* idx, uint32_t* sc, uint32_t* keys,
                            int32_t* blocks, float* partials, const AttnPlan& p, cudaStream_t stream) {
    const int nblk = (L + bc - 1) / bc;
    const int nblk_stride = (ldL + bc - 1) / bc;
    int P = 2;
    while (P < nblk) P <<= 1;
    if (P > 2 * kSelThreads) return cudaErrorInvalidValue;
    int bc_shift = 0;
    while ((1 << bc_shift) < bc) ++bc_shift;
    const bool select_here = attn_dims_in_split(Hq, Hkv, T, per_query_head);
    cudaError_t e = cudaSuccess;
    if (!select_here) e = launch_attn_dims(Q, B, Hq, Hkv, T, k, per_query_head, p.nsets, idx, sc, stream);
    if (e != cudaSuccess) return e;
    e = launch_pdl(ctx_score_kernel, dim3((nblk + kScoreBlocks - 1) / kScoreBlocks, B * p.nsets), dim3(128), 0,
                   stream, Q, means, Hq, Hkv, T, nblk, nblk_stride, per_query_head, keys);
    if (e != cudaSuccess) return e;
    if (P <= kSelThreads)
        e = launch_pdl(ctx_select_reg_kernel, dim3(B * p.nsets), dim3(P < 32 ? 32 : P), 0, stream,
                       (const uint32_t*)keys, nblk, kc, blocks);
    else
        e = launch_pdl(ctx_select_kernel, dim3(B * p.nsets), dim3(kSelThreads), (size_t)P * sizeof(uint64_t), stream,
                       (const uint32_t*)keys, nblk, P, kc, blocks);
    if (e != cudaSuccess) return e;
    return launch_attn_split_ctx(Q, Kt, V, B, Hq, Hkv, T, L, ldL, k, causal, scale, per_query_head, O, idx,
                                 (int)select_here, blocks, bc_shift, kc, partials, p, stream);
}

}  // namespace rmm
