// rmm_score.cu -- step 1 of the reduced product: the per-slice input score.
//
// s_h = max over tokens t of |X[t,h]|  (cf-1.com post on input-adaptive
// matrix-product reduction, §5.1: a cheap score taken from the current
// activations; one common score for all tokens of the call, §8).
//
// |x| is taken on the bf16 bit pattern with the sign cleared, an integer that
// orders exactly like the magnitude of a finite value, so the maximum is
// exact and independent of the reduction order.
//
// One pass over X [T, H] (HBM-bound: T*H*2 bytes read).  Each CTA owns a
// 64-wide channel strip and a strided subset of 64-token tiles; it folds its
// strip's maximum into the score vector s32[h] with atomicMax (the vector
// starts at zero: the select kernel clears it after reading).  On the GEMM
// path the same pass also writes the
// full transpose X^T [H, ldT] (through a shared-memory tile) so that a kept
// slice of X is one contiguous row that TMA can gather; this is a transposed
// copy of all of X, never a compacted copy of the kept part.
#include "rmm_common.cuh"
#include "rmm_internal.h"

namespace rmm {

namespace {

constexpr int kTileT = 128;  // tokens per tile
constexpr int kTileH = 64;  // channels per strip
constexpr int kThreads = 256;

template <bool kWriteXt, bool kVec>
__global__ void __launch_bounds__(kThreads)
    score_kernel(const uint16_t* __restrict__ X, int T, int H, uint32_t* __restrict__ s32,
                 uint16_t* __restrict__ Xt, int ldT) {
    // Rows of 66 elements (33 words): the transposed reads of 8 rows that are
    // 8 apart then fall on distinct bank groups (2-way conflicts at most).
    __shared__ __align__(16) uint16_t tile[kTileT][kTileH + 2];
    __shared__ uint16_t red[32][kTileH];
    constexpr int kPasses = kTileT / 32;  // 16-byte loads in flight per thread

    pdl_wait();
    pdl_launch_dependents();
    const int tid = threadIdx.x;
    const int cg = tid & 7;    // 8-channel group within the strip
    const int row = tid >> 3;  // 0..31
    const int h0 = blockIdx.x * kTileH;
    const int hc = h0 + cg * 8;

    uint32_t mx[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) mx[i] = 0;

    for (int t0 = blockIdx.y * kTileT; t0 < T; t0 += gridDim.y * kTileT) {
        // issue all of this thread's loads of the tile before using any
        uint4 q[kPasses];
#pragma unroll
        for (int p = 0; p < kPasses; ++p) {
            const int t = t0 + p * 32 + row;
            if (kVec && t < T && hc + 8 <= H) {
                q[p] = ld_nc_v4(X + (size_t)t * H + hc);
            } else {
                uint16_t w[8];
#pragma unroll
                for (int i = 0; i < 8; ++i)
                    w[i] = (t < T && hc + i < H) ? X[(size_t)t * H + hc + i] : (uint16_t)0;
                q[p] = make_uint4(w[0] | ((uint32_t)w[1] << 16), w[2] | ((uint32_t)w[3] << 16),
                                  w[4] | ((uint32_t)w[5] << 16), w[6] | ((uint32_t)w[7] << 16));
            }
        }
#pragma unroll
        for (int p = 0; p < kPasses; ++p) {
            const int r = p * 32 + row;
            uint16_t v[8];
            v[0] = q[p].x & 0xFFFF; v[1] = q[p].x >> 16;
            v[2] = q[p].y & 0xFFFF; v[3] = q[p].y >> 16;
            v[4] = q[p].z & 0xFFFF; v[5] = q[p].z >> 16;
            v[6] = q[p].w & 0xFFFF; v[7] = q[p].w >> 16;
#pragma unroll
            for (int i = 0; i < 8; ++i) mx[i] = max(mx[i], (uint32_t)(v[i] & 0x7FFF));
            if (kWriteXt) {
                uint32_t* d = reinterpret_cast<uint32_t*>(&tile[r][cg * 8]);
                d[0] = v[0] | ((uint32_t)v[1] << 16);
                d[1] = v[2] | ((uint32_t)v[3] << 16);
                d[2] = v[4] | ((uint32_t)v[5] << 16);
                d[3] = v[6] | ((uint32_t)v[7] << 16);
            }
        }
        if (kWriteXt) {
            __syncthreads();
            // transposed write-out: 16 threads per channel row, 8 tokens each
            const int tc = tid & 15;
#pragma unroll
            for (int p = 0; p < kTileH / 16; ++p) {
                const int hl = p * 16 + (tid >> 4);
                const int h = h0 + hl;
                const int tt = t0 + tc * 8;
                if (h < H && tt < T) {
                    uint16_t w[8];
#pragma unroll
                    for (int i = 0; i < 8; ++i) w[i] = tile[tc * 8 + i][hl];
                    uint16_t* dst = Xt + (size_t)h * ldT + tt;
                    if (tt + 8 <= T) {
                        uint4 q;
                        q.x = w[0] | ((uint32_t)w[1] << 16);
                        q.y = w[2] | ((uint32_t)w[3] << 16);
                        q.z = w[4] | ((uint32_t)w[5] << 16);
                        q.w = w[6] | ((uint32_t)w[7] << 16);
                        *reinterpret_cast<uint4*>(dst) = q;
                    } else {
                        for (int i = 0; i < 8 && tt + i < T; ++i) dst[i] = w[i];
                    }
                }
            }
            __syncthreads();
        }
    }

    // fold the 32 row-threads that share each channel group
#pragma unroll
    for (int i = 0; i < 8; ++i) red[row][cg * 8 + i] = (uint16_t)mx[i];
    __syncthreads();
    if (tid < kTileH) {
        uint32_t m = 0;
#pragma unroll 8
        for (int r = 0; r < 32; ++r) m = max(m, (uint32_t)red[r][tid]);
        const int h = h0 + tid;
        if (s32 && h < H && m > 0) atomicMax(s32 + h, m);
    }
}

// The score pass with the X^T copy, transposing in registers (H % 8 == 0,
// X 16-byte aligned).  A CTA of 4 warps covers 64 tokens x 128 channels (about
// seven CTAs per SM: one wave for the prefill shapes);
// lane (g, half) of warp w loads 8 channels x 8 tokens (eight 16-byte loads,
// all in flight), transposes the 8 x 8 block of bf16 with byte permutes and
// stores 8 rows of X^T, 8 tokens each; lanes g and g + 16 fill the two halves
// of one 32-byte sector.  No shared-memory tile.
constexpr int kXtThreads = 128;
constexpr int kXtTokens = 16 * (kXtThreads / 32);

__global__ void __launch_bounds__(kXtThreads)
    score_xt_kernel(const uint16_t* __restrict__ X, int T, int H, uint32_t* __restrict__ s32,
                    uint16_t* __restrict__ Xt, int ldT) {
    __shared__ uint32_t red[kXtThreads / 32][128];
    pdl_wait();
    pdl_launch_dependents();
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int g = lane & 15, half = lane >> 4;
    const int h = blockIdx.x * 128 + 8 * g;                   // first of the thread's 8 channels
    const int tb = blockIdx.y * kXtTokens + 16 * warp + 8 * half;  // first of its 8 tokens
    const bool hok = h < H;                                   // H % 8 == 0: all 8 channels valid
    uint4 q[8];
#pragma unroll
    for (int i = 0; i < 8; ++i)
        q[i] = (hok && tb + i < T) ? ld_nc_v4(X + (size_t)(tb + i) * H + h) : make_uint4(0u, 0u, 0u, 0u);
    uint32_t mx[8];
#pragma unroll
    for (int c = 0; c < 8; ++c) mx[c] = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const uint32_t w[4] = {q[i].x, q[i].y, q[i].z, q[i].w};
#pragma unroll
        for (int m = 0; m < 4; ++m) {
            mx[2 * m] = max(mx[2 * m], w[m] & 0x7FFFu);
            mx[2 * m + 1] = max(mx[2 * m + 1], (w[m] >> 16) & 0x7FFFu);
        }
    }
    // 8 x 8 transpose: o[j] holds channel h + j for tokens tb .. tb + 7
    uint32_t o[8][4];
#pragma unroll
    for (int n = 0; n < 4; ++n) {
        const uint32_t a[4] = {q[2 * n].x, q[2 * n].y, q[2 * n].z, q[2 * n].w};
        const uint32_t bb[4] = {q[2 * n + 1].x, q[2 * n + 1].y, q[2 * n + 1].z, q[2 * n + 1].w};
#pragma unroll
        for (int m = 0; m < 4; ++m) {
            o[2 * m][n] = __byte_perm(a[m], bb[m], 0x5410);      // low halves: channel 2m
            o[2 * m + 1][n] = __byte_perm(a[m], bb[m], 0x7632);  // high halves: channel 2m+1
        }
    }
    if (hok && tb < T) {
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            uint16_t* dst = Xt + (size_t)(h + j) * ldT + tb;
            if (tb + 8 <= T) {
                *reinterpret_cast<uint4*>(dst) = make_uint4(o[j][0], o[j][1], o[j][2], o[j][3]);
            } else {
#pragma unroll
                for (int i = 0; i < 8; ++i)
                    if (tb + i < T) dst[i] = (uint16_t)((i & 1) ? (o[j][i >> 1] >> 16) : (o[j][i >> 1] & 0xFFFFu));
            }
        }
    }
    // channel maxima: the two token halves of a lane pair, then the 8 warps
#pragma unroll
    for (int c = 0; c < 8; ++c) mx[c] = max(mx[c], __shfl_xor_sync(0xffffffffu, mx[c], 16));
    if (half == 0) {
#pragma unroll
        for (int c = 0; c < 8; ++c) red[warp][8 * g + c] = mx[c];
    }
    __syncthreads();
    if (tid < 128) {
        uint32_t m = 0;
#pragma unroll
        for (int w = 0; w < kXtThreads / 32; ++w) m = max(m, red[w][tid]);
        const int hh = blockIdx.x * 128 + tid;
        if (s32 && hh < H && m > 0) atomicMax(s32 + hh, m);
    }
}

}  // namespace

cudaError_t launch_score(const uint16_t* X, int T, int H, uint32_t* s32, uint16_t* Xt, int ldT,
                         int num_sms, cudaStream_t stream) {
    // enough CTAs to keep ~16 per SM in flight; each takes one or more 64-token tiles
    const int strips = (H + kTileH - 1) / kTileH;
    const int tiles = (T + kTileT - 1) / kTileT;
    int ty = (16 * num_sms + strips - 1) / strips;
    if (ty > tiles) ty = tiles;
    if (ty > 65535) ty = 65535;
    if (ty < 1) ty = 1;
    dim3 grid(strips, ty);
    const bool vec = (H % 8 == 0) && ((reinterpret_cast<uintptr_t>(X) & 15) == 0);
    if (Xt && vec) {
        const int by = (T + kXtTokens - 1) / kXtTokens;
        if (by <= 65535)
            return launch_pdl(score_xt_kernel, dim3((H + 127) / 128, by), dim3(kXtThreads), 0, stream, X, T, H, s32,
                              Xt, ldT);
    }
    auto kern = Xt ? (vec ? score_kernel<true, true> : score_kernel<true, false>)
                   : (vec ? score_kernel<false, true> : score_kernel<false, false>);
    return launch_pdl(kern, grid, dim3(kThreads), 0, stream, X, T, H, s32, Xt, ldT);
}

}  // namespace rmm
