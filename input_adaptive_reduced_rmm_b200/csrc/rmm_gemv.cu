// rmm_gemv.cu -- step 3 for decode-sized T (T <= 16): the reduced product as a
// split-K GEMV that streams only the kept rows of W^T.
//
// Y[t,n] = sum_{j<k} X[t, idx_j] * Wt[idx_j, n]
//
// At decode a step emits one token, so the product is GEMV-like and bound by
// memory traffic (GEMM primer, tangquanwei.github.io 'GEMM', section 7); the
// reduction cuts that traffic to the k kept weight rows (k*N*2 bytes).  Each
// kept slice h is one contiguous row of W^T (N*2 bytes).
//
// Grid: (column blocks of 256/512 outputs) x (splits of the kept list).  A CTA
// stages its split's indices and the matching X values in shared memory,
// then each thread streams 16-byte pieces of kept rows (8 outputs) with
// non-allocating loads, accumulating T x 8 fp32 sums.  Row groups inside the
// CTA are folded through shared memory; splits are folded deterministically
// (fixed order 0..S-1) by the last CTA of each column block to finish, found
// with a counter that it resets to zero afterwards.
#include "rmm_common.cuh"
#include "rmm_internal.h"

namespace rmm {

namespace {

constexpr int kThreads = 256;

__device__ __forceinline__ void unpack8(const uint4& w, float (&f)[8]) {
    f[0] = __uint_as_float(w.x << 16);
    f[1] = __uint_as_float(w.x & 0xFFFF0000u);
    f[2] = __uint_as_float(w.y << 16);
    f[3] = __uint_as_float(w.y & 0xFFFF0000u);
    f[4] = __uint_as_float(w.z << 16);
    f[5] = __uint_as_float(w.z & 0xFFFF0000u);
    f[6] = __uint_as_float(w.w << 16);
    f[7] = __uint_as_float(w.w & 0xFFFF0000u);
}

template <int TT, int TPR>
__global__ void __launch_bounds__(kThreads)
    gemv_kernel(const uint16_t* __restrict__ X, int T, int H, const uint16_t* __restrict__ Wt,
                int N, const int32_t* __restrict__ idx, int k, uint16_t* __restrict__ Y,
                float* __restrict__ partials, unsigned* __restrict__ counters,
                int rows_per_split) {
    constexpr int RG = kThreads / TPR;  // row groups
    constexpr int COLS = TPR * 8;       // outputs per CTA
    constexpr int U = (TT >= 8) ? 4 : 8;  // kept rows in flight per thread

    extern __shared__ float smem[];
    float* xs = smem;                                        // [rows][TT]
    int* sidx = reinterpret_cast<int*>(xs + rows_per_split * TT);  // [rows]
    float* red = reinterpret_cast<float*>(sidx + rows_per_split);  // [TT][COLS]
    __shared__ int is_last;

    pdl_wait();
    pdl_launch_dependents();
    const int tid = threadIdx.x;
    const int rg = tid / TPR, ct = tid % TPR;
    const int split = blockIdx.y;
    const int j0 = split * rows_per_split;
    const int nr = max(0, min(k, j0 + rows_per_split) - j0);
    const int n = blockIdx.x * COLS + ct * 8;

    for (int i = tid; i < nr; i += kThreads) sidx[i] = idx[j0 + i];
    __syncthreads();
    for (int e = tid; e < nr * TT; e += kThreads) {
        const int i = e / TT, t = e - (e / TT) * TT;
        xs[e] = (t < T) ? bf16_bits_to_float(X[(size_t)t * H + sidx[i]]) : 0.0f;
    }
    __syncthreads();

    float acc[TT][8];
#pragma unroll
    for (int t = 0; t < TT; ++t)
#pragma unroll
        for (int c = 0; c < 8; ++c) acc[t][c] = 0.0f;

    if (n < N) {
        const uint16_t* wcol = Wt + n;
        int i = rg;
        for (; i + (U - 1) * RG < nr; i += U * RG) {
            uint4 w[U];
#pragma unroll
            for (int u = 0; u < U; ++u) w[u] = ld_nc_v4(wcol + (size_t)sidx[i + u * RG] * N);
#pragma unroll
            for (int u = 0; u < U; ++u) {
                float wf[8];
                unpack8(w[u], wf);
                const float* xr = xs + (i + u * RG) * TT;
#pragma unroll
                for (int t = 0; t < TT; ++t) {
                    const float xv = xr[t];
#pragma unroll
                    for (int c = 0; c < 8; ++c) acc[t][c] = fmaf(xv, wf[c], acc[t][c]);
                }
            }
        }
        for (; i < nr; i += RG) {
            uint4 w = ld_nc_v4(wcol + (size_t)sidx[i] * N);
            float wf[8];
            unpack8(w, wf);
            const float* xr = xs + i * TT;
#pragma unroll
            for (int t = 0; t < TT; ++t) {
                const float xv = xr[t];
#pragma unroll
                for (int c = 0; c < 8; ++c) acc[t][c] = fmaf(xv, wf[c], acc[t][c]);
            }
        }
    }

    // fold the row groups into row group 0 (fixed order: deterministic)
    for (int r = 1; r < RG; ++r) {
        if (rg == r) {
#pragma unroll
            for (int t = 0; t < TT; ++t)
#pragma unroll
                for (int c = 0; c < 8; ++c) red[t * COLS + ct * 8 + c] = acc[t][c];
        }
        __syncthreads();
        if (rg == 0) {
#pragma unroll
            for (int t = 0; t < TT; ++t)
#pragma unroll
                for (int c = 0; c < 8; ++c) acc[t][c] += red[t * COLS + ct * 8 + c];
        }
        __syncthreads();
    }

    if (gridDim.y == 1) {
        if (rg == 0 && n < N) {
#pragma unroll
            for (int t = 0; t < TT; ++t) {
                if (t < T) {
                    uint4 o;
                    o.x = pack_bf16x2(acc[t][0], acc[t][1]);
                    o.y = pack_bf16x2(acc[t][2], acc[t][3]);
                    o.z = pack_bf16x2(acc[t][4], acc[t][5]);
                    o.w = pack_bf16x2(acc[t][6], acc[t][7]);
                    *reinterpret_cast<uint4*>(Y + (size_t)t * N + n) = o;
                }
            }
        }
        return;
    }

    if (rg == 0 && n < N) {
#pragma unroll
        for (int t = 0; t < TT; ++t) {
            if (t < T) {
                float4* dst = reinterpret_cast<float4*>(partials + ((size_t)split * T + t) * N + n);
                dst[0] = make_float4(acc[t][0], acc[t][1], acc[t][2], acc[t][3]);
                dst[1] = make_float4(acc[t][4], acc[t][5], acc[t][6], acc[t][7]);
            }
        }
    }
    __threadfence();
    __syncthreads();
    if (tid == 0) {
        const unsigned prev = atomicAdd(&counters[blockIdx.x], 1u);
        is_last = (prev == gridDim.y - 1);
    }
    __syncthreads();
    if (!is_last) return;
    __threadfence();
    const int S = gridDim.y;
    constexpr int Q4 = COLS / 4;
    for (int e = tid; e < T * Q4; e += kThreads) {
        const int t = e / Q4, c4 = e - (e / Q4) * Q4;
        const int nn = blockIdx.x * COLS + c4 * 4;
        if (nn >= N) continue;
        float4 s = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int sp = 0; sp < S; ++sp) {
            const float4 v =
                __ldcg(reinterpret_cast<const float4*>(partials + ((size_t)sp * T + t) * N + nn));
            s.x += v.x;
            s.y += v.y;
            s.z += v.z;
            s.w += v.w;
        }
        uint2 o;
        o.x = pack_bf16x2(s.x, s.y);
        o.y = pack_bf16x2(s.z, s.w);
        *reinterpret_cast<uint2*>(Y + (size_t)t * N + nn) = o;
    }
    if (tid == 0) counters[blockIdx.x] = 0;  // leave the counter ready for the next call
}

template <int TT, int TPR>
cudaError_t launch_t(const uint16_t* X, int T, int H, const uint16_t* Wt, int N,
                     const int32_t* idx, int k, uint16_t* Y, float* partials, unsigned* counters,
                     const GemvPlan& p, cudaStream_t stream) {
    const size_t smem = (size_t)p.rows_per_split * TT * sizeof(float) +
                        (size_t)p.rows_per_split * sizeof(int) + (size_t)TT * TPR * 8 * sizeof(float);
    auto kern = gemv_kernel<TT, TPR>;
    if (smem > 48 * 1024) {
        cudaError_t e =
            cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
    }
    dim3 grid(p.col_blocks, p.splits);
    return launch_pdl(kern, grid, dim3(kThreads), smem, stream, X, T, H, Wt, N, idx, k, Y, partials,
                      counters, p.rows_per_split);
}

template <int TT>
cudaError_t launch_tt(const uint16_t* X, int T, int H, const uint16_t* Wt, int N,
                      const int32_t* idx, int k, uint16_t* Y, float* partials, unsigned* counters,
                      const GemvPlan& p, cudaStream_t stream) {
    if (p.cols_per_cta == 512)
        return launch_t<TT, 64>(X, T, H, Wt, N, idx, k, Y, partials, counters, p, stream);
    return launch_t<TT, 32>(X, T, H, Wt, N, idx, k, Y, partials, counters, p, stream);
}

}  // namespace

GemvPlan gemv_plan(int T, int N, int k, int num_sms, int forced_splits) {
    GemvPlan p;
    p.cols_per_cta = (N >= 8192) ? 512 : 256;
    p.col_blocks = (N + p.cols_per_cta - 1) / p.cols_per_cta;
    const int target = num_sms * (T <= 4 ? 4 : 2);
    int splits = forced_splits > 0 ? forced_splits : (target + p.col_blocks - 1) / p.col_blocks;
    const int max_splits = forced_splits > 0 ? k : (k / 32 > 1 ? k / 32 : 1);
    if (splits > max_splits) splits = max_splits;
    if (splits > 1024) splits = 1024;
    if (splits < 1) splits = 1;
    p.rows_per_split = (k + splits - 1) / splits;
    p.splits = (k + p.rows_per_split - 1) / p.rows_per_split;
    return p;
}

size_t gemv_smem_bytes(const GemvPlan& p, int T) {
    const int TT = T <= 1 ? 1 : T <= 2 ? 2 : T <= 4 ? 4 : T <= 8 ? 8 : 16;
    return (size_t)p.rows_per_split * TT * sizeof(float) + (size_t)p.rows_per_split * sizeof(int) +
           (size_t)TT * p.cols_per_cta * sizeof(float);
}

size_t gemv_partials_bytes(const GemvPlan& p, int T, int N) {
    return p.splits > 1 ? (size_t)p.splits * T * N * sizeof(float) : 0;
}

cudaError_t launch_gemv(const uint16_t* X, int T, int H, const uint16_t* Wt, int N,
                        const int32_t* idx, int k, uint16_t* Y, float* partials,
                        unsigned* counters, const GemvPlan& p, int* /*status*/,
                        cudaStream_t stream) {
    if (T <= 1) return launch_tt<1>(X, T, H, Wt, N, idx, k, Y, partials, counters, p, stream);
    if (T <= 2) return launch_tt<2>(X, T, H, Wt, N, idx, k, Y, partials, counters, p, stream);
    if (T <= 4) return launch_tt<4>(X, T, H, Wt, N, idx, k, Y, partials, counters, p, stream);
    if (T <= 8) return launch_tt<8>(X, T, H, Wt, N, idx, k, Y, partials, counters, p, stream);
    return launch_tt<16>(X, T, H, Wt, N, idx, k, Y, partials, counters, p, stream);
}

}  // namespace rmm
