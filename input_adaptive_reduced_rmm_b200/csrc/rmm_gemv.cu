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
// Work: for the members p of a group of products sharing X (e.g. q, k, v) the
// kept list is cut into S splits of at most 512 rows and each member's outputs
// into column blocks of COLS (256 for T <= 4, narrower for wider T).  One CTA =
// (member, column block) along x, split along y; x varies fastest, so the CTAs
// running at the same moment read neighbouring 512-byte pieces of the same
// kept rows.  S gives a grid of ~6 CTAs per SM (~12 above 100 MB of kept
// weights) in several waves: measured on B200, such grids sustain 5.4-5.8
// TB/s on scattered kept rows, while fewer, longer-running CTAs lose to
// ramp-up and ramp-down and shorter ones to their set-up.
//
// A CTA stages its split's kept indices in shared memory, issues its first
// batch of weight loads and only then gathers the X values beside them, so
// both latencies overlap; it streams 16-byte pieces of the kept rows with
// non-allocating loads (16, 8 or 4 rows in flight per thread, packed fp32x2 FMAs),
// folds its row groups (shuffles, then the warps in a fixed order) and writes
// its fp32 partial sums -- or, with one split, Y itself.  A second launch,
// chained by programmatic dependent launch, adds the S partials of every
// output in split order and writes Y: no fences, counters or atomics on the
// streaming CTAs, a deterministic result, and the fold's launch latency hidden
// behind the product.
#include "rmm_common.cuh"
#include "rmm_internal.h"

namespace rmm {

namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kMaxRowsPerItem = 512;
constexpr int kFoldCols = 256;  // outputs of one fold CTA (32 threads x 8 columns)
constexpr int kFoldGroups = kThreads / (kFoldCols / 8);

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

// (d0, d1) = (a * b0 + d0, a * b1 + d1), one packed fp32x2 FMA, round to nearest
__device__ __forceinline__ void fma2(float& d0, float& d1, float a, float b0, float b1) {
    asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
        "mov.b64 ra, {%2, %2};\n\t"
        "mov.b64 rb, {%3, %4};\n\t"
        "mov.b64 rd, {%0, %1};\n\t"
        "fma.rn.f32x2 rd, ra, rb, rd;\n\t"
        "mov.b64 {%0, %1}, rd;\n\t}"
        : "+f"(d0), "+f"(d1)
        : "f"(a), "f"(b0), "f"(b1));
}

template <int TT>
__device__ __forceinline__ void fma_row(float (&acc)[TT][8], const uint4& w, const float* xr) {
    float wf[8];
    unpack8(w, wf);
#pragma unroll
    for (int t = 0; t < TT; ++t) {
        const float xv = xr[t];
#pragma unroll
        for (int c = 0; c < 8; c += 2) fma2(acc[t][c], acc[t][c + 1], xv, wf[c], wf[c + 1]);
    }
}

__device__ __forceinline__ void store_bf16x8(uint16_t* dst, const float* s) {
    uint4 o;
    o.x = pack_bf16x2(s[0], s[1]);
    o.y = pack_bf16x2(s[2], s[3]);
    o.z = pack_bf16x2(s[4], s[5]);
    o.w = pack_bf16x2(s[6], s[7]);
    *reinterpret_cast<uint4*>(dst) = o;
}

// member of a group whose prefix range holds x
__device__ __forceinline__ int member_of(const int* start, int count, int x) {
    int p = 0;
#pragma unroll
    for (int i = 1; i < kMaxGroupGemv; ++i)
        if (i < count && x >= start[i]) p = i;
    return p;
}

template <int TT, int COLS, int U>
__global__ void __launch_bounds__(kThreads, (TT <= 4) ? 3 : 1)
    gemv_kernel(const uint16_t* __restrict__ X, int T, int H, const int32_t* __restrict__ idx, int k,
                const __grid_constant__ GemvGroup g, float* __restrict__ partials) {
    constexpr int TPR = COLS / 8;         // threads per kept-row piece
    constexpr int RG = kThreads / TPR;    // row groups
    constexpr int WCOLS = (COLS < 256) ? COLS : 256;  // columns held by one warp after its shuffle fold
    constexpr int P8 = COLS / 8;

    extern __shared__ float smem[];
    float* xs = smem;                                               // [kMaxRowsPerItem][TT]
    int* sidx = reinterpret_cast<int*>(xs + kMaxRowsPerItem * TT);  // [kMaxRowsPerItem]
    float* fold = reinterpret_cast<float*>(sidx + kMaxRowsPerItem); // [kWarps][TT][WCOLS]
    float* part = fold + kWarps * TT * WCOLS;                       // [TT][COLS]

    pdl_wait();
    pdl_launch_dependents();
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int rg = tid / TPR, ct = tid % TPR;
    const int p = member_of(g.item_start, g.count, blockIdx.x);
    const int cb = blockIdx.x - g.item_start[p];
    const int sp = blockIdx.y;
    const int N = g.N[p];
    const int ld = g.ld[p];
    const int rows = g.rows_per_split[p];
    const int j0 = sp * rows;
    const int nr = max(0, min(k, j0 + rows) - j0);
    const int n0 = cb * COLS;

    // 1. the split's kept indices (idx null: every slice kept, the identity list)
    for (int i = tid; i < nr; i += kThreads) sidx[i] = idx ? __ldg(idx + j0 + i) : j0 + i;
    __syncthreads();

    // 2. the first batch of weight pieces in flight, then the X values beside them
    const int n = n0 + ct * 8;
    const bool col_ok = n < N;  // N % 8 == 0: the whole 16-byte piece is in range
    const uint16_t* wcol = g.Wt[p] + (col_ok ? n : 0);
    uint4 w[U];
    int i = rg;
#pragma unroll
    for (int u = 0; u < U; ++u)
        w[u] = (col_ok && i + u * RG < nr) ? ld_nc_v4(wcol + (size_t)sidx[i + u * RG] * ld)
                                           : make_uint4(0u, 0u, 0u, 0u);
    for (int e0 = tid; e0 < nr * TT; e0 += 4 * kThreads) {
        uint16_t v[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const int e = e0 + q * kThreads;
            const int r = e / TT, t = e - (e / TT) * TT;
            v[q] = (e < nr * TT && t < T) ? X[(size_t)t * H + sidx[r]] : (uint16_t)0;
        }
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const int e = e0 + q * kThreads;
            if (e < nr * TT) xs[e] = bf16_bits_to_float(v[q]);
        }
    }
    __syncthreads();

    // 3. stream the kept rows
    float acc[TT][8];
#pragma unroll
    for (int t = 0; t < TT; ++t)
#pragma unroll
        for (int c = 0; c < 8; ++c) acc[t][c] = 0.0f;
    for (;;) {
#pragma unroll
        for (int u = 0; u < U; ++u)
            if (i + u * RG < nr) fma_row<TT>(acc, w[u], xs + (i + u * RG) * TT);
        i += U * RG;
        if (i >= nr) break;
#pragma unroll
        for (int u = 0; u < U; ++u)
            w[u] = (col_ok && i + u * RG < nr) ? ld_nc_v4(wcol + (size_t)sidx[i + u * RG] * ld)
                                               : make_uint4(0u, 0u, 0u, 0u);
    }

    // 4. fold the row groups: shuffles inside a warp, then the warps in order
#pragma unroll
    for (int off = TPR; off < 32; off <<= 1)
#pragma unroll
        for (int t = 0; t < TT; ++t)
#pragma unroll
            for (int c = 0; c < 8; ++c) acc[t][c] += __shfl_xor_sync(0xffffffffu, acc[t][c], off);
    if (lane * 8 < WCOLS) {
#pragma unroll
        for (int t = 0; t < TT; ++t)
#pragma unroll
            for (int c = 0; c < 8; ++c) fold[(warp * TT + t) * WCOLS + lane * 8 + c] = acc[t][c];
    }
    __syncthreads();
    constexpr int WPR = (TPR > 32) ? TPR / 32 : 1;  // warps per row group
    for (int o = tid; o < TT * COLS; o += kThreads) {
        const int t = o / COLS, col = o - (o / COLS) * COLS;
        const int wsel = col / WCOLS;
        float s = 0.0f;
#pragma unroll
        for (int w2 = 0; w2 < kWarps; ++w2)
            if (w2 % WPR == wsel) s += fold[(w2 * TT + t) * WCOLS + (col - wsel * WCOLS)];
        part[o] = s;
    }
    __syncthreads();

    // 5. Y itself with one split, else this split's partial sums
    if (g.splits[p] == 1) {
        uint16_t* Y = g.Y[p];
        for (int o8 = tid; o8 < TT * P8; o8 += kThreads) {
            const int t = o8 / P8, c8 = o8 - (o8 / P8) * P8;
            const int nn = n0 + c8 * 8;
            if (t < T && nn < N) store_bf16x8(Y + (size_t)t * ld + nn, part + t * COLS + c8 * 8);
        }
        return;
    }
    float* pbase = partials + g.partial_off[p];
    for (int o8 = tid; o8 < TT * P8; o8 += kThreads) {
        const int t = o8 / P8, c8 = o8 - (o8 / P8) * P8;
        const int nn = n0 + c8 * 8;
        if (t < T && nn < N) {
            float4* dst = reinterpret_cast<float4*>(pbase + ((size_t)sp * T + t) * N + nn);
            const float* s = part + t * COLS + c8 * 8;
            __stcg(dst, make_float4(s[0], s[1], s[2], s[3]));
            __stcg(dst + 1, make_float4(s[4], s[5], s[6], s[7]));
        }
    }
}

// Y[t, n..n+8) = sum over splits s (in order) of the partials.  One CTA = 256
// columns of one member and one token; its 8 thread groups take consecutive
// ranges of the splits (four splits' loads in flight at a time) and the range
// sums are added in range order.
// With g.swiglu the grid covers member 0's column blocks and each CTA folds
// both members at the same columns, then writes Y[0] = bf16(silu(g) * u) from
// the bf16-rounded gate and up values (the arithmetic of swiglu_kernel).
__device__ __forceinline__ void fold_member(const GemvGroup& g, int p, int t, int n, int c, int grp, int T,
                                            const float* __restrict__ partials, float4 (*gs)[kFoldCols / 8][2],
                                            float (&tot)[8]) {
    const int N = g.N[p], S = g.splits[p];
    const bool live = n < N;
    float s[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    if (live) {
        const float* b = partials + g.partial_off[p] + (size_t)t * N + n;
        const size_t stride = (size_t)T * N;
        const int s_hi = (grp + 1) * S / kFoldGroups;
        for (int s0 = grp * S / kFoldGroups; s0 < s_hi; s0 += 4) {
            float4 v[4][2];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                if (s0 + u < s_hi) {
                    v[u][0] = __ldcg(reinterpret_cast<const float4*>(b + (s0 + u) * stride));
                    v[u][1] = __ldcg(reinterpret_cast<const float4*>(b + (s0 + u) * stride + 4));
                }
            }
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                if (s0 + u < s_hi) {
                    s[0] += v[u][0].x; s[1] += v[u][0].y; s[2] += v[u][0].z; s[3] += v[u][0].w;
                    s[4] += v[u][1].x; s[5] += v[u][1].y; s[6] += v[u][1].z; s[7] += v[u][1].w;
                }
            }
        }
    }
    gs[grp][c][0] = make_float4(s[0], s[1], s[2], s[3]);
    gs[grp][c][1] = make_float4(s[4], s[5], s[6], s[7]);
    __syncthreads();
#pragma unroll
    for (int e = 0; e < 8; ++e) tot[e] = 0.f;
    if (grp == 0 && live) {
#pragma unroll
        for (int q = 0; q < kFoldGroups; ++q) {
            const float4 a = gs[q][c][0], d = gs[q][c][1];
            tot[0] += a.x; tot[1] += a.y; tot[2] += a.z; tot[3] += a.w;
            tot[4] += d.x; tot[5] += d.y; tot[6] += d.z; tot[7] += d.w;
        }
    }
    __syncthreads();  // gs may be reused by the next member
}

__global__ void __launch_bounds__(kThreads)
    gemv_fold_kernel(const __grid_constant__ GemvGroup g, int T, const float* __restrict__ partials) {
    __shared__ float4 gs[kFoldGroups][kFoldCols / 8][2];
    pdl_wait();
    pdl_launch_dependents();
    const int tid = threadIdx.x;
    const int p = member_of(g.fold_start, g.count, blockIdx.x);
    const int c = tid % (kFoldCols / 8);
    const int n = (blockIdx.x - g.fold_start[p]) * kFoldCols + c * 8;
    const int grp = tid / (kFoldCols / 8);
    const int t = blockIdx.y;
    const bool live = n < g.N[p];
    float tot[8];
    fold_member(g, p, t, n, c, grp, T, partials, gs, tot);
    if (g.swiglu) {
        float up[8];
        fold_member(g, 1, t, n, c, grp, T, partials, gs, up);
        if (grp == 0 && live) {
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const float gv = bf16_bits_to_float(float_to_bf16_bits(tot[e]));
                const float uv = bf16_bits_to_float(float_to_bf16_bits(up[e]));
                tot[e] = gv / (1.0f + expf(-gv)) * uv;
            }
        }
    }
    if (grp == 0 && live) store_bf16x8(g.Y[p] + (size_t)t * g.ld[p] + n, tot);
}

template <int TT>
cudaError_t launch_tt(const uint16_t* X, int T, int H, const int32_t* idx, int k, const GemvGroup& g,
                      float* partials, cudaStream_t stream) {
    constexpr int COLS = TT <= 4 ? 256 : TT <= 8 ? 128 : 64;  // gemv_cols_for
    if (g.cols != COLS) return cudaErrorInvalidValue;
    const size_t smem = gemv_smem_bytes(COLS, T);
    // kept rows in flight per thread: 16 for long splits of one or two tokens
    constexpr int U_SHORT = TT >= 8 ? 4 : 8;
    constexpr int U_LONG = TT <= 2 ? 16 : U_SHORT;
    auto kern = g.rows_per_split[0] >= 192 ? gemv_kernel<TT, COLS, U_LONG> : gemv_kernel<TT, COLS, U_SHORT>;
    cudaError_t e = ensure_smem_limit(kern, smem);
    if (e != cudaSuccess) return e;
    e = launch_pdl(kern, dim3(g.item_start[g.count], g.splits[0]), dim3(kThreads), smem, stream, X, T, H, idx, k, g,
                   partials);
    if (e != cudaSuccess || g.splits[0] == 1) return e;
    // with the SwiGLU epilogue only member 0's column blocks (each folds both members)
    return launch_pdl(gemv_fold_kernel, dim3(g.fold_start[g.swiglu ? 1 : g.count], T), dim3(kThreads), 0, stream, g,
                      T, static_cast<const float*>(partials));
}

// Splits before rounding to whole rows; never decreases as k grows.  Measured
// on B200 (one token, graph replays, kept rows scattered): a grid of ~6 CTAs
// per SM streams best up to ~100 MB of kept weights (4096 -> 14336 at r=0.5:
// 896 CTAs of 128 rows, 14.0 us) and ~12 per SM above (8192 -> 28672: 1792
// CTAs of 256 rows, 40.7 us, 5.8 TB/s); fewer, longer CTAs lose to ramp-up and
// ramp-down, more, shorter ones to their set-up.  At least 32 rows per split.
int initial_splits(const GemvGroup& g, int T, int k, int forced_splits, int num_sms) {
    const int cols = gemv_cols_for(T);
    int blocks = 0;
    size_t n_total = 0;
    for (int p = 0; p < g.count; ++p) {
        blocks += (g.N[p] + cols - 1) / cols;
        n_total += (size_t)g.N[p];
    }
    if (blocks < 1) blocks = 1;
    const size_t kept_bytes = (size_t)k * n_total * 2;
    const int per_sm = T <= 4 ? (kept_bytes > (size_t)100 << 20 ? 12 : 6) : 2;
    const int target = num_sms * per_sm;
    int S = forced_splits > 0 ? forced_splits : (target + blocks - 1) / blocks;
    const int max_by_rows = (k + 31) / 32;
    if (forced_splits <= 0 && S > max_by_rows) S = max_by_rows;
    const int min_splits = (k + kMaxRowsPerItem - 1) / kMaxRowsPerItem;
    if (S < min_splits) S = min_splits;
    if (S > k) S = k;
    if (S > 65535) S = 65535;
    if (S < 1) S = 1;
    return S;
}

}  // namespace

int gemv_cols_for(int T) { return T <= 4 ? 256 : T <= 8 ? 128 : 64; }

size_t gemv_smem_bytes(int cols, int T) {
    const int TT = T <= 1 ? 1 : T <= 2 ? 2 : T <= 4 ? 4 : T <= 8 ? 8 : 16;
    const int wcols = cols < 256 ? cols : 256;
    return (size_t)kMaxRowsPerItem * TT * sizeof(float) + (size_t)kMaxRowsPerItem * sizeof(int) +
           ((size_t)kWarps * TT * wcols + (size_t)TT * cols) * sizeof(float);
}

size_t gemv_partials_bound(const GemvGroup& g, int T, int H, int forced_splits, int num_sms) {
    const int S = initial_splits(g, T, H, forced_splits, num_sms);
    if (S <= 1) return 0;
    size_t n = 0;
    for (int p = 0; p < g.count; ++p) n += (size_t)g.N[p];
    return (size_t)S * T * n * sizeof(float);
}

size_t gemv_group_plan(GemvGroup& g, int T, int k, int forced_splits, int num_sms) {
    g.cols = gemv_cols_for(T);
    int S = initial_splits(g, T, k, forced_splits, num_sms);
    const int rows = (k + S - 1) / S;
    S = (k + rows - 1) / rows;
    size_t part = 0;
    g.item_start[0] = 0;
    g.fold_start[0] = 0;
    for (int p = 0; p < g.count; ++p) {
        if (g.ld[p] == 0) g.ld[p] = g.N[p];
        g.rows_per_split[p] = rows;
        g.splits[p] = S;
        g.col_blocks[p] = (g.N[p] + g.cols - 1) / g.cols;
        g.item_start[p + 1] = g.item_start[p] + g.col_blocks[p];
        g.fold_start[p + 1] = g.fold_start[p] + (g.N[p] + kFoldCols - 1) / kFoldCols;
        g.partial_off[p] = part;
        if (S > 1) part += (size_t)S * T * g.N[p];
    }
    for (int p = g.count + 1; p <= kMaxGroupGemv; ++p) {
        g.item_start[p] = g.item_start[g.count];
        g.fold_start[p] = g.fold_start[g.count];
    }
    return part * sizeof(float);
}

cudaError_t launch_gemv(const uint16_t* X, int T, int H, const int32_t* idx, int k, const GemvGroup& g,
                        float* partials, int num_sms, cudaStream_t stream) {
    (void)num_sms;
    if (g.count < 1 || g.count > kMaxGroupGemv) return cudaErrorInvalidValue;
    if (T <= 1) return launch_tt<1>(X, T, H, idx, k, g, partials, stream);
    if (T <= 2) return launch_tt<2>(X, T, H, idx, k, g, partials, stream);
    if (T <= 4) return launch_tt<4>(X, T, H, idx, k, g, partials, stream);
    if (T <= 8) return launch_tt<8>(X, T, H, idx, k, g, partials, stream);
    return launch_tt<16>(X, T, H, idx, k, g, partials, stream);
}

}  // namespace rmm
