// rmm_layer.cu -- the elementwise and layout glue of one decoder layer around
// the reduced products: residual add + RMSNorm, SwiGLU, the q/k/v split into
// attention heads with the KV-cache append, and the attention output back to
// token-major rows.
//
// The layer anatomy (RMSNorm in place of LayerNorm, a residual stream through
// every block, a gated SwiGLU MLP) follows the 'Numerical Linear Algebra for
// LLMs' paper digest (ai-feeds.com), section 'Method: key modules'.  Every
// intermediate is bf16 between ops; arithmetic inside an op is fp32.  All of
// it is memory bound and moves each byte once, with 16-byte accesses.
#include "rmm_common.cuh"
#include "rmm_internal.h"

namespace rmm {

namespace {

__device__ __forceinline__ void unpack8f(const uint4& w, float (&f)[8]) {
    f[0] = __uint_as_float(w.x << 16);
    f[1] = __uint_as_float(w.x & 0xFFFF0000u);
    f[2] = __uint_as_float(w.y << 16);
    f[3] = __uint_as_float(w.y & 0xFFFF0000u);
    f[4] = __uint_as_float(w.z << 16);
    f[5] = __uint_as_float(w.z & 0xFFFF0000u);
    f[6] = __uint_as_float(w.w << 16);
    f[7] = __uint_as_float(w.w & 0xFFFF0000u);
}

__device__ __forceinline__ uint4 pack8f(const float (&f)[8]) {
    return make_uint4(pack_bf16x2(f[0], f[1]), pack_bf16x2(f[2], f[3]), pack_bf16x2(f[4], f[5]),
                      pack_bf16x2(f[6], f[7]));
}

constexpr int kNormThreads = 256;
constexpr int kNormMaxVec = 8;  // 16-byte pieces per thread held in registers (H <= 16384)

// One CTA per row: h = bf16(x + r) (r optional), written to Hsum when asked;
// y = bf16(h * rsqrt(mean(h^2) + eps) * w) (w optional, else 1), written to Y
// when asked.  The row stays in registers between the two passes.
__global__ void __launch_bounds__(kNormThreads)
    add_rmsnorm_kernel(const uint16_t* __restrict__ X, const uint16_t* __restrict__ R, int H, float eps,
                       const uint16_t* __restrict__ Wn, uint16_t* __restrict__ Hsum, uint16_t* __restrict__ Y) {
    pdl_wait();
    pdl_launch_dependents();
    __shared__ float red[kNormThreads / 32];
    const size_t row = blockIdx.x;
    const int nvec = H / 8;
    float v[kNormMaxVec][8];
    float ss = 0.f;
#pragma unroll
    for (int i = 0; i < kNormMaxVec; ++i) {
        const int c = threadIdx.x + i * kNormThreads;
        if (c < nvec) {
            unpack8f(ld_nc_v4(X + row * H + c * 8), v[i]);
            if (R) {
                float r[8];
                unpack8f(ld_nc_v4(R + row * H + c * 8), r);
#pragma unroll
                for (int e = 0; e < 8; ++e) v[i][e] += r[e];
            }
            const uint4 hb = pack8f(v[i]);  // the residual stream is bf16
            if (Hsum) *reinterpret_cast<uint4*>(Hsum + row * H + c * 8) = hb;
            unpack8f(hb, v[i]);
#pragma unroll
            for (int e = 0; e < 8; ++e) ss += v[i][e] * v[i][e];
        }
    }
    if (!Y) return;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = ss;
    __syncthreads();
    float tot = 0.f;
#pragma unroll
    for (int w = 0; w < kNormThreads / 32; ++w) tot += red[w];
    const float inv = rsqrtf(tot / (float)H + eps);
#pragma unroll
    for (int i = 0; i < kNormMaxVec; ++i) {
        const int c = threadIdx.x + i * kNormThreads;
        if (c < nvec) {
            float y[8], w[8];
            if (Wn) unpack8f(ld_nc_v4(Wn + c * 8), w);
#pragma unroll
            for (int e = 0; e < 8; ++e) y[e] = v[i][e] * inv * (Wn ? w[e] : 1.0f);
            *reinterpret_cast<uint4*>(Y + row * H + c * 8) = pack8f(y);
        }
    }
}

// out = bf16(silu(g) * u), silu(z) = z / (1 + e^-z); 8 elements per thread
__global__ void __launch_bounds__(256)
    swiglu_kernel(const uint16_t* __restrict__ G, const uint16_t* __restrict__ U, size_t n8,
                  uint16_t* __restrict__ Out) {
    pdl_wait();
    pdl_launch_dependents();
    for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n8; i += (size_t)gridDim.x * blockDim.x) {
        float g[8], u[8], o[8];
        unpack8f(ld_nc_v4(G + i * 8), g);
        unpack8f(ld_nc_v4(U + i * 8), u);
#pragma unroll
        for (int e = 0; e < 8; ++e) o[e] = g[e] / (1.0f + expf(-g[e])) * u[e];
        *reinterpret_cast<uint4*>(Out + i * 8) = pack8f(o);
    }
}

constexpr int kTokTile = 64;  // tokens per CTA in the head relayouts

// Token-major projections -> attention layouts, for one head per blockIdx.y
// (query heads first, then KV heads) and 64 tokens per blockIdx.x:
//   Q[h, t, :]          = Yq[t, h*d : h*d+d]
//   Kt[g, j, L0 + t]    = Yk[t, g*d + j]      (d-major key cache: transposed)
//   V[g, L0 + t, :]     = Yv[t, g*d : g*d+d]
__global__ void __launch_bounds__(256)
    qkv_heads_kernel(const uint16_t* __restrict__ Yq, const uint16_t* __restrict__ Yk,
                     const uint16_t* __restrict__ Yv, int T, int Hq, int Hkv, uint16_t* __restrict__ Q,
                     uint16_t* __restrict__ Kt, uint16_t* __restrict__ V, int ldL, int L0) {
    pdl_wait();
    pdl_launch_dependents();
    constexpr int d = 128;
    __shared__ uint16_t tile[kTokTile][d + 8];
    const int t0 = blockIdx.x * kTokTile;
    const int hh = blockIdx.y;
    const int tid = threadIdx.x;
    if (hh < Hq) {  // Q: straight 256-byte row copies
        for (int e = tid; e < kTokTile * (d / 8); e += blockDim.x) {
            const int t = t0 + e / (d / 8), c = e % (d / 8);
            if (t < T)
                *reinterpret_cast<uint4*>(Q + ((size_t)hh * T + t) * d + c * 8) =
                    ld_nc_v4(Yq + (size_t)t * Hq * d + hh * d + c * 8);
        }
        return;
    }
    const int g = hh - Hq;
    for (int e = tid; e < kTokTile * (d / 8); e += blockDim.x) {
        const int tl = e / (d / 8), c = e % (d / 8), t = t0 + tl;
        if (t < T) {
            *reinterpret_cast<uint4*>(V + ((size_t)g * ldL + L0 + t) * d + c * 8) =
                ld_nc_v4(Yv + (size_t)t * Hkv * d + g * d + c * 8);
            const uint4 k = ld_nc_v4(Yk + (size_t)t * Hkv * d + g * d + c * 8);
            uint32_t* dst = reinterpret_cast<uint32_t*>(&tile[tl][c * 8]);
            dst[0] = k.x;
            dst[1] = k.y;
            dst[2] = k.z;
            dst[3] = k.w;
        }
    }
    __syncthreads();
    // transposed write: one key dim j per row of Kt, 64 consecutive positions
    for (int e = tid; e < d * kTokTile; e += blockDim.x) {
        const int j = e / kTokTile, tl = e % kTokTile, t = t0 + tl;
        if (t < T) Kt[((size_t)g * d + j) * ldL + L0 + t] = tile[tl][j];
    }
}

// O[h, t, :] (attention heads) -> A[t, h*d : h*d+d] (token-major rows)
__global__ void __launch_bounds__(256)
    heads_to_tokens_kernel(const uint16_t* __restrict__ O, int Hq, int T, uint16_t* __restrict__ A) {
    pdl_wait();
    pdl_launch_dependents();
    constexpr int d = 128;
    const size_t n = (size_t)Hq * T * (d / 8);
    for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x) {
        const int c = (int)(i % (d / 8));
        const size_t ht = i / (d / 8);
        const int t = (int)(ht % T), h = (int)(ht / T);
        *reinterpret_cast<uint4*>(A + ((size_t)t * Hq + h) * d + c * 8) = ld_nc_v4(O + ht * d + c * 8);
    }
}

int grid_for(size_t items, int threads, int num_sms) {
    size_t g = (items + threads - 1) / threads;
    const size_t cap = (size_t)num_sms * 8;
    if (g > cap) g = cap;
    return g < 1 ? 1 : (int)g;
}

}  // namespace

cudaError_t launch_add_rmsnorm(const uint16_t* X, const uint16_t* R, int T, int H, float eps, const uint16_t* Wn,
                               uint16_t* Hsum, uint16_t* Y, cudaStream_t stream) {
    if (T < 1 || H < 8 || H % 8 != 0 || H / 8 > kNormMaxVec * kNormThreads) return cudaErrorInvalidValue;
    return launch_pdl(add_rmsnorm_kernel, dim3(T), dim3(kNormThreads), 0, stream, X, R, H, eps, Wn, Hsum, Y);
}

cudaError_t launch_swiglu(const uint16_t* G, const uint16_t* U, size_t n, uint16_t* Out, int num_sms,
                          cudaStream_t stream) {
    if (n == 0 || n % 8 != 0) return cudaErrorInvalidValue;
    return launch_pdl(swiglu_kernel, dim3(grid_for(n / 8, 256, num_sms)), dim3(256), 0, stream, G, U, n / 8, Out);
}

cudaError_t launch_qkv_heads(const uint16_t* Yq, const uint16_t* Yk, const uint16_t* Yv, int T, int Hq, int Hkv,
                             uint16_t* Q, uint16_t* Kt, uint16_t* V, int ldL, int L0, cudaStream_t stream) {
    if (T < 1 || Hq < 1 || Hkv < 1 || L0 < 0 || L0 + T > ldL) return cudaErrorInvalidValue;
    return launch_pdl(qkv_heads_kernel, dim3((T + kTokTile - 1) / kTokTile, Hq + Hkv), dim3(256), 0, stream, Yq, Yk,
                      Yv, T, Hq, Hkv, Q, Kt, V, ldL, L0);
}

cudaError_t launch_heads_to_tokens(const uint16_t* O, int Hq, int T, uint16_t* A, int num_sms, cudaStream_t stream) {
    if (T < 1 || Hq < 1) return cudaErrorInvalidValue;
    return launch_pdl(heads_to_tokens_kernel, dim3(grid_for((size_t)Hq * T * 16, 256, num_sms)), dim3(256), 0,
                      stream, O, Hq, T, A);
}

}  // namespace rmm
