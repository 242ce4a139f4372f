// rmm_glue.cu -- small helper kernels around the reduced product.
//
//   transpose_kernel  W [N, H] -> W^T [H, N], once per weight, so that a kept
//                     contraction slice h of the weight is one contiguous row
//                     (the product streams or gathers whole kept rows).
//   pad_idx_kernel    copies a caller's kept list and pads it with the
//                     out-of-range index H to a multiple of the GEMM K-block;
//                     with no list given, the identity list 0..k-1 (keep
//                     ratio 1: every slice kept), optionally copied out.
#include "rmm_common.cuh"
#include "rmm_internal.h"

namespace rmm {

namespace {

constexpr int kTile = 64;

__global__ void __launch_bounds__(256)
    transpose_kernel(const uint16_t* __restrict__ W, uint16_t* __restrict__ Wt, int N, int H) {
    pdl_wait();
    __shared__ uint16_t tile[kTile][kTile + 2];
    const int h0 = blockIdx.x * kTile, n0 = blockIdx.y * kTile;
    const int tx = threadIdx.x & 63, ty = threadIdx.x >> 6;  // 64 x 4
    for (int i = ty; i < kTile; i += 4) {
        const int n = n0 + i, h = h0 + tx;
        tile[i][tx] = (n < N && h < H) ? W[(size_t)n * H + h] : (uint16_t)0;
    }
    __syncthreads();
    for (int i = ty; i < kTile; i += 4) {
        const int h = h0 + i, n = n0 + tx;
        if (h < H && n < N) Wt[(size_t)h * N + n] = tile[tx][i];
    }
}

__global__ void pad_idx_kernel(const int32_t* __restrict__ src, int k, int H,
                               int32_t* __restrict__ dst, int pad_to, int32_t* __restrict__ dst_copy) {
    pdl_wait();
    pdl_launch_dependents();
    for (int j = blockIdx.x * blockDim.x + threadIdx.x; j < pad_to; j += gridDim.x * blockDim.x) {
        const int32_t v = (j < k) ? (src ? src[j] : j) : H;
        dst[j] = v;
        if (dst_copy && j < k) dst_copy[j] = v;
    }
}

}  // namespace

cudaError_t launch_transpose(const uint16_t* W, uint16_t* Wt, int N, int H, cudaStream_t stream) {
    dim3 grid((H + kTile - 1) / kTile, (N + kTile - 1) / kTile);
    transpose_kernel<<<grid, 256, 0, stream>>>(W, Wt, N, H);
    return cudaGetLastError();
}

cudaError_t launch_pad_idx(const int32_t* src, int k, int H, int32_t* dst, int pad_to, cudaStream_t stream,
                           int32_t* dst_copy) {
    const int blocks = (pad_to + 255) / 256;
    return launch_pdl(pad_idx_kernel, dim3(blocks < 1 ? 1 : blocks), dim3(256), 0, stream, src, k, H, dst,
                      pad_to, dst_copy);
}

}  // namespace rmm
