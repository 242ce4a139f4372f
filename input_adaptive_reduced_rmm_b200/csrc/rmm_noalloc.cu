// rmm_noalloc.cu -- the decode-sized reduced linear map with library-owned scratch.
//
// Some callers cannot hand the library a workspace: they run where allocating
// device memory is not theirs to do -- a plugin whose host framework owns every
// allocation and only lends it input and output buffers, or an inference loop
// under a fixed memory budget that must not grow once serving has started.
// rmm_linear_decode_noalloc serves them: the same score -> kept set -> split-K
// GEMV path as rmm_linear for T <= 16, but every intermediate (the score
// vector, the kept list, the split partial sums) lives in one file-scope
// __device__ array of fixed size that every GPU loading the library holds
// until the process exits.  Nothing is allocated or freed.
//
// Host code never uses the array's name as a device address: on first use on
// a device (with that device current) the address is obtained once with
// cudaGetSymbolAddress, checked, cached per device, and passed to the kernels.
// That first call on a device should come before any stream capture.
#include <string.h>

#include <mutex>

#include "rmm_common.cuh"
#include "rmm_internal.h"

namespace rmm {
namespace {

constexpr size_t kNoAllocScratchBytes = size_t(4) << 20;  // 4 MiB per device
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

std::mutex g_noalloc_mu;
void* g_noalloc_ptr[kMaxDevices] = {};

size_t up256(size_t v) { return (v + 255) / 256 * 256; }

// Device address of the scratch array on the current device (set up once per device).
rmm_status noalloc_scratch(uint8_t** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return RMM_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return RMM_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> g(g_noalloc_mu);
    if (!g_noalloc_ptr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return RMM_ERR_CUDA;
        g_noalloc_ptr[dev] = p;
    }
    *out = static_cast<uint8_t*>(g_noalloc_ptr[dev]);
    return RMM_OK;
}

// Zero the words a call needs to start at zero (the score vector, which the
// score pass folds into with atomicMax); the scratch keeps whatever the
// previous call left there.
__global__ void noalloc_clear_kernel(unsigned* words, int n) {
    pdl_wait();
    pdl_launch_dependents();
    for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x) words[i] = 0;
}

}  // namespace
}  // namespace rmm

using namespace rmm;

extern "C" rmm_status rmm_linear_decode_noalloc(const void* X, const void* Wt, int T, int H, int N,
                                                double r, void* Y, int32_t* idx_out,
                                                rmm_stream_t stream) {
    if (!X || !Wt || !Y || T < 1 || H < 1 || H > 65535 || N < 8 || N % 8 != 0) return RMM_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(X) | reinterpret_cast<uintptr_t>(Wt) | reinterpret_cast<uintptr_t>(Y)) & 15)
        return RMM_ERR_INVALID_ARG;
    if (T > kGemvMaxT || N > (1 << 20)) return RMM_ERR_UNSUPPORTED;  // beyond the scratch's sizing
    const int k = rmm_k_for(H, r);
    if (k < 1) return RMM_ERR_INVALID_ARG;

    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) != cudaSuccess) return RMM_ERR_CUDA;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return RMM_ERR_CUDA;
    uint8_t* scratch = nullptr;
    rmm_status st = noalloc_scratch(&scratch);
    if (st != RMM_OK) return st;

    // scratch layout: score vector | kept list | split partials
    const size_t off_s32 = 0;
    const size_t off_idx = off_s32 + up256((size_t)H * sizeof(uint32_t));
    const size_t off_partials = off_idx + up256(((size_t)H + 2 * kGemmBK) * sizeof(int32_t));
    if (off_partials >= kNoAllocScratchBytes) return RMM_ERR_UNSUPPORTED;
    const size_t room = kNoAllocScratchBytes - off_partials;
    if (gemv_smem_bytes(gemv_cols_for(T), T) > kGemvMaxSmemBytes) return RMM_ERR_UNSUPPORTED;

    // Plan for the output columns [c0, c0 + w): the default splits when their
    // partial sums fit, else fewer; false when even the fewest do not fit.
    auto plan_for = [&](GemvGroup& g, int c0, int w) {
        memset(&g, 0, sizeof g);
        g.count = 1;
        g.Wt[0] = static_cast<const uint16_t*>(Wt) + c0;
        g.Y[0] = static_cast<uint16_t*>(Y) + c0;
        g.N[0] = w;
        g.ld[0] = N;
        size_t part = gemv_group_plan(g, T, k, 0, sms);
        if (part > room) {
            const int splits = (int)(room / ((size_t)T * w * sizeof(float)));
            g.ld[0] = N;
            part = gemv_group_plan(g, T, k, splits < 2 ? 1 : splits, sms);
        }
        return part <= room;
    };
    // columns per launch: all N when the partial sums fit, else halves of it
    // (multiples of 8 columns, so every launch keeps 16-byte alignment)
    GemvGroup g;
    int chunk = N;
    while (!plan_for(g, 0, chunk)) {
        if (chunk <= 64) return RMM_ERR_UNSUPPORTED;
        chunk = (chunk / 2 + 7) / 8 * 8;
    }

    cudaStream_t s = static_cast<cudaStream_t>(stream);
    // the score vector must start at zero
    noalloc_clear_kernel<<<(int)((off_idx / 4 + 255) / 256), 256, 0, s>>>(reinterpret_cast<unsigned*>(scratch),
                                                                         (int)(off_idx / 4));
    if (cudaGetLastError() != cudaSuccess) return RMM_ERR_CUDA;

    uint32_t* s32 = reinterpret_cast<uint32_t*>(scratch + off_s32);
    int32_t* idx = reinterpret_cast<int32_t*>(scratch + off_idx);
    // the score vector was just cleared; the select clears it again after reading
    cudaError_t e = (T == 1) ? launch_select(static_cast<const uint16_t*>(X), T, nullptr, 0, H, k, idx, k, idx_out,
                                             nullptr, s)
                             : launch_score(static_cast<const uint16_t*>(X), T, H, s32, nullptr, 0, sms, s);
    if (e == cudaSuccess && T > 1) e = launch_select(nullptr, 0, s32, 1, H, k, idx, k, idx_out, nullptr, s);
    if (e != cudaSuccess) return RMM_ERR_CUDA;
    // one product per column chunk, one after another through the same partials
    for (int c0 = 0; c0 < N; c0 += chunk) {
        const int w = (N - c0 < chunk) ? N - c0 : chunk;
        if (!plan_for(g, c0, w)) return RMM_ERR_UNSUPPORTED;
        if (launch_gemv(static_cast<const uint16_t*>(X), T, H, idx, k, g,
                        reinterpret_cast<float*>(scratch + off_partials), sms, s) != cudaSuccess)
            return RMM_ERR_CUDA;
    }
    return RMM_OK;
}
