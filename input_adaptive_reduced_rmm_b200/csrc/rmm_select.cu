// rmm_select.cu -- step 2 of the reduced product: the kept set.
//
// Keeps the k = ceil(r*H) slices with the largest scores under the total
// order (score desc, index asc) and emits them in ascending index order
// (cf-1.com post on input-adaptive matrix-product reduction, §5.2 score ->
// top-k; §6.1 demo: top-k followed by a sort so the kept slices keep their
// original order).
//
// One CTA of 1024 threads, scores resident in shared memory:
//   1. read the score vector into shared memory (and clear it for the next
//      call when it is the library's own accumulator);
//   2. radix select on the key: a 256-bin histogram of s>>8 finds the bin of
//      the k-th largest score, a 256-bin histogram of s&255 inside that bin
//      finds the threshold score s*; c_gt = #{s > s*}, need = k - c_gt;
//   3. ordered compaction: every thread owns a contiguous run of indices, one
//      block-wide scan of packed (#gt, #eq) counts gives each run its output
//      offset, and index h is kept iff s_h > s*, or s_h == s* and fewer than
//      `need` equal scores precede it -- which yields the ascending list
//      directly, with ties resolved toward the lower index.
#include "rmm_common.cuh"
#include "rmm_internal.h"

namespace rmm {

namespace {

constexpr int kThreads = 1024;
constexpr int kWarps = kThreads / 32;

// Inclusive block-wide sum of one value per thread (all threads participate).
__device__ __forceinline__ uint32_t block_inclusive_scan(uint32_t v, uint32_t* warp_tot) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        uint32_t n = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += n;
    }
    if (lane == 31) warp_tot[warp] = v;
    __syncthreads();
    if (warp == 0) {
        uint32_t w = (lane < kWarps) ? warp_tot[lane] : 0;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            uint32_t n = __shfl_up_sync(0xffffffffu, w, o);
            if (lane >= o) w += n;
        }
        warp_tot[lane] = w;  // inclusive prefix over warps
    }
    __syncthreads();
    uint32_t base = (warp > 0) ? warp_tot[warp - 1] : 0;
    __syncthreads();  // warp_tot may be reused by the caller
    return base + v;
}

// Within one warp: given counts cnt[b] of nbins bins, find the bin holding the
// k-th largest element counting from the top bin down.  Returns the bin and
// the number of elements in higher bins (via *above).
__device__ __forceinline__ int warp_find_bin(const int* cnt, int nbins, int k, int* above) {
    const int lane = threadIdx.x & 31;
    const int per = nbins / 32;  // bins per lane, lane 0 owns the highest bins
    int hi = nbins - 1 - lane * per;
    int sum = 0;
    for (int i = 0; i < per; ++i) sum += cnt[hi - i];
    int incl = sum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        int n = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += n;
    }
    int run = incl - sum;  // elements in bins above this lane's run
    int found = -1, found_above = 0;
    if (run < k && run + sum >= k) {
        for (int i = 0; i < per; ++i) {
            int b = hi - i;
            if (run + cnt[b] >= k) {
                found = b;
                found_above = run;
                break;
            }
            run += cnt[b];
        }
    }
    unsigned m = __ballot_sync(0xffffffffu, found >= 0);
    int src = __ffs(m) - 1;
    *above = __shfl_sync(0xffffffffu, found_above, src);
    return __shfl_sync(0xffffffffu, found, src);
}

// Histogram of 8-bit bins over the keys: bin = (key >> shift) & 255 for keys
// with key >> 8 == match (all keys when match == ~0).  Lanes holding the same
// bin are merged with __match_any_sync so each distinct bin costs one shared
// atomic per warp and chunk.
__device__ __forceinline__ void warp_histogram(const uint16_t* s, int H, int shift, uint32_t match,
                                               int* hist) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    for (int h0 = warp * 32; h0 < H; h0 += kThreads) {
        const int h = h0 + lane;
        uint32_t bin = 0xFFFFFFFFu;  // "no bin"
        if (h < H) {
            const uint32_t v = s[h];
            if (match == 0xFFFFFFFFu || (v >> 8) == match) bin = (v >> shift) & 0xFFu;
        }
        const unsigned same = __match_any_sync(0xffffffffu, bin);
        if (bin != 0xFFFFFFFFu && lane == __ffs(same) - 1) atomicAdd(&hist[bin], __popc(same));
    }
}

__global__ void __launch_bounds__(kThreads)
    select_kernel(uint32_t* __restrict__ s32, int clear_input, int H, int k, int32_t* __restrict__ idx,
                  int pad_to, int32_t* __restrict__ idx_copy, uint32_t* __restrict__ s_out) {
    extern __shared__ uint16_t s[];  // H keys
    __shared__ int hist_hi[256];
    __shared__ int hist_fine[256];
    __shared__ uint32_t warp_tot[32];
    __shared__ int sh_thresh, sh_need;

    pdl_wait();
    pdl_launch_dependents();
    const int tid = threadIdx.x;
    if (tid < 256) hist_hi[tid] = 0;
    if (tid < 256) hist_fine[tid] = 0;

    // 1. load the scores
    for (int h = tid; h < H; h += kThreads) {
        const uint32_t m = s32[h] & 0xFFFFu;
        if (clear_input) s32[h] = 0;
        s[h] = (uint16_t)m;
        if (s_out) s_out[h] = m;
    }
    __syncthreads();

    // 2a. coarse histogram of s >> 8 (256 bins; keys are < 2^16, and < 2^15
    //     for finite bf16 magnitudes).  Scores of one input crowd into a few
    //     exponent bins, so equal bins are merged per warp first.
    warp_histogram(s, H, 8, 0xFFFFFFFFu, hist_hi);
    __syncthreads();
    if (tid < 32) {
        int above;
        int b = warp_find_bin(hist_hi, 256, k, &above);
        if (tid == 0) {
            sh_thresh = b;
            sh_need = k - above;  // elements still to take from bin b downward
        }
    }
    __syncthreads();
    const int bhi = sh_thresh;
    const int k2 = sh_need;
    // 2b. fine histogram of the low 8 bits inside the coarse bin
    warp_histogram(s, H, 0, (uint32_t)bhi, hist_fine);
    __syncthreads();
    if (tid < 32) {
        int above;
        int b = warp_find_bin(hist_fine, 256, k2, &above);
        if (tid == 0) {
            sh_thresh = (bhi << 8) | b;
            sh_need = k2 - above;  // equal-to-threshold elements to keep
        }
    }
    __syncthreads();
    const uint32_t thr = (uint32_t)sh_thresh;
    const uint32_t need = (uint32_t)sh_need;

    // 3. ordered compaction over contiguous runs
    const int per = (H + kThreads - 1) / kThreads;
    const int lo = min(H, tid * per), hi = min(H, lo + per);
    uint32_t gt = 0, eq = 0;
    for (int h = lo; h < hi; ++h) {
        uint32_t v = s[h];
        gt += (v > thr);
        eq += (v == thr);
    }
    // pack (gt, eq) in one word: both totals are <= H <= 65535
    uint32_t incl = block_inclusive_scan((gt << 16) | eq, warp_tot);
    uint32_t excl = incl - ((gt << 16) | eq);
    uint32_t gt_before = excl >> 16, eq_before = excl & 0xFFFFu;
    for (int h = lo; h < hi; ++h) {
        uint32_t v = s[h];
        if (v > thr) {
            const uint32_t pos = gt_before + min(eq_before, need);
            idx[pos] = h;
            if (idx_copy) idx_copy[pos] = h;
            ++gt_before;
        } else if (v == thr) {
            if (eq_before < need) {
                idx[gt_before + eq_before] = h;
                if (idx_copy) idx_copy[gt_before + eq_before] = h;
            }
            ++eq_before;
        }
    }
    for (int j = k + tid; j < pad_to; j += kThreads) idx[j] = H;
}

}  // namespace

cudaError_t launch_select(uint32_t* s32, int clear_input, int H, int k, int32_t* idx, int pad_to,
                          int32_t* idx_copy, uint32_t* s_out, cudaStream_t stream) {
    const size_t smem = ((size_t)H * sizeof(uint16_t) + 15) & ~(size_t)15;
    if (smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(select_kernel,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
    }
    return launch_pdl(select_kernel, dim3(1), dim3(kThreads), smem, stream, s32, clear_input, H, k, idx,
                      pad_to, idx_copy, s_out);
}

}  // namespace rmm
