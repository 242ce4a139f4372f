// rmm_select.cu -- step 2 of the reduced product: the kept set.
//
// Keeps the k = ceil(r*H) slices with the largest scores under the total
// order (score desc, index asc) and emits them in ascending index order
// (cf-1.com post on input-adaptive matrix-product reduction, §5.2 score ->
// top-k; §6.1 demo: top-k followed by a sort so the kept slices keep their
// original order).
//
// Up to H = 16384: one CTA of 1024 threads (above: the same steps on a
// cluster of CTAs, select_cluster_kernel); keys are 16-bit (bf16 magnitude
// bits):
//   1. every thread loads its strided share of the keys into registers, all
//      loads in flight at once (from X for one token, else from the score
//      vector, which is cleared behind the read when it is the library's own
//      accumulator), while the CTA clears a 128 KB shared histogram;
//   2. one shared-memory atomic per key counts it in a histogram over all
//      2^16 key values (two 16-bit counts per word).  Exact bins: a warp's
//      keys rarely share a value, so the atomics hardly ever serialise, even
//      though an activation's magnitudes crowd into a few exponents;
//   3. the threshold s* = the k-th largest key: per-warp sums of 32 ranges of
//      2048 keys, then one warp descends from the top through the range, a
//      32-word chunk of it and a word of that chunk; c_gt = #{s > s*} comes
//      out of the descent and need = k - c_gt;
//   4. ordered compaction straight from the registers: ballots count each
//      warp's greater and equal keys per row of 1024 slices, one block-wide
//      scan of the packed (#gt, #eq) counts gives every warp-row its output
//      offset, and the ballots rank each key inside it.  Index h is kept iff
//      s_h > s*, or s_h == s* and fewer than `need` equal scores precede it --
//      which yields the ascending list directly, with ties resolved toward the
//      lower index.
#include "rmm_common.cuh"
#include "rmm_internal.h"

namespace rmm {

namespace {

constexpr int kThreads = 1024;
constexpr int kWarps = kThreads / 32;
constexpr int kHistWords = 32768;  // 2^16 keys, two 16-bit counts per word
constexpr size_t kSmemBytes = kHistWords * sizeof(uint32_t);  // then the compaction's counts
// Larger H: the selection runs on a cluster of CTAs.  Measured on B200 (ncu,
// one select): H = 28672 takes 9.6 us on 8 CTAs against 19.7 us on one; at
// H = 14336 both take ~9.5 us, and at 4096 one CTA is faster (5.8 against 8.2
// us): the cluster's barriers and per-CTA histogram sweeps are a fixed cost.
constexpr int kClusterMinH = 16384;
static_assert(kWarps == 32, "the descent takes one range per warp");

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

__device__ __forceinline__ uint32_t warp_inclusive_scan(uint32_t v) {
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        uint32_t n = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += n;
    }
    return v;
}

// Keys this thread holds: key e is slice tid + e * kThreads.  E <= 16 keys are
// held one per register, more two per register (even e low half, odd e high).
template <int E>
struct Keys {
    static constexpr bool kPacked = E > 16;
    static constexpr int R = kPacked ? E / 2 : E;
    uint32_t v[R];

    __device__ __forceinline__ uint32_t get(int e) const {
        if (kPacked) return (e & 1) ? (v[e / 2] >> 16) : (v[e / 2] & 0xFFFFu);
        return v[e];
    }

    // Read the keys -- the fold of X's T rows, or the score vector (cleared
    // behind the read when asked) -- into registers; up to 16 loads are in
    // flight per thread.  Slices past H get key 0 and are never counted.
    // `meanwhile` runs once, after the first loads are issued and before any
    // is used.
    // Keys of slices base + (tid + e * kThreads) for e < E, those below `count`.
    template <class F>
    __device__ __forceinline__ void load(const uint16_t* __restrict__ X, int T, uint32_t* __restrict__ s32,
                                         int clear_input, int H, uint32_t* __restrict__ s_out, F&& meanwhile,
                                         int base = 0, int count = -1) {
        const int tid = threadIdx.x;
        if (count < 0) count = H;
        constexpr int B = E < 16 ? E : 16;
#pragma unroll
        for (int b0 = 0; b0 < E; b0 += B) {
            uint32_t raw[B];
#pragma unroll
            for (int u = 0; u < B; ++u) {
                const int hl = tid + (b0 + u) * kThreads;
                raw[u] = 0;
                if (hl < count) raw[u] = X ? (uint32_t)X[base + hl] : s32[base + hl];
            }
            if (b0 == 0) meanwhile();
#pragma unroll
            for (int u = 0; u < B; ++u) raw[u] &= X ? 0x7FFFu : 0xFFFFu;
            if (X) {
                for (int t = 1; t < T; ++t) {
#pragma unroll
                    for (int u = 0; u < B; ++u) {
                        const int hl = tid + (b0 + u) * kThreads;
                        if (hl < count) raw[u] = max(raw[u], (uint32_t)(X[(size_t)t * H + base + hl] & 0x7FFFu));
                    }
                }
            }
#pragma unroll
            for (int u = 0; u < B; ++u) {
                const int e = b0 + u;
                const int hl = tid + e * kThreads;
                if (hl < count) {
                    if (!X && clear_input) s32[base + hl] = 0;
                    if (s_out) s_out[base + hl] = raw[u];
                }
                if (kPacked) {
                    if (e & 1) v[e / 2] |= raw[u] << 16;
                    else v[e / 2] = raw[u];
                } else {
                    v[e] = raw[u];
                }
            }
        }
    }
};

// Warp 0: the k-th largest key from the histogram.  hist word w counts key 2w
// in its low half and key 2w+1 in its high half; range_tot[r] counts the keys
// of words [1024 r, 1024 r + 1024).  Lane l looks at the (31 - l)-th piece, so
// that lane order runs from the largest keys down; at each level the first
// lane whose running count reaches k names the piece holding s*, and `above`
// accumulates the keys in the pieces above it.
__device__ __forceinline__ void descend(const uint32_t* hist, const uint32_t* range_tot, uint32_t k,
                                        uint32_t* thr_out, uint32_t* above_out) {
    const int lane = threadIdx.x & 31;
    // ranges of 1024 words
    uint32_t c = range_tot[31 - lane];
    uint32_t incl = warp_inclusive_scan(c);
    int L = __ffs(__ballot_sync(0xffffffffu, incl >= k)) - 1;
    uint32_t above = __shfl_sync(0xffffffffu, incl - c, L);
    const int r = 31 - L;
    // chunks of 32 words inside the range (read rotated: 4-way bank conflicts at most)
    const uint4* chunk = reinterpret_cast<const uint4*>(hist + r * 1024 + (31 - lane) * 32);
    uint32_t w = 0;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        const uint4 x = chunk[(j + lane) & 7];
        w += x.x + x.y + x.z + x.w;
    }
    c = (w & 0xFFFFu) + (w >> 16);
    incl = warp_inclusive_scan(c);
    L = __ffs(__ballot_sync(0xffffffffu, above + incl >= k)) - 1;
    above += __shfl_sync(0xffffffffu, incl - c, L);
    const int cw = r * 1024 + (31 - L) * 32;
    // words of the chunk
    const uint32_t wv = hist[cw + 31 - lane];
    c = (wv & 0xFFFFu) + (wv >> 16);
    incl = warp_inclusive_scan(c);
    L = __ffs(__ballot_sync(0xffffffffu, above + incl >= k)) - 1;
    above += __shfl_sync(0xffffffffu, incl - c, L);
    const uint32_t wsel = __shfl_sync(0xffffffffu, wv, L);
    const uint32_t b = (uint32_t)(cw + 31 - L);
    const uint32_t n_odd = wsel >> 16;  // count of key 2b+1, the larger of the word's two
    if (above + n_odd >= k) {
        *thr_out = 2 * b + 1;
    } else {
        above += n_odd;
        *thr_out = 2 * b;
    }
    *above_out = above;
}

template <int E>  // keys per thread: H <= E * kThreads
__global__ void __launch_bounds__(kThreads, 1)
    select_kernel(const uint16_t* __restrict__ X, int T, uint32_t* __restrict__ s32, int clear_input, int H,
                  int k, int32_t* __restrict__ idx, int pad_to, int32_t* __restrict__ idx_copy,
                  uint32_t* __restrict__ s_out) {
    extern __shared__ __align__(16) uint32_t hist[];  // kHistWords; later the H keys
    __shared__ uint32_t range_tot[32];
    __shared__ uint32_t warp_tot[32];
    __shared__ uint32_t sh_thr, sh_need;

    pdl_wait();
    pdl_launch_dependents();
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

    // 1. the keys into registers; the histogram is cleared while they arrive
    Keys<E> keys;
    keys.load(X, T, s32, clear_input, H, s_out, [&] {
        uint4* h4 = reinterpret_cast<uint4*>(hist);
#pragma unroll
        for (int i = 0; i < kHistWords / 4 / kThreads; ++i) h4[tid + i * kThreads] = make_uint4(0u, 0u, 0u, 0u);
    });
    __syncthreads();

    // 2. exact histogram
#pragma unroll
    for (int e = 0; e < E; ++e) {
        const int h = tid + e * kThreads;
        if (h < H) {
            const uint32_t key = keys.get(e);
            atomicAdd(&hist[key >> 1], (key & 1u) ? 0x10000u : 1u);
        }
    }
    __syncthreads();

    // 3. per-range totals (warp w: words [1024 w, 1024 w + 1024)), then the descent
    {
        const uint4* q = reinterpret_cast<const uint4*>(hist + warp * 1024);
        uint32_t w = 0;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const uint4 x = q[lane + 32 * j];
            w += x.x + x.y + x.z + x.w;
        }
        const uint32_t c = __reduce_add_sync(0xffffffffu, (w & 0xFFFFu) + (w >> 16));
        if (lane == 0) range_tot[warp] = c;
    }
    __syncthreads();
    if (warp == 0) {
        uint32_t thr, above;
        descend(hist, range_tot, (uint32_t)k, &thr, &above);
        if (lane == 0) {
            sh_thr = thr;
            sh_need = (uint32_t)k - above;
        }
    }
    __syncthreads();
    const uint32_t thr = sh_thr;
    const uint32_t need = sh_need;

    // 4. ordered compaction.  Slice h = tid + 1024 e, so index order is
    //    (e, warp, lane).  Each warp counts its greater and equal keys of every
    //    row e with two ballots and stores them packed (#gt << 16 | #eq, both
    //    totals < 2^16) at cnt[e * 32 + warp]; one block-wide scan turns the
    //    counts into exclusive prefixes in index order; the ballots again rank
    //    each key inside its warp.
    uint32_t* cnt = hist;  // E * 32 words, over the histogram
    const uint32_t lt_mask = (1u << lane) - 1u;
#pragma unroll
    for (int e = 0; e < E; ++e) {
        const int h = tid + e * kThreads;
        const uint32_t v = keys.get(e);
        const uint32_t bg = __ballot_sync(0xffffffffu, h < H && v > thr);
        const uint32_t be = __ballot_sync(0xffffffffu, h < H && v == thr);
        if (lane == 0) cnt[e * 32 + warp] = ((uint32_t)__popc(bg) << 16) | (uint32_t)__popc(be);
    }
    __syncthreads();
    {
        constexpr int P = (E * 32 + kThreads - 1) / kThreads;  // entries per thread
        uint32_t x[P], sum = 0;
#pragma unroll
        for (int p = 0; p < P; ++p) {
            const int i = tid * P + p;
            x[p] = (i < E * 32) ? cnt[i] : 0u;
            sum += x[p];
        }
        uint32_t run = block_inclusive_scan(sum, warp_tot) - sum;
#pragma unroll
        for (int p = 0; p < P; ++p) {
            const int i = tid * P + p;
            if (i < E * 32) cnt[i] = run;
            run += x[p];
        }
    }
    __syncthreads();
#pragma unroll
    for (int e = 0; e < E; ++e) {
        const int h = tid + e * kThreads;
        const uint32_t v = keys.get(e);
        const bool is_gt = h < H && v > thr;
        const bool is_eq = h < H && v == thr;
        const uint32_t bg = __ballot_sync(0xffffffffu, is_gt);
        const uint32_t be = __ballot_sync(0xffffffffu, is_eq);
        const uint32_t base = cnt[e * 32 + warp];
        const uint32_t g_rank = (base >> 16) + __popc(bg & lt_mask);
        const uint32_t e_rank = (base & 0xFFFFu) + __popc(be & lt_mask);
        if (is_gt || (is_eq && e_rank < need)) {
            const uint32_t pos = g_rank + min(e_rank, need);
            idx[pos] = h;
            if (idx_copy) idx_copy[pos] = h;
        }
    }
    for (int j = k + tid; j < pad_to; j += kThreads) idx[j] = H;
}

// u32 at a shared-memory address of the cluster window
__device__ __forceinline__ uint32_t ld_shared_cluster_u32(uint32_t addr) {
    uint32_t v;
    asm volatile("ld.shared::cluster.u32 %0, [%1];" : "=r"(v) : "r"(addr) : "memory");
    return v;
}

__device__ __forceinline__ uint32_t cluster_nctarank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_nctarank;" : "=r"(r));
    return r;
}

// The same selection spread over a cluster of C CTAs (one SM could not keep up:
// every key costs a few dozen instructions across 1024 threads).  CTA c takes
// the contiguous slices [c * slice, c * slice + slice) and builds its own 2^16
// histogram; the descent to s* adds the CTAs' counts at each level (32 ranges,
// 32 chunks, 32 words) read through distributed shared memory, one cluster
// barrier per level; in the compaction each CTA places its keys after the
// #gt and #eq of the CTAs before it (index order = CTA order).  A final
// cluster barrier keeps every CTA's counts readable until all have read them.
template <int E>  // keys per thread: slice <= E * kThreads
__global__ void __launch_bounds__(kThreads, 1)
    select_cluster_kernel(const uint16_t* __restrict__ X, int T, uint32_t* __restrict__ s32, int clear_input, int H,
                          int k, int32_t* __restrict__ idx, int pad_to, int32_t* __restrict__ idx_copy,
                          uint32_t* __restrict__ s_out, int slice) {
    extern __shared__ __align__(16) uint32_t hist[];  // kHistWords; later the compaction's counts
    __shared__ uint32_t lvl0[32], lvl1[32], lvl2lo[32], lvl2hi[32];  // this CTA's counts per descent piece
    __shared__ uint32_t warp_tot[32];
    __shared__ uint32_t cta_tot;  // this CTA's #gt << 16 | #eq
    __shared__ uint32_t sh_r, sh_cw, sh_thr, sh_need, sh_above, sh_gt_before, sh_eq_before;

    pdl_wait();
    pdl_launch_dependents();
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const uint32_t C = cluster_nctarank(), c = cluster_ctarank();
    const int base = (int)c * slice;
    const int count = max(0, min(H - base, slice));

    // 1. this CTA's keys into registers while its histogram is cleared
    Keys<E> keys;
    keys.load(X, T, s32, clear_input, H, s_out, [&] {
        uint4* h4 = reinterpret_cast<uint4*>(hist);
#pragma unroll
        for (int i = 0; i < kHistWords / 4 / kThreads; ++i) h4[tid + i * kThreads] = make_uint4(0u, 0u, 0u, 0u);
    }, base, count);
    __syncthreads();

    // 2. exact histogram of this CTA's keys
#pragma unroll
    for (int e = 0; e < E; ++e) {
        if (tid + e * kThreads < count) {
            const uint32_t key = keys.get(e);
            atomicAdd(&hist[key >> 1], (key & 1u) ? 0x10000u : 1u);
        }
    }
    __syncthreads();

    // 3. the descent: piece p of a level covers larger keys as p grows; lane l
    //    looks at piece 31 - l, so lane order runs from the largest keys down
    {
        const uint4* q = reinterpret_cast<const uint4*>(hist + warp * 1024);
        uint32_t w = 0;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const uint4 x = q[lane + 32 * j];
            w += x.x + x.y + x.z + x.w;
        }
        const uint32_t cnt = __reduce_add_sync(0xffffffffu, (w & 0xFFFFu) + (w >> 16));
        if (lane == 0) lvl0[warp] = cnt;
    }
    cluster_sync();
    if (warp == 0) {
        // ranges of 1024 words, summed over the cluster
        uint32_t cnt = 0;
        for (uint32_t j = 0; j < C; ++j) cnt += ld_shared_cluster_u32(mapa_shared(smem_addr(&lvl0[31 - lane]), j));
        uint32_t incl = warp_inclusive_scan(cnt);
        const int L = __ffs(__ballot_sync(0xffffffffu, incl >= (uint32_t)k)) - 1;
        const uint32_t above = __shfl_sync(0xffffffffu, incl - cnt, L);
        const int r = 31 - L;
        // this CTA's 32 chunks (32 words each) of range r
        const uint4* ch = reinterpret_cast<const uint4*>(hist + r * 1024 + lane * 32);
        uint32_t w = 0;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const uint4 x = ch[(j + lane) & 7];
            w += x.x + x.y + x.z + x.w;
        }
        lvl1[lane] = (w & 0xFFFFu) + (w >> 16);
        if (lane == 0) {
            sh_r = (uint32_t)r;
            sh_above = above;
        }
    }
    cluster_sync();
    if (warp == 0) {
        const int r = (int)sh_r;
        uint32_t above = sh_above;
        uint32_t cnt = 0;
        for (uint32_t j = 0; j < C; ++j) cnt += ld_shared_cluster_u32(mapa_shared(smem_addr(&lvl1[31 - lane]), j));
        const uint32_t incl = warp_inclusive_scan(cnt);
        const int L = __ffs(__ballot_sync(0xffffffffu, above + incl >= (uint32_t)k)) - 1;
        above += __shfl_sync(0xffffffffu, incl - cnt, L);
        const int cw = r * 1024 + (31 - L) * 32;
        // this CTA's 32 words of chunk cw: key 2w in the low half, 2w+1 in the high half
        const uint32_t wv = hist[cw + lane];
        lvl2lo[lane] = wv & 0xFFFFu;
        lvl2hi[lane] = wv >> 16;
        if (lane == 0) {
            sh_cw = (uint32_t)cw;
            sh_above = above;
        }
    }
    cluster_sync();
    if (warp == 0) {
        const int cw = (int)sh_cw;
        uint32_t above = sh_above;
        uint32_t lo = 0, hi = 0;
        for (uint32_t j = 0; j < C; ++j) {
            lo += ld_shared_cluster_u32(mapa_shared(smem_addr(&lvl2lo[31 - lane]), j));
            hi += ld_shared_cluster_u32(mapa_shared(smem_addr(&lvl2hi[31 - lane]), j));
        }
        const uint32_t cnt = lo + hi;
        const uint32_t incl = warp_inclusive_scan(cnt);
        const int L = __ffs(__ballot_sync(0xffffffffu, above + incl >= (uint32_t)k)) - 1;
        above += __shfl_sync(0xffffffffu, incl - cnt, L);
        const uint32_t n_odd = __shfl_sync(0xffffffffu, hi, L);  // key 2b+1, the larger of the word's two
        const uint32_t b = (uint32_t)(cw + 31 - L);
        if (lane == 0) {
            uint32_t thr;
            if (above + n_odd >= (uint32_t)k) {
                thr = 2 * b + 1;
            } else {
                above += n_odd;
                thr = 2 * b;
            }
            sh_thr = thr;
            sh_need = (uint32_t)k - above;
        }
    }
    __syncthreads();
    const uint32_t thr = sh_thr;
    const uint32_t need = sh_need;

    // 4. ordered compaction inside the CTA (as in the one-CTA kernel), then
    //    after the #gt / #eq of the CTAs before this one
    uint32_t* cnt = hist;  // E * 32 words, over the histogram
    const uint32_t lt_mask = (1u << lane) - 1u;
#pragma unroll
    for (int e = 0; e < E; ++e) {
        const bool ok = tid + e * kThreads < count;
        const uint32_t v = keys.get(e);
        const uint32_t bg = __ballot_sync(0xffffffffu, ok && v > thr);
        const uint32_t be = __ballot_sync(0xffffffffu, ok && v == thr);
        if (lane == 0) cnt[e * 32 + warp] = ((uint32_t)__popc(bg) << 16) | (uint32_t)__popc(be);
    }
    __syncthreads();
    {
        constexpr int P = (E * 32 + kThreads - 1) / kThreads;  // entries per thread
        uint32_t x[P], sum = 0;
#pragma unroll
        for (int p = 0; p < P; ++p) {
            const int i = tid * P + p;
            x[p] = (i < E * 32) ? cnt[i] : 0u;
            sum += x[p];
        }
        uint32_t run = block_inclusive_scan(sum, warp_tot) - sum;
#pragma unroll
        for (int p = 0; p < P; ++p) {
            const int i = tid * P + p;
            if (i < E * 32) cnt[i] = run;
            run += x[p];
        }
        if (tid == kThreads - 1) cta_tot = run;  // the CTA's totals (the last thread's inclusive sum)
    }
    cluster_sync();
    if (warp == 0) {
        uint32_t g = 0, q = 0;
        if ((uint32_t)lane < c) {
            const uint32_t t = ld_shared_cluster_u32(mapa_shared(smem_addr(&cta_tot), (uint32_t)lane));
            g = t >> 16;
            q = t & 0xFFFFu;
        }
        g = __reduce_add_sync(0xffffffffu, g);
        q = __reduce_add_sync(0xffffffffu, q);
        if (lane == 0) {
            sh_gt_before = g;
            sh_eq_before = q;
        }
    }
    __syncthreads();
    const uint32_t gt_before = sh_gt_before, eq_before = sh_eq_before;
#pragma unroll
    for (int e = 0; e < E; ++e) {
        const int hl = tid + e * kThreads;
        const bool ok = hl < count;
        const uint32_t v = keys.get(e);
        const bool is_gt = ok && v > thr;
        const bool is_eq = ok && v == thr;
        const uint32_t bg = __ballot_sync(0xffffffffu, is_gt);
        const uint32_t be = __ballot_sync(0xffffffffu, is_eq);
        const uint32_t bc = cnt[e * 32 + warp];
        const uint32_t g_rank = gt_before + (bc >> 16) + __popc(bg & lt_mask);
        const uint32_t e_rank = eq_before + (bc & 0xFFFFu) + __popc(be & lt_mask);
        if (is_gt || (is_eq && e_rank < need)) {
            const uint32_t pos = g_rank + min(e_rank, need);
            idx[pos] = base + hl;
            if (idx_copy) idx_copy[pos] = base + hl;
        }
    }
    if (c == 0)
        for (int j = k + tid; j < pad_to; j += kThreads) idx[j] = H;
    cluster_sync();  // every CTA has read the others' counts
}

template <int E>
cudaError_t launch_cluster_e(const uint16_t* X, int T, uint32_t* s32, int clear_input, int H, int k, int32_t* idx,
                             int pad_to, int32_t* idx_copy, uint32_t* s_out, int C, int slice,
                             cudaStream_t stream) {
    cudaError_t e = ensure_smem_limit(select_cluster_kernel<E>, kSmemBytes);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(C);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = kSmemBytes;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = C;
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    return cudaLaunchKernelEx(&cfg, select_cluster_kernel<E>, X, T, s32, clear_input, H, k, idx, pad_to, idx_copy,
                              s_out, slice);
}

template <int E>
cudaError_t launch_e(const uint16_t* X, int T, uint32_t* s32, int clear_input, int H, int k, int32_t* idx,
                     int pad_to, int32_t* idx_copy, uint32_t* s_out, cudaStream_t stream) {
    cudaError_t e = ensure_smem_limit(select_kernel<E>, kSmemBytes);
    if (e != cudaSuccess) return e;
    return launch_pdl(select_kernel<E>, dim3(1), dim3(kThreads), kSmemBytes, stream, X, T, s32, clear_input, H, k,
                      idx, pad_to, idx_copy, s_out);
}

}  // namespace

cudaError_t launch_select(const uint16_t* X, int T, uint32_t* s32, int clear_input, int H, int k, int32_t* idx,
                          int pad_to, int32_t* idx_copy, uint32_t* s_out, cudaStream_t stream) {
    if (H < 1 || H > 65535 || k < 1 || k > H) return cudaErrorInvalidValue;
    if (H > kClusterMinH) {
        // a cluster of up to 8 CTAs, at least 2048 slices each
        const int C = min(8, (H + 2047) / 2048);
        const int slice = (H + C - 1) / C;
        if (slice <= 2 * kThreads)
            return launch_cluster_e<2>(X, T, s32, clear_input, H, k, idx, pad_to, idx_copy, s_out, C, slice, stream);
        if (slice <= 4 * kThreads)
            return launch_cluster_e<4>(X, T, s32, clear_input, H, k, idx, pad_to, idx_copy, s_out, C, slice, stream);
        return launch_cluster_e<8>(X, T, s32, clear_input, H, k, idx, pad_to, idx_copy, s_out, C, slice, stream);
    }
    // the fewest keys per thread that cover H
    if (H <= 4 * kThreads) return launch_e<4>(X, T, s32, clear_input, H, k, idx, pad_to, idx_copy, s_out, stream);
    if (H <= 8 * kThreads) return launch_e<8>(X, T, s32, clear_input, H, k, idx, pad_to, idx_copy, s_out, stream);
    if (H <= 16 * kThreads) return launch_e<16>(X, T, s32, clear_input, H, k, idx, pad_to, idx_copy, s_out, stream);
    if (H <= 32 * kThreads) return launch_e<32>(X, T, s32, clear_input, H, k, idx, pad_to, idx_copy, s_out, stream);
    return launch_e<64>(X, T, s32, clear_input, H, k, idx, pad_to, idx_copy, s_out, stream);
}

}  // namespace rmm
