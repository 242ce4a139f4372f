// rmm_attn.cu -- attention with Q K^T reduced along the head dimension.
//
// For each (batch b, KV head g) -- or each query head, on request:
//   s_j   = max over the group's query heads q and all t < T of |Q[b,q,t,j]|
//   S_g   = top-k of s, k = ceil(r*d), ties to the lower index, ascending
//   logit = scale * sum_{j in S_g} Q[b,q,t,j] * Kt[b,g,j,l]
//   O     = softmax_l(logit) . V[b,g,l,:]          (all d dims, fp32 softmax)
// (cf-1.com post on input-adaptive matrix-product reduction, §3.3: reduce
// inside a head rather than dropping heads; paper abstract: attention-side
// products reduced along their contraction dimension.)
//
// The key cache is stored d-major (Kt [B, Hkv, d, ldL]) so a kept head
// dimension is one contiguous row of L keys: the logits pass reads exactly
// k of the d rows, and V is read in full.
//
// Kernels:
//   attn_score_kernel   column max of |Q| over a set's query rows, many CTAs,
//                       atomicMax into a per-set score vector (long chunks)
//   attn_select_kernel  one CTA per kept set: the scores (or, for short
//                       chunks, the column max itself), then an exact
//                       rank-based top-k of the d scores
//   attn_split_kernel   one CTA per (set, split of L, block of query tokens):
//                       logits for a 1024-key sub-block (each thread 4 keys,
//                       8-byte loads of kept K^T rows), online softmax in fp32,
//                       P.V with 16-byte loads of V rows; writes the split's
//                       running max, sum and unnormalised output
//   attn_combine_kernel merges the splits (flash-decoding style) into bf16 O.
// Prefill chunks of 16 or more tokens run on the tensor cores instead
// (rmm_attn_tc.cu); the split pass serves decode.
#include <math.h>

#include "rmm_common.cuh"
#include "rmm_internal.h"

namespace rmm {

namespace {

constexpr int D = 128;        // the head dimension the kernels handle
constexpr int kThreads = 256;
constexpr int SB = 1024;      // keys per sub-block
constexpr int RMAX = 8;       // query rows per CTA (at most)
constexpr int PSTRIDE = D + 2;  // floats per split partial: m, l, O[d]

// ---------------------------------------------------------------- selection

// Column max of |Q| over a set's stacked query rows (its heads x T tokens),
// spread over many CTAs: CTA (set of batch b, chunk of 64 rows); 16-byte loads,
// 16 row lanes x 16 dim chunks; folded into sc[set][d] with atomicMax (sc
// starts at zero: the select kernel clears it after reading).
__global__ void __launch_bounds__(256)
    attn_score_kernel(const uint16_t* __restrict__ Q, int Hq, int Hkv, int T, int per_query_head,
                      uint32_t* __restrict__ sc) {
    __shared__ uint32_t red[16][D];
    const int nsets = per_query_head ? Hq : Hkv;
    const int set = blockIdx.x % nsets;
    const int b = blockIdx.x / nsets;
    const int nq = per_query_head ? 1 : Hq / Hkv;
    const int q_lo = per_query_head ? set : set * nq;
    const int nrows = nq * T;
    const int c16 = threadIdx.x & 15, rl = threadIdx.x >> 4;
    pdl_wait();
    pdl_launch_dependents();
    uint32_t m[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    const int r0 = blockIdx.y * 64;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int r = r0 + rl + 16 * i;
        if (r < nrows) {
            const int q = q_lo + r / T, t = r % T;
            const uint4 v = ld_nc_v4(Q + (((size_t)b * Hq + q) * T + t) * D + c16 * 8);
            const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                m[2 * e] = max(m[2 * e], w[e] & 0x7FFFu);
                m[2 * e + 1] = max(m[2 * e + 1], (w[e] >> 16) & 0x7FFFu);
            }
        }
    }
#pragma unroll
    for (int e = 0; e < 8; ++e) red[rl][c16 * 8 + e] = m[e];
    __syncthreads();
    if (threadIdx.x < D) {
        uint32_t mm = 0;
#pragma unroll
        for (int i = 0; i < 16; ++i) mm = max(mm, red[i][threadIdx.x]);
        if (mm > 0) atomicMax(sc + (size_t)blockIdx.x * D + threadIdx.x, mm);
    }
}

// The kept head dimensions of set (b, set), computed by the CTA's first D
// threads (thread j = dimension j; the others only pass the barriers): the
// scores from sc (cleared after reading) or, with sc null, the column max of
// |Q| over the set's rows, then an exact rank-based top-k under (score desc,
// index asc), written in ascending order to out (shared or global).
__device__ __forceinline__ void select_dims_cta(const uint16_t* __restrict__ Q, int Hq, int Hkv, int T, int k,
                                                int per_query_head, int b, int set, uint32_t* __restrict__ sc,
                                                uint32_t* sv, int* warp_cnt, int32_t* out) {
    const int G = Hq / Hkv;
    const int q_lo = per_query_head ? set : set * G;
    const int nrows = (per_query_head ? 1 : G) * T;
    const int j = threadIdx.x;
    uint32_t m = 0;
    if (j < D) {
        const int nsets = per_query_head ? Hq : Hkv;
        const size_t so = ((size_t)b * nsets + set) * D + j;
        if (sc) {
            m = sc[so];
            sc[so] = 0;
        } else {
#pragma unroll 8
            for (int r = 0; r < nrows; ++r)  // rows q_lo + r / T, token r % T: all loads independent
                m = max(m, (uint32_t)(Q[(((size_t)b * Hq + q_lo + r / T) * T + r % T) * D + j] & 0x7FFF));
        }
        sv[j] = m;
    }
    __syncthreads();
    bool keep = false;
    if (j < D) {
        // rank under (score desc, index asc): number of entries that beat j
        int rank = 0;
#pragma unroll 16
        for (int i = 0; i < D; ++i) {
            const uint32_t v = sv[i];
            rank += (v > m) || (v == m && i < j);
        }
        keep = rank < k;
    }
    const unsigned ball = __ballot_sync(0xffffffffu, keep);
    const int lane = j & 31, w = j >> 5;
    if (j < D && lane == 0) warp_cnt[w] = __popc(ball);
    __syncthreads();
    if (j < D) {
        int pos = __popc(ball & ((1u << lane) - 1u));
        for (int i = 0; i < w; ++i) pos += warp_cnt[i];
        if (keep) out[pos] = j;
    }
}

// One CTA per kept set (long chunks; short decode chunks select inside the
// split pass instead).
__global__ void __launch_bounds__(D)
    attn_select_kernel(const uint16_t* __restrict__ Q, int Hq, int Hkv, int T, int k,
                       int per_query_head, uint32_t* __restrict__ sc, int32_t* __restrict__ idx) {
    __shared__ uint32_t sv[D];
    __shared__ int warp_cnt[D / 32];
    const int nsets = per_query_head ? Hq : Hkv;
    pdl_wait();
    pdl_launch_dependents();
    select_dims_cta(Q, Hq, Hkv, T, k, per_query_head, blockIdx.x / nsets, blockIdx.x % nsets, sc, sv, warp_cnt,
                    idx + (size_t)blockIdx.x * k);
}

// ---------------------------------------------------------------- split pass

// kCtx: the keys are the kept context blocks only.  The split then runs over
// Lv = kc * 2^bc_shift virtual positions: position v is key
// blocks[set][v >> bc_shift] * 2^bc_shift + (v mod 2^bc_shift) of the cache, and
// positions at or past L (the ragged last block) are masked.  Without kCtx,
// Lv = L and position v is key v.
// kRows (4 or 8): query rows per CTA; 4 when a set has at most 4 rows per
// call (decode with up to 4 query heads per KV head), halving the registers.
template <bool kCtx, int kRows>
__global__ void __launch_bounds__(kThreads, kRows == 4 ? 2 : 1)
    attn_split_kernel(const uint16_t* __restrict__ Q, const uint16_t* __restrict__ Kt,
                      const uint16_t* __restrict__ V, int Hq, int Hkv, int T, int L, int ldL, int k,
                      int causal, float scale, int per_query_head, int32_t* __restrict__ idx, int select_here,
                      float* __restrict__ partials, int chunk, int tq, int Lv,
                      const int32_t* __restrict__ blocks, int bc_shift, int kc) {
    __shared__ float qs[kRows][D];      // scaled kept query values
    __shared__ int sidx[D];
    // One buffer, two uses: logits/probabilities of the current sub-block
    // [kRows][SB] inside the key loop, the cross-warp fold of P.V [8][kRows][D]
    // after it (both 32 KB).
    __shared__ float buf[kRows * SB];
    float (*lg)[SB] = reinterpret_cast<float (*)[SB]>(buf);
    float (*red)[kRows][D] = reinterpret_cast<float (*)[kRows][D]>(buf);
    static_assert(8 * kRows * D <= kRows * SB, "fold buffer must fit in the logits buffer");
    __shared__ float m_run[kRows], l_run[kRows], alpha[kRows];

    const int nsets = per_query_head ? Hq : Hkv;
    const int set = blockIdx.x % nsets;
    const int b = blockIdx.x / nsets;
    const int G = Hq / Hkv;
    const int g = per_query_head ? set / G : set;
    const int q_lo = per_query_head ? set : set * G;
    const int nq = per_query_head ? 1 : G;
    const int split = blockIdx.y;
    const int nsplit = gridDim.y;
    const int t0 = blockIdx.z * tq;
    const int l_begin = split * chunk;
    const int l_end = min(Lv, l_begin + chunk);
    const int32_t* __restrict__ set_blocks = kCtx ? blocks + (size_t)blockIdx.x * kc : nullptr;
    const int bc_mask = (1 << bc_shift) - 1;
    // cache position of virtual position v (4-aligned v gives a 4-aligned position)
    auto key_pos = [&](int v) -> int {
        if constexpr (kCtx) return (__ldg(set_blocks + (v >> bc_shift)) << bc_shift) + (v & bc_mask);
        return v;
    };
    const int R = nq * tq;  // rows: r = qi * tq + ti
    const int tid = threadIdx.x;
    pdl_wait();
    pdl_launch_dependents();

    if (select_here) {
        // short decode chunk: every CTA of the set ranks the d dims itself (a
        // few hundred instructions), the first one also writes the kept list
        __shared__ uint32_t sv[D];
        __shared__ int warp_cnt[kThreads / 32];
        select_dims_cta(Q, Hq, Hkv, T, k, per_query_head, b, set, nullptr, sv, warp_cnt, sidx);
        __syncthreads();
        if (split == 0 && blockIdx.z == 0)
            for (int i = tid; i < k; i += kThreads) idx[(size_t)blockIdx.x * k + i] = sidx[i];
    } else {
        for (int i = tid; i < k; i += kThreads) sidx[i] = idx[(size_t)blockIdx.x * k + i];
        __syncthreads();
    }
#pragma unroll
    for (int e = tid; e < kRows * D; e += kThreads) {
        const int r = e / D, jj = e % D;
        float v = 0.0f;
        if (r < R && jj < k) {
            const int qi = r / tq, ti = r % tq, t = t0 + ti;
            if (t < T) v = scale * bf16_bits_to_float(Q[(((size_t)(b * Hq + q_lo + qi)) * T + t) * D + sidx[jj]]);
        }
        qs[r][jj] = v;
    }
    if (tid < kRows) {
        m_run[tid] = -INFINITY;
        l_run[tid] = 0.0f;
    }
    __syncthreads();

    // last key each row may see
    int last[kRows];
#pragma unroll
    for (int r = 0; r < kRows; ++r) {
        const int ti = (r < R) ? r % tq : 0;
        const int t = t0 + ti;
        last[r] = (r < R && t < T) ? (causal ? (L - T + t) : (L - 1)) : -1;
    }

    const uint16_t* kbase = Kt + ((size_t)(b * Hkv + g) * D) * ldL;
    const uint16_t* vbase = V + ((size_t)(b * Hkv + g) * ldL) * D;

    // P.V mapping: 16 column groups of 8 dims x 16 key groups
    const int cgp = tid & 15, kg = tid >> 4;
    float acc[kRows][8];
#pragma unroll
    for (int r = 0; r < kRows; ++r)
#pragma unroll
        for (int c = 0; c < 8; ++c) acc[r][c] = 0.0f;

    for (int l0 = l_begin; l0 < l_end; l0 += SB) {
        // with context blocks, the sub-block's scattered V rows start towards L2
        // now, so that the P.V pass after the logits finds them there: line q of
        // the sub-block (a V row is two 128-byte lines) is requested by thread
        // q mod 256.  (For contiguous keys the same prefetch competes with the
        // K loads on the critical path and measured slower: not done.)
        if constexpr (kCtx) {
            const int nk = min(SB, l_end - l0);
            for (int q = tid; q < 2 * nk; q += kThreads) {
                const int lv = key_pos(l0 + (q >> 1));
                if (lv < L) prefetch_l2(vbase + (size_t)lv * D + (q & 1) * 64);
            }
        }
        // ---- logits: thread owns keys l0 + 4*tid .. +3
        const int l = l0 + tid * 4;
        const int lp = l < l_end ? key_pos(l) : L;  // cache position of the thread's first key
        float s4[kRows][4];
#pragma unroll
        for (int r = 0; r < kRows; ++r)
#pragma unroll
            for (int c = 0; c < 4; ++c) s4[r][c] = 0.0f;
        if (lp < L) {  // lp + 3 < roundup(L, 4) <= ldL: the 8-byte load stays in the row
            // kUnrollK kept rows per step: their loads are all in flight before the FMAs
            constexpr int kUnrollK = 8;
            for (int jj0 = 0; jj0 < k; jj0 += kUnrollK) {
                uint2 kv[kUnrollK];
#pragma unroll
                for (int u = 0; u < kUnrollK; ++u)
                    kv[u] = jj0 + u < k ? ld_nc_v2(kbase + (size_t)sidx[jj0 + u] * ldL + lp) : make_uint2(0u, 0u);
#pragma unroll
                for (int u = 0; u < kUnrollK; ++u) {
                    const float k0 = __uint_as_float(kv[u].x << 16), k1 = __uint_as_float(kv[u].x & 0xFFFF0000u);
                    const float k2 = __uint_as_float(kv[u].y << 16), k3 = __uint_as_float(kv[u].y & 0xFFFF0000u);
#pragma unroll
                    for (int r = 0; r < kRows; ++r) {
                        const float qv = qs[r][jj0 + u];  // zero past k
                        s4[r][0] = fmaf(qv, k0, s4[r][0]);
                        s4[r][1] = fmaf(qv, k1, s4[r][1]);
                        s4[r][2] = fmaf(qv, k2, s4[r][2]);
                        s4[r][3] = fmaf(qv, k3, s4[r][3]);
                    }
                }
            }
        }
#pragma unroll
        for (int r = 0; r < kRows; ++r)
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                const int lc = lp + c;
                lg[r][tid * 4 + c] = (l + c < l_end && lc < L && lc <= last[r]) ? s4[r][c] : -INFINITY;
            }
        __syncthreads();

        // ---- online softmax, one warp per row
        const int warp = tid >> 5, lane = tid & 31;
        for (int r = warp; r < kRows; r += kThreads / 32) {
            float mx = -INFINITY;
            for (int i = lane; i < SB; i += 32) mx = fmaxf(mx, lg[r][i]);
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
            const float m_old = m_run[r];
            const float m_new = fmaxf(m_old, mx);
            float sum = 0.0f;
            if (m_new == -INFINITY) {
                for (int i = lane; i < SB; i += 32) lg[r][i] = 0.0f;
            } else {
                for (int i = lane; i < SB; i += 32) {
                    const float p = __expf(lg[r][i] - m_new);
                    lg[r][i] = p;
                    sum += p;
                }
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
            if (lane == 0) {
                const float a = (m_old == -INFINITY) ? 0.0f : __expf(m_old - m_new);
                alpha[r] = (m_new == -INFINITY) ? 1.0f : a;
                l_run[r] = l_run[r] * alpha[r] + sum;
                m_run[r] = m_new;
            }
        }
        __syncthreads();

        // ---- P.V
#pragma unroll
        for (int r = 0; r < kRows; ++r) {
            const float a = alpha[r];
#pragma unroll
            for (int c = 0; c < 8; ++c) acc[r][c] *= a;
        }
        const int nkeys = min(SB, l_end - l0);
        // kUnrollV V rows per step, their loads in flight together
        constexpr int kUnrollV = kRows == 4 ? 8 : 4;
        for (int i0 = kg; i0 < nkeys; i0 += 16 * kUnrollV) {
            uint4 v[kUnrollV];
#pragma unroll
            for (int u = 0; u < kUnrollV; ++u) {
                const int i = i0 + 16 * u;
                const int lv = i < nkeys ? key_pos(l0 + i) : L;
                // a masked key (probability 0) past the cache's end is not loaded
                v[u] = lv < L ? ld_nc_v4(vbase + (size_t)lv * D + cgp * 8) : make_uint4(0u, 0u, 0u, 0u);
            }
#pragma unroll
            for (int u = 0; u < kUnrollV; ++u) {
                const int i = i0 + 16 * u;
                if (i >= nkeys) break;
                float vf[8];
                vf[0] = __uint_as_float(v[u].x << 16); vf[1] = __uint_as_float(v[u].x & 0xFFFF0000u);
                vf[2] = __uint_as_float(v[u].y << 16); vf[3] = __uint_as_float(v[u].y & 0xFFFF0000u);
                vf[4] = __uint_as_float(v[u].z << 16); vf[5] = __uint_as_float(v[u].z & 0xFFFF0000u);
                vf[6] = __uint_as_float(v[u].w << 16); vf[7] = __uint_as_float(v[u].w & 0xFFFF0000u);
#pragma unroll
                for (int r = 0; r < kRows; ++r) {
                    const float p = lg[r][i];
#pragma unroll
                    for (int c = 0; c < 8; ++c) acc[r][c] = fmaf(p, vf[c], acc[r][c]);
                }
            }
        }
        __syncthreads();  // lg is rewritten by the next sub-block
    }

    // fold the 16 key groups: pairs within a warp by shuffle, then 8 warps via smem
#pragma unroll
    for (int r = 0; r < kRows; ++r)
#pragma unroll
        for (int c = 0; c < 8; ++c) acc[r][c] += __shfl_xor_sync(0xffffffffu, acc[r][c], 16);
    const int warp = tid >> 5, lane = tid & 31;
    if (lane < 16) {
#pragma unroll
        for (int r = 0; r < kRows; ++r)
#pragma unroll
            for (int c = 0; c < 8; ++c) red[warp][r][cgp * 8 + c] = acc[r][c];
    }
    __syncthreads();
    for (int e = tid; e < R * D; e += kThreads) {
        const int r = e / D, c = e % D;
        const int qi = r / tq, ti = r % tq, t = t0 + ti;
        if (t >= T) continue;
        float o = 0.0f;
#pragma unroll
        for (int w = 0; w < 8; ++w) o += red[w][r][c];
        const size_t row = ((size_t)(b * Hq + q_lo + qi)) * T + t;
        float* dst = partials + (row * nsplit + split) * PSTRIDE;
        dst[2 + c] = o;
        if (c == 0) {
            dst[0] = m_run[r];
            dst[1] = l_run[r];
        }
    }
}

// ---------------------------------------------------------------- combine

constexpr int kMaxSplits = 1024;
constexpr int kCombineGroups = 4;  // split groups per row, D threads each

// One CTA per output row: the splits' maxima and sums are read once into
// shared memory (all loads in flight together); then thread (group g, column
// c) adds the weighted column c of the splits s = g (mod 4), eight loads in
// flight, and the four groups are added in a fixed order.
__global__ void __launch_bounds__(kCombineGroups * D)
    attn_combine_kernel(const float* __restrict__ partials, int nsplit, uint16_t* __restrict__ O) {
    __shared__ float sm[kMaxSplits], sl[kMaxSplits];
    __shared__ float red[kCombineGroups * D / 32];
    __shared__ float part_num[kCombineGroups][D], part_den[kCombineGroups][D];
    pdl_wait();
    pdl_launch_dependents();
    const size_t row = blockIdx.x;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int c = tid % D, grp = tid / D;
    const float* p = partials + row * nsplit * PSTRIDE;
    float mx = -INFINITY;
    for (int s = tid; s < nsplit; s += kCombineGroups * D) {
        const float2 ml = *reinterpret_cast<const float2*>(p + (size_t)s * PSTRIDE);
        sm[s] = ml.x;
        sl[s] = ml.y;
        mx = fmaxf(mx, ml.x);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    if (lane == 0) red[warp] = mx;
    __syncthreads();
    float M = red[0];
#pragma unroll
    for (int w = 1; w < kCombineGroups * D / 32; ++w) M = fmaxf(M, red[w]);
    // weights: exp(m_s - M), zero for a split that saw no key
    for (int s = tid; s < nsplit; s += kCombineGroups * D)
        sm[s] = (sm[s] == -INFINITY) ? 0.0f : __expf(sm[s] - M);
    __syncthreads();
    float num = 0.0f, den = 0.0f;
#pragma unroll 8
    for (int s = grp; s < nsplit; s += kCombineGroups) {
        const float w = sm[s];
        den = fmaf(w, sl[s], den);
        num = fmaf(w, p[(size_t)s * PSTRIDE + 2 + c], num);
    }
    part_num[grp][c] = num;
    part_den[grp][c] = den;
    __syncthreads();
    if (grp == 0) {
        float n = part_num[0][c], d = part_den[0][c];
#pragma unroll
        for (int g = 1; g < kCombineGroups; ++g) {
            n += part_num[g][c];
            d += part_den[g][c];
        }
        // a row that saw no key (only with kept context blocks) is zero
        O[row * D + c] = float_to_bf16_bits(d > 0.0f ? n / d : 0.0f);
    }
}

}  // namespace

AttnPlan attn_plan(int B, int Hq, int Hkv, int T, int L, int per_query_head, int num_sms) {
    AttnPlan p;
    p.nsets = per_query_head ? Hq : Hkv;
    const int nq = per_query_head ? 1 : Hq / Hkv;
    p.rows = (nq <= 4 && nq * T <= 4) ? 4 : RMAX;
    p.tq = p.rows / nq;
    if (p.tq < 1) p.tq = 1;
    if (p.tq > T) p.tq = T;
    const long long base = (long long)B * p.nsets * ((T + p.tq - 1) / p.tq);
    const long long target = 2LL * num_sms;
    long long ns = (target + base - 1) / base;
    if (ns < 1) ns = 1;
    int chunk = (int)((L + ns - 1) / ns);
    if (chunk < 256) chunk = 256;
    chunk = (chunk + 3) & ~3;
    p.chunk = chunk;
    p.nsplit = (L + chunk - 1) / chunk;
    return p;
}

size_t attn_partials_bytes(const AttnPlan& p, int B, int Hq, int T) {
    return (size_t)B * Hq * T * p.nsplit * PSTRIDE * sizeof(float);
}

bool attn_dims_in_split(int Hq, int Hkv, int T, int per_query_head) {
    const int nq = per_query_head ? 1 : Hq / Hkv;
    return nq * T < 64;
}

cudaError_t launch_attn_dims(const uint16_t* Q, int B, int Hq, int Hkv, int T, int k, int per_query_head, int nsets,
                             int32_t* idx, uint32_t* sc, cudaStream_t stream) {
    // the kept sets: the column max over many CTAs when the chunk is long
    const int nq = per_query_head ? 1 : Hq / Hkv;
    cudaError_t e;
    const bool wide = !attn_dims_in_split(Hq, Hkv, T, per_query_head);
    if (wide) {
        e = launch_pdl(attn_score_kernel, dim3(B * nsets, (nq * T + 63) / 64), dim3(256), 0, stream, Q, Hq, Hkv, T,
                       per_query_head, sc);
        if (e != cudaSuccess) return e;
    }
    return launch_pdl(attn_select_kernel, dim3(B * nsets), dim3(D), 0, stream, Q, Hq, Hkv, T, k, per_query_head,
                      wide ? sc : (uint32_t*)nullptr, idx);
}

cudaError_t launch_attn_split_ctx(const uint16_t* Q, const uint16_t* Kt, const uint16_t* V, int B, int Hq, int Hkv,
                                  int T, int L, int ldL, int k, int causal, float scale, int per_query_head,
                                  uint16_t* O, int32_t* idx, int select_here, const int32_t* blocks, int bc_shift,
                                  int kc, float* partials, const AttnPlan& p, cudaStream_t stream) {
    const int nq = per_query_head ? 1 : Hq / Hkv;
    if (nq > RMAX || p.nsplit > kMaxSplits) return cudaErrorInvalidValue;
    dim3 grid(B * p.nsets, p.nsplit, (T + p.tq - 1) / p.tq);
    cudaError_t e = launch_pdl(p.rows == 4 ? attn_split_kernel<true, 4> : attn_split_kernel<true, RMAX>, grid,
                               dim3(kThreads), 0, stream, Q, Kt, V, Hq, Hkv, T, L, ldL, k, causal, scale,
                               per_query_head, idx, select_here, partials, p.chunk, p.tq, kc << bc_shift, blocks,
                               bc_shift, kc);
    if (e != cudaSuccess) return e;
    return launch_pdl(attn_combine_kernel, dim3(B * Hq * T), dim3(kCombineGroups * D), 0, stream, (const float*)partials, p.nsplit,
                      O);
}

cudaError_t launch_attn(const uint16_t* Q, const uint16_t* Kt, const uint16_t* V, int B, int Hq,
                        int Hkv, int T, int L, int ldL, int k, int causal, float scale,
                        int per_query_head, uint16_t* O, int32_t* idx, float* partials, uint32_t* sc,
                        int* status, int path, const AttnPlan& p, cudaStream_t stream) {
    const int nq = per_query_head ? 1 : Hq / Hkv;
    const bool tc = path == 2 || (path == 0 && attn_tc_supported(T, k));
    // short decode chunks select their dims inside the split pass
    const bool select_here = !tc && attn_dims_in_split(Hq, Hkv, T, per_query_head);
    cudaError_t e = cudaSuccess;
    if (!select_here) e = launch_attn_dims(Q, B, Hq, Hkv, T, k, per_query_head, p.nsets, idx, sc, stream);
    if (e != cudaSuccess) return e;
    if (tc)
        return launch_attn_tc(Q, Kt, V, B, Hq, Hkv, T, L, ldL, k, causal, scale, per_query_head, idx, O, status,
                              stream);
    if (nq > RMAX || p.nsplit > kMaxSplits) return cudaErrorInvalidValue;
    dim3 grid(B * p.nsets, p.nsplit, (T + p.tq - 1) / p.tq);
    e = launch_pdl(p.rows == 4 ? attn_split_kernel<false, 4> : attn_split_kernel<false, RMAX>, grid, dim3(kThreads), 0,
                   stream, Q, Kt, V, Hq, Hkv, T, L, ldL, k, causal, scale, per_query_head, idx, (int)select_here,
                   partials, p.chunk, p.tq, L, (const int32_t*)nullptr, 0, 0);
    if (e != cudaSuccess) return e;
    return launch_pdl(attn_combine_kernel, dim3(B * Hq * T), dim3(kCombineGroups * D), 0, stream, (const float*)partials, p.nsplit,
                      O);
}

}  // namespace rmm
