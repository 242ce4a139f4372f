// rmm_attn_tc.cu -- the prefill chunk of the reduced attention on the tensor
// cores (tcgen05, accumulators in TMEM).
//
// For one (batch b, query head h) and 128 query rows t0 .. t0+127, with the
// head's kept set S (k of the d = 128 head dims, padded to kp = roundup(k, 16)
// with dims whose query values are zero):
//   S_j = Q[:, S] K_j[:, S]^T    over key blocks j of 128 keys   (M=128, N=128, K=kp)
//   O  += P_j V_j                P_j = exp(S_j - m) in bf16      (M=128, N=128, K=128)
// with a causal mask (query t sits at key position L - T + t) and an fp32
// online softmax.  The reduction along the head dimension and the full
// softmax.V follow the cf-1.com post on input-adaptive matrix-product
// reduction, §3.3 (reduce inside a head) and the paper abstract (attention
// products reduced along their contraction dimension).
//
// Operands in shared memory, 128-byte swizzled: the gathered query tile and
// the key block are MN-major (a kept dim is one row of 128 tokens / keys --
// the d-major key cache makes each kept dim of a key block one contiguous
// 256-byte segment); V blocks are MN-major (a key is one row of d values).
// TMEM holds two S buffers (columns 0-127, 128-255), O (256-383), P
// (384-447) and the softmax warps' row exchange (448-453).  The softmax
// threads write P_j there, two bf16 keys per 32-bit column, each thread its
// own row, and the P.V product reads it as its A operand straight from tensor
// memory (K-major by definition), so P never passes through shared memory.
//
// Warp roles (384 threads):
//   0-7  softmax: warps q and q+4 own query rows 32q .. 32q+31 (their TMEM
//        lanes), one row per thread, and split the 128 columns; reads S_j,
//        masks, keeps a running reference max m and sum l; P_j to TMEM.
//        O is rescaled in TMEM only when a row's block max exceeds m
//        by more than 2^8 (the reference max is then raised), so P stays below
//        256 and most blocks need no rescale.  At the end O / l goes to HBM.
//   8    MMA: one thread keeps two S blocks ahead of the softmax and issues
//        P_j V_j as soon as P_j is written; tcgen05.commit releases buffers.
//   9-11 producers: the query tile once (kept dims gathered), then per key
//        block the kp kept rows of K^T with 16-byte cp.async (zero-filled past
//        the valid keys) and the 128 x 128 V tile with two TMA tile loads
//        (a 3-D map over [head][key][dim]: keys past L read as zero), three
//        stages.
// Every wait is bounded: on expiry the kernel records RMM_ERR_TIMEOUT, every
// role leaves its loop, in-flight tensor-core work drains, TMEM is freed.
#include <math.h>

#include "rmm_common.cuh"
#include "rmm_internal.h"

namespace rmm {

namespace {

constexpr int D = 128;
constexpr int BQ = 128;   // query rows per CTA (= TMEM lanes)
constexpr int BKV = 128;  // keys per block
constexpr int KV_STAGES_MAX = 3;  // key/value stages (231 KB of shared memory at kp = 128)
constexpr int kSoftmaxWarps = 8;  // two per TMEM lane quarter, each on 64 of the 128 columns
constexpr int kSoftmaxThreads = 32 * kSoftmaxWarps;
constexpr int kMmaWarp = kSoftmaxWarps;
constexpr int kProdWarps = 3;
constexpr int kProdThreads = 32 * kProdWarps;
constexpr int kThreadsTc = 32 * (kSoftmaxWarps + 1 + kProdWarps);  // 12 warps: three per SM sub-partition
constexpr int V_CHUNK = BKV * 128;     // 64 dims x 128 key rows (bytes)
constexpr int V_BYTES = 2 * V_CHUNK;   // 32 KB
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t TM_S0 = 0, TM_O = 256, TM_P = 384;  // P: 128 keys as 64 packed columns
// The two softmax warps of a lane quarter exchange row values through TMEM
// columns TM_X .. TM_X+5: block maxima [block parity][half], then row sums [half].
constexpr uint32_t TM_X = 448;
constexpr float kRescaleLog2 = 8.0f;   // rescale O when a block max exceeds the reference by 2^8

struct __align__(8) Bars {
    uint64_t q_full;
    uint64_t kv_full[KV_STAGES_MAX];
    uint64_t kv_empty[KV_STAGES_MAX];
    uint64_t s_full[2];
    uint64_t s_empty[2];
    uint64_t p_full;
    uint64_t p_empty;
    uint64_t o_full;
    uint64_t drain;
    uint64_t pair[4];  // per TMEM lane quarter: the two softmax warps on those rows meet here
    uint32_t tmem_base;
    int abort_flag;
};

// 2^x with the hardware approximation (ex2.approx.ftz: ~2 ulp; -inf gives 0);
// P is rounded to bf16 right after, so its error is far below that rounding.
__device__ __forceinline__ float fast_exp2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// 2^x on the FMA pipe, for x <= 8 (P's range): round-to-nearest range
// reduction x = n + f, |f| <= 1/2, by adding 1.5 * 2^23 (the integer n lands
// in the low mantissa bits); 2^f = e^(f ln 2) by its Taylor expansion to
// degree 4 (remainder < 6e-5 relative for |f ln 2| <= 0.35, well below the
// bf16 rounding of P); n is added to the exponent bits.  x below -126 is
// clamped (2^-126 is zero for P's purposes).  Half of each row's
// exponentials run here instead of on the special-function unit, whose
// throughput otherwise bounds the softmax.
__device__ __forceinline__ float poly_exp2(float x) {
    x = fmaxf(x, -126.0f);
    const float t = x + 12582912.0f;
    const float f = x - (t - 12582912.0f);
    float p = fmaf(f, 0.0096181291076285f, 0.0555041086648216f);
    p = fmaf(p, f, 0.2402265069591007f);
    p = fmaf(p, f, 0.6931471805599453f);
    p = fmaf(p, f, 1.0f);
    const int n = __float_as_int(t) - 0x4B400000;
    return __int_as_float(__float_as_int(p) + (n << 23));
}

// Byte offset of 16-byte chunk c16 (along M/N) of row j (along K) in the
// 128-byte-swizzled MN-major layout whose 64-element groups are `chunk` apart.
__device__ __forceinline__ uint32_t swz(int j, int c16, int chunk) {
    return (uint32_t)((c16 >> 3) * chunk + j * 128 + (((c16 & 7) ^ (j & 7)) << 4));
}

// Softmax pass 1 for one row and 64 columns (col0 .. col0+63) of a key block:
// the max of the raw logits (scale > 0) in 8 independent chains.  kMask: keys
// past the cache end or (causal) past the row's position count as -inf.
template <bool kMask>
__device__ __forceinline__ float row_max64(uint32_t scol, int key0, int L, int causal, int pos) {
    uint32_t r[2][32];
    tmem_ld_32x32b_x32(scol, r[0]);
    tmem_ld_32x32b_x32(scol + 32, r[1]);
    tmem_ld_wait();
    float mx[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) mx[e] = -INFINITY;
#pragma unroll
    for (int q = 0; q < 2; ++q)
#pragma unroll
        for (int c = 0; c < 32; ++c) {
            float x = __uint_as_float(r[q][c]);
            if (kMask) {
                const int key = key0 + q * 32 + c;
                if (!(key < L && (!causal || key <= pos))) x = -INFINITY;
            }
            mx[c & 7] = fmaxf(mx[c & 7], x);
        }
    return fmaxf(fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])), fmaxf(fmaxf(mx[4], mx[5]), fmaxf(mx[6], mx[7])));
}

// Softmax pass 2 for the same 64 columns: p = 2^(s * scale_log2 - m) (one FMA
// and an exponential, half of them on the FMA pipe; masked logits give 0),
// their sum, and P (bf16) into the 32 TMEM columns at pcol of the row's lane
// (column c holds keys 2c and 2c+1 of the 64), written 32 keys at a time.
template <bool kMask>
__device__ __forceinline__ float row_exp64(uint32_t scol, int key0, int L, int causal, int pos, float scale_log2,
                                           float neg_m, uint32_t pcol) {
    uint32_t r[2][32];
    tmem_ld_32x32b_x32(scol, r[0]);
    tmem_ld_32x32b_x32(scol + 32, r[1]);
    tmem_ld_wait();
    float sm[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    uint32_t pk[2][16];
#pragma unroll
    for (int c8 = 0; c8 < 8; ++c8) {
        float p[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            const int c = c8 * 8 + e;
            const float x = fmaf(__uint_as_float(r[c >> 5][c & 31]), scale_log2, neg_m);
            float v = (e & 1) ? poly_exp2(x) : fast_exp2(x);
            if (kMask) {
                const int key = key0 + c;
                if (!(key < L && (!causal || key <= pos))) v = 0.0f;
            }
            p[e] = v;
            sm[e] += v;
        }
        pk[c8 >> 2][(c8 & 3) * 4 + 0] = pack_bf16x2(p[0], p[1]);
        pk[c8 >> 2][(c8 & 3) * 4 + 1] = pack_bf16x2(p[2], p[3]);
        pk[c8 >> 2][(c8 & 3) * 4 + 2] = pack_bf16x2(p[4], p[5]);
        pk[c8 >> 2][(c8 & 3) * 4 + 3] = pack_bf16x2(p[6], p[7]);
        if ((c8 & 3) == 3) tmem_st_32x32b_x16(pcol + (c8 >> 2) * 16, pk[c8 >> 2]);
    }
    tmem_st_wait();
    return ((sm[0] + sm[1]) + (sm[2] + sm[3])) + ((sm[4] + sm[5]) + (sm[6] + sm[7]));
}

__global__ void __launch_bounds__(kThreadsTc, 1)
    attn_tc_kernel(const uint16_t* __restrict__ Q, const uint16_t* __restrict__ Kt,
                   const __grid_constant__ CUtensorMap vmap, int Hq, int Hkv, int T, int L, int ldL, int k, int kp,
                   int causal, float scale_log2, int per_query_head, const int32_t* __restrict__ idx,
                   uint16_t* __restrict__ O, int* status) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~static_cast<uintptr_t>(1023));
    const int QK_BYTES = kp * 256;  // a gathered query tile or key block
    const int ks = KV_STAGES_MAX;   // key/value stages
    uint8_t* sV = smem;                                   // ks x 32 KB (1024-aligned)
    uint8_t* sQ = sV + ks * V_BYTES;                      // kp x 256
    uint8_t* sK = sQ + QK_BYTES;                          // ks x kp x 256
    int* sidx = reinterpret_cast<int*>(sK + ks * QK_BYTES);  // kp kept dims
    Bars* bars = reinterpret_cast<Bars*>(sidx + D);
    volatile int* abort_flag = &bars->abort_flag;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int n_tiles = (T + BQ - 1) / BQ;
    // heads vary fastest in launch order, so the longest (latest) tiles of every
    // head are launched before any shorter tile: a short tail
    const int tile = n_tiles - 1 - (int)blockIdx.y;
    const int h = blockIdx.x, b = blockIdx.z;
    const int G = Hq / Hkv;
    const int g = h / G;
    const int nsets = per_query_head ? Hq : Hkv;
    const int set = per_query_head ? h : g;
    const int t0 = tile * BQ;
    // key blocks this tile needs
    int last_key = L - 1;
    if (causal) last_key = min(last_key, L - T + min(t0 + BQ - 1, T - 1));
    const int nkb = last_key / BKV + 1;

    if (tid == 0) {
        mbar_init(smem_addr(&bars->q_full), kProdThreads);
        for (int s = 0; s < ks; ++s) {
            // the producers' cp.async arrivals + one arrival that expects the V tile's bytes
            mbar_init(smem_addr(&bars->kv_full[s]), kProdThreads + 1);
            mbar_init(smem_addr(&bars->kv_empty[s]), 1);
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(smem_addr(&bars->s_full[s]), 1);
            mbar_init(smem_addr(&bars->s_empty[s]), kSoftmaxThreads);
        }
        mbar_init(smem_addr(&bars->p_full), kSoftmaxThreads);
        mbar_init(smem_addr(&bars->p_empty), 1);
        mbar_init(smem_addr(&bars->o_full), 1);
        mbar_init(smem_addr(&bars->drain), 1);
        for (int q = 0; q < 4; ++q) mbar_init(smem_addr(&bars->pair[q]), 64);
        bars->abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == kMmaWarp) {
        tmem_alloc(smem_addr(&bars->tmem_base), TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = bars->tmem_base;
    if (tid == 32 * (kMmaWarp + 1)) tma_prefetch_desc(&vmap);
    pdl_wait();  // Q, the caches and the kept sets come from the preceding kernels
    pdl_launch_dependents();

    if (warp > kMmaWarp) {
        // ------------------------------------------------------------ producers
        const int pt = tid - 32 * (kMmaWarp + 1);
        const int32_t* S = idx + ((size_t)b * nsets + set) * k;
        for (int j = pt; j < kp; j += kProdThreads) sidx[j] = j < k ? __ldg(S + j) : -1;
        asm volatile("bar.sync 1, %0;" ::"r"(kProdThreads));
        // the query tile: 128 tokens x 128 dims staged row-major in the (not yet
        // used) first V stage with coalesced 16-byte copies, then the kp kept
        // dims gathered from there into the MN-major operand, 8 tokens per chunk
        const uint16_t* Qh = Q + ((size_t)b * Hq + h) * T * D;
        const uint32_t qstage = smem_addr(sV);
        for (int it = pt; it < BQ * 16; it += kProdThreads) {
            const int tr = it >> 4, c16 = it & 15;
            const bool ok = t0 + tr < T;
            cp_async_16(qstage + tr * 256 + c16 * 16, ok ? Qh + (size_t)(t0 + tr) * D + c16 * 8 : Qh, ok ? 16u : 0u);
        }
        cp_async_wait_all();
        asm volatile("bar.sync 1, %0;" ::"r"(kProdThreads));
        const uint16_t* qs = reinterpret_cast<const uint16_t*>(sV);
        for (int it = pt; it < kp * 16; it += kProdThreads) {
            // consecutive lanes take consecutive kept dims of one 8-token chunk:
            // their reads fall in different banks (lanes on one dim and different
            // chunks would all hit one bank: the staged rows are 256 B apart)
            const int jr = it % kp, c16 = it / kp;
            const int dim = sidx[jr];
            uint16_t v[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) v[e] = dim >= 0 ? qs[(c16 * 8 + e) * D + dim] : (uint16_t)0;
            const uint4 w = make_uint4(v[0] | ((uint32_t)v[1] << 16), v[2] | ((uint32_t)v[3] << 16),
                                       v[4] | ((uint32_t)v[5] << 16), v[6] | ((uint32_t)v[7] << 16));
            st_shared_v4(smem_addr(sQ) + swz(jr, c16, kp * 128), w);
        }
        fence_proxy_async_smem();
        asm volatile("bar.sync 1, %0;" ::"r"(kProdThreads));  // staging read before V lands there
        mbar_arrive(smem_addr(&bars->q_full));
        const uint16_t* Kg = Kt + ((size_t)b * Hkv + g) * D * ldL;
        const int vplane = b * Hkv + g;
        int issued = 0;  // key blocks whose loads were issued
        for (int j = 0; j < nkb; ++j) {
            const int s = j % ks;
            const uint32_t ph = (uint32_t)(j / ks) & 1u;
            if (!mbar_wait(smem_addr(&bars->kv_empty[s]), ph ^ 1u, status, abort_flag)) break;
            const int kb0 = j * BKV;
            const uint32_t full = smem_addr(&bars->kv_full[s]);
            if (pt == 0) {
                // V: two 64-dim x 128-key boxes, the swizzled layout the P.V MMA reads
                // (keys past L are outside the map and read as zero; P is 0 there)
                mbar_arrive_expect_tx(full, V_BYTES);
                const uint32_t vst = smem_addr(sV + s * V_BYTES);
                tma_load_3d(vst, &vmap, full, 0, kb0, vplane);
                tma_load_3d(vst + V_CHUNK, &vmap, full, 64, kb0, vplane);
            }
            const uint32_t kst = smem_addr(sK + s * QK_BYTES);
            for (int it = pt; it < kp * 16; it += kProdThreads) {
                const int jr = it >> 4, c16 = it & 15;
                const int key = kb0 + c16 * 8;
                const int dim = sidx[jr];
                const bool ok = dim >= 0 && key < ldL;
                cp_async_16(kst + swz(jr, c16, kp * 128), ok ? Kg + (size_t)dim * ldL + key : Kg, ok ? 16u : 0u);
            }
            cp_async_arrive_noinc(full);
            issued = j + 1;
        }
        cp_async_wait_all();
        // no V tile may still be landing in shared memory when the CTA leaves
        // (after an abort; otherwise every issued block was consumed): wait,
        // bounded, for the last phase of each stage that was issued
        if (pt == 0) {
            volatile int no_abort = 0;
            for (int j = max(0, issued - ks); j < issued; ++j)
                mbar_wait(smem_addr(&bars->kv_full[j % ks]), (uint32_t)(j / ks) & 1u, status, &no_abort);
        }
    } else if (warp == kMmaWarp) {
        // ------------------------------------------------------------ MMA issuer
        bool ok = __all_sync(0xffffffffu, mbar_wait(smem_addr(&bars->q_full), 0, status, abort_flag));
        const uint32_t idesc_s = idesc_bf16_f32(BQ, BKV, 1, 1);  // Q_S and K_S both MN-major
        const uint32_t idesc_pv = idesc_bf16_f32(BQ, D, 0, 1);   // P K-major, V MN-major
        const uint32_t qbase = smem_addr(sQ);
        fence_proxy_async_smem();
        tc_fence_after();
        // S_j into TMEM buffer j & 1, once block j has landed and the softmax has
        // read S_{j-2} from that buffer
        auto issue_s = [&](int j) -> bool {
            const int s = j % ks, sb = j & 1;
            bool got = mbar_wait(smem_addr(&bars->kv_full[s]), (uint32_t)(j / ks) & 1u, status, abort_flag);
            got = got && mbar_wait(smem_addr(&bars->s_empty[sb]), ((uint32_t)(j >> 1) & 1u) ^ 1u, status, abort_flag);
            if (!__all_sync(0xffffffffu, got)) return false;  // the warp leaves together
            fence_proxy_async_smem();  // the producers' cp.async data, read by the tensor cores
            tc_fence_after();
            if (lane == 0) {
                const uint32_t kbase = smem_addr(sK + s * QK_BYTES);
                for (int kk = 0; kk < kp / 16; ++kk)
                    umma_f16(tmem + TM_S0 + sb * BKV, smem_desc_sw128(qbase + kk * 2048, kp * 128, 1024),
                             smem_desc_sw128(kbase + kk * 2048, kp * 128, 1024), idesc_s, kk > 0 ? 1u : 0u);
                umma_commit(smem_addr(&bars->s_full[sb]));
            }
            __syncwarp();
            return true;
        };
        // two S blocks ahead; then, per block, P_j V_j as soon as P_j is written and
        // S_{j+2} after it, so a late key block never holds back a ready P.V
        if (ok && nkb > 0) ok = issue_s(0);
        if (ok && nkb > 1) ok = issue_s(1);
        for (int j = 0; ok && j < nkb; ++j) {
            const int sp = j % ks;
            if (!__all_sync(0xffffffffu, mbar_wait(smem_addr(&bars->p_full), (uint32_t)j & 1u, status, abort_flag))) {
                ok = false;
                break;
            }
            tc_fence_after();
            if (lane == 0) {
                const uint32_t vbase = smem_addr(sV + sp * V_BYTES);
#pragma unroll
                for (int kk = 0; kk < BKV / 16; ++kk)
                    umma_f16_tmem_a(tmem + TM_O, tmem + TM_P + kk * 8, smem_desc_sw128(vbase + kk * 2048, V_CHUNK, 1024),
                                    idesc_pv, (j > 0 || kk > 0) ? 1u : 0u);
                umma_commit(smem_addr(&bars->p_empty));
                umma_commit(smem_addr(&bars->kv_empty[sp]));
            }
            __syncwarp();
            if (j + 2 < nkb) ok = issue_s(j + 2);
        }
        if (lane == 0) {
            if (ok) umma_commit(smem_addr(&bars->o_full));
            umma_commit(smem_addr(&bars->drain));  // everything issued so far has completed
        }
        __syncwarp();
        // wait for the issued MMAs even after an abort (they finish on their own) so
        // that TMEM is never freed under them; only the time limit ends this wait
        volatile int no_abort = 0;
        mbar_wait(smem_addr(&bars->drain), 0, status, &no_abort, kWaitLimitNs);
    } else {
        // ------------------------------------------------------------ softmax + epilogue
        // warps q and q + 4 share TMEM lanes 32q .. 32q+31 (query rows) and take
        // columns 0-63 and 64-127 of S, of P (one atom each) and of O; the row max
        // is combined through TMEM (columns TM_X..) with one barrier per pair and block,
        // the row sums are kept per half and added at the end
        const int quarter = warp & 3, half = warp >> 2;
        const int i = quarter * 32 + lane;  // query row inside the tile = TMEM lane
        const int t = t0 + i;
        const int pos = L - T + t;
        const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
        const uint32_t pair_mb = smem_addr(&bars->pair[quarter]);  // the two warps on these rows
        int pair_phase = 0;
        float m_use = -INFINITY, l_half = 0.0f;
        bool ok = true;
        for (int j = 0; j < nkb; ++j) {
            const int sb = j & 1;
            // waits and branches around tcgen05.ld/st (.sync.aligned: the whole warp,
            // converged) are decided warp-wide
            if (!__all_sync(0xffffffffu,
                            mbar_wait(smem_addr(&bars->s_full[sb]), (uint32_t)(j >> 1) & 1u, status, abort_flag))) {
                ok = false;
                break;
            }
            tc_fence_after();
            const int key0 = j * BKV + half * 64;
            // mask only where the warp's rows cross the diagonal or the cache end
            const bool full = __all_sync(0xffffffffu, key0 + 63 < L && (!causal || key0 + 63 <= pos));
            const uint32_t scol = tmem + lane_base + TM_S0 + sb * BKV + half * 64;
            const float m_mine = full ? row_max64<false>(scol, key0, L, causal, pos)
                                      : row_max64<true>(scol, key0, L, causal, pos);
            tmem_st_32x32b_x1(tmem + lane_base + TM_X + (j & 1) * 2 + half, __float_as_uint(m_mine));
            tmem_st_wait();
            tc_fence_before();
            // meet the partner warp (bounded, like every wait here)
            mbar_arrive(pair_mb);
            if (!__all_sync(0xffffffffu, mbar_wait(pair_mb, (uint32_t)(pair_phase++) & 1u, status, abort_flag))) {
                ok = false;
                break;
            }
            tc_fence_after();
            const float m_blk = fmaxf(m_mine, __uint_as_float(tmem_ld_32x32b_x1(
                                                  tmem + lane_base + TM_X + (j & 1) * 2 + (half ^ 1)))) *
                                scale_log2;
            const bool resc = m_blk > m_use + kRescaleLog2;
            const float m_new = resc ? m_blk : m_use;
            const float alpha = resc ? exp2f(m_use - m_new) : 1.0f;  // exp2(-inf) = 0 on the first block
            const float neg_m = (m_new == -INFINITY) ? 0.0f : -m_new;
            // P_{j-1} V_{j-1} has finished: O is final for the earlier blocks and P is free
            if (!__all_sync(0xffffffffu,
                            mbar_wait(smem_addr(&bars->p_empty), ((uint32_t)j & 1u) ^ 1u, status, abort_flag))) {
                ok = false;
                break;
            }
            tc_fence_after();
            if (j > 0 && __any_sync(0xffffffffu, resc)) {
#pragma unroll 1
                for (int q = 0; q < 2; ++q) {
                    uint32_t o[32];
                    const uint32_t oc = tmem + lane_base + TM_O + half * 64 + q * 32;
                    tmem_ld_32x32b_x32(oc, o);
                    tmem_ld_wait();
#pragma unroll
                    for (int c = 0; c < 32; ++c) o[c] = __float_as_uint(__uint_as_float(o[c]) * alpha);
                    tmem_st_32x32b_x32(oc, o);
                }
                tmem_st_wait();
            }
            m_use = m_new;
            const uint32_t pcol = tmem + lane_base + TM_P + half * 32;
            const float rs = full ? row_exp64<false>(scol, key0, L, causal, pos, scale_log2, neg_m, pcol)
                                  : row_exp64<true>(scol, key0, L, causal, pos, scale_log2, neg_m, pcol);
            tc_fence_before();
            mbar_arrive(smem_addr(&bars->s_empty[sb]));  // S_j fully read
            l_half = l_half * alpha + rs;
            tc_fence_before();
            mbar_arrive(smem_addr(&bars->p_full));
        }
        const bool done = ok && __all_sync(0xffffffffu, mbar_wait(smem_addr(&bars->o_full), 0, status, abort_flag));
        // the two halves' row sums
        tmem_st_32x32b_x1(tmem + lane_base + TM_X + 4 + half, __float_as_uint(l_half));
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(pair_mb);
        const bool met = __all_sync(0xffffffffu, mbar_wait(pair_mb, (uint32_t)pair_phase & 1u, status, abort_flag));
        if (done && met) {
            tc_fence_after();
            const float l_other = __uint_as_float(tmem_ld_32x32b_x1(tmem + lane_base + TM_X + 4 + (half ^ 1)));
            const float inv = 1.0f / (half == 0 ? l_half + l_other : l_other + l_half);  // half 0's sum first
            uint16_t* orow = O + (((size_t)b * Hq + h) * T + (t < T ? t : 0)) * D + half * 64;
#pragma unroll 1
            for (int q = 0; q < 2; ++q) {
                uint32_t o[32];
                tmem_ld_32x32b_x32(tmem + lane_base + TM_O + half * 64 + q * 32, o);
                tmem_ld_wait();
                if (t < T) {
#pragma unroll
                    for (int v = 0; v < 4; ++v) {
                        const uint4 w = make_uint4(
                            pack_bf16x2(__uint_as_float(o[v * 8 + 0]) * inv, __uint_as_float(o[v * 8 + 1]) * inv),
                            pack_bf16x2(__uint_as_float(o[v * 8 + 2]) * inv, __uint_as_float(o[v * 8 + 3]) * inv),
                            pack_bf16x2(__uint_as_float(o[v * 8 + 4]) * inv, __uint_as_float(o[v * 8 + 5]) * inv),
                            pack_bf16x2(__uint_as_float(o[v * 8 + 6]) * inv, __uint_as_float(o[v * 8 + 7]) * inv));
                        *reinterpret_cast<uint4*>(orow + q * 32 + v * 8) = w;
                    }
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == kMmaWarp) tmem_dealloc(tmem, TMEM_COLS);
}

// The FMA-pipe exponential on its own, for its direct test.
__global__ void exp2_fma_kernel(const float* __restrict__ x, float* __restrict__ y, int n) {
    for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x) y[i] = poly_exp2(x[i]);
}

size_t attn_tc_smem_bytes(int kp) {
    const int ks = KV_STAGES_MAX;
    return 1024 + (size_t)ks * V_BYTES + (size_t)(1 + ks) * kp * 256 + D * sizeof(int) + sizeof(Bars);
}

}  // namespace

cudaError_t launch_exp2_fma(const float* x, float* y, int n, cudaStream_t stream) {
    const int blocks = (n + 255) / 256 < 1184 ? (n + 255) / 256 : 1184;
    exp2_fma_kernel<<<blocks, 256, 0, stream>>>(x, y, n);
    return cudaGetLastError();
}

bool attn_tc_supported(int T, int k) { return T >= kAttnTcMinT && k >= 1 && k <= D; }

cudaError_t launch_attn_tc(const uint16_t* Q, const uint16_t* Kt, const uint16_t* V, int B, int Hq, int Hkv, int T,
                           int L, int ldL, int k, int causal, float scale, int per_query_head, const int32_t* idx,
                           uint16_t* O, int* status, cudaStream_t stream) {
    const int kp = (k + 15) / 16 * 16;
    const size_t smem = attn_tc_smem_bytes(kp);
    // V [B * Hkv][ldL][d] as [plane][key][dim], only the L valid keys of a plane
    CUtensorMap vmap;
    if (!tiled_map_3d(V, D, (uint64_t)L, (uint64_t)B * Hkv, D, (uint64_t)ldL * D, BKV, &vmap))
        return cudaErrorInvalidValue;
    cudaError_t e = ensure_smem_limit(attn_tc_kernel, smem);
    if (e != cudaSuccess) return e;
    dim3 grid(Hq, (T + BQ - 1) / BQ, B);
    return launch_pdl(attn_tc_kernel, grid, dim3(kThreadsTc), smem, stream, Q, Kt, vmap, Hq, Hkv, T, L, ldL, k, kp,
                      causal, scale * 1.4426950408889634f, per_query_head, idx, O, status);
}

}  // namespace rmm
