// rmm_gemm.cu -- step 3 for prefill-sized T: the reduced product on the
// 5th-generation tensor cores (tcgen05, accumulators in TMEM).
//
// Y[t,n] = sum_{j<k} X[t, idx_j] * Wt[idx_j, n]        (fp32 accumulate, bf16 out)
//
// The reduced product is a dense contraction over the k kept slices
// (cf-1.com post on input-adaptive matrix-product reduction, §5.3: the
// smaller dense product; paper abstract: slices along the contraction
// dimension).  Instead of gathering the kept slices into compacted copies
// in memory (the post's demo does this, and §8 of the post names the copy
// traffic as the method's first cost), the producer warp gathers them straight
// into shared memory with TMA tile::gather4: each instruction brings four
// kept rows (of X^T or of W^T) x 64 elements, so a K-block of 64 kept slices is
// 16 gathers per 64-wide column group.  Both operands land MN-major in the
// 128-byte-swizzled canonical layout that tcgen05.mma reads directly.
//
// Persistent, warp-specialised, one CTA per SM:
//   warp 0     TMA producer (all 32 lanes issue gathers; 4-stage ring)
//   warp 1     TMEM allocator and MMA issuer (one thread issues
//              tcgen05.mma 128x256x16; tcgen05.commit frees ring slots and
//              signals finished accumulators)
//   warps 2-5  epilogue: tcgen05.ld 32 lanes x 32 columns -> bf16 -> global
// Two 256-column fp32 accumulators (all 512 TMEM columns) let the epilogue of
// one tile overlap the main loop of the next.  Tiles are walked M-fastest so
// CTAs running at the same time share W^T column blocks in L2.
//
// Tail handling: the kept list is padded with the index H (out of range) to a
// multiple of 64; TMA zero-fills out-of-range rows, so padded slices add 0.
// Rows t >= T of the last M tile are zero-filled the same way and not stored.
//
// Every wait is bounded (rmm_common.cuh): a stalled pipeline reports
// RMM_ERR_TIMEOUT through the status word and the CTA drains its in-flight
// copies, releases TMEM and exits.
#include "rmm_common.cuh"
#include "rmm_internal.h"

namespace rmm {

namespace {

constexpr int BM = 128;
constexpr int BN = 256;
constexpr int BK = kGemmBK;  // 64
constexpr int STAGES = 4;
constexpr int CHUNK_BYTES = BK * 128;           // BK rows x 64 bf16 (one swizzle-atom column)
constexpr int A_STAGE_BYTES = (BM / 64) * CHUNK_BYTES;  // 16 KB
constexpr int B_STAGE_BYTES = (BN / 64) * CHUNK_BYTES;  // 32 KB
constexpr uint32_t STAGE_TX = A_STAGE_BYTES + B_STAGE_BYTES;
constexpr int TMEM_COLS = 2 * BN;
constexpr int kThreads = 192;
constexpr int kEpilogueWarps = 4;

struct __align__(8) Barriers {
    uint64_t full[STAGES];
    uint64_t empty[STAGES];
    uint64_t tfull[2];
    uint64_t tempty[2];
    uint64_t never;  // watchdog self-test: nothing ever arrives here
    uint32_t tmem_base;
    int abort_flag;
};

constexpr size_t kSmemBytes = 1024 /*alignment slack*/ + (size_t)STAGES * (A_STAGE_BYTES + B_STAGE_BYTES) +
                              sizeof(Barriers);

__global__ void __launch_bounds__(kThreads, 1)
    gemm_kernel(const __grid_constant__ CUtensorMap map_xt, const __grid_constant__ CUtensorMap map_wt,
                const int32_t* __restrict__ idx, int k, int T, int H, int N,
                uint16_t* __restrict__ Y, int* status, int debug_timeout) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~static_cast<uintptr_t>(1023));
    uint8_t* sA = smem;
    uint8_t* sB = smem + STAGES * A_STAGE_BYTES;
    Barriers* bars = reinterpret_cast<Barriers*>(sB + STAGES * B_STAGE_BYTES);
    volatile int* abort_flag = &bars->abort_flag;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int m_tiles = (T + BM - 1) / BM;
    const int n_tiles = (N + BN - 1) / BN;
    const int num_tiles = m_tiles * n_tiles;
    const int nkb = (k + BK - 1) / BK;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(smem_addr(&bars->full[s]), 1);
            mbar_init(smem_addr(&bars->empty[s]), 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(smem_addr(&bars->tfull[a]), 1);
            mbar_init(smem_addr(&bars->tempty[a]), kEpilogueWarps);
        }
        mbar_init(smem_addr(&bars->never), 1);
        bars->abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&map_xt);
        tma_prefetch_desc(&map_wt);
    }
    if (warp == 1) {
        tmem_alloc(smem_addr(&bars->tmem_base), TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = bars->tmem_base;

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        int stage = 0;
        uint32_t phase = 0;
        uint32_t armed_mask = 0, armed_parity = 0;  // per stage: armed at least once / parity armed
        bool ok = true;
        const int g = lane & 15;     // group of 4 kept slices within the K-block
        const int half = lane >> 4;  // which 64-wide column groups this lane gathers
        for (int tile = blockIdx.x; ok && tile < num_tiles; tile += gridDim.x) {
            const int m0 = (tile % m_tiles) * BM;
            const int n0 = (tile / m_tiles) * BN;
            for (int kb = 0; kb < nkb; ++kb) {
                const uint32_t full = smem_addr(&bars->full[stage]);
                if (!mbar_wait(smem_addr(&bars->empty[stage]), phase ^ 1, status, abort_flag)) {
                    ok = false;
                    break;
                }
                if (lane == 0) mbar_arrive_expect_tx(full, STAGE_TX);
                __syncwarp();
                armed_mask |= 1u << stage;
                armed_parity = (armed_parity & ~(1u << stage)) | (phase << stage);
                const int j = kb * BK + g * 4;
                const int r0 = __ldg(idx + j), r1 = __ldg(idx + j + 1);
                const int r2 = __ldg(idx + j + 2), r3 = __ldg(idx + j + 3);
                const uint32_t a_dst =
                    smem_addr(sA + stage * A_STAGE_BYTES + half * CHUNK_BYTES + g * 512);
                tma_gather4(a_dst, &map_xt, full, m0 + half * 64, r0, r1, r2, r3);
#pragma unroll
                for (int c = half; c < BN / 64; c += 2) {
                    const uint32_t b_dst =
                        smem_addr(sB + stage * B_STAGE_BYTES + c * CHUNK_BYTES + g * 512);
                    tma_gather4(b_dst, &map_wt, full, n0 + c * 64, r0, r1, r2, r3);
                }
                if (++stage == STAGES) {
                    stage = 0;
                    phase ^= 1;
                }
            }
        }
        // Drain: every armed stage's copies must land before the CTA exits
        // (a no-op on the normal path, where the MMA warp consumed them all).
        if (lane == 0) {
            for (int s = 0; s < STAGES; ++s) {
                if (armed_mask & (1u << s)) {
                    int tmp_abort = 0;  // drain even after an abort
                    mbar_wait(smem_addr(&bars->full[s]), (armed_parity >> s) & 1u, status,
                              &tmp_abort, kDebugWaitLimitNs);
                }
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        constexpr uint32_t idesc = idesc_bf16_f32_mn_mn(BM, BN);
        int stage = 0;
        uint32_t phase = 0;
        int acc = 0;
        uint32_t acc_phase = 0;
        bool ok = true;
        if (debug_timeout) {
            // Watchdog self-test: wait on a barrier nothing signals; this runs
            // out after the debug limit, records RMM_ERR_TIMEOUT and aborts.
            ok = mbar_wait(smem_addr(&bars->never), 0, status, abort_flag, kDebugWaitLimitNs);
        }
        for (int tile = blockIdx.x; ok && tile < num_tiles; tile += gridDim.x) {
            if (!mbar_wait(smem_addr(&bars->tempty[acc]), acc_phase ^ 1, status, abort_flag)) break;
            tc_fence_after();
            const uint32_t d_tmem = tmem_base + (uint32_t)(acc * BN);
            for (int kb = 0; kb < nkb; ++kb) {
                if (!mbar_wait(smem_addr(&bars->full[stage]), phase, status, abort_flag)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                if (lane == 0) {
                    const uint32_t a_base = smem_addr(sA + stage * A_STAGE_BYTES);
                    const uint32_t b_base = smem_addr(sB + stage * B_STAGE_BYTES);
#pragma unroll
                    for (int kk = 0; kk < BK / 16; ++kk) {
                        // 16 kept slices = 2 groups of 8 rows = 2 x 1024 bytes
                        const uint64_t adesc = smem_desc_sw128(a_base + kk * 2048, CHUNK_BYTES, 1024);
                        const uint64_t bdesc = smem_desc_sw128(b_base + kk * 2048, CHUNK_BYTES, 1024);
                        umma_f16(d_tmem, adesc, bdesc, idesc, (kb | kk) != 0 ? 1u : 0u);
                    }
                    umma_commit(smem_addr(&bars->empty[stage]));
                }
                __syncwarp();
                if (++stage == STAGES) {
                    stage = 0;
                    phase ^= 1;
                }
            }
            if (!ok) break;
            if (lane == 0) umma_commit(smem_addr(&bars->tfull[acc]));
            __syncwarp();
            if (++acc == 2) {
                acc = 0;
                acc_phase ^= 1;
            }
        }
    } else {
        // ------------------------------------------------------------ epilogue
        const int q = warp & 3;  // TMEM lane quarter this warp may access
        int acc = 0;
        uint32_t acc_phase = 0;
        for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x) {
            const int m0 = (tile % m_tiles) * BM;
            const int n0 = (tile / m_tiles) * BN;
            if (!mbar_wait(smem_addr(&bars->tfull[acc]), acc_phase, status, abort_flag)) break;
            tc_fence_after();
            const int row = m0 + q * 32 + lane;
            uint16_t* yrow = Y + (size_t)row * N;
#pragma unroll 1
            for (int cc = 0; cc < BN / 32; ++cc) {
                uint32_t r[32];
                tmem_ld_32x32b_x32(tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * BN + cc * 32), r);
                tmem_ld_wait();
                if (row < T) {
#pragma unroll
                    for (int v = 0; v < 4; ++v) {
                        const int nn = n0 + cc * 32 + v * 8;
                        if (nn < N) {
                            uint4 o;
                            o.x = pack_bf16x2(__uint_as_float(r[v * 8 + 0]), __uint_as_float(r[v * 8 + 1]));
                            o.y = pack_bf16x2(__uint_as_float(r[v * 8 + 2]), __uint_as_float(r[v * 8 + 3]));
                            o.z = pack_bf16x2(__uint_as_float(r[v * 8 + 4]), __uint_as_float(r[v * 8 + 5]));
                            o.w = pack_bf16x2(__uint_as_float(r[v * 8 + 6]), __uint_as_float(r[v * 8 + 7]));
                            *reinterpret_cast<uint4*>(yrow + nn) = o;
                        }
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_addr(&bars->tempty[acc]));
            if (++acc == 2) {
                acc = 0;
                acc_phase ^= 1;
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem_base, TMEM_COLS);
}

}  // namespace

size_t gemm_smem_bytes() { return kSmemBytes; }

cudaError_t launch_gemm(const CUtensorMap& map_xt, const CUtensorMap& map_wt, const int32_t* idx,
                        int k, int T, int H, int N, uint16_t* Y, int* status, int debug_timeout,
                        int num_sms, cudaStream_t stream) {
    cudaError_t e = cudaFuncSetAttribute(gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)kSmemBytes);
    if (e != cudaSuccess) return e;
    const int tiles = ((T + BM - 1) / BM) * ((N + BN - 1) / BN);
    const int grid = tiles < num_sms ? tiles : num_sms;
    gemm_kernel<<<grid, kThreads, kSmemBytes, stream>>>(map_xt, map_wt, idx, k, T, H, N, Y, status,
                                                         debug_timeout);
    return cudaGetLastError();
}

}  // namespace rmm
