// rmm_gemm.cu -- step 3 for prefill-sized T: the reduced product on the
// 5th-generation tensor cores (tcgen05, accumulators in TMEM).
//
// Y[t,n] = sum_{j<k} X[t, idx_j] * Wt[idx_j, n]        (fp32 accumulate, bf16 out)
//
// The reduced product is a dense contraction over the k kept slices
// (cf-1.com post on input-adaptive matrix-product reduction, §5.3: the
// smaller dense product; paper abstract: slices along the contraction
// dimension).  The post's demo gathers the kept slices into compacted copies
// in memory, and its §8 names that copy traffic as the method's first cost;
// here the kept slices go straight from their home rows into shared memory,
// and no compacted copy exists anywhere in HBM.
//
// Two kernels live here.  The default is the CTA-pair kernel (namespace
// `pair`, described at its definition): a cluster of two CTAs computes a
// 256 x 512 tile with tcgen05 cta_group::2, its operands gathered by cp.async
// or, for kept sets made of whole 64-slice runs, loaded by TMA tile copies.
// The single-CTA kernel described next is kept for comparison (rmm_options.
// gemm_producer 1 and 2).
//
// A kept slice h is one contiguous row of W^T [H, N] and one contiguous row of
// X^T [H, T] (written by the score pass).  For a 128 x 256 output tile and a
// K-block of 64 kept slices the operands are 64 rows x 256 columns of W^T
// (512 B per row) and 64 rows x 128 columns of X^T (256 B per row), placed
// MN-major in the 128-byte-swizzled canonical layout that tcgen05.mma reads:
// each 64-column group is a block of 64 rows x 128 B, and 16-byte chunk c of
// row j sits at chunk position c ^ (j mod 8).
//
// Two producers fill that layout (template parameter):
//   cp.async (default)  many warps; one warp instruction moves one 512-B row
//                       segment (16 B per lane) into its swizzled place; each
//                       thread's copies arrive on the stage barrier through
//                       cp.async.mbarrier.arrive.  Padded slices (index H) and
//                       columns past N or T are zero-filled.
//   TMA tile::gather4   one warp; each instruction brings four kept rows x 64
//                       columns (measured on B200: ~75 SM cycles of TMA time
//                       per instruction, 96 per stage, which caps this
//                       producer near 155 TFLOP/s -- kept for comparison).
//
// Persistent, warp-specialised, one CTA per SM (21 warps):
//   warps 0-15   producer (measured: the copy-issue rate per warp is the
//                limit, so the 96 row copies of a stage are spread over 16
//                warps, 6 per warp, fully unrolled with precomputed offsets)
//   warps 16-19  epilogue: tcgen05.ld 32 lanes x 32 columns -> bf16 -> global
//                (warp w reads TMEM lanes 32*(w%4) .. +31)
//   warp 20      TMEM allocator and MMA issuer (one thread issues
//              tcgen05.mma 128x256x16, tcgen05.commit frees ring slots and
//              signals finished accumulators)
// Two 256-column fp32 accumulators (all 512 TMEM columns) let the epilogue of
// one tile overlap the main loop of the next.  Tiles are walked M-fastest so
// CTAs running at the same time share W^T column blocks in L2.
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
constexpr int CHUNK_BYTES = BK * 128;                   // BK rows x 64 bf16 (one swizzle-atom column)
constexpr int A_STAGE_BYTES = (BM / 64) * CHUNK_BYTES;  // 16 KB
constexpr int B_STAGE_BYTES = (BN / 64) * CHUNK_BYTES;  // 32 KB
constexpr uint32_t STAGE_TX = A_STAGE_BYTES + B_STAGE_BYTES;
constexpr int TMEM_COLS = 2 * BN;
constexpr int kProducerWarps = 16;
constexpr int kRowsB = BK / kProducerWarps;        // W^T row copies per producer warp and stage
constexpr int kRowsA = BK / (2 * kProducerWarps);  // X^T double-row copies per producer warp and stage
static_assert(BK % (2 * kProducerWarps) == 0, "row copies must divide evenly over the producer warps");
constexpr int kProducerThreads = 32 * kProducerWarps;
constexpr int kEpilogueWarps = 4;
constexpr int kMmaWarp = kProducerWarps + kEpilogueWarps;
constexpr int kThreads = 32 * (kMmaWarp + 1);

struct __align__(8) Barriers {
    uint64_t full[STAGES];
    uint64_t empty[STAGES];
    uint64_t tfull[2];
    uint64_t tempty[2];
    uint64_t never;  // watchdog self-test: nothing ever arrives here
    uint32_t tmem_base;
    int abort_flag;
};

constexpr size_t kSmemBytes =
    1024 /*alignment slack*/ + (size_t)STAGES * (A_STAGE_BYTES + B_STAGE_BYTES) + sizeof(Barriers);

// Byte offset, inside a stage's operand block, of 16-byte chunk c16 (counted
// along M/N from the tile start) of kept row j, in the 128-byte-swizzled
// MN-major canonical layout.
__device__ __forceinline__ uint32_t swz_offset(int j, int c16) {
    return (uint32_t)((c16 >> 3) * CHUNK_BYTES + j * 128 + (((c16 & 7) ^ (j & 7)) << 4));
}

struct TileCoord {
    int p, m0, n0;
};

// Tile t of the group: product p with tile_start[p] <= t < tile_start[p+1],
// walked M-fastest inside the product so concurrent CTAs share W^T columns.
__device__ __forceinline__ TileCoord decode_tile(const GemmGroup& g, int t, int m_tiles) {
    int p = 0;
#pragma unroll
    for (int i = 1; i < kMaxGroup; ++i)
        if (i < g.count && t >= g.tile_start[i]) p = i;
    const int local = t - g.tile_start[p];
    TileCoord c;
    c.p = p;
    c.m0 = (local % m_tiles) * BM;
    c.n0 = (local / m_tiles) * BN;
    return c;
}

template <bool kTmaGather>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_kernel(const __grid_constant__ CUtensorMap map_xt, const __grid_constant__ CUtensorMap map_wt,
                const uint16_t* __restrict__ Xt, int ldT, const __grid_constant__ GemmGroup group,
                const int32_t* __restrict__ idx, int k, int T, int H, int* status, int debug_timeout) {
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
    const int num_tiles = group.tile_start[group.count];
    const int nkb = (k + BK - 1) / BK;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(smem_addr(&bars->full[s]), kTmaGather ? 1 : kProducerThreads);
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
    if (kTmaGather && warp == 0 && lane == 0) {
        tma_prefetch_desc(&map_xt);
        tma_prefetch_desc(&map_wt);
    }
    if (warp == kMmaWarp) {
        tmem_alloc(smem_addr(&bars->tmem_base), TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = bars->tmem_base;
    pdl_wait();  // the kept list and X^T come from the preceding kernels
    pdl_launch_dependents();

    if (warp < kProducerWarps) {
        // ------------------------------------------------------------ producer
        int stage = 0;
        uint32_t phase = 0;
        uint32_t armed_mask = 0, armed_parity = 0;  // TMA producer: stages armed / parity armed
        bool ok = true;
        // Kept indices of a K-block live in registers, two per lane
        // (idx[kb*64 + lane], idx[kb*64 + 32 + lane]); they are fetched two
        // K-blocks ahead so their latency never sits on the copy-issue path.
        // The K-block sequence repeats 0..nkb-1 for every tile.
        int q0a = 0, q1a = 0, q0b = 0, q1b = 0, next_kb = 0;
        if (!kTmaGather) {
            q0a = __ldg(idx + lane);
            q1a = __ldg(idx + 32 + lane);
            next_kb = (1 < nkb) ? 1 : 0;
            q0b = __ldg(idx + next_kb * BK + lane);
            q1b = __ldg(idx + next_kb * BK + 32 + lane);
            next_kb = (next_kb + 1 < nkb) ? next_kb + 1 : 0;
        }
        // swizzled shared-memory offsets of this thread's copies: fixed for every stage
        uint32_t b_off[kRowsB], a_off[kRowsA];
#pragma unroll
        for (int i = 0; i < kRowsB; ++i) b_off[i] = swz_offset(warp + kProducerWarps * i, lane);
#pragma unroll
        for (int i = 0; i < kRowsA; ++i)
            a_off[i] = swz_offset(2 * (warp + kProducerWarps * i) + (lane >> 4), lane & 15);
        for (int tile = blockIdx.x; ok && tile < num_tiles; tile += gridDim.x) {
            const TileCoord tc = decode_tile(group, tile, m_tiles);
            const int m0 = tc.m0, n0 = tc.n0;
            const int N = group.N[tc.p];
            const uint16_t* __restrict__ Wt = group.Wt[tc.p];
            if (kTmaGather && warp != 0) break;
            const int b_col = n0 + lane * 8;          // this lane's W^T columns
            const int a_col = m0 + (lane & 15) * 8;   // this lane's X^T columns (tokens)
            const bool b_col_ok = b_col < N;
            const bool a_col_ok = a_col < T;
            for (int kb = 0; kb < nkb; ++kb) {
                const uint32_t full = smem_addr(&bars->full[stage]);
                if (!mbar_wait(smem_addr(&bars->empty[stage]), phase ^ 1, status, abort_flag)) {
                    ok = false;
                    break;
                }
                const uint32_t a_stage = smem_addr(sA + stage * A_STAGE_BYTES);
                const uint32_t b_stage = smem_addr(sB + stage * B_STAGE_BYTES);
                if constexpr (kTmaGather) {
                    if (lane == 0) mbar_arrive_expect_tx(full, STAGE_TX);
                    __syncwarp();
                    armed_mask |= 1u << stage;
                    armed_parity = (armed_parity & ~(1u << stage)) | (phase << stage);
                    const int g = lane & 15, half = lane >> 4;
                    const int j = kb * BK + g * 4;
                    const int r0 = __ldg(idx + j), r1 = __ldg(idx + j + 1);
                    const int r2 = __ldg(idx + j + 2), r3 = __ldg(idx + j + 3);
                    tma_gather4(a_stage + half * CHUNK_BYTES + g * 512, &map_xt, full, m0 + half * 64, r0,
                                r1, r2, r3);
#pragma unroll
                    for (int c = half; c < BN / 64; c += 2)
                        tma_gather4(b_stage + c * CHUNK_BYTES + g * 512, &map_wt, full, n0 + c * 64, r0, r1,
                                    r2, r3);
                } else {
                    // kept indices of this K-block (the list is padded with H)
                    const int v0 = q0a, v1 = q1a;
                    q0a = q0b;
                    q1a = q1b;
                    q0b = __ldg(idx + next_kb * BK + lane);
                    q1b = __ldg(idx + next_kb * BK + 32 + lane);
                    next_kb = (next_kb + 1 < nkb) ? next_kb + 1 : 0;
                    // W^T: 64 rows x 32 chunks; warp w copies rows w + PW*i (one
                    // 512-B row segment per warp instruction, lane = 16-B chunk)
#pragma unroll
                    for (int i = 0; i < kRowsB; ++i) {
                        const int jr = warp + kProducerWarps * i;  // warp-uniform
                        const int h = __shfl_sync(0xffffffffu, jr < 32 ? v0 : v1, jr & 31);
                        const bool ok_copy = b_col_ok && h < H;
                        const uint16_t* src = ok_copy ? Wt + (size_t)h * N + b_col : Wt;
                        cp_async_16(b_stage + b_off[i], src, ok_copy ? 16u : 0u);
                    }
                    // X^T: 64 rows x 16 chunks; a warp instruction covers two rows
#pragma unroll
                    for (int i = 0; i < kRowsA; ++i) {
                        const int jr = 2 * (warp + kProducerWarps * i) + (lane >> 4);
                        const int h0v = __shfl_sync(0xffffffffu, v0, jr & 31);
                        const int h1v = __shfl_sync(0xffffffffu, v1, jr & 31);
                        const int h = jr < 32 ? h0v : h1v;
                        const bool ok_copy = a_col_ok && h < H;
                        const uint16_t* src = ok_copy ? Xt + (size_t)h * ldT + a_col : Xt;
                        cp_async_16(a_stage + a_off[i], src, ok_copy ? 16u : 0u);
                    }
                    cp_async_arrive_noinc(full);
                }
                if (++stage == STAGES) {
                    stage = 0;
                    phase ^= 1;
                }
            }
        }
        if constexpr (kTmaGather) {
            // Drain: every armed stage's copies must land before the CTA exits
            // (a no-op on the normal path, where the MMA warp consumed them all).
            if (warp == 0 && lane == 0) {
                for (int s = 0; s < STAGES; ++s) {
                    if (armed_mask & (1u << s)) {
                        int tmp_abort = 0;  // drain even after an abort
                        mbar_wait(smem_addr(&bars->full[s]), (armed_parity >> s) & 1u, status, &tmp_abort,
                                  kDebugWaitLimitNs);
                    }
                }
            }
        } else {
            cp_async_wait_all();
        }
    } else if (warp == kMmaWarp) {
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
                if (!kTmaGather) fence_proxy_async_smem();  // cp.async wrote the stage
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
        const int q = warp & 3;  // TMEM lane quarter (four consecutive warps cover all four)
        int acc = 0;
        uint32_t acc_phase = 0;
        for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x) {
            const TileCoord tc = decode_tile(group, tile, m_tiles);
            const int m0 = tc.m0, n0 = tc.n0;
            const int N = group.N[tc.p];
            uint16_t* __restrict__ Y = group.Y[tc.p];
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
    if (warp == kMmaWarp) tmem_dealloc(tmem_base, TMEM_COLS);
}


// ============================================================================
// CTA-pair variant (tcgen05 cta_group::2): a cluster of two CTAs on one TPC
// computes a 256 x 512 output tile.  CTA r of the pair stages rows
// [128r, 128r+128) of the X^T tile and the contiguous column half
// [256r, 256r+256) of the W^T tile (48 KB per 64-slice stage, 4 stages).  The
// leader (r = 0) issues, per 16-slice step, two tcgen05.mma.cta_group::2
// 256x256x16: "lo" on the first 128 columns of each CTA's half, "hi" on the
// second 128; each reads A from both CTAs by rows and B by column halves, and
// accumulates rows [128r, 128r+128) in CTA r's TMEM (lo in columns 0..255, hi
// in 256..511: all of TMEM).  Per SM this gathers 5.7 KB of operands per MFLOP
// (11.4 KB for the single-CTA 128 x 256 tile), which matters because the
// cp.async gather rate per SM is this kernel's measured bound; a kept W^T row
// still arrives as one 512-byte segment per warp instruction.
//
// TMEM column c of a CTA holds output column
//   n0 + 256 * ((c mod 256) / 128) + 128 * (c / 256) + (c mod 128)
// (lo/hi, then which CTA's half the MMA took the 128 columns from).
//
// Synchronisation across the pair:
//   full[s]       local: the CTA's own 512 producer threads (cp.async arrive)
//   pair_full[s]  leader only: the peer's MMA warp relays "peer stage s full"
//                 (cluster-scope release/acquire, after a proxy fence)
//   empty[s]      both: the leader commits to its own and the peer's barrier
//   tfull         both: the leader commits to its own and the peer's barrier
//   tempty        leader only: 4 local + 4 remote epilogue-warp arrivals
// The single accumulator is not double-buffered (it fills TMEM), so a tile's
// epilogue does not overlap the next tile's main loop.
// An abort (bounded wait ran out) is raised in both CTAs' flags.
namespace pair {

constexpr int BM2 = 256;                 // tile rows (two CTAs x 128)
constexpr int BN2 = 512;                 // tile columns (two CTAs x 256)
constexpr int HALF_M = 128;              // rows staged per CTA
constexpr int HALF_N = 256;              // columns staged per CTA
constexpr int STAGES2 = 4;
constexpr int A2_STAGE_BYTES = (HALF_M / 64) * CHUNK_BYTES;  // 16 KB
constexpr int B2_STAGE_BYTES = (HALF_N / 64) * CHUNK_BYTES;  // 32 KB
constexpr int TMEM_COLS2 = 512;

struct __align__(8) Barriers2 {
    uint64_t full[STAGES2];
    uint64_t pair_full[STAGES2];
    uint64_t empty[STAGES2];
    uint64_t tfull;
    uint64_t tempty;
    uint64_t never;
    uint32_t tmem_base;
    int abort_flag;
};

constexpr int EPI_STAGE_BYTES = 32 * 128;  // one epilogue warp's 32 rows x 64 bf16 columns
// Eight epilogue warps: warps w and w + 4 share TMEM lane quarter w % 4 and
// drain the lower and upper 256 accumulator columns, halving the time the
// MMA waits for the (single, TMEM-filling) accumulator between tiles.
constexpr int kEpiWarps2 = 8;
constexpr int kMmaWarp2 = kProducerWarps + kEpiWarps2;
constexpr int kThreads2 = 32 * (kMmaWarp2 + 1);
constexpr size_t kSmemBytes2 =
    1024 + (size_t)STAGES2 * (A2_STAGE_BYTES + B2_STAGE_BYTES) + (size_t)kEpiWarps2 * EPI_STAGE_BYTES +
    sizeof(Barriers2);

__device__ __forceinline__ TileCoord decode_tile2(const GemmGroup& g, int t, int m_tiles) {
    int p = 0;
#pragma unroll
    for (int i = 1; i < kMaxGroup; ++i)
        if (i < g.count && t >= g.tile_start[i]) p = i;
    const int local = t - g.tile_start[p];
    TileCoord c;
    c.p = p;
    c.m0 = (local % m_tiles) * BM2;
    c.n0 = (local / m_tiles) * BN2;
    return c;
}

// Work unit u: a whole tile (u < units_full), or one K-range of a tile of the
// split last wave; part = the unit's slot in the fp32 partials, -1 if whole.
struct Unit {
    TileCoord tc;
    int kb0, kb1, part;
};

__device__ __forceinline__ Unit decode_unit(const GemmGroup& g, int u, int m_tiles, int nkb) {
    Unit r;
    if (u < g.units_full) {
        r.tc = decode_tile2(g, u, m_tiles);
        r.kb0 = 0;
        r.kb1 = nkb;
        r.part = -1;
    } else {
        const int v = u - g.units_full;
        const int sp = v % g.tail_splits;
        r.tc = decode_tile2(g, g.units_full + v / g.tail_splits, m_tiles);
        r.kb0 = sp * nkb / g.tail_splits;
        r.kb1 = (sp + 1) * nkb / g.tail_splits;
        r.part = v;
    }
    return r;
}

// kTmaRows: every 64-slice K-block of the kept list is 64 contiguous slices
// (block-granular kept sets whose block is a multiple of 64), so one thread
// loads each stage with six TMA tile loads (two 64-token boxes of X^T, four
// 64-column boxes of W^T, 64 rows each) instead of the cp.async gather.
template <bool kTmaRows>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads2, 1)
    gemm_pair_kernel(const uint16_t* __restrict__ Xt, int ldT, const __grid_constant__ GemmGroup group,
                     const __grid_constant__ GemmOutMaps ymaps, const __grid_constant__ GemmInMaps imaps,
                     const int32_t* __restrict__ idx, int k, int T, int H, int* status, int debug_timeout) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~static_cast<uintptr_t>(1023));
    uint8_t* sA = smem;
    uint8_t* sB = smem + STAGES2 * A2_STAGE_BYTES;
    uint8_t* sE = sB + STAGES2 * B2_STAGE_BYTES;  // epilogue staging, one block per epilogue warp
    Barriers2* bars = reinterpret_cast<Barriers2*>(sE + kEpiWarps2 * EPI_STAGE_BYTES);
    volatile int* abort_flag = &bars->abort_flag;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();  // 0 = leader
    const uint32_t peer = rank ^ 1u;
    const int m_tiles = (T + BM2 - 1) / BM2;
    const int num_units = group.units;
    const int nkb = (k + BK - 1) / BK;
    const int cluster_id = blockIdx.x >> 1;
    const int num_clusters = gridDim.x >> 1;
    const uint32_t peer_abort = mapa_shared(smem_addr(&bars->abort_flag), peer);

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES2; ++s) {
            mbar_init(smem_addr(&bars->full[s]), kTmaRows ? 1 : kProducerThreads);
            mbar_init(smem_addr(&bars->pair_full[s]), 1);
            mbar_init(smem_addr(&bars->empty[s]), 1);
        }
        mbar_init(smem_addr(&bars->tfull), 1);
        mbar_init(smem_addr(&bars->tempty), 2 * kEpiWarps2);
        mbar_init(smem_addr(&bars->never), 1);
        bars->abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == kMmaWarp2) {
        tmem_alloc_pair(smem_addr(&bars->tmem_base), TMEM_COLS2);
        tmem_relinquish_pair();
    }
    tc_fence_before();
    cluster_sync();  // barriers of both CTAs initialised, TMEM allocated in both
    tc_fence_after();
    const uint32_t tmem_base = bars->tmem_base;
    pdl_wait();  // the kept list and X^T come from the preceding kernels
    pdl_launch_dependents();

    if (kTmaRows && warp < kProducerWarps) {
        // ------------------------------------------------------------ TMA producer (both CTAs)
        if (warp == 0 && lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            uint32_t issued_phase[STAGES2];
            bool issued[STAGES2];
            for (int s = 0; s < STAGES2; ++s) issued[s] = false;
            bool ok = true;
            for (int u = cluster_id; ok && u < num_units; u += num_clusters) {
                const Unit ux = decode_unit(group, u, m_tiles, nkb);
                const TileCoord tc = ux.tc;
                const int a_col = tc.m0 + HALF_M * (int)rank;
                const int b_col = tc.n0 + HALF_N * (int)rank;
                int row_next = __ldg(idx + ux.kb0 * BK);  // first slice of the K-block: its 64 rows are contiguous
                for (int kb = ux.kb0; kb < ux.kb1; ++kb) {
                    const int row = row_next;
                    if (kb + 1 < ux.kb1) row_next = __ldg(idx + (kb + 1) * BK);
                    const uint32_t full = smem_addr(&bars->full[stage]);
                    if (!mbar_wait(smem_addr(&bars->empty[stage]), phase ^ 1, status, abort_flag)) {
                        st_shared_cluster_u32(peer_abort, 1);
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(full, A2_STAGE_BYTES + B2_STAGE_BYTES);
                    const uint32_t a_stage = smem_addr(sA + stage * A2_STAGE_BYTES);
                    const uint32_t b_stage = smem_addr(sB + stage * B2_STAGE_BYTES);
#pragma unroll
                    for (int i = 0; i < HALF_M / 64; ++i)
                        tma_load_2d(a_stage + i * CHUNK_BYTES, &imaps.xt, full, a_col + 64 * i, row);
#pragma unroll
                    for (int i = 0; i < HALF_N / 64; ++i)
                        tma_load_2d(b_stage + i * CHUNK_BYTES, &imaps.wt[tc.p], full, b_col + 64 * i, row);
                    issued[stage] = true;
                    issued_phase[stage] = phase;
                    if (++stage == STAGES2) {
                        stage = 0;
                        phase ^= 1;
                    }
                }
            }
            // no copy may still be landing in shared memory when the CTA leaves
            volatile int no_abort = 0;
            for (int s = 0; s < STAGES2; ++s)
                if (issued[s]) mbar_wait(smem_addr(&bars->full[s]), issued_phase[s], status, &no_abort);
        }
    } else if (warp < kProducerWarps) {
        // ------------------------------------------------------------ producer (both CTAs)
        int stage = 0;
        uint32_t phase = 0;
        bool ok = true;
        // kept indices of the (unit, K-block) sequence this pair walks, two
        // K-blocks ahead of use; past the last unit any in-range block will do
        int pu = cluster_id, pkb = 0, pkb1 = 1 << 30;
        if (pu < num_units) {
            const Unit x = decode_unit(group, pu, m_tiles, nkb);
            pkb = x.kb0;
            pkb1 = x.kb1;
        }
        auto advance = [&]() {
            if (++pkb >= pkb1) {
                pu += num_clusters;
                pkb = 0;
                pkb1 = 1 << 30;
                if (pu < num_units) {
                    const Unit x = decode_unit(group, pu, m_tiles, nkb);
                    pkb = x.kb0;
                    pkb1 = x.kb1;
                }
            }
        };
        auto kq = [&]() { return pu < num_units ? pkb : 0; };
        int q0a = __ldg(idx + kq() * BK + lane), q1a = __ldg(idx + kq() * BK + 32 + lane);
        advance();
        int q0b = __ldg(idx + kq() * BK + lane), q1b = __ldg(idx + kq() * BK + 32 + lane);
        uint32_t b_off[kRowsB], a_off[kRowsA];
#pragma unroll
        for (int i = 0; i < kRowsB; ++i) b_off[i] = swz_offset(warp + kProducerWarps * i, lane);
#pragma unroll
        for (int i = 0; i < kRowsA; ++i)
            a_off[i] = swz_offset(2 * (warp + kProducerWarps * i) + (lane >> 4), lane & 15);
        for (int u = cluster_id; ok && u < num_units; u += num_clusters) {
            const Unit ux = decode_unit(group, u, m_tiles, nkb);
            const TileCoord tc = ux.tc;
            const int N = group.N[tc.p];
            const uint16_t* __restrict__ Wt = group.Wt[tc.p];
            const int a_col = tc.m0 + HALF_M * (int)rank + (lane & 15) * 8;  // tokens
            const int b_col = tc.n0 + HALF_N * (int)rank + lane * 8;         // output features
            const bool a_col_ok = a_col < T;
            const bool b_col_ok = b_col < N;
            for (int kb = ux.kb0; kb < ux.kb1; ++kb) {
                const uint32_t full = smem_addr(&bars->full[stage]);
                if (!mbar_wait(smem_addr(&bars->empty[stage]), phase ^ 1, status, abort_flag)) {
                    st_shared_cluster_u32(peer_abort, 1);
                    ok = false;
                    break;
                }
                const uint32_t a_stage = smem_addr(sA + stage * A2_STAGE_BYTES);
                const uint32_t b_stage = smem_addr(sB + stage * B2_STAGE_BYTES);
                const int v0 = q0a, v1 = q1a;
                q0a = q0b;
                q1a = q1b;
                advance();
                q0b = __ldg(idx + kq() * BK + lane);
                q1b = __ldg(idx + kq() * BK + 32 + lane);
                // W^T: one 512-B row segment per warp instruction
#pragma unroll
                for (int i = 0; i < kRowsB; ++i) {
                    const int jr = warp + kProducerWarps * i;  // warp-uniform
                    const int h = __shfl_sync(0xffffffffu, jr < 32 ? v0 : v1, jr & 31);
                    const bool ok_b = b_col_ok && h < H;
                    cp_async_16(b_stage + b_off[i], ok_b ? Wt + (size_t)h * N + b_col : Wt, ok_b ? 16u : 0u);
                }
                // X^T: two 256-B row segments per warp instruction
#pragma unroll
                for (int i = 0; i < kRowsA; ++i) {
                    const int jr = 2 * (warp + kProducerWarps * i) + (lane >> 4);
                    const int h0v = __shfl_sync(0xffffffffu, v0, jr & 31);
                    const int h1v = __shfl_sync(0xffffffffu, v1, jr & 31);
                    const int h = jr < 32 ? h0v : h1v;
                    const bool ok_a = a_col_ok && h < H;
                    cp_async_16(a_stage + a_off[i], ok_a ? Xt + (size_t)h * ldT + a_col : Xt, ok_a ? 16u : 0u);
                }
                cp_async_arrive_noinc(full);
                if (++stage == STAGES2) {
                    stage = 0;
                    phase ^= 1;
                }
            }
        }
        cp_async_wait_all();
    } else if (warp == kMmaWarp2) {
        int stage = 0;
        uint32_t phase = 0;
        bool ok = true;
        if (rank == 1) {
            // ------------------------------------------------------------ relay (peer CTA)
            if (lane == 0) {
                const uint32_t leader_pair_full0 = mapa_shared(smem_addr(&bars->pair_full[0]), 0);
                for (int u = cluster_id; ok && u < num_units; u += num_clusters) {
                    const Unit ux = decode_unit(group, u, m_tiles, nkb);
                    for (int kb = ux.kb0; kb < ux.kb1; ++kb) {
                        if (!mbar_wait(smem_addr(&bars->full[stage]), phase, status, abort_flag)) {
                            st_shared_cluster_u32(peer_abort, 1);
                            ok = false;
                            break;
                        }
                        fence_proxy_async_smem();  // the peer's cp.async data, read by the leader's MMA
                        mbar_arrive_cluster(leader_pair_full0 + stage * (uint32_t)sizeof(uint64_t));
                        if (++stage == STAGES2) {
                            stage = 0;
                            phase ^= 1;
                        }
                    }
                }
            }
            __syncwarp();
        } else {
            // ------------------------------------------------------------ MMA issuer (leader)
            constexpr uint32_t idesc = idesc_bf16_f32_mn_mn(BM2, 256);
            uint32_t acc_phase = 0;
            const uint32_t empty0_local = smem_addr(&bars->empty[0]);
            const uint32_t empty0_peer = mapa_shared(empty0_local, 1);
            const uint32_t tfull_local = smem_addr(&bars->tfull);
            const uint32_t tfull_peer = mapa_shared(tfull_local, 1);
            if (debug_timeout) {
                ok = mbar_wait(smem_addr(&bars->never), 0, status, abort_flag, kDebugWaitLimitNs);
                if (!ok) st_shared_cluster_u32(peer_abort, 1);
            }
            for (int u = cluster_id; ok && u < num_units; u += num_clusters) {
                const Unit ux = decode_unit(group, u, m_tiles, nkb);
                if (!mbar_wait_cluster(smem_addr(&bars->tempty), acc_phase ^ 1, status, abort_flag)) {
                    st_shared_cluster_u32(peer_abort, 1);
                    break;
                }
                tc_fence_after();
                for (int kb = ux.kb0; kb < ux.kb1; ++kb) {
                    if (!mbar_wait(smem_addr(&bars->full[stage]), phase, status, abort_flag) ||
                        !mbar_wait_cluster(smem_addr(&bars->pair_full[stage]), phase, status, abort_flag)) {
                        st_shared_cluster_u32(peer_abort, 1);
                        ok = false;
                        break;
                    }
                    fence_proxy_async_smem();
                    tc_fence_after();
                    if (lane == 0) {
                        const uint32_t a_base = smem_addr(sA + stage * A2_STAGE_BYTES);
                        const uint32_t b_base = smem_addr(sB + stage * B2_STAGE_BYTES);
#pragma unroll
                        for (int kk = 0; kk < BK / 16; ++kk) {
                            const uint32_t accumulate = (kb != ux.kb0 || kk != 0) ? 1u : 0u;
                            const uint64_t adesc = smem_desc_sw128(a_base + kk * 2048, CHUNK_BYTES, 1024);
                            const uint64_t blo = smem_desc_sw128(b_base + kk * 2048, CHUNK_BYTES, 1024);
                            const uint64_t bhi = smem_desc_sw128(b_base + 2 * CHUNK_BYTES + kk * 2048, CHUNK_BYTES, 1024);
                            umma_f16_pair(tmem_base, adesc, blo, idesc, accumulate);
                            umma_f16_pair(tmem_base + 256u, adesc, bhi, idesc, accumulate);
                        }
                        const uint32_t eoff = stage * (uint32_t)sizeof(uint64_t);
                        umma_commit_pair(empty0_local + eoff);
                        umma_commit_pair(empty0_peer + eoff);
                    }
                    __syncwarp();
                    if (++stage == STAGES2) {
                        stage = 0;
                        phase ^= 1;
                    }
                }
                if (!ok) break;
                if (lane == 0) {
                    umma_commit_pair(tfull_local);
                    umma_commit_pair(tfull_peer);
                }
                __syncwarp();
                acc_phase ^= 1;
            }
        }
    } else {
        // ------------------------------------------------------------ epilogue (both CTAs)
        const int q = warp & 3;                            // TMEM lane quarter
        const int e = warp - kProducerWarps;               // 0..7
        const int c64_begin = (e / 4) * (TMEM_COLS2 / 128);  // this warp's half of the columns
        uint32_t acc_phase = 0;
        const uint32_t tempty_leader = mapa_shared(smem_addr(&bars->tempty), 0);
        for (int u = cluster_id; u < num_units; u += num_clusters) {
            const Unit ux = decode_unit(group, u, m_tiles, nkb);
            const TileCoord tc = ux.tc;
            if (!mbar_wait(smem_addr(&bars->tfull), acc_phase, status, abort_flag)) {
                st_shared_cluster_u32(peer_abort, 1);
                break;
            }
            tc_fence_after();
            const int rbase = tc.m0 + HALF_M * (int)rank + q * 32;  // first row of this warp
            const uint32_t stg = smem_addr(sE + e * EPI_STAGE_BYTES);
            // 64 TMEM columns at a time: the 64 output columns they hold are contiguous
#pragma unroll 1
            for (int c64 = c64_begin; c64 < c64_begin + TMEM_COLS2 / 128; ++c64) {
                const int c = c64 * 64;
                const int lcol = 256 * ((c & 255) >> 7) + 128 * (c >> 8) + (c & 127);  // column inside the tile
                if (ux.part < 0) {
                    // the previous block's TMA store has finished reading the staging area
                    if (lane == 0) bulk_wait_read_all();
                    __syncwarp();
                }
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    uint32_t r[32];
                    tmem_ld_32x32b_x32(tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(c + 32 * h), r);
                    tmem_ld_wait();
                    if (ux.part >= 0) {
                        // a K-range of a split tile: fp32 partials in the lanes' order, one
                        // 512-byte store per instruction: [cta][warp][32-col chunk][v][lane][4]
                        float4* dst = reinterpret_cast<float4*>(group.partials + (size_t)ux.part * BM2 * BN2) +
                                      ((((int)rank * kEpilogueWarps + q) * (TMEM_COLS2 / 32) + 2 * c64 + h) * 8) * 32 +
                                      lane;
#pragma unroll
                        for (int v = 0; v < 8; ++v)
                            __stcg(dst + v * 32,
                                   make_float4(__uint_as_float(r[4 * v]), __uint_as_float(r[4 * v + 1]),
                                               __uint_as_float(r[4 * v + 2]), __uint_as_float(r[4 * v + 3])));
                    } else {
                        // bf16 row pieces into shared memory, 16-byte chunks XOR-swizzled by row
#pragma unroll
                        for (int j = 0; j < 4; ++j) {
                            const int ch = 4 * h + j;
                            uint4 o;
                            o.x = pack_bf16x2(__uint_as_float(r[j * 8 + 0]), __uint_as_float(r[j * 8 + 1]));
                            o.y = pack_bf16x2(__uint_as_float(r[j * 8 + 2]), __uint_as_float(r[j * 8 + 3]));
                            o.z = pack_bf16x2(__uint_as_float(r[j * 8 + 4]), __uint_as_float(r[j * 8 + 5]));
                            o.w = pack_bf16x2(__uint_as_float(r[j * 8 + 6]), __uint_as_float(r[j * 8 + 7]));
                            st_shared_v4(stg + lane * 128 + ((ch ^ (lane & 7)) << 4), o);
                        }
                    }
                }
                if (ux.part < 0) {
                    // the staged 32 x 64 block goes out as one TMA tile store (rows past
                    // T and columns past N are clipped by the map)
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) {
                        tma_store_2d(&ymaps.m[tc.p], stg, tc.n0 + lcol, rbase);
                        bulk_commit();
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(tempty_leader);
            acc_phase ^= 1;
        }
        if (lane == 0) bulk_wait_all();  // this warp's tile stores have completed
        __syncwarp();
    }

    tc_fence_before();
    cluster_sync();  // the leader's last MMAs and the peer's last TMEM reads are done
    tc_fence_after();
    if (warp == kMmaWarp2) tmem_dealloc_pair(tmem_base, TMEM_COLS2);
}

// Y = the sum, in split order, of the fp32 partials of each split tile.  The
// epilogue left them in its lanes' order, [cta][warp][32-column chunk][v][lane]
// float4s; here warp w of a CTA takes one (cta, warp, chunk, column octet) and
// lane l the row that epilogue lane l held, so every load is 512 contiguous
// bytes.  64 CTAs of 8 warps cover one 256 x 512 tile.
__global__ void __launch_bounds__(256)
    gemm_fold_kernel(const __grid_constant__ GemmGroup group, int T) {
    pdl_wait();
    pdl_launch_dependents();
    const int m_tiles = (T + BM2 - 1) / BM2;
    const int lane = threadIdx.x & 31;
    const int tail = blockIdx.x / 64;
    const int item = (blockIdx.x % 64) * 8 + (threadIdx.x >> 5);  // 0..511
    const int vp = item % 4, cc = (item / 4) % (TMEM_COLS2 / 32), qw = (item / 64) % kEpilogueWarps;
    const int rk = item / (4 * (TMEM_COLS2 / 32) * kEpilogueWarps);
    const int lrow = rk * HALF_M + qw * 32 + lane;
    const int c = cc * 32 + vp * 8;  // TMEM column of the octet
    const int lcol = 256 * ((c & 255) >> 7) + 128 * (c >> 8) + (c & 127);
    const TileCoord tc = decode_tile2(group, group.units_full + tail, m_tiles);
    const int row = tc.m0 + lrow, col = tc.n0 + lcol;
    const int N = group.N[tc.p];
    if (row >= T || col >= N) return;
    const int S = group.tail_splits;
    const size_t off = ((size_t)((rk * kEpilogueWarps + qw) * (TMEM_COLS2 / 32) + cc) * 8 + 2 * vp) * 32 + lane;
    const float4* src = reinterpret_cast<const float4*>(group.partials + (size_t)tail * S * BM2 * BN2) + off;
    float a[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    for (int s0 = 0; s0 < S; s0 += 4) {
        float4 v[4][2];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            if (s0 + u < S) {
                const float4* q = src + (size_t)(s0 + u) * (BM2 * BN2 / 4);
                v[u][0] = __ldcg(q);
                v[u][1] = __ldcg(q + 32);
            }
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            if (s0 + u < S) {
                a[0] += v[u][0].x; a[1] += v[u][0].y; a[2] += v[u][0].z; a[3] += v[u][0].w;
                a[4] += v[u][1].x; a[5] += v[u][1].y; a[6] += v[u][1].z; a[7] += v[u][1].w;
            }
        }
    }
    uint4 o;
    o.x = pack_bf16x2(a[0], a[1]);
    o.y = pack_bf16x2(a[2], a[3]);
    o.z = pack_bf16x2(a[4], a[5]);
    o.w = pack_bf16x2(a[6], a[7]);
    *reinterpret_cast<uint4*>(group.Y[tc.p] + (size_t)row * N + col) = o;
}

}  // namespace pair

}  // namespace

size_t gemm_smem_bytes() { return kSmemBytes; }

int gemm_group_tiles(GemmGroup& g, int T, int pair) {
    const int bm = pair ? pair::BM2 : BM, bn = pair ? pair::BN2 : BN;
    const int m_tiles = (T + bm - 1) / bm;
    g.tile_start[0] = 0;
    for (int p = 0; p < g.count; ++p) g.tile_start[p + 1] = g.tile_start[p] + m_tiles * ((g.N[p] + bn - 1) / bn);
    for (int p = g.count + 1; p <= kMaxGroup; ++p) g.tile_start[p] = g.tile_start[g.count];
    g.units_full = g.units = g.tile_start[g.count];
    g.tail_splits = 1;
    g.partials = nullptr;
    return g.tile_start[g.count];
}

size_t gemm_pair_partial_bytes(int num_sms) {
    const int pairs = num_sms / 2 > 0 ? num_sms / 2 : 1;
    return (size_t)pairs * pair::BM2 * pair::BN2 * sizeof(float);
}

// Whole tiles fill every full wave over the pairs; the R tiles of the last,
// partial wave are each cut into s = min(pairs / R, 8) K-ranges (at least one
// K-block each), so that wave takes about 1/s of a tile's time instead of a
// whole one.
cudaError_t launch_gemm_pair(const uint16_t* Xt, int ldT, const GemmGroup& group, const GemmOutMaps& ymaps,
                             const GemmInMaps* imaps, const int32_t* idx, int k, int T, int H, float* partials,
                             int* status, int debug_timeout, int num_sms, cudaStream_t stream) {
    if (group.count < 1 || group.count > kMaxGroup) return cudaErrorInvalidValue;
    auto kern = imaps ? pair::gemm_pair_kernel<true> : pair::gemm_pair_kernel<false>;
    cudaError_t e = ensure_smem_limit(kern, pair::kSmemBytes2);
    if (e != cudaSuccess) return e;
    GemmInMaps no_maps;
    if (!imaps) {
        memset(&no_maps, 0, sizeof no_maps);
        imaps = &no_maps;
    }
    const int tiles = group.tile_start[group.count];
    const int nkb = (k + BK - 1) / BK;
    const int pairs = num_sms / 2 > 0 ? num_sms / 2 : 1;
    GemmGroup g = group;
    g.units_full = g.units = tiles;
    g.tail_splits = 1;
    g.partials = partials;
    const int R = tiles % pairs;
    if (partials && R > 0) {
        // at most 8 ranges: beyond that the fold's reads of the partials cost
        // more than the shorter tail saves
        int s = pairs / R;
        if (s > 8) s = 8;
        if (s > nkb) s = nkb;
        if (s > 1) {
            g.units_full = tiles - R;
            g.tail_splits = s;
            g.units = g.units_full + R * s;
        }
    }
    int clusters = pairs < g.units ? pairs : g.units;
    if (clusters < 1) clusters = 1;
    e = launch_pdl(kern, dim3(2 * clusters), dim3(pair::kThreads2), pair::kSmemBytes2, stream, Xt, ldT, g, ymaps,
                   *imaps, idx, k, T, H, status, debug_timeout);
    if (e != cudaSuccess || g.tail_splits == 1) return e;
    return launch_pdl(pair::gemm_fold_kernel, dim3(R * (pair::BM2 / 4)), dim3(256), 0, stream, g, T);
}

cudaError_t launch_gemm(const CUtensorMap& map_xt, const CUtensorMap& map_wt, const uint16_t* Xt,
                        int ldT, const GemmGroup& group, const int32_t* idx, int k, int T, int H,
                        int* status, int debug_timeout, int tma_gather, int num_sms,
                        cudaStream_t stream) {
    if (group.count < 1 || group.count > kMaxGroup || (tma_gather && group.count != 1))
        return cudaErrorInvalidValue;
    auto kern = tma_gather ? gemm_kernel<true> : gemm_kernel<false>;
    cudaError_t e = ensure_smem_limit(kern, kSmemBytes);
    if (e != cudaSuccess) return e;
    const int tiles = group.tile_start[group.count];
    const int grid = tiles < num_sms ? tiles : num_sms;
    return launch_pdl(kern, dim3(grid), dim3(kThreads), kSmemBytes, stream, map_xt, map_wt, Xt, ldT, group, idx,
                      k, T, H, status, debug_timeout);
}

}  // namespace rmm
