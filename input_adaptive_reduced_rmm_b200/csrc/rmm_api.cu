// rmm_api.cu -- the extern "C" entry points of librmm (declared in rmm.h):
// argument validation, workspace layout, path choice, tensor-map cache and
// launches.  Everything here is host code; all arithmetic runs in the kernels.
#include <math.h>
#include <string.h>

#include <mutex>
#include <unordered_map>

#include "rmm_common.cuh"
#include "rmm_internal.h"

namespace rmm {

cudaError_t ensure_smem_limit_fn(const void* kern, size_t bytes) {
    if (bytes == 0) return cudaSuccess;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) dev = -1;
    static std::mutex mu;
    static std::unordered_map<uint64_t, size_t> done;  // (device, kernel) -> limit set
    const uint64_t key = (reinterpret_cast<uint64_t>(kern) << 8) ^ (uint64_t)(dev & 0xFF);
    {
        std::lock_guard<std::mutex> g(mu);
        auto it = done.find(key);
        if (it != done.end() && it->second >= bytes) return cudaSuccess;
    }
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
    if (e != cudaSuccess) return e;
    std::lock_guard<std::mutex> g(mu);
    size_t& v = done[key];
    if (bytes > v) v = bytes;
    return cudaSuccess;
}

namespace {

constexpr size_t kAlign = 256;
constexpr size_t kStatusBytes = 256;  // status word (int32 at offset 0) + reserved

size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

int num_sms_current() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 148;
    static int cache[64] = {0};
    if (dev >= 0 && dev < 64 && cache[dev] > 0) return cache[dev];
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
        n = 148;
    if (dev >= 0 && dev < 64) cache[dev] = n;
    return n;
}

const rmm_options& opts_or_default(const rmm_options* o) {
    static const rmm_options d = {16, 0, 0, 0, 0, 0, 0, 0, 0, nullptr, nullptr};
    return o ? *o : d;
}

bool opts_valid(const rmm_options* o) {
    if (!o) return true;
    if (o->t_gemv < 0 || o->t_gemv > kGemvMaxT) return false;
    if (o->gemv_splits < 0) return false;
    if (o->gemm_producer < 0 || o->gemm_producer > 2) return false;
    if (o->attn_path < 0 || o->attn_path > 2) return false;
    if (o->block_size < 0) return false;
    if (o->block_score < 0 || o->block_score > 1 || (o->block_score == 1 && o->block_size == 0)) return false;
    if (o->swiglu_pair < 0 || o->swiglu_pair > 1) return false;
    return true;
}

// ---------------------------------------------------------------- layout

struct LinearLayout {
    bool gemv;
    int ldT;           // leading dimension of X^T (GEMM path)
    GemvGroup plan;    // GEMV path
    size_t s32, idx, partials, xt, total;
};

// Workspace layout for `count` products of one activation matrix [T, H] with
// kept count k (k = H gives the largest layout, used by the size queries).
LinearLayout linear_layout(int T, int H, const int* Ns, int count, int k, const rmm_options& o, int sms) {
    LinearLayout L{};
    L.gemv = T <= o.t_gemv;
    size_t off = kStatusBytes;
    L.s32 = off;
    off += align_up((size_t)H * sizeof(uint32_t), kAlign);
    L.idx = off;
    off += align_up(((size_t)H + 2 * kGemmBK) * sizeof(int32_t), kAlign);
    if (L.gemv) {
        memset(&L.plan, 0, sizeof L.plan);
        L.plan.count = count;
        for (int p = 0; p < count; ++p) L.plan.N[p] = Ns[p];
        size_t part = gemv_group_plan(L.plan, T, k, o.gemv_splits, sms);
        if (k == H) part = gemv_partials_bound(L.plan, T, H, o.gemv_splits, sms);  // size query: any k
        L.partials = off;
        off += align_up(part, kAlign);
    } else {
        L.ldT = (T + 7) / 8 * 8;
        L.xt = off;
        off += align_up((size_t)H * L.ldT * sizeof(uint16_t), kAlign);
        L.partials = off;  // fp32 partials of the split last wave (CTA-pair GEMM)
        off += align_up(gemm_pair_partial_bytes(sms), kAlign);
    }
    L.total = off;
    return L;
}

// ---------------------------------------------------------------- tensor maps

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

struct MapKey {
    const void* ptr;
    uint64_t rows, cols, ld, box_rows;
    bool operator==(const MapKey& o) const {
        return ptr == o.ptr && rows == o.rows && cols == o.cols && ld == o.ld && box_rows == o.box_rows;
    }
};
struct MapKeyHash {
    size_t operator()(const MapKey& k) const {
        size_t h = std::hash<const void*>()(k.ptr);
        h ^= std::hash<uint64_t>()(k.rows * 1000003ull + k.cols * 7919ull + k.ld * 31ull + k.box_rows) + 0x9e3779b9 +
             (h << 6) + (h >> 2);
        return h;
    }
};

// A tiled map over a bf16 matrix [rows, cols] (leading dimension ld elements):
// box = box_rows rows x 64 columns (128 bytes), 128-byte swizzle; loads read
// zeros and stores skip elements outside the matrix.  Cached by (pointer,
// shape, box).  box_rows 1 is the row-gather map of the TMA producer; 32 the
// output tile of one GEMM epilogue warp.
bool tiled_map(const void* base, uint64_t rows, uint64_t cols, uint64_t ld, uint32_t box_rows, CUtensorMap* out) {
    static std::mutex mu;
    static std::unordered_map<MapKey, CUtensorMap, MapKeyHash> cache;
    const MapKey key{base, rows, cols, ld, box_rows};
    {
        std::lock_guard<std::mutex> g(mu);
        auto it = cache.find(key);
        if (it != cache.end()) {
            *out = it->second;
            return true;
        }
    }
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    CUtensorMap m;
    memset(&m, 0, sizeof m);
    const cuuint64_t dims[2] = {cols, rows};
    const cuuint64_t strides[1] = {ld * sizeof(uint16_t)};
    const cuuint32_t box[2] = {64, box_rows};
    const cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(&m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides,
                    box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return false;
    std::lock_guard<std::mutex> g(mu);
    if (cache.size() > 4096) cache.clear();
    cache[key] = m;
    *out = m;
    return true;
}

rmm_status cuda_status(cudaError_t e) { return e == cudaSuccess ? RMM_OK : RMM_ERR_CUDA; }

bool row_gather_map(const void* base, uint64_t rows, uint64_t cols, uint64_t ld, CUtensorMap* out) {
    return tiled_map(base, rows, cols, ld, 1, out);
}

bool group_args_ok(const void* X, int T, int H, int count, const void* const* Wts, const int* Ns,
                   void* const* Ys) {
    if (!X || !Wts || !Ns || !Ys || count < 1 || count > kMaxGroup) return false;
    if (T < 1 || T > (1 << 20) || H < 1 || H > 65535 || !aligned16(X)) return false;
    for (int p = 0; p < count; ++p) {
        if (!Wts[p] || !Ys[p] || Ns[p] < 8 || Ns[p] % 8 != 0) return false;
        if (!aligned16(Wts[p]) || !aligned16(Ys[p])) return false;
    }
    return true;
}

// The product step for every member of the group, on the chosen path.
rmm_status run_product_kernels(const void* X, int T, int H, int count, const void* const* Wts,
                               const int* Ns, void* const* Ys, const int32_t* idx_padded, int k,
                               uint8_t* ws, const LinearLayout& L, const rmm_options& o,
                               cudaStream_t s) {
    int* status = reinterpret_cast<int*>(ws);
    const int sms = num_sms_current();
    // the gated-MLP epilogue when it is not fused into the GEMV fold:
    // Ys[0] = bf16(silu(Ys[0]) * Ys[1]) after the products
    auto swiglu_after = [&]() -> rmm_status {
        return cuda_status(launch_swiglu(static_cast<const uint16_t*>(Ys[0]), static_cast<const uint16_t*>(Ys[1]),
                                         (size_t)T * Ns[0], static_cast<uint16_t*>(Ys[0]), sms, s));
    };
    if (L.gemv) {
        GemvGroup g = L.plan;
        for (int p = 0; p < count; ++p) {
            g.Wt[p] = static_cast<const uint16_t*>(Wts[p]);
            g.Y[p] = static_cast<uint16_t*>(Ys[p]);
        }
        g.swiglu = o.swiglu_pair;  // fused into the fold of the split partials
        (void)status;
        rmm_status st = cuda_status(launch_gemv(static_cast<const uint16_t*>(X), T, H, idx_padded, k, g,
                                                reinterpret_cast<float*>(ws + L.partials), sms, s));
        if (st == RMM_OK && o.swiglu_pair && g.splits[0] == 1) st = swiglu_after();  // no fold to fuse into
        return st;
    }
    if (o.swiglu_pair) {
        rmm_options o2 = o;
        o2.swiglu_pair = 0;
        rmm_status st = run_product_kernels(X, T, H, count, Wts, Ns, Ys, idx_padded, k, ws, L, o2, s);
        return st == RMM_OK ? swiglu_after() : st;
    }
    if (o.gemm_producer == 1 && count != 1) return RMM_ERR_UNSUPPORTED;
    GemmGroup g;
    memset(&g, 0, sizeof g);
    g.count = count;
    for (int p = 0; p < count; ++p) {
        g.Wt[p] = static_cast<const uint16_t*>(Wts[p]);
        g.Y[p] = static_cast<uint16_t*>(Ys[p]);
        g.N[p] = Ns[p];
    }
    if (o.gemm_producer == 0) {  // default: CTA-pair tcgen05 GEMM
        gemm_group_tiles(g, T, 1);
        GemmOutMaps ym;
        memset(&ym, 0, sizeof ym);
        for (int p = 0; p < count; ++p)
            if (!tiled_map(Ys[p], (uint64_t)T, (uint64_t)Ns[p], (uint64_t)Ns[p], 32, &ym.m[p])) return RMM_ERR_CUDA;
        const uint16_t* xt = reinterpret_cast<const uint16_t*>(ws + L.xt);
        // block-granular sets in runs of 64 slices: every K-block is 64 contiguous
        // rows, loaded by TMA tile copies
        GemmInMaps im;
        const bool tma_rows = o.block_size > 0 && o.block_size % kGemmBK == 0;
        if (tma_rows) {
            memset(&im, 0, sizeof im);
            if (!tiled_map(xt, (uint64_t)H, (uint64_t)T, (uint64_t)L.ldT, kGemmBK, &im.xt)) return RMM_ERR_CUDA;
            for (int p = 0; p < count; ++p)
                if (!tiled_map(Wts[p], (uint64_t)H, (uint64_t)Ns[p], (uint64_t)Ns[p], kGemmBK, &im.wt[p]))
                    return RMM_ERR_CUDA;
        }
        return cuda_status(launch_gemm_pair(xt, L.ldT, g, ym, tma_rows ? &im : nullptr, idx_padded, k, T, H,
                                            reinterpret_cast<float*>(ws + L.partials), status,
                                            o.debug_timeout_test, sms, s));
    }
    gemm_group_tiles(g, T, 0);
    CUtensorMap mx, mw;
    memset(&mx, 0, sizeof mx);
    memset(&mw, 0, sizeof mw);
    const uint16_t* xt = reinterpret_cast<const uint16_t*>(ws + L.xt);
    if (o.gemm_producer == 1) {
        if (!row_gather_map(xt, (uint64_t)H, (uint64_t)T, (uint64_t)L.ldT, &mx)) return RMM_ERR_CUDA;
        if (!row_gather_map(Wts[0], (uint64_t)H, (uint64_t)Ns[0], (uint64_t)Ns[0], &mw)) return RMM_ERR_CUDA;
    }
    return cuda_status(launch_gemm(mx, mw, xt, L.ldT, g, idx_padded, k, T, H, status,
                                   o.debug_timeout_test, o.gemm_producer == 1, sms, s));
}

// Records a caller's timing event; while the stream is being captured into a
// CUDA graph the record becomes an event node of the graph (so a replay times
// the product kernels too).
cudaError_t record_product_event(void* ev, cudaStream_t s) {
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(s, &cs) != cudaSuccess) return cudaErrorUnknown;
    return cudaEventRecordWithFlags(static_cast<cudaEvent_t>(ev), s,
                                    cs == cudaStreamCaptureStatusActive ? cudaEventRecordExternal
                                                                        : cudaEventRecordDefault);
}

rmm_status run_products(const void* X, int T, int H, int count, const void* const* Wts, const int* Ns,
                        void* const* Ys, const int32_t* idx_padded, int k, uint8_t* ws,
                        const LinearLayout& L, const rmm_options& o, cudaStream_t s) {
    if (o.product_event_begin && record_product_event(o.product_event_begin, s) != cudaSuccess) return RMM_ERR_CUDA;
    rmm_status st = run_product_kernels(X, T, H, count, Wts, Ns, Ys, idx_padded, k, ws, L, o, s);
    if (st == RMM_OK && o.product_event_end && record_product_event(o.product_event_end, s) != cudaSuccess)
        return RMM_ERR_CUDA;
    return st;
}

// score (+ X^T) -> kept set -> products, shared by rmm_linear and rmm_linear_group.
rmm_status linear_group(const void* X, int T, int H, double r, int count, const void* const* Wts,
                        const int* Ns, void* const* Ys, int32_t* idx_out, void* workspace,
                        size_t workspace_bytes, rmm_stream_t stream, const rmm_options* options) {
    if (!group_args_ok(X, T, H, count, Wts, Ns, Ys) || !opts_valid(options)) return RMM_ERR_INVALID_ARG;
    const rmm_options& o = opts_or_default(options);
    if (o.swiglu_pair && (count != 2 || Ns[0] != Ns[1])) return RMM_ERR_INVALID_ARG;
    const int bsz = o.block_size;
    if (!block_size_ok(H, bsz)) return RMM_ERR_UNSUPPORTED;
    const bool mean_blocks = bsz > 0 && o.block_score == 1;
    if (mean_blocks && T > kGemvMaxT) return RMM_ERR_UNSUPPORTED;
    // kept slices: ceil(r*H), or ceil(r*H/block) whole blocks
    const int kb = bsz ? rmm_k_for(H / bsz, r) : 0;
    const int k = bsz ? (kb < 1 ? -1 : kb * bsz) : rmm_k_for(H, r);
    if (k < 1) return RMM_ERR_INVALID_ARG;
    const int sms = num_sms_current();
    const LinearLayout L = linear_layout(T, H, Ns, count, k, o, sms);
    if (!workspace || workspace_bytes < L.total || !aligned16(workspace)) return RMM_ERR_WORKSPACE;
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    uint32_t* s32 = reinterpret_cast<uint32_t*>(ws + L.s32);
    int32_t* idx = reinterpret_cast<int32_t*>(ws + L.idx);
    const int pad_to = (k + kGemmBK - 1) / kGemmBK * kGemmBK;
    cudaError_t e;
    if (bsz) {
        // block-granular: the score pass (with X^T on the GEMM path; not needed
        // for mean-magnitude blocks on the GEMV path), then the blocks
        e = cudaSuccess;
        if (!mean_blocks || !L.gemv)
            e = launch_score(static_cast<const uint16_t*>(X), T, H, s32,
                             L.gemv ? nullptr : reinterpret_cast<uint16_t*>(ws + L.xt), L.ldT, sms, s);
        if (e == cudaSuccess)
            e = launch_block_select(s32, mean_blocks ? static_cast<const uint16_t*>(X) : nullptr, T, H, bsz, kb, idx,
                                    idx_out, nullptr, s);
        if (e == cudaSuccess && pad_to > k) e = launch_pad_idx(idx, k, H, idx, pad_to, s);
    } else if (L.gemv && k == H) {
        // every slice kept (ratio 1): the kept list is 0..H-1 whatever the
        // scores, so neither score nor select runs, and the GEMV reads the
        // identity list implicitly; the list is written only when asked for
        e = idx_out ? launch_pad_idx(nullptr, k, H, idx, pad_to, s, idx_out) : cudaSuccess;
        if (e != cudaSuccess) return RMM_ERR_CUDA;
        return run_products(X, T, H, count, Wts, Ns, Ys, nullptr, k, ws, L, o, s);
    } else if (L.gemv && T == 1) {
        // one token: the select kernel reads the score straight from X
        e = launch_select(static_cast<const uint16_t*>(X), T, nullptr, 0, H, k, idx, pad_to, idx_out, nullptr, s);
    } else if (L.gemv) {
        // a few tokens: the score pass spreads the fold over the GPU, no X^T
        e = launch_score(static_cast<const uint16_t*>(X), T, H, s32, nullptr, 0, sms, s);
        if (e == cudaSuccess) e = launch_select(nullptr, 0, s32, 1, H, k, idx, pad_to, idx_out, nullptr, s);
    } else {
        e = launch_score(static_cast<const uint16_t*>(X), T, H, s32, reinterpret_cast<uint16_t*>(ws + L.xt), L.ldT,
                         sms, s);
        if (e == cudaSuccess) e = launch_select(nullptr, 0, s32, 1, H, k, idx, pad_to, idx_out, nullptr, s);
    }
    if (e != cudaSuccess) return RMM_ERR_CUDA;
    return run_products(X, T, H, count, Wts, Ns, Ys, idx, k, ws, L, o, s);
}

}  // namespace

// A 3-D tiled map over a bf16 tensor [n2][n1][n0] (innermost n0, row stride
// ld1 elements, plane stride ld2 elements): box = 64 x box1 x 1 elements,
// 128-byte swizzle; loads read zeros outside the tensor.  Cached like the
// 2-D maps.
bool tiled_map_3d(const void* base, uint64_t n0, uint64_t n1, uint64_t n2, uint64_t ld1, uint64_t ld2,
                  uint32_t box1, CUtensorMap* out) {
    struct Key3 {
        const void* ptr;
        uint64_t n0, n1, n2, ld1, ld2, box1;
        bool operator==(const Key3& o) const {
            return ptr == o.ptr && n0 == o.n0 && n1 == o.n1 && n2 == o.n2 && ld1 == o.ld1 && ld2 == o.ld2 &&
                   box1 == o.box1;
        }
    };
    struct Hash3 {
        size_t operator()(const Key3& k) const {
            size_t h = std::hash<const void*>()(k.ptr);
            h ^= std::hash<uint64_t>()(((k.n0 * 1000003ull + k.n1) * 7919ull + k.n2) * 31ull + k.ld1 * 131ull +
                                       k.ld2 * 17ull + k.box1) + 0x9e3779b9 + (h << 6) + (h >> 2);
            return h;
        }
    };
    static std::mutex mu;
    static std::unordered_map<Key3, CUtensorMap, Hash3> cache;
    const Key3 key{base, n0, n1, n2, ld1, ld2, box1};
    {
        std::lock_guard<std::mutex> g(mu);
        auto it = cache.find(key);
        if (it != cache.end()) {
            *out = it->second;
            return true;
        }
    }
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    CUtensorMap m;
    memset(&m, 0, sizeof m);
    const cuuint64_t dims[3] = {n0, n1, n2};
    const cuuint64_t strides[2] = {ld1 * sizeof(uint16_t), ld2 * sizeof(uint16_t)};
    const cuuint32_t box[3] = {64, box1, 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = fn(&m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return false;
    std::lock_guard<std::mutex> g(mu);
    if (cache.size() > 4096) cache.clear();
    cache[key] = m;
    *out = m;
    return true;
}

}  // namespace rmm

using namespace rmm;

extern "C" {

const char* rmm_status_string(rmm_status s) {
    switch (s) {
        case RMM_OK: return "RMM_OK";
        case RMM_ERR_INVALID_ARG: return "RMM_ERR_INVALID_ARG";
        case RMM_ERR_UNSUPPORTED: return "RMM_ERR_UNSUPPORTED";
        case RMM_ERR_WORKSPACE: return "RMM_ERR_WORKSPACE";
        case RMM_ERR_CUDA: return "RMM_ERR_CUDA";
        case RMM_ERR_TIMEOUT: return "RMM_ERR_TIMEOUT";
    }
    return "RMM_ERR_UNKNOWN";
}

int rmm_k_for(int H, double r) {
    if (H < 1 || !(r > 0.0) || !(r <= 1.0)) return -1;
    double kk = ceil(r * (double)H);
    long k = (long)kk;
    if (k < 1) k = 1;
    if (k > H) k = H;
    return (int)k;
}

rmm_status rmm_workspace_init(void* ws, size_t bytes, rmm_stream_t stream) {
    if (!ws || bytes < kStatusBytes) return RMM_ERR_INVALID_ARG;
    return cuda_status(cudaMemsetAsync(ws, 0, bytes, static_cast<cudaStream_t>(stream)));
}

rmm_status rmm_get_status(void* ws, rmm_stream_t stream) {
    if (!ws) return RMM_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (cudaStreamSynchronize(s) != cudaSuccess) return RMM_ERR_CUDA;
    int code = 0;
    if (cudaMemcpy(&code, ws, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return RMM_ERR_CUDA;
    if (code != 0) {
        if (cudaMemsetAsync(ws, 0, sizeof(int), s) != cudaSuccess) return RMM_ERR_CUDA;
        if (cudaStreamSynchronize(s) != cudaSuccess) return RMM_ERR_CUDA;
    }
    return static_cast<rmm_status>(code);
}

rmm_status rmm_transpose_weight(const void* W, void* Wt, int N, int H, rmm_stream_t stream) {
    if (!W || !Wt || N < 1 || H < 1) return RMM_ERR_INVALID_ARG;
    const char* a = static_cast<const char*>(W);
    const char* b = static_cast<const char*>(Wt);
    const size_t bytes = (size_t)N * H * sizeof(uint16_t);
    if (a < b + bytes && b < a + bytes) return RMM_ERR_INVALID_ARG;
    return cuda_status(launch_transpose(static_cast<const uint16_t*>(W), static_cast<uint16_t*>(Wt),
                                        N, H, static_cast<cudaStream_t>(stream)));
}

size_t rmm_linear_workspace_bytes(int T, int H, int N, const rmm_options* options) {
    if (T < 1 || H < 1 || N < 1 || !opts_valid(options)) return 0;
    const rmm_options& o = opts_or_default(options);
    return linear_layout(T, H, &N, 1, H, o, num_sms_current()).total;
}

size_t rmm_linear_group_workspace_bytes(int T, int H, int count, const int* Ns, const rmm_options* options) {
    if (T < 1 || H < 1 || count < 1 || count > kMaxGroup || !Ns || !opts_valid(options)) return 0;
    for (int p = 0; p < count; ++p)
        if (Ns[p] < 1) return 0;
    const rmm_options& o = opts_or_default(options);
    return linear_layout(T, H, Ns, count, H, o, num_sms_current()).total;
}

rmm_status rmm_linear(const void* X, const void* Wt, int T, int H, int N, double r, void* Y,
                      int32_t* idx_out, void* workspace, size_t workspace_bytes,
                      rmm_stream_t stream, const rmm_options* options) {
    const void* Wts[1] = {Wt};
    void* Ys[1] = {Y};
    return linear_group(X, T, H, r, 1, Wts, &N, Ys, idx_out, workspace, workspace_bytes, stream, options);
}

rmm_status rmm_linear_group(const void* X, int T, int H, double r, int count, const void* const* Wts,
                            const int* Ns, void* const* Ys, int32_t* idx_out, void* workspace,
                            size_t workspace_bytes, rmm_stream_t stream, const rmm_options* options) {
    return linear_group(X, T, H, r, count, Wts, Ns, Ys, idx_out, workspace, workspace_bytes, stream, options);
}

rmm_status rmm_score(const void* X, int T, int H, uint32_t* s_out, void* workspace,
                     size_t workspace_bytes, rmm_stream_t stream) {
    if (!X || !s_out || T < 1 || H < 1 || H > 65535 || !aligned16(X)) return RMM_ERR_INVALID_ARG;
    const size_t off_s32 = kStatusBytes;
    const size_t off_idx = off_s32 + align_up((size_t)H * 4, kAlign);
    const size_t need = off_idx + align_up(((size_t)H + 2 * kGemmBK) * 4, kAlign);
    if (!workspace || workspace_bytes < need) return RMM_ERR_WORKSPACE;
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    uint32_t* s32 = reinterpret_cast<uint32_t*>(ws + off_s32);
    int32_t* idx = reinterpret_cast<int32_t*>(ws + off_idx);
    cudaError_t e = launch_score(static_cast<const uint16_t*>(X), T, H, s32, nullptr, 0, num_sms_current(), s);
    if (e != cudaSuccess) return RMM_ERR_CUDA;
    return cuda_status(launch_select(nullptr, 0, s32, 1, H, H, idx, H, nullptr, s_out, s));
}

rmm_status rmm_select(const uint32_t* sc, int H, int k, int32_t* idx_out, void* /*workspace*/,
                      size_t /*workspace_bytes*/, rmm_stream_t stream) {
    if (!sc || !idx_out || H < 1 || H > 65535 || k < 1 || k > H) return RMM_ERR_INVALID_ARG;
    return cuda_status(launch_select(nullptr, 0, const_cast<uint32_t*>(sc), 0, H, k, idx_out, k, nullptr, nullptr,
                                     static_cast<cudaStream_t>(stream)));
}

rmm_status rmm_gemm_reduced(const void* X, const void* Wt, const int32_t* idx, int k, int T, int H,
                            int N, void* Y, void* workspace, size_t workspace_bytes,
                            rmm_stream_t stream, const rmm_options* options) {
    const void* Wts[1] = {Wt};
    void* Ys[1] = {Y};
    if (!group_args_ok(X, T, H, 1, Wts, &N, Ys) || !idx || k < 1 || k > H || !opts_valid(options))
        return RMM_ERR_INVALID_ARG;
    const rmm_options& o = opts_or_default(options);
    if (o.swiglu_pair) return RMM_ERR_INVALID_ARG;  // a pair epilogue needs a group of two
    const int sms = num_sms_current();
    const LinearLayout L = linear_layout(T, H, &N, 1, k, o, sms);
    if (!workspace || workspace_bytes < L.total || !aligned16(workspace)) return RMM_ERR_WORKSPACE;
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (L.gemv) return run_products(X, T, H, 1, Wts, &N, Ys, idx, k, ws, L, o, s);
    // GEMM path: X^T (written by the score pass, scores not accumulated) and
    // the kept list padded to the K-block
    cudaError_t e = launch_score(static_cast<const uint16_t*>(X), T, H, nullptr,
                                 reinterpret_cast<uint16_t*>(ws + L.xt), L.ldT, sms, s);
    if (e != cudaSuccess) return RMM_ERR_CUDA;
    int32_t* idx_pad = reinterpret_cast<int32_t*>(ws + L.idx);
    const int pad_to = (k + kGemmBK - 1) / kGemmBK * kGemmBK;
    e = launch_pad_idx(idx, k, H, idx_pad, pad_to, s);
    if (e != cudaSuccess) return RMM_ERR_CUDA;
    return run_products(X, T, H, 1, Wts, &N, Ys, idx_pad, k, ws, L, o, s);
}

size_t rmm_attn_workspace_bytes(int B, int Hq, int Hkv, int T, int L, int d,
                                const rmm_options* options) {
    if (B < 1 || Hq < 1 || Hkv < 1 || T < 1 || L < T || d != 128 || Hq % Hkv != 0 ||
        !opts_valid(options))
        return 0;
    const rmm_options& o = opts_or_default(options);
    const AttnPlan p = attn_plan(B, Hq, Hkv, T, L, o.attn_per_query_head, num_sms_current());
    return kStatusBytes + 2 * align_up((size_t)B * p.nsets * d * sizeof(int32_t), kAlign) +
           align_up(attn_partials_bytes(p, B, Hq, T), kAlign);
}

rmm_status rmm_attn_qk(const void* Q, const void* Kt, const void* V, int B, int Hq, int Hkv, int T,
                       int L, int ldL, int d, double r, int causal, float scale, void* O,
                       int32_t* idx_out, void* workspace, size_t workspace_bytes,
                       rmm_stream_t stream, const rmm_options* options) {
    if (!Q || !Kt || !V || !O || B < 1 || Hq < 1 || Hkv < 1 || T < 1 || L < T || ldL < L ||
        ldL % 8 != 0 || Hq % Hkv != 0 || !opts_valid(options))
        return RMM_ERR_INVALID_ARG;
    if (!aligned16(Q) || !aligned16(Kt) || !aligned16(V) || !aligned16(O)) return RMM_ERR_INVALID_ARG;
    if (!(scale > 0.0f) || !isfinite(scale)) return RMM_ERR_INVALID_ARG;
    if (d != 128) return RMM_ERR_UNSUPPORTED;
    const int k = rmm_k_for(d, r);
    if (k < 1) return RMM_ERR_INVALID_ARG;
    const rmm_options& o = opts_or_default(options);
    if (!o.attn_per_query_head && Hq / Hkv > 8) return RMM_ERR_UNSUPPORTED;
    const AttnPlan p = attn_plan(B, Hq, Hkv, T, L, o.attn_per_query_head, num_sms_current());
    // workspace: status | kept sets | per-set score vectors (zero between calls) | split partials
    const size_t idx_bytes = align_up((size_t)B * p.nsets * d * sizeof(int32_t), kAlign);
    const size_t need = kStatusBytes + 2 * idx_bytes + align_up(attn_partials_bytes(p, B, Hq, T), kAlign);
    if (!workspace || workspace_bytes < need || !aligned16(workspace)) return RMM_ERR_WORKSPACE;
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    int32_t* idx = idx_out ? idx_out : reinterpret_cast<int32_t*>(ws + kStatusBytes);
    uint32_t* sc = reinterpret_cast<uint32_t*>(ws + kStatusBytes + idx_bytes);
    float* partials = reinterpret_cast<float*>(ws + kStatusBytes + 2 * idx_bytes);
    return cuda_status(launch_attn(static_cast<const uint16_t*>(Q), static_cast<const uint16_t*>(Kt),
                                   static_cast<const uint16_t*>(V), B, Hq, Hkv, T, L, ldL, k,
                                   causal ? 1 : 0, scale, o.attn_per_query_head,
                                   static_cast<uint16_t*>(O), idx, partials, sc, reinterpret_cast<int*>(ws),
                                   o.attn_path, p, static_cast<cudaStream_t>(stream)));
}

// ---------------------------------------------------------------- context blocks

rmm_status rmm_ctx_block_means(const void* Kt, int B, int Hkv, int d, int L, int ldL, int block, int blk_begin,
                               int blk_end, float* means, rmm_stream_t stream) {
    if (!Kt || !means || B < 1 || Hkv < 1 || L < 1 || ldL < L || ldL % 8 != 0 || !ctx_block_ok(block))
        return RMM_ERR_INVALID_ARG;
    if (!aligned16(Kt) || !aligned16(means)) return RMM_ERR_INVALID_ARG;
    if (blk_begin < 0 || blk_end <= blk_begin || blk_end > (L + block - 1) / block) return RMM_ERR_INVALID_ARG;
    if (d != 128) return RMM_ERR_UNSUPPORTED;
    return cuda_status(launch_ctx_means(static_cast<const uint16_t*>(Kt), B, Hkv, L, ldL, block, blk_begin, blk_end,
                                        means, static_cast<cudaStream_t>(stream)));
}

namespace {

// workspace of rmm_attn_ctx: status | idx | dims scores (zero between calls) |
// block keys | kept blocks | split partials
struct CtxLayout {
    size_t idx, sc, keys, blocks, partials, total;
};

CtxLayout ctx_layout(int B, int Hq, int T, int d, int nblk, int kc, const AttnPlan& p) {
    CtxLayout c;
    size_t off = kStatusBytes;
    c.idx = off;
    off += align_up((size_t)B * p.nsets * d * sizeof(int32_t), kAlign);
    c.sc = off;
    off += align_up((size_t)B * p.nsets * d * sizeof(uint32_t), kAlign);
    c.keys = off;
    off += align_up((size_t)B * p.nsets * nblk * sizeof(uint32_t), kAlign);
    c.blocks = off;
    off += align_up((size_t)B * p.nsets * kc * sizeof(int32_t), kAlign);
    c.partials = off;
    off += align_up(attn_partials_bytes(p, B, Hq, T), kAlign);
    c.total = off;
    return c;
}

}  // namespace

size_t rmm_attn_ctx_workspace_bytes(int B, int Hq, int Hkv, int T, int L, int d, int block, double r_ctx,
                                    const rmm_options* options) {
    if (B < 1 || Hq < 1 || Hkv < 1 || T < 1 || L < T || d != 128 || Hq % Hkv != 0 || !ctx_block_ok(block) ||
        !opts_valid(options))
        return 0;
    const int nblk = (L + block - 1) / block;
    const int kc = rmm_k_for(nblk, r_ctx);
    if (kc < 1) return 0;
    const rmm_options& o = opts_or_default(options);
    const AttnPlan p = attn_plan(B, Hq, Hkv, T, kc * block, o.attn_per_query_head, num_sms_current());
    return ctx_layout(B, Hq, T, d, nblk, kc, p).total;
}

rmm_status rmm_attn_ctx(const void* Q, const void* Kt, const void* V, const float* means, int B, int Hq, int Hkv,
                        int T, int L, int ldL, int d, double r, double r_ctx, int block, int causal, float scale,
                        void* O, int32_t* idx_out, int32_t* blocks_out, void* workspace, size_t workspace_bytes,
                        rmm_stream_t stream, const rmm_options* options) {
    if (!Q || !Kt || !V || !means || !O || B < 1 || Hq < 1 || Hkv < 1 || T < 1 || L < T || ldL < L ||
        ldL % 8 != 0 || Hq % Hkv != 0 || !ctx_block_ok(block) || !opts_valid(options))
        return RMM_ERR_INVALID_ARG;
    if (!aligned16(Q) || !aligned16(Kt) || !aligned16(V) || !aligned16(O) || !aligned16(means))
        return RMM_ERR_INVALID_ARG;
    if (!(scale > 0.0f) || !isfinite(scale)) return RMM_ERR_INVALID_ARG;
    if (d != 128) return RMM_ERR_UNSUPPORTED;
    const int k = rmm_k_for(d, r);
    const int nblk = (L + block - 1) / block;
    const int kc = rmm_k_for(nblk, r_ctx);
    if (k < 1 || kc < 1) return RMM_ERR_INVALID_ARG;
    const rmm_options& o = opts_or_default(options);
    if (T > kCtxMaxT || nblk > kCtxMaxBlocks || (!o.attn_per_query_head && Hq / Hkv > 8))
        return RMM_ERR_UNSUPPORTED;
    const AttnPlan p = attn_plan(B, Hq, Hkv, T, kc * block, o.attn_per_query_head, num_sms_current());
    const CtxLayout c = ctx_layout(B, Hq, T, d, nblk, kc, p);
    if (!workspace || workspace_bytes < c.total || !aligned16(workspace)) return RMM_ERR_WORKSPACE;
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    int32_t* idx = idx_out ? idx_out : reinterpret_cast<int32_t*>(ws + c.idx);
    int32_t* blocks = blocks_out ? blocks_out : reinterpret_cast<int32_t*>(ws + c.blocks);
    return cuda_status(launch_attn_ctx(
        static_cast<const uint16_t*>(Q), static_cast<const uint16_t*>(Kt), static_cast<const uint16_t*>(V), means, B,
        Hq, Hkv, T, L, ldL, k, block, kc, causal ? 1 : 0, scale, o.attn_per_query_head, static_cast<uint16_t*>(O),
        idx, reinterpret_cast<uint32_t*>(ws + c.sc), reinterpret_cast<uint32_t*>(ws + c.keys), blocks,
        reinterpret_cast<float*>(ws + c.partials), p, static_cast<cudaStream_t>(stream)));
}

rmm_status rmm_add_rmsnorm(const void* X, const void* R, int T, int H, float eps, const void* weight, void* Hsum,
                           void* Y, rmm_stream_t stream) {
    if (!X || (!Hsum && !Y) || T < 1 || H < 8 || H % 8 != 0 || H > 16384 || !(eps >= 0.0f)) return RMM_ERR_INVALID_ARG;
    if (!aligned16(X) || (R && !aligned16(R)) || (weight && !aligned16(weight)) || (Hsum && !aligned16(Hsum)) ||
        (Y && !aligned16(Y)))
        return RMM_ERR_INVALID_ARG;
    return cuda_status(launch_add_rmsnorm(static_cast<const uint16_t*>(X), static_cast<const uint16_t*>(R), T, H, eps,
                                          static_cast<const uint16_t*>(weight), static_cast<uint16_t*>(Hsum),
                                          static_cast<uint16_t*>(Y), static_cast<cudaStream_t>(stream)));
}

rmm_status rmm_swiglu(const void* G, const void* U, int64_t n, void* Out, rmm_stream_t stream) {
    if (!G || !U || !Out || n < 8 || n % 8 != 0) return RMM_ERR_INVALID_ARG;
    if (!aligned16(G) || !aligned16(U) || !aligned16(Out)) return RMM_ERR_INVALID_ARG;
    return cuda_status(launch_swiglu(static_cast<const uint16_t*>(G), static_cast<const uint16_t*>(U), (size_t)n,
                                     static_cast<uint16_t*>(Out), num_sms_current(),
                                     static_cast<cudaStream_t>(stream)));
}

rmm_status rmm_qkv_heads(const void* Yq, const void* Yk, const void* Yv, int T, int Hq, int Hkv, int d, void* Q,
                         void* Kt, void* V, int ldL, int L0, rmm_stream_t stream) {
    if (!Yq || !Yk || !Yv || !Q || !Kt || !V || T < 1 || Hq < 1 || Hkv < 1 || L0 < 0 || L0 + T > ldL)
        return RMM_ERR_INVALID_ARG;
    if (d != 128) return RMM_ERR_UNSUPPORTED;
    if (!aligned16(Yq) || !aligned16(Yk) || !aligned16(Yv) || !aligned16(Q) || !aligned16(V)) return RMM_ERR_INVALID_ARG;
    return cuda_status(launch_qkv_heads(static_cast<const uint16_t*>(Yq), static_cast<const uint16_t*>(Yk),
                                        static_cast<const uint16_t*>(Yv), T, Hq, Hkv, static_cast<uint16_t*>(Q),
                                        static_cast<uint16_t*>(Kt), static_cast<uint16_t*>(V), ldL, L0,
                                        static_cast<cudaStream_t>(stream)));
}

rmm_status rmm_heads_to_tokens(const void* O, int Hq, int T, int d, void* A, rmm_stream_t stream) {
    if (!O || !A || Hq < 1 || T < 1) return RMM_ERR_INVALID_ARG;
    if (d != 128) return RMM_ERR_UNSUPPORTED;
    if (!aligned16(O) || !aligned16(A)) return RMM_ERR_INVALID_ARG;
    return cuda_status(launch_heads_to_tokens(static_cast<const uint16_t*>(O), Hq, T, static_cast<uint16_t*>(A),
                                              num_sms_current(), static_cast<cudaStream_t>(stream)));
}

rmm_status rmm_selftest_exp2_fma(const float* x, float* y, int n, rmm_stream_t stream) {
    if (!x || !y || n < 1) return RMM_ERR_INVALID_ARG;
    return cuda_status(launch_exp2_fma(x, y, n, static_cast<cudaStream_t>(stream)));
}

}  // extern "C"
