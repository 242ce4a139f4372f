/*
 * rmm.h -- C ABI of librmm: Reduced Matrix Multiplication (RMM) on B200 (sm_100a).
 *
 * The method (Reduced Matrix Multiplication: Input-Adaptive Matrix-Product
 * Reduction for LLM Inference, Lan, Li, Zhou -- abstract): a training-free,
 * input-adaptive reduction of each Transformer matrix product: the slices
 * of the contraction dimension that the current input makes most significant
 * are kept, their share set by one retention ratio r.  For a projection Y = X W^T (X [T,H] activations,
 * W [N,H] weights; cf-1.com post on input-adaptive matrix-product reduction,
 * §2) the library
 *   1. scores every contraction index h by s_h = max_t |X[t,h]| (post §5.1:
 *      a cheap score from the current activations),
 *   2. keeps the top k = ceil(r*H) indices S, ties going to the lower index,
 *      emitted in ascending order (post §5.2, and the §6.1 demo's sort after
 *      top-k),
 *   3. computes Y ~= X[:,S] W[:,S]^T (post §5.3: the smaller dense product)
 *      without writing any compacted copy of X or W to memory.
 * Attention's Q K^T is reduced the same way along the head dimension (post
 * §3.3: reduce inside heads), followed by an unreduced softmax(.) V.
 *
 * Conventions for every entry point:
 *   - All tensors are device pointers owned by the caller; the library never
 *     allocates or frees memory and never synchronises, except
 *     rmm_get_status().  Work is enqueued on `stream` (a cudaStream_t; NULL =
 *     the legacy default stream) and runs asynchronously.
 *   - bf16 tensors are passed as `void*` holding IEEE bfloat16 bit patterns,
 *     row-major with the stated leading dimension.
 *   - Argument errors are detected on the host before anything is launched
 *     and returned as RMM_ERR_INVALID_ARG / RMM_ERR_UNSUPPORTED /
 *     RMM_ERR_WORKSPACE; a failed launch returns RMM_ERR_CUDA.
 *   - Device-side errors (a bounded wait that ran out) are written to a status
 *     word at the start of the workspace and read by rmm_get_status().
 *   - Inputs must be finite; NaN or Inf in X or Q gives an unspecified kept set.
 *   - Workspaces must be zero-filled once before first use (rmm_workspace_init
 *     does this); the library leaves them reusable after every successful call.
 *     One workspace must not be used by two calls that may run concurrently.
 */
#ifndef RMM_H_
#define RMM_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* A cudaStream_t, passed opaquely so that this header needs no CUDA headers. */
typedef void* rmm_stream_t;

typedef enum {
    RMM_OK = 0,
    RMM_ERR_INVALID_ARG = 1, /* null pointer, bad size, r outside (0,1], misaligned pointer */
    RMM_ERR_UNSUPPORTED = 2, /* a valid shape the library does not handle (e.g. d != 128) */
    RMM_ERR_WORKSPACE = 3,   /* workspace null or smaller than the *_workspace_bytes() query */
    RMM_ERR_CUDA = 4,        /* a CUDA launch or runtime call failed */
    RMM_ERR_TIMEOUT = 5      /* a bounded device-side wait ran out (reported by rmm_get_status) */
} rmm_status;

/* Optional knobs; pass NULL for the defaults. */
typedef struct rmm_options {
    /* Largest T that takes the split-K GEMV (decode) path; larger T takes the
     * tcgen05 GEMM.  Default 16; valid range 0..16. */
    int t_gemv;
    /* Attention kept-set granularity: 0 (default) = one set per (batch, KV
     * head) over the stacked queries of its group; 1 = one set per query head. */
    int attn_per_query_head;
    /* Split count of the decode GEMV; 0 = automatic. */
    int gemv_splits;
    /* Watchdog self-test: nonzero makes the reduced GEMM wait, with a 50 ms
     * limit, on a barrier that nothing signals; the call then reports
     * RMM_ERR_TIMEOUT through rmm_get_status() and leaves Y unspecified. */
    int debug_timeout_test;
    /* Operand producer of the reduced GEMM: 0 (default) = the CTA-pair
     * kernel, sixteen warps per CTA gathering the kept rows with 16-byte
     * cp.async into the swizzled layout; 1 = single-CTA kernel with TMA
     * tile::gather4 (one instruction per four kept rows x 64 columns);
     * 2 = single-CTA kernel with the cp.async producer. */
    int gemm_producer;
    /* Attention kernel for the product: 0 (default) = tensor cores (tcgen05)
     * for query chunks of 16 or more tokens, the CUDA-core split pass for
     * shorter ones (decode); 1 = always the split pass; 2 = always the tensor
     * cores. */
    int attn_path;
    /* Granularity of the kept set of rmm_linear / rmm_linear_group: 0
     * (default) = single contraction slices; 16, 32, 64, 128 or 256 = blocks
     * of that many consecutive slices (H a multiple of it, at most 1024
     * blocks), as in the FFN demo of the cf-1.com post (§6.1, 64-wide blocks).
     * A block scores the largest of its slices' scores; kb = ceil(r * H /
     * block_size) blocks are kept under (score desc, block index asc); idx_out
     * then receives their k = kb * block_size slices, ascending. */
    int block_size;
    /* Block score with block_size > 0: 0 (default) = the largest of the
     * block's slice scores; 1 = the block's mean magnitude over all T tokens,
     * the score of the FFN demo (cf-1.com post §5.1, §6.1), computed in single
     * precision in one order (tokens ascending, within a token the block's
     * slices ascending, then one correctly rounded division by T*block_size).
     * 1 requires T <= 16 (RMM_ERR_UNSUPPORTED otherwise). */
    int block_score;
    /* Gated-MLP epilogue for a group of two products of the same width (gate
     * and up of a SwiGLU MLP, the gated FFN of the cf-1.com post §6.1):
     * nonzero makes rmm_linear_group write Ys[0][t,n] = bf16(silu(g) * u) with
     * g = bf16(Y_gate[t,n]), u = bf16(Y_up[t,n]), silu(z) = z / (1 + e^-z), the
     * same bits as rmm_swiglu applied to the two products; Ys[1] serves as
     * scratch (its contents unspecified).  On the split-K GEMV path the fold
     * of the split partial sums applies it (no extra launch); otherwise the
     * SwiGLU kernel runs after the products.  Requires count == 2 and
     * Ns[0] == Ns[1] (RMM_ERR_INVALID_ARG otherwise). */
    int swiglu_pair;
    /* Optional pair of cudaEvent_t handles (NULL: none) recorded on the
     * stream immediately before and after the reduced-product kernel (GEMV or
     * GEMM) of rmm_linear / rmm_gemm_reduced, so that a caller can time that
     * kernel alone inside a longer sequence of calls.  During CUDA-graph
     * capture they are recorded as external event nodes of the graph. */
    void* product_event_begin;
    void* product_event_end;
} rmm_options;

/* Human-readable name of a status code (static storage). */
const char* rmm_status_string(rmm_status status);

/* Number of kept slices for retention ratio r (paper abstract: one retention
 * ratio sets the share of each product that is kept): ceil(r*H) in double,
 * clamped to [1, H].  Returns -1 if r is not in (0, 1] or H < 1. */
int rmm_k_for(int H, double r);

/* Zero-fill a workspace (device memory, `bytes` long) on `stream`.  Needed
 * once before the first call that uses it. */
rmm_status rmm_workspace_init(void* workspace, size_t bytes, rmm_stream_t stream);

/* Read and clear the device status word of a workspace: synchronises
 * `stream`, returns RMM_OK or the first device-side error recorded since the
 * last call (RMM_ERR_TIMEOUT), or RMM_ERR_CUDA if the stream itself failed. */
rmm_status rmm_get_status(void* workspace, rmm_stream_t stream);

/* W^T from W: W bf16 [N, H] row-major -> Wt bf16 [H, N] row-major, so that a
 * kept slice h of the weight is one contiguous row of N elements.  Done once
 * per weight (outside any timed region).  W and Wt must not overlap. */
rmm_status rmm_transpose_weight(const void* W, void* Wt, int N, int H, rmm_stream_t stream);

/* Workspace bytes needed by rmm_linear / rmm_gemm_reduced / rmm_score /
 * rmm_select for these sizes and options. */
size_t rmm_linear_workspace_bytes(int T, int H, int N, const rmm_options* options);

/* The reduced linear map Y ~= X[:,S] W[:,S]^T with S the k = ceil(r*H) kept
 * slices (cf-1.com post §2, §5.1-§5.3; paper abstract).
 *   X        bf16 [T, H] row-major (leading dimension H), 16-byte aligned
 *   Wt       bf16 [H, N] row-major (leading dimension N) = W^T, 16-byte aligned
 *   T        tokens, 1 <= T <= 2^20
 *   H        contraction size, 1 <= H <= 65535
 *   N        output features, 8 <= N, N % 8 == 0
 *   r        retention ratio in (0, 1]
 *   Y        bf16 [T, N] row-major, 16-byte aligned (written)
 *   idx_out  int32 [k] or NULL: receives the kept set S, ascending
 *   workspace, workspace_bytes: >= rmm_linear_workspace_bytes(T, H, N, options)
 * T <= options.t_gemv runs score -> select -> split-K GEMV; larger T runs
 * score (+ X^T) -> select -> tcgen05 GEMM.  Accumulation is fp32, Y is
 * rounded to bf16 (round to nearest even). */
rmm_status rmm_linear(const void* X, const void* Wt, int T, int H, int N, double r, void* Y,
                      int32_t* idx_out, void* workspace, size_t workspace_bytes,
                      rmm_stream_t stream, const rmm_options* options);

/* Several projections of the same activations (e.g. q, k, v of one layer, or
 * gate and up): since the score depends only on X, they share one kept set
 * (cf-1.com post §8: one common set per batch), so the score pass, the kept
 * set and (GEMM path) X^T are computed once and the products of all members
 * run in one launch.  Y_p ~= X[:,S] W_p[:,S]^T for p < count.
 *   X, T, H, r: as for rmm_linear
 *   count: 1..4 members
 *   Wts[p]: bf16 W_p^T [H, Ns[p]], Ys[p]: bf16 [T, Ns[p]] (host arrays of
 *           device pointers; Ns[p] % 8 == 0)
 *   idx_out: int32 [k] or NULL (the shared kept set, ascending)
 *   workspace_bytes >= rmm_linear_group_workspace_bytes(T, H, count, Ns, options)
 * With options.gemm_producer == 1 only count == 1 is supported. */
size_t rmm_linear_group_workspace_bytes(int T, int H, int count, const int* Ns,
                                        const rmm_options* options);
rmm_status rmm_linear_group(const void* X, int T, int H, double r, int count, const void* const* Wts,
                            const int* Ns, void* const* Ys, int32_t* idx_out, void* workspace,
                            size_t workspace_bytes, rmm_stream_t stream, const rmm_options* options);

/* Step 1 alone, the score (cf-1.com post §5.1: a cheap importance score of
 * every contraction index from the current activations; §8: one score for the
 * whole batch): s_out[h] = max_t |X[t,h]| as the bf16 magnitude key (bit
 * pattern with the sign cleared; -0 and +0 both give 0).  X bf16 [T, H],
 * s_out uint32 [H].  T >= 1. */
rmm_status rmm_score(const void* X, int T, int H, uint32_t* s_out, void* workspace,
                     size_t workspace_bytes, rmm_stream_t stream);

/* Step 2 alone, the kept set (cf-1.com post §5.2: scores turned into a top-k
 * set; §6.1: the top-k indices sorted so the kept slices keep their order):
 * the k indices of the largest scores under (score desc, index asc), written
 * to idx_out [k] in ascending order.  s: uint32 [H], each < 65536;
 * 1 <= k <= H <= 65535. */
rmm_status rmm_select(const uint32_t* s, int H, int k, int32_t* idx_out, void* workspace,
                      size_t workspace_bytes, rmm_stream_t stream);

/* Step 3 alone, the reduced product for a given kept set (cf-1.com post §5.3:
 * the gathered slices in one smaller dense product; §2: the output keeps its
 * shape): Y[t,n] = sum_{j<k} X[t,idx[j]] * Wt[idx[j],n].
 * idx: int32 [k], distinct values in [0, H) (any order).  Same layouts and
 * path choice as rmm_linear. */
rmm_status rmm_gemm_reduced(const void* X, const void* Wt, const int32_t* idx, int k, int T,
                            int H, int N, void* Y, void* workspace, size_t workspace_bytes,
                            rmm_stream_t stream, const rmm_options* options);

/* Workspace bytes needed by rmm_attn_qk for these sizes. */
size_t rmm_attn_workspace_bytes(int B, int Hq, int Hkv, int T, int L, int d,
                                const rmm_options* options);

/* Reduced attention (cf-1.com post §3.3; paper abstract: attention products
 * reduced along their contraction dimension).  For each (batch b, KV head g):
 *   s_j = max over the group's query heads q and all t < T of |Q[b,q,t,j]|,
 *   S_g = top-k of s (k = ceil(r*d), ties to the lower index),
 *   logit[q,t,l] = scale * sum_{j in S_g} Q[b,q,t,j] * Kt[b,g,j,l],
 *   O[b,q,t,:] = softmax_l(logit) . V[b,g,l,:]   (full d, fp32 softmax).
 * Queries sit at positions L-T .. L-1; with causal != 0 query t sees keys
 * l <= L-T+t.
 *   Q   bf16 [B, Hq, T, d]
 *   Kt  bf16 [B, Hkv, d, ldL]  (d-major key cache: a kept dim is one row)
 *   V   bf16 [B, Hkv, ldL, d]
 *   O   bf16 [B, Hq, T, d] (written)
 *   idx_out int32 [B, Hkv, k] (or [B, Hq, k] with attn_per_query_head) or NULL
 * Requirements: d == 128, Hq % Hkv == 0, 1 <= T <= L <= ldL, ldL % 8 == 0,
 * 16-byte aligned pointers. */
rmm_status rmm_attn_qk(const void* Q, const void* Kt, const void* V, int B, int Hq, int Hkv,
                       int T, int L, int ldL, int d, double r, int causal, float scale, void* O,
                       int32_t* idx_out, void* workspace, size_t workspace_bytes,
                       rmm_stream_t stream, const rmm_options* options);

/* ---------------------------------------------------------------- context blocks
 *
 * Reduction of Q K^T along the sequence (cf-1.com post §3.1: in generation,
 * cut the cached keys into blocks, score the blocks cheaply, run the full
 * Q K^T only on the blocks that may draw attention; §7: the gain grows with
 * the context).  Block j holds positions [j*block, min(L, (j+1)*block)),
 * block in {32, 64, 128, 256}; its summary is its mean key; a kept set's
 * score for block j is the largest dot product of one of the set's query
 * rows with that mean; the kc = ceil(r_ctx * nblk) best blocks are kept
 * (ties to the lower block index); dropped keys take no part in the softmax.
 * Mean and score are computed in single precision in a fixed order (float
 * sums over l ascending, one correctly rounded division, an fmaf chain over
 * the d dims ascending) so the kept blocks are reproducible exactly. */

/* means[b][g][j][c] = (sum over l in block j of Kt[b][g][c][l]) / n_j, fp32,
 * for the blocks j in [blk_begin, blk_end) (other blocks untouched: refresh
 * the block that receives a new key after each append).
 *   Kt    bf16 [B, Hkv, d, ldL], the first L positions valid
 *   means fp32 [B, Hkv, ceil(ldL / block), d] (caller-owned)
 * Requirements: d == 128, 1 <= L <= ldL, ldL % 8 == 0, 0 <= blk_begin <
 * blk_end <= ceil(L / block), 16-byte aligned pointers. */
rmm_status rmm_ctx_block_means(const void* Kt, int B, int Hkv, int d, int L, int ldL, int block, int blk_begin,
                               int blk_end, float* means, rmm_stream_t stream);

/* Workspace bytes needed by rmm_attn_ctx for these sizes. */
size_t rmm_attn_ctx_workspace_bytes(int B, int Hq, int Hkv, int T, int L, int d, int block, double r_ctx,
                                    const rmm_options* options);

/* Reduced attention with both reductions: the kept head dimensions of
 * rmm_attn_qk (k = ceil(r*d) per set) and the kept context blocks (kc =
 * ceil(r_ctx * ceil(L/block)) per set), then softmax over the kept keys and
 * O = P . V over the full d.  A query row that may attend to no kept key
 * (possible only with causal chunks) gets O = 0.  Same layouts, scale and
 * causal rule as rmm_attn_qk; means as written by rmm_ctx_block_means for
 * every block below ceil(L / block).
 *   idx_out    int32 [B, nsets, k] or NULL (kept head dimensions, ascending)
 *   blocks_out int32 [B, nsets, kc] or NULL (kept blocks, ascending)
 * nsets = Hkv, or Hq with options.attn_per_query_head.  Runs the CUDA-core
 * split pass: T <= 16 (decode and short chunks), ceil(L/block) <= 2048,
 * Hq / Hkv <= 8 for per-KV-head sets; RMM_ERR_UNSUPPORTED otherwise. */
rmm_status rmm_attn_ctx(const void* Q, const void* Kt, const void* V, const float* means, int B, int Hq, int Hkv,
                        int T, int L, int ldL, int d, double r, double r_ctx, int block, int causal, float scale,
                        void* O, int32_t* idx_out, int32_t* blocks_out, void* workspace, size_t workspace_bytes,
                        rmm_stream_t stream, const rmm_options* options);

/* The decode-sized reduced linear map without a workspace.  The pages have
 * no counterpart to this entry point; it exists for callers that cannot give
 * the library device memory of its own: a plugin whose host framework owns
 * every allocation and only lends it input and output buffers, or a serving
 * loop under a fixed memory budget that must not grow once it has started.
 * Computes exactly what rmm_linear computes on its split-K GEMV path
 * (score -> kept set -> reduced product), but all intermediates live in a
 * fixed 4 MiB array inside the library: every GPU that loads the library
 * holds that array until the process exits.  Nothing is allocated or freed.
 *   X, Wt, T, H, N, r, Y, idx_out: as for rmm_linear.
 * Limits: T <= 16 (decode sizes), H <= 65535, N % 8 == 0, N <= 2^20; sizes
 * beyond these return RMM_ERR_UNSUPPORTED with nothing launched.  Large T*N
 * use fewer splits so that the partial sums fit in the array.
 * The first call on a device (with that device current) looks up the array's
 * device address once; make that first call before any stream capture.
 * Every call uses the same array: calls that may overlap on the GPU (on
 * different streams, or from different threads) race and must not be
 * issued; calls in one stream are ordered and safe.  The array keeps the
 * previous call's contents; each call clears what must start at zero. */
rmm_status rmm_linear_decode_noalloc(const void* X, const void* Wt, int T, int H, int N, double r,
                                     void* Y, int32_t* idx_out, rmm_stream_t stream);

/* ---------------------------------------------------------------- decoder-layer glue
 *
 * The memory-bound ops that sit between the reduced products of one decoder
 * layer: RMSNorm in place of LayerNorm, a residual stream through every block
 * and a gated SwiGLU MLP ('Numerical Linear Algebra for LLMs' paper digest,
 * ai-feeds.com, section 'Method: key modules').  All tensors are bf16
 * row-major device buffers owned by the caller, 16-byte aligned; arithmetic
 * inside an op is fp32, every output is rounded to bf16 (round to nearest
 * even).  Calls are asynchronous on `stream`; argument errors are returned
 * before anything is launched. */

/* Hsum = X + R and Y = RMSNorm(Hsum) * weight for each of the T rows of H:
 *   Hsum[t,h] = bf16(X[t,h] + R[t,h])        (R NULL: Hsum = X)
 *   Y[t,h]    = bf16(Hsum[t,h] / sqrt(mean_h Hsum[t,h]^2 + eps) * weight[h])
 * weight NULL means 1; Hsum or Y may be NULL to skip that output (not both).
 * Requires H % 8 == 0 and 8 <= H <= 16384.  Y may alias X. */
rmm_status rmm_add_rmsnorm(const void* X, const void* R, int T, int H, float eps, const void* weight,
                           void* Hsum, void* Y, rmm_stream_t stream);

/* Out[i] = bf16(silu(G[i]) * U[i]), silu(z) = z / (1 + exp(-z)), for n
 * elements (n % 8 == 0). */
rmm_status rmm_swiglu(const void* G, const void* U, int64_t n, void* Out, rmm_stream_t stream);

/* The q/k/v projections of T tokens (token-major, as rmm_linear_group writes
 * them) into the attention layouts of rmm_attn_qk (batch 1), appending the new
 * keys and values to the caches at positions L0 .. L0+T-1:
 *   Yq [T, Hq*d] -> Q  [Hq, T, d]
 *   Yk [T, Hkv*d] -> Kt [Hkv, d, ldL]  (Kt[g, j, L0+t] = Yk[t, g*d+j])
 *   Yv [T, Hkv*d] -> V  [Hkv, ldL, d]  (V[g, L0+t, :] = Yv[t, g*d : g*d+d])
 * Requires d == 128 and L0 + T <= ldL; cache positions outside the append are
 * not touched. */
rmm_status rmm_qkv_heads(const void* Yq, const void* Yk, const void* Yv, int T, int Hq, int Hkv, int d,
                         void* Q, void* Kt, void* V, int ldL, int L0, rmm_stream_t stream);

/* Attention output back to token-major rows for the o projection:
 * A[t, h*d + j] = O[h, t, j] for O [Hq, T, d] (batch 1), d == 128. */
rmm_status rmm_heads_to_tokens(const void* O, int Hq, int T, int d, void* A, rmm_stream_t stream);

/* ---------------------------------------------------------------- self-test
 *
 * y[i] = 2^x[i] as the tensor-core attention's softmax computes half of its
 * exponentials: on the FMA pipe, by a round-to-nearest split x = n + f
 * (|f| <= 1/2), the Taylor series of e^(f ln 2) to degree 4 and n added to
 * the exponent.  The softmax only evaluates x <= 8; below -126 the result is
 * 2^-126.  Stated bound: relative error below 6e-5 on [-126, 8].  It exists so
 * that the bound can be checked directly; x and y are fp32 device buffers of
 * n elements (n >= 1).  The pages have no counterpart: the exponential is an
 * implementation detail of the softmax (cf-1.com post §3.3 keeps softmax.V
 * exact in form). */
rmm_status rmm_selftest_exp2_fma(const float* x, float* y, int n, rmm_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* RMM_H_ */
