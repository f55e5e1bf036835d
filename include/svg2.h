/*
 * libsvg2 — SVG2 semantic-aware permuted sparse attention for one DiT attention layer,
 * hand-written CUDA for NVIDIA B200 (sm_100a).
 *
 * Method: "Sparse VideoGen2: Accelerate Video Generation with Sparse Attention via Semantic-Aware
 * Permutation" (wiki summary page, sections Key claims and Method; paper sections 4.1-4.3).
 * Per (batch, head) the layer clusters Q and K with k-means (Method (1)), scores cluster pairs
 * from centroids and keeps K clusters per Q cluster by top-p (Method (3); section 4.2, Eq. 1-2),
 * permutes Q, K, V into cluster-contiguous order (Method (2); section 4.1), runs attention over
 * the kept variable-size blocks only (Method (4); section 4.3, Fig. 7(b)) and scatters the output
 * rows back to token order (Method (2), "final inverse-permutation of the rows").
 *
 * Conventions shared by every entry point
 *   - Every pointer argument is a DEVICE pointer unless stated otherwise; the caller owns all
 *     memory.  The library never allocates device memory: scratch comes from the caller's
 *     workspace `ws` of `ws_bytes` bytes (size from svg2_workspace_size), 256-byte aligned.
 *   - Tensors are contiguous row-major [B, H, N, d] (d innermost); per-head vectors are
 *     [B, H, n].  d is 64 or 128.  bf16 tensors hold raw bfloat16 values.
 *   - `stream` is a cudaStream_t (NULL = legacy default stream).  Calls are asynchronous on it:
 *     arguments are validated on the host first and a bad one returns an error before any launch;
 *     a failed launch returns SVG2_ERR_CUDA.  Device-side errors (a bounded wait that ran out,
 *     an out-of-range label) are latched in a status word at the start of `ws` and read with
 *     svg2_check_status.  No kernel traps or waits without a bound.
 *   - The library keeps no global state (the one exception is the fixed scratch array of
 *     svg2_sparse_attn_noalloc, described there), is reentrant, and never lets a C++ exception
 *     cross the C boundary.  Return values are svg2_status codes.
 */
#ifndef SVG2_H_
#define SVG2_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define SVG2_API __attribute__((visibility("default")))
#else
#define SVG2_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  SVG2_OK = 0,
  SVG2_ERR_INVALID_ARG = 1,   /* null pointer, size out of range, bad enum value */
  SVG2_ERR_UNSUPPORTED = 2,   /* d / dtype / sizes beyond the library's limits */
  SVG2_ERR_WORKSPACE = 3,     /* ws too small or misaligned */
  SVG2_ERR_CUDA = 4,          /* a CUDA runtime or driver call failed */
  SVG2_ERR_DEVICE_TIMEOUT = 5,/* a bounded device wait ran out (read via svg2_check_status) */
  SVG2_ERR_DEVICE_BOUNDS = 6  /* a device index check failed, e.g. a label >= k */
} svg2_status;

typedef enum { SVG2_BF16 = 0, SVG2_F32 = 1 } svg2_dtype;

/* k-means initialisation.  GIVEN: start from the centroids already in the `centroids` buffer —
 * this is also the warm start of the pages' centroid cache (section 4.3, Fig. 7(a)): pass the
 * previous denoising step's centroids.  KMEANSPP: k-means++ seeding from the data (Method (1)). */
typedef enum { SVG2_INIT_GIVEN = 0, SVG2_INIT_KMEANSPP = 1 } svg2_init;

/* k-means++ seeding looks at S = seed_tokens candidate tokens (0, or seed_tokens >= N: all N tokens):
 * one per stratum of the token order, stratum j = [floor(j N / S), floor((j + 1) N / S)), at offset
 * floor(r_j w_j / 2^32) inside it, w_j its width and r_j = (j * 2654435769) mod 2^32.  The offsets
 * vary from stratum to stratum, so the candidates do not line up with the rows and columns of the
 * video grid the tokens come from.  The Lloyd iterations always use all tokens.  This default keeps
 * the seeding cheap on video-length layers. */
#define SVG2_DEFAULT_SEED_TOKENS 16384

/* Largest sizes the library supports.  Besides these, B*H <= 65535 (several kernels give the (b,h)
 * planes a grid dimension of their own) and B*H*N < 2^31 (token rows across all planes are indexed
 * with 32-bit integers); larger sizes return SVG2_ERR_UNSUPPORTED. */
#define SVG2_MAX_CLUSTERS 1024
#define SVG2_MAX_TOKENS (1 << 24)

/* Human-readable name of a status code (static string, never NULL). */
SVG2_API const char* svg2_status_string(int status);

/* Bytes of workspace that svg2_layer needs for these sizes; every other entry point needs at
 * most this much for the same sizes.  Returns SVG2_ERR_INVALID_ARG / UNSUPPORTED on bad sizes. */
SVG2_API int svg2_workspace_size(int B, int H, int N, int d, int nQ, int nK, size_t* bytes);

/* Reads and clears the device status word in `ws` after synchronising `stream`.
 * *device_status receives the latched svg2_status (SVG2_OK if none); where/info (optional, may be
 * NULL) receive a kernel tag and two integers for diagnostics. */
SVG2_API int svg2_check_status(void* ws, void* stream, int* device_status, uint32_t* where, uint32_t* info);

/* Diagnostics: sets, stream-ordered on `stream`, the budget in SM clock cycles of the bounded
 * waits inside the tensor-core attention (svg2_sparse_attn, svg2_dense_attn, the layer calls) and
 * the tensor-core k-means assignment that later calls make with this workspace.  0 restores the
 * default (about 0.5 s at the boost clock); values above the default are clamped to it, so the
 * setting can only make a wait give up sooner.  A wait that runs out latches
 * SVG2_ERR_DEVICE_TIMEOUT (read with svg2_check_status); the kernel then stops issuing work, waits
 * for its own copies and tensor-core operations already in flight, frees its tensor memory and
 * exits, so later calls on the same workspace run normally.  The value lives in the status area
 * at the start of `ws` (bytes 16..23), which, like the status word, must be zero when the
 * workspace is first used (torch.zeros / cudaMemset); svg2_check_status does not clear it.  The
 * k-means++ seeding keeps the default budget whatever this says.  No counterpart on the pages:
 * it exists so that the give-up path of those waits can be tested.
 *   ws      256-byte aligned workspace; returns SVG2_ERR_INVALID_ARG if NULL or misaligned. */
SVG2_API int svg2_set_wait_budget(void* ws, uint64_t cycles, void* stream);

/*
 * Batched k-means (Method (1); Key claims section 4.1 and 4.3) on X [B, H, N, d] per (b, h):
 * `iters` >= 1 Lloyd iterations — assignment label_t = argmin_c ||x_t - c||^2 (ties to the lower
 * c) as a tensor-core distance GEMM fused with the argmin, then c_j = mean of its members (an empty
 * cluster keeps its centroid) as a segmented sum divided by the count.
 *   X          bf16 or f32 per `dtype`.
 *   init       SVG2_INIT_GIVEN (centroids holds the start, e.g. the previous step's cache) or
 *              SVG2_INIT_KMEANSPP (seeding from the data; `u` must then hold B*H*k uniforms in
 *              [0,1), float64, one per seed, and seeds are chosen by fixed-point D^2 sampling).
 *   seed_tokens  k-means++ candidates: seed_tokens tokens, one per stratum of the token order (0 =
 *              all tokens; see SVG2_DEFAULT_SEED_TOKENS); the candidate count must be >= k.
 *   centroids  float32 [B, H, k, d], in (GIVEN) and out (final centroids).
 *   labels     int32 [B, H, N], out: labels of the last assignment (the ones the final centroids
 *              were computed from).
 *   counts     int32 [B, H, k], out: cluster sizes under those labels.
 *   perm       int32 [B, H, N], out (optional, may be NULL): stable sort of the token indices by
 *              label, perm[j] = token at permuted row j.
 *   offsets    int32 [B, H, k+1], out (optional): exclusive scan of counts.
 * 1 <= k <= min(N, SVG2_MAX_CLUSTERS). */
SVG2_API int svg2_kmeans(const void* X, int dtype, int B, int H, int N, int d, int k, int iters, int init,
                const double* u, int seed_tokens, float* centroids, int32_t* labels, int32_t* counts, int32_t* perm,
                int32_t* offsets, void* ws, size_t ws_bytes, void* stream);

/*
 * k-means++ seeding alone (Method (1): the cold start of svg2_kmeans with SVG2_INIT_KMEANSPP).
 * Per (b, h): seed 0 is candidate floor(u_0 * S); seed s is the first candidate whose running sum
 * of floor(D^2 / M0 * 2^32) exceeds floor(u_s * U), where D^2 is the float64 squared distance to
 * the nearest earlier seed, M0 the largest D^2 after seed 0 and U the sum of all weights (a
 * uniform pick when U = 0).  Candidates as in SVG2_DEFAULT_SEED_TOKENS's note (0 = all tokens).
 *   u          float64 [B, H, k] uniforms in [0, 1).
 *   centroids  float32 [B, H, k, d], out: the seed rows.
 * Same sizes, dtype and workspace rules as svg2_kmeans; the candidate count must be >= k. */
SVG2_API int svg2_kmeanspp(const void* X, int dtype, int B, int H, int N, int d, int k, const double* u,
                  int seed_tokens, float* centroids, void* ws, size_t ws_bytes, void* stream);

/*
 * Critical-cluster selection (section 4.2, Eq. 1-2; Method (3)).  Per (b, h, Q-cluster i):
 * l_ij = (cq_i . ck_j) * scale, w_ij = count_k[j] * exp(l_ij - max_j l_ij) over non-empty j
 * (w = 0 for empty j), then top-p: the shortest prefix of the K clusters ordered by (w desc, j asc)
 * whose weight reaches p of the row total, in fixed point: u_j = floor(w_j / max w * 2^32),
 * T = ceil(p * sum u), keep until the running sum >= T.  top_p >= 1 keeps every non-empty cluster.
 *   cq float32 [B,H,nQ,d]; ck float32 [B,H,nK,d]; count_k int32 [B,H,nK].
 *   weights   float32 [B,H,nQ,nK], out (optional, may be NULL).
 *   mask      uint8 [B,H,nQ,nK], out: 1 where the pair is kept.
 *   sel_count int32 [B,H,nQ], out: number of kept K clusters per Q cluster.
 *   sel_idx   int32 [B,H,nQ,nK], out: the kept K-cluster indices in ascending order in the first
 *             sel_count entries of each row (rest unspecified).
 *   stream_len int32 [B,H,nQ], out (optional): number of keys kept per Q cluster.
 * nQ, nK in [1, SVG2_MAX_CLUSTERS]; 0 < top_p. */
SVG2_API int svg2_select(const float* cq, const float* ck, const int32_t* count_k, int B, int H, int nQ, int nK,
                int d, float top_p, float scale, float* weights, uint8_t* mask, int32_t* sel_count,
                int32_t* sel_idx, int32_t* stream_len, void* ws, size_t ws_bytes, void* stream);

/* The top-p step of svg2_select alone, on given float32 weights [B,H,nQ,nK] (same outputs). */
SVG2_API int svg2_select_from_weights(const float* weights, const int32_t* count_k, int B, int H, int nQ, int nK,
                             float top_p, uint8_t* mask, int32_t* sel_count, int32_t* sel_idx,
                             int32_t* stream_len, void* ws, size_t ws_bytes, void* stream);

/*
 * Stable counting sort of labels (Method (2)): per (b,h), counts [k], offsets [k+1] (exclusive
 * scan) and perm [N] with perm[j] = original token of permuted row j, in (label asc, token asc).
 * labels int32 [B,H,N] in [0,k) (a label out of range latches SVG2_ERR_DEVICE_BOUNDS). */
SVG2_API int svg2_sort(const int32_t* labels, int B, int H, int N, int k, int32_t* perm, int32_t* offsets,
              int32_t* counts, void* ws, size_t ws_bytes, void* stream);

/* Row gather applying a permutation (Method (2)): Xp[b,h,j,:] = X[b,h,perm[b,h,j],:].
 * X bf16 or f32 per dtype; Xp is always bf16 (f32 input is rounded to nearest even). */
SVG2_API int svg2_gather(const void* X, int dtype, const int32_t* perm, int B, int H, int N, int d, void* Xp,
                void* stream);

/* svg2_sort of `labels` followed by svg2_gather of X: cluster-contiguous bf16 Xp. */
SVG2_API int svg2_permute(const void* X, int dtype, const int32_t* labels, int B, int H, int N, int d, int k,
                 void* Xp, int32_t* perm, int32_t* offsets, int32_t* counts, void* ws, size_t ws_bytes,
                 void* stream);

/*
 * Variable-block-size sparse attention (Method (4); section 4.3, Fig. 7(b)) on permuted bf16
 * Qp, Kp, Vp [B,H,N,d] (d = 128): a query row of Q cluster i (rows [q_off[i], q_off[i+1]))
 * attends, with one softmax, to the keys of every kept K cluster j (rows [k_off[j], k_off[j+1]))
 * listed in sel_idx[i][0..sel_count[i]).  Online softmax on tcgen05/TMEM tiles; the kept
 * clusters are gathered into one packed key stream, so ragged cluster edges cost no padding.
 *   q_off int32 [B,H,nQ+1]; k_off int32 [B,H,nK+1]; sel_count/sel_idx as from svg2_select.
 *   perm_q   optional int32 [B,H,N]: if given, output row r is written to token perm_q[r]
 *            (the inverse permutation fused into the epilogue); if NULL, O is in permuted order.
 *   O        bf16 [B,H,N,d], out.  scale multiplies q.k (usually 1/sqrt(d)). */
SVG2_API int svg2_sparse_attn(const void* Qp, const void* Kp, const void* Vp, const int32_t* q_off,
                     const int32_t* k_off, const int32_t* sel_count, const int32_t* sel_idx, int B, int H,
                     int N, int d, int nQ, int nK, float scale, const int32_t* perm_q, void* O, void* ws,
                     size_t ws_bytes, void* stream);

/*
 * Per-head E4M3 quantisation for the FP8 attention variant (the project's roadmap item "Support FP8
 * attention", GitHub README, Open-source Plan; the pages fix no scaling scheme, this is the plainest:
 * one scale per (b,h) plane).  E4M3 is the OCP 8-bit floating point format with 4 exponent bits
 * (bias 7), 3 mantissa bits, no infinities and 448 as its largest finite magnitude.  Per plane:
 *   amax = max |x| (NaN entries ignored); inv = fl32(448 / amax); scale[bh] = fl32(amax / 448)
 *   (inv = scale = 1 when amax == 0); X8[bh, r, :] = E4M3(fl32(X[bh, perm[r], :] * inv)), rounded
 *   to nearest even, saturating at +-448.
 * A code c stands for E4M3(c) * scale[bh].
 *   X      [B,H,N,d] bf16 or f32 (dtype), 16-byte aligned.
 *   perm   optional int32 [B,H,N] (NULL: the identity); entries outside [0, N) leave their row unwritten.
 *   X8     uint8 [B,H,N,d], out, 16-byte aligned.  scale  float [B,H], out.
 * Three kernels on `stream`, no workspace.  Errors: SVG2_ERR_INVALID_ARG (null or unaligned
 * pointers, bad dtype), SVG2_ERR_UNSUPPORTED (sizes), SVG2_ERR_CUDA (launch). */
SVG2_API int svg2_quantize_e4m3(const void* X, int dtype, const int32_t* perm, int B, int H, int N, int d, void* X8,
                                float* scale, void* stream);

/*
 * The FP8 variant of svg2_sparse_attn (project roadmap item "Support FP8 attention"): the same
 * variable-block sparse attention on E4M3 codes, with the products on the tensor core's 8-bit path
 * (tcgen05 kind::f8f6f4).  Computes softmax(scale * q.k) v over the dequantised values
 * q = E4M3(Qp8) * scale_q[bh] (likewise k, v); P is handed to the PV product as E4M3 (its values
 * stay within [0, 256] by the lazy rescale), accumulation is float32, O is bf16.
 *   Qp8, Kp8, Vp8  uint8 E4M3 codes [B,H,N,d], d = 128, permuted as for svg2_sparse_attn (16-byte aligned).
 *   scale_q, scale_k, scale_v  float [B,H]: the planes' dequantisation scales (svg2_quantize_e4m3).
 *   Other arguments, workspace and errors as svg2_sparse_attn; d != 128 gives SVG2_ERR_UNSUPPORTED. */
SVG2_API int svg2_sparse_attn_fp8(const void* Qp8, const void* Kp8, const void* Vp8, const float* scale_q,
                                  const float* scale_k, const float* scale_v, const int32_t* q_off,
                                  const int32_t* k_off, const int32_t* sel_count, const int32_t* sel_idx, int B,
                                  int H, int N, int d, int nQ, int nK, float scale, const int32_t* perm_q, void* O,
                                  void* ws, size_t ws_bytes, void* stream);

/*
 * Dense attention, O = softmax(scale * Q K^T) V per (b,h) over all N keys, on the same tcgen05
 * kernel as svg2_sparse_attn: the one-cluster case (one Q cluster and one K cluster holding every
 * token in its original order), so no permutation and no k-means.  This is the layer the pages run
 * for the first denoising steps before the sparse one takes over (Method; the dense warm-up) and the
 * reference the sparse layer is compared with at top-p = 1.
 *   Q, K, V  bf16 [B,H,N,d] (d = 128 or 64), row-major; O bf16 [B,H,N,d], out (may not alias Q, K, V).
 *   ws       at least svg2_dense_attn_workspace_size() bytes, 256-byte aligned; holds the status
 *            word (read with svg2_check_status) and the work plan.
 * Errors: SVG2_ERR_INVALID_ARG (null or unaligned pointers, non-finite scale), SVG2_ERR_UNSUPPORTED
 * (sizes), SVG2_ERR_WORKSPACE, SVG2_ERR_CUDA (launch). */
SVG2_API int svg2_dense_attn_workspace_size(int B, int H, int N, int d, size_t* bytes);
SVG2_API int svg2_dense_attn(const void* Q, const void* K, const void* V, int B, int H, int N, int d, float scale,
                             void* O, void* ws, size_t ws_bytes, void* stream);

/* Inverse permutation of output rows (Method (2)): O[b,h,perm[b,h,j],:] = Op[b,h,j,:], bf16. */
SVG2_API int svg2_unpermute(const void* Op, const int32_t* perm, int B, int H, int N, int d, void* O, void* stream);

/* Parameters of one layer call. */
typedef struct {
  int nQ, nK;          /* clusters for Q and for K */
  int iters;           /* Lloyd iterations per call (>= 1) */
  int init;            /* svg2_init: GIVEN = warm start from cq/ck, KMEANSPP = cold start */
  float top_p;         /* (0, 1]; >= 1 keeps every pair */
  float scale;         /* softmax scale, usually 1/sqrt(d) */
  int seed_tokens;     /* k-means++ candidates, as in svg2_kmeans (0 = all tokens) */
  int fuse_unpermute;  /* 1: write O in token order from the attention epilogue (default path);
                          0: write permuted rows, then run svg2_unpermute */
  int attn_fp8;        /* 0: bf16 attention; 1: the FP8 variant (d = 128): the gathers write per-head
                          E4M3 codes of Q, K, V (as svg2_quantize_e4m3) and svg2_sparse_attn_fp8 runs */
} svg2_params;

/* Optional device buffers for the layer's intermediate results.  Any NULL field is kept inside
 * the workspace instead.  Shapes as in the per-stage calls above. */
typedef struct {
  int32_t *labels_q, *labels_k, *count_q, *count_k, *perm_q, *perm_k, *q_off, *k_off;
  float* weights;
  uint8_t* mask;
  int32_t *sel_count, *sel_idx, *stream_len;
} svg2_layer_outputs;

/*
 * One SVG2 attention layer (Method (1)-(4)): k-means on Q (nQ) and on K (nK), selection, permute,
 * sparse attention and inverse permutation, all enqueued on `stream` with no host synchronisation.
 *   Q, K, V   [B,H,N,d] bf16 or f32 (dtype), d = 128 for the tensor-core attention.
 *   uq, uk    float64 uniforms [B,H,nQ] / [B,H,nK] for k-means++ (ignored for GIVEN; may be NULL).
 *   cq, ck    float32 centroid caches [B,H,nQ,d] / [B,H,nK,d]: in for GIVEN (warm start), out always.
 *   O         bf16 [B,H,N,d], out, in token order.
 *   outs      optional (may be NULL), see svg2_layer_outputs. */
SVG2_API int svg2_layer(const void* Q, const void* K, const void* V, int dtype, int B, int H, int N, int d,
               const svg2_params* params, const double* uq, const double* uk, float* cq, float* ck, void* O,
               const svg2_layer_outputs* outs, void* ws, size_t ws_bytes, void* stream);

/*
 * svg2_layer for inputs and output in host memory, with the transfers overlapped with the work:
 * on `copy_stream` K (in two halves of the planes), then Q, then V (per attention group) are copied
 * to the caller's device staging buffers while, on `stream`, the k-means of each half of K starts
 * as soon as that half has landed and that of Q as soon as Q has (K's k-means, with more clusters,
 * is the longer one and hides Q's upload), and each group's K/V gathers wait only for its own V; the
 * attention then runs in groups of `heads_per_group` (b,h) planes (0 = all at once; the last
 * `heads_per_group` planes go in halves, quarters, ... down to one plane, so that the one copy
 * back that nothing overlaps is small) and each group's output is copied back while the next
 * group is computed.  Host buffers must be
 * page-locked (cudaHostAlloc / cudaHostRegister) for the copies to be asynchronous.  The copies
 * start only after the work already enqueued on `stream`; on return everything is enqueued and
 * `stream` waits for the last copy, so synchronising `stream` covers the whole call.
 * `copy_stream` may be NULL or equal to `stream` (no overlap).  Results equal svg2_layer's.
 *   Qh, Kh, Vh   host [B,H,N,d] (dtype); Oh host bf16 [B,H,N,d], out.
 *   Qd, Kd, Vd   device staging buffers [B,H,N,d] (dtype); Od device bf16 [B,H,N,d] (caller-owned).
 *   uq, uk, cq, ck, params, ws as in svg2_layer (device memory). */
SVG2_API int svg2_layer_host(const void* Qh, const void* Kh, const void* Vh, void* Oh, void* Qd, void* Kd,
                             void* Vd, void* Od, int dtype, int B, int H, int N, int d, const svg2_params* params,
                             const double* uq, const double* uk, float* cq, float* ck, int heads_per_group,
                             void* ws, size_t ws_bytes, void* stream, void* copy_stream);

/*
 * svg2_sparse_attn without a workspace, for callers that cannot allocate device memory at call
 * time (no cudaMalloc and no caching allocator available to them, e.g. code that must not grow
 * its memory footprint once running).  The paper has no counterpart; this is an interface
 * convenience.  Same inputs, outputs and semantics as svg2_sparse_attn, but its scratch — the
 * attention work plan and a status word — is a fixed 1 MiB array inside the library, which every
 * GPU that loads the library keeps until the process exits.  Sizes whose plan needs more than that
 * (about B*H*(ceil(N/256) + nQ) * 16 bytes plus a few KB) return SVG2_ERR_UNSUPPORTED.
 * The call allocates nothing.  Its first call on a device looks up the array's device address
 * (once per device, with that device current); make that first call before any stream capture.
 * All calls share the one array and it keeps the last call's contents, so calls whose kernels
 * may overlap on the GPU (different streams, or other threads) race: serialise them.
 *   device_status  optional 16-byte, 16-byte-aligned caller-owned device word that must start at
 *                  zero; device-side errors (SVG2_ERR_DEVICE_*) are latched there.  If NULL, the
 *                  library's own word is used (cleared at every call) and such errors are not
 *                  reported to the caller. */
SVG2_API int svg2_sparse_attn_noalloc(const void* Qp, const void* Kp, const void* Vp, const int32_t* q_off,
                                      const int32_t* k_off, const int32_t* sel_count, const int32_t* sel_idx,
                                      int B, int H, int N, int d, int nQ, int nK, float scale,
                                      const int32_t* perm_q, void* O, uint32_t* device_status, void* stream);

/*
 * Self-test of the tensor-core building blocks (not part of the method): C = A * B^T for
 * bf16 A [128, 128] and B [n, 128] (n in {64, 128, 256}), loaded by TMA with 128-byte swizzle,
 * multiplied by tcgen05.mma into TMEM (float32); then P = bf16(C[:, :128]) is written back to
 * TMEM and multiplied by V [128, 128] (bf16, row-major: keys x d) from shared memory as
 * O = P * V, exercising the TMEM-operand form used by the attention.  Outputs C float32
 * [128, n] and O float32 [128, 128].  ws holds the status word. */
SVG2_API int svg2_selftest_mma(const void* A, const void* Bm, int n, const void* V, float* C, float* O, void* ws,
                      size_t ws_bytes, void* stream);

/*
 * Denoising-loop driver: the schedule the pages run around the layer.  Over num_steps denoising
 * steps and num_layers attention layers, steps 0 .. dense_steps-1 run dense attention
 * (svg2_dense_attn; the pages keep full attention for the first steps); a layer's first sparse
 * step starts its k-means cold (k-means++ seeding and layer.iters Lloyd iterations); its later
 * steps start warm from the centroids it left at its previous sparse step, with warm_iters
 * iterations (the centroid cache across steps of Key claims section 4.3, Fig. 7(a)).
 * The driver holds host state only (the schedule, which layers' caches hold centroids) and does
 * not touch the GPU except through the layer calls it makes.  Its centroid cache is caller-owned
 * device memory: num_layers x [B,H,nQ,d] then [B,H,nK,d] float32, svg2_driver_cache_bytes()
 * bytes, 16-byte aligned, bound with svg2_driver_bind_cache (binding marks every layer cold;
 * svg2_driver_reset does the same for a new video).  One driver serves one stream at a time.
 * Errors: SVG2_ERR_INVALID_ARG (null handle or pointers, step or layer out of range, bad config),
 * SVG2_ERR_UNSUPPORTED (d), SVG2_ERR_WORKSPACE (no or too small cache, workspace), and the errors
 * of the layer calls.
 */
typedef struct svg2_driver svg2_driver;
typedef struct {
  int num_steps, num_layers;
  int dense_steps;    /* steps 0 .. dense_steps-1 run dense attention (0 <= dense_steps <= num_steps) */
  int warm_iters;     /* Lloyd iterations of a warm-started k-means (>= 1; 2 in the pages) */
  svg2_params layer;  /* the sparse layer; layer.iters is the cold start's, layer.init is ignored */
} svg2_driver_config;
typedef enum { SVG2_STEP_DENSE = 0, SVG2_STEP_COLD = 1, SVG2_STEP_WARM = 2 } svg2_step_kind;

SVG2_API int svg2_driver_create(const svg2_driver_config* cfg, int B, int H, int N, int d, svg2_driver** out);
SVG2_API int svg2_driver_destroy(svg2_driver* drv);
SVG2_API int svg2_driver_cache_bytes(const svg2_driver* drv, size_t* bytes);
SVG2_API int svg2_driver_bind_cache(svg2_driver* drv, float* cache, size_t bytes);
SVG2_API int svg2_driver_reset(svg2_driver* drv);
/* Bytes of workspace that both the dense and the sparse layer calls of this driver fit in. */
SVG2_API int svg2_driver_workspace_size(const svg2_driver* drv, size_t* bytes);
/* What svg2_driver_layer(step, layer) will run now: a svg2_step_kind in *kind. */
SVG2_API int svg2_driver_plan(const svg2_driver* drv, int step, int layer, int* kind);
/* Runs layer `layer` of step `step` on bf16 Q, K, V [B,H,N,d] into O (bf16, token order), on
 * `stream`: dense, cold (uq, uk: the k-means++ uniforms as in svg2_layer) or warm, per
 * svg2_driver_plan.  A sparse call that returns SVG2_OK leaves the layer's cache warm. */
SVG2_API int svg2_driver_layer(svg2_driver* drv, int step, int layer, const void* Q, const void* K, const void* V,
                               const double* uq, const double* uk, void* O, void* ws, size_t ws_bytes,
                               void* stream);

#ifdef __cplusplus
}
#endif

#endif /* SVG2_H_ */
