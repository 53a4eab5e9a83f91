/*
 * psa.h -- C ABI of the B200 (sm_100a) block-sparse prefill attention library
 * (PISA-style block routing with a 0th-order term for unselected blocks).
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - Tensors are row-major, contiguous.  Q, K, V and the output are
 *    [B, H, N, d] bf16, passed as raw 16-bit patterns (psa_bf16_t).
 *    Pooled statistics are [B, H, M, d] float32 with M = N / 64.
 *    Block I of a head is tokens [64 I, 64 I + 64).
 *  - Every pointer argument is a DEVICE pointer owned by the caller, except
 *    where a comment says "host".  The library never allocates device memory
 *    and never frees what it is given.
 *  - Every call is asynchronous on `stream` (a cudaStream_t passed as void*;
 *    NULL = the legacy default stream) and returns a status code.  The
 *    forward path's kernels are programmatic dependent launches: each may
 *    start its setup while the kernel before it on the stream drains, and
 *    waits on the device before touching memory, so stream order holds for
 *    every read and write; captured into a CUDA graph they become
 *    programmatic edges.
 *  - Arguments are validated on the host before any launch: a bad argument
 *    returns an error code and launches nothing.  The tensors must live on
 *    the CURRENT device (cudaSetDevice): a call whose main input or output
 *    is memory of another device returns PSA_ERR_DEVICE, one given host
 *    memory returns PSA_ERR_ARG.  Conditions that only the
 *    device can see (a malformed block list, a bounded wait that ran out) are
 *    recorded in the status word inside the caller's workspace; read it with
 *    psa_read_status().
 *  - Supported: block_size == 64, d in {64, 128}, N a positive multiple of
 *    64, M = N / 64 <= 16384, B * H * N * d < 2^31.
 *
 * Rows of a block list ("CSR") are ordered (b, h, I) row-major: row
 * r = (b * H + h) * M + I.  row_ptr has B*H*M + 1 int32 entries, col_idx
 * holds the listed key blocks J of each row in ascending order.
 *
 * Citations name the web page and the section that defines the operation.
 */
#ifndef PSA_H
#define PSA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define PSA_API __attribute__((visibility("default")))
#else
#define PSA_API
#endif

typedef uint16_t psa_bf16_t; /* raw bfloat16 bits */

enum psa_status {
    PSA_OK = 0,
    PSA_ERR_ARG = 1,          /* null pointer, non-positive size, bad flag      */
    PSA_ERR_SHAPE = 2,        /* N not a multiple of block_size, sizes too big */
    PSA_ERR_UNSUPPORTED = 3,  /* block_size != 64, d not in {64, 128}, M > 16384 */
    PSA_ERR_CAPACITY = 4,     /* workspace or col_idx capacity too small       */
    PSA_ERR_CUDA = 5,         /* a CUDA runtime / driver call failed           */
    PSA_ERR_TIMEOUT = 6,      /* device: a bounded wait ran out (kernel quit)   */
    PSA_ERR_CSR = 7,          /* device: a listed block is out of range or repeated */
    PSA_ERR_DEVICE = 8        /* no sm_100 device current, or a tensor of another device */
};

/* Text for a status code (static storage, never NULL). */
PSA_API const char* psa_status_string(int status);

/* Library version: major * 10000 + minor * 100 + patch. */
PSA_API int psa_version(void);

/*
 * Bytes of device workspace that the routers, psa_attn and psa_dense need
 * for a problem of this shape (one workspace serves them all).  Besides
 * O(B*H*M*d) of pooled data it holds the block-score matrices of as many
 * heads as fit 256 MB (at least one head: 4*M*ceil(M/128)*128 bytes).  The
 * workspace must be 256-byte aligned and is owned by the caller; calls that
 * share one workspace must be ordered on one stream.  Returns 0 for invalid
 * sizes.
 */
PSA_API size_t psa_workspace_size(int B, int H, int N, int d);

/*
 * Worst-case number of listed blocks over all rows (the col_idx capacity
 * that can never overflow): B*H*M*M, or B*H*M*(M+1)/2 when causal.
 */
PSA_API size_t psa_route_capacity(int B, int H, int M, int causal);

/*
 * a1. Pooling [PISA summary, "How are candidate blocks narrowed": a
 * representative query and key per block and the sum of the values;
 * FlashPrefill summary, 2.a "Block approximation": average-pooled keys].
 *   qbar[b,h,I,:] = mean of q over block I     (float32, [B,H,M,d])
 *   kbar[b,h,J,:] = mean of k over block J     (float32, [B,H,M,d])
 *   vsum[b,h,J,:] = sum  of v over block J     (float32, [B,H,M,d])
 * Accumulates in float32.  Errors: PSA_ERR_ARG, PSA_ERR_SHAPE,
 * PSA_ERR_UNSUPPORTED, PSA_ERR_CUDA.
 */
PSA_API int psa_pool(const psa_bf16_t* q, const psa_bf16_t* k, const psa_bf16_t* v,
             int B, int H, int N, int d, int block_size,
             float* qbar, float* kbar, float* vsum, void* stream);

/*
 * a2 + a3. Block scores and top-k routing [PISA summary, "How are candidate
 * blocks narrowed" and usage line `density=0.15`].
 *   s_IJ = qbar_I . kbar_J / sqrt(d) (float32), candidates J < M, or J <= I
 *   when causal.  Row I keeps k = clamp(ceil(fl32(density * M)), 1, #cand)
 *   blocks: the k highest scores, ties to the smaller J; when causal the
 *   diagonal block takes one of the k slots and the other k-1 are the best
 *   J < I.  Lists ascending.
 * Outputs: row_ptr [B*H*M + 1], col_idx [capacity] (device int32),
 * *nnz_out (device int32) = total listed, and, when row_max is not NULL,
 * row_max [B*H*M] (device float32) = max over the candidates of s_IJ, the
 * softmax stabiliser psa_attn can take instead of computing its own.
 * `workspace` (device, 256-byte aligned, psa_workspace_size(B,H,64*M,d)
 * bytes) holds the score matrices: the scores are one tensor-core product
 * per head at fp32 accuracy (each fp32 operand split into three bf16 parts),
 * written to the workspace and then selected from; heads go in batches that
 * fit it.  The call resets the workspace status word; a bounded device wait
 * that runs out records PSA_ERR_TIMEOUT there (psa_read_status).
 * Errors: PSA_ERR_ARG, PSA_ERR_UNSUPPORTED, PSA_ERR_CAPACITY (capacity
 * below the exact total, which the host knows for top-k, or workspace too
 * small), PSA_ERR_CUDA.
 */
PSA_API int psa_route_topk(const float* qbar, const float* kbar,
                   int B, int H, int M, int d, float density, int causal,
                   int* row_ptr, int* col_idx, size_t capacity, int* nnz_out,
                   float* row_max, void* workspace, size_t workspace_bytes,
                   void* stream);

/*
 * a2 + a4. Block scores and sorting-free threshold routing [FlashPrefill
 * summary, 2.b "Max-based dynamic thresholding": thresh_I = alpha *
 * max_J Score_IJ].  Keeps J iff s_IJ >= alpha * max over candidates
 * (float32), plus the diagonal block I, plus block 0 when keep_first.
 * Lists ascending.  The total is data dependent: *nnz_out (device) receives
 * the exact total; if it exceeds `capacity`, rows past the capacity are cut
 * (row_ptr stays a valid, truncated CSR) and the caller must retry with a
 * larger col_idx.  psa_route_capacity() never overflows.  row_max
 * (nullable) as for psa_route_topk: the row maxima the threshold is taken of.
 * `workspace` (device, psa_workspace_size(B,H,64*M,d) bytes) holds the
 * score matrices (as for psa_route_topk) and the row counts and bit masks
 * between the launches; the call resets its status word.  Errors:
 * PSA_ERR_ARG, PSA_ERR_UNSUPPORTED, PSA_ERR_CAPACITY (workspace too small),
 * PSA_ERR_CUDA.
 */
PSA_API int psa_route_thresh(const float* qbar, const float* kbar,
                     int B, int H, int M, int d, float alpha, int causal,
                     int keep_first, int* row_ptr, int* col_idx, size_t capacity,
                     int* nnz_out, float* row_max, void* workspace,
                     size_t workspace_bytes, void* stream);

/*
 * a4, probability reading. The same max-based rule with the block attention
 * score read as the softmax of the row's block scores [FlashPrefill summary,
 * 2.b "Max-based dynamic thresholding"; the summary does not say which
 * score it means]: keep J iff p_IJ >= alpha * max_J p_IJ with p_IJ
 * proportional to e^{s_IJ}, i.e. s_IJ >= max_J s_IJ + ln(alpha) (float32,
 * ln(alpha) rounded to float32), plus the diagonal block I, plus block 0
 * when keep_first.  alpha must be positive and finite (alpha >= 1 keeps the
 * row maximum and the forced blocks only).  Outputs, workspace, capacity
 * and errors as psa_route_thresh; row_max (nullable) is still the row
 * maximum of s_IJ.
 */
PSA_API int psa_route_thresh_prob(const float* qbar, const float* kbar,
                          int B, int H, int M, int d, float alpha, int causal,
                          int keep_first, int* row_ptr, int* col_idx, size_t capacity,
                          int* nnz_out, float* row_max, void* workspace,
                          size_t workspace_bytes, void* stream);

/*
 * a5 - a7. Exact attention on the listed blocks plus the 0th-order term of
 * every other candidate, in one softmax [PISA summary, routing table and
 * "Why approximating unselected blocks keeps softmax intact"; FlashPrefill
 * summary, 2.c "Index-driven physical jumping" for the addressing].
 *   For query i of block I: z_ij = q_i.k_j / sqrt(d) over the tokens of the
 *   listed blocks (causal: j <= i inside the diagonal block), and
 *   a_iJ = q_i.kbar_J / sqrt(d) for each unlisted candidate J (causal:
 *   J < I).  out_i = (sum e^z v_j + sum e^a vsum_J) /
 *                    (sum e^z + 64 sum e^a),  lse_i = ln of that denominator
 *   (natural log, including the common stabiliser).
 * Inputs: q, k, v bf16 [B,H,N,d]; kbar, vsum float32 [B,H,M,d] from
 * psa_pool; row_ptr / col_idx from a router or from the caller, where
 * col_capacity is the number of int32 entries col_idx points to (a row whose
 * row_ptr range leaves [0, col_capacity] is treated as empty and recorded as
 * PSA_ERR_CSR, so the kernel never reads past the caller's buffer).
 * row_max (float32 [B*H*M], nullable) is the router's row maximum of s_IJ;
 * the kernel builds each row's softmax stabiliser from it, and computes the
 * same quantity itself from q and kbar when it is NULL.  It only shifts the
 * exponents: any finite values give the same result up to rounding, rows
 * whose sum would leave the fp32 range are recomputed exactly.
 * Outputs: out bf16 [B,H,N,d]; lse float32 [B,H,N] (may be NULL).
 * A malformed list entry is recorded as PSA_ERR_CSR in the workspace
 * status: an entry out of range (J >= M, or J > I when causal) is skipped,
 * a repeated entry is counted each time it appears.
 * Errors: PSA_ERR_ARG, PSA_ERR_SHAPE, PSA_ERR_UNSUPPORTED, PSA_ERR_CAPACITY
 * (workspace too small), PSA_ERR_DEVICE, PSA_ERR_CUDA.
 */
PSA_API int psa_attn(const psa_bf16_t* q, const psa_bf16_t* k, const psa_bf16_t* v,
             const float* kbar, const float* vsum,
             const int* row_ptr, const int* col_idx, size_t col_capacity,
             const float* row_max, int B, int H, int N, int d, int block_size, int causal,
             psa_bf16_t* out, float* lse,
             void* workspace, size_t workspace_bytes, void* stream);

/*
 * f-1. The global statistic of the first-order ("hyd") correction [PISA
 * summary, "Why approximating unselected blocks keeps softmax intact" and
 * FAQ "Why a global first-order correction?": to first order around the
 * block-mean key, an unselected block J adds e^{a_iJ} H_J^T q_i / sqrt(d) to
 * the numerator, H_J = sum_{j in J} (k_j - kbar_J) v_j^T, and the pages use
 * one global statistic in place of the per-block matrices; reading taken:
 * the mean of H_J over the blocks of a head]:
 *   hstat[b,h] = (1/M) sum_J sum_{j in J} (k_j - kbar_J) v_j^T
 * float32 [B,H,d,d], row = key feature, column = value feature.
 * Inputs: k, v bf16 [B,H,N,d]; kbar, vsum float32 [B,H,M,d] from psa_pool.
 * `workspace` (psa_workspace_size bytes) holds the partial sums; the call
 * resets its status word.  Errors: PSA_ERR_ARG, PSA_ERR_SHAPE,
 * PSA_ERR_UNSUPPORTED, PSA_ERR_CAPACITY, PSA_ERR_DEVICE, PSA_ERR_CUDA.
 */
PSA_API int psa_hyd_stat(const psa_bf16_t* k, const psa_bf16_t* v, const float* kbar, const float* vsum,
                         int B, int H, int N, int d, float* hstat, void* workspace, size_t workspace_bytes,
                         void* stream);

/*
 * f-1. Attention with the first-order correction of the unselected blocks
 * [same sources as psa_hyd_stat]: psa_attn's output plus, for each query,
 *   sum_{J unlisted candidate} e^{a_iJ} (hstat^T q_i) / sqrt(d)
 * in the numerator (the denominator is psa_attn's), i.e.
 *   out_i = out0_i + w_i (q_i^T hstat) / sqrt(d),
 *   w_i = sum_J e^{a_iJ} / den_i,
 * with out0 and den the 0th-order output and denominator; lse is
 * psa_attn's.  hstat: float32 [B,H,d,d] from psa_hyd_stat (any statistic of
 * that shape may be passed).  Other arguments, workspace and errors as
 * psa_attn.
 */
PSA_API int psa_attn_hyd(const psa_bf16_t* q, const psa_bf16_t* k, const psa_bf16_t* v,
                         const float* kbar, const float* vsum, const float* hstat,
                         const int* row_ptr, const int* col_idx, size_t col_capacity,
                         const float* row_max, int B, int H, int N, int d, int block_size, int causal,
                         psa_bf16_t* out, float* lse, void* workspace, size_t workspace_bytes, void* stream);

/*
 * f-4. Gradients of the 0th-order attention of psa_attn for fixed block
 * lists [PISA summary, "Minimal usage": the simplified 0th-order version
 * supports training].  With out, lse the outputs of psa_attn on the same
 * inputs and lists, and dout = dL/dout, it writes dq, dk, dv (bf16
 * [B,H,N,d], fp32 accumulation):
 *   D_i = dout_i . out_i,  p_ij = e^{z_ij - lse_i},  pi_iJ = e^{a_iJ - lse_i}
 *   dS_ij = p_ij (dout_i . v_j - D_i)          (listed keys)
 *   dA_iJ = pi_iJ (dout_i . vsum_J - 64 D_i)   (unlisted candidates)
 *   dq_i = (sum_j dS_ij k_j + sum_J dA_iJ kbar_J) / sqrt(d)
 *   dk_j = sum_i dS_ij q_i / sqrt(d) + dkbar_J / 64,  dkbar_J = sum_i dA_iJ q_i / sqrt(d)
 *   dv_j = sum_i p_ij dout_i + dvsum_J,            dvsum_J = sum_i pi_iJ dout_i
 * (block J of token j; the pooling spreads the pseudo-key gradients over the
 * block's tokens).  The routing carries no gradient.  Inputs as psa_attn
 * (kbar, vsum from psa_pool; lse float32 [B,H,N] required, dout bf16
 * [B,H,N,d]); outputs dq, dk, dv bf16 [B,H,N,d].  A list entry that repeats
 * a block or leaves the candidates is recorded as PSA_ERR_CSR in the
 * workspace status word and left out.  `workspace` as psa_attn (the call
 * resets its status word).  Errors as psa_attn.
 */
PSA_API int psa_attn_bwd(const psa_bf16_t* q, const psa_bf16_t* k, const psa_bf16_t* v,
                         const float* kbar, const float* vsum,
                         const int* row_ptr, const int* col_idx, size_t col_capacity,
                         int B, int H, int N, int d, int block_size, int causal,
                         const psa_bf16_t* out, const float* lse, const psa_bf16_t* dout,
                         psa_bf16_t* dq, psa_bf16_t* dk, psa_bf16_t* dv,
                         void* workspace, size_t workspace_bytes, void* stream);

/*
 * Dense attention (density = 1: every candidate block exact) through the
 * same tensor-core kernel: the comparison baseline [PISA summary, "first
 * check: compare dense and PISA outputs on the same seed and input";
 * FlashAttention blog, section 1].  out = softmax(q k^T / sqrt(d)) v with
 * the causal mask when `causal`.  Needs a workspace (it pools the keys to
 * pick its softmax stabiliser).  Errors as psa_attn.
 */
PSA_API int psa_dense(const psa_bf16_t* q, const psa_bf16_t* k, const psa_bf16_t* v,
              int B, int H, int N, int d, int causal,
              psa_bf16_t* out, float* lse,
              void* workspace, size_t workspace_bytes, void* stream);

/*
 * Attention without a workspace, for callers that cannot allocate device
 * memory (the method's sources have no counterpart: this is an interface
 * choice).  Same computation, arguments and errors as psa_attn, minus the
 * workspace: the scratch (bf16 pooled keys and value sums, status word,
 * fixup lists, per-query denominators of the fixup rerun) lives in a 16 MiB
 * array inside the library, so shapes need
 * 256 + 8*B*H*M + 256*B*H*M + 4*B*H*M*d bytes (each part rounded up to 256
 * bytes) to fit in 16 MiB, else PSA_ERR_CAPACITY.  The first call on a device looks up the
 * array's device address (make it before any stream capture); so does the
 * first call after a device reset, which loads the library's device code
 * anew.  Every call on a device shares the array: calls whose work overlaps
 * on the GPU race.
 * `status` (device int, nullable) receives the device status word of this
 * call (PSA_OK, PSA_ERR_CSR or PSA_ERR_TIMEOUT) in stream order.  Never
 * allocates device memory.
 */
PSA_API int psa_attn_noalloc(const psa_bf16_t* q, const psa_bf16_t* k, const psa_bf16_t* v,
                             const float* kbar, const float* vsum,
                             const int* row_ptr, const int* col_idx, size_t col_capacity,
                             const float* row_max, int B, int H, int N, int d, int block_size,
                             int causal, psa_bf16_t* out, float* lse, int* status, void* stream);

/*
 * Test hook for the failure path (the method's sources have no counterpart;
 * never needed in normal use).  With on = 1, the next psa_attn call (only
 * that one, in this process) launches a kernel whose first block withholds
 * one internal hand-off, so the bounded waits behind it run out: the call
 * itself returns PSA_OK, the kernel stops within a few seconds and records
 * PSA_ERR_TIMEOUT in the workspace status word, and later calls run normally
 * on the same context.  on = 0 cancels a pending request.  Errors: PSA_ERR_ARG.
 */
PSA_API int psa_test_stall_next_attn(int on);

/*
 * Synchronises `stream`, then copies the device status word of `workspace`
 * into *status (host pointer): PSA_OK, or the first device-side error
 * recorded since the last call that reset it (the routers, psa_attn and
 * psa_dense reset it at their start).  Returns PSA_OK or PSA_ERR_CUDA.
 */
PSA_API int psa_read_status(const void* workspace, int* status, void* stream);

/*
 * Synchronises `stream`, then reports (host pointers) how often the last
 * psa_attn / psa_attn_hyd / psa_dense call on `workspace` left its fast path
 * (an implementation detail with no counterpart in the method's sources):
 *   *rerun = query blocks (64 rows each) with a row whose softmax
 *            denominator, under the kernel's fixed per-block stabiliser,
 *            left [2^-60, 2^60]; they were recomputed on the tensor cores
 *            with each query's own stabiliser (from the first pass's sum);
 *   *exact = those of them that the rerun still could not bring into range
 *            (a first-pass sum that was not finite), recomputed by the
 *            exact two-pass CUDA-core path.
 * Returns PSA_OK, PSA_ERR_ARG or PSA_ERR_CUDA.
 */
PSA_API int psa_read_fixup_count(const void* workspace, int* rerun, int* exact, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* PSA_H */
