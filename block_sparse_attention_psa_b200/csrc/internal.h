// internal.h -- launch helpers shared between the C-ABI layer (api.cu) and
// the kernel files.  Not part of the public interface.
#pragma once

#include <cstddef>
#include <cstdint>
#include <initializer_list>
#include <utility>
#include <cuda.h>
#include <cuda_runtime.h>

namespace psa {

// Launch with programmatic stream serialization: the kernel may be scheduled
// while the previous kernel of the stream is still running (after that one
// calls grid_dep_launch() in every CTA); the kernel itself calls
// grid_dep_wait() before touching global memory.
template <typename... KArgs, typename... Args>
cudaError_t launch_chained(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                           Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

constexpr int kBlock = 64;        // tokens per block (the only supported size)
constexpr int kMaxBlocks = 16384; // M limit (bitmaps and score rows on chip)

// Workspace layout (byte offsets, each 256-aligned).  The header holds the
// status word and the fixup counter.
struct WorkspaceLayout {
  size_t header = 0;        // int status, fixup_count, fixup_count2, sched[2]; ... (256 B, zeroed per call)
  size_t fixup_list = 0;    // int [B*H*M]   units flagged by the attention sweep
  size_t fixup_list2 = 0;   // int [B*H*M]   units still flagged by the rerun
  size_t row_lse2 = 0;      // fp32 [B*H*N] per query log2 denominator of the sweep
  size_t kbar_bf16 = 0;     // bf16 [B*H*M*d]
  size_t vsum_bf16 = 0;     // bf16 [B*H*M*d] (value sums)
  size_t row_count = 0;     // int [B*H*M]     (threshold routing)
  size_t row_bits = 0;      // uint32 [B*H*M*ceil(M/32)]
  size_t q_split = 0;       // bf16 [3][B*H*M*d] (three-part split of qbar, routing)
  size_t k_split = 0;       // bf16 [3][B*H*M*d] (same for kbar)
  size_t hyd_w = 0;         // fp32 [B*H*N] (first-order mode: 0th-order share per query)
  size_t hyd_partial = 0;   // fp32 partial statistics of the first-order mode
  size_t bwd_part = 0;      // fp32 partial pseudo-key gradients of the backward (two halves)
  size_t scores = 0;        // fp32 [score_heads][M][Mp] block scores of one batch of heads
  int score_heads = 0;      // heads per routing batch
  size_t total = 0;
};
WorkspaceLayout workspace_layout(long long BH, long long M, long long d);

// Routing scratch inside the workspace.
struct RouteScratch {
  uint16_t* q_split;
  uint16_t* k_split;
  float* scores;
  int heads_per_batch;
  int* status;
};

// score.cu: block scores s_IJ = qbar_I . kbar_J / sqrt(d) on the tensor cores
int score_stride(int M);  // Mp: M rounded up to the 128-column score tile
// three-way bf16 split of two fp32 arrays of n values each, in one launch
cudaError_t launch_split3(const float* x0, const float* x1, long long n, uint16_t* out0, uint16_t* out1,
                          cudaStream_t st);
struct ScorePlan {
  CUtensorMap mq, mk;  // the split operands, 128-row x 64-feature boxes
  int BH = 0, M = 0, d = 0, Mp = 0;
  cudaError_t init(const uint16_t* q_split, const uint16_t* k_split, int BH, int M, int d);
  // scores of heads [bh0, bh0 + nh) into scores[nh][M][Mp]
  cudaError_t run(int bh0, int nh, int causal, float* scores, int* status, cudaStream_t st) const;
};

// pool.cu
cudaError_t launch_pool(const uint16_t* q, const uint16_t* k, const uint16_t* v, int BH, int M, int d,
                        float* qbar, float* kbar, float* vsum, cudaStream_t st);
cudaError_t launch_pool_keys_bf16(const uint16_t* k, int BH, int M, int d, uint16_t* kbar_bf16,
                                  cudaStream_t st);
// zero the 256-byte header of a workspace (a chained launch, in place of a memset)
cudaError_t launch_zero_header(void* workspace, cudaStream_t st);
cudaError_t launch_stats_to_bf16(const float* kbar, const float* vsum, long long n, uint16_t* kbar_bf16,
                                 uint16_t* vsum_bf16, cudaStream_t st);

// route.cu
cudaError_t launch_route_topk(const float* qbar, const float* kbar, int BH, int M, int d, int k0, int causal,
                              int* row_ptr, int* col_idx, long long total, int* nnz_out, float* row_max,
                              const RouteScratch& w, cudaStream_t st);
// threshold thr_I = a_mul * max_J s_IJ + a_add (one fma)
cudaError_t launch_route_thresh(const float* qbar, const float* kbar, int BH, int M, int d, float a_mul,
                                float a_add, int causal, int keep_first, int* row_ptr, int* col_idx, long long capacity,
                                int* nnz_out, int* row_count, uint32_t* row_bits, float* row_max,
                                const RouteScratch& w, cudaStream_t st);

// attn.cu
struct AttnLaunch {
  const uint16_t* q;
  const uint16_t* k;
  const uint16_t* v;
  const uint16_t* kbar_bf16;
  const uint16_t* vsum_bf16;
  const int* row_ptr;   // null in dense mode
  const int* col_idx;   // null in dense mode
  long long col_cap;
  const float* row_max; // per row max block score (nullable: computed in the kernel)
  uint16_t* out;
  float* lse;
  int BH, N, M, d, causal, dense;
  int* status;
  int* fixup_count;   // units the first pass flagged (rerun with per-query stabilisers)
  int* fixup_list;
  int* fixup_count2;  // units the rerun still flagged (exact CUDA-core path)
  int* fixup_list2;
  float* row_lse2;    // [BH * N]: per query, the first pass's log2 denominator
  int* sched;         // [2] zeroed ticket counters of the attention sweep and of its rerun
  int stall;  // failure-path test hook (0 in normal use)
  int hyd = 0;             // first-order mode: also write hyd_w (per query, 0th-order share)
  float* hyd_w = nullptr;  // [BH * N] fp32 (hyd mode only)
};
cudaError_t launch_attn(const AttnLaunch& a, cudaStream_t st);

// bwd.cu: gradients of the 0th-order attention for fixed block lists
struct BwdLaunch {
  const uint16_t* q;
  const uint16_t* k;
  const uint16_t* v;
  const uint16_t* kbar_bf16;
  const uint16_t* vsum_bf16;
  const int* row_ptr;
  const int* col_idx;
  long long col_cap;
  const uint16_t* out;   // the forward's output
  const float* lse;      // the forward's lse (natural log)
  const uint16_t* dout;
  uint16_t* dq;
  uint16_t* dk;
  uint16_t* dv;
  int BH, N, M, d, causal;
  int* status;
  int* sched;            // ticket counter of the dk, dv item scheduler (zeroed header word)
  // workspace
  uint32_t* bits;        // [BH*M][ceil(M/32)]
  float* nlse2;          // [BH*N]
  float* delta;          // [BH*N]
  float* part_dvs;       // partial pseudo-key gradients
  float* part_dkb;
  float* dvsum;          // [BH*M*d]
  float* dkbar;          // [BH*M*d]
};
size_t bwd_partial_bytes(int BH, int M, int d);
cudaError_t launch_bwd(const BwdLaunch& a, cudaStream_t st);

// hyd.cu: the first-order correction
// partial matrices of the statistic kernel (bytes, for the workspace)
size_t hyd_partial_bytes(int BH, int M, int d);
// hstat[BH][d][d] = mean over the blocks J of sum_{j in J} (k_j - kbar_J) v_j^T
cudaError_t launch_hyd_stat(const uint16_t* k, const uint16_t* v, const float* kbar, const float* vsum, int BH,
                            int N, int d, float* partial, float* hstat, int* status, cudaStream_t st);
// out[i] += w[i] * (q_i^T H) / sqrt(d), in place
cudaError_t launch_hyd_apply(const uint16_t* q, const float* hstat, const float* w, uint16_t* out, int BH, int N,
                             int d, int* status, cudaStream_t st);

// api.cu: one-shot flag set by psa_test_stall_next_attn, taken by the next psa_attn
int take_stall_request();

// api.cu: driver entry point for cuTensorMapEncodeTiled (resolved once)
CUresult encode_tensor_map_3d_bf16(CUtensorMap* map, const void* base, uint64_t inner, uint64_t rows,
                                   uint64_t outer, uint32_t box_inner, uint32_t box_rows);
int device_sm_count();
// PSA_OK if the current device is sm_100 and every non-null pointer names
// device (or managed) memory of that device; else PSA_ERR_DEVICE / PSA_ERR_ARG.
int check_device_pointers(std::initializer_list<const void*> ptrs);

}  // namespace psa
