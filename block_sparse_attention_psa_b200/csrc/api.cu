// api.cu -- the C ABI declared in include/psa.h: argument validation on the
// host, workspace layout, TMA descriptor encoding and kernel launches.
#include <climits>
#include <atomic>
#include <cmath>
#include <cstring>
#include <initializer_list>
#include <mutex>

#include "internal.h"
#include "psa.h"

namespace psa {

static size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

WorkspaceLayout workspace_layout(long long BH, long long M, long long d) {
  WorkspaceLayout L;
  size_t o = 256;
  L.header = 0;
  L.fixup_list = o;
  o += align256(static_cast<size_t>(BH * M) * 4);
  L.fixup_list2 = o;
  o += align256(static_cast<size_t>(BH * M) * 4);
  L.row_lse2 = o;
  o += align256(static_cast<size_t>(BH * M * 64) * 4);
  L.kbar_bf16 = o;
  o += align256(static_cast<size_t>(BH * M * d) * 2);
  L.vsum_bf16 = o;
  o += align256(static_cast<size_t>(BH * M * d) * 2);
  L.row_count = o;
  o += align256(static_cast<size_t>(BH * M) * 4);
  L.row_bits = o;
  o += align256(static_cast<size_t>(BH * M * ((M + 31) / 32)) * 4);
  L.q_split = o;
  o += align256(static_cast<size_t>(3 * BH * M * d) * 2);
  L.k_split = o;
  o += align256(static_cast<size_t>(3 * BH * M * d) * 2);
  L.hyd_w = o;
  o += align256(static_cast<size_t>(BH * M * 64) * 4);
  L.hyd_partial = o;
  o += align256(psa::hyd_partial_bytes(static_cast<int>(BH), static_cast<int>(M), static_cast<int>(d)));
  L.bwd_part = o;
  o += 2 * align256(psa::bwd_partial_bytes(static_cast<int>(BH), static_cast<int>(M), static_cast<int>(d)));
  // block scores of as many heads as fit 256 MB (at least one)
  const size_t head_scores = static_cast<size_t>(M) * score_stride(static_cast<int>(M)) * 4;
  const long long fit = static_cast<long long>((size_t(256) << 20) / head_scores);
  L.score_heads = static_cast<int>(fit < 1 ? 1 : (fit > BH ? BH : fit));
  L.scores = o;
  o += align256(head_scores * L.score_heads);
  L.total = o;
  return L;
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  });
  return fn;
}

CUresult encode_tensor_map_3d_bf16(CUtensorMap* map, const void* base, uint64_t inner, uint64_t rows,
                                   uint64_t outer, uint32_t box_inner, uint32_t box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return CUDA_ERROR_NOT_FOUND;
  const cuuint64_t dims[3] = {inner, rows, outer};
  const cuuint64_t strides[2] = {inner * 2, inner * rows * 2};
  const cuuint32_t box[3] = {box_inner, box_rows, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
}

int device_sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 1;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n < 1) return 1;
  return n;
}

// The current device must be an sm_100 part, and the memory each pointer
// names must live on it: a kernel launched on the current device would
// otherwise address another GPU's memory (or host memory) through its TMA
// descriptors and bulk stores.  Host and unregistered memory is rejected.
int check_device_pointers(std::initializer_list<const void*> ptrs) {
  int dev = 0, major = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return PSA_ERR_DEVICE;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess)
    return PSA_ERR_DEVICE;
  if (major != 10) return PSA_ERR_DEVICE;
  for (const void* p : ptrs) {
    if (!p) continue;
    cudaPointerAttributes at;
    if (cudaPointerGetAttributes(&at, p) != cudaSuccess) {
      cudaGetLastError();  // clear the sticky-free error of the query
      return PSA_ERR_ARG;
    }
    if (at.type != cudaMemoryTypeDevice && at.type != cudaMemoryTypeManaged) return PSA_ERR_ARG;
    if (at.type == cudaMemoryTypeDevice && at.device != dev) return PSA_ERR_DEVICE;
  }
  return PSA_OK;
}

std::atomic<int> g_stall_request{0};

int take_stall_request() { return g_stall_request.exchange(0); }

}  // namespace psa

using psa::kBlock;
using psa::kMaxBlocks;

namespace {

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int check_shape(int B, int H, int N, int d, int block_size) {
  if (B <= 0 || H <= 0 || N <= 0 || d <= 0) return PSA_ERR_ARG;
  if (block_size != kBlock) return PSA_ERR_UNSUPPORTED;
  if (d != 64 && d != 128) return PSA_ERR_UNSUPPORTED;
  if (N % kBlock) return PSA_ERR_SHAPE;
  if (N / kBlock > kMaxBlocks) return PSA_ERR_UNSUPPORTED;
  if (static_cast<long long>(B) * H * N * d >= (1LL << 31)) return PSA_ERR_SHAPE;
  return PSA_OK;
}

int check_device(std::initializer_list<const void*> ptrs) { return psa::check_device_pointers(ptrs); }

int cuda_status(cudaError_t e) { return e == cudaSuccess ? PSA_OK : PSA_ERR_CUDA; }

long long causal_prefix(long long I, long long k0) {
  if (I <= k0) return I * (I + 1) / 2;
  return k0 * (k0 + 1) / 2 + (I - k0) * k0;
}

}  // namespace

namespace {

psa::RouteScratch route_scratch(char* ws, const psa::WorkspaceLayout& L) {
  psa::RouteScratch w;
  w.q_split = reinterpret_cast<uint16_t*>(ws + L.q_split);
  w.k_split = reinterpret_cast<uint16_t*>(ws + L.k_split);
  w.scores = reinterpret_cast<float*>(ws + L.scores);
  w.heads_per_batch = L.score_heads;
  w.status = reinterpret_cast<int*>(ws + L.header);
  return w;
}

// Shared by both threshold routers: thr_I = a_mul * max_J s_IJ + a_add.
int route_thresh_common(const float* qbar, const float* kbar, int B, int H, int M, int d, float a_mul, float a_add,
                        int causal, int keep_first, int* row_ptr, int* col_idx, size_t capacity, int* nnz_out,
                        float* row_max, void* workspace, size_t workspace_bytes, void* stream) {
  if (!qbar || !kbar || !row_ptr || !col_idx || !nnz_out || !workspace) return PSA_ERR_ARG;
  if (reinterpret_cast<uintptr_t>(row_max) & 3u) return PSA_ERR_ARG;
  if (M <= 0) return PSA_ERR_ARG;
  if (M > kMaxBlocks) return PSA_ERR_UNSUPPORTED;
  int s = check_shape(B, H, M * kBlock, d, kBlock);
  if (s != PSA_OK) return s;
  if ((causal != 0 && causal != 1) || (keep_first != 0 && keep_first != 1)) return PSA_ERR_ARG;
  if (!aligned16(qbar) || !aligned16(kbar) || (reinterpret_cast<uintptr_t>(workspace) & 255u)) return PSA_ERR_ARG;
  const long long bh = static_cast<long long>(B) * H;
  const psa::WorkspaceLayout L = psa::workspace_layout(bh, M, d);
  if (workspace_bytes < L.total) return PSA_ERR_CAPACITY;
  if ((s = check_device({qbar, row_ptr, workspace})) != PSA_OK) return s;
  const long long cap = capacity > static_cast<size_t>(INT_MAX) ? INT_MAX : static_cast<long long>(capacity);
  char* ws = static_cast<char*>(workspace);
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (psa::launch_zero_header(ws, st) != cudaSuccess) return PSA_ERR_CUDA;
  return cuda_status(psa::launch_route_thresh(qbar, kbar, static_cast<int>(bh), M, d, a_mul, a_add, causal,
                                              keep_first, row_ptr, col_idx, cap, nnz_out,
                                              reinterpret_cast<int*>(ws + L.row_count),
                                              reinterpret_cast<uint32_t*>(ws + L.row_bits), row_max,
                                              route_scratch(ws, L), st));
}

// psa_attn, and with `hstat` the first-order mode of psa_attn_hyd
int attn_common(const psa_bf16_t* q, const psa_bf16_t* k, const psa_bf16_t* v, const float* kbar,
                const float* vsum, const float* hstat, const int* row_ptr, const int* col_idx, size_t col_capacity,
                const float* row_max, int B, int H, int N, int d, int block_size, int causal, psa_bf16_t* out,
                float* lse, void* workspace, size_t workspace_bytes, void* stream) {
  if (!q || !k || !v || !kbar || !vsum || !row_ptr || !col_idx || !out || !workspace) return PSA_ERR_ARG;
  int s = check_shape(B, H, N, d, block_size);
  if (s != PSA_OK) return s;
  if (causal != 0 && causal != 1) return PSA_ERR_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || !aligned16(kbar) ||
      !aligned16(vsum) || (reinterpret_cast<uintptr_t>(workspace) & 255u) ||
      (lse && (reinterpret_cast<uintptr_t>(lse) & 3u)) || (reinterpret_cast<uintptr_t>(row_max) & 3u) ||
      (reinterpret_cast<uintptr_t>(hstat) & 15u))
    return PSA_ERR_ARG;
  const long long bh = static_cast<long long>(B) * H;
  const int M = N / kBlock;
  const psa::WorkspaceLayout L = psa::workspace_layout(bh, M, d);
  if (workspace_bytes < L.total) return PSA_ERR_CAPACITY;
  if ((s = check_device({q, out, workspace})) != PSA_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  char* ws = static_cast<char*>(workspace);
  cudaError_t e = psa::launch_zero_header(ws, st);
  if (e != cudaSuccess) return PSA_ERR_CUDA;
  uint16_t* kb16 = reinterpret_cast<uint16_t*>(ws + L.kbar_bf16);
  uint16_t* vb16 = reinterpret_cast<uint16_t*>(ws + L.vsum_bf16);
  e = psa::launch_stats_to_bf16(kbar, vsum, bh * M * d, kb16, vb16, st);
  if (e != cudaSuccess) return PSA_ERR_CUDA;
  psa::AttnLaunch a;
  a.q = q;
  a.k = k;
  a.v = v;
  a.kbar_bf16 = kb16;
  a.vsum_bf16 = vb16;
  a.row_ptr = row_ptr;
  a.col_idx = col_idx;
  a.col_cap = col_capacity > static_cast<size_t>(LLONG_MAX) ? LLONG_MAX : static_cast<long long>(col_capacity);
  a.row_max = row_max;
  a.stall = psa::take_stall_request();
  a.out = out;
  a.lse = lse;
  a.BH = static_cast<int>(bh);
  a.N = N;
  a.M = M;
  a.d = d;
  a.causal = causal;
  a.dense = 0;
  a.status = reinterpret_cast<int*>(ws);
  a.fixup_count = reinterpret_cast<int*>(ws) + 1;
  a.fixup_list = reinterpret_cast<int*>(ws + L.fixup_list);
  a.fixup_count2 = reinterpret_cast<int*>(ws) + 2;
  a.sched = reinterpret_cast<int*>(ws) + 3;
  a.fixup_list2 = reinterpret_cast<int*>(ws + L.fixup_list2);
  a.row_lse2 = reinterpret_cast<float*>(ws + L.row_lse2);
  a.hyd = hstat != nullptr;
  a.hyd_w = hstat ? reinterpret_cast<float*>(ws + L.hyd_w) : nullptr;
  if ((e = psa::launch_attn(a, st)) != cudaSuccess) return PSA_ERR_CUDA;
  if (hstat)
    e = psa::launch_hyd_apply(q, hstat, a.hyd_w, out, a.BH, N, d, a.status, st);
  return cuda_status(e);
}

}  // namespace

extern "C" {

const char* psa_status_string(int status) {
  switch (status) {
    case PSA_OK: return "ok";
    case PSA_ERR_ARG: return "invalid argument (null pointer, non-positive size or bad flag)";
    case PSA_ERR_SHAPE: return "bad shape (N not a multiple of block_size, or tensor too large)";
    case PSA_ERR_UNSUPPORTED: return "unsupported configuration (block_size != 64, d not in {64,128}, M > 16384)";
    case PSA_ERR_CAPACITY: return "capacity too small (workspace or block-list buffer)";
    case PSA_ERR_CUDA: return "a CUDA runtime call failed";
    case PSA_ERR_TIMEOUT: return "device: a bounded wait ran out and the kernel stopped";
    case PSA_ERR_CSR: return "device: a block list entry was out of range or repeated";
    case PSA_ERR_DEVICE: return "no sm_100 (B200) device is current, or a tensor lives on another device";
    default: return "unknown status";
  }
}

int psa_version(void) { return 200; }

size_t psa_workspace_size(int B, int H, int N, int d) {
  if (check_shape(B, H, N, d, kBlock) != PSA_OK) return 0;
  return psa::workspace_layout(static_cast<long long>(B) * H, N / kBlock, d).total;
}

size_t psa_route_capacity(int B, int H, int M, int causal) {
  if (B <= 0 || H <= 0 || M <= 0) return 0;
  const size_t bh = static_cast<size_t>(B) * H, m = static_cast<size_t>(M);
  return causal ? bh * m * (m + 1) / 2 : bh * m * m;
}

int psa_pool(const psa_bf16_t* q, const psa_bf16_t* k, const psa_bf16_t* v, int B, int H, int N, int d,
             int block_size, float* qbar, float* kbar, float* vsum, void* stream) {
  if (!q || !k || !v || !qbar || !kbar || !vsum) return PSA_ERR_ARG;
  int s = check_shape(B, H, N, d, block_size);
  if (s != PSA_OK) return s;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(qbar) || !aligned16(kbar) ||
      !aligned16(vsum))
    return PSA_ERR_ARG;
  if ((s = check_device({q, qbar})) != PSA_OK) return s;
  return cuda_status(psa::launch_pool(q, k, v, B * H, N / kBlock, d, qbar, kbar, vsum,
                                      static_cast<cudaStream_t>(stream)));
}

int psa_route_topk(const float* qbar, const float* kbar, int B, int H, int M, int d, float density, int causal,
                   int* row_ptr, int* col_idx, size_t capacity, int* nnz_out, float* row_max, void* workspace,
                   size_t workspace_bytes, void* stream) {
  if (!qbar || !kbar || !row_ptr || !col_idx || !nnz_out || !workspace) return PSA_ERR_ARG;
  if (reinterpret_cast<uintptr_t>(row_max) & 3u) return PSA_ERR_ARG;
  if (M <= 0) return PSA_ERR_ARG;
  if (M > kMaxBlocks) return PSA_ERR_UNSUPPORTED;
  int s = check_shape(B, H, M * kBlock, d, kBlock);
  if (s != PSA_OK) return s;
  if (!(density >= 0.0f) || std::isinf(density)) return PSA_ERR_ARG;
  if (causal != 0 && causal != 1) return PSA_ERR_ARG;
  if (!aligned16(qbar) || !aligned16(kbar) || (reinterpret_cast<uintptr_t>(workspace) & 255u)) return PSA_ERR_ARG;
  // k = clamp(ceil(fl32(density * M)), 1, #candidates): single-precision product
  volatile float prod = density * static_cast<float>(M);
  double kc = std::ceil(static_cast<double>(prod));
  long long k0 = kc < 1.0 ? 1 : (kc > M ? M : static_cast<long long>(kc));
  const long long bh = static_cast<long long>(B) * H;
  const long long total = causal ? bh * causal_prefix(M, k0) : bh * M * k0;
  if (total > INT_MAX || static_cast<size_t>(total) > capacity) return PSA_ERR_CAPACITY;
  const psa::WorkspaceLayout L = psa::workspace_layout(bh, M, d);
  if (workspace_bytes < L.total) return PSA_ERR_CAPACITY;
  if ((s = check_device({qbar, row_ptr, workspace})) != PSA_OK) return s;
  char* ws = static_cast<char*>(workspace);
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (psa::launch_zero_header(ws, st) != cudaSuccess) return PSA_ERR_CUDA;
  return cuda_status(psa::launch_route_topk(qbar, kbar, static_cast<int>(bh), M, d, static_cast<int>(k0),
                                            causal, row_ptr, col_idx, total, nnz_out, row_max,
                                            route_scratch(ws, L), st));
}

int psa_route_thresh(const float* qbar, const float* kbar, int B, int H, int M, int d, float alpha, int causal,
                     int keep_first, int* row_ptr, int* col_idx, size_t capacity, int* nnz_out, float* row_max,
                     void* workspace, size_t workspace_bytes, void* stream) {
  if (!std::isfinite(alpha)) return PSA_ERR_ARG;
  return route_thresh_common(qbar, kbar, B, H, M, d, alpha, 0.0f, causal, keep_first, row_ptr, col_idx, capacity,
                             nnz_out, row_max, workspace, workspace_bytes, stream);
}

int psa_route_thresh_prob(const float* qbar, const float* kbar, int B, int H, int M, int d, float alpha,
                          int causal, int keep_first, int* row_ptr, int* col_idx, size_t capacity, int* nnz_out,
                          float* row_max, void* workspace, size_t workspace_bytes, void* stream) {
  if (!(alpha > 0.0f) || !std::isfinite(alpha)) return PSA_ERR_ARG;
  const float log_alpha = static_cast<float>(std::log(static_cast<double>(alpha)));
  return route_thresh_common(qbar, kbar, B, H, M, d, 1.0f, log_alpha, causal, keep_first, row_ptr, col_idx,
                             capacity, nnz_out, row_max, workspace, workspace_bytes, stream);
}

int psa_attn(const psa_bf16_t* q, const psa_bf16_t* k, const psa_bf16_t* v, const float* kbar, const float* vsum,
             const int* row_ptr, const int* col_idx, size_t col_capacity, const float* row_max, int B, int H,
             int N, int d, int block_size, int causal, psa_bf16_t* out, float* lse, void* workspace,
             size_t workspace_bytes, void* stream) {
  return attn_common(q, k, v, kbar, vsum, nullptr, row_ptr, col_idx, col_capacity, row_max, B, H, N, d, block_size,
                     causal, out, lse, workspace, workspace_bytes, stream);
}

int psa_attn_hyd(const psa_bf16_t* q, const psa_bf16_t* k, const psa_bf16_t* v, const float* kbar,
                 const float* vsum, const float* hstat, const int* row_ptr, const int* col_idx, size_t col_capacity,
                 const float* row_max, int B, int H, int N, int d, int block_size, int causal, psa_bf16_t* out,
                 float* lse, void* workspace, size_t workspace_bytes, void* stream) {
  if (!hstat) return PSA_ERR_ARG;
  return attn_common(q, k, v, kbar, vsum, hstat, row_ptr, col_idx, col_capacity, row_max, B, H, N, d, block_size,
                     causal, out, lse, workspace, workspace_bytes, stream);
}

int psa_attn_bwd(const psa_bf16_t* q, const psa_bf16_t* k, const psa_bf16_t* v, const float* kbar,
                 const float* vsum, const int* row_ptr, const int* col_idx, size_t col_capacity, int B, int H, int N,
                 int d, int block_size, int causal, const psa_bf16_t* out, const float* lse, const psa_bf16_t* dout,
                 psa_bf16_t* dq, psa_bf16_t* dk, psa_bf16_t* dv, void* workspace, size_t workspace_bytes,
                 void* stream) {
  if (!q || !k || !v || !kbar || !vsum || !row_ptr || !col_idx || !out || !lse || !dout || !dq || !dk || !dv ||
      !workspace)
    return PSA_ERR_ARG;
  int s = check_shape(B, H, N, d, block_size);
  if (s != PSA_OK) return s;
  if (causal != 0 && causal != 1) return PSA_ERR_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(kbar) || !aligned16(vsum) || !aligned16(out) ||
      !aligned16(dout) || !aligned16(dq) || !aligned16(dk) || !aligned16(dv) ||
      (reinterpret_cast<uintptr_t>(lse) & 3u) || (reinterpret_cast<uintptr_t>(workspace) & 255u))
    return PSA_ERR_ARG;
  const long long bh = static_cast<long long>(B) * H;
  const int M = N / kBlock;
  const psa::WorkspaceLayout L = psa::workspace_layout(bh, M, d);
  if (workspace_bytes < L.total) return PSA_ERR_CAPACITY;
  if ((s = check_device({q, dout, dq, workspace})) != PSA_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  char* ws = static_cast<char*>(workspace);
  if (psa::launch_zero_header(ws, st) != cudaSuccess) return PSA_ERR_CUDA;
  uint16_t* kb16 = reinterpret_cast<uint16_t*>(ws + L.kbar_bf16);
  uint16_t* vb16 = reinterpret_cast<uint16_t*>(ws + L.vsum_bf16);
  if (psa::launch_stats_to_bf16(kbar, vsum, bh * M * d, kb16, vb16, st) != cudaSuccess) return PSA_ERR_CUDA;
  psa::BwdLaunch a;
  a.q = q;
  a.k = k;
  a.v = v;
  a.kbar_bf16 = kb16;
  a.vsum_bf16 = vb16;
  a.row_ptr = row_ptr;
  a.col_idx = col_idx;
  a.col_cap = col_capacity > static_cast<size_t>(LLONG_MAX) ? LLONG_MAX : static_cast<long long>(col_capacity);
  a.out = out;
  a.lse = lse;
  a.dout = dout;
  a.dq = dq;
  a.dk = dk;
  a.dv = dv;
  a.BH = static_cast<int>(bh);
  a.N = N;
  a.M = M;
  a.d = d;
  a.causal = causal;
  a.status = reinterpret_cast<int*>(ws);
  a.sched = reinterpret_cast<int*>(ws) + 8;
  // scratch of the backward: regions the forward calls use only within a call
  a.bits = reinterpret_cast<uint32_t*>(ws + L.row_bits);
  a.nlse2 = reinterpret_cast<float*>(ws + L.row_lse2);
  a.delta = reinterpret_cast<float*>(ws + L.hyd_w);
  a.dvsum = reinterpret_cast<float*>(ws + L.q_split);
  a.dkbar = reinterpret_cast<float*>(ws + L.k_split);
  const size_t part = (psa::bwd_partial_bytes(a.BH, M, d) + 255) & ~static_cast<size_t>(255);
  a.part_dvs = reinterpret_cast<float*>(ws + L.bwd_part);
  a.part_dkb = reinterpret_cast<float*>(ws + L.bwd_part + part);
  return cuda_status(psa::launch_bwd(a, st));
}

int psa_hyd_stat(const psa_bf16_t* k, const psa_bf16_t* v, const float* kbar, const float* vsum, int B, int H,
                 int N, int d, float* hstat, void* workspace, size_t workspace_bytes, void* stream) {
  if (!k || !v || !kbar || !vsum || !hstat || !workspace) return PSA_ERR_ARG;
  int s = check_shape(B, H, N, d, kBlock);
  if (s != PSA_OK) return s;
  if (!aligned16(k) || !aligned16(v) || !aligned16(kbar) || !aligned16(vsum) || !aligned16(hstat) ||
      (reinterpret_cast<uintptr_t>(workspace) & 255u))
    return PSA_ERR_ARG;
  const long long bh = static_cast<long long>(B) * H;
  const int M = N / kBlock;
  const psa::WorkspaceLayout L = psa::workspace_layout(bh, M, d);
  if (workspace_bytes < L.total) return PSA_ERR_CAPACITY;
  if ((s = check_device({k, hstat, workspace})) != PSA_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  char* ws = static_cast<char*>(workspace);
  if (psa::launch_zero_header(ws, st) != cudaSuccess) return PSA_ERR_CUDA;
  return cuda_status(psa::launch_hyd_stat(k, v, kbar, vsum, static_cast<int>(bh), N, d,
                                          reinterpret_cast<float*>(ws + L.hyd_partial), hstat,
                                          reinterpret_cast<int*>(ws), st));
}

int psa_dense(const psa_bf16_t* q, const psa_bf16_t* k, const psa_bf16_t* v, int B, int H, int N, int d,
              int causal, psa_bf16_t* out, float* lse, void* workspace, size_t workspace_bytes, void* stream) {
  if (!q || !k || !v || !out || !workspace) return PSA_ERR_ARG;
  int s = check_shape(B, H, N, d, kBlock);
  if (s != PSA_OK) return s;
  if (causal != 0 && causal != 1) return PSA_ERR_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) ||
      (reinterpret_cast<uintptr_t>(workspace) & 255u) || (lse && (reinterpret_cast<uintptr_t>(lse) & 3u)))
    return PSA_ERR_ARG;
  const long long bh = static_cast<long long>(B) * H;
  const int M = N / kBlock;
  const psa::WorkspaceLayout L = psa::workspace_layout(bh, M, d);
  if (workspace_bytes < L.total) return PSA_ERR_CAPACITY;
  if ((s = check_device({q, out, workspace})) != PSA_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  char* ws = static_cast<char*>(workspace);
  cudaError_t e = psa::launch_zero_header(ws, st);
  if (e != cudaSuccess) return PSA_ERR_CUDA;
  uint16_t* kb16 = reinterpret_cast<uint16_t*>(ws + L.kbar_bf16);
  e = psa::launch_pool_keys_bf16(k, static_cast<int>(bh), M, d, kb16, st);
  if (e != cudaSuccess) return PSA_ERR_CUDA;
  psa::AttnLaunch a;
  std::memset(&a, 0, sizeof(a));
  a.q = q;
  a.k = k;
  a.v = v;
  a.kbar_bf16 = kb16;
  a.vsum_bf16 = kb16;
  a.out = out;
  a.lse = lse;
  a.BH = static_cast<int>(bh);
  a.N = N;
  a.M = M;
  a.d = d;
  a.causal = causal;
  a.dense = 1;
  a.status = reinterpret_cast<int*>(ws);
  a.fixup_count = reinterpret_cast<int*>(ws) + 1;
  a.fixup_list = reinterpret_cast<int*>(ws + L.fixup_list);
  a.fixup_count2 = reinterpret_cast<int*>(ws) + 2;
  a.sched = reinterpret_cast<int*>(ws) + 3;
  a.fixup_list2 = reinterpret_cast<int*>(ws + L.fixup_list2);
  a.row_lse2 = reinterpret_cast<float*>(ws + L.row_lse2);
  return cuda_status(psa::launch_attn(a, st));
}

int psa_test_stall_next_attn(int on) {
  if (on != 0 && on != 1) return PSA_ERR_ARG;
  psa::g_stall_request.store(on);
  return PSA_OK;
}

int psa_read_fixup_count(const void* workspace, int* rerun, int* exact, void* stream) {
  if (!workspace || !rerun || !exact) return PSA_ERR_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(st) != cudaSuccess) return PSA_ERR_CUDA;
  int v[2] = {0, 0};
  if (cudaMemcpy(v, static_cast<const int*>(workspace) + 1, sizeof(v), cudaMemcpyDeviceToHost) != cudaSuccess)
    return PSA_ERR_CUDA;
  *rerun = v[0];
  *exact = v[1];
  return PSA_OK;
}

int psa_read_status(const void* workspace, int* status, void* stream) {
  if (!workspace || !status) return PSA_ERR_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(st) != cudaSuccess) return PSA_ERR_CUDA;
  int v = 0;
  if (cudaMemcpy(&v, workspace, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return PSA_ERR_CUDA;
  *status = v;
  return PSA_OK;
}

}  // extern "C"
