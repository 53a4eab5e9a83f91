// noalloc.cu -- psa_attn_noalloc: the attention step without a caller
// workspace, for callers that cannot allocate device memory.
//
// Some callers cannot call cudaMalloc (or any allocating routine) at the
// point where they run attention: plugins inside frameworks whose device
// memory all comes from the framework's own pool, or real-time and
// safety-critical loops that forbid allocation after start-up.  This entry point needs nothing from them but
// the inputs and outputs: its scratch (the bf16 copies of the pooled keys
// and value sums, the status word, the fixup lists and the per-query
// denominators the fixup rerun starts from) lives in one file-scope device
// array below.
//
// That array is shared by every call on a device and keeps the previous
// call's contents; the parts that must start at zero (status word, fixup
// counter) are cleared by each call.  Two calls whose kernels overlap on the
// GPU (different streams, no ordering between them) therefore race on it.
#include <climits>
#include <mutex>

#include "internal.h"
#include "psa.h"

namespace {

// 16 MiB of scratch, 256-byte aligned.  Every GPU that loads this library
// holds it until the process exits.
constexpr size_t kNoAllocScratchBytes = size_t(16) << 20;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_setup_mutex;
// per device: the device address of the array in the context it was looked
// up in, and that context's unique id (ids are never reused, so a reset
// device, whose next context reloads the module, is set up again)
void* g_scratch_ptr[kMaxDevices] = {};
unsigned long long g_scratch_ctx[kMaxDevices] = {};

size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

// Scratch bytes the attention step needs: header, the first fixup list, bf16
// pooled keys and bf16 value sums, the second fixup list and the per-query
// log2 denominators of the first pass.
size_t scratch_bytes(long long BH, long long M, long long d) {
  return 256 + 2 * align256(static_cast<size_t>(BH * M) * 4) + 2 * align256(static_cast<size_t>(BH * M * d) * 2) +
         align256(static_cast<size_t>(BH * M * 64) * 4);
}

typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long*);

// Unique id of the current device's context (0 if it cannot be read).
unsigned long long current_context_id() {
  static CtxGetCurrentFn get_current = nullptr;
  static CtxGetIdFn get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<CtxGetCurrentFn>(p);
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<CtxGetIdFn>(p);
  });
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (!get_current || !get_id || get_current(&ctx) != CUDA_SUCCESS || !ctx || get_id(ctx, &id) != CUDA_SUCCESS)
    return 0;
  return id;
}

// Device address of the scratch array on the current device.  The host-side
// symbol is only a stand-in, never a device address: the address is looked up
// with the device current, once per device context (the first call on a
// device, and the first after a device reset), and cached.
int scratch_for_current_device(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return PSA_ERR_DEVICE;
  // the device's primary context, current on this thread (cudaSetDevice
  // initialises it, so the context id below is the one kernels run in)
  if (cudaSetDevice(dev) != cudaSuccess) return PSA_ERR_DEVICE;
  const unsigned long long ctx = current_context_id();
  std::lock_guard<std::mutex> lock(g_setup_mutex);
  if (!g_scratch_ptr[dev] || ctx == 0 || g_scratch_ctx[dev] != ctx) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess || !ptr) return PSA_ERR_CUDA;
    g_scratch_ptr[dev] = ptr;
    g_scratch_ctx[dev] = ctx;
  }
  *out = g_scratch_ptr[dev];
  return PSA_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

extern "C" {

int psa_attn_noalloc(const psa_bf16_t* q, const psa_bf16_t* k, const psa_bf16_t* v, const float* kbar,
                     const float* vsum, const int* row_ptr, const int* col_idx, size_t col_capacity,
                     const float* row_max, int B, int H, int N, int d, int block_size, int causal, psa_bf16_t* out,
                     float* lse, int* status, void* stream) {
  if (!q || !k || !v || !kbar || !vsum || !row_ptr || !col_idx || !out) return PSA_ERR_ARG;
  if (B <= 0 || H <= 0 || N <= 0 || d <= 0) return PSA_ERR_ARG;
  if (block_size != psa::kBlock || (d != 64 && d != 128)) return PSA_ERR_UNSUPPORTED;
  if (N % psa::kBlock) return PSA_ERR_SHAPE;
  if (N / psa::kBlock > psa::kMaxBlocks) return PSA_ERR_UNSUPPORTED;
  if (static_cast<long long>(B) * H * N * d >= (1LL << 31)) return PSA_ERR_SHAPE;
  if (causal != 0 && causal != 1) return PSA_ERR_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || !aligned16(kbar) ||
      !aligned16(vsum) || (lse && (reinterpret_cast<uintptr_t>(lse) & 3u)) ||
      (status && (reinterpret_cast<uintptr_t>(status) & 3u)) || (reinterpret_cast<uintptr_t>(row_max) & 3u))
    return PSA_ERR_ARG;
  const long long bh = static_cast<long long>(B) * H;
  const int M = N / psa::kBlock;
  if (scratch_bytes(bh, M, d) > kNoAllocScratchBytes) return PSA_ERR_CAPACITY;  // shape too large
  int s = psa::check_device_pointers({q, out});
  if (s != PSA_OK) return s;
  void* base = nullptr;
  s = scratch_for_current_device(&base);
  if (s != PSA_OK) return s;
  char* ws = static_cast<char*>(base);
  const size_t off_fix = 256;
  const size_t off_kb = off_fix + align256(static_cast<size_t>(bh * M) * 4);
  const size_t off_vs = off_kb + align256(static_cast<size_t>(bh * M * d) * 2);
  const size_t off_fix2 = off_vs + align256(static_cast<size_t>(bh * M * d) * 2);
  const size_t off_lse2 = off_fix2 + align256(static_cast<size_t>(bh * M) * 4);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // the status word and the fixup counter must start at zero on every call
  if (psa::launch_zero_header(ws, st) != cudaSuccess) return PSA_ERR_CUDA;
  uint16_t* kb16 = reinterpret_cast<uint16_t*>(ws + off_kb);
  uint16_t* vs16 = reinterpret_cast<uint16_t*>(ws + off_vs);
  if (psa::launch_stats_to_bf16(kbar, vsum, bh * M * d, kb16, vs16, st) != cudaSuccess) return PSA_ERR_CUDA;
  psa::AttnLaunch a;
  a.q = q;
  a.k = k;
  a.v = v;
  a.kbar_bf16 = kb16;
  a.vsum_bf16 = vs16;
  a.row_ptr = row_ptr;
  a.col_idx = col_idx;
  a.col_cap = col_capacity > static_cast<size_t>(LLONG_MAX) ? LLONG_MAX : static_cast<long long>(col_capacity);
  a.row_max = row_max;
  a.stall = 0;
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
  a.fixup_list = reinterpret_cast<int*>(ws + off_fix);
  a.fixup_count2 = reinterpret_cast<int*>(ws) + 2;
  a.sched = reinterpret_cast<int*>(ws) + 3;
  a.fixup_list2 = reinterpret_cast<int*>(ws + off_fix2);
  a.row_lse2 = reinterpret_cast<float*>(ws + off_lse2);
  if (psa::launch_attn(a, st) != cudaSuccess) return PSA_ERR_CUDA;
  if (status && cudaMemcpyAsync(status, ws, sizeof(int), cudaMemcpyDeviceToDevice, st) != cudaSuccess)
    return PSA_ERR_CUDA;
  return PSA_OK;
}

}  // extern "C"
