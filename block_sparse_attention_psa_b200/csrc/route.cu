// route.cu -- a2..a4: block scores and the two routers.
//
// Scores: PISA summary (kodorricoding.tistory.com/108), "How are candidate
// blocks narrowed": one score per (query block, key block) from the block
// representatives, s_IJ = qbar_I . kbar_J / sqrt(d), computed in fp32.
// Top-k: the same section and the usage line (`density`).  Threshold:
// FlashPrefill summary, 2.b "Max-based dynamic thresholding",
// thresh_I = alpha * max_J s_IJ, no sort and no cumulative sum.
//
// A CTA of 256 threads scores R consecutive query blocks of one head against
// every candidate key block (kbar rows are read once per CTA and reused for
// the R rows), keeps the scores in shared memory, and then one warp per row
// selects.  Top-k finds the k-th largest score exactly by a 32-step bitwise
// search over the order-preserving integer image of the fp32 scores (ties
// resolved by ascending J), so it needs no sort; both routers write the
// list in ascending J with warp ballots, and, when asked, each row's largest
// candidate score (the attention step's softmax stabiliser).
#include "internal.h"
#include "sm100.cuh"

namespace psa {
namespace {

__device__ __forceinline__ uint32_t order_key(float s) {
  const uint32_t b = __float_as_uint(s);
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

__device__ __forceinline__ uint32_t lanemask_lt() {
  uint32_t m;
  asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
  return m;
}

// Sum over i < I of min(k0, i + 1): start of row I inside its head for causal
// top-k (k0 >= 1).
__host__ __device__ inline long long causal_prefix(long long I, long long k0) {
  if (I <= k0) return I * (I + 1) / 2;
  return k0 * (k0 + 1) / 2 + (I - k0) * k0;
}

// Scores of rows [I0, I0 + rows) of head bh into ss[r * M + J], J < jmax.
// Thread t owns key J0 + t of each 256-key chunk and accumulates its R dot
// products over the features in order.  The kbar rows reach it through
// shared memory, 16 features of 256 keys at a time: loaded with coalesced
// 16-byte loads (read straight from global memory, every lane of a warp
// would touch a different cache line) into rows padded to 20 floats, so the
// per-thread 16-byte reads are free of bank conflicts.  The next slice is
// fetched into registers while the current one is consumed.
constexpr int kSliceF = 16;            // features per slice
constexpr int kSliceStride = 20;       // padded row, floats
constexpr int kChunkJ = 256;           // keys per chunk (one per thread)

template <int R, int D>
__device__ void score_rows(const float* __restrict__ qbar, const float* __restrict__ kbar, int bh, int M,
                           int I0, int rows, int jmax, float tau, float* sq, float* sk, float* ss) {
  static_assert(D % kSliceF == 0, "slices");
  constexpr int kSlices = D / kSliceF;
  const int tid = threadIdx.x;
  for (int e = tid; e < R * D; e += blockDim.x)
    sq[e] = e < rows * D ? qbar[(static_cast<size_t>(bh) * M + I0) * D + e] : 0.f;
  const float* kb = kbar + static_cast<size_t>(bh) * M * D;
  const float4* sq4 = reinterpret_cast<const float4*>(sq);
  for (int J0 = 0; J0 < jmax; J0 += kChunkJ) {
    // slice loader: float4 e = i * 256 + tid covers key row e / 4, features 4 (e % 4) ..
    float4 pre[4];
    auto fetch = [&](int s) {
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int e = i * 256 + tid, row = e >> 2, c4 = e & 3;
        pre[i] = J0 + row < jmax
                     ? __ldg(reinterpret_cast<const float4*>(kb + static_cast<size_t>(J0 + row) * D + s * kSliceF) + c4)
                     : make_float4(0.f, 0.f, 0.f, 0.f);
      }
    };
    auto stash = [&](float* buf) {
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int e = i * 256 + tid, row = e >> 2, c4 = e & 3;
        *reinterpret_cast<float4*>(buf + row * kSliceStride + 4 * c4) = pre[i];
      }
    };
    float acc[R];
#pragma unroll
    for (int r = 0; r < R; ++r) acc[r] = 0.f;
    fetch(0);
    __syncthreads();  // previous chunk's readers are done with both buffers
    stash(sk);
#pragma unroll 1
    for (int s = 0; s < kSlices; ++s) {
      float* cur = sk + (s & 1) * kChunkJ * kSliceStride;
      if (s + 1 < kSlices) fetch(s + 1);
      __syncthreads();
      const float4* kr = reinterpret_cast<const float4*>(cur + tid * kSliceStride);
#pragma unroll
      for (int c = 0; c < kSliceF / 4; ++c) {
        const float4 kv = kr[c];
#pragma unroll
        for (int r = 0; r < R; ++r) {
          const float4 qv = sq4[r * (D / 4) + s * (kSliceF / 4) + c];
          acc[r] = fmaf(qv.x, kv.x, acc[r]);
          acc[r] = fmaf(qv.y, kv.y, acc[r]);
          acc[r] = fmaf(qv.z, kv.z, acc[r]);
          acc[r] = fmaf(qv.w, kv.w, acc[r]);
        }
      }
      if (s + 1 < kSlices) stash(sk + ((s + 1) & 1) * kChunkJ * kSliceStride);
    }
    const int J = J0 + tid;
    if (J < jmax) {
#pragma unroll
      for (int r = 0; r < R; ++r)
        if (r < rows) ss[r * M + J] = acc[r] * tau + 0.0f;  // +0 folds -0 into +0
    }
  }
  __syncthreads();
}

template <int R, int D>
__global__ void __launch_bounds__(256) route_topk_kernel(const float* __restrict__ qbar,
                                                         const float* __restrict__ kbar, int BH, int M,
                                                         float tau, int k0, int causal, int* __restrict__ row_ptr,
                                                         int* __restrict__ col_idx, long long total,
                                                         int* __restrict__ nnz_out, float* __restrict__ row_max) {
  extern __shared__ float sm[];
  const int bh = blockIdx.y;
  const int I0 = blockIdx.x * R;
  const int rows = min(R, M - I0);
  const int jmax = causal ? min(M, I0 + rows) : M;
  float* sq = sm;
  float* sk = sq + R * D;
  float* ss = sk + 2 * kChunkJ * kSliceStride;
  score_rows<R, D>(qbar, kbar, bh, M, I0, rows, jmax, tau, sq, sk, ss);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  if (warp >= rows) return;
  const int I = I0 + warp;
  const long long row = static_cast<long long>(bh) * M + I;
  const float* s = ss + warp * M;
  const int cand = causal ? I + 1 : M;
  const int kk = max(1, min(k0, cand));
  // causal: the diagonal takes one slot, the rest come from J < I
  const int n = causal ? I : M;
  const int krest = causal ? kk - 1 : kk;
  if (row_max) {
    float m = -INFINITY;
    for (int J = lane; J < cand; J += 32) m = fmaxf(m, s[J]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if (lane == 0) row_max[row] = m;
  }

  uint32_t T = 0;
  if (krest > 0) {
    for (int bit = 31; bit >= 0; --bit) {
      const uint32_t t = T | (1u << bit);
      int cnt = 0;
      for (int J = lane; J < n; J += 32) cnt += order_key(s[J]) >= t;
      cnt = __reduce_add_sync(0xffffffffu, cnt);
      if (cnt >= krest) {
        T = t;
        // exactly krest keys are >= T: they are the selection (every key equal
        // to T is in it, so the tie rule below takes them all)
        if (cnt == krest) break;
      }
    }
  }
  int gt = 0;
  if (krest > 0)
    for (int J = lane; J < n; J += 32) gt += order_key(s[J]) > T;
  gt = __reduce_add_sync(0xffffffffu, gt);
  const int need_eq = krest - gt;

  long long start;
  if (causal) {
    const long long k0c = max(k0, 1);
    start = static_cast<long long>(bh) * causal_prefix(M, k0c) + causal_prefix(I, k0c);
  } else {
    start = row * kk;
  }
  int pos = 0, eq_seen = 0;
  const uint32_t lt = lanemask_lt();
  for (int J0 = 0; J0 < cand; J0 += 32) {
    const int J = J0 + lane;
    bool gtf = false, eqf = false;
    if (J < n && krest > 0) {
      const uint32_t key = order_key(s[J]);
      gtf = key > T;
      eqf = key == T;
    }
    const uint32_t eqm = __ballot_sync(0xffffffffu, eqf);
    const bool in = gtf || (eqf && eq_seen + __popc(eqm & lt) < need_eq) || (causal && J == I);
    eq_seen += __popc(eqm);
    const uint32_t m = __ballot_sync(0xffffffffu, in);
    if (in) col_idx[start + pos + __popc(m & lt)] = J;
    pos += __popc(m);
  }
  if (lane == 0) {
    row_ptr[row] = static_cast<int>(start);
    if (row == static_cast<long long>(BH) * M - 1) {
      row_ptr[row + 1] = static_cast<int>(total);
      *nnz_out = static_cast<int>(total);
    }
  }
}

template <int R, int D>
__global__ void __launch_bounds__(256) route_thresh_kernel(const float* __restrict__ qbar,
                                                           const float* __restrict__ kbar, int M,
                                                           float tau, float a_mul, float a_add, int causal,
                                                           int keep_first,
                                                           int* __restrict__ row_count,
                                                           uint32_t* __restrict__ row_bits,
                                                           float* __restrict__ row_max) {
  extern __shared__ float sm[];
  const int bh = blockIdx.y;
  const int I0 = blockIdx.x * R;
  const int rows = min(R, M - I0);
  const int jmax = causal ? min(M, I0 + rows) : M;
  float* sq = sm;
  float* sk = sq + R * D;
  float* ss = sk + 2 * kChunkJ * kSliceStride;
  score_rows<R, D>(qbar, kbar, bh, M, I0, rows, jmax, tau, sq, sk, ss);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  if (warp >= rows) return;
  const int I = I0 + warp;
  const long long row = static_cast<long long>(bh) * M + I;
  const float* s = ss + warp * M;
  const int cand = causal ? I + 1 : M;
  float m = -INFINITY;
  for (int J = lane; J < cand; J += 32) m = fmaxf(m, s[J]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  // logit rule: alpha * max (a_mul = alpha, a_add = 0, the product exactly as
  // alpha * m); probability rule: max + ln(alpha) (a_mul = 1, a_add = ln alpha)
  const float thr = fmaf(a_mul, m, a_add);
  if (row_max && lane == 0) row_max[row] = m;
  const int nw = (M + 31) / 32;
  uint32_t* bits = row_bits + row * nw;
  int cnt = 0;
  for (int J0 = 0; J0 < cand; J0 += 32) {
    const int J = J0 + lane;
    const bool in = J < cand && (s[J] >= thr || J == I || (keep_first && J == 0));
    const uint32_t w = __ballot_sync(0xffffffffu, in);
    if (lane == 0) bits[J0 / 32] = w;
    cnt += __popc(w);
  }
  if (lane == 0) row_count[row] = cnt;
}

// Exclusive scan of the row counts into row_ptr (one CTA of 1024 threads),
// clamped to the capacity so that a too-small col_idx still yields a valid,
// truncated list; *nnz_out gets the exact total (saturated at INT_MAX).
__global__ void __launch_bounds__(1024) scan_rows_kernel(const int* __restrict__ count, long long n,
                                                         long long capacity, int* __restrict__ row_ptr,
                                                         int* __restrict__ nnz_out) {
  constexpr int kItems = 8;
  __shared__ long long warp_tot[32];
  __shared__ long long carry_s;
  const int tid = threadIdx.x, lane = tid % 32, warp = tid / 32;
  if (tid == 0) carry_s = 0;
  __syncthreads();
  for (long long base = 0; base < n; base += 1024LL * kItems) {
    long long v[kItems];
    long long tsum = 0;
#pragma unroll
    for (int i = 0; i < kItems; ++i) {
      const long long idx = base + static_cast<long long>(tid) * kItems + i;
      v[i] = idx < n ? count[idx] : 0;
      tsum += v[i];
    }
    long long incl = tsum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const long long y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    if (lane == 31) warp_tot[warp] = incl;
    __syncthreads();
    if (warp == 0) {
      long long w = warp_tot[lane];
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const long long y = __shfl_up_sync(0xffffffffu, w, o);
        if (lane >= o) w += y;
      }
      warp_tot[lane] = w;  // inclusive over warps
    }
    __syncthreads();
    const long long carry = carry_s;
    long long run = carry + (warp ? warp_tot[warp - 1] : 0) + incl - tsum;
#pragma unroll
    for (int i = 0; i < kItems; ++i) {
      const long long idx = base + static_cast<long long>(tid) * kItems + i;
      if (idx < n) row_ptr[idx] = static_cast<int>(run < capacity ? run : capacity);
      run += v[i];
    }
    __syncthreads();
    if (tid == 0) carry_s = carry + warp_tot[31];
    __syncthreads();
  }
  if (tid == 0) {
    const long long tot = carry_s;
    row_ptr[n] = static_cast<int>(tot < capacity ? tot : capacity);
    *nnz_out = static_cast<int>(tot < 0x7fffffffLL ? tot : 0x7fffffffLL);
  }
}

// One warp per row: expand the row's bit mask into ascending J entries.
__global__ void __launch_bounds__(256) compact_rows_kernel(const uint32_t* __restrict__ row_bits,
                                                           const int* __restrict__ row_ptr, long long nrows,
                                                           int M, int causal, int* __restrict__ col_idx) {
  const int lane = threadIdx.x % 32;
  const long long row = blockIdx.x * 8LL + threadIdx.x / 32;
  if (row >= nrows) return;
  const int I = static_cast<int>(row % M);
  const int cand = causal ? I + 1 : M;
  const int nw = (M + 31) / 32;
  const uint32_t* bits = row_bits + row * nw;
  const int start = row_ptr[row], end = row_ptr[row + 1];
  const uint32_t lt = lanemask_lt();
  int pos = start;
  for (int J0 = 0; J0 < cand; J0 += 32) {
    const uint32_t w = bits[J0 / 32];
    const int J = J0 + lane;
    const bool in = J < cand && ((w >> lane) & 1u);
    const uint32_t m = __ballot_sync(0xffffffffu, in);
    const int at = pos + __popc(m & lt);
    if (in && at < end) col_idx[at] = J;
    pos += __popc(m);
  }
}

// shared memory of a router CTA: R query rows, the two kbar slices, R score rows
size_t route_smem(int R, int M, int d) {
  return (static_cast<size_t>(R) * (M + d) + 2 * kChunkJ * kSliceStride) * sizeof(float);
}

int rows_per_cta(int M, int d) {
  for (int R = 8; R > 1; R >>= 1)
    if (route_smem(R, M, d) <= 200 * 1024) return R;
  return 1;
}

template <typename K>
cudaError_t set_smem(K kernel, size_t bytes) {
  return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(bytes));
}

}  // namespace

cudaError_t launch_route_topk(const float* qbar, const float* kbar, int BH, int M, int d, int k0, int causal,
                              int* row_ptr, int* col_idx, long long total, int* nnz_out, float* row_max,
                              cudaStream_t st) {
  const int R = rows_per_cta(M, d);
  const size_t smem = route_smem(R, M, d);
  const dim3 grid((M + R - 1) / R, BH);
  const float tau = 1.0f / sqrtf(static_cast<float>(d));
  cudaError_t e;
#define PSA_TOPK(RR)                                                                                   \
  case RR:                                                                                             \
    if (d == 128) {                                                                                    \
      if ((e = set_smem(route_topk_kernel<RR, 128>, smem)) != cudaSuccess) return e;                   \
      route_topk_kernel<RR, 128><<<grid, 256, smem, st>>>(qbar, kbar, BH, M, tau, k0, causal, row_ptr, \
                                                           col_idx, total, nnz_out, row_max);          \
    } else {                                                                                           \
      if ((e = set_smem(route_topk_kernel<RR, 64>, smem)) != cudaSuccess) return e;                    \
      route_topk_kernel<RR, 64><<<grid, 256, smem, st>>>(qbar, kbar, BH, M, tau, k0, causal, row_ptr,  \
                                                          col_idx, total, nnz_out, row_max);           \
    }                                                                                                  \
    break;
  if (d != 64 && d != 128) return cudaErrorInvalidValue;
  switch (R) {
    PSA_TOPK(8)
    PSA_TOPK(4)
    PSA_TOPK(2)
    PSA_TOPK(1)
    default:
      return cudaErrorInvalidValue;
  }
#undef PSA_TOPK
  return cudaGetLastError();
}

cudaError_t launch_route_thresh(const float* qbar, const float* kbar, int BH, int M, int d, float a_mul,
                                float a_add, int causal, int keep_first, int* row_ptr, int* col_idx, long long capacity,
                                int* nnz_out, int* row_count, uint32_t* row_bits, float* row_max,
                                cudaStream_t st) {
  const int R = rows_per_cta(M, d);
  const size_t smem = route_smem(R, M, d);
  const dim3 grid((M + R - 1) / R, BH);
  const float tau = 1.0f / sqrtf(static_cast<float>(d));
  cudaError_t e;
#define PSA_THRESH(RR)                                                                                 \
  case RR:                                                                                             \
    if (d == 128) {                                                                                    \
      if ((e = set_smem(route_thresh_kernel<RR, 128>, smem)) != cudaSuccess) return e;                 \
      route_thresh_kernel<RR, 128><<<grid, 256, smem, st>>>(qbar, kbar, M, tau, a_mul, a_add, causal,  \
                                                             keep_first, row_count, row_bits, row_max); \
    } else {                                                                                           \
      if ((e = set_smem(route_thresh_kernel<RR, 64>, smem)) != cudaSuccess) return e;                  \
      route_thresh_kernel<RR, 64><<<grid, 256, smem, st>>>(qbar, kbar, M, tau, a_mul, a_add, causal,   \
                                                            keep_first, row_count, row_bits, row_max);  \
    }                                                                                                  \
    break;
  if (d != 64 && d != 128) return cudaErrorInvalidValue;
  switch (R) {
    PSA_THRESH(8)
    PSA_THRESH(4)
    PSA_THRESH(2)
    PSA_THRESH(1)
    default:
      return cudaErrorInvalidValue;
  }
#undef PSA_THRESH
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  const long long nrows = static_cast<long long>(BH) * M;
  scan_rows_kernel<<<1, 1024, 0, st>>>(row_count, nrows, capacity, row_ptr, nnz_out);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  compact_rows_kernel<<<static_cast<unsigned>((nrows + 7) / 8), 256, 0, st>>>(row_bits, row_ptr, nrows, M,
                                                                               causal, col_idx);
  return cudaGetLastError();
}

}  // namespace psa
