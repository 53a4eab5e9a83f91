// route.cu -- a3/a4: the two routers, on the block scores of score.cu.
//
// Scores: PISA summary (kodorricoding.tistory.com/108), "How are candidate
// blocks narrowed": one score per (query block, key block) from the block
// representatives, s_IJ = qbar_I . kbar_J / sqrt(d), computed at fp32
// accuracy on the tensor cores (score.cu).  Top-k: the same section and the
// usage line (`density`).  Threshold: FlashPrefill summary, 2.b "Max-based
// dynamic thresholding", thresh_I = alpha * max_J s_IJ, no sort and no
// cumulative sum.
//
// A CTA of 256 threads copies the score rows of R consecutive query blocks
// of one head into shared memory, and then one warp per row selects.  Top-k
// finds the k-th largest score exactly by a radix select over the four 8-bit
// digits of the order-preserving integer image of the fp32 scores (one
// 256-bucket warp histogram per digit; ties resolved by ascending J), so it
// needs no sort; both routers write the list in ascending J with warp
// ballots, and, when asked, each row's largest candidate score (the
// attention step's softmax stabiliser).  Heads are routed in batches whose
// score matrices fit the workspace.
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

// Inverse of order_key.
__device__ __forceinline__ float key_float(uint32_t k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7fffffffu) : ~k);
}

// The bucket of a 256-bucket histogram that holds the need-th largest key
// (counting from the top bucket down): its digit, and how many keys the
// buckets above it hold.  Lane l scans buckets 255 - 8l down to 248 - 8l.
__device__ __forceinline__ void pick_bucket(const int* hist, int lane, int need, int& digit, int& above) {
  int c[8], sum = 0;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    c[i] = hist[255 - 8 * lane - i];
    sum += c[i];
  }
  int incl = sum;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  const int excl = incl - sum;
  const bool mine = excl < need && incl >= need;
  const int src = __ffs(__ballot_sync(0xffffffffu, mine)) - 1;
  int dg = 0, ab = 0;
  if (mine) {
    int run = excl;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      if (run + c[i] >= need) {
        dg = 255 - 8 * lane - i;
        ab = run;
        break;
      }
      run += c[i];
    }
  }
  digit = __shfl_sync(0xffffffffu, dg, src);
  above = __shfl_sync(0xffffffffu, ab, src);
}

// Sum over i < I of min(k0, i + 1): start of row I inside its head for causal
// top-k (k0 >= 1).
__host__ __device__ inline long long causal_prefix(long long I, long long k0) {
  if (I <= k0) return I * (I + 1) / 2;
  return k0 * (k0 + 1) / 2 + (I - k0) * k0;
}

// Score row I0 + warp of local head hl, candidates J < jmax, into
// ss[warp * Mp + J]: each warp copies the row it then selects from (row
// stride Mp, a multiple of 128, so the copy moves coalesced float4s).  With
// Keys the row is stored as the order keys of the scores.
template <bool Keys>
__device__ __forceinline__ void load_row(const float* __restrict__ scores, int M, int Mp, int hl, int I, int jmax,
                                         float* ss_row) {
  const int lane = threadIdx.x % 32;
  const int q4 = (jmax + 3) / 4;
  const float4* src = reinterpret_cast<const float4*>(scores + (static_cast<size_t>(hl) * M + I) * Mp);
  float4* dst = reinterpret_cast<float4*>(ss_row);
  auto put = [&](int c, float4 x) {
    if (Keys)
      x = make_float4(__uint_as_float(order_key(x.x)), __uint_as_float(order_key(x.y)),
                      __uint_as_float(order_key(x.z)), __uint_as_float(order_key(x.w)));
    dst[c] = x;
  };
  int c = lane;
  for (; c + 96 < q4; c += 128) {
    const float4 x0 = __ldg(src + c), x1 = __ldg(src + c + 32), x2 = __ldg(src + c + 64), x3 = __ldg(src + c + 96);
    put(c, x0);
    put(c + 32, x1);
    put(c + 64, x2);
    put(c + 96, x3);
  }
  for (; c < q4; c += 32) put(c, __ldg(src + c));
  __syncwarp();
}

template <int R>
__global__ void __launch_bounds__(256, 4) route_topk_kernel(const float* __restrict__ scores, int Mp, int bh0,
                                                         int BH, int M, int k0, int causal,
                                                         int* __restrict__ row_ptr, int* __restrict__ col_idx,
                                                         long long total, int* __restrict__ nnz_out,
                                                         float* __restrict__ row_max) {
  extern __shared__ float ss[];  // [R][Mp] score rows, then [R][256] histograms
  grid_dep_launch();
  grid_dep_wait();
  const int hl = blockIdx.y, bh = bh0 + hl;
  const int I0 = blockIdx.x * R;
  const int rows = min(R, M - I0);
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  if (warp >= rows) return;
  const int I = I0 + warp;
  const int cand = causal ? I + 1 : M;
  load_row<true>(scores, M, Mp, hl, I, cand, ss + warp * Mp);
  const long long row = static_cast<long long>(bh) * M + I;
  const uint32_t* sk = reinterpret_cast<const uint32_t*>(ss + warp * Mp);  // order keys
  int* hist = reinterpret_cast<int*>(ss + R * Mp) + warp * 256;
  const int kk = max(1, min(k0, cand));
  // causal: the diagonal takes one slot, the rest come from J < I
  const int n = causal ? I : M;
  const int krest = causal ? kk - 1 : kk;
  // T = the krest-th largest order key among J < n, exactly: a radix
  // select over four 8-bit digits, high to low.  Each pass histograms the
  // digit of the keys that share the prefix fixed so far, then finds the
  // bucket that holds the krest-th key by a scan from the top bucket down.  The keys in
  // the buckets above the chosen ones are exactly the keys above T, so the
  // rank left at the end is the number of keys equal to T to take.  The
  // first pass also takes the row maximum (the diagonal J = I = n is the
  // one candidate outside J < n, when causal).
  uint32_t T = 0;
  int need_eq = 0;
  uint32_t mk = causal ? sk[I] : 0u;
  if (krest > 0) {
    uint32_t prefix = 0;
    int need = krest;  // rank of T among the keys that share `prefix`
#pragma unroll 1
    for (int shift = 24; shift >= 0; shift -= 8) {
      for (int b = lane; b < 256; b += 32) hist[b] = 0;
      __syncwarp();
      const uint32_t hi = shift == 24 ? 0u : 0xffffffffu << (shift + 8);
      if (shift == 24) {
        // first digit (sign and leading exponent bits): every key counts
        for (int J0 = 0; J0 < n; J0 += 32) {
          const int J = J0 + lane;
          int digit = 256;  // no key
          if (J < n) {
            const uint32_t key = sk[J];
            mk = max(mk, key);
            digit = static_cast<int>(key >> 24);
          }
          if (digit < 256) atomicAdd(&hist[digit], 1);
        }
      } else {
        // later digits: only the keys that share the prefix count
        for (int J = lane; J < n; J += 32) {
          const uint32_t key = sk[J];
          if ((key & hi) == prefix) atomicAdd(&hist[(key >> shift) & 255u], 1);
        }
      }
      __syncwarp();
      int digit, above;
      pick_bucket(hist, lane, need, digit, above);
      prefix |= static_cast<uint32_t>(digit) << shift;
      need -= above;
      __syncwarp();
    }
    T = prefix;
    need_eq = need;
  } else if (row_max) {
    for (int J = lane; J < n; J += 32) mk = max(mk, sk[J]);
  }
  if (row_max) {
    mk = __reduce_max_sync(0xffffffffu, mk);
    if (lane == 0) row_max[row] = key_float(mk);
  }

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
      const uint32_t key = sk[J];
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

template <int R>
__global__ void __launch_bounds__(256, 4) route_thresh_kernel(const float* __restrict__ scores, int Mp, int bh0,
                                                           int M, float a_mul, float a_add, int causal,
                                                           int keep_first,
                                                           int* __restrict__ row_count,
                                                           uint32_t* __restrict__ row_bits,
                                                           float* __restrict__ row_max) {
  extern __shared__ float ss[];  // [R][Mp] score rows
  grid_dep_launch();
  grid_dep_wait();
  const int hl = blockIdx.y, bh = bh0 + hl;
  const int I0 = blockIdx.x * R;
  const int rows = min(R, M - I0);
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  if (warp >= rows) return;
  const int I = I0 + warp;
  const int cand = causal ? I + 1 : M;
  load_row<false>(scores, M, Mp, hl, I, cand, ss + warp * Mp);
  const long long row = static_cast<long long>(bh) * M + I;
  const float* s = ss + warp * Mp;
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
  grid_dep_launch();
  grid_dep_wait();
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
  grid_dep_launch();
  grid_dep_wait();
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

// shared memory of a router CTA: R score rows of stride Mp (+ R 256-bucket
// histograms for top-k)
size_t route_smem(int R, int Mp) { return static_cast<size_t>(R) * (Mp + 256) * sizeof(float); }

int rows_per_cta(int Mp) {
  for (int R = 8; R > 1; R >>= 1)
    if (route_smem(R, Mp) <= 200 * 1024) return R;
  return 1;
}

template <typename K>
cudaError_t set_smem(K kernel, size_t bytes) {
  return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(bytes));
}

// Split both operands and prepare the score tiles of every head.
cudaError_t prepare_scores(const float* qbar, const float* kbar, int BH, int M, int d, const RouteScratch& w,
                           ScorePlan& plan, cudaStream_t st) {
  if (d != 64 && d != 128) return cudaErrorInvalidValue;
  const long long n = static_cast<long long>(BH) * M * d;
  const cudaError_t e = launch_split3(qbar, kbar, n, w.q_split, w.k_split, st);
  if (e != cudaSuccess) return e;
  return plan.init(w.q_split, w.k_split, BH, M, d);
}

}  // namespace

cudaError_t launch_route_topk(const float* qbar, const float* kbar, int BH, int M, int d, int k0, int causal,
                              int* row_ptr, int* col_idx, long long total, int* nnz_out, float* row_max,
                              const RouteScratch& w, cudaStream_t st) {
  ScorePlan plan;
  cudaError_t e = prepare_scores(qbar, kbar, BH, M, d, w, plan, st);
  if (e != cudaSuccess) return e;
  const int Mp = plan.Mp;
  const int R = rows_per_cta(Mp);
  const size_t smem = route_smem(R, Mp);
  for (int h0 = 0; h0 < BH; h0 += w.heads_per_batch) {
    const int nh = BH - h0 < w.heads_per_batch ? BH - h0 : w.heads_per_batch;
    if ((e = plan.run(h0, nh, causal, w.scores, w.status, st)) != cudaSuccess) return e;
    const dim3 grid((M + R - 1) / R, nh);
#define PSA_TOPK(RR)                                                                                         \
  case RR:                                                                                                   \
    if ((e = set_smem(route_topk_kernel<RR>, smem)) != cudaSuccess) return e;                                \
    e = launch_chained(route_topk_kernel<RR>, grid, dim3(256), smem, st, w.scores, Mp, h0, BH, M, k0, causal, \
                       row_ptr, col_idx, total, nnz_out, row_max);                                           \
    break;
    switch (R) {
      PSA_TOPK(8)
      PSA_TOPK(4)
      PSA_TOPK(2)
      PSA_TOPK(1)
      default:
        return cudaErrorInvalidValue;
    }
#undef PSA_TOPK
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

cudaError_t launch_route_thresh(const float* qbar, const float* kbar, int BH, int M, int d, float a_mul,
                                float a_add, int causal, int keep_first, int* row_ptr, int* col_idx, long long capacity,
                                int* nnz_out, int* row_count, uint32_t* row_bits, float* row_max,
                                const RouteScratch& w, cudaStream_t st) {
  ScorePlan plan;
  cudaError_t e = prepare_scores(qbar, kbar, BH, M, d, w, plan, st);
  if (e != cudaSuccess) return e;
  const int Mp = plan.Mp;
  const int R = rows_per_cta(Mp);
  const size_t smem = route_smem(R, Mp);
  for (int h0 = 0; h0 < BH; h0 += w.heads_per_batch) {
    const int nh = BH - h0 < w.heads_per_batch ? BH - h0 : w.heads_per_batch;
    if ((e = plan.run(h0, nh, causal, w.scores, w.status, st)) != cudaSuccess) return e;
    const dim3 grid((M + R - 1) / R, nh);
#define PSA_THRESH(RR)                                                                                       \
  case RR:                                                                                                   \
    if ((e = set_smem(route_thresh_kernel<RR>, smem)) != cudaSuccess) return e;                              \
    e = launch_chained(route_thresh_kernel<RR>, grid, dim3(256), smem, st, w.scores, Mp, h0, M, a_mul, a_add, \
                       causal, keep_first, row_count, row_bits, row_max);                                    \
    break;
    switch (R) {
      PSA_THRESH(8)
      PSA_THRESH(4)
      PSA_THRESH(2)
      PSA_THRESH(1)
      default:
        return cudaErrorInvalidValue;
    }
#undef PSA_THRESH
    if (e != cudaSuccess) return e;
  }
  const long long nrows = static_cast<long long>(BH) * M;
  if ((e = launch_chained(scan_rows_kernel, dim3(1), dim3(1024), 0, st, static_cast<const int*>(row_count), nrows,
                         capacity, row_ptr, nnz_out)) != cudaSuccess)
    return e;
  return launch_chained(compact_rows_kernel, dim3(static_cast<unsigned>((nrows + 7) / 8)), dim3(256), 0, st,
                        static_cast<const uint32_t*>(row_bits), static_cast<const int*>(row_ptr), nrows, M, causal,
                        col_idx);
}

}  // namespace psa
