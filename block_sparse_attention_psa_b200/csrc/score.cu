// score.cu -- a2: the block-score matrix s_IJ = qbar_I . kbar_J / sqrt(d) of
// every head on the tensor cores, at fp32 accuracy.
//
// Scores: PISA summary (kodorricoding.tistory.com/108), "How are candidate
// blocks narrowed": one score per (query block, key block) pair from the
// block representatives.  For one head this is the dense product
// Qbar . Kbar^T (M x M, inner dimension d), so it runs as tcgen05 MMAs.
//
// Precision.  The routers must reproduce an fp64 ranking up to a 1e-4
// relative band, which bf16 or tf32 products alone do not reach.  Each fp32
// operand x is therefore split into three bf16 parts x = x0 + x1 + x2 + r
// (x0 = bf16(x), x1 = bf16(x - x0), x2 = bf16(x - x0 - x1), |r| <= 2^-24 |x|
// or so; every difference is exact in fp32), and the product is taken as
//   q.k ~= q2.k0 + q1.k1 + q0.k2 + q1.k0 + q0.k1 + q0.k0,
// dropping only the terms of relative size 2^-24 and below.  The six
// products are bf16 x bf16 MMAs accumulated in fp32 in TMEM, smallest terms
// first; the result carries the rounding of an fp32 dot product.
//
// Layout.  The split operands are bf16 [3][B*H*M][d] (part, row, feature),
// read by TMA in 128-row x 64-feature boxes with the 128-byte swizzle.  One
// CTA computes one 128 x 128 tile (query blocks I0.., key blocks J0..) of
// one head: all six part boxes of both operands land in shared memory at
// once (192 KB at d = 128, 96 KB at d = 64), one thread issues the 6 * d/16
// MMAs (M = 128, N = 128, K = 16) into 128 TMEM columns, and the four warps
// read the tile back (one query row per thread) and store it, scaled by
// 1/sqrt(d), into the score matrix [heads][M][Mp] (Mp = M rounded up to 128,
// so every tile column exists).  Causal tiles wholly above the diagonal are
// skipped.
#include <cuda_bf16.h>

#include "internal.h"
#include "sm100.cuh"

namespace psa {
namespace {

constexpr int kTile = 128;          // query rows and key columns of a tile
constexpr int kBoxBytes = kTile * 64 * 2;  // one 128-row x 64-feature bf16 box

template <int D>
struct ScoreCfg {
  static constexpr int kChunks = D / 64;                   // 64-feature boxes per row
  static constexpr int kOpBytes = 3 * kChunks * kBoxBytes; // one operand, all three parts
  static constexpr int kSmem = 2 * kOpBytes + 1024 + 64;   // + 1 KB alignment slack + barriers
  static constexpr uint32_t kIdesc = idesc_bf16_f32(128, 128, 0, 0);
};

// Three-way bf16 split of n fp32 values (n % 4 == 0): out[p * n + i] is part p of x[i].
__global__ void __launch_bounds__(256) split3_kernel(const float4* __restrict__ x, long long n4,
                                                     uint2* __restrict__ out) {
  const long long n = n4 * 4;
  for (long long i = blockIdx.x * 256LL + threadIdx.x; i < n4; i += static_cast<long long>(gridDim.x) * 256) {
    const float4 v = x[i];
    const float xs[4] = {v.x, v.y, v.z, v.w};
    uint16_t p[3][4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      float r = xs[j];
#pragma unroll
      for (int s = 0; s < 3; ++s) {
        const __nv_bfloat16 b = __float2bfloat16_rn(r);
        p[s][j] = __bfloat16_as_ushort(b);
        r = r - __bfloat162float(b);  // exact
      }
    }
#pragma unroll
    for (int s = 0; s < 3; ++s)
      out[(s * n) / 4 + i] = make_uint2(p[s][0] | (static_cast<uint32_t>(p[s][1]) << 16),
                                        p[s][2] | (static_cast<uint32_t>(p[s][3]) << 16));
  }
}

template <int D>
__global__ void __launch_bounds__(128) score_tc_kernel(const __grid_constant__ CUtensorMap tmQ,
                                                       const __grid_constant__ CUtensorMap tmK, int M, int Mp,
                                                       int bh0, int causal, float tau,
                                                       float* __restrict__ scores, int* status) {
  using C = ScoreCfg<D>;
  const int tj = blockIdx.x, ti = blockIdx.y, hl = blockIdx.z;
  if (causal && tj > ti) return;  // every J of the tile is above every I
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;                 // query parts  [3][kChunks][128 x 64]
  uint8_t* sB = smem + C::kOpBytes;   // key parts    [3][kChunks][128 x 64]
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + 2 * C::kOpBytes);
  uint64_t* load_bar = bars;
  uint64_t* mma_bar = bars + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  if (threadIdx.x == 0) {
    mbar_init(load_bar, 1);
    mbar_init(mma_bar, 1);
    *abort_flag = 0;
    fence_barrier_init();
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, kTile);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tmem_slot;

  const int I0 = ti * kTile, J0 = tj * kTile;
  const int rowQ = (bh0 + hl) * M + I0, rowK = (bh0 + hl) * M + J0;
  bool ok = true;
  if (threadIdx.x == 0) {
    mbar_arrive_expect_tx(load_bar, 2 * C::kOpBytes);
#pragma unroll
    for (int p = 0; p < 3; ++p)
#pragma unroll
      for (int c = 0; c < C::kChunks; ++c) {
        const int box = p * C::kChunks + c;
        tma_load_3d(&tmQ, sA + box * kBoxBytes, load_bar, 64 * c, rowQ, p);
        tma_load_3d(&tmK, sB + box * kBoxBytes, load_bar, 64 * c, rowK, p);
      }
    ok = mbar_wait(load_bar, 0, abort_flag, status);
    if (ok) {
      tc_fence_after();
      const uint64_t dA0 = sdesc_sw128(smem_u32(sA), 16, 1024);
      const uint64_t dB0 = sdesc_sw128(smem_u32(sB), 16, 1024);
      constexpr uint64_t kPart = (C::kChunks * kBoxBytes) >> 4;  // one part, 16-byte units
      // (query part, key part), smallest products first
      constexpr int kPairs[6][2] = {{2, 0}, {1, 1}, {0, 2}, {1, 0}, {0, 1}, {0, 0}};
#pragma unroll
      for (int pr = 0; pr < 6; ++pr) {
        const uint64_t a = dA0 + kPairs[pr][0] * kPart, b = dB0 + kPairs[pr][1] * kPart;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint64_t off = (kk >> 2) * (kBoxBytes >> 4) + (kk & 3) * 2;
          tc_mma_bf16(tbase, a + off, b + off, C::kIdesc, (pr == 0 && kk == 0) ? 0u : 1u);
        }
      }
      tc_commit(mma_bar);
    } else {
      // a load that never landed: wait a bounded time for it before the CTA exits
      const long long t0 = clock64();
      while (!mbar_try_wait(load_bar, 0) && clock64() - t0 < kWaitCycles) {
      }
    }
  }
  __syncwarp();
  ok = mbar_wait(mma_bar, 0, abort_flag, status);
  if (ok) {
    tc_fence_after();
    const int r = warp * 32 + lane;  // TMEM lane = query row of the tile
    const int I = I0 + r;
    float* dst = scores + (static_cast<size_t>(hl) * M + I) * Mp + J0;
#pragma unroll 1
    for (int c = 0; c < kTile / 32; ++c) {
      float v[32];
      tmem_ld32(tbase + (static_cast<uint32_t>(warp * 32) << 16) + 32 * c, v);
      tc_wait_ld();
      if (I < M) {
#pragma unroll
        for (int j = 0; j < 32; j += 4)
          *reinterpret_cast<float4*>(dst + 32 * c + j) =
              make_float4(v[j] * tau + 0.0f, v[j + 1] * tau + 0.0f, v[j + 2] * tau + 0.0f, v[j + 3] * tau + 0.0f);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tbase, kTile);
  }
}

template <int D>
cudaError_t launch_score_tiles(const CUtensorMap& mq, const CUtensorMap& mk, int M, int Mp, int bh0, int nh,
                               int causal, float tau, float* scores, int* status, cudaStream_t st) {
  using C = ScoreCfg<D>;
  cudaError_t e = cudaFuncSetAttribute(score_tc_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmem);
  if (e != cudaSuccess) return e;
  const int nt = (M + kTile - 1) / kTile;
  score_tc_kernel<D><<<dim3(nt, nt, nh), 128, C::kSmem, st>>>(mq, mk, M, Mp, bh0, causal, tau, scores, status);
  return cudaGetLastError();
}

}  // namespace

int score_stride(int M) { return (M + kTile - 1) / kTile * kTile; }

cudaError_t launch_split3(const float* x, long long n, uint16_t* out, cudaStream_t st) {
  const long long n4 = n / 4;
  if (n4 == 0) return cudaSuccess;
  const long long want = (n4 + 255) / 256;
  const int grid = static_cast<int>(want < 148LL * 16 ? want : 148LL * 16);
  split3_kernel<<<grid, 256, 0, st>>>(reinterpret_cast<const float4*>(x), n4, reinterpret_cast<uint2*>(out));
  return cudaGetLastError();
}

cudaError_t ScorePlan::init(const uint16_t* qs, const uint16_t* ks, int BH_, int M_, int d_) {
  BH = BH_;
  M = M_;
  d = d_;
  Mp = score_stride(M);
  const uint64_t rows = static_cast<uint64_t>(BH) * M;
  if (encode_tensor_map_3d_bf16(&mq, qs, d, rows, 3, 64, kTile) != CUDA_SUCCESS) return cudaErrorInvalidValue;
  if (encode_tensor_map_3d_bf16(&mk, ks, d, rows, 3, 64, kTile) != CUDA_SUCCESS) return cudaErrorInvalidValue;
  return cudaSuccess;
}

cudaError_t ScorePlan::run(int bh0, int nh, int causal, float* scores, int* status, cudaStream_t st) const {
  const float tau = 1.0f / sqrtf(static_cast<float>(d));
  if (d == 128) return launch_score_tiles<128>(mq, mk, M, Mp, bh0, nh, causal, tau, scores, status, st);
  if (d == 64) return launch_score_tiles<64>(mq, mk, M, Mp, bh0, nh, causal, tau, scores, status, st);
  return cudaErrorInvalidValue;
}

}  // namespace psa
