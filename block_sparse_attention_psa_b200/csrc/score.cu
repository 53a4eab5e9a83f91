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
// one head, 64 features at a time: the six part boxes of the chunk (96 KB)
// land in shared memory, one thread issues the 6 x 4 MMAs (M = 128, N = 128,
// K = 16) of the chunk into 128 TMEM columns, and the buffer is refilled once
// they have read it.  Two CTAs fit on an SM, so one CTA's loads overlap the
// other's MMAs and stores.  The four warps then read the tile back (one query
// row per thread), stage it in the freed buffer, and store it, scaled by
// 1/sqrt(d), row by row with coalesced 512-byte writes into the score matrix
// [heads][M][Mp] (Mp = M rounded up to 128, so every tile column exists).
// Causal tiles wholly above the diagonal are skipped.
#include <cuda_bf16.h>

#include "internal.h"
#include "sm100.cuh"

namespace psa {
namespace {

constexpr int kTile = 128;          // query rows and key columns of a tile
constexpr int kBoxBytes = kTile * 64 * 2;  // one 128-row x 64-feature bf16 box

constexpr int kChunkBytes = 6 * kBoxBytes;  // three query + three key part boxes of one chunk
constexpr int kStageStride = kTile + 4;     // staged tile row, floats (16-byte rows, no bank conflicts)
constexpr int kScoreSmem = kChunkBytes + 1024 + 64;  // + alignment slack + barriers
static_assert(kTile * kStageStride * 4 <= kChunkBytes, "the staged tile fits the operand buffer");
constexpr uint32_t kScoreIdesc = idesc_bf16_f32(128, 128, 0, 0);

// Three-way bf16 split of two arrays of n fp32 values each (n % 4 == 0):
// out_t[p * n + i] is part p of x_t[i].
__global__ void __launch_bounds__(256) split3_kernel(const float4* __restrict__ x0, const float4* __restrict__ x1,
                                                     long long n4, uint2* __restrict__ out0,
                                                     uint2* __restrict__ out1) {
  grid_dep_launch();
  grid_dep_wait();
  for (long long t = blockIdx.x * 256LL + threadIdx.x; t < 2 * n4; t += static_cast<long long>(gridDim.x) * 256) {
    const bool second = t >= n4;
    const long long i = second ? t - n4 : t;
    const float4 v = (second ? x1 : x0)[i];
    uint2* out = second ? out1 : out0;
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
      out[s * n4 + i] = make_uint2(p[s][0] | (static_cast<uint32_t>(p[s][1]) << 16),
                                   p[s][2] | (static_cast<uint32_t>(p[s][3]) << 16));
  }
}

template <int D>
__global__ void __launch_bounds__(128) score_tc_kernel(const __grid_constant__ CUtensorMap tmQ,
                                                       const __grid_constant__ CUtensorMap tmK, int M, int Mp,
                                                       int bh0, int causal, float tau,
                                                       float* __restrict__ scores, int* status) {
  constexpr int kChunks = D / 64;
  const int tj = blockIdx.x, ti = blockIdx.y, hl = blockIdx.z;
  if (causal && tj > ti) return;  // every J of the tile is above every I (an exit counts as the trigger)
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;                  // query parts of one chunk [3][128 x 64]
  uint8_t* sB = smem + 3 * kBoxBytes;  // key parts of one chunk   [3][128 x 64]
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kChunkBytes);
  uint64_t* load_bar = bars;      // chunk c landed: phase c (issuing thread only)
  uint64_t* mma_bar = bars + 1;   // chunk c's MMAs done, buffer free: phase c (issuing thread only)
  uint64_t* done_bar = bars + 2;  // the whole tile is in TMEM: one phase (every thread)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 3);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  if (threadIdx.x == 0) {
    mbar_init(load_bar, 1);
    mbar_init(mma_bar, 1);
    mbar_init(done_bar, 1);
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
  grid_dep_launch();
  grid_dep_wait();

  const int I0 = ti * kTile, J0 = tj * kTile;
  const int rowQ = (bh0 + hl) * M + I0, rowK = (bh0 + hl) * M + J0;
  if (threadIdx.x == 0) {
    const uint64_t dA0 = sdesc_sw128(smem_u32(sA), 16, 1024);
    const uint64_t dB0 = sdesc_sw128(smem_u32(sB), 16, 1024);
    constexpr uint64_t kPart = kBoxBytes >> 4;  // one part box, 16-byte units
    // (query part, key part), smallest products first
    constexpr int kPairs[6][2] = {{2, 0}, {1, 1}, {0, 2}, {1, 0}, {0, 1}, {0, 0}};
    bool ok = true;
#pragma unroll 1
    for (int c = 0; c < kChunks && ok; ++c) {
      // the buffer is free once the previous chunk's MMAs have read it
      if (c > 0 && !(ok = mbar_wait(mma_bar, (c - 1) & 1, abort_flag, status))) break;
      mbar_arrive_expect_tx(load_bar, kChunkBytes);
#pragma unroll
      for (int p = 0; p < 3; ++p) {
        tma_load_3d(&tmQ, sA + p * kBoxBytes, load_bar, 64 * c, rowQ, p);
        tma_load_3d(&tmK, sB + p * kBoxBytes, load_bar, 64 * c, rowK, p);
      }
      if (!(ok = mbar_wait(load_bar, c & 1, abort_flag, status))) {
        // a load that never landed: wait a bounded time for it before the CTA exits
        const long long t0 = clock64();
        while (!mbar_try_wait(load_bar, c & 1) && clock64() - t0 < kWaitCycles) {
        }
        break;
      }
      tc_fence_after();
#pragma unroll
      for (int pr = 0; pr < 6; ++pr) {
        const uint64_t a = dA0 + kPairs[pr][0] * kPart, b = dB0 + kPairs[pr][1] * kPart;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          tc_mma_bf16(tbase, a + kk * 2, b + kk * 2, kScoreIdesc, (c == 0 && pr == 0 && kk == 0) ? 0u : 1u);
      }
      tc_commit(c + 1 < kChunks ? mma_bar : done_bar);
    }
  }
  __syncwarp();
  // the tile is complete and the buffer is free
  const bool ok = mbar_wait(done_bar, 0, abort_flag, status);
  if (ok) {
    tc_fence_after();
    float* stage = reinterpret_cast<float*>(smem);
    const int r = warp * 32 + lane;  // TMEM lane = query row of the tile
#pragma unroll 1
    for (int c = 0; c < kTile / 32; ++c) {
      float v[32];
      tmem_ld32(tbase + (static_cast<uint32_t>(warp * 32) << 16) + 32 * c, v);
      tc_wait_ld();
#pragma unroll
      for (int j = 0; j < 32; j += 4)
        *reinterpret_cast<float4*>(stage + r * kStageStride + 32 * c + j) =
            make_float4(v[j] * tau + 0.0f, v[j + 1] * tau + 0.0f, v[j + 2] * tau + 0.0f, v[j + 3] * tau + 0.0f);
    }
  }
  __syncthreads();
  if (ok) {
    const float* stage = reinterpret_cast<const float*>(smem);
    const int rows = M - I0 < kTile ? M - I0 : kTile;
    for (int r = warp; r < rows; r += 4) {
      float4* dst = reinterpret_cast<float4*>(scores + (static_cast<size_t>(hl) * M + I0 + r) * Mp + J0);
      dst[lane] = *reinterpret_cast<const float4*>(stage + r * kStageStride + 4 * lane);
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
  cudaError_t e = cudaFuncSetAttribute(score_tc_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, kScoreSmem);
  if (e != cudaSuccess) return e;
  const int nt = (M + kTile - 1) / kTile;
  return launch_chained(score_tc_kernel<D>, dim3(nt, nt, nh), dim3(128), kScoreSmem, st, mq, mk, M, Mp, bh0, causal,
                        tau, scores, status);
}

}  // namespace

int score_stride(int M) { return (M + kTile - 1) / kTile * kTile; }

cudaError_t launch_split3(const float* x0, const float* x1, long long n, uint16_t* out0, uint16_t* out1,
                          cudaStream_t st) {
  const long long n4 = n / 4;
  if (n4 == 0) return cudaSuccess;
  const long long want = (2 * n4 + 255) / 256;
  const int grid = static_cast<int>(want < 148LL * 16 ? want : 148LL * 16);
  return launch_chained(split3_kernel, dim3(grid), dim3(256), 0, st, reinterpret_cast<const float4*>(x0),
                        reinterpret_cast<const float4*>(x1), n4, reinterpret_cast<uint2*>(out0),
                        reinterpret_cast<uint2*>(out1));
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
