// pool.cu -- a1: per-block statistics of Q, K and V.
//
// PISA summary (kodorricoding.tistory.com/108), "How are candidate blocks
// narrowed": a representative query and key per block and the sum of the
// values.  FlashPrefill summary, 2.a "Block approximation": the key block is
// represented by its average-pooled vector.
//
// One pass over Q, K and V (HBM-bound): each CTA streams whole 64-row blocks
// with 16-byte loads, sums in fp32 registers, reduces across the row groups
// of a warp with shuffles and across warps through shared memory.
#include <cuda_bf16.h>

#include "internal.h"
#include "sm100.cuh"

namespace psa {
namespace {

__device__ __forceinline__ void add_bf16x8(float (&acc)[8], const uint4 w) {
  const uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    acc[2 * i] += __uint_as_float(u[i] << 16);
    acc[2 * i + 1] += __uint_as_float(u[i] & 0xffff0000u);
  }
}

__device__ __forceinline__ uint16_t f2bf(float x) {
  return __bfloat16_as_ushort(__float2bfloat16_rn(x));
}

// NT = number of input tensors pooled (3: q, k, v; 1: k only, bf16 mean out).
// A work item is one tensor of one block (64 rows), so a grid-stride loop
// has 3x more, smaller items than blocks: the last wave of CTAs is then a
// small part of the pass even when the block count is only a few times the
// number of resident CTAs.
template <int D, int NT>
__global__ void __launch_bounds__(256) pool_kernel(const uint4* __restrict__ q, const uint4* __restrict__ k,
                                                   const uint4* __restrict__ v, int nblk,
                                                   float* __restrict__ qbar, float* __restrict__ kbar,
                                                   float* __restrict__ vsum, uint16_t* __restrict__ kbar_bf16) {
  constexpr int kChunks = D / 8;           // 16-byte chunks per row
  constexpr int kGroups = 256 / kChunks;   // row groups per CTA
  constexpr int kRows = 64 / kGroups;      // rows per thread per block
  __shared__ float red[8][D];
  const int c = threadIdx.x % kChunks;
  const int g = threadIdx.x / kChunks;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int items = nblk * NT;
  grid_dep_launch();
  grid_dep_wait();

  for (int it = blockIdx.x; it < items; it += gridDim.x) {
    const int blk = it / NT, t = it - blk * NT;
    const uint4* src = NT == 1 ? k : (t == 0 ? q : (t == 1 ? k : v));
    const size_t base = static_cast<size_t>(blk) * 64 * kChunks;
    uint4 w[kRows];
#pragma unroll
    for (int r = 0; r < kRows; ++r) w[r] = __ldcs(src + base + static_cast<size_t>(g + r * kGroups) * kChunks + c);
    float acc[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] = 0.f;
#pragma unroll
    for (int r = 0; r < kRows; ++r) add_bf16x8(acc, w[r]);
    // lanes that hold the same chunk differ by multiples of kChunks
#pragma unroll
    for (int o = kChunks; o < 32; o <<= 1)
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[i] += __shfl_xor_sync(0xffffffffu, acc[i], o);
    if (lane < kChunks) {
#pragma unroll
      for (int i = 0; i < 8; ++i) red[warp][c * 8 + i] = acc[i];
    }
    __syncthreads();
    for (int col = threadIdx.x; col < D; col += 256) {
      float s = 0.f;
#pragma unroll
      for (int wi = 0; wi < 8; ++wi) s += red[wi][col];
      const size_t o = static_cast<size_t>(blk) * D + col;
      if (NT == 3) {
        if (t == 0) qbar[o] = s * (1.0f / 64.0f);
        else if (t == 1) kbar[o] = s * (1.0f / 64.0f);
        else vsum[o] = s;
      } else {
        kbar_bf16[o] = f2bf(s * (1.0f / 64.0f));
      }
    }
    __syncthreads();
  }
}

// Zero the 256-byte header of a call's workspace (status word, counters).
__global__ void zero_header_kernel(int4* __restrict__ header) {
  grid_dep_launch();
  grid_dep_wait();
  if (threadIdx.x < 16) header[threadIdx.x] = make_int4(0, 0, 0, 0);
}

__global__ void stats_to_bf16_kernel(const float4* __restrict__ kbar, const float4* __restrict__ vsum,
                                     long long n4, uint2* __restrict__ kb, uint2* __restrict__ vb) {
  grid_dep_launch();
  grid_dep_wait();
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < n4;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    const float4 a = kbar[i];
    const float4 s = vsum[i];
    kb[i] = make_uint2(f2bf(a.x) | (static_cast<uint32_t>(f2bf(a.y)) << 16),
                       f2bf(a.z) | (static_cast<uint32_t>(f2bf(a.w)) << 16));
    vb[i] = make_uint2(f2bf(s.x) | (static_cast<uint32_t>(f2bf(s.y)) << 16),
                       f2bf(s.z) | (static_cast<uint32_t>(f2bf(s.w)) << 16));
  }
}

int pool_grid(long long items) {
  const int cap = device_sm_count() * 8;
  return items < cap ? static_cast<int>(items) : cap;
}

}  // namespace

cudaError_t launch_pool(const uint16_t* q, const uint16_t* k, const uint16_t* v, int BH, int M, int d,
                        float* qbar, float* kbar, float* vsum, cudaStream_t st) {
  const int nblk = BH * M;
  const dim3 grid(pool_grid(3LL * nblk));
  auto* Q = reinterpret_cast<const uint4*>(q);
  auto* K = reinterpret_cast<const uint4*>(k);
  auto* V = reinterpret_cast<const uint4*>(v);
  uint16_t* none = nullptr;
  if (d == 128) return launch_chained(pool_kernel<128, 3>, grid, dim3(256), 0, st, Q, K, V, nblk, qbar, kbar, vsum, none);
  return launch_chained(pool_kernel<64, 3>, grid, dim3(256), 0, st, Q, K, V, nblk, qbar, kbar, vsum, none);
}

cudaError_t launch_pool_keys_bf16(const uint16_t* k, int BH, int M, int d, uint16_t* kbar_bf16,
                                  cudaStream_t st) {
  const int nblk = BH * M;
  const dim3 grid(pool_grid(nblk));
  auto* K = reinterpret_cast<const uint4*>(k);
  const uint4* none = nullptr;
  float* nonef = nullptr;
  if (d == 128)
    return launch_chained(pool_kernel<128, 1>, grid, dim3(256), 0, st, none, K, none, nblk, nonef, nonef, nonef,
                          kbar_bf16);
  return launch_chained(pool_kernel<64, 1>, grid, dim3(256), 0, st, none, K, none, nblk, nonef, nonef, nonef,
                        kbar_bf16);
}

cudaError_t launch_stats_to_bf16(const float* kbar, const float* vsum, long long n, uint16_t* kbar_bf16,
                                 uint16_t* vsum_bf16, cudaStream_t st) {
  const long long n4 = n / 4;  // n = B*H*M*d, d in {64, 128}
  long long blocks = (n4 + 255) / 256;
  const long long cap = device_sm_count() * 16LL;
  if (blocks > cap) blocks = cap;
  if (blocks < 1) blocks = 1;
  return launch_chained(stats_to_bf16_kernel, dim3(static_cast<unsigned>(blocks)), dim3(256), 0, st,
                        reinterpret_cast<const float4*>(kbar), reinterpret_cast<const float4*>(vsum), n4,
                        reinterpret_cast<uint2*>(kbar_bf16), reinterpret_cast<uint2*>(vsum_bf16));
}

cudaError_t launch_zero_header(void* workspace, cudaStream_t st) {
  return launch_chained(zero_header_kernel, dim3(1), dim3(32), 0, st, static_cast<int4*>(workspace));
}

}  // namespace psa
