// hyd.cu -- f-1: the first-order correction of the unselected blocks.
//
// PISA summary (kodorricoding.tistory.com/108), "Why approximating
// unselected blocks keeps softmax intact" and the FAQ "Why a global
// first-order correction?": beyond the 0th-order term around the block-mean
// key, the expansion of e^{q.k/sqrt(d)} to first order adds, for every
// unselected block J, e^{a_iJ} H^T q_i / sqrt(d) to the numerator, where the
// per-block statistic is H_J = sum_{j in J} (k_j - kbar_J) v_j^T; the
// denominator gains nothing (the deviations sum to zero over a block).  The
// pages replace the per-block matrices by one global statistic; the reading
// taken here is H = the mean of H_J over the blocks of a head.  Then
//   out_i = out0_i + w_i * (q_i^T H) / sqrt(d),
//   w_i   = sum_{J unselected} e^{a_iJ} / den_i,
// with out0 the 0th-order output and den_i its denominator.  The attention
// kernel's hyd mode writes out0 and w (one extra tensor-core product per
// pooled tile gives the column sums of the 0th-order weights); the two
// kernels here compute H and apply the correction.
//
// Statistic.  For one head, sum_J H_J = K^T V - Kbar^T Vsum (Kbar, Vsum the
// [M, d] pooled means and sums).  K^T V (inner dimension N) runs on the
// tensor cores: a CTA streams the K and V blocks of a range of key blocks
// through a 4-stage TMA ring and accumulates D[d x d] += K_J^T V_J in TMEM
// (both operands MN-major, 64 tokens per block); its epilogue subtracts the
// range's kbar_J vsum_J^T in fp32 on the CUDA cores and writes a partial
// matrix.  A second launch sums the partials of each head in a fixed order
// and divides by M (deterministic).  HBM: one read of K and V.
//
// Correction.  Per 128-query tile, X = Q_tile . H on the tensor cores (A =
// the query tile, K-major, by TMA; B = H split into two bf16 parts h0 + h1,
// h1 = bf16(H - h0), built in shared memory from the fp32 statistic, so the
// product carries ~2^-16 relative error); the output tile comes in by TMA
// next to the query tile, each epilogue thread adds w_i * X_i / sqrt(d) to its
// query row in shared memory, and a TMA store writes the tile back.  A CTA
// serves tiles of one head only, so H is built once per CTA.
#include <cuda_bf16.h>

#include "internal.h"
#include "sm100.cuh"

namespace psa {
namespace {

// ------------------------------------------------------------------ statistic
constexpr int kStatThreads = 128;
constexpr int kStatStages = 4;

template <int D>
struct StatCfg {
  static constexpr int kTileBytes = 64 * D * 2;        // one 64-token block of K or V
  static constexpr int kStageBytes = 2 * kTileBytes;   // K then V
  static constexpr int kSmem = kStatStages * kStageBytes + 1024 + 256;
  // D[128 x D] += K_J^T (M = key features, K = tokens) . V_J (N = value
  // features): both operands MN-major.  At d = 64 the A view repeats its
  // 64-feature atom (rows 64..127 of D duplicate rows 0..63 and are unused).
  static constexpr uint32_t kIdesc = idesc_bf16_f32(128, D, 1, 1);
  // the epilogue stages 64 blocks of kbar and vsum (fp32) in the ring
  static_assert(2 * 64 * D * 4 <= kStatStages * kStageBytes, "epilogue staging fits the ring");
};

template <int D>
__global__ void __launch_bounds__(kStatThreads)
    hyd_stat_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                    const float* __restrict__ kbar, const float* __restrict__ vsum, int M, int per,
                    int chunks, float* __restrict__ partial, int* status) {
  using C = StatCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kStatStages * C::kStageBytes);
  uint64_t* full = bars;                    // [stages] K and V of a block landed
  uint64_t* empty = bars + kStatStages;     // [stages] the block's MMAs are done
  uint64_t* done = bars + 2 * kStatStages;  // every MMA of the CTA is done
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * kStatStages + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x / 32;
  const int chunk = blockIdx.x, bh = blockIdx.y;
  const int J0 = chunk * per;
  const int J1 = min(M, J0 + per);
  const int nblk = J1 - J0;  // >= 1 by construction of the grid

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStatStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(done, 1);
    *abort_flag = 0;
    fence_barrier_init();
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 128);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tmem_slot;

  if (threadIdx.x == 0) {
    // ---------------------------------------------------------- TMA producer
    int issued[kStatStages] = {};
    bool ok = true;
    for (int i = 0; i < nblk && ok; ++i) {
      const int s = i % kStatStages;
      if (i >= kStatStages && !(ok = mbar_wait(&empty[s], ((i / kStatStages) - 1) & 1, abort_flag, status))) break;
      uint8_t* dst = smem + s * C::kStageBytes;
      mbar_arrive_expect_tx(&full[s], C::kStageBytes);
      const int y = 64 * (J0 + i);
#pragma unroll
      for (int c = 0; c < D / 64; ++c) {
        tma_load_3d(&tmK, dst + c * 8192, &full[s], 64 * c, y, bh);
        tma_load_3d(&tmV, dst + C::kTileBytes + c * 8192, &full[s], 64 * c, y, bh);
      }
      ++issued[s];
    }
    // no bulk copy may still be writing shared memory when the CTA leaves
    for (int s = 0; s < kStatStages; ++s) {
      if (issued[s] == 0) continue;
      const long long t0 = clock64();
      while (!mbar_try_wait(&full[s], (issued[s] - 1) & 1) && clock64() - t0 < kWaitCycles) {
      }
    }
  } else if (threadIdx.x == 32) {
    // ---------------------------------------------------------- MMA issuer
    const uint64_t a0 = sdesc_sw128(smem_u32(smem), D == 128 ? 8192 : 0, 1024);
    const uint64_t b0 = sdesc_sw128(smem_u32(smem + C::kTileBytes), 8192, 1024);
    constexpr uint64_t kStage16 = C::kStageBytes >> 4;
    for (int i = 0; i < nblk; ++i) {
      const int s = i % kStatStages;
      if (!mbar_wait(&full[s], (i / kStatStages) & 1, abort_flag, status)) break;
      tc_fence_after();
      const uint64_t a = a0 + s * kStage16, b = b0 + s * kStage16;
#pragma unroll
      for (int kk = 0; kk < 4; ++kk)  // 16 tokens per step: 16 rows of 128 B
        tc_mma_bf16(tbase, a + 128 * kk, b + 128 * kk, C::kIdesc, (i > 0 || kk > 0) ? 1u : 0u);
      tc_commit(&empty[s]);
    }
    tc_commit(done);
  }
  __syncwarp();
  // ------------------------------------------------------------ epilogue
  // thread t = TMEM lane t = key feature t of the partial matrix.  Every MMA
  // is done and every load has landed, so the ring's shared memory is free:
  // the range's kbar and vsum rows are staged there (64 blocks at a time,
  // coalesced), and each thread accumulates its row of sum_J kbar_J vsum_J^T
  // from shared memory in fp32.
  const bool ok = mbar_wait(done, 0, abort_flag, status);
  tc_fence_after();
  const int t = threadIdx.x;
  constexpr int kStageBlocks = 64;
  float* kb_s = reinterpret_cast<float*>(smem);                // [64][D]
  float* vs_s = kb_s + kStageBlocks * D;                       // [64][D]
  float corr[D];
#pragma unroll
  for (int i = 0; i < D; ++i) corr[i] = 0.f;
  const size_t head = static_cast<size_t>(bh) * M;
  for (int Jc = J0; Jc < J1; Jc += kStageBlocks) {
    const int n = min(kStageBlocks, J1 - Jc);
    __syncthreads();  // the previous range is consumed
    const float4* kb4 = reinterpret_cast<const float4*>(kbar + (head + Jc) * D);
    const float4* vs4 = reinterpret_cast<const float4*>(vsum + (head + Jc) * D);
    for (int e = t; e < n * D / 4; e += kStatThreads) {
      reinterpret_cast<float4*>(kb_s)[e] = __ldg(kb4 + e);
      reinterpret_cast<float4*>(vs_s)[e] = __ldg(vs4 + e);
    }
    __syncthreads();
    if (t < D) {
      for (int J = 0; J < n; ++J) {
        const float kb = kb_s[J * D + t];
        const float4* row = reinterpret_cast<const float4*>(vs_s + J * D);
#pragma unroll
        for (int i = 0; i < D / 4; ++i) {
          const float4 x = row[i];
          corr[4 * i] = fmaf(kb, x.x, corr[4 * i]);
          corr[4 * i + 1] = fmaf(kb, x.y, corr[4 * i + 1]);
          corr[4 * i + 2] = fmaf(kb, x.z, corr[4 * i + 2]);
          corr[4 * i + 3] = fmaf(kb, x.w, corr[4 * i + 3]);
        }
      }
    }
  }
  if (ok && t < D) {
    float* dst = partial + (static_cast<size_t>(bh) * chunks + chunk) * D * D + static_cast<size_t>(t) * D;
#pragma unroll
    for (int c = 0; c < D / 32; ++c) {
      float acc[32];
      tmem_ld32(tbase + (static_cast<uint32_t>(warp * 32) << 16) + 32 * c, acc);
      tc_wait_ld();
      float4* out4 = reinterpret_cast<float4*>(dst + 32 * c);
#pragma unroll
      for (int i = 0; i < 8; ++i)
        out4[i] = make_float4(acc[4 * i] - corr[32 * c + 4 * i], acc[4 * i + 1] - corr[32 * c + 4 * i + 1],
                              acc[4 * i + 2] - corr[32 * c + 4 * i + 2], acc[4 * i + 3] - corr[32 * c + 4 * i + 3]);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tbase, 128);
  }
}

// hstat[bh] = (1/M) * sum over the chunks of partial[bh][chunk], in chunk order.
__global__ void __launch_bounds__(256) hyd_reduce_kernel(const float* __restrict__ partial, int chunks, int dd,
                                                         float inv_m, float* __restrict__ hstat) {
  const int bh = blockIdx.y;
  const int e = blockIdx.x * 256 + threadIdx.x;
  if (e >= dd) return;
  const float* p = partial + static_cast<size_t>(bh) * chunks * dd + e;
  float s = 0.f;
  for (int c = 0; c < chunks; ++c) s += p[static_cast<size_t>(c) * dd];
  hstat[static_cast<size_t>(bh) * dd + e] = s * inv_m;
}

// ------------------------------------------------------------------ correction
constexpr int kApplyThreads = 192;  // warp 0 TMA, warp 1 MMA, warps 2..5 epilogue
constexpr int kApplyStages = 2;

template <int D>
struct ApplyCfg {
  static constexpr int kTileBytes = 128 * D * 2;  // 128 rows of q (or out): D/64 boxes of 16 KB
  static constexpr int kStageBytes = 2 * kTileBytes;
  static constexpr int kHBytes = D * D * 2;     // one bf16 part of H
  static constexpr int kOffH = kApplyStages * kStageBytes;
  static constexpr int kSmem = kOffH + 2 * kHBytes + 1024 + 256;
  // X[128 queries x D] = Q (A, K-major) . H (B: N = value features, K = key
  // features, MN-major)
  static constexpr uint32_t kIdesc = idesc_bf16_f32(128, D, 0, 1);
};

// out[i] += w_i * (q_i^T H) tau for the 128-query tiles [t0, t0 + per) of
// head blockIdx.y.  A stage holds the query tile and the output tile (both by
// TMA, 128-byte swizzle); the MMA warp computes X = Q H into one of two TMEM
// buffers; the epilogue warps (one query row per thread) add w X tau to the
// output rows in shared memory, and one thread writes the tile back with a
// TMA store, after which the stage is free again.
template <int D>
__global__ void __launch_bounds__(kApplyThreads)
    hyd_apply_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmO,
                     const float* __restrict__ hstat, const float* __restrict__ wts, int N, int per, float tau,
                     int* status) {
  using C = ApplyCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sH = smem + C::kOffH;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kOffH + 2 * C::kHBytes);
  uint64_t* full = bars;                              // [stages] q and out tiles landed
  uint64_t* stage_free = bars + kApplyStages;         // [stages] the out tile is written back
  uint64_t* acc_full = bars + 2 * kApplyStages;       // [2] X in TMEM buffer (commit)
  uint64_t* acc_empty = bars + 2 * kApplyStages + 2;  // [2] X read (4 epilogue warps)
  uint64_t* drain = bars + 2 * kApplyStages + 4;      // teardown of the MMA issuer
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * kApplyStages + 5);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int bh = blockIdx.y;
  const int ntile = (N + 127) / 128;
  const int t0 = blockIdx.x * per;
  const int t1 = min(ntile, t0 + per);
  const int nt = t1 - t0;  // >= 1 by construction of the grid

  // H of this head as two bf16 parts, in the MN-major 128-byte-swizzled
  // layout of the B operand: part p, value-feature atom n/64, key-feature
  // row k (128 bytes), 16-byte chunk ((n % 64) / 8) ^ (k % 8)
  {
    const float* Hh = hstat + static_cast<size_t>(bh) * D * D;
    for (int e = threadIdx.x; e < D * D; e += kApplyThreads) {
      const int k = e / D, n = e % D;
      const float h = Hh[e];
      const __nv_bfloat16 h0 = __float2bfloat16_rn(h);
      const __nv_bfloat16 h1 = __float2bfloat16_rn(h - __bfloat162float(h0));
      const int off = (n / 64) * (D * 128) + k * 128 + ((((n % 64) / 8) ^ (k % 8)) << 4) + (n % 8) * 2;
      *reinterpret_cast<__nv_bfloat16*>(sH + off) = h0;
      *reinterpret_cast<__nv_bfloat16*>(sH + C::kHBytes + off) = h1;
    }
  }
  fence_async_shared();
  if (threadIdx.x == 0) {
    for (int s = 0; s < kApplyStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&stage_free[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], 4);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmO);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 256);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tmem_slot;

  if (warp == 0) {
    // ---------------------------------------------------------- TMA producer
    if (lane == 0) {
      int issued[kApplyStages] = {};
      for (int i = 0; i < nt; ++i) {
        const int s = i % kApplyStages;
        if (i >= kApplyStages &&
            !mbar_wait(&stage_free[s], ((i / kApplyStages) - 1) & 1, abort_flag, status))
          break;
        uint8_t* dst = smem + s * C::kStageBytes;
        mbar_arrive_expect_tx(&full[s], C::kStageBytes);
        const int y = 128 * (t0 + i);
#pragma unroll
        for (int c = 0; c < D / 64; ++c) {
          tma_load_3d(&tmQ, dst + c * 16384, &full[s], 64 * c, y, bh);
          tma_load_3d(&tmO, dst + C::kTileBytes + c * 16384, &full[s], 64 * c, y, bh);
        }
        ++issued[s];
      }
      for (int s = 0; s < kApplyStages; ++s) {
        if (issued[s] == 0) continue;
        const long long c0 = clock64();
        while (!mbar_try_wait(&full[s], (issued[s] - 1) & 1) && clock64() - c0 < kWaitCycles) {
        }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA issuer
    if (lane == 0) {
      const uint64_t a0 = sdesc_sw128(smem_u32(smem), 16, 1024);
      const uint64_t b0 = sdesc_sw128(smem_u32(sH), D * 128, 1024);
      constexpr uint64_t kStage16 = C::kStageBytes >> 4, kH16 = C::kHBytes >> 4;
      for (int i = 0; i < nt; ++i) {
        const int s = i % kApplyStages, b = i & 1;
        if (!mbar_wait(&full[s], (i / kApplyStages) & 1, abort_flag, status)) break;
        if (i >= 2 && !mbar_wait(&acc_empty[b], ((i >> 1) - 1) & 1, abort_flag, status)) break;
        tc_fence_after();
        const uint32_t dt = tbase + D * b;
        const uint64_t a = a0 + s * kStage16;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          // A: 16 key features = 32 bytes inside a 64-feature box (boxes 16 KB apart);
          // B: 16 key-feature rows of 128 bytes
          const uint64_t ak = a + (kk >> 2) * 1024 + (kk & 3) * 2;
          tc_mma_bf16(dt, ak, b0 + 128 * kk, C::kIdesc, kk > 0 ? 1u : 0u);
          tc_mma_bf16(dt, ak, b0 + kH16 + 128 * kk, C::kIdesc, 1u);
        }
        tc_commit(&acc_full[b]);
      }
      // every MMA must finish before TMEM is freed
      tc_commit(drain);
      const long long c0 = clock64();
      while (!mbar_try_wait(drain, 0) && clock64() - c0 < kWaitCycles) {
      }
    }
    __syncwarp();
  } else {
    // ---------------------------------------------------------- epilogue
    const int quarter = warp & 3;            // TMEM lanes 32*quarter .. +31
    const int r = quarter * 32 + lane;       // query row of the tile
    const int et = threadIdx.x - 64;         // 0..127 over the epilogue warps
    const size_t head = static_cast<size_t>(bh) * N;
    for (int i = 0; i < nt; ++i) {
      const int s = i % kApplyStages, b = i & 1;
      if (!mbar_wait(&acc_full[b], (i >> 1) & 1, abort_flag, status)) break;
      tc_fence_after();
      const int qi = 128 * (t0 + i) + r;
      const float sc = (qi < N ? wts[head + qi] : 0.f) * tau;
      uint8_t* otile = smem + s * C::kStageBytes + C::kTileBytes;
#pragma unroll 1
      for (int c = 0; c < D / 32; ++c) {
        float x[32];
        tmem_ld32(tbase + D * b + (static_cast<uint32_t>(quarter * 32) << 16) + 32 * c, x);
        tc_wait_ld();
        if (sc != 0.f) {
          // features 32c .. 32c+31: box c/2, 16-byte pieces 4(c%2) .. +3 of row r
          uint8_t* row = otile + (c >> 1) * 16384 + r * 128;
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            uint4* piece = reinterpret_cast<uint4*>(row + ((((c & 1) * 4 + j) ^ (r & 7)) << 4));
            uint4 o = *piece;
            uint32_t u[4] = {o.x, o.y, o.z, o.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const float lo = __uint_as_float(u[e] << 16) + sc * x[8 * j + 2 * e];
              const float hi = __uint_as_float(u[e] & 0xffff0000u) + sc * x[8 * j + 2 * e + 1];
              u[e] = pack_bf16x2(lo, hi);
            }
            *piece = make_uint4(u[0], u[1], u[2], u[3]);
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[b]);
      // write the tile back (rows past N are clipped by the TMA unit)
      fence_async_shared();
      named_barrier_sync(1, 128);
      if (et == 0) {
#pragma unroll
        for (int c = 0; c < D / 64; ++c) tma_store_3d(&tmO, otile + c * 16384, 64 * c, 128 * (t0 + i), bh);
        bulk_commit();
        bulk_wait_read0();  // the store has read the tile: the stage may be refilled
        mbar_arrive(&stage_free[s]);
      }
    }
    if (et == 0) bulk_wait0();
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tbase, 256);
  }
}

// One CTA per SM (the ring holds an SM's shared memory): as many chunks of
// key blocks per head as keep the grid within one wave.
int stat_chunks(int BH, int M, int& per) {
  const int sms = device_sm_count();
  int want = sms / BH;
  if (want < 1) want = 1;
  if (want > M) want = M;
  per = (M + want - 1) / want;
  return (M + per - 1) / per;
}

template <int D>
cudaError_t launch_stat_d(const uint16_t* k, const uint16_t* v, const float* kbar, const float* vsum, int BH,
                          int N, float* partial, float* hstat, int* status, cudaStream_t st) {
  using C = StatCfg<D>;
  const int M = N / 64;
  CUtensorMap mk, mv;
  if (encode_tensor_map_3d_bf16(&mk, k, D, N, BH, 64, 64) != CUDA_SUCCESS ||
      encode_tensor_map_3d_bf16(&mv, v, D, N, BH, 64, 64) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  int per = 1;
  const int chunks = stat_chunks(BH, M, per);
  cudaError_t e = cudaFuncSetAttribute(hyd_stat_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmem);
  if (e != cudaSuccess) return e;
  hyd_stat_kernel<D><<<dim3(chunks, BH), kStatThreads, C::kSmem, st>>>(mk, mv, kbar, vsum, M, per, chunks,
                                                                       partial, status);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  hyd_reduce_kernel<<<dim3((D * D + 255) / 256, BH), 256, 0, st>>>(partial, chunks, D * D, 1.0f / M, hstat);
  return cudaGetLastError();
}

template <int D>
cudaError_t launch_apply_d(const uint16_t* q, const float* hstat, const float* w, uint16_t* out, int BH, int N,
                           int* status, cudaStream_t st) {
  using C = ApplyCfg<D>;
  CUtensorMap mq, mo;
  if (encode_tensor_map_3d_bf16(&mq, q, D, N, BH, 64, 128) != CUDA_SUCCESS ||
      encode_tensor_map_3d_bf16(&mo, out, D, N, BH, 64, 128) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  const int ntile = (N + 127) / 128;
  const int sms = device_sm_count();
  int want = sms / BH;  // one CTA per SM, one wave
  if (want < 1) want = 1;
  if (want > ntile) want = ntile;
  const int per = (ntile + want - 1) / want;
  const int chunks = (ntile + per - 1) / per;
  cudaError_t e = cudaFuncSetAttribute(hyd_apply_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmem);
  if (e != cudaSuccess) return e;
  hyd_apply_kernel<D><<<dim3(chunks, BH), kApplyThreads, C::kSmem, st>>>(
      mq, mo, hstat, w, N, per, 1.0f / sqrtf(static_cast<float>(D)), status);
  return cudaGetLastError();
}

}  // namespace

size_t hyd_partial_bytes(int BH, int M, int d) {
  int per = 1;
  // the grid is sized for the largest device this library supports (the
  // chunk count only grows with the SM count), so the workspace never
  // depends on the device it is used on
  const int sms = 256;
  int want = (2 * sms + BH - 1) / BH;
  if (want < 1) want = 1;
  if (want > M) want = M;
  per = (M + want - 1) / want;
  const size_t chunks = static_cast<size_t>((M + per - 1) / per);
  return static_cast<size_t>(BH) * chunks * d * d * 4;
}

cudaError_t launch_hyd_stat(const uint16_t* k, const uint16_t* v, const float* kbar, const float* vsum, int BH,
                            int N, int d, float* partial, float* hstat, int* status, cudaStream_t st) {
  return d == 128 ? launch_stat_d<128>(k, v, kbar, vsum, BH, N, partial, hstat, status, st)
                  : launch_stat_d<64>(k, v, kbar, vsum, BH, N, partial, hstat, status, st);
}

cudaError_t launch_hyd_apply(const uint16_t* q, const float* hstat, const float* w, uint16_t* out, int BH, int N,
                             int d, int* status, cudaStream_t st) {
  return d == 128 ? launch_apply_d<128>(q, hstat, w, out, BH, N, status, st)
                  : launch_apply_d<64>(q, hstat, w, out, BH, N, status, st);
}

}  // namespace psa
