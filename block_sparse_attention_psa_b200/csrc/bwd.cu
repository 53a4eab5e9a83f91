// bwd.cu -- f-4: gradients of the 0th-order block-sparse attention for fixed
// block lists (the training-support variant of the PISA summary, "Minimal
// usage": the simplified 0th-order version supports training).
//
// Forward, for query i of block I (lists S_I, other candidates U_I):
//   out_i = sum_{j listed} p_ij v_j + sum_{J in U_I} pi_iJ vsum_J,
//   p_ij = e^{z_ij - lse_i}, pi_iJ = e^{a_iJ - lse_i},
//   z_ij = tau q_i.k_j, a_iJ = tau q_i.kbar_J, tau = 1/sqrt(d),
// with kbar_J the mean and vsum_J the sum of block J's keys and values.
// With D_i = dO_i . out_i (the usual softmax identity):
//   dS_ij = p_ij (dO_i.v_j - D_i)                (listed keys)
//   dA_iJ = pi_iJ (dO_i.vsum_J - 64 D_i)         (pseudo-key of block J)
//   dq_i   = tau (sum_j dS_ij k_j + sum_J dA_iJ kbar_J)
//   dk_j   = tau sum_i dS_ij q_i + dkbar_J / 64,  dkbar_J = tau sum_i dA_iJ q_i
//   dv_j   = sum_i p_ij dO_i + dvsum_J,           dvsum_J = sum_i pi_iJ dO_i
// (the last terms of dk and dv reach every token j of block J through the
// mean and the sum of the pooling).  Routing is a selection and carries no
// gradient.
//
// Launches: delta (D_i and -lse_i log2 e), the listed-block bitmaps, the
// pseudo-key gradients per tile of 128 pooled keys (partial sums over ranges
// of query blocks, then a fixed-order reduction), dq per query block, and dk,
// dv per key block.  The three gradient kernels run on the tensor cores
// (tcgen05, TMEM accumulators, TMA operands) with one layout: warps 0-7 read
// and write TMEM rows and do the elementwise work (warps w and w + 4 share
// lane quarter w % 4, each taking half of a row's 64 columns), warp 8 loads
// by TMA, warp 9 issues the score products and owns TMEM, warp 10 issues the
// accumulations; the dq and dk, dv kernels draw their units and items from
// dynamic schedulers.  Every product keeps M = 128 rows:
//   pseudo: S^T = Kbar_t Q_I^T, dP^T = Vsum_t dO_I^T   [128 pooled keys x 64 q]
//           dVsum_t += Pi^T dO_I, dKbar_t += dA^T Q_I   [128 x d]
//   dq:     S^T = K_t Q_I^T, dP^T = V_t dO_I^T           [128 keys x 64 q]
//           dq^T += K_t^T dS^T                           [d x 64 q]
//   dk, dv: S = Q_p K_J^T, dP = dO_p V_J^T               [128 q (two query blocks) x 64 keys]
//           dV^T += dO_p^T P, dK^T += Q_p^T dS           [d x 64 keys]
// Every wait is bounded; a wait that runs out records PSA_ERR_TIMEOUT.
#include <cuda_bf16.h>

#include "internal.h"
#include "sm100.cuh"

namespace psa {
namespace {

// Warps 0-7 elementwise, 8 TMA, 9 the score products (and TMEM), 10 the
// accumulations: the scores of the next step and the accumulations of the
// current one issue from two threads (an issue waits for the tensor core to
// accept it).
constexpr int kBwdThreads = 352;
constexpr int kWarpTma = 8, kWarpMma = 9, kWarpAcc = 10;
constexpr float kLog2e = 1.4426950408889634f;

struct BwdArgs {
  const int* row_ptr;
  const int* col_idx;
  long long col_cap;
  const uint32_t* bits;   // [BH*M][nw] listed blocks of each row
  const float* nlse2;     // [BH*N] -lse * log2(e)
  const float* delta;     // [BH*N] dO . out
  int BH, M, N, nw, causal;
  float sl;               // log2(e) / sqrt(d)
  float tau;              // 1 / sqrt(d)
  int* status;
  int* sched;             // ticket counter of the dk, dv item scheduler (zero at the call's start)
};

// 32 bf16 (columns 32*half ..) of row r of a 128-byte-swizzled tile (row r,
// 16-byte chunk c at (c ^ (r % 8)) * 16)
__device__ __forceinline__ void store_half_row(uint8_t* tile, int r, int half, const uint32_t (&pk)[16]) {
  const uint32_t base = smem_u32(tile) + r * 128;
#pragma unroll
  for (int c = 0; c < 4; ++c)
    st_shared_v4(base + (((4 * half + c) ^ (r & 7)) << 4), pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
}

// Bounded wait for a copy's completion during teardown (ignores the abort flag).
__device__ __forceinline__ void drain_wait(uint64_t* bar, uint32_t parity) {
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, parity) && clock64() - t0 < kWaitCycles) {
  }
}

// ------------------------------------------------------------------ delta
// D_i = dO_i . out_i and -lse_i log2(e); 8 lanes per row.
template <int D>
__global__ void __launch_bounds__(256) bwd_delta_kernel(const uint4* __restrict__ out, const uint4* __restrict__ dout,
                                                        const float* __restrict__ lse, long long rows,
                                                        float* __restrict__ delta, float* __restrict__ nlse2) {
  constexpr int kPer = D / 64;  // 16-byte chunks per lane
  for (long long g = blockIdx.x * 256LL + threadIdx.x; g < rows * 8; g += static_cast<long long>(gridDim.x) * 256) {
    const long long row = g >> 3;
    const int sub = static_cast<int>(g & 7);
    float acc = 0.f;
#pragma unroll
    for (int j = 0; j < kPer; ++j) {
      const uint4 a = __ldg(out + row * (D / 8) + sub * kPer + j);
      const uint4 b = __ldg(dout + row * (D / 8) + sub * kPer + j);
      const uint32_t ua[4] = {a.x, a.y, a.z, a.w}, ub[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        acc = fmaf(__uint_as_float(ua[e] << 16), __uint_as_float(ub[e] << 16), acc);
        acc = fmaf(__uint_as_float(ua[e] & 0xffff0000u), __uint_as_float(ub[e] & 0xffff0000u), acc);
      }
    }
    acc += __shfl_xor_sync(0xffffffffu, acc, 4);
    acc += __shfl_xor_sync(0xffffffffu, acc, 2);
    acc += __shfl_xor_sync(0xffffffffu, acc, 1);
    if (sub == 0) {
      delta[row] = acc;
      nlse2[row] = -lse[row] * kLog2e;
    }
  }
}

// ------------------------------------------------------------------ bitmaps
// One warp per row: bits[row][J / 32] bit J % 32 set iff J is listed; a
// malformed row (range out of bounds, entry out of range, repeat) is recorded
// as PSA_ERR_CSR and its bad entries are left out.
__global__ void __launch_bounds__(256) bwd_bits_kernel(const int* __restrict__ row_ptr,
                                                       const int* __restrict__ col_idx, long long col_cap, int M,
                                                       int nw, int causal, long long nrows,
                                                       uint32_t* __restrict__ bits, int* status) {
  const int lane = threadIdx.x % 32;
  const long long row = blockIdx.x * 8LL + threadIdx.x / 32;
  if (row >= nrows) return;
  uint32_t* b = bits + row * nw;
  for (int w = lane; w < nw; w += 32) b[w] = 0u;
  __syncwarp();
  const int I = static_cast<int>(row % M);
  const int cand = causal ? I + 1 : M;
  const int a = row_ptr[row], e = row_ptr[row + 1];
  if (a < 0 || e < a || static_cast<long long>(e) > col_cap || e - a > cand) {
    if (lane == 0) record_status(status, kStatusCsr);
    return;
  }
  for (int i = a + lane; i < e; i += 32) {
    const int J = col_idx[i];
    if (J < 0 || J >= cand) {
      record_status(status, kStatusCsr);
      continue;
    }
    const uint32_t bit = 1u << (J & 31);
    if (atomicOr(&b[J >> 5], bit) & bit) record_status(status, kStatusCsr);
  }
}

__device__ __forceinline__ bool listed(const BwdArgs& g, int bh, int I, int J) {
  const uint32_t w = __ldg(g.bits + (static_cast<size_t>(bh) * g.M + I) * g.nw + (J >> 5));
  return (w >> (J & 31)) & 1u;
}

// ------------------------------------------------------------------ pseudo-key gradients
template <int D>
struct PseudoCfg {
  static constexpr int kTile = 128 * D * 2;  // 128 pooled rows (bf16 kbar or vsum)
  static constexpr int kQ = 64 * D * 2;      // one 64-row block of q or dO
  static constexpr int kStage = (2 * kQ + 512 + 1023) / 1024 * 1024;  // q, dO, -lse log2e [64], D [64]
  static constexpr int kBuf = 128 * 128;     // one 128 x 64 bf16 operand
  static constexpr int kOffVs = kTile, kOffStage = 2 * kTile;
  static constexpr int kOffPi = kOffStage + 2 * kStage, kOffDa = kOffPi + kBuf;
  static constexpr int kOffBars = kOffDa + kBuf;
  static constexpr int kSmem = kOffBars + 256 + 1024;
  static constexpr uint32_t kIdescS = idesc_bf16_f32(128, 64, 0, 0);
  static constexpr uint32_t kIdescAcc = idesc_bf16_f32(128, D, 0, 1);
};

// Item = (head, tile of 128 pooled keys, range of query blocks): partial
// dvsum and dkbar (tau applied) of the tile over the range.
template <int D>
__global__ void __launch_bounds__(kBwdThreads, 1)
    bwd_pseudo_kernel(const __grid_constant__ CUtensorMap tmKb, const __grid_constant__ CUtensorMap tmVs,
                      const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmDO,
                      const BwdArgs g, int tiles, int chunks, int per, float* __restrict__ part_dvs,
                      float* __restrict__ part_dkb) {
  using C = PseudoCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sKb = smem;
  uint8_t* sVs = smem + C::kOffVs;
  uint8_t* sPi = smem + C::kOffPi;
  uint8_t* sDa = smem + C::kOffDa;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kOffBars);
  uint64_t* kv_full = bars + 0;
  uint64_t* full = bars + 1;        // [2] stage landed
  uint64_t* stage_free = bars + 3;  // [2] the stage's accumulation MMAs are done
  uint64_t* s_full = bars + 5;      // [2] S^T, dP^T ready
  uint64_t* s_empty = bars + 7;     // [2] read by the 4 elementwise warps
  uint64_t* pd_full = bars + 9;     // Pi^T, dA^T written (4 warps)
  uint64_t* pd_free = bars + 10;    // their MMAs are done
  uint64_t* done = bars + 11;       // every accumulation MMA is done
  uint64_t* drain_s = bars + 12;    // teardown of the scores issuer
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 13);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int item = blockIdx.x;
  const int chunk = item % chunks, tile = (item / chunks) % tiles, bh = item / (chunks * tiles);
  int start = chunk * per;
  const int end = min(g.M, start + per);
  if (g.causal) start = max(start, tile * 128 + 1);  // J < I for some J of the tile
  const int n = max(0, end - start);

  if (threadIdx.x == 0) {
    mbar_init(kv_full, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&stage_free[i], 1);
      mbar_init(&s_full[i], 1);
      mbar_init(&s_empty[i], 8);
    }
    mbar_init(pd_full, 8);
    mbar_init(pd_free, 1);
    mbar_init(done, 1);
    mbar_init(drain_s, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == kWarpMma) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tmem_slot;
  const uint32_t t_acc_vs = tbase + 256, t_acc_kb = tbase + 256 + D;

  if (warp == kWarpTma) {
    if (lane == 0 && n > 0) {
      // the tile's pooled keys and value sums, once
      mbar_arrive_expect_tx(kv_full, 2 * C::kTile);
#pragma unroll
      for (int c = 0; c < D / 64; ++c) {
        tma_load_3d(&tmKb, sKb + c * 16384, kv_full, 64 * c, tile * 128, bh);
        tma_load_3d(&tmKb, sKb + c * 16384 + 8192, kv_full, 64 * c, tile * 128 + 64, bh);
        tma_load_3d(&tmVs, sVs + c * 16384, kv_full, 64 * c, tile * 128, bh);
        tma_load_3d(&tmVs, sVs + c * 16384 + 8192, kv_full, 64 * c, tile * 128 + 64, bh);
      }
      int issued[2] = {0, 0};
      for (int i = 0; i < n; ++i) {
        const int s = i & 1;
        if (i >= 2 && !mbar_wait(&stage_free[s], ((i >> 1) - 1) & 1, abort_flag, g.status)) break;
        uint8_t* st = smem + C::kOffStage + s * C::kStage;
        const int I = start + i;
        mbar_arrive_expect_tx(&full[s], 2 * C::kQ + 512);
#pragma unroll
        for (int c = 0; c < D / 64; ++c) {
          tma_load_3d(&tmQ, st + c * 8192, &full[s], 64 * c, 64 * I, bh);
          tma_load_3d(&tmDO, st + C::kQ + c * 8192, &full[s], 64 * c, 64 * I, bh);
        }
        const size_t r0 = static_cast<size_t>(bh) * g.N + 64 * I;
        bulk_load(st + 2 * C::kQ, g.nlse2 + r0, 256, &full[s]);
        bulk_load(st + 2 * C::kQ + 256, g.delta + r0, 256, &full[s]);
        ++issued[s];
      }
      drain_wait(kv_full, 0);
      for (int s = 0; s < 2; ++s)
        if (issued[s]) drain_wait(&full[s], (issued[s] - 1) & 1);
    }
    __syncwarp();
  } else if (warp == kWarpMma) {
    // ---------------------------------------------------------- scores issuer
    if (lane == 0) {
      bool ok = n == 0 || mbar_wait(kv_full, 0, abort_flag, g.status);
      const uint64_t dKb = sdesc_sw128(smem_u32(sKb), 16, 1024);
      const uint64_t dVs = sdesc_sw128(smem_u32(sVs), 16, 1024);
      const uint64_t dStage = sdesc_sw128(smem_u32(smem + C::kOffStage), 16, 1024);
      constexpr uint64_t kSt16 = C::kStage >> 4, kQ16 = C::kQ >> 4;
      for (int i = 0; ok && i < n; ++i) {
        const int s = i & 1, b = i & 1;
        if (!(ok = mbar_wait(&full[s], (i >> 1) & 1, abort_flag, g.status))) break;
        if (i >= 2 && !(ok = mbar_wait(&s_empty[b], ((i >> 1) - 1) & 1, abort_flag, g.status))) break;
        tc_fence_after();
        const uint64_t q = dStage + s * kSt16, o = q + kQ16;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint64_t ka = (kk >> 2) * 1024 + (kk & 3) * 2, kb = (kk >> 2) * 512 + (kk & 3) * 2;
          tc_mma_bf16(tbase + 128 * b, dKb + ka, q + kb, C::kIdescS, kk > 0 ? 1u : 0u);
          tc_mma_bf16(tbase + 128 * b + 64, dVs + ka, o + kb, C::kIdescS, kk > 0 ? 1u : 0u);
        }
        tc_commit(&s_full[b]);
      }
      tc_commit(drain_s);
      drain_wait(drain_s, 0);
    }
    __syncwarp();
  } else if (warp == kWarpAcc) {
    // ---------------------------------------------------------- accumulation issuer
    // dVsum_t += Pi^T dO and dKbar_t += dA^T Q of every step once its Pi^T and
    // dA^T are written; `done` completes after the last (the elementwise
    // warps saw every step's scores complete before writing its Pi^T, dA^T)
    if (lane == 0) {
      // the q / dO tiles as MN-major B operands: N = D (atoms of 64 features 8 KB apart)
      const uint64_t dStageMN = sdesc_sw128(smem_u32(smem + C::kOffStage), 8192, 1024);
      const uint64_t dPi = sdesc_sw128(smem_u32(sPi), 16, 1024);
      const uint64_t dDa = sdesc_sw128(smem_u32(sDa), 16, 1024);
      constexpr uint64_t kSt16 = C::kStage >> 4, kQ16 = C::kQ >> 4;
      bool ok = true;
      for (int j = 0; ok && j < n; ++j) {
        const int sj = j & 1;
        if (!(ok = mbar_wait(pd_full, j & 1, abort_flag, g.status))) break;
        tc_fence_after();
        const uint64_t q = dStageMN + sj * kSt16, o = q + kQ16;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {  // K = 64 queries
          const uint32_t acc = (j > 0 || kk > 0) ? 1u : 0u;
          tc_mma_bf16(t_acc_vs, dPi + kk * 2, o + 128 * kk, C::kIdescAcc, acc);
          tc_mma_bf16(t_acc_kb, dDa + kk * 2, q + 128 * kk, C::kIdescAcc, acc);
        }
        tc_commit(pd_free);
        tc_commit(&stage_free[sj]);
      }
      tc_commit(done);
      drain_wait(done, 0);
    }
    __syncwarp();
  } else if (warp < 8) {
    // ------------------------------------------------------------ elementwise
    const int quarter = warp & 3, half = warp >> 2;
    const int j = quarter * 32 + lane;       // TMEM lane = pooled key of the tile
    const int c0 = 32 * half;                // this thread's 32 query columns
    const int J = tile * 128 + j;
    const uint32_t lane_addr = static_cast<uint32_t>(quarter * 32) << 16;
    for (int i = 0; i < n; ++i) {
      const int s = i & 1, b = i & 1;
      const int I = start + i;
      const int pcand = g.causal ? I : g.M;
      const bool valid = J < pcand && !listed(g, bh, I, J);
      mbar_wait(&full[s], (i >> 1) & 1, abort_flag, g.status);
      mbar_wait(&s_full[b], (i >> 1) & 1, abort_flag, g.status);
      tc_fence_after();
      float sv[32], dp[32];
      tmem_ld32(tbase + lane_addr + 128 * b + c0, sv);
      tmem_ld32(tbase + lane_addr + 128 * b + 64 + c0, dp);
      tc_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&s_empty[b]);
      const float* nl = reinterpret_cast<const float*>(smem + C::kOffStage + s * C::kStage + 2 * C::kQ) + c0;
      const float* dl = nl + 64;
      uint32_t pi[16], da[16];
#pragma unroll
      for (int q = 0; q < 32; q += 2) {
        float e0 = valid ? ex2_approx(fmaf(sv[q], g.sl, nl[q])) : 0.f;
        float e1 = valid ? ex2_approx(fmaf(sv[q + 1], g.sl, nl[q + 1])) : 0.f;
        pi[q / 2] = pack_bf16x2(e0, e1);
        da[q / 2] = pack_bf16x2(e0 * (dp[q] - 64.f * dl[q]), e1 * (dp[q + 1] - 64.f * dl[q + 1]));
      }
      if (i >= 1) mbar_wait(pd_free, (i - 1) & 1, abort_flag, g.status);
      store_half_row(sPi, j, half, pi);
      store_half_row(sDa, j, half, da);
      fence_async_shared();
      __syncwarp();
      if (lane == 0) mbar_arrive(pd_full);
    }
    // partial sums of this item: row j of the tile, D features
    const bool ok = n == 0 || mbar_wait(done, 0, abort_flag, g.status);
    tc_fence_after();
    float* dvs = part_dvs + (static_cast<size_t>(item) * 128 + j) * D;
    float* dkb = part_dkb + (static_cast<size_t>(item) * 128 + j) * D;
#pragma unroll 1
    for (int c = half * (D / 64); c < (half + 1) * (D / 64); ++c) {  // this half's D/2 features
      float a[32], k[32];
      if (n > 0 && ok) {
        tmem_ld32(t_acc_vs + lane_addr + 32 * c, a);
        tmem_ld32(t_acc_kb + lane_addr + 32 * c, k);
        tc_wait_ld();
      } else {
#pragma unroll
        for (int e = 0; e < 32; ++e) a[e] = k[e] = 0.f;
      }
#pragma unroll
      for (int e = 0; e < 32; e += 4) {
        *reinterpret_cast<float4*>(dvs + 32 * c + e) = make_float4(a[e], a[e + 1], a[e + 2], a[e + 3]);
        *reinterpret_cast<float4*>(dkb + 32 * c + e) =
            make_float4(g.tau * k[e], g.tau * k[e + 1], g.tau * k[e + 2], g.tau * k[e + 3]);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == kWarpMma) {
    tc_fence_after();
    tmem_dealloc(tbase, 512);
  }
}

// dvsum / dkbar [BH][M][D] = sum over the chunks of the items' partials, in
// chunk order.
__global__ void __launch_bounds__(256) bwd_pseudo_reduce_kernel(const float* __restrict__ part_dvs,
                                                                const float* __restrict__ part_dkb, int M, int D,
                                                                int tiles, int chunks, float* __restrict__ dvsum,
                                                                float* __restrict__ dkbar) {
  const int bh = blockIdx.y;
  const long long e = blockIdx.x * 256LL + threadIdx.x;  // (J, f) of this head
  if (e >= static_cast<long long>(M) * D) return;
  const int J = static_cast<int>(e / D), f = static_cast<int>(e % D);
  const int tile = J / 128, r = J % 128;
  float a = 0.f, k = 0.f;
  for (int c = 0; c < chunks; ++c) {
    const size_t o = ((static_cast<size_t>((bh * tiles + tile) * chunks + c)) * 128 + r) * D + f;
    a += part_dvs[o];
    k += part_dkb[o];
  }
  const size_t o = (static_cast<size_t>(bh) * M + J) * D + f;
  dvsum[o] = a;
  dkbar[o] = k;
}

// ------------------------------------------------------------------ dq
// A unit is one query block: its steps are the forward's tile stream (pooled
// tiles of 128 unlisted candidates, then pairs of listed blocks).  The key
// rows of a step stay in shared memory until dq^T += K^T dS^T has read them,
// after the elementwise work, so they get a 3-slot ring; the value rows are
// free once dP^T is issued (2 slots); q and dO of a unit have one stage
// (released when its last S^T / dP^T is done) and its -lse log2e and D two
// small slots (released by the elementwise warps).  The MMA warp issues
// whichever of "scores of the next step" and "dq of the oldest step" is ready.
template <int D>
struct DqCfg {
  static constexpr int kQ = 64 * D * 2;
  static constexpr int kTile = 128 * D * 2;  // 128 key (or value) rows
  static constexpr int kKSlots = 3, kVSlots = 2;
  static constexpr int kOffK = 2 * kQ;                     // q, dO at 0, kQ
  static constexpr int kOffV = kOffK + kKSlots * kTile;
  static constexpr int kOffDs = kOffV + kVSlots * kTile;
  static constexpr int kOffNl = kOffDs + 128 * 128;         // [2][-lse log2e 64, D 64]
  static constexpr int kOffBars = kOffNl + 2 * 512;
  static constexpr int kSmem = kOffBars + 512 + 1024;  // 512 B: barriers, TMEM slot, unit ring
  static_assert(kSmem <= 232448, "shared memory of one CTA");
  static constexpr uint32_t kIdescS = idesc_bf16_f32(128, 64, 0, 0);
  // dq^T [D x 64 q] += K^T (A: M = features, MN-major) . dS^T (B: N = q, MN-major)
  static constexpr uint32_t kIdescAcc = idesc_bf16_f32(128, 64, 1, 1);
};

struct DqUnit {
  int bh, I, rp, nsel, cand, pcand, n_a2, n_e, ntiles;
};

__device__ __forceinline__ DqUnit dq_unit(int u, const BwdArgs& g) {
  DqUnit x;
  x.bh = u / g.M;
  x.I = u - x.bh * g.M;
  const int row = u;
  x.cand = g.causal ? x.I + 1 : g.M;
  x.pcand = g.causal ? x.I : g.M;
  const int a = __ldg(g.row_ptr + row), b = __ldg(g.row_ptr + row + 1);
  if (a < 0 || b < a || static_cast<long long>(b) > g.col_cap || b - a > x.cand) {
    x.rp = 0;
    x.nsel = 0;
  } else {
    x.rp = a;
    x.nsel = b - a;
  }
  x.n_a2 = (x.pcand > 0 && x.nsel < x.cand) ? (x.pcand + 127) / 128 : 0;
  x.n_e = (x.nsel + 1) / 2;
  if (x.n_a2 + x.n_e == 0) x.n_e = 1;  // one (empty) product keeps dq defined
  x.ntiles = x.n_a2 + x.n_e;
  return x;
}

template <int D>
__global__ void __launch_bounds__(kBwdThreads, 1)
    bwd_dq_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmDO,
                  const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                  const __grid_constant__ CUtensorMap tmKb, const __grid_constant__ CUtensorMap tmVs,
                  const BwdArgs g, __nv_bfloat16* __restrict__ dq) {
  using C = DqCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sDs = smem + C::kOffDs;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kOffBars);
  uint64_t* u_full = bars + 0;     // [2] by unit parity: q, dO, -lse log2e, D landed
  uint64_t* u_free = bars + 2;     // q, dO stage: the unit's last S^T / dP^T done
  uint64_t* nl_free = bars + 3;    // [2] -lse log2e, D slot read by the 8 elementwise warps
  uint64_t* k_full = bars + 5;     // [3] key rows of a step landed
  uint64_t* k_free = bars + 8;     // [3] the step's dq MMA is done
  uint64_t* v_full = bars + 11;    // [2] value rows landed
  uint64_t* v_free = bars + 13;    // [2] the step's dP^T is done
  uint64_t* s_full = bars + 15;    // [2] S^T, dP^T ready
  uint64_t* s_empty = bars + 17;   // [2] read by the 8 elementwise warps
  uint64_t* ds_full = bars + 19;   // dS^T written (8 warps)
  uint64_t* ds_free = bars + 20;   // its MMA is done
  uint64_t* dq_full = bars + 21;   // [2] a unit's dq^T is complete
  uint64_t* dq_empty = bars + 23;  // [2] read by the 8 elementwise warps
  uint64_t* drain = bars + 25;     // [2] teardown of the two issuers
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 27);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  volatile int* uring = reinterpret_cast<volatile int*>(bars + 28);  // [4] unit ids in flight
  uint64_t* id_full = bars + 30;   // [4] a unit id published (producer)
  uint64_t* id_empty = bars + 34;  // [4] read by its 10 consumers (both issuers, 8 elementwise warps)

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int units = g.BH * g.M;
  // Dynamic unit scheduler, as in the forward: a CTA's first unit comes from
  // blockIdx.x, each later one from the next ticket of the call's counter;
  // ticket t is query block M - 1 - t % M of head t / M (largest first, so
  // long causal units start early).  The producer publishes the CTA's ul-th
  // unit in slot ul % 4; the other roles read the slots in order; -1 ends.
  auto publish = [&](int ul) -> int {
    int t;
    if (ul == 0) {
      t = static_cast<int>(blockIdx.x) < units ? static_cast<int>(blockIdx.x) : -1;
    } else {
      t = static_cast<int>(gridDim.x) + atomicAdd(g.sched + 1, 1);
      if (t >= units) t = -1;
    }
    const int u = t < 0 ? -1 : (t / g.M) * g.M + g.M - 1 - t % g.M;
    const int slot = ul & 3;
    if (ul >= 4 && !mbar_wait(&id_empty[slot], ((ul >> 2) - 1) & 1, abort_flag, g.status)) return -1;
    uring[slot] = u;
    mbar_arrive(&id_full[slot]);
    return u;
  };
  auto fetch = [&](int ul) -> int {  // by lane 0 of a consuming warp
    const int slot = ul & 3;
    if (!mbar_wait(&id_full[slot], (ul >> 2) & 1, abort_flag, g.status)) return -1;
    const int u = uring[slot];
    mbar_arrive(&id_empty[slot]);
    return u;
  };
  if (threadIdx.x == 0) {
    for (int i = 0; i < 4; ++i) {
      mbar_init(&id_full[i], 1);
      mbar_init(&id_empty[i], 10);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&u_full[i], 1);
      mbar_init(&nl_free[i], 8);
      mbar_init(&v_full[i], 1);
      mbar_init(&v_free[i], 1);
      mbar_init(&s_full[i], 1);
      mbar_init(&s_empty[i], 8);
      mbar_init(&dq_full[i], 1);
      mbar_init(&dq_empty[i], 8);
    }
    for (int i = 0; i < 3; ++i) {
      mbar_init(&k_full[i], 1);
      mbar_init(&k_free[i], 1);
    }
    mbar_init(u_free, 1);
    mbar_init(ds_full, 8);
    mbar_init(ds_free, 1);
    mbar_init(&drain[0], 1);
    mbar_init(&drain[1], 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == kWarpMma) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tmem_slot;

  if (warp == kWarpTma) {
    // ---------------------------------------------------------- producer
    if (lane == 0) {
      int si = 0;
      int k_iss[3] = {0, 0, 0}, v_iss[2] = {0, 0}, u_iss[2] = {0, 0};
      bool ok = true;
      for (int ul = 0; ok; ++ul) {
        const int u = publish(ul);
        if (u < 0) break;
        const DqUnit x = dq_unit(u, g);
        const int ub = ul & 1;
        // q, dO stage: the previous unit's scores are done; its -lse / D slot: read
        if (ul >= 1 && !(ok = mbar_wait(u_free, (ul - 1) & 1, abort_flag, g.status))) break;
        if (ul >= 2 && !(ok = mbar_wait(&nl_free[ub], ((ul >> 1) - 1) & 1, abort_flag, g.status))) break;
        mbar_arrive_expect_tx(&u_full[ub], 2 * C::kQ + 512);
#pragma unroll
        for (int c = 0; c < D / 64; ++c) {
          tma_load_3d(&tmQ, smem + c * 8192, &u_full[ub], 64 * c, 64 * x.I, x.bh);
          tma_load_3d(&tmDO, smem + C::kQ + c * 8192, &u_full[ub], 64 * c, 64 * x.I, x.bh);
        }
        const size_t r0 = static_cast<size_t>(x.bh) * g.N + 64 * x.I;
        bulk_load(smem + C::kOffNl + ub * 512, g.nlse2 + r0, 256, &u_full[ub]);
        bulk_load(smem + C::kOffNl + ub * 512 + 256, g.delta + r0, 256, &u_full[ub]);
        ++u_iss[ub];
        for (int t = 0; ok && t < x.ntiles; ++t, ++si) {
          const CUtensorMap *mk, *mv;
          int y0, y1;
          if (t < x.n_a2) {
            mk = &tmKb;
            mv = &tmVs;
            y0 = 128 * t;
            y1 = y0 + 64;
          } else {
            mk = &tmK;
            mv = &tmV;
            const int e2 = 2 * (t - x.n_a2);
            int j1 = e2 < x.nsel ? __ldg(g.col_idx + x.rp + e2) : 0;
            int j2 = e2 + 1 < x.nsel ? __ldg(g.col_idx + x.rp + e2 + 1) : j1;
            j1 = min(max(j1, 0), g.M - 1);
            j2 = min(max(j2, 0), g.M - 1);
            y0 = 64 * j1;
            y1 = 64 * j2;
          }
          const int ks = si % 3, vs = si & 1;
          if (si >= 3 && !(ok = mbar_wait(&k_free[ks], ((si / 3) - 1) & 1, abort_flag, g.status))) break;
          uint8_t* kd = smem + C::kOffK + ks * C::kTile;
          mbar_arrive_expect_tx(&k_full[ks], C::kTile);
#pragma unroll
          for (int c = 0; c < D / 64; ++c) {
            tma_load_3d(mk, kd + c * 16384, &k_full[ks], 64 * c, y0, x.bh);
            tma_load_3d(mk, kd + c * 16384 + 8192, &k_full[ks], 64 * c, y1, x.bh);
          }
          ++k_iss[ks];
          if (si >= 2 && !(ok = mbar_wait(&v_free[vs], ((si >> 1) - 1) & 1, abort_flag, g.status))) break;
          uint8_t* vd = smem + C::kOffV + vs * C::kTile;
          mbar_arrive_expect_tx(&v_full[vs], C::kTile);
#pragma unroll
          for (int c = 0; c < D / 64; ++c) {
            tma_load_3d(mv, vd + c * 16384, &v_full[vs], 64 * c, y0, x.bh);
            tma_load_3d(mv, vd + c * 16384 + 8192, &v_full[vs], 64 * c, y1, x.bh);
          }
          ++v_iss[vs];
        }
      }
      for (int b = 0; b < 3; ++b)
        if (k_iss[b]) drain_wait(&k_full[b], (k_iss[b] - 1) & 1);
      for (int b = 0; b < 2; ++b) {
        if (v_iss[b]) drain_wait(&v_full[b], (v_iss[b] - 1) & 1);
        if (u_iss[b]) drain_wait(&u_full[b], (u_iss[b] - 1) & 1);
      }
    }
    __syncwarp();
  } else if (warp == kWarpMma) {
    // ---------------------------------------------------------- scores issuer
    // S^T = K_t Q^T and dP^T = V_t dO^T of every step, in order
    if (lane == 0) {
      const uint64_t dQ = sdesc_sw128(smem_u32(smem), 16, 1024);
      const uint64_t dO = sdesc_sw128(smem_u32(smem + C::kQ), 16, 1024);
      const uint64_t dK = sdesc_sw128(smem_u32(smem + C::kOffK), 16, 1024);
      const uint64_t dV = sdesc_sw128(smem_u32(smem + C::kOffV), 16, 1024);
      constexpr uint64_t kT16 = C::kTile >> 4;
      int si = 0;
      bool ok = true;
      for (int ul = 0; ok; ++ul) {
        const int u = fetch(ul);
        if (u < 0) break;
        const DqUnit x = dq_unit(u, g);
        const int ub = ul & 1;
        if (!(ok = mbar_wait(&u_full[ub], (ul >> 1) & 1, abort_flag, g.status))) break;
        for (int t = 0; t < x.ntiles; ++t, ++si) {
          const int ks = si % 3, vs = si & 1, b = si & 1;
          if (!(ok = mbar_wait(&k_full[ks], (si / 3) & 1, abort_flag, g.status))) break;
          if (!(ok = mbar_wait(&v_full[vs], (si >> 1) & 1, abort_flag, g.status))) break;
          if (si >= 2 && !(ok = mbar_wait(&s_empty[b], ((si >> 1) - 1) & 1, abort_flag, g.status))) break;
          tc_fence_after();
          const uint64_t kt = dK + ks * kT16, vt = dV + vs * kT16;
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint64_t ka = (kk >> 2) * 1024 + (kk & 3) * 2, kb = (kk >> 2) * 512 + (kk & 3) * 2;
            tc_mma_bf16(tbase + 128 * b, kt + ka, dQ + kb, C::kIdescS, kk > 0 ? 1u : 0u);
            tc_mma_bf16(tbase + 128 * b + 64, vt + ka, dO + kb, C::kIdescS, kk > 0 ? 1u : 0u);
          }
          tc_commit(&s_full[b]);
          tc_commit(&v_free[vs]);
          if (t == x.ntiles - 1) tc_commit(u_free);
        }
      }
      tc_commit(&drain[0]);
      drain_wait(&drain[0], 0);
    }
    __syncwarp();
  } else if (warp == kWarpAcc) {
    // ---------------------------------------------------------- dq issuer
    // dq^T += K_t^T dS^T of every step, in order, once its dS^T is written (a
    // unit's first step also once the epilogue of the unit two before has read
    // the dq^T buffer it overwrites); each frees the dS^T tile and the key slot
    if (lane == 0) {
      // key rows as the MN-major A of dq^T: M = features (64-feature atoms 16 KB apart)
      const uint64_t dKmn = sdesc_sw128(smem_u32(smem + C::kOffK), D == 128 ? 16384 : 0, 1024);
      const uint64_t dDs = sdesc_sw128(smem_u32(sDs), 16, 1024);
      constexpr uint64_t kT16 = C::kTile >> 4;
      int si = 0;
      bool ok = true;
      for (int ul = 0; ok; ++ul) {
        const int u = fetch(ul);
        if (u < 0) break;
        const DqUnit x = dq_unit(u, g);
        const int ub = ul & 1;
        for (int t = 0; t < x.ntiles; ++t, ++si) {
          if (!(ok = mbar_wait(ds_full, si & 1, abort_flag, g.status))) break;
          if (t == 0 && ul >= 2 && !(ok = mbar_wait(&dq_empty[ub], ((ul >> 1) - 1) & 1, abort_flag, g.status))) break;
          tc_fence_after();
          const uint32_t t_dq = tbase + 256 + 64 * ub;
          const uint64_t a = dKmn + (si % 3) * kT16;
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)  // K = 128 key rows
            tc_mma_bf16(t_dq, a + 128 * kk, dDs + 128 * kk, C::kIdescAcc, (t > 0 || kk > 0) ? 1u : 0u);
          tc_commit(ds_free);
          tc_commit(&k_free[si % 3]);
          if (t == x.ntiles - 1) tc_commit(&dq_full[ub]);
        }
      }
      tc_commit(&drain[1]);
      drain_wait(&drain[1], 0);
    }
    __syncwarp();
  } else if (warp < 8) {
    // ------------------------------------------------------------ elementwise
    const int quarter = warp & 3, half = warp >> 2;
    const int r = quarter * 32 + lane;  // TMEM lane: key row of S^T, feature row of dq^T
    const int c0 = 32 * half;           // this thread's 32 query columns
    const uint32_t lane_addr = static_cast<uint32_t>(quarter * 32) << 16;
    int sc = 0;
    for (int ul = 0;; ++ul) {
      int u = -1;
      if (lane == 0) u = fetch(ul);
      u = __shfl_sync(0xffffffffu, u, 0);
      if (u < 0) break;
      const DqUnit x = dq_unit(u, g);
      const int ub = ul & 1;
      if (!mbar_wait(&u_full[ub], (ul >> 1) & 1, abort_flag, g.status)) break;
      const float* nl = reinterpret_cast<const float*>(smem + C::kOffNl + ub * 512);
      const float* dl = nl + 64;
      bool stop = false;
      // what decides this thread's row of step t: the listed-block bitmap word
      // (pooled tile) or the listed block (exact tile); loaded a step ahead so
      // the load's latency stays off the step's critical path
      auto fetch_row = [&](int t) -> int {
        if (t < x.n_a2) {
          const int J = 128 * t + r;
          return J < x.pcand ? static_cast<int>(__ldg(g.bits + (static_cast<size_t>(x.bh) * g.M + x.I) * g.nw +
                                                      (J >> 5)))
                             : -1;
        }
        const int idx = 2 * (t - x.n_a2) + (r >> 6);
        return idx < x.nsel ? __ldg(g.col_idx + x.rp + idx) : -1;
      };
      int next_row = fetch_row(0);
      for (int t = 0; t < x.ntiles; ++t, ++sc) {
        const int b = sc & 1;
        const bool pooled = t < x.n_a2;
        const int cur_row = next_row;
        if (t + 1 < x.ntiles) next_row = fetch_row(t + 1);
        bool valid, diag = false;
        if (pooled) {
          const int J = 128 * t + r;
          valid = J < x.pcand && !((static_cast<uint32_t>(cur_row) >> (J & 31)) & 1u);
        } else {
          const int J = cur_row;
          valid = J >= 0 && J < x.cand;
          diag = g.causal && J == x.I;
        }
        if (!mbar_wait(&s_full[b], (sc >> 1) & 1, abort_flag, g.status)) {
          stop = true;
          break;
        }
        tc_fence_after();
        float sv[32], dp[32];
        tmem_ld32(tbase + lane_addr + 128 * b + c0, sv);
        tmem_ld32(tbase + lane_addr + 128 * b + 64 + c0, dp);
        tc_wait_ld();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&s_empty[b]);
        const float wD = pooled ? 64.f : 1.f;
        const int kj = r & 63;
        uint32_t ds[16];
#pragma unroll
        for (int q = 0; q < 32; q += 2) {
          const int qq = c0 + q;
          float e0 = valid ? ex2_approx(fmaf(sv[q], g.sl, nl[qq])) : 0.f;
          float e1 = valid ? ex2_approx(fmaf(sv[q + 1], g.sl, nl[qq + 1])) : 0.f;
          if (diag) {
            e0 = kj <= qq ? e0 : 0.f;
            e1 = kj <= qq + 1 ? e1 : 0.f;
          }
          ds[q / 2] = pack_bf16x2(e0 * (dp[q] - wD * dl[qq]), e1 * (dp[q + 1] - wD * dl[qq + 1]));
        }
        if (sc >= 1) mbar_wait(ds_free, (sc - 1) & 1, abort_flag, g.status);
        store_half_row(sDs, r, half, ds);
        fence_async_shared();
        __syncwarp();
        if (lane == 0) mbar_arrive(ds_full);
      }
      if (stop) break;
      __syncwarp();
      if (lane == 0) mbar_arrive(&nl_free[ub]);  // this unit's -lse / D slot is read
      // dq of the unit: feature row r, this thread's 32 query columns
      if (!mbar_wait(&dq_full[ub], (ul >> 1) & 1, abort_flag, g.status)) break;
      tc_fence_after();
      if (r < D) {  // warp-uniform
        __nv_bfloat16* dst = dq + (static_cast<size_t>(x.bh) * g.N + 64 * x.I + c0) * D + r;
        float v[32];
        tmem_ld32(tbase + lane_addr + 256 + 64 * ub + c0, v);
        tc_wait_ld();
#pragma unroll
        for (int q = 0; q < 32; ++q) dst[static_cast<size_t>(q) * D] = __float2bfloat16_rn(g.tau * v[q]);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&dq_empty[ub]);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == kWarpMma) {
    tc_fence_after();
    tmem_dealloc(tbase, 512);
  }
}

// ------------------------------------------------------------------ dk, dv
template <int D>
struct KvCfg {
  static constexpr int kBlk = 64 * D * 2;          // one 64-row block of K or V
  static constexpr int kPair = 128 * D * 2;        // two query blocks of q or dO
  static constexpr int kStage = (2 * kPair + 1024 + 64 + 1023) / 1024 * 1024;  // q, dO, -lse log2e [128], D [128], meta
  static constexpr int kOffStage = 2 * kBlk;
  static constexpr int kOffP = kOffStage + 2 * kStage;
  static constexpr int kOffDs = kOffP + 128 * 128;
  static constexpr int kOffBal = kOffDs + 128 * 128;            // ballots of the listing scan [M / 32]
  static constexpr int kOffBars = kOffBal + kMaxBlocks / 8;
  static constexpr int kSmem = kOffBars + 256 + 1024;
  static_assert(kSmem <= 232448, "shared memory of one CTA");
  static constexpr uint32_t kIdescS = idesc_bf16_f32(128, 64, 0, 0);    // [128 q x 64 keys]
  static constexpr uint32_t kIdescAcc = idesc_bf16_f32(128, 64, 1, 1);  // [D x 64 keys] += [D x 128 q] . [128 q x 64]
};

struct KvMeta {
  int Ia, Ib, last, pad;
};

template <int D>
__global__ void __launch_bounds__(kBwdThreads, 1)
    bwd_dkdv_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmDO,
                    const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                    const BwdArgs g, const float* __restrict__ dkbar, const float* __restrict__ dvsum,
                    __nv_bfloat16* __restrict__ dk, __nv_bfloat16* __restrict__ dv) {
  using C = KvCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sK = smem;
  uint8_t* sV = smem + C::kBlk;
  uint8_t* sP = smem + C::kOffP;
  uint8_t* sDs = smem + C::kOffDs;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kOffBars);
  uint64_t* item_full = bars + 0;   // K_J, V_J landed
  uint64_t* item_free = bars + 1;   // every MMA of the item is done
  uint64_t* full = bars + 2;        // [2] a step's rows landed (or an empty step posted)
  uint64_t* stage_free = bars + 4;  // [2] the step's MMAs are done
  uint64_t* s_full = bars + 6;      // [2]
  uint64_t* s_empty = bars + 8;     // [2] (4 warps)
  uint64_t* pd_full = bars + 10;    // P, dS written (4 warps)
  uint64_t* pd_free = bars + 11;
  uint64_t* acc_full = bars + 12;   // dK^T, dV^T of the item complete
  uint64_t* acc_empty = bars + 13;  // read by the 4 warps
  uint64_t* drain = bars + 14;     // [2] teardown of the two issuers
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 16);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  volatile int* iring = reinterpret_cast<volatile int*>(bars + 17);  // [4] item ids in flight
  uint64_t* id_full = bars + 19;    // [4] an item id published (producer)
  uint64_t* id_empty = bars + 23;   // [4] read by its 10 consumers (both issuers, 8 elementwise warps)

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int items = g.BH * g.M;
  // Dynamic item scheduler: a CTA's first item is blockIdx.x, each later one
  // the next ticket of the call's counter (after the grid's first items), so
  // CTAs that drew key blocks listed by few query blocks take more of them.
  // The producer draws and publishes the CTA's il-th item in slot il % 4;
  // every other role reads the slots in order; -1 ends the sequence.
  auto publish = [&](int il) -> int {
    int it;
    if (il == 0) {
      it = static_cast<int>(blockIdx.x) < items ? static_cast<int>(blockIdx.x) : -1;
    } else {
      it = static_cast<int>(gridDim.x) + atomicAdd(g.sched, 1);
      if (it >= items) it = -1;
    }
    const int slot = il & 3;
    if (il >= 4 && !mbar_wait(&id_empty[slot], ((il >> 2) - 1) & 1, abort_flag, g.status)) return -1;
    iring[slot] = it;
    mbar_arrive(&id_full[slot]);
    return it;
  };
  auto fetch = [&](int il) -> int {  // by lane 0 of a consuming warp
    const int slot = il & 3;
    if (!mbar_wait(&id_full[slot], (il >> 2) & 1, abort_flag, g.status)) return -1;
    const int it = iring[slot];
    mbar_arrive(&id_empty[slot]);
    return it;
  };
  if (threadIdx.x == 0) {
    for (int i = 0; i < 4; ++i) {
      mbar_init(&id_full[i], 1);
      mbar_init(&id_empty[i], 10);
    }
    mbar_init(item_full, 1);
    mbar_init(item_free, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&stage_free[i], 1);
      mbar_init(&s_full[i], 1);
      mbar_init(&s_empty[i], 8);
    }
    mbar_init(pd_full, 8);
    mbar_init(pd_free, 1);
    mbar_init(acc_full, 1);
    mbar_init(acc_empty, 8);
    mbar_init(&drain[0], 1);
    mbar_init(&drain[1], 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == kWarpMma) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tmem_slot;
  const uint32_t t_dk = tbase + 256, t_dv = tbase + 320;
  auto stage = [&](int s) { return smem + C::kOffStage + s * C::kStage; };
  auto meta = [&](int s) { return reinterpret_cast<volatile KvMeta*>(stage(s) + 2 * C::kPair + 1024); };

  if (warp == kWarpTma) {
    // ---------------------------------------------------------- producer
    // the query blocks that list key block J, in pairs
    int sc = 0;
    int st_issued[2] = {0, 0}, it_issued = 0;
    bool ok = true;
    for (int il = 0; ok; ++il) {
      int it = -1;
      if (lane == 0) it = publish(il);
      it = __shfl_sync(0xffffffffu, it, 0);
      if (it < 0) break;
      const int bh = it / g.M, J = it - bh * g.M;
      if (lane == 0) {
        if (il >= 1) ok = mbar_wait(item_free, (il - 1) & 1, abort_flag, g.status);
        if (ok) {
          mbar_arrive_expect_tx(item_full, 2 * C::kBlk);
#pragma unroll
          for (int c = 0; c < D / 64; ++c) {
            tma_load_3d(&tmK, sK + c * 8192, item_full, 64 * c, 64 * J, bh);
            tma_load_3d(&tmV, sV + c * 8192, item_full, 64 * c, 64 * J, bh);
          }
          ++it_issued;
        }
      }
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) break;
      // the rows that list J: one ballot per 32 rows, eight independent bitmap
      // loads per lane in flight, the ballots kept in shared memory
      const int I0 = g.causal ? J : 0;
      const int ngroups = (g.M - I0 + 31) / 32;
      uint32_t* bal = reinterpret_cast<uint32_t*>(smem + C::kOffBal);
      int cnt = 0;
      for (int g0 = 0; g0 < ngroups; g0 += 8) {
        bool on[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const int I = I0 + 32 * (g0 + u) + lane;
          on[u] = g0 + u < ngroups && I < g.M && listed(g, bh, I, J);
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const uint32_t w = __ballot_sync(0xffffffffu, on[u]);
          if (g0 + u < ngroups) {
            if (lane == 0) bal[g0 + u] = w;
            cnt += __popc(w);
          }
        }
      }
      __syncwarp();
      const int nsteps = cnt == 0 ? 1 : (cnt + 1) / 2;
      int k = 0, pending = -1;
      auto emit = [&](int Ia, int Ib) {
        if (lane == 0 && ok) {
          const int s = sc & 1;
          if (sc >= 2) ok = mbar_wait(&stage_free[s], ((sc >> 1) - 1) & 1, abort_flag, g.status);
          if (ok) {
            volatile KvMeta* m = meta(s);
            m->Ia = Ia;
            m->Ib = Ib;
            m->last = k == nsteps - 1;
            if (Ia >= 0) {
              const int ib = Ib >= 0 ? Ib : Ia;  // a missing second block repeats the first (masked)
              uint8_t* st = stage(s);
              mbar_arrive_expect_tx(&full[s], 2 * C::kPair + 1024);
#pragma unroll
              for (int c = 0; c < D / 64; ++c) {
                tma_load_3d(&tmQ, st + c * 16384, &full[s], 64 * c, 64 * Ia, bh);
                tma_load_3d(&tmQ, st + c * 16384 + 8192, &full[s], 64 * c, 64 * ib, bh);
                tma_load_3d(&tmDO, st + C::kPair + c * 16384, &full[s], 64 * c, 64 * Ia, bh);
                tma_load_3d(&tmDO, st + C::kPair + c * 16384 + 8192, &full[s], 64 * c, 64 * ib, bh);
              }
              const size_t ra = static_cast<size_t>(bh) * g.N + 64 * Ia, rb = static_cast<size_t>(bh) * g.N + 64 * ib;
              bulk_load(st + 2 * C::kPair, g.nlse2 + ra, 256, &full[s]);
              bulk_load(st + 2 * C::kPair + 256, g.nlse2 + rb, 256, &full[s]);
              bulk_load(st + 2 * C::kPair + 512, g.delta + ra, 256, &full[s]);
              bulk_load(st + 2 * C::kPair + 768, g.delta + rb, 256, &full[s]);
            } else {
              mbar_arrive(&full[s]);
            }
            ++st_issued[s];
          }
        }
        ++sc;
        ++k;
      };
      for (int gi = 0; gi < ngroups; ++gi) {
        uint32_t m = bal[gi];
        while (m) {
          const int l = __ffs(m) - 1;
          m &= m - 1;
          const int I = I0 + 32 * gi + l;
          if (pending < 0) {
            pending = I;
          } else {
            emit(pending, I);
            pending = -1;
          }
        }
      }
      __syncwarp();
      if (pending >= 0) emit(pending, -1);
      if (cnt == 0) emit(-1, -1);
      ok = __shfl_sync(0xffffffffu, ok, 0);
    }
    if (lane == 0) {
      if (it_issued) drain_wait(item_full, (it_issued - 1) & 1);
      for (int b = 0; b < 2; ++b)
        if (st_issued[b]) drain_wait(&full[b], (st_issued[b] - 1) & 1);
    }
    __syncwarp();
  } else if (warp == kWarpMma) {
    // ---------------------------------------------------------- scores issuer
    // S = Q_p K_J^T and dP = dO_p V_J^T of every step, in order: a step's
    // rows landed and its S / dP buffer read by the elementwise warps.
    if (lane == 0) {
      const uint64_t dK = sdesc_sw128(smem_u32(sK), 16, 1024);
      const uint64_t dV = sdesc_sw128(smem_u32(sV), 16, 1024);
      const uint64_t dSt = sdesc_sw128(smem_u32(stage(0)), 16, 1024);
      constexpr uint64_t kSt16 = C::kStage >> 4, kPair16 = C::kPair >> 4;
      int sc = 0;
      bool ok = true;
      for (int il = 0; ok; ++il) {
        if (fetch(il) < 0) break;
        if (!(ok = mbar_wait(item_full, il & 1, abort_flag, g.status))) break;
        for (;;) {
          const int s = sc & 1, b = sc & 1;
          if (!(ok = mbar_wait(&full[s], (sc >> 1) & 1, abort_flag, g.status))) break;
          if (sc >= 2 && !(ok = mbar_wait(&s_empty[b], ((sc >> 1) - 1) & 1, abort_flag, g.status))) break;
          volatile KvMeta* m = meta(s);
          const bool has = m->Ia >= 0;
          const bool last = m->last != 0;
          tc_fence_after();
          if (has) {
            const uint64_t q = dSt + s * kSt16, o = q + kPair16;
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
              const uint64_t ka = (kk >> 2) * 1024 + (kk & 3) * 2, kb = (kk >> 2) * 512 + (kk & 3) * 2;
              tc_mma_bf16(tbase + 128 * b, q + ka, dK + kb, C::kIdescS, kk > 0 ? 1u : 0u);
              tc_mma_bf16(tbase + 128 * b + 64, o + ka, dV + kb, C::kIdescS, kk > 0 ? 1u : 0u);
            }
          }
          tc_commit(&s_full[b]);
          ++sc;
          if (last) break;
        }
      }
      tc_commit(&drain[0]);
      drain_wait(&drain[0], 0);
    }
    __syncwarp();
  } else if (warp == kWarpAcc) {
    // ---------------------------------------------------------- accumulation issuer
    // dV^T += dO_p^T P and dK^T += Q_p^T dS of every step, in order, once its P
    // and dS are written (and, for an item's first step, once the epilogue has
    // read the previous item's accumulators); each frees the step's stage and
    // the P / dS tiles, and the item's last frees K_J, V_J and completes the item.
    if (lane == 0) {
      const uint64_t dStMN = sdesc_sw128(smem_u32(stage(0)), D == 128 ? 16384 : 0, 1024);
      const uint64_t dP = sdesc_sw128(smem_u32(sP), 16, 1024);
      const uint64_t dDs = sdesc_sw128(smem_u32(sDs), 16, 1024);
      constexpr uint64_t kSt16 = C::kStage >> 4, kPair16 = C::kPair >> 4;
      int sc = 0;
      bool ok = true;
      for (int il = 0; ok; ++il) {
        if (fetch(il) < 0) break;
        bool first = true, acc_started = false;
        for (;;) {
          const int ss = sc & 1;
          if (!(ok = mbar_wait(pd_full, sc & 1, abort_flag, g.status))) break;
          volatile KvMeta* m = meta(ss);
          const bool has = m->Ia >= 0;
          const bool last = m->last != 0;
          if (first && il >= 1 && !(ok = mbar_wait(acc_empty, (il - 1) & 1, abort_flag, g.status))) break;
          tc_fence_after();
          if (has) {
            const uint64_t q = dStMN + ss * kSt16, o = q + kPair16;
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {  // K = 128 query rows
              const uint32_t acc = (acc_started || kk > 0) ? 1u : 0u;
              tc_mma_bf16(t_dv, o + 128 * kk, dP + 128 * kk, C::kIdescAcc, acc);
              tc_mma_bf16(t_dk, q + 128 * kk, dDs + 128 * kk, C::kIdescAcc, acc);
            }
            acc_started = true;
          }
          tc_commit(pd_free);
          tc_commit(&stage_free[ss]);
          if (last) {
            tc_commit(acc_full);
            tc_commit(item_free);
          }
          first = false;
          ++sc;
          if (last) break;
        }
      }
      tc_commit(&drain[1]);
      drain_wait(&drain[1], 0);
    }
    __syncwarp();
  } else if (warp < 8) {
    // ---------------------------------------------------------- elementwise
    const int quarter = warp & 3, half = warp >> 2;
    const int r = quarter * 32 + lane;  // TMEM lane: query row of the pair (S, dP); feature row (dK^T, dV^T)
    const int c0 = 32 * half;           // this thread's 32 key columns
    const uint32_t lane_addr = static_cast<uint32_t>(quarter * 32) << 16;
    int sc = 0;
    bool ok = true;
    for (int il = 0; ok; ++il) {
      int it = -1;
      if (lane == 0) it = fetch(il);
      it = __shfl_sync(0xffffffffu, it, 0);
      if (it < 0) break;
      const int bh = it / g.M, J = it - bh * g.M;
      bool any = false;
      for (;;) {
        const int s = sc & 1, b = sc & 1;
        if (!(ok = mbar_wait(&full[s], (sc >> 1) & 1, abort_flag, g.status))) break;
        volatile KvMeta* m = meta(s);
        const int Ia = m->Ia, Ib = m->Ib;
        const bool last = m->last != 0;
        const int Irow = (r >> 6) ? Ib : Ia;
        const bool valid = Irow >= 0;
        const bool diag = g.causal && Irow == J;
        const int i = r & 63;
        any = any || Ia >= 0;
        if (!(ok = mbar_wait(&s_full[b], (sc >> 1) & 1, abort_flag, g.status))) break;
        tc_fence_after();
        float sv[32], dp[32];
        tmem_ld32(tbase + lane_addr + 128 * b + c0, sv);
        tmem_ld32(tbase + lane_addr + 128 * b + 64 + c0, dp);
        tc_wait_ld();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&s_empty[b]);
        const float* nlv = reinterpret_cast<const float*>(stage(s) + 2 * C::kPair);
        const float nl = nlv[r], dl = nlv[128 + r];  // [-lse log2e of both blocks][D of both blocks]
        uint32_t pk[16], dsk[16];
#pragma unroll
        for (int j = 0; j < 32; j += 2) {
          const int jj = c0 + j;  // key within block J
          float e0 = valid ? ex2_approx(fmaf(sv[j], g.sl, nl)) : 0.f;
          float e1 = valid ? ex2_approx(fmaf(sv[j + 1], g.sl, nl)) : 0.f;
          if (diag) {
            e0 = jj <= i ? e0 : 0.f;
            e1 = jj + 1 <= i ? e1 : 0.f;
          }
          pk[j / 2] = pack_bf16x2(e0, e1);
          dsk[j / 2] = pack_bf16x2(e0 * (dp[j] - dl), e1 * (dp[j + 1] - dl));
        }
        if (sc >= 1) mbar_wait(pd_free, (sc - 1) & 1, abort_flag, g.status);
        store_half_row(sP, r, half, pk);
        store_half_row(sDs, r, half, dsk);
        fence_async_shared();
        __syncwarp();
        if (lane == 0) mbar_arrive(pd_full);
        ++sc;
        if (last) break;
      }
      if (!ok) break;
      if (!(ok = mbar_wait(acc_full, il & 1, abort_flag, g.status))) break;
      tc_fence_after();
      if (r < D) {  // warp-uniform
        const size_t pj = (static_cast<size_t>(bh) * g.M + J) * D + r;
        const float kb = dkbar[pj] * (1.0f / 64.0f), vs = dvsum[pj];
        const size_t o = (static_cast<size_t>(bh) * g.N + 64 * J + c0) * D + r;
        float a[32], c[32];
        tmem_ld32(t_dk + lane_addr + c0, a);
        tmem_ld32(t_dv + lane_addr + c0, c);
        tc_wait_ld();
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          const size_t oj = o + static_cast<size_t>(j) * D;
          dk[oj] = __float2bfloat16_rn((any ? g.tau * a[j] : 0.f) + kb);
          dv[oj] = __float2bfloat16_rn((any ? c[j] : 0.f) + vs);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(acc_empty);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == kWarpMma) {
    tc_fence_after();
    tmem_dealloc(tbase, 512);
  }
}

// One CTA per SM: as many ranges of query blocks per (head, tile) as keep
// the grid within one wave.
int pseudo_chunks(int BH, int tiles, int M, int& per) {
  const int items = BH * tiles;
  int want = device_sm_count() / items;
  if (want < 1) want = 1;
  if (want > M) want = M;
  per = (M + want - 1) / want;
  return (M + per - 1) / per;
}

template <typename K>
cudaError_t set_smem(K kernel, int bytes) {
  return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
}

template <int D>
cudaError_t launch_bwd_d(const BwdLaunch& a, cudaStream_t st) {
  const int BH = a.BH, N = a.N, M = a.M;
  CUtensorMap mq, mdo, mk, mv, mkb, mvs;
  if (encode_tensor_map_3d_bf16(&mq, a.q, D, N, BH, 64, 64) != CUDA_SUCCESS ||
      encode_tensor_map_3d_bf16(&mdo, a.dout, D, N, BH, 64, 64) != CUDA_SUCCESS ||
      encode_tensor_map_3d_bf16(&mk, a.k, D, N, BH, 64, 64) != CUDA_SUCCESS ||
      encode_tensor_map_3d_bf16(&mv, a.v, D, N, BH, 64, 64) != CUDA_SUCCESS ||
      encode_tensor_map_3d_bf16(&mkb, a.kbar_bf16, D, M, BH, 64, 64) != CUDA_SUCCESS ||
      encode_tensor_map_3d_bf16(&mvs, a.vsum_bf16, D, M, BH, 64, 64) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  BwdArgs g;
  g.row_ptr = a.row_ptr;
  g.col_idx = a.col_idx;
  g.col_cap = a.col_cap;
  g.bits = a.bits;
  g.nlse2 = a.nlse2;
  g.delta = a.delta;
  g.BH = BH;
  g.M = M;
  g.N = N;
  g.nw = (M + 31) / 32;
  g.causal = a.causal;
  g.sl = kLog2e / sqrtf(static_cast<float>(D));
  g.tau = 1.0f / sqrtf(static_cast<float>(D));
  g.status = a.status;
  g.sched = a.sched;
  const int sms = device_sm_count();
  cudaError_t e;
  // delta and -lse log2 e
  {
    const long long rows = static_cast<long long>(BH) * N;
    long long blocks = (rows * 8 + 255) / 256;
    if (blocks > sms * 16LL) blocks = sms * 16LL;
    bwd_delta_kernel<D><<<static_cast<unsigned>(blocks), 256, 0, st>>>(
        reinterpret_cast<const uint4*>(a.out), reinterpret_cast<const uint4*>(a.dout), a.lse, rows, a.delta, a.nlse2);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  // listed-block bitmaps
  {
    const long long nrows = static_cast<long long>(BH) * M;
    bwd_bits_kernel<<<static_cast<unsigned>((nrows + 7) / 8), 256, 0, st>>>(a.row_ptr, a.col_idx, a.col_cap, M, g.nw,
                                                                           a.causal, nrows, a.bits, a.status);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  // pseudo-key gradients
  {
    const int tiles = (M + 127) / 128;
    int per = 1;
    const int chunks = pseudo_chunks(BH, tiles, M, per);
    if ((e = set_smem(bwd_pseudo_kernel<D>, PseudoCfg<D>::kSmem)) != cudaSuccess) return e;
    bwd_pseudo_kernel<D><<<BH * tiles * chunks, kBwdThreads, PseudoCfg<D>::kSmem, st>>>(
        mkb, mvs, mq, mdo, g, tiles, chunks, per, a.part_dvs, a.part_dkb);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    const long long md = static_cast<long long>(M) * D;
    bwd_pseudo_reduce_kernel<<<dim3(static_cast<unsigned>((md + 255) / 256), BH), 256, 0, st>>>(
        a.part_dvs, a.part_dkb, M, D, tiles, chunks, a.dvsum, a.dkbar);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  // dq
  {
    if ((e = set_smem(bwd_dq_kernel<D>, DqCfg<D>::kSmem)) != cudaSuccess) return e;
    const int units = BH * M;
    bwd_dq_kernel<D><<<units < sms ? units : sms, kBwdThreads, DqCfg<D>::kSmem, st>>>(
        mq, mdo, mk, mv, mkb, mvs, g, reinterpret_cast<__nv_bfloat16*>(a.dq));
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  // dk, dv
  {
    if ((e = set_smem(bwd_dkdv_kernel<D>, KvCfg<D>::kSmem)) != cudaSuccess) return e;
    const int items = BH * M;
    bwd_dkdv_kernel<D><<<items < sms ? items : sms, kBwdThreads, KvCfg<D>::kSmem, st>>>(
        mq, mdo, mk, mv, g, a.dkbar, a.dvsum, reinterpret_cast<__nv_bfloat16*>(a.dk),
        reinterpret_cast<__nv_bfloat16*>(a.dv));
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace

size_t bwd_partial_bytes(int BH, int M, int d) {
  // chunk count sized for up to 256 SMs (it only grows with the SM count)
  const int tiles = (M + 127) / 128;
  const int items = BH * tiles;
  int want = (2 * 256 + items - 1) / items;
  if (want < 1) want = 1;
  if (want > M) want = M;
  const int per = (M + want - 1) / want;
  const size_t chunks = static_cast<size_t>((M + per - 1) / per);
  return static_cast<size_t>(items) * chunks * 128 * d * 4;
}

cudaError_t launch_bwd(const BwdLaunch& a, cudaStream_t st) {
  return a.d == 128 ? launch_bwd_d<128>(a, st) : launch_bwd_d<64>(a, st);
}

}  // namespace psa
