// Per-block fidelity of a block mask: the true token-level attention mass of
// every 64 x 64 block, and the share of it a mask keeps.  This is the check
// the pith.science review of "∇NABLA: Neighborhood Adaptive Block-Level Attention"
// (arXiv 2507.13546v2) asks of Algorithm 1's pooling proxy: what fraction of
// the attention mass of dense attention (§2.1, Eq. 2-3) falls inside the
// retained blocks.
//
//   A[b, h, i, j] = mean over the valid query tokens s of block i of
//                   sum over the keys t of block j of softmax_t(q_s . k_t / sqrt(D))
//   recall[b, h, i] = sum_j M[i, j] A[i, j]
//
// block_mass_kernel: one unit = a pair of query blocks (a 128-row Q tile, so
// the S products run at M = 128), every key block visited twice: the first
// pass accumulates each row's log-sum-exp online (log2 domain), the second
// sums exp2(s * log2(e) / sqrt(D) - lse2) over each key block's 64 columns,
// reduces the row sums of each warp with shuffles and stores them per warp in
// shared memory; at the end of the unit the two warps of each query block
// are added and divided by its number of valid rows.  S = Q K^T on tcgen05
// (operands by TMA, 128-byte swizzle, accumulator in TMEM, double-buffered);
// no V and no P V product.
//
// Warp roles (192 threads): warp 0 TMA producer (Q per unit, a 3-deep ring of
// K tiles), warp 1 TMEM owner and MMA issuer, warps 2-5 one thread per row.
#include <cuda.h>
#include <cuda_bf16.h>
#include <math.h>

#include "internal.cuh"
#include "sm100.cuh"

namespace nabla {
namespace {

using namespace sm100;

constexpr int kStages = 3;
constexpr int kThreads = 192;
constexpr uint32_t kTmemCols = 128;
constexpr uint64_t kDrainLimitNs = 1000000000ull;

template <int D>
struct MassLayout {
  static constexpr int kHalves = D / 64;
  static constexpr uint32_t kQHalf = 128 * 128;  // 128 rows x 128 B
  static constexpr uint32_t kKHalf = 64 * 128;   // 64 rows x 128 B
  static constexpr uint32_t kQBytes = kHalves * kQHalf;
  static constexpr uint32_t kKBytes = kHalves * kKHalf;
  static constexpr uint32_t q_off = 0;
  static constexpr uint32_t k_off = kQBytes;
  static constexpr uint32_t bar_off = k_off + kStages * kKBytes;
  // q_full, q_empty, k_full[3], k_empty[3], s_full[2], s_free[2], unit_done,
  // parts_read, drain
  static constexpr int kNumBars = 2 + 2 * kStages + 4 + 3;
  static constexpr uint32_t misc_off = bar_off + kNumBars * 8;
  static constexpr uint32_t part_off = (misc_off + 16 + 15) & ~15u;  // float [4 warps][nb]
  static size_t bytes(int nb) { return part_off + (size_t)4 * nb * sizeof(float); }
};

template <int D>
__global__ void __launch_bounds__(kThreads, 2)
    block_mass_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                      int n_units, int S, int nb, int npairs, float scale_log2, float* __restrict__ mass,
                      int32_t* __restrict__ status, uint64_t limit_ns) {
  using L = MassLayout<D>;
  extern __shared__ __align__(1024) uint8_t smem[];
  if (smem_u32(smem) & 1023u) {
    if (threadIdx.x == 0) atomicCAS(status, 0, (int32_t)NABLA_ERR_UNSUPPORTED);
    return;
  }
  uint64_t* bars = (uint64_t*)(smem + L::bar_off);
  uint64_t* q_full = bars;
  uint64_t* q_empty = bars + 1;
  uint64_t* k_full = bars + 2;
  uint64_t* k_empty = k_full + kStages;
  uint64_t* s_full = k_empty + kStages;  // [2]
  uint64_t* s_free = s_full + 2;         // [2]: the softmax threads hold S in registers
  uint64_t* unit_done = s_free + 2;      // per unit: every warp stored its block sums
  uint64_t* parts_read = unit_done + 1;  // per unit: the sums were written out
  uint64_t* drain = parts_read + 1;
  uint32_t* tmem_slot = (uint32_t*)(smem + L::misc_off);
  volatile int* abort_flag = (volatile int*)(smem + L::misc_off + 4);
  float* part = (float*)(smem + L::part_off);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    mbar_init(q_empty, 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(k_full + s, 1);
      mbar_init(k_empty + s, 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(s_full + b, 1);
      mbar_init(s_free + b, 128);
    }
    mbar_init(unit_done, 128);
    mbar_init(parts_read, 128);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t smem_base = smem_u32(smem);
  const int steps = 2 * nb;  // per unit: two passes over every key block

  if (warp == 0) {
    // ------------------------------------------------------------- producer
    if (lane == 0) {
      uint32_t g = 0, u_local = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < n_units && ok; u += gridDim.x, ++u_local) {
        const int bh = u / npairs, p = u - bh * npairs;
        if (u_local > 0 && !(ok = mbar_wait(q_empty, (u_local - 1) & 1, abort_flag, limit_ns))) break;
        mbar_expect_tx(q_full, L::kQBytes);
#pragma unroll
        for (int h = 0; h < L::kHalves; ++h)
          tma_load_3d(smem + L::q_off + h * L::kQHalf, &tm_q, q_full, h * 64, p * 128, bh);
        for (int t = 0; t < steps; ++t, ++g) {
          const int j = t < nb ? t : t - nb;
          const uint32_t ks = g % kStages, use = g / kStages;
          if (use > 0 && !(ok = mbar_wait(k_empty + ks, (use - 1) & 1, abort_flag, limit_ns))) break;
          mbar_expect_tx(k_full + ks, L::kKBytes);
#pragma unroll
          for (int h = 0; h < L::kHalves; ++h)
            tma_load_3d(smem + L::k_off + ks * L::kKBytes + h * L::kKHalf, &tm_k, k_full + ks, h * 64, j * 64, bh);
        }
      }
      if (u_local > 0) mbar_wait(q_full, (u_local - 1) & 1, nullptr, kDrainLimitNs);
      for (uint32_t i = (g > kStages ? g - kStages : 0); i < g; ++i)
        mbar_wait(k_full + i % kStages, (i / kStages) & 1, nullptr, kDrainLimitNs);
    }
  } else if (warp == 1) {
    // ----------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(128, 64, 0, 0);
      const uint32_t qbase = smem_base + L::q_off;
      uint32_t g = 0, u_local = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < n_units && ok; u += gridDim.x, ++u_local) {
        if (!(ok = mbar_wait(q_full, u_local & 1, abort_flag, limit_ns))) break;
        tc_fence_after();
        for (int t = 0; t < steps && ok; ++t, ++g) {
          const uint32_t ks = g % kStages, sb = g & 1;
          if (!(ok = mbar_wait(k_full + ks, (g / kStages) & 1, abort_flag, limit_ns))) break;
          // buffer sb is free once every softmax thread loaded S of step g - 2
          if (g >= 2 && !(ok = mbar_wait(s_free + sb, ((g - 2) >> 1) & 1, abort_flag, limit_ns))) break;
          tc_fence_after();
          const uint32_t kbase = smem_base + L::k_off + ks * L::kKBytes;
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t koff = (kk & 3) * 32;  // 16 bf16 = 32 B inside the 128-B row
            mma_ss(tmem + sb * 64, desc_sw128(qbase + (kk >> 2) * L::kQHalf + koff, 16, 1024),
                   desc_sw128(kbase + (kk >> 2) * L::kKHalf + koff, 16, 1024), idesc, kk > 0 ? 1u : 0u);
          }
          mma_commit(k_empty + ks);
          mma_commit(s_full + sb);
        }
        mma_commit(q_empty);
      }
      mma_commit(drain);
    }
  } else {
    // ----------------------------------------------- one thread per query row
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const int tid = threadIdx.x - 64;
    const uint32_t lane_base = tmem + ((uint32_t)(quarter * 32) << 16);
    uint32_t g = 0, u_local = 0;
    bool ok = true;
    for (int u = blockIdx.x; u < n_units && ok; u += gridDim.x, ++u_local) {
      const int bh = u / npairs, p = u - bh * npairs;
      const bool valid = p * 128 + row < S;
      float m = -INFINITY, l = 0.f, lse2 = 0.f;
      for (int t = 0; t < steps; ++t, ++g) {
        const int j = t < nb ? t : t - nb;
        const uint32_t sb = g & 1;
        const bool w1 = mbar_wait(s_full + sb, (g >> 1) & 1, abort_flag, limit_ns);
        if (!__all_sync(0xffffffffu, w1)) { ok = false; break; }
        tc_fence_after();
        uint32_t r0[32], r1[32];
        tmem_ld32(lane_base + sb * 64, r0);
        tmem_ld32(lane_base + sb * 64 + 32, r1);
        tmem_ld_wait();
        tc_fence_before();
        mbar_arrive(s_free + sb);
        const int kv_lim = j == nb - 1 ? S - j * 64 : 64;
        float x[64];
#pragma unroll
        for (int c = 0; c < 32; ++c) {
          x[c] = c < kv_lim ? __uint_as_float(r0[c]) * scale_log2 : -INFINITY;
          x[c + 32] = c + 32 < kv_lim ? __uint_as_float(r1[c]) * scale_log2 : -INFINITY;
        }
        if (t < nb) {
          // pass 1: running max and sum of exp2 over the row
          float mx = x[0];
#pragma unroll
          for (int c = 1; c < 64; ++c) mx = fmaxf(mx, x[c]);
          const float mn = fmaxf(m, mx);
          float sum = 0.f;
#pragma unroll
          for (int c = 0; c < 64; ++c) sum += ex2(x[c] - mn);
          l = l * ex2(m - mn) + sum;
          m = mn;
          if (t == nb - 1) lse2 = m + log2f(l);
        } else {
          // pass 2: this row's mass on key block j, summed over the warp's rows
          float sum = 0.f;
#pragma unroll
          for (int c = 0; c < 64; ++c) sum += ex2(x[c] - lse2);
          sum = valid ? sum : 0.f;
#pragma unroll
          for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
          if (lane == 0) part[quarter * nb + j] = sum;
        }
      }
      if (!ok) break;
      // all four warps stored their sums: write the unit's two rows of A
      mbar_arrive(unit_done);
      const bool w2 = mbar_wait(unit_done, u_local & 1, abort_flag, limit_ns);
      if (!__all_sync(0xffffffffu, w2)) { ok = false; break; }
      const int i0 = 2 * p;
      const float n0 = (float)min(64, S - i0 * 64);
      const bool has1 = i0 + 1 < nb;
      const float n1 = has1 ? (float)min(64, S - (i0 + 1) * 64) : 1.f;
      float* row0 = mass + ((long long)bh * nb + i0) * nb;
      for (int jj = tid; jj < nb; jj += 128) {
        row0[jj] = (part[jj] + part[nb + jj]) / n0;
        if (has1) row0[nb + jj] = (part[2 * nb + jj] + part[3 * nb + jj]) / n1;
      }
      mbar_arrive(parts_read);
      const bool w3 = mbar_wait(parts_read, u_local & 1, abort_flag, limit_ns);
      if (!__all_sync(0xffffffffu, w3)) { ok = false; break; }
    }
  }

  // ------------------------------------------------------------- teardown
  __syncthreads();
  if (warp == 1) {
    if (lane == 0) mbar_wait(drain, 0, nullptr, kDrainLimitNs);
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
  if (threadIdx.x == 0 && *abort_flag) atomicCAS(status, 0, (int32_t)NABLA_ERR_TIMEOUT);
}

// recall[row] = sum of mass[row][j] over the kept blocks j of the row
__global__ void __launch_bounds__(256) recall_kernel(const float* __restrict__ mass, const uint32_t* __restrict__ bits,
                                                     long long rows, int nb, int W, float* __restrict__ recall) {
  const long long row = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  const float* a = mass + row * nb;
  const uint32_t* b = bits + row * W;
  float acc = 0.f;
  for (int j = lane; j < nb; j += 32)
    if ((b[j >> 5] >> (j & 31)) & 1u) acc += a[j];
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
  if (lane == 0) recall[row] = acc;
}

template <int D>
cudaError_t run_mass(const Dims& d, const void* q, const void* k, float* mass, int32_t* ws_header,
                     cudaStream_t st) {
  CUtensorMap tq, tk;
  if (!make_map_bf16(&tq, q, d, 128) || !make_map_bf16(&tk, k, d, 64)) return cudaErrorInvalidValue;
  const int n_units = (int)(d.BH() * d.npairs);
  const size_t smem = MassLayout<D>::bytes(d.nb);
  auto kern = block_mass_kernel<D>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const int grid = std::min(n_units, 2 * sm_count());
  const float scale_log2 = 1.4426950408889634f / sqrtf((float)D);
  kern<<<grid, kThreads, smem, st>>>(tq, tk, n_units, d.S, d.nb, d.npairs, scale_log2, mass,
                                     ws_header + kWsStatus, wait_limit_ns());
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_block_mass(const Dims& d, const void* q, const void* k, float* mass, int32_t* ws_header,
                              cudaStream_t st) {
  if (d.dtype != NABLA_BF16) return cudaErrorInvalidValue;
  if (d.D == 128) return run_mass<128>(d, q, k, mass, ws_header, st);
  return run_mass<64>(d, q, k, mass, ws_header, st);
}

cudaError_t launch_mask_recall(const Dims& d, const float* mass, const uint32_t* bits, float* recall,
                               cudaStream_t st) {
  const long long rows = d.BH() * d.nb;
  recall_kernel<<<(unsigned)((rows * 32 + 255) / 256), 256, 0, st>>>(mass, bits, rows, d.nb, d.W, recall);
  return cudaGetLastError();
}

}  // namespace nabla
