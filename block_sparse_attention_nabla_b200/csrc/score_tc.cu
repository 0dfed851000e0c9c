// Reduced attention logits of Algorithm 1 ("∇NABLA: Neighborhood Adaptive
// Block-Level Attention", §3.1.2) on the 5th-generation tensor cores:
//
//     L[b, h, i, j] = (Qa_i . Ka_j) / sqrt(D)
//
// for all query blocks i and key blocks j of every (b, h).  The selection
// needs these logits to about fp32 accuracy, more than one tf32 product
// gives, so each pooled vector x is split as x = hi + lo with hi the nearest
// tf32 value and lo = x - hi (exact in fp32), and
//
//     Qa . Ka ~= Qa_hi . Ka_hi + Qa_hi . Ka_lo + Qa_lo . Ka_hi
//
// (the dropped lo . lo term and the tf32 truncation of lo are below 2^-21 of
// the product) is accumulated in fp32 in TMEM.
//
// Persistent kernel, one CTA per SM, each taking the 128 x 128 tiles of L in
// a fixed round-robin share (head-major order).  Warp 0 streams the operand
// sub-chunks (32 dimensions = one 128-byte swizzle row of A_hi, A_lo, B_hi,
// B_lo: 64 KB) through a ring of kStages stages with TMA; warp 1 owns TMEM
// and issues the 12 MMAs of every sub-chunk into one of two 128-column
// accumulators; warps 2-5 drain the other accumulator, one TMEM lane (row)
// per thread, and write the tile through a shared-memory staging tile of
// their own in whole 128-byte row segments.  So the loads of the next
// sub-chunks, the MMAs of this tile and the epilogue of the previous one
// overlap, where one tile per CTA ran them in sequence.
//
// The kernel is launched behind the pooling with programmatic stream
// serialization, so its CTAs start as the pooling's leave the SMs: before the
// first tile of a head the producer waits (bounded) until the pooling has
// counted all of that head's blocks.  After each tile every epilogue warp
// counts it for the selection, which is launched behind this kernel the same
// way and runs beside it, head by head.
#include <cuda.h>
#include <cudaTypedefs.h>

#include "internal.cuh"
#include "sm100.cuh"

namespace nabla {
namespace {

using namespace sm100;

constexpr int kSubK = 32;                             // fp32 elements per 128-byte swizzle row
constexpr int kStages = 2;
constexpr int kThreads = 192;
constexpr uint32_t kOpBytes = 128 * 128;              // one operand sub-chunk: 128 rows x 128 B
constexpr uint32_t kStageBytes = 4 * kOpBytes;        // A_hi, A_lo, B_hi, B_lo
constexpr uint32_t kEpiOff = kStages * kStageBytes;   // 4 warps x [32 rows][128 B]
constexpr uint32_t kBarOff = kEpiOff + 4 * 4096;
// full[S], empty[S], acc_full[2], acc_empty[2], drain
constexpr int kNumBars = 2 * kStages + 2 + 2 + 1;
constexpr uint32_t kMiscOff = kBarOff + kNumBars * 8;  // TMEM slot, abort flag
constexpr uint32_t kGemmSmem = kMiscOff + 16;
constexpr uint64_t kDrainNs = 1000000000ull;

template <int D>
__global__ void __launch_bounds__(kThreads, 1) score_gemm_kernel(
    const __grid_constant__ CUtensorMap tm_qhi, const __grid_constant__ CUtensorMap tm_qlo,
    const __grid_constant__ CUtensorMap tm_khi, const __grid_constant__ CUtensorMap tm_klo,
    float* __restrict__ L, int nb, int ldl, int T, long long n_tiles, float scale, int32_t* __restrict__ counters,
    int pool_goal, int32_t* __restrict__ status, uint64_t limit_ns) {
  constexpr int kSub = D / kSubK;
  extern __shared__ __align__(1024) uint8_t smem[];
  if (smem_u32(smem) & 1023u) {
    if (threadIdx.x == 0) atomicCAS(status, 0, (int32_t)NABLA_ERR_UNSUPPORTED);
    return;
  }
  uint64_t* full = (uint64_t*)(smem + kBarOff);
  uint64_t* empty = full + kStages;
  uint64_t* acc_full = empty + kStages;
  uint64_t* acc_empty = acc_full + 2;
  uint64_t* drain = acc_empty + 2;
  uint32_t* tmem_slot = (uint32_t*)(smem + kMiscOff);
  volatile int* abort_flag = (volatile int*)(smem + kMiscOff + 4);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(full + s, 1);
      mbar_init(empty + s, 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(acc_full + b, 1);
      mbar_init(acc_empty + b, 128);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tm_qhi);
    tma_prefetch_desc(&tm_qlo);
    tma_prefetch_desc(&tm_khi);
    tma_prefetch_desc(&tm_klo);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 256);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  pdl_launch_dependents();
  const uint32_t tmem = *tmem_slot;
  const uint32_t sbase = smem_u32(smem);
  const long long per_bh = (long long)T * T;

  if (warp == 0) {
    // ---------------------------------------------------------- producer
    if (lane == 0) {
      uint32_t g = 0;  // sub-chunks issued by this CTA
      bool ok = true;
      int ready_bh = -1;  // the last head whose pooled vectors are known complete
      for (long long t = blockIdx.x; t < n_tiles && ok; t += gridDim.x) {
        const int bh = (int)(t / per_bh);
        const int r = (int)(t - (long long)bh * per_bh);
        const int m0 = (r / T) * 128, n0 = (r % T) * 128;
        if (bh != ready_bh) {
          if (!(ok = wait_counter(counters + 2 * bh, pool_goal, abort_flag, limit_ns))) break;
          fence_proxy_async_global();  // the TMA reads below see the pooled vectors
          ready_bh = bh;
        }
        for (int s = 0; s < kSub; ++s, ++g) {
          const uint32_t st = g % kStages, use = g / kStages;
          if (use > 0 && !(ok = mbar_wait(empty + st, (use - 1) & 1, abort_flag, limit_ns))) break;
          uint8_t* dst = smem + st * kStageBytes;
          mbar_expect_tx(full + st, kStageBytes);
          tma_load_3d(dst + 0 * kOpBytes, &tm_qhi, full + st, s * kSubK, m0, bh);
          tma_load_3d(dst + 1 * kOpBytes, &tm_qlo, full + st, s * kSubK, m0, bh);
          tma_load_3d(dst + 2 * kOpBytes, &tm_khi, full + st, s * kSubK, n0, bh);
          tma_load_3d(dst + 3 * kOpBytes, &tm_klo, full + st, s * kSubK, n0, bh);
        }
      }
      // let every copy this thread issued land before the CTA exits
      for (uint32_t i = (g > kStages ? g - kStages : 0); i < g; ++i)
        mbar_wait(full + i % kStages, (i / kStages) & 1, nullptr, kDrainNs);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_tf32_f32(128, 128);
      uint32_t g = 0, lt = 0;
      bool ok = true;
      for (long long t = blockIdx.x; t < n_tiles && ok; t += gridDim.x, ++lt) {
        const uint32_t ab = lt & 1;
        // the epilogue has drained this accumulator's previous tile
        if (lt >= 2 && !(ok = mbar_wait(acc_empty + ab, ((lt >> 1) - 1) & 1, abort_flag, limit_ns))) break;
        tc_fence_after();
        const uint32_t acc = tmem + ab * 128;
        for (int s = 0; s < kSub; ++s, ++g) {
          const uint32_t st = g % kStages;
          if (!(ok = mbar_wait(full + st, (g / kStages) & 1, abort_flag, limit_ns))) break;
          tc_fence_after();
          const uint32_t base = sbase + st * kStageBytes;
#pragma unroll
          for (int kk = 0; kk < kSubK / 8; ++kk) {  // 8 tf32 = 32 bytes per MMA
            const uint64_t ahi = desc_sw128(base + 0 * kOpBytes + kk * 32, 16, 1024);
            const uint64_t alo = desc_sw128(base + 1 * kOpBytes + kk * 32, 16, 1024);
            const uint64_t bhi = desc_sw128(base + 2 * kOpBytes + kk * 32, 16, 1024);
            const uint64_t blo = desc_sw128(base + 3 * kOpBytes + kk * 32, 16, 1024);
            mma_ss_tf32(acc, ahi, bhi, idesc, (s > 0 || kk > 0) ? 1u : 0u);
            mma_ss_tf32(acc, ahi, blo, idesc, 1u);
            mma_ss_tf32(acc, alo, bhi, idesc, 1u);
          }
          mma_commit(empty + st);
        }
        if (ok) mma_commit(acc_full + ab);
      }
    }
  } else {
    // --------------------------------------------------------- epilogue
    // Each warp moves its 32 rows out of TMEM in 32 x 32 chunks through a
    // shared-memory tile of its own (16-byte chunk k of row r sits at
    // k ^ (r & 7), so the writes and reads are conflict-free), so that every
    // global store writes whole 128-byte row segments.
    const int quarter = warp & 3;
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    uint8_t* tile = smem + kEpiOff + quarter * 4096;  // [32 rows][128 B]
    const int rsub = lane >> 3, q = lane & 7;
    uint32_t lt = 0;
    for (long long t = blockIdx.x; t < n_tiles; t += gridDim.x, ++lt) {
      const uint32_t ab = lt & 1;
      const bool w = mbar_wait(acc_full + ab, (lt >> 1) & 1, abort_flag, limit_ns);
      if (!__all_sync(0xffffffffu, w)) break;
      tc_fence_after();
      const int bh = (int)(t / per_bh);
      const int r = (int)(t - (long long)bh * per_bh);
      const int m0 = (r / T) * 128, n0 = (r % T) * 128;
      const uint32_t taddr = tmem + ab * 128 + lane_off;
#pragma unroll 1
      for (int c0 = 0; c0 < 128; c0 += 32) {
        uint32_t v[32];
        tmem_ld32(taddr + c0, v);
        tmem_ld_wait();
        if (c0 == 96) {
          // the accumulator is read: the issuer may start the tile after next
          tc_fence_before();
          mbar_arrive(acc_empty + ab);
        }
        __syncwarp();  // the previous chunk's reads of the staging tile are done
#pragma unroll
        for (int kc = 0; kc < 8; ++kc)
          *reinterpret_cast<float4*>(tile + lane * 128 + ((kc ^ (lane & 7)) << 4)) =
              make_float4(__uint_as_float(v[4 * kc]) * scale, __uint_as_float(v[4 * kc + 1]) * scale,
                          __uint_as_float(v[4 * kc + 2]) * scale, __uint_as_float(v[4 * kc + 3]) * scale);
        __syncwarp();
        const int col = n0 + c0 + 4 * q;
#pragma unroll
        for (int kc = 0; kc < 8; ++kc) {
          const int rr = 4 * kc + rsub;  // row of the warp's 32; lanes 8 rsub .. 8 rsub + 7 cover its 128 bytes
          const float4 x = *reinterpret_cast<const float4*>(tile + rr * 128 + ((q ^ (rr & 7)) << 4));
          const int m = m0 + quarter * 32 + rr;
          if (m < nb && col < nb) {
            float* dst = L + ((long long)bh * nb + m) * ldl + col;
            if (col + 4 <= nb) {
              *reinterpret_cast<float4*>(dst) = x;
            } else {
              dst[0] = x.x;
              if (col + 1 < nb) dst[1] = x.y;
              if (col + 2 < nb) dst[2] = x.z;
            }
          }
        }
      }
      // count the tile for the selection: every lane's stores before lane 0's release
      __threadfence();
      __syncwarp();
      if (lane == 0) atomicAdd(counters + 2 * bh + 1, 1);
    }
  }

  // ------------------------------------------------------------- teardown
  __syncthreads();
  if (warp == 1) {
    if (lane == 0) {
      // a run that gave up may still have MMAs in flight: let them finish
      mma_commit(drain);
      mbar_wait(drain, 0, nullptr, kDrainNs);
    }
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
  if (threadIdx.x == 0 && *abort_flag) atomicCAS(status, 0, (int32_t)NABLA_ERR_TIMEOUT);
}

template <int D>
cudaError_t run(const Dims& d, const float* qhi, const float* qlo, const float* khi, const float* klo,
                float* L, int ldl, int32_t* counters, int pool_goal, int32_t* status, cudaStream_t st) {
  CUtensorMap a, b, c, e;
  if (!make_map_pooled_f32(&a, qhi, d) || !make_map_pooled_f32(&b, qlo, d) ||
      !make_map_pooled_f32(&c, khi, d) || !make_map_pooled_f32(&e, klo, d))
    return cudaErrorInvalidValue;
  auto kern = score_gemm_kernel<D>;
  cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kGemmSmem);
  if (err != cudaSuccess) return err;
  // the largest shared-memory configuration, so that the builder's kernels fit side by side
  err = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, (int)cudaSharedmemCarveoutMaxShared);
  if (err != cudaSuccess) return err;
  const int T = (d.nb + 127) / 128;
  const long long n_tiles = (long long)T * T * d.BH();
  const int grid = (int)std::min<long long>(n_tiles, sm_count());
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = kGemmSmem;
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, a, b, c, e, L, d.nb, ldl, T, n_tiles, 1.0f / sqrtf((float)d.D), counters,
                            pool_goal, status, wait_limit_ns());
}

}  // namespace

cudaError_t launch_score_gemm(const Dims& d, const float* qhi, const float* qlo, const float* khi,
                              const float* klo, float* L, int ldl, int32_t* counters, int pool_goal,
                              int32_t* status, cudaStream_t st) {
  if (d.D == 128) return run<128>(d, qhi, qlo, khi, klo, L, ldl, counters, pool_goal, status, st);
  return run<64>(d, qhi, qlo, khi, klo, L, ldl, counters, pool_goal, status, st);
}

}  // namespace nabla
