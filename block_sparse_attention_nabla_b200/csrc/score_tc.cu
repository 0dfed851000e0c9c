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
// One CTA computes one 128 x 128 tile of L: warp 0 streams the four operand
// sub-chunks (32 dimensions = one 128-byte swizzle row) with TMA, warp 1 owns
// TMEM and issues the MMAs, then all four warps write the tile to the logits
// buffer through shared memory in coalesced row segments.
#include <cuda.h>
#include <cudaTypedefs.h>

#include "internal.cuh"
#include "sm100.cuh"

namespace nabla {
namespace {

using namespace sm100;

constexpr int kSubK = 32;  // fp32 elements per 128-byte swizzle row
constexpr uint32_t kOpBytes = 128 * 128;            // one operand sub-chunk: 128 rows x 128 B
constexpr uint32_t kStageBytes = 4 * kOpBytes;      // A_hi, A_lo, B_hi, B_lo
constexpr uint32_t kBarOff = kStageBytes;
constexpr uint32_t kMiscOff = kBarOff + 4 * 8;      // full, empty, done, drain
constexpr uint32_t kGemmSmem = kMiscOff + 16;
constexpr uint64_t kDrainNs = 1000000000ull;

template <int D>
__global__ void __launch_bounds__(128) score_gemm_kernel(
    const __grid_constant__ CUtensorMap tm_qhi, const __grid_constant__ CUtensorMap tm_qlo,
    const __grid_constant__ CUtensorMap tm_khi, const __grid_constant__ CUtensorMap tm_klo,
    float* __restrict__ L, int nb, int ldl, float scale, int32_t* __restrict__ status, uint64_t limit_ns) {
  constexpr int kSub = D / kSubK;
  extern __shared__ __align__(1024) uint8_t smem[];
  if (smem_u32(smem) & 1023u) {
    if (threadIdx.x == 0) atomicCAS(status, 0, (int32_t)NABLA_ERR_UNSUPPORTED);
    return;
  }
  uint64_t* full = (uint64_t*)(smem + kBarOff);
  uint64_t* empty = full + 1;
  uint64_t* done = full + 2;
  uint64_t* drain = full + 3;
  uint32_t* tmem_slot = (uint32_t*)(smem + kMiscOff);
  volatile int* abort_flag = (volatile int*)(smem + kMiscOff + 4);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n0 = blockIdx.x * 128, m0 = blockIdx.y * 128, bh = blockIdx.z;

  if (threadIdx.x == 0) {
    mbar_init(full, 1);
    mbar_init(empty, 1);
    mbar_init(done, 1);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 128);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t sbase = smem_u32(smem);

  if (warp == 0 && lane == 0) {
    // producer: one stage, refilled once the MMAs of the previous sub-chunk completed
    int issued = 0;
    for (int s = 0; s < kSub; ++s) {
      if (s > 0 && !mbar_wait(empty, (s - 1) & 1, abort_flag, limit_ns)) break;
      mbar_expect_tx(full, kStageBytes);
      tma_load_3d(smem + 0 * kOpBytes, &tm_qhi, full, s * kSubK, m0, bh);
      tma_load_3d(smem + 1 * kOpBytes, &tm_qlo, full, s * kSubK, m0, bh);
      tma_load_3d(smem + 2 * kOpBytes, &tm_khi, full, s * kSubK, n0, bh);
      tma_load_3d(smem + 3 * kOpBytes, &tm_klo, full, s * kSubK, n0, bh);
      ++issued;
    }
    if (issued > 0) mbar_wait(full, (issued - 1) & 1, nullptr, kDrainNs);
  } else if (warp == 1 && lane == 0) {
    constexpr uint32_t idesc = idesc_tf32_f32(128, 128);
    bool ok = true;
    for (int s = 0; s < kSub && ok; ++s) {
      if (!(ok = mbar_wait(full, s & 1, abort_flag, limit_ns))) break;
      tc_fence_after();
#pragma unroll
      for (int kk = 0; kk < kSubK / 8; ++kk) {  // 8 tf32 = 32 bytes per MMA
        const uint64_t ahi = desc_sw128(sbase + 0 * kOpBytes + kk * 32, 16, 1024);
        const uint64_t alo = desc_sw128(sbase + 1 * kOpBytes + kk * 32, 16, 1024);
        const uint64_t bhi = desc_sw128(sbase + 2 * kOpBytes + kk * 32, 16, 1024);
        const uint64_t blo = desc_sw128(sbase + 3 * kOpBytes + kk * 32, 16, 1024);
        mma_ss_tf32(tmem, ahi, bhi, idesc, (s > 0 || kk > 0) ? 1u : 0u);
        mma_ss_tf32(tmem, ahi, blo, idesc, 1u);
        mma_ss_tf32(tmem, alo, bhi, idesc, 1u);
      }
      mma_commit(empty);
    }
    if (ok) mma_commit(done);
  }
  // epilogue: each warp moves its 32 rows out of TMEM in 32 x 32 chunks
  // through a shared-memory tile of its own (the operand stage is free once
  // the MMAs are done; 16-byte chunk k of row r sits at k ^ (r & 7), so the
  // writes and reads are conflict-free), so that every global store writes
  // whole 128-byte row segments instead of 32 rows' 16-byte pieces.
  __syncwarp();
  const bool w = mbar_wait(done, 0, abort_flag, limit_ns);
  if (__all_sync(0xffffffffu, w)) {
    tc_fence_after();
    const uint32_t taddr = tmem + ((uint32_t)(warp * 32) << 16);
    uint8_t* tile = smem + warp * 4096;  // [32 rows][128 B]
    const int rsub = lane >> 3, q = lane & 7;
#pragma unroll 1
    for (int c0 = 0; c0 < 128; c0 += 32) {
      uint32_t v[32];
      tmem_ld32(taddr + c0, v);
      tmem_ld_wait();
      __syncwarp();  // the previous chunk's reads of the tile are done
#pragma unroll
      for (int k = 0; k < 8; ++k)
        *reinterpret_cast<float4*>(tile + lane * 128 + ((k ^ (lane & 7)) << 4)) =
            make_float4(__uint_as_float(v[4 * k]) * scale, __uint_as_float(v[4 * k + 1]) * scale,
                        __uint_as_float(v[4 * k + 2]) * scale, __uint_as_float(v[4 * k + 3]) * scale);
      __syncwarp();
      const int col = n0 + c0 + 4 * q;
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const int r = 4 * k + rsub;  // row of the warp's 32; lanes 8 rsub .. 8 rsub + 7 cover its 128 bytes
        const float4 x = *reinterpret_cast<const float4*>(tile + r * 128 + ((q ^ (r & 7)) << 4));
        const int m = m0 + warp * 32 + r;
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
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    if (lane == 0) {
      // a run that gave up may still have MMAs in flight: let them finish
      mma_commit(drain);
      mbar_wait(drain, 0, nullptr, kDrainNs);
    }
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 128);
  }
  if (threadIdx.x == 0 && *abort_flag) atomicCAS(status, 0, (int32_t)NABLA_ERR_TIMEOUT);
}

template <int D>
cudaError_t run(const Dims& d, const float* qhi, const float* qlo, const float* khi, const float* klo,
                float* L, int ldl, int32_t* status, cudaStream_t st) {
  CUtensorMap a, b, c, e;
  if (!make_map_pooled_f32(&a, qhi, d) || !make_map_pooled_f32(&b, qlo, d) ||
      !make_map_pooled_f32(&c, khi, d) || !make_map_pooled_f32(&e, klo, d))
    return cudaErrorInvalidValue;
  auto kern = score_gemm_kernel<D>;
  cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kGemmSmem);
  if (err != cudaSuccess) return err;
  const int t = (d.nb + 127) / 128;
  kern<<<dim3(t, t, (unsigned)d.BH()), 128, kGemmSmem, st>>>(a, b, c, e, L, d.nb, ldl,
                                                              1.0f / sqrtf((float)d.D), status,
                                                              wait_limit_ns());
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_score_gemm(const Dims& d, const float* qhi, const float* qlo, const float* khi,
                              const float* klo, float* L, int ldl, int32_t* status, cudaStream_t st) {
  if (d.D == 128) return run<128>(d, qhi, qlo, khi, klo, L, ldl, status, st);
  return run<64>(d, qhi, qlo, khi, klo, L, ldl, status, st);
}

}  // namespace nabla
