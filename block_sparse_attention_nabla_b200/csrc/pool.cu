// Block averaging of Algorithm 1 ("∇NABLA: Neighborhood Adaptive Block-Level
// Attention", §3.1.2): the mean of Q and of K over every block of N = 64
// tokens, the HBM-bound step of the mask builder (it reads Q and K once).
//
// A block of one (b, h) is 64 consecutive rows of D elements, one contiguous
// run of 64 * D * sizeof(T) bytes (16 KB for bf16 at D = 128), so each block
// arrives in shared memory with a single bulk copy (cp.async.bulk): one lane
// of a producer warp keeps a ring of kStages blocks in flight, and D consumer
// threads, one per column, sum the block's valid rows of their column in fp64
// straight from shared memory and free the slot.  The loads cost no
// instructions of the consumers and stay in flight while they add, which is
// what a warp-per-block loop with register loads could not sustain.
//
// Items are (b, h, tensor, block) in head-major order, dealt round-robin to a
// persistent grid of all the CTAs that fit (three per SM).  Outputs per
// block: the mean in fp64 (the selection ranks near-equal entries by fp64
// logits) and as a pair of fp32 values hi + lo with hi the nearest tf32 value
// (operands of the tensor-core score GEMM).  A partial last block divides by
// its number of valid tokens.  Each consumer warp adds, once per head, the
// number of that head's items it has written to the head's counter (a
// release).  The score GEMM is launched behind this kernel with programmatic
// stream serialization: its CTAs take SMs as this kernel's CTAs leave them and
// wait on the counter of each head before they read its pooled vectors.
#include <cuda_bf16.h>

#include "internal.cuh"
#include "sm100.cuh"

namespace nabla {
namespace {

using namespace sm100;

constexpr int kPoolStages = 4;
// Consumer groups: group g reduces the items it = g, g + kGroups, ... of its
// CTA (stage it % kPoolStages).  One group per CTA with three CTAs per SM is
// the fastest measured (273 us at 720p against 407 us with two groups).
constexpr int kGroups = 1;
constexpr uint64_t kPoolDrainNs = 1000000000ull;

template <typename T, int D>
struct PoolLayout {
  static constexpr uint32_t kStageBytes = 64u * D * sizeof(T);
  static constexpr uint32_t bar_off = kPoolStages * kStageBytes;   // full[S], empty[S]
  static constexpr uint32_t misc_off = bar_off + 2 * kPoolStages * 8;
  static constexpr uint32_t bytes = misc_off + 16;
  static constexpr int kThreads = 32 + kGroups * D;                 // producer warp + groups of one thread per column
};

__device__ __forceinline__ float to_float(float x) { return x; }
__device__ __forceinline__ float to_float(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T, int D>
__global__ void __launch_bounds__(PoolLayout<T, D>::kThreads)
    pool_bulk_kernel(const T* __restrict__ q, const T* __restrict__ k, double* __restrict__ qa,
                     double* __restrict__ ka, float* __restrict__ qhi, float* __restrict__ qlo,
                     float* __restrict__ khi, float* __restrict__ klo, int S, int nb, long long n_items,
                     int32_t* __restrict__ counters, int32_t* __restrict__ status, uint64_t limit_ns) {
  using L = PoolLayout<T, D>;
  extern __shared__ __align__(128) uint8_t smem[];
  uint64_t* full = (uint64_t*)(smem + L::bar_off);
  uint64_t* empty = full + kPoolStages;
  volatile int* abort_flag = (volatile int*)(smem + L::misc_off);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kPoolStages; ++s) {
      mbar_init(full + s, 1);
      mbar_init(empty + s, D);  // every thread of the group that reads it releases the slot
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  pdl_launch_dependents();
  const long long per_bh = 2ll * nb;  // Q blocks then K blocks of one (b, h)

  if (warp == 0) {
    if (lane == 0) {
      long long it = 0;
      for (long long item = blockIdx.x; item < n_items; item += gridDim.x, ++it) {
        const uint32_t s = (uint32_t)(it % kPoolStages), use = (uint32_t)(it / kPoolStages);
        if (use > 0 && !mbar_wait(empty + s, (use - 1) & 1, abort_flag, limit_ns)) break;
        const long long bh = item / per_bh;
        const int r = (int)(item - bh * per_bh);
        const bool isk = r >= nb;
        const int i = isk ? r - nb : r;
        const int valid = min(kBlock, S - i * kBlock);
        const T* src = (isk ? k : q) + (bh * S + (long long)i * kBlock) * D;
        const uint32_t bytes = (uint32_t)valid * D * sizeof(T);  // a multiple of 128
        mbar_expect_tx(full + s, bytes);
        bulk_load(smem + s * L::kStageBytes, src, bytes, full + s);
      }
      // let every copy issued land before the CTA exits: the last use of each
      // slot completes after the earlier ones
      for (long long j = (it > kPoolStages ? it - kPoolStages : 0); j < it; ++j)
        mbar_wait(full + (j % kPoolStages), (uint32_t)((j / kPoolStages) & 1), nullptr, kPoolDrainNs);
    }
  } else {
    const int ct = threadIdx.x - 32;
    const int grp = ct / D, col = ct - grp * D;
    long long it = grp;
    long long cur_bh = -1;
    int done_items = 0;  // items of head cur_bh this warp has written
    // publish this warp's finished items of head cur_bh: every lane's stores
    // are ordered before lane 0's release
    auto publish = [&]() {
      if (done_items > 0) {
        __threadfence();
        __syncwarp();
        if (lane == 0) atomicAdd(counters + 2 * cur_bh, done_items);
      }
      done_items = 0;
    };
    for (long long item = blockIdx.x + (long long)grp * gridDim.x; item < n_items;
         item += (long long)kGroups * gridDim.x, it += kGroups) {
      const uint32_t s = (uint32_t)(it % kPoolStages);
      const bool ok = mbar_wait(full + s, (uint32_t)((it / kPoolStages) & 1), abort_flag, limit_ns);
      if (!__all_sync(0xffffffffu, ok)) break;
      const long long bh = item / per_bh;
      if (bh != cur_bh) {
        publish();
        cur_bh = bh;
      }
      const int r = (int)(item - bh * per_bh);
      const bool isk = r >= nb;
      const int i = isk ? r - nb : r;
      const int valid = min(kBlock, S - i * kBlock);
      const T* tile = reinterpret_cast<const T*>(smem + s * L::kStageBytes) + col;
      double acc0 = 0.0, acc1 = 0.0;  // two chains: even and odd rows
      if (valid == kBlock) {
#pragma unroll 16
        for (int row = 0; row < kBlock; row += 2) {
          acc0 += (double)to_float(tile[row * D]);
          acc1 += (double)to_float(tile[(row + 1) * D]);
        }
      } else {
        for (int row = 0; row < valid; ++row) acc0 += (double)to_float(tile[row * D]);
      }
      mbar_arrive(empty + s);
      const double mean = (acc0 + acc1) / (double)valid;
      const float f = (float)mean;
      const float h = to_tf32(f);
      const long long o = (bh * nb + i) * D + col;
      (isk ? ka : qa)[o] = mean;
      (isk ? khi : qhi)[o] = h;
      (isk ? klo : qlo)[o] = f - h;
      ++done_items;
    }
    publish();
  }
  __syncthreads();
  if (threadIdx.x == 0 && *abort_flag) atomicCAS(status, 0, (int32_t)NABLA_ERR_TIMEOUT);
}

template <typename T, int D>
cudaError_t run_pool(const Dims& d, const T* q, const T* k, double* qa, double* ka, float* qhi, float* qlo,
                     float* khi, float* klo, int32_t* counters, int32_t* status, cudaStream_t st) {
  using L = PoolLayout<T, D>;
  auto kern = pool_bulk_kernel<T, D>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)L::bytes);
  if (e != cudaSuccess) return e;
  // the largest shared-memory configuration, so that the builder's kernels fit side by side
  e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, (int)cudaSharedmemCarveoutMaxShared);
  if (e != cudaSuccess) return e;
  // all the CTAs that fit at once: the pooling needs that many blocks in
  // flight to stream Q and K at the HBM rate
  int per_sm = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, L::kThreads, L::bytes) != cudaSuccess ||
      per_sm < 1)
    per_sm = 1;
  const long long n_items = 2 * d.BH() * d.nb;
  const int grid = (int)std::min<long long>(n_items, (long long)sm_count() * per_sm);
  kern<<<grid, L::kThreads, L::bytes, st>>>(q, k, qa, ka, qhi, qlo, khi, klo, d.S, d.nb, n_items, counters,
                                            status, wait_limit_ns());
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_pool(const Dims& d, const void* q, const void* k, double* qa, double* ka, float* qhi,
                        float* qlo, float* khi, float* klo, int32_t* counters, int32_t* status, cudaStream_t st) {
  if (d.dtype == NABLA_BF16) {
    const auto* qq = (const __nv_bfloat16*)q;
    const auto* kk = (const __nv_bfloat16*)k;
    if (d.D == 128) return run_pool<__nv_bfloat16, 128>(d, qq, kk, qa, ka, qhi, qlo, khi, klo, counters, status, st);
    return run_pool<__nv_bfloat16, 64>(d, qq, kk, qa, ka, qhi, qlo, khi, klo, counters, status, st);
  }
  const auto* qq = (const float*)q;
  const auto* kk = (const float*)k;
  if (d.D == 128) return run_pool<float, 128>(d, qq, kk, qa, ka, qhi, qlo, khi, klo, counters, status, st);
  return run_pool<float, 64>(d, qq, kk, qa, ka, qhi, qlo, khi, klo, counters, status, st);
}

}  // namespace nabla
