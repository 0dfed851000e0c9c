// Eq. 1 of "∇NABLA: Neighborhood Adaptive Block-Level Attention" (§2.1),
//
//     Q = X W_Q,   K = X W_K,   V = X W_V,
//
// on the 5th-generation tensor cores, with the block averaging of Algorithm 1
// (§3.1.2) fused into the epilogue: the kernel that writes Q and K also
// writes their 64-token block means, so the mask builder does not read Q and
// K again.
//
// X [B, S, C] bf16 (hidden states, token-major); W^T [3, H D, C] bf16 (one row
// per output feature n = h D + d of Q, K, V: the transposed W of Eq. 1, the
// layout of a linear layer's weight).  Outputs Q, K, V [B, H, S, D] bf16,
// accumulated in fp32, and for Q and K the block means of the stored (bf16)
// values in fp64 and as the tf32 hi / lo pairs the score GEMM reads, exactly
// as the pooling kernel computes them from Q and K in memory.
//
// Persistent kernel, one CTA per SM, tiles of 128 tokens (two 64-token blocks
// of one sample) x 256 output features, taken in a fixed round-robin share of
// a grouped order (16 token tiles per group, all feature tiles of a group
// before the next): the CTAs of one wave share their X and W tiles in L2
// (at C = 5120 a wave holds 16 X tiles and about 9 W tiles, 45 MB, the
// smallest such working set), and W is read from DRAM about once per group.  Warp 0 streams 64-feature slices of X and W^T (16 + 32 KB) through a
// 4-stage TMA ring; warp 1 owns TMEM and issues four K = 16 MMAs per slice
// (M = 128, N = 256, both operands K-major in shared memory, the shape that
// runs at the full tensor rate) into one of two 256-column accumulators;
// warps 2-5 drain the other accumulator, one TMEM lane (token) per thread,
// 64 columns at a time: round to bf16, stage the 128 x 64 chunk in shared
// memory, store it to Q, K or V in whole 128-byte row segments, and sum each
// column of each 64-token block from the same staging tile in fp64.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cudaTypedefs.h>

#include "internal.cuh"
#include "sm100.cuh"

namespace nabla {
namespace {

using namespace sm100;

constexpr int kTileM = 128;                              // tokens per tile
constexpr int kTileN = 256;                              // output features per tile
constexpr int kTileK = 64;                               // hidden features per stage (128-byte rows)
constexpr int kStages = 4;
constexpr int kThreads = 192;                            // producer, MMA issuer, 4 epilogue warps
constexpr int kGroupM = 16;                              // token tiles per raster group
constexpr int kChunk = 64;                               // accumulator columns per epilogue pass
constexpr uint32_t kABytes = kTileM * 128;               // X slice: 128 rows x 128 B
constexpr uint32_t kBBytes = kTileN * 128;               // W^T slice: 256 rows x 128 B
constexpr uint32_t kStageBytes = kABytes + kBBytes;
constexpr uint32_t kStagingBytes = kTileM * kChunk * 2;  // one bf16 chunk: 128 rows x 128 B
constexpr uint32_t kEpiOff = kStages * kStageBytes;      // two staging tiles
constexpr uint32_t kBarOff = kEpiOff + 2 * kStagingBytes;
// full[S], empty[S], acc_full[2], acc_empty[2], drain
constexpr int kNumBars = 2 * kStages + 2 + 2 + 1;
constexpr uint32_t kMiscOff = kBarOff + kNumBars * 8;    // TMEM slot, abort flag
constexpr uint32_t kSmem = kMiscOff + 16;
constexpr uint32_t kTmemCols = 512;                      // two 128 x 256 fp32 accumulators
constexpr uint64_t kDrainNs = 1000000000ull;
static_assert(kSmem <= 227 * 1024, "shared memory");
static_assert(kTileN % kChunk == 0 && kTileK * 2 == 128, "tile shape");

// Tile t of the grouped order -> (sample b, token tile mt, feature tile nt).
// Token tiles are numbered over (b, mt); a group is kGroupM consecutive ones
// (fewer in the last group), and inside a group the feature tile varies
// slowest.
struct TileOrder {
  long long m_tiles;  // B * n_mt
  int n_mt, n_nt;
  __device__ __forceinline__ void decode(long long t, int& b, int& mt, int& nt) const {
    const long long per_group = (long long)kGroupM * n_nt;
    const long long g = t / per_group;
    const long long m0 = g * kGroupM;
    const int gm = (int)min((long long)kGroupM, m_tiles - m0);
    const int r = (int)(t - g * per_group);
    nt = r / gm;
    const long long m = m0 + (r - nt * gm);
    b = (int)(m / n_mt);
    mt = (int)(m - (long long)b * n_mt);
  }
};

// AND of p over the `count` threads that reach named barrier `id` (a barrier
// of its own, so every participant gets the same answer).
__device__ __forceinline__ bool bar_and(uint32_t id, uint32_t count, bool p) {
  uint32_t r;
  asm volatile(
      "{\n .reg .pred pi, po;\n setp.ne.u32 pi, %1, 0;\n barrier.red.and.pred po, %2, %3, pi;\n"
      " selp.u32 %0, 1, 0, po;\n}"
      : "=r"(r)
      : "r"((uint32_t)p), "r"(id), "r"(count)
      : "memory");
  return r != 0u;
}

__device__ __forceinline__ void bar_sync(uint32_t id, uint32_t count) {
  asm volatile("barrier.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}

// Element (row, col) of a staged bf16 chunk: row r holds 128 bytes, its
// 16-byte piece k stored at k ^ (r & 7).
__device__ __forceinline__ double staged(const uint8_t* tile, int row, int col) {
  const uint16_t u = *reinterpret_cast<const uint16_t*>(tile + row * 128 + ((((col >> 3) ^ (row & 7))) << 4) +
                                                        (col & 7) * 2);
  return (double)__uint_as_float((uint32_t)u << 16);
}

struct ProjOut {
  __nv_bfloat16* qkv[3];
  double* mean[2];  // Qa, Ka
  float* hi[2];
  float* lo[2];
};

__global__ void __launch_bounds__(kThreads, 1)
    qkv_project_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_w,
                       ProjOut out, int S, int H, int D, int nb, int n_kb, long long n_tiles, TileOrder order,
                       int32_t* __restrict__ status, uint64_t limit_ns) {
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
    tma_prefetch_desc(&tm_x);
    tma_prefetch_desc(&tm_w);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t sbase = smem_u32(smem);

  if (warp == 0) {
    // ---------------------------------------------------------- producer
    if (lane == 0) {
      uint32_t g = 0;  // slices issued by this CTA
      bool ok = true;
      for (long long t = blockIdx.x; t < n_tiles && ok; t += gridDim.x) {
        int b, mt, nt;
        order.decode(t, b, mt, nt);
        for (int kb = 0; kb < n_kb; ++kb, ++g) {
          const uint32_t st = g % kStages, use = g / kStages;
          if (use > 0 && !(ok = mbar_wait(empty + st, (use - 1) & 1, abort_flag, limit_ns))) break;
          uint8_t* dst = smem + st * kStageBytes;
          mbar_expect_tx(full + st, kStageBytes);
          tma_load_3d(dst, &tm_x, full + st, kb * kTileK, mt * kTileM, b);
          tma_load_3d(dst + kABytes, &tm_w, full + st, kb * kTileK, nt * kTileN, 0);
        }
      }
      // let every copy this thread issued land before the CTA exits
      for (uint32_t i = (g > kStages ? g - kStages : 0); i < g; ++i)
        mbar_wait(full + i % kStages, (i / kStages) & 1, nullptr, kDrainNs);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(kTileM, kTileN, 0, 0);
      uint32_t g = 0, lt = 0;
      bool ok = true;
      for (long long t = blockIdx.x; t < n_tiles && ok; t += gridDim.x, ++lt) {
        const uint32_t ab = lt & 1;
        // the epilogue has drained this accumulator's previous tile
        if (lt >= 2 && !(ok = mbar_wait(acc_empty + ab, ((lt >> 1) - 1) & 1, abort_flag, limit_ns))) break;
        tc_fence_after();
        const uint32_t acc = tmem + ab * kTileN;
        for (int kb = 0; kb < n_kb; ++kb, ++g) {
          const uint32_t st = g % kStages;
          if (!(ok = mbar_wait(full + st, (g / kStages) & 1, abort_flag, limit_ns))) break;
          tc_fence_after();
          const uint32_t a_base = sbase + st * kStageBytes, b_base = a_base + kABytes;
#pragma unroll
          for (int kk = 0; kk < kTileK / 16; ++kk)  // 16 bf16 = 32 bytes of the 128-byte row per MMA
            mma_ss(acc, desc_sw128(a_base + kk * 32, 16, 1024), desc_sw128(b_base + kk * 32, 16, 1024), idesc,
                   (kb > 0 || kk > 0) ? 1u : 0u);
          mma_commit(empty + st);
        }
        if (ok) mma_commit(acc_full + ab);
      }
    }
  } else {
    // --------------------------------------------------------- epilogue
    const int et = threadIdx.x - 64;          // 0 .. 127
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;      // token row of the tile == TMEM lane
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    const int HD = H * D;
    uint32_t lt = 0, chunk = 0;
    for (long long t = blockIdx.x; t < n_tiles; t += gridDim.x, ++lt) {
      const uint32_t ab = lt & 1;
      const bool w = mbar_wait(acc_full + ab, (lt >> 1) & 1, abort_flag, limit_ns);
      // all four warps go on or stop together: they meet at named barriers below
      if (!bar_and(1, 128, w)) break;
      tc_fence_after();
      int b, mt, nt;
      order.decode(t, b, mt, nt);
      const uint32_t taddr = tmem + ab * kTileN + lane_off;
#pragma unroll 1
      for (int c = 0; c < kTileN / kChunk; ++c) {
        uint32_t v0[32], v1[32];
        tmem_ld32(taddr + c * kChunk, v0);
        tmem_ld32(taddr + c * kChunk + 32, v1);
        tmem_ld_wait();
        if (c == kTileN / kChunk - 1) {
          // the accumulator is read: the issuer may start the tile after next
          tc_fence_before();
          mbar_arrive(acc_empty + ab);
        }
        const int f0 = nt * kTileN + c * kChunk;  // first output feature of the chunk
        if (f0 >= 3 * HD) continue;               // past the last feature (same for every thread)
        uint8_t* tile = smem + kEpiOff + (chunk & 1) * kStagingBytes;
        ++chunk;
        uint32_t w32[32];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          w32[i] = pack_bf16x2(__uint_as_float(v0[2 * i]), __uint_as_float(v0[2 * i + 1]));
          w32[16 + i] = pack_bf16x2(__uint_as_float(v1[2 * i]), __uint_as_float(v1[2 * i + 1]));
        }
#pragma unroll
        for (int k = 0; k < 8; ++k)
          *reinterpret_cast<uint4*>(tile + row * 128 + ((k ^ (row & 7)) << 4)) =
              make_uint4(w32[4 * k], w32[4 * k + 1], w32[4 * k + 2], w32[4 * k + 3]);
        bar_sync(1, 128);  // the chunk is staged (and the one before it in this buffer was read)
        const int which = f0 / HD, h = (f0 - which * HD) / D, d0 = f0 % D;
        const long long bh = (long long)b * H + h;
        __nv_bfloat16* dst = which == 0 ? out.qkv[0] : which == 1 ? out.qkv[1] : out.qkv[2];
        // this warp's 32 rows: lanes 8 j .. 8 j + 7 store one row's 128 bytes
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int rr = quarter * 32 + 4 * i + (lane >> 3), q16 = lane & 7;
          const int s = mt * kTileM + rr;
          if (s < S) {
            const uint4 val = *reinterpret_cast<const uint4*>(tile + rr * 128 + ((q16 ^ (rr & 7)) << 4));
            *reinterpret_cast<uint4*>(dst + (bh * S + s) * D + d0 + q16 * 8) = val;
          }
        }
        if (which < 2) {
          // block means of Q or K: thread et sums column et % 64 of block et / 64
          // (rows past S are zero and are not counted)
          const int blk = et >> 6, col = et & 63;
          const int i = mt * 2 + blk;
          if (i < nb) {
            const int valid = min(kBlock, S - i * kBlock);
            const uint8_t* base = tile + blk * 64 * 128;
            double acc0 = 0.0, acc1 = 0.0;  // even and odd rows, as the pooling kernel adds them
            if (valid == kBlock) {
#pragma unroll 16
              for (int r = 0; r < kBlock; r += 2) {
                acc0 += staged(base, r, col);
                acc1 += staged(base, r + 1, col);
              }
            } else {
              for (int r = 0; r < valid; ++r) acc0 += staged(base, r, col);
            }
            const double mean = (acc0 + acc1) / (double)valid;
            const float f = (float)mean;
            const float hv = to_tf32(f);
            const long long o = (bh * nb + i) * D + d0 + col;
            (which == 0 ? out.mean[0] : out.mean[1])[o] = mean;
            (which == 0 ? out.hi[0] : out.hi[1])[o] = hv;
            (which == 0 ? out.lo[0] : out.lo[1])[o] = f - hv;
          }
        }
      }
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
    tmem_dealloc(tmem, kTmemCols);
  }
  if (threadIdx.x == 0 && *abort_flag) atomicCAS(status, 0, (int32_t)NABLA_ERR_TIMEOUT);
}

}  // namespace

cudaError_t launch_qkv_project(const Dims& d, int C, const void* x, const void* wt, void* q, void* k, void* v,
                               double* qa, double* ka, float* qhi, float* qlo, float* khi, float* klo,
                               int32_t* status, cudaStream_t st) {
  const int HD = d.H * d.D;
  CUtensorMap tx, tw;
  if (!make_map_bf16_rows(&tx, x, C, d.S, d.B, kTileM) || !make_map_bf16_rows(&tw, wt, C, 3 * HD, 1, kTileN))
    return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(qkv_project_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmem);
  if (e != cudaSuccess) return e;
  TileOrder order;
  order.n_mt = (d.S + kTileM - 1) / kTileM;
  order.n_nt = (3 * HD + kTileN - 1) / kTileN;
  order.m_tiles = (long long)d.B * order.n_mt;
  const long long n_tiles = order.m_tiles * order.n_nt;
  const int grid = (int)std::min<long long>(n_tiles, sm_count());
  ProjOut out;
  out.qkv[0] = (__nv_bfloat16*)q;
  out.qkv[1] = (__nv_bfloat16*)k;
  out.qkv[2] = (__nv_bfloat16*)v;
  out.mean[0] = qa;
  out.mean[1] = ka;
  out.hi[0] = qhi;
  out.hi[1] = khi;
  out.lo[0] = qlo;
  out.lo[1] = klo;
  qkv_project_kernel<<<grid, kThreads, kSmem, st>>>(tx, tw, out, d.S, d.H, d.D, d.nb, (C + kTileK - 1) / kTileK,
                                                    n_tiles, order, status, wait_limit_ns());
  return cudaGetLastError();
}

}  // namespace nabla
