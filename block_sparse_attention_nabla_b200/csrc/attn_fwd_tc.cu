// Block-sparse attention forward on the 5th-generation tensor cores (sm_100a).
//
// Computes Eq. 4 of "∇NABLA: Neighborhood Adaptive Block-Level Attention"
// (§2.2), softmax(Q K^T / sqrt(D) + M) V, over the kept 64 x 64 tiles of the
// NABLA mask (§3.1.2-3.1.3) only.
//
// Work unit: a pair of query blocks (2p, 2p + 1) of one (b, h) = a 128-row Q
// tile, so every MMA runs at M = 128.  The unit visits the union of the two
// blocks' kept key blocks in ascending order; rows whose own block did not keep
// a visited key block see it as -inf.  Units come from the mask builder's work
// list (grouped by head so a head's K and V stay in L2, most expensive first);
// the grid is persistent, one CTA per SM, units assigned round-robin.
//
// Warp roles (192 threads):
//   warp 0      TMA producer: Q tile per unit, K and V tiles through an
//               NS-stage ring, plus the (key block, membership) of each stage;
//   warp 1      TMEM owner and MMA issuer: S = Q K^T into one of two TMEM S
//               buffers, then O += P V with P read from TMEM;
//   warps 2-5   softmax and epilogue, one thread per row: load S from TMEM,
//               online softmax in the log2 domain, write P (bf16) over S in
//               TMEM, rescale O only when the running max grows by more than
//               2^8 (exact after the final division), finally O / l and LSE.
// TMEM columns: [0, 64) S0 / P0, [64, 128) S1 / P1, [128, 128 + D) O.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cudaTypedefs.h>
#include <math.h>

#include "internal.cuh"
#include "sm100.cuh"

namespace nabla {
namespace {

using namespace sm100;

constexpr int kStages = 4;
constexpr int kThreads = 192;
constexpr uint32_t kTmemCols = 256;
constexpr uint32_t kOCol = 128;
constexpr float kRescaleLog2 = 8.0f;
// Bound of the teardown waits for this CTA's own copies and MMAs in flight;
// independent of the (tunable) limit of the pipeline waits.
constexpr uint64_t kDrainLimitNs = 1000000000ull;

template <int D>
struct FwdLayout {
  static constexpr int kHalves = D / 64;                    // 128-byte swizzle atoms along D
  static constexpr uint32_t kQHalf = 128 * 128;             // bytes: 128 rows x 128 B
  static constexpr uint32_t kKVHalf = 64 * 128;             // bytes: 64 rows x 128 B
  static constexpr uint32_t kQBytes = kHalves * kQHalf;
  static constexpr uint32_t kKVBytes = kHalves * kKVHalf;
  static constexpr uint32_t q_off = 0;
  static constexpr uint32_t k_off = q_off + kQBytes;
  static constexpr uint32_t v_off = k_off + kStages * kKVBytes;
  static constexpr uint32_t bar_off = v_off + kStages * kKVBytes;
  // barriers: q_full, q_empty, k_full[S], v_full[S], kv_empty[S], s_full[2], p_full[2], o_done, drain
  static constexpr int kNumBars = 2 + 3 * kStages + 2 + 2 + 2;
  static constexpr uint32_t meta_off = bar_off + kNumBars * 8;
  static constexpr uint32_t misc_off = meta_off + kStages * 4;
  static constexpr uint32_t bytes = misc_off + 16;
  static constexpr uint32_t alloc_bytes = bytes + 1024;     // slack for 1024-byte alignment
};

struct Bars {
  uint64_t* q_full;
  uint64_t* q_empty;
  uint64_t* k_full;
  uint64_t* v_full;
  uint64_t* kv_empty;
  uint64_t* s_full;
  uint64_t* p_full;
  uint64_t* o_done;
  uint64_t* drain;
};

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    fwd_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_v, const int32_t* __restrict__ cnt,
                  const int32_t* __restrict__ idx, const int32_t* __restrict__ work, int n_units,
                  int S, int nb, int npairs, float scale_log2, __nv_bfloat16* __restrict__ out,
                  float* __restrict__ lse, int32_t* __restrict__ status, uint64_t limit_ns) {
  using L = FwdLayout<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint64_t* bars = (uint64_t*)(smem + L::bar_off);
  Bars b;
  b.q_full = bars;
  b.q_empty = bars + 1;
  b.k_full = bars + 2;
  b.v_full = b.k_full + kStages;
  b.kv_empty = b.v_full + kStages;
  b.s_full = b.kv_empty + kStages;
  b.p_full = b.s_full + 2;
  b.o_done = b.p_full + 2;
  b.drain = b.o_done + 1;
  volatile int32_t* meta = (volatile int32_t*)(smem + L::meta_off);
  uint32_t* tmem_slot = (uint32_t*)(smem + L::misc_off);
  volatile int* abort_flag = (volatile int*)(smem + L::misc_off + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(b.q_full, 1);
    mbar_init(b.q_empty, 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(b.k_full + s, 1);
      mbar_init(b.v_full + s, 1);
      mbar_init(b.kv_empty + s, 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(b.s_full + s, 1);
      mbar_init(b.p_full + s, 128);
    }
    mbar_init(b.o_done, 1);
    mbar_init(b.drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
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

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      uint32_t kv_iter = 0, q_iter = 0;
      int last_use[kStages];
      for (int s = 0; s < kStages; ++s) last_use[s] = -1;
      bool ok = true;
      for (int u = blockIdx.x; u < n_units && ok; u += gridDim.x) {
        const int unit = work[2 * u];
        const int bh = unit / npairs, p = unit - bh * npairs;
        if (q_iter > 0 && !(ok = mbar_wait(b.q_empty, (q_iter - 1) & 1, abort_flag, limit_ns))) break;
        mbar_expect_tx(b.q_full, L::kQBytes);
#pragma unroll
        for (int h = 0; h < L::kHalves; ++h)
          tma_load_3d(smem + L::q_off + h * L::kQHalf, &tm_q, b.q_full, h * 64, p * 128, bh);
        ++q_iter;
        const long long ra = (long long)bh * nb + 2 * p;
        const int na = cnt[ra];
        const int nbb = (2 * p + 1 < nb) ? cnt[ra + 1] : 0;
        const int32_t* la = idx + ra * nb;
        const int32_t* lb = la + nb;
        int ia = 0, ib = 0;
        while (ia < na || ib < nbb) {
          const int ja = ia < na ? la[ia] : 0x7fffffff;
          const int jb = ib < nbb ? lb[ib] : 0x7fffffff;
          const int j = min(ja, jb);
          const int flags = (ja == j ? 1 : 0) | (jb == j ? 2 : 0);
          ia += ja == j;
          ib += jb == j;
          const uint32_t stage = kv_iter % kStages, use = kv_iter / kStages;
          if (use > 0 && !(ok = mbar_wait(b.kv_empty + stage, (use - 1) & 1, abort_flag, limit_ns))) break;
          meta[stage] = j | (flags << 30);
          mbar_expect_tx(b.k_full + stage, L::kKVBytes);
#pragma unroll
          for (int h = 0; h < L::kHalves; ++h)
            tma_load_3d(smem + L::k_off + stage * L::kKVBytes + h * L::kKVHalf, &tm_k, b.k_full + stage,
                        h * 64, j * 64, bh);
          mbar_expect_tx(b.v_full + stage, L::kKVBytes);
#pragma unroll
          for (int h = 0; h < L::kHalves; ++h)
            tma_load_3d(smem + L::v_off + stage * L::kKVBytes + h * L::kKVHalf, &tm_v, b.v_full + stage,
                        h * 64, j * 64, bh);
          last_use[stage] = (int)use;
          ++kv_iter;
        }
      }
      // Let every copy this thread issued land before the CTA exits.
      if (q_iter > 0) mbar_wait(b.q_full, (q_iter - 1) & 1, nullptr, kDrainLimitNs);
      for (int s = 0; s < kStages; ++s)
        if (last_use[s] >= 0) {
          mbar_wait(b.k_full + s, last_use[s] & 1, nullptr, kDrainLimitNs);
          mbar_wait(b.v_full + s, last_use[s] & 1, nullptr, kDrainLimitNs);
        }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_s = idesc_bf16_f32(128, 64, 0, 0);
      constexpr uint32_t idesc_o = idesc_bf16_f32(128, D, 0, 1);
      uint32_t kv_iter = 0, q_iter = 0, g_iter = 0;
      bool ok = true;
      auto issue_pv = [&](uint32_t t) -> bool {
        const uint32_t g = g_iter + t;
        const uint32_t sb = g & 1;
        if (!mbar_wait(b.p_full + sb, (g >> 1) & 1, abort_flag, limit_ns)) return false;
        const uint32_t kv = kv_iter + t, stage = kv % kStages;
        if (!mbar_wait(b.v_full + stage, (kv / kStages) & 1, abort_flag, limit_ns)) return false;
        tc_fence_after();
        const uint32_t vbase = smem_base + L::v_off + stage * L::kKVBytes;
#pragma unroll
        for (int ks = 0; ks < 4; ++ks) {
          const uint64_t bdesc = desc_sw128(vbase + ks * 16 * 128, L::kKVHalf, 1024);
          mma_ts(tmem + kOCol, tmem + sb * 64 + ks * 8, bdesc, idesc_o, (t > 0 || ks > 0) ? 1u : 0u);
        }
        mma_commit(b.o_done);
        mma_commit(b.kv_empty + stage);
        return true;
      };
      for (int u = blockIdx.x; u < n_units && ok; u += gridDim.x) {
        const uint32_t n = (uint32_t)work[2 * u + 1];
        if (!(ok = mbar_wait(b.q_full, q_iter & 1, abort_flag, limit_ns))) break;
        ++q_iter;
        tc_fence_after();
        for (uint32_t t = 0; t < n && ok; ++t) {
          const uint32_t kv = kv_iter + t, stage = kv % kStages;
          if (!(ok = mbar_wait(b.k_full + stage, (kv / kStages) & 1, abort_flag, limit_ns))) break;
          tc_fence_after();
          const uint32_t sb = (g_iter + t) & 1;
          const uint32_t kbase = smem_base + L::k_off + stage * L::kKVBytes;
          const uint32_t qbase = smem_base + L::q_off;
#pragma unroll
          for (int ks = 0; ks < D / 16; ++ks) {
            const uint32_t koff = (ks & 3) * 32;  // 16 bf16 = 32 B inside the 128-B row
            const uint64_t adesc = desc_sw128(qbase + (ks >> 2) * L::kQHalf + koff, 16, 1024);
            const uint64_t bdesc = desc_sw128(kbase + (ks >> 2) * L::kKVHalf + koff, 16, 1024);
            mma_ss(tmem + sb * 64, adesc, bdesc, idesc_s, ks > 0 ? 1u : 0u);
          }
          mma_commit(b.s_full + sb);
          if (t >= 1) ok = issue_pv(t - 1);
        }
        if (ok && n >= 1) ok = issue_pv(n - 1);
        mma_commit(b.q_empty);
        kv_iter += n;
        g_iter += n;
      }
    }
  } else {
    // ------------------------------------------------- softmax + epilogue
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;  // row of the 128-row tile == TMEM lane
    const uint32_t lane_base = tmem + ((uint32_t)(quarter * 32) << 16);
    uint32_t kv_iter = 0, g_iter = 0;
    bool ok = true;
    for (int u = blockIdx.x; u < n_units && ok; u += gridDim.x) {
      const int unit = work[2 * u];
      const uint32_t n = (uint32_t)work[2 * u + 1];
      const int bh = unit / npairs, p = unit - bh * npairs;
      const int qrow = p * 128 + row;
      const int my_flag = row < 64 ? 1 : 2;
      float m = -INFINITY, l = 0.f;
      for (uint32_t t = 0; t < n; ++t) {
        const uint32_t g = g_iter + t, sb = g & 1;
        const uint32_t kv = kv_iter + t, stage = kv % kStages;
        bool w1 = mbar_wait(b.s_full + sb, (g >> 1) & 1, abort_flag, limit_ns);
        bool w2 = w1 && mbar_wait(b.k_full + stage, (kv / kStages) & 1, abort_flag, limit_ns);
        if (!__all_sync(0xffffffffu, w2)) { ok = false; break; }
        tc_fence_after();
        const int mt = meta[stage];
        const int j = mt & 0x3fffffff;
        const bool mine = ((mt >> 30) & my_flag) != 0;
        const int kv_lim = (j == nb - 1) ? S - j * 64 : 64;
        uint32_t r0[32], r1[32];
        tmem_ld32(lane_base + sb * 64, r0);
        tmem_ld32(lane_base + sb * 64 + 32, r1);
        tmem_ld_wait();
        float s[64];
        float rmax = -INFINITY;
#pragma unroll
        for (int c = 0; c < 32; ++c) {
          s[c] = (mine && c < kv_lim) ? __uint_as_float(r0[c]) * scale_log2 : -INFINITY;
          s[c + 32] = (mine && c + 32 < kv_lim) ? __uint_as_float(r1[c]) * scale_log2 : -INFINITY;
          rmax = fmaxf(rmax, fmaxf(s[c], s[c + 32]));
        }
        float corr = 1.f;
        bool rescale = false;
        if (rmax > -INFINITY) {
          if (m == -INFINITY) {
            m = rmax;
          } else if (rmax > m + kRescaleLog2) {
            corr = ex2(m - rmax);
            m = rmax;
            rescale = true;
          }
        }
        uint32_t pk[32];
        float psum = 0.f;
        if (m == -INFINITY) {
#pragma unroll
          for (int c = 0; c < 32; ++c) pk[c] = 0u;
        } else {
#pragma unroll
          for (int c = 0; c < 32; ++c) {
            const float p0 = ex2(s[2 * c] - m), p1 = ex2(s[2 * c + 1] - m);
            psum += p0 + p1;
            pk[c] = pack_bf16x2(p0, p1);
          }
        }
        l = l * corr + psum;
        tmem_st32(lane_base + sb * 64, pk);
        tmem_st_wait();
        if (t >= 1) {
          const bool w3 = mbar_wait(b.o_done, (g - 1) & 1, abort_flag, limit_ns);
          if (!__all_sync(0xffffffffu, w3)) { ok = false; break; }
          tc_fence_after();
          if (__any_sync(0xffffffffu, rescale)) {
#pragma unroll
            for (int c0 = 0; c0 < D; c0 += 32) {
              uint32_t ov[32];
              tmem_ld32(lane_base + kOCol + c0, ov);
              tmem_ld_wait();
              if (rescale)
#pragma unroll
                for (int c = 0; c < 32; ++c) ov[c] = __float_as_uint(__uint_as_float(ov[c]) * corr);
              tmem_st32(lane_base + kOCol + c0, ov);
            }
            tmem_st_wait();
          }
        }
        tc_fence_before();
        mbar_arrive(b.p_full + sb);
      }
      if (!ok) break;
      // epilogue
      if (n >= 1) {
        const bool w4 = mbar_wait(b.o_done, (g_iter + n - 1) & 1, abort_flag, limit_ns);
        if (!__all_sync(0xffffffffu, w4)) { ok = false; break; }
        tc_fence_after();
      }
      const float inv = l > 0.f ? 1.f / l : 0.f;
      const bool valid = qrow < S;
      __nv_bfloat16* orow = out + ((long long)bh * S + qrow) * D;
#pragma unroll
      for (int c0 = 0; c0 < D; c0 += 32) {
        uint32_t ov[32];
        if (n >= 1) {
          tmem_ld32(lane_base + kOCol + c0, ov);
          tmem_ld_wait();
        } else {
#pragma unroll
          for (int c = 0; c < 32; ++c) ov[c] = 0u;
        }
        uint4 pkd[4];
        uint32_t* pw = reinterpret_cast<uint32_t*>(pkd);
#pragma unroll
        for (int c = 0; c < 16; ++c)
          pw[c] = pack_bf16x2(__uint_as_float(ov[2 * c]) * inv, __uint_as_float(ov[2 * c + 1]) * inv);
        if (valid) {
          uint4* dst = reinterpret_cast<uint4*>(orow + c0);
#pragma unroll
          for (int e = 0; e < 4; ++e) dst[e] = pkd[e];
        }
      }
      if (valid && lse) lse[(long long)bh * S + qrow] = l > 0.f ? (m + log2f(l)) * 0.69314718055994531f : -INFINITY;
      tc_fence_before();
      kv_iter += n;
      g_iter += n;
    }
  }

  // ------------------------------------------------------------- teardown
  __syncthreads();
  if (warp == 1) {
    if (lane == 0) {
      mma_commit(b.drain);
      mbar_wait(b.drain, 0, nullptr, kDrainLimitNs);
    }
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
  if (threadIdx.x == 0 && *abort_flag) atomicCAS(status, 0, (int32_t)NABLA_ERR_TIMEOUT);
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    cudaDriverEntryPointQueryResult q;
    void* p = nullptr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = (PFN_cuTensorMapEncodeTiled_v12000)p;
  }
  return fn;
}

// 3-D view {D, S, B*H} of a [B, H, S, D] bf16 tensor; box {64, rows, 1};
// 128-byte swizzle; rows beyond S read as zero.
bool make_map(CUtensorMap* map, const void* base, const Dims& d, int rows) {
  auto enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[3] = {(cuuint64_t)d.D, (cuuint64_t)d.S, (cuuint64_t)d.BH()};
  cuuint64_t strides[2] = {(cuuint64_t)d.D * 2, (cuuint64_t)d.S * d.D * 2};
  cuuint32_t box[3] = {64, (cuuint32_t)rows, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides,
                   box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

int sm_count() {
  static int n = 0;
  if (!n) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (n <= 0) n = 148;
  }
  return n;
}

template <int D>
cudaError_t run(const Dims& d, const void* q, const void* k, const void* v, const int32_t* cnt,
                const int32_t* idx, const int32_t* work, void* o, float* lse, int32_t* ws_header,
                cudaStream_t st) {
  CUtensorMap tq, tk, tv;
  if (!make_map(&tq, q, d, 128) || !make_map(&tk, k, d, 64) || !make_map(&tv, v, d, 64))
    return cudaErrorInvalidValue;
  const int n_units = (int)(d.BH() * d.npairs);
  const int grid = std::min(n_units, sm_count());
  auto kern = fwd_tc_kernel<D>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)FwdLayout<D>::alloc_bytes);
  if (e != cudaSuccess) return e;
  const float scale_log2 = 1.4426950408889634f / sqrtf((float)D);
  kern<<<grid, kThreads, FwdLayout<D>::alloc_bytes, st>>>(tq, tk, tv, cnt, idx, work, n_units, d.S,
                                                          d.nb, d.npairs, scale_log2,
                                                          (__nv_bfloat16*)o, lse, ws_header + kWsStatus,
                                                          wait_limit_ns());
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attn_fwd_tc(const Dims& d, const void* q, const void* k, const void* v,
                               const int32_t* cnt, const int32_t* idx, const int32_t* work,
                               void* o, float* lse, int32_t* ws_header, cudaStream_t st) {
  if (d.dtype != NABLA_BF16) return cudaErrorInvalidValue;
  if (d.D == 128) return run<128>(d, q, k, v, cnt, idx, work, o, lse, ws_header, st);
  return run<64>(d, q, k, v, cnt, idx, work, o, lse, ws_header, st);
}

}  // namespace nabla
