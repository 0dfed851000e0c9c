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
// list (grouped by head so a head's K and V stay in L2, most expensive first)
// and are drawn in list order by a persistent grid of two CTAs per SM: each
// CTA takes the next unit (a global counter) when it is ready for one, so the
// CTAs finish together; one thread issuing tcgen05 MMAs cannot keep the
// tensor core busy with these tile shapes, two can.
//
// Warp roles (224 threads per CTA):
//   warp 0      Q and K producer: draws the next unit and hands its index to
//               the other roles through a 4-slot ring; TMA of the unit's Q tile
//               and of the K tiles
//               of its key blocks (3-deep ring; a slot is refilled as soon as
//               its S = Q K^T completes); it walks the OR of the pair's two
//               bitmask rows (the softmax threads walk the same rows to learn
//               each tile's key block and membership);
//   warp 6      V producer: the same walk, V tiles into a 2-deep ring (a slot
//               is refilled once its O += P V completes);
//   warp 1      TMEM owner and MMA issuer.  S of the next tile is issued before
//               the P V of the current one, into the other of two TMEM S
//               buffers, so the softmax of one tile overlaps the MMAs of its
//               neighbours;
//   warps 2-5   softmax and epilogue, one thread per row: load S, online
//               softmax in the log2 domain, write P (bf16) over S; rescale O
//               only when the running max grows by more than 2^8 (exact after
//               the final division); finally O / l and LSE.
// TMEM columns: [0, 64) S0 / P0, [64, 128) S1 / P1, [128, 128 + D) O.
//
// Residual mode (a caller that trains passes o_res): the softmax threads also
// write P_lo = bf16(P - bf16(P)) into the upper 32 columns of the S buffer, the
// issuer adds O += P_lo V after O += P V, and the epilogue writes, beside the
// bf16 O, its rounding residual bf16(O - bf16(O)).  O + o_res then carries the
// softmax-weighted sum at about 2^-16 relative instead of 2^-9, which the
// backward needs for Delta = rowsum(dO * O) in rows whose softmax is nearly
// one-hot (there dS = P (dP - Delta) cancels).
#include <cuda.h>
#include <cuda_bf16.h>
#include <cudaTypedefs.h>
#include <math.h>

#include "internal.cuh"
#include "sm100.cuh"

namespace nabla {
namespace {

using namespace sm100;

constexpr int kKStages = 3;
constexpr int kVStages = 2;
constexpr int kCtasPerSm = 2;
constexpr int kThreads = 224;
constexpr uint32_t kTmemCols = 256;
constexpr uint32_t kOCol = 128;
constexpr float kRescaleLog2 = 8.0f;
// Units in flight between the producer that draws them and the other roles.
constexpr int kUnitRing = 4;
// Bound of the teardown waits for this CTA's own copies and MMAs in flight;
// independent of the (tunable) limit of the pipeline waits.
constexpr uint64_t kDrainLimitNs = 1000000000ull;

template <int D>
struct FwdLayout {
  static constexpr int kHalves = D / 64;                    // 128-byte swizzle atoms along D
  static constexpr uint32_t kQHalf = 128 * 128;             // bytes: 128 rows x 128 B
  static constexpr uint32_t kKVHalf = 64 * 128;             // bytes: 64 rows x 128 B
  static constexpr uint32_t kQBytes = kHalves * kQHalf;
  static constexpr uint32_t kKVBytes = kHalves * kKVHalf;   // one K or V tile
  static constexpr uint32_t q_off = 0;
  static constexpr uint32_t k_off = q_off + kQBytes;
  static constexpr uint32_t v_off = k_off + kKStages * kKVBytes;
  static constexpr uint32_t bar_off = v_off + kVStages * kKVBytes;
  // q_full, q_empty, k_full[K], k_empty[K], v_full[V], v_empty[V], s_full[2],
  // p_full[2], o_done, o_final, drain, unit_full[R], unit_empty[R]
  static constexpr int kNumBars = 2 + 2 * kKStages + 2 * kVStages + 2 + 2 + 3 + 2 * kUnitRing;
  static constexpr uint32_t misc_off = bar_off + kNumBars * 8;   // TMEM slot, abort flag
  static constexpr uint32_t ids_off = misc_off + 16;             // unit indices [R]
  static constexpr uint32_t bytes = ids_off + 4 * kUnitRing;
};

struct Bars {
  uint64_t *q_full, *q_empty, *k_full, *k_empty, *v_full, *v_empty, *s_full, *p_full, *o_done,
      *o_final, *drain, *unit_full, *unit_empty;
};

// Walks the key blocks of one unit in ascending order: the set bits of the OR
// of the unit's two bitmask rows, with the membership of each.
struct UnitWalk {
  const uint32_t* ra;
  const uint32_t* rb;
  int W;
  template <typename F>
  __device__ __forceinline__ bool run(F&& f) const {
    for (int w = 0; w < W; ++w) {
      const uint32_t wa = ra[w], wb = rb ? rb[w] : 0u;
      uint32_t un = wa | wb;
      while (un) {
        const int bit = __ffs(un) - 1;
        un &= un - 1u;
        const int flags = (int)((wa >> bit) & 1u) | (int)(((wb >> bit) & 1u) << 1);
        if (!f(w * 32 + bit, flags)) return false;
      }
    }
    return true;
  }
};

// The same walk as an iterator, for the softmax threads (which follow the
// producer's order without waiting on it); the next bitmask words are
// fetched one word ahead.
struct WalkIter {
  const uint32_t* ra;
  const uint32_t* rb;
  int W, w;
  uint32_t wa, wb, un, na, nbw;
  __device__ __forceinline__ WalkIter(const uint32_t* a, const uint32_t* b, int W_) : ra(a), rb(b), W(W_), w(0) {
    wa = W > 0 ? ra[0] : 0u;
    wb = (W > 0 && rb) ? rb[0] : 0u;
    un = wa | wb;
    na = W > 1 ? ra[1] : 0u;
    nbw = (W > 1 && rb) ? rb[1] : 0u;
  }
  __device__ __forceinline__ void next(int& j, int& flags) {
    while (un == 0u && w + 1 < W) {
      ++w;
      wa = na;
      wb = nbw;
      un = wa | wb;
      na = w + 1 < W ? ra[w + 1] : 0u;
      nbw = (w + 1 < W && rb) ? rb[w + 1] : 0u;
    }
    const int bit = __ffs(un) - 1;
    un &= un - 1u;
    j = w * 32 + bit;
    flags = (int)((wa >> bit) & 1u) | (int)(((wb >> bit) & 1u) << 1);
  }
};

template <int D, bool kRes>
__global__ void __launch_bounds__(kThreads, kCtasPerSm)
    fwd_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_v, const uint32_t* __restrict__ bits,
                  const int32_t* __restrict__ work, int n_units, int S, int nb, int W, int npairs,
                  float scale_log2, __nv_bfloat16* __restrict__ out, __nv_bfloat16* __restrict__ out_res,
                  float* __restrict__ lse,
                  int32_t* __restrict__ unit_ctr, int32_t* __restrict__ status, uint64_t limit_ns) {
  using L = FwdLayout<D>;
  extern __shared__ __align__(1024) uint8_t smem[];
  // The 128-byte swizzle atoms must start on 1024-byte boundaries.
  if (smem_u32(smem) & 1023u) {
    if (threadIdx.x == 0) atomicCAS(status, 0, (int32_t)NABLA_ERR_UNSUPPORTED);
    return;
  }
  uint64_t* bars = (uint64_t*)(smem + L::bar_off);
  Bars b;
  b.q_full = bars;
  b.q_empty = bars + 1;
  b.k_full = bars + 2;
  b.k_empty = b.k_full + kKStages;
  b.v_full = b.k_empty + kKStages;
  b.v_empty = b.v_full + kVStages;
  b.s_full = b.v_empty + kVStages;
  b.p_full = b.s_full + 2;
  b.o_done = b.p_full + 2;
  b.o_final = b.o_done + 1;
  b.drain = b.o_final + 1;
  b.unit_full = b.drain + 1;
  b.unit_empty = b.unit_full + kUnitRing;
  uint32_t* tmem_slot = (uint32_t*)(smem + L::misc_off);
  volatile int* abort_flag = (volatile int*)(smem + L::misc_off + 4);
  int32_t* unit_ids = (int32_t*)(smem + L::ids_off);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(b.q_full, 1);
    mbar_init(b.q_empty, 1);
    for (int s = 0; s < kKStages; ++s) {
      mbar_init(b.k_full + s, 1);
      mbar_init(b.k_empty + s, 1);
    }
    for (int s = 0; s < kVStages; ++s) {
      mbar_init(b.v_full + s, 1);
      mbar_init(b.v_empty + s, 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(b.s_full + s, 1);
      mbar_init(b.p_full + s, 128);
    }
    mbar_init(b.o_done, 1);
    mbar_init(b.o_final, 1);
    mbar_init(b.drain, 1);
    for (int s = 0; s < kUnitRing; ++s) {
      mbar_init(b.unit_full + s, 1);
      mbar_init(b.unit_empty + s, 2 + 128);  // V producer, MMA issuer, softmax threads
    }
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
    // ---------------------------------------------------- Q and K producer
    if (lane == 0) {
      uint32_t q_iter = 0, g = 0, ku = 0;
      bool ok = true;
      while (ok) {
        // draw the next unit of the work list (-1: none left) and hand its
        // index to the other roles through the ring
        const uint32_t us = ku % kUnitRing;
        if (ku >= kUnitRing && !(ok = mbar_wait(b.unit_empty + us, (ku / kUnitRing - 1) & 1, abort_flag, limit_ns)))
          break;
        const int drawn = atomicAdd(unit_ctr, 1);
        const int u = drawn < n_units ? drawn : -1;
        unit_ids[us] = u;
        mbar_arrive(b.unit_full + us);
        ++ku;
        if (u < 0) break;
        const int unit = work[2 * u];
        const int bh = unit / npairs, p = unit - bh * npairs;
        if (q_iter > 0 && !(ok = mbar_wait(b.q_empty, (q_iter - 1) & 1, abort_flag, limit_ns))) break;
        mbar_expect_tx(b.q_full, L::kQBytes);
#pragma unroll
        for (int h = 0; h < L::kHalves; ++h)
          tma_load_3d(smem + L::q_off + h * L::kQHalf, &tm_q, b.q_full, h * 64, p * 128, bh);
        ++q_iter;
        const uint32_t* ra = bits + ((long long)bh * nb + 2 * p) * W;
        UnitWalk walk{ra, 2 * p + 1 < nb ? ra + W : nullptr, W};
        ok = walk.run([&](int j, int) -> bool {
          const uint32_t ks = g % kKStages, use = g / kKStages;
          if (use > 0 && !mbar_wait(b.k_empty + ks, (use - 1) & 1, abort_flag, limit_ns)) return false;
          mbar_expect_tx(b.k_full + ks, L::kKVBytes);
#pragma unroll
          for (int h = 0; h < L::kHalves; ++h)
            tma_load_3d(smem + L::k_off + ks * L::kKVBytes + h * L::kKVHalf, &tm_k, b.k_full + ks, h * 64,
                        j * 64, bh);
          ++g;
          return true;
        });
      }
      // Let every copy this thread issued land before the CTA exits (the last
      // use of each slot completes after all earlier ones).
      if (q_iter > 0) mbar_wait(b.q_full, (q_iter - 1) & 1, nullptr, kDrainLimitNs);
      for (uint32_t i = (g > kKStages ? g - kKStages : 0); i < g; ++i)
        mbar_wait(b.k_full + i % kKStages, (i / kKStages) & 1, nullptr, kDrainLimitNs);
    }
  } else if (warp == 6) {
    // ------------------------------------------------------------ V producer
    if (lane == 0) {
      uint32_t g = 0, ku = 0;
      bool ok = true;
      while (ok) {
        const uint32_t us = ku % kUnitRing;
        if (!(ok = mbar_wait(b.unit_full + us, (ku / kUnitRing) & 1, abort_flag, limit_ns))) break;
        const int u = unit_ids[us];
        mbar_arrive(b.unit_empty + us);
        ++ku;
        if (u < 0) break;
        const int unit = work[2 * u];
        const int bh = unit / npairs, p = unit - bh * npairs;
        const uint32_t* ra = bits + ((long long)bh * nb + 2 * p) * W;
        UnitWalk walk{ra, 2 * p + 1 < nb ? ra + W : nullptr, W};
        ok = walk.run([&](int j, int) -> bool {
          const uint32_t vs = g % kVStages, use = g / kVStages;
          if (use > 0 && !mbar_wait(b.v_empty + vs, (use - 1) & 1, abort_flag, limit_ns)) return false;
          mbar_expect_tx(b.v_full + vs, L::kKVBytes);
#pragma unroll
          for (int h = 0; h < L::kHalves; ++h)
            tma_load_3d(smem + L::v_off + vs * L::kKVBytes + h * L::kKVHalf, &tm_v, b.v_full + vs, h * 64,
                        j * 64, bh);
          ++g;
          return true;
        });
      }
      for (uint32_t i = (g > kVStages ? g - kVStages : 0); i < g; ++i)
        mbar_wait(b.v_full + i % kVStages, (i / kVStages) & 1, nullptr, kDrainLimitNs);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_s = idesc_bf16_f32(128, 64, 0, 0);
      constexpr uint32_t idesc_o = idesc_bf16_f32(128, D, 0, 1);
      uint32_t g_iter = 0, q_iter = 0;
      bool ok = true;
      uint32_t unit_first = 0;
      auto issue_pv = [&](uint32_t h) -> bool {
        const uint32_t sb = h & 1;
        if (!mbar_wait(b.p_full + sb, (h >> 1) & 1, abort_flag, limit_ns)) return false;
        const uint32_t vs = h % kVStages;
        if (!mbar_wait(b.v_full + vs, (h / kVStages) & 1, abort_flag, limit_ns)) return false;
        tc_fence_after();
        const uint32_t vbase = smem_base + L::v_off + vs * L::kKVBytes;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          const uint64_t bdesc = desc_sw128(vbase + kk * 16 * 128, L::kKVHalf, 1024);
          mma_ts(tmem + kOCol, tmem + sb * 64 + kk * 8, bdesc, idesc_o, (h > unit_first || kk > 0) ? 1u : 0u);
        }
        if constexpr (kRes) {
          // O += P_lo V: the bf16 remainder of P, kept in the S buffer's
          // upper 32 columns, so that O carries P at about 2^-16 relative
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint64_t bdesc = desc_sw128(vbase + kk * 16 * 128, L::kKVHalf, 1024);
            mma_ts(tmem + kOCol, tmem + sb * 64 + 32 + kk * 8, bdesc, idesc_o, 1u);
          }
        }
        mma_commit(b.v_empty + vs);
        mma_commit(b.o_done);
        return true;
      };
      uint32_t ku = 0;
      while (ok) {
        const uint32_t us = ku % kUnitRing;
        if (!(ok = mbar_wait(b.unit_full + us, (ku / kUnitRing) & 1, abort_flag, limit_ns))) break;
        const int u = unit_ids[us];
        mbar_arrive(b.unit_empty + us);
        ++ku;
        if (u < 0) break;
        const uint32_t n = (uint32_t)work[2 * u + 1];
        if (!(ok = mbar_wait(b.q_full, q_iter & 1, abort_flag, limit_ns))) break;
        ++q_iter;
        tc_fence_after();
        unit_first = g_iter;
        const uint32_t qbase = smem_base + L::q_off;
        for (uint32_t t = 0; t < n && ok; ++t) {
          const uint32_t g = g_iter + t, ks = g % kKStages, sb = g & 1;
          if (!(ok = mbar_wait(b.k_full + ks, (g / kKStages) & 1, abort_flag, limit_ns))) break;
          tc_fence_after();
          const uint32_t kbase = smem_base + L::k_off + ks * L::kKVBytes;
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t koff = (kk & 3) * 32;  // 16 bf16 = 32 B inside the 128-B row
            const uint64_t adesc = desc_sw128(qbase + (kk >> 2) * L::kQHalf + koff, 16, 1024);
            const uint64_t bdesc = desc_sw128(kbase + (kk >> 2) * L::kKVHalf + koff, 16, 1024);
            mma_ss(tmem + sb * 64, adesc, bdesc, idesc_s, kk > 0 ? 1u : 0u);
          }
          mma_commit(b.k_empty + ks);
          mma_commit(b.s_full + sb);
          if (t >= 1) ok = issue_pv(g - 1);
        }
        if (ok && n >= 1) ok = issue_pv(g_iter + n - 1);
        // only a unit with tiles signals its O: for one without, the issuer
        // runs ahead of the softmax threads, and two such signals in a row
        // could put o_final two phases past a waiter
        if (ok && n >= 1) mma_commit(b.o_final);
        mma_commit(b.q_empty);
        g_iter += n;
      }
    }
  } else {
    // ------------------------------------------------- softmax + epilogue
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;  // row of the 128-row tile == TMEM lane
    const uint32_t lane_base = tmem + ((uint32_t)(quarter * 32) << 16);
    const int my_flag = row < 64 ? 1 : 2;
    uint32_t g_iter = 0, finals = 0;  // finals: units with tiles, i.e. o_final phases
    bool ok = true;
    uint32_t ku = 0;
    while (ok) {
      const uint32_t us = ku % kUnitRing;
      const bool wu = mbar_wait(b.unit_full + us, (ku / kUnitRing) & 1, abort_flag, limit_ns);
      if (!__all_sync(0xffffffffu, wu)) { ok = false; break; }
      const int u = unit_ids[us];
      mbar_arrive(b.unit_empty + us);
      ++ku;
      if (u < 0) break;
      const int unit = work[2 * u];
      const uint32_t n = (uint32_t)work[2 * u + 1];
      const int bh = unit / npairs, p = unit - bh * npairs;
      const int qrow = p * 128 + row;
      float m = -INFINITY, l = 0.f;
      const uint32_t* ra = bits + ((long long)bh * nb + 2 * p) * W;
      WalkIter walk(ra, 2 * p + 1 < nb ? ra + W : nullptr, W);
      for (uint32_t t = 0; t < n; ++t) {
        const uint32_t g = g_iter + t, sb = g & 1;
        int j, flags;
        walk.next(j, flags);
        const bool w1 = mbar_wait(b.s_full + sb, (g >> 1) & 1, abort_flag, limit_ns);
        if (!__all_sync(0xffffffffu, w1)) { ok = false; break; }
        tc_fence_after();
        // All 32 rows of a warp belong to the same query block of the pair,
        // so `mine` is warp-uniform: a warp whose block did not keep key
        // block j only writes P = 0.
        const bool mine = (flags & my_flag) != 0;
        uint32_t pk[32];
        uint32_t plo[kRes ? 32 : 1];
        float corr = 1.f;
        bool rescale = false;
        if (mine) {
          uint32_t r0[32], r1[32];
          tmem_ld32(lane_base + sb * 64, r0);
          tmem_ld32(lane_base + sb * 64 + 32, r1);
          tmem_ld_wait();
          float sc[64];
#pragma unroll
          for (int c = 0; c < 32; ++c) {
            sc[c] = __uint_as_float(r0[c]);
            sc[c + 32] = __uint_as_float(r1[c]);
          }
          const int kv_lim = (j == nb - 1) ? S - j * 64 : 64;
          if (kv_lim < 64) {
#pragma unroll
            for (int c = 0; c < 64; ++c)
              if (c >= kv_lim) sc[c] = -INFINITY;
          }
          float mx0 = sc[0], mx1 = sc[1];
#pragma unroll
          for (int c = 2; c < 62; c += 4) {
            mx0 = fmax3(mx0, sc[c], sc[c + 1]);
            mx1 = fmax3(mx1, sc[c + 2], sc[c + 3]);
          }
          const float rmax = fmax3(mx0, mx1, fmaxf(sc[62], sc[63])) * scale_log2;
          if (m == -INFINITY) {
            m = rmax;
          } else if (rmax > m + kRescaleLog2) {
            corr = ex2(m - rmax);
            m = rmax;
            rescale = true;
          }
          const uint64_t sc2 = f2pack(scale_log2, scale_log2);
          const uint64_t nm2 = f2pack(-m, -m);
          uint64_t acc2 = f2pack(0.f, 0.f), acc2b = f2pack(0.f, 0.f);
#pragma unroll
          for (int c = 0; c < 32; ++c) {
            float x0, x1;
            f2unpack(ffma2(f2pack(sc[2 * c], sc[2 * c + 1]), sc2, nm2), x0, x1);
            const float p0 = ex2(x0), p1 = ex2(x1);
            if (c & 1) acc2b = fadd2(acc2b, f2pack(p0, p1));
            else acc2 = fadd2(acc2, f2pack(p0, p1));
            pk[c] = pack_bf16x2(p0, p1);
            if constexpr (kRes) {
              // p minus its bf16 value is exact in fp32; its bf16 rounding
              // leaves about 2^-9 of that, i.e. 2^-17 of p
              const float h0 = __uint_as_float(pk[c] << 16), h1 = __uint_as_float(pk[c] & 0xffff0000u);
              plo[c] = pack_bf16x2(p0 - h0, p1 - h1);
            }
          }
          float s0, s1, s2, s3;
          f2unpack(acc2, s0, s1);
          f2unpack(acc2b, s2, s3);
          l = l * corr + ((s0 + s1) + (s2 + s3));
        } else {
#pragma unroll
          for (int c = 0; c < 32; ++c) pk[c] = 0u;
          if constexpr (kRes) {
#pragma unroll
            for (int c = 0; c < 32; ++c) plo[c] = 0u;
          }
        }
        tmem_st32(lane_base + sb * 64, pk);
        if constexpr (kRes) tmem_st32(lane_base + sb * 64 + 32, plo);
        if (__any_sync(0xffffffffu, rescale)) {
          // O must hold the sum over tiles < g before it is scaled.  S of
          // tile g completed, and it was issued after P V of tile g - 2, so
          // o_done has completed phase g - 2 and at most phase g - 1: waiting
          // for the parity of phase g - 1 is unambiguous even though this
          // thread does not wait on o_done every tile.  (rescale implies
          // t >= 1.)
          const bool w3 = mbar_wait(b.o_done, (g - 1) & 1, abort_flag, limit_ns);
          if (!__all_sync(0xffffffffu, w3)) { ok = false; break; }
          tc_fence_after();
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
        }
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(b.p_full + sb);
      }
      if (!ok) break;
      // epilogue: o_final completes once per unit with tiles, after its
      // last P V; a unit without tiles writes O = 0 and LSE = -inf at once
      if (n >= 1) {
        const bool w4 = mbar_wait(b.o_final, finals & 1, abort_flag, limit_ns);
        if (!__all_sync(0xffffffffu, w4)) { ok = false; break; }
        ++finals;
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
        if constexpr (kRes) {
          // the rounding residual O - bf16(O), itself rounded to bf16
          uint4 rkd[4];
          uint32_t* rw = reinterpret_cast<uint32_t*>(rkd);
#pragma unroll
          for (int c = 0; c < 16; ++c) {
            const float o0 = __uint_as_float(ov[2 * c]) * inv, o1 = __uint_as_float(ov[2 * c + 1]) * inv;
            rw[c] = pack_bf16x2(o0 - __uint_as_float(pw[c] << 16), o1 - __uint_as_float(pw[c] & 0xffff0000u));
          }
          if (valid) {
            uint4* dst = reinterpret_cast<uint4*>(out_res + ((long long)bh * S + qrow) * D + c0);
#pragma unroll
            for (int e = 0; e < 4; ++e) dst[e] = rkd[e];
          }
        }
      }
      if (valid && lse) lse[(long long)bh * S + qrow] = l > 0.f ? (m + log2f(l)) * 0.69314718055994531f : -INFINITY;
      tc_fence_before();
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

template <int D, bool kRes>
cudaError_t run(const Dims& d, const void* q, const void* k, const void* v, const uint32_t* bits,
                const int32_t* work, void* o, void* o_res, float* lse, int32_t* ws_header, cudaStream_t st) {
  CUtensorMap tq, tk, tv;
  if (!make_map_bf16(&tq, q, d, 128) || !make_map_bf16(&tk, k, d, 64) || !make_map_bf16(&tv, v, d, 64))
    return cudaErrorInvalidValue;
  const int n_units = (int)(d.BH() * d.npairs);
  const int grid = std::min(n_units, kCtasPerSm * sm_count());
  auto kern = fwd_tc_kernel<D, kRes>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)FwdLayout<D>::bytes);
  if (e != cudaSuccess) return e;
  const float scale_log2 = 1.4426950408889634f / sqrtf((float)D);
  kern<<<grid, kThreads, FwdLayout<D>::bytes, st>>>(tq, tk, tv, bits, work, n_units, d.S, d.nb, d.W,
                                                    d.npairs, scale_log2, (__nv_bfloat16*)o,
                                                    (__nv_bfloat16*)o_res, lse, ws_header + kWsUnitCounter,
                                                    ws_header + kWsStatus, wait_limit_ns());
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attn_fwd_tc(const Dims& d, const void* q, const void* k, const void* v,
                               const uint32_t* bits, const int32_t* work, void* o, void* o_res, float* lse,
                               int32_t* ws_header, cudaStream_t st) {
  if (d.dtype != NABLA_BF16) return cudaErrorInvalidValue;
  if (o_res) {
    if (d.D == 128) return run<128, true>(d, q, k, v, bits, work, o, o_res, lse, ws_header, st);
    return run<64, true>(d, q, k, v, bits, work, o, o_res, lse, ws_header, st);
  }
  if (d.D == 128) return run<128, false>(d, q, k, v, bits, work, o, nullptr, lse, ws_header, st);
  return run<64, false>(d, q, k, v, bits, work, o, nullptr, lse, ws_header, st);
}

}  // namespace nabla
