// Mask builder kernels: Algorithm 1 "NABLA Sparse Mask Generation" of
// "∇NABLA: Neighborhood Adaptive Block-Level Attention" (§3.1.2), the STA
// union of §3.1.3, and the index structures the attention kernels walk.
//
//   select_kernel      row softmax of the reduced scores Qa Ka^T / sqrt(D)
//                      (pooling: pool.cu; scores: score_tc.cu), CDF
//                      binarisation, STA OR, bitmask + compact index lists
//   lists_kernel       bitmask -> compact index lists (external masks)
//   transpose_kernel   per key block, the query blocks that attend to it
//   work_kernel        per (b, h): query-block pairs sorted by cost
#include <cuda_bf16.h>
#include <math.h>

#include "internal.cuh"
#include "sm100.cuh"

namespace nabla {
namespace {

constexpr unsigned kFull = 0xffffffffu;

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(kFull, v, off);
  return v;
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) v = fmaxf(v, __shfl_xor_sync(kFull, v, off));
  return v;
}

__device__ __forceinline__ int warp_sum_i(int v) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(kFull, v, off);
  return v;
}

__device__ __forceinline__ unsigned lanemask_lt() {
  unsigned m;
  asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
  return m;
}

// ------------------------------------------------------------------ select
// One warp per row of the reduced map (one query block of one (b, h)); the
// logits L[i][j] = (Qa_i . Ka_j) / sqrt(D) come from the tensor-core score
// GEMM (score_tc.cu).  Per row: max, e_j = exp(L_j - max), s = sum e_j.  Block
// j is kept iff the mass of the entries ranked above it is <= thr * s:
// Algorithm 1's ascending cumulative sum compared with 1 - thr, stated through
// the mass above each entry.  The fp32 cut-off is the smallest float bit
// pattern u with sum_{e_k > u} e_k <= thr * s (binary search; positive floats
// order like their bit patterns), taken on the top 16 bits: the cut-off
// bucket is the smallest 16-bit prefix p with sum_{prefix(e_k) > p} e_k <=
// thr * s.  Entries above the bucket are kept, entries below dropped, and the
// entries of the bucket (relative width <= 2^-7: a handful at a thousand
// blocks per row, up to ~100 at 8,192) are ranked by their fp64 logits (ties:
// higher block index first, as a stable ascending sort leaves them; fp32
// cannot order entries closer than its rounding error) and kept in rank order
// while the mass above them stays <= thr * s; a bucket of more than
// kMaxCand entries is decided in fp32 instead.  Then the STA window is OR-ed in and bits / cnt / idx are
// written.  The row's values live in registers (NPL per lane, nb <= 32 NPL),
// else in the logits buffer.
constexpr int kMaxCand = 128;

struct SelectCtx {
  const double* qa_h;
  const double* ka_h;
  int nb, W;
  float thr;
  int topk;  // > 0: fixed-budget rule, keep the topk largest entries (thr unused)
  const int32_t* coords;  // [nb][3] or null
  int hT, hH, hW;
  int (*cand_j)[kMaxCand];
  float (*cand_e)[kMaxCand];
  double (*cand_lg)[kMaxCand];
};

// fp64 logits Qa_row . Ka_j (unscaled: a positive factor keeps the order) of
// the n <= 32 candidates cand[0..n): one warp-wide dot product each, lane l
// taking dimensions l, l + 32, ...; lane b returns candidate b's logit.  The
// xor butterfly leaves the same sum in every lane.
template <int D>
__device__ __forceinline__ double candidate_logits(const double* __restrict__ qrow,
                                                   const double* __restrict__ ka_h, const int* cand, int n,
                                                   int lane) {
  constexpr int VD = D / 32;
  double qv[VD];
#pragma unroll
  for (int v = 0; v < VD; ++v) qv[v] = qrow[lane + 32 * v];
  double mine = -1e300;
  for (int b0 = 0; b0 < n; b0 += 4) {
    double part[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      part[u] = 0.0;
      if (b0 + u < n) {
        const double* krow = ka_h + (long long)cand[b0 + u] * D;
#pragma unroll
        for (int v = 0; v < VD; ++v) part[u] = fma(qv[v], krow[lane + 32 * v], part[u]);
      }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1)
#pragma unroll
      for (int u = 0; u < 4; ++u) part[u] += __shfl_xor_sync(kFull, part[u], off);
#pragma unroll
    for (int u = 0; u < 4; ++u)
      if (lane == b0 + u) mine = part[u];
  }
  return mine;
}

// Warp-wide selection of one row.  NPL > 0: the row's exponentials live in
// registers, ev[t] for block 32 t + lane (nb <= 32 NPL); NPL == 0: they stay in
// shared memory (Lr).
template <int D, int NPL>
__device__ __forceinline__ void select_row(const SelectCtx& c, float* Lr, int row, uint32_t* brow,
                                           int32_t* irow, int32_t* cntp, int warp, int lane) {
  const int nb = c.nb, W = c.W;
  constexpr int NR = NPL > 0 ? NPL : 1;
  float ev[NR];
  float mx = -INFINITY, s = 0.f;
  if constexpr (NPL > 0) {
#pragma unroll
    for (int t = 0; t < NPL; ++t) {
      const int j = t * 32 + lane;
      ev[t] = (t < W && j < nb) ? Lr[j] : -INFINITY;
      mx = fmaxf(mx, ev[t]);
    }
    mx = warp_max(mx);
#pragma unroll
    for (int t = 0; t < NPL; ++t) {
      ev[t] = (t < W && t * 32 + lane < nb) ? expf(ev[t] - mx) : 0.f;
      s += ev[t];
    }
  } else {
    for (int j = lane; j < nb; j += 32) mx = fmaxf(mx, Lr[j]);
    mx = warp_max(mx);
    for (int j = lane; j < nb; j += 32) {
      const float e = expf(Lr[j] - mx);
      Lr[j] = e;
      s += e;
    }
  }
  s = warp_sum(s);
  // Both rules keep an entry iff the weight of the entries ranked above it is
  // <= limit: weight e and limit thr * s for the CDF rule, weight 1 and limit
  // topk - 1 for the fixed budget (exactly topk entries kept).
  const bool tk = c.topk > 0;
  const float limit = tk ? (float)(min(c.topk, nb) - 1) : c.thr * s;
  // Weight of the entries whose bit pattern, shifted right by `sh`, exceeds u:
  // for e >= 0 that is e > the float whose pattern is u's bucket top.
  auto mass_above = [&](uint32_t u, int sh) -> float {
    const float tv = __uint_as_float((u << sh) | ((1u << sh) - 1u));
    float f[4] = {0.f, 0.f, 0.f, 0.f};  // independent partial sums: short add chains
    if constexpr (NPL > 0) {
#pragma unroll
      for (int t = 0; t < NPL; ++t)
        if (ev[t] > tv) f[t & 3] += tk ? 1.f : ev[t];
    } else {
      for (int j = lane; j < nb; j += 32) {
        const float e = Lr[j];
        if (e > tv) f[0] += tk ? 1.f : e;
      }
    }
    return warp_sum((f[0] + f[1]) + (f[2] + f[3]));
  };
  // Binary search over the top 16 bits of the pattern: the smallest prefix p
  // whose strictly higher prefixes hold mass <= limit.  e_max = 1 has prefix
  // 0x3F80, so the mass above prefix 0x3F80 is 0.  Entries above the cut-off
  // bucket (prefix > p) are kept and entries below it dropped; the entries
  // of bucket p are ranked below.  p == 0 means every block is kept.
  // Lower end: entries at or below u = (1 - thr) s / (2 nb) hold at most
  // nb u = (1 - thr) s / 2 of the mass, so every prefix below prefix(u) still
  // has more than thr s above it (by half the dropped mass, far beyond fp32
  // rounding of the sums) and cannot be the cut-off.
  uint32_t lo = 0u, hi = 0x3F80u;
  if (!tk && c.thr < 1.f) lo = min(__float_as_uint((1.f - c.thr) * s / (float)(2 * nb)) >> 16, hi);
  while (lo < hi) {
    const uint32_t mid = lo + ((hi - lo) >> 1);
    if (mass_above(mid, 16) <= limit) hi = mid; else lo = mid + 1u;
  }
  const uint32_t pcut = lo;
  // 0 keep all, 1 ranked bucket, 2 fp32 rule at bits >= cut32.  The fixed
  // budget ranks bucket 0 too (entries whose e underflowed stay ordered by
  // their logits).
  int mode = (pcut == 0u && !tk) ? 0 : 1;
  uint32_t cut32 = 0u;
  uint64_t keepbits = 0;          // register path: ranked-candidate decisions by t
  if (mode == 1) {
    float above = 0.f;
    int ncand = 0;
    auto visit = [&](int t, float e) {
      const int j = t * 32 + lane;
      const uint32_t pre = __float_as_uint(e) >> 16;
      above += pre > pcut ? (tk ? 1.f : e) : 0.f;
      const bool isc = j < nb && pre == pcut;
      const uint32_t word = __ballot_sync(kFull, isc);
      const int slot = ncand + __popc(word & lanemask_lt());
      if (isc && slot < kMaxCand) {
        c.cand_j[warp][slot] = j;
        c.cand_e[warp][slot] = e;
      }
      ncand += __popc(word);
    };
    if constexpr (NPL > 0) {
#pragma unroll
      for (int t = 0; t < NPL; ++t)
        if (t < W) visit(t, ev[t]);
    } else {
      for (int t = 0; t < W; ++t) visit(t, t * 32 + lane < nb ? Lr[t * 32 + lane] : 0.f);
    }
    above = warp_sum(above);
    __syncwarp();
    if (ncand > kMaxCand) {
      // too many entries in one bucket to rank at once: finish the search on
      // the low 16 bits and keep the fp32 decision bits(e) >= cut32
      uint32_t l2 = pcut << 16, h2 = (pcut << 16) | 0xFFFFu;
      while (l2 < h2) {
        const uint32_t mid = l2 + ((h2 - l2) >> 1);
        if (mass_above(mid, 0) <= limit) h2 = mid; else l2 = mid + 1u;
      }
      cut32 = l2;
      mode = 2;
    } else {
      if (ncand <= 32) {
        // one candidate per lane: fp64 logits and ranking through shuffles
        const bool act = lane < ncand;
        const int cj = act ? c.cand_j[warp][lane] : 0;
        const float ce = act ? c.cand_e[warp][lane] : 0.f;
        const double lg = candidate_logits<D>(c.qa_h + (long long)row * D, c.ka_h, c.cand_j[warp], ncand, lane);
        float mass = above;
        for (int b2 = 0; b2 < ncand; ++b2) {
          const double lb = __shfl_sync(kFull, lg, b2);
          const int jb = __shfl_sync(kFull, cj, b2);
          const float eb = __shfl_sync(kFull, ce, b2);
          if (lb > lg || (lb == lg && jb > cj)) mass += tk ? 1.f : eb;
        }
        const bool kp = act && mass <= limit;
        // hand each candidate's decision to the lane that owns its block
        const uint32_t kmask = __ballot_sync(kFull, kp);
        for (int b2 = 0; b2 < ncand; ++b2) {
          const int jb = __shfl_sync(kFull, cj, b2);
          if ((jb & 31) == lane) {
            const bool kb = (kmask >> b2) & 1u;
            if constexpr (NPL > 0) {
              if (kb) keepbits |= 1ull << (jb >> 5);
            } else {
              Lr[jb] = kb ? 2.f : 0.f;  // 2 sits in a bucket above any e <= 1
            }
          }
        }
      } else {
        // larger buckets (long rows): the same ranking with the candidates'
        // logits in shared memory, 32 candidates at a time
        // fp64 logits of the candidates, 32 at a time (lane b of a group
        // returns candidate b's), kept in shared memory
        const double* qrow = c.qa_h + (long long)row * D;
        for (int c0 = 0; c0 < ncand; c0 += 32) {
          const int nc = min(32, ncand - c0);
          const double lg = candidate_logits<D>(qrow, c.ka_h, c.cand_j[warp] + c0, nc, lane);
          if (lane < nc) c.cand_lg[warp][c0 + lane] = lg;
        }
        __syncwarp();
        // a candidate is kept iff the weight above the bucket plus that of the
        // candidates ranked above it is <= limit
        for (int c0 = 0; c0 < ncand; c0 += 32) {
          const int ci = c0 + lane;
          const bool act = ci < ncand;
          const int cj = act ? c.cand_j[warp][ci] : 0;
          const double lg = act ? c.cand_lg[warp][ci] : 0.0;
          float mass = above;
          for (int b2 = 0; b2 < ncand; ++b2) {
            const double lb = c.cand_lg[warp][b2];
            const int jb = c.cand_j[warp][b2];
            if (lb > lg || (lb == lg && jb > cj)) mass += tk ? 1.f : c.cand_e[warp][b2];
          }
          const bool kp = act && mass <= limit;
          // hand each candidate's decision to the lane that owns its block
          const uint32_t kmask = __ballot_sync(kFull, kp);
          const int nc = min(32, ncand - c0);
          for (int b2 = 0; b2 < nc; ++b2) {
            const int jb = c.cand_j[warp][c0 + b2];
            if ((jb & 31) == lane) {
              const bool kb = (kmask >> b2) & 1u;
              if constexpr (NPL > 0) {
                if (kb) keepbits |= 1ull << (jb >> 5);
              } else {
                Lr[jb] = kb ? 2.f : 0.f;  // 2 sits in a bucket above any e <= 1
              }
            }
          }
        }
      }
      __syncwarp();
    }
  }

  int running = 0;
  const bool use_sta = c.coords != nullptr;
  const int ti = use_sta ? c.coords[3 * row] : 0, yi = use_sta ? c.coords[3 * row + 1] : 0,
            xi = use_sta ? c.coords[3 * row + 2] : 0;
  auto emit = [&](int t, float e, bool ranked_keep) {
    const int j = t * 32 + lane;
    bool keep = false;
    if (j < nb) {
      if (mode == 0) keep = true;
      else if (mode == 1) keep = (__float_as_uint(e) >> 16) > pcut || ranked_keep;
      else keep = __float_as_uint(e) >= cut32;
      if (use_sta && !keep)
        keep = abs(c.coords[3 * j] - ti) <= c.hT && abs(c.coords[3 * j + 1] - yi) <= c.hH &&
               abs(c.coords[3 * j + 2] - xi) <= c.hW;
    }
    const uint32_t word = __ballot_sync(kFull, keep);
    if (lane == 0) brow[t] = word;
    if (keep) irow[running + __popc(word & lanemask_lt())] = j;
    running += __popc(word);
  };
  if constexpr (NPL > 0) {
#pragma unroll
    for (int t = 0; t < NPL; ++t)
      if (t < W) emit(t, ev[t], (keepbits >> t) & 1ull);
  } else {
    for (int t = 0; t < W; ++t) emit(t, t * 32 + lane < nb ? Lr[t * 32 + lane] : 0.f, false);
  }
  if (lane == 0) *cntp = running;
}

// Launched behind the score GEMM with programmatic stream serialization: the
// warp of a row starts once the GEMM has counted all tiles of the row's head
// (and the pooling all its blocks; a bounded wait that runs out records
// NABLA_ERR_TIMEOUT and the row is built from whatever is there).
template <int D, int NPL>
__global__ void __launch_bounds__(256) select_rows_kernel(
    const float* __restrict__ L, int ldl, const double* __restrict__ qa, const double* __restrict__ ka,
    long long rows, int nb, int W, float thr, int topk, const int32_t* __restrict__ coords, int hT, int hH,
    int hW, uint32_t* __restrict__ bits, int32_t* __restrict__ cnt, int32_t* __restrict__ idx,
    const int32_t* __restrict__ counters, int pool_goal, int score_goal, int32_t* __restrict__ status,
    uint64_t limit_ns) {
  __shared__ int cand_j[8][kMaxCand];
  __shared__ float cand_e[8][kMaxCand];
  __shared__ double cand_lg[8][kMaxCand];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const long long grow = (long long)blockIdx.x * 8 + warp;  // (b * H + h) * nb + i
  if (grow >= rows) return;
  const long long bh = grow / nb;
  if (lane == 0) {
    const bool ok = sm100::wait_counter(counters + 2 * bh + 1, score_goal, nullptr, limit_ns) &&
                    sm100::wait_counter(counters + 2 * bh, pool_goal, nullptr, limit_ns);
    if (!ok) atomicCAS(status, 0, (int32_t)NABLA_ERR_TIMEOUT);
  }
  __syncwarp();
  const int row = (int)(grow - bh * nb);
  SelectCtx ctx{qa + bh * nb * D, ka + bh * nb * D, nb, W, thr, topk, coords, hT, hH, hW, cand_j, cand_e, cand_lg};
  float* Lr = const_cast<float*>(L) + grow * ldl;
  uint32_t* brow = bits + grow * W;
  int32_t* irow = idx + grow * nb;
  select_row<D, NPL>(ctx, Lr, row, brow, irow, cnt + grow, warp, lane);
}

template <int D>
cudaError_t launch_select_rows(unsigned grid, cudaStream_t st, const float* L, int ldl, const double* qa,
                               const double* ka, long long rows, int nb, int W, float thr, int topk,
                               const int32_t* coords, int hT, int hH, int hW, uint32_t* bits, int32_t* cnt,
                               int32_t* idx, const int32_t* counters, int pool_goal, int score_goal,
                               int32_t* status) {
  // registers per lane hold ceil(nb / 32) values, rounded up to a few sizes
  auto k = W <= 8 ? select_rows_kernel<D, 8>
         : W <= 16 ? select_rows_kernel<D, 16>
         : W <= 24 ? select_rows_kernel<D, 24>
         : W <= 40 ? select_rows_kernel<D, 40>
         : W <= 64 ? select_rows_kernel<D, 64>
                   : select_rows_kernel<D, 0>;
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(256);
  {
    // the SM keeps its largest shared-memory configuration, so the builder's
    // kernels can be resident side by side
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributePreferredSharedMemoryCarveout,
                                         (int)cudaSharedmemCarveoutMaxShared);
    if (e != cudaSuccess) return e;
  }
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, k, L, ldl, qa, ka, rows, nb, W, thr, topk, coords, hT, hH, hW, bits, cnt, idx,
                            counters, pool_goal, score_goal, status, wait_limit_ns());
}

// ----------------------------------------------------------- STA-only masks
// The sliding-tile mask alone (§2.2, Eq. 5; the STA rows of Table 1): one warp
// per row (b, h, i); bit j is set iff block j lies in the window around block
// i, the same test as the STA union of the selection.  Every row keeps at
// least its own block.
__global__ void __launch_bounds__(256) sta_bits_kernel(const int32_t* __restrict__ coords, long long rows,
                                                       int nb, int W, int hT, int hH, int hW,
                                                       uint32_t* __restrict__ bits) {
  const long long grow = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (grow >= rows) return;  // uniform across the warp
  const int i = (int)(grow % nb);
  const int ti = coords[3 * i], yi = coords[3 * i + 1], xi = coords[3 * i + 2];
  uint32_t* brow = bits + grow * W;
  for (int t = 0; t < W; ++t) {
    const int j = t * 32 + lane;
    const bool keep = j < nb && abs(coords[3 * j] - ti) <= hT && abs(coords[3 * j + 1] - yi) <= hH &&
                      abs(coords[3 * j + 2] - xi) <= hW;
    const uint32_t word = __ballot_sync(kFull, keep);
    if (lane == 0) brow[t] = word;
  }
}

// ------------------------------------------------------ lists from a bitmask
__global__ void __launch_bounds__(256) lists_kernel(const uint32_t* __restrict__ bits, long long rows,
                                                    int nb, int W, int32_t* __restrict__ cnt,
                                                    int32_t* __restrict__ idx) {
  const long long row = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  const uint32_t* brow = bits + row * W;
  int32_t* irow = idx + row * nb;
  int running = 0;
  for (int t = 0; t < W; ++t) {
    const int j = t * 32 + lane;
    uint32_t word = brow[t];
    if (t == W - 1 && (nb & 31)) word &= (1u << (nb & 31)) - 1u;
    if ((word >> lane) & 1u) irow[running + __popc(word & lanemask_lt())] = j;
    running += __popc(word);
  }
  if (lane == 0) cnt[row] = running;
}

// --------------------------------------------------- transposed (CSC) lists
__global__ void __launch_bounds__(256) transpose_kernel(const uint32_t* __restrict__ bits,
                                                        long long cols, int nb, int W,
                                                        int32_t* __restrict__ cnt_t,
                                                        int32_t* __restrict__ idx_t) {
  const long long gcol = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (gcol >= cols) return;
  const long long bh = gcol / nb;
  const int j = (int)(gcol - bh * nb);
  const uint32_t* bm = bits + bh * nb * W + (j >> 5);
  int32_t* irow = idx_t + gcol * nb;
  int running = 0;
  for (int i0 = 0; i0 < nb; i0 += 32) {
    const int i = i0 + lane;
    const bool keep = i < nb && ((bm[(long long)i * W] >> (j & 31)) & 1u);
    const uint32_t word = __ballot_sync(kFull, keep);
    if (keep) irow[running + __popc(word & lanemask_lt())] = i;
    running += __popc(word);
  }
  if (lane == 0) cnt_t[gcol] = running;
}

// ---------------------------------------------------------------- work list
// One CTA per (b, h): cost of each query-block pair = popcount of the union of
// its two rows; bitonic sort of (nb - cost, pair) ascending = cost descending,
// pair ascending among equal costs.
__global__ void __launch_bounds__(1024) work_kernel(const uint32_t* __restrict__ bits, int nb, int W,
                                                    int npairs, int p2, int32_t* __restrict__ work) {
  extern __shared__ unsigned long long keys[];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nwarp = blockDim.x >> 5;
  const long long bh = blockIdx.x;
  const uint32_t* rb = bits + bh * nb * W;
  // costs, four pairs in flight per warp (the bitmask words come from L2)
  for (int p0 = 4 * warp; p0 < npairs; p0 += 4 * nwarp) {
    int c[4] = {0, 0, 0, 0};
    for (int w = lane; w < W; w += 32) {
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int p = p0 + u;
        if (p < npairs) {
          const uint32_t a = rb[(long long)(2 * p) * W + w];
          const uint32_t b = 2 * p + 1 < nb ? rb[(long long)(2 * p + 1) * W + w] : 0u;
          c[u] += __popc(a | b);
        }
      }
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int cu = warp_sum_i(c[u]);
      if (lane == 0 && p0 + u < npairs) keys[p0 + u] = ((unsigned long long)(nb - cu) << 32) | (unsigned)(p0 + u);
    }
  }
  for (int p = npairs + tid; p < p2; p += blockDim.x) keys[p] = ~0ull;
  __syncthreads();
  // ascending bitonic sort of keys[0, p2) (distinct keys: the pair index is
  // in the low word)
  if (p2 <= (int)blockDim.x) {
    // one key per thread in a register: exchanges within a warp by shuffle,
    // across warps through shared memory
    unsigned long long key = tid < p2 ? keys[tid] : ~0ull;
    for (int kk = 2; kk <= p2; kk <<= 1) {
      for (int jj = kk >> 1; jj > 0; jj >>= 1) {
        unsigned long long other;
        if (jj >= 32) {
          __syncthreads();
          keys[tid] = key;
          __syncthreads();
          other = keys[tid ^ jj];
        } else {
          other = __shfl_xor_sync(kFull, key, jj);
        }
        const bool up = (tid & kk) == 0, lower = (tid & jj) == 0;
        key = (lower == up) ? (key < other ? key : other) : (key < other ? other : key);
      }
    }
    __syncthreads();
    keys[tid] = key;
    __syncthreads();
  } else {
    for (int kk = 2; kk <= p2; kk <<= 1) {
      for (int jj = kk >> 1; jj > 0; jj >>= 1) {
        for (int i = tid; i < p2; i += blockDim.x) {
          const int ixj = i ^ jj;
          if (ixj > i) {
            const unsigned long long a = keys[i], b = keys[ixj];
            const bool up = (i & kk) == 0;
            if ((a > b) == up) { keys[i] = b; keys[ixj] = a; }
          }
        }
        __syncthreads();
      }
    }
  }
  for (int r = tid; r < npairs; r += blockDim.x) {
    const unsigned long long key = keys[r];
    const int p = (int)(key & 0xffffffffu);
    const int cost = nb - (int)(key >> 32);
    work[(bh * npairs + r) * 2] = (int32_t)(bh * npairs + p);
    work[(bh * npairs + r) * 2 + 1] = cost;
  }
}

template <typename Kern>
cudaError_t set_smem(Kern k, size_t bytes) {
  if (bytes <= 48 * 1024) return cudaSuccess;
  return cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
}

}  // namespace

cudaError_t launch_select(const Dims& d, const float* L, int ldl, const double* qa, const double* ka,
                          float thr, const nabla_sta* sta, uint32_t* bits, int32_t* cnt, int32_t* idx,
                          const int32_t* counters, int pool_goal, int32_t* status, cudaStream_t st,
                          int topk) {
  const long long rows = d.BH() * d.nb;
  const unsigned grid = (unsigned)((rows + 7) / 8);
  const bool use_sta = sta && sta->block_coords;
  const int32_t* coords = use_sta ? sta->block_coords : nullptr;
  const int hT = use_sta ? sta->wT / 2 : 0, hH = use_sta ? sta->wH / 2 : 0, hW = use_sta ? sta->wW / 2 : 0;
  if (d.D == 128)
    return launch_select_rows<128>(grid, st, L, ldl, qa, ka, rows, d.nb, d.W, thr, topk, coords, hT, hH, hW, bits,
                                   cnt, idx, counters, pool_goal, score_target(d), status);
  return launch_select_rows<64>(grid, st, L, ldl, qa, ka, rows, d.nb, d.W, thr, topk, coords, hT, hH, hW, bits, cnt,
                                idx, counters, pool_goal, score_target(d), status);
}

cudaError_t launch_sta_bits(const Dims& d, const nabla_sta& sta, uint32_t* bits, cudaStream_t st) {
  const long long rows = d.BH() * d.nb;
  const long long blocks = (rows * 32 + 255) / 256;
  sta_bits_kernel<<<(unsigned)blocks, 256, 0, st>>>(sta.block_coords, rows, d.nb, d.W, sta.wT / 2, sta.wH / 2,
                                                    sta.wW / 2, bits);
  return cudaGetLastError();
}

cudaError_t launch_lists_from_bits(const Dims& d, const uint32_t* bits, int32_t* cnt, int32_t* idx,
                                   cudaStream_t st) {
  const long long rows = d.BH() * d.nb;
  const long long blocks = (rows * 32 + 255) / 256;
  lists_kernel<<<(unsigned)blocks, 256, 0, st>>>(bits, rows, d.nb, d.W, cnt, idx);
  return cudaGetLastError();
}

cudaError_t launch_transpose_lists(const Dims& d, const uint32_t* bits, int32_t* cnt_t,
                                   int32_t* idx_t, cudaStream_t st) {
  const long long cols = d.BH() * d.nb;
  const long long blocks = (cols * 32 + 255) / 256;
  transpose_kernel<<<(unsigned)blocks, 256, 0, st>>>(bits, cols, d.nb, d.W, cnt_t, idx_t);
  return cudaGetLastError();
}

cudaError_t launch_work_list(const Dims& d, const uint32_t* bits, int32_t* work, cudaStream_t st) {
  int p2 = 1;
  while (p2 < d.npairs) p2 <<= 1;
  // one key per thread in the register sort (p2 <= 1024), p2 keys otherwise
  const size_t smem = sizeof(unsigned long long) * std::max(p2, 1024);
  cudaError_t e = set_smem(work_kernel, smem);
  if (e != cudaSuccess) return e;
  work_kernel<<<(unsigned)d.BH(), 1024, smem, st>>>(bits, d.nb, d.W, d.npairs, p2, work);
  return cudaGetLastError();
}

}  // namespace nabla
