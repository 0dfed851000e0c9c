// Mask builder kernels: Algorithm 1 "NABLA Sparse Mask Generation" of
// "∇NABLA: Neighborhood Adaptive Block-Level Attention" (§3.1.2), the STA
// union of §3.1.3, and the index structures the attention kernels walk.
//
//   pool_kernel        block averaging of Q and K (reads Q and K once; the
//                      HBM-bound part of the builder)
//   select_kernel      reduced scores Qa Ka^T / sqrt(D), row softmax, CDF
//                      binarisation, STA OR, bitmask + compact index lists
//   lists_kernel       bitmask -> compact index lists (external masks)
//   transpose_kernel   per key block, the query blocks that attend to it
//   work_kernel        per (b, h): query-block pairs sorted by cost
#include <cuda_bf16.h>
#include <math.h>

#include "internal.cuh"

namespace nabla {
namespace {

constexpr unsigned kFull = 0xffffffffu;

__device__ __forceinline__ uint4 ld_stream(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

__device__ __forceinline__ void add_chunk(const uint4& u, float (&acc)[8]) {
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    float2 f = __bfloat1622float2(h[e]);
    acc[2 * e] += f.x;
    acc[2 * e + 1] += f.y;
  }
}

__device__ __forceinline__ void add_chunk(const uint4& u, float (&acc)[4]) {
  acc[0] += __uint_as_float(u.x);
  acc[1] += __uint_as_float(u.y);
  acc[2] += __uint_as_float(u.z);
  acc[3] += __uint_as_float(u.w);
}

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

// ------------------------------------------------------------------ pooling
// One warp per 64-token block of Q or K, no CTA-wide barriers: each lane owns
// one 16-byte column chunk and sums its rows in fp64 from 16-byte loads, eight
// loads in flight per lane; lanes that hold the same chunk for different rows
// are combined by shuffles.  The means are written in fp64 (the selection
// ranks near-equal entries by fp64 logits) and rounded to fp32 (operands of
// the score GEMM).  The tail block divides by its number of valid tokens.
template <typename T, int D>
__global__ void __launch_bounds__(256) pool_kernel(const T* __restrict__ q, const T* __restrict__ k,
                                                   double* __restrict__ qa, double* __restrict__ ka,
                                                   float* __restrict__ qa32, float* __restrict__ ka32,
                                                   int S, int nb, long long per_tensor) {
  constexpr int VE = 16 / sizeof(T);  // elements per 16-byte chunk
  constexpr int CH = D / VE;          // chunks per row (8, 16 or 32)
  constexpr int RPI = 32 / CH;        // rows covered by one warp-wide load
  constexpr int NL = kBlock / RPI;    // loads per lane for a full block
  constexpr int UNR = NL < 8 ? NL : 8;
  const int lane = threadIdx.x & 31;
  const int c = lane % CH, r0 = lane / CH;
  const long long nwarps = (long long)gridDim.x * (blockDim.x >> 5);
  for (long long item = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); item < 2 * per_tensor;
       item += nwarps) {
    const bool isk = item >= per_tensor;
    const long long it = isk ? item - per_tensor : item;  // (b * H + h) * nb + i
    const long long bh = it / nb;
    const int i = (int)(it - bh * nb);
    const T* src = (isk ? k : q) + (bh * S + (long long)i * kBlock) * D + c * VE;
    const int valid = min(kBlock, S - i * kBlock);
    double acc[VE];
#pragma unroll
    for (int e = 0; e < VE; ++e) acc[e] = 0.0;
#pragma unroll
    for (int p0 = 0; p0 < NL; p0 += UNR) {
      uint4 v[UNR];
#pragma unroll
      for (int p = 0; p < UNR; ++p) {
        const int r = r0 + (p0 + p) * RPI;
        v[p] = r < valid ? ld_stream(src + (long long)r * D) : make_uint4(0, 0, 0, 0);
      }
#pragma unroll
      for (int p = 0; p < UNR; ++p) {
        float f[VE];
#pragma unroll
        for (int e = 0; e < VE; ++e) f[e] = 0.f;
        add_chunk(v[p], f);
#pragma unroll
        for (int e = 0; e < VE; ++e) acc[e] += (double)f[e];
      }
    }
#pragma unroll
    for (int off = CH; off < 32; off <<= 1)
#pragma unroll
      for (int e = 0; e < VE; ++e) acc[e] += __shfl_xor_sync(kFull, acc[e], off);
    if (lane < CH) {
      double* dst = (isk ? ka : qa) + it * D + c * VE;
      float* dst32 = (isk ? ka32 : qa32) + it * D + c * VE;
#pragma unroll
      for (int e = 0; e < VE; ++e) {
        const double mean = acc[e] / (double)valid;
        dst[e] = mean;
        dst32[e] = (float)mean;
      }
    }
  }
}

// ------------------------------------------------------------ score + select
// One CTA handles R query blocks of one (b, h).
//   phase 1: L[r][j] = (Qa_r . Ka_j) * (1/sqrt(D)) in fp32 from the fp32
//            pooled vectors, staged in shared memory (the map is never written
//            to HBM); Ka chunks are double-buffered with cp.async;
//   phase 2: one warp per row: max, e_j = exp(L_j - max), s = sum e_j.  Block
//            j is kept iff the mass of the entries ranked above it is
//            <= thr * s: Algorithm 1's ascending cumulative sum compared with
//            1 - thr, stated through the mass above each entry.  The fp32
//            cut-off is the smallest float bit pattern u with
//            sum_{e_k > u} e_k <= thr * s (binary search; positive floats
//            order like their bit patterns).  fp32 cannot order entries whose
//            values differ by less than its rounding error, so the entries
//            within a relative 2^-12 of the cut-off value are ranked again by
//            their fp64 logits (ties: higher block index first, as a stable
//            ascending sort leaves them) and kept in rank order while the mass
//            above them stays <= thr * s;
//   then OR the STA window and emit bits / cnt / idx.
// The row's values live in registers (NPL per lane, nb <= 32 NPL) during the
// search, else in shared memory.
constexpr float kWindow = 1.0f / 4096.0f;
constexpr int kMaxCand = 32;
constexpr int KC = 32;  // Ka rows per GEMM chunk

struct SelectCtx {
  const double* qa_h;
  const double* ka_h;
  int nb, W;
  float thr;
  const int* Ct;
  const int* Cy;
  const int* Cx;
  bool use_sta;
  int hT, hH, hW;
  int (*cand_j)[kMaxCand];
  float (*cand_e)[kMaxCand];
};

template <int D>
__device__ __forceinline__ double logit64(const double* qrow, const double* krow) {
  double dot = 0.0;
#pragma unroll 8
  for (int d = 0; d < D; ++d) dot = fma(qrow[d], krow[d], dot);
  return dot;
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
  const float limit = c.thr * s;
  // e_max = exp(0) = 1, so every entry's bit pattern is <= 0x3F800000 and
  // the mass strictly above 0x3F800001 is 0 <= limit.
  uint32_t lo = 0u, hi = 0x3F800001u;
  while (lo < hi) {
    const uint32_t mid = lo + ((hi - lo) >> 1);
    float f = 0.f;
    if constexpr (NPL > 0) {
#pragma unroll
      for (int t = 0; t < NPL; ++t) f += __float_as_uint(ev[t]) > mid ? ev[t] : 0.f;
    } else {
      for (int j = lane; j < nb; j += 32) {
        const float e = Lr[j];
        f += __float_as_uint(e) > mid ? e : 0.f;
      }
    }
    f = warp_sum(f);
    if (f <= limit) hi = mid; else lo = mid + 1u;
  }

  // Decision: keep everything if lo == 0; otherwise keep e > vhi, drop
  // e < vlo, and settle the candidates in [vlo, vhi] by fp64 rank (or by the
  // fp32 rule bits(e) >= lo when there are more than kMaxCand of them).
  const float vcut = __uint_as_float(lo);
  const float vhi = vcut * (1.f + kWindow), vlo = vcut * (1.f - kWindow);
  int mode = lo == 0u ? 0 : 1;  // 0 keep all, 1 ranked candidates, 2 fp32 rule
  uint64_t keepbits = 0;        // register path: ranked-candidate decisions by t
  if (mode == 1) {
    float above = 0.f;
    int ncand = 0;
    auto visit = [&](int t, float e) {
      const int j = t * 32 + lane;
      above += e > vhi ? e : 0.f;
      const bool isc = j < nb && e >= vlo && e <= vhi;
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
      mode = 2;
    } else {
      const bool act = lane < ncand;
      const int cj = act ? c.cand_j[warp][lane] : 0;
      const float ce = act ? c.cand_e[warp][lane] : 0.f;
      const double lg = act ? logit64<D>(c.qa_h + (long long)row * D, c.ka_h + (long long)cj * D) : -1e300;
      float mass = above;
      for (int b2 = 0; b2 < ncand; ++b2) {
        const double lb = __shfl_sync(kFull, lg, b2);
        const int jb = __shfl_sync(kFull, cj, b2);
        const float eb = __shfl_sync(kFull, ce, b2);
        if (lb > lg || (lb == lg && jb > cj)) mass += eb;
      }
      const bool kp = act && mass <= limit;
      // hand each candidate's decision to the lane that owns its block
      const uint32_t kmask = __ballot_sync(kFull, kp);
      for (int b2 = 0; b2 < ncand; ++b2) {
        const int jb = __shfl_sync(kFull, cj, b2);
        const bool kb = (kmask >> b2) & 1u;
        if (kb && (jb & 31) == lane) {
          if constexpr (NPL > 0) keepbits |= 1ull << (jb >> 5);
          else Lr[jb] = 2.f;  // > vhi: kept by the emission rule below
        } else if (!kb && (jb & 31) == lane) {
          if constexpr (NPL == 0) Lr[jb] = 0.f;
        }
      }
      __syncwarp();
    }
  }

  int running = 0;
  const int ti = c.use_sta ? c.Ct[row] : 0, yi = c.use_sta ? c.Cy[row] : 0, xi = c.use_sta ? c.Cx[row] : 0;
  auto emit = [&](int t, float e, bool ranked_keep) {
    const int j = t * 32 + lane;
    bool keep = false;
    if (j < nb) {
      if (mode == 0) keep = true;
      else if (mode == 1) keep = e > vhi || ranked_keep;
      else keep = __float_as_uint(e) >= lo;
      if (c.use_sta && !keep)
        keep = abs(c.Ct[j] - ti) <= c.hT && abs(c.Cy[j] - yi) <= c.hH && abs(c.Cx[j] - xi) <= c.hW;
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

__device__ __forceinline__ void cp_async16(void* dst, const void* src, bool valid) {
  const uint32_t d = (uint32_t)__cvta_generic_to_shared(dst);
  const int n = valid ? 16 : 0;
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(d), "l"(src), "r"(n) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }

template <int R, int D>
__global__ void __launch_bounds__(256, 1) select_kernel(
    const float* __restrict__ qa32, const float* __restrict__ ka32, const double* __restrict__ qa,
    const double* __restrict__ ka, int nb, int W, int ldl, float thr, float scale,
    const int32_t* __restrict__ coords, int hT, int hH, int hW, uint32_t* __restrict__ bits,
    int32_t* __restrict__ cnt, int32_t* __restrict__ idx) {
  extern __shared__ float4 smem4[];
  constexpr int LD = D + 4;  // padded Qa/Ka row: LD / 4 is odd -> conflict-free float4 rows
  constexpr int RG = R / 2;  // row pairs
  constexpr int CT = 256 / RG;
  constexpr int CPT = KC / CT > 0 ? KC / CT : 1;
  __shared__ int cand_j[8][kMaxCand];
  __shared__ float cand_e[8][kMaxCand];
  float* Ls = reinterpret_cast<float*>(smem4);
  float* Qs = Ls + R * ldl;
  float* Ks = Qs + R * LD;  // two buffers of KC rows
  int* Ct = reinterpret_cast<int*>(Ks + 2 * KC * LD);
  int* Cy = Ct + nb;
  int* Cx = Cy + nb;
  const bool use_sta = coords != nullptr;

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const long long bh = blockIdx.y;
  const int row0 = blockIdx.x * R;
  const float* qa_h = qa32 + bh * nb * D;
  const float* ka_h = ka32 + bh * nb * D;

  auto load_chunk = [&](int c0, int buf) {
    float* dstb = Ks + buf * KC * LD;
    for (int e = tid; e < KC * (D / 4); e += 256) {
      const int r = e / (D / 4), c4 = e % (D / 4);
      const bool ok = c0 + r < nb;
      const float* src = ka_h + (long long)(ok ? c0 + r : 0) * D + c4 * 4;
      cp_async16(dstb + r * LD + c4 * 4, src, ok);
    }
    cp_async_commit();
  };

  for (int e = tid; e < R * (D / 4); e += 256) {
    const int r = e / (D / 4), c4 = e % (D / 4);
    const bool ok = row0 + r < nb;
    cp_async16(Qs + r * LD + c4 * 4, qa_h + (long long)(ok ? row0 + r : 0) * D + c4 * 4, ok);
  }
  load_chunk(0, 0);
  if (use_sta)
    for (int j = tid; j < nb; j += 256) {
      Ct[j] = coords[3 * j];
      Cy[j] = coords[3 * j + 1];
      Cx[j] = coords[3 * j + 2];
    }

  const int tr = tid / CT, tc = tid % CT;
  for (int c0 = 0, buf = 0; c0 < nb; c0 += KC, buf ^= 1) {
    cp_async_wait_all();
    __syncthreads();
    if (c0 + KC < nb) load_chunk(c0 + KC, buf ^ 1);
    const float* Kb = Ks + buf * KC * LD;
    float acc0[CPT], acc1[CPT];
#pragma unroll
    for (int j = 0; j < CPT; ++j) acc0[j] = acc1[j] = 0.f;
    if (tc < KC) {
#pragma unroll 4
      for (int kk = 0; kk < D; kk += 4) {
        const float4 a0 = *reinterpret_cast<const float4*>(Qs + (2 * tr) * LD + kk);
        const float4 a1 = *reinterpret_cast<const float4*>(Qs + (2 * tr + 1) * LD + kk);
#pragma unroll
        for (int j = 0; j < CPT; ++j) {
          const float4 bv = *reinterpret_cast<const float4*>(Kb + (tc + CT * j) * LD + kk);
          acc0[j] = fmaf(a0.x, bv.x, acc0[j]);
          acc0[j] = fmaf(a0.y, bv.y, acc0[j]);
          acc0[j] = fmaf(a0.z, bv.z, acc0[j]);
          acc0[j] = fmaf(a0.w, bv.w, acc0[j]);
          acc1[j] = fmaf(a1.x, bv.x, acc1[j]);
          acc1[j] = fmaf(a1.y, bv.y, acc1[j]);
          acc1[j] = fmaf(a1.z, bv.z, acc1[j]);
          acc1[j] = fmaf(a1.w, bv.w, acc1[j]);
        }
      }
#pragma unroll
      for (int j = 0; j < CPT; ++j) {
        const int col = c0 + tc + CT * j;
        if (col < nb) {
          Ls[(2 * tr) * ldl + col] = acc0[j] * scale;
          Ls[(2 * tr + 1) * ldl + col] = acc1[j] * scale;
        }
      }
    }
    __syncthreads();
  }

  SelectCtx ctx{qa + bh * nb * D, ka + bh * nb * D, nb, W, thr, Ct, Cy, Cx, use_sta, hT, hH, hW, cand_j, cand_e};
  for (int r = warp; r < R; r += 8) {
    const int row = row0 + r;
    if (row >= nb) break;
    float* Lr = Ls + r * ldl;
    const long long grow = bh * nb + row;
    uint32_t* brow = bits + grow * W;
    int32_t* irow = idx + grow * nb;
    if (W <= 16) select_row<D, 16>(ctx, Lr, row, brow, irow, cnt + grow, warp, lane);
    else if (W <= 40) select_row<D, 40>(ctx, Lr, row, brow, irow, cnt + grow, warp, lane);
    else if (W <= 64) select_row<D, 64>(ctx, Lr, row, brow, irow, cnt + grow, warp, lane);
    else select_row<D, 0>(ctx, Lr, row, brow, irow, cnt + grow, warp, lane);
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
  for (int p = warp; p < npairs; p += nwarp) {
    int c = 0;
    const bool has_b = 2 * p + 1 < nb;
    for (int w = lane; w < W; w += 32) {
      const uint32_t a = rb[(long long)(2 * p) * W + w];
      const uint32_t b = has_b ? rb[(long long)(2 * p + 1) * W + w] : 0u;
      c += __popc(a | b);
    }
    c = warp_sum_i(c);
    if (lane == 0) keys[p] = ((unsigned long long)(nb - c) << 32) | (unsigned)p;
  }
  for (int p = npairs + tid; p < p2; p += blockDim.x) keys[p] = ~0ull;
  __syncthreads();
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

int num_sms() {
  static int sms = 0;
  if (!sms) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (sms <= 0) sms = 148;
  }
  return sms;
}

constexpr size_t kSmemLimit = 227 * 1024 - 4096;  // dynamic part; the kernel also has ~2 KB static

template <int R, int D>
size_t select_smem(int nb, int ldl) {
  return sizeof(float) * ((size_t)R * ldl + (size_t)R * (D + 4) + 2 * KC * (D + 4)) + 3 * sizeof(int) * nb;
}

template <int R, int D>
cudaError_t run_select(const Dims& d, const float* qa32, const float* ka32, const double* qa,
                       const double* ka, float thr, const nabla_sta* sta, uint32_t* bits,
                       int32_t* cnt, int32_t* idx, cudaStream_t st, int ldl) {
  const size_t smem = select_smem<R, D>(d.nb, ldl);
  auto kern = select_kernel<R, D>;
  cudaError_t e = set_smem(kern, smem);
  if (e != cudaSuccess) return e;
  const bool use_sta = sta && sta->block_coords;
  dim3 grid((d.nb + R - 1) / R, (unsigned)d.BH());
  kern<<<grid, 256, smem, st>>>(qa32, ka32, qa, ka, d.nb, d.W, ldl, thr, 1.0f / sqrtf((float)d.D),
                                use_sta ? sta->block_coords : nullptr, use_sta ? sta->wT / 2 : 0,
                                use_sta ? sta->wH / 2 : 0, use_sta ? sta->wW / 2 : 0, bits, cnt, idx);
  return cudaGetLastError();
}

template <int D>
cudaError_t select_d(const Dims& d, const float* qa32, const float* ka32, const double* qa,
                     const double* ka, float thr, const nabla_sta* sta, uint32_t* bits,
                     int32_t* cnt, int32_t* idx, cudaStream_t st) {
  const int ldl = (d.nb + 3) & ~3;
  if (select_smem<32, D>(d.nb, ldl) <= kSmemLimit)
    return run_select<32, D>(d, qa32, ka32, qa, ka, thr, sta, bits, cnt, idx, st, ldl);
  if (select_smem<16, D>(d.nb, ldl) <= kSmemLimit)
    return run_select<16, D>(d, qa32, ka32, qa, ka, thr, sta, bits, cnt, idx, st, ldl);
  if (select_smem<8, D>(d.nb, ldl) <= kSmemLimit)
    return run_select<8, D>(d, qa32, ka32, qa, ka, thr, sta, bits, cnt, idx, st, ldl);
  return cudaErrorInvalidConfiguration;
}

}  // namespace

cudaError_t launch_pool(const Dims& d, const void* q, const void* k, double* qa, double* ka,
                        float* qa32, float* ka32, cudaStream_t st) {
  const long long per = d.BH() * d.nb;
  const long long warps = 2 * per;
  const int grid = (int)std::min<long long>((warps + 7) / 8, (long long)num_sms() * 8);
  if (d.dtype == NABLA_BF16) {
    if (d.D == 128)
      pool_kernel<__nv_bfloat16, 128><<<grid, 256, 0, st>>>((const __nv_bfloat16*)q, (const __nv_bfloat16*)k, qa, ka, qa32, ka32, d.S, d.nb, per);
    else
      pool_kernel<__nv_bfloat16, 64><<<grid, 256, 0, st>>>((const __nv_bfloat16*)q, (const __nv_bfloat16*)k, qa, ka, qa32, ka32, d.S, d.nb, per);
  } else {
    if (d.D == 128)
      pool_kernel<float, 128><<<grid, 256, 0, st>>>((const float*)q, (const float*)k, qa, ka, qa32, ka32, d.S, d.nb, per);
    else
      pool_kernel<float, 64><<<grid, 256, 0, st>>>((const float*)q, (const float*)k, qa, ka, qa32, ka32, d.S, d.nb, per);
  }
  return cudaGetLastError();
}

cudaError_t launch_select(const Dims& d, const float* qa32, const float* ka32, const double* qa,
                          const double* ka, float thr, const nabla_sta* sta, uint32_t* bits,
                          int32_t* cnt, int32_t* idx, cudaStream_t st) {
  if (d.D == 128) return select_d<128>(d, qa32, ka32, qa, ka, thr, sta, bits, cnt, idx, st);
  return select_d<64>(d, qa32, ka32, qa, ka, thr, sta, bits, cnt, idx, st);
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
  const size_t smem = sizeof(unsigned long long) * p2;
  cudaError_t e = set_smem(work_kernel, smem);
  if (e != cudaSuccess) return e;
  work_kernel<<<(unsigned)d.BH(), 1024, smem, st>>>(bits, d.nb, d.W, d.npairs, p2, work);
  return cudaGetLastError();
}

}  // namespace nabla
