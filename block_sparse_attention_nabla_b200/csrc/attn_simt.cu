// CUDA-core block-sparse attention in fp32 arithmetic: the forward and
// backward of Eq. 4 ("∇NABLA: Neighborhood Adaptive Block-Level Attention",
// §2.2) restricted to the kept 64 x 64 tiles.  Serves fp32 inputs, where the
// tensor cores would lose precision, and the backward of bf16 inputs.
//
// Forward: one CTA per (b, h, query block); it walks the block's compact list
// of kept key blocks with an online softmax.  Backward: Delta = rowsum(dO * O);
// dK and dV by one CTA per key block walking the transposed lists; dQ by one
// CTA per query block walking the row lists.  Neither uses atomics, so the
// result does not depend on scheduling.
//
// Thread layout of every 64 x 64 tile: thread t owns row t / 4 and the
// columns (t % 4) + 4 m.
#include <cuda_bf16.h>
#include <math.h>

#include "internal.cuh"

namespace nabla {
namespace {

template <typename T> __device__ __forceinline__ float to_f(T x);
template <> __device__ __forceinline__ float to_f<float>(float x) { return x; }
template <> __device__ __forceinline__ float to_f<__nv_bfloat16>(__nv_bfloat16 x) { return __bfloat162float(x); }
template <typename T> __device__ __forceinline__ T from_f(float x);
template <> __device__ __forceinline__ float from_f<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float x) { return __float2bfloat16_rn(x); }

// Loads rows [row0, row0 + 64) of a [S, D] matrix into a [64][D + 1] fp32
// tile; rows at or beyond S become zero.
template <typename T, int D>
__device__ __forceinline__ void load_tile(float* dst, const T* src, int row0, int S) {
  constexpr int LD = D + 1;
  for (int e = threadIdx.x; e < 64 * D; e += blockDim.x) {
    const int r = e / D, c = e % D;
    const int row = row0 + r;
    dst[r * LD + c] = row < S ? to_f(src[(long long)row * D + c]) : 0.f;
  }
}

template <typename T, int D>
__global__ void __launch_bounds__(256) fwd_kernel(const T* __restrict__ q, const T* __restrict__ k,
                                                  const T* __restrict__ v,
                                                  const int32_t* __restrict__ cnt,
                                                  const int32_t* __restrict__ idx, T* __restrict__ o,
                                                  float* __restrict__ lse, int S, int nb, float scale) {
  extern __shared__ float sm[];
  constexpr int LD = D + 1, E = D / 4;
  float* Qs = sm;
  float* Ks = Qs + 64 * LD;
  float* Vs = Ks + 64 * LD;
  float* Ps = Vs + 64 * LD;  // [64][65]
  const long long bh = blockIdx.y;
  const int i = blockIdx.x;
  const int tid = threadIdx.x, r = tid >> 2, part = tid & 3;
  const T* qh = q + bh * S * (long long)D;
  const T* kh = k + bh * S * (long long)D;
  const T* vh = v + bh * S * (long long)D;
  load_tile<T, D>(Qs, qh, i * 64, S);
  float m = -INFINITY, l = 0.f, acc[E];
#pragma unroll
  for (int e = 0; e < E; ++e) acc[e] = 0.f;
  const int n = cnt[bh * nb + i];
  const int32_t* list = idx + (bh * nb + i) * (long long)nb;
  for (int t = 0; t < n; ++t) {
    const int j = list[t];
    __syncthreads();
    load_tile<T, D>(Ks, kh, j * 64, S);
    load_tile<T, D>(Vs, vh, j * 64, S);
    __syncthreads();
    float sc[16], tmax = -INFINITY;
#pragma unroll
    for (int mm = 0; mm < 16; ++mm) {
      const int c = part + 4 * mm;
      float dot = 0.f;
#pragma unroll 8
      for (int d = 0; d < D; ++d) dot = fmaf(Qs[r * LD + d], Ks[c * LD + d], dot);
      dot = j * 64 + c < S ? dot * scale : -INFINITY;
      sc[mm] = dot;
      tmax = fmaxf(tmax, dot);
    }
    tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, 1));
    tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, 2));
    const float mnew = fmaxf(m, tmax);
    const float corr = expf(m - mnew);
    float psum = 0.f;
#pragma unroll
    for (int mm = 0; mm < 16; ++mm) {
      const float p = expf(sc[mm] - mnew);
      Ps[r * 65 + part + 4 * mm] = p;
      psum += p;
    }
    psum += __shfl_xor_sync(0xffffffffu, psum, 1);
    psum += __shfl_xor_sync(0xffffffffu, psum, 2);
    l = l * corr + psum;
    m = mnew;
#pragma unroll
    for (int e = 0; e < E; ++e) acc[e] *= corr;
    __syncwarp();
    for (int c = 0; c < 64; ++c) {
      const float p = Ps[r * 65 + c];
#pragma unroll
      for (int e = 0; e < E; ++e) acc[e] = fmaf(p, Vs[c * LD + part + 4 * e], acc[e]);
    }
  }
  const int row = i * 64 + r;
  if (row < S) {
    const float inv = l > 0.f ? 1.f / l : 0.f;
    T* orow = o + (bh * S + row) * (long long)D;
#pragma unroll
    for (int e = 0; e < E; ++e) orow[part + 4 * e] = from_f<T>(acc[e] * inv);
    if (part == 0 && lse) lse[bh * S + row] = l > 0.f ? m + logf(l) : -INFINITY;
  }
}

// Delta_r = sum_d dO[r][d] * O[r][d], one warp per row; O plus its rounding
// residual when the forward wrote one (bf16 only, o_res may be NULL).
template <typename T, int D>
__global__ void __launch_bounds__(256) delta_kernel(const T* __restrict__ o, const T* __restrict__ o_res,
                                                    const T* __restrict__ dout, float* __restrict__ delta,
                                                    long long rows) {
  const long long row = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  float s = 0.f;
  for (int d = lane; d < D; d += 32) {
    float od = to_f(o[row * D + d]);
    if (o_res) od += to_f(o_res[row * D + d]);
    s = fmaf(od, to_f(dout[row * D + d]), s);
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
  if (lane == 0) delta[row] = s;
}

// Recomputes P and dS = P * (dP - Delta) of one tile into Ps / dSs.
// Qs, dOs hold the query block (rows), Ks, Vs the key block (columns).
template <int D>
__device__ __forceinline__ void tile_p_ds(const float* Qs, const float* dOs, const float* Ks,
                                          const float* Vs, const float* lse_s, const float* dl_s,
                                          float* Ps, float* dSs, int q0, int k0, int S,
                                          float scale) {
  constexpr int LD = D + 1;
  const int tid = threadIdx.x, r = tid >> 2, part = tid & 3;
  const bool rv = q0 + r < S;
#pragma unroll 2
  for (int mm = 0; mm < 16; ++mm) {
    const int c = part + 4 * mm;
    float s = 0.f, dp = 0.f;
#pragma unroll 8
    for (int d = 0; d < D; ++d) {
      s = fmaf(Qs[r * LD + d], Ks[c * LD + d], s);
      dp = fmaf(dOs[r * LD + d], Vs[c * LD + d], dp);
    }
    const float p = (rv && k0 + c < S) ? expf(s * scale - lse_s[r]) : 0.f;
    Ps[r * 65 + c] = p;
    dSs[r * 65 + c] = p * (dp - dl_s[r]);
  }
}

template <typename T, int D>
__global__ void __launch_bounds__(256) dkdv_kernel(
    const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
    const T* __restrict__ dout, const float* __restrict__ lse, const float* __restrict__ delta,
    const int32_t* __restrict__ cnt_t, const int32_t* __restrict__ idx_t, T* __restrict__ dk,
    T* __restrict__ dv, int S, int nb, float scale) {
  extern __shared__ float sm[];
  constexpr int LD = D + 1, E = D / 4;
  float* Ks = sm;
  float* Vs = Ks + 64 * LD;
  float* Qs = Vs + 64 * LD;
  float* dOs = Qs + 64 * LD;
  float* Ps = dOs + 64 * LD;
  float* dSs = Ps + 64 * 65;
  float* lse_s = dSs + 64 * 65;
  float* dl_s = lse_s + 64;
  const long long bh = blockIdx.y;
  const int j = blockIdx.x;
  const int tid = threadIdx.x, c = tid >> 2, part = tid & 3;
  const long long base = bh * S * (long long)D;
  load_tile<T, D>(Ks, k + base, j * 64, S);
  load_tile<T, D>(Vs, v + base, j * 64, S);
  float adk[E], adv[E];
#pragma unroll
  for (int e = 0; e < E; ++e) adk[e] = adv[e] = 0.f;
  const int n = cnt_t[bh * nb + j];
  const int32_t* list = idx_t + (bh * nb + j) * (long long)nb;
  for (int t = 0; t < n; ++t) {
    const int i = list[t];
    __syncthreads();
    load_tile<T, D>(Qs, q + base, i * 64, S);
    load_tile<T, D>(dOs, dout + base, i * 64, S);
    if (tid < 64) {
      const int row = i * 64 + tid;
      lse_s[tid] = row < S ? lse[bh * S + row] : 0.f;
      dl_s[tid] = row < S ? delta[bh * S + row] : 0.f;
    }
    __syncthreads();
    tile_p_ds<D>(Qs, dOs, Ks, Vs, lse_s, dl_s, Ps, dSs, i * 64, j * 64, S, scale);
    __syncthreads();
    for (int rr = 0; rr < 64; ++rr) {
      const float p = Ps[rr * 65 + c], ds = dSs[rr * 65 + c];
#pragma unroll
      for (int e = 0; e < E; ++e) {
        adv[e] = fmaf(p, dOs[rr * LD + part + 4 * e], adv[e]);
        adk[e] = fmaf(ds, Qs[rr * LD + part + 4 * e], adk[e]);
      }
    }
  }
  const int row = j * 64 + c;
  if (row < S) {
#pragma unroll
    for (int e = 0; e < E; ++e) {
      dk[base + (long long)row * D + part + 4 * e] = from_f<T>(adk[e] * scale);
      dv[base + (long long)row * D + part + 4 * e] = from_f<T>(adv[e]);
    }
  }
}

template <typename T, int D>
__global__ void __launch_bounds__(256) dq_kernel(
    const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
    const T* __restrict__ dout, const float* __restrict__ lse, const float* __restrict__ delta,
    const int32_t* __restrict__ cnt, const int32_t* __restrict__ idx, T* __restrict__ dq, int S,
    int nb, float scale) {
  extern __shared__ float sm[];
  constexpr int LD = D + 1, E = D / 4;
  float* Qs = sm;
  float* dOs = Qs + 64 * LD;
  float* Ks = dOs + 64 * LD;
  float* Vs = Ks + 64 * LD;
  float* Ps = Vs + 64 * LD;
  float* dSs = Ps + 64 * 65;
  float* lse_s = dSs + 64 * 65;
  float* dl_s = lse_s + 64;
  const long long bh = blockIdx.y;
  const int i = blockIdx.x;
  const int tid = threadIdx.x, r = tid >> 2, part = tid & 3;
  const long long base = bh * S * (long long)D;
  load_tile<T, D>(Qs, q + base, i * 64, S);
  load_tile<T, D>(dOs, dout + base, i * 64, S);
  if (tid < 64) {
    const int row = i * 64 + tid;
    lse_s[tid] = row < S ? lse[bh * S + row] : 0.f;
    dl_s[tid] = row < S ? delta[bh * S + row] : 0.f;
  }
  float adq[E];
#pragma unroll
  for (int e = 0; e < E; ++e) adq[e] = 0.f;
  const int n = cnt[bh * nb + i];
  const int32_t* list = idx + (bh * nb + i) * (long long)nb;
  for (int t = 0; t < n; ++t) {
    const int j = list[t];
    __syncthreads();
    load_tile<T, D>(Ks, k + base, j * 64, S);
    load_tile<T, D>(Vs, v + base, j * 64, S);
    __syncthreads();
    tile_p_ds<D>(Qs, dOs, Ks, Vs, lse_s, dl_s, Ps, dSs, i * 64, j * 64, S, scale);
    __syncwarp();
    for (int cc = 0; cc < 64; ++cc) {
      const float ds = dSs[r * 65 + cc];
#pragma unroll
      for (int e = 0; e < E; ++e) adq[e] = fmaf(ds, Ks[cc * LD + part + 4 * e], adq[e]);
    }
  }
  const int row = i * 64 + r;
  if (row < S) {
#pragma unroll
    for (int e = 0; e < E; ++e) dq[base + (long long)row * D + part + 4 * e] = from_f<T>(adq[e] * scale);
  }
}

template <typename Kern>
cudaError_t prep(Kern k, size_t bytes) {
  return cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
}

template <typename T, int D>
cudaError_t fwd_t(const Dims& d, const void* q, const void* k, const void* v, const int32_t* cnt,
                  const int32_t* idx, void* o, float* lse, cudaStream_t st) {
  const size_t smem = sizeof(float) * (3 * 64 * (D + 1) + 64 * 65);
  auto kern = fwd_kernel<T, D>;
  cudaError_t e = prep(kern, smem);
  if (e != cudaSuccess) return e;
  kern<<<dim3(d.nb, (unsigned)d.BH()), 256, smem, st>>>((const T*)q, (const T*)k, (const T*)v, cnt,
                                                        idx, (T*)o, lse, d.S, d.nb,
                                                        1.0f / sqrtf((float)D));
  return cudaGetLastError();
}

template <typename T, int D>
cudaError_t bwd_t(const Dims& d, const void* q, const void* k, const void* v, const void* o,
                  const void* o_res, const void* dout, const float* lse, const int32_t* cnt, const int32_t* idx,
                  const int32_t* cnt_t, const int32_t* idx_t, float* delta, void* dq, void* dk,
                  void* dv, cudaStream_t st) {
  const float scale = 1.0f / sqrtf((float)D);
  const long long rows = d.BH() * d.S;
  delta_kernel<T, D><<<(unsigned)((rows * 32 + 255) / 256), 256, 0, st>>>((const T*)o, (const T*)o_res,
                                                                           (const T*)dout, delta, rows);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const size_t smem = sizeof(float) * (4 * 64 * (D + 1) + 2 * 64 * 65 + 128);
  auto k1 = dkdv_kernel<T, D>;
  if ((e = prep(k1, smem)) != cudaSuccess) return e;
  k1<<<dim3(d.nb, (unsigned)d.BH()), 256, smem, st>>>((const T*)q, (const T*)k, (const T*)v,
                                                      (const T*)dout, lse, delta, cnt_t, idx_t,
                                                      (T*)dk, (T*)dv, d.S, d.nb, scale);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  auto k2 = dq_kernel<T, D>;
  if ((e = prep(k2, smem)) != cudaSuccess) return e;
  k2<<<dim3(d.nb, (unsigned)d.BH()), 256, smem, st>>>((const T*)q, (const T*)k, (const T*)v,
                                                      (const T*)dout, lse, delta, cnt, idx, (T*)dq,
                                                      d.S, d.nb, scale);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attn_fwd_simt(const Dims& d, const void* q, const void* k, const void* v,
                                 const int32_t* cnt, const int32_t* idx, void* o, float* lse,
                                 cudaStream_t st) {
  if (d.dtype != NABLA_FP32) return cudaErrorInvalidValue;
  if (d.D == 128) return fwd_t<float, 128>(d, q, k, v, cnt, idx, o, lse, st);
  return fwd_t<float, 64>(d, q, k, v, cnt, idx, o, lse, st);
}

cudaError_t launch_attn_bwd_simt(const Dims& d, const void* q, const void* k, const void* v,
                                 const void* o, const void* o_res, const void* dout, const float* lse,
                                 const int32_t* cnt, const int32_t* idx, const int32_t* cnt_t,
                                 const int32_t* idx_t, float* delta, void* dq, void* dk, void* dv,
                                 cudaStream_t st) {
  if (d.dtype == NABLA_FP32) {
    if (d.D == 128)
      return bwd_t<float, 128>(d, q, k, v, o, o_res, dout, lse, cnt, idx, cnt_t, idx_t, delta, dq, dk, dv, st);
    return bwd_t<float, 64>(d, q, k, v, o, o_res, dout, lse, cnt, idx, cnt_t, idx_t, delta, dq, dk, dv, st);
  }
  if (d.D == 128)
    return bwd_t<__nv_bfloat16, 128>(d, q, k, v, o, o_res, dout, lse, cnt, idx, cnt_t, idx_t, delta, dq, dk, dv, st);
  return bwd_t<__nv_bfloat16, 64>(d, q, k, v, o, o_res, dout, lse, cnt, idx, cnt_t, idx_t, delta, dq, dk, dv, st);
}

}  // namespace nabla
