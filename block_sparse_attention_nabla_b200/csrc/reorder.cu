// Fractal token reordering of "∇NABLA: Neighborhood Adaptive Block-Level
// Attention" (§3.1.1, Figure 3) and its inverse.
//
// A DiT applies the permutation to its token sequence at the input stage, so
// that the P x P spatial patches of every latent frame become contiguous runs
// of tokens (64-token blocks of the mask builder when P = 8), and inverts it at
// the output stage; frames keep their temporal order.  Edge patches of a frame
// whose height or width is not a multiple of P hold their valid tokens,
// row-major.
//
// The kernel is a row gather: output row r takes input row src(r), both rows
// of row_bytes bytes moved with 16-byte loads and stores.  It is bound by HBM
// (each row read once and written once); the index arithmetic is a handful of
// integer divisions per row.  Writes are sequential, reads are whole rows.
#include <cuda_runtime.h>

#include "internal.cuh"

namespace nabla {
namespace {

// Position f of a frame's fractal order -> raster index y * W + x.  A row of
// patches spans P * W tokens (the last one ph * W); inside it each patch to
// the left of column px holds P * ph tokens, and the patch itself pw per row.
__device__ __forceinline__ int raster_of_fractal(int f, int H, int W, int P) {
  const int py = f / (P * W);
  const int rem = f - py * P * W;
  const int ph = min(P, H - py * P);
  const int px = rem / (P * ph);
  const int rem2 = rem - px * P * ph;
  const int pw = min(P, W - px * P);
  const int dy = rem2 / pw;
  const int dx = rem2 - dy * pw;
  return (py * P + dy) * W + px * P + dx;
}

// Raster index y * W + x -> position in the frame's fractal order.
__device__ __forceinline__ int fractal_of_raster(int r, int H, int W, int P) {
  const int y = r / W, x = r - (r / W) * W;
  const int py = y / P, px = x / P;
  const int ph = min(P, H - py * P), pw = min(P, W - px * P);
  return py * P * W + px * P * ph + (y - py * P) * pw + (x - px * P);
}

__device__ __forceinline__ uint4 ld_stream(const uint4* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

// G lanes move one row (G = 32 for rows of >= 32 chunks of 16 bytes, fewer
// for short rows, so that no lane idles); UNR chunks in flight per lane.
template <int UNR>
__global__ void __launch_bounds__(256) reorder_kernel(const uint4* __restrict__ x, uint4* __restrict__ y,
                                                      long long rows, int HW, int H, int W, int P, int vec,
                                                      int G, int inverse) {
  const int lane = threadIdx.x & 31;
  const int gl = lane % G;
  const long long groups_per_cta = (blockDim.x >> 5) * (32 / G);
  const long long ngroups = (long long)gridDim.x * groups_per_cta;
  for (long long r = blockIdx.x * groups_per_cta + (threadIdx.x >> 5) * (32 / G) + lane / G; r < rows;
       r += ngroups) {
    const long long frame = r / HW;
    const int i = (int)(r - frame * HW);
    const int s = inverse ? fractal_of_raster(i, H, W, P) : raster_of_fractal(i, H, W, P);
    const uint4* src = x + (frame * HW + s) * vec;
    uint4* dst = y + r * vec;
    for (int v0 = gl; v0 < vec; v0 += G * UNR) {
      uint4 t[UNR];
#pragma unroll
      for (int u = 0; u < UNR; ++u)
        if (v0 + G * u < vec) t[u] = ld_stream(src + v0 + G * u);
#pragma unroll
      for (int u = 0; u < UNR; ++u)
        if (v0 + G * u < vec) __stcs(dst + v0 + G * u, t[u]);
    }
  }
}

}  // namespace

cudaError_t launch_fractal_reorder(const void* x, void* y, int B, int T, int H, int W, int P,
                                   size_t row_bytes, int inverse, cudaStream_t st) {
  const long long HW = (long long)H * W;
  const long long rows = (long long)B * T * HW;
  const int vec = (int)(row_bytes / 16);
  int G = 1;
  while (G < 32 && G < vec) G <<= 1;
  const long long groups = 8 * (32 / G);  // per 256-thread CTA
  const long long want = (rows + groups - 1) / groups;
  const int grid = (int)std::min<long long>(want, (long long)sm_count() * 8);
  reorder_kernel<8><<<grid, 256, 0, st>>>((const uint4*)x, (uint4*)y, rows, (int)HW, H, W, P, vec, G,
                                          inverse);
  return cudaGetLastError();
}

}  // namespace nabla
