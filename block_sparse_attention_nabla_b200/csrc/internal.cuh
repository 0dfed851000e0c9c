// Internal declarations shared by the translation units of libnabla.so.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/nabla.h"

namespace nabla {

constexpr int kBlock = 64;         // N of Algorithm 1: tokens per block
constexpr int kMaxBlocks = 8192;   // nb limit (S <= 524,288); keeps per-row state on chip

// Derived sizes of one problem.
struct Dims {
  int B, H, S, D, nb, W, npairs, dtype;
  long long BH() const { return (long long)B * H; }
};

inline Dims make_dims(const nabla_shape& s) {
  Dims d;
  d.B = s.B; d.H = s.H; d.S = s.S; d.D = s.D; d.dtype = s.dtype;
  d.nb = (s.S + kBlock - 1) / kBlock;
  d.W = (d.nb + 31) / 32;
  d.npairs = (d.nb + 1) / 2;
  return d;
}

// Workspace layout: a 256-byte header (status word, scheduler counters), the
// per-(b, h) progress counters through which the builder's kernels hand heads
// on to each other, the
// pooled Qa / Ka in fp64 and as tf32 hi / lo pairs ([B, H, nb, D] each), the
// reduced logits L (fp32 [B, H, nb, ldl], ldl = nb rounded up to 4) and, for
// the backward, the per-row Delta = rowsum(dO * O) (fp32 [B, H, S]) and the
// block-padded per-row LSE / ln 2 and Delta of the tensor-core backward (fp32
// [B, H, nb * 64] each).
struct WsLayout {
  size_t header = 0;
  size_t counters = 0;  // int32 [B * H][2]: pooled items, score tiles (the builder's hand-off), zeroed per call
  size_t qa = 0, ka = 0, qhi = 0, qlo = 0, khi = 0, klo = 0, logits = 0, delta = 0, lse2p = 0, deltap = 0;
  int ldl = 0;
  size_t total = 0;
};

inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

inline WsLayout ws_layout(const Dims& d, bool want_bwd) {
  WsLayout w;
  size_t off = 256;
  w.counters = off; off = align256(off + (size_t)d.BH() * 2 * sizeof(int32_t));
  size_t pooled = (size_t)d.BH() * d.nb * d.D * sizeof(double);
  w.qa = off; off = align256(off + pooled);
  w.ka = off; off = align256(off + pooled);
  w.qhi = off; off = align256(off + pooled / 2);
  w.qlo = off; off = align256(off + pooled / 2);
  w.khi = off; off = align256(off + pooled / 2);
  w.klo = off; off = align256(off + pooled / 2);
  w.ldl = (d.nb + 3) & ~3;
  w.logits = off; off = align256(off + (size_t)d.BH() * d.nb * w.ldl * sizeof(float));
  if (want_bwd) {
    w.delta = off; off = align256(off + (size_t)d.BH() * d.S * sizeof(float));
    w.lse2p = off; off = align256(off + (size_t)d.BH() * d.nb * 64 * sizeof(float));
    w.deltap = off; off = align256(off + (size_t)d.BH() * d.nb * 64 * sizeof(float));
  }
  w.total = off;
  return w;
}

// Header words (int32 index into the workspace).
enum : int { kWsStatus = 0, kWsUnitCounter = 1 };  // both zeroed at the start of every call

uint64_t wait_limit_ns();

// Tensor maps (tmaps.cu).  make_map_bf16: 3-D view {D, S, B*H} of a
// [B, H, S, D] bf16 tensor, box {64, box_rows, 1}, 128-byte swizzle, rows
// beyond S read as zero.  make_map_pooled_f32: view {D, nb, B*H} of a
// [B, H, nb, D] fp32 array, box {32, 128, 1}, 128-byte swizzle.
bool make_map_bf16(CUtensorMap* map, const void* base, const Dims& d, int box_rows);
bool make_map_pooled_f32(CUtensorMap* map, const float* base, const Dims& d);
// make_map_bf16_rows: 3-D view {inner, rows, outer} of a contiguous bf16 array
// (inner a multiple of 8), box {64, box_rows, 1}, 128-byte swizzle; elements
// outside the array read as zero.
bool make_map_bf16_rows(CUtensorMap* map, const void* base, int inner, long long rows, int outer, int box_rows);
int sm_count();

// Records the message nabla_last_error() returns in the calling thread (an
// empty message clears it); status is for the reader's benefit only.
void record_error(nabla_status status, const char* fmt, ...);

// Argument checks shared by the entry points (abi.cu).  Each returns NABLA_OK
// or records a message and returns the error status the header documents.
nabla_status check_shape(const nabla_shape* s);                  // sizes, block, dtype, D, nb, B * H
nabla_status check_tensor(const void* p, const char* name);      // non-NULL, 16-byte aligned
nabla_status check_i32(const void* p, const char* name);         // non-NULL, 4-byte aligned
nabla_status check_mask_out(const nabla_mask* m, bool need_bits);  // required lists present, aligned
// thr in (0, 1] (topk == 0) or topk >= 1, and an optional STA window.
nabla_status check_selection(float thr, int32_t topk, const nabla_sta* sta);

// ---------------------------------------------------------------- launchers
// Each returns the cudaError_t of its launches (cudaSuccess if all enqueued).

// The mask builder is a chain of three kernels launched back to back on one
// stream: pooling, the score GEMM and the selection.  Each of the last two is
// launched with programmatic stream serialization, so it starts while its
// predecessor still runs, and takes a head (b, h) only once the predecessor
// has counted all of that head's work done in `counters` (int32 [B * H][2],
// zeroed before the pooling: [0] pooled items, [1] score tiles).  status: the
// workspace status word (a bounded wait that ran out sets NABLA_ERR_TIMEOUT).
cudaError_t launch_pool(const Dims& d, const void* q, const void* k, double* qa, double* ka,
                        float* qhi, float* qlo, float* khi, float* klo, int32_t* counters, int32_t* status,
                        cudaStream_t st);
// pool_goal: the count of pooled items that marks a head ready, pool_target(d)
// behind the pooling kernel, 0 when the pooled vectors are already in place
// (written by the Eq. 1 projection before the build).
cudaError_t launch_score_gemm(const Dims& d, const float* qhi, const float* qlo, const float* khi,
                              const float* klo, float* L, int ldl, int32_t* counters, int pool_goal,
                              int32_t* status, cudaStream_t st);
// topk > 0 selects the fixed-budget rule (the topk largest entries per row)
// instead of the CDF rule with thr.
cudaError_t launch_select(const Dims& d, const float* L, int ldl, const double* qa, const double* ka,
                          float thr, const nabla_sta* sta, uint32_t* bits, int32_t* cnt, int32_t* idx,
                          const int32_t* counters, int pool_goal, int32_t* status, cudaStream_t st,
                          int topk = 0);
// Targets of the counters: every pooled item is counted once by each of the
// pooling kernel's D / 32 consumer warps, every score tile once by each of the
// GEMM's four epilogue warps.
inline int pool_target(const Dims& d) { return 2 * d.nb * (d.D / 32); }
inline int score_target(const Dims& d) { const int T = (d.nb + 127) / 128; return 4 * T * T; }
// STA-only bitmask (every sample and head): the sliding-tile window alone.
cudaError_t launch_sta_bits(const Dims& d, const nabla_sta& sta, uint32_t* bits, cudaStream_t st);
cudaError_t launch_lists_from_bits(const Dims& d, const uint32_t* bits, int32_t* cnt,
                                   int32_t* idx, cudaStream_t st);
cudaError_t launch_transpose_lists(const Dims& d, const uint32_t* bits, int32_t* cnt_t,
                                   int32_t* idx_t, cudaStream_t st);
cudaError_t launch_work_list(const Dims& d, const uint32_t* bits, int32_t* work, cudaStream_t st);

cudaError_t launch_attn_fwd_simt(const Dims& d, const void* q, const void* k, const void* v,
                                 const int32_t* cnt, const int32_t* idx, void* o, float* lse,
                                 cudaStream_t st);
cudaError_t launch_attn_bwd_simt(const Dims& d, const void* q, const void* k, const void* v,
                                 const void* o, const void* o_res, const void* dout, const float* lse,
                                 const int32_t* cnt, const int32_t* idx, const int32_t* cnt_t,
                                 const int32_t* idx_t, float* delta, void* dq, void* dk, void* dv,
                                 cudaStream_t st);
cudaError_t launch_block_mass(const Dims& d, const void* q, const void* k, float* mass, int32_t* ws_header,
                              cudaStream_t st);
cudaError_t launch_mask_recall(const Dims& d, const float* mass, const uint32_t* bits, float* recall,
                               cudaStream_t st);
cudaError_t launch_fractal_reorder(const void* x, void* y, int B, int T, int H, int W, int P,
                                   size_t row_bytes, int inverse, cudaStream_t st);
// o_res: NULL, or [B, H, S, D] bf16 for the rounding residual of O (residual mode).
cudaError_t launch_attn_fwd_tc(const Dims& d, const void* q, const void* k, const void* v,
                               const uint32_t* bits, const int32_t* work, void* o, void* o_res, float* lse,
                               int32_t* ws_header, cudaStream_t st);

// bf16, D = 128 only.  lse2p / deltap: workspace [B*H][nb*64] fp32 each.
cudaError_t launch_attn_bwd_tc(const Dims& d, const void* q, const void* k, const void* v, const void* o,
                               const void* o_res, const void* dout, const float* lse, const uint32_t* bits, const int32_t* cnt,
                               const int32_t* idx, const int32_t* cnt_t, float* lse2p, float* deltap, void* dq,
                               void* dk, void* dv, int32_t* ws_header, cudaStream_t st);

// Eq. 1 projection with the block pooling fused (qkv_tc.cu): x [B, S, C] and
// wt [3, H D, C] bf16 (C a multiple of 8); q, k, v [B, H, S, D] bf16; the
// pooled Q and K into the builder's workspace arrays (same values as
// launch_pool computes from q and k).
cudaError_t launch_qkv_project(const Dims& d, int C, const void* x, const void* wt, void* q, void* k, void* v,
                               double* qa, double* ka, float* qhi, float* qlo, float* khi, float* klo,
                               int32_t* status, cudaStream_t st);

cudaError_t launch_wait_selftest(int32_t* status, uint64_t limit_ns, cudaStream_t st);

}  // namespace nabla
