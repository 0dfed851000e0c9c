// extern "C" entry points of libnabla.so: argument validation, workspace
// layout, kernel dispatch and error reporting.  Declarations and the contract
// of every call are in include/nabla.h.
#include <algorithm>
#include <atomic>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <string>

#include "internal.cuh"

namespace nabla {
namespace {

thread_local std::string g_last_error;
std::atomic<uint64_t> g_wait_limit_ns{0};

nabla_status fail(nabla_status s, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return s;
}

nabla_status cuda_fail(cudaError_t e, const char* what) {
  return fail(NABLA_ERR_CUDA, "%s: %s (%s)", what, cudaGetErrorName(e), cudaGetErrorString(e));
}

bool aligned(const void* p, size_t a) { return ((uintptr_t)p % a) == 0; }

nabla_status check_ws(const Dims& d, bool bwd, const void* ws, size_t bytes) {
  const size_t need = ws_layout(d, bwd).total;
  if (!ws) return fail(NABLA_ERR_WORKSPACE, "workspace is NULL (%zu bytes needed)", need);
  if (!aligned(ws, 256)) return fail(NABLA_ERR_WORKSPACE, "workspace must be 256-byte aligned");
  if (bytes < need)
    return fail(NABLA_ERR_WORKSPACE, "workspace has %zu bytes, %zu needed", bytes, need);
  return NABLA_OK;
}

#define NABLA_TRY(expr)                   \
  do {                                    \
    nabla_status _s = (expr);             \
    if (_s != NABLA_OK) return _s;        \
  } while (0)

#define NABLA_CUDA(expr, what)                      \
  do {                                              \
    cudaError_t _e = (expr);                        \
    if (_e != cudaSuccess) return cuda_fail(_e, what); \
  } while (0)

// Builds cnt / idx is done by the caller; this adds the transposed lists and
// the work list, which both derive from the bitmask.
nabla_status emit_derived(const Dims& d, const uint32_t* bits, const nabla_mask* out,
                          cudaStream_t st) {
  if (out->cnt_t || out->idx_t) {
    NABLA_TRY(check_i32(out->cnt_t, "mask.cnt_t"));
    NABLA_TRY(check_i32(out->idx_t, "mask.idx_t"));
    NABLA_CUDA(launch_transpose_lists(d, bits, out->cnt_t, out->idx_t, st), "transpose lists");
  }
  NABLA_CUDA(launch_work_list(d, bits, out->work, st), "work list");
  return NABLA_OK;
}

nabla_status reset_status(void* ws, cudaStream_t st) {
  NABLA_CUDA(cudaMemsetAsync(ws, 0, 256, st), "clear workspace header");
  return NABLA_OK;
}

}  // namespace

nabla_status check_shape(const nabla_shape* s) {
  if (!s) return fail(NABLA_ERR_INVALID_ARG, "shape is NULL");
  if (s->B < 1 || s->H < 1 || s->S < 1 || s->D < 1)
    return fail(NABLA_ERR_INVALID_ARG, "B, H, S, D must be >= 1 (got %d, %d, %d, %d)", s->B, s->H,
                s->S, s->D);
  if (s->block != kBlock)
    return fail(NABLA_ERR_UNSUPPORTED, "block must be %d (got %d)", kBlock, s->block);
  if (s->dtype != NABLA_BF16 && s->dtype != NABLA_FP32)
    return fail(NABLA_ERR_INVALID_ARG, "dtype must be NABLA_BF16 or NABLA_FP32 (got %d)", s->dtype);
  if (s->D != 64 && s->D != 128)
    return fail(NABLA_ERR_UNSUPPORTED, "head dimension D must be 64 or 128 (got %d)", s->D);
  const long long nb = (s->S + kBlock - 1) / kBlock;
  if (nb > kMaxBlocks)
    return fail(NABLA_ERR_UNSUPPORTED, "S = %d gives %lld blocks; at most %d are supported", s->S,
                nb, kMaxBlocks);
  if ((long long)s->B * s->H > (1ll << 30))
    return fail(NABLA_ERR_UNSUPPORTED, "B * H too large");
  return NABLA_OK;
}

nabla_status check_tensor(const void* p, const char* name) {
  if (!p) return fail(NABLA_ERR_INVALID_ARG, "%s is NULL", name);
  if (!aligned(p, 16)) return fail(NABLA_ERR_INVALID_ARG, "%s is not 16-byte aligned", name);
  return NABLA_OK;
}

nabla_status check_i32(const void* p, const char* name) {
  if (!p) return fail(NABLA_ERR_INVALID_ARG, "%s is NULL", name);
  if (!aligned(p, 4)) return fail(NABLA_ERR_INVALID_ARG, "%s is not 4-byte aligned", name);
  return NABLA_OK;
}

nabla_status check_mask_out(const nabla_mask* m, bool need_bits) {
  if (!m) return fail(NABLA_ERR_INVALID_ARG, "mask is NULL");
  if (need_bits) NABLA_TRY(check_i32(m->bits, "mask.bits"));
  NABLA_TRY(check_i32(m->cnt, "mask.cnt"));
  NABLA_TRY(check_i32(m->idx, "mask.idx"));
  NABLA_TRY(check_i32(m->work, "mask.work"));
  if ((m->cnt_t == nullptr) != (m->idx_t == nullptr))
    return fail(NABLA_ERR_INVALID_ARG, "mask.cnt_t and mask.idx_t must both be set or both NULL");
  return NABLA_OK;
}

nabla_status check_selection(float thr, int32_t topk, const nabla_sta* sta) {
  if (topk < 0) return fail(NABLA_ERR_INVALID_ARG, "topk must be >= 1 (got %d)", topk);
  if (topk == 0 && !(thr > 0.f && thr <= 1.f))
    return fail(NABLA_ERR_INVALID_ARG, "thr must lie in (0, 1] (got %g)", (double)thr);
  if (sta && sta->block_coords) {
    NABLA_TRY(check_i32(sta->block_coords, "sta.block_coords"));
    if (sta->wT < 1 || sta->wH < 1 || sta->wW < 1)
      return fail(NABLA_ERR_INVALID_ARG, "STA window sizes must be >= 1 (got %d, %d, %d)", sta->wT,
                  sta->wH, sta->wW);
  }
  return NABLA_OK;
}

void record_error(nabla_status, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
}

uint64_t wait_limit_ns() {
  const uint64_t v = g_wait_limit_ns.load(std::memory_order_relaxed);
  return v ? v : 2000000000ull;
}

}  // namespace nabla

using namespace nabla;

extern "C" {

int32_t nabla_abi_version(void) { return NABLA_ABI_VERSION; }

const char* nabla_last_error(void) { return g_last_error.c_str(); }

void nabla_set_wait_limit_ns(uint64_t ns) { g_wait_limit_ns.store(ns, std::memory_order_relaxed); }

size_t nabla_workspace_size(const nabla_shape* shape, int32_t want_bwd) {
  if (check_shape(shape) != NABLA_OK) return 0;
  return ws_layout(make_dims(*shape), want_bwd != 0).total;
}

static nabla_status build_mask_impl(const nabla_shape* shape, const void* q, const void* k, float thr,
                                    int32_t topk, const nabla_sta* sta, const nabla_mask* out,
                                    void* workspace, size_t workspace_bytes, nabla_stream_t stream) {
  NABLA_TRY(check_shape(shape));
  const Dims d = make_dims(*shape);
  NABLA_TRY(check_tensor(q, "q"));
  NABLA_TRY(check_tensor(k, "k"));
  NABLA_TRY(check_selection(thr, topk, sta));
  NABLA_TRY(check_mask_out(out, true));
  NABLA_TRY(check_ws(d, false, workspace, workspace_bytes));
  cudaStream_t st = (cudaStream_t)stream;
  const WsLayout L = ws_layout(d, false);
  char* ws = (char*)workspace;
  double* qa = (double*)(ws + L.qa);
  double* ka = (double*)(ws + L.ka);
  float* qhi = (float*)(ws + L.qhi);
  float* qlo = (float*)(ws + L.qlo);
  float* khi = (float*)(ws + L.khi);
  float* klo = (float*)(ws + L.klo);
  float* logits = (float*)(ws + L.logits);
  int32_t* status = (int32_t*)workspace + kWsStatus;
  int32_t* counters = (int32_t*)(ws + L.counters);
  NABLA_TRY(reset_status(workspace, st));
  NABLA_CUDA(cudaMemsetAsync(counters, 0, (size_t)d.BH() * 2 * sizeof(int32_t), st), "clear builder counters");
  NABLA_CUDA(launch_pool(d, q, k, qa, ka, qhi, qlo, khi, klo, counters, status, st), "pooling kernel");
  NABLA_CUDA(launch_score_gemm(d, qhi, qlo, khi, klo, logits, L.ldl, counters, pool_target(d), status, st),
             "score GEMM kernel");
  NABLA_CUDA(launch_select(d, logits, L.ldl, qa, ka, topk ? 1.f : thr, sta, out->bits, out->cnt, out->idx,
                           counters, pool_target(d), status, st, topk),
             "select kernel");
  return emit_derived(d, out->bits, out, st);
}

nabla_status nabla_build_mask(const nabla_shape* shape, const void* q, const void* k, float thr,
                              const nabla_sta* sta, const nabla_mask* out, void* workspace,
                              size_t workspace_bytes, nabla_stream_t stream) {
  g_last_error.clear();
  return build_mask_impl(shape, q, k, thr, 0, sta, out, workspace, workspace_bytes, stream);
}

nabla_status nabla_build_mask_topk(const nabla_shape* shape, const void* q, const void* k, int32_t topk,
                                   const nabla_sta* sta, const nabla_mask* out, void* workspace,
                                   size_t workspace_bytes, nabla_stream_t stream) {
  g_last_error.clear();
  if (topk < 1) return fail(NABLA_ERR_INVALID_ARG, "topk must be >= 1 (got %d)", topk);
  return build_mask_impl(shape, q, k, 1.f, topk, sta, out, workspace, workspace_bytes, stream);
}

nabla_status nabla_qkv_project(const nabla_shape* shape, int32_t C, const void* x, const void* wt, void* q,
                               void* k, void* v, void* workspace, size_t workspace_bytes, nabla_stream_t stream) {
  g_last_error.clear();
  NABLA_TRY(check_shape(shape));
  const Dims d = make_dims(*shape);
  if (d.dtype != NABLA_BF16)
    return fail(NABLA_ERR_UNSUPPORTED, "nabla_qkv_project runs on the tensor cores: bf16 only");
  if (C < 8 || C % 8 != 0) return fail(NABLA_ERR_INVALID_ARG, "C must be a positive multiple of 8 (got %d)", C);
  if (C > (1 << 20)) return fail(NABLA_ERR_UNSUPPORTED, "C = %d is above the limit of 1048576", C);
  NABLA_TRY(check_tensor(x, "x"));
  NABLA_TRY(check_tensor(wt, "wt"));
  NABLA_TRY(check_tensor(q, "q"));
  NABLA_TRY(check_tensor(k, "k"));
  NABLA_TRY(check_tensor(v, "v"));
  NABLA_TRY(check_ws(d, false, workspace, workspace_bytes));
  if ((long long)3 * d.H * d.D > (1ll << 31) - 1)
    return fail(NABLA_ERR_UNSUPPORTED, "3 * H * D = %lld output features is above 2^31 - 1", 3ll * d.H * d.D);
  {
    // the outputs may overlap neither the inputs, each other nor the workspace
    const unsigned long long nqkv = (unsigned long long)d.BH() * d.S * d.D * 2;
    struct Range { const void* p; unsigned long long n; const char* name; } r[6] = {
        {x, (unsigned long long)d.B * d.S * C * 2, "x"}, {wt, 3ull * d.H * d.D * C * 2, "wt"},
        {q, nqkv, "q"}, {k, nqkv, "k"}, {v, nqkv, "v"}, {workspace, workspace_bytes, "workspace"}};
    for (int i = 2; i < 5; ++i)
      for (int j = 0; j < 6; ++j) {
        if (j == i) continue;
        const uintptr_t a = (uintptr_t)r[i].p, b = (uintptr_t)r[j].p;
        if (a < b + r[j].n && b < a + r[i].n)
          return fail(NABLA_ERR_INVALID_ARG, "%s overlaps %s", r[i].name, r[j].name);
      }
  }
  cudaStream_t st = (cudaStream_t)stream;
  const WsLayout L = ws_layout(d, false);
  char* ws = (char*)workspace;
  NABLA_TRY(reset_status(workspace, st));
  NABLA_CUDA(launch_qkv_project(d, C, x, wt, q, k, v, (double*)(ws + L.qa), (double*)(ws + L.ka),
                                (float*)(ws + L.qhi), (float*)(ws + L.qlo), (float*)(ws + L.khi),
                                (float*)(ws + L.klo), (int32_t*)workspace + kWsStatus, st),
             "projection kernel");
  return NABLA_OK;
}

nabla_status nabla_build_mask_pooled(const nabla_shape* shape, float thr, const nabla_sta* sta,
                                     const nabla_mask* out, void* workspace, size_t workspace_bytes,
                                     nabla_stream_t stream) {
  g_last_error.clear();
  NABLA_TRY(check_shape(shape));
  const Dims d = make_dims(*shape);
  NABLA_TRY(check_selection(thr, 0, sta));
  NABLA_TRY(check_mask_out(out, true));
  NABLA_TRY(check_ws(d, false, workspace, workspace_bytes));
  cudaStream_t st = (cudaStream_t)stream;
  const WsLayout L = ws_layout(d, false);
  char* ws = (char*)workspace;
  int32_t* status = (int32_t*)workspace + kWsStatus;
  int32_t* counters = (int32_t*)(ws + L.counters);
  // the pooled vectors are in place: the score GEMM and the selection wait
  // for no pooling (goal 0), only the selection for the GEMM's tiles
  NABLA_CUDA(cudaMemsetAsync(counters, 0, (size_t)d.BH() * 2 * sizeof(int32_t), st), "clear builder counters");
  NABLA_CUDA(launch_score_gemm(d, (const float*)(ws + L.qhi), (const float*)(ws + L.qlo),
                               (const float*)(ws + L.khi), (const float*)(ws + L.klo), (float*)(ws + L.logits),
                               L.ldl, counters, 0, status, st),
             "score GEMM kernel");
  NABLA_CUDA(launch_select(d, (const float*)(ws + L.logits), L.ldl, (const double*)(ws + L.qa),
                           (const double*)(ws + L.ka), thr, sta, out->bits, out->cnt, out->idx, counters, 0, status,
                           st),
             "select kernel");
  return emit_derived(d, out->bits, out, st);
}

nabla_status nabla_fractal_reorder(const void* x, void* y, int32_t B, int32_t T, int32_t H, int32_t W,
                                   int32_t P, size_t row_bytes, int32_t inverse, nabla_stream_t stream) {
  g_last_error.clear();
  NABLA_TRY(check_tensor(x, "x"));
  NABLA_TRY(check_tensor(y, "y"));
  if (B < 1 || T < 1 || H < 1 || W < 1 || P < 1)
    return fail(NABLA_ERR_INVALID_ARG, "B, T, H, W, P must be >= 1 (got %d, %d, %d, %d, %d)", B, T, H, W, P);
  if (row_bytes == 0 || row_bytes % 16 != 0)
    return fail(NABLA_ERR_INVALID_ARG, "row_bytes must be a positive multiple of 16 (got %zu)", row_bytes);
  if (inverse != 0 && inverse != 1) return fail(NABLA_ERR_INVALID_ARG, "inverse must be 0 or 1 (got %d)", inverse);
  if ((long long)H * W > (1ll << 30) || row_bytes / 16 > (1ull << 30))
    return fail(NABLA_ERR_UNSUPPORTED, "frame of %d x %d tokens or rows of %zu bytes too large", H, W, row_bytes);
  const unsigned long long bytes = (unsigned long long)B * T * H * W * row_bytes;
  const uintptr_t xs = (uintptr_t)x, ys = (uintptr_t)y;
  if (xs < ys + bytes && ys < xs + bytes) return fail(NABLA_ERR_INVALID_ARG, "x and y overlap");
  NABLA_CUDA(launch_fractal_reorder(x, y, B, T, H, W, P, row_bytes, inverse, (cudaStream_t)stream),
             "fractal reorder kernel");
  return NABLA_OK;
}

nabla_status nabla_block_mass(const nabla_shape* shape, const void* q, const void* k, float* mass,
                              void* workspace, size_t workspace_bytes, nabla_stream_t stream) {
  g_last_error.clear();
  NABLA_TRY(check_shape(shape));
  const Dims d = make_dims(*shape);
  if (d.dtype != NABLA_BF16)
    return fail(NABLA_ERR_UNSUPPORTED, "nabla_block_mass runs on the tensor cores: bf16 inputs only");
  NABLA_TRY(check_tensor(q, "q"));
  NABLA_TRY(check_tensor(k, "k"));
  NABLA_TRY(check_i32(mass, "mass"));
  if (!workspace || !aligned(workspace, 256) || workspace_bytes < 256)
    return fail(NABLA_ERR_WORKSPACE, "workspace must be >= 256 bytes and 256-byte aligned");
  cudaStream_t st = (cudaStream_t)stream;
  NABLA_TRY(reset_status(workspace, st));
  NABLA_CUDA(launch_block_mass(d, q, k, mass, (int32_t*)workspace, st), "block mass kernel");
  return NABLA_OK;
}

nabla_status nabla_mask_recall(const nabla_shape* shape, const float* mass, const uint32_t* bits,
                               float* recall, nabla_stream_t stream) {
  g_last_error.clear();
  NABLA_TRY(check_shape(shape));
  const Dims d = make_dims(*shape);
  NABLA_TRY(check_i32(mass, "mass"));
  NABLA_TRY(check_i32(bits, "bits"));
  NABLA_TRY(check_i32(recall, "recall"));
  NABLA_CUDA(launch_mask_recall(d, mass, bits, recall, (cudaStream_t)stream), "recall kernel");
  return NABLA_OK;
}

nabla_status nabla_build_sta_mask(const nabla_shape* shape, const nabla_sta* sta, const nabla_mask* out,
                                  nabla_stream_t stream) {
  g_last_error.clear();
  NABLA_TRY(check_shape(shape));
  const Dims d = make_dims(*shape);
  if (!sta || !sta->block_coords) return fail(NABLA_ERR_INVALID_ARG, "sta and sta->block_coords are required");
  NABLA_TRY(check_i32(sta->block_coords, "sta.block_coords"));
  if (sta->wT < 1 || sta->wH < 1 || sta->wW < 1)
    return fail(NABLA_ERR_INVALID_ARG, "STA window sizes must be >= 1 (got %d, %d, %d)", sta->wT, sta->wH,
                sta->wW);
  NABLA_TRY(check_mask_out(out, true));
  cudaStream_t st = (cudaStream_t)stream;
  NABLA_CUDA(launch_sta_bits(d, *sta, out->bits, st), "STA mask kernel");
  NABLA_CUDA(launch_lists_from_bits(d, out->bits, out->cnt, out->idx, st), "lists kernel");
  return emit_derived(d, out->bits, out, st);
}

nabla_status nabla_mask_from_bits(const nabla_shape* shape, const uint32_t* bits,
                                  const nabla_mask* out, void* workspace, size_t workspace_bytes,
                                  nabla_stream_t stream) {
  g_last_error.clear();
  NABLA_TRY(check_shape(shape));
  const Dims d = make_dims(*shape);
  NABLA_TRY(check_i32(bits, "bits"));
  NABLA_TRY(check_mask_out(out, false));
  NABLA_TRY(check_ws(d, false, workspace, workspace_bytes));
  cudaStream_t st = (cudaStream_t)stream;
  NABLA_TRY(reset_status(workspace, st));
  NABLA_CUDA(launch_lists_from_bits(d, bits, out->cnt, out->idx, st), "lists kernel");
  return emit_derived(d, bits, out, st);
}

nabla_status nabla_attn_fwd(const nabla_shape* shape, const void* q, const void* k, const void* v,
                            const nabla_mask* mask, void* o, void* o_res, float* lse, void* workspace,
                            size_t workspace_bytes, nabla_stream_t stream) {
  g_last_error.clear();
  NABLA_TRY(check_shape(shape));
  const Dims d = make_dims(*shape);
  NABLA_TRY(check_tensor(q, "q"));
  NABLA_TRY(check_tensor(k, "k"));
  NABLA_TRY(check_tensor(v, "v"));
  NABLA_TRY(check_tensor(o, "o"));
  if (o_res) {
    NABLA_TRY(check_tensor(o_res, "o_res"));
    if (d.dtype != NABLA_BF16)
      return fail(NABLA_ERR_INVALID_ARG, "o_res applies to bf16 only (an fp32 O needs no residual)");
  }
  if (lse && !aligned(lse, 4)) return fail(NABLA_ERR_INVALID_ARG, "lse is not 4-byte aligned");
  NABLA_TRY(check_mask_out(mask, true));
  NABLA_TRY(check_ws(d, false, workspace, workspace_bytes));
  cudaStream_t st = (cudaStream_t)stream;
  NABLA_TRY(reset_status(workspace, st));
  if (d.dtype == NABLA_BF16)
    NABLA_CUDA(launch_attn_fwd_tc(d, q, k, v, mask->bits, mask->work, o, o_res, lse, (int32_t*)workspace, st),
               "tensor-core attention forward");
  else
    NABLA_CUDA(launch_attn_fwd_simt(d, q, k, v, mask->cnt, mask->idx, o, lse, st),
               "fp32 attention forward");
  return NABLA_OK;
}

nabla_status nabla_attn_bwd(const nabla_shape* shape, const void* q, const void* k, const void* v,
                            const void* o, const void* o_res, const void* dout, const float* lse,
                            const nabla_mask* mask, void* dq, void* dk, void* dv, void* workspace,
                            size_t workspace_bytes, nabla_stream_t stream) {
  g_last_error.clear();
  NABLA_TRY(check_shape(shape));
  const Dims d = make_dims(*shape);
  NABLA_TRY(check_tensor(q, "q"));
  NABLA_TRY(check_tensor(k, "k"));
  NABLA_TRY(check_tensor(v, "v"));
  NABLA_TRY(check_tensor(o, "o"));
  NABLA_TRY(check_tensor(dout, "dout"));
  if (o_res) {
    NABLA_TRY(check_tensor(o_res, "o_res"));
    if (d.dtype != NABLA_BF16)
      return fail(NABLA_ERR_INVALID_ARG, "o_res applies to bf16 only (an fp32 O needs no residual)");
  }
  NABLA_TRY(check_tensor(dq, "dq"));
  NABLA_TRY(check_tensor(dk, "dk"));
  NABLA_TRY(check_tensor(dv, "dv"));
  NABLA_TRY(check_i32(lse, "lse"));
  NABLA_TRY(check_mask_out(mask, true));
  if (!mask->cnt_t) return fail(NABLA_ERR_INVALID_ARG, "backward needs mask.cnt_t and mask.idx_t");
  NABLA_TRY(check_ws(d, true, workspace, workspace_bytes));
  cudaStream_t st = (cudaStream_t)stream;
  const WsLayout L = ws_layout(d, true);
  NABLA_TRY(reset_status(workspace, st));
  char* ws = (char*)workspace;
  if (d.dtype == NABLA_BF16 && d.D == 128)
    NABLA_CUDA(launch_attn_bwd_tc(d, q, k, v, o, o_res, dout, lse, mask->bits, mask->cnt, mask->idx, mask->cnt_t,
                                  (float*)(ws + L.lse2p), (float*)(ws + L.deltap), dq, dk, dv,
                                  (int32_t*)ws, st),
               "tensor-core attention backward");
  else
    NABLA_CUDA(launch_attn_bwd_simt(d, q, k, v, o, o_res, dout, lse, mask->cnt, mask->idx, mask->cnt_t,
                                    mask->idx_t, (float*)(ws + L.delta), dq, dk, dv, st),
               "attention backward");
  return NABLA_OK;
}

nabla_status nabla_selftest_wait_timeout(void* workspace, uint64_t limit_ns, nabla_stream_t stream) {
  g_last_error.clear();
  if (!workspace) return fail(NABLA_ERR_WORKSPACE, "workspace is NULL");
  if (!aligned(workspace, 256)) return fail(NABLA_ERR_WORKSPACE, "workspace must be 256-byte aligned");
  if (limit_ns == 0 || limit_ns > 10000000000ull)
    return fail(NABLA_ERR_INVALID_ARG, "limit_ns must lie in [1, 1e10] (got %llu)",
                (unsigned long long)limit_ns);
  cudaStream_t st = (cudaStream_t)stream;
  NABLA_TRY(reset_status(workspace, st));
  NABLA_CUDA(launch_wait_selftest((int32_t*)workspace + kWsStatus, limit_ns, st), "wait self-test");
  return NABLA_OK;
}

nabla_status nabla_workspace_status(const void* workspace, int32_t* host_status,
                                    nabla_stream_t stream) {
  g_last_error.clear();
  if (!workspace || !host_status)
    return fail(NABLA_ERR_INVALID_ARG, "workspace and host_status must not be NULL");
  cudaStream_t st = (cudaStream_t)stream;
  NABLA_CUDA(cudaMemcpyAsync(host_status, workspace, sizeof(int32_t), cudaMemcpyDeviceToHost, st),
             "read status word");
  NABLA_CUDA(cudaStreamSynchronize(st), "synchronise stream");
  return NABLA_OK;
}

// Tile coordinate of the first token of every 64-token block.  Inside a
// frame of H_lat x W_lat tokens the P x P patches follow in row-major patch
// order, each patch's tokens contiguous (an edge patch cut by the frame holds
// only its valid tokens); frames follow in time order.  Patch row py starts at
// token py * P * W_lat of its frame (every patch row above it is P tokens
// high), and inside that row, whose patches are ph = min(P, H_lat - py * P)
// tokens high, patch px starts at px * ph * P (every patch left of it is P
// tokens wide).  The tile coordinate of any token of patch (py, px) of frame t
// is (t, py, px).
nabla_status nabla_sta_block_coords(int32_t T, int32_t H_lat, int32_t W_lat, int32_t P, int32_t S,
                                    int32_t* coords_host) {
  g_last_error.clear();
  if (!coords_host) return fail(NABLA_ERR_INVALID_ARG, "coords_host is NULL");
  if (T < 1 || H_lat < 1 || W_lat < 1 || P < 1 || S < 1)
    return fail(NABLA_ERR_INVALID_ARG, "T, H_lat, W_lat, P and S must be >= 1 (got %d, %d, %d, %d, %d)", T,
                H_lat, W_lat, P, S);
  const long long frame = (long long)H_lat * W_lat;
  const long long tokens = frame * T;
  const long long nb = ((long long)S + kBlock - 1) / kBlock;
  if (tokens > 0x7fffffffll)
    return fail(NABLA_ERR_INVALID_ARG, "T * H_lat * W_lat = %lld tokens is beyond int32", tokens);
  if ((nb - 1) * kBlock >= tokens)
    return fail(NABLA_ERR_INVALID_ARG,
                "S = %d gives %lld blocks, but block %lld would start past the %lld tokens of the latent", S,
                nb, nb - 1, tokens);
  const long long patch_row = (long long)P * W_lat;
  for (long long i = 0; i < nb; ++i) {
    const long long n = i * kBlock;
    const long long t = n / frame, r = n - t * frame;
    const long long py = r / patch_row, rr = r - py * patch_row;
    const long long ph = std::min<long long>(P, H_lat - py * P);
    const long long px = rr / (ph * P);
    coords_host[3 * i] = (int32_t)t;
    coords_host[3 * i + 1] = (int32_t)py;
    coords_host[3 * i + 2] = (int32_t)px;
  }
  return NABLA_OK;
}

}  // extern "C"
