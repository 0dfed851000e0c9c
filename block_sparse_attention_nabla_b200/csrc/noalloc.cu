// Mask builder entry point that allocates nothing: nabla_build_mask_noalloc.
//
// Some callers cannot allocate device memory when they build a mask: a serving
// process that reserved all device memory up front and forbids side
// allocations while a request runs, a plug-in loaded into such a host, or code
// that must not call cudaMalloc because it may synchronise the device and
// stall streams that other work depends on.  They still own the inputs and the
// mask outputs; only the builder's scratch (the pooled Qa / Ka and the status
// word) comes from the static array below instead of a caller workspace.
//
// The array lives in every GPU that loads this library until the process
// exits.  The first call on a device loads the module that holds it (CUDA
// loads modules lazily), which commits the 32 MiB on that device; callers make
// that first call, or nabla_build_mask_noalloc_status, at start-up, before they
// reserve the rest of the device memory.  The status word at the start of the
// array reports a bounded wait that ran out in the pooling or the score GEMM, and
// nabla_build_mask_noalloc_status reads it back.  Every call shares the array
// and it keeps the last call's contents, so calls whose work overlaps on the
// GPU (different streams, or different host threads on one device) race on
// it; callers serialise them.
#include <mutex>

#include "internal.cuh"

namespace nabla {
namespace {

// 32 MiB: a 256-byte header (status word), the pooled vectors (fp64 and tf32
// hi / lo pairs) and the reduced logits.
constexpr size_t kNoAllocScratchBytes = 32u << 20;
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

std::mutex g_setup_mutex;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of the static array on the current device.  The name
// g_noalloc_scratch means something else in host code, so the address is asked
// for once per device, with that device current, and cached.
nabla_status scratch_on_current_device(void** out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) {
    record_error(NABLA_ERR_CUDA, "cudaGetDevice failed: %s", cudaGetErrorString(e));
    return NABLA_ERR_CUDA;
  }
  if (dev < 0 || dev >= kMaxDevices) {
    record_error(NABLA_ERR_UNSUPPORTED, "device %d is beyond the %d devices this entry point serves",
                 dev, kMaxDevices);
    return NABLA_ERR_UNSUPPORTED;
  }
  std::lock_guard<std::mutex> lock(g_setup_mutex);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || !p) {
      record_error(NABLA_ERR_CUDA, "cudaGetSymbolAddress of the static scratch failed: %s",
                   cudaGetErrorString(e));
      return NABLA_ERR_CUDA;
    }
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return NABLA_OK;
}

}  // namespace
}  // namespace nabla

using namespace nabla;

extern "C" NABLA_API nabla_status nabla_build_mask_noalloc(const nabla_shape* shape, const void* q,
                                                           const void* k, float thr,
                                                           const nabla_sta* sta,
                                                           const nabla_mask* out,
                                                           nabla_stream_t stream) {
  record_error(NABLA_OK, "");
  // the same checks, with the same messages, as nabla_build_mask
  nabla_status chk = check_shape(shape);
  if (chk == NABLA_OK) chk = check_tensor(q, "q");
  if (chk == NABLA_OK) chk = check_tensor(k, "k");
  if (chk == NABLA_OK) chk = check_selection(thr, 0, sta);
  if (chk == NABLA_OK) chk = check_mask_out(out, true);
  if (chk != NABLA_OK) return chk;
  const Dims d = make_dims(*shape);
  const WsLayout L = ws_layout(d, false);
  if (L.total > kNoAllocScratchBytes) {
    record_error(NABLA_ERR_UNSUPPORTED,
                 "this shape needs %zu bytes of scratch; the static scratch of "
                 "nabla_build_mask_noalloc holds %zu (B * H * (nb * (32 D + 4 nb) + 8) bytes, nb = ceil(S / 64), plus about 2 KB, must fit); "
                 "use nabla_build_mask with a workspace",
                 L.total, kNoAllocScratchBytes);
    return NABLA_ERR_UNSUPPORTED;
  }
  void* scratch = nullptr;
  const nabla_status st0 = scratch_on_current_device(&scratch);
  if (st0 != NABLA_OK) return st0;
  cudaStream_t st = (cudaStream_t)stream;
  char* ws = (char*)scratch;
  int32_t* status = (int32_t*)ws + kWsStatus;
  int32_t* counters = (int32_t*)(ws + L.counters);
  cudaError_t e = cudaMemsetAsync(ws, 0, 256, st);  // the status word starts at zero
  if (e == cudaSuccess) e = cudaMemsetAsync(counters, 0, (size_t)d.BH() * 2 * sizeof(int32_t), st);
  if (e == cudaSuccess)
    e = launch_pool(d, q, k, (double*)(ws + L.qa), (double*)(ws + L.ka), (float*)(ws + L.qhi),
                    (float*)(ws + L.qlo), (float*)(ws + L.khi), (float*)(ws + L.klo), counters, status, st);
  if (e == cudaSuccess)
    e = launch_score_gemm(d, (const float*)(ws + L.qhi), (const float*)(ws + L.qlo),
                          (const float*)(ws + L.khi), (const float*)(ws + L.klo), (float*)(ws + L.logits),
                          L.ldl, counters, pool_target(d), status, st);
  if (e == cudaSuccess)
    e = launch_select(d, (const float*)(ws + L.logits), L.ldl, (const double*)(ws + L.qa),
                      (const double*)(ws + L.ka), thr, sta, out->bits, out->cnt, out->idx, counters,
                      pool_target(d), status, st);
  if (e == cudaSuccess && out->cnt_t) e = launch_transpose_lists(d, out->bits, out->cnt_t, out->idx_t, st);
  if (e == cudaSuccess) e = launch_work_list(d, out->bits, out->work, st);
  if (e != cudaSuccess) {
    record_error(NABLA_ERR_CUDA, "nabla_build_mask_noalloc launch failed: %s", cudaGetErrorString(e));
    return NABLA_ERR_CUDA;
  }
  return NABLA_OK;
}

extern "C" NABLA_API nabla_status nabla_build_mask_noalloc_status(int32_t* host_status,
                                                                  nabla_stream_t stream) {
  record_error(NABLA_OK, "");
  if (!host_status) {
    record_error(NABLA_ERR_INVALID_ARG, "host_status is NULL");
    return NABLA_ERR_INVALID_ARG;
  }
  void* scratch = nullptr;
  const nabla_status st0 = scratch_on_current_device(&scratch);
  if (st0 != NABLA_OK) return st0;
  cudaStream_t st = (cudaStream_t)stream;
  cudaError_t e = cudaMemcpyAsync(host_status, (const int32_t*)scratch + kWsStatus, sizeof(int32_t),
                                  cudaMemcpyDeviceToHost, st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) {
    record_error(NABLA_ERR_CUDA, "reading the static scratch's status word failed: %s", cudaGetErrorString(e));
    return NABLA_ERR_CUDA;
  }
  return NABLA_OK;
}
