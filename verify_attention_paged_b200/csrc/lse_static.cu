// Partial + merge passes on a library-owned, statically allocated device
// scratch area, for callers that must not allocate device memory.
//
// Some callers cannot call cudaMalloc at the point where they run
// attention: engines whose device memory is carved up once at start-up by
// a host framework (plugin and custom-op hosts that hand a kernel only its
// inputs and outputs) and real-time serving loops whose device memory is
// fixed at start-up, so that nothing may be allocated after warm-up.  This
// entry point gives
// them the whole call (lse_attn_run, then lse_attn_merge) with the
// workspace taken from a file-scope __device__ array instead of caller
// memory.  It allocates nothing.
#include <cuda_runtime.h>

#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>

#include "lse_internal.h"

// The scratch: LSE_STATIC_SCRATCH_BYTES per GPU, resident on every device
// that loads this library until the process exits.
static __device__ __align__(256) unsigned char g_lse_static_scratch[LSE_STATIC_SCRATCH_BYTES];

namespace {

constexpr int kMaxDevices = 64;
std::mutex g_setup_mutex;
void *g_scratch_addr[kMaxDevices] = {};

int fail_msg(char **err, int status, const char *msg) {
  if (err) {
    const size_t n = strlen(msg) + 1;
    char *m = static_cast<char *>(malloc(n));  // host string for the caller (lse_free)
    if (m) memcpy(m, msg, n);
    *err = m;
  }
  return status;
}

// Device address of the scratch array on the current device.  Host code
// only sees a stand-in for the symbol, so the address is asked from the
// runtime once per device, with that device current.
int scratch_address(void **out, char **err) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fail_msg(err, LSE_ERR_CUDA, cudaGetErrorString(e));
  if (dev < 0 || dev >= kMaxDevices)
    return fail_msg(err, LSE_ERR_UNSUPPORTED, "device ordinal beyond the static scratch table");
  std::lock_guard<std::mutex> lock(g_setup_mutex);
  if (!g_scratch_addr[dev]) {
    void *p = nullptr;
    e = cudaGetSymbolAddress(&p, g_lse_static_scratch);
    if (e != cudaSuccess || !p) {
      char buf[256];
      snprintf(buf, sizeof buf, "cudaGetSymbolAddress(static scratch): %s",
               cudaGetErrorString(e));
      return fail_msg(err, LSE_ERR_CUDA, buf);
    }
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return LSE_OK;
}

}  // namespace

extern "C" LSE_API int lse_attn_forward_static(
    const lse_attn_plan_t *plan, const float *q, const int32_t *k_pages,
    const int32_t *v_pages, const int32_t *seq_lens, const int32_t *row_offsets,
    const uint64_t *row_masks, float softmax_scale, float *out, float *lse_out, void *stream,
    char **err) {
  if (!plan) return fail_msg(err, LSE_ERR_INVALID_ARG, "plan is NULL");
  if (plan->ws_bytes > (size_t)LSE_STATIC_SCRATCH_BYTES) {
    char buf[256];
    snprintf(buf, sizeof buf,
             "plan needs %zu bytes of workspace; the static scratch holds %zu "
             "(use lse_attn_run / lse_attn_merge with a caller workspace)",
             plan->ws_bytes, (size_t)LSE_STATIC_SCRATCH_BYTES);
    return fail_msg(err, LSE_ERR_UNSUPPORTED, buf);
  }
  void *ws = nullptr;
  int st = scratch_address(&ws, err);
  if (st) return st;
  // the device error word must start at zero for this call; everything else
  // the passes read is written by this call first
  cudaError_t e = cudaMemsetAsync(ws, 0, sizeof(uint32_t), reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return fail_msg(err, LSE_ERR_CUDA, cudaGetErrorString(e));
  st = lse_attn_run(plan, q, k_pages, v_pages, seq_lens, row_offsets, row_masks, softmax_scale,
                    ws, stream, err);
  if (st) return st;
  return lse_attn_merge(plan, seq_lens, row_offsets, ws, out, lse_out, stream, err);
}

// The first 32-bit word of the scratch is the device error word of the
// latest static call on this device (the passes OR their LSE_DEVERR_* bits
// into it).  Read it, then clear it, in stream order.
extern "C" LSE_API int lse_attn_static_read_error(void *stream, uint32_t *device_error,
                                                  char **err) {
  if (!device_error) return fail_msg(err, LSE_ERR_INVALID_ARG, "device_error is NULL");
  void *ws = nullptr;
  int st = scratch_address(&ws, err);
  if (st) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  uint32_t v = 0;
  cudaError_t e = cudaMemcpyAsync(&v, ws, sizeof v, cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e == cudaSuccess) e = cudaMemsetAsync(ws, 0, sizeof v, s);
  if (e != cudaSuccess) return fail_msg(err, LSE_ERR_CUDA, cudaGetErrorString(e));
  *device_error = v;
  return LSE_OK;
}
