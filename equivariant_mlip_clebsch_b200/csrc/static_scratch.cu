// static_scratch.cu -- backward entry point for callers that cannot allocate.
//
// cgtp_backward needs a scratch buffer (the per-edge messages of the
// two-pass dx, plus per-slice dY parts for wide plans) and takes it from the
// caller.  Some callers have no way to provide one: a simulation engine that
// sizes all of its device memory once at start-up and forbids later
// allocation, or an embedding runtime that owns no device allocator and must
// not pull in one (PyTorch's included).  cgtp_backward_static_scratch serves
// them from a fixed array that lives in this library's device image instead.
//
// The array is a file-scope __device__ variable, so every GPU on which the
// library's device code is loaded holds it until the process exits.  Host
// code cannot use the variable's name as a device address; the address is
// obtained once per device with cudaGetSymbolAddress, with that device
// current, on the first call made on that device.
#include <cuda_runtime.h>

#include <cstdio>
#include <mutex>
#include <string>

#include "internal.hpp"

namespace {

constexpr size_t kScratchBytes = size_t(CGTP_STATIC_SCRATCH_BYTES);

static __device__ __align__(256) unsigned char g_backward_scratch[CGTP_STATIC_SCRATCH_BYTES];

std::mutex g_mu;
void* g_addr[256] = {nullptr};

// Device address of g_backward_scratch on the current device, looked up once.
cgtp_status scratch_address(void** out) {
  int dev = -1;
  CGTP_CUDA_TRY(cudaGetDevice(&dev));
  if (dev < 0 || dev >= 256) return cgtp::fail(CGTP_ERR_CUDA, "device ordinal out of range");
  std::lock_guard<std::mutex> g(g_mu);
  if (!g_addr[dev]) {
    void* p = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&p, g_backward_scratch);
    if (e != cudaSuccess || !p)
      return cgtp::fail(CGTP_ERR_CUDA, std::string("cudaGetSymbolAddress(static scratch): ") +
                                           cudaGetErrorString(e));
    g_addr[dev] = p;
  }
  *out = g_addr[dev];
  return CGTP_OK;
}

}  // namespace

extern "C" cgtp_status cgtp_backward_static_scratch(
    cgtp_plan plan, int64_t n_recv, int64_t n_send, int64_t E, const int32_t* rowptr,
    const int32_t* col, const int32_t* rowptr_T, const int32_t* perm_T, const float* x,
    const float* Y, const float* W, const float* grad_out, float* grad_x, float* grad_W,
    float* grad_Y, cgtp_stream stream) {
  cgtp::NvtxRange nvtx_range("cgtp_backward_static_scratch");
  if (!plan) return cgtp::fail(CGTP_ERR_NULL, "plan is NULL");
  const cgtp::Plan& P = *reinterpret_cast<const cgtp::Plan*>(plan);
  // every host check first: a call with the wrong device current, a bad size
  // or pointer is refused before the array's address is looked up
  cgtp_status st = cgtp::backward_validate(P, n_recv, n_send, E, rowptr, col, rowptr_T, perm_T, x, Y, W,
                                           grad_out, grad_x, grad_W, grad_Y);
  if (st != CGTP_OK) return st;
  // only the scratch this call uses counts against the array: a grad_W-only
  // call needs none, whatever the graph's size
  const size_t need = cgtp::backward_scratch_bytes(P, E, grad_x != nullptr, grad_Y != nullptr, nullptr);
  if (need > kScratchBytes) {
    char msg[200];
    std::snprintf(msg, sizeof msg,
                  "this backward needs %zu bytes of scratch; the static scratch holds %zu bytes "
                  "(CGTP_STATIC_SCRATCH_BYTES): use cgtp_backward with a workspace",
                  need, kScratchBytes);
    return cgtp::fail(CGTP_ERR_WORKSPACE, msg);
  }
  void* ws = nullptr;
  if (need > 0) {
    st = scratch_address(&ws);
    if (st != CGTP_OK) return st;
  }
  // the scratch needs no initial contents: every byte the backward reads
  // from it is written earlier in the same call
  return cgtp::backward_impl(plan, n_recv, n_send, E, rowptr, col, rowptr_T, perm_T, x, Y, W,
                             grad_out, grad_x, grad_W, grad_Y, ws, need > 0 ? kScratchBytes : 0, stream,
                             /*allow_timing=*/false, /*eid=*/nullptr, /*graph_checks=*/true);
}
