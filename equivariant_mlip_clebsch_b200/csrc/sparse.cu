// sparse.cu -- BranchIP sparse evaluation of the CGTP convolution.
//
// The BranchIP page (section "BranchIP", the Branchlegro paragraph): a router
// gives every edge a continuation gate f_e in [0, 1] that multiplies the
// edge's feature before the TP; at inference the zero-gated edges are
// omitted from the TP ("sparse evaluation") and the skipped per-edge outputs
// are zero-padded to the full edge set, which reproduces the dense
// evaluation exactly.  Here the gate scales the edge's whole TP term (the
// convolution is linear in Y_e, so it is applied to the edge's harmonics).
//
// Device steps, all deterministic (scans, no atomics), no host round trip:
//   1. compaction: the active edges (f_e > 0) in receiver order -> the
//      receiver CSR over them (rowptr_A, col_A), their full-set ids (eid)
//      and their gated harmonics Y_A = f_e Y_e; with the transpose, the
//      sender lists over them (rowptr_TA, perm_TA, compact ids);
//   2. the plan's forward / backward kernels over the compact edges, reading
//      W rows (writing grad_W rows) of the full set through eid;
//   3. (backward) padding: grad_Y = f_e dL/dY'_A, grad_gate = <Y_e, dL/dY'_A>
//      on active edges, zeros (and zero grad_W rows) on the skipped ones.
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>
#include <string>

#include "internal.hpp"

namespace cgtp {

namespace {

constexpr int kScanThreads = 512;
constexpr int kScanItems = 8;  // consecutive elements per thread
constexpr int kTile = kScanThreads * kScanItems;

__device__ __forceinline__ bool active(const float* __restrict__ f, int64_t e) { return __ldg(f + e) > 0.f; }

// Exclusive scan of one value per thread over the block; returns the
// thread's offset and (through total) the block's sum.  Every thread of the
// block must call it (it synchronises the block).
__device__ __forceinline__ int block_exclusive_scan(int v, int* total) {
  constexpr int kWarps = kScanThreads / 32;
  __shared__ int warp_off[kWarps];
  __shared__ int tot;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int t = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += t;
  }
  if (lane == 31) warp_off[warp] = incl;  // the warp's total
  __syncthreads();
  if (warp == 0) {
    const int w = lane < kWarps ? warp_off[lane] : 0;
    int wi = w;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int t = __shfl_up_sync(0xffffffffu, wi, o);
      if (lane >= o) wi += t;
    }
    if (lane < kWarps) warp_off[lane] = wi - w;  // exclusive offset of each warp
    if (lane == kWarps - 1) tot = wi;
  }
  __syncthreads();
  const int off = warp_off[warp] + incl - v;
  *total = tot;
  __syncthreads();  // warp_off and tot are reused by the next call
  return off;
}

// Step 1a: per tile, the number of active edges in edge order and in the
// transpose (sender) order.
__global__ void __launch_bounds__(kScanThreads) active_count_kernel(int64_t E, const float* __restrict__ f,
                                                                     const int32_t* __restrict__ perm_T,
                                                                     int32_t* __restrict__ blk) {
  const int64_t base = (int64_t)blockIdx.x * kTile + (int64_t)threadIdx.x * kScanItems;
  int c = 0, cT = 0;
#pragma unroll
  for (int k = 0; k < kScanItems; ++k) {
    const int64_t e = base + k;
    if (e < E) {
      c += active(f, e);
      if (perm_T) cT += active(f, __ldg(perm_T + e));
    }
  }
  int tot = 0, totT = 0;
  block_exclusive_scan(c, &tot);
  block_exclusive_scan(cT, &totT);
  if (threadIdx.x == 0) {
    blk[2 * blockIdx.x] = tot;
    blk[2 * blockIdx.x + 1] = totT;
  }
}

// Step 1b: exclusive scan of the tile counts (one block, in chunks), and the
// totals at pos[E] / posT[E].
__global__ void __launch_bounds__(kScanThreads) active_scan_kernel(int64_t ntiles, int32_t* __restrict__ blk,
                                                                    int64_t E, int32_t* __restrict__ pos,
                                                                    int32_t* __restrict__ posT) {
  int carry = 0, carryT = 0;
  for (int64_t b0 = 0; b0 < ntiles; b0 += kScanThreads) {
    const int64_t b = b0 + threadIdx.x;
    const int v = b < ntiles ? blk[2 * b] : 0;
    const int vT = b < ntiles ? blk[2 * b + 1] : 0;
    int tot = 0, totT = 0;
    const int o = block_exclusive_scan(v, &tot);
    const int oT = block_exclusive_scan(vT, &totT);
    if (b < ntiles) {
      blk[2 * b] = carry + o;
      blk[2 * b + 1] = carryT + oT;
    }
    carry += tot;
    carryT += totT;
  }
  if (threadIdx.x == 0) {
    pos[E] = carry;
    if (posT) posT[E] = carryT;
  }
}

// Step 1c: every edge's exclusive position among the active ones (pos), in
// edge order and in sender order (posT); the active edges' ids and senders.
__global__ void __launch_bounds__(kScanThreads) active_place_kernel(int64_t E, const float* __restrict__ f,
                                                                     const int32_t* __restrict__ col,
                                                                     const int32_t* __restrict__ perm_T,
                                                                     const int32_t* __restrict__ blk,
                                                                     int32_t* __restrict__ pos,
                                                                     int32_t* __restrict__ posT,
                                                                     int32_t* __restrict__ eid,
                                                                     int32_t* __restrict__ col_A) {
  const int64_t base = (int64_t)blockIdx.x * kTile + (int64_t)threadIdx.x * kScanItems;
  bool a[kScanItems], aT[kScanItems];
  int c = 0, cT = 0;
#pragma unroll
  for (int k = 0; k < kScanItems; ++k) {
    const int64_t e = base + k;
    a[k] = e < E && active(f, e);
    aT[k] = perm_T && e < E && active(f, __ldg(perm_T + e));
    c += a[k];
    cT += aT[k];
  }
  int tot = 0, totT = 0;
  int p = block_exclusive_scan(c, &tot) + blk[2 * blockIdx.x];
  int pT = block_exclusive_scan(cT, &totT) + blk[2 * blockIdx.x + 1];
#pragma unroll
  for (int k = 0; k < kScanItems; ++k) {
    const int64_t e = base + k;
    if (e < E) {
      pos[e] = p;
      if (a[k]) {
        eid[p] = (int32_t)e;
        col_A[p] = __ldg(col + e);
      }
      p += a[k];
      if (perm_T) {
        posT[e] = pT;
        pT += aT[k];
      }
    }
  }
}

// Step 1d: the compact CSRs from the positions, and the gated harmonics of
// the active edges.  Grid-stride over max(n_recv + 1, n_send + 1, E * D_e).
__global__ void __launch_bounds__(256) active_finish_kernel(
    int64_t n_recv, int64_t n_send, int64_t E, int De, const int32_t* __restrict__ rowptr,
    const int32_t* __restrict__ rowptr_T, const int32_t* __restrict__ perm_T, const float* __restrict__ f,
    const float* __restrict__ Y, const int32_t* __restrict__ pos, const int32_t* __restrict__ posT,
    int32_t* __restrict__ rowptr_A, int32_t* __restrict__ rowptr_TA, int32_t* __restrict__ perm_TA,
    float* __restrict__ Y_A) {
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  const int64_t t0 = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  for (int64_t i = t0; i <= n_recv; i += stride) rowptr_A[i] = pos[rowptr[i]];
  if (perm_T) {
    for (int64_t j = t0; j <= n_send; j += stride) rowptr_TA[j] = posT[rowptr_T[j]];
    for (int64_t t = t0; t < E; t += stride) {
      const int32_t e = __ldg(perm_T + t);
      if (active(f, e)) perm_TA[posT[t]] = pos[e];
    }
  }
  const int64_t n = E * De;
  for (int64_t k = t0; k < n; k += stride) {
    const int64_t e = k / De;
    if (active(f, e)) Y_A[(int64_t)pos[e] * De + (k - e * De)] = __ldg(f + e) * __ldg(Y + k);
  }
}

// Step 3 (backward): one warp per edge of the full set.  Active edge e at
// compact position p: grad_Y[e] = f_e dYA[p], grad_gate[e] = <Y[e], dYA[p]>;
// skipped edges: zeros in grad_Y, grad_gate and their grad_W row.
__global__ void __launch_bounds__(256) sparse_pad_kernel(int64_t E, int De, int64_t U, const float* __restrict__ f,
                                                          const float* __restrict__ Y,
                                                          const int32_t* __restrict__ pos,
                                                          const float* __restrict__ dYA, float* __restrict__ grad_W,
                                                          float* __restrict__ grad_Y,
                                                          float* __restrict__ grad_gate) {
  const int lane = threadIdx.x & 31;
  const int64_t warps = (int64_t)gridDim.x * (blockDim.x >> 5);
  for (int64_t e = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5; e < E; e += warps) {
    const int32_t p = pos[e];
    const bool on = pos[e + 1] > p;
    const float fe = __ldg(f + e);
    float dot = 0.f;
    for (int t = lane; t < De; t += 32) {
      const float d = on ? dYA[(int64_t)p * De + t] : 0.f;
      if (grad_Y) grad_Y[e * De + t] = on ? fe * d : 0.f;
      dot = fmaf(__ldg(Y + e * De + t), d, dot);
    }
    if (grad_gate) {
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, o);
      if (lane == 0) grad_gate[e] = on ? dot : 0.f;
    }
    if (grad_W && !on) {
      float* row = grad_W + e * U;
      for (int64_t k = lane; k < U; k += 32) row[k] = 0.f;
    }
  }
}

// Workspace layout of the sparse entry points (256-byte aligned pieces).
struct SparseLayout {
  size_t pos, posT, blk, rowptr_A, col_A, eid, rowptr_TA, perm_TA, Y_A, dY_A, bwd, total;
};

SparseLayout sparse_layout(const Plan& P, int64_t n_recv, int64_t n_send, int64_t E) {
  auto r256 = [](size_t v) { return (v + 255) & ~size_t(255); };
  const size_t ntiles = (size_t)((E + kTile - 1) / kTile);
  SparseLayout L;
  size_t o = 0;
  L.pos = o;
  o += r256((size_t)(E + 1) * 4);
  L.posT = o;
  o += r256((size_t)(E + 1) * 4);
  L.blk = o;
  o += r256(std::max<size_t>(1, 2 * ntiles) * 4);
  L.rowptr_A = o;
  o += r256((size_t)(n_recv + 1) * 4);
  L.col_A = o;
  o += r256((size_t)std::max<int64_t>(E, 1) * 4);
  L.eid = o;
  o += r256((size_t)std::max<int64_t>(E, 1) * 4);
  L.rowptr_TA = o;
  o += r256((size_t)(n_send + 1) * 4);
  L.perm_TA = o;
  o += r256((size_t)std::max<int64_t>(E, 1) * 4);
  L.Y_A = o;
  o += r256((size_t)std::max<int64_t>(E, 1) * P.D_e * 4);
  L.dY_A = o;
  o += r256((size_t)std::max<int64_t>(E, 1) * P.D_e * 4);
  L.bwd = o;
  o += r256(backward_scratch_bytes(P, E, true, true, nullptr));
  L.total = o;
  return L;
}

struct Compact {
  int32_t *pos, *posT, *rowptr_A, *col_A, *eid, *rowptr_TA, *perm_TA;
  float *Y_A, *dY_A;
  void* bwd;
  size_t bwd_bytes;
};

Compact carve(const SparseLayout& L, void* ws) {
  char* b = reinterpret_cast<char*>(ws);
  Compact c;
  c.pos = reinterpret_cast<int32_t*>(b + L.pos);
  c.posT = reinterpret_cast<int32_t*>(b + L.posT);
  c.rowptr_A = reinterpret_cast<int32_t*>(b + L.rowptr_A);
  c.col_A = reinterpret_cast<int32_t*>(b + L.col_A);
  c.eid = reinterpret_cast<int32_t*>(b + L.eid);
  c.rowptr_TA = reinterpret_cast<int32_t*>(b + L.rowptr_TA);
  c.perm_TA = reinterpret_cast<int32_t*>(b + L.perm_TA);
  c.Y_A = reinterpret_cast<float*>(b + L.Y_A);
  c.dY_A = reinterpret_cast<float*>(b + L.dY_A);
  c.bwd = b + L.bwd;
  c.bwd_bytes = L.total - L.bwd;
  return c;
}

// Step 1 on the stream: four launches.
cudaError_t launch_compaction(const Plan& P, int64_t n_recv, int64_t n_send, int64_t E, const int32_t* rowptr,
                              const int32_t* col, const int32_t* rowptr_T, const int32_t* perm_T,
                              const float* gate, const float* Y, const SparseLayout& L, void* ws,
                              cudaStream_t s) {
  Compact c = carve(L, ws);
  int32_t* blk = reinterpret_cast<int32_t*>(reinterpret_cast<char*>(ws) + L.blk);
  const int64_t ntiles = (E + kTile - 1) / kTile;
  const int32_t* pT = rowptr_T ? perm_T : nullptr;  // the transpose only when it is needed
  if (ntiles > 0) {
    active_count_kernel<<<(unsigned)ntiles, kScanThreads, 0, s>>>(E, gate, pT, blk);
  }
  active_scan_kernel<<<1, kScanThreads, 0, s>>>(ntiles, blk, E, c.pos, pT ? c.posT : nullptr);
  if (ntiles > 0) {
    active_place_kernel<<<(unsigned)ntiles, kScanThreads, 0, s>>>(E, gate, col, pT, blk, c.pos, c.posT, c.eid,
                                                                  c.col_A);
  }
  const int64_t work = std::max<int64_t>({n_recv + 1, pT ? n_send + 1 : 0, E * P.D_e, 1});
  const int64_t blocks = std::min<int64_t>((work + 255) / 256, (int64_t)P.num_sms * 8);
  active_finish_kernel<<<(unsigned)blocks, 256, 0, s>>>(n_recv, n_send, E, (int)P.D_e, rowptr, rowptr_T, pT, gate,
                                                        Y, c.pos, c.posT, c.rowptr_A, c.rowptr_TA, c.perm_TA, c.Y_A);
  return cudaGetLastError();
}

bool aligned16(const void* p) { return ((uintptr_t)p & 15) == 0; }

cgtp_status sparse_checks(const Plan& P, int64_t n_recv, int64_t n_send, int64_t E, const int32_t* rowptr,
                          const float* gate, void* workspace, size_t workspace_bytes, size_t need) {
  if (n_recv < 0 || n_send < 0 || E < 0 || n_recv >= (int64_t(1) << 31) || n_send >= (int64_t(1) << 31) ||
      E >= (int64_t(1) << 31) - 1)
    return fail(CGTP_ERR_SIZE, "sizes out of range");
  cgtp_status st = check_plan_device(P);
  if (st != CGTP_OK) return st;
  if (n_recv > 0 && !rowptr) return fail(CGTP_ERR_NULL, "rowptr is NULL");
  if (E > 0 && !gate) return fail(CGTP_ERR_NULL, "gate is NULL");
  if (!workspace || workspace_bytes < need)
    return fail(CGTP_ERR_WORKSPACE, "workspace of " + std::to_string(need) + " bytes required");
  if ((uintptr_t)workspace & 255) return fail(CGTP_ERR_ALIGN, "workspace must be 256-byte aligned");
  return CGTP_OK;
}

}  // namespace

}  // namespace cgtp

using namespace cgtp;

extern "C" {

cgtp_status cgtp_sparse_workspace_size(cgtp_plan plan, int64_t n_recv, int64_t n_send, int64_t E, size_t* bytes) {
  if (!plan || !bytes) return fail(CGTP_ERR_NULL, "null argument");
  if (n_recv < 0 || n_send < 0 || E < 0) return fail(CGTP_ERR_SIZE, "negative size");
  *bytes = sparse_layout(*reinterpret_cast<const Plan*>(plan), n_recv, n_send, E).total;
  return CGTP_OK;
}

cgtp_status cgtp_sparse_forward(cgtp_plan plan, int64_t n_recv, int64_t n_send, int64_t E, const int32_t* rowptr,
                                const int32_t* col, const float* x, const float* Y, const float* W,
                                const float* gate, float* out, void* workspace, size_t workspace_bytes,
                                cgtp_stream stream) {
  NvtxRange nvtx_range("cgtp_sparse_forward");
  if (!plan) return fail(CGTP_ERR_NULL, "plan is NULL");
  const Plan& P = *reinterpret_cast<const Plan*>(plan);
  const SparseLayout L = sparse_layout(P, std::max<int64_t>(n_recv, 0), std::max<int64_t>(n_send, 0),
                                       std::max<int64_t>(E, 0));
  cgtp_status st = sparse_checks(P, n_recv, n_send, E, rowptr, gate, workspace, workspace_bytes, L.total);
  if (st != CGTP_OK) return st;
  if (n_recv == 0) return CGTP_OK;
  if (E > 0 && (!col || !x || !Y || !W)) return fail(CGTP_ERR_NULL, "col, x, Y or W is NULL");
  for (const void* p : {(const void*)x, (const void*)Y, (const void*)W, (const void*)out, (const void*)gate})
    if (p && !aligned16(p)) return fail(CGTP_ERR_ALIGN, "float arrays must be 16-byte aligned");
  if (E > 0) {
    st = check_graph(const_cast<Plan&>(P), n_recv, n_send, E, rowptr, col, nullptr, nullptr, stream);
    if (st != CGTP_OK) return st;
  }
  cudaStream_t s = (cudaStream_t)stream;
  CGTP_CUDA_TRY(launch_compaction(P, n_recv, n_send, E, rowptr, col, nullptr, nullptr, gate, Y, L, workspace, s));
  const Compact c = carve(L, workspace);
  // E (the full count) bounds the compact edges; the kernels read the
  // compact count from rowptr_A on the device
  return forward_impl(plan, n_recv, n_send, E, c.rowptr_A, c.col_A, x, c.Y_A, W, E > 0 ? c.eid : nullptr, out,
                      stream, false);
}

cgtp_status cgtp_sparse_backward(cgtp_plan plan, int64_t n_recv, int64_t n_send, int64_t E, const int32_t* rowptr,
                                 const int32_t* col, const int32_t* rowptr_T, const int32_t* perm_T,
                                 const float* x, const float* Y, const float* W, const float* gate,
                                 const float* grad_out, float* grad_x, float* grad_W, float* grad_Y,
                                 float* grad_gate, void* workspace, size_t workspace_bytes, cgtp_stream stream) {
  NvtxRange nvtx_range("cgtp_sparse_backward");
  if (!plan) return fail(CGTP_ERR_NULL, "plan is NULL");
  const Plan& P = *reinterpret_cast<const Plan*>(plan);
  const SparseLayout L = sparse_layout(P, std::max<int64_t>(n_recv, 0), std::max<int64_t>(n_send, 0),
                                       std::max<int64_t>(E, 0));
  cgtp_status st = sparse_checks(P, n_recv, n_send, E, rowptr, gate, workspace, workspace_bytes, L.total);
  if (st != CGTP_OK) return st;
  st = backward_validate(P, n_recv, n_send, E, rowptr, col, rowptr_T, perm_T, x, Y, W, grad_out, grad_x, grad_W,
                         grad_Y);
  if (st != CGTP_OK) return st;
  for (const void* p : {(const void*)gate, (const void*)grad_gate})
    if (p && !aligned16(p)) return fail(CGTP_ERR_ALIGN, "float arrays must be 16-byte aligned");
  cudaStream_t s = (cudaStream_t)stream;
  if (E == 0) {  // no edges: grad_x is zero, the per-edge outputs are empty
    return backward_impl(plan, n_recv, n_send, 0, rowptr, col, rowptr_T, perm_T, x, Y, W, grad_out, grad_x,
                         nullptr, nullptr, nullptr, 0, stream, true, nullptr, false);
  }
  st = check_graph(const_cast<Plan&>(P), n_recv, n_send, E, rowptr, col, grad_x ? rowptr_T : nullptr,
                   grad_x ? perm_T : nullptr, stream);
  if (st != CGTP_OK) return st;
  CGTP_CUDA_TRY(launch_compaction(P, n_recv, n_send, E, rowptr, col, grad_x ? rowptr_T : nullptr,
                                  grad_x ? perm_T : nullptr, gate, Y, L, workspace, s));
  const Compact c = carve(L, workspace);
  const bool want_dy = grad_Y || grad_gate;
  st = backward_impl(plan, n_recv, n_send, E, c.rowptr_A, c.col_A, c.rowptr_TA, c.perm_TA, x, c.Y_A, W, grad_out,
                     grad_x, grad_W, want_dy ? c.dY_A : nullptr, c.bwd, c.bwd_bytes, stream, true, c.eid, false);
  if (st != CGTP_OK) return st;
  if (!want_dy && !grad_W) return CGTP_OK;
  const int64_t blocks = std::min<int64_t>((E + 7) / 8, (int64_t)P.num_sms * 8);
  sparse_pad_kernel<<<(unsigned)blocks, 256, 0, s>>>(E, (int)P.D_e, P.U, gate, Y, c.pos,
                                                     want_dy ? c.dY_A : nullptr, grad_W, grad_Y, grad_gate);
  CGTP_CUDA_TRY(cudaGetLastError());
  return CGTP_OK;
}

}  // extern "C"
