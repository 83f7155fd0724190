// capi.cpp -- the extern "C" surface of libcgtp (declared in include/cgtp.h).
// Argument marshalling and validation only; the work runs in the kernels.
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <string>

#include "double_backward.hpp"
#include "internal.hpp"

namespace cgtp {

static thread_local std::string t_err = "no error";

void set_error(const std::string& msg) { t_err = msg; }

cgtp_status fail(cgtp_status s, const std::string& msg) {
  t_err = std::string(cgtp_status_string(s)) + ": " + msg;
  return s;
}

cgtp_status neighbor_list_impl(int64_t, const double*, const double*, double, int32_t*, int32_t*,
                               int32_t*, float*, int64_t*);
cgtp_status csr_transpose_impl(int64_t, int64_t, int64_t, const int32_t*, const int32_t*, int32_t*,
                               int32_t*);

void destroy_plan_device(Plan& P) {
  for (auto& t : P.tlog) {
    cudaEventDestroy(t.a);
    cudaEventDestroy(t.b);
  }
  for (auto e : P.tpool) cudaEventDestroy(e);
  P.tlog.clear();
  P.tpool.clear();
  jit_unload(P.fwd);
  jit_unload(P.bwd);
  jit_unload(P.bwd_er);
  jit_unload(P.fwd_tan);
  jit_unload(P.fwd_acc);
  jit_unload(P.bwd_tan);
  for (void** p : {&P.d_fwd_ent, &P.d_bwd_ent}) {
    if (*p) cudaFree(*p);
    *p = nullptr;
  }
  if (P.d_err) cudaFree(P.d_err);
  P.d_err = nullptr;
  if (P.d_csr) cudaFree(P.d_csr);
  P.d_csr = nullptr;
}

static bool aligned16(const void* p) { return ((uintptr_t)p & 15) == 0; }

static cgtp_status check_device(const Plan& P) {
  int dev = -1;
  CGTP_CUDA_TRY(cudaGetDevice(&dev));
  if (dev != P.device)
    return fail(CGTP_ERR_CUDA, "plan was created on device " + std::to_string(P.device) +
                                   " but device " + std::to_string(dev) + " is current");
  if (P.host_only) return fail(CGTP_ERR_CUDA, "plan was built without a device (compile-only)");
  return CGTP_OK;
}

static const char* kKindName[] = {"sph_harm",     "cgtp_fwd",  "cgtp_bwd",     "bwd_reduce",  "sph_harm_bwd",
                                  "zero_fill",    "cgtp_fwd_tan", "cgtp_bwd_tan", "cgtp_fwd_acc"};

// Brackets one internal launch with events when timing is on.
struct TimedScope {
  Plan& P;
  int kind;
  cudaStream_t s;
  cudaEvent_t a = nullptr, b = nullptr;
  static cudaEvent_t take(Plan& P) {
    if (!P.tpool.empty()) {
      cudaEvent_t e = P.tpool.back();
      P.tpool.pop_back();
      return e;
    }
    cudaEvent_t e = nullptr;
    if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
    return e;
  }
  TimedScope(Plan& P_, int k, cudaStream_t st, bool allowed = true) : P(P_), kind(k), s(st) {
    if (!allowed || !P.timing) return;
    std::lock_guard<std::mutex> g(P.tmu);
    a = take(P);
    b = take(P);
    if (a) cudaEventRecord(a, s);
  }
  ~TimedScope() {
    if (!a || !b) return;
    cudaEventRecord(b, s);
    std::lock_guard<std::mutex> g(P.tmu);
    P.tlog.push_back({kind, a, b});
  }
};

// Persistent grid: about one wave of resident CTAs; each walks the slices in
// order and, inside a slice, the receivers blockIdx.x, + gridDim.x, ...
static unsigned persistent_grid(int blocks_per_sm, int num_sms, int64_t n_recv) {
  const int64_t T = std::max<int64_t>(1, (int64_t)blocks_per_sm * num_sms);
  return (unsigned)std::max<int64_t>(1, std::min<int64_t>(T, n_recv));
}

// Backward workspace: the per-edge messages for dx [E x D_in] and the
// per-slice dY partials [S x E x D_e] when S > 1.  Returns the total bytes;
// the partials' offset through the pointer when given.
static size_t bwd_workspace_layout(const Plan& P, int64_t E, size_t* off_dyp) {
  auto r256 = [](size_t v) { return (v + 255) & ~size_t(255); };
  size_t b = r256((size_t)E * P.D_in * sizeof(float));
  if (off_dyp) *off_dyp = b;
  if (P.bcfg.S > 1) b += r256((size_t)P.bcfg.S * E * P.D_e * sizeof(float));
  return b;
}

// Double-backward workspace: the backward's own workspace, then one scratch
// buffer per output (grad_out, x, W, Y) for a term added to an earlier one.
struct DbwdLayout {
  size_t bwd, f, x, w, y, total;
};
static DbwdLayout dbwd_workspace_layout(const Plan& P, int64_t n_recv, int64_t n_send, int64_t E) {
  auto r256 = [](size_t v) { return (v + 255) & ~size_t(255); };
  DbwdLayout L;
  L.bwd = 0;
  L.f = r256(bwd_workspace_layout(P, E, nullptr));
  L.x = L.f + r256((size_t)n_recv * P.D_out * sizeof(float));
  L.w = L.x + r256((size_t)n_send * P.D_in * sizeof(float));
  L.y = L.w + r256((size_t)E * P.U * sizeof(float));
  L.total = L.y + r256((size_t)E * P.D_e * sizeof(float));
  return L;
}

}  // namespace cgtp

using namespace cgtp;

extern "C" {

const char* cgtp_status_string(cgtp_status s) {
  switch (s) {
    case CGTP_OK: return "CGTP_OK";
    case CGTP_ERR_NULL: return "CGTP_ERR_NULL";
    case CGTP_ERR_ALIGN: return "CGTP_ERR_ALIGN";
    case CGTP_ERR_IRREPS_PARSE: return "CGTP_ERR_IRREPS_PARSE";
    case CGTP_ERR_IRREPS_MISMATCH: return "CGTP_ERR_IRREPS_MISMATCH";
    case CGTP_ERR_LMAX: return "CGTP_ERR_LMAX";
    case CGTP_ERR_SIZE: return "CGTP_ERR_SIZE";
    case CGTP_ERR_INVALID_CSR: return "CGTP_ERR_INVALID_CSR";
    case CGTP_ERR_CUDA: return "CGTP_ERR_CUDA";
    case CGTP_ERR_OOM: return "CGTP_ERR_OOM";
    case CGTP_ERR_TIMEOUT: return "CGTP_ERR_TIMEOUT";
    case CGTP_ERR_JIT: return "CGTP_ERR_JIT";
    case CGTP_ERR_WORKSPACE: return "CGTP_ERR_WORKSPACE";
  }
  return "CGTP_ERR_UNKNOWN";
}

const char* cgtp_last_error(void) { return t_err.c_str(); }

cgtp_status cgtp_plan_create(const char* irreps_in, const char* irreps_edge, const char* irreps_out,
                             int lmax, cgtp_plan* out) {
  NvtxRange nvtx_range("cgtp_plan_create");
  if (!out) return fail(CGTP_ERR_NULL, "out is NULL");
  *out = nullptr;
  if (!irreps_in || !irreps_edge || !irreps_out) return fail(CGTP_ERR_NULL, "irreps string is NULL");
  std::unique_ptr<Plan> P;
  try {
    P.reset(new Plan());
  } catch (...) {
    return fail(CGTP_ERR_OOM, "host allocation failed");
  }
  P->irreps_in_s = irreps_in;
  P->irreps_edge_s = irreps_edge;
  P->irreps_out_s = irreps_out;
  P->lmax = lmax;
  cgtp_status st;
  try {
    st = build_paths(*P);
    if (st != CGTP_OK) return st;
    P->host_only = std::getenv("CGTP_JIT_COMPILE_ONLY") != nullptr;
    if (!P->host_only) {
      CGTP_CUDA_TRY(cudaGetDevice(&P->device));
      CGTP_CUDA_TRY(cudaDeviceGetAttribute(&P->num_sms, cudaDevAttrMultiProcessorCount, P->device));
      CGTP_CUDA_TRY(cudaFree(0));  // make the primary context current
      if (cudaMalloc(&P->d_err, sizeof(int)) != cudaSuccess) return fail(CGTP_ERR_OOM, "cudaMalloc");
      CGTP_CUDA_TRY(cudaMemset(P->d_err, 0, sizeof(int)));
      if (cudaMalloc(&P->d_csr, sizeof(int)) != cudaSuccess) return fail(CGTP_ERR_OOM, "cudaMalloc");
      CGTP_CUDA_TRY(upload_sph_norm());  // once per device, before any capture
      if (const char* d = std::getenv("CGTP_DEBUG"); d && *d && *d != '0') P->checks.store(CGTP_CHECK_GRAPH);
    }
    if (const char* v = std::getenv("CGTP_BWD_TFORM"); v && *v == '0') P->bwd_tform = false;
    if (const char* v = std::getenv("CGTP_FWD_PACKED"); v && (*v == '0' || *v == '1')) P->fwd_packed = *v - '0';
    if (const char* v = std::getenv("CGTP_DBWD_FWD")) {
      if (std::string(v) == "tangent") P->dbwd_fwd_sum = 0;
      if (std::string(v) == "sum") P->dbwd_fwd_sum = 1;
    }
    st = build_forward(*P);  // leaves the forward compiling on a host thread
    if (st == CGTP_OK) st = build_backward(*P);
    if (st == CGTP_OK)
      st = finish_forward(*P);
    else
      P->fwd_pending.reset();  // joins; its result is not needed
  } catch (const std::exception& e) {
    P->fwd_pending.reset();
    destroy_plan_device(*P);
    return fail(CGTP_ERR_OOM, std::string("exception in plan create: ") + e.what());
  }
  if (st != CGTP_OK) {
    destroy_plan_device(*P);
    return st;
  }
  *out = reinterpret_cast<cgtp_plan>(P.release());
  return CGTP_OK;
}

cgtp_status cgtp_plan_destroy(cgtp_plan plan) {
  if (!plan) return CGTP_OK;
  Plan* P = reinterpret_cast<Plan*>(plan);
  destroy_plan_device(*P);
  delete P;
  return CGTP_OK;
}

cgtp_status cgtp_plan_info(cgtp_plan plan, int64_t* d_in, int64_t* d_edge, int64_t* d_out,
                           int64_t* n_weights, int64_t* n_paths) {
  if (!plan) return fail(CGTP_ERR_NULL, "plan is NULL");
  const Plan* P = reinterpret_cast<const Plan*>(plan);
  if (d_in) *d_in = P->D_in;
  if (d_edge) *d_edge = P->D_e;
  if (d_out) *d_out = P->D_out;
  if (n_weights) *n_weights = P->U;
  if (n_paths) *n_paths = (int64_t)P->paths.size();
  return CGTP_OK;
}

cgtp_status cgtp_plan_paths(cgtp_plan plan, int32_t* table) {
  if (!plan || !table) return fail(CGTP_ERR_NULL, "null argument");
  const Plan* P = reinterpret_cast<const Plan*>(plan);
  for (size_t k = 0; k < P->paths.size(); ++k) {
    const Path& p = P->paths[k];
    const int32_t row[8] = {p.l1, p.l2, p.l3, p.mul, p.x_off, p.k0, p.o_off, p.c_off};
    std::memcpy(table + 8 * k, row, sizeof row);
  }
  return CGTP_OK;
}

cgtp_status cgtp_plan_coefficients(cgtp_plan plan, double* coeff, int64_t* n_coeff) {
  if (!plan || !n_coeff) return fail(CGTP_ERR_NULL, "null argument");
  const Plan* P = reinterpret_cast<const Plan*>(plan);
  *n_coeff = (int64_t)P->coeff.size();
  if (coeff) std::memcpy(coeff, P->coeff.data(), P->coeff.size() * sizeof(double));
  return CGTP_OK;
}

cgtp_status cgtp_real_cg(int l1, int l2, int l3, double* C) {
  if (!C) return fail(CGTP_ERR_NULL, "C is NULL");
  if (l1 < 0 || l2 < 0 || l1 > 12 || l2 > 12) return fail(CGTP_ERR_LMAX, "degrees must be in 0..12");
  std::vector<double> v;
  if (!real_cg_block(l1, l2, l3, v)) return fail(CGTP_ERR_SIZE, "triangle rule violated");
  std::memcpy(C, v.data(), v.size() * sizeof(double));
  return CGTP_OK;
}

cgtp_status cgtp_sph_harm(cgtp_plan plan, int64_t E, const float* r, float* Y, cgtp_stream stream) {
  NvtxRange nvtx_range("cgtp_sph_harm");
  if (!plan) return fail(CGTP_ERR_NULL, "plan is NULL");
  const Plan* P = reinterpret_cast<const Plan*>(plan);
  if (E < 0 || E >= (int64_t(1) << 31)) return fail(CGTP_ERR_SIZE, "E out of range");
  if (E == 0) return CGTP_OK;
  if (!r || !Y) return fail(CGTP_ERR_NULL, "r or Y is NULL");
  if (!aligned16(r) || !aligned16(Y)) return fail(CGTP_ERR_ALIGN, "r and Y must be 16-byte aligned");
  cgtp_status st = check_device(*P);
  if (st != CGTP_OK) return st;
  {
    TimedScope ts(*const_cast<Plan*>(P), 0, (cudaStream_t)stream);
    CGTP_CUDA_TRY(launch_sph_harm(P->L, E, r, Y, (cudaStream_t)stream));
  }
  return CGTP_OK;
}

cgtp_status cgtp_sph_harm_backward(cgtp_plan plan, int64_t E, const float* r, const float* grad_Y,
                                   float* grad_r, cgtp_stream stream) {
  NvtxRange nvtx_range("cgtp_sph_harm_backward");
  if (!plan) return fail(CGTP_ERR_NULL, "plan is NULL");
  const Plan* P = reinterpret_cast<const Plan*>(plan);
  if (E < 0 || E >= (int64_t(1) << 31)) return fail(CGTP_ERR_SIZE, "E out of range");
  if (E == 0) return CGTP_OK;
  if (!r || !grad_Y || !grad_r) return fail(CGTP_ERR_NULL, "r, grad_Y or grad_r is NULL");
  if (!aligned16(r) || !aligned16(grad_Y) || !aligned16(grad_r))
    return fail(CGTP_ERR_ALIGN, "r, grad_Y and grad_r must be 16-byte aligned");
  cgtp_status st = check_device(*P);
  if (st != CGTP_OK) return st;
  {
    TimedScope ts(*const_cast<Plan*>(P), 4, (cudaStream_t)stream);
    CGTP_CUDA_TRY(launch_sph_harm_backward(P->L, E, r, grad_Y, grad_r, (cudaStream_t)stream));
  }
  return CGTP_OK;
}

cgtp_status cgtp_edge_forces(int64_t n_atoms, int64_t E, const int32_t* rowptr, const int32_t* rowptr_T,
                             const int32_t* perm_T, const float* grad_r, float* forces, cgtp_stream stream) {
  NvtxRange nvtx_range("cgtp_edge_forces");
  if (n_atoms < 0 || E < 0 || n_atoms >= (int64_t(1) << 31) || E >= (int64_t(1) << 31))
    return fail(CGTP_ERR_SIZE, "sizes out of range");
  if (n_atoms == 0) return CGTP_OK;
  if (!rowptr || !rowptr_T || !forces) return fail(CGTP_ERR_NULL, "rowptr, rowptr_T or forces is NULL");
  if (E > 0 && (!perm_T || !grad_r)) return fail(CGTP_ERR_NULL, "perm_T or grad_r is NULL");
  CGTP_CUDA_TRY(launch_edge_forces(n_atoms, rowptr, rowptr_T, perm_T, grad_r, forces, (cudaStream_t)stream));
  return CGTP_OK;
}

cgtp_status cgtp_edge_virial(int64_t E, const float* r, const float* grad_r, float* virial, cgtp_stream stream) {
  NvtxRange nvtx_range("cgtp_edge_virial");
  if (E < 0 || E >= (int64_t(1) << 31)) return fail(CGTP_ERR_SIZE, "E out of range");
  if (!virial) return fail(CGTP_ERR_NULL, "virial is NULL");
  if (E > 0 && (!r || !grad_r)) return fail(CGTP_ERR_NULL, "r or grad_r is NULL");
  if (E > 0 && (!aligned16(r) || !aligned16(grad_r)))
    return fail(CGTP_ERR_ALIGN, "r and grad_r must be 16-byte aligned");
  CGTP_CUDA_TRY(launch_edge_virial(E, r, grad_r, virial, (cudaStream_t)stream));
  return CGTP_OK;
}

cgtp_status cgtp_forward(cgtp_plan plan, int64_t n_recv, int64_t n_send, int64_t E,
                         const int32_t* rowptr, const int32_t* col, const float* x, const float* Y,
                         const float* W, float* out, cgtp_stream stream) {
  NvtxRange nvtx_range("cgtp_forward");
  return cgtp::forward_impl(plan, n_recv, n_send, E, rowptr, col, x, Y, W, nullptr, out, stream, true);
}

cgtp_status cgtp_backward_workspace_size(cgtp_plan plan, int64_t n_recv, int64_t n_send, int64_t E,
                                         size_t* bytes) {
  if (!plan || !bytes) return fail(CGTP_ERR_NULL, "null argument");
  const Plan* P = reinterpret_cast<const Plan*>(plan);
  if (n_recv < 0 || n_send < 0 || E < 0) return fail(CGTP_ERR_SIZE, "negative size");
  *bytes = bwd_workspace_layout(*P, E, nullptr);
  return CGTP_OK;
}

cgtp_status cgtp_backward(cgtp_plan plan, int64_t n_recv, int64_t n_send, int64_t E,
                          const int32_t* rowptr, const int32_t* col, const int32_t* rowptr_T,
                          const int32_t* perm_T, const float* x, const float* Y, const float* W,
                          const float* grad_out, float* grad_x, float* grad_W, float* grad_Y,
                          void* workspace, size_t workspace_bytes, cgtp_stream stream) {
  NvtxRange nvtx_range("cgtp_backward");
  return cgtp::backward_impl(plan, n_recv, n_send, E, rowptr, col, rowptr_T, perm_T, x, Y, W,
                             grad_out, grad_x, grad_W, grad_Y, workspace, workspace_bytes, stream,
                             true, nullptr, true);
}

}  // extern "C"

namespace cgtp {

// The double backward's tangent kernels, built once per plan under its lock
// (CGTP_DBWD_COMPOSE=1 at build time keeps the composition of plain calls).
// Returns whether they are available; a build failure is remembered, not
// returned: the composition remains.
static bool ensure_tangent(Plan& P) {
  std::lock_guard<std::mutex> g(P.tan_mu);
  if (P.tan_state != 0) return P.tan_state > 0;
  if (const char* v = std::getenv("CGTP_DBWD_COMPOSE"); v && *v && *v != '0') {
    P.tan_state = -1;
    P.tan_msg = "tangent kernels switched off (CGTP_DBWD_COMPOSE)";
    return false;
  }
  if (P.fwd_roles.empty() || P.bwd_roles.empty()) {
    P.tan_state = -1;
    P.tan_msg = "no paths";
    return false;
  }
  // gg_out: the tangent forward, or the sum of one plain and two
  // accumulating forwards.  Which is faster depends on the plan (Lmax 3: the
  // tangent forward 1773 us against 3 x 453; Case 5: 1019 against 1193), so
  // both are built unless CGTP_DBWD_FWD fixes one, and the first double
  // backward timed outside stream capture chooses (dbwd_fwd_sum).
  std::string fsrc, asrc, bsrc;
  cgtp_status st = CGTP_OK;
  if (P.dbwd_fwd_sum != 1) {
    st = build_forward_tangent(P, P.fwd_tan, &fsrc);
    if (st != CGTP_OK && P.dbwd_fwd_sum < 0) {  // e.g. doubled stages too large: the sum remains
      jit_unload(P.fwd_tan);
      P.dbwd_fwd_sum = 1;
      st = CGTP_OK;
    }
  }
  if (st == CGTP_OK && P.dbwd_fwd_sum != 0) st = build_forward_accumulate(P, P.fwd_acc, &asrc);
  if (st == CGTP_OK) st = build_backward_tangent(P, P.bwd_tan, &bsrc);
  if (st != CGTP_OK) {
    P.tan_msg = cgtp_last_error();
    jit_unload(P.fwd_tan);
    jit_unload(P.fwd_acc);
    jit_unload(P.bwd_tan);
    P.tan_state = -1;
    return false;
  }
  if (const char* d = std::getenv("CGTP_DUMP_SOURCE")) {
    for (auto [name, src] : {std::pair<const char*, std::string*>{"/fwd_tan.cu", &fsrc}, {"/fwd_acc.cu", &asrc},
                             {"/bwd_tan.cu", &bsrc}}) {
      if (src->empty()) continue;
      if (FILE* f = std::fopen((std::string(d) + name).c_str(), "w")) {
        std::fputs(src->c_str(), f);
        std::fclose(f);
      }
    }
  }
  P.tan_state = 1;
  return true;
}

cgtp_status forward_impl(cgtp_plan plan, int64_t n_recv, int64_t n_send, int64_t E, const int32_t* rowptr,
                         const int32_t* col, const float* x, const float* Y, const float* W, const int32_t* eid,
                         float* out, cgtp_stream stream, bool graph_checks) {
  if (!plan) return fail(CGTP_ERR_NULL, "plan is NULL");
  Plan* P = reinterpret_cast<Plan*>(plan);
  if (n_recv < 0 || n_send < 0 || E < 0 || n_recv >= (int64_t(1) << 31) ||
      n_send >= (int64_t(1) << 31) || E >= (int64_t(1) << 31) - 1)
    return fail(CGTP_ERR_SIZE, "sizes out of range");
  if (n_recv == 0) return CGTP_OK;
  if (!rowptr || !out) return fail(CGTP_ERR_NULL, "rowptr or out is NULL");
  if (E > 0 && (!col || !Y || !W || !x)) return fail(CGTP_ERR_NULL, "col, x, Y or W is NULL");
  if (E > 0 && n_send == 0) return fail(CGTP_ERR_SIZE, "edges without senders");
  for (const void* p : {(const void*)x, (const void*)Y, (const void*)W, (const void*)out})
    if (p && !aligned16(p)) return fail(CGTP_ERR_ALIGN, "float arrays must be 16-byte aligned");
  cgtp_status st = check_device(*P);
  if (st != CGTP_OK) return st;
  if (graph_checks && E > 0) {
    st = check_graph(*P, n_recv, n_send, E, rowptr, col, nullptr, nullptr, stream);
    if (st != CGTP_OK) return st;
  }
  cudaStream_t s = (cudaStream_t)stream;
  if (P->fwd_roles.empty()) {
    CGTP_CUDA_TRY(cudaMemsetAsync(out, 0, (size_t)n_recv * P->D_out * sizeof(float), s));
    return CGTP_OK;
  }
  int nr = (int)n_recv;
  // persistent CTAs: about one wave of resident CTAs, each walking its slice's
  // receivers first, first + stride, ...
  void* args[] = {&rowptr, &col, &x, &Y, &W, &eid, &out, &P->d_fwd_ent, &nr, &P->d_err};
  TimedScope ts(*P, 1, s);
  return jit_launch(P->fwd, dim3(persistent_grid(P->fwd.blocks_per_sm, P->num_sms, n_recv)), args, s);
}

cgtp_status check_plan_device(const Plan& P) { return check_device(P); }

cgtp_status check_graph(Plan& P, int64_t n_recv, int64_t n_send, int64_t E, const int32_t* rowptr,
                        const int32_t* col, const int32_t* rowptr_T, const int32_t* perm_T, cgtp_stream stream,
                        bool always) {
  if ((!always && !(P.checks.load() & CGTP_CHECK_GRAPH)) || (n_recv == 0 && E == 0)) return CGTP_OK;
  if (!rowptr || (E > 0 && !col)) return fail(CGTP_ERR_NULL, "rowptr or col is NULL");
  if (!rowptr_T || !perm_T) rowptr_T = nullptr, perm_T = nullptr;
  cudaStream_t s = (cudaStream_t)stream;
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  CGTP_CUDA_TRY(cudaStreamIsCapturing(s, &cs));
  if (cs != cudaStreamCaptureStatusNone)
    return fail(CGTP_ERR_CUDA, "the graph checks wait for their result; turn them off under stream capture");
  std::lock_guard<std::mutex> g(P.csr_mu);  // one result word per plan
  int h = 0;
  CGTP_CUDA_TRY(cudaMemsetAsync(P.d_csr, 0, sizeof(int), s));
  CGTP_CUDA_TRY(launch_csr_check(P.num_sms, n_recv, n_send, E, rowptr, col, rowptr_T, perm_T, P.d_csr, s));
  CGTP_CUDA_TRY(cudaMemcpyAsync(&h, P.d_csr, sizeof(int), cudaMemcpyDeviceToHost, s));
  CGTP_CUDA_TRY(cudaStreamSynchronize(s));
  if (h == 0) return CGTP_OK;
  static const char* what[] = {"rowptr does not run from 0 to E", "rowptr decreases",
                               "a col entry lies outside [0, n_send)", "rowptr_T does not run from 0 to E",
                               "rowptr_T decreases", "a perm_T entry lies outside [0, E)",
                               "a perm_T entry lists an edge of another sender",
                               "perm_T is not ascending within a sender"};
  std::string msg = "graph checks failed:";
  for (int b = 0; b < 8; ++b)
    if (h & (1 << b)) msg += std::string(" ") + what[b] + ";";
  return fail(CGTP_ERR_INVALID_CSR, msg);
}

// The scratch bytes one backward call uses: the per-edge messages when grad_x
// is wanted (first), and the slice parts of dY when grad_Y is wanted from a
// plan of several slices (after the messages, or at offset 0 without them).
size_t backward_scratch_bytes(const Plan& P, int64_t E, bool want_x, bool want_Y, size_t* off_dyp) {
  auto r256 = [](size_t v) { return (v + 255) & ~size_t(255); };
  const size_t msg = want_x ? r256((size_t)E * P.D_in * sizeof(float)) : 0;
  if (off_dyp) *off_dyp = msg;
  const size_t parts = (want_Y && P.bcfg.S > 1) ? r256((size_t)P.bcfg.S * E * P.D_e * sizeof(float)) : 0;
  return msg + parts;
}

cgtp_status backward_validate(const Plan& P, int64_t n_recv, int64_t n_send, int64_t E, const int32_t* rowptr,
                              const int32_t* col, const int32_t* rowptr_T, const int32_t* perm_T, const float* x,
                              const float* Y, const float* W, const float* grad_out, const float* grad_x,
                              const float* grad_W, const float* grad_Y) {
  if (n_recv < 0 || n_send < 0 || E < 0 || n_recv >= (int64_t(1) << 31) ||
      n_send >= (int64_t(1) << 31) || E >= (int64_t(1) << 31) - 1)
    return fail(CGTP_ERR_SIZE, "sizes out of range");
  cgtp_status st = check_device(P);
  if (st != CGTP_OK) return st;
  for (const void* p : {(const void*)x, (const void*)Y, (const void*)W, (const void*)grad_out,
                        (const void*)grad_x, (const void*)grad_W, (const void*)grad_Y})
    if (p && !aligned16(p)) return fail(CGTP_ERR_ALIGN, "float arrays must be 16-byte aligned");
  if (E == 0) return CGTP_OK;
  if (!rowptr || !col || !x || !Y || !W || !grad_out)
    return fail(CGTP_ERR_NULL, "rowptr, col, x, Y, W or grad_out is NULL");
  if (grad_x && (!rowptr_T || !perm_T)) return fail(CGTP_ERR_NULL, "grad_x needs rowptr_T and perm_T");
  return CGTP_OK;
}

cgtp_status backward_impl(cgtp_plan plan, int64_t n_recv, int64_t n_send, int64_t E,
                          const int32_t* rowptr, const int32_t* col, const int32_t* rowptr_T,
                          const int32_t* perm_T, const float* x, const float* Y, const float* W,
                          const float* grad_out, float* grad_x, float* grad_W, float* grad_Y,
                          void* workspace, size_t workspace_bytes, cgtp_stream stream,
                          bool allow_timing, const int32_t* eid, bool graph_checks) {
  if (!plan) return fail(CGTP_ERR_NULL, "plan is NULL");
  Plan* P = reinterpret_cast<Plan*>(plan);
  cgtp_status st = backward_validate(*P, n_recv, n_send, E, rowptr, col, rowptr_T, perm_T, x, Y, W, grad_out,
                                     grad_x, grad_W, grad_Y);
  if (st != CGTP_OK) return st;
  if (graph_checks && E > 0) {
    st = check_graph(*P, n_recv, n_send, E, rowptr, col, grad_x ? rowptr_T : nullptr, grad_x ? perm_T : nullptr,
                     stream);
    if (st != CGTP_OK) return st;
  }
  cudaStream_t s = (cudaStream_t)stream;
  if (grad_x && n_send > 0 && (E == 0 || P->bwd_roles.empty()))
    CGTP_CUDA_TRY(cudaMemsetAsync(grad_x, 0, (size_t)n_send * P->D_in * sizeof(float), s));
  if (E == 0) return CGTP_OK;
  if (P->bwd_roles.empty()) {
    if (grad_W) CGTP_CUDA_TRY(cudaMemsetAsync(grad_W, 0, (size_t)E * P->U * sizeof(float), s));
    if (grad_Y) CGTP_CUDA_TRY(cudaMemsetAsync(grad_Y, 0, (size_t)E * P->D_e * sizeof(float), s));
    return CGTP_OK;
  }
  size_t off_dyp = 0;
  const size_t need = backward_scratch_bytes(*P, E, grad_x != nullptr, grad_Y != nullptr, &off_dyp);
  const bool need_ws = need > 0;
  if (need_ws && (!workspace || workspace_bytes < need))
    return fail(CGTP_ERR_WORKSPACE, "workspace of " + std::to_string(need) + " bytes required");
  if (need_ws && ((uintptr_t)workspace & 255))
    return fail(CGTP_ERR_ALIGN, "workspace must be 256-byte aligned");
  char* wsb = reinterpret_cast<char*>(workspace);
  float* m = grad_x ? reinterpret_cast<float*>(wsb) : nullptr;
  float* dyp = nullptr;
  if (grad_Y) dyp = P->bcfg.S > 1 ? reinterpret_cast<float*>(wsb + off_dyp) : grad_Y;
  if (m && P->bwd_irrep_gap) {  // hidden irreps without paths receive zero gradient
    TimedScope ts(*P, 5, s, allow_timing);
    CGTP_CUDA_TRY(cudaMemsetAsync(m, 0, (size_t)E * P->D_in * sizeof(float), s));
  }
  if (n_recv > 0) {
    int nr = (int)n_recv;
    // few receivers per CTA: equal edge ranges keep the CTAs' work even
    unsigned G = persistent_grid(P->bwd.blocks_per_sm, P->num_sms, n_recv);
    const bool er = P->bwd_er.function && n_recv <= 8 * (int64_t)G;
    JitKernel& JK = er ? P->bwd_er : P->bwd;
    if (er) G = persistent_grid(P->bwd_er.blocks_per_sm, P->num_sms, n_recv);
    int e_stride = (int)E;  // the slices' dY parts lie E edges apart
    void* args[] = {&rowptr, &col, &x, &Y, &W, &eid, &grad_out, &grad_W, &dyp, &m, &P->d_bwd_ent, &nr, &P->d_err,
                    &e_stride};
    TimedScope ts(*P, 2, s, allow_timing);
    st = jit_launch(JK, dim3(G), args, s);
    if (st != CGTP_OK) return st;
  }
  if (grad_x || (grad_Y && P->bcfg.S > 1)) {
    TimedScope ts(*P, 3, s, allow_timing);
    CGTP_CUDA_TRY(launch_bwd_reduce(n_send, P->D_in, rowptr_T, perm_T, m, grad_x, P->bcfg.S, E * P->D_e, dyp,
                                    (grad_Y && P->bcfg.S > 1) ? grad_Y : nullptr, s));
  }
  return CGTP_OK;
}


}  // namespace cgtp

extern "C" {

cgtp_status cgtp_plan_describe(cgtp_plan plan, char* buf, size_t n, size_t* needed) {
  if (!plan) return fail(CGTP_ERR_NULL, "plan is NULL");
  const Plan* P = reinterpret_cast<const Plan*>(plan);
  std::string t;
  t += "irreps_in=" + P->irreps_in_s + " irreps_edge=" + P->irreps_edge_s + " irreps_out=" +
       P->irreps_out_s + "\n";
  t += "D_in=" + std::to_string(P->D_in) + " D_e=" + std::to_string(P->D_e) + " D_out=" +
       std::to_string(P->D_out) + " U=" + std::to_string(P->U) + " paths=" +
       std::to_string(P->paths.size()) + "\n";
  auto cfg = [&](const char* nm, const FwdConfig& F, const JitKernel& k, size_t nroles) {
    t += std::string(nm) + ": roles=" + std::to_string(nroles) + " slices=" + std::to_string(F.S) +
         " warps=" + std::to_string(F.nw) + "+2 chunk=" + std::to_string(F.B) + " stages=" +
         std::to_string(F.stages) + " w_smem=" + std::to_string((int)F.w_smem) + " x_smem=" +
         std::to_string((int)F.x_smem) + " nacc=" + std::to_string(F.nacc) + " smem=" +
         std::to_string(k.smem) + " threads=" + std::to_string(k.threads);
    char hx[40];
    std::snprintf(hx, sizeof hx, " hash=%016llx\n", k.hash);
    t += hx;
    for (size_t s = 0; s < F.slice_roles.size(); ++s) {
      t += "  slice " + std::to_string(s) + ":";
      for (int r : F.slice_roles[s]) t += " " + std::to_string(r);
      t += "\n";
    }
    t += k.log;
    if (!k.log.empty() && k.log.back() != '\n') t += "\n";
  };
  cfg("forward", P->fcfg, P->fwd, P->fwd_roles.size());
  for (size_t r = 0; r < P->fwd_roles.size(); ++r) {
    const FwdRole& q = P->fwd_roles[r];
    t += "  frole " + std::to_string(r) + ": irrep " + std::to_string(q.irrep) + " u0=" +
         std::to_string(q.u0) + " R=" + std::to_string(q.R) + " paths=" +
         std::to_string(q.paths.size()) + " cost=" + std::to_string((int)q.cost) + "\n";
  }
  cfg("backward", P->bcfg, P->bwd, P->bwd_roles.size());
  t += std::string("forward form=") + (P->fcfg.packed ? "packed" : "scalar") + "\n";
  t += std::string("backward form=") + (P->bwd_tform ? "cg_first" : "staged_chat") + "\n";
  for (size_t r = 0; r < P->bwd_roles.size(); ++r) {
    const BwdRole& q = P->bwd_roles[r];
    t += "  brole " + std::to_string(r) + ": irrep " + std::to_string(q.irrep) + " u0=" +
         std::to_string(q.u0) + " R=" + std::to_string(q.R) + " ph=" + std::to_string(q.ph) + "/" +
         std::to_string(q.nph) + " cost=" + std::to_string((int)q.cost) + "\n";
  }
  if (P->tan_state > 0)
    t += std::string("double backward forward=") +
         (P->dbwd_fwd_sum < 0 ? "undecided" : P->dbwd_fwd_sum ? "sum" : "tangent") + "\n";
  for (const JitKernel* k : {&P->fwd_tan, &P->fwd_acc, &P->bwd_tan}) {  // double-backward kernels, once built
    if (k->name.empty()) continue;
    char hx[64];
    std::snprintf(hx, sizeof hx, " smem=%d threads=%d hash=%016llx\n", k->smem, k->threads, k->hash);
    t += k->name + " (double backward):" + std::string(hx) + k->log;
    if (!k->log.empty() && k->log.back() != '\n') t += "\n";
  }
  {  // the edge-range variant of the backward (same roles and layout)
    char hx[40];
    std::snprintf(hx, sizeof hx, " hash=%016llx\n", P->bwd_er.hash);
    t += "backward (edge ranges, for at most 8 receivers per CTA):" + std::string(hx) + P->bwd_er.log;
    if (!P->bwd_er.log.empty() && P->bwd_er.log.back() != '\n') t += "\n";
  }
  if (needed) *needed = t.size() + 1;
  if (buf && n > 0) {
    const size_t k = std::min(n - 1, t.size());
    std::memcpy(buf, t.data(), k);
    buf[k] = '\0';
  }
  return CGTP_OK;
}

cgtp_status cgtp_plan_prepare_double_backward(cgtp_plan plan, int* tangent) {
  NvtxRange nvtx_range("cgtp_plan_prepare_double_backward");
  if (!plan) return fail(CGTP_ERR_NULL, "plan is NULL");
  Plan* P = reinterpret_cast<Plan*>(plan);
  if (!P->host_only) {  // a compile-only plan builds (and checks) the kernels' code only
    cgtp_status st = check_device(*P);
    if (st != CGTP_OK) return st;
  }
  const bool ok = ensure_tangent(*P);
  if (tangent) *tangent = ok ? 1 : 0;
  return CGTP_OK;
}

cgtp_status cgtp_plan_set_checks(cgtp_plan plan, int flags) {
  if (!plan) return fail(CGTP_ERR_NULL, "plan is NULL");
  if (flags & ~CGTP_CHECK_GRAPH) return fail(CGTP_ERR_SIZE, "unknown check flags");
  reinterpret_cast<Plan*>(plan)->checks.store(flags);
  return CGTP_OK;
}

cgtp_status cgtp_validate_graph(cgtp_plan plan, int64_t n_recv, int64_t n_send, int64_t E,
                                const int32_t* rowptr, const int32_t* col, const int32_t* rowptr_T,
                                const int32_t* perm_T, cgtp_stream stream) {
  NvtxRange nvtx_range("cgtp_validate_graph");
  if (!plan) return fail(CGTP_ERR_NULL, "plan is NULL");
  Plan* P = reinterpret_cast<Plan*>(plan);
  if (n_recv < 0 || n_send < 0 || E < 0 || n_recv >= (int64_t(1) << 31) ||
      n_send >= (int64_t(1) << 31) || E >= (int64_t(1) << 31) - 1)
    return fail(CGTP_ERR_SIZE, "sizes out of range");
  if ((rowptr_T == nullptr) != (perm_T == nullptr)) return fail(CGTP_ERR_NULL, "rowptr_T and perm_T go together");
  cgtp_status st = check_device(*P);
  if (st != CGTP_OK) return st;
  return check_graph(*P, n_recv, n_send, E, rowptr, col, rowptr_T, perm_T, stream, true);
}

cgtp_status cgtp_plan_set_timing(cgtp_plan plan, int enable) {
  if (!plan) return fail(CGTP_ERR_NULL, "plan is NULL");
  Plan* P = reinterpret_cast<Plan*>(plan);
  P->timing.store(enable != 0);
  return CGTP_OK;
}

cgtp_status cgtp_plan_kernel_times(cgtp_plan plan, int max, char* names, double* ms,
                                   int64_t* launches, int* n) {
  if (!plan || !n) return fail(CGTP_ERR_NULL, "null argument");
  Plan* P = reinterpret_cast<Plan*>(plan);
  const int K = (int)(sizeof(kKindName) / sizeof(kKindName[0]));
  std::vector<double> tot(K, 0.0);
  std::vector<int64_t> cnt(K, 0);
  std::vector<Plan::TimedLaunch> log;
  {
    std::lock_guard<std::mutex> g(P->tmu);
    log.swap(P->tlog);
  }
  cgtp_status st = CGTP_OK;
  for (auto& t : log) {
    float v = 0.f;
    if (st == CGTP_OK) {
      cudaError_t e = cudaEventSynchronize(t.b);
      if (e == cudaSuccess) e = cudaEventElapsedTime(&v, t.a, t.b);
      if (e != cudaSuccess) st = fail(CGTP_ERR_CUDA, std::string("event timing: ") + cudaGetErrorString(e));
    }
    tot[t.kind] += v;
    cnt[t.kind] += 1;
  }
  {
    std::lock_guard<std::mutex> g(P->tmu);
    for (auto& t : log) {
      P->tpool.push_back(t.a);
      P->tpool.push_back(t.b);
    }
  }
  int k = 0;
  for (int q = 0; q < K; ++q) {
    if (cnt[q] == 0) continue;
    if (k < max) {
      if (names) std::snprintf(names + 32 * k, 32, "%s", kKindName[q]);
      if (ms) ms[k] = tot[q];
      if (launches) launches[k] = cnt[q];
    }
    ++k;
  }
  *n = k;
  return st;
}

cgtp_status cgtp_plan_check_device_error(cgtp_plan plan, int* code) {
  if (!plan || !code) return fail(CGTP_ERR_NULL, "null argument");
  Plan* P = reinterpret_cast<Plan*>(plan);
  cgtp_status st = check_device(*P);
  if (st != CGTP_OK) return st;
  CGTP_CUDA_TRY(cudaDeviceSynchronize());
  int v = 0;
  CGTP_CUDA_TRY(cudaMemcpy(&v, P->d_err, sizeof(int), cudaMemcpyDeviceToHost));
  CGTP_CUDA_TRY(cudaMemset(P->d_err, 0, sizeof(int)));
  *code = v;
  if (v != 0) return fail(CGTP_ERR_TIMEOUT, "a bounded wait inside a kernel expired");
  return CGTP_OK;
}

cgtp_status cgtp_double_backward_workspace_size(cgtp_plan plan, int64_t n_recv, int64_t n_send, int64_t E,
                                                size_t* bytes) {
  if (!plan || !bytes) return fail(CGTP_ERR_NULL, "null argument");
  if (n_recv < 0 || n_send < 0 || E < 0) return fail(CGTP_ERR_SIZE, "negative size");
  *bytes = dbwd_workspace_layout(*reinterpret_cast<const Plan*>(plan), n_recv, n_send, E).total;
  return CGTP_OK;
}

cgtp_status cgtp_double_backward(cgtp_plan plan, int64_t n_recv, int64_t n_send, int64_t E,
                                 const int32_t* rowptr, const int32_t* col, const int32_t* rowptr_T,
                                 const int32_t* perm_T, const float* x, const float* Y, const float* W,
                                 const float* grad_out, const float* h_x, const float* h_W, const float* h_Y,
                                 float* gg_out, float* gx, float* gW, float* gY, void* workspace,
                                 size_t workspace_bytes, cgtp_stream stream) {
  NvtxRange nvtx_range("cgtp_double_backward");
  if (!plan) return fail(CGTP_ERR_NULL, "plan is NULL");
  Plan* P = reinterpret_cast<Plan*>(plan);
  if (n_recv < 0 || n_send < 0 || E < 0 || n_recv >= (int64_t(1) << 31) ||
      n_send >= (int64_t(1) << 31) || E >= (int64_t(1) << 31) - 1)
    return fail(CGTP_ERR_SIZE, "sizes out of range");
  cgtp_status st = check_device(*P);
  if (st != CGTP_OK) return st;
  for (const void* p : {(const void*)x, (const void*)Y, (const void*)W, (const void*)grad_out, (const void*)h_x,
                        (const void*)h_W, (const void*)h_Y, (const void*)gg_out, (const void*)gx, (const void*)gW,
                        (const void*)gY})
    if (p && !aligned16(p)) return fail(CGTP_ERR_ALIGN, "float arrays must be 16-byte aligned");
  if (n_recv > 0 && !rowptr) return fail(CGTP_ERR_NULL, "rowptr is NULL");
  if (E > 0 && (!col || !x || !Y || !W || !grad_out))
    return fail(CGTP_ERR_NULL, "col, x, Y, W or grad_out is NULL");
  if (gx && (h_W || h_Y) && E > 0 && (!rowptr_T || !perm_T))
    return fail(CGTP_ERR_NULL, "grad_x needs rowptr_T and perm_T");
  if (n_recv > 0 && E > 0) {
    const bool need_T = gx && (h_W || h_Y);
    st = check_graph(*P, n_recv, n_send, E, rowptr, col, need_T ? rowptr_T : nullptr, need_T ? perm_T : nullptr,
                     stream);
    if (st != CGTP_OK) return st;
  }
  const DbwdLayout L = dbwd_workspace_layout(*P, n_recv, n_send, E);
  if (!workspace || workspace_bytes < L.total)
    return fail(CGTP_ERR_WORKSPACE, "workspace of " + std::to_string(L.total) + " bytes required");
  if ((uintptr_t)workspace & 255) return fail(CGTP_ERR_ALIGN, "workspace must be 256-byte aligned");
  char* ws = reinterpret_cast<char*>(workspace);
  float* tF = reinterpret_cast<float*>(ws + L.f);
  float* tX = reinterpret_cast<float*>(ws + L.x);
  float* tW = reinterpret_cast<float*>(ws + L.w);
  float* tY = reinterpret_cast<float*>(ws + L.y);
  cudaStream_t cs = (cudaStream_t)stream;
  if (h_x && h_W && h_Y && E > 0 && n_recv > 0 && ensure_tangent(*P)) {
    // one tangent forward and one tangent backward: the derivatives along
    // (h_x, h_Y, h_W) of the forward and of the backward at fixed grad_out
    int nr = (int)n_recv;
    const int32_t* no_eid = nullptr;
    if (gg_out) {
      // d grad_out along (h_x, h_Y, h_W): the tangent forward, or (the
      // forward is trilinear) one plain forward with h_x plus two
      // accumulating forwards with h_Y and h_W
      auto run_tangent = [&]() -> cgtp_status {
        void* args[] = {&rowptr, &col, &x, &Y, &W, &no_eid, &gg_out, &P->d_fwd_ent, &nr, &P->d_err, &h_x, &h_Y, &h_W};
        TimedScope ts(*P, 6, cs);
        return jit_launch(P->fwd_tan, dim3(persistent_grid(P->fwd_tan.blocks_per_sm, P->num_sms, n_recv)), args, cs);
      };
      auto run_sum = [&]() -> cgtp_status {
        cgtp_status r = forward_impl(plan, n_recv, n_send, E, rowptr, col, h_x, Y, W, nullptr, gg_out, stream, false);
        const float* ins[2][3] = {{x, h_Y, W}, {x, Y, h_W}};
        for (auto& in : ins) {
          if (r != CGTP_OK) break;
          void* args[] = {&rowptr, &col, &in[0], &in[1], &in[2], &no_eid, &gg_out, &P->d_fwd_ent, &nr, &P->d_err};
          TimedScope ts(*P, 8, cs);
          r = jit_launch(P->fwd_acc, dim3(persistent_grid(P->fwd_acc.blocks_per_sm, P->num_sms, n_recv)), args, cs);
        }
        return r;
      };
      int mode = P->dbwd_fwd_sum.load();
      if (mode < 0) {
        cudaStreamCaptureStatus capst = cudaStreamCaptureStatusNone;
        CGTP_CUDA_TRY(cudaStreamIsCapturing(cs, &capst));
        if (capst != cudaStreamCaptureStatusNone) {
          mode = 0;  // no timing under capture: the tangent forward, undecided
        } else {
          // run each way once untimed (first launches carry one-time costs),
          // then time each once on this call's inputs and keep the faster;
          // the chosen one runs last, so every call's gg_out comes from it
          std::lock_guard<std::mutex> g(P->tan_mu);
          if (P->dbwd_fwd_sum < 0) {
            st = run_tangent();
            if (st == CGTP_OK) st = run_sum();
            if (st != CGTP_OK) return st;
            cudaEvent_t ev[3];
            for (auto& e : ev) CGTP_CUDA_TRY(cudaEventCreate(&e));
            cudaEventRecord(ev[0], cs);
            st = run_tangent();
            cudaEventRecord(ev[1], cs);
            if (st == CGTP_OK) st = run_sum();
            cudaEventRecord(ev[2], cs);
            float t_tan = 0.f, t_sum = 0.f;
            if (st == CGTP_OK && cudaEventSynchronize(ev[2]) == cudaSuccess &&
                cudaEventElapsedTime(&t_tan, ev[0], ev[1]) == cudaSuccess &&
                cudaEventElapsedTime(&t_sum, ev[1], ev[2]) == cudaSuccess)
              P->dbwd_fwd_sum = t_sum < t_tan ? 1 : 0;
            for (auto& e : ev) cudaEventDestroy(e);
            if (st != CGTP_OK) return st;
          }
          mode = std::max(0, P->dbwd_fwd_sum.load());
        }
      }
      st = mode == 1 ? run_sum() : run_tangent();
      if (st != CGTP_OK) return st;
    }
    if (gx || gW || gY) {
      size_t off_dyp = 0;
      backward_scratch_bytes(*P, E, gx != nullptr, gY != nullptr, &off_dyp);
      float* m = gx ? reinterpret_cast<float*>(ws + L.bwd) : nullptr;
      float* dyp = gY ? (P->bcfg.S > 1 ? reinterpret_cast<float*>(ws + L.bwd + off_dyp) : gY) : nullptr;
      if (m && P->bwd_irrep_gap) CGTP_CUDA_TRY(cudaMemsetAsync(m, 0, (size_t)E * P->D_in * sizeof(float), cs));
      int e_stride = (int)E;
      void* args[] = {&rowptr, &col, &x, &Y, &W, &no_eid, &grad_out, &gW, &dyp, &m, &P->d_bwd_ent, &nr, &P->d_err,
                      &e_stride, &h_x, &h_Y, &h_W};
      {
        TimedScope ts(*P, 7, cs);
        st = jit_launch(P->bwd_tan, dim3(persistent_grid(P->bwd_tan.blocks_per_sm, P->num_sms, n_recv)), args, cs);
        if (st != CGTP_OK) return st;
      }
      if (gx || (gY && P->bcfg.S > 1)) {
        TimedScope ts(*P, 3, cs);
        CGTP_CUDA_TRY(launch_bwd_reduce(n_send, P->D_in, rowptr_T, perm_T, m, gx, P->bcfg.S, E * P->D_e, dyp,
                                        (gY && P->bcfg.S > 1) ? gY : nullptr, cs));
      }
    }
    return CGTP_OK;
  }
  // the term structure (double_backward.hpp) on the library's kernels
  struct DeviceOps {
    cgtp_plan plan;
    int64_t n_recv, n_send, E;
    const int32_t *rowptr, *col, *rowptr_T, *perm_T;
    const float* g;
    void* bws;
    size_t bw_bytes;
    cgtp_stream stream;
    int forward(const float* xx, const float* yy, const float* ww, float* out) {
      return forward_impl(plan, n_recv, n_send, E, rowptr, col, xx, yy, ww, nullptr, out, stream, false);
    }
    int backward(const float* xx, const float* yy, const float* ww, float* ox, float* ow, float* oy) {
      return backward_impl(plan, n_recv, n_send, E, rowptr, col, rowptr_T, perm_T, xx, yy, ww, g, ox, ow, oy, bws,
                           bw_bytes, stream, true, nullptr, false);
    }
    int add(float* dst, const float* src, int64_t n) {
      CGTP_CUDA_TRY(launch_add(n, src, dst, (cudaStream_t)stream));
      return CGTP_OK;
    }
    int zero(float* dst, int64_t n) {
      CGTP_CUDA_TRY(cudaMemsetAsync(dst, 0, (size_t)n * sizeof(float), (cudaStream_t)stream));
      return CGTP_OK;
    }
  } ops{plan, n_recv, n_send, E, rowptr, col, rowptr_T, perm_T, grad_out, ws + L.bwd, L.f - L.bwd, stream};
  const DbwdDims dims{n_recv, n_send, E, P->D_in, P->D_e, P->D_out, P->U};
  return (cgtp_status)compose_double_backward(ops, dims, x, Y, W, h_x, h_W, h_Y, gg_out, gx, gW, gY, tF, tX, tW,
                                              tY);
}

cgtp_status cgtp_fma_peak_sink_floats(int64_t* floats) {
  if (!floats) return fail(CGTP_ERR_NULL, "floats is NULL");
  int dev = 0, sms = 0;
  CGTP_CUDA_TRY(cudaGetDevice(&dev));
  CGTP_CUDA_TRY(cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev));
  *floats = fma_peak_sink_floats(sms);
  return CGTP_OK;
}

cgtp_status cgtp_fma_peak(int64_t iters, float* sink, int64_t sink_floats, cgtp_stream stream, double* flops) {
  if (!sink || !flops) return fail(CGTP_ERR_NULL, "sink or flops is NULL");
  if (iters < 1 || iters > (int64_t(1) << 24)) return fail(CGTP_ERR_SIZE, "iters must be in 1..2^24");
  int dev = 0, sms = 0;
  CGTP_CUDA_TRY(cudaGetDevice(&dev));
  CGTP_CUDA_TRY(cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev));
  if (sink_floats < fma_peak_sink_floats(sms))
    return fail(CGTP_ERR_SIZE, "sink holds fewer floats than cgtp_fma_peak_sink_floats");
  CGTP_CUDA_TRY(launch_fma_peak(sms, iters, 1.0f - 1e-7f, 1e-7f, sink, (cudaStream_t)stream, flops));
  return CGTP_OK;
}

cgtp_status cgtp_neighbor_list(int64_t N, const double* pos, const double* box, double rc,
                               int32_t* rowptr, int32_t* col, int32_t* shift, float* r,
                               int64_t* n_edges) {
  try {
    return neighbor_list_impl(N, pos, box, rc, rowptr, col, shift, r, n_edges);
  } catch (const std::exception& e) {
    return fail(CGTP_ERR_OOM, e.what());
  }
}

cgtp_status cgtp_csr_transpose(int64_t n_recv, int64_t n_send, int64_t E, const int32_t* rowptr,
                               const int32_t* col, int32_t* rowptr_T, int32_t* perm_T) {
  try {
    return csr_transpose_impl(n_recv, n_send, E, rowptr, col, rowptr_T, perm_T);
  } catch (const std::exception& e) {
    return fail(CGTP_ERR_OOM, e.what());
  }
}

}  // extern "C"
