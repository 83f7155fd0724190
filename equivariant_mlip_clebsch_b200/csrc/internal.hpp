// internal.hpp -- shared declarations of the libcgtp host code.
#pragma once

#include <cuda_runtime.h>

#include <atomic>
#include <cstdint>
#include <memory>
#include <mutex>
#include <string>
#include <thread>
#include <vector>

#include <nvtx3/nvToolsExt.h>

#include "cgtp.h"

namespace cgtp {

// An NVTX range over one C-ABI call, named after the entry point: it shows
// each call (and the kernels it launched) on a profiler's timeline.  NVTX v3
// is header-only and does nothing unless a profiling tool is attached.
struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
  NvtxRange(const NvtxRange&) = delete;
  NvtxRange& operator=(const NvtxRange&) = delete;
};

// ---------------------------------------------------------------- errors
void set_error(const std::string& msg);
cgtp_status fail(cgtp_status s, const std::string& msg);

// A failed runtime call returns CGTP_ERR_CUDA and clears the runtime's
// per-thread last error, so that a non-sticky failure here (an invalid launch
// configuration, say) is reported once, through the status, and not again by
// the caller's next unrelated CUDA check.
#define CGTP_CUDA_TRY(expr)                                                          \
  do {                                                                               \
    cudaError_t _e = (expr);                                                         \
    if (_e != cudaSuccess) {                                                         \
      (void)cudaGetLastError();                                                      \
      return ::cgtp::fail(CGTP_ERR_CUDA, std::string(#expr) + ": " + cudaGetErrorString(_e)); \
    }                                                                                \
  } while (0)

// ---------------------------------------------------------------- irreps
struct Irrep {
  int mul;
  int l;
  int parity;  // +1 even, -1 odd
};
bool parse_irreps(const char* s, std::vector<Irrep>& out, std::string& err);

// ---------------------------------------------------------------- CG
// Real CG block [2l1+1][2l2+1][2l3+1] in FP64 (see cgtp.h for conventions).
bool real_cg_block(int l1, int l2, int l3, std::vector<double>& C);

// ---------------------------------------------------------------- paths
struct Path {
  int l1, l2, l3;
  int irrep;  // index of the hidden irrep
  int mul;
  int x_off;  // hidden block offset in a row of x
  int k0;     // W column of channel 0
  int o_off;  // out offset of channel 0
  int c_off;  // offset into the FP64 coefficient array
  int out_irrep;
};

// One warp's share of the forward: channels [u0, u0 + 32*R) of one hidden
// irrep for a group of its paths (accumulators live in registers).
struct FwdRole {
  int irrep;
  int u0;
  int R;
  std::vector<int> paths;  // indices into Plan::paths
  double cost;
};

// One warp's share of the backward: channels [u0, u0 + 32*R) of one hidden
// irrep, every path of that irrep, the edges of a chunk with b % nph == ph.
struct BwdRole {
  int irrep;
  int u0;
  int R;
  int ph, nph;
  double cost;
};

struct JitKernel {
  void* module = nullptr;    // CUmodule
  void* function = nullptr;  // CUfunction
  int threads = 0;
  int smem = 0;
  std::string name;
  std::string log;
  unsigned long long hash = 0;  // of the generated source and compile options
  int blocks_per_sm = 0;        // resident CTAs per SM (occupancy query)
};

// A compiled kernel before loading: building needs no CUDA context and may
// run on any thread; loading uses the calling thread's current context.
struct JitBinary {
  std::string cubin, log, err;  // err: the failing thread's message
  unsigned long long hash = 0;
};

// A kernel compiling on a host thread during plan creation; the destructor
// joins, so no exit path leaves the thread running.
struct PendingCompile {
  std::thread th;
  std::string src;
  JitBinary bin;
  cgtp_status st = CGTP_OK;
  void join() {
    if (th.joinable()) th.join();
  }
  ~PendingCompile() { join(); }
};

struct FwdConfig {
  int S = 1;             // slices (each CTA walks them in turn)
  int nw = 0;            // consumer warps per CTA
  int B = 4;             // edges per chunk
  int stages = 3;        // ring depth
  bool w_smem = true;    // W row pieces staged by bulk copy (16-byte aligned)
  bool x_smem = true;    // x blocks staged by bulk copy
  bool generic = false;  // forward roles of one path, one function per (2l1+1, 2l3+1) shape
  bool packed = false;   // forward roles with packed FMAs over an m1-major Chat
  int nacc = 0;          // accumulator registers per thread
  std::vector<std::vector<int>> slice_roles;  // role ids per slice
};

struct Plan {
  std::string irreps_in_s, irreps_edge_s, irreps_out_s;
  std::vector<Irrep> in, edge, out;
  int lmax = 0, L = 0;
  int64_t D_in = 0, D_e = 0, D_out = 0, U = 0;
  std::vector<int> x_off, out_off, chan_base;
  std::vector<Path> paths;
  std::vector<double> coeff;  // concatenated real CG blocks (FP64)
  int device = -1;
  int num_sms = 0;

  // forward
  std::vector<FwdRole> fwd_roles;
  FwdConfig fcfg;
  JitKernel fwd;
  // Chat build tables per slice (device): entry -> (dst offset, term begin, term count)
  void* d_fwd_ent = nullptr;   // int4 [n]
  std::vector<int> fwd_ent_begin;  // per slice, into d_fwd_ent (size S+1)
  std::vector<int> fwd_chs;        // Chat floats per edge per slice

  // backward
  std::vector<BwdRole> bwd_roles;
  FwdConfig bcfg;
  JitKernel bwd;     // CTAs walk receivers blockIdx.x, + gridDim.x, ...
  JitKernel bwd_er;  // CTAs take equal edge ranges (for few receivers per CTA)
  void* d_bwd_ent = nullptr;
  std::vector<int> bwd_ent_begin;
  std::vector<int> bwd_chs;
  bool bwd_irrep_gap = false;  // some hidden irrep has no path
  // backward roles contract grad_out with the CG table first and then with
  // Y, so no Chat is staged; CGTP_BWD_TFORM=0 at plan creation selects the
  // staged-Chat form instead (kept for comparison)
  bool bwd_tform = true;
  // forward roles with float2 accumulators and packed FMAs: -1 chosen by the
  // planner, 0 off, 1 on (CGTP_FWD_PACKED at plan creation)
  int fwd_packed = -1;
  // double backward: gg_out from the tangent forward (0) or as one plain and
  // two accumulating forwards (1); -1: chosen by timing both on the first
  // all-cotangent call outside stream capture (CGTP_DBWD_FWD=tangent|sum at
  // plan creation fixes it)
  std::atomic<int> dbwd_fwd_sum{-1};

  // tangent kernels of the double backward, built on first use (tan_state:
  // 0 not built, 1 ready, -1 unavailable: the composition is used)
  JitKernel fwd_tan, bwd_tan;
  JitKernel fwd_acc;  // accumulating forward (double backward on packed plans)
  std::mutex tan_mu;
  int tan_state = 0;
  std::string tan_msg;

  int* d_err = nullptr;  // device error word
  // device checks of the graph before each call (cgtp_plan_set_checks;
  // CGTP_DEBUG=1 at plan creation): flags, the result word, its lock
  std::atomic<int> checks{0};
  int* d_csr = nullptr;
  std::mutex csr_mu;
  // kernel timing (cgtp_plan_set_timing)
  std::atomic<bool> timing{false};  // read by launches on any thread
  std::mutex tmu;
  struct TimedLaunch {
    int kind;
    cudaEvent_t a, b;
  };
  std::vector<TimedLaunch> tlog;
  std::vector<cudaEvent_t> tpool;
  bool host_only = false;  // built for compile checks only: no device state
  int L_sh = 0;
  // the forward's compile while the backward is built (reads the fields
  // above; the last member, so it is joined before they are destroyed)
  std::unique_ptr<PendingCompile> fwd_pending;
};

// The forward and backward behind the C ABI.  eid (nullable, device int32
// [E]): the full-set ids of the listed edges, whose W rows (and grad_W rows)
// the kernels read (write) instead of row e (the sparse evaluation's active
// edges); NULL for the plain convolution.
// graph_checks: run the plan's graph checks (when on) on this call's graph.
cgtp_status forward_impl(cgtp_plan plan, int64_t n_recv, int64_t n_send, int64_t E, const int32_t* rowptr,
                         const int32_t* col, const float* x, const float* Y, const float* W, const int32_t* eid,
                         float* out, cgtp_stream stream, bool graph_checks);
cgtp_status backward_impl(cgtp_plan plan, int64_t n_recv, int64_t n_send, int64_t E,
                          const int32_t* rowptr, const int32_t* col, const int32_t* rowptr_T,
                          const int32_t* perm_T, const float* x, const float* Y, const float* W,
                          const float* grad_out, float* grad_x, float* grad_W, float* grad_Y,
                          void* workspace, size_t workspace_bytes, cgtp_stream stream,
                          bool allow_timing, const int32_t* eid, bool graph_checks);

// The plan's device is current and the plan has device state.
cgtp_status check_plan_device(const Plan& P);
// With the plan's CSR checks on: runs them on the stream, waits for their
// result and returns CGTP_ERR_INVALID_CSR (with the failed checks in the
// message) before any kernel reads through the graph.  OK when checks are off.
cgtp_status check_graph(Plan& P, int64_t n_recv, int64_t n_send, int64_t E, const int32_t* rowptr,
                        const int32_t* col, const int32_t* rowptr_T, const int32_t* perm_T, cgtp_stream stream,
                        bool always = false);
// Host checks of a backward call (sizes, device, alignment, required pointers).
cgtp_status backward_validate(const Plan& P, int64_t n_recv, int64_t n_send, int64_t E, const int32_t* rowptr,
                              const int32_t* col, const int32_t* rowptr_T, const int32_t* perm_T, const float* x,
                              const float* Y, const float* W, const float* grad_out, const float* grad_x,
                              const float* grad_W, const float* grad_Y);
// Scratch bytes a backward call uses for the gradients it is asked for (at
// most cgtp_backward_workspace_size); off_dyp receives the dY parts' offset.
size_t backward_scratch_bytes(const Plan& P, int64_t E, bool want_x, bool want_Y, size_t* off_dyp);

// construction steps
cgtp_status build_paths(Plan& P);
cgtp_status build_forward(Plan& P);
cgtp_status build_backward(Plan& P);
cgtp_status finish_forward(Plan& P);  // joins the forward's compile and loads it
// tangent kernels (the double backward): built and loaded on the calling thread
cgtp_status build_forward_accumulate(Plan& P, JitKernel& out, std::string* src_out);
cgtp_status build_forward_tangent(Plan& P, JitKernel& out, std::string* src);
cgtp_status build_backward_tangent(Plan& P, JitKernel& out, std::string* src);
void destroy_plan_device(Plan& P);

// JIT
cgtp_status jit_build(const std::string& src, const std::string& name, JitBinary& b);
cgtp_status jit_load(const JitBinary& b, const std::string& name, JitKernel& k);
cgtp_status jit_compile(const std::string& src, const std::string& name, JitKernel& k);
cgtp_status jit_launch(const JitKernel& k, dim3 grid, void** args, cudaStream_t stream);
void jit_unload(JitKernel& k);

// generic CUDA kernels (kernels.cu)
cudaError_t launch_sph_harm(int L, int64_t E, const float* r, float* Y, cudaStream_t s);
// dr = sum_t dY_t dY_t/dr per edge (harmonics up to L), and the per-atom forces
// F = sum over receiver edges - sum over sender edges of dr.
cudaError_t launch_sph_harm_backward(int L, int64_t E, const float* r, const float* dY, float* dr,
                                     cudaStream_t s);
cudaError_t launch_edge_forces(int64_t n_atoms, const int32_t* rowptr, const int32_t* rowptr_T,
                               const int32_t* perm_T, const float* G, float* F, cudaStream_t s);
cudaError_t launch_edge_virial(int64_t E, const float* r, const float* G, float* V, cudaStream_t s);
cudaError_t launch_add(int64_t n, const float* src, float* dst, cudaStream_t s);
// c_norm of the harmonics kernels, uploaded once per device (plan creation)
cudaError_t upload_sph_norm();
// The graph's device checks (bits in *flag, see kernels.cu); the sender
// lists are checked when rowptr_T and perm_T are given.
cudaError_t launch_csr_check(int num_sms, int64_t n_recv, int64_t n_send, int64_t E, const int32_t* rowptr,
                             const int32_t* col, const int32_t* rowptr_T, const int32_t* perm_T, int* flag,
                             cudaStream_t s);
// FP32 FMA throughput probe: 2 CTAs per SM; flops receives the launch's FLOPs
int64_t fma_peak_sink_floats(int num_sms);
cudaError_t launch_fma_peak(int num_sms, int64_t iters, float m, float c, float* sink, cudaStream_t s,
                            double* flops);

// dx row sums over the transpose edge list and the dY slice sums, one launch;
// either part is skipped when its output is null (or S == 1 for dY).
cudaError_t launch_bwd_reduce(int64_t n_send, int64_t width, const int32_t* rowptr_T, const int32_t* perm_T,
                              const float* m, float* dx, int S, int64_t ny, const float* parts, float* dy,
                              cudaStream_t s);

}  // namespace cgtp
