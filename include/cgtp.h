/*
 * cgtp.h -- C ABI of the B200 Clebsch-Gordan tensor-product (CGTP)
 * convolution library (libcgtp.so).
 *
 * The operation is the CGTP convolution that the LunaTP page (arXiv
 * 2610.18393, Abstract) names as the core cost of equivariant interatomic
 * potentials, with the irreps configurations of its Table 1 and the outputs
 * of its Table 11 (forward x'; backward x-bar, y-bar, w-bar).  The pages give
 * no formula; this library computes, for a receiver-sorted edge list i <- j,
 *
 *   out[i, o_off(p) + u (2l3+1) + m3] =
 *       sum_{e in row i} W[e, k0(p) + u]
 *         sum_{m1,m2} C_p[m1,m2,m3] x[col e, x_off(p) + u (2l1+1) + m1] Y[e, l2^2 + m2]
 *
 * over every path p = (hidden irrep l1, edge irrep l2 -> l3) allowed by the
 * triangle rule and parity, with channelwise ("uvu") weights W per edge.
 *
 * Conventions
 *   - Real spherical harmonics, component normalisation (sum_m Y_lm^2 = 2l+1),
 *     m = -l..l, no Condon-Shortley phase: Y_1(r) = sqrt(3) (y, z, x)/|r|.
 *   - Real CG blocks in that basis, sum C^2 = 2 l3 + 1, first non-zero entry
 *     (lexicographic m1, m2, m3) positive.
 *   - Paths: for each hidden irrep in order, each edge irrep in order, each l3
 *     from |l1-l2| to l1+l2 ascending, kept when (l3, p1 p2) is an output
 *     irrep.  Its channels are appended to that output block in this order;
 *     every output block must receive exactly its declared multiplicity.
 *   - W column k is the global output channel (output irreps in order).
 *
 * Layouts (all row-major, FP32 unless stated, device memory unless stated)
 *   x    [n_send, d_in]    hidden irrep blocks in order, each [mul, 2l+1]
 *   Y    [E, d_edge]       d_edge = (L+1)^2, degree l at columns l^2..l^2+2l
 *   W    [E, n_weights]
 *   out  [n_recv, d_out]   output irrep blocks in order, each [mul, 2l+1]
 *   rowptr [n_recv+1] int32 (receiver CSR), col [E] int32 sender per edge
 *   rowptr_T [n_send+1], perm_T [E] int32: edge ids grouped by sender,
 *   ascending inside each sender (see cgtp_csr_transpose).
 *
 * Ownership: the caller owns every buffer.  A plan owns its own host tables,
 * device tables and compiled kernels from cgtp_plan_create to
 * cgtp_plan_destroy.  Forward and backward allocate nothing; the backward's
 * scratch is a caller-provided workspace (cgtp_backward_workspace_size).
 *
 * Errors: every entry point returns a cgtp_status.  Arguments are validated
 * on the host before any launch (null pointers, 16-byte alignment of float
 * arrays, sizes, irreps, lmax).  No exception crosses the ABI.  What the ABI
 * cannot see is trusted: each device buffer holds at least the elements its
 * layout above implies (the Python binding checks dtype, element count and
 * device of every tensor before the call), and the graph is a valid CSR
 * (rowptr non-decreasing from 0 to E, every col in [0, n_send), perm_T a
 * permutation grouped by sender) -- cgtp_csr_transpose checks exactly this
 * on the host while it builds rowptr_T and perm_T, and a plan's device
 * graph checks (cgtp_plan_set_checks, or CGTP_DEBUG) check it before each
 * call.
 * cgtp_last_error() returns a message for the calling thread's last failure.
 * Calls are ordered on the given stream; a plan may be used from several
 * threads for concurrent launches.
 */
#ifndef CGTP_H_
#define CGTP_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct cgtp_plan_s* cgtp_plan;
typedef void* cgtp_stream; /* a cudaStream_t; NULL means the legacy default stream */

typedef enum {
  CGTP_OK = 0,
  CGTP_ERR_NULL = 1,            /* a required pointer is NULL */
  CGTP_ERR_ALIGN = 2,           /* a float array is not 16-byte aligned */
  CGTP_ERR_IRREPS_PARSE = 3,    /* an irreps string does not parse */
  CGTP_ERR_IRREPS_MISMATCH = 4, /* output multiplicities disagree with the paths */
  CGTP_ERR_LMAX = 5,            /* some l exceeds lmax, or lmax > 6 */
  CGTP_ERR_SIZE = 6,            /* a size is negative, too large, or inconsistent */
  CGTP_ERR_INVALID_CSR = 7,     /* rowptr/col/perm inconsistent (host or device checks) */
  CGTP_ERR_CUDA = 8,            /* a CUDA runtime or driver call failed */
  CGTP_ERR_OOM = 9,             /* host or device allocation failed in plan create */
  CGTP_ERR_TIMEOUT = 10,        /* a bounded wait inside a kernel gave up */
  CGTP_ERR_JIT = 11,            /* runtime compilation of a kernel failed */
  CGTP_ERR_WORKSPACE = 12       /* backward workspace missing or too small */
} cgtp_status;

/* Human-readable name of a status.  Never NULL. */
const char* cgtp_status_string(cgtp_status s);

/* Detail of the calling thread's most recent non-OK status.  Never NULL. */
const char* cgtp_last_error(void);

/* Build a plan on the CURRENT CUDA device.
 *   irreps_in   hidden irreps, e.g. "128x0e+64x1o"  (LunaTP Table 1 "Hidden irreps")
 *   irreps_edge exactly "1x0?+1x1?+...+1xL?" (Table 1 "Edge irreps"); the parity
 *               letters only select paths, the harmonics are the true Y_l
 *   irreps_out  output irreps (Table 1 "Output irreps"), each (l, parity) once
 *   lmax        upper bound on every l in the three strings, 0 <= lmax <= 6
 * Parses and checks the irreps, enumerates the paths, builds the real CG
 * tables in FP64 (rounded to FP32 for the device), generates and compiles the
 * path-specialised forward and backward kernels for sm_100a, and uploads the
 * tables.  On failure *out is set to NULL.
 * Capacity: the backward keeps the grad_out rows of all paths of one hidden
 * irrep in shared memory, beside two edge stages, within the 227 KB a CTA
 * can hold: a plan whose single hidden irrep feeds more than roughly 30,000
 * output floats per atom (mul x the sum of 2 l3 + 1 over its paths; 256x6e
 * against L = 6 edges feeds 51,456) is refused with CGTP_ERR_SIZE.
 * Errors: NULL, IRREPS_PARSE, IRREPS_MISMATCH, LMAX, SIZE, CUDA, OOM, JIT. */
cgtp_status cgtp_plan_create(const char* irreps_in, const char* irreps_edge,
                             const char* irreps_out, int lmax, cgtp_plan* out);

/* Release every resource of the plan.  NULL is accepted.  The caller must
 * ensure no launch using the plan is still running. */
cgtp_status cgtp_plan_destroy(cgtp_plan plan);

/* Sizes of the plan: row widths of x (d_in), Y (d_edge), out (d_out), the
 * number of W columns (n_weights = total output channels) and of paths.
 * Any output pointer may be NULL. */
cgtp_status cgtp_plan_info(cgtp_plan plan, int64_t* d_in, int64_t* d_edge, int64_t* d_out,
                           int64_t* n_weights, int64_t* n_paths);

/* Host copy of the path table: n_paths rows of 8 int32
 *   l1, l2, l3, mul, x_off, k0, o_off, c_off
 * (c_off = offset of the path's [2l1+1][2l2+1][2l3+1] block in the
 * coefficient array that cgtp_plan_coefficients returns). */
cgtp_status cgtp_plan_paths(cgtp_plan plan, int32_t* table);

/* Host copy of the plan's real CG blocks in FP64, concatenated in path order;
 * n_coeff receives the total length (call with coeff == NULL to size it). */
cgtp_status cgtp_plan_coefficients(cgtp_plan plan, double* coeff, int64_t* n_coeff);

/* Host-only: the library's real CG block C[2l1+1][2l2+1][2l3+1] in FP64 for
 * one coupling l1 (x) l2 -> l3 (each l <= 12).  Needs no GPU. */
cgtp_status cgtp_real_cg(int l1, int l2, int l3, double* C);

/* Real spherical harmonics of the edge vectors (L = the plan's edge degree).
 *   r [E,3] FP32 device, Y [E, d_edge] FP32 device (overwritten).
 * r need not be normalised; r = 0 gives Y_00 = 1 and zeros elsewhere.
 * Source: Table 1 edge irreps and Fig. 1 (Lmax = 6) of the LunaTP page. */
cgtp_status cgtp_sph_harm(cgtp_plan plan, int64_t E, const float* r, float* Y,
                          cgtp_stream stream);

/* The harmonics' step of the force chain (after the backward's grad_Y):
 *   grad_r[e][k] = sum_t grad_Y[e][t] dY_t(r_e)/dr_k
 * r [E,3], grad_Y [E, d_edge], grad_r [E,3]: FP32 device, 16-byte aligned;
 * grad_r is overwritten; r = 0 gives grad_r = 0.  Forces are minus the
 * position gradient of the energy (BranchIP page, its force definition).
 * The pages print no formula for this step; it is the chain rule through
 * the harmonics of cgtp_sph_harm.  Errors: NULL, SIZE, ALIGN, CUDA (also for a
 * plan of another device or a compile-only plan). */
cgtp_status cgtp_sph_harm_backward(cgtp_plan plan, int64_t E, const float* r, const float* grad_Y,
                                   float* grad_r, cgtp_stream stream);

/* Per-atom forces from the edge-vector gradient, for edges
 * r_e = pos[col[e]] - pos[i] + shift (receiver CSR rowptr, sender lists
 * rowptr_T/perm_T as from cgtp_csr_transpose; all int32 device arrays):
 *   forces[a] = sum over a's receiver edges of grad_r[e]
 *             - sum over a's sender edges of grad_r[e]      (= -dL/dpos[a]).
 * grad_r [E,3], forces [n_atoms,3]: FP32 device; forces overwritten; each
 * sum in edge order (bitwise reproducible, no atomics).  Needs no plan. */
cgtp_status cgtp_edge_forces(int64_t n_atoms, int64_t E, const int32_t* rowptr, const int32_t* rowptr_T,
                             const int32_t* perm_T, const float* grad_r, float* forces,
                             cgtp_stream stream);

/* Strain derivative of the loss (the virial), for stresses, from the same
 * edge-vector gradient as cgtp_edge_forces:
 *   virial[3a+b] = sum_e grad_r[e][a] r[e][b]   (a, b = x, y, z)
 * which is dL/d eps_ab when every edge vector (and so the cell) is strained
 * as r_e -> (1 + eps) r_e; the stress is virial / cell volume.  The pages
 * name stresses beside forces as derivatives of the energy (BranchIP page,
 * its MLIP background) but print no formula: this is the chain rule through
 * the edge vectors, the same reading as the forces.
 * r, grad_r [E,3] FP32 device, 16-byte aligned; virial [9] FP32 device,
 * overwritten (zeros for E = 0).  Products and sums in FP64, in an order fixed
 * by E (bitwise reproducible, no atomics).  Needs no plan.
 * Errors: SIZE (E < 0 or E >= 2^31), NULL, ALIGN, CUDA. */
cgtp_status cgtp_edge_virial(int64_t E, const float* r, const float* grad_r, float* virial,
                             cgtp_stream stream);

/* Forward CGTP convolution (the x' of LunaTP Table 11), formula above.
 *   n_recv receivers, n_send senders, E edges (0 <= E < 2^31)
 *   rowptr [n_recv+1], col [E] (int32, device); x [n_send, d_in];
 *   Y [E, d_edge]; W [E, n_weights]; out [n_recv, d_out] (overwritten;
 *   receivers without edges get zeros).
 * Each receiver's row is accumulated on chip and stored once: no atomics, and
 * the result is bitwise reproducible run to run. */
cgtp_status cgtp_forward(cgtp_plan plan, int64_t n_recv, int64_t n_send, int64_t E,
                         const int32_t* rowptr, const int32_t* col, const float* x,
                         const float* Y, const float* W, float* out, cgtp_stream stream);

/* Bytes of device workspace cgtp_backward needs for these sizes. */
cgtp_status cgtp_backward_workspace_size(cgtp_plan plan, int64_t n_recv, int64_t n_send,
                                         int64_t E, size_t* bytes);

/* Backward of the forward above given grad_out = dL/dout [n_recv, d_out]
 * (the x-bar, w-bar, y-bar of LunaTP Table 11):
 *   grad_x [n_send, d_in], grad_W [E, n_weights], grad_Y [E, d_edge]
 * each overwritten; any of the three may be NULL to skip it.  The sender-major
 * sum for grad_x goes through the transpose edge list (rowptr_T, perm_T,
 * needed only when grad_x != NULL) and the workspace; no atomics, bitwise
 * reproducible.  workspace must hold cgtp_backward_workspace_size bytes and be
 * 256-byte aligned (NULL is accepted when grad_W is the only output wanted). */
cgtp_status cgtp_backward(cgtp_plan plan, int64_t n_recv, int64_t n_send, int64_t E,
                          const int32_t* rowptr, const int32_t* col, const int32_t* rowptr_T,
                          const int32_t* perm_T, const float* x, const float* Y,
                          const float* W, const float* grad_out, float* grad_x, float* grad_W,
                          float* grad_Y, void* workspace, size_t workspace_bytes,
                          cgtp_stream stream);

/* Text report of the plan: paths, warp roles, slices, chunk and ring sizes,
 * shared memory, threads and the kernel assembler's register/spill lines.
 * Writes at most n bytes (NUL-terminated); *needed receives the full length
 * including the NUL.  buf may be NULL to query the length. */
cgtp_status cgtp_plan_describe(cgtp_plan plan, char* buf, size_t n, size_t* needed);

/* Per-kernel timing.  While enabled, every launch made through the plan
 * (harmonics, forward, backward and its reduction kernels) is bracketed by a
 * pair of CUDA events recorded on the caller's stream.  cgtp_plan_kernel_times
 * waits for those events and returns, per kernel name, the summed device time
 * in milliseconds and the launch count since the previous call (which resets
 * them).  names receives up to max entries of 32 bytes each. */
cgtp_status cgtp_plan_set_timing(cgtp_plan plan, int enable);

/* Device checks of the graph (off by default; on for every plan created
 * while the environment variable CGTP_DEBUG is set to anything but "0").
 * With CGTP_CHECK_GRAPH set, every convolution call of the plan (forward,
 * backward, its static-scratch form, the double backward and the sparse
 * evaluation) first checks on the device, on the call's stream, that rowptr
 * runs non-decreasing from 0 to E and every col lies in [0, n_send), and,
 * when the call reads the sender lists (grad_x wanted), that rowptr_T runs
 * non-decreasing from 0 to E and perm_T lists, for each sender, ids of its own
 * edges in strictly ascending order (which makes it a permutation).  The
 * call then WAITS for the result (a stream synchronize: not usable under
 * stream capture, which is refused with CGTP_ERR_CUDA) and returns
 * CGTP_ERR_INVALID_CSR, naming the failed checks, before any kernel reads
 * through the graph.  The checks read only the arrays' declared extents
 * (n_recv + 1, E, n_send + 1 entries); the sender lists are walked only
 * after their bounds passed.  flags: 0 or CGTP_CHECK_GRAPH.
 * Errors: NULL, SIZE (unknown flags). */
#define CGTP_CHECK_GRAPH 1
cgtp_status cgtp_plan_set_checks(cgtp_plan plan, int flags);

/* The same device graph checks once, whatever the plan's flags: rowptr
 * [n_recv+1] runs non-decreasing from 0 to E and every col [E] lies in
 * [0, n_send); when rowptr_T [n_send+1] and perm_T [E] are both given, they
 * form the sender lists as above (both NULL: not checked).  On the stream;
 * the call waits for the result, so it is refused under stream capture
 * (CGTP_ERR_CUDA).  A caller that builds a graph once and calls the
 * convolutions many times can validate it here instead of turning the
 * per-call checks on.  Errors: NULL, SIZE, INVALID_CSR (naming the failed
 * checks), CUDA. */
cgtp_status cgtp_validate_graph(cgtp_plan plan, int64_t n_recv, int64_t n_send, int64_t E,
                                const int32_t* rowptr, const int32_t* col, const int32_t* rowptr_T,
                                const int32_t* perm_T, cgtp_stream stream);
cgtp_status cgtp_plan_kernel_times(cgtp_plan plan, int max, char* names, double* ms,
                                   int64_t* launches, int* n);

/* Size of the fixed device scratch of cgtp_backward_static_scratch: 64 MiB. */
#define CGTP_STATIC_SCRATCH_BYTES (64u << 20)

/* cgtp_backward without a caller workspace, for callers that cannot allocate
 * device memory when they call it: e.g. a simulation engine that sizes all of
 * its device memory once at start-up and forbids later allocation, or an
 * embedding runtime that owns no device allocator.  (The pages have no
 * counterpart; this is an interface convenience.)
 *
 * Same arguments, outputs and errors as cgtp_backward, minus the workspace.
 * The scratch is a fixed array of CGTP_STATIC_SCRATCH_BYTES inside the
 * library's device code: every GPU that loads the library holds it until the
 * process exits.  The call allocates nothing (no cudaMalloc/cudaFree, no
 * library allocator).  Only the scratch the requested gradients use counts
 * against the array: the per-edge messages (E x d_in floats) when grad_x is
 * wanted, and the slice parts of grad_Y for plans of several slices; a
 * grad_W-only call uses none.  A call that needs more is rejected with
 * CGTP_ERR_WORKSPACE before any launch, and every argument check of
 * cgtp_backward runs before the array is touched.
 *   - The first call on a device looks up the array's device address with
 *     that device current (cudaGetSymbolAddress) and caches it; make that
 *     first call before any stream capture on the device.
 *   - All calls share the one array and it keeps the last call's contents
 *     (nothing in it has to start at zero).  Calls whose launches overlap on
 *     the GPU (different streams, or different threads without ordering)
 *     race on it; order them on one stream.
 *   - Kernel timing (cgtp_plan_set_timing) does not record these launches. */
cgtp_status cgtp_backward_static_scratch(cgtp_plan plan, int64_t n_recv, int64_t n_send,
                                         int64_t E, const int32_t* rowptr, const int32_t* col,
                                         const int32_t* rowptr_T, const int32_t* perm_T,
                                         const float* x, const float* Y, const float* W,
                                         const float* grad_out, float* grad_x, float* grad_W,
                                         float* grad_Y, cgtp_stream stream);

/* Reads and clears the plan's device error word on the current device
 * (synchronises the device).  *code is 0 when every bounded wait of the
 * kernels launched since the last call completed; CGTP_ERR_TIMEOUT is
 * returned otherwise. */
cgtp_status cgtp_plan_check_device_error(cgtp_plan plan, int* code);

/* ---- BranchIP sparse evaluation -------------------------------------- */

/* The BranchIP page (section "BranchIP", the Branchlegro paragraph) gives
 * every edge a continuation gate f_e in [0, 1] that multiplies the edge's
 * feature before the TP; at inference the zero-gated edges are omitted from
 * the TP and the skipped per-edge outputs are zero-padded to the full edge
 * set ("sparse evaluation"), which reproduces the dense evaluation exactly.
 * Here the gate scales each edge's whole TP term:
 *   out[i] = sum_{e in row i} f_e TP(x[col e], Y[e], W[e])
 * (the convolution is linear in each input, so this is the gate applied to
 * any one of them), and only the edges with f_e > 0 are evaluated.
 *   gate [E] FP32 device, 16-byte aligned; f_e > 0 marks an active edge (a
 *   NaN gate is inactive).  Other arguments and layouts as for cgtp_forward /
 *   cgtp_backward; the graph is the full (ungated) CSR.
 * Steps, all on the stream and deterministic (no atomics, no host sync): a
 * scan compacts the active edges (receiver CSR, their ids, their gated
 * harmonics f_e Y_e, and with grad_x the sender lists) into the workspace;
 * the plan's kernels run over them, reading W rows and writing grad_W rows
 * of the full set through the edge ids; the backward then pads.
 * Workspace: cgtp_sparse_workspace_size bytes, 256-byte aligned, caller
 * owned; nothing in it needs initialising, and a call leaves nothing in it
 * that a later call needs (each call compacts again).
 * Backward outputs (each nullable = skipped), overwritten over the FULL edge
 * set: grad_x [n_send, d_in]; grad_W [E, n_weights] = f_e dL/dW' (zero rows
 * for skipped edges); grad_Y [E, d_edge] (zero rows for skipped edges);
 * grad_gate [E] = <g[i], TP_e> on active edges and 0 on skipped ones (the
 * sparse path builds no backward branch for them; exact for a loss that
 * reaches the gate through a function with zero slope where it is zero, the
 * page's flat-zero gate).  rowptr_T/perm_T are needed only with grad_x.
 * Errors: NULL, SIZE, ALIGN, WORKSPACE, CUDA (also for a plan of another
 * device or a compile-only plan). */
cgtp_status cgtp_sparse_workspace_size(cgtp_plan plan, int64_t n_recv, int64_t n_send, int64_t E,
                                       size_t* bytes);
cgtp_status cgtp_sparse_forward(cgtp_plan plan, int64_t n_recv, int64_t n_send, int64_t E,
                                const int32_t* rowptr, const int32_t* col, const float* x,
                                const float* Y, const float* W, const float* gate, float* out,
                                void* workspace, size_t workspace_bytes, cgtp_stream stream);
cgtp_status cgtp_sparse_backward(cgtp_plan plan, int64_t n_recv, int64_t n_send, int64_t E,
                                 const int32_t* rowptr, const int32_t* col, const int32_t* rowptr_T,
                                 const int32_t* perm_T, const float* x, const float* Y,
                                 const float* W, const float* gate, const float* grad_out,
                                 float* grad_x, float* grad_W, float* grad_Y, float* grad_gate,
                                 void* workspace, size_t workspace_bytes, cgtp_stream stream);

/* ---- measurement ----------------------------------------------------- */

/* FP32 FMA throughput probe of the current device, the measured FP32 peak
 * that the FP32-bound workloads (Lmax >= 4) are compared with.  It is not
 * part of the convolution: the pages quote only relative speedups, and the
 * roofline of the FP32-bound kernels needs the device's own FMA rate.
 * cgtp_fma_peak launches, on the given stream, 2 CTAs per SM of 512 threads,
 * each running 8 independent FMA chains for iters x 16 steps, and stores each
 * thread's chain sum in sink (device FP32, at least
 * cgtp_fma_peak_sink_floats elements; contents meaningless).  *flops
 * receives the launch's floating-point operations (2 per FMA); the caller
 * times the launch (CUDA events on the same stream) and divides.
 * Errors: NULL, SIZE (iters outside 1..2^24, sink too small), CUDA. */
cgtp_status cgtp_fma_peak_sink_floats(int64_t* floats);
cgtp_status cgtp_fma_peak(int64_t iters, float* sink, int64_t sink_floats, cgtp_stream stream,
                          double* flops);

/* ---- graph utilities (host, no GPU needed) ----------------------------- */

/* Second-order backward ("double backward"; LunaTP Table 11 lists its
 * outputs h_x and h_y, and its Figure 5 trains through it with a Hessian
 * objective; no formula is printed): given cotangents of the
 * backward's outputs, h_x [n_send, d_in], h_W [E, n_weights], h_Y [E, d_edge]
 * (each nullable = zero), the gradients of
 *   S = <h_x, grad_x> + <h_W, grad_W> + <h_Y, grad_Y>
 * (grad_* the backward at x, Y, W with cotangent grad_out) with respect to
 * grad_out, x, W and Y.  The convolution is linear in each of x, Y, W, so
 *   S = <grad_out, fwd(h_x, Y, W) + fwd(x, Y, h_W) + fwd(x, h_Y, W)>
 * and the gradients are forwards and backwards of this library with one
 * argument replaced by its cotangent:
 *   gg_out = fwd(h_x, Y, W) + fwd(x, Y, h_W) + fwd(x, h_Y, W)
 *   gx = bwd_x(Y, h_W) + bwd_x(h_Y, W)      gW = bwd_W(h_x, Y) + bwd_W(x, h_Y)
 *   gY = bwd_Y(h_x, W) + bwd_Y(x, h_W)       (all with grad_out)
 * Outputs gg_out [n_recv, d_out], gx, gW, gY (shapes of grad_out, x, W, Y;
 * each nullable = not computed) are overwritten and must not alias inputs.
 * workspace: cgtp_double_backward_workspace_size bytes, 256-byte aligned.
 * Graph arrays as for cgtp_backward (rowptr_T/perm_T needed for gx).
 * Errors: NULL, SIZE, ALIGN, WORKSPACE, CUDA (also for a plan of another
 * device or a compile-only plan). */
cgtp_status cgtp_double_backward_workspace_size(cgtp_plan plan, int64_t n_recv, int64_t n_send, int64_t E,
                                                size_t* bytes);

/* With all three cotangents given, cgtp_double_backward replaces the calls
 * above by one tangent backward, compiled with every W, x and Y piece staged
 * beside its direction (h_W, h_x, h_Y), which gives
 * d/dt bwd(x + t h_x, Y + t h_Y, W + t h_W; grad_out) = (gx, gW, gY) in one
 * pass, and forms gg_out = d/dt fwd(x + t h_x, Y + t h_Y, W + t h_W) either
 * by the tangent forward (one pass, built the same way) or by one plain
 * forward with h_x plus two passes of an accumulating forward with h_Y and
 * h_W (the forward is trilinear).  Which of the two is faster depends on the
 * plan: unless CGTP_DBWD_FWD=tangent|sum at plan creation fixes it, both are
 * built, and the first such call made outside stream capture runs each once
 * untimed, times each once, keeps the faster for the plan and runs it last,
 * so that every call's gg_out comes from the kept form.  That first call
 * therefore does three times the forward work and waits on the host for its
 * timing events; under stream capture before that choice, the tangent
 * forward runs.  The kernels are compiled on the plan's first such call;
 * cgtp_plan_prepare_double_backward compiles them ahead (call it before any
 * stream capture).  *tangent (may be NULL) receives 1 when they are
 * available, 0 when the plan keeps the composition (a tangent backward whose
 * stages do not fit shared memory at its roles' edge phases, or
 * CGTP_DBWD_COMPOSE set at the first call).  Errors: NULL, CUDA. */
cgtp_status cgtp_plan_prepare_double_backward(cgtp_plan plan, int* tangent);
cgtp_status cgtp_double_backward(cgtp_plan plan, int64_t n_recv, int64_t n_send, int64_t E,
                                 const int32_t* rowptr, const int32_t* col, const int32_t* rowptr_T,
                                 const int32_t* perm_T, const float* x, const float* Y, const float* W,
                                 const float* grad_out, const float* h_x, const float* h_W, const float* h_Y,
                                 float* gg_out, float* gx, float* gW, float* gY, void* workspace,
                                 size_t workspace_bytes, cgtp_stream stream);

/* Periodic neighbour list by cell list, FP64.  Host pointers.
 * Edge i <- j with image n (integers, |n_a| <= ceil(rc / box_a)) exists iff
 * (i,j,n) != (i,i,0) and |(pos_j + n*box) - pos_i|^2 < rc^2, each component
 * formed as (pos_j[a] + n_a*box[a]) - pos_i[a] and the square summed x, y, z
 * in that order, all in FP64 (so every decision is exactly reproducible).
 * Edges are ordered by (receiver i, sender j, n_x, n_y, n_z).  Positions must
 * lie in [0, box).  Call with col == NULL to get *n_edges (and rowptr); then
 * with col/shift/r sized for it.  r [E,3] FP32 = the rounded edge vectors,
 * shift [E,3] int32 = n.  rowptr has N+1 entries.  Receivers are split over
 * host threads (CGTP_HOST_THREADS, default the hardware threads, one below
 * 4096 atoms); the result does not depend on their number. */
cgtp_status cgtp_neighbor_list(int64_t N, const double* pos, const double* box, double rc,
                               int32_t* rowptr, int32_t* col, int32_t* shift, float* r,
                               int64_t* n_edges);

/* Transpose of a receiver CSR: rowptr_T [n_send+1] and perm_T [E] listing, for
 * every sender, the ids of its edges in ascending order.  Host pointers.
 * Checks the CSR on the way: CGTP_ERR_INVALID_CSR when rowptr does not run
 * non-decreasing from 0 to E or a col entry lies outside [0, n_send). */
cgtp_status cgtp_csr_transpose(int64_t n_recv, int64_t n_send, int64_t E,
                               const int32_t* rowptr, const int32_t* col, int32_t* rowptr_T,
                               int32_t* perm_T);

#ifdef __cplusplus
}
#endif

#endif /* CGTP_H_ */
