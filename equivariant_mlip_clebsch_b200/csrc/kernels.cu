// kernels.cu -- the kernels that do not depend on the path structure:
// real spherical harmonics of the edge vectors and their gradient, the force
// and strain-derivative (virial) assembly from the edge-vector gradient, and
// the deterministic closing reductions of the backward (sender-major row sums,
// slice sums) in one launch.
#include <cooperative_groups.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstdlib>
#include <mutex>

#include "internal.hpp"

namespace cgtp {

namespace {

// Programmatic dependent launch (as for the generated kernels): wait for the
// previous kernel on the stream and its writes, then let the next one launch.
__device__ __forceinline__ void grid_dependency_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void grid_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

template <class... KArgs, class... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, unsigned block, cudaStream_t s, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(block);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

// Normalisation of the component-normalised real harmonics:
//   N_l0 = sqrt(2l+1),  N_lm = sqrt(2l+1) sqrt(2 (l-m)!/(l+m)!)  (m > 0)
// index l*(l+1)/2 + m, l <= 6.
__constant__ float c_norm[28];
constexpr int kMaxDevices = 256;
std::atomic<bool> g_norm_ready[kMaxDevices];
std::mutex g_norm_mu;

template <int L>
__global__ void __launch_bounds__(128) sph_harm_kernel(int64_t E, const float* __restrict__ r,
                                                       float* __restrict__ Y) {
  grid_dependency_wait();
  grid_launch_dependents();
  constexpr int D = (L + 1) * (L + 1);
  __shared__ float tile[128 * D];
  const int64_t e0 = (int64_t)blockIdx.x * 128;
  const int64_t e = e0 + threadIdx.x;
  float* y = tile + threadIdx.x * D;
  if (e < E) {
    const float rx = r[3 * e], ry = r[3 * e + 1], rz = r[3 * e + 2];
    const float r2 = rx * rx + ry * ry + rz * rz;
    if (r2 == 0.f) {
      y[0] = 1.f;
#pragma unroll
      for (int t = 1; t < D; ++t) y[t] = 0.f;
    } else {
      const float inv = rsqrtf(r2);
      const float x = rx * inv, yy = ry * inv, z = rz * inv;
      // C_m + i S_m = (x + i y)^m  (= sin^m(theta) e^{i m phi})
      float Cm[L + 1], Sm[L + 1];
      Cm[0] = 1.f;
      Sm[0] = 0.f;
#pragma unroll
      for (int m = 1; m <= L; ++m) {
        Cm[m] = x * Cm[m - 1] - yy * Sm[m - 1];
        Sm[m] = x * Sm[m - 1] + yy * Cm[m - 1];
      }
      // Q_l^m(z) = P_l^m(z) / (1 - z^2)^(m/2) without the Condon-Shortley
      // phase: Q_m^m = (2m-1)!!, Q_{m+1}^m = (2m+1) z Q_m^m,
      // (l-m) Q_l^m = (2l-1) z Q_{l-1}^m - (l+m-1) Q_{l-2}^m
#pragma unroll
      for (int m = 0; m <= L; ++m) {
        float qmm = 1.f;
#pragma unroll
        for (int k = 1; k <= m; ++k) qmm *= (float)(2 * k - 1);
        float q2 = 0.f, q1 = qmm;
#pragma unroll
        for (int l = m; l <= L; ++l) {
          float q;
          if (l == m)
            q = qmm;
          else if (l == m + 1)
            q = (float)(2 * m + 1) * z * qmm;
          else
            q = ((float)(2 * l - 1) * z * q1 - (float)(l + m - 1) * q2) / (float)(l - m);
          if (l > m) {
            q2 = q1;
            q1 = q;
          }
          const float nq = c_norm[l * (l + 1) / 2 + m] * q;
          if (m == 0) {
            y[l * l + l] = nq;
          } else {
            y[l * l + l + m] = nq * Cm[m];
            y[l * l + l - m] = nq * Sm[m];
          }
        }
      }
    }
  }
  __syncthreads();
  const int64_t n = (E - e0 < 128 ? E - e0 : 128) * D;
  float* dst = Y + e0 * D;
  for (int t = threadIdx.x; t < n; t += 128) dst[t] = tile[t];
}

// dL/dr of the harmonics, one thread per edge:
//   dr[e] = sum_t dY[e][t] dY_t/dr(r_e).
// Y_lm = N_lm Q_l^m(z) C_m(x,y) (or S_m) on the unit vector u = r/|r| (the
// Cartesian form of sph_harm_kernel).  Any smooth extension F of Y off the
// sphere has the same tangential gradient, so with g = sum_t dY_t grad_u F_t:
//   dr = (g - (g.u) u) / |r|,
// where grad C_m = m (C_{m-1}, -S_{m-1}, 0), grad S_m = m (S_{m-1}, C_{m-1}, 0),
// and Q' follows from differentiating the z recurrence:
//   (l-m) Q_l' = (2l-1)(Q_{l-1} + z Q_{l-1}') - (l+m-1) Q_{l-2}'.
// dY rows are staged through shared memory (coalesced); r = 0 gives dr = 0.
template <int L>
__global__ void __launch_bounds__(128) sph_harm_backward_kernel(int64_t E, const float* __restrict__ r,
                                                                const float* __restrict__ dY,
                                                                float* __restrict__ dr) {
  grid_dependency_wait();
  grid_launch_dependents();
  constexpr int D = (L + 1) * (L + 1);
  __shared__ float tile[128 * D];
  __shared__ float otile[128 * 3];
  const int64_t e0 = (int64_t)blockIdx.x * 128;
  const int64_t n = (E - e0 < 128 ? E - e0 : 128);
  for (int64_t t = threadIdx.x; t < n * D; t += 128) tile[t] = dY[e0 * D + t];
  __syncthreads();
  const int64_t e = e0 + threadIdx.x;
  if (e < E) {
    const float* g_in = tile + threadIdx.x * D;
    const float rx = r[3 * e], ry = r[3 * e + 1], rz = r[3 * e + 2];
    const float r2 = rx * rx + ry * ry + rz * rz;
    float gx = 0.f, gy = 0.f, gz = 0.f, inv = 0.f, x = 0.f, yy = 0.f, z = 0.f;
    if (r2 > 0.f) {
      inv = rsqrtf(r2);
      x = rx * inv;
      yy = ry * inv;
      z = rz * inv;
      float Cm[L + 1], Sm[L + 1];
      Cm[0] = 1.f;
      Sm[0] = 0.f;
#pragma unroll
      for (int m = 1; m <= L; ++m) {
        Cm[m] = x * Cm[m - 1] - yy * Sm[m - 1];
        Sm[m] = x * Sm[m - 1] + yy * Cm[m - 1];
      }
#pragma unroll
      for (int m = 0; m <= L; ++m) {
        float qmm = 1.f;
#pragma unroll
        for (int k = 1; k <= m; ++k) qmm *= (float)(2 * k - 1);
        float q2 = 0.f, q1 = qmm, d2 = 0.f, d1 = 0.f;
#pragma unroll
        for (int l = m; l <= L; ++l) {
          float q, dq;
          if (l == m) {
            q = qmm;
            dq = 0.f;
          } else if (l == m + 1) {
            q = (float)(2 * m + 1) * z * qmm;
            dq = (float)(2 * m + 1) * qmm;
          } else {
            q = ((float)(2 * l - 1) * z * q1 - (float)(l + m - 1) * q2) / (float)(l - m);
            dq = ((float)(2 * l - 1) * (q1 + z * d1) - (float)(l + m - 1) * d2) / (float)(l - m);
          }
          if (l > m) {
            q2 = q1;
            q1 = q;
            d2 = d1;
            d1 = dq;
          }
          const float nn = c_norm[l * (l + 1) / 2 + m];
          if (m == 0) {
            const float w = g_in[l * l + l] * nn;
            gz = fmaf(w, dq, gz);
          } else {
            const float wc = g_in[l * l + l + m] * nn, ws = g_in[l * l + l - m] * nn;
            const float fm = (float)m;
            // F_c = Q C_m, F_s = Q S_m
            gx = fmaf(q * fm, fmaf(wc, Cm[m - 1], ws * Sm[m - 1]), gx);
            gy = fmaf(q * fm, fmaf(ws, Cm[m - 1], -wc * Sm[m - 1]), gy);
            gz = fmaf(dq, fmaf(wc, Cm[m], ws * Sm[m]), gz);
          }
        }
      }
      const float gu = gx * x + gy * yy + gz * z;
      gx = (gx - gu * x) * inv;
      gy = (gy - gu * yy) * inv;
      gz = (gz - gu * z) * inv;
    }
    otile[3 * threadIdx.x] = gx;
    otile[3 * threadIdx.x + 1] = gy;
    otile[3 * threadIdx.x + 2] = gz;
  }
  __syncthreads();
  for (int64_t t = threadIdx.x; t < n * 3; t += 128) dr[e0 * 3 + t] = otile[t];
}

// Forces from the edge-vector gradient, one thread per atom a:
//   F[a] = sum over a's receiver edges of G[e] - sum over a's sender edges of G[e]
// (r_e = pos_sender - pos_receiver + shift, F = -dL/dpos), each sum in edge
// order: bitwise reproducible.
__global__ void __launch_bounds__(128) edge_forces_kernel(int64_t n_atoms, const int32_t* __restrict__ rowptr,
                                                          const int32_t* __restrict__ rowptr_T,
                                                          const int32_t* __restrict__ perm_T,
                                                          const float* __restrict__ G, float* __restrict__ F) {
  grid_dependency_wait();
  grid_launch_dependents();
  const int64_t a = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (a >= n_atoms) return;
  float fx = 0.f, fy = 0.f, fz = 0.f;
  for (int e = rowptr[a]; e < rowptr[a + 1]; ++e) {
    fx += G[3 * (int64_t)e];
    fy += G[3 * (int64_t)e + 1];
    fz += G[3 * (int64_t)e + 2];
  }
  float sx = 0.f, sy = 0.f, sz = 0.f;
  for (int t = rowptr_T[a]; t < rowptr_T[a + 1]; ++t) {
    const int64_t e = perm_T[t];
    sx += G[3 * e];
    sy += G[3 * e + 1];
    sz += G[3 * e + 2];
  }
  F[3 * a] = fx - sx;
  F[3 * a + 1] = fy - sy;
  F[3 * a + 2] = fz - sz;
}

// Strain derivative of the loss from the edge-vector gradient:
//   V[3a+b] = sum_e G[e][a] r[e][b]      (= dL/d eps_ab for r_e -> (1 + eps) r_e).
// One cluster of kVirCtas CTAs.  Thread t of the cluster takes the groups of
// four edges t, t + kVirCtas*kVirThreads, ... (three float4 loads per array and
// group: 48 bytes, 16-byte aligned when r and G are), and the last E % 4 edges
// one each; products and sums are in FP64.  Each CTA sums its warps in warp
// order, then CTA 0 adds the CTAs' sums in rank order through distributed
// shared memory, so the result depends on E only (no atomics).
constexpr int kVirCtas = 8;
constexpr int kVirThreads = 512;

__global__ void __cluster_dims__(kVirCtas, 1, 1) __launch_bounds__(kVirThreads)
    edge_virial_kernel(int64_t E, const float* __restrict__ r, const float* __restrict__ G, float* __restrict__ V) {
  namespace cg = cooperative_groups;
  grid_dependency_wait();
  grid_launch_dependents();
  __shared__ double warp_sum[kVirThreads / 32][9];
  __shared__ double cta_sum[9];
  cg::cluster_group cluster = cg::this_cluster();
  const int64_t t = (int64_t)cluster.block_rank() * kVirThreads + threadIdx.x;
  constexpr int64_t kStride = (int64_t)kVirCtas * kVirThreads;
  double acc[9];
#pragma unroll
  for (int k = 0; k < 9; ++k) acc[k] = 0.0;
  const int64_t groups = E / 4;
  for (int64_t q = t; q < groups; q += kStride) {
    float rf[12], gf[12];
    const float4* r4 = reinterpret_cast<const float4*>(r + 12 * q);
    const float4* g4 = reinterpret_cast<const float4*>(G + 12 * q);
#pragma unroll
    for (int v = 0; v < 3; ++v) {
      const float4 a = __ldg(r4 + v), b = __ldg(g4 + v);
      rf[4 * v] = a.x, rf[4 * v + 1] = a.y, rf[4 * v + 2] = a.z, rf[4 * v + 3] = a.w;
      gf[4 * v] = b.x, gf[4 * v + 1] = b.y, gf[4 * v + 2] = b.z, gf[4 * v + 3] = b.w;
    }
#pragma unroll
    for (int k = 0; k < 4; ++k)
#pragma unroll
      for (int a = 0; a < 3; ++a)
#pragma unroll
        for (int b = 0; b < 3; ++b) acc[3 * a + b] += (double)gf[3 * k + a] * (double)rf[3 * k + b];
  }
  if (t < E - 4 * groups) {
    const int64_t e = 4 * groups + t;
#pragma unroll
    for (int a = 0; a < 3; ++a)
#pragma unroll
      for (int b = 0; b < 3; ++b) acc[3 * a + b] += (double)G[3 * e + a] * (double)r[3 * e + b];
  }
#pragma unroll
  for (int k = 0; k < 9; ++k)
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) acc[k] += __shfl_xor_sync(0xffffffffu, acc[k], off);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (lane == 0)
#pragma unroll
    for (int k = 0; k < 9; ++k) warp_sum[warp][k] = acc[k];
  __syncthreads();
  if (threadIdx.x < 9) {
    double s = 0.0;
    for (int w = 0; w < kVirThreads / 32; ++w) s += warp_sum[w][threadIdx.x];
    cta_sum[threadIdx.x] = s;
  }
  cluster.sync();  // every CTA's cta_sum is written
  if (cluster.block_rank() == 0 && threadIdx.x < 9) {
    double s = 0.0;
    for (unsigned q = 0; q < (unsigned)kVirCtas; ++q) s += cluster.map_shared_rank(cta_sum, q)[threadIdx.x];
    V[threadIdx.x] = (float)s;
  }
  cluster.sync();  // no CTA leaves (and frees its shared memory) before CTA 0 has read it
}

// dst += src over n floats (grid-stride), for the sums of the double
// backward's terms.
__global__ void __launch_bounds__(256) add_kernel(int64_t n, const float* __restrict__ src, float* __restrict__ dst) {
  grid_dependency_wait();
  grid_launch_dependents();
  const int64_t stride = (int64_t)gridDim.x * 256;
  for (int64_t i = (int64_t)blockIdx.x * 256 + threadIdx.x; i < n; i += stride) dst[i] += src[i];
}

// Device checks of the graph (a plan's CSR checks, cgtp_plan_set_checks).
// Bits of the flag word: 1 rowptr does not run from 0 to E, 2 rowptr
// decreases, 4 a col outside [0, n_send), 8 rowptr_T does not run from 0 to E,
// 16 rowptr_T decreases, 32 a perm_T entry outside [0, E), 64 a perm_T entry
// whose edge has another sender, 128 perm_T not strictly ascending within a
// sender.  Phase 1 reads only the arrays' own extents; phase 2 (the sender
// lists) runs only when phase 1 found nothing, so its loops follow validated
// bounds.
__global__ void __launch_bounds__(256) csr_check_kernel(int64_t n_recv, int64_t n_send, int64_t E,
                                                        const int32_t* __restrict__ rowptr,
                                                        const int32_t* __restrict__ col,
                                                        const int32_t* __restrict__ rowptr_T,
                                                        int* __restrict__ flag) {
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  const int64_t t0 = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  int bad = 0;
  if (t0 == 0) {
    if (rowptr[0] != 0 || rowptr[n_recv] != E) bad |= 1;
    if (rowptr_T && (rowptr_T[0] != 0 || rowptr_T[n_send] != E)) bad |= 8;
  }
  for (int64_t i = t0; i < n_recv; i += stride)
    if (rowptr[i] > rowptr[i + 1]) bad |= 2;
  for (int64_t e = t0; e < E; e += stride) {
    const int32_t j = col[e];
    if (j < 0 || j >= n_send) bad |= 4;
  }
  if (rowptr_T)
    for (int64_t j = t0; j < n_send; j += stride)
      if (rowptr_T[j] > rowptr_T[j + 1]) bad |= 16;
  if (bad) atomicOr(flag, bad);
}

__global__ void __launch_bounds__(256) csr_perm_check_kernel(int64_t n_send, int64_t E,
                                                             const int32_t* __restrict__ col,
                                                             const int32_t* __restrict__ rowptr_T,
                                                             const int32_t* __restrict__ perm_T,
                                                             int* __restrict__ flag) {
  if (*(volatile int*)flag) return;  // phase 1 failed: the bounds below are not trusted
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  int bad = 0;
  for (int64_t j = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; j < n_send; j += stride) {
    int32_t prev = -1;
    for (int32_t t = rowptr_T[j]; t < rowptr_T[j + 1]; ++t) {
      const int32_t e = perm_T[t];
      if (e < 0 || e >= E) {
        bad |= 32;
        break;
      }
      if (col[e] != j) bad |= 64;
      if (e <= prev) bad |= 128;
      prev = e;
    }
  }
  if (bad) atomicOr(flag, bad);
}

// FP32 FMA throughput probe (the measured FP32 peak the Lmax >= 4 workloads
// are compared with).  Every thread runs kFmaChains independent dependency
// chains a <- a * m + c, kFmaUnroll steps per loop trip; with 512 threads per
// CTA and two CTAs per SM each scheduler has eight warps of eight independent
// FMAs in flight, more than the pipeline latency needs.  m and c come from
// the caller (the compiler cannot fold the chains); the chains' sum is stored
// per thread so that none is dead.  FLOPs = 2 x threads x iters x chains x unroll.
constexpr int kFmaChains = 8;
constexpr int kFmaUnroll = 16;
constexpr int kFmaThreads = 512;

__global__ void __launch_bounds__(kFmaThreads) fma_peak_kernel(int64_t iters, float m, float c,
                                                               float* __restrict__ sink) {
  float a[kFmaChains];
#pragma unroll
  for (int k = 0; k < kFmaChains; ++k) a[k] = (float)(threadIdx.x + k) * 1e-3f;
  for (int64_t it = 0; it < iters; ++it) {
#pragma unroll
    for (int u = 0; u < kFmaUnroll; ++u)
#pragma unroll
      for (int k = 0; k < kFmaChains; ++k) a[k] = fmaf(a[k], m, c);
  }
  float s = 0.f;
#pragma unroll
  for (int k = 0; k < kFmaChains; ++k) s += a[k];
  sink[(int64_t)blockIdx.x * kFmaThreads + threadIdx.x] = s;
}

// The backward's closing reductions in one launch (the block form; the warp
// form, bwd_reduce_rows_kernel, below).
//  blocks [0, n_send): dx[j][c] = sum over sender j's edges of m[perm_T[t]][c].
//    Two groups of 128 threads take the even and the odd positions t0 + 2k of
//    the sender's list, eight rows in flight each; the two partial sums are
//    added in a fixed order, so the result is bitwise reproducible.
//  blocks [n_send, n_send + dy_blocks): dY = sum over the S slice partials.
constexpr int kEpiThreads = 256;

__device__ __forceinline__ void add4(float4& a, const float4 v) {
  a.x += v.x;
  a.y += v.y;
  a.z += v.z;
  a.w += v.w;
}

__global__ void __launch_bounds__(kEpiThreads) bwd_reduce_kernel(
    int64_t n_send, int64_t width, const int32_t* __restrict__ rowptr_T, const int32_t* __restrict__ perm_T,
    const float* __restrict__ m, float* __restrict__ dx, int S, int64_t ny, const float* __restrict__ parts,
    float* __restrict__ dy) {
  grid_dependency_wait();
  grid_launch_dependents();
  __shared__ float4 part[128];
  const int64_t blk = blockIdx.x;
  if (blk >= n_send || dx == nullptr) {
    const int64_t b0 = dx ? blk - n_send : blk;
    const int64_t nblk = (int64_t)gridDim.x - (dx ? n_send : 0);
    for (int64_t k = b0 * kEpiThreads + threadIdx.x; k < ny; k += nblk * kEpiThreads) {
      float acc = 0.f;
      for (int q = 0; q < S; ++q) acc += parts[(int64_t)q * ny + k];
      dy[k] = acc;
    }
    return;
  }
  const int64_t j = blk;
  const int t0 = rowptr_T[j], t1 = rowptr_T[j + 1];
  const int g = threadIdx.x >> 7, c0 = threadIdx.x & 127;
  if ((width & 3) == 0) {
    const int64_t w4 = width >> 2;
    for (int64_t cb = 0; cb < w4; cb += 128) {
      const int64_t c = cb + c0;
      float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
      if (c < w4) {
        int t = t0 + g;
        for (; t + 14 < t1; t += 16) {
          float4 v[8];
#pragma unroll
          for (int k = 0; k < 8; ++k)
            v[k] = __ldcs(reinterpret_cast<const float4*>(m + (int64_t)__ldg(perm_T + t + 2 * k) * width) + c);
#pragma unroll
          for (int k = 0; k < 8; ++k) add4(acc, v[k]);
        }
        for (; t < t1; t += 2) add4(acc, __ldcs(reinterpret_cast<const float4*>(m + (int64_t)__ldg(perm_T + t) * width) + c));
      }
      if (g == 1) part[c0] = acc;
      __syncthreads();
      if (g == 0 && c < w4) {
        const float4 o = part[c0];
        add4(acc, o);
        reinterpret_cast<float4*>(dx + j * width)[c] = acc;
      }
      __syncthreads();
    }
  } else {
    float* pf = reinterpret_cast<float*>(part);
    for (int64_t cb = 0; cb < width; cb += 128) {
      const int64_t c = cb + c0;
      float acc = 0.f;
      if (c < width)
        for (int t = t0 + g; t < t1; t += 2) acc += __ldcs(m + (int64_t)perm_T[t] * width + c);
      if (g == 1) pf[c0] = acc;
      __syncthreads();
      if (g == 0 && c < width) dx[j * width + c] = acc + pf[c0];
      __syncthreads();
    }
  }
}

// The same reductions with dx taken by warps (rows of a multiple of 4 floats):
// warp w of blocks [0, dx_blocks) takes sender j = w / nchunk and the float4
// columns [32 (w % nchunk), +32) of its row, reading the sender's message rows
// in batches of eight predicated loads and adding them in list order (a lane
// past the list adds zero), so the result is bitwise reproducible; blocks
// from dx_blocks on sum the dY slice partials as above.
__global__ void __launch_bounds__(kEpiThreads) bwd_reduce_rows_kernel(
    int64_t n_send, int64_t w4, int64_t nchunk, int64_t dx_blocks, const int32_t* __restrict__ rowptr_T,
    const int32_t* __restrict__ perm_T, const float4* __restrict__ m, float4* __restrict__ dx, int S, int64_t ny,
    const float* __restrict__ parts, float* __restrict__ dy) {
  grid_dependency_wait();
  grid_launch_dependents();
  const int64_t blk = blockIdx.x;
  if (blk >= dx_blocks) {
    const int64_t nblk = (int64_t)gridDim.x - dx_blocks;
    for (int64_t k = (blk - dx_blocks) * kEpiThreads + threadIdx.x; k < ny; k += nblk * kEpiThreads) {
      float acc = 0.f;
      for (int q = 0; q < S; ++q) acc += parts[(int64_t)q * ny + k];
      dy[k] = acc;
    }
    return;
  }
  const int64_t item = blk * (kEpiThreads / 32) + (threadIdx.x >> 5);
  if (item >= n_send * nchunk) return;
  const int64_t j = item / nchunk;
  const int64_t c = (item % nchunk) * 32 + (threadIdx.x & 31);
  if (c >= w4) return;
  const int t0 = __ldg(rowptr_T + j), t1 = __ldg(rowptr_T + j + 1);
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int t = t0; t < t1; t += 8) {
    float4 v[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      v[k] = make_float4(0.f, 0.f, 0.f, 0.f);
      if (t + k < t1) v[k] = __ldcs(m + (int64_t)__ldg(perm_T + t + k) * w4 + c);
    }
#pragma unroll
    for (int k = 0; k < 8; ++k) add4(acc, v[k]);
  }
  dx[j * w4 + c] = acc;
}

}  // namespace

// Uploads c_norm to the current device once (plan creation calls this with
// the plan's device current).  A synchronous copy: it must not run inside a
// stream capture, which is why the launches below never do it themselves.
cudaError_t upload_sph_norm() {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  if (g_norm_ready[dev].load(std::memory_order_acquire)) return cudaSuccess;
  std::lock_guard<std::mutex> g(g_norm_mu);
  if (g_norm_ready[dev].load(std::memory_order_relaxed)) return cudaSuccess;
  float h[28];
  for (int l = 0; l <= 6; ++l)
    for (int m = 0; m <= l; ++m) {
      double f = 1.0;  // (l-m)!/(l+m)!
      for (int k = l - m + 1; k <= l + m; ++k) f /= (double)k;
      h[l * (l + 1) / 2 + m] = (float)(std::sqrt(2.0 * l + 1.0) * (m == 0 ? 1.0 : std::sqrt(2.0 * f)));
    }
  e = cudaMemcpyToSymbol(c_norm, h, sizeof h);
  if (e == cudaSuccess) g_norm_ready[dev].store(true, std::memory_order_release);
  return e;
}

cudaError_t launch_sph_harm(int L, int64_t E, const float* r, float* Y, cudaStream_t s) {
  if (E == 0) return cudaSuccess;
  const dim3 grid((unsigned)((E + 127) / 128));
  switch (L) {
    case 0: return launch_pdl(sph_harm_kernel<0>, grid, 128, s, E, r, Y);
    case 1: return launch_pdl(sph_harm_kernel<1>, grid, 128, s, E, r, Y);
    case 2: return launch_pdl(sph_harm_kernel<2>, grid, 128, s, E, r, Y);
    case 3: return launch_pdl(sph_harm_kernel<3>, grid, 128, s, E, r, Y);
    case 4: return launch_pdl(sph_harm_kernel<4>, grid, 128, s, E, r, Y);
    case 5: return launch_pdl(sph_harm_kernel<5>, grid, 128, s, E, r, Y);
    case 6: return launch_pdl(sph_harm_kernel<6>, grid, 128, s, E, r, Y);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_sph_harm_backward(int L, int64_t E, const float* r, const float* dY, float* dr,
                                     cudaStream_t s) {
  if (E == 0) return cudaSuccess;
  const dim3 grid((unsigned)((E + 127) / 128));
  switch (L) {
    case 0: return launch_pdl(sph_harm_backward_kernel<0>, grid, 128, s, E, r, dY, dr);
    case 1: return launch_pdl(sph_harm_backward_kernel<1>, grid, 128, s, E, r, dY, dr);
    case 2: return launch_pdl(sph_harm_backward_kernel<2>, grid, 128, s, E, r, dY, dr);
    case 3: return launch_pdl(sph_harm_backward_kernel<3>, grid, 128, s, E, r, dY, dr);
    case 4: return launch_pdl(sph_harm_backward_kernel<4>, grid, 128, s, E, r, dY, dr);
    case 5: return launch_pdl(sph_harm_backward_kernel<5>, grid, 128, s, E, r, dY, dr);
    case 6: return launch_pdl(sph_harm_backward_kernel<6>, grid, 128, s, E, r, dY, dr);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_edge_forces(int64_t n_atoms, const int32_t* rowptr, const int32_t* rowptr_T,
                               const int32_t* perm_T, const float* G, float* F, cudaStream_t s) {
  if (n_atoms == 0) return cudaSuccess;
  return launch_pdl(edge_forces_kernel, dim3((unsigned)((n_atoms + 127) / 128)), 128, s, n_atoms, rowptr, rowptr_T,
                    perm_T, G, F);
}

cudaError_t launch_edge_virial(int64_t E, const float* r, const float* G, float* V, cudaStream_t s) {
  return launch_pdl(edge_virial_kernel, dim3(kVirCtas), kVirThreads, s, E, r, G, V);
}

cudaError_t launch_csr_check(int num_sms, int64_t n_recv, int64_t n_send, int64_t E, const int32_t* rowptr,
                             const int32_t* col, const int32_t* rowptr_T, const int32_t* perm_T, int* flag,
                             cudaStream_t s) {
  const int64_t work = std::max<int64_t>({n_recv, n_send, E, 1});
  const unsigned blocks = (unsigned)std::min<int64_t>((work + 255) / 256, (int64_t)num_sms * 8);
  csr_check_kernel<<<blocks, 256, 0, s>>>(n_recv, n_send, E, rowptr, col, rowptr_T, flag);
  if (rowptr_T && perm_T)
    csr_perm_check_kernel<<<blocks, 256, 0, s>>>(n_send, E, col, rowptr_T, perm_T, flag);
  return cudaGetLastError();
}

int64_t fma_peak_sink_floats(int num_sms) { return (int64_t)num_sms * 2 * kFmaThreads; }

cudaError_t launch_fma_peak(int num_sms, int64_t iters, float m, float c, float* sink, cudaStream_t s,
                            double* flops) {
  const int64_t blocks = (int64_t)num_sms * 2;
  *flops = 2.0 * (double)blocks * kFmaThreads * (double)iters * kFmaChains * kFmaUnroll;
  fma_peak_kernel<<<(unsigned)blocks, kFmaThreads, 0, s>>>(iters, m, c, sink);
  return cudaGetLastError();
}

cudaError_t launch_add(int64_t n, const float* src, float* dst, cudaStream_t s) {
  if (n <= 0) return cudaSuccess;
  const int64_t blocks = std::min<int64_t>((n + 255) / 256, 148 * 8);
  return launch_pdl(add_kernel, dim3((unsigned)blocks), 256, s, n, src, dst);
}

cudaError_t launch_bwd_reduce(int64_t n_send, int64_t width, const int32_t* rowptr_T, const int32_t* perm_T,
                              const float* m, float* dx, int S, int64_t ny, const float* parts, float* dy,
                              cudaStream_t s) {
  const int64_t nx = (dx && width > 0) ? n_send : 0;
  const int64_t ndy = (dy && S > 1 && ny > 0) ? std::min<int64_t>((ny + kEpiThreads - 1) / kEpiThreads, 148 * 4) : 0;
  if (nx + ndy == 0) return cudaSuccess;
  // dx by warps when their items fill the GPU (at least 32 warps per SM;
  // measured on B200: Lmax 3 108.9 -> 102.6 us, Lmax 2 wide 41.4 -> 33.6,
  // Lmax 6 62.1 -> 59.8; with fewer items, Lmax 2 14.9 -> 16.8, the block
  // form stays).  CGTP_REDUCE_ROWS=0/1 forces either form.
  static const int force = [] {
    const char* v = std::getenv("CGTP_REDUCE_ROWS");
    return v && (*v == '0' || *v == '1') ? *v - '0' : -1;
  }();
  const int64_t w4 = width / 4, nchunk = (w4 + 31) / 32;
  bool rows = false;
  if (nx > 0 && width % 4 == 0) {
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    rows = force >= 0 ? force == 1 : nx * nchunk >= 32 * (int64_t)sms;
  }
  if (rows) {
    const int64_t dx_blocks = (nx * nchunk + kEpiThreads / 32 - 1) / (kEpiThreads / 32);
    return launch_pdl(bwd_reduce_rows_kernel, dim3((unsigned)(dx_blocks + ndy)), kEpiThreads, s, nx, w4, nchunk,
                      dx_blocks, rowptr_T, perm_T, reinterpret_cast<const float4*>(m), reinterpret_cast<float4*>(dx),
                      S, ndy ? ny : (int64_t)0, parts, dy);
  }
  return launch_pdl(bwd_reduce_kernel, dim3((unsigned)(nx + ndy)), kEpiThreads, s, nx, width, rowptr_T, perm_T, m,
                    nx ? dx : nullptr, S, ndy ? ny : (int64_t)0, parts, dy);
}

}  // namespace cgtp
