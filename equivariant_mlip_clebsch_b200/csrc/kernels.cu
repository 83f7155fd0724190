// kernels.cu -- the kernels that do not depend on the path structure:
// real spherical harmonics of the edge vectors, and the two deterministic
// reductions of the backward (sender-major row sums, slice sums).
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>

#include "internal.hpp"

namespace cgtp {

namespace {

// Normalisation of the component-normalised real harmonics:
//   N_l0 = sqrt(2l+1),  N_lm = sqrt(2l+1) sqrt(2 (l-m)!/(l+m)!)  (m > 0)
// index l*(l+1)/2 + m, l <= 6.
__constant__ float c_norm[28];
bool g_norm_ready[64] = {false};

template <int L>
__global__ void __launch_bounds__(128) sph_harm_kernel(int64_t E, const float* __restrict__ r,
                                                       float* __restrict__ Y) {
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

// dx[j][c] = sum over the sender's edges t (ascending) of m[perm_T[t]][c];
// the sum runs in edge order (bitwise reproducible), four rows in flight.
__global__ void __launch_bounds__(128) segment_rows_kernel(int64_t width,
                                                           const int32_t* __restrict__ rowptr_T,
                                                           const int32_t* __restrict__ perm_T,
                                                           const float* __restrict__ m,
                                                           float* __restrict__ dx) {
  const int64_t j = blockIdx.x;
  const int t0 = rowptr_T[j], t1 = rowptr_T[j + 1];
  if ((width & 3) == 0) {
    const int64_t w4 = width >> 2;
    for (int64_t c = threadIdx.x + (int64_t)blockIdx.y * 128; c < w4; c += 128 * (int64_t)gridDim.y) {
      float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
      int t = t0;
      for (; t + 4 <= t1; t += 4) {
        float4 v[4];
#pragma unroll
        for (int k = 0; k < 4; ++k)
          v[k] = __ldcs(reinterpret_cast<const float4*>(m + (int64_t)__ldg(perm_T + t + k) * width) + c);
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          acc.x += v[k].x;
          acc.y += v[k].y;
          acc.z += v[k].z;
          acc.w += v[k].w;
        }
      }
      for (; t < t1; ++t) {
        const float4 v = __ldcs(reinterpret_cast<const float4*>(m + (int64_t)__ldg(perm_T + t) * width) + c);
        acc.x += v.x;
        acc.y += v.y;
        acc.z += v.z;
        acc.w += v.w;
      }
      reinterpret_cast<float4*>(dx + j * width)[c] = acc;
    }
  } else {
    for (int64_t c = threadIdx.x + (int64_t)blockIdx.y * 128; c < width; c += 128 * (int64_t)gridDim.y) {
      float acc = 0.f;
      for (int t = t0; t < t1; ++t) acc += __ldcs(m + (int64_t)perm_T[t] * width + c);
      dx[j * width + c] = acc;
    }
  }
}

__global__ void sum_slices_kernel(int S, int64_t n, const float* __restrict__ parts,
                                  float* __restrict__ dst) {
  for (int64_t k = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; k < n;
       k += (int64_t)gridDim.x * blockDim.x) {
    float acc = 0.f;
    for (int s = 0; s < S; ++s) acc += parts[(int64_t)s * n + k];
    dst[k] = acc;
  }
}

}  // namespace

static cudaError_t ensure_norm() {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev >= 0 && dev < 64 && g_norm_ready[dev]) return cudaSuccess;
  float h[28];
  for (int l = 0; l <= 6; ++l)
    for (int m = 0; m <= l; ++m) {
      double f = 1.0;  // (l-m)!/(l+m)!
      for (int k = l - m + 1; k <= l + m; ++k) f /= (double)k;
      h[l * (l + 1) / 2 + m] = (float)(std::sqrt(2.0 * l + 1.0) * (m == 0 ? 1.0 : std::sqrt(2.0 * f)));
    }
  e = cudaMemcpyToSymbol(c_norm, h, sizeof h);
  if (e == cudaSuccess && dev >= 0 && dev < 64) g_norm_ready[dev] = true;
  return e;
}

cudaError_t launch_sph_harm(int L, int64_t E, const float* r, float* Y, cudaStream_t s) {
  cudaError_t e = ensure_norm();
  if (e != cudaSuccess) return e;
  if (E == 0) return cudaSuccess;
  const dim3 grid((unsigned)((E + 127) / 128));
  switch (L) {
    case 0: sph_harm_kernel<0><<<grid, 128, 0, s>>>(E, r, Y); break;
    case 1: sph_harm_kernel<1><<<grid, 128, 0, s>>>(E, r, Y); break;
    case 2: sph_harm_kernel<2><<<grid, 128, 0, s>>>(E, r, Y); break;
    case 3: sph_harm_kernel<3><<<grid, 128, 0, s>>>(E, r, Y); break;
    case 4: sph_harm_kernel<4><<<grid, 128, 0, s>>>(E, r, Y); break;
    case 5: sph_harm_kernel<5><<<grid, 128, 0, s>>>(E, r, Y); break;
    case 6: sph_harm_kernel<6><<<grid, 128, 0, s>>>(E, r, Y); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

cudaError_t launch_segment_rows(int64_t n_send, int64_t width, const int32_t* rowptr_T,
                                const int32_t* perm_T, const float* m, float* dx, cudaStream_t s) {
  if (n_send == 0 || width == 0) return cudaSuccess;
  const int64_t cols = (width & 3) == 0 ? width / 4 : width;
  const unsigned gy = (unsigned)((cols + 127) / 128);
  segment_rows_kernel<<<dim3((unsigned)n_send, gy), 128, 0, s>>>(width, rowptr_T, perm_T, m, dx);
  return cudaGetLastError();
}

cudaError_t launch_sum_slices(int S, int64_t n, const float* parts, float* dst, cudaStream_t s) {
  if (n == 0) return cudaSuccess;
  const int64_t blocks = std::min<int64_t>((n + 255) / 256, 148 * 16);
  sum_slices_kernel<<<(unsigned)blocks, 256, 0, s>>>(S, n, parts, dst);
  return cudaGetLastError();
}

}  // namespace cgtp
