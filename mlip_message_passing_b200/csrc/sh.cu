// Standalone real spherical harmonics of edge vectors (the same device routine the
// convolution evaluates in registers).
#include "kernels.cuh"

namespace e3b {

template <int LY, typename T>
__global__ void sh_kernel(int64_t n, const T* __restrict__ vec, int norm, T* __restrict__ out) {
  constexpr int NY = (LY + 1) * (LY + 1);
  for (int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < n; i += int64_t(gridDim.x) * blockDim.x) {
    T Y[NY];
    sh_eval<LY, T>(vec[3 * i], vec[3 * i + 1], vec[3 * i + 2], norm, Y);
#pragma unroll
    for (int m = 0; m < NY; ++m) out[i * NY + m] = Y[m];
  }
}

// Forward-mode dual number with three tangents: v + d . (dx, dy, dz).
template <typename T>
struct Dual3 {
  T v, d[3];
  __device__ Dual3() {}
  __device__ Dual3(double c) : v(T(c)), d{T(0), T(0), T(0)} {}
  __device__ Dual3(T val, int k) : v(val), d{T(0), T(0), T(0)} { d[k] = T(1); }
};
template <typename T>
__device__ __forceinline__ Dual3<T> operator+(const Dual3<T>& a, const Dual3<T>& b) {
  Dual3<T> r;
  r.v = a.v + b.v;
#pragma unroll
  for (int k = 0; k < 3; ++k) r.d[k] = a.d[k] + b.d[k];
  return r;
}
template <typename T>
__device__ __forceinline__ Dual3<T> operator-(const Dual3<T>& a, const Dual3<T>& b) {
  Dual3<T> r;
  r.v = a.v - b.v;
#pragma unroll
  for (int k = 0; k < 3; ++k) r.d[k] = a.d[k] - b.d[k];
  return r;
}
template <typename T>
__device__ __forceinline__ Dual3<T> operator*(const Dual3<T>& a, const Dual3<T>& b) {
  Dual3<T> r;
  r.v = a.v * b.v;
#pragma unroll
  for (int k = 0; k < 3; ++k) r.d[k] = a.v * b.d[k] + a.d[k] * b.v;
  return r;
}

// grad_vec[i] = sum_m grad_y[i, m] dY_m/dvec.  Y depends on vec through u = vec / r only, so
// dY/dvec = (1/r) (I - u u^T) grad_u P(u) with P the polynomials of sh_poly, differentiated by
// evaluating them on dual numbers seeded with the unit tangents.
template <int LY, typename T>
__global__ void sh_bwd_kernel(int64_t n, const T* __restrict__ vec, int norm, const T* __restrict__ gy,
                              T* __restrict__ gv) {
  constexpr int NY = (LY + 1) * (LY + 1);
  for (int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < n; i += int64_t(gridDim.x) * blockDim.x) {
    const T vx = vec[3 * i], vy = vec[3 * i + 1], vz = vec[3 * i + 2];
    const T r2 = vx * vx + vy * vy + vz * vz;
    const T inv = r2 > T(0) ? rsqrt_t(r2) : T(0);
    const T u[3] = {vx * inv, vy * inv, vz * inv};
    Dual3<T> Y[NY];
    sh_poly<LY, Dual3<T>>(Dual3<T>(u[0], 0), Dual3<T>(u[1], 1), Dual3<T>(u[2], 2), Y);
    T gu[3] = {T(0), T(0), T(0)};
#pragma unroll
    for (int l = 1; l <= LY; ++l) {
      const T c = sh_norm_factor<T>(norm, l);
#pragma unroll
      for (int m = 0; m < 2 * l + 1; ++m) {
        const T g = c * gy[i * NY + l * l + m];
#pragma unroll
        for (int k = 0; k < 3; ++k) gu[k] = fma(g, Y[l * l + m].d[k], gu[k]);
      }
    }
    const T radial = gu[0] * u[0] + gu[1] * u[1] + gu[2] * u[2];
#pragma unroll
    for (int k = 0; k < 3; ++k) gv[3 * i + k] = inv * (gu[k] - radial * u[k]);
  }
}

template <typename T>
static void sh_bwd_launch(int lmax, int64_t n, const void* vec, int norm, const void* gy, void* gv, cudaStream_t s) {
  const int blocks = int(std::min<int64_t>((n + 255) / 256, int64_t(sm_count()) * 16));
  const T* v = static_cast<const T*>(vec);
  const T* g = static_cast<const T*>(gy);
  T* o = static_cast<T*>(gv);
  switch (lmax) {
    case 0: sh_bwd_kernel<0, T><<<blocks, 256, 0, s>>>(n, v, norm, g, o); break;
    case 1: sh_bwd_kernel<1, T><<<blocks, 256, 0, s>>>(n, v, norm, g, o); break;
    case 2: sh_bwd_kernel<2, T><<<blocks, 256, 0, s>>>(n, v, norm, g, o); break;
    default: sh_bwd_kernel<3, T><<<blocks, 256, 0, s>>>(n, v, norm, g, o); break;
  }
}

template <typename T>
static void sh_launch(int lmax, int64_t n, const void* vec, int norm, void* out, cudaStream_t s) {
  const int blocks = int(std::min<int64_t>((n + 255) / 256, int64_t(sm_count()) * 16));
  const T* v = static_cast<const T*>(vec);
  T* o = static_cast<T*>(out);
  switch (lmax) {
    case 0: sh_kernel<0, T><<<blocks, 256, 0, s>>>(n, v, norm, o); break;
    case 1: sh_kernel<1, T><<<blocks, 256, 0, s>>>(n, v, norm, o); break;
    case 2: sh_kernel<2, T><<<blocks, 256, 0, s>>>(n, v, norm, o); break;
    default: sh_kernel<3, T><<<blocks, 256, 0, s>>>(n, v, norm, o); break;
  }
}

}  // namespace e3b

using namespace e3b;

extern "C" e3_status e3_spherical_harmonics(int32_t lmax, int64_t n, const void* vec, e3_sh_norm sh_norm,
                                            e3_dtype dtype, void* out, void* stream) {
  clear_error();
  if (lmax < 0 || lmax > E3_LMAX) return fail(E3_ERR_UNSUPPORTED, "lmax %d not in [0, %d]", lmax, E3_LMAX);
  if (n < 0) return fail(E3_ERR_SHAPE, "n < 0");
  if (dtype != E3_F32 && dtype != E3_F64) return fail(E3_ERR_INVALID_ARG, "bad dtype");
  if (sh_norm < E3_SH_COMPONENT || sh_norm > E3_SH_NORM) return fail(E3_ERR_INVALID_ARG, "bad sh_norm");
  if (n == 0) return E3_OK;
  const size_t es = dtype == E3_F64 ? 8 : 4;
  if (vec == nullptr || out == nullptr) return fail(E3_ERR_INVALID_ARG, "NULL pointer");
  if ((reinterpret_cast<uintptr_t>(vec) % es) || (reinterpret_cast<uintptr_t>(out) % es))
    return fail(E3_ERR_INVALID_ARG, "pointer not aligned to its element size");
  e3_status st = ensure_device_tables();
  if (st != E3_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (dtype == E3_F32)
    sh_launch<float>(lmax, n, vec, sh_norm, out, s);
  else
    sh_launch<double>(lmax, n, vec, sh_norm, out, s);
  const cudaError_t err = cudaGetLastError();
  if (err != cudaSuccess) return fail(E3_ERR_CUDA, "harmonics launch failed: %s", cudaGetErrorString(err));
  return E3_OK;
}

extern "C" e3_status e3_spherical_harmonics_backward(int32_t lmax, int64_t n, const void* vec, e3_sh_norm sh_norm,
                                                     const void* grad_y, e3_dtype dtype, void* grad_vec,
                                                     void* stream) {
  clear_error();
  if (lmax < 0 || lmax > E3_LMAX) return fail(E3_ERR_UNSUPPORTED, "lmax %d not in [0, %d]", lmax, E3_LMAX);
  if (n < 0) return fail(E3_ERR_SHAPE, "n < 0");
  if (dtype != E3_F32 && dtype != E3_F64) return fail(E3_ERR_INVALID_ARG, "bad dtype");
  if (sh_norm < E3_SH_COMPONENT || sh_norm > E3_SH_NORM) return fail(E3_ERR_INVALID_ARG, "bad sh_norm");
  if (n == 0) return E3_OK;
  const size_t es = dtype == E3_F64 ? 8 : 4;
  if (vec == nullptr || grad_y == nullptr || grad_vec == nullptr) return fail(E3_ERR_INVALID_ARG, "NULL pointer");
  if ((reinterpret_cast<uintptr_t>(vec) % es) || (reinterpret_cast<uintptr_t>(grad_y) % es) ||
      (reinterpret_cast<uintptr_t>(grad_vec) % es))
    return fail(E3_ERR_INVALID_ARG, "pointer not aligned to its element size");
  e3_status st = ensure_device_tables();
  if (st != E3_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (dtype == E3_F32)
    sh_bwd_launch<float>(lmax, n, vec, sh_norm, grad_y, grad_vec, s);
  else
    sh_bwd_launch<double>(lmax, n, vec, sh_norm, grad_y, grad_vec, s);
  const cudaError_t err = cudaGetLastError();
  if (err != cudaSuccess) return fail(E3_ERR_CUDA, "harmonics backward launch failed: %s", cudaGetErrorString(err));
  return E3_OK;
}
