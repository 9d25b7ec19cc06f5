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

// Second order.  For upstream u (a gradient with respect to grad_vec), the backward of
// grad_vec = J(vec)^T gy is
//     d/dgy  = J(vec) u                       (the harmonics' directional derivative along u)
//     d/dvec = grad_vec (gy . J(vec) u)       (a Hessian-vector product)
// Both come from evaluating Y on nested dual numbers: the outer number carries the derivative
// along u, its parts are Dual3 numbers carrying the three derivatives with respect to vec; the
// direction vec / |vec| is formed on these numbers (1 / sqrt by its own derivative rules), so
// the radial projection of the first order is included.
template <typename T>
struct DualU {  // a + b e with e^2 = 0, parts of type T
  T a, b;
};
template <typename T>
__device__ __forceinline__ DualU<T> operator+(const DualU<T>& x, const DualU<T>& y) { return {x.a + y.a, x.b + y.b}; }
template <typename T>
__device__ __forceinline__ DualU<T> operator-(const DualU<T>& x, const DualU<T>& y) { return {x.a - y.a, x.b - y.b}; }
template <typename T>
__device__ __forceinline__ DualU<T> operator*(const DualU<T>& x, const DualU<T>& y) {
  return {x.a * y.a, x.a * y.b + x.b * y.a};
}
template <typename T>
struct DualUCast {  // constants of sh_poly as nested duals
  static __device__ __forceinline__ DualU<Dual3<T>> make(double c) { return {Dual3<T>(c), Dual3<T>(0.0)}; }
};
template <typename T>
struct DU {  // DualU<Dual3<T>> with the constructor from a double that sh_poly needs
  DualU<Dual3<T>> q;
  __device__ DU() {}
  __device__ DU(double c) : q{Dual3<T>(c), Dual3<T>(0.0)} {}
  __device__ DU(const DualU<Dual3<T>>& v) : q(v) {}
};
template <typename T>
__device__ __forceinline__ DU<T> operator+(const DU<T>& x, const DU<T>& y) { return DU<T>(x.q + y.q); }
template <typename T>
__device__ __forceinline__ DU<T> operator-(const DU<T>& x, const DU<T>& y) { return DU<T>(x.q - y.q); }
template <typename T>
__device__ __forceinline__ DU<T> operator*(const DU<T>& x, const DU<T>& y) { return DU<T>(x.q * y.q); }

// 1 / sqrt(s) on a Dual3 (value and its three derivatives).
template <typename T>
__device__ __forceinline__ Dual3<T> rsqrt_d3(const Dual3<T>& s) {
  Dual3<T> r;
  r.v = rsqrt_t(s.v);
  const T dv = T(-0.5) * r.v * r.v * r.v;  // d(s^-1/2)/ds
#pragma unroll
  for (int k = 0; k < 3; ++k) r.d[k] = dv * s.d[k];
  return r;
}
// 1 / sqrt(s) on the nested dual: the outer derivative scales by the same first derivative, taken
// as a Dual3 so that its own vec-derivatives are right.
template <typename T>
__device__ __forceinline__ DU<T> rsqrt_du(const DU<T>& s) {
  const Dual3<T> r = rsqrt_d3(s.q.a);
  // d(s^-1/2)/ds = -1/2 s^-3/2 = -1/2 r^3 (a Dual3)
  const Dual3<T> d = Dual3<T>(-0.5) * r * r * r;
  return DU<T>(DualU<Dual3<T>>{r, d * s.q.b});
}

template <int LY, typename T>
__global__ void sh_bwd2_kernel(int64_t n, const T* __restrict__ vec, int norm, const T* __restrict__ gy,
                               const T* __restrict__ u, T* __restrict__ d_gy, T* __restrict__ d_vec) {
  constexpr int NY = (LY + 1) * (LY + 1);
  for (int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < n; i += int64_t(gridDim.x) * blockDim.x) {
    DU<T> c[3];
    T r2 = T(0);
#pragma unroll
    for (int k = 0; k < 3; ++k) {
      const T vk = vec[3 * i + k];
      r2 += vk * vk;
      c[k] = DU<T>(DualU<Dual3<T>>{Dual3<T>(vk, k), Dual3<T>(0.0)});
      c[k].q.b.v = u[3 * i + k];  // the derivative along u
    }
    DU<T> Y[NY];
    if (r2 > T(0)) {
      const DU<T> inv = rsqrt_du(c[0] * c[0] + c[1] * c[1] + c[2] * c[2]);
      sh_poly<LY, DU<T>>(c[0] * inv, c[1] * inv, c[2] * inv, Y);
    } else {  // Y^0 = 1, Y^(l>0) = 0 at the origin: no derivatives
#pragma unroll
      for (int m = 0; m < NY; ++m) Y[m] = DU<T>(m == 0 ? 1.0 : 0.0);
    }
    T hv[3] = {T(0), T(0), T(0)};
#pragma unroll
    for (int l = 0; l <= LY; ++l) {
      const T cn = sh_norm_factor<T>(norm, l);
#pragma unroll
      for (int m = 0; m < 2 * l + 1; ++m) {
        const int j = l * l + m;
        d_gy[i * NY + j] = cn * Y[j].q.b.v;  // (J u)_j
        const T g = cn * gy[i * NY + j];
#pragma unroll
        for (int k = 0; k < 3; ++k) hv[k] = fma(g, Y[j].q.b.d[k], hv[k]);
      }
    }
#pragma unroll
    for (int k = 0; k < 3; ++k) d_vec[3 * i + k] = hv[k];
  }
}

template <typename T>
static void sh_bwd2_launch(int lmax, int64_t n, const void* vec, int norm, const void* gy, const void* u, void* dgy,
                           void* dvec, cudaStream_t s) {
  const int blocks = int(std::min<int64_t>((n + 255) / 256, int64_t(sm_count()) * 16));
  const T* v = static_cast<const T*>(vec);
  const T* g = static_cast<const T*>(gy);
  const T* uu = static_cast<const T*>(u);
  T* a = static_cast<T*>(dgy);
  T* b = static_cast<T*>(dvec);
  switch (lmax) {
    case 0: sh_bwd2_kernel<0, T><<<blocks, 256, 0, s>>>(n, v, norm, g, uu, a, b); break;
    case 1: sh_bwd2_kernel<1, T><<<blocks, 256, 0, s>>>(n, v, norm, g, uu, a, b); break;
    case 2: sh_bwd2_kernel<2, T><<<blocks, 256, 0, s>>>(n, v, norm, g, uu, a, b); break;
    default: sh_bwd2_kernel<3, T><<<blocks, 256, 0, s>>>(n, v, norm, g, uu, a, b); break;
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

extern "C" e3_status e3_spherical_harmonics_double_backward(int32_t lmax, int64_t n, const void* vec,
                                                            e3_sh_norm sh_norm, const void* grad_y,
                                                            const void* u, e3_dtype dtype, void* d_grad_y,
                                                            void* d_vec, void* stream) {
  clear_error();
  if (lmax < 0 || lmax > E3_LMAX) return fail(E3_ERR_UNSUPPORTED, "lmax %d not in [0, %d]", lmax, E3_LMAX);
  if (n < 0) return fail(E3_ERR_SHAPE, "n < 0");
  if (dtype != E3_F32 && dtype != E3_F64) return fail(E3_ERR_INVALID_ARG, "bad dtype");
  if (sh_norm < E3_SH_COMPONENT || sh_norm > E3_SH_NORM) return fail(E3_ERR_INVALID_ARG, "bad sh_norm");
  if (n == 0) return E3_OK;
  const size_t es = dtype == E3_F64 ? 8 : 4;
  const void* ptrs[5] = {vec, grad_y, u, d_grad_y, d_vec};
  for (const void* q : ptrs) {
    if (q == nullptr) return fail(E3_ERR_INVALID_ARG, "NULL pointer");
    if (reinterpret_cast<uintptr_t>(q) % es) return fail(E3_ERR_INVALID_ARG, "pointer not aligned to its element size");
  }
  e3_status st = ensure_device_tables();
  if (st != E3_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (dtype == E3_F32)
    sh_bwd2_launch<float>(lmax, n, vec, sh_norm, grad_y, u, d_grad_y, d_vec, s);
  else
    sh_bwd2_launch<double>(lmax, n, vec, sh_norm, grad_y, u, d_grad_y, d_vec, s);
  const cudaError_t err = cudaGetLastError();
  if (err != cudaSuccess) return fail(E3_ERR_CUDA, "harmonics double backward launch failed: %s", cudaGetErrorString(err));
  return E3_OK;
}
