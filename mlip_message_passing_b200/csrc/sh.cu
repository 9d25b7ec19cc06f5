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
