// Tensor product in the uuu connection mode (e3nn course, "Curriculum at a glance", lesson 03b:
// an instruction may tie the channel of both inputs and of the output, with one weight per path
// and channel):
//
//   out[b, p, u, m3] = alpha_p w[b, p, u] sum_{m1, m2} C_p[m1, m2, m3] x[b, l1, u, m1] y[b, l2, u, m2]
//
// Channels never mix, so one thread owns one (sample, channel) pair: it reads that channel's x
// and y components once, evaluates every path of the compiled set with the coefficients at
// compile-time constant-bank offsets, and writes the channel's outputs (forward) or its gradients
// (backward: grad_x, grad_y and grad_w of one (b, u) need nothing from other threads).  The work
// is a few hundred FMAs per (b, u) against (NX + NY + P + NO) elements of traffic, so the kernel
// is bound by HBM.  Neighbouring threads are neighbouring channels, whose components are adjacent
// in the mul_ir layout: when C is a multiple of 32 a warp's 32 channels of one block form one
// contiguous run of 32 (2l + 1) elements, which the warp moves through a shared-memory buffer so
// that every global access instruction covers whole 128-byte lines (RUN kernels); otherwise each
// thread reads and writes its own components.
#include <climits>

#include "kernels.cuh"

namespace e3b {

namespace {

template <typename T, int L, int N>
__device__ __forceinline__ void load_channel(const T* __restrict__ row, int C, int u, T (&v)[N]) {
  static_for<0, L + 1>([&](auto lc) {
    constexpr int l = decltype(lc)::value;
    const T* p = row + int64_t(C) * (l * l) + int64_t(u) * (2 * l + 1);
    static_for<0, 2 * l + 1>([&](auto mc) { v[l * l + decltype(mc)::value] = __ldg(p + decltype(mc)::value); });
  });
}

template <typename T, int L, int N>
__device__ __forceinline__ void store_channel(T* __restrict__ row, int C, int u, const T (&v)[N]) {
  static_for<0, L + 1>([&](auto lc) {
    constexpr int l = decltype(lc)::value;
    T* p = row + int64_t(C) * (l * l) + int64_t(u) * (2 * l + 1);
    static_for<0, 2 * l + 1>([&](auto mc) { p[decltype(mc)::value] = v[l * l + decltype(mc)::value]; });
  });
}

constexpr int UUU_THREADS = 128;

// Run transfers: lane L owns channel u0 + L, whose D components sit at [L D, L D + D) of the
// run; memory holds the run as 32 D contiguous elements starting at `run`.
template <typename T, int D>
__device__ __forceinline__ void run_load(const T* __restrict__ run, T* buf, int lane, T* v) {
#pragma unroll
  for (int j = 0; j < D; ++j) buf[lane + 32 * j] = __ldg(run + lane + 32 * j);
  __syncwarp();
#pragma unroll
  for (int m = 0; m < D; ++m) v[m] = buf[lane * D + m];
  __syncwarp();
}

template <typename T, int D>
__device__ __forceinline__ void run_store(T* __restrict__ run, T* buf, int lane, const T* v) {
#pragma unroll
  for (int m = 0; m < D; ++m) buf[lane * D + m] = v[m];
  __syncwarp();
#pragma unroll
  for (int j = 0; j < D; ++j) run[lane + 32 * j] = buf[lane + 32 * j];
  __syncwarp();
}

// Components of channel u of every block l = 0..L of a row (RUN: through the warp's buffer).
template <bool RUN, typename T, int L, int N>
__device__ __forceinline__ void get_channel(const T* __restrict__ row, int C, int u, int lane, T* buf, T (&v)[N]) {
  if constexpr (RUN) {
    static_for<0, L + 1>([&](auto lc) {
      constexpr int l = decltype(lc)::value;
      run_load<T, 2 * l + 1>(row + int64_t(C) * (l * l) + int64_t(u - lane) * (2 * l + 1), buf, lane, v + l * l);
    });
  } else {
    load_channel<T, L>(row, C, u, v);
  }
}

template <bool RUN, typename T, int L, int N>
__device__ __forceinline__ void put_channel(T* __restrict__ row, int C, int u, int lane, T* buf, const T (&v)[N]) {
  if constexpr (RUN) {
    static_for<0, L + 1>([&](auto lc) {
      constexpr int l = decltype(lc)::value;
      run_store<T, 2 * l + 1>(row + int64_t(C) * (l * l) + int64_t(u - lane) * (2 * l + 1), buf, lane, v + l * l);
    });
  } else {
    store_channel<T, L>(row, C, u, v);
  }
}

template <class CF, bool RUN>
__global__ void __launch_bounds__(UUU_THREADS) uuu_fwd_kernel(const UuuArgs a) {
  using T = typename CF::T;
  __shared__ T sbuf[UUU_THREADS / 32][32 * 7];
  const int lane = threadIdx.x & 31;
  T* buf = sbuf[threadIdx.x >> 5];
  const int64_t t = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
  if (t >= a.B * a.C) return;  // RUN: C % 32 == 0, so whole warps leave together
  const int64_t b = t / a.C;
  const int u = int(t - b * a.C);
  T X[CF::NX], Y[CF::NY];
  get_channel<RUN, T, CF::LX>(static_cast<const T*>(a.x) + b * a.dim1, a.C, u, lane, buf, X);
  get_channel<RUN, T, CF::LY>(static_cast<const T*>(a.y) + b * a.dim2, a.C, u, lane, buf, Y);
  const T* w = static_cast<const T*>(a.w) + b * a.w_stride + u;
  T* out = static_cast<T*>(a.out) + b * a.dim_out;
  static_for<0, CF::P>([&](auto pc) {
    constexpr int P = decltype(pc)::value;
    using PC = PathC<CF, P>;
    constexpr int L1 = PC::L1, L2 = PC::L2, L3 = PC::L3;
    const T s = T(a.alpha[P]) * __ldg(w + int64_t(P) * a.C);
    T o[PC::D3];
    static_for<0, PC::D3>([&](auto m3c) {
      constexpr int M3 = decltype(m3c)::value - L3;
      T v = T(0);
      static_for<-L1, L1 + 1>([&](auto m1c) {
        constexpr int M1 = decltype(m1c)::value;
        if constexpr (a_nz(L1, L2, L3, M1, M3))
          v = fma(a_entry<T, L1, L2, L3, M1, M3>(Y), X[L1 * L1 + L1 + M1], v);
      });
      o[M3 + L3] = s * v;
    });
    T* ob = out + int64_t(a.C) * PC::OUT;
    if constexpr (RUN) {
      run_store<T, PC::D3>(ob + int64_t(u - lane) * PC::D3, buf, lane, o);
    } else {
#pragma unroll
      for (int m = 0; m < PC::D3; ++m) ob[int64_t(u) * PC::D3 + m] = o[m];
    }
  });
}

template <class CF, bool RUN>
__global__ void __launch_bounds__(UUU_THREADS) uuu_bwd_kernel(const UuuArgs a) {
  using T = typename CF::T;
  __shared__ T sbuf[UUU_THREADS / 32][32 * 7];
  const int lane = threadIdx.x & 31;
  T* buf = sbuf[threadIdx.x >> 5];
  const int64_t t = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
  if (t >= a.B * a.C) return;  // RUN: C % 32 == 0, so whole warps leave together
  const int64_t b = t / a.C;
  const int u = int(t - b * a.C);
  T X[CF::NX], Y[CF::NY], dX[CF::NX], dY[CF::NY];
  get_channel<RUN, T, CF::LX>(static_cast<const T*>(a.x) + b * a.dim1, a.C, u, lane, buf, X);
  get_channel<RUN, T, CF::LY>(static_cast<const T*>(a.y) + b * a.dim2, a.C, u, lane, buf, Y);
#pragma unroll
  for (int i = 0; i < CF::NX; ++i) dX[i] = T(0);
#pragma unroll
  for (int i = 0; i < CF::NY; ++i) dY[i] = T(0);
  const T* w = static_cast<const T*>(a.w) + b * a.w_stride + u;
  const T* g = static_cast<const T*>(a.grad_out) + b * a.dim_out;
  T* gw = a.grad_w ? static_cast<T*>(a.grad_w) + b * a.w_stride + u : nullptr;
  if constexpr (RUN) {
    // ask L2 for every path's grad_out run and weight line of this warp now: the loop below reads
    // them one path after the other, and each would otherwise wait on HBM in turn
    static_for<0, CF::P>([&](auto pc) {
      constexpr int P = decltype(pc)::value;
      using PC = PathC<CF, P>;
      const T* run = g + int64_t(a.C) * PC::OUT + int64_t(u - lane) * PC::D3;
      if (lane * 128 < int(32 * PC::D3 * sizeof(T))) asm volatile("prefetch.global.L2 [%0];" ::"l"(run + lane * 128 / int(sizeof(T))));
      if (lane == 31) asm volatile("prefetch.global.L2 [%0];" ::"l"(w + int64_t(P) * a.C));
    });
  }
  static_for<0, CF::P>([&](auto pc) {
    constexpr int P = decltype(pc)::value;
    using PC = PathC<CF, P>;
    constexpr int L1 = PC::L1, L2 = PC::L2, L3 = PC::L3;
    T G[PC::D3];
    const T* gb = g + int64_t(a.C) * PC::OUT;
    if constexpr (RUN) {
      run_load<T, PC::D3>(gb + int64_t(u - lane) * PC::D3, buf, lane, G);
    } else {
#pragma unroll
      for (int m = 0; m < PC::D3; ++m) G[m] = __ldg(gb + int64_t(u) * PC::D3 + m);
    }
    const T al = T(a.alpha[P]);
    const T q = al * __ldg(w + int64_t(P) * a.C);
    T z = T(0);  // sum C x y g: the path's weight gradient over alpha
    static_for<-L1, L1 + 1>([&](auto m1c) {
      constexpr int M1 = decltype(m1c)::value;
      static_for<-L2, L2 + 1>([&](auto m2c) {
        constexpr int M2 = decltype(m2c)::value;
        static_for<-L3, L3 + 1>([&](auto m3c) {
          constexpr int M3 = decltype(m3c)::value;
          if constexpr (cg_nz(L1, L2, L3, M1, M2, M3)) {
            constexpr int I = cg_index(L1, L2, L3, M1, M2, M3);
            const T s = CGT<T>::template get<I>() * G[M3 + L3];
            const T xv = X[L1 * L1 + L1 + M1], yv = Y[L2 * L2 + L2 + M2];
            z = fma(s, xv * yv, z);
            dX[L1 * L1 + L1 + M1] = fma(s * q, yv, dX[L1 * L1 + L1 + M1]);
            dY[L2 * L2 + L2 + M2] = fma(s * q, xv, dY[L2 * L2 + L2 + M2]);
          }
        });
      });
    });
    if (gw) gw[int64_t(P) * a.C] = al * z;
  });
  if (a.grad_x) put_channel<RUN, T, CF::LX>(static_cast<T*>(a.grad_x) + b * a.dim1, a.C, u, lane, buf, dX);
  if (a.grad_y) put_channel<RUN, T, CF::LY>(static_cast<T*>(a.grad_y) + b * a.dim2, a.C, u, lane, buf, dY);
}

template <class CF>
e3_status launch_uuu_cfg(const UuuArgs& a, bool backward) {
  constexpr int threads = UUU_THREADS;
  const int64_t blocks = (a.B * a.C + threads - 1) / threads;
  if (blocks > INT_MAX) return fail(E3_ERR_SHAPE, "B x C = %lld is too large", (long long)(a.B * a.C));
  const cudaStream_t s = static_cast<cudaStream_t>(a.stream);
  const bool run = a.C % 32 == 0;
  if (backward) {
    if (run)
      uuu_bwd_kernel<CF, true><<<unsigned(blocks), threads, 0, s>>>(a);
    else
      uuu_bwd_kernel<CF, false><<<unsigned(blocks), threads, 0, s>>>(a);
  } else {
    if (run)
      uuu_fwd_kernel<CF, true><<<unsigned(blocks), threads, 0, s>>>(a);
    else
      uuu_fwd_kernel<CF, false><<<unsigned(blocks), threads, 0, s>>>(a);
  }
  const cudaError_t err = cudaGetLastError();
  if (err != cudaSuccess) return fail(E3_ERR_CUDA, "uuu launch failed: %s", cudaGetErrorString(err));
  return E3_OK;
}

}  // namespace

e3_status upload_tables_uuu(const double* t64, const float* t32) {
  const cudaError_t err = upload_tables(t64, t32);
  if (err != cudaSuccess) return fail(E3_ERR_CUDA, "uploading the CG table failed: %s", cudaGetErrorString(err));
  return E3_OK;
}

e3_status launch_uuu(const e3_plan* plan, const UuuArgs& a, bool backward) {
#define E3_U(A, B, C)                                                                    \
  if (plan->LX == A && plan->LY == B && plan->LO == C) {                                 \
    if (plan->dtype == E3_F32) return launch_uuu_cfg<Cfg<A, B, C, float>>(a, backward);  \
    return launch_uuu_cfg<Cfg<A, B, C, double>>(a, backward);                            \
  }
  E3_CONFIGS(E3_U)
#undef E3_U
  return fail(E3_ERR_UNSUPPORTED, "degrees (%d, %d, %d) are not compiled", plan->LX, plan->LY, plan->LO);
}

}  // namespace e3b
