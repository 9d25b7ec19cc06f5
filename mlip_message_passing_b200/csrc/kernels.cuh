// Kernels for the channelwise ("uvu") Clebsch-Gordan tensor product and the message-passing
// convolution, forward and backward, for sm_100a.
//
// What is computed (e3nn course, "Curriculum at a glance", lessons 03a/03b/06a; E3J, sections
// E.1 and E.2.2): for an edge e with sender s, receiver n, harmonics Y_e and weights w_e,
//     msg[p, u, m3] = alpha_p * w[e, p, u] * sum_{m1, m2} C_p[m1, m2, m3] x[s, l1(p), u, m1] Y_e[l2(p), m2]
//     out[n]        = scale * sum_{e : dst_e = n} msg_e
// and the transposes of this trilinear map for the backward pass.
//
// Work decomposition (B200: FP32 FMA issue is the co-bottleneck with HBM for l <= 3):
//   * A_p[m1, m3] = sum_m2 C_p[m1, m2, m3] Y[m2] is formed once per edge and path in registers;
//     the CG values come from __constant__ memory at compile-time offsets, so they enter the
//     FFMA as constant-bank operands and cost no load instruction.  Only the structural
//     nonzeros of C and of A are visited (selection rules in cg_pattern.h).
//   * A thread owns 4 consecutive channels x one compile-time group of paths, so one A entry
//     feeds 4 FMAs and the accumulators (<= 80) stay in registers.
//   * Channels are the fastest thread index; when C/4 < 32 the remaining lanes of a warp take
//     different edges of the same receiver ("slices") and are summed with a fixed butterfly at
//     the end, so the reduction order is fixed and the result is bitwise repeatable.
//   * Forward: one CTA per (receiver segment, path group); the receiver's in-edges are
//     consecutive in memory (receiver CSR), so the weight rows stream contiguously and x[src]
//     rows are gathered from L2.  No floating-point atomics, no [E, dim_out] message tensor.
//   * Backward: one one-warp CTA per (sender segment, path group), walking the sender CSR; A
//     is recomputed, never stored; grad_w and grad_y are edge-local writes; grad_x is reduced
//     in registers in a fixed order.  All groups run in one launch; the groups of one unit are
//     ordered by a progress counter (the first group to touch a grad_x or grad_y block stores
//     it, later groups add).
//   * A row (a receiver's in-edges, a sender's out-edges) of more than SEG_EDGES edges is cut
//     into segments, each its own unit, so a hub does not serialise on one CTA; the segments'
//     partial sums join the row in segment order through progress counters.  CTAs take tickets
//     in start order, and every wait is on a CTA with an earlier ticket: no deadlock.
#pragma once

#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>
#include <type_traits>

#include "cg_pattern.h"
#include "internal.h"

namespace e3b {

// Each translation unit that includes this header gets its own copy of the coefficient
// tables (internal linkage); upload_tables() fills the copy of the including unit.
static __constant__ float c_cg32[CG_TABLE_SIZE];
static __constant__ double c_cg64[CG_TABLE_SIZE];

constexpr int MAXP = 64;  // paths per plan (34 at l <= 3)
constexpr int K = 4;      // channels per thread

template <typename T>
struct CGT;
template <>
struct CGT<float> {
  template <int I>
  static __device__ __forceinline__ float get() {
    static_assert(I >= 0 && I < CG_TABLE_SIZE, "CG index");
    return c_cg32[I];
  }
};
template <>
struct CGT<double> {
  template <int I>
  static __device__ __forceinline__ double get() {
    static_assert(I >= 0 && I < CG_TABLE_SIZE, "CG index");
    return c_cg64[I];
  }
};

template <int B, int E, typename F>
__device__ __forceinline__ void static_for(F&& f) {
  if constexpr (B < E) {
    f(std::integral_constant<int, B>());
    static_for<B + 1, E>(f);
  }
}

template <int N, int I = 0, typename F>
__device__ __forceinline__ void dispatch(int g, F&& f) {
  if constexpr (I < N) {
    if (g == I)
      f(std::integral_constant<int, I>());
    else
      dispatch<N, I + 1>(g, f);
  }
}

__device__ __forceinline__ void record_error(int* status, int code) { atomicCAS(status, 0, code); }

__device__ __forceinline__ float rsqrt_t(float v) { return rsqrtf(v); }
__device__ __forceinline__ double rsqrt_t(double v) { return rsqrt(v); }

// --------------------------------------------------------------------- configuration ---
template <int LX_, int LY_, int LO_, typename T_>
struct Cfg {
  static constexpr int LX = LX_, LY = LY_, LO = LO_;
  using T = T_;
  static constexpr PathTable PT = make_path_table(LX, LY, LO, GROUP_OUT_CAP);
  static constexpr int P = PT.n;
  static constexpr int G = PT.ngroups;
  static constexpr int NY = (LY + 1) * (LY + 1);
  static constexpr int NX = (LX + 1) * (LX + 1);
  static constexpr int NO = PT.out_dim;
  static_assert(P <= MAXP, "too many paths");
};

template <class CF, int GI>
struct Grp {
  static constexpr int PB = CF::PT.gbegin[GI];
  static constexpr int PE = CF::PT.gbegin[GI + 1];
  static constexpr int NP = PE - PB;
  static_assert(NP >= 1, "empty path group");
  static constexpr int L1A = CF::PT.l1[PB];
  static constexpr int L1B = CF::PT.l1[PE - 1];
  static constexpr int XB = L1A * L1A;                    // first per-channel x index used
  static constexpr int NXG = (L1B + 1) * (L1B + 1) - XB;  // per-channel x values used
  static constexpr int OB = CF::PT.out_off[PB];
  static constexpr int NOG = CF::PT.out_off[PE] - OB;
};

template <class CF, int P>
struct PathC {
  static constexpr int L1 = CF::PT.l1[P];
  static constexpr int L2 = CF::PT.l2[P];
  static constexpr int L3 = CF::PT.l3[P];
  static constexpr int D1 = 2 * L1 + 1, D3 = 2 * L3 + 1;
  static constexpr int OUT = CF::PT.out_off[P];  // per-channel offset
};

// A_p[m1, m3] for one (m1, m3): sum over the pattern m2 of C[m1, m2, m3] * Y[l2, m2].
template <typename T, int L1, int L2, int L3, int M1, int M3, int NY>
__device__ __forceinline__ T a_entry(const T (&Y)[NY]) {
  T v = T(0);
  static_for<-L2, L2 + 1>([&](auto m2c) {
    constexpr int M2 = decltype(m2c)::value;
    if constexpr (cg_nz(L1, L2, L3, M1, M2, M3)) {
      constexpr int I = cg_index(L1, L2, L3, M1, M2, M3);
      v = fma(CGT<T>::template get<I>(), Y[L2 * L2 + L2 + M2], v);
    }
  });
  return v;
}

__device__ __forceinline__ float2 lo2(float4 v) { return make_float2(v.x, v.y); }
__device__ __forceinline__ float2 hi2(float4 v) { return make_float2(v.z, v.w); }

// ----------------------------------------------------------------- memory helpers ---
// 16-byte vector moves between global memory and register arrays.
template <typename T, int N>
__device__ __forceinline__ void ld16(T (&r)[N], const T* __restrict__ p, bool stream) {
  if constexpr (std::is_same<T, float>::value) {
    static_assert(N % 4 == 0, "float chunk");
#pragma unroll
    for (int i = 0; i < N / 4; ++i) {
      const float4 v = stream ? __ldcs(reinterpret_cast<const float4*>(p) + i)
                              : __ldg(reinterpret_cast<const float4*>(p) + i);
      r[4 * i] = v.x;
      r[4 * i + 1] = v.y;
      r[4 * i + 2] = v.z;
      r[4 * i + 3] = v.w;
    }
  } else {
    static_assert(N % 2 == 0, "double chunk");
#pragma unroll
    for (int i = 0; i < N / 2; ++i) {
      const double2 v = stream ? __ldcs(reinterpret_cast<const double2*>(p) + i)
                               : __ldg(reinterpret_cast<const double2*>(p) + i);
      r[2 * i] = v.x;
      r[2 * i + 1] = v.y;
    }
  }
}

// The same through L2 only (coherent): for values another CTA of the same launch wrote.
template <typename T, int N>
__device__ __forceinline__ void ld16_l2(T (&r)[N], const T* __restrict__ p) {
  if constexpr (std::is_same<T, float>::value) {
    static_assert(N % 4 == 0, "float chunk");
#pragma unroll
    for (int i = 0; i < N / 4; ++i) {
      const float4 v = __ldcg(reinterpret_cast<const float4*>(p) + i);
      r[4 * i] = v.x;
      r[4 * i + 1] = v.y;
      r[4 * i + 2] = v.z;
      r[4 * i + 3] = v.w;
    }
  } else {
    static_assert(N % 2 == 0, "double chunk");
#pragma unroll
    for (int i = 0; i < N / 2; ++i) {
      const double2 v = __ldcg(reinterpret_cast<const double2*>(p) + i);
      r[2 * i] = v.x;
      r[2 * i + 1] = v.y;
    }
  }
}

template <typename T, int N>
__device__ __forceinline__ void st16(T* __restrict__ p, const T (&r)[N]) {
  if constexpr (std::is_same<T, float>::value) {
#pragma unroll
    for (int i = 0; i < N / 4; ++i)
      __stcs(reinterpret_cast<float4*>(p) + i, make_float4(r[4 * i], r[4 * i + 1], r[4 * i + 2], r[4 * i + 3]));
  } else {
#pragma unroll
    for (int i = 0; i < N / 2; ++i) __stcs(reinterpret_cast<double2*>(p) + i, make_double2(r[2 * i], r[2 * i + 1]));
  }
}

// x values of the group's degree range for channels 4cb..4cb+3 of row `row`:
// xr[k][j] = x[row, block l, channel 4cb+k, m] with j = l*l + (m + l) - XB.
template <class CF, class GR, typename T>
__device__ __forceinline__ void load_x(T (&xr)[K][GR::NXG], const T* __restrict__ xrow, int C, int cb) {
  static_for<GR::L1A, GR::L1B + 1>([&](auto lc) {
    constexpr int L = decltype(lc)::value;
    constexpr int D = 2 * L + 1;
    T t[K * D];
    ld16(t, xrow + size_t(C) * (L * L) + size_t(4 * cb) * D, false);
#pragma unroll
    for (int k = 0; k < K; ++k)
#pragma unroll
      for (int m = 0; m < D; ++m) xr[k][L * L - GR::XB + m] = t[k * D + m];
  });
}

// ------------------------------------------------------------ spherical harmonics ---
// Component-normalised harmonics of a unit vector (x, y, z) as polynomials, Y[0] = 1.  T may be
// a forward-mode dual number: the harmonics backward differentiates this routine.
template <int LY, typename T>
__device__ __forceinline__ void sh_poly(T x, T y, T z, T (&Y)[(LY + 1) * (LY + 1)]) {
  Y[0] = T(1);
  if constexpr (LY >= 1) {
    const T s3 = T(1.7320508075688772935);
    Y[1] = s3 * y;
    Y[2] = s3 * z;
    Y[3] = s3 * x;
    if constexpr (LY >= 2) {
      const T s15 = T(3.8729833462074168852), s5h = T(1.1180339887498948482);
      Y[4] = s15 * x * y;
      Y[5] = s15 * y * z;
      Y[6] = s5h * (T(2) * z * z - x * x - y * y);
      Y[7] = s15 * x * z;
      Y[8] = T(0.5) * s15 * (x * x - y * y);
      if constexpr (LY >= 3) {
        const T c70 = T(2.0916500663351888699);   // sqrt(70)/4
        const T c105 = T(10.246950765959598383);  // sqrt(105)
        const T c42 = T(1.6201851746019650147);   // sqrt(42)/4
        const T c7 = T(1.3228756555322952953);    // sqrt(7)/2
        const T x2 = x * x, y2 = y * y, z2 = z * z;
        const T f = T(4) * z2 - x2 - y2;            // 5 z^2 - r^2 on the sphere
        Y[9] = c70 * y * (T(3) * x2 - y2);
        Y[10] = c105 * x * y * z;
        Y[11] = c42 * y * f;
        Y[12] = c7 * z * (T(2) * z2 - T(3) * x2 - T(3) * y2);
        Y[13] = c42 * x * f;
        Y[14] = T(0.5) * c105 * z * (x2 - y2);
        Y[15] = c70 * x * (x2 - T(3) * y2);
      }
    }
  }
}

// Factor of degree l that turns component-normalised harmonics into normalisation `norm`:
// integral 1/sqrt(4 pi) for every degree, norm 1/sqrt(2l+1) for l > 0.
template <typename T>
__device__ __forceinline__ T sh_norm_factor(int norm, int l) {
  if (norm == E3_SH_INTEGRAL) return T(0.28209479177387814347);
  if (norm == E3_SH_NORM && l > 0) return rsqrt_t(T(2 * l + 1));
  return T(1);
}

// Real harmonics, component normalisation (sum_m Y_lm^2 = 2l+1 on the unit sphere), m = -l..l,
// z the pole, no Condon-Shortley phase (e3nn course, lesson 02b), of the direction of (vx, vy,
// vz), scaled to normalisation `norm`.  r = 0 gives Y^0 = 1 (scaled) and zero for l > 0: every
// l > 0 polynomial vanishes at the origin.
template <int LY, typename T>
__device__ __forceinline__ void sh_eval(T vx, T vy, T vz, int norm, T (&Y)[(LY + 1) * (LY + 1)]) {
  T x = T(0), y = T(0), z = T(0);
  if constexpr (LY >= 1) {
    const T r2 = vx * vx + vy * vy + vz * vz;
    const T inv = r2 > T(0) ? rsqrt_t(r2) : T(0);
    x = vx * inv;
    y = vy * inv;
    z = vz * inv;
  }
  sh_poly<LY, T>(x, y, z, Y);
  if (norm != E3_SH_COMPONENT) {
#pragma unroll
    for (int l = 0; l <= LY; ++l) {
      const T c = sh_norm_factor<T>(norm, l);
#pragma unroll
      for (int m = 0; m < 2 * l + 1; ++m) Y[l * l + m] *= c;
    }
  }
}

template <class CF, typename T>
__device__ __forceinline__ void load_y(T (&Y)[CF::NY], const T* __restrict__ y, const T* __restrict__ vec,
                                       int norm, int64_t e) {
  if (y != nullptr) {
#pragma unroll
    for (int i = 0; i < CF::NY; ++i) Y[i] = __ldg(y + e * CF::NY + i);
  } else {
    const T vx = __ldg(vec + 3 * e), vy = __ldg(vec + 3 * e + 1), vz = __ldg(vec + 3 * e + 2);
    sh_eval<CF::LY, T>(vx, vy, vz, norm, Y);
  }
}

// ========================================================================== forward ===
struct KFwd {
  const int32_t* row_ptr;
  const int32_t* src;
  const void* x;
  const void* y;
  const void* vec;
  const void* w;
  void* out;
  int64_t n_rows, n_edges, w_stride;
  int C, sh_norm, n_chunks, stages;
  int* status;
  // convolution: ticket counter and per (row, group) progress counters (zero at launch), the
  // receiver units of the topology buffer and their number, and the grid's bound on it
  int* ticket;
  int* flags;
  const int4* uinfo;
  const int32_t* unseg;
  const int32_t* n_units;
  int64_t units_max;
  unsigned long long wait_ns;  // limit of every bounded wait
  int first_ticket;            // first ticket drawn (0; a test withholds tickets by raising it)
  double pscale[MAXP];  // scale * alpha_p
};

template <class CF, int GI>
struct FwdAcc {
  using T = typename CF::T;
  using GR = Grp<CF, GI>;
  T acc[K][GR::NOG];

  __device__ __forceinline__ void zero() {
#pragma unroll
    for (int k = 0; k < K; ++k)
#pragma unroll
      for (int o = 0; o < GR::NOG; ++o) acc[k][o] = T(0);
  }

  // acc += w (x) A x for one edge
  __device__ __forceinline__ void edge(const T (&xr)[K][GR::NXG], const T (&wr)[K][GR::NP], const T (&Y)[CF::NY]) {
    static_for<GR::PB, GR::PE>([&](auto pc) {
      constexpr int P = decltype(pc)::value;
      using PC = PathC<CF, P>;
      constexpr int L1 = PC::L1, L2 = PC::L2, L3 = PC::L3, D1 = PC::D1, D3 = PC::D3;
      constexpr int XO = L1 * L1 - GR::XB, OO = PC::OUT - GR::OB, PW = P - GR::PB;
      if constexpr (D1 < D3) {
        // scale x by the weight first (fewer multiplies), then acc += A^T xs
        T xs[K][D1];
#pragma unroll
        for (int k = 0; k < K; ++k)
#pragma unroll
          for (int m1 = 0; m1 < D1; ++m1) xs[k][m1] = wr[k][PW] * xr[k][XO + m1];
        static_for<0, D3>([&](auto m3c) {
          constexpr int M3I = decltype(m3c)::value;
          T a[D1];
          static_for<0, D1>([&](auto m1c) {
            constexpr int M1I = decltype(m1c)::value;
            if constexpr (a_nz(L1, L2, L3, M1I - L1, M3I - L3))
              a[M1I] = a_entry<T, L1, L2, L3, M1I - L1, M3I - L3>(Y);
          });
#pragma unroll
          for (int k = 0; k < K; ++k) {
            T t = acc[k][OO + M3I];
            static_for<0, D1>([&](auto m1c) {
              constexpr int M1I = decltype(m1c)::value;
              if constexpr (a_nz(L1, L2, L3, M1I - L1, M3I - L3)) t = fma(a[M1I], xs[k][M1I], t);
            });
            acc[k][OO + M3I] = t;
          }
        });
      } else {
        // t = A^T x, then acc += w t
        static_for<0, D3>([&](auto m3c) {
          constexpr int M3I = decltype(m3c)::value;
          T a[D1];
          static_for<0, D1>([&](auto m1c) {
            constexpr int M1I = decltype(m1c)::value;
            if constexpr (a_nz(L1, L2, L3, M1I - L1, M3I - L3))
              a[M1I] = a_entry<T, L1, L2, L3, M1I - L1, M3I - L3>(Y);
          });
#pragma unroll
          for (int k = 0; k < K; ++k) {
            T t = T(0);
            static_for<0, D1>([&](auto m1c) {
              constexpr int M1I = decltype(m1c)::value;
              if constexpr (a_nz(L1, L2, L3, M1I - L1, M3I - L3)) t = fma(a[M1I], xr[k][XO + M1I], t);
            });
            acc[k][OO + M3I] = fma(wr[k][PW], t, acc[k][OO + M3I]);
          }
        });
      }
    });
  }

  // The same contraction reading each path's weights and x block from the staged slices just
  // before use (sw: the group's weight slice, path PB first; sx: x blocks L1A..L1B), so that
  // only one path's operands are live at a time.
  __device__ __forceinline__ void edge_smem(const T* sw, const T* sx, const T (&Y)[CF::NY], int C, int cb) {
    static_for<GR::PB, GR::PE>([&](auto pc) {
      constexpr int P = decltype(pc)::value;
      using PC = PathC<CF, P>;
      constexpr int L1 = PC::L1, L2 = PC::L2, L3 = PC::L3, D1 = PC::D1, D3 = PC::D3;
      constexpr int OO = PC::OUT - GR::OB;
      T wk[K];
      lds16(wk, sw + size_t(P - GR::PB) * C + 4 * cb);
      T xk[K * D1];
      lds16(xk, sx + size_t(C) * (L1 * L1 - GR::XB) + size_t(4 * cb) * D1);
      if constexpr (D1 < D3) {
        T xs[K][D1];
#pragma unroll
        for (int k = 0; k < K; ++k)
#pragma unroll
          for (int m1 = 0; m1 < D1; ++m1) xs[k][m1] = wk[k] * xk[k * D1 + m1];
        static_for<0, D3>([&](auto m3c) {
          constexpr int M3I = decltype(m3c)::value;
          T a[D1];
          static_for<0, D1>([&](auto m1c) {
            constexpr int M1I = decltype(m1c)::value;
            if constexpr (a_nz(L1, L2, L3, M1I - L1, M3I - L3)) a[M1I] = a_entry<T, L1, L2, L3, M1I - L1, M3I - L3>(Y);
          });
#pragma unroll
          for (int k = 0; k < K; ++k) {
            T t = acc[k][OO + M3I];
            static_for<0, D1>([&](auto m1c) {
              constexpr int M1I = decltype(m1c)::value;
              if constexpr (a_nz(L1, L2, L3, M1I - L1, M3I - L3)) t = fma(a[M1I], xs[k][M1I], t);
            });
            acc[k][OO + M3I] = t;
          }
        });
      } else {
        static_for<0, D3>([&](auto m3c) {
          constexpr int M3I = decltype(m3c)::value;
          T a[D1];
          static_for<0, D1>([&](auto m1c) {
            constexpr int M1I = decltype(m1c)::value;
            if constexpr (a_nz(L1, L2, L3, M1I - L1, M3I - L3)) a[M1I] = a_entry<T, L1, L2, L3, M1I - L1, M3I - L3>(Y);
          });
#pragma unroll
          for (int k = 0; k < K; ++k) {
            T t = T(0);
            static_for<0, D1>([&](auto m1c) {
              constexpr int M1I = decltype(m1c)::value;
              if constexpr (a_nz(L1, L2, L3, M1I - L1, M3I - L3)) t = fma(a[M1I], xk[k * D1 + M1I], t);
            });
            acc[k][OO + M3I] = fma(wk[k], t, acc[k][OO + M3I]);
          }
        });
      }
    });
  }

  // out[row, path blocks of the group, channels 4cb..] += pscale_p * acc (a later row segment)
  __device__ __forceinline__ void store_add(T* __restrict__ orow, int C, int cb, const double* pscale) {
    static_for<GR::PB, GR::PE>([&](auto pc) {
      constexpr int P = decltype(pc)::value;
      using PC = PathC<CF, P>;
      constexpr int D3 = PC::D3, OO = PC::OUT - GR::OB;
      const T s = T(pscale[P]);
      T* p = orow + size_t(C) * PC::OUT + size_t(4 * cb) * D3;
      T t[K * D3];
      ld16_l2(t, p);
#pragma unroll
      for (int k = 0; k < K; ++k)
#pragma unroll
        for (int m = 0; m < D3; ++m) t[k * D3 + m] += s * acc[k][OO + m];
      st16(p, t);
    });
  }

  // out[row, path blocks of the group, channels 4cb..] = pscale_p * acc
  __device__ __forceinline__ void store(T* __restrict__ orow, int C, int cb, const double* pscale) {
    static_for<GR::PB, GR::PE>([&](auto pc) {
      constexpr int P = decltype(pc)::value;
      using PC = PathC<CF, P>;
      constexpr int D3 = PC::D3, OO = PC::OUT - GR::OB;
      const T s = T(pscale[P]);
      T t[K * D3];
#pragma unroll
      for (int k = 0; k < K; ++k)
#pragma unroll
        for (int m = 0; m < D3; ++m) t[k * D3 + m] = s * acc[k][OO + m];
      st16(orow + size_t(C) * PC::OUT + size_t(4 * cb) * D3, t);
    });
  }

  // sum over the slices of a warp (lanes that differ in the bits from CB up), fixed butterfly
  __device__ __forceinline__ void reduce_slices(int CB) {
    for (int off = CB; off < 32; off <<= 1)
#pragma unroll
      for (int k = 0; k < K; ++k)
#pragma unroll
        for (int o = 0; o < GR::NOG; ++o) acc[k][o] += __shfl_xor_sync(0xffffffffu, acc[k][o], off);
  }
};

// The forward accumulator of the float convolution with paired FP32 arithmetic: acc[q][o] holds
// channels (4cb + 2q, 4cb + 2q + 1) of output o in one register pair, so each fma.rn.f32x2 does
// the work of two FFMA (the kernels are bound by FP32 issue).  The staged x slices are
// component-major inside each degree block ([m][u], see transpose_blocks_kernel), so one 16-byte
// shared load gives two channel pairs of one component.  An entry A[m1, m3] is built once per
// thread with scalar FMAs (constant-bank coefficients) and duplicated into a pair; keeping the
// harmonics scalar saves the registers a duplicated copy would hold (measured faster).  The loop
// runs over m1 outside and m3 inside, so the accumulators of one row are independent; per channel
// every operation and its order are those of FwdAcc, so the results are bitwise the same.
template <class CF, int GI>
struct FwdAcc2 {
  using GR = Grp<CF, GI>;
  float2 acc[2][GR::NOG];

  __device__ __forceinline__ void zero() {
#pragma unroll
    for (int q = 0; q < 2; ++q)
#pragma unroll
      for (int o = 0; o < GR::NOG; ++o) acc[q][o] = make_float2(0.f, 0.f);
  }

  // sw: the group's weight slice ([path][u]); sx: x blocks L1A..L1B, each [m][u]
  __device__ __forceinline__ void edge_smem(const float* sw, const float* sx, const float (&Y)[CF::NY], int C,
                                            int cb) {
    static_for<GR::PB, GR::PE>([&](auto pc) {
      constexpr int P = decltype(pc)::value;
      using PC = PathC<CF, P>;
      constexpr int L1 = PC::L1, L2 = PC::L2, L3 = PC::L3, D1 = PC::D1, D3 = PC::D3;
      constexpr int OO = PC::OUT - GR::OB;
      const float4 w4 = *reinterpret_cast<const float4*>(sw + size_t(P - GR::PB) * C + 4 * cb);
      const float2 w2[2] = {lo2(w4), hi2(w4)};
      float2 x2[2][D1];
#pragma unroll
      for (int m1 = 0; m1 < D1; ++m1) {
        const float4 v = *reinterpret_cast<const float4*>(sx + size_t(C) * (L1 * L1 - GR::XB + m1) + 4 * cb);
        x2[0][m1] = lo2(v);
        x2[1][m1] = hi2(v);
      }
      if constexpr (D1 < D3) {
        static_for<0, D1>([&](auto m1c) {
          constexpr int M1I = decltype(m1c)::value;
          const float2 xs[2] = {__fmul2_rn(w2[0], x2[0][M1I]), __fmul2_rn(w2[1], x2[1][M1I])};
          static_for<0, D3>([&](auto m3c) {
            constexpr int M3I = decltype(m3c)::value;
            if constexpr (a_nz(L1, L2, L3, M1I - L1, M3I - L3)) {
              const float a1 = a_entry<float, L1, L2, L3, M1I - L1, M3I - L3>(Y);
              const float2 a = make_float2(a1, a1);
              acc[0][OO + M3I] = __ffma2_rn(a, xs[0], acc[0][OO + M3I]);
              acc[1][OO + M3I] = __ffma2_rn(a, xs[1], acc[1][OO + M3I]);
            }
          });
        });
      } else {
        float2 t[2][D3];
#pragma unroll
        for (int q = 0; q < 2; ++q)
#pragma unroll
          for (int m3 = 0; m3 < D3; ++m3) t[q][m3] = make_float2(0.f, 0.f);
        static_for<0, D1>([&](auto m1c) {
          constexpr int M1I = decltype(m1c)::value;
          static_for<0, D3>([&](auto m3c) {
            constexpr int M3I = decltype(m3c)::value;
            if constexpr (a_nz(L1, L2, L3, M1I - L1, M3I - L3)) {
              const float a1 = a_entry<float, L1, L2, L3, M1I - L1, M3I - L3>(Y);
              const float2 a = make_float2(a1, a1);
              t[0][M3I] = __ffma2_rn(a, x2[0][M1I], t[0][M3I]);
              t[1][M3I] = __ffma2_rn(a, x2[1][M1I], t[1][M3I]);
            }
          });
        });
#pragma unroll
        for (int q = 0; q < 2; ++q)
#pragma unroll
          for (int m3 = 0; m3 < D3; ++m3) acc[q][OO + m3] = __ffma2_rn(w2[q], t[q][m3], acc[q][OO + m3]);
      }
    });
  }

  __device__ __forceinline__ float ch(int k, int o) const { return (k & 1) ? acc[k >> 1][o].y : acc[k >> 1][o].x; }

  __device__ __forceinline__ void store_add(float* __restrict__ orow, int C, int cb, const double* pscale) {
    static_for<GR::PB, GR::PE>([&](auto pc) {
      constexpr int P = decltype(pc)::value;
      using PC = PathC<CF, P>;
      constexpr int D3 = PC::D3, OO = PC::OUT - GR::OB;
      const float s = float(pscale[P]);
      float* p = orow + size_t(C) * PC::OUT + size_t(4 * cb) * D3;
      float t[K * D3];
      ld16_l2(t, p);
#pragma unroll
      for (int k = 0; k < K; ++k)
#pragma unroll
        for (int m = 0; m < D3; ++m) t[k * D3 + m] += s * ch(k, OO + m);
      st16(p, t);
    });
  }

  __device__ __forceinline__ void store(float* __restrict__ orow, int C, int cb, const double* pscale) {
    static_for<GR::PB, GR::PE>([&](auto pc) {
      constexpr int P = decltype(pc)::value;
      using PC = PathC<CF, P>;
      constexpr int D3 = PC::D3, OO = PC::OUT - GR::OB;
      const float s = float(pscale[P]);
      float t[K * D3];
#pragma unroll
      for (int k = 0; k < K; ++k)
#pragma unroll
        for (int m = 0; m < D3; ++m) t[k * D3 + m] = s * ch(k, OO + m);
      st16(orow + size_t(C) * PC::OUT + size_t(4 * cb) * D3, t);
    });
  }

  __device__ __forceinline__ void reduce_slices(int CB) {
    for (int off = CB; off < 32; off <<= 1)
#pragma unroll
      for (int q = 0; q < 2; ++q)
#pragma unroll
        for (int o = 0; o < GR::NOG; ++o) {
          acc[q][o].x += __shfl_xor_sync(0xffffffffu, acc[q][o].x, off);
          acc[q][o].y += __shfl_xor_sync(0xffffffffu, acc[q][o].y, off);
        }
  }
};

// Paired arithmetic is used by the float convolution (its x and grad_out are transposed to
// component-major blocks first); double precision and the tensor product keep FwdAcc.
template <class CF, bool CONV>
constexpr bool paired() {
  return CONV && std::is_same<typename CF::T, float>::value;
}

// ------------------------------------------------------------ async copy machinery ---
// One thread per CTA streams the weight and x slices of upcoming edges into a ring of shared
// memory stages with cp.async.bulk (1-D TMA, no multicast); completion is tracked by one
// mbarrier per stage (transaction bytes).  Every wait is bounded: after the launch's wait_ns
// nanoseconds of the global timer (one second unless a test sets it lower) the kernel records
// E3_ERR_TIMEOUT and stops issuing work.
constexpr int FWD_WIN = 64;  // in-edges whose sender ids and harmonics are staged at once

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_fence_init() { asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory"); }
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)), "r"(bytes) : "memory");
}
__device__ __forceinline__ bool mbar_test_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(smem_addr(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
// try_wait with a suspend-time hint: the warp is parked until the phase completes or about
// 20 microseconds pass, instead of polling.
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(smem_addr(bar)), "r"(parity), "r"(20000u)
      : "memory");
  return ok != 0;
}
__device__ __forceinline__ unsigned long long global_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                   smem_addr(dst)),
               "l"(src), "r"(bytes), "r"(smem_addr(bar))
               : "memory");
}
// Bring [p, p + bytes) into L2 ahead of its bulk copy (16-byte aligned, multiple of 16).
__device__ __forceinline__ void prefetch_l2(const void* p, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}

// bounded wait; false after wait_ns (the error is recorded).  The common case -- the copy
// landed while the previous stage was being consumed -- costs one test.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, int* status, unsigned long long wait_ns) {
  if (mbar_test_wait(bar, parity)) return true;
  const unsigned long long t0 = global_ns();
  do {
    for (int i = 0; i < 16; ++i)
      if (mbar_try_wait(bar, parity)) return true;
  } while (global_ns() - t0 < wait_ns);
  record_error(status, E3_ERR_TIMEOUT);
  return false;
}

// Bounded wait (one thread) until *flag >= v (acquire); false after wait_ns nanoseconds of the
// global timer, with E3_ERR_TIMEOUT recorded.
__device__ __forceinline__ bool wait_flag_geq(const int* flag, int v, int* status, unsigned long long wait_ns) {
  const unsigned long long t0 = global_ns();
  int cur;
  while (true) {
    asm volatile("ld.acquire.gpu.global.s32 %0, [%1];" : "=r"(cur) : "l"(flag) : "memory");
    if (cur >= v) return true;
    if (global_ns() - t0 > wait_ns) {
      record_error(status, E3_ERR_TIMEOUT);
      return false;
    }
    __nanosleep(64);
  }
}

template <typename T, int N>
__device__ __forceinline__ void lds16(T (&r)[N], const T* p) {
  if constexpr (std::is_same<T, float>::value) {
#pragma unroll
    for (int i = 0; i < N / 4; ++i) {
      const float4 v = reinterpret_cast<const float4*>(p)[i];
      r[4 * i] = v.x;
      r[4 * i + 1] = v.y;
      r[4 * i + 2] = v.z;
      r[4 * i + 3] = v.w;
    }
  } else {
#pragma unroll
    for (int i = 0; i < N / 2; ++i) {
      const double2 v = reinterpret_cast<const double2*>(p)[i];
      r[2 * i] = v.x;
      r[2 * i + 1] = v.y;
    }
  }
}

// Byte sizes of one edge's slices for group GI: weights of the group's paths (all channels)
// and x blocks l1 in [L1A, L1B] (all channels); both are contiguous in global memory.
template <class CF, int GI>
struct FwdSlice {
  using T = typename CF::T;
  using GR = Grp<CF, GI>;
  static __host__ __device__ constexpr uint32_t wbytes(int C) { return uint32_t(GR::NP) * C * sizeof(T); }
  static __host__ __device__ constexpr uint32_t xbytes(int C) { return uint32_t(GR::NXG) * C * sizeof(T); }
};

template <class CF, int I = 0>
__host__ __device__ constexpr uint32_t max_slice_bytes(int C) {
  if constexpr (I >= CF::G) {
    return 0;
  } else {
    const uint32_t a = FwdSlice<CF, I>::wbytes(C) + FwdSlice<CF, I>::xbytes(C);
    const uint32_t b = max_slice_bytes<CF, I + 1>(C);
    return a > b ? a : b;
  }
}

// Shared memory of the forward CTA.
template <class CF>
struct FwdSmem {
  using T = typename CF::T;
  static constexpr int NYP = (CF::NY + 3) & ~3;  // harmonics row padded to 16 bytes (float)
  static __host__ __device__ size_t ysh_off() { return 0; }
  static __host__ __device__ size_t src_off() { return sizeof(T) * size_t(FWD_WIN) * NYP; }
  static __host__ __device__ size_t bar_off() { return src_off() + sizeof(int32_t) * FWD_WIN; }
  static __host__ __device__ size_t flag_off(int S) { return bar_off() + 8 * size_t(S); }
  static __host__ __device__ size_t stage_off(int S) { return (flag_off(S) + 16 + 127) & ~size_t(127); }
  static __host__ __device__ size_t stage_bytes(int C, int NS) { return size_t(NS) * max_slice_bytes<CF>(C); }
  static __host__ __device__ size_t total(int C, int NS, int S) { return stage_off(S) + size_t(S) * stage_bytes(C, NS); }
};

// Stage sender ids (checked) and harmonics of edges [e0 + ws, e0 + ws + cnt) into shared
// memory.  Shared by every path group, so it is kept out of line (one copy of the code).
template <class CF, bool CONV>
__device__ __noinline__ void fwd_stage_window(const KFwd& a, int64_t e0, int64_t ws, int cnt,
                                              typename CF::T* ysh, int32_t* src_s) {
  using T = typename CF::T;
  constexpr int NYP = FwdSmem<CF>::NYP;
  const T* __restrict__ y = static_cast<const T*>(a.y);
  const T* __restrict__ vec = static_cast<const T*>(a.vec);
  for (int i = threadIdx.x; i < cnt; i += blockDim.x) {
    const int64_t e = e0 + ws + i;
    if constexpr (CONV) {
      const int32_t s = __ldg(a.src + e);
      const bool ok = uint32_t(s) < uint32_t(a.n_rows);
      if (!ok) record_error(a.status, E3_ERR_INDEX);
      src_s[i] = ok ? s : -1;
    }
    T Yl[CF::NY];
    load_y<CF>(Yl, y, vec, a.sh_norm, e);
#pragma unroll
    for (int m = 0; m < CF::NY; ++m) ysh[i * NYP + m] = Yl[m];
  }
}

template <class CF, int GI, bool CONV, int CC>
__device__ __forceinline__ void fwd_group(const KFwd& a, int64_t unit, int64_t e0_in, int64_t e1_in, int64_t seg,
                                          int64_t nseg, unsigned char* smem) {
  using T = typename CF::T;
  using GR = Grp<CF, GI>;
  using SM = FwdSmem<CF>;
  constexpr int NYP = SM::NYP;
  const int C = CC > 0 ? CC : a.C;  // compile-time for the specialised multiplicities
  const int CB = C >> 2;
  const int tid = threadIdx.x;
  const int cb = CB >= 32 ? tid : tid % CB;
  const int slice = CB >= 32 ? 0 : tid / CB;
  const int NS = CB >= 32 ? 1 : 32 / CB;
  const int S = a.stages;
  const T* __restrict__ x = static_cast<const T*>(a.x);
  const T* __restrict__ w = static_cast<const T*>(a.w);
  T* __restrict__ out = static_cast<T*>(a.out);
  const size_t xrow = size_t(CF::NX) * C, orow = size_t(CF::NO) * C;
  const uint32_t WB = FwdSlice<CF, GI>::wbytes(C), XB = FwdSlice<CF, GI>::xbytes(C);
  const uint32_t SLOT = WB + XB;
  const size_t STAGE = SM::stage_bytes(C, NS);

  T* ysh = reinterpret_cast<T*>(smem + SM::ysh_off());
  int32_t* src_s = reinterpret_cast<int32_t*>(smem + SM::src_off());
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + SM::bar_off());
  volatile int* s_abort = reinterpret_cast<volatile int*>(smem + SM::flag_off(S));
  unsigned char* stages = smem + SM::stage_off(S);

  // edges handled by this CTA: segment `seg` of receiver `unit`'s in-edges (convolution; the
  // topology build checked the row pointers)
  int64_t e0, e1;
  if constexpr (CONV) {
    e0 = e0_in;
    e1 = e1_in;
  } else {
    const int64_t per = (a.n_rows + a.n_chunks - 1) / a.n_chunks;
    e0 = unit * per;
    e1 = e0 + per < a.n_rows ? e0 + per : a.n_rows;
    if (e0 > e1) e0 = e1;
  }
  if (tid == 0) {
    for (int i = 0; i < S; ++i) mbar_init(&bars[i], 1);
    *s_abort = 0;
    mbar_fence_init();
  }
  __syncthreads();

  typename std::conditional<paired<CF, CONV>(), FwdAcc2<CF, GI>, FwdAcc<CF, GI>>::type f;
  f.zero();
  T Y[CF::NY];
  // ring state: identical in every thread, advanced uniformly
  int prod_slot = 0, cons_slot = 0;
  uint32_t cons_phase = 0, issued = 0, consumed = 0;
  bool alive = true;
  const int64_t deg = e1 - e0;

  for (int64_t ws = 0; ws < deg && alive; ws += FWD_WIN) {
    const int cnt = int(deg - ws < FWD_WIN ? deg - ws : FWD_WIN);
    fwd_stage_window<CF, CONV>(a, e0, ws, cnt, ysh, src_s);
    __syncthreads();
    const int steps = (cnt + NS - 1) / NS;
    // producer: thread 0 posts the expected bytes, then thread j (< edges in the step) copies
    // the weights and the x slice of the step's j-th edge.  An edge whose sender id is out of
    // range copies row 0 instead (the edge is skipped by the consumer), so the byte count of
    // a stage depends only on its number of edges.
    auto issue = [&](int st) {
      uint64_t* bar = &bars[prod_slot];
      unsigned char* dst = stages + size_t(prod_slot) * STAGE;
      const int nv = min(NS, cnt - st * NS);
      if (tid == 0) mbar_arrive_expect_tx(bar, uint32_t(nv) * SLOT);
      __syncwarp();
      if (tid < nv) {
        const int r = st * NS + tid;
        const int64_t e = e0 + ws + r;
        int64_t row = e;
        if constexpr (CONV) row = max(src_s[r], 0);
        unsigned char* d = dst + size_t(tid) * SLOT;
        bulk_load(d, w + e * a.w_stride + size_t(GR::PB) * C, WB, bar);
        bulk_load(d + WB, x + size_t(row) * xrow + size_t(GR::XB) * C, XB, bar);
      }
      prod_slot = prod_slot + 1 == S ? 0 : prod_slot + 1;
      ++issued;
    };
    for (int st = 0; st < S && st < steps; ++st) issue(st);

    for (int st = 0; st < steps; ++st) {
      const int slot = cons_slot;
      const bool ok = mbar_wait(&bars[slot], cons_phase, a.status, a.wait_ns);
      if (!ok) *s_abort = 1;
      cons_slot = cons_slot + 1 == S ? 0 : cons_slot + 1;
      if (cons_slot == 0) cons_phase ^= 1u;
      ++consumed;
      const int r = st * NS + slice;
      const bool mine = ok && r < cnt && (!CONV || src_s[r] >= 0);
      if (mine) {
        const T* sl = reinterpret_cast<const T*>(stages + size_t(slot) * STAGE + size_t(slice) * SLOT);
        const T* xs = sl + WB / sizeof(T);
        {
          T yp[NYP];
          lds16(yp, ysh + r * NYP);
#pragma unroll
          for (int m = 0; m < CF::NY; ++m) Y[m] = yp[m];
        }
        if constexpr (!CONV) f.zero();
        f.edge_smem(sl, xs, Y, C, cb);
        if constexpr (!CONV) f.store(out + size_t(e0 + ws + r) * orow, C, cb, a.pscale);
      }
      __syncthreads();  // every thread is done with this stage (and sees an abort)
      if (*s_abort) {
        alive = false;
        break;
      }
      if (st + S < steps) issue(st + S);
    }
    __syncthreads();  // window staging buffers are reused by the next window
  }
  // a row split into segments: its segments add their partial sums in segment order
  int* seg_flag = (CONV && nseg > 1) ? a.flags + unit * CF::G + GI : nullptr;
  if (!alive) {
    // a wait gave up: let the copies in flight land (bounded) before the CTA exits
    if (tid == 0)
      for (uint32_t q = consumed - 1; q < issued; ++q) mbar_wait(&bars[q % S], (q / S) & 1u, a.status, a.wait_ns);
    __syncthreads();
    if (seg_flag != nullptr && tid == 0)  // later segments must not wait for this one in vain
      asm volatile("st.release.gpu.global.s32 [%0], %1;" ::"l"(seg_flag), "r"(int(seg + 1)) : "memory");
    return;
  }
  if constexpr (CONV) {
    if (CB < 32) f.reduce_slices(CB);
    if (seg_flag == nullptr) {
      if (slice == 0) f.store(out + size_t(unit) * orow, C, cb, a.pscale);
    } else {
      // wait (bounded) until the earlier segments of this row and group have added theirs; the
      // segment that waits drew a later ticket than those it waits for, so they are resident or
      // finished
      if (tid == 0 && seg > 0) wait_flag_geq(seg_flag, int(seg), a.status, a.wait_ns);
      __syncthreads();
      if (slice == 0) {
        if (seg == 0)
          f.store(out + size_t(unit) * orow, C, cb, a.pscale);
        else
          f.store_add(out + size_t(unit) * orow, C, cb, a.pscale);
      }
      __threadfence();
      __syncthreads();
      if (tid == 0) asm volatile("st.release.gpu.global.s32 [%0], %1;" ::"l"(seg_flag), "r"(int(seg + 1)) : "memory");
    }
  }
}

// Register budget of the forward: path sets with output degree <= 2 fit in 128 registers per
// thread (16 resident warps per SM, CTAs of up to 256 threads, multiplicity <= 1024); the l <= 3
// set gets 168 (12 warps per SM, CTAs of up to 64 threads, multiplicity <= 256): measured on the
// large convolution, 7.9 ms against 9.0 ms with the compiler's choice of 252.
template <class CF>
constexpr int fwd_max_threads() {
  return CF::LO <= 2 ? 256 : 64;
}
template <class CF>
constexpr int fwd_min_blocks() {
  return CF::LO <= 2 ? 2 : 6;
}

template <class CF, bool CONV, int CC>
__global__ void __launch_bounds__(fwd_max_threads<CF>(), fwd_min_blocks<CF>()) fwd_kernel(const __grid_constant__ KFwd a) {
  extern __shared__ __align__(128) unsigned char smem_raw[];
  // group-major order, so the CTAs resident on an SM at any time mostly run the same path group
  // and share its (large, fully unrolled) code
  if constexpr (CONV) {
    // a ticket per CTA (tickets follow the order CTAs start in): group, then row segment; a row's
    // later segments wait for its earlier ones, which hold earlier tickets
    __shared__ int s_ticket;
    if (threadIdx.x == 0) s_ticket = atomicAdd(a.ticket, 1) + a.first_ticket;
    __syncthreads();
    const int t = s_ticket;
    const int g = int(t / a.units_max);
    const int64_t u = t % a.units_max;
    const int4 inf = a.uinfo[u];  // {row, first edge, end edge, segment}; in bounds for u < units_max
    const int64_t nseg = a.unseg[u];
    if (u >= *a.n_units) return;  // the grid covers an upper bound of the units
    dispatch<CF::G>(g, [&](auto gi) {
      fwd_group<CF, decltype(gi)::value, CONV, CC>(a, inf.x, inf.y, inf.z, inf.w, nseg, smem_raw);
    });
  } else {
    const int64_t units = int64_t(gridDim.x) / CF::G;
    const int g = int(blockIdx.x / units);
    const int64_t unit = blockIdx.x % units;
    dispatch<CF::G>(g, [&](auto gi) { fwd_group<CF, decltype(gi)::value, CONV, CC>(a, unit, 0, 0, 0, 1, smem_raw); });
  }
}

// ========================================================================= backward ===
struct KBwd {
  const int32_t* row_ptr_src;
  const int32_t* perm_src;
  const int32_t* dst;
  const void* x;
  const void* y;
  const void* vec;
  const void* w;
  const void* grad_out;
  void* grad_x;
  void* grad_y;
  void* grad_w;
  int64_t n_nodes, n_edges;
  int64_t units;        // senders (convolution) or sample ranges (tensor product)
  int C, sh_norm, n_chunks, stages;
  int* status;
  int* ticket;          // CTA ticket counter (zero at launch)
  int* done;            // per unit: path groups finished (zero at launch)
  int* chain;           // convolution, per sender split into segments: (group, segment) pairs that
                        // have added their grad_x, in group-major order (zero at launch)
  const int4* uinfo;    // convolution: sender units of the topology buffer
  const int32_t* unseg;
  const int32_t* n_units;
  unsigned long long wait_ns;  // limit of every bounded wait
  int first_ticket;            // first ticket drawn (0; a test withholds tickets by raising it)
  double scale;
  double alpha[MAXP];
  float alpha_f[MAXP];    // the same path weights rounded once, for the float kernels
  float2 alpha_f2[MAXP];  // {alpha_f, alpha_f}: operands of the paired float arithmetic
  float2 salpha_f2[MAXP]; // {float(scale) * alpha_f, same}: the grad_w factor, rounded as the scalar code rounds it
};

// Which path groups touch x block l1 / harmonics block l2 (the first toucher stores, later
// groups accumulate; blocks no group touches are zero-filled by group 0).
template <class CF>
__host__ __device__ constexpr int first_group_l1(int l) {
  for (int g = 0; g < CF::G; ++g)
    for (int p = CF::PT.gbegin[g]; p < CF::PT.gbegin[g + 1]; ++p)
      if (CF::PT.l1[p] == l) return g;
  return -1;
}
template <class CF>
__host__ __device__ constexpr int first_group_l2(int l) {
  for (int g = 0; g < CF::G; ++g)
    for (int p = CF::PT.gbegin[g]; p < CF::PT.gbegin[g + 1]; ++p)
      if (CF::PT.l2[p] == l) return g;
  return -1;
}
template <class CF, int GI>
__host__ __device__ constexpr bool group_has_l2(int l) {
  for (int p = CF::PT.gbegin[GI]; p < CF::PT.gbegin[GI + 1]; ++p)
    if (CF::PT.l2[p] == l) return true;
  return false;
}

constexpr int BWD_WIN = 64;  // out-edges whose ids and harmonics are staged at once (a typical sender in one window)

// A group that adds to grad_y blocks an earlier group stored stages the edge's grad_y row with
// its other slices, so the read-modify-write does not wait on a global load (rows whose byte
// size is not a multiple of 16 cannot be bulk-copied and are read directly).
template <class CF, int GI>
__host__ __device__ constexpr bool bwd_stage_gy() {
  bool acc = false;
  for (int l = 0; l <= CF::LY; ++l) acc = acc || (group_has_l2<CF, GI>(l) && first_group_l2<CF>(l) != GI);
  return acc && (CF::NY * sizeof(typename CF::T)) % 16 == 0;
}

// Byte sizes of one edge's staged slices in the backward of group GI: weights of the group's
// paths, grad_out of the receiver for the group's outputs, (tensor product only) the x slice,
// and the grad_y row when bwd_stage_gy() holds and grad_y is requested.
template <class CF, int GI>
struct BwdSlice {
  using T = typename CF::T;
  using GR = Grp<CF, GI>;
  static __host__ __device__ constexpr uint32_t wbytes(int C) { return uint32_t(GR::NP) * C * sizeof(T); }
  static __host__ __device__ constexpr uint32_t gbytes(int C) { return uint32_t(GR::NOG) * C * sizeof(T); }
  static __host__ __device__ constexpr uint32_t xbytes(int C, bool conv) {
    return conv ? 0u : uint32_t(GR::NXG) * C * sizeof(T);
  }
  static __host__ __device__ constexpr uint32_t ybytes(bool dy) {
    return dy && bwd_stage_gy<CF, GI>() ? uint32_t(CF::NY * sizeof(T)) : 0u;
  }
  static __host__ __device__ constexpr uint32_t slot(int C, bool conv, bool dy) {
    return wbytes(C) + gbytes(C) + xbytes(C, conv) + ybytes(dy);
  }
};

template <class CF, int GI>
struct BwdSmem {
  using T = typename CF::T;
  static constexpr int NYP = (CF::NY + 3) & ~3;
  static __host__ __device__ size_t ysh_off() { return 0; }
  static __host__ __device__ size_t eid_off() { return sizeof(T) * size_t(BWD_WIN) * NYP; }
  static __host__ __device__ size_t did_off() { return eid_off() + sizeof(int32_t) * BWD_WIN; }
  static __host__ __device__ size_t bar_off() { return did_off() + sizeof(int32_t) * BWD_WIN; }
  static __host__ __device__ size_t flag_off(int S) { return bar_off() + 8 * size_t(S); }
  static __host__ __device__ size_t stage_off(int S) { return (flag_off(S) + 16 + 127) & ~size_t(127); }
  static __host__ __device__ size_t stage_bytes(int C, int NS, bool conv, bool dy) {
    return size_t(NS) * BwdSlice<CF, GI>::slot(C, conv, dy);
  }
  static __host__ __device__ size_t total(int C, int NS, int S, bool conv, bool dy) {
    return stage_off(S) + size_t(S) * stage_bytes(C, NS, conv, dy);
  }
};

// Per-edge backward of one path group with grad_out read from shared memory (sg: the group's
// outputs, channels in mul_ir order).  Accumulates alpha_p w t into dx, returns this thread's
// unreduced grad_y contribution in dY and writes grad_w (scaled) when gw != nullptr.  FL = 1:
// grad_w and grad_y are both requested, known at compile time, so that no per-path test
// separates one path's work from the next in the schedule.
template <class CF, int GI, int FL>
__device__ __forceinline__ void bwd_edge(const typename CF::T (&xr)[K][Grp<CF, GI>::NXG],
                                         const typename CF::T* sw,
                                         const typename CF::T (&Y)[CF::NY], const typename CF::T* sg,
                                         typename CF::T (&dx)[K][Grp<CF, GI>::NXG], typename CF::T (&dY)[CF::NY],
                                         bool want_dy, typename CF::T* __restrict__ gw, int C, int cb,
                                         const double* alpha, const float* alpha_f, typename CF::T scale) {
  using T = typename CF::T;
  using GR = Grp<CF, GI>;
#pragma unroll
  for (int i = 0; i < CF::NY; ++i) dY[i] = T(0);
  static_for<GR::PB, GR::PE>([&](auto pc) {
    constexpr int P = decltype(pc)::value;
    using PC = PathC<CF, P>;
    constexpr int L1 = PC::L1, L2 = PC::L2, L3 = PC::L3, D1 = PC::D1, D3 = PC::D3;
    constexpr int XO = L1 * L1 - GR::XB, PW = P - GR::PB;
    T wk[K];
    lds16(wk, sw + size_t(PW) * C + 4 * cb);
    T g[K][D3];
    {
      T t4[K * D3];
      lds16(t4, sg + size_t(C) * (PC::OUT - GR::OB) + size_t(4 * cb) * D3);
#pragma unroll
      for (int k = 0; k < K; ++k)
#pragma unroll
        for (int m = 0; m < D3; ++m) g[k][m] = t4[k * D3 + m];
    }
    const T al = std::is_same<T, float>::value ? T(alpha_f[P]) : T(alpha[P]);
    T wa[K];
#pragma unroll
    for (int k = 0; k < K; ++k) wa[k] = al * wk[k];
    // t[k][m1] = sum_m3 A[m1, m3] g[k][m3]
    T t[K][D1];
#pragma unroll
    for (int k = 0; k < K; ++k)
#pragma unroll
      for (int m1 = 0; m1 < D1; ++m1) t[k][m1] = T(0);
    static_for<0, D3>([&](auto m3c) {
      constexpr int M3I = decltype(m3c)::value;
      T a[D1];
      static_for<0, D1>([&](auto m1c) {
        constexpr int M1I = decltype(m1c)::value;
        if constexpr (a_nz(L1, L2, L3, M1I - L1, M3I - L3)) a[M1I] = a_entry<T, L1, L2, L3, M1I - L1, M3I - L3>(Y);
      });
#pragma unroll
      for (int k = 0; k < K; ++k)
        static_for<0, D1>([&](auto m1c) {
          constexpr int M1I = decltype(m1c)::value;
          if constexpr (a_nz(L1, L2, L3, M1I - L1, M3I - L3)) t[k][M1I] = fma(a[M1I], g[k][M3I], t[k][M1I]);
        });
    });
    if (FL == 1 || gw != nullptr) {  // grad_w[e, p, u] = scale alpha_p sum_m1 x[u, m1] t[u, m1]
      T o[K];
#pragma unroll
      for (int k = 0; k < K; ++k) {
        T s = T(0);
#pragma unroll
        for (int m1 = 0; m1 < D1; ++m1) s = fma(xr[k][XO + m1], t[k][m1], s);
        o[k] = scale * al * s;
      }
      st16(gw + size_t(P) * C + 4 * cb, o);
    }
#pragma unroll
    for (int k = 0; k < K; ++k)  // grad_x += alpha_p w t
#pragma unroll
      for (int m1 = 0; m1 < D1; ++m1) dx[k][XO + m1] = fma(wa[k], t[k][m1], dx[k][XO + m1]);
    if (FL == 1 || want_dy) {  // grad_y[m2] += sum_{m1,m3} C[m1,m2,m3] sum_k alpha_p w_k x_k[m1] g_k[m3]
      // the weight scales the shorter of the x and grad_out blocks
      constexpr bool SX = D1 <= D3;
      T xw[K][SX ? D1 : 1], gw_[K][SX ? 1 : D3];
#pragma unroll
      for (int k = 0; k < K; ++k) {
        if constexpr (SX) {
#pragma unroll
          for (int m1 = 0; m1 < D1; ++m1) xw[k][m1] = wa[k] * xr[k][XO + m1];
        } else {
#pragma unroll
          for (int m3 = 0; m3 < D3; ++m3) gw_[k][m3] = wa[k] * g[k][m3];
        }
      }
      static_for<0, D1>([&](auto m1c) {
        constexpr int M1I = decltype(m1c)::value;
        static_for<0, D3>([&](auto m3c) {
          constexpr int M3I = decltype(m3c)::value;
          if constexpr (a_nz(L1, L2, L3, M1I - L1, M3I - L3)) {
            T z = T(0);
#pragma unroll
            for (int k = 0; k < K; ++k) {
              if constexpr (SX)
                z = fma(xw[k][M1I], g[k][M3I], z);
              else
                z = fma(xr[k][XO + M1I], gw_[k][M3I], z);
            }
            static_for<-L2, L2 + 1>([&](auto m2c) {
              constexpr int M2 = decltype(m2c)::value;
              if constexpr (cg_nz(L1, L2, L3, M1I - L1, M2, M3I - L3)) {
                constexpr int I = cg_index(L1, L2, L3, M1I - L1, M2, M3I - L3);
                dY[L2 * L2 + L2 + M2] = fma(CGT<T>::template get<I>(), z, dY[L2 * L2 + L2 + M2]);
              }
            });
          }
        });
      });
    }
  });
}

// Per-edge backward of group GI for the float convolution with paired FP32 arithmetic (see
// FwdAcc2): xr2 and dx2 hold channels (4cb + 2q, 4cb + 2q + 1) of one x component in a register
// pair, and the staged grad_out slice sg is component-major inside each path block ([m3][u]).
// Per channel the operations and their order are those of bwd_edge, except the grad_y product,
// whose sum over the thread's four channels is formed as two pair sums added at the end.
template <class CF, int GI, int FL>
__device__ __forceinline__ void bwd_edge2(const float2 (&xr2)[2][Grp<CF, GI>::NXG], const float* sw,
                                          const float (&Y)[CF::NY], const float* sg,
                                          float2 (&dx2)[2][Grp<CF, GI>::NXG], float (&dY)[CF::NY], bool want_dy,
                                          float* __restrict__ gw, int C, int cb, const float2* alpha2,
                                          const float2* salpha2) {
  using GR = Grp<CF, GI>;
#pragma unroll
  for (int i = 0; i < CF::NY; ++i) dY[i] = 0.f;
  static_for<GR::PB, GR::PE>([&](auto pc) {
    constexpr int P = decltype(pc)::value;
    using PC = PathC<CF, P>;
    constexpr int L1 = PC::L1, L2 = PC::L2, L3 = PC::L3, D1 = PC::D1, D3 = PC::D3;
    constexpr int XO = L1 * L1 - GR::XB, PW = P - GR::PB;
    const float4 w4 = *reinterpret_cast<const float4*>(sw + size_t(PW) * C + 4 * cb);
    float2 g2[2][D3];
#pragma unroll
    for (int m3 = 0; m3 < D3; ++m3) {
      const float4 v = *reinterpret_cast<const float4*>(sg + size_t(C) * (PC::OUT - GR::OB + m3) + 4 * cb);
      g2[0][m3] = lo2(v);
      g2[1][m3] = hi2(v);
    }
    const float2 wa2[2] = {__fmul2_rn(alpha2[P], lo2(w4)), __fmul2_rn(alpha2[P], hi2(w4))};
    // t[q][m1] = sum_m3 A[m1, m3] g[q][m3]
    float2 t2[2][D1];
#pragma unroll
    for (int q = 0; q < 2; ++q)
#pragma unroll
      for (int m1 = 0; m1 < D1; ++m1) t2[q][m1] = make_float2(0.f, 0.f);
    static_for<0, D3>([&](auto m3c) {
      constexpr int M3I = decltype(m3c)::value;
      float2 a[D1];
      static_for<0, D1>([&](auto m1c) {
        constexpr int M1I = decltype(m1c)::value;
        if constexpr (a_nz(L1, L2, L3, M1I - L1, M3I - L3)) {
          const float a1 = a_entry<float, L1, L2, L3, M1I - L1, M3I - L3>(Y);
          a[M1I] = make_float2(a1, a1);
        }
      });
#pragma unroll
      for (int q = 0; q < 2; ++q)
        static_for<0, D1>([&](auto m1c) {
          constexpr int M1I = decltype(m1c)::value;
          if constexpr (a_nz(L1, L2, L3, M1I - L1, M3I - L3)) t2[q][M1I] = __ffma2_rn(a[M1I], g2[q][M3I], t2[q][M1I]);
        });
    });
    if (FL == 1 || gw != nullptr) {  // grad_w[e, p, u] = scale alpha_p sum_m1 x[u, m1] t[u, m1]
      float2 o2[2];
#pragma unroll
      for (int q = 0; q < 2; ++q) {
        float2 s2 = make_float2(0.f, 0.f);
#pragma unroll
        for (int m1 = 0; m1 < D1; ++m1) s2 = __ffma2_rn(xr2[q][XO + m1], t2[q][m1], s2);
        o2[q] = __fmul2_rn(salpha2[P], s2);
      }
      __stcs(reinterpret_cast<float4*>(gw + size_t(P) * C + 4 * cb), make_float4(o2[0].x, o2[0].y, o2[1].x, o2[1].y));
    }
#pragma unroll
    for (int q = 0; q < 2; ++q)  // grad_x += alpha_p w t
#pragma unroll
      for (int m1 = 0; m1 < D1; ++m1) dx2[q][XO + m1] = __ffma2_rn(wa2[q], t2[q][m1], dx2[q][XO + m1]);
    if (FL == 1 || want_dy) {  // grad_y[m2] += sum_{m1,m3} C[m1,m2,m3] sum_u alpha_p w_u x_u[m1] g_u[m3]
      constexpr bool SX = D1 <= D3;  // the weight scales the shorter of the x and grad_out blocks
      float2 xw2[2][SX ? D1 : 1], gw2[2][SX ? 1 : D3];
#pragma unroll
      for (int q = 0; q < 2; ++q) {
        if constexpr (SX) {
#pragma unroll
          for (int m1 = 0; m1 < D1; ++m1) xw2[q][m1] = __fmul2_rn(wa2[q], xr2[q][XO + m1]);
        } else {
#pragma unroll
          for (int m3 = 0; m3 < D3; ++m3) gw2[q][m3] = __fmul2_rn(wa2[q], g2[q][m3]);
        }
      }
      static_for<0, D1>([&](auto m1c) {
        constexpr int M1I = decltype(m1c)::value;
        static_for<0, D3>([&](auto m3c) {
          constexpr int M3I = decltype(m3c)::value;
          if constexpr (a_nz(L1, L2, L3, M1I - L1, M3I - L3)) {
            float2 z2;
            if constexpr (SX)
              z2 = __ffma2_rn(xw2[1][M1I], g2[1][M3I], __fmul2_rn(xw2[0][M1I], g2[0][M3I]));
            else
              z2 = __ffma2_rn(xr2[1][XO + M1I], gw2[1][M3I], __fmul2_rn(xr2[0][XO + M1I], gw2[0][M3I]));
            const float z = z2.x + z2.y;
            static_for<-L2, L2 + 1>([&](auto m2c) {
              constexpr int M2 = decltype(m2c)::value;
              if constexpr (cg_nz(L1, L2, L3, M1I - L1, M2, M3I - L3)) {
                constexpr int I = cg_index(L1, L2, L3, M1I - L1, M2, M3I - L3);
                dY[L2 * L2 + L2 + M2] = fmaf(c_cg32[I], z, dY[L2 * L2 + L2 + M2]);
              }
            });
          }
        });
      });
    }
  });
}

// grad_y components that group GI produces: every component of each harmonics block l2 that
// one of its paths uses, ascending; VP = that count rounded up to a power of two.
template <class CF, int GI>
struct YUse {
  struct Tab {
    int n;
    int comp[16];
  };
  static constexpr Tab make() {
    Tab t{};
    for (int l = 0; l <= CF::LY; ++l)
      if (group_has_l2<CF, GI>(l))
        for (int i = 0; i < 2 * l + 1; ++i) t.comp[t.n++] = l * l + i;
    return t;
  }
  static constexpr Tab TAB = make();
  static constexpr int NU = TAB.n;
  static constexpr int VP = NU <= 1 ? 1 : (NU <= 2 ? 2 : (NU <= 4 ? 4 : (NU <= 8 ? 8 : 16)));
  static constexpr bool CONTIG = [] {
    for (int i = 0; i < TAB.n; ++i)
      if (TAB.comp[i] != TAB.comp[0] + i) return false;
    return true;
  }();
  // harmonics component of used index u (u < NU)
  static __device__ __forceinline__ int comp_of(int u) {
    if constexpr (CONTIG) {
      constexpr int C0 = TAB.comp[0];
      return C0 + u;
    } else {
      int m = 0;
      static_for<0, NU>([&](auto qc) {
        constexpr int Q = decltype(qc)::value;
        constexpr int MQ = TAB.comp[Q];
        if (u == Q) m = MQ;
      });
      return m;
    }
  }
};

// Sum v[0..VP) over the W lanes of a slice (lane bits below W) by recursive halving: after
// each level a lane keeps half of its values and adds its partner's copy of that half.  On
// return v[0..max(VP/W, 1)) hold totals of components reduce_scatter_base(W, cb) + j (the same
// base for lanes that differ only in the bits below W/VP when VP < W).
template <typename T, int VP>
__device__ __forceinline__ void reduce_scatter(T (&v)[VP], int W, int cb) {
  int len = VP;
#pragma unroll
  for (int lvl = 0; lvl < 5; ++lvl) {
    const int o = W >> (lvl + 1);
    if (o < 1) break;
    const bool up = (cb & o) != 0;
    if (len > 1) {
      const int half = len / 2;
#pragma unroll
      for (int i = 0; i < VP / 2; ++i) {
        if (i >= half) break;
        const T send = up ? v[i] : v[i + half];
        const T keep = up ? v[i + half] : v[i];
        v[i] = keep + __shfl_xor_sync(0xffffffffu, send, o);
      }
      len = half;
    } else {
      v[0] += __shfl_xor_sync(0xffffffffu, v[0], o);
    }
  }
}

// First component a lane holds after reduce_scatter (fixed per lane).
template <int VP>
__device__ __forceinline__ int reduce_scatter_base(int W, int cb) {
  int base = 0, len = VP;
  for (int lvl = 0; lvl < 5; ++lvl) {
    const int o = W >> (lvl + 1);
    if (o < 1 || len <= 1) break;
    len /= 2;
    if (cb & o) base += len;
  }
  return base;
}

// Store / accumulate rules of group GI for grad_y blocks (bit l2) and grad_x blocks (bit l1).
template <class CF, int GI>
struct BwdMasks {
  static constexpr unsigned YS = [] {
    unsigned m = 0;
    for (int l = 0; l <= CF::LY; ++l) m |= (first_group_l2<CF>(l) == GI ? 1u : 0u) << l;
    return m;
  }();
  static constexpr unsigned YZ = [] {
    unsigned m = 0;
    if (GI == 0)
      for (int l = 0; l <= CF::LY; ++l) m |= (first_group_l2<CF>(l) < 0 ? 1u : 0u) << l;
    return m;
  }();
};

__device__ __forceinline__ int block_of(int m) { return m >= 9 ? 3 : (m >= 4 ? 2 : (m >= 1 ? 1 : 0)); }

// grad_x of one row for the group's degree blocks (first toucher stores, later groups add);
// group 0 also zero-fills the blocks no group touches.
template <class CF, int GI>
__device__ __forceinline__ void bwd_put_dx(typename CF::T* __restrict__ row, const typename CF::T (&dx)[K][Grp<CF, GI>::NXG],
                                           int C, int cb, typename CF::T scale, bool seg0 = true) {
  using T = typename CF::T;
  using GR = Grp<CF, GI>;
  static_for<GR::L1A, GR::L1B + 1>([&](auto lc) {
    constexpr int L = decltype(lc)::value;
    constexpr int D = 2 * L + 1;
    T* p = row + size_t(C) * (L * L) + size_t(4 * cb) * D;
    T v[K * D];
    // the first segment of the first group touching block L stores, every later one adds
    const bool store = first_group_l1<CF>(L) == GI && seg0;
    if (!store) ld16_l2(v, p);
#pragma unroll
    for (int k = 0; k < K; ++k)
#pragma unroll
      for (int m = 0; m < D; ++m) {
        const T s = scale * dx[k][L * L - GR::XB + m];
        if (store)
          v[k * D + m] = s;
        else
          v[k * D + m] += s;
      }
    st16(p, v);
  });
  if (GI == 0 && seg0) {
    static_for<0, CF::LX + 1>([&](auto lc) {
      constexpr int L = decltype(lc)::value;
      constexpr int D = 2 * L + 1;
      if constexpr (first_group_l1<CF>(L) < 0) {
        T v[K * D];
#pragma unroll
        for (int i = 0; i < K * D; ++i) v[i] = T(0);
        st16(row + size_t(C) * (L * L) + size_t(4 * cb) * D, v);
      }
    });
  }
}

// Ordering of the path groups of one unit.  Group GI of a unit adds to grad_x / grad_y blocks
// that groups < GI of the same unit stored, so it starts only once done[unit] == GI (acquire),
// and publishes done[unit] = GI + 1 after its writes (release).  The CTA that waits drew its
// ticket after the CTA it waits for (tickets are group-major), so that CTA is resident or
// finished and the chain ends at group 0: no deadlock, whatever order the hardware schedules
// CTAs in.  The wait is bounded; on timeout the error is recorded and the group proceeds.
__device__ __forceinline__ void bwd_wait_turn(const KBwd& a, int64_t unit, int gi) {
  if (gi > 0 && threadIdx.x == 0) wait_flag_geq(a.done + unit, gi, a.status, a.wait_ns);
  __syncwarp();
  // later bulk copies (async proxy) read what the earlier group wrote (generic proxy)
  asm volatile("fence.proxy.async;" ::: "memory");
}

__device__ __forceinline__ void bwd_end_turn(const KBwd& a, int64_t unit, int gi) {
  __threadfence();
  __syncwarp();
  if (threadIdx.x == 0)
    asm volatile("st.release.gpu.global.s32 [%0], %1;" ::"l"(a.done + unit), "r"(gi + 1) : "memory");
}

// Backward of path group GI for one unit.  Convolution: one CTA (one warp) per sender,
// walking its out-edges through the sender CSR; tensor product: one CTA per sample range.
// FL = 1: grad_w and grad_y are both non-null (the caller checked).
template <class CF, int GI, bool CONV, int CC, int FL>
__device__ __forceinline__ void bwd_group(const KBwd& a, const int64_t u, const int64_t n, const int64_t j0_in,
                                          const int64_t j1_in, const int64_t seg, const int64_t nseg,
                                          unsigned char* smem) {
  using T = typename CF::T;
  using GR = Grp<CF, GI>;
  using SM = BwdSmem<CF, GI>;
  using MK = BwdMasks<CF, GI>;
  constexpr int NYP = SM::NYP;
  const int C = CC > 0 ? CC : a.C;  // compile-time for the specialised multiplicities
  const int CB = C >> 2;            // CB <= 32: one warp covers every channel
  const int lane = threadIdx.x;
  const int cb = lane % CB, slice = lane / CB, NS = 32 / CB;
  const int S = a.stages;
  const T* __restrict__ x = static_cast<const T*>(a.x);
  const T* __restrict__ y = static_cast<const T*>(a.y);
  const T* __restrict__ vec = static_cast<const T*>(a.vec);
  const T* __restrict__ w = static_cast<const T*>(a.w);
  const T* __restrict__ g = static_cast<const T*>(a.grad_out);
  T* __restrict__ gx = static_cast<T*>(a.grad_x);
  T* __restrict__ gy = static_cast<T*>(a.grad_y);
  T* __restrict__ gwp = static_cast<T*>(a.grad_w);
  const size_t xrow = size_t(CF::NX) * C, orow = size_t(CF::NO) * C, wrow = size_t(CF::P) * C;
  const T scale = T(a.scale);
  const bool want_dy = FL == 1 || gy != nullptr;
  const uint32_t WB = BwdSlice<CF, GI>::wbytes(C), GB = BwdSlice<CF, GI>::gbytes(C);
  const uint32_t XB = BwdSlice<CF, GI>::xbytes(C, CONV), YB = BwdSlice<CF, GI>::ybytes(want_dy);
  const uint32_t SLOT = WB + GB + XB + YB;
  const size_t STAGE = size_t(NS) * SLOT;
  T* ysh = reinterpret_cast<T*>(smem + SM::ysh_off());
  int32_t* eid = reinterpret_cast<int32_t*>(smem + SM::eid_off());
  int32_t* did = reinterpret_cast<int32_t*>(smem + SM::did_off());
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + SM::bar_off());
  volatile int* s_abort = reinterpret_cast<volatile int*>(smem + SM::flag_off(S));
  unsigned char* stages = smem + SM::stage_off(S);

  // unit u: segment `seg` (of nseg) of sender n's out-edges (convolution), or sample range n
  int64_t j0, j1;
  if constexpr (CONV) {
    j0 = j0_in;  // the topology build checked the row pointers
    j1 = j1_in;
  } else {
    const int64_t per = (a.n_nodes + a.n_chunks - 1) / a.n_chunks;
    j0 = n * per;
    j1 = j0 + per < a.n_nodes ? j0 + per : a.n_nodes;
    if (j0 > j1) j0 = j1;
  }
  if (lane == 0) {
    for (int i = 0; i < S; ++i) mbar_init(&bars[i], 1);
    *s_abort = 0;
    mbar_fence_init();
  }
  bwd_wait_turn(a, u, GI);
  __syncthreads();

  T xr[K][GR::NXG], dx[K][GR::NXG], Y[CF::NY], dY[CF::NY];
  float2 xr2[2][GR::NXG], dx2[2][GR::NXG];  // paired float convolution: channel pairs of x, grad_x
#pragma unroll
  for (int k = 0; k < K; ++k)
#pragma unroll
    for (int j = 0; j < GR::NXG; ++j) dx[k][j] = T(0);
  if constexpr (CONV) load_x<CF, GR>(xr, x + size_t(n) * xrow, C, cb);
  if constexpr (paired<CF, CONV>()) {
#pragma unroll
    for (int q = 0; q < 2; ++q)
#pragma unroll
      for (int j = 0; j < GR::NXG; ++j) {
        xr2[q][j] = make_float2(xr[2 * q][j], xr[2 * q + 1][j]);
        dx2[q][j] = make_float2(0.f, 0.f);
      }
  }
  // grad_y components this lane writes after the per-edge reduction (fixed per lane)
  const int ybase = reduce_scatter_base<YUse<CF, GI>::VP>(CB, cb);
  const int yheld = YUse<CF, GI>::VP >= CB ? YUse<CF, GI>::VP / CB : 1;
  const bool ywriter = YUse<CF, GI>::VP >= CB || (cb & (CB / YUse<CF, GI>::VP - 1)) == 0;

  int prod_slot = 0, cons_slot = 0;
  uint32_t cons_phase = 0, issued = 0, consumed = 0;
  bool alive = true;
  const int64_t deg = j1 - j0;
  for (int64_t ws = 0; ws < deg && alive; ws += BWD_WIN) {
    const int cnt = int(deg - ws < BWD_WIN ? deg - ws : BWD_WIN);
    for (int i = lane; i < cnt; i += 32) {
      int64_t e = j0 + ws + i;
      int64_t d = e;
      bool ok = true;
      if constexpr (CONV) {
        e = __ldg(a.perm_src + e);
        ok = e >= 0 && e < a.n_edges;
        d = ok ? __ldg(a.dst + e) : 0;
        ok = ok && d >= 0 && d < a.n_nodes;
        if (!ok) record_error(a.status, E3_ERR_INDEX);
      }
      eid[i] = ok ? int32_t(e) : -1;
      did[i] = ok ? int32_t(d) : 0;
      T Yl[CF::NY];
      if (ok) {
        load_y<CF>(Yl, y, vec, a.sh_norm, e);
      } else {
#pragma unroll
        for (int m = 0; m < CF::NY; ++m) Yl[m] = T(0);
      }
#pragma unroll
      for (int m = 0; m < CF::NY; ++m) ysh[i * NYP + m] = Yl[m];
    }
    __syncthreads();
    const int steps = (cnt + NS - 1) / NS;
    // producer: lane 0 posts the expected bytes, then lane j (< edges in the step) copies the
    // slices of the step's j-th edge: weights, grad_out of the receiver, x for the tensor
    // product, the grad_y row to add to.  An edge with an id out of range copies edge 0 /
    // node 0 instead (the consumer skips it), so a stage's byte count depends only on its
    // number of edges.
    auto issue = [&](int st) {
      uint64_t* bar = &bars[prod_slot];
      unsigned char* dst = stages + size_t(prod_slot) * STAGE;
      const int nv = min(NS, cnt - st * NS);
      if (lane == 0) mbar_arrive_expect_tx(bar, uint32_t(nv) * SLOT);
      __syncwarp();
      if (lane < nv) {
        const int r = st * NS + lane;
        const int64_t e = max(eid[r], 0);
        unsigned char* d = dst + size_t(lane) * SLOT;
        bulk_load(d, w + e * wrow + size_t(GR::PB) * C, WB, bar);
        bulk_load(d + WB, g + size_t(did[r]) * orow + size_t(GR::OB) * C, GB, bar);
        if (XB > 0) bulk_load(d + WB + GB, x + size_t(e) * xrow + size_t(GR::XB) * C, XB, bar);
        if (YB > 0) bulk_load(d + WB + GB + XB, gy + size_t(e) * CF::NY, YB, bar);
      }
      prod_slot = prod_slot + 1 == S ? 0 : prod_slot + 1;
      ++issued;
    };
    for (int st = 0; st < S && st < steps; ++st) issue(st);

    for (int st = 0; st < steps; ++st) {
      {
        // the weight rows of the edges the next copy will fetch go to L2 now, so that copy
        // does not wait on DRAM
        const int rp = (st + S) * NS + lane;
        if (lane < NS && rp < cnt) prefetch_l2(w + max(eid[rp], 0) * wrow + size_t(GR::PB) * C, WB);
      }
      const int slot = cons_slot;
      const bool okw = mbar_wait(&bars[slot], cons_phase, a.status, a.wait_ns);
      if (!okw) *s_abort = 1;
      cons_slot = cons_slot + 1 == S ? 0 : cons_slot + 1;
      if (cons_slot == 0) cons_phase ^= 1u;
      ++consumed;
      const int r = st * NS + slice;
      const bool mine = okw && r < cnt && eid[r] >= 0;
      const int64_t e = mine ? eid[r] : 0;
      const T* sl = reinterpret_cast<const T*>(stages + size_t(slot) * STAGE + size_t(slice) * SLOT);
      if (mine) {
        if constexpr (!CONV) {
          const T* xs = sl + (WB + GB) / sizeof(T);
          static_for<GR::L1A, GR::L1B + 1>([&](auto lc) {
            constexpr int L = decltype(lc)::value;
            constexpr int D = 2 * L + 1;
            T t[K * D];
            lds16(t, xs + size_t(C) * (L * L - GR::XB) + size_t(4 * cb) * D);
#pragma unroll
            for (int k = 0; k < K; ++k)
#pragma unroll
              for (int m = 0; m < D; ++m) xr[k][L * L - GR::XB + m] = t[k * D + m];
          });
#pragma unroll
          for (int k = 0; k < K; ++k)
#pragma unroll
            for (int j = 0; j < GR::NXG; ++j) dx[k][j] = T(0);
        }
        {
          T yp[NYP];
          lds16(yp, ysh + r * NYP);
#pragma unroll
          for (int m = 0; m < CF::NY; ++m) Y[m] = yp[m];
        }
        if constexpr (paired<CF, CONV>())
          bwd_edge2<CF, GI, FL>(xr2, sl, Y, sl + WB / sizeof(T), dx2, dY, want_dy,
                                (FL == 1 || gwp) ? gwp + e * wrow : nullptr, C, cb, a.alpha_f2, a.salpha_f2);
        else
          bwd_edge<CF, GI, FL>(xr, sl, Y, sl + WB / sizeof(T), dx, dY, want_dy,
                               (FL == 1 || gwp) ? gwp + e * wrow : nullptr, C, cb, a.alpha, a.alpha_f, scale);
      } else {
#pragma unroll
        for (int m = 0; m < CF::NY; ++m) dY[m] = T(0);
      }
      if (want_dy) {
        // sum the group's components over the channel lanes of the slice, then each lane
        // writes the components it holds (first group of a block stores, later ones add)
        using YU = YUse<CF, GI>;
        T v[YU::VP];
        static_for<0, YU::VP>([&](auto uc) {
          constexpr int U = decltype(uc)::value;
          if constexpr (U < YU::NU) {
            constexpr int M = YU::TAB.comp[U];
            v[U] = dY[M];
          } else {
            v[U] = T(0);
          }
        });
        reduce_scatter<T, YU::VP>(v, CB, cb);
        if (mine && ywriter) {
#pragma unroll
          for (int j = 0; j < YU::VP; ++j) {
            if (j >= yheld) break;
            const int u = ybase + j;
            if (u >= YU::NU) break;
            const int m = YU::comp_of(u);
            T* p = gy + e * CF::NY + m;
            if (MK::YS & (1u << block_of(m)))
              *p = scale * v[j];
            else if (YB > 0)
              *p = sl[(WB + GB + XB) / sizeof(T) + m] + scale * v[j];
            else
              *p = __ldcg(p) + scale * v[j];
          }
          // group 0 also zero-fills harmonics blocks that no path uses
          if constexpr (MK::YZ != 0u) {
            if (cb == 0)
              for (int m = 0; m < CF::NY; ++m)
                if (MK::YZ & (1u << block_of(m))) gy[e * CF::NY + m] = T(0);
          }
        }
      }
      if constexpr (!CONV) {
        if (mine && gx != nullptr) bwd_put_dx<CF, GI>(gx + size_t(e) * xrow, dx, C, cb, scale);
      }
      __syncthreads();  // every thread is done with this stage (and sees an abort)
      if (*s_abort) {
        alive = false;
        break;
      }
      if (st + S < steps) issue(st + S);
    }
    __syncthreads();
  }
  // a sender split into segments adds its grad_x in (group, segment) order through a.chain
  int* chain = (CONV && nseg > 1) ? a.chain + n : nullptr;
  const int pos = int(GI * nseg + seg);
  if (!alive) {
    // a wait gave up: let the copies in flight land (bounded) before the CTA exits
    if (lane == 0)
      for (uint32_t q = consumed - 1; q < issued; ++q) mbar_wait(&bars[q % S], (q / S) & 1u, a.status, a.wait_ns);
    __syncthreads();
    if (chain != nullptr && lane == 0)  // later pairs must not wait for this one in vain
      asm volatile("st.release.gpu.global.s32 [%0], %1;" ::"l"(chain), "r"(pos + 1) : "memory");
    bwd_end_turn(a, u, GI);
    return;
  }
  if constexpr (CONV) {
    if (gx != nullptr) {
      if constexpr (paired<CF, CONV>()) {
        for (int off = CB; off < 32; off <<= 1)
#pragma unroll
          for (int q = 0; q < 2; ++q)
#pragma unroll
            for (int j = 0; j < GR::NXG; ++j) {
              dx2[q][j].x += __shfl_xor_sync(0xffffffffu, dx2[q][j].x, off);
              dx2[q][j].y += __shfl_xor_sync(0xffffffffu, dx2[q][j].y, off);
            }
#pragma unroll
        for (int q = 0; q < 2; ++q)
#pragma unroll
          for (int j = 0; j < GR::NXG; ++j) {
            dx[2 * q][j] = dx2[q][j].x;
            dx[2 * q + 1][j] = dx2[q][j].y;
          }
      } else {
        for (int off = CB; off < 32; off <<= 1)
#pragma unroll
          for (int k = 0; k < K; ++k)
#pragma unroll
            for (int j = 0; j < GR::NXG; ++j) dx[k][j] += __shfl_xor_sync(0xffffffffu, dx[k][j], off);
      }
      // wait (bounded) for the earlier (group, segment) pairs of this sender; they drew
      // earlier tickets, so they are resident or finished
      if (chain != nullptr && lane == 0 && pos > 0) wait_flag_geq(chain, pos, a.status, a.wait_ns);
      __syncwarp();
      if (slice == 0) bwd_put_dx<CF, GI>(gx + size_t(n) * xrow, dx, C, cb, scale, seg == 0);
      if (chain != nullptr) {
        __threadfence();
        __syncwarp();
        if (lane == 0) asm volatile("st.release.gpu.global.s32 [%0], %1;" ::"l"(chain), "r"(pos + 1) : "memory");
      }
    } else if (chain != nullptr && lane == 0) {
      asm volatile("st.release.gpu.global.s32 [%0], %1;" ::"l"(chain), "r"(pos + 1) : "memory");
    }
  }
  bwd_end_turn(a, u, GI);
}

// All path groups in one launch: every CTA draws a ticket; tickets are group-major (all units
// of group 0, then group 1, ...), so at any time the SMs mostly run one group's code and the
// next group's CTAs fill the SMs that the previous group's last CTAs leave idle.
// Register budget: the largest float group body alone needs about 168 registers; the bound
// keeps the merged kernel there (12 resident warps per SM by registers).  Double precision
// keeps the compiler's choice.
template <class CF>
constexpr int bwd_min_blocks() {
  return std::is_same<typename CF::T, float>::value ? 12 : 1;
}

template <class CF, bool CONV, int CC>
__global__ void __launch_bounds__(32, bwd_min_blocks<CF>()) bwd_kernel(const __grid_constant__ KBwd a) {
  extern __shared__ __align__(128) unsigned char smem[];
  int t = 0;
  if (threadIdx.x == 0) t = atomicAdd(a.ticket, 1) + a.first_ticket;
  t = __shfl_sync(0xffffffffu, t, 0);
  const int g = int(t / a.units);
  const int64_t u = t % a.units;
  if constexpr (CONV) {
    const int4 inf = a.uinfo[u];  // {sender, first edge, end edge, segment}; in bounds for u < units
    const int64_t nseg = a.unseg[u];
    if (u >= *a.n_units) return;  // the grid covers an upper bound of the units
    // the specialised multiplicities carry a copy with every gradient requested
    if (CC > 0 && a.grad_w != nullptr && a.grad_y != nullptr) {
      dispatch<CF::G>(g, [&](auto gc) {
        bwd_group<CF, decltype(gc)::value, CONV, CC, (CC > 0 ? 1 : 0)>(a, u, inf.x, inf.y, inf.z, inf.w, nseg, smem);
      });
    } else {
      dispatch<CF::G>(g, [&](auto gc) {
        bwd_group<CF, decltype(gc)::value, CONV, CC, 0>(a, u, inf.x, inf.y, inf.z, inf.w, nseg, smem);
      });
    }
  } else {
    dispatch<CF::G>(g, [&](auto gc) { bwd_group<CF, decltype(gc)::value, CONV, CC, 0>(a, u, u, 0, 0, 0, 1, smem); });
  }
}

// ============================================================ layout transposition ===
// Rows of blocks, block b holding C channels x D_b components.  in: mul_ir ([u][m] inside a
// block, the boundary's layout); out: component-major ([m][u] inside a block, the same block
// offsets).  The paired float kernels stage these copies, so that one 16-byte shared-memory load
// gives two channel pairs of one component.  Each thread writes 4 consecutive channels of one
// component (a 16-byte store); the reads of a block hit L1 after its first touch.
struct TransposeArgs {
  const float* in;
  float* out;
  int64_t rows;
  int row_len;  // floats per row
  int C;
  int nblk;
  int D[MAXP];
  int off[MAXP];  // float offset of block b in a row
};

static __global__ void __launch_bounds__(128) transpose_blocks_kernel(const __grid_constant__ TransposeArgs a) {
  for (int64_t r = blockIdx.x; r < a.rows; r += gridDim.x) {
    const float* __restrict__ in = a.in + r * a.row_len;
    float* __restrict__ out = a.out + r * a.row_len;
    for (int b = 0; b < a.nblk; ++b) {
      const int D = a.D[b], n = a.C * D;
      const float* __restrict__ ib = in + a.off[b];
      float* __restrict__ ob = out + a.off[b];
      for (int i = 4 * int(threadIdx.x); i < n; i += 4 * int(blockDim.x)) {
        const int m = i / a.C, u = i - m * a.C;  // C % 4 == 0: i .. i + 3 share m
        const float* p = ib + u * D + m;
        __stcg(reinterpret_cast<float4*>(ob + i), make_float4(__ldg(p), __ldg(p + D), __ldg(p + 2 * D), __ldg(p + 3 * D)));
      }
    }
  }
}

// Component-major copy of `rows` rows whose blocks have the given degrees, on `stream`.
static inline e3_status transpose_blocks(const float* in, float* out, int64_t rows, int C, const int* degs, int nblk,
                                         cudaStream_t stream) {
  if (rows <= 0) return E3_OK;
  TransposeArgs t{};
  t.in = in;
  t.out = out;
  t.rows = rows;
  t.C = C;
  t.nblk = nblk;
  int off = 0;
  for (int b = 0; b < nblk; ++b) {
    t.D[b] = 2 * degs[b] + 1;
    t.off[b] = off;
    off += C * t.D[b];
  }
  t.row_len = off;
  const int64_t grid = std::min<int64_t>(rows, int64_t(sm_count()) * 16);
  transpose_blocks_kernel<<<unsigned(grid), 128, 0, stream>>>(t);
  const cudaError_t err = cudaGetLastError();
  if (err != cudaSuccess) return fail(E3_ERR_CUDA, "transpose launch failed: %s", cudaGetErrorString(err));
  return E3_OK;
}

// =================================================================== host launchers ===
template <class CF, int CC>
e3_status launch_fwd_cc(const e3_plan* plan, const FwdArgs& h, bool conv) {
  KFwd a{};
  a.row_ptr = h.row_ptr;
  a.src = h.src;
  a.x = h.x;
  a.y = h.y;
  a.vec = h.vec;
  a.w = h.w;
  a.out = h.out;
  a.n_rows = h.n_rows;
  a.n_edges = h.n_edges;
  a.w_stride = h.w_stride;
  a.C = plan->C;
  a.sh_norm = h.sh_norm;
  e3_status st = E3_OK;
  a.status = plan->status;  // this plan's status word
  a.wait_ns = test_wait_limit_ns();
  a.first_ticket = test_first_ticket();
  for (int p = 0; p < plan->n_paths; ++p) a.pscale[p] = h.scale * plan->alpha[p];
  const int CB = plan->C / 4;
  const int threads = CB >= 32 ? CB : 32;
  const int NS = CB >= 32 ? 1 : 32 / CB;
  if (threads > fwd_max_threads<CF>())
    return fail(E3_ERR_UNSUPPORTED, "forward: multiplicity %d needs %d threads per CTA, at most %d compiled", plan->C,
                threads, fwd_max_threads<CF>());
  // ring depth: as deep as 3 stages while the CTAs that fit by registers also fit in shared memory
  auto kern = conv ? fwd_kernel<CF, true, CC> : fwd_kernel<CF, false, CC>;
  cudaFuncAttributes fa{};
  cudaError_t err = cudaFuncGetAttributes(&fa, kern);
  if (err != cudaSuccess) return fail(E3_ERR_CUDA, "cudaFuncGetAttributes: %s", cudaGetErrorString(err));
  const int regs = fa.numRegs > 0 ? fa.numRegs : 255;
  int ctas = 65536 / (((regs + 7) & ~7) * ((threads + 31) & ~31));
  ctas = std::max(1, std::min(ctas, 32));
  const size_t budget = size_t(225) * 1024 / ctas;
  int S = 3;
  while (S > 2 && FwdSmem<CF>::total(plan->C, NS, S) + 1024 > budget) --S;
  a.stages = S;
  const size_t smem = FwdSmem<CF>::total(plan->C, NS, S);
  if (smem > size_t(227) * 1024) return fail(E3_ERR_UNSUPPORTED, "forward needs %zu bytes of shared memory", smem);
  int64_t units;
  if (conv) {
    // receiver units from the topology buffer; zeroed ticket and progress counters
    const TopoPart T = topo_dst(h.n_rows, h.n_edges);
    const ConvCounters Cn = conv_counters(h.n_rows, h.n_edges, CF::G);
    const unsigned char* topo = static_cast<const unsigned char*>(h.topo);
    unsigned char* ws = static_cast<unsigned char*>(h.workspace);
    a.ticket = reinterpret_cast<int*>(ws);
    a.flags = reinterpret_cast<int*>(ws + Cn.flags);
    a.uinfo = reinterpret_cast<const int4*>(topo + T.info);
    a.unseg = reinterpret_cast<const int32_t*>(topo + T.nseg);
    a.n_units = reinterpret_cast<const int32_t*>(topo + T.units);
    a.units_max = seg_units_max(h.n_rows, h.n_edges);
    cudaError_t e2 = cudaMemsetAsync(ws, 0, Cn.chain, static_cast<cudaStream_t>(h.stream));
    if (e2 != cudaSuccess) return fail(E3_ERR_CUDA, "cudaMemsetAsync: %s", cudaGetErrorString(e2));
    if constexpr (paired<CF, true>()) {  // x in component-major blocks, after the counters
      int degs[CF::LX + 1];
      for (int l = 0; l <= CF::LX; ++l) degs[l] = l;
      float* xt = reinterpret_cast<float*>(ws + Cn.total);
      st = transpose_blocks(static_cast<const float*>(h.x), xt, h.n_rows, plan->C, degs, CF::LX + 1,
                            static_cast<cudaStream_t>(h.stream));
      if (st != E3_OK) return st;
      a.x = xt;
    }
    units = a.units_max;
    a.n_chunks = 0;
  } else {
    const int64_t n_units = (h.n_rows + NS - 1) / NS;
    units = std::min<int64_t>(n_units, int64_t(sm_count()) * ctas);
    a.n_chunks = int(units);
  }
  const int64_t blocks = units * CF::G;
  if (blocks >= (int64_t(1) << 31)) return fail(E3_ERR_SHAPE, "grid too large");
  err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
  if (err != cudaSuccess) return fail(E3_ERR_CUDA, "cudaFuncSetAttribute: %s", cudaGetErrorString(err));
  kern<<<unsigned(blocks), threads, smem, static_cast<cudaStream_t>(h.stream)>>>(a);
  err = cudaGetLastError();
  if (err != cudaSuccess) return fail(E3_ERR_CUDA, "forward launch failed: %s", cudaGetErrorString(err));
  return E3_OK;
}

// Shared memory of the merged backward: the largest of the groups' layouts.
template <class CF, int GI = 0>
size_t bwd_smem_max(int C, int NS, int S, bool conv, bool dy) {
  if constexpr (GI < CF::G) {
    return std::max(BwdSmem<CF, GI>::total(C, NS, S, conv, dy), bwd_smem_max<CF, GI + 1>(C, NS, S, conv, dy));
  } else {
    return 0;
  }
}

template <class CF, int CC>
e3_status launch_bwd_cc(const e3_plan* plan, const BwdArgs& h, bool conv) {
  KBwd a{};
  a.row_ptr_src = h.row_ptr_src;
  a.perm_src = h.perm_src;
  a.dst = h.dst;
  a.x = h.x;
  a.y = h.y;
  a.vec = h.vec;
  a.w = h.w;
  a.grad_out = h.grad_out;
  a.grad_x = h.grad_x;
  a.grad_y = h.grad_y;
  a.grad_w = h.grad_w;
  a.n_nodes = h.n_nodes;
  a.n_edges = h.n_edges;
  a.C = plan->C;
  a.sh_norm = h.sh_norm;
  a.scale = h.scale;
  e3_status st = E3_OK;
  a.status = plan->status;  // this plan's status word
  a.wait_ns = test_wait_limit_ns();
  a.first_ticket = test_first_ticket();
  for (int p = 0; p < plan->n_paths; ++p) {
    a.alpha[p] = plan->alpha[p];
    a.alpha_f[p] = float(plan->alpha[p]);
    a.alpha_f2[p] = make_float2(a.alpha_f[p], a.alpha_f[p]);
    const float sal = float(h.scale) * a.alpha_f[p];
    a.salpha_f2[p] = make_float2(sal, sal);
  }
  const int CB = plan->C / 4;
  if (CB > 32) return fail(E3_ERR_UNSUPPORTED, "the backward kernels need a multiplicity of at most 128");
  const int NS = 32 / CB;
  int64_t units;
  const cudaStream_t s = static_cast<cudaStream_t>(h.stream);
  unsigned char* ws = static_cast<unsigned char*>(h.workspace);
  cudaError_t err = cudaSuccess;
  if (conv) {
    // units are sender segments of the topology buffer; zeroed ticket and counters
    const TopoPart T = topo_src(h.n_nodes, h.n_edges);
    const ConvCounters Cn = conv_counters(h.n_nodes, h.n_edges, CF::G);
    const unsigned char* topo = static_cast<const unsigned char*>(h.topo);
    units = seg_units_max(h.n_nodes, h.n_edges);
    a.n_chunks = 0;
    a.ticket = reinterpret_cast<int*>(ws);
    a.done = reinterpret_cast<int*>(ws + Cn.flags);
    a.chain = reinterpret_cast<int*>(ws + Cn.chain);
    a.uinfo = reinterpret_cast<const int4*>(topo + T.info);
    a.unseg = reinterpret_cast<const int32_t*>(topo + T.nseg);
    a.n_units = reinterpret_cast<const int32_t*>(topo + T.units);
    err = cudaMemsetAsync(ws, 0, Cn.total, s);
    if (err != cudaSuccess) return fail(E3_ERR_CUDA, "cudaMemsetAsync: %s", cudaGetErrorString(err));
    if constexpr (paired<CF, true>()) {  // grad_out in component-major path blocks, after the counters
      int degs[CF::P];
      for (int p = 0; p < CF::P; ++p) degs[p] = CF::PT.l3[p];
      float* gt = reinterpret_cast<float*>(ws + Cn.total);
      st = transpose_blocks(static_cast<const float*>(h.grad_out), gt, h.n_nodes, plan->C, degs, CF::P, s);
      if (st != E3_OK) return st;
      a.grad_out = gt;
    }
  } else {
    const int64_t n_units = (h.n_nodes + NS - 1) / NS;
    units = std::min<int64_t>(n_units, int64_t(sm_count()) * 16);
    a.n_chunks = int(units);
    if (units == 0) return E3_OK;
    if (h.workspace_bytes < backward_workspace_bytes(units)) return fail(E3_ERR_INVALID_ARG, "workspace too small");
    a.ticket = reinterpret_cast<int*>(ws);
    a.done = reinterpret_cast<int*>(ws + 16);
    err = cudaMemsetAsync(ws, 0, 16 + 4 * size_t(units), s);
    if (err != cudaSuccess) return fail(E3_ERR_CUDA, "cudaMemsetAsync: %s", cudaGetErrorString(err));
  }
  const int64_t blocks = units * CF::G;
  if (blocks >= (int64_t(1) << 31)) return fail(E3_ERR_SHAPE, "grid too large");
  a.units = units;

  auto kern = conv ? bwd_kernel<CF, true, CC> : bwd_kernel<CF, false, CC>;
  cudaFuncAttributes fa{};
  err = cudaFuncGetAttributes(&fa, kern);
  if (err != cudaSuccess) return fail(E3_ERR_CUDA, "cudaFuncGetAttributes: %s", cudaGetErrorString(err));
  const int regs = fa.numRegs > 0 ? fa.numRegs : 255;
  const int ctas = std::max(1, std::min(32, 65536 / (((regs + 7) & ~7) * 32)));
  const size_t budget = size_t(225) * 1024 / ctas;
  // Ring depth: two stages when they cost no resident CTAs, else one.  A backward step is
  // long enough that more resident warps hide the copy latency better than a second stage
  // does (measured on the water-box workload: 8 CTAs/SM with two stages are slower than 12
  // with one).
  const bool dy = a.grad_y != nullptr;
  int S = 2;
  while (S > 1 && bwd_smem_max<CF>(a.C, NS, S, conv, dy) + 1024 > budget) --S;
  a.stages = S;
  const size_t smem = bwd_smem_max<CF>(a.C, NS, S, conv, dy);
  if (smem > size_t(227) * 1024) return fail(E3_ERR_UNSUPPORTED, "backward needs %zu bytes of shared memory", smem);
  err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
  if (err != cudaSuccess) return fail(E3_ERR_CUDA, "cudaFuncSetAttribute: %s", cudaGetErrorString(err));
  kern<<<unsigned(blocks), 32, smem, s>>>(a);
  err = cudaGetLastError();
  if (err != cudaSuccess) return fail(E3_ERR_CUDA, "backward launch failed: %s", cudaGetErrorString(err));
  return E3_OK;
}

// Multiplicities compiled with C as a constant (all channel address arithmetic folds to
// immediates); any other multiplicity runs the kernels with C read from the arguments.
template <class CF>
constexpr int spec_c(int i) {
  if constexpr (!std::is_same<typename CF::T, float>::value) {
    return 0;
  } else if constexpr (CF::LX == 2 && CF::LY == 3 && CF::LO == 2) {
    return i == 0 ? 64 : (i == 1 ? 128 : 0);
  } else if constexpr (CF::LX == 3 && CF::LY == 3 && CF::LO == 3) {
    return i == 0 ? 128 : 0;
  } else if constexpr (CF::LX == 1 && CF::LY == 2 && CF::LO == 2) {
    return i == 0 ? 8 : 0;
  } else {
    return 0;
  }
}

template <class CF>
e3_status launch_fwd_cfg(const e3_plan* plan, const FwdArgs& h, bool conv) {
  if constexpr (spec_c<CF>(0) > 0)
    if (plan->C == spec_c<CF>(0)) return launch_fwd_cc<CF, spec_c<CF>(0)>(plan, h, conv);
  if constexpr (spec_c<CF>(1) > 0)
    if (plan->C == spec_c<CF>(1)) return launch_fwd_cc<CF, spec_c<CF>(1)>(plan, h, conv);
  return launch_fwd_cc<CF, 0>(plan, h, conv);
}

template <class CF>
e3_status launch_bwd_cfg(const e3_plan* plan, const BwdArgs& h, bool conv) {
  if constexpr (spec_c<CF>(0) > 0)
    if (plan->C == spec_c<CF>(0)) return launch_bwd_cc<CF, spec_c<CF>(0)>(plan, h, conv);
  if constexpr (spec_c<CF>(1) > 0)
    if (plan->C == spec_c<CF>(1)) return launch_bwd_cc<CF, spec_c<CF>(1)>(plan, h, conv);
  return launch_bwd_cc<CF, 0>(plan, h, conv);
}

// Fill this unit's copy of the coefficient tables on the current device.
static inline cudaError_t upload_tables(const double* t64, const float* t32) {
  cudaError_t err = cudaMemcpyToSymbol(c_cg64, t64, sizeof(double) * CG_TABLE_SIZE);
  if (err == cudaSuccess) err = cudaMemcpyToSymbol(c_cg32, t32, sizeof(float) * CG_TABLE_SIZE);
  return err;
}

}  // namespace e3b
