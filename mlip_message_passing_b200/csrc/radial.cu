// Radial network of the point convolution on the fifth-generation tensor cores (sm_100a).
//
// What is computed (e3nn course, "Curriculum at a glance", lessons 05b and 06a; the path weights
// of an edge are a learned function of its length): for an edge vector v with r = |v|,
//     f_n = sqrt(2/c) sin(n pi r / c) / r * u(r / c),  n = 1 .. n_basis   (Bessel basis x envelope)
//     u(d) = 1 - (p+1)(p+2)/2 d^p + p(p+2) d^(p+1) - p(p+1)/2 d^(p+2)  for d < 1, else 0
//     h = SiLU(f W1),  w = h W2                                            (no biases)
// with W1 [n_basis, hidden] and W2 [hidden, n_out]; w [E, n_out] are the convolution's weights.
//
// The second layer is the dense contraction [E, hidden] x [hidden, n_out] (for the large
// convolution 1.26 M x 64 x 4352), the one GEMM-shaped step on this path, so it runs on tcgen05:
//   * a CTA takes tiles of 128 edges; each thread computes its edge's features and hidden layer
//     on the CUDA cores and writes them to shared memory as the MMA's A operand (K-major, the
//     canonical no-swizzle layout of 8-row x 16-byte core matrices);
//   * W2 is split once (e3_radial_prepare) into tf32 high and low parts laid out as B operand
//     tiles of 128 output columns; a tile is one contiguous bulk copy (cp.async.bulk, no multicast)
//     into a two-stage shared-memory ring;
//   * float32 accuracy from tf32 inputs: w = A_hi B_hi + A_hi B_lo + A_lo B_hi (the three-pass
//     split product; the dropped A_lo B_lo term is below 2^-21 of each product), accumulated in
//     float32 in tensor memory (TMEM), 128 lanes = 128 edges, one 128-column accumulator per
//     output tile, two of them so that the next tile's MMAs run while this tile's epilogue
//     (tcgen05.ld, then 16-byte stores to w) drains the other.
// One thread issues the MMAs and commits them to an mbarrier; every wait is bounded and records
// E3_ERR_TIMEOUT; TMEM is released before the CTA exits.
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>

#include "internal.h"
#include "tc_sm100.cuh"

namespace e3b {
namespace {

constexpr int RT_M = 128;         // edges per tile: the MMA's M, one TMEM lane per edge
constexpr int RT_N = 128;         // output columns per tile: the MMA's N
constexpr int RT_STAGES = 2;      // B tiles in flight (ring of shared-memory stages)
constexpr int RT_ACC = 2;         // TMEM accumulators (one per stage)
constexpr int RT_KMAX = 64;       // hidden width (the MMA's K) at most
constexpr int RT_BASIS_MAX = 16;  // Bessel functions at most
constexpr int RT_MATH_WARPS = 8;  // warps w and w + 4 read TMEM lanes 32 (w % 4) .. + 31
constexpr int RT_THREADS = 32 * RT_MATH_WARPS + 64;  // + one MMA warp + one B producer warp
constexpr int RT_TMEM_COLS = RT_ACC * RT_N;

struct RadialArgs {
  int64_t E;
  const float* vec;
  const float* w1;
  const unsigned char* prep;
  float* out;
  int* status;
  unsigned long long wait_ns;
  float cutoff, bessel_norm;
  int n_basis, p, K, n_out, n_tiles;
};

struct RadialSmem {
  static __host__ __device__ size_t a_bytes(int K) { return size_t(RT_M) * K * 4; }   // one of hi, lo
  static __host__ __device__ size_t b_bytes(int K) { return size_t(2) * RT_N * K * 4; }  // a tile: hi + lo
  static __host__ __device__ size_t b_off(int K) { return 2 * a_bytes(K); }
  static __host__ __device__ size_t w1_off(int K) { return b_off(K) + RT_STAGES * b_bytes(K); }  // (W1 is read through L1)
  static __host__ __device__ size_t stage_off(int K) { return w1_off(K); }
  // per warp, a 32-row x 32-column block of the accumulator on its way to global memory; the
  // 16-byte chunk j of row r sits at chunk j ^ (r % 8), so writes by row and reads by column group
  // are both free of bank conflicts
  static constexpr int STAGE_LD = 32;
  static __host__ __device__ size_t stage_bytes() { return size_t(RT_MATH_WARPS) * 32 * STAGE_LD * 4; }
  static __host__ __device__ size_t bar_off(int K) { return stage_off(K) + stage_bytes(); }
  static __host__ __device__ size_t total(int K) { return bar_off(K) + 8 * (2 * RT_STAGES + 2 * RT_ACC + 2) + 16; }
};

// Bessel features times the envelope of edge e (zeros past the last edge).
__device__ __forceinline__ void radial_features(const RadialArgs& a, int64_t e, float (&f)[RT_BASIS_MAX]) {
#pragma unroll
  for (int n = 0; n < RT_BASIS_MAX; ++n) f[n] = 0.f;
  if (e >= a.E) return;
  const float vx = __ldg(a.vec + 3 * e), vy = __ldg(a.vec + 3 * e + 1), vz = __ldg(a.vec + 3 * e + 2);
  const float r = sqrtf(vx * vx + vy * vy + vz * vz);
  const float d = r / a.cutoff;
  if (!(d < 1.f)) return;  // the envelope is zero from the cutoff on
  float dp = 1.f;
  for (int i = 0; i < a.p; ++i) dp *= d;
  const float p = float(a.p);
  const float env = 1.f - 0.5f * (p + 1.f) * (p + 2.f) * dp + p * (p + 2.f) * dp * d - 0.5f * p * (p + 1.f) * dp * d * d;
  const float pi_c = 3.14159265358979323846f / a.cutoff;
#pragma unroll
  for (int n = 0; n < RT_BASIS_MAX; ++n) {
    if (n < a.n_basis) {
      const float k = float(n + 1) * pi_c;
      f[n] = a.bessel_norm * env * (r > 1e-12f ? sinf(k * r) / r : k);
    }
  }
}

// Bulk copy of B tile nt into stage s (one thread).
__device__ __forceinline__ void request_tile(unsigned char* Bs, const unsigned char* prep, int nt, uint32_t s,
                                             uint32_t bbytes, uint64_t* bfull) {
  bulk_copy(Bs + size_t(s) * bbytes, prep + size_t(nt) * bbytes, bbytes, &bfull[s]);
}

// The three-pass product of one column tile (one thread): B stage s, accumulator ac.
__device__ __forceinline__ void issue_mma(const RadialArgs& a, uint32_t tmem, uint32_t idesc, uint32_t a_hi,
                                          uint32_t a_lo, uint32_t b_hi, uint32_t b_lo, uint32_t ac) {
  const uint32_t d = tmem + ac * RT_N;
  for (int ks = 0; ks < a.K / 8; ++ks) {
    const uint32_t o = uint32_t(ks) * 256;  // one K step: two 128-byte core matrices along K
    mma_tf32(d, smem_desc(a_hi + o, a.K), smem_desc(b_hi + o, a.K), idesc, ks > 0 ? 1u : 0u);
    mma_tf32(d, smem_desc(a_hi + o, a.K), smem_desc(b_lo + o, a.K), idesc, 1u);
    mma_tf32(d, smem_desc(a_lo + o, a.K), smem_desc(b_hi + o, a.K), idesc, 1u);
  }
}

// The RT_N / 2 accumulator columns [cbeg, cbeg + RT_N / 2) of this warp's 32 TMEM lanes (edges
// e0 .. e0 + 31) to w[e, RT_N nt + cbeg ..], 32 columns at a time: each thread loads its lane's
// values (warp-collective: every thread takes part) and writes them as a row of the warp's
// staging block; then each store instruction of the warp writes four whole 128-byte row segments
// (lane l: row l / 8 + 4 i, columns 4 (l % 8) ..), so no sector of w is written in parts.
__device__ __forceinline__ void store_tile(const RadialArgs& a, int64_t e0, int nt, int cbeg, uint32_t lane_base,
                                           float* stage) {
  const int lane = threadIdx.x & 31;
  const int c0 = nt * RT_N;
  constexpr int LD = RadialSmem::STAGE_LD;
  constexpr int H = RT_N / 64;  // 32-column chunks of this warp's half of the tile
  uint32_t v[H][32];
#pragma unroll
  for (int h = 0; h < H; ++h) tmem_ld32_nowait(lane_base + uint32_t(cbeg + 32 * h), v[h]);
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int h = 0; h < H; ++h) {
    const int c = cbeg + 32 * h;
#pragma unroll
    for (int j = 0; j < 8; ++j)
      *reinterpret_cast<float4*>(stage + lane * LD + 4 * (j ^ (lane & 7))) =
          make_float4(__uint_as_float(v[h][4 * j]), __uint_as_float(v[h][4 * j + 1]), __uint_as_float(v[h][4 * j + 2]),
                      __uint_as_float(v[h][4 * j + 3]));
    __syncwarp();
    const int col = c0 + c + 4 * (lane & 7);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int row = (lane >> 3) + 4 * i;
      const int64_t e = e0 + row;
      if (e < a.E && col < a.n_out)  // n_out % 4 == 0: a group of 4 is all in or all out
        *reinterpret_cast<float4*>(a.out + e * a.n_out + col) =
            *reinterpret_cast<const float4*>(stage + row * LD + 4 * ((lane & 7) ^ (row & 7)));
    }
    __syncwarp();
  }
}

// Warp-specialised: warps 0 .. RT_MATH_WARPS-1 compute the hidden layer into the A operand and
// drain the accumulators to w; warp RT_MATH_WARPS issues the MMAs; the next warp streams the B
// tiles.  They meet only on mbarriers, each wait bounded:
//   bfull[s] / bempty[s]      B stage s landed / read by its MMAs (tcgen05.commit)
//   accfull[c] / accempty[c]  accumulator c written (tcgen05.commit) / drained (one arrive per math warp)
//   afull / aempty            A of an edge tile written (one arrive per math warp) / read by its MMAs
// A consumer waits on parity (use & 1) of a full barrier; a producer waits on parity
// ((use & 1) ^ 1) of an empty one, which a fresh barrier passes at once.
__global__ void __launch_bounds__(RT_THREADS, 1) radial_kernel(const __grid_constant__ RadialArgs a) {
  extern __shared__ __align__(1024) unsigned char sm[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int K = a.K;
  unsigned char* As = sm;
  unsigned char* Bs = sm + RadialSmem::b_off(K);
  float* stage = reinterpret_cast<float*>(sm + RadialSmem::stage_off(K));
  uint64_t* bfull = reinterpret_cast<uint64_t*>(sm + RadialSmem::bar_off(K));
  uint64_t* bempty = bfull + RT_STAGES;
  uint64_t* accfull = bempty + RT_STAGES;
  uint64_t* accempty = accfull + RT_ACC;
  uint64_t* afull = accempty + RT_ACC;
  uint64_t* aempty = afull + 1;
  uint32_t* tslot = reinterpret_cast<uint32_t*>(aempty + 1);
  volatile int* s_abort = reinterpret_cast<volatile int*>(tslot + 1);
  const uint32_t ABYTES = uint32_t(RadialSmem::a_bytes(K)), BBYTES = uint32_t(RadialSmem::b_bytes(K));

  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(saddr(tslot)),
                 "r"(RT_TMEM_COLS));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  if (tid == 0) {
    for (int i = 0; i < RT_STAGES; ++i) {
      bar_init(&bfull[i], 1);
      bar_init(&bempty[i], 1);
    }
    for (int i = 0; i < RT_ACC; ++i) {
      bar_init(&accfull[i], 1);
      bar_init(&accempty[i], RT_MATH_WARPS);
    }
    bar_init(afull, RT_MATH_WARPS);
    bar_init(aempty, 1);
    *s_abort = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  fence_before_sync();
  __syncthreads();
  fence_after_sync();
  const uint32_t tmem = *tslot;
  const int64_t n_etiles = (a.E + RT_M - 1) / RT_M;

  if (warp < RT_MATH_WARPS) {
    // ------------------------------------------------------------- math warps
    uint32_t qq = 0, etn = 0;
    for (int64_t et = blockIdx.x; et < n_etiles && !warp_aborted(s_abort); et += gridDim.x, ++etn) {
      // A of the previous edge tile has been read by all its MMAs
      if (!warp_wait(aempty, (etn & 1u) ^ 1u, a.status, a.wait_ns)) {
        *s_abort = 1;
        break;
      }
      const int row = tid & (RT_M - 1);  // two threads per edge: each writes half of the hidden units
      const int64_t e = et * RT_M + row;
      float f[RT_BASIS_MAX];
      radial_features(a, e, f);
      const int kh = K / 2;  // a multiple of 4
      for (int k = (tid >> 7) * kh; k < (tid >> 7) * kh + kh; k += 4) {
        float hk[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          float sum = 0.f;
#pragma unroll
          for (int n = 0; n < RT_BASIS_MAX; ++n)
            if (n < a.n_basis) sum = fmaf(f[n], __ldg(a.w1 + n * K + k + j), sum);
          hk[j] = e < a.E ? sum / (1.f + expf(-sum)) : 0.f;
        }
        float4 hi, lo;
        hi.x = to_tf32(hk[0]);
        hi.y = to_tf32(hk[1]);
        hi.z = to_tf32(hk[2]);
        hi.w = to_tf32(hk[3]);
        lo.x = to_tf32(hk[0] - hi.x);
        lo.y = to_tf32(hk[1] - hi.y);
        lo.z = to_tf32(hk[2] - hi.z);
        lo.w = to_tf32(hk[3] - hi.w);
        *reinterpret_cast<float4*>(As + kmajor_off(row, k, K)) = hi;
        *reinterpret_cast<float4*>(As + ABYTES + kmajor_off(row, k, K)) = lo;
      }
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // the tensor core reads A through the async proxy
      __syncwarp();
      if (lane == 0) asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(saddr(afull)) : "memory");
      for (int nt = 0; nt < a.n_tiles; ++nt, ++qq) {
        const uint32_t ac = qq % RT_ACC;
        if (!warp_wait(&accfull[ac], (qq / RT_ACC) & 1u, a.status, a.wait_ns)) {
          *s_abort = 1;
          break;
        }
        fence_after_sync();
        // warps w and w + 4 share TMEM lanes 32 (w % 4) ..; each takes half of the columns
        store_tile(a, et * RT_M + (warp & 3) * 32, nt, (warp >> 2) * (RT_N / 2),
                   tmem + (uint32_t((warp & 3) * 32) << 16) + ac * RT_N, stage + warp * 32 * RadialSmem::STAGE_LD);
        fence_before_sync();
        __syncwarp();
        if (lane == 0) asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(saddr(&accempty[ac])) : "memory");
      }
    }
    __syncwarp();
  } else if (warp == RT_MATH_WARPS) {
    // ------------------------------------------------------------- MMA warp (one thread)
    if (lane == 0) {
      const uint32_t idesc = idesc_tf32(RT_M, RT_N);
      const uint32_t a_hi = saddr(As), a_lo = saddr(As + ABYTES);
      uint32_t qq = 0, etn = 0;
      int64_t last = -1;  // 0: the last commit went to aempty, else accfull / bempty of tile last - 1
      for (int64_t et = blockIdx.x; et < n_etiles && !*s_abort; et += gridDim.x, ++etn) {
        if (!bar_wait(afull, etn & 1u, a.status, a.wait_ns)) {
          *s_abort = 1;
          break;
        }
        fence_after_sync();
        for (int nt = 0; nt < a.n_tiles && !*s_abort; ++nt, ++qq) {
          const uint32_t s = qq % RT_STAGES, ac = qq % RT_ACC;
          if (!bar_wait(&bfull[s], (qq / RT_STAGES) & 1u, a.status, a.wait_ns) ||
              !bar_wait(&accempty[ac], ((qq / RT_ACC) & 1u) ^ 1u, a.status, a.wait_ns)) {
            *s_abort = 1;
            break;
          }
          fence_after_sync();
          const uint32_t b_hi = saddr(Bs + size_t(s) * BBYTES), b_lo = b_hi + BBYTES / 2;
          issue_mma(a, tmem, idesc, a_hi, a_lo, b_hi, b_lo, ac);
          mma_commit(&bempty[s]);
          mma_commit(&accfull[ac]);
          last = int64_t(qq) + 1;
        }
        if (*s_abort) break;
        mma_commit(aempty);
        last = 0;
      }
      if (*s_abort && last > 0) {
        // let the last committed MMA group finish (bounded) before the tensor memory is released
        const uint32_t lq = uint32_t(last - 1);
        bar_wait(&accfull[lq % RT_ACC], (lq / RT_ACC) & 1u, a.status, a.wait_ns);
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------- B producer (one thread)
    if (lane == 0) {
      uint32_t i = 0;
      for (int64_t et = blockIdx.x; et < n_etiles && !*s_abort; et += gridDim.x) {
        for (int nt = 0; nt < a.n_tiles; ++nt, ++i) {
          const uint32_t s = i % RT_STAGES;
          if (!bar_wait(&bempty[s], ((i / RT_STAGES) & 1u) ^ 1u, a.status, a.wait_ns)) {
            *s_abort = 1;
            break;
          }
          request_tile(Bs, a.prep, nt, s, BBYTES, bfull);
        }
        if (*s_abort) break;
      }
      if (*s_abort) {
        // let the copies in flight land (bounded) before the CTA exits
        for (uint32_t k = i >= RT_STAGES ? i - RT_STAGES : 0; k < i; ++k)
          bar_wait(&bfull[k % RT_STAGES], (k / RT_STAGES) & 1u, a.status, a.wait_ns);
      }
    }
    __syncwarp();
  }
  fence_before_sync();
  __syncthreads();
  fence_after_sync();
  if (warp == 0) asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(RT_TMEM_COLS));
}

// W2 [K, n_out] (row-major) -> B operand tiles: for each tile of 128 output columns, the tf32 high
// part then the low part, each [128 columns (rows of the K-major block) x K]; columns past n_out
// are zero.
__global__ void radial_prep_kernel(int K, int n_out, int n_tiles, const float* __restrict__ w2,
                                   unsigned char* __restrict__ prep) {
  const int64_t total = int64_t(n_tiles) * RT_N * K;
  for (int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < total; i += int64_t(gridDim.x) * blockDim.x) {
    const int k = int(i % K);
    const int64_t n = i / K;
    const int t = int(n / RT_N), row = int(n % RT_N);
    const float v = n < n_out ? __ldg(w2 + int64_t(k) * n_out + n) : 0.f;
    const float hi = to_tf32(v), lo = to_tf32(v - hi);
    unsigned char* tile = prep + size_t(t) * RadialSmem::b_bytes(K);
    *reinterpret_cast<float*>(tile + kmajor_off(row, k, K)) = hi;
    *reinterpret_cast<float*>(tile + RadialSmem::b_bytes(K) / 2 + kmajor_off(row, k, K)) = lo;
  }
}

size_t prep_bytes(int hidden, int n_out) {
  const int n_tiles = (n_out + RT_N - 1) / RT_N;
  return size_t(n_tiles) * RadialSmem::b_bytes(hidden);
}

e3_status check_radial_shape(int hidden, int n_out) {
  if (hidden < 8 || hidden > RT_KMAX || hidden % 8 != 0)
    return fail(E3_ERR_UNSUPPORTED, "hidden width %d: the kernel needs a multiple of 8 in [8, %d]", hidden, RT_KMAX);
  if (n_out < 4 || n_out % 4 != 0) return fail(E3_ERR_SHAPE, "n_out %d must be a positive multiple of 4", n_out);
  return E3_OK;
}

}  // namespace
}  // namespace e3b

using namespace e3b;

extern "C" e3_status e3_radial_prep_size(int32_t hidden, int32_t n_out, size_t* bytes) {
  clear_error();
  if (bytes == nullptr) return fail(E3_ERR_INVALID_ARG, "bytes is NULL");
  const e3_status st = check_radial_shape(hidden, n_out);
  if (st != E3_OK) return st;
  *bytes = prep_bytes(hidden, n_out);
  return E3_OK;
}

extern "C" e3_status e3_radial_prepare(int32_t hidden, int32_t n_out, const float* w2, void* prep, size_t prep_size,
                                       void* stream) {
  clear_error();
  e3_status st = check_radial_shape(hidden, n_out);
  if (st != E3_OK) return st;
  if (w2 == nullptr || prep == nullptr) return fail(E3_ERR_INVALID_ARG, "NULL pointer");
  if (reinterpret_cast<uintptr_t>(prep) % 16 != 0) return fail(E3_ERR_INVALID_ARG, "prep is not 16-byte aligned");
  if (prep_size < prep_bytes(hidden, n_out)) return fail(E3_ERR_SHAPE, "prep buffer of %zu bytes, need %zu", prep_size,
                                                         prep_bytes(hidden, n_out));
  const int n_tiles = (n_out + RT_N - 1) / RT_N;
  const int64_t total = int64_t(n_tiles) * RT_N * hidden;
  const int blocks = int(std::min<int64_t>((total + 255) / 256, 148 * 8));
  radial_prep_kernel<<<blocks, 256, 0, static_cast<cudaStream_t>(stream)>>>(hidden, n_out, n_tiles, w2,
                                                                            static_cast<unsigned char*>(prep));
  const cudaError_t err = cudaGetLastError();
  if (err != cudaSuccess) return fail(E3_ERR_CUDA, "prep launch failed: %s", cudaGetErrorString(err));
  return E3_OK;
}

extern "C" e3_status e3_radial_weights(int64_t E, const float* edge_vec, double cutoff, int32_t n_basis,
                                       int32_t envelope_p, int32_t hidden, const float* w1, const void* prep,
                                       int32_t n_out, float* w, void* stream) {
  clear_error();
  e3_status st = check_radial_shape(hidden, n_out);
  if (st != E3_OK) return st;
  if (E < 0 || E >= (int64_t(1) << 40)) return fail(E3_ERR_SHAPE, "E = %lld out of range", (long long)E);
  if (n_basis < 1 || n_basis > RT_BASIS_MAX) return fail(E3_ERR_UNSUPPORTED, "n_basis %d not in [1, %d]", n_basis, RT_BASIS_MAX);
  if (envelope_p < 1 || envelope_p > 32) return fail(E3_ERR_INVALID_ARG, "envelope order %d not in [1, 32]", envelope_p);
  if (!(cutoff > 0.0) || !(cutoff < 1e30)) return fail(E3_ERR_INVALID_ARG, "cutoff must be positive and finite");
  if (E == 0) return E3_OK;
  if (edge_vec == nullptr || w1 == nullptr || prep == nullptr || w == nullptr) return fail(E3_ERR_INVALID_ARG, "NULL pointer");
  if (reinterpret_cast<uintptr_t>(prep) % 16 != 0 || reinterpret_cast<uintptr_t>(w) % 16 != 0)
    return fail(E3_ERR_INVALID_ARG, "prep and w must be 16-byte aligned");
  if (reinterpret_cast<uintptr_t>(edge_vec) % 4 != 0 || reinterpret_cast<uintptr_t>(w1) % 4 != 0)
    return fail(E3_ERR_INVALID_ARG, "edge_vec and w1 must be 4-byte aligned");
  RadialArgs a{};
  a.E = E;
  a.vec = edge_vec;
  a.w1 = w1;
  a.prep = static_cast<const unsigned char*>(prep);
  a.out = w;
  st = device_status_ptr(&a.status);
  if (st != E3_OK) return st;
  a.wait_ns = test_wait_limit_ns();
  a.cutoff = float(cutoff);
  a.bessel_norm = float(std::sqrt(2.0 / cutoff));
  a.n_basis = n_basis;
  a.p = envelope_p;
  a.K = hidden;
  a.n_out = n_out;
  a.n_tiles = (n_out + RT_N - 1) / RT_N;
  const size_t smem = RadialSmem::total(hidden);
  cudaError_t err = cudaFuncSetAttribute(radial_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
  if (err != cudaSuccess) return fail(E3_ERR_CUDA, "cudaFuncSetAttribute: %s", cudaGetErrorString(err));
  const int64_t tiles = (E + RT_M - 1) / RT_M;
  const int grid = int(std::min<int64_t>(tiles, sm_count()));
  radial_kernel<<<grid, RT_THREADS, smem, static_cast<cudaStream_t>(stream)>>>(a);
  err = cudaGetLastError();
  if (err != cudaSuccess) return fail(E3_ERR_CUDA, "radial launch failed: %s", cudaGetErrorString(err));
  return E3_OK;
}
