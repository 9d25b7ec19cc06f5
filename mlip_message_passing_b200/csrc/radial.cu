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

namespace e3b {
namespace {

constexpr int RT_M = 128;         // edges per tile: the MMA's M, one TMEM lane per edge
constexpr int RT_N = 128;         // output columns per tile: the MMA's N
constexpr int RT_KMAX = 64;       // hidden width (the MMA's K) at most
constexpr int RT_BASIS_MAX = 16;  // Bessel functions at most
constexpr int RT_THREADS = 128;   // four warps; warp w reads TMEM lanes 32w .. 32w + 31
constexpr int RT_TMEM_COLS = 2 * RT_N;

// Byte offset of element (row, k) of a K-major operand block with K columns, in the canonical
// no-swizzle layout: 8-row x 16-byte core matrices; the core matrices along K are LBO = 128 bytes
// apart (so one MMA K-step of 8 tf32 values spans 256 bytes), 8-row groups SBO = 32 K bytes apart.
__host__ __device__ constexpr uint32_t kmajor_off(int row, int k, int K) {
  return uint32_t((row >> 3) * (K * 32) + (k >> 2) * 128 + (row & 7) * 16 + (k & 3) * 4);
}

// Shared-memory matrix descriptor: start address, LBO, SBO (16-byte units), the descriptor
// version of this architecture (bit 46), no swizzle (bits 61-63 zero).
__device__ __forceinline__ uint64_t smem_desc(uint32_t saddr, int K) {
  const uint64_t lbo = 128u >> 4, sbo = uint64_t(K * 32) >> 4;
  return uint64_t((saddr >> 4) & 0x3FFFu) | (lbo << 16) | (sbo << 32) | (uint64_t(1) << 46);
}

// Instruction descriptor of kind::tf32: float32 accumulator (bits 4-5 = 1), A and B tf32 (bits
// 7-9 and 10-12 = 2), both K-major, N / 8 at bits 17-22, M / 16 at bits 24-28.
constexpr uint32_t idesc_tf32(int M, int N) {
  return (1u << 4) | (2u << 7) | (2u << 10) | (uint32_t(N >> 3) << 17) | (uint32_t(M >> 4) << 24);
}

__device__ __forceinline__ uint32_t saddr(const void* p) { return static_cast<uint32_t>(__cvta_generic_to_shared(p)); }

__device__ __forceinline__ float to_tf32(float x) {
  uint32_t r;
  asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
  return __uint_as_float(r);
}

__device__ __forceinline__ unsigned long long now_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ void bar_init(uint64_t* b, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(saddr(b)), "r"(count) : "memory");
}

__device__ __forceinline__ bool bar_test(uint64_t* b, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(saddr(b)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Bounded wait for phase `parity` of barrier b; false (E3_ERR_TIMEOUT recorded) after wait_ns.
__device__ __forceinline__ bool bar_wait(uint64_t* b, uint32_t parity, int* status, unsigned long long wait_ns) {
  if (bar_test(b, parity)) return true;
  const unsigned long long t0 = now_ns();
  while (!bar_test(b, parity)) {
    if (now_ns() - t0 > wait_ns) {
      atomicCAS(status, 0, int(E3_ERR_TIMEOUT));
      return false;
    }
  }
  return true;
}

__device__ __forceinline__ void bulk_copy(void* dst, const void* src, uint32_t bytes, uint64_t* b) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(saddr(b)), "r"(bytes) : "memory");
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                   saddr(dst)),
               "l"(src), "r"(bytes), "r"(saddr(b))
               : "memory");
}

__device__ __forceinline__ void mma_tf32(uint32_t tmem_d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t accumulate) {
  const uint32_t mask = 0;  // no output lane disabled
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::tf32 [%0], %1, %2, %3, {%5, %5, %5, %5}, p;\n}\n" ::"r"(tmem_d),
      "l"(a), "l"(b), "r"(idesc), "r"(accumulate), "r"(mask));
}

__device__ __forceinline__ void mma_commit(uint64_t* b) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(saddr(b))
               : "memory");
}

__device__ __forceinline__ void fence_before_sync() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void fence_after_sync() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// 32 consecutive accumulator columns of this thread's TMEM lane.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&v)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]), "=r"(v[8]),
        "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15]), "=r"(v[16]),
        "=r"(v[17]), "=r"(v[18]), "=r"(v[19]), "=r"(v[20]), "=r"(v[21]), "=r"(v[22]), "=r"(v[23]), "=r"(v[24]),
        "=r"(v[25]), "=r"(v[26]), "=r"(v[27]), "=r"(v[28]), "=r"(v[29]), "=r"(v[30]), "=r"(v[31])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

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
  static __host__ __device__ size_t w1_off(int K) { return b_off(K) + 2 * b_bytes(K); }
  static __host__ __device__ size_t bar_off(int K) { return w1_off(K) + size_t(RT_BASIS_MAX) * RT_KMAX * 4; }
  static __host__ __device__ size_t total(int K) { return bar_off(K) + 64; }
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

// Thread 0: bulk copy of B tile nt into the next stage of the ring (copies counts the requests).
__device__ __forceinline__ void request_tile(unsigned char* Bs, const unsigned char* prep, int nt, uint32_t bbytes,
                                             uint64_t* bbar, uint32_t& copies) {
  const uint32_t s = copies & 1u;
  bulk_copy(Bs + size_t(s) * bbytes, prep + size_t(nt) * bbytes, bbytes, &bbar[s]);
  ++copies;
}

// Thread 0: the three-pass product of column tile number qq (stage and accumulator qq & 1) once
// its B tile has landed; false if that wait gave up.
__device__ __forceinline__ bool issue_tile(const RadialArgs& a, uint32_t qq, uint32_t tmem, uint32_t idesc,
                                           uint32_t a_hi, uint32_t a_lo, unsigned char* Bs, uint32_t bbytes,
                                           uint64_t* bbar, uint64_t* mbar, int64_t& last_commit) {
  const uint32_t s = qq & 1u;
  if (!bar_wait(&bbar[s], (qq >> 1) & 1u, a.status, a.wait_ns)) return false;
  fence_after_sync();
  const uint32_t b_hi = saddr(Bs + size_t(s) * bbytes), b_lo = b_hi + bbytes / 2;
  const uint32_t d = tmem + s * RT_N;
  for (int ks = 0; ks < a.K / 8; ++ks) {
    const uint32_t o = uint32_t(ks) * 256;  // one K step: two 128-byte core matrices along K
    mma_tf32(d, smem_desc(a_hi + o, a.K), smem_desc(b_hi + o, a.K), idesc, ks > 0 ? 1u : 0u);
    mma_tf32(d, smem_desc(a_hi + o, a.K), smem_desc(b_lo + o, a.K), idesc, 1u);
    mma_tf32(d, smem_desc(a_lo + o, a.K), smem_desc(b_hi + o, a.K), idesc, 1u);
  }
  mma_commit(&mbar[s]);
  last_commit = int64_t(qq);
  return true;
}

// Every thread: the 128 accumulator columns of its TMEM lane (edge e) to w[e, 128 nt ..]; the
// loads are warp-collective, so threads past the last edge load too and store nothing.
__device__ __forceinline__ void store_tile(const RadialArgs& a, int64_t e, int nt, uint32_t lane_base) {
  const int c0 = nt * RT_N;
  float* orow = a.out + (e < a.E ? e : 0) * a.n_out;
#pragma unroll
  for (int c = 0; c < RT_N; c += 32) {
    uint32_t v[32];
    tmem_ld32(lane_base + uint32_t(c), v);
    if (e < a.E) {
#pragma unroll
      for (int j = 0; j < 32; j += 4) {
        const int col = c0 + c + j;
        if (col < a.n_out)  // n_out % 4 == 0: a group of 4 is all in or all out
          __stcs(reinterpret_cast<float4*>(orow + col),
                 make_float4(__uint_as_float(v[j]), __uint_as_float(v[j + 1]), __uint_as_float(v[j + 2]),
                             __uint_as_float(v[j + 3])));
      }
    }
  }
}

__global__ void __launch_bounds__(RT_THREADS, 1) radial_kernel(const __grid_constant__ RadialArgs a) {
  extern __shared__ __align__(1024) unsigned char sm[];
  const int tid = threadIdx.x, warp = tid >> 5;
  const int K = a.K;
  unsigned char* As = sm;
  unsigned char* Bs = sm + RadialSmem::b_off(K);
  float* w1s = reinterpret_cast<float*>(sm + RadialSmem::w1_off(K));
  uint64_t* bbar = reinterpret_cast<uint64_t*>(sm + RadialSmem::bar_off(K));  // B tile landed, per stage
  uint64_t* mbar = bbar + 2;                                                 // MMAs done, per accumulator
  uint32_t* tslot = reinterpret_cast<uint32_t*>(bbar + 4);
  volatile int* s_abort = reinterpret_cast<volatile int*>(tslot + 1);
  const uint32_t ABYTES = uint32_t(RadialSmem::a_bytes(K)), BBYTES = uint32_t(RadialSmem::b_bytes(K));

  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(saddr(tslot)),
                 "r"(RT_TMEM_COLS));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  if (tid == 0) {
    for (int i = 0; i < 4; ++i) bar_init(&bbar[i], 1);
    *s_abort = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  for (int i = tid; i < a.n_basis * K; i += RT_THREADS) w1s[i] = __ldg(a.w1 + i);
  fence_before_sync();
  __syncthreads();
  fence_after_sync();
  const uint32_t tmem = *tslot;
  const uint32_t idesc = idesc_tf32(RT_M, RT_N);
  const uint32_t a_hi = saddr(As), a_lo = saddr(As + ABYTES);

  uint32_t q = 0;            // (edge tile, column tile) pairs started by this CTA: identical in every thread
  uint32_t copies = 0;       // B tiles requested (thread 0's count)
  int64_t last_commit = -1;  // sequence number of the last committed MMA group (thread 0's)
  bool alive = true;
  const int64_t n_etiles = (a.E + RT_M - 1) / RT_M;
  for (int64_t et = blockIdx.x; et < n_etiles && alive; et += gridDim.x) {
    // ---- features of this thread's edge, then its hidden layer four units at a time, written as
    // the A operand rows (tf32 hi / lo).  Every MMA that read A has completed: each column tile's
    // completion was waited for in the previous edge tile.
    const int64_t e = et * RT_M + tid;
    float f[RT_BASIS_MAX];
    radial_features(a, e, f);
    for (int k = 0; k < K; k += 4) {
      float hk[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        float s = 0.f;
#pragma unroll
        for (int n = 0; n < RT_BASIS_MAX; ++n)
          if (n < a.n_basis) s = fmaf(f[n], w1s[n * K + k + j], s);
        hk[j] = e < a.E ? s / (1.f + expf(-s)) : 0.f;
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
      *reinterpret_cast<float4*>(As + kmajor_off(tid, k, K)) = hi;
      *reinterpret_cast<float4*>(As + ABYTES + kmajor_off(tid, k, K)) = lo;
    }
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // the tensor core reads A through the async proxy
    fence_before_sync();
    __syncthreads();
    fence_after_sync();

    // ---- column tiles: MMA(nt + 1) is issued before the epilogue of nt
    const uint32_t q0 = q;
    if (tid == 0) {
      request_tile(Bs, a.prep, 0, BBYTES, bbar, copies);
      if (a.n_tiles > 1) request_tile(Bs, a.prep, 1, BBYTES, bbar, copies);
      if (!issue_tile(a, q0, tmem, idesc, a_hi, a_lo, Bs, BBYTES, bbar, mbar, last_commit)) *s_abort = 1;
    }
    for (int nt = 0; nt < a.n_tiles; ++nt) {
      const uint32_t qq = q0 + uint32_t(nt), s = qq & 1u;
      if (tid == 0 && !*s_abort && nt + 1 < a.n_tiles &&
          !issue_tile(a, qq + 1, tmem, idesc, a_hi, a_lo, Bs, BBYTES, bbar, mbar, last_commit))
        *s_abort = 1;
      // this tile's MMAs done: its accumulator is readable and its B stage is free.  The flag
      // is made uniform over the CTA, so the warp-collective TMEM loads below are taken by all
      // threads or by none.
      const bool done = __syncthreads_and(bar_wait(&mbar[s], (qq >> 1) & 1u, a.status, a.wait_ns) ? 1 : 0) != 0;
      if (!done) *s_abort = 1;
      fence_after_sync();
      if (tid == 0 && done && nt + 2 < a.n_tiles) request_tile(Bs, a.prep, nt + 2, BBYTES, bbar, copies);
      if (done) store_tile(a, e, nt, tmem + (uint32_t(warp * 32) << 16) + s * RT_N);
      fence_before_sync();
      __syncthreads();
      fence_after_sync();
      if (*s_abort) {
        alive = false;
        break;
      }
    }
    q += uint32_t(a.n_tiles);
  }
  if (!alive && tid == 0) {
    // a wait gave up: let the last copy of each stage and the last committed MMA group (whose
    // completion implies every earlier one) finish, bounded, before the tensor memory is released
    for (uint32_t i = copies >= 2 ? copies - 2 : 0; i < copies; ++i)
      bar_wait(&bbar[i & 1u], (i >> 1) & 1u, a.status, a.wait_ns);
    if (last_commit >= 0)
      bar_wait(&mbar[uint32_t(last_commit) & 1u], (uint32_t(last_commit) >> 1) & 1u, a.status, a.wait_ns);
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
