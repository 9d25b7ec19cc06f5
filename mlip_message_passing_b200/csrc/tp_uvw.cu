// Fully connected ("uvw") tensor product with shared weights on the fifth-generation tensor cores.
//
// What is computed (e3nn course, "Curriculum at a glance", lesson 03b: in the uvw mode every
// channel u of x and v of y feeds every output channel w, one weight per (path, u, v, w)).  With y
// of one channel per degree (the harmonics of an edge, or any single-channel feature) this is
//     out[b, o, w, m3] = sum_{p -> o} alpha_p sum_u W_p[u, w] T_p[b, u, m3],
//     T_p[b, u, m3]   = sum_{m1, m2} C_p[m1, m2, m3] x[b, l1(p), u, m1] y[b, l2(p), m2],
// for each output block o a dense contraction over K = (path, u): rows (sample, m3), columns w.
// The backward's grad_x has the same shape with x and grad_out exchanged:
//     grad_x[b, l1, u, m1] = sum_{p: l1(p) = l1} alpha_p sum_w W_p[u, w] S_p[b, w, m1],
//     S_p[b, w, m1]       = sum_{m2, m3} C_p[m1, m2, m3] g[b, o(p), w, m3] y[b, l2(p), m2].
// Both run in one warp-specialised tcgen05 kernel (uvw_gemm_kernel):
//   * a tile is 128 accumulator rows of one target block of degree l: BT = floor(128 / D)
//     samples x D = 2 l + 1 components, row b_local D + m;
//   * eight math warps compute the A operand (alpha_p T_p, or alpha_p S_p) for 32 input channels
//     at a time on the CUDA cores, as tf32 high and low parts, into a ring of shared-memory
//     stages (K-major, the canonical no-swizzle layout of 8-row x 16-byte core matrices); a
//     thread keeps its samples' coupling sum_m2 C y in registers over all chunks of a term;
//   * the weights, split per call into tf32 high and low parts and laid out as B operand chunks of
//     32 input channels (uvw_prep_kernel), stream in by bulk copy (cp.async.bulk, no multicast);
//   * one thread issues A_hi B_hi + A_hi B_lo + A_lo B_hi per 8-wide K step (the three-pass split
//     product: float32 accuracy from tf32 inputs) into float32 accumulators in TMEM, 128 lanes x
//     N columns each: the main products go round-robin by chunk into UV_NBIG accumulators and the
//     two small correction products into one more, so that no accumulator takes more than a third
//     of the additions of a long K (a tile sums up to ~1300 products, and every addition in the
//     tensor core rounds); after the last chunk of a tile the math warps load and add the
//     accumulators (tcgen05.ld, float32) and store the sum.
// Every wait is bounded (E3_ERR_TIMEOUT) and TMEM is released before the CTA exits.
// grad_w, a contraction over samples, runs in a second tcgen05 kernel (both operands written by the
// math warps); grad_y contracts Z_p = W_p g (this kernel, plain role) with x on the CUDA cores.
#include <climits>

#include "kernels.cuh"
#include "tc_sm100.cuh"

namespace e3b {
namespace {

constexpr int UV_M = 128;          // accumulator rows per tile (TMEM lanes)
constexpr int UV_KC = 32;          // input channels per K chunk
constexpr int UV_NMAX = 128;       // output channels (the MMA's N) at most
constexpr int UV_STAGES = 3;       // A and B chunks in flight
constexpr int UV_MATH_WARPS = 8;
constexpr int UV_THREADS = 32 * UV_MATH_WARPS + 64;  // + one MMA warp + one B producer warp
constexpr int UV_NBIG = 3;       // accumulators of the main products (round-robin by chunk)
constexpr int UV_TMEM_COLS = 512;  // (UV_NBIG + 1) x UV_NMAX columns, rounded up to a power of two
constexpr uint32_t UV_A_BYTES = UV_M * UV_KC * 4;             // one of hi, lo
constexpr uint32_t UV_B_BYTES_MAX = 2 * UV_NMAX * UV_KC * 4;  // hi + lo

// What the math warps put into the A operand (see produce_term).
enum UvwRole { ROLE_FWD = 0, ROLE_GX = 1, ROLE_PLAIN = 2 };

struct UvwSmem {
  static constexpr size_t a_off(int s) { return size_t(s) * 2 * UV_A_BYTES; }
  static constexpr size_t b_off(int s) { return size_t(UV_STAGES) * 2 * UV_A_BYTES + size_t(s) * UV_B_BYTES_MAX; }
  static constexpr size_t bar_off() { return b_off(UV_STAGES); }
  // afull, aempty, bfull, bempty [UV_STAGES] each, accfull, accempty; then the TMEM slot and the abort flag
  static constexpr size_t total() { return bar_off() + 8 * (4 * UV_STAGES + 2) + 16; }
};

__device__ __forceinline__ int find_target(const UvwGemmArgs& a, int tile) {
  int t = 0;
  while (t + 1 < a.n_targets && tile >= a.tg[t + 1].tile_begin) ++t;
  return t;
}

// A operand of every chunk of one term (32 input channels [32 kc, 32 kc + 32) per chunk) for the
// samples of a tile.  Thread (warp w, lane): channels ul = 16 (w % 2) + 4 (lane / 8) .. + 3 of a
// chunk, samples b_local = 8 (w / 2) + lane % 8 + 32 i (i < NSLOT).  The coupling of each of its
// samples, cm[i][t] = sum_m2 C[..] y[m2] (input component i, target component t), is formed once
// and kept in registers for the term's chunks.  The eight lanes of one store phase hold eight
// consecutive samples, whose rows differ modulo 8 (D is odd), so the 16-byte stores are free of
// bank conflicts.  Returns false when a wait gave up (the abort flag is then set).
template <int LI, int L2, int LT, int ROLE>
__device__ __forceinline__ bool produce_term(const UvwGemmArgs& a, int bt, int64_t b0, const UvwTerm& tm,
                                             const UvwTerm* next, int nk, unsigned char* sm, uint64_t* aempty,
                                             uint64_t* afull, uint32_t& q, volatile int* s_abort, int warp, int lane) {
  constexpr int DI = 2 * LI + 1, DT = 2 * LT + 1, NY2 = (L2 + 1) * (L2 + 1);
  constexpr int NSLOT = (UV_M / DT + 31) / 32;
  const int ul = 16 * (warp & 1) + 4 * (lane >> 3);
  float cm[NSLOT][DI][DT];
  const float* inrow[NSLOT];
  bool valid[NSLOT];
#pragma unroll
  for (int k = 0; k < NSLOT; ++k) {
    const int bl = 8 * (warp >> 1) + (lane & 7) + 32 * k;
    const int64_t b = b0 + bl;
    valid[k] = bl < bt && b < a.B;
    inrow[k] = a.in + (valid[k] ? b * a.in_stride + tm.in_off : 0);
    float Y[NY2];
#pragma unroll
    for (int m = 0; m < 2 * L2 + 1; ++m)
      Y[L2 * L2 + m] = (ROLE != ROLE_PLAIN && valid[k]) ? __ldg(a.y + b * a.y_stride + L2 * L2 + m) : 0.f;
    static_for<0, DI>([&](auto ic) {
      static_for<0, DT>([&](auto tc) {
        constexpr int I = decltype(ic)::value, T = decltype(tc)::value;
        if constexpr (ROLE == ROLE_PLAIN) {
          cm[k][I][T] = I == T ? tm.alpha : 0.f;  // the input itself (DT == DI)
        } else if constexpr (ROLE == ROLE_FWD) {
          if constexpr (a_nz(LI, L2, LT, I - LI, T - LT))
            cm[k][I][T] = tm.alpha * a_entry<float, LI, L2, LT, I - LI, T - LT>(Y);
          else
            cm[k][I][T] = 0.f;
        } else {
          if constexpr (a_nz(LT, L2, LI, T - LT, I - LI))
            cm[k][I][T] = tm.alpha * a_entry<float, LT, L2, LI, T - LT, I - LI>(Y);
          else
            cm[k][I][T] = 0.f;
        }
      });
    });
  }
  for (int kc = 0; kc < nk; ++kc, ++q) {
    const uint32_t s = q % UV_STAGES;
    if (!warp_wait(&aempty[s], ((q / UV_STAGES) & 1u) ^ 1u, a.status, a.wait_ns)) {
      *s_abort = 1;
      return false;
    }
    unsigned char* As = sm + UvwSmem::a_off(int(s));
    if (kc + 1 < nk) {
      // ask L2 for the next chunk's runs now, so that their loads do not wait on HBM
#pragma unroll
      for (int k = 0; k < NSLOT; ++k) {
        if (!valid[k]) continue;
        const float* ip = inrow[k] + (int64_t(kc + 1) * UV_KC + ul) * DI;
        asm volatile("prefetch.global.L2 [%0];" ::"l"(ip));
        asm volatile("prefetch.global.L2 [%0];" ::"l"(ip + 4 * DI - 1));
      }
    } else if (next != nullptr) {
      // the last chunk of this term: the next term's first chunk (same samples, another block)
      const int dn = 2 * next->l_in + 1;
#pragma unroll
      for (int k = 0; k < NSLOT; ++k) {
        if (!valid[k]) continue;
        const float* ip = inrow[k] - tm.in_off + next->in_off + int64_t(ul) * dn;
        asm volatile("prefetch.global.L2 [%0];" ::"l"(ip));
        asm volatile("prefetch.global.L2 [%0];" ::"l"(ip + 4 * dn - 1));
      }
    }
#pragma unroll
    for (int k = 0; k < NSLOT; ++k) {
      if (!valid[k]) continue;
      const int bl = 8 * (warp >> 1) + (lane & 7) + 32 * k;
      float in[4 * DI];  // channels u .. u + 3, components contiguous: one run of 4 DI floats
      const float4* ip = reinterpret_cast<const float4*>(inrow[k] + (int64_t(kc) * UV_KC + ul) * DI);
#pragma unroll
      for (int j = 0; j < DI; ++j) {
        const float4 v = __ldg(ip + j);
        in[4 * j] = v.x;
        in[4 * j + 1] = v.y;
        in[4 * j + 2] = v.z;
        in[4 * j + 3] = v.w;
      }
#pragma unroll
      for (int t = 0; t < DT; ++t) {
        float v[4];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          if constexpr (ROLE == ROLE_PLAIN) {
            v[c] = tm.alpha * in[c * DI + t];
          } else {
            float acc = 0.f;
#pragma unroll
            for (int i = 0; i < DI; ++i) acc = fmaf(cm[k][i][t], in[c * DI + i], acc);
            v[c] = acc;
          }
        }
        float4 hi, lo;
        hi.x = to_tf32(v[0]);
        hi.y = to_tf32(v[1]);
        hi.z = to_tf32(v[2]);
        hi.w = to_tf32(v[3]);
        lo.x = to_tf32(v[0] - hi.x);
        lo.y = to_tf32(v[1] - hi.y);
        lo.z = to_tf32(v[2] - hi.z);
        lo.w = to_tf32(v[3] - hi.w);
        const uint32_t off = kmajor_off(bl * DT + t, ul, UV_KC);
        *reinterpret_cast<float4*>(As + off) = hi;
        *reinterpret_cast<float4*>(As + UV_A_BYTES + off) = lo;
      }
    }
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // the tensor core reads A through the async proxy
    __syncwarp();
    if (lane == 0) asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(saddr(&afull[s])) : "memory");
  }
  return true;
}

template <int ROLE>
__device__ __forceinline__ bool produce_term_any(const UvwGemmArgs& a, const UvwTarget& tg, int64_t b0,
                                                 const UvwTerm& tm, const UvwTerm* next, int nk, unsigned char* sm,
                                                 uint64_t* aempty, uint64_t* afull, uint32_t& q,
                                                 volatile int* s_abort, int warp, int lane) {
  bool ok = true;
  if constexpr (ROLE == ROLE_PLAIN) {
    dispatch<E3_LMAX + 1>(tm.l_in, [&](auto lic) {
      constexpr int LI = decltype(lic)::value;
      ok = produce_term<LI, 0, LI, ROLE>(a, tg.bt, b0, tm, next, nk, sm, aempty, afull, q, s_abort, warp, lane);
    });
  } else {
    dispatch<E3_LMAX + 1>(tm.l_in, [&](auto lic) {
      dispatch<E3_LMAX + 1>(tm.l2, [&](auto l2c) {
        dispatch<E3_LMAX + 1>(tg.l, [&](auto ltc) {
          constexpr int LI = decltype(lic)::value, L2 = decltype(l2c)::value, LT = decltype(ltc)::value;
          if constexpr (triangle(LI, L2, LT))
            ok = produce_term<LI, L2, LT, ROLE>(a, tg.bt, b0, tm, next, nk, sm, aempty, afull, q, s_abort, warp,
                                                lane);
        });
      });
    });
  }
  return ok;
}

// Accumulator rows 32 (w % 4) + lane of this warp to the target block: warps w and w + 4 share
// the lanes and take alternate 32-column groups; the value is the sum of the correction
// accumulator and the nbig main accumulators in use.  Every lane joins each tcgen05.ld
// (warp-collective); rows past the tile's samples store nothing.
__device__ __forceinline__ void store_rows(const UvwGemmArgs& a, const UvwTarget& tg, int64_t b0, uint32_t tmem,
                                           int nbig, int warp, int lane) {
  const int D = 2 * tg.l + 1;
  const int r = 32 * (warp & 3) + lane;
  const int bl = r / D, m = r - bl * D;
  const int64_t b = b0 + bl;
  const bool ok = bl < tg.bt && b < a.B;
  float* dst = a.out + (ok ? b * a.out_stride + tg.off + m : 0);
  const uint32_t lane_base = tmem + (uint32_t(32 * (warp & 3)) << 16);
  for (int c = 32 * (warp >> 2); c < a.N; c += 64) {
    uint32_t v[32];
    float sum[32];
    tmem_ld32_nowait(lane_base + uint32_t(UV_NBIG * UV_NMAX + c), v);
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int i = 0; i < 32; ++i) sum[i] = __uint_as_float(v[i]);
    for (int k = 0; k < nbig; ++k) {
      tmem_ld32_nowait(lane_base + uint32_t(k * UV_NMAX + c), v);
      asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
      for (int i = 0; i < 32; ++i) sum[i] += __uint_as_float(v[i]);
    }
    if (ok) {
#pragma unroll
      for (int i = 0; i < 32; ++i) dst[int64_t(c + i) * D] = sum[i];
    }
  }
}

// A target block that no path writes: its rows are zero.
__device__ __forceinline__ void zero_rows(const UvwGemmArgs& a, const UvwTarget& tg, int64_t b0, int tid) {
  const int D = 2 * tg.l + 1;
  const int64_t n = int64_t(tg.bt) * a.N * D;
  for (int64_t i = tid; i < n; i += 32 * UV_MATH_WARPS) {
    const int64_t bl = i / (int64_t(a.N) * D);
    const int64_t b = b0 + bl;
    if (b < a.B) a.out[b * a.out_stride + tg.off + (i - bl * a.N * D)] = 0.f;
  }
}

// Warp-specialised: warps 0 .. 7 produce A chunks and drain the accumulator; warp 8 issues the
// MMAs; warp 9 streams the B chunks.  They meet on mbarriers, each wait bounded:
//   afull[s] / aempty[s]   A chunk in stage s written (one arrive per math warp) / read by its MMAs
//   bfull[s] / bempty[s]   B chunk in stage s landed / read by its MMAs
//   accfull / accempty     the tile's accumulator complete (tcgen05.commit) / drained
// A consumer waits on parity (use & 1) of a full barrier; a producer on parity ((use & 1) ^ 1) of
// an empty one, which a fresh barrier passes at once.  Tiles of targets without paths are zeroed
// by the math warps and skipped by the other two roles (they count no barrier phases).
template <int ROLE>
__global__ void __launch_bounds__(UV_THREADS, 1) uvw_gemm_kernel(const __grid_constant__ UvwGemmArgs a) {
  extern __shared__ __align__(1024) unsigned char sm[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  uint64_t* afull = reinterpret_cast<uint64_t*>(sm + UvwSmem::bar_off());
  uint64_t* aempty = afull + UV_STAGES;
  uint64_t* bfull = aempty + UV_STAGES;
  uint64_t* bempty = bfull + UV_STAGES;
  uint64_t* accfull = bempty + UV_STAGES;
  uint64_t* accempty = accfull + 1;
  uint32_t* tslot = reinterpret_cast<uint32_t*>(accempty + 1);
  volatile int* s_abort = reinterpret_cast<volatile int*>(tslot + 1);
  const int nk = a.k_in / UV_KC;

  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(saddr(tslot)),
                 "r"(UV_TMEM_COLS));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  if (tid == 0) {
    for (int i = 0; i < UV_STAGES; ++i) {
      bar_init(&afull[i], UV_MATH_WARPS);
      bar_init(&aempty[i], 1);
      bar_init(&bfull[i], 1);
      bar_init(&bempty[i], 1);
    }
    bar_init(accfull, 1);
    bar_init(accempty, UV_MATH_WARPS);
    *s_abort = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  fence_before_sync();
  __syncthreads();
  fence_after_sync();
  const uint32_t tmem = *tslot;

  if (warp < UV_MATH_WARPS) {
    // ------------------------------------------------------------- math warps
    uint32_t q = 0, tn = 0;
    for (int tile = blockIdx.x; tile < a.total_tiles && !warp_aborted(s_abort); tile += gridDim.x) {
      const UvwTarget& tg = a.tg[find_target(a, tile)];
      const int64_t b0 = int64_t(tile - tg.tile_begin) * tg.bt;
      if (tg.term_begin == tg.term_end) {
        zero_rows(a, tg, b0, tid);
        continue;
      }
      bool ok = true;
      for (int j = tg.term_begin; j < tg.term_end && ok; ++j)
        ok = produce_term_any<ROLE>(a, tg, b0, a.term[j], j + 1 < tg.term_end ? &a.term[j + 1] : nullptr, nk, sm,
                                    aempty, afull, q, s_abort, warp, lane);
      if (!ok) break;
      if (!warp_wait(accfull, tn & 1u, a.status, a.wait_ns)) {
        *s_abort = 1;
        break;
      }
      fence_after_sync();
      const int chunks = (tg.term_end - tg.term_begin) * nk;
      store_rows(a, tg, b0, tmem, chunks < UV_NBIG ? chunks : UV_NBIG, warp, lane);
      fence_before_sync();
      __syncwarp();
      if (lane == 0) asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(saddr(accempty)) : "memory");
      ++tn;
    }
    __syncwarp();
  } else if (warp == UV_MATH_WARPS) {
    // ------------------------------------------------------------- MMA warp (one thread)
    if (lane == 0) {
      const uint32_t idesc = idesc_tf32(UV_M, a.N);
      const uint32_t bhalf = a.b_chunk_bytes / 2;
      uint32_t q = 0, tn = 0;
      int64_t last = -1;  // chunk index + 1 of the last commit (its aempty phase), or -1
      for (int tile = blockIdx.x; tile < a.total_tiles && !*s_abort; tile += gridDim.x) {
        const UvwTarget& tg = a.tg[find_target(a, tile)];
        if (tg.term_begin == tg.term_end) continue;
        if (!bar_wait(accempty, (tn & 1u) ^ 1u, a.status, a.wait_ns)) {
          *s_abort = 1;
          break;
        }
        fence_after_sync();
        uint32_t ci = 0;  // chunk of this tile
        for (int j = tg.term_begin; j < tg.term_end && !*s_abort; ++j) {
          for (int kc = 0; kc < nk; ++kc, ++q, ++ci) {
            const uint32_t s = q % UV_STAGES, ph = (q / UV_STAGES) & 1u;
            if (!bar_wait(&afull[s], ph, a.status, a.wait_ns) || !bar_wait(&bfull[s], ph, a.status, a.wait_ns)) {
              *s_abort = 1;
              break;
            }
            fence_after_sync();
            const uint32_t a_hi = saddr(sm + UvwSmem::a_off(int(s))), a_lo = a_hi + UV_A_BYTES;
            const uint32_t b_hi = saddr(sm + UvwSmem::b_off(int(s))), b_lo = b_hi + bhalf;
            const uint32_t big = tmem + (ci % UV_NBIG) * UV_NMAX, small = tmem + UV_NBIG * UV_NMAX;
#pragma unroll
            for (int ks = 0; ks < UV_KC / 8; ++ks) {
              const uint32_t o = uint32_t(ks) * 256;  // one K step: two 128-byte core matrices along K
              mma_tf32(big, smem_desc(a_hi + o, UV_KC), smem_desc(b_hi + o, UV_KC), idesc,
                       (ci < UV_NBIG && ks == 0) ? 0u : 1u);
              mma_tf32(small, smem_desc(a_hi + o, UV_KC), smem_desc(b_lo + o, UV_KC), idesc,
                       (ci == 0 && ks == 0) ? 0u : 1u);
              mma_tf32(small, smem_desc(a_lo + o, UV_KC), smem_desc(b_hi + o, UV_KC), idesc, 1u);
            }
            mma_commit(&aempty[s]);
            mma_commit(&bempty[s]);
            last = int64_t(q) + 1;
          }
        }
        if (*s_abort) break;
        mma_commit(accfull);
        ++tn;
      }
      if (*s_abort && last > 0) {
        // let the last committed MMA group finish (bounded) before the tensor memory is released
        const uint32_t lq = uint32_t(last - 1);
        bar_wait(&aempty[lq % UV_STAGES], (lq / UV_STAGES) & 1u, a.status, a.wait_ns);
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------- B producer (one thread)
    if (lane == 0) {
      uint32_t q = 0;
      for (int tile = blockIdx.x; tile < a.total_tiles && !*s_abort; tile += gridDim.x) {
        const UvwTarget& tg = a.tg[find_target(a, tile)];
        for (int j = tg.term_begin; j < tg.term_end && !*s_abort; ++j) {
          for (int kc = 0; kc < nk; ++kc, ++q) {
            const uint32_t s = q % UV_STAGES;
            if (!bar_wait(&bempty[s], ((q / UV_STAGES) & 1u) ^ 1u, a.status, a.wait_ns)) {
              *s_abort = 1;
              break;
            }
            bulk_copy(sm + UvwSmem::b_off(int(s)), a.prep + size_t(a.term[j].chunk0 + kc) * a.b_chunk_bytes,
                      a.b_chunk_bytes, &bfull[s]);
          }
        }
      }
      if (*s_abort) {
        // let the copies in flight land (bounded) before the CTA exits
        for (uint32_t k = q >= UV_STAGES ? q - UV_STAGES : 0; k < q; ++k)
          bar_wait(&bfull[k % UV_STAGES], (k / UV_STAGES) & 1u, a.status, a.wait_ns);
      }
    }
    __syncwarp();
  }
  fence_before_sync();
  __syncthreads();
  fence_after_sync();
  if (warp == 0) asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(UV_TMEM_COLS));
}

// Shared weights W [P][C][Cout] -> B chunks of 32 input channels, tf32 high part then low part,
// each [N rows x 32] K-major: the forward's chunks (p, kc) hold rows w, k = u - 32 kc; the
// backward's (after all forward chunks) rows u, k = w - 32 kc.
__global__ void uvw_prep_kernel(int P, int C, int Co, const float* __restrict__ w, unsigned char* __restrict__ prep) {
  const int64_t total = int64_t(P) * C * Co;
  const uint32_t fwd_bytes = 2u * uint32_t(Co) * UV_KC * 4, bwd_bytes = 2u * uint32_t(C) * UV_KC * 4;
  unsigned char* bwd = prep + size_t(P) * (C / UV_KC) * fwd_bytes;
  for (int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < total; i += int64_t(gridDim.x) * blockDim.x) {
    const int wc = int(i % Co);
    const int64_t pu = i / Co;
    const int u = int(pu % C), p = int(pu / C);
    const float v = __ldg(w + i);
    const float hi = to_tf32(v), lo = to_tf32(v - hi);
    unsigned char* f = prep + (size_t(p) * (C / UV_KC) + u / UV_KC) * fwd_bytes;
    *reinterpret_cast<float*>(f + kmajor_off(wc, u % UV_KC, UV_KC)) = hi;
    *reinterpret_cast<float*>(f + fwd_bytes / 2 + kmajor_off(wc, u % UV_KC, UV_KC)) = lo;
    unsigned char* g = bwd + (size_t(p) * (Co / UV_KC) + wc / UV_KC) * bwd_bytes;
    *reinterpret_cast<float*>(g + kmajor_off(u, wc % UV_KC, UV_KC)) = hi;
    *reinterpret_cast<float*>(g + bwd_bytes / 2 + kmajor_off(u, wc % UV_KC, UV_KC)) = lo;
  }
}

// ------------------------------------------------------------- grad_w (tensor cores) ---
// grad_W_p[u, w] = alpha_p sum_k T_p[k, u] g_p[k, w] over k = (sample, m3): a contraction whose K runs
// over the samples.  A tile is one path and GT_CHUNKS chunks of K; a chunk holds SK = floor(32 / D3)
// samples' D3 components (the last 32 - SK D3 positions stay zero).  The math warps write both
// operands of a chunk (A[u][k] = T_p, B[w][k] = the grad_out block, tf32 high and low parts) after
// putting the chunk's couplings sum_m2 C y in shared memory; one thread issues the three-pass MMAs
// into four TMEM accumulators as in the forward; after a tile the math warps add the accumulators
// and add alpha_p times them into grad_w (zeroed first) with atomics.  A tile sums at most
// 64 x 32 products per accumulator row, so no accumulator takes more than ~90 additions.
constexpr int GT_CHUNKS = 64;
constexpr int GT_STAGES = 3;
constexpr int GT_THREADS = 32 * UV_MATH_WARPS + 32;  // + the MMA warp
constexpr uint32_t GT_A_BYTES = UV_M * UV_KC * 4;     // one of hi, lo
constexpr uint32_t GT_B_BYTES = UV_NMAX * UV_KC * 4;  // one of hi, lo
constexpr int GT_CM = 32 * 7 * 7;                     // couplings of one chunk: SK x DI x D3 <= 32 x 7 x 7 floats

struct GtSmem {
  static constexpr size_t a_off(int s) { return size_t(s) * 2 * (GT_A_BYTES + GT_B_BYTES); }
  static constexpr size_t b_off(int s) { return a_off(s) + 2 * GT_A_BYTES; }
  static constexpr size_t cm_off() { return a_off(GT_STAGES); }                  // two buffers
  static constexpr size_t bar_off() { return cm_off() + 2 * GT_CM * 4; }
  // full, empty [GT_STAGES] each, accfull, accempty; then the TMEM slot and the abort flag
  static constexpr size_t total() { return bar_off() + 8 * (2 * GT_STAGES + 2) + 16; }
};

__device__ __forceinline__ int gt_find_path(const UvwBwdArgs& a, int tile) {
  int p = 0;
  while (p + 1 < a.P && tile >= a.path[p + 1].tile_begin) ++p;
  return p;
}

// One chunk (chunk index ch of the path) of path pp: couplings, then A and B into stage As / Bs.
template <int L1, int L2, int L3>
__device__ __noinline__ void gt_chunk(const UvwBwdArgs& a, const UvwPath& pp, int64_t ch, unsigned char* As,
                                      unsigned char* Bs, float* cmS, int tid) {
  constexpr int D1 = 2 * L1 + 1, D3 = 2 * L3 + 1, NY2 = (L2 + 1) * (L2 + 1), SK = UV_KC / D3;
  const int64_t bbase = ch * SK;
  if (tid < SK) {
    // couplings of sample tid: cm[i][t] = sum_m2 C[i, m2, t] y[m2]
    const int64_t b = bbase + tid;
    float Y[NY2];
#pragma unroll
    for (int m = 0; m < 2 * L2 + 1; ++m) Y[L2 * L2 + m] = b < a.B ? __ldg(a.y + b * a.dim2 + L2 * L2 + m) : 0.f;
    float* cm = cmS + tid * D1 * D3;
    static_for<0, D1>([&](auto ic) {
      static_for<0, D3>([&](auto tc) {
        constexpr int I = decltype(ic)::value, T = decltype(tc)::value;
        if constexpr (a_nz(L1, L2, L3, I - L1, T - L3))
          cm[I * D3 + T] = a_entry<float, L1, L2, L3, I - L1, T - L3>(Y);
        else
          cm[I * D3 + T] = 0.f;
      });
    });
  } else {
    // the next chunk's x and grad_out rows into L2 (one 128-byte line per thread and pass)
    const int64_t nb = bbase + SK;
    const int xl = (a.C * D1 * 4 + 127) / 128, gl = (a.Co * D3 * 4 + 127) / 128;
    for (int i = tid - SK; i < SK * (xl + gl); i += 32 * UV_MATH_WARPS - SK) {
      const int sl = i / (xl + gl), j = i - sl * (xl + gl);
      const int64_t b = nb + sl;
      if (b >= a.B) continue;
      const float* ptr = j < xl ? a.x + b * a.dim1 + pp.x_off + 32 * j : a.g + b * a.dim_out + pp.g_off + 32 * (j - xl);
      asm volatile("prefetch.global.L2 [%0];" ::"l"(ptr));
    }
  }
  asm volatile("bar.sync 1, %0;" ::"r"(32 * UV_MATH_WARPS) : "memory");
  // A[u][s D3 + m3] = T_p[b_s, u, m3] for channels u, u + 1 of sample s
  const int nq = a.C / 2;
  for (int task = tid; task < SK * nq; task += 32 * UV_MATH_WARPS) {
    const int sl = task / nq, u = 2 * (task - sl * nq);
    const int64_t b = bbase + sl;
    float T[2][D3];
#pragma unroll
    for (int c = 0; c < 2; ++c)
#pragma unroll
      for (int t = 0; t < D3; ++t) T[c][t] = 0.f;
    if (b < a.B) {
      const float2* xp = reinterpret_cast<const float2*>(a.x + b * a.dim1 + pp.x_off + int64_t(u) * D1);
      float xv[2 * D1];
#pragma unroll
      for (int j = 0; j < D1; ++j) {
        const float2 v = __ldg(xp + j);
        xv[2 * j] = v.x, xv[2 * j + 1] = v.y;
      }
      const float* cm = cmS + sl * D1 * D3;
#pragma unroll
      for (int i = 0; i < D1; ++i)
#pragma unroll
        for (int t = 0; t < D3; ++t) {
          const float cv = cm[i * D3 + t];
#pragma unroll
          for (int c = 0; c < 2; ++c) T[c][t] = fmaf(cv, xv[c * D1 + i], T[c][t]);
        }
    }
#pragma unroll
    for (int c = 0; c < 2; ++c)
#pragma unroll
      for (int t = 0; t < D3; ++t) {
        const float hi = to_tf32(T[c][t]), lo = to_tf32(T[c][t] - hi);
        const uint32_t off = kmajor_off(u + c, sl * D3 + t, UV_KC);
        *reinterpret_cast<float*>(As + off) = hi;
        *reinterpret_cast<float*>(As + GT_A_BYTES + off) = lo;
      }
  }
  // B[w][s D3 + m3] = g[b_s, o(p), w, m3]
  for (int task = tid; task < SK * a.Co; task += 32 * UV_MATH_WARPS) {
    const int sl = task / a.Co, w = task - sl * a.Co;
    const int64_t b = bbase + sl;
    const float* gp = a.g + (b < a.B ? b * a.dim_out + pp.g_off + int64_t(w) * D3 : 0);
#pragma unroll
    for (int t = 0; t < D3; ++t) {
      const float v = b < a.B ? __ldg(gp + t) : 0.f;
      const float hi = to_tf32(v), lo = to_tf32(v - hi);
      const uint32_t off = kmajor_off(w, sl * D3 + t, UV_KC);
      *reinterpret_cast<float*>(Bs + off) = hi;
      *reinterpret_cast<float*>(Bs + GT_B_BYTES + off) = lo;
    }
  }
}

__global__ void __launch_bounds__(GT_THREADS, 1) uvw_grad_w_tc_kernel(const __grid_constant__ UvwBwdArgs a) {
  extern __shared__ __align__(1024) unsigned char sm[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  uint64_t* full = reinterpret_cast<uint64_t*>(sm + GtSmem::bar_off());
  uint64_t* empty = full + GT_STAGES;
  uint64_t* accfull = empty + GT_STAGES;
  uint64_t* accempty = accfull + 1;
  uint32_t* tslot = reinterpret_cast<uint32_t*>(accempty + 1);
  volatile int* s_abort = reinterpret_cast<volatile int*>(tslot + 1);
  float* cmS = reinterpret_cast<float*>(sm + GtSmem::cm_off());

  // the operand positions no chunk writes (k past SK D3, rows past C or Co) stay zero
  for (size_t i = size_t(tid) * 16; i < GtSmem::cm_off(); i += size_t(GT_THREADS) * 16)
    *reinterpret_cast<float4*>(sm + i) = make_float4(0.f, 0.f, 0.f, 0.f);
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(saddr(tslot)),
                 "r"(UV_TMEM_COLS));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  if (tid == 0) {
    for (int i = 0; i < GT_STAGES; ++i) {
      bar_init(&full[i], UV_MATH_WARPS);
      bar_init(&empty[i], 1);
    }
    bar_init(accfull, 1);
    bar_init(accempty, UV_MATH_WARPS);
    *s_abort = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  fence_before_sync();
  __syncthreads();
  fence_after_sync();
  const uint32_t tmem = *tslot;

  // tiles in stride: a CTA's tiles mix paths of every degree (a contiguous range would leave the
  // CTAs with degree-0 paths, whose chunks hold 32 samples, far behind: measured 2x slower)
  if (warp < UV_MATH_WARPS) {
    uint32_t q = 0, tn = 0;
    bool ok = true;
    for (int tile = blockIdx.x; tile < a.total_tiles && ok; tile += gridDim.x, ++tn) {
      const UvwPath& pp = a.path[gt_find_path(a, tile)];
      const int64_t ch0 = int64_t(tile - pp.tile_begin) * GT_CHUNKS;
      const int nck = int(pp.chunks - ch0 < GT_CHUNKS ? pp.chunks - ch0 : GT_CHUNKS);
      for (int c = 0; c < nck; ++c, ++q) {
        const uint32_t s = q % GT_STAGES;
        // every math warp takes the same waits in the same order, so the block barrier inside the
        // chunk is reached by all of them or (after an abort flag, read once per chunk) by none
        const bool wok = warp_wait(&empty[s], ((q / GT_STAGES) & 1u) ^ 1u, a.status, a.wait_ns);
        if (!wok) *s_abort = 1;
        asm volatile("bar.sync 2, %0;" ::"r"(32 * UV_MATH_WARPS) : "memory");
        if (*s_abort) {
          ok = false;
          break;
        }
        unsigned char* As = sm + GtSmem::a_off(int(s));
        unsigned char* Bs = sm + GtSmem::b_off(int(s));
        float* cm = cmS + (q & 1u) * GT_CM;
        dispatch<E3_LMAX + 1>(pp.l1, [&](auto l1c) {
          dispatch<E3_LMAX + 1>(pp.l2, [&](auto l2c) {
            dispatch<E3_LMAX + 1>(pp.l3, [&](auto l3c) {
              constexpr int L1 = decltype(l1c)::value, L2 = decltype(l2c)::value, L3 = decltype(l3c)::value;
              if constexpr (triangle(L1, L2, L3)) gt_chunk<L1, L2, L3>(a, pp, ch0 + c, As, Bs, cm, tid);
            });
          });
        });
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // the tensor core reads through the async proxy
        __syncwarp();
        if (lane == 0) asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(saddr(&full[s])) : "memory");
      }
      if (!ok) break;
      const bool aok = warp_wait(accfull, tn & 1u, a.status, a.wait_ns);
      if (!aok) *s_abort = 1;
      asm volatile("bar.sync 2, %0;" ::"r"(32 * UV_MATH_WARPS) : "memory");  // one verdict for all math warps
      if (*s_abort) break;
      fence_after_sync();
      const int u = 32 * (warp & 3) + lane;
      const int nbig = nck < UV_NBIG ? nck : UV_NBIG;
      const uint32_t lane_base = tmem + (uint32_t(32 * (warp & 3)) << 16);
      for (int cc = 32 * (warp >> 2); cc < a.Co; cc += 64) {
        uint32_t v[32];
        float sum[32];
        tmem_ld32_nowait(lane_base + uint32_t(UV_NBIG * UV_NMAX + cc), v);
        asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
        for (int i = 0; i < 32; ++i) sum[i] = __uint_as_float(v[i]);
        for (int k = 0; k < nbig; ++k) {
          tmem_ld32_nowait(lane_base + uint32_t(k * UV_NMAX + cc), v);
          asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
          for (int i = 0; i < 32; ++i) sum[i] += __uint_as_float(v[i]);
        }
        if (u < a.C) {
          float* dst = a.grad_w + pp.w_off + int64_t(u) * a.Co + cc;
#pragma unroll
          for (int i = 0; i < 32; ++i) atomicAdd(dst + i, pp.alpha * sum[i]);
        }
      }
      fence_before_sync();
      __syncwarp();
      if (lane == 0) asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(saddr(accempty)) : "memory");
    }
    __syncwarp();
  } else if (lane == 0) {
    // ------------------------------------------------------------- MMA thread
    const uint32_t idesc = idesc_tf32(UV_M, a.Co);
    uint32_t q = 0, tn = 0;
    int64_t last = -1;
    for (int tile = blockIdx.x; tile < a.total_tiles && !*s_abort; tile += gridDim.x, ++tn) {
      const UvwPath& pp = a.path[gt_find_path(a, tile)];
      const int64_t ch0 = int64_t(tile - pp.tile_begin) * GT_CHUNKS;
      const int nck = int(pp.chunks - ch0 < GT_CHUNKS ? pp.chunks - ch0 : GT_CHUNKS);
      if (!bar_wait(accempty, (tn & 1u) ^ 1u, a.status, a.wait_ns)) {
        *s_abort = 1;
        break;
      }
      fence_after_sync();
      for (int c = 0; c < nck; ++c, ++q) {
        const uint32_t s = q % GT_STAGES;
        if (!bar_wait(&full[s], (q / GT_STAGES) & 1u, a.status, a.wait_ns)) {
          *s_abort = 1;
          break;
        }
        fence_after_sync();
        const uint32_t a_hi = saddr(sm + GtSmem::a_off(int(s))), a_lo = a_hi + GT_A_BYTES;
        const uint32_t b_hi = saddr(sm + GtSmem::b_off(int(s))), b_lo = b_hi + GT_B_BYTES;
        const uint32_t big = tmem + (uint32_t(c) % UV_NBIG) * UV_NMAX, small = tmem + UV_NBIG * UV_NMAX;
#pragma unroll
        for (int ks = 0; ks < UV_KC / 8; ++ks) {
          const uint32_t o = uint32_t(ks) * 256;
          mma_tf32(big, smem_desc(a_hi + o, UV_KC), smem_desc(b_hi + o, UV_KC), idesc, (c < UV_NBIG && ks == 0) ? 0u : 1u);
          mma_tf32(small, smem_desc(a_hi + o, UV_KC), smem_desc(b_lo + o, UV_KC), idesc, (c == 0 && ks == 0) ? 0u : 1u);
          mma_tf32(small, smem_desc(a_lo + o, UV_KC), smem_desc(b_hi + o, UV_KC), idesc, 1u);
        }
        mma_commit(&empty[s]);
        last = int64_t(q) + 1;
      }
      if (*s_abort) break;
      mma_commit(accfull);
    }
    if (*s_abort && last > 0) {
      const uint32_t lq = uint32_t(last - 1);
      bar_wait(&empty[lq % GT_STAGES], (lq / GT_STAGES) & 1u, a.status, a.wait_ns);
    }
  }
  fence_before_sync();
  __syncthreads();
  fence_after_sync();
  if (warp == 0) asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(UV_TMEM_COLS));
}

// ------------------------------------------------------------------ grad_y ---
// grad_y[b, l2, m2] = sum_p alpha_p sum_{m1, m3} C_p[m1, m2, m3] sum_u x[b, u, m1] Z_p[b, u, m3],
// Z_p[b, u, m3] = sum_w W_p[u, w] g[b, o(p), w, m3].  Z (every path, a batch of samples) comes from
// the tensor-core kernel in its plain role; here a CTA of C threads (thread u) takes one sample,
// contracts its x and Z rows with the coefficients path by path, and sums over the channels with
// warp shuffles and shared-memory atomics into the sample's grad_y.
constexpr int GY_NY = (E3_LMAX + 1) * (E3_LMAX + 1);

template <int L1, int L2, int L3>
__device__ __forceinline__ void gy_path(const UvwBwdArgs& a, const UvwPath& pp, int64_t b, const float* zrow, float* qS) {
  constexpr int D1 = 2 * L1 + 1, D2 = 2 * L2 + 1, D3 = 2 * L3 + 1;
  const int u = threadIdx.x;
  float xv[D1], zv[D3];
#pragma unroll
  for (int m = 0; m < D1; ++m) xv[m] = __ldg(a.x + b * a.dim1 + pp.x_off + int64_t(u) * D1 + m);
#pragma unroll
  for (int m = 0; m < D3; ++m) zv[m] = __ldg(zrow + int64_t(pp.z_off) * a.C + int64_t(u) * D3 + m);
  float c[D2];
#pragma unroll
  for (int m = 0; m < D2; ++m) c[m] = 0.f;
  static_for<-L1, L1 + 1>([&](auto m1c) {
    static_for<-L2, L2 + 1>([&](auto m2c) {
      static_for<-L3, L3 + 1>([&](auto m3c) {
        constexpr int M1 = decltype(m1c)::value, M2 = decltype(m2c)::value, M3 = decltype(m3c)::value;
        if constexpr (cg_nz(L1, L2, L3, M1, M2, M3)) {
          constexpr int I = cg_index(L1, L2, L3, M1, M2, M3);
          c[M2 + L2] = fmaf(CGT<float>::template get<I>() * xv[M1 + L1], zv[M3 + L3], c[M2 + L2]);
        }
      });
    });
  });
#pragma unroll
  for (int m = 0; m < D2; ++m) {
    float v = pp.alpha * c[m];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    if ((threadIdx.x & 31) == 0) atomicAdd(&qS[L2 * L2 + m], v);
  }
}

__global__ void __launch_bounds__(UV_NMAX) uvw_grad_y_kernel(const __grid_constant__ UvwBwdArgs a, const float* z,
                                                             int64_t z_stride, int64_t b0) {
  __shared__ float qS[GY_NY];
  const int64_t b = b0 + blockIdx.x;
  if (threadIdx.x < GY_NY) qS[threadIdx.x] = 0.f;
  __syncthreads();
  const float* zrow = z + int64_t(blockIdx.x) * z_stride;
  for (int p = 0; p < a.P; ++p) {
    const UvwPath& pp = a.path[p];
    dispatch<E3_LMAX + 1>(pp.l1, [&](auto l1c) {
      dispatch<E3_LMAX + 1>(pp.l2, [&](auto l2c) {
        dispatch<E3_LMAX + 1>(pp.l3, [&](auto l3c) {
          constexpr int L1 = decltype(l1c)::value, L2 = decltype(l2c)::value, L3 = decltype(l3c)::value;
          if constexpr (triangle(L1, L2, L3)) gy_path<L1, L2, L3>(a, pp, b, zrow, qS);
        });
      });
    });
  }
  __syncthreads();
  if (threadIdx.x < a.dim2) a.grad_y[b * a.dim2 + threadIdx.x] = qS[threadIdx.x];
}

}  // namespace

e3_status upload_tables_uvw(const double* t64, const float* t32) {
  const cudaError_t err = upload_tables(t64, t32);
  if (err != cudaSuccess) return fail(E3_ERR_CUDA, "uploading the CG table failed: %s", cudaGetErrorString(err));
  return E3_OK;
}

size_t uvw_prep_bytes(int P, int C, int Co) { return size_t(16) * P * C * Co; }

e3_status launch_uvw_prep(int P, int C, int Co, const float* w, void* prep, void* stream) {
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int64_t total = int64_t(P) * C * Co;
  const int blocks = int(std::min<int64_t>((total + 255) / 256, 4 * 148));
  uvw_prep_kernel<<<blocks, 256, 0, s>>>(P, C, Co, w, static_cast<unsigned char*>(prep));
  const cudaError_t err = cudaGetLastError();
  if (err != cudaSuccess) return fail(E3_ERR_CUDA, "uvw prep launch failed: %s", cudaGetErrorString(err));
  return E3_OK;
}

e3_status launch_uvw_gemm(const UvwGemmArgs& a, int role, void* stream) {
  if (a.total_tiles <= 0 || a.B == 0) return E3_OK;
  if (a.N % 32 != 0 || a.N > UV_NMAX || a.k_in % UV_KC != 0) return fail(E3_ERR_UNSUPPORTED, "uvw channel counts");
  const size_t smem = UvwSmem::total();
  cudaError_t err =
      role == ROLE_FWD  ? cudaFuncSetAttribute(uvw_gemm_kernel<ROLE_FWD>, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem))
      : role == ROLE_GX ? cudaFuncSetAttribute(uvw_gemm_kernel<ROLE_GX>, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem))
                        : cudaFuncSetAttribute(uvw_gemm_kernel<ROLE_PLAIN>, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
  if (err != cudaSuccess) return fail(E3_ERR_CUDA, "uvw smem attribute: %s", cudaGetErrorString(err));
  const int grid = std::min(a.total_tiles, sm_count());
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (role == ROLE_FWD)
    uvw_gemm_kernel<ROLE_FWD><<<grid, UV_THREADS, smem, s>>>(a);
  else if (role == ROLE_GX)
    uvw_gemm_kernel<ROLE_GX><<<grid, UV_THREADS, smem, s>>>(a);
  else
    uvw_gemm_kernel<ROLE_PLAIN><<<grid, UV_THREADS, smem, s>>>(a);
  err = cudaGetLastError();
  if (err != cudaSuccess) return fail(E3_ERR_CUDA, "uvw launch failed: %s", cudaGetErrorString(err));
  return E3_OK;
}

}  // namespace e3b

namespace e3b {

e3_status launch_uvw_grad_w(const UvwBwdArgs& in, void* stream) {
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t err = cudaMemsetAsync(in.grad_w, 0, sizeof(float) * size_t(in.P) * in.C * in.Co, s);
  if (err != cudaSuccess) return fail(E3_ERR_CUDA, "zeroing grad_w failed: %s", cudaGetErrorString(err));
  if (in.B == 0) return E3_OK;
  UvwBwdArgs a = in;
  int64_t tiles = 0;
  for (int p = 0; p < a.P; ++p) {
    const int64_t sk = UV_KC / (2 * a.path[p].l3 + 1);
    a.path[p].chunks = (a.B + sk - 1) / sk;
    a.path[p].tile_begin = int32_t(tiles);
    tiles += (a.path[p].chunks + GT_CHUNKS - 1) / GT_CHUNKS;
  }
  if (tiles >= INT_MAX) return fail(E3_ERR_SHAPE, "B too large");
  a.total_tiles = int32_t(tiles);
  const size_t smem = GtSmem::total();
  err = cudaFuncSetAttribute(uvw_grad_w_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
  if (err != cudaSuccess) return fail(E3_ERR_CUDA, "uvw grad_w smem attribute: %s", cudaGetErrorString(err));
  const int grid = int(std::min<int64_t>(tiles, sm_count()));
  uvw_grad_w_tc_kernel<<<grid, GT_THREADS, smem, s>>>(a);
  err = cudaGetLastError();
  if (err != cudaSuccess) return fail(E3_ERR_CUDA, "uvw grad_w launch failed: %s", cudaGetErrorString(err));
  return E3_OK;
}

e3_status launch_uvw_grad_y(const UvwBwdArgs& a, const float* z, int64_t z_stride, int64_t b0, int64_t nb,
                            void* stream) {
  if (nb <= 0) return E3_OK;
  if (nb > INT_MAX) return fail(E3_ERR_SHAPE, "batch too large");
  uvw_grad_y_kernel<<<unsigned(nb), a.C, 0, static_cast<cudaStream_t>(stream)>>>(a, z, z_stride, b0);
  const cudaError_t err = cudaGetLastError();
  if (err != cudaSuccess) return fail(E3_ERR_CUDA, "uvw grad_y launch failed: %s", cudaGetErrorString(err));
  return E3_OK;
}

}  // namespace e3b
