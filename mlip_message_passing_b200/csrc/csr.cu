// Receiver / sender CSR segmentation of an edge list, and a row gather, for sm_100a.
//
// E3J, section E.2.2: the convolution aggregates messages per receiver over a CSR adjacency
// so that no atomics are needed; section C.2: aggregation must be deterministic.  The
// segmentation here is integer-only and bit-exact: perm_dst is the stable sort of the edges
// by receiver, perm_src the stable sort of that order by sender, and the row pointers are
// exclusive prefix sums of the degree counts.
//
// The stable sorts are least-significant-digit radix sorts with 8-bit digits over the
// ceil(log2 N) bits that a node id can use.  Each pass: per-tile digit counts, one exclusive
// scan over the (digit, tile) table in digit-major order, then a scatter in which every tile
// ranks its elements stably (tile rounds of 256 elements in input order, warp-level match of
// equal digits, per-warp counts combined in warp order).  Counting uses integer atomics in
// shared memory only; ranks never depend on thread scheduling, so the output is unique.
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <mutex>

#include "internal.h"

namespace e3b {

constexpr int RS_THREADS = 256;
constexpr int RS_ROUNDS = 8;  // rounds of 256 elements per tile
constexpr int RS_TILE = RS_THREADS * RS_ROUNDS;
constexpr int RS_RADIX = 256;

__device__ __forceinline__ void rs_error(int* status, int code) { atomicCAS(status, 0, code); }

// key of element i: keys[j] with j = gather ? gather[i] : i; when `other` is given, an edge whose
// id in either array is -1 (padding) gets the key `pad` (one past the largest node id), so the
// stable sort puts padding edges after every valid edge, in element order
__device__ __forceinline__ uint32_t rs_key(const int32_t* __restrict__ keys, const int32_t* __restrict__ other,
                                           const int32_t* __restrict__ gather, int64_t i, uint32_t pad) {
  const int64_t j = gather ? int64_t(__ldg(gather + i)) : i;
  const int32_t k = __ldg(keys + j);
  if (other != nullptr && (k == -1 || __ldg(other + j) == -1)) return pad;
  return uint32_t(k);
}

// counts[d * n_tiles + tile] = number of elements of `tile` whose digit is d
__global__ void __launch_bounds__(RS_THREADS) rs_count(const int32_t* __restrict__ keys,
                                                       const int32_t* __restrict__ other,
                                                       const int32_t* __restrict__ gather, uint32_t pad, int64_t n,
                                                       int shift, int n_tiles, int32_t* __restrict__ counts) {
  __shared__ int32_t h[RS_RADIX];
  h[threadIdx.x] = 0;
  __syncthreads();
  const int64_t base = int64_t(blockIdx.x) * RS_TILE;
  for (int r = 0; r < RS_ROUNDS; ++r) {
    const int64_t i = base + int64_t(r) * RS_THREADS + threadIdx.x;
    if (i < n) atomicAdd(&h[(rs_key(keys, other, gather, i, pad) >> shift) & 0xff], 1);
  }
  __syncthreads();
  counts[int64_t(threadIdx.x) * n_tiles + blockIdx.x] = h[threadIdx.x];
}

// In-place exclusive scan of a[0..n) by one CTA of 1024 threads (chunked serial sums, then a
// block scan of the chunk totals).  total (optional) receives the sum.
__global__ void __launch_bounds__(1024) exclusive_scan_1cta(int32_t* __restrict__ a, int64_t n,
                                                            int32_t* __restrict__ total) {
  __shared__ int32_t part[1024];
  const int t = threadIdx.x;
  const int64_t chunk = (n + 1023) / 1024;
  const int64_t b = t * chunk, e = b + chunk < n ? b + chunk : n;
  int32_t s = 0;
  for (int64_t i = b; i < e; ++i) s += a[i];
  part[t] = s;
  __syncthreads();
  for (int off = 1; off < 1024; off <<= 1) {
    const int32_t v = t >= off ? part[t - off] : 0;
    __syncthreads();
    part[t] += v;
    __syncthreads();
  }
  int32_t run = part[t] - s;  // exclusive prefix of this chunk
  for (int64_t i = b; i < e; ++i) {
    const int32_t v = a[i];
    a[i] = run;
    run += v;
  }
  if (total != nullptr && t == 1023) *total = part[1023];
}

// Stable scatter of one pass.  offsets: exclusive scan of counts (digit-major).
__global__ void __launch_bounds__(RS_THREADS) rs_scatter(const int32_t* __restrict__ keys,
                                                         const int32_t* __restrict__ other,
                                                         const int32_t* __restrict__ gather, uint32_t pad,
                                                         const int32_t* __restrict__ vals_in, int64_t n, int shift,
                                                         int n_tiles, const int32_t* __restrict__ offsets,
                                                         int32_t* __restrict__ keys_out,
                                                         int32_t* __restrict__ vals_out) {
  __shared__ int32_t run[RS_RADIX];              // running count per digit in this tile
  __shared__ int32_t wc[RS_THREADS / 32][RS_RADIX];  // per-warp counts of the current round
  const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
  run[t] = offsets[int64_t(t) * n_tiles + blockIdx.x];
  const int64_t base = int64_t(blockIdx.x) * RS_TILE;
  for (int r = 0; r < RS_ROUNDS; ++r) {
    for (int q = t; q < (RS_THREADS / 32) * RS_RADIX; q += RS_THREADS) (&wc[0][0])[q] = 0;
    __syncthreads();
    const int64_t i = base + int64_t(r) * RS_THREADS + t;
    const bool ok = i < n;
    uint32_t key = 0;
    int d = RS_RADIX;  // sentinel: no element
    if (ok) {
      key = rs_key(keys, other, gather, i, pad);
      d = int((key >> shift) & 0xff);
    }
    const unsigned peers = __match_any_sync(0xffffffffu, d);
    const int rank_in_warp = __popc(peers & ((1u << lane) - 1u));
    if (ok && rank_in_warp == 0) wc[warp][d] = __popc(peers);
    __syncthreads();
    if (ok) {
      int32_t pos = run[d] + rank_in_warp;
      for (int w = 0; w < warp; ++w) pos += wc[w][d];
      if (keys_out) keys_out[pos] = int32_t(key);
      vals_out[pos] = vals_in ? __ldg(vals_in + i) : int32_t(i);
    }
    __syncthreads();
    {
      int32_t add = 0;
      for (int w = 0; w < RS_THREADS / 32; ++w) add += wc[w][t];
      run[t] += add;
    }
    __syncthreads();
  }
}

// degree counts (row_ptr[id] += 1); padding edges (-1 in ids or other) are skipped, other ids
// outside [0, N) are reported and skipped
__global__ void degree_count(const int32_t* __restrict__ ids, const int32_t* __restrict__ other, int64_t n, int64_t N,
                             int32_t* __restrict__ row_ptr, int* status) {
  for (int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < n; i += int64_t(gridDim.x) * blockDim.x) {
    const int32_t v = __ldg(ids + i);
    if (v == -1 || __ldg(other + i) == -1) continue;
    if (v < 0 || v >= N) {
      rs_error(status, E3_ERR_INDEX);
      continue;
    }
    atomicAdd(row_ptr + v, 1);
  }
}

__global__ void gather_rows_kernel(int64_t n_rows, int64_t n_in_rows, int64_t row_words, bool vec16,
                                   const int32_t* __restrict__ perm, const uint32_t* __restrict__ in,
                                   uint32_t* __restrict__ out, int* status) {
  const int64_t per_row = vec16 ? row_words / 4 : row_words;
  const int64_t total = n_rows * per_row;
  for (int64_t q = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; q < total; q += int64_t(gridDim.x) * blockDim.x) {
    const int64_t r = q / per_row, c = q % per_row;
    const int32_t s = __ldg(perm + r);
    if (s < 0 || s >= n_in_rows) {
      rs_error(status, E3_ERR_INDEX);
      continue;
    }
    if (vec16)
      reinterpret_cast<uint4*>(out)[r * per_row + c] = __ldg(reinterpret_cast<const uint4*>(in) + int64_t(s) * per_row + c);
    else
      out[r * row_words + c] = __ldg(in + int64_t(s) * row_words + c);
  }
}

// out[idx[r], :] += in[r, :] for rows r < n_rows of `words` elements of T; the indices of one call
// are distinct (the caller's contract), so no two threads touch one element and the result does
// not depend on scheduling.
template <typename T>
__global__ void add_rows_kernel(int64_t n_rows, int64_t n_out_rows, int64_t words, const int32_t* __restrict__ idx,
                                const T* __restrict__ in, T* __restrict__ out, int* status) {
  const int64_t total = n_rows * words;
  for (int64_t q = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; q < total; q += int64_t(gridDim.x) * blockDim.x) {
    const int64_t r = q / words, c = q % words;
    const int32_t d = __ldg(idx + r);
    if (d < 0 || d >= n_out_rows) {
      rs_error(status, E3_ERR_INDEX);
      continue;
    }
    out[int64_t(d) * words + c] += in[q];
  }
}

// ------------------------------------------------------------------- node reordering ---
// Morton (Z-order) code of a position: each coordinate quantised to 10 bits inside the box
// (scale = 1024 / extent in double, floor, clamp), bit b of axis k goes to bit 3 b + k.
constexpr int MORTON_BITS = 10;
template <typename T>
__global__ void morton_code_kernel(int64_t n, const T* __restrict__ pos, double lo0, double lo1, double lo2,
                                   double s0, double s1, double s2, int32_t* __restrict__ codes) {
  for (int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < n; i += int64_t(gridDim.x) * blockDim.x) {
    const double lo[3] = {lo0, lo1, lo2}, sc[3] = {s0, s1, s2};
    uint32_t code = 0;
#pragma unroll
    for (int k = 0; k < 3; ++k) {
      const double f = floor((double(pos[3 * i + k]) - lo[k]) * sc[k]);
      const uint32_t q = f < 0.0 ? 0u : (f > double((1 << MORTON_BITS) - 1) ? uint32_t((1 << MORTON_BITS) - 1) : uint32_t(f));
#pragma unroll
      for (int b = 0; b < MORTON_BITS; ++b) code |= ((q >> b) & 1u) << (3 * b + k);
    }
    codes[i] = int32_t(code);
  }
}

// inv[perm[i]] = i (entries out of range are reported and skipped)
__global__ void invert_perm_kernel(int64_t n, const int32_t* __restrict__ perm, int32_t* __restrict__ inv,
                                   int* status) {
  for (int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < n; i += int64_t(gridDim.x) * blockDim.x) {
    const int32_t p = perm[i];
    if (p < 0 || p >= n) {
      atomicCAS(status, 0, int(E3_ERR_INDEX));
      continue;
    }
    inv[p] = int32_t(i);
  }
}

// out[i] = map[ids[i]] (ids out of range are reported and give -1)
__global__ void remap_ids_kernel(int64_t n, const int32_t* __restrict__ ids, int64_t N, const int32_t* __restrict__ map,
                                 int32_t* __restrict__ out, int* status) {
  for (int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < n; i += int64_t(gridDim.x) * blockDim.x) {
    const int32_t id = ids[i];
    if (id < 0 || id >= N) {
      atomicCAS(status, 0, int(E3_ERR_INDEX));
      out[i] = -1;
      continue;
    }
    out[i] = __ldg(map + id);
  }
}

// Segments per row, in processing order: entry i counts the segments of row order[i] (row i
// without an order); at least one, so that every row is written; seg_start[N] = 0 for the scan.
// A row whose pointers are out of range, or an order entry out of range, counts one (empty)
// segment.
__global__ void seg_count_kernel(int64_t N, int64_t E, const int32_t* __restrict__ row_ptr,
                                 const int32_t* __restrict__ order, int32_t* __restrict__ seg_start) {
  for (int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i <= N; i += int64_t(gridDim.x) * blockDim.x) {
    if (i == N) {
      seg_start[N] = 0;
      continue;
    }
    const int64_t n = order != nullptr ? int64_t(order[i]) : i;
    int64_t deg = 0;
    if (n >= 0 && n < N) {
      const int64_t r0 = row_ptr[n], r1 = row_ptr[n + 1];
      if (r0 >= 0 && r1 >= r0 && r1 <= E) deg = r1 - r0;
    }
    seg_start[i] = deg <= SEG_EDGES ? 1 : int32_t((deg + SEG_EDGES - 1) / SEG_EDGES);
  }
}

// The units of each row in processing order: {row, first edge, end edge, segment} and the row's
// segment count; the number of units goes to *units.  Rows whose pointers are out of range, and
// order entries out of range, record E3_ERR_INDEX and get empty units; units beyond units_max
// (row pointers that overlap) record E3_ERR_INDEX and are dropped.
__global__ void unit_fill_kernel(int64_t N, int64_t E, int64_t units_max, const int32_t* __restrict__ row_ptr,
                                 const int32_t* __restrict__ order, const int32_t* __restrict__ seg_start,
                                 int4* __restrict__ info, int32_t* __restrict__ nseg, int32_t* __restrict__ units,
                                 int* status) {
  for (int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < N; i += int64_t(gridDim.x) * blockDim.x) {
    int64_t n = order != nullptr ? int64_t(order[i]) : i;
    int64_t r0 = 0, r1 = 0;
    if (n < 0 || n >= N) {
      atomicCAS(status, 0, int(E3_ERR_INDEX));
      n = 0;
    } else {
      r0 = row_ptr[n];
      r1 = row_ptr[n + 1];
      if (r0 < 0 || r1 < r0 || r1 > E) {
        atomicCAS(status, 0, int(E3_ERR_INDEX));
        r0 = r1 = 0;
      }
    }
    const int32_t u0 = seg_start[i], k = seg_start[i + 1] - u0;
    for (int32_t s = 0; s < k; ++s) {
      if (u0 < 0 || int64_t(u0) + s >= units_max) {
        atomicCAS(status, 0, int(E3_ERR_INDEX));
        break;
      }
      const int64_t e0 = r0 + int64_t(s) * SEG_EDGES;
      const int64_t e1 = e0 + SEG_EDGES < r1 ? e0 + SEG_EDGES : r1;
      info[u0 + s] = make_int4(int(n), int(e0 < e1 ? e0 : e1), int(e1), s);
      nseg[u0 + s] = k;
    }
    if (i == N - 1) *units = int32_t(seg_start[N] < units_max ? seg_start[N] : units_max);
  }
}

// rows [*first_row, n_rows) of 4-byte words set to zero (padding positions after the last row)
__global__ void zero_tail_kernel(const int32_t* __restrict__ first_row, int64_t n_rows, int64_t row_words,
                                 uint32_t* __restrict__ p) {
  const int64_t start = *first_row;
  if (start < 0 || start >= n_rows) return;
  const int64_t total = (n_rows - start) * row_words;
  uint32_t* q = p + start * row_words;
  for (int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < total; i += int64_t(gridDim.x) * blockDim.x)
    q[i] = 0u;
}

// ------------------------------------------------------------------------ host side ---
static int64_t n_tiles_of(int64_t E) { return (E + RS_TILE - 1) / RS_TILE; }
static size_t align256(size_t b) { return (b + 255) & ~size_t(255); }

static size_t csr_ws_bytes(int64_t E) {
  const int64_t nt = n_tiles_of(E) > 0 ? n_tiles_of(E) : 1;
  return 4 * align256(sizeof(int32_t) * size_t(E > 0 ? E : 1)) + align256(sizeof(int32_t) * size_t(RS_RADIX) * nt);
}

static int key_bits(int64_t N) {
  int b = 1;
  while ((int64_t(1) << b) < N) ++b;
  return b;
}

// Stable sort of element indices 0..n by key(i) (see rs_key); writes the sorted indices to vals_final.
static e3_status radix_sort(const int32_t* keys, const int32_t* other, const int32_t* gather, uint32_t pad, int64_t n,
                            int bits, int32_t* vals_final, int32_t* ka, int32_t* va, int32_t* kb, int32_t* vb,
                            int32_t* counts, cudaStream_t s) {
  const int n_tiles = int(n_tiles_of(n));
  const int passes = (bits + 7) / 8;
  const int32_t* kin = keys;
  const int32_t* oin = other;
  const int32_t* gin = gather;
  const int32_t* vin = nullptr;
  for (int p = 0; p < passes; ++p) {
    const bool last = p == passes - 1;
    int32_t* kout = last ? nullptr : (p % 2 == 0 ? ka : kb);
    int32_t* vout = last ? vals_final : (p % 2 == 0 ? va : vb);
    rs_count<<<n_tiles, RS_THREADS, 0, s>>>(kin, oin, gin, pad, n, 8 * p, n_tiles, counts);
    exclusive_scan_1cta<<<1, 1024, 0, s>>>(counts, int64_t(RS_RADIX) * n_tiles, nullptr);
    rs_scatter<<<n_tiles, RS_THREADS, 0, s>>>(kin, oin, gin, pad, vin, n, 8 * p, n_tiles, counts, kout, vout);
    kin = kout;  // later passes read the (padding-resolved) keys the scatter wrote
    oin = nullptr;
    gin = nullptr;
    vin = vout;
  }
  const cudaError_t err = cudaGetLastError();
  if (err != cudaSuccess) return fail(E3_ERR_CUDA, "radix sort launch failed: %s", cudaGetErrorString(err));
  return E3_OK;
}

e3_status build_topo_part(int64_t N, int64_t E, const int32_t* row_ptr, const int32_t* order, unsigned char* base,
                          const TopoPart& t, void* stream) {
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int32_t* units = reinterpret_cast<int32_t*>(base + t.units);
  cudaError_t err = cudaMemsetAsync(units, 0, 16, s);
  if (err != cudaSuccess) return fail(E3_ERR_CUDA, "memset failed: %s", cudaGetErrorString(err));
  if (N <= 0) return E3_OK;
  int* status = nullptr;
  e3_status st = device_status_ptr(&status);
  if (st != E3_OK) return st;
  int32_t* seg_start = reinterpret_cast<int32_t*>(base + t.seg_start);
  const int blocks = int(std::min<int64_t>((N + 256) / 256, 148 * 8));
  seg_count_kernel<<<blocks, 256, 0, s>>>(N, E, row_ptr, order, seg_start);
  exclusive_scan_1cta<<<1, 1024, 0, s>>>(seg_start, N + 1, nullptr);
  unit_fill_kernel<<<blocks, 256, 0, s>>>(N, E, seg_units_max(N, E), row_ptr, order, seg_start,
                                          reinterpret_cast<int4*>(base + t.info),
                                          reinterpret_cast<int32_t*>(base + t.nseg), units, status);
  err = cudaGetLastError();
  if (err != cudaSuccess) return fail(E3_ERR_CUDA, "topology launch failed: %s", cudaGetErrorString(err));
  return E3_OK;
}

e3_status zero_rows_after(const int32_t* first_row, int64_t n_rows, int64_t row_bytes, void* ptr, void* stream) {
  if (n_rows <= 0 || row_bytes <= 0) return E3_OK;
  zero_tail_kernel<<<148 * 4, 256, 0, static_cast<cudaStream_t>(stream)>>>(first_row, n_rows, row_bytes / 4,
                                                                            static_cast<uint32_t*>(ptr));
  const cudaError_t err = cudaGetLastError();
  if (err != cudaSuccess) return fail(E3_ERR_CUDA, "zero launch failed: %s", cudaGetErrorString(err));
  return E3_OK;
}

}  // namespace e3b

using namespace e3b;

extern "C" e3_status e3_csr_workspace_size(int64_t N, int64_t E, size_t* bytes) {
  clear_error();
  if (bytes == nullptr) return fail(E3_ERR_INVALID_ARG, "bytes is NULL");
  if (N < 0 || E < 0 || N >= (int64_t(1) << 31) || E >= (int64_t(1) << 31))
    return fail(E3_ERR_SHAPE, "N or E out of range");
  *bytes = csr_ws_bytes(E);
  return E3_OK;
}

extern "C" e3_status e3_csr_build(int64_t N, int64_t E, const int32_t* src, const int32_t* dst, int32_t* perm_dst,
                                  int32_t* row_ptr_dst, int32_t* perm_src, int32_t* row_ptr_src, void* workspace,
                                  size_t ws_bytes, void* stream) {
  clear_error();
  if (N < 0 || E < 0 || N >= (int64_t(1) << 31) || E >= (int64_t(1) << 31))
    return fail(E3_ERR_SHAPE, "N or E out of range");
  if (row_ptr_dst == nullptr || row_ptr_src == nullptr) return fail(E3_ERR_INVALID_ARG, "row_ptr array is NULL");
  if (E > 0 && (src == nullptr || dst == nullptr || perm_dst == nullptr || perm_src == nullptr))
    return fail(E3_ERR_INVALID_ARG, "edge array is NULL");
  if (E > 0 && N == 0) return fail(E3_ERR_SHAPE, "edges without nodes");
  if (E > 0 && (workspace == nullptr || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0))
    return fail(E3_ERR_INVALID_ARG, "workspace is NULL or not 256-byte aligned");
  if (E > 0 && ws_bytes < csr_ws_bytes(E))
    return fail(E3_ERR_SHAPE, "workspace of %zu bytes, need %zu", ws_bytes, csr_ws_bytes(E));
  int* status = nullptr;
  e3_status st = device_status_ptr(&status);
  if (st != E3_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t err = cudaMemsetAsync(row_ptr_dst, 0, sizeof(int32_t) * size_t(N + 1), s);
  if (err == cudaSuccess) err = cudaMemsetAsync(row_ptr_src, 0, sizeof(int32_t) * size_t(N + 1), s);
  if (err != cudaSuccess) return fail(E3_ERR_CUDA, "memset failed: %s", cudaGetErrorString(err));
  if (E == 0) return E3_OK;
  const int blocks = int(std::min<int64_t>((E + 255) / 256, 148 * 8));
  degree_count<<<blocks, 256, 0, s>>>(dst, src, E, N, row_ptr_dst, status);
  degree_count<<<blocks, 256, 0, s>>>(src, dst, E, N, row_ptr_src, status);
  // row_ptr[n] = c_n for n < N and row_ptr[N] = 0: one exclusive scan over N + 1 entries
  // gives row_ptr[n] = sum_{m < n} c_m and row_ptr[N] = E
  exclusive_scan_1cta<<<1, 1024, 0, s>>>(row_ptr_dst, N + 1, nullptr);
  exclusive_scan_1cta<<<1, 1024, 0, s>>>(row_ptr_src, N + 1, nullptr);
  err = cudaGetLastError();
  if (err != cudaSuccess) return fail(E3_ERR_CUDA, "count launch failed: %s", cudaGetErrorString(err));

  char* ws = static_cast<char*>(workspace);
  const size_t eb = align256(sizeof(int32_t) * size_t(E));
  int32_t* ka = reinterpret_cast<int32_t*>(ws);
  int32_t* va = reinterpret_cast<int32_t*>(ws + eb);
  int32_t* kb = reinterpret_cast<int32_t*>(ws + 2 * eb);
  int32_t* vb = reinterpret_cast<int32_t*>(ws + 3 * eb);
  int32_t* counts = reinterpret_cast<int32_t*>(ws + 4 * eb);
  const int bits = key_bits(N + 1);  // padding edges take key N
  st = radix_sort(dst, src, nullptr, uint32_t(N), E, bits, perm_dst, ka, va, kb, vb, counts, s);
  if (st != E3_OK) return st;
  st = radix_sort(src, dst, perm_dst, uint32_t(N), E, bits, perm_src, ka, va, kb, vb, counts, s);
  return st;
}

extern "C" e3_status e3_gather_rows(int64_t n_rows, int64_t n_in_rows, int64_t row_bytes, const int32_t* perm,
                                    const void* in, void* out, void* stream) {
  clear_error();
  if (n_rows < 0 || n_in_rows < 0 || row_bytes < 0 || row_bytes % 4 != 0)
    return fail(E3_ERR_SHAPE, "bad sizes (row_bytes must be a multiple of 4)");
  if (n_rows == 0 || row_bytes == 0) return E3_OK;
  if (perm == nullptr || in == nullptr || out == nullptr) return fail(E3_ERR_INVALID_ARG, "NULL pointer");
  if ((reinterpret_cast<uintptr_t>(in) & 3u) || (reinterpret_cast<uintptr_t>(out) & 3u))
    return fail(E3_ERR_INVALID_ARG, "in/out not 4-byte aligned");
  int* status = nullptr;
  e3_status st = device_status_ptr(&status);
  if (st != E3_OK) return st;
  const bool vec16 = row_bytes % 16 == 0 && (reinterpret_cast<uintptr_t>(in) & 15u) == 0 &&
                     (reinterpret_cast<uintptr_t>(out) & 15u) == 0;
  const int64_t words = row_bytes / 4;
  const int64_t total = n_rows * (vec16 ? words / 4 : words);
  const int blocks = int(std::min<int64_t>((total + 255) / 256, 148 * 16));
  gather_rows_kernel<<<blocks, 256, 0, static_cast<cudaStream_t>(stream)>>>(
      n_rows, n_in_rows, words, vec16, perm, static_cast<const uint32_t*>(in), static_cast<uint32_t*>(out), status);
  const cudaError_t err = cudaGetLastError();
  if (err != cudaSuccess) return fail(E3_ERR_CUDA, "gather launch failed: %s", cudaGetErrorString(err));
  return E3_OK;
}

extern "C" e3_status e3_add_rows(int64_t n_rows, int64_t n_out_rows, int64_t row_elems, e3_dtype dtype,
                                 const int32_t* idx, const void* in, void* out, void* stream) {
  clear_error();
  if (n_rows < 0 || n_out_rows < 0 || row_elems < 0) return fail(E3_ERR_SHAPE, "negative size");
  if (dtype != E3_F32 && dtype != E3_F64) return fail(E3_ERR_INVALID_ARG, "bad dtype %d", int(dtype));
  if (n_rows == 0 || row_elems == 0) return E3_OK;
  if (idx == nullptr || in == nullptr || out == nullptr) return fail(E3_ERR_INVALID_ARG, "NULL pointer");
  const size_t es = dtype == E3_F64 ? 8 : 4;
  if ((reinterpret_cast<uintptr_t>(in) % es) || (reinterpret_cast<uintptr_t>(out) % es))
    return fail(E3_ERR_INVALID_ARG, "in/out not aligned to the element size");
  int* status = nullptr;
  e3_status st = device_status_ptr(&status);
  if (st != E3_OK) return st;
  const int64_t total = n_rows * row_elems;
  const int blocks = int(std::min<int64_t>((total + 255) / 256, 148 * 16));
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (dtype == E3_F32)
    add_rows_kernel<float><<<blocks, 256, 0, s>>>(n_rows, n_out_rows, row_elems, idx, static_cast<const float*>(in),
                                                  static_cast<float*>(out), status);
  else
    add_rows_kernel<double><<<blocks, 256, 0, s>>>(n_rows, n_out_rows, row_elems, idx,
                                                   static_cast<const double*>(in), static_cast<double*>(out), status);
  const cudaError_t err = cudaGetLastError();
  if (err != cudaSuccess) return fail(E3_ERR_CUDA, "add_rows launch failed: %s", cudaGetErrorString(err));
  return E3_OK;
}

// ------------------------------------------------------------ no-allocation variant ---
// e3_csr_build_static: the same CSR build with its scratch in a fixed device array that the
// library owns, for callers that cannot allocate device memory themselves.  The array is
// sized for E3_CSR_STATIC_MAX_EDGES edges and lives on every device that loads the library
// until the process exits.
namespace e3b {

constexpr size_t static_align256(size_t b) { return (b + 255) & ~size_t(255); }
constexpr size_t kStaticTiles = (size_t(E3_CSR_STATIC_MAX_EDGES) + RS_TILE - 1) / RS_TILE;
constexpr size_t kStaticScratchBytes =
    4 * static_align256(sizeof(int32_t) * size_t(E3_CSR_STATIC_MAX_EDGES)) +
    static_align256(sizeof(int32_t) * size_t(RS_RADIX) * kStaticTiles);

static __device__ __align__(256) unsigned char g_csr_scratch[kStaticScratchBytes];

static std::mutex g_scratch_mutex;
static void* g_scratch_ptr[64] = {};

// Device address of g_csr_scratch on the current device (looked up once per device; the
// name g_csr_scratch is only a host-side stand-in and must never be passed to a kernel).
static e3_status static_scratch(void** ptr) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return fail(E3_ERR_CUDA, "cudaGetDevice failed");
  if (dev < 0 || dev >= 64) return fail(E3_ERR_UNSUPPORTED, "device index %d", dev);
  std::lock_guard<std::mutex> lock(g_scratch_mutex);
  if (g_scratch_ptr[dev] == nullptr) {
    void* p = nullptr;
    const cudaError_t err = cudaGetSymbolAddress(&p, g_csr_scratch);
    if (err != cudaSuccess || p == nullptr)
      return fail(E3_ERR_CUDA, "cudaGetSymbolAddress(csr scratch) failed: %s", cudaGetErrorString(err));
    g_scratch_ptr[dev] = p;
  }
  *ptr = g_scratch_ptr[dev];
  return E3_OK;
}

}  // namespace e3b

extern "C" e3_status e3_csr_build_static(int64_t N, int64_t E, const int32_t* src, const int32_t* dst,
                                         int32_t* perm_dst, int32_t* row_ptr_dst, int32_t* perm_src,
                                         int32_t* row_ptr_src, void* stream) {
  clear_error();
  if (E > int64_t(E3_CSR_STATIC_MAX_EDGES))
    return fail(E3_ERR_SHAPE, "e3_csr_build_static: %lld edges exceed the built-in scratch limit of %d edges; "
                "use e3_csr_build with a caller-provided workspace", (long long)E, E3_CSR_STATIC_MAX_EDGES);
  if (E < 0 || N < 0) return fail(E3_ERR_SHAPE, "N or E out of range");
  if (csr_ws_bytes(E) > kStaticScratchBytes)
    return fail(E3_ERR_SHAPE, "e3_csr_build_static: scratch too small for %lld edges", (long long)E);
  void* ws = nullptr;
  const e3_status st = static_scratch(&ws);
  if (st != E3_OK) return st;
  return e3_csr_build(N, E, src, dst, perm_dst, row_ptr_dst, perm_src, row_ptr_src, ws, kStaticScratchBytes,
                      stream);
}

// ------------------------------------------------------------------- node reordering ---
static size_t morton_ws_bytes(int64_t N) { return align256(sizeof(int32_t) * size_t(N > 0 ? N : 1)) + csr_ws_bytes(N); }

extern "C" e3_status e3_morton_workspace_size(int64_t N, size_t* bytes) {
  clear_error();
  if (bytes == nullptr) return fail(E3_ERR_INVALID_ARG, "bytes is NULL");
  if (N < 0 || N >= (int64_t(1) << 31)) return fail(E3_ERR_SHAPE, "N out of range");
  *bytes = morton_ws_bytes(N);
  return E3_OK;
}

extern "C" e3_status e3_morton_order(int64_t N, const void* pos, e3_dtype dtype, const double* lo, const double* extent,
                                     int32_t* perm, void* workspace, size_t ws_bytes, void* stream) {
  clear_error();
  if (N < 0 || N >= (int64_t(1) << 31)) return fail(E3_ERR_SHAPE, "N out of range");
  if (dtype != E3_F32 && dtype != E3_F64) return fail(E3_ERR_INVALID_ARG, "bad dtype");
  if (lo == nullptr || extent == nullptr) return fail(E3_ERR_INVALID_ARG, "lo or extent is NULL");
  for (int k = 0; k < 3; ++k)
    if (!(extent[k] > 0.0) || !std::isfinite(extent[k]) || !std::isfinite(lo[k]))
      return fail(E3_ERR_INVALID_ARG, "box extent must be positive and finite");
  if (N == 0) return E3_OK;
  if (pos == nullptr || perm == nullptr) return fail(E3_ERR_INVALID_ARG, "NULL pointer");
  if (reinterpret_cast<uintptr_t>(pos) % (dtype == E3_F64 ? 8 : 4)) return fail(E3_ERR_INVALID_ARG, "pos not aligned");
  if (workspace == nullptr || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
    return fail(E3_ERR_INVALID_ARG, "workspace is NULL or not 256-byte aligned");
  if (ws_bytes < morton_ws_bytes(N)) return fail(E3_ERR_SHAPE, "workspace of %zu bytes, need %zu", ws_bytes, morton_ws_bytes(N));
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  char* ws = static_cast<char*>(workspace);
  int32_t* codes = reinterpret_cast<int32_t*>(ws);
  char* sort_ws = ws + align256(sizeof(int32_t) * size_t(N));
  const size_t eb = align256(sizeof(int32_t) * size_t(N));
  int32_t* ka = reinterpret_cast<int32_t*>(sort_ws);
  int32_t* va = reinterpret_cast<int32_t*>(sort_ws + eb);
  int32_t* kb = reinterpret_cast<int32_t*>(sort_ws + 2 * eb);
  int32_t* vb = reinterpret_cast<int32_t*>(sort_ws + 3 * eb);
  int32_t* counts = reinterpret_cast<int32_t*>(sort_ws + 4 * eb);
  const double scale[3] = {double(1 << MORTON_BITS) / extent[0], double(1 << MORTON_BITS) / extent[1],
                           double(1 << MORTON_BITS) / extent[2]};
  const int blocks = int(std::min<int64_t>((N + 255) / 256, 148 * 8));
  if (dtype == E3_F32)
    morton_code_kernel<float><<<blocks, 256, 0, s>>>(N, static_cast<const float*>(pos), lo[0], lo[1], lo[2], scale[0],
                                                     scale[1], scale[2], codes);
  else
    morton_code_kernel<double><<<blocks, 256, 0, s>>>(N, static_cast<const double*>(pos), lo[0], lo[1], lo[2],
                                                      scale[0], scale[1], scale[2], codes);
  const cudaError_t err = cudaGetLastError();
  if (err != cudaSuccess) return fail(E3_ERR_CUDA, "morton code launch failed: %s", cudaGetErrorString(err));
  return radix_sort(codes, nullptr, nullptr, 0u, N, 3 * MORTON_BITS, perm, ka, va, kb, vb, counts, s);
}

extern "C" e3_status e3_invert_permutation(int64_t N, const int32_t* perm, int32_t* inv, void* stream) {
  clear_error();
  if (N < 0 || N >= (int64_t(1) << 31)) return fail(E3_ERR_SHAPE, "N out of range");
  if (N == 0) return E3_OK;
  if (perm == nullptr || inv == nullptr) return fail(E3_ERR_INVALID_ARG, "NULL pointer");
  int* status = nullptr;
  e3_status st = device_status_ptr(&status);
  if (st != E3_OK) return st;
  const int blocks = int(std::min<int64_t>((N + 255) / 256, 148 * 8));
  invert_perm_kernel<<<blocks, 256, 0, static_cast<cudaStream_t>(stream)>>>(N, perm, inv, status);
  const cudaError_t err = cudaGetLastError();
  if (err != cudaSuccess) return fail(E3_ERR_CUDA, "invert launch failed: %s", cudaGetErrorString(err));
  return E3_OK;
}

extern "C" e3_status e3_remap_ids(int64_t n, const int32_t* ids, int64_t N, const int32_t* map, int32_t* out,
                                  void* stream) {
  clear_error();
  if (n < 0 || N < 0 || n >= (int64_t(1) << 31) || N >= (int64_t(1) << 31)) return fail(E3_ERR_SHAPE, "n or N out of range");
  if (n == 0) return E3_OK;
  if (ids == nullptr || map == nullptr || out == nullptr) return fail(E3_ERR_INVALID_ARG, "NULL pointer");
  int* status = nullptr;
  e3_status st = device_status_ptr(&status);
  if (st != E3_OK) return st;
  const int blocks = int(std::min<int64_t>((n + 255) / 256, 148 * 8));
  remap_ids_kernel<<<blocks, 256, 0, static_cast<cudaStream_t>(stream)>>>(n, ids, N, map, out, status);
  const cudaError_t err = cudaGetLastError();
  if (err != cudaSuccess) return fail(E3_ERR_CUDA, "remap launch failed: %s", cudaGetErrorString(err));
  return E3_OK;
}

// ------------------------------------------------------------------- convolution units ---
extern "C" e3_status e3_conv_topology_size(int64_t N, int64_t E, size_t* bytes) {
  clear_error();
  if (bytes == nullptr) return fail(E3_ERR_INVALID_ARG, "bytes is NULL");
  if (N < 0 || E < 0 || N >= (int64_t(1) << 31) || E >= (int64_t(1) << 31)) return fail(E3_ERR_SHAPE, "N or E out of range");
  *bytes = topo_bytes(N, E);
  return E3_OK;
}

extern "C" e3_status e3_conv_topology_build(int64_t N, int64_t E, const int32_t* row_ptr_dst, const int32_t* row_ptr_src,
                                            void* topo, size_t topo_bytes_, void* stream) {
  return e3_conv_topology_build_ordered(N, E, row_ptr_dst, row_ptr_src, nullptr, topo, topo_bytes_, stream);
}

extern "C" e3_status e3_conv_topology_build_ordered(int64_t N, int64_t E, const int32_t* row_ptr_dst,
                                                    const int32_t* row_ptr_src, const int32_t* order, void* topo,
                                                    size_t topo_bytes_, void* stream) {
  clear_error();
  if (N < 0 || E < 0 || N >= (int64_t(1) << 31) || E >= (int64_t(1) << 31)) return fail(E3_ERR_SHAPE, "N or E out of range");
  if (topo == nullptr || (reinterpret_cast<uintptr_t>(topo) & 15u) != 0)
    return fail(E3_ERR_INVALID_ARG, "topology buffer is NULL or not 16-byte aligned");
  if (topo_bytes_ < topo_bytes(N, E)) return fail(E3_ERR_SHAPE, "topology buffer of %zu bytes, need %zu", topo_bytes_, topo_bytes(N, E));
  if (N > 0 && (row_ptr_dst == nullptr || row_ptr_src == nullptr)) return fail(E3_ERR_INVALID_ARG, "row_ptr array is NULL");
  unsigned char* base = static_cast<unsigned char*>(topo);
  e3_status st = build_topo_part(N, E, row_ptr_dst, order, base, topo_dst(N, E), stream);
  if (st != E3_OK) return st;
  return build_topo_part(N, E, row_ptr_src, order, base, topo_src(N, E), stream);
}
