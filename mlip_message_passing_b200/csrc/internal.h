// Internal declarations shared by the host library (host.cpp) and the CUDA translation units.
#pragma once

#include <cstdint>
#include <string>
#include <vector>

#include "../../include/e3b.h"

struct e3_plan {
  int device = 0;
  e3_dtype dtype = E3_F32;
  e3_weight_mode wmode = E3_W_PER_SAMPLE;
  e3_mode mode = E3_UVU;
  int C = 0;                      // common multiplicity of the x irreps (and of y in uuu)
  int LX = 0, LY = 0, LO = 0;     // degree range of x, y and the output
  int n_paths = 0;
  std::vector<int> l1, l2, l3;    // per path
  std::vector<double> alpha;      // per path
  int64_t dim1 = 0, dim2 = 0, dim_out = 0, weight_numel = 0;
  std::string irreps_out;
  // uvw: output channels, per path the output block and offsets, the weight staging buffer
  int Co = 0;
  std::vector<int> io, x_off, g_off, z_off;
  std::vector<int> out_l, out_off;  // per output block
  void* uvw_prep = nullptr;
  size_t uvw_prep_size = 0;
  void* uvw_z = nullptr;            // Z of a batch of samples for grad_y
  int64_t uvw_z_row = 0, uvw_z_batch = 0;
  int* status = nullptr;            // this plan's device status word (its kernels record errors here)
  ~e3_plan();
};

namespace e3b {

// Path sets (LX, LY, LO) with compiled kernels.
#define E3_CONFIGS(X) X(1, 1, 2) X(1, 2, 2) X(2, 3, 2) X(3, 3, 3)

// Thread-local error message; returns `st` so callers can `return fail(st, ...)`.
e3_status fail(e3_status st, const char* fmt, ...);
void clear_error();

// Real-basis CG (ladder construction), dense [2l1+1][2l2+1][2l3+1], row-major.
std::vector<double> real_cg_ladder(int l1, int l2, int l3);

// Packed table (cg_pattern.h layout) in double precision, generated once per process.
const std::vector<double>& packed_cg_table();

// Is (LX, LY, LO) compiled?
bool degrees_supported(int LX, int LY, int LO);
const char* supported_list();

// Device side (dispatch.cu): upload the CG tables to the current device if not done yet.
e3_status ensure_device_tables();
// Address of the current device's status word (dispatch.cu).
e3_status device_status_ptr(int** ptr);
// Number of SMs of the current device.
int sm_count();
// Limit of every bounded device wait (nanoseconds) and the first ticket the ticketed kernels
// draw, as set by e3_set_test_knobs (defaults: one second, 0).
unsigned long long test_wait_limit_ns();
int test_first_ticket();

// Launchers (dispatch.cu, per path set in tp_conv_l*.cu).  Arguments are validated by the caller.
struct FwdArgs {
  int64_t n_rows;            // nodes (conv) or samples (tp)
  int64_t n_edges;           // conv only
  const int32_t* row_ptr;    // conv only (receiver CSR)
  const int32_t* src;        // conv only
  const void* x;
  const void* y;             // harmonics, or NULL when vec is given
  const void* vec;           // edge vectors [E, 3] or NULL
  int sh_norm;
  const void* w;
  int64_t w_stride;          // weight_numel, or 0 for shared weights
  double scale;
  void* out;
  const void* topo;          // conv only: topology buffer (receiver part used)
  void* workspace;           // conv only: conv_counters
  void* stream;
};
e3_status launch_forward(const e3_plan* plan, const FwdArgs& a, bool conv);

struct BwdArgs {
  int64_t n_nodes;           // senders (conv) or samples (tp)
  int64_t n_edges;
  const int32_t* row_ptr_dst; // conv only: row_ptr_dst[N] = first padding position
  const int32_t* row_ptr_src; // conv only
  const int32_t* perm_src;    // conv only
  const int32_t* dst;         // conv only
  const void* x;
  const void* y;
  const void* vec;
  int sh_norm;
  const void* w;
  const void* grad_out;
  double scale;
  void* grad_x;
  void* grad_y;
  void* grad_w;
  const void* topo;          // conv only: topology buffer (sender part used)
  void* workspace;           // conv: conv_counters; tp: e3_backward_workspace_size(n_nodes) bytes
  size_t workspace_bytes;
  void* stream;
};
// Bytes of backward workspace for n units: 16-byte ticket counter + one int per unit.
inline size_t backward_workspace_bytes(int64_t n) { return (size_t(16) + 4 * size_t(n) + 255) & ~size_t(255); }

// Row segmentation of the convolution: no CTA walks more than SEG_EDGES edges of one row; a row
// of deg edges has max(1, ceil(deg / SEG_EDGES)) segments, each a work unit.
constexpr int64_t SEG_EDGES = 256;
inline int64_t seg_units_max(int64_t N, int64_t E) { return N + E / SEG_EDGES + 1; }
inline size_t al16(size_t b) { return (b + 15) & ~size_t(15); }

// Topology buffer (built once per topology by e3_conv_topology_build), one part per direction
// (receivers: dst, senders: src), each
//   units (int, padded to 16 B) | info [units_max] int4 {row, first edge, end edge, segment} |
//   nseg [units_max] int (segments of the unit's row) | seg_start [N + 1] int (scratch)
struct TopoPart {
  size_t units, info, nseg, seg_start, end;
};
inline TopoPart topo_part(int64_t N, int64_t E, size_t base) {
  const int64_t U = seg_units_max(N, E);
  TopoPart t{};
  t.units = base;
  t.info = base + 16;
  t.nseg = t.info + al16(16 * size_t(U));
  t.seg_start = t.nseg + al16(4 * size_t(U));
  t.end = t.seg_start + al16(4 * size_t(N + 1));
  return t;
}
inline TopoPart topo_dst(int64_t N, int64_t E) { return topo_part(N, E, 0); }
inline TopoPart topo_src(int64_t N, int64_t E) { return topo_part(N, E, topo_dst(N, E).end); }
inline size_t topo_bytes(int64_t N, int64_t E) { return (topo_src(N, E).end + 255) & ~size_t(255); }
// Fill one direction's part from row_ptr [N + 1], rows in the processing order `order` (a
// permutation of 0..N-1, or NULL for 0..N-1); rows with out-of-range pointers record E3_ERR_INDEX
// and get empty units; stream-ordered.
e3_status build_topo_part(int64_t N, int64_t E, const int32_t* row_ptr, const int32_t* order, unsigned char* base,
                          const TopoPart& t, void* stream);

// Per-call counters of a convolution launch (zeroed by the call):
//   ticket (16 B) | flags [units_max * G] int | chain [N] int
struct ConvCounters {
  size_t flags, chain, total;
};
inline ConvCounters conv_counters(int64_t N, int64_t E, int G) {
  ConvCounters c{};
  c.flags = 16;
  c.chain = c.flags + al16(4 * size_t(seg_units_max(N, E)) * size_t(G));
  c.total = (c.chain + al16(4 * size_t(N)) + 255) & ~size_t(255);
  return c;
}
// path groups of a plan's kernels
int plan_groups(const e3_plan* plan);
// Workspace of one convolution call: the counters, then, for float plans, room for a
// component-major copy of x (forward) or of grad_out (backward), which the paired kernels stage.
inline size_t conv_workspace_bytes(const e3_plan* plan, int64_t N, int64_t E, int groups) {
  size_t b = conv_counters(N, E, groups).total;
  if (plan->dtype == E3_F32) {
    const int64_t row = plan->dim1 > plan->dim_out ? plan->dim1 : plan->dim_out;
    b += (size_t(N) * size_t(row) * 4 + 255) & ~size_t(255);
  }
  return b;
}
e3_status launch_backward(const e3_plan* plan, const BwdArgs& a, bool conv);

// uuu tensor product (tp_uuu.cu): one thread per (sample, channel).
constexpr int UUU_MAXP = 64;
struct UuuArgs {
  int64_t B;
  int C;
  int64_t dim1, dim2, dim_out;
  const void* x;
  const void* y;
  const void* w;
  int64_t w_stride;          // weight_numel, or 0 for shared weights (forward only)
  void* out;                 // forward
  const void* grad_out;      // backward
  void* grad_x;              // backward, each optional
  void* grad_y;
  void* grad_w;
  void* stream;
  double alpha[UUU_MAXP];
};
e3_status upload_tables_uuu(const double* t64, const float* t32);
e3_status launch_uuu(const e3_plan* plan, const UuuArgs& a, bool backward);
// uvw tensor product with shared weights (tp_uvw.cu).
// The tcgen05 contraction: per target block (an output block in the forward, an x block for
// grad_x) the sum over its terms (paths) of alpha_p (coupled input) x W_p.
constexpr int UVW_MAXT = 64;
constexpr int UVW_MAXP = 64;
struct UvwTarget {
  int32_t off;          // offset of the block in a row of the result
  int32_t l;            // its degree
  int32_t bt;           // samples per tile: floor(128 / (2 l + 1))
  int32_t tile_begin;   // first tile of this target in the launch
  int32_t term_begin, term_end;
};
struct UvwTerm {
  int32_t in_off;       // offset of the input block (x block, or grad_out block) in an input row
  int32_t l_in, l2;     // its degree and the degree of y
  int32_t chunk0;       // first B chunk of the path in the prepared weights
  float alpha;
};
struct UvwGemmArgs {
  int64_t B;
  const float* in;
  int64_t in_stride;
  int32_t k_in;         // input channels of every term (the K of one term)
  const float* y;
  int64_t y_stride;
  float* out;
  int64_t out_stride;
  int32_t N;            // channels of the result (the MMA's N)
  const unsigned char* prep;
  uint32_t b_chunk_bytes;
  int32_t n_targets, total_tiles;
  UvwTarget tg[UVW_MAXT];
  UvwTerm term[UVW_MAXP];
  int* status;
  unsigned long long wait_ns;
};
// grad_w and grad_y on the CUDA cores: every path's degrees and offsets.
struct UvwPath {
  int32_t l1, l2, l3;
  int32_t x_off, g_off;  // offsets of the path's x block and output block in their rows
  int32_t z_off;         // per-channel offset of the path's block in a row of Z (sum of earlier 2 l3 + 1)
  int64_t w_off;         // offset of W_p [C][Cout] in the shared weights
  float alpha;
  int64_t chunks;        // grad_w: K chunks of this path (filled by the launcher)
  int32_t tile_begin;    // grad_w: first tile of this path
};
struct UvwBwdArgs {
  int64_t B;
  int32_t C, Co, P;
  const float* x;
  int64_t dim1;
  const float* y;
  int64_t dim2;
  const float* w;
  const float* g;
  int64_t dim_out;
  float* grad_w;
  float* grad_y;
  int* status;
  unsigned long long wait_ns;
  int32_t total_tiles;   // grad_w (filled by the launcher)
  UvwPath path[UVW_MAXP];
};
e3_status upload_tables_uvw(const double* t64, const float* t32);
size_t uvw_prep_bytes(int P, int C, int Co);
e3_status launch_uvw_prep(int P, int C, int Co, const float* w, void* prep, void* stream);
// role: 0 forward (A = alpha C-coupled x), 1 grad_x (A = alpha C-coupled grad_out), 2 plain (A = the input)
e3_status launch_uvw_gemm(const UvwGemmArgs& a, int role, void* stream);
e3_status launch_uvw_grad_w(const UvwBwdArgs& a, void* stream);
// grad_y of samples [b0, b0 + nb) from Z (row r = sample b0 + r, z_stride floats per row)
e3_status launch_uvw_grad_y(const UvwBwdArgs& a, const float* z, int64_t z_stride, int64_t b0, int64_t nb,
                            void* stream);

// Zero rows [*first_row, n_rows) of a row-major array of row_bytes-byte rows (first_row read on
// the device: the padding positions after the last CSR row).
e3_status zero_rows_after(const int32_t* first_row, int64_t n_rows, int64_t row_bytes, void* ptr, void* stream);

}  // namespace e3b
