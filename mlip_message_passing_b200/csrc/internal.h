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
  int C = 0;                      // common multiplicity of the x irreps
  int LX = 0, LY = 0, LO = 0;     // degree range of x, y and the output
  int n_paths = 0;
  std::vector<int> l1, l2, l3;    // per path
  std::vector<double> alpha;      // per path
  int64_t dim1 = 0, dim2 = 0, dim_out = 0, weight_numel = 0;
  std::string irreps_out;
};

namespace e3b {

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
  void* workspace;           // e3_backward_workspace_size(n_nodes) bytes
  size_t workspace_bytes;
  void* stream;
};
// Bytes of backward workspace for n units: 16-byte ticket counter + one int per unit.
inline size_t backward_workspace_bytes(int64_t n) { return (size_t(16) + 4 * size_t(n) + 255) & ~size_t(255); }
e3_status launch_backward(const e3_plan* plan, const BwdArgs& a, bool conv);
// Zero rows [*first_row, n_rows) of a row-major array of row_bytes-byte rows (first_row read on
// the device: the padding positions after the last CSR row).
e3_status zero_rows_after(const int32_t* first_row, int64_t n_rows, int64_t row_bytes, void* ptr, void* stream);

}  // namespace e3b
