// Host side of the library: irreps strings, instruction validation, the Clebsch-Gordan table
// (ladder construction), plans, and argument checking for every C-ABI entry point that
// launches work.  No CUDA kernels live here.
#include <cuda_runtime.h>

#include <algorithm>
#include <climits>
#include <cmath>
#include <complex>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <new>
#include <string>
#include <vector>

#include "cg_pattern.h"
#include "internal.h"

namespace e3b {

// ------------------------------------------------------------------------- errors ---
static thread_local std::string g_last_error;

e3_status fail(e3_status st, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof buf, fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return st;
}

void clear_error() { g_last_error.clear(); }

// ------------------------------------------------------------------ irreps strings ---
// e3nn course, "Curriculum at a glance", lesson 02a: terms "<mul>x<l><p>" joined by '+';
// a bare "<l><p>" has multiplicity 1.
struct IrrepT {
  int mul, l, p;
};

static bool parse_irreps(const char* s, std::vector<IrrepT>* out, std::string* why) {
  out->clear();
  if (s == nullptr) {
    *why = "NULL irreps string";
    return false;
  }
  const char* c = s;
  auto skip = [&] {
    while (*c == ' ' || *c == '\t') ++c;
  };
  skip();
  if (*c == '\0') {
    *why = "empty irreps string";
    return false;
  }
  while (true) {
    skip();
    long a = -1, b = -1;
    if (*c < '0' || *c > '9') {
      *why = std::string("expected a digit at '") + c + "'";
      return false;
    }
    a = 0;
    while (*c >= '0' && *c <= '9') {
      a = a * 10 + (*c - '0');
      if (a > 1000000) {
        *why = "number too large";
        return false;
      }
      ++c;
    }
    skip();
    if (*c == 'x') {
      ++c;
      skip();
      if (*c < '0' || *c > '9') {
        *why = std::string("expected a degree after 'x' at '") + c + "'";
        return false;
      }
      b = 0;
      while (*c >= '0' && *c <= '9') {
        b = b * 10 + (*c - '0');
        if (b > 1000) {
          *why = "degree too large";
          return false;
        }
        ++c;
      }
    } else {
      b = a;
      a = 1;
    }
    if (*c != 'e' && *c != 'o') {
      *why = std::string("expected parity 'e' or 'o' at '") + c + "'";
      return false;
    }
    if (a <= 0) {
      *why = "multiplicity must be positive";
      return false;
    }
    out->push_back({int(a), int(b), *c == 'e' ? 1 : -1});
    ++c;
    skip();
    if (*c == '\0') break;
    if (*c != '+') {
      *why = std::string("expected '+' at '") + c + "'";
      return false;
    }
    ++c;
  }
  return true;
}

static std::string irreps_to_string(const std::vector<IrrepT>& v) {
  std::string s;
  for (size_t i = 0; i < v.size(); ++i) {
    if (i) s += "+";
    s += std::to_string(v[i].mul) + "x" + std::to_string(v[i].l) + (v[i].p > 0 ? "e" : "o");
  }
  return s;
}

// ------------------------------------------------------ CG: the ladder construction ---
// E3J, section G.2: the top-spin vector |l3, l3> of V_l1 (x) V_l2 solves J+ v = 0 restricted
// to m1 + m2 = l3, a two-term (triangular) recurrence; the lower vectors follow by applying
// J- = J1- + J2- and normalising.  The standard angular-momentum matrix elements are
//   J+ |j m> = sqrt(j(j+1) - m(m+1)) |j m+1>,   J- |j m> = sqrt(j(j+1) - m(m-1)) |j m-1>.
// The complex-basis result is then moved to the real basis of the harmonics (the same change
// of basis that defines the real harmonics from the complex ones), normalised to Frobenius
// norm 1 and given the sign of the library convention (see e3b.h).

static double jp(int j, int m) { return std::sqrt(double(j * (j + 1) - m * (m + 1))); }
static double jm(int j, int m) { return std::sqrt(double(j * (j + 1) - m * (m - 1))); }

// cc[(m1+l1)][(m2+l2)][(m3+l3)]: coefficient of |m1>|m2> in |l3 m3>, Condon-Shortley phase.
static std::vector<double> complex_cg_ladder(int l1, int l2, int l3) {
  const int d1 = 2 * l1 + 1, d2 = 2 * l2 + 1, d3 = 2 * l3 + 1;
  std::vector<double> cc(size_t(d1) * d2 * d3, 0.0);
  auto at = [&](int m1, int m2, int m3) -> double& {
    return cc[(size_t(m1 + l1) * d2 + (m2 + l2)) * d3 + (m3 + l3)];
  };
  // top state: a[m1] with m2 = l3 - m1; a_{m1+1} = -a_{m1} jp(l1, m1) / jp(l2, l3 - m1 - 1)
  const int lo = std::max(-l1, l3 - l2), hi = std::min(l1, l3 + l2);
  std::vector<double> a(size_t(hi - lo + 1), 0.0);
  a[0] = 1.0;
  for (int m1 = lo; m1 < hi; ++m1) a[m1 + 1 - lo] = -a[m1 - lo] * jp(l1, m1) / jp(l2, l3 - m1 - 1);
  double nrm = 0.0;
  for (double v : a) nrm += v * v;
  nrm = std::sqrt(nrm);
  const double sgn = a[hi - lo] >= 0 ? 1.0 : -1.0;  // <l1 l1; l2 l3-l1 | l3 l3> > 0
  for (int m1 = lo; m1 <= hi; ++m1) at(m1, l3 - m1, l3) = sgn * a[m1 - lo] / nrm;
  // lowering
  for (int m3 = l3; m3 > -l3; --m3) {
    const double inv = 1.0 / jm(l3, m3);
    for (int m1 = -l1; m1 <= l1; ++m1)
      for (int m2 = -l2; m2 <= l2; ++m2) {
        const double v = at(m1, m2, m3);
        if (v == 0.0) continue;
        if (m1 > -l1) at(m1 - 1, m2, m3 - 1) += v * jm(l1, m1) * inv;
        if (m2 > -l2) at(m1, m2 - 1, m3 - 1) += v * jm(l2, m2) * inv;
      }
  }
  return cc;
}

// U with Y_real = U Y_complex for the real harmonics of e3b.h (m>0: cos, m<0: sin, no
// Condon-Shortley phase), rows real m, columns complex m.
static std::vector<std::complex<double>> real_from_complex(int l) {
  const int d = 2 * l + 1;
  std::vector<std::complex<double>> U(size_t(d) * d, 0.0);
  const double r = 1.0 / std::sqrt(2.0);
  for (int m = -l; m <= l; ++m) {
    auto u = [&](int mc) -> std::complex<double>& { return U[size_t(m + l) * d + (mc + l)]; };
    if (m > 0) {
      u(-m) = r;
      u(m) = ((m & 1) ? -r : r);
    } else if (m == 0) {
      u(0) = 1.0;
    } else {
      const int k = -m;
      u(-k) = std::complex<double>(0.0, r);
      u(k) = std::complex<double>(0.0, (k & 1) ? r : -r);
    }
  }
  return U;
}

std::vector<double> real_cg_ladder(int l1, int l2, int l3) {
  const int d1 = 2 * l1 + 1, d2 = 2 * l2 + 1, d3 = 2 * l3 + 1;
  const std::vector<double> cc = complex_cg_ladder(l1, l2, l3);
  const auto U1 = real_from_complex(l1), U2 = real_from_complex(l2), U3 = real_from_complex(l3);
  // C_R[i][j][k] = sum conj(U1[i][a]) conj(U2[j][b]) U3[k][c] cc[a][b][c]
  std::vector<std::complex<double>> cr(size_t(d1) * d2 * d3, 0.0);
  for (int i = 0; i < d1; ++i)
    for (int j = 0; j < d2; ++j)
      for (int k = 0; k < d3; ++k) {
        std::complex<double> s = 0.0;
        for (int a = 0; a < d1; ++a) {
          const auto u1 = std::conj(U1[size_t(i) * d1 + a]);
          if (u1 == 0.0) continue;
          for (int b = 0; b < d2; ++b) {
            const auto u2 = std::conj(U2[size_t(j) * d2 + b]);
            if (u2 == 0.0) continue;
            for (int c = 0; c < d3; ++c) {
              const double v = cc[(size_t(a) * d2 + b) * d3 + c];
              if (v == 0.0) continue;
              s += u1 * u2 * U3[size_t(k) * d3 + c] * v;
            }
          }
        }
        cr[(size_t(i) * d2 + j) * d3 + k] = s;
      }
  double re = 0.0, im = 0.0;
  for (const auto& z : cr) {
    re = std::max(re, std::fabs(z.real()));
    im = std::max(im, std::fabs(z.imag()));
  }
  const bool use_re = re >= im;
  std::vector<double> t(cr.size());
  double nrm = 0.0;
  for (size_t q = 0; q < cr.size(); ++q) {
    t[q] = use_re ? cr[q].real() : cr[q].imag();
    nrm += t[q] * t[q];
  }
  nrm = std::sqrt(nrm);
  for (double& v : t) v /= nrm;
  double ref = 0.0;
  if (((l1 + l2 + l3) & 1) == 0) {
    ref = t[(size_t(l1) * d2 + l2) * d3 + l3];
  } else {
    for (double v : t)
      if (std::fabs(v) > 1e-12) {
        ref = v;
        break;
      }
  }
  if (ref < 0)
    for (double& v : t) v = -v;
  for (double& v : t)
    if (std::fabs(v) < 1e-15) v = 0.0;
  return t;
}

const std::vector<double>& packed_cg_table() {
  static std::vector<double> table;
  static std::once_flag once;
  std::call_once(once, [] {
    table.assign(CG_TABLE_SIZE, 0.0);
    for (int l1 = 0; l1 <= E3_LMAX; ++l1)
      for (int l2 = 0; l2 <= E3_LMAX; ++l2)
        for (int l3 = 0; l3 <= E3_LMAX; ++l3) {
          if (!triangle(l1, l2, l3)) continue;
          const auto t = real_cg_ladder(l1, l2, l3);
          const int d2 = 2 * l2 + 1, d3 = 2 * l3 + 1;
          for (int m1 = -l1; m1 <= l1; ++m1)
            for (int m2 = -l2; m2 <= l2; ++m2)
              for (int m3 = -l3; m3 <= l3; ++m3) {
                const double v = t[(size_t(m1 + l1) * d2 + (m2 + l2)) * d3 + (m3 + l3)];
                const int idx = cg_index(l1, l2, l3, m1, m2, m3);
                if (idx >= 0) {
                  table[idx] = v;
                } else if (std::fabs(v) > 1e-12) {
                  // the selection rules of cg_pattern.h would be wrong; never expected
                  std::fprintf(stderr, "e3b: CG entry outside pattern (%d %d %d | %d %d %d) = %g\n",
                               l1, l2, l3, m1, m2, m3, v);
                }
              }
        }
  });
  return table;
}

// ------------------------------------------------------------- compiled path sets ---
static const int kSupported[][3] = {{1, 1, 2}, {1, 2, 2}, {2, 3, 2}, {3, 3, 3}};

bool degrees_supported(int LX, int LY, int LO) {
  for (const auto& s : kSupported)
    if (s[0] == LX && s[1] == LY && s[2] == LO) return true;
  return false;
}

const char* supported_list() {
  static std::string s;
  static std::once_flag once;
  std::call_once(once, [] {
    for (const auto& t : kSupported) {
      if (!s.empty()) s += " ";
      s += std::to_string(t[0]) + "," + std::to_string(t[1]) + "," + std::to_string(t[2]);
    }
  });
  return s.c_str();
}

}  // namespace e3b

using namespace e3b;

// ===================================================================== C ABI: plans ===

extern "C" const char* e3_last_error(void) { return e3b::g_last_error.c_str(); }

extern "C" const char* e3_supported(void) { return supported_list(); }

extern "C" e3_status e3_cg_dense(int32_t l1, int32_t l2, int32_t l3, double* out) {
  clear_error();
  if (out == nullptr) return fail(E3_ERR_INVALID_ARG, "e3_cg_dense: out is NULL");
  if (l1 < 0 || l2 < 0 || l3 < 0 || l1 > E3_LMAX || l2 > E3_LMAX || l3 > E3_LMAX)
    return fail(E3_ERR_UNSUPPORTED, "e3_cg_dense: degrees must lie in [0, %d]", E3_LMAX);
  if (!triangle(l1, l2, l3)) return fail(E3_ERR_INSTRUCTION, "e3_cg_dense: triangle rule violated");
  const auto t = real_cg_ladder(l1, l2, l3);
  std::memcpy(out, t.data(), t.size() * sizeof(double));
  return E3_OK;
}

// Live plans, so that e3_device_status can drain their status words too.
static std::mutex g_plans_mu;
static std::vector<e3_plan*> g_plans;

e3_plan::~e3_plan() {
  {
    std::lock_guard<std::mutex> lock(g_plans_mu);
    for (size_t i = 0; i < g_plans.size(); ++i)
      if (g_plans[i] == this) {
        g_plans.erase(g_plans.begin() + long(i));
        break;
      }
  }
  if (uvw_prep != nullptr || uvw_z != nullptr || status != nullptr) {
    int cur = -1;
    const bool restore = cudaGetDevice(&cur) == cudaSuccess && cur != device;
    if (restore) cudaSetDevice(device);
    if (uvw_prep != nullptr) cudaFree(uvw_prep);
    if (uvw_z != nullptr) cudaFree(uvw_z);
    if (status != nullptr) cudaFree(status);
    if (restore) cudaSetDevice(cur);
  }
}

// The plan's own status word (zeroed), and its entry in the list of live plans.
static e3_status plan_attach_status(e3_plan* plan) {
  if (cudaMalloc(reinterpret_cast<void**>(&plan->status), 256) != cudaSuccess) {
    plan->status = nullptr;
    return fail(E3_ERR_CUDA, "allocating the plan's status word failed");
  }
  if (cudaMemset(plan->status, 0, 256) != cudaSuccess) return fail(E3_ERR_CUDA, "zeroing the plan's status word failed");
  std::lock_guard<std::mutex> lock(g_plans_mu);
  g_plans.push_back(plan);
  return E3_OK;
}

// Plan of the fully connected (uvw) mode: x = Cx0+..+CxLx, y = 1x0+..+1xLy, output blocks of one
// multiplicity Co; instructions given, or every (i1, i2, i_out) that the triangle and parity rules
// allow, in that loop order.  Shared float32 weights W_p[u][w] (v has one value), alpha_p =
// sqrt((2 l3 + 1) / (C n_out)).
static e3_status create_uvw(const std::vector<IrrepT>& ir1, const std::vector<IrrepT>& ir2,
                            const std::vector<IrrepT>& irf, bool have_out, const e3_instruction* instr,
                            int32_t n_instr, e3_dtype dtype, e3_weight_mode wmode, e3_plan** plan_out) {
  if (!have_out) return fail(E3_ERR_INSTRUCTION, "the uvw mode needs irreps_out");
  struct Ins {
    int i1, i2, io;
    double pw;
  };
  std::vector<Ins> ins;
  if (n_instr == 0) {
    for (int i1 = 0; i1 < int(ir1.size()); ++i1)
      for (int i2 = 0; i2 < int(ir2.size()); ++i2)
        for (int io = 0; io < int(irf.size()); ++io)
          if (triangle(ir1[i1].l, ir2[i2].l, irf[io].l) && irf[io].p == ir1[i1].p * ir2[i2].p)
            ins.push_back({i1, i2, io, -1.0});
  } else {
    for (int q = 0; q < n_instr; ++q) {
      const auto& s = instr[q];
      if (s.i_in1 < 0 || s.i_in1 >= int(ir1.size()) || s.i_in2 < 0 || s.i_in2 >= int(ir2.size()) || s.i_out < 0 ||
          s.i_out >= int(irf.size()))
        return fail(E3_ERR_INSTRUCTION, "instruction %d: index out of range", q);
      const auto &a = ir1[s.i_in1], &b = ir2[s.i_in2], &c = irf[s.i_out];
      if (!triangle(a.l, b.l, c.l))
        return fail(E3_ERR_INSTRUCTION, "instruction %d: triangle rule |l1-l2| <= l3 <= l1+l2 fails (%d,%d,%d)", q,
                    a.l, b.l, c.l);
      if (c.p != a.p * b.p) return fail(E3_ERR_INSTRUCTION, "instruction %d: parity rule p3 = p1 p2 fails", q);
      if (!s.has_weight) return fail(E3_ERR_UNSUPPORTED, "instruction %d: paths without weights have no kernel", q);
      ins.push_back({s.i_in1, s.i_in2, s.i_out, s.path_weight});
    }
  }
  if (ins.empty()) return fail(E3_ERR_INSTRUCTION, "no allowed path between the inputs and irreps_out");
  if (dtype != E3_F32) return fail(E3_ERR_UNSUPPORTED, "uvw kernels compute in float32 (tf32 tensor cores, three passes)");
  if (wmode != E3_W_SHARED) return fail(E3_ERR_UNSUPPORTED, "uvw kernels take shared weights");
  const int C = ir1[0].mul;
  for (int i = 0; i < int(ir1.size()); ++i)
    if (ir1[i].l != i || ir1[i].mul != C)
      return fail(E3_ERR_UNSUPPORTED,
                  "irreps_in1 must be Cx0+Cx1+..+CxLx (one block per degree, ascending, common multiplicity)");
  for (int i = 0; i < int(ir2.size()); ++i)
    if (ir2[i].l != i || ir2[i].mul != 1) return fail(E3_ERR_UNSUPPORTED, "irreps_in2 must be 1x0+1x1+..+1xLy");
  const int Co = irf[0].mul;
  for (const auto& c : irf)
    if (c.mul != Co) return fail(E3_ERR_UNSUPPORTED, "uvw output blocks need one common multiplicity");
  if (C % 32 != 0 || C > 128 || Co % 32 != 0 || Co > 128)
    return fail(E3_ERR_UNSUPPORTED, "uvw kernels need multiplicities in {32, 64, 96, 128} (got %d and %d)", C, Co);
  const int LX = int(ir1.size()) - 1, LY = int(ir2.size()) - 1;
  int LO = 0;
  for (const auto& c : irf) LO = std::max(LO, c.l);
  if (LX > E3_LMAX || LY > E3_LMAX || LO > E3_LMAX) return fail(E3_ERR_UNSUPPORTED, "degrees above %d have no kernel", E3_LMAX);
  if (int(ins.size()) > UVW_MAXP || int(irf.size()) > UVW_MAXT)
    return fail(E3_ERR_UNSUPPORTED, "at most %d paths and %d output blocks", UVW_MAXP, UVW_MAXT);

  auto* plan = new (std::nothrow) e3_plan();
  if (plan == nullptr) return fail(E3_ERR_INVALID_ARG, "out of host memory");
  if (cudaGetDevice(&plan->device) != cudaSuccess) {
    delete plan;
    return fail(E3_ERR_CUDA, "cudaGetDevice failed");
  }
  plan->dtype = dtype;
  plan->wmode = wmode;
  plan->mode = E3_UVW;
  plan->C = C;
  plan->Co = Co;
  plan->LX = LX;
  plan->LY = LY;
  plan->LO = LO;
  plan->n_paths = int(ins.size());
  for (const auto& c : irf) {
    plan->out_off.push_back(int(plan->dim_out));
    plan->out_l.push_back(c.l);
    plan->dim_out += int64_t(c.mul) * (2 * c.l + 1);
  }
  std::vector<int> n_out(irf.size(), 0);
  for (const auto& s : ins) n_out[s.io] += 1;
  for (const auto& s : ins) {
    const int l1 = ir1[s.i1].l, l3 = irf[s.io].l;
    plan->z_off.push_back(int(plan->uvw_z_row));
    plan->uvw_z_row += 2 * l3 + 1;
    plan->l1.push_back(l1);
    plan->l2.push_back(ir2[s.i2].l);
    plan->l3.push_back(l3);
    plan->io.push_back(s.io);
    plan->x_off.push_back(C * l1 * l1);
    plan->g_off.push_back(plan->out_off[s.io]);
    plan->alpha.push_back(s.pw >= 0 ? s.pw : std::sqrt((2.0 * l3 + 1.0) / (double(C) * n_out[s.io])));
  }
  plan->dim1 = int64_t(C) * (LX + 1) * (LX + 1);
  plan->dim2 = int64_t(LY + 1) * (LY + 1);
  plan->weight_numel = int64_t(plan->n_paths) * C * Co;
  plan->irreps_out = irreps_to_string(irf);
  packed_cg_table();
  e3_status st = ensure_device_tables();
  if (st == E3_OK) {
    plan->uvw_prep_size = uvw_prep_bytes(plan->n_paths, C, Co);
    if (cudaMalloc(&plan->uvw_prep, plan->uvw_prep_size) != cudaSuccess) {
      plan->uvw_prep = nullptr;
      st = fail(E3_ERR_CUDA, "allocating the weight staging buffer (%zu bytes) failed", plan->uvw_prep_size);
    }
  }
  if (st == E3_OK) {
    // grad_y goes through Z_p = W_p g for every path, a batch of samples at a time (<= 256 MiB)
    plan->uvw_z_row *= C;
    plan->uvw_z_batch = std::max<int64_t>(128, std::min<int64_t>(16384, (int64_t(1) << 28) / (4 * plan->uvw_z_row)));
    if (cudaMalloc(&plan->uvw_z, size_t(plan->uvw_z_batch) * plan->uvw_z_row * 4) != cudaSuccess) {
      plan->uvw_z = nullptr;
      st = fail(E3_ERR_CUDA, "allocating the grad_y staging buffer failed");
    }
  }
  if (st == E3_OK) st = plan_attach_status(plan);
  if (st != E3_OK) {
    delete plan;
    return st;
  }
  *plan_out = plan;
  return E3_OK;
}

extern "C" e3_status e3_plan_create(const char* irreps_in1, const char* irreps_in2,
                                    const char* irreps_out, const e3_instruction* instr,
                                    int32_t n_instr, e3_mode mode, e3_dtype dtype,
                                    e3_weight_mode wmode, e3_plan** plan_out) {
  clear_error();
  if (plan_out == nullptr) return fail(E3_ERR_INVALID_ARG, "plan output pointer is NULL");
  *plan_out = nullptr;
  if (dtype != E3_F32 && dtype != E3_F64) return fail(E3_ERR_INVALID_ARG, "bad dtype %d", int(dtype));
  if (wmode != E3_W_PER_SAMPLE && wmode != E3_W_SHARED)
    return fail(E3_ERR_INVALID_ARG, "bad weight mode %d", int(wmode));
  if (mode != E3_UVU && mode != E3_UVW && mode != E3_UUU && mode != E3_UUW)
    return fail(E3_ERR_INVALID_ARG, "bad connection mode %d", int(mode));
  if (n_instr < 0 || (n_instr > 0 && instr == nullptr))
    return fail(E3_ERR_INVALID_ARG, "bad instruction list");

  std::vector<IrrepT> ir1, ir2, irf;
  std::string why;
  if (!parse_irreps(irreps_in1, &ir1, &why)) return fail(E3_ERR_IRREPS_PARSE, "irreps_in1: %s", why.c_str());
  if (!parse_irreps(irreps_in2, &ir2, &why)) return fail(E3_ERR_IRREPS_PARSE, "irreps_in2: %s", why.c_str());
  const bool have_out = irreps_out != nullptr && irreps_out[strspn(irreps_out, " \t")] != '\0';
  if (have_out && !parse_irreps(irreps_out, &irf, &why))
    return fail(E3_ERR_IRREPS_PARSE, "irreps_out: %s", why.c_str());
  if (n_instr > 0 && !have_out)
    return fail(E3_ERR_INSTRUCTION, "explicit instructions need irreps_out");
  if (mode == E3_UVW) return create_uvw(ir1, ir2, irf, have_out, instr, n_instr, dtype, wmode, plan_out);

  // instructions: (i1, i2, i_out, alpha_override); output irreps
  struct Ins {
    int i1, i2, io;
    double pw;
  };
  std::vector<Ins> ins;
  std::vector<IrrepT> out_irreps;
  if (n_instr == 0) {
    for (int i1 = 0; i1 < int(ir1.size()); ++i1)
      for (int i2 = 0; i2 < int(ir2.size()); ++i2) {
        const auto &a = ir1[i1], &b = ir2[i2];
        for (int l3 = std::abs(a.l - b.l); l3 <= a.l + b.l; ++l3) {
          const int p3 = a.p * b.p;
          bool ok = !have_out;
          for (const auto& f : irf) ok = ok || (f.l == l3 && f.p == p3);
          if (!ok) continue;
          ins.push_back({i1, i2, int(out_irreps.size()), -1.0});
          out_irreps.push_back({a.mul, l3, p3});  // uvu and uuu: output channel u of x
        }
      }
    if (ins.empty()) return fail(E3_ERR_INSTRUCTION, "no allowed path between the inputs and the output filter");
  } else {
    out_irreps = irf;
    for (int q = 0; q < n_instr; ++q) {
      const auto& s = instr[q];
      if (s.i_in1 < 0 || s.i_in1 >= int(ir1.size()) || s.i_in2 < 0 || s.i_in2 >= int(ir2.size()) ||
          s.i_out < 0 || s.i_out >= int(out_irreps.size()))
        return fail(E3_ERR_INSTRUCTION, "instruction %d: index out of range", q);
      const auto &a = ir1[s.i_in1], &b = ir2[s.i_in2], &c = out_irreps[s.i_out];
      if (!triangle(a.l, b.l, c.l))
        return fail(E3_ERR_INSTRUCTION, "instruction %d: triangle rule |l1-l2| <= l3 <= l1+l2 fails (%d,%d,%d)",
                    q, a.l, b.l, c.l);
      if (c.p != a.p * b.p)
        return fail(E3_ERR_INSTRUCTION, "instruction %d: parity rule p3 = p1 p2 fails", q);
      if ((mode == E3_UVU || mode == E3_UUU) && c.mul != a.mul)
        return fail(E3_ERR_INSTRUCTION, "instruction %d: %s needs mul_out == mul_in1", q, mode == E3_UVU ? "uvu" : "uuu");
      if (mode == E3_UUU && b.mul != a.mul)
        return fail(E3_ERR_INSTRUCTION, "instruction %d: uuu needs mul_in2 == mul_in1", q);
      if (!s.has_weight)
        return fail(E3_ERR_UNSUPPORTED, "instruction %d: paths without weights have no kernel", q);
      ins.push_back({s.i_in1, s.i_in2, s.i_out, s.path_weight});
    }
  }
  if (mode != E3_UVU && mode != E3_UUU)
    return fail(E3_ERR_UNSUPPORTED, "the uvu, uuu and uvw connection modes have kernels; this mode has none");

  // layout the kernels are compiled for
  const int C = ir1[0].mul;
  for (int i = 0; i < int(ir1.size()); ++i)
    if (ir1[i].l != i || ir1[i].mul != C)
      return fail(E3_ERR_UNSUPPORTED,
                  "irreps_in1 must be Cx0+Cx1+..+CxLx (one block per degree, ascending, common multiplicity)");
  const int mul2 = mode == E3_UUU ? C : 1;
  for (int i = 0; i < int(ir2.size()); ++i)
    if (ir2[i].l != i || ir2[i].mul != mul2)
      return fail(E3_ERR_UNSUPPORTED, mode == E3_UUU ? "irreps_in2 must be Cx0+Cx1+..+CxLy in the uuu mode"
                                                      : "irreps_in2 must be 1x0+1x1+..+1xLy");
  const int LX = int(ir1.size()) - 1, LY = int(ir2.size()) - 1;
  if (mode == E3_UVU && (C % 4 != 0 || !((C / 4) <= 32 ? (32 % (C / 4) == 0) : ((C / 4) % 32 == 0))))
    return fail(E3_ERR_UNSUPPORTED, "multiplicity %d: kernels need C in {4, 8, 16, 32, 64} or a multiple of 128", C);
  int LO = 0;
  for (const auto& s : ins) LO = std::max(LO, out_irreps[s.io].l);
  if (LX > E3_LMAX || LY > E3_LMAX || LO > E3_LMAX)
    return fail(E3_ERR_UNSUPPORTED, "degrees above %d have no kernel", E3_LMAX);
  // the instruction list must be the full enumeration for (LX, LY, LO), uncollapsed, with
  // output blocks in instruction order
  const int P = n_paths(LX, LY, LO);
  bool same = int(ins.size()) == P && int(out_irreps.size()) == P;
  for (int p = 0; same && p < P; ++p) {
    same = ir1[ins[p].i1].l == path_l(LX, LY, LO, p, 0) && ir2[ins[p].i2].l == path_l(LX, LY, LO, p, 1) &&
           out_irreps[ins[p].io].l == path_l(LX, LY, LO, p, 2) && ins[p].io == p;
  }
  if (!same)
    return fail(E3_ERR_UNSUPPORTED,
                "kernels need every path with l3 <= %d, one output block per instruction in order", LO);
  if (!degrees_supported(LX, LY, LO))
    return fail(E3_ERR_UNSUPPORTED, "(Lx, Ly, Lo) = (%d, %d, %d) is not compiled; compiled: %s", LX, LY, LO,
                supported_list());

  auto* plan = new (std::nothrow) e3_plan();
  if (plan == nullptr) return fail(E3_ERR_INVALID_ARG, "out of host memory");
  if (cudaGetDevice(&plan->device) != cudaSuccess) {
    delete plan;
    return fail(E3_ERR_CUDA, "cudaGetDevice failed");
  }
  plan->dtype = dtype;
  plan->wmode = wmode;
  plan->mode = mode;
  plan->C = C;
  plan->LX = LX;
  plan->LY = LY;
  plan->LO = LO;
  plan->n_paths = P;
  std::vector<int> n_out(out_irreps.size(), 0);
  for (const auto& s : ins) n_out[s.io] += 1;
  for (int p = 0; p < P; ++p) {
    const auto &b = ir2[ins[p].i2], &c = out_irreps[ins[p].io];
    plan->l1.push_back(ir1[ins[p].i1].l);
    plan->l2.push_back(b.l);
    plan->l3.push_back(c.l);
    // default path weight: unit second moment of every output component for unit-variance
    // inputs; the fan-in of one output element is mul_in2 channels in uvu and one in uuu
    const double fan_in = mode == E3_UUU ? 1.0 : double(b.mul);
    plan->alpha.push_back(ins[p].pw >= 0 ? ins[p].pw : std::sqrt((2.0 * c.l + 1.0) / (fan_in * n_out[ins[p].io])));
  }
  for (const auto& a : ir1) plan->dim1 += int64_t(a.mul) * (2 * a.l + 1);
  for (const auto& b : ir2) plan->dim2 += int64_t(b.mul) * (2 * b.l + 1);
  for (const auto& c : out_irreps) plan->dim_out += int64_t(c.mul) * (2 * c.l + 1);
  plan->weight_numel = int64_t(P) * C;
  plan->irreps_out = irreps_to_string(out_irreps);
  packed_cg_table();
  e3_status st = ensure_device_tables();
  if (st == E3_OK) st = plan_attach_status(plan);
  if (st != E3_OK) {
    delete plan;
    return st;
  }
  *plan_out = plan;
  return E3_OK;
}

extern "C" e3_status e3_plan_destroy(e3_plan* plan) {
  clear_error();
  delete plan;
  return E3_OK;
}

extern "C" e3_status e3_plan_info(const e3_plan* plan, int64_t* dim_in1, int64_t* dim_in2, int64_t* dim_out,
                                  int64_t* weight_numel, int32_t* n_paths_out) {
  clear_error();
  if (plan == nullptr) return fail(E3_ERR_INVALID_ARG, "plan is NULL");
  if (dim_in1) *dim_in1 = plan->dim1;
  if (dim_in2) *dim_in2 = plan->dim2;
  if (dim_out) *dim_out = plan->dim_out;
  if (weight_numel) *weight_numel = plan->weight_numel;
  if (n_paths_out) *n_paths_out = plan->n_paths;
  return E3_OK;
}

extern "C" e3_status e3_plan_irreps_out(const e3_plan* plan, char* buf, size_t buf_len, size_t* needed) {
  clear_error();
  if (plan == nullptr) return fail(E3_ERR_INVALID_ARG, "plan is NULL");
  const size_t n = plan->irreps_out.size() + 1;
  if (needed) *needed = n;
  if (buf != nullptr) {
    if (buf_len < n) return fail(E3_ERR_SHAPE, "buffer of %zu bytes, need %zu", buf_len, n);
    std::memcpy(buf, plan->irreps_out.c_str(), n);
  }
  return E3_OK;
}

extern "C" e3_status e3_plan_paths(const e3_plan* plan, int32_t* lls, double* alpha) {
  clear_error();
  if (plan == nullptr) return fail(E3_ERR_INVALID_ARG, "plan is NULL");
  for (int p = 0; p < plan->n_paths; ++p) {
    if (lls) {
      lls[3 * p] = plan->l1[p];
      lls[3 * p + 1] = plan->l2[p];
      lls[3 * p + 2] = plan->l3[p];
    }
    if (alpha) alpha[p] = plan->alpha[p];
  }
  return E3_OK;
}

static e3_status check_plan_device(const e3_plan* plan);

// Read and clear the status words `words` (device pointers) in stream order after synchronising
// `stream`; the first nonzero one is the result.
static e3_status drain_status(const std::vector<int*>& words, void* stream, const char* who) {
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  std::vector<int> h(words.size(), 0);
  for (size_t i = 0; i < words.size(); ++i)
    if (cudaMemcpyAsync(&h[i], words[i], sizeof(int), cudaMemcpyDeviceToHost, s) != cudaSuccess ||
        cudaMemsetAsync(words[i], 0, sizeof(int), s) != cudaSuccess)
      return fail(E3_ERR_CUDA, "reading a status word failed: %s", cudaGetErrorString(cudaGetLastError()));
  if (cudaStreamSynchronize(s) != cudaSuccess)
    return fail(E3_ERR_CUDA, "reading a status word failed: %s", cudaGetErrorString(cudaGetLastError()));
  for (int v : h)
    if (v != E3_OK)
      return fail(static_cast<e3_status>(v), "%s reported %s", who,
                  v == E3_ERR_INDEX ? "an index out of range" : (v == E3_ERR_TIMEOUT ? "a wait that gave up" : "an error"));
  return E3_OK;
}

extern "C" e3_status e3_device_status(void* stream) {
  clear_error();
  int* d = nullptr;
  e3_status st = device_status_ptr(&d);
  if (st != E3_OK) return st;
  int dev = -1;
  cudaGetDevice(&dev);
  std::vector<int*> words{d};
  {
    std::lock_guard<std::mutex> lock(g_plans_mu);
    for (e3_plan* p : g_plans)
      if (p->device == dev && p->status != nullptr) words.push_back(p->status);
  }
  return drain_status(words, stream, "device");
}

extern "C" e3_status e3_plan_status(const e3_plan* plan, void* stream) {
  clear_error();
  const e3_status st = check_plan_device(plan);
  if (st != E3_OK) return st;
  if (plan->status == nullptr) return fail(E3_ERR_INVALID_ARG, "plan has no status word");
  return drain_status({plan->status}, stream, "plan");
}

// ========================================================= C ABI: compute entry points ===

static bool misaligned(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) != 0; }

static e3_status check_plan_device(const e3_plan* plan) {
  if (plan == nullptr) return fail(E3_ERR_INVALID_ARG, "plan is NULL");
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return fail(E3_ERR_CUDA, "cudaGetDevice failed");
  if (dev != plan->device)
    return fail(E3_ERR_INVALID_ARG, "plan belongs to device %d but device %d is current", plan->device, dev);
  return E3_OK;
}

#define E3_REQ(ptr, name)                                                        \
  do {                                                                           \
    if ((ptr) == nullptr) return fail(E3_ERR_INVALID_ARG, "%s is NULL", name);   \
    if (misaligned(ptr)) return fail(E3_ERR_INVALID_ARG, "%s is not 16-byte aligned", name); \
  } while (0)
#define E3_OPT(ptr, name)                                                        \
  do {                                                                           \
    if ((ptr) != nullptr && misaligned(ptr))                                     \
      return fail(E3_ERR_INVALID_ARG, "%s is not 16-byte aligned", name);        \
  } while (0)

static UuuArgs uuu_args(const e3_plan* plan, int64_t B, const void* x, const void* y, const void* w,
                        int64_t w_stride, void* stream) {
  UuuArgs u{};
  u.B = B;
  u.C = plan->C;
  u.dim1 = plan->dim1;
  u.dim2 = plan->dim2;
  u.dim_out = plan->dim_out;
  u.x = x;
  u.y = y;
  u.w = w;
  u.w_stride = w_stride;
  u.stream = stream;
  for (int p = 0; p < plan->n_paths && p < UUU_MAXP; ++p) u.alpha[p] = plan->alpha[p];
  return u;
}

// Launch arguments of the uvw contraction.  Forward: targets are the output blocks, terms the paths
// into each, input x.  grad_x: targets are the x blocks, terms the paths out of each, input grad_out.
// Roles of the uvw contraction kernel.
enum { UVW_FWD = 0, UVW_GX = 1, UVW_PLAIN = 2 };

// Launch arguments of the uvw contraction.  Forward: targets are the output blocks, terms the paths
// into each, input x.  grad_x: targets are the x blocks, terms the paths out of each, input grad_out.
// Plain (for grad_y): one target per path, its Z_p block (C channels), input grad_out.
static e3_status uvw_gemm_args(const e3_plan* plan, int64_t B, int role, const void* in, const void* y, void* out,
                               UvwGemmArgs* a) {
  *a = UvwGemmArgs{};
  const bool fwd = role == UVW_FWD;
  const int P = plan->n_paths, C = plan->C, Co = plan->Co;
  a->B = B;
  a->in = static_cast<const float*>(in);
  a->in_stride = fwd ? plan->dim1 : plan->dim_out;
  a->k_in = fwd ? C : Co;
  a->y = static_cast<const float*>(y);
  a->y_stride = plan->dim2;
  a->out = static_cast<float*>(out);
  a->out_stride = fwd ? plan->dim_out : (role == UVW_GX ? plan->dim1 : plan->uvw_z_row);
  a->N = fwd ? Co : C;
  const size_t fwd_chunk = size_t(2) * Co * 32 * 4, bwd_chunk = size_t(2) * C * 32 * 4;
  a->prep = static_cast<const unsigned char*>(plan->uvw_prep) + (fwd ? 0 : size_t(P) * (C / 32) * fwd_chunk);
  a->b_chunk_bytes = uint32_t(fwd ? fwd_chunk : bwd_chunk);
  const int nt = fwd ? int(plan->out_l.size()) : (role == UVW_GX ? plan->LX + 1 : P);
  int64_t tiles = 0;
  int nterm = 0;
  for (int t = 0; t < nt; ++t) {
    UvwTarget& tg = a->tg[t];
    tg.l = fwd ? plan->out_l[t] : (role == UVW_GX ? t : plan->l3[t]);
    tg.off = fwd ? plan->out_off[t] : (role == UVW_GX ? C * t * t : C * plan->z_off[t]);
    tg.bt = 128 / (2 * tg.l + 1);
    tg.tile_begin = int32_t(tiles);
    tg.term_begin = nterm;
    for (int p = 0; p < P; ++p) {
      if ((fwd ? plan->io[p] : (role == UVW_GX ? plan->l1[p] : p)) != t) continue;
      UvwTerm& tm = a->term[nterm++];
      tm.in_off = fwd ? plan->x_off[p] : plan->g_off[p];
      tm.l_in = fwd ? plan->l1[p] : plan->l3[p];
      tm.l2 = role == UVW_PLAIN ? 0 : plan->l2[p];
      tm.chunk0 = fwd ? p * (C / 32) : p * (Co / 32);
      tm.alpha = role == UVW_PLAIN ? 1.f : float(plan->alpha[p]);
    }
    tg.term_end = nterm;
    tiles += (B + tg.bt - 1) / tg.bt;
  }
  if (tiles >= INT32_MAX) return fail(E3_ERR_SHAPE, "B = %lld is too large", (long long)B);
  a->n_targets = nt;
  a->total_tiles = int32_t(tiles);
  a->wait_ns = test_wait_limit_ns();
  a->status = plan->status;
  return E3_OK;
}

static UvwBwdArgs uvw_bwd_args(const e3_plan* plan, int64_t B, const void* x, const void* y, const void* w,
                               const void* g, void* grad_w, void* grad_y) {
  UvwBwdArgs a{};
  a.B = B;
  a.C = plan->C;
  a.Co = plan->Co;
  a.P = plan->n_paths;
  a.x = static_cast<const float*>(x);
  a.dim1 = plan->dim1;
  a.y = static_cast<const float*>(y);
  a.dim2 = plan->dim2;
  a.w = static_cast<const float*>(w);
  a.g = static_cast<const float*>(g);
  a.dim_out = plan->dim_out;
  a.grad_w = static_cast<float*>(grad_w);
  a.grad_y = static_cast<float*>(grad_y);
  a.wait_ns = test_wait_limit_ns();
  a.status = plan->status;
  for (int p = 0; p < plan->n_paths; ++p) {
    UvwPath& q = a.path[p];
    q.l1 = plan->l1[p];
    q.l2 = plan->l2[p];
    q.l3 = plan->l3[p];
    q.x_off = plan->x_off[p];
    q.g_off = plan->g_off[p];
    q.z_off = plan->z_off[p];
    q.w_off = int64_t(p) * plan->C * plan->Co;
    q.alpha = float(plan->alpha[p]);
  }
  return a;
}

extern "C" e3_status e3_tp_forward(const e3_plan* plan, int64_t B, const void* x, const void* y, const void* w,
                                   void* out, void* stream) {
  clear_error();
  e3_status st = check_plan_device(plan);
  if (st != E3_OK) return st;
  if (B < 0 || B >= (int64_t(1) << 31)) return fail(E3_ERR_SHAPE, "B = %lld out of range", (long long)B);
  if (B == 0) return E3_OK;
  E3_REQ(x, "x");
  E3_REQ(y, "y");
  E3_REQ(w, "w");
  E3_REQ(out, "out");
  FwdArgs a{};
  a.n_rows = B;
  a.x = x;
  a.y = y;
  a.vec = nullptr;
  a.sh_norm = E3_SH_COMPONENT;
  a.w = w;
  a.w_stride = plan->wmode == E3_W_SHARED ? 0 : plan->weight_numel;
  a.scale = 1.0;
  a.out = out;
  a.stream = stream;
  if (plan->mode == E3_UUU) {
    UuuArgs u = uuu_args(plan, B, x, y, w, a.w_stride, stream);
    u.out = out;
    return launch_uuu(plan, u, false);
  }
  if (plan->mode == E3_UVW) {
    st = launch_uvw_prep(plan->n_paths, plan->C, plan->Co, static_cast<const float*>(w), plan->uvw_prep, stream);
    if (st != E3_OK) return st;
    UvwGemmArgs g;
    st = uvw_gemm_args(plan, B, UVW_FWD, x, y, out, &g);
    if (st != E3_OK) return st;
    return launch_uvw_gemm(g, UVW_FWD, stream);
  }
  return launch_forward(plan, a, false);
}

extern "C" e3_status e3_backward_workspace_size(int64_t n, size_t* bytes) {
  clear_error();
  if (bytes == nullptr) return fail(E3_ERR_INVALID_ARG, "bytes is NULL");
  if (n < 0 || n >= (int64_t(1) << 31)) return fail(E3_ERR_SHAPE, "n = %lld out of range", (long long)n);
  *bytes = backward_workspace_bytes(n);
  return E3_OK;
}

int e3b::plan_groups(const e3_plan* plan) { return make_path_table(plan->LX, plan->LY, plan->LO, GROUP_OUT_CAP).ngroups; }

extern "C" e3_status e3_conv_workspace_size(const e3_plan* plan, int64_t N, int64_t E, size_t* bytes) {
  clear_error();
  if (plan == nullptr || bytes == nullptr) return fail(E3_ERR_INVALID_ARG, "plan or bytes is NULL");
  if (N < 0 || E < 0 || N >= (int64_t(1) << 31) || E >= (int64_t(1) << 31)) return fail(E3_ERR_SHAPE, "N or E out of range");
  if (plan->mode != E3_UVU) return fail(E3_ERR_UNSUPPORTED, "the convolution has kernels for the uvu mode only");
  *bytes = conv_workspace_bytes(plan, N, E, plan_groups(plan));
  return E3_OK;
}

static e3_status check_conv_workspace(const e3_plan* plan, int64_t N, int64_t E, const void* topo, const void* ws,
                                      size_t ws_bytes) {
  if (topo == nullptr) return fail(E3_ERR_INVALID_ARG, "topology buffer is NULL");
  if (reinterpret_cast<uintptr_t>(topo) % 16 != 0) return fail(E3_ERR_INVALID_ARG, "topology buffer is not 16-byte aligned");
  if (ws == nullptr) return fail(E3_ERR_INVALID_ARG, "workspace is NULL");
  if (reinterpret_cast<uintptr_t>(ws) % 16 != 0) return fail(E3_ERR_INVALID_ARG, "workspace is not 16-byte aligned");
  const size_t need = conv_workspace_bytes(plan, N, E, plan_groups(plan));
  if (ws_bytes < need) return fail(E3_ERR_INVALID_ARG, "workspace of %zu bytes, need %zu", ws_bytes, need);
  return E3_OK;
}

static e3_status check_workspace(int64_t n, const void* ws, size_t ws_bytes) {
  if (ws == nullptr) return fail(E3_ERR_INVALID_ARG, "workspace is NULL");
  if (reinterpret_cast<uintptr_t>(ws) % 16 != 0) return fail(E3_ERR_INVALID_ARG, "workspace is not 16-byte aligned");
  if (ws_bytes < backward_workspace_bytes(n))
    return fail(E3_ERR_INVALID_ARG, "workspace of %zu bytes, need %zu", ws_bytes, backward_workspace_bytes(n));
  return E3_OK;
}

extern "C" e3_status e3_tp_backward(const e3_plan* plan, int64_t B, const void* x, const void* y, const void* w,
                                    const void* grad_out, void* grad_x, void* grad_y, void* grad_w,
                                    void* workspace, size_t workspace_bytes, void* stream) {
  clear_error();
  e3_status st = check_plan_device(plan);
  if (st != E3_OK) return st;
  if (plan->wmode == E3_W_SHARED && plan->mode != E3_UVW)
    return fail(E3_ERR_UNSUPPORTED, "backward with shared weights has no kernel");
  if (B < 0 || B >= (int64_t(1) << 31)) return fail(E3_ERR_SHAPE, "B = %lld out of range", (long long)B);
  if (B == 0) return E3_OK;
  E3_REQ(x, "x");
  E3_REQ(y, "y");
  E3_REQ(w, "w");
  E3_REQ(grad_out, "grad_out");
  E3_OPT(grad_x, "grad_x");
  E3_OPT(grad_y, "grad_y");
  E3_OPT(grad_w, "grad_w");
  if (!grad_x && !grad_y && !grad_w) return E3_OK;
  st = check_workspace(B, workspace, workspace_bytes);
  if (st != E3_OK) return st;
  BwdArgs a{};
  a.workspace = workspace;
  a.workspace_bytes = workspace_bytes;
  a.n_nodes = B;
  a.n_edges = B;
  a.x = x;
  a.y = y;
  a.sh_norm = E3_SH_COMPONENT;
  a.w = w;
  a.grad_out = grad_out;
  a.scale = 1.0;
  a.grad_x = grad_x;
  a.grad_y = grad_y;
  a.grad_w = grad_w;
  a.stream = stream;
  if (plan->mode == E3_UVW) {
    if (grad_x || grad_y) {
      st = launch_uvw_prep(plan->n_paths, plan->C, plan->Co, static_cast<const float*>(w), plan->uvw_prep, stream);
      if (st != E3_OK) return st;
    }
    if (grad_x) {
      UvwGemmArgs g;
      st = uvw_gemm_args(plan, B, UVW_GX, grad_out, y, grad_x, &g);
      if (st == E3_OK) st = launch_uvw_gemm(g, UVW_GX, stream);
      if (st != E3_OK) return st;
    }
    const UvwBwdArgs b = uvw_bwd_args(plan, B, x, y, w, grad_out, grad_w, grad_y);
    if (grad_w) {
      st = launch_uvw_grad_w(b, stream);
      if (st != E3_OK) return st;
    }
    if (grad_y) {
      // Z_p = W_p g for a batch of samples on the tensor cores, then the contraction with x
      for (int64_t b0 = 0; b0 < B; b0 += plan->uvw_z_batch) {
        const int64_t nb = std::min<int64_t>(plan->uvw_z_batch, B - b0);
        UvwGemmArgs g;
        st = uvw_gemm_args(plan, nb, UVW_PLAIN, static_cast<const float*>(grad_out) + b0 * plan->dim_out, y,
                           plan->uvw_z, &g);
        if (st == E3_OK) st = launch_uvw_gemm(g, UVW_PLAIN, stream);
        if (st == E3_OK)
          st = launch_uvw_grad_y(b, static_cast<const float*>(plan->uvw_z), plan->uvw_z_row, b0, nb, stream);
        if (st != E3_OK) return st;
      }
    }
    return E3_OK;
  }
  if (plan->mode == E3_UUU) {
    UuuArgs u = uuu_args(plan, B, x, y, w, plan->weight_numel, stream);
    u.grad_out = grad_out;
    u.grad_x = grad_x;
    u.grad_y = grad_y;
    u.grad_w = grad_w;
    return launch_uuu(plan, u, true);
  }
  return launch_backward(plan, a, false);
}

static e3_status check_conv_common(const e3_plan* plan, int64_t N, int64_t E, const void* y, const void* vec,
                                   e3_sh_norm sh_norm) {
  if (plan->mode != E3_UVU) return fail(E3_ERR_UNSUPPORTED, "the convolution has kernels for the uvu mode only");
  if (N < 0 || N >= (int64_t(1) << 31)) return fail(E3_ERR_SHAPE, "N = %lld out of range", (long long)N);
  if (E < 0 || E >= (int64_t(1) << 31)) return fail(E3_ERR_SHAPE, "E = %lld out of range", (long long)E);
  if (E > 0 && (y == nullptr) == (vec == nullptr)) return fail(E3_ERR_INVALID_ARG, "give exactly one of y and edge_vec");
  if (vec != nullptr && (sh_norm < E3_SH_COMPONENT || sh_norm > E3_SH_NORM))
    return fail(E3_ERR_INVALID_ARG, "bad sh_norm %d", int(sh_norm));
  if (vec != nullptr && (reinterpret_cast<uintptr_t>(vec) % (plan->dtype == E3_F64 ? 8 : 4)) != 0)
    return fail(E3_ERR_INVALID_ARG, "edge_vec is not aligned to its element size");
  return E3_OK;
}

extern "C" e3_status e3_conv_forward(const e3_plan* plan, int64_t N, int64_t E, const int32_t* row_ptr_dst,
                                     const int32_t* src, const void* x, const void* y, const void* edge_vec,
                                     e3_sh_norm sh_norm, const void* w, double out_scale, void* out,
                                     const void* topo, void* workspace, size_t workspace_bytes, void* stream) {
  clear_error();
  e3_status st = check_plan_device(plan);
  if (st != E3_OK) return st;
  st = check_conv_common(plan, N, E, y, edge_vec, sh_norm);
  if (st != E3_OK) return st;
  if (N == 0) return E3_OK;
  E3_REQ(out, "out");
  if (row_ptr_dst == nullptr) return fail(E3_ERR_INVALID_ARG, "row_ptr_dst is NULL");
  if (E > 0) {
    E3_REQ(x, "x");
    E3_REQ(w, "w");
    E3_OPT(y, "y");
    if (src == nullptr) return fail(E3_ERR_INVALID_ARG, "src is NULL");
  }
  if (!std::isfinite(out_scale)) return fail(E3_ERR_INVALID_ARG, "out_scale is not finite");
  st = check_conv_workspace(plan, N, E, topo, workspace, workspace_bytes);
  if (st != E3_OK) return st;
  FwdArgs a{};
  a.topo = topo;
  a.workspace = workspace;
  a.n_rows = N;
  a.n_edges = E;
  a.row_ptr = row_ptr_dst;
  a.src = src;
  a.x = x;
  a.y = y;
  a.vec = edge_vec;
  a.sh_norm = sh_norm;
  a.w = w;
  a.w_stride = plan->wmode == E3_W_SHARED ? 0 : plan->weight_numel;
  a.scale = out_scale;
  a.out = out;
  a.stream = stream;
  return launch_forward(plan, a, true);
}

extern "C" e3_status e3_conv_backward(const e3_plan* plan, int64_t N, int64_t E, const int32_t* row_ptr_dst,
                                      const int32_t* src, const int32_t* dst, const int32_t* row_ptr_src,
                                      const int32_t* perm_src, const void* x, const void* y, const void* edge_vec,
                                      e3_sh_norm sh_norm, const void* w, const void* grad_out, double out_scale,
                                      void* grad_x, void* grad_y, void* grad_w, const void* topo, void* workspace,
                                      size_t workspace_bytes,
                                      void* stream) {
  clear_error();
  (void)src;
  e3_status st = check_plan_device(plan);
  if (st != E3_OK) return st;
  if (plan->wmode == E3_W_SHARED) return fail(E3_ERR_UNSUPPORTED, "backward with shared weights has no kernel");
  st = check_conv_common(plan, N, E, y, edge_vec, sh_norm);
  if (st != E3_OK) return st;
  E3_OPT(grad_x, "grad_x");
  E3_OPT(grad_y, "grad_y");
  E3_OPT(grad_w, "grad_w");
  if (!grad_x && !grad_y && !grad_w) return E3_OK;
  if (N == 0) {  // without nodes every edge is padding: zero gradients
    const size_t es = plan->dtype == E3_F64 ? 8 : 4;
    cudaError_t err = cudaSuccess;
    if (E > 0 && grad_w != nullptr)
      err = cudaMemsetAsync(grad_w, 0, size_t(E) * es * plan->weight_numel, static_cast<cudaStream_t>(stream));
    if (err == cudaSuccess && E > 0 && grad_y != nullptr)
      err = cudaMemsetAsync(grad_y, 0, size_t(E) * es * plan->dim2, static_cast<cudaStream_t>(stream));
    if (err != cudaSuccess) return fail(E3_ERR_CUDA, "memset failed: %s", cudaGetErrorString(err));
    return E3_OK;
  }
  if (row_ptr_src == nullptr) return fail(E3_ERR_INVALID_ARG, "row_ptr_src is NULL");
  if (E > 0) {
    E3_REQ(x, "x");
    E3_REQ(w, "w");
    E3_REQ(grad_out, "grad_out");
    E3_OPT(y, "y");
    if (dst == nullptr || perm_src == nullptr) return fail(E3_ERR_INVALID_ARG, "dst or perm_src is NULL");
  }
  if (!std::isfinite(out_scale)) return fail(E3_ERR_INVALID_ARG, "out_scale is not finite");
  st = check_conv_workspace(plan, N, E, topo, workspace, workspace_bytes);
  if (st != E3_OK) return st;
  BwdArgs a{};
  a.topo = topo;
  a.workspace = workspace;
  a.workspace_bytes = workspace_bytes;
  a.n_nodes = N;
  a.n_edges = E;
  a.row_ptr_dst = row_ptr_dst;
  a.row_ptr_src = row_ptr_src;
  a.perm_src = perm_src;
  a.dst = dst;
  a.x = x;
  a.y = y;
  a.vec = edge_vec;
  a.sh_norm = sh_norm;
  a.w = w;
  a.grad_out = grad_out;
  a.scale = out_scale;
  a.grad_x = grad_x;
  a.grad_y = grad_y;
  a.grad_w = grad_w;
  a.stream = stream;
  st = launch_backward(plan, a, true);
  if (st != E3_OK) return st;
  // padding edges (receiver-order positions from row_ptr_dst[N] on) get zero gradients
  const size_t es = plan->dtype == E3_F64 ? 8 : 4;
  if (E > 0 && grad_w != nullptr) {
    st = zero_rows_after(row_ptr_dst + N, E, int64_t(es) * plan->weight_numel, grad_w, stream);
    if (st != E3_OK) return st;
  }
  if (E > 0 && grad_y != nullptr) st = zero_rows_after(row_ptr_dst + N, E, int64_t(es) * plan->dim2, grad_y, stream);
  return st;
}
