// Per-device state (status word, coefficient tables, SM count) and dispatch of a plan to the
// translation unit compiled for its path set.
#include <cuda_runtime.h>

#include <atomic>
#include <cstdint>
#include <mutex>
#include <vector>

#include "cg_pattern.h"
#include "internal.h"

namespace e3b {

#define E3_DECL(A, B, C)                                                              \
  e3_status upload_tables_l##A##B##C(const double* t64, const float* t32);            \
  e3_status launch_fwd_l##A##B##C(const e3_plan* plan, const FwdArgs& a, bool conv);   \
  e3_status launch_bwd_l##A##B##C(const e3_plan* plan, const BwdArgs& a, bool conv);
E3_CONFIGS(E3_DECL)
#undef E3_DECL

__device__ int g_status;  // first device-side error since the last e3_device_status()

static std::mutex g_dev_mutex;
static uint64_t g_ready = 0;  // bit per device
static int* g_status_ptr[64] = {};
static int g_sms[64] = {};

e3_status ensure_device_tables() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return fail(E3_ERR_CUDA, "cudaGetDevice failed");
  if (dev < 0 || dev >= 64) return fail(E3_ERR_UNSUPPORTED, "device index %d", dev);
  std::lock_guard<std::mutex> lock(g_dev_mutex);
  if (g_ready & (uint64_t(1) << dev)) return E3_OK;
  const std::vector<double>& t = packed_cg_table();
  const std::vector<float> tf(t.begin(), t.end());
#define E3_UP(A, B, C)                                                               \
  {                                                                                  \
    const e3_status st = upload_tables_l##A##B##C(t.data(), tf.data());              \
    if (st != E3_OK) return st;                                                      \
  }
  E3_CONFIGS(E3_UP)
#undef E3_UP
  {
    e3_status st = upload_tables_uuu(t.data(), tf.data());
    if (st == E3_OK) st = upload_tables_uvw(t.data(), tf.data());
    if (st != E3_OK) return st;
  }
  const int zero = 0;
  cudaError_t err = cudaMemcpyToSymbol(g_status, &zero, sizeof(int));
  if (err == cudaSuccess) err = cudaGetSymbolAddress(reinterpret_cast<void**>(&g_status_ptr[dev]), g_status);
  if (err == cudaSuccess) err = cudaDeviceGetAttribute(&g_sms[dev], cudaDevAttrMultiProcessorCount, dev);
  if (err != cudaSuccess) return fail(E3_ERR_CUDA, "device set-up failed: %s", cudaGetErrorString(err));
  g_ready |= uint64_t(1) << dev;
  return E3_OK;
}

e3_status device_status_ptr(int** ptr) {
  const e3_status st = ensure_device_tables();
  if (st != E3_OK) return st;
  int dev = 0;
  cudaGetDevice(&dev);
  *ptr = g_status_ptr[dev];
  return E3_OK;
}

static std::atomic<long long> g_wait_limit_ns{1000000000ll};
static std::atomic<int> g_first_ticket{0};

unsigned long long test_wait_limit_ns() { return static_cast<unsigned long long>(g_wait_limit_ns.load()); }
int test_first_ticket() { return g_first_ticket.load(); }

int sm_count() {
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64 || g_sms[dev] == 0) return 148;
  return g_sms[dev];
}

e3_status launch_forward(const e3_plan* plan, const FwdArgs& a, bool conv) {
#define E3_F(A, B, C) \
  if (plan->LX == A && plan->LY == B && plan->LO == C) return launch_fwd_l##A##B##C(plan, a, conv);
  E3_CONFIGS(E3_F)
#undef E3_F
  return fail(E3_ERR_UNSUPPORTED, "degrees (%d, %d, %d) are not compiled", plan->LX, plan->LY, plan->LO);
}

e3_status launch_backward(const e3_plan* plan, const BwdArgs& a, bool conv) {
#define E3_B(A, B, C) \
  if (plan->LX == A && plan->LY == B && plan->LO == C) return launch_bwd_l##A##B##C(plan, a, conv);
  E3_CONFIGS(E3_B)
#undef E3_B
  return fail(E3_ERR_UNSUPPORTED, "degrees (%d, %d, %d) are not compiled", plan->LX, plan->LY, plan->LO);
}

}  // namespace e3b

extern "C" e3_status e3_set_test_knobs(int64_t wait_limit_ns, int32_t first_ticket) {
  e3b::clear_error();
  if (wait_limit_ns < 0 || first_ticket < 0) return e3b::fail(E3_ERR_INVALID_ARG, "negative knob");
  e3b::g_wait_limit_ns.store(wait_limit_ns == 0 ? 1000000000ll : wait_limit_ns);
  e3b::g_first_ticket.store(first_ticket);
  return E3_OK;
}
