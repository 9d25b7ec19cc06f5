// Kernels of the (3, 3, 3) path set: x degrees 0..3, harmonics 0..3, outputs up to 3.
#include "kernels.cuh"

namespace e3b {

e3_status upload_tables_l333(const double* t64, const float* t32) {
  const cudaError_t err = upload_tables(t64, t32);
  if (err != cudaSuccess) return fail(E3_ERR_CUDA, "uploading the CG table failed: %s", cudaGetErrorString(err));
  return E3_OK;
}

e3_status launch_fwd_l333(const e3_plan* plan, const FwdArgs& a, bool conv) {
  if (plan->dtype == E3_F32) return launch_fwd_cfg<Cfg<3, 3, 3, float>>(plan, a, conv);
  return launch_fwd_cfg<Cfg<3, 3, 3, double>>(plan, a, conv);
}

e3_status launch_bwd_l333(const e3_plan* plan, const BwdArgs& a, bool conv) {
  if (plan->dtype == E3_F32) return launch_bwd_cfg<Cfg<3, 3, 3, float>>(plan, a, conv);
  return launch_bwd_cfg<Cfg<3, 3, 3, double>>(plan, a, conv);
}

}  // namespace e3b
