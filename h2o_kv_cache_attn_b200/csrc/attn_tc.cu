// Tensor-core (tcgen05 / TMEM / TMA) path of chunked cache attention with
// summed weights.  Not enabled in this build: every request takes the CUDA-core
// path in attn_simt.cu.
#include "h2okv_internal.cuh"

namespace h2okv {

bool tc_path_supported(const h2okv_cache_desc &) { return false; }

void tc_plan(const h2okv_cache_desc &d, TcPlan *plan) {
  plan->enabled = tc_path_supported(d);
  plan->tiles_per_head = (d.max_chunk + 127) / 128;
  plan->max_splits = 1;
}

int launch_attn_tc(h2okv_cache *, const void *, int, int64_t, void *, float *, float *, float *,
                   cudaStream_t) {
  return set_error(H2OKV_ERR_UNSUPPORTED, "tensor-core path not built");
}

}  // namespace h2okv
