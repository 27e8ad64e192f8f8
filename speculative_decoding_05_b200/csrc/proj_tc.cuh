// proj_tc.cuh -- tensor-core (tcgen05) projection path for large batches.
#pragma once

#include "proj_simt.cuh"

namespace dspark {

struct TcPlan {
  int V, r, B, K;
};

inline bool tc_supported(int V, int r, int B) {
  (void)V;
  (void)r;
  (void)B;
  return false;
}

inline dspark_status tc_plan_draft(TcPlan&, const float*, const void*, const void*, int, int, int,
                                   int) {
  return DSPARK_ERR_UNSUPPORTED;
}
inline dspark_status tc_plan_residual(TcPlan&, const float*, const float*, const void*, const void*,
                                      int, int, int, int) {
  return DSPARK_ERR_UNSUPPORTED;
}
inline void tc_launch_draft(const TcPlan&, int, const int32_t*, const int32_t*, const float*, float*,
                            float2*, unsigned*, cudaStream_t) {}
inline void tc_launch_residual(const TcPlan&, const ResInfo*, const float*, float2*, unsigned*,
                               cudaStream_t) {}

}  // namespace dspark
