// proj.cuh -- internal entry points of the tensor-core projections (proj_tc.cu).
#pragma once

#include "common.cuh"

namespace csa {

size_t out_proj_workspace(int64_t M, int G, int r);
unsigned int read_proj_tc_status();

}  // namespace csa
