// calibrate_dp.h -- launchers of the data-parallel calibration (calibrate.cu).
#pragma once

#include <cuda_runtime.h>

#include "../../include/tri.h"

namespace tri {

cudaError_t launch_calibrate_sums(const void* q, tri_dtype dt, int64_t n_heads, int64_t n_tok,
                                  double* sums, void* ws, cudaStream_t s);
cudaError_t launch_calibrate_finish(const double* sums, int64_t n_heads, int64_t n_tok,
                                    float* stats, cudaStream_t s);

}  // namespace tri
