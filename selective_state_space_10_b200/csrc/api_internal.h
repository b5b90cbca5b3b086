// api_internal.h -- declarations shared between the library's C-ABI translation units.
#pragma once

#include "ssd.h"

namespace ssd {

ssd_status prefill_into_workspace(const ssd_dims *dims, ssd_dtype dtype, const void *x, const float *dt,
                                  const float *A, const void *B, const void *C, const float *D, int chunk,
                                  float *y, float *final_state, void *workspace, size_t workspace_bytes,
                                  ssd_stream_t stream);

}  // namespace ssd
