// Prefix launchers with a rotation base for the block's query rows that is
// separate from the number of cached keys (prefix_tc.cu, prefix_fp32.cu).
#pragma once

#include <cuda_runtime.h>

#include "launch.h"

namespace fbk {

// qpos: device int32 [b], row t of sequence b is rotated at qpos[b] + t; NULL
// rotates at prefix_lens[b] + t (the block right after its prefix).
// gate: NULL, or the flag that decides at run time whether the launches do
// anything (see PrefixGate).
cudaError_t launch_prefix_tc_at(const Geometry &g, const __nv_bfloat16 *q, const int *qpos, const Workspace &ws,
                                int shares, cudaStream_t st, const PrefixGate *gate = nullptr);
cudaError_t launch_prefix_fp32_at(const Geometry &g, const __nv_bfloat16 *q, const int *qpos, const Workspace &ws,
                                  int shares, cudaStream_t st);

}  // namespace fbk
