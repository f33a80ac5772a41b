// Launcher of the FACache step for a sequence's unchanged rows
// (facache_rows.cu), called by the C ABI (abi.cu).
#pragma once

#include <cuda_runtime.h>

#include "common.cuh"

namespace fbk {

struct FacRowsArgs {
  const __nv_bfloat16 *q;   // [b, U, Hq, d], after RoPE
  fbk_partial state;        // [b, Hq, U, d], [b, Hq, U]
  const __nv_bfloat16 *kb;  // [b, B, Hkv, d], before RoPE
  const __nv_bfloat16 *vb;  // [b, B, Hkv, d]
  const int *block_pos;     // [b]: c0
  __nv_bfloat16 *out;       // [b, U, Hq, d]
  float *lse;               // [b, Hq, U] or null
  int n_rows;               // U
  int ctas_per_unit;        // set by the launcher
};

// One launch; sms = the device's SM count.
cudaError_t launch_facache_rows(const Geometry &g, const FacRowsArgs &a, int sms, cudaStream_t st);

// Writes the rotation base of each chunk of U's rows of one sequence (kernel
// parameters only; see facache_rows.cu).
cudaError_t launch_chunk_positions(int *pos, int n_before, int n_after, int c0, int cmax, int blk, cudaStream_t st);

}  // namespace fbk
