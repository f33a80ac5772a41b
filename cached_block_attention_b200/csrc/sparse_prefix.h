// Launchers of the sparse block-external attention kernels (sparse_prefix.cu),
// called by the C ABI (abi.cu).
#pragma once

#include <cuda_runtime.h>

#include "common.cuh"

namespace fbk {

// Mean key per logical page and kv-head: means [b, max_pages, Hkv, d] fp32.
cudaError_t launch_page_means(const Geometry &g, float *means, cudaStream_t st);

// Page scores and the top-k pages per sequence; qrot [b, B, Hq, d] fp32 and
// scores [b, Hkv, max_pages] fp32 are scratch; kept_table [b, k] and kept_lens [b].
cudaError_t launch_select_pages(const Geometry &g, const __nv_bfloat16 *q, const float *means, int k, float *qrot,
                                float *scores, int *kept_table, int *kept_lens, int sms, cudaStream_t st);

// Residual of dense minus sparse (rows = b * Hq * B), and its application.
cudaError_t launch_residual_capture(int rows, int d, const fbk_partial &dense, const fbk_partial &sparse, float *r_o,
                                    float *r_lse, int sms, cudaStream_t st);
cudaError_t launch_residual_apply(int rows, int d, const fbk_partial &sparse, const float *r_o, const float *r_lse,
                                  const fbk_partial &ext, int sms, cudaStream_t st);

}  // namespace fbk
