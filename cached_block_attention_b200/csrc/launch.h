// Host-side launchers of the kernels, called by the C ABI (abi.cu).
#pragma once

#include <cuda_runtime.h>

#include "common.cuh"

namespace fbk {

// Launch with programmatic stream serialization (see pdl_wait / pdl_release):
// the kernel may start while its stream predecessor finishes, and waits for it
// on the device before touching its results.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                       Args... args) {
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, args...);
}

struct TmaMaps;  // defined in prefix_tc.cu

// fp32 CUDA-core prefix kernel (FBK_FP32_CHECK): one CTA per share.
cudaError_t launch_prefix_fp32(const Geometry &g, const __nv_bfloat16 *q, const Workspace &ws,
                               int shares, cudaStream_t st);


// Fixed-order LSE reduction of the per-share states into the prefix state.
cudaError_t launch_split_reduce(const Geometry &g, const Workspace &ws, int shares,
                                const fbk_partial &out, cudaStream_t st);

// In-block attention + merge with the prefix state + normalisation.
cudaError_t launch_block_merge(const Geometry &g, const __nv_bfloat16 *q,
                               const __nv_bfloat16 *kb, const __nv_bfloat16 *vb,
                               const fbk_partial &pfx, void *out, float *lse, bool f32_out,
                               cudaStream_t st);

// RoPE + append of the finished block, then prefix_lens += B.
cudaError_t launch_commit(const Geometry &g, const __nv_bfloat16 *kb, const __nv_bfloat16 *vb,
                          __nv_bfloat16 *kc, __nv_bfloat16 *vc, int *lens, cudaStream_t st);

// Uncached full attention (fp32, CUDA cores).
cudaError_t launch_full_ref(const Geometry &g, const __nv_bfloat16 *q, const __nv_bfloat16 *kb,
                            const __nv_bfloat16 *vb, void *out, float *lse, bool f32_out,
                            cudaStream_t st);

}  // namespace fbk
