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

// A prefix computation run only when a device flag asks for it (the adaptive
// refresh of fbk_decode_block_adaptive). Each kernel of the computation reads
// *gate after waiting for its predecessor and returns at once when it is 0;
// when it runs, the query rotation also writes *mark = 1 and *last = step.
struct PrefixGate {
  const int *gate;
  int *mark;
  int *last;
  int step;
};

// The drift statistic of the adaptive refresh, computed by the step kernel
// (off when q_base is NULL): for every block row, the share of its softmax
// mass on the prefix times 1 - cos(queries of step next_step, queries of step
// *last_refresh), rows of q_base + step * q_stride. The maximum goes to
// *drift_out (atomic, non-negative), and when it exceeds theta the kernel sets
// next_flags[0 .. n_next) to 1. Block 0 clears *clear after its wait.
struct DriftArgs {
  const __nv_bfloat16 *q_base;
  long long q_stride;
  const int *last_refresh;
  int next_step;  // -1: no decision at this step
  int *clear;
  int *next_flags;
  int n_next;
  float theta;
  float *drift_out;
};

// fp32 CUDA-core prefix kernel (FBK_FP32_CHECK): one CTA per share.
cudaError_t launch_prefix_fp32(const Geometry &g, const __nv_bfloat16 *q, const Workspace &ws,
                               int shares, cudaStream_t st);


// Fixed-order LSE reduction of the per-share states into the prefix state.
cudaError_t launch_split_reduce(const Geometry &g, const Workspace &ws, int shares,
                                const fbk_partial &out, cudaStream_t st, const int *gate = nullptr);

// In-block attention + merge with the prefix state + normalisation; drift:
// NULL, or the adaptive refresh's statistic (bf16 path only).
cudaError_t launch_block_merge(const Geometry &g, const __nv_bfloat16 *q,
                               const __nv_bfloat16 *kb, const __nv_bfloat16 *vb,
                               const fbk_partial &pfx, void *out, float *lse, bool f32_out,
                               cudaStream_t st, const DriftArgs *drift = nullptr);

// Start of an adaptive block: flags [2][n] = (1..., 0...), last_refresh [n] =
// 0, drift and refreshed [steps][n] = 0.
cudaError_t launch_adaptive_init(int *flags, int *last_refresh, float *drift, int *refreshed, int n_layers,
                                 int steps, cudaStream_t st);

// RoPE + append of the finished block, then prefix_lens += B.
cudaError_t launch_commit(const Geometry &g, const __nv_bfloat16 *kb, const __nv_bfloat16 *vb,
                          __nv_bfloat16 *kc, __nv_bfloat16 *vc, int *lens, cudaStream_t st);

// Uncached full attention (fp32, CUDA cores).
cudaError_t launch_full_ref(const Geometry &g, const __nv_bfloat16 *q, const __nv_bfloat16 *kb,
                            const __nv_bfloat16 *vb, void *out, float *lse, bool f32_out,
                            cudaStream_t st);

}  // namespace fbk
