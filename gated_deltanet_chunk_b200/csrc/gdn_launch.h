// gdn_launch.h -- launchers of the libgdn.so kernels (host side, internal).
#pragma once

#include <cuda_runtime.h>

#include "gdn_common.cuh"

namespace gdn {

// fp32 CUDA-core chunked forward; dk in {64,128}, chunk in {64,128}, dv % 32 == 0.
cudaError_t launch_chunk_simt(const ChunkArgs& a, int dk, int chunk, int io_bf16, cudaStream_t s);

// Tensor-core chunked forward (tcgen05 + TMA): bf16 io, Dk = Dv = 128, chunk 64.
bool chunk_tc_supported(int dk, int dv, int chunk, int io_bf16);
cudaError_t launch_chunk_tc(const ChunkArgs& a, int64_t total_tokens, cudaStream_t s);
// One CTA whose bounded wait on a barrier nothing arrives on expires after
// limit_ns and records kStatusTimeout in *status.
cudaError_t launch_selftest_wait(uint64_t limit_ns, unsigned int* status, cudaStream_t s);

// One-token decode step; dk, dv in {64,128}.
cudaError_t launch_recurrent_step(const StepArgs& a, int dk, int dv, int io_bf16, cudaStream_t s);

// Gated RMSNorm rows: y = o / sqrt(mean(o^2) + eps) * w * silu(z); dim in {64,128}; y may be o.
cudaError_t launch_gated_rmsnorm(const void* o, const void* z, const float* w, float eps, void* y,
                                 int64_t rows, int dim, int io_bf16, cudaStream_t s);

// Causal depthwise conv1d + SiLU of q|k|v: prefill (with the final conv_state
// when state_out is set) and the one-token decode update; ksize in [1, 4].
cudaError_t launch_conv_fwd(const ConvArgs& a, int io_bf16, cudaStream_t s);
cudaError_t launch_conv_update(const ConvArgs& a, int io_bf16, cudaStream_t s);

}  // namespace gdn
