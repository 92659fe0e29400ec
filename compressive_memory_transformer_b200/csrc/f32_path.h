// f32_path.h — internal interface of the fp32 SIMT forward (see f32_path.cu).
#pragma once
#include <cstddef>
#include <cuda_runtime.h>

namespace infini {

size_t f32_workspace_bytes(int BH, int S, int d);

// Launches the fp32 forward on `stream`. `workspace` holds f32_workspace_bytes()
// bytes (256-byte aligned). Requires L >= 1, N >= 1, 1 <= d <= 128.
cudaError_t f32_forward_launch(const float* q, const float* k, const float* v, const float* beta,
                               const float* M_in, const float* z_in, float* out, float* M_out,
                               float* z_out, int BH, int H, long long L, int N, int d, int mode,
                               void* workspace, cudaStream_t stream);

}  // namespace infini
