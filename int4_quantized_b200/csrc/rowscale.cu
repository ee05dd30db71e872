// rowscale.cu -- scales of groups that span whole rows, spread to one scale per row.
//
// A group of g = c * K consecutive weights of an [N][K] matrix covers c whole rows (for
// g = N * K, the whole matrix: the INT4_TENSOR format of the "量化推理：INT8/INT4 ..." page),
// so row n takes scale n / c. qgemm expands such scales into its workspace and then runs
// the one-scale-per-row path on them; the values are those of the stored scales, copied.
#include <cuda_runtime.h>

#include <cstdint>

namespace q4 {
namespace {

__global__ void __launch_bounds__(256) expand_row_scales(const float *__restrict__ scales, int64_t rows_per_scale,
                                                         int64_t N, float *__restrict__ out) {
    for (int64_t n = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; n < N; n += (int64_t)gridDim.x * blockDim.x)
        out[n] = scales[n / rows_per_scale];
}

}  // namespace

cudaError_t launch_expand_row_scales(const float *scales, int64_t rows_per_scale, int64_t N, float *out,
                                     cudaStream_t st) {
    if (N <= 0) return cudaSuccess;
    const int64_t want = (N + 255) / 256;
    const unsigned blocks = (unsigned)(want < 4096 ? want : 4096);
    expand_row_scales<<<blocks, 256, 0, st>>>(scales, rows_per_scale, N, out);
    return cudaGetLastError();
}

}  // namespace q4
