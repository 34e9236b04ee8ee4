// Test-only kernel: the mask's float64 exponential (exp_nonpos) and CUDA's
// exp on the same arguments, so that the test can compare them.
#include <cuda_runtime.h>

#include "../adaptive_block_sparse_fractal_b200/csrc/exp_nonpos.cuh"

__global__ void both(const double *x, double *mine, double *cuda, int n) {
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i < n) {
        mine[i] = nabla::exp_nonpos(x[i]);
        cuda[i] = exp(x[i]);
    }
}

extern "C" int exp_check(const double *x, double *mine, double *cuda, int n) {
    both<<<(n + 255) / 256, 256>>>(x, mine, cuda, n);
    return static_cast<int>(cudaGetLastError());
}
