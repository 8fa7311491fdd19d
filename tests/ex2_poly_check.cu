// Accuracy check of the library's FMA-pipe 2^x (ex2_poly2) against CUDA's
// exp2f over a dense range of inputs.  Built and run by test_gpu_ex2_poly.py.
#include <cstdio>
#include <cmath>
#include "../sparse_attention_long_block_b200/csrc/tc_ptx.cuh"

__global__ void k(const float *x, float *y, float *ref, int n) {
    const int i = 2 * (blockIdx.x * blockDim.x + threadIdx.x);
    if (i + 1 >= n) return;
    float a, b;
    vnsa::ptx::ex2_poly2(a, b, x[i], x[i + 1]);
    y[i] = a;
    y[i + 1] = b;
    ref[i] = exp2f(x[i]);
    ref[i + 1] = exp2f(x[i + 1]);
}

int main() {
    const int n = 1 << 22;
    float *hx = new float[n], *hy = new float[n], *hr = new float[n];
    for (int i = 0; i < n; ++i) hx[i] = -124.0f + 132.0f * (float)i / (float)(n - 1);  // [-124, 8]
    float *dx, *dy, *dr;
    cudaMalloc(&dx, n * 4);
    cudaMalloc(&dy, n * 4);
    cudaMalloc(&dr, n * 4);
    cudaMemcpy(dx, hx, n * 4, cudaMemcpyHostToDevice);
    k<<<n / 512, 256>>>(dx, dy, dr, n);
    cudaMemcpy(hy, dy, n * 4, cudaMemcpyDeviceToHost);
    cudaMemcpy(hr, dr, n * 4, cudaMemcpyDeviceToHost);
    double worst = 0;
    for (int i = 0; i < n; ++i) {
        const double rel = fabs((double)hy[i] / (double)hr[i] - 1.0);
        if (rel > worst) worst = rel;
    }
    // clamping: -inf and very negative inputs give a tiny positive value
    float sx[2] = {-INFINITY, -1000.f}, sy[2];
    cudaMemcpy(dx, sx, 8, cudaMemcpyHostToDevice);
    k<<<1, 1>>>(dx, dy, dr, 2);
    cudaMemcpy(sy, dy, 8, cudaMemcpyDeviceToHost);
    printf("max_rel_err %.3e clamp %.3e %.3e err %s\n", worst, sy[0], sy[1],
           cudaGetErrorString(cudaGetLastError()));
    return 0;
}
