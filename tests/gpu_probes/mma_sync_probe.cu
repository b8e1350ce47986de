// mma_sync_probe.cu -- test-only kernel: one warp computes a 16x16x16 fp32
// product with the library's 3xTF32 m16n8k8 mma.sync helper, to check the
// fragment layout it assumes.  Not part of the library.
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../gated_delta_rule_135_b200/csrc/warp_mma.cuh"

namespace {
__global__ void probe(const float* P, const float* Q, float* D, int half) {
    __shared__ __align__(16) float sP[16 * 20], sQ[16 * 20], sD[16 * 20];
    const int lane = threadIdx.x;
    for (int e = lane; e < 256; e += 32) {
        sP[(e / 16) * 20 + e % 16] = P[e];
        sQ[(e / 16) * 20 + e % 16] = Q[e];
    }
    __syncwarp();
    float acc[2][4] = {};
    if (half) kda::warpmma::mm16_acc_h(sP, 20, sQ, 20, acc);
    else kda::warpmma::mm16_acc(sP, 20, sQ, 20, acc);
    kda::warpmma::store16(sD, 20, acc, 1.f);
    __syncwarp();
    for (int e = lane; e < 256; e += 32) D[e] = sD[(e / 16) * 20 + e % 16];
}
}  // namespace

extern "C" int mma_sync_probe(const float* P, const float* Q, float* D, int half) {
    probe<<<1, 32>>>(P, Q, D, half);
    return cudaDeviceSynchronize() == cudaSuccess ? 0 : -1;
}
