// lq_fp32.cuh -- entering and reading back the FP32-state reference path
// (bits = 32): the state is stored as it is, so init copies S0 into the
// blobs and read-back copies it out.  The decode step of this path (and of
// the per-step baselines) is dense_step_kernel in lq_dense.cuh.
#pragma once

#include "lq_common.cuh"

namespace lq {

constexpr int kFp32Cols = 32;      // value columns per CTA
constexpr int kFp32Threads = 128;  // 16 row groups x 8 column quads

struct Fp32Args {
    uint8_t *state;
    const float *S0;
    float *S_out;
    Layout L;
    Flags F;
    const void *q, *k, *v;
    const float *beta, *decay;
    float *out;
    int num_heads;
};

template <int D, int MODE>
__global__ void __launch_bounds__(256) fp32_copy_kernel(Fp32Args A) {
    const size_t head = blockIdx.x;
    uint8_t *blob = A.state + head * A.L.blob;
    float *S = reinterpret_cast<float *>(blob + kHdrBytes);
    const float4 *src = reinterpret_cast<const float4 *>(MODE == 1 ? A.S0 + head * (size_t)D * D : S);
    float4 *dst = reinterpret_cast<float4 *>(MODE == 1 ? S : A.S_out + head * (size_t)D * D);
    for (int x = threadIdx.x; x < D * D / 4; x += 256) dst[x] = src[x];
    if (MODE == 1 && threadIdx.x == 0) {
        uint32_t *h = reinterpret_cast<uint32_t *>(blob);
        h[0] = 0u; h[1] = 0u; h[2] = 0u; h[3] = kMagic;
        *reinterpret_cast<float *>(blob + kHdrG) = 1.f;
    }
}

}  // namespace lq
