// lq_fp32.cuh -- the FP32-state reference path (bits = 32): every decode
// token reads the dense FP32 state of each head from HBM, updates it and
// writes it back.  This is the cost LeapQuant removes (news post "Linear
// attention has to move state every token it generates; LeapQuant
// compresses it to 8-bit without losing accuracy", second paragraph); the
// library keeps it as the comparison point for throughput and accuracy.
//
// One CTA of 4*D threads per (slot, head): thread 0 bulk-copies the D x D
// state into shared memory; thread t owns rows TI*(t%16).. and columns
// 4*(t/16).. (TI = D/16), forms S' = D_t S in registers, the column sums
// S'^T k and S'^T q go through shared memory, and the thread writes
// S' + k u^T straight back with 16-byte stores.
#pragma once

#include "lq_common.cuh"

namespace lq {

template <int D>
__host__ __device__ constexpr uint32_t fp32_smem_bytes() {
    // bar/hdr 128 | k, q, a, u [D] | partials 2 x [16][D] | state D*D
    return 128u + (4u * D + 32u * D) * 4u + (uint32_t)D * D * 4u;
}

struct Fp32Args {
    uint8_t *state;
    const float *S0;
    float *S_out;
    Layout L;
    Flags F;
    const void *q, *k, *v;
    const float *beta, *decay;
    float *out;
};

template <int D>
__global__ void __launch_bounds__(4 * D) fp32_decode_kernel(Fp32Args A) {
    constexpr int TI = D / 16;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int ic = tid & 15, jc = tid >> 4, i0 = TI * ic, j0 = 4 * jc;
    const size_t head = blockIdx.x;
    const Flags &F = A.F;
    uint8_t *blob = A.state + head * A.L.blob;
    float *S = reinterpret_cast<float *>(blob + kHdrBytes);

    extern __shared__ __align__(128) uint8_t smem[];
    uint64_t *bar = reinterpret_cast<uint64_t *>(smem);
    uint32_t *s_hdr = reinterpret_cast<uint32_t *>(smem + 16);
    float *s_k = reinterpret_cast<float *>(smem + 128);
    float *s_q = s_k + D, *s_a = s_q + D, *s_u = s_a + D;
    float *s_pk = s_u + D;            // [16][D]
    float *s_pq = s_pk + 16 * D;      // [16][D]
    float *s_S = s_pq + 16 * D;       // [D][D]

    if (tid == 0) {
        const uint4 h = *reinterpret_cast<const uint4 *>(blob);
        const bool run = h.w == kMagic && h.y == 0;
        s_hdr[0] = run ? 1u : 0u;
        if (h.w != kMagic && h.y == 0) set_status(blob, LQ_DEV_CORRUPT);
        if (run) {
            mbar_init(&bar[0], 1);
            fence_mbar_init();
            mbar_arrive_expect_tx(&bar[0], (uint32_t)D * D * 4u);
            bulk_g2s(s_S, S, (uint32_t)D * D * 4u, &bar[0]);
        }
    }
    float vv = 0.f, kq = 0.f;
    if (tid < D) {
        const size_t o = head * D + tid;
        const float kv = load_in(A.k, o, F.bf16_in), qv = load_in(A.q, o, F.bf16_in);
        vv = load_in(A.v, o, F.bf16_in);
        s_k[tid] = kv;
        s_q[tid] = qv;
        s_a[tid] = F.kda ? A.decay[o] : A.decay[head];
        kq = kv * qv;
    }
    const float bt = A.beta[head];
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) kq += __shfl_xor_sync(0xFFFFFFFFu, kq, off);
    if (lane == 0) s_pk[warp] = kq;  // scratch until the partials are written
    __syncthreads();
    if (!s_hdr[0]) {
        if (tid < D) A.out[head * D + tid] = 0.f;
        return;
    }
    float kq_all = 0.f;
#pragma unroll
    for (int w = 0; w < D / 32; ++w) kq_all += s_pk[w];
    if (!__syncthreads_and(mbar_wait_bounded(&bar[0], 0))) {
        if (tid < D) A.out[head * D + tid] = 0.f;
        if (tid == 0) {
            set_status(blob, LQ_DEV_TIMEOUT);
            mbar_wait_bounded(&bar[0], 0);
        }
        return;
    }

    float Sd[TI][4];
    float pk[4] = {0.f, 0.f, 0.f, 0.f}, pq[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int ii = 0; ii < TI; ++ii) {
        const int i = i0 + ii;
        const float4 r4 = *reinterpret_cast<const float4 *>(s_S + (size_t)i * D + j0);
        const float a = s_a[i], kk = s_k[i], qq = s_q[i];
        Sd[ii][0] = a * r4.x; Sd[ii][1] = a * r4.y; Sd[ii][2] = a * r4.z; Sd[ii][3] = a * r4.w;
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) {
            pk[jj] = fmaf(Sd[ii][jj], kk, pk[jj]);
            pq[jj] = fmaf(Sd[ii][jj], qq, pq[jj]);
        }
    }
    *reinterpret_cast<float4 *>(s_pk + ic * D + j0) = make_float4(pk[0], pk[1], pk[2], pk[3]);
    *reinterpret_cast<float4 *>(s_pq + ic * D + j0) = make_float4(pq[0], pq[1], pq[2], pq[3]);
    __syncthreads();
    if (tid < D) {
        float a = 0.f, b = 0.f;
#pragma unroll
        for (int r = 0; r < 16; ++r) {
            a += s_pk[r * D + tid];
            b += s_pq[r * D + tid];
        }
        const float u = bt * (vv - a);
        s_u[tid] = u;
        A.out[head * D + tid] = fmaf(kq_all, u, b);
    }
    __syncthreads();
    const float4 u4 = *reinterpret_cast<const float4 *>(s_u + j0);
    const float uu[4] = {u4.x, u4.y, u4.z, u4.w};
#pragma unroll
    for (int ii = 0; ii < TI; ++ii) {
        const float kk = s_k[i0 + ii];
        float4 o4;
        o4.x = fmaf(kk, uu[0], Sd[ii][0]);
        o4.y = fmaf(kk, uu[1], Sd[ii][1]);
        o4.z = fmaf(kk, uu[2], Sd[ii][2]);
        o4.w = fmaf(kk, uu[3], Sd[ii][3]);
        *reinterpret_cast<float4 *>(S + (size_t)(i0 + ii) * D + j0) = o4;
    }
}

// init (MODE 1): S0 -> blob with a fresh header; dequant (MODE 2): blob -> S_out
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
