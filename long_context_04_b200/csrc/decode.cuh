// One-token decode step (jvyan.cn article, section 2 "compute optimisation":
// length-1 requests run as their own kernel on their own CUDA stream):
//     KV <- KV + k v^T,   o = q^T KV,   optional RMSNorm of o over D.
//
// HBM-bound: per (sequence, head) the fp32 D x D state is read and written
// once (8 D^2 bytes) against 4 D^2 flops.  One CTA of 256 threads owns one
// (sequence, head); thread t owns 4 consecutive columns (one float4) of
// D / (256 / (D/4)) rows, so each warp instruction moves whole 512-byte (D=128)
// rows.  All of a thread's float4 loads are issued before any use (D^2/1024
// loads in flight per thread), with streaming cache hints since the state is
// touched once per step.  Column partial sums of q^T KV are reduced across the
// row groups in shared memory; the RMSNorm sum uses warp shuffles.
#pragma once

#include "la_device.cuh"

namespace la {

template <typename T>
__device__ __forceinline__ float to_f32(T x);
template <>
__device__ __forceinline__ float to_f32<float>(float x) { return x; }
template <>
__device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 x) { return __bfloat162float(x); }
template <typename T>
__device__ __forceinline__ T from_f32(float x);
template <>
__device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <>
__device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) { return __float2bfloat16_rn(x); }

template <int D, typename T>
__global__ void __launch_bounds__(256)
    decode_step_kernel(const T *__restrict__ q, const T *__restrict__ k, const T *__restrict__ v,
                       float *__restrict__ state, T *__restrict__ o, int rmsnorm) {
    constexpr int C4 = D / 4;            // float4 per state row
    constexpr int RG = 256 / C4;         // row groups
    constexpr int RPT = D / RG;          // rows per thread
    __shared__ float sq[D], sk[D];
    __shared__ float red[RG][D];
    __shared__ float ssum[8];

    const int bh = blockIdx.x;
    const int tid = threadIdx.x;
    const int c4 = tid % C4, rg = tid / C4;
    const size_t vec = (size_t)bh * D;
    float4 *S = reinterpret_cast<float4 *>(state + (size_t)bh * D * D);

    float4 x[RPT];
#pragma unroll
    for (int t = 0; t < RPT; ++t) x[t] = __ldcs(&S[(size_t)(rg + RG * t) * C4 + c4]);

    if (tid < D) {
        sq[tid] = to_f32(q[vec + tid]);
        sk[tid] = to_f32(k[vec + tid]);
    }
    const float v0 = to_f32(v[vec + 4 * c4 + 0]), v1 = to_f32(v[vec + 4 * c4 + 1]),
                v2 = to_f32(v[vec + 4 * c4 + 2]), v3 = to_f32(v[vec + 4 * c4 + 3]);
    __syncthreads();

    float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
#pragma unroll
    for (int t = 0; t < RPT; ++t) {
        const int r = rg + RG * t;
        const float kr = sk[r], qr = sq[r];
        x[t].x = fmaf(kr, v0, x[t].x);
        x[t].y = fmaf(kr, v1, x[t].y);
        x[t].z = fmaf(kr, v2, x[t].z);
        x[t].w = fmaf(kr, v3, x[t].w);
        __stcs(&S[(size_t)r * C4 + c4], x[t]);
        a0 = fmaf(qr, x[t].x, a0);
        a1 = fmaf(qr, x[t].y, a1);
        a2 = fmaf(qr, x[t].z, a2);
        a3 = fmaf(qr, x[t].w, a3);
    }
    red[rg][4 * c4 + 0] = a0;
    red[rg][4 * c4 + 1] = a1;
    red[rg][4 * c4 + 2] = a2;
    red[rg][4 * c4 + 3] = a3;
    __syncthreads();

    float out = 0.f;
    if (tid < D) {
#pragma unroll
        for (int g = 0; g < RG; ++g) out += red[g][tid];
    }
    float scale = 1.f;
    if (rmsnorm) {
        float ss = tid < D ? out * out : 0.f;
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
        if ((tid & 31) == 0) ssum[tid >> 5] = ss;
        __syncthreads();
        float tot = 0.f;
#pragma unroll
        for (int w = 0; w < D / 32; ++w) tot += ssum[w];
        scale = rsqrtf(tot * (1.0f / D) + 1e-6f);
    }
    if (tid < D) o[vec + tid] = from_f32<T>(out * scale);
}

// state_dst[slot(s)][h] = state_ws[s][h]; one CTA per (s, h).
__global__ void __launch_bounds__(256)
    state_copy_kernel(const float4 *__restrict__ src, float4 *__restrict__ dst,
                      const int *__restrict__ seq_to_slot, int H, int n4, int num_slots) {
    const int s = blockIdx.x / H, h = blockIdx.x % H;
    const int slot = seq_to_slot != nullptr ? seq_to_slot[s] : s;
    if (slot < 0 || slot >= num_slots) {
        if (threadIdx.x == 0) record_fault(DEV_RANGE);
        return;
    }
    const float4 *a = src + (size_t)blockIdx.x * n4;
    float4 *b = dst + ((size_t)slot * H + h) * n4;
    for (int i = threadIdx.x; i < n4; i += blockDim.x) b[i] = __ldcs(&a[i]);
}

// dst[s][h] = 0 (the final state of sequences with no tokens); one CTA per (s, h).
__global__ void __launch_bounds__(256) state_zero_kernel(float4 *__restrict__ dst, int n4) {
    float4 *b = dst + (size_t)blockIdx.x * n4;
    for (int i = threadIdx.x; i < n4; i += blockDim.x) b[i] = make_float4(0.f, 0.f, 0.f, 0.f);
}

}  // namespace la
