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
#include "../../include/lightning_attention.h"

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

// One (sequence, head) of one token.  S is that pair's D x D state: read when
// `read` (else the step starts from zero), written back when `write`.
template <int D, typename T>
__device__ __forceinline__ void decode_one(const T *__restrict__ q, const T *__restrict__ k,
                                           const T *__restrict__ v, T *__restrict__ o,
                                           float4 *__restrict__ S, bool read, bool write,
                                           int rmsnorm) {
    constexpr int C4 = D / 4;            // float4 per state row
    constexpr int RG = 256 / C4;         // row groups
    constexpr int RPT = D / RG;          // rows per thread
    __shared__ float sq[D], sk[D];
    __shared__ float red[RG][D];
    __shared__ float ssum[8];

    const int tid = threadIdx.x;
    const int c4 = tid % C4, rg = tid / C4;

    float4 x[RPT];
#pragma unroll
    for (int t = 0; t < RPT; ++t)
        x[t] = read ? __ldcs(&S[(size_t)(rg + RG * t) * C4 + c4]) : make_float4(0.f, 0.f, 0.f, 0.f);

    if (tid < D) {
        sq[tid] = to_f32(q[tid]);
        sk[tid] = to_f32(k[tid]);
    }
    const float v0 = to_f32(v[4 * c4 + 0]), v1 = to_f32(v[4 * c4 + 1]),
                v2 = to_f32(v[4 * c4 + 2]), v3 = to_f32(v[4 * c4 + 3]);
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
        if (write) __stcs(&S[(size_t)r * C4 + c4], x[t]);
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
    if (tid < D) o[tid] = from_f32<T>(out * scale);
}

template <int D, typename T>
__global__ void __launch_bounds__(256)
    decode_step_kernel(const T *__restrict__ q, const T *__restrict__ k, const T *__restrict__ v,
                       float *__restrict__ state, T *__restrict__ o, int rmsnorm) {
    const size_t bh = blockIdx.x;
    decode_one<D, T>(q + bh * D, k + bh * D, v + bh * D, o + bh * D,
                     reinterpret_cast<float4 *>(state + bh * D * D), true, true, rmsnorm);
}

// The one-token sequences of a prefill call: entry i is the token row and the
// state index of one of them; with `identity` set, entry i is row i, state i.
struct OneTokenTable {
    int identity;
    int row[LA_MAX_VARLEN_SEQS];
    int sid[LA_MAX_VARLEN_SEQS];
};

// A prefill's one-token sequences as decode steps: one CTA per (sequence, head),
// reading q, k, v and writing o at the sequence's row of the packed [T, H, D]
// arrays.  The state of sequence s (state_ws[s], when given) is read with
// `read` and written back with `write`; a one-token prefill is exactly one
// decode step from its initial state (or from zero).
template <int D, typename T>
__global__ void __launch_bounds__(256)
    decode_rows_kernel(const T *__restrict__ q, const T *__restrict__ k, const T *__restrict__ v,
                       T *__restrict__ o, float *__restrict__ state_ws, int H, int read, int write,
                       int rmsnorm, const __grid_constant__ OneTokenTable tab) {
    const int i = blockIdx.x / H, h = blockIdx.x % H;
    const int row = tab.identity ? i : tab.row[i];
    const int sid = tab.identity ? i : tab.sid[i];
    const size_t vec = ((size_t)row * H + h) * D;
    float4 *S = state_ws != nullptr
                    ? reinterpret_cast<float4 *>(state_ws + ((size_t)sid * H + h) * D * D)
                    : nullptr;
    decode_one<D, T>(q + vec, k + vec, v + vec, o + vec, S, read != 0 && S != nullptr,
                     write != 0 && S != nullptr, rmsnorm);
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
