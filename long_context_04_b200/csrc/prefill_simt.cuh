// Lightning-attention prefill for fp32 inputs: CUDA-core FFMA, no tensor cores.
//
// Same block algorithm as the bf16 path (MiniMax-01, CSDN digest section 2.1;
// mizuki blog appendix "key concepts"): per block b of BETA tokens,
//     O_b = [(Q_b K_b^T) (.) M] V_b + Q_b KV,     KV += K_b^T V_b,
// on the CUDA cores (TF32 tensor cores would not meet a 1e-5 relative error).
// Inputs, outputs, scores and the state are stored in fp32; every dot product
// is accumulated in fp64 registers (an fp32 x fp32 product is exact in fp64),
// so a row whose sum cancels -- a one-token sequence with q.k near zero, say --
// still comes out within a few fp32 roundings.
// One CTA (256 threads) owns one (sequence, head); K_b, V_b and the D x D
// state stay in shared memory, query rows are processed 16 at a time.
#pragma once

#include "prefill_tc.cuh"  // SeqTable

namespace la {

template <int BETA, int D>
struct SimtCfg {
    static constexpr int THREADS = 256;
    static constexpr int RT = 16;  // query rows per tile
    static constexpr int SMEM_FLOATS = 2 * BETA * D + D * D + RT * D + RT * BETA + RT * D;
    static constexpr int SMEM_BYTES = SMEM_FLOATS * 4;
};

template <int BETA, int D>
__global__ void __launch_bounds__(256)
    prefill_simt_kernel(const float *__restrict__ q, const float *__restrict__ k,
                        const float *__restrict__ v, float *__restrict__ o,
                        float *state, const float *state_in, int H, int rmsnorm,
                        const __grid_constant__ SeqTable seqs) {
    using C = SimtCfg<BETA, D>;
    extern __shared__ float sm[];
    float *sK = sm;                       // [BETA][D]
    float *sV = sK + BETA * D;            // [BETA][D]
    float *sKV = sV + BETA * D;           // [D][D]
    float *sQ = sKV + D * D;              // [RT][D]
    float *sS = sQ + C::RT * D;           // [RT][BETA]
    float *sO = sS + C::RT * BETA;        // [RT][D]

    const int tid = threadIdx.x;
    const int h = blockIdx.x % H;
    const int rank = blockIdx.x / H;
    int start, len, sid;
    seqs.get(rank, start, len, sid);

    // KV starts at the sequence's initial state (state_in may alias state: this CTA
    // reads its slice here and writes it back only at the end)
    const float *x0 = state_in != nullptr ? state_in + ((size_t)sid * H + h) * D * D : nullptr;
    for (int x = tid; x < D * D; x += C::THREADS) sKV[x] = x0 != nullptr ? x0[x] : 0.f;

    for (int p0 = 0; p0 < len; p0 += BETA) {
        const int nv = min(BETA, len - p0);
        __syncthreads();
        for (int x = tid; x < BETA * D; x += C::THREADS) {
            const int rr = x / D, d = x % D;
            const size_t g = ((size_t)(start + p0 + rr) * H + h) * D + d;
            sK[x] = rr < nv ? k[g] : 0.f;
            sV[x] = rr < nv ? v[g] : 0.f;
        }
        __syncthreads();
        for (int r0 = 0; r0 < nv; r0 += C::RT) {
            for (int x = tid; x < C::RT * D; x += C::THREADS) {
                const int rr = x / D, d = x % D;
                sQ[x] = r0 + rr < nv ? q[((size_t)(start + p0 + r0 + rr) * H + h) * D + d] : 0.f;
            }
            __syncthreads();
            // S = Q_tile K_b^T with the causal mask (key c <= query row)
            for (int x = tid; x < C::RT * BETA; x += C::THREADS) {
                const int rr = x / BETA, c = x % BETA;
                double acc = 0.0;
                if (c <= r0 + rr) {
#pragma unroll 8
                    for (int d = 0; d < D; ++d)
                        acc = fma((double)sQ[rr * D + d], (double)sK[c * D + d], acc);
                }
                sS[x] = (float)acc;
            }
            __syncthreads();
            // O = S V_b + Q_tile KV
            for (int x = tid; x < C::RT * D; x += C::THREADS) {
                const int rr = x / D, j = x % D;
                double intra = 0.0, inter = 0.0;
                const int cmax = min(r0 + rr, BETA - 1);
                for (int c = 0; c <= cmax; ++c)
                    intra = fma((double)sS[rr * BETA + c], (double)sV[c * D + j], intra);
#pragma unroll 8
                for (int i = 0; i < D; ++i)
                    inter = fma((double)sQ[rr * D + i], (double)sKV[i * D + j], inter);
                sO[x] = (float)(intra + inter);
            }
            __syncthreads();
            // optional RMSNorm per row, then store: one warp per row
            const int warp = tid >> 5, lane = tid & 31;
            for (int rr = warp; rr < C::RT; rr += C::THREADS / 32) {
                if (r0 + rr >= nv) continue;
                float scale = 1.f;
                if (rmsnorm) {
                    double ss = 0.0;
                    for (int j = lane; j < D; j += 32)
                        ss = fma((double)sO[rr * D + j], (double)sO[rr * D + j], ss);
#pragma unroll
                    for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
                    scale = (float)(1.0 / sqrt(ss / (double)D + 1e-6));
                }
                float *dst = o + ((size_t)(start + p0 + r0 + rr) * H + h) * D;
                for (int j = lane; j < D; j += 32) dst[j] = sO[rr * D + j] * scale;
            }
            __syncthreads();
        }
        // KV += K_b^T V_b
        for (int x = tid; x < D * D; x += C::THREADS) {
            const int i = x / D, j = x % D;
            double acc = (double)sKV[x];
            for (int c = 0; c < nv; ++c) acc = fma((double)sK[c * D + i], (double)sV[c * D + j], acc);
            sKV[x] = (float)acc;
        }
    }
    __syncthreads();
    if (state != nullptr) {
        float *dst = state + ((size_t)sid * H + h) * D * D;
        for (int x = tid; x < D * D; x += C::THREADS) dst[x] = sKV[x];
    }
}

}  // namespace la
