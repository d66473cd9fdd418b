// The local state of a chunk, state = K^T V, without the attention output; and the
// exclusive prefix of chunk states over ranks.
//
// These are steps 1 and 3 of LASP+, the sequence-parallel scheme the pages name for
// lightning attention (mizuki blog, section 5 "pretraining" and appendix "key
// concepts": local prefix sums of the chunk states, an all-gather, after which each
// chunk runs from the sum of the states before it; jvyan.cn article, section 3).
// Step 2 is the all-gather; step 4 is the ordinary prefill started from that sum.
//
// chunk_state_tc_kernel<D> (bf16): one CTA per (sequence, head, 64-column value
// slice).  Per block of 128 tokens the K tile (128 x D) and the value slice (128 x 64)
// arrive by TMA in a ring; one thread issues dKV_b = K_b^T V_b as tcgen05 MMAs with
// M = D (key dims), N = 64, K = 128 tokens into one of two TMEM accumulators, and the
// epilogue adds each block's accumulator into an fp32 state held in registers, as the
// prefill kernels do: one long fp32 accumulation chain inside the tensor core drifts
// measurably over tens of thousands of tokens.  Value rows past the sequence end are
// zeroed in shared memory before their block's MMAs.  HBM traffic: 4 D bytes per
// token-head (K, V).
//
// chunk_state_simt_kernel<D> (fp32): one CTA per (sequence, head), K_b and V_b staged
// in shared memory, fp64 accumulation of every dot product, fp32 state.
//
// state_prefix_kernel: out[s][h] = sum_{r < rank} gathered[r][s][h], r ascending.
#pragma once

#include "prefill_tc.cuh"

namespace la {

struct ChunkStateParams {
    CUtensorMap tmap_k;    // K as [T][H*D], box 64 columns x 128 rows
    CUtensorMap tmap_v;    // V, the same
    float *state;          // [S][H][D][D]
    int H;
    unsigned long long timeout_ns;
    SeqTable seqs;
};

template <int D>
struct ChunkCfg {
    static constexpr int BETA = 128;
    static constexpr int NVS = D / 64;              // value slices (CTAs) per (sequence, head)
    static constexpr int DB = D / 64;               // 64-column boxes of K
    static constexpr int BOX = BETA * 128;          // 128 rows x 128 B
    static constexpr int STAGE = (DB + 1) * BOX;    // K boxes, then the value slice
    static constexpr int NST = 4;
    static constexpr int OFF_MISC = NST * STAGE;
    static constexpr int MISC = 1024;
    static constexpr int SMEM_BYTES = 1024 + OFF_MISC + MISC;
    static_assert(SMEM_BYTES <= 227 * 1024, "shared memory budget");
    static constexpr int TMEM_COLS = 128;          // two accumulators of 64 columns
    static constexpr int GROUP = 128;               // epilogue threads
    static constexpr int THREADS = 64 + GROUP;
    static constexpr uint32_t ID_KV = idesc_bf16_f32(D, 64, 1, 1);
};

struct ChunkMisc {
    uint64_t full[4];
    uint64_t empty[4];
    uint64_t tail_landed; // the partial last block's tiles have landed (single phase)
    uint64_t zeroed;      // value rows past the sequence end zeroed (single phase)
    uint64_t acc_full[2]; // block j's accumulator (buffer j % 2) complete
    uint64_t acc_free[2]; // the epilogue has read buffer j % 2
    uint64_t done;        // every MMA complete (single phase)
    uint32_t tmem_base;
    int abort_flag;
};

template <int D>
__global__ void __launch_bounds__(ChunkCfg<D>::THREADS, 1)
    chunk_state_tc_kernel(const __grid_constant__ ChunkStateParams p) {
    using C = ChunkCfg<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    ChunkMisc *m = reinterpret_cast<ChunkMisc *>(smem + C::OFF_MISC);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int vs = blockIdx.x % C::NVS;
    const int unit = blockIdx.x / C::NVS;
    const int h = unit % p.H, rank = unit / p.H;
    int seq_start, seq_len, sid;
    p.seqs.get(rank, seq_start, seq_len, sid);
    const int nb = (seq_len + C::BETA - 1) / C::BETA;
    const int tail_rows = nb > 0 ? seq_len - (nb - 1) * C::BETA : C::BETA;  // rows of the last block
    const uint64_t tlimit = p.timeout_ns;
    volatile int *abort_flag = &m->abort_flag;

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::NST; ++s) {
            mbar_init(&m->full[s], 1);
            mbar_init(&m->empty[s], 1);
        }
        mbar_init(&m->tail_landed, 1);
        mbar_init(&m->zeroed, C::GROUP);
        mbar_init(&m->done, 1);
        for (int i = 0; i < 2; ++i) {
            mbar_init(&m->acc_full[i], 1);
            mbar_init(&m->acc_free[i], C::GROUP);
        }
        m->abort_flag = 0;
        fence_mbarrier_init_cluster();
        tma_prefetch_desc(&p.tmap_k);
        tma_prefetch_desc(&p.tmap_v);
    }
    if (warp == 1) {
        tmem_alloc(&m->tmem_base, C::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = m->tmem_base;
    auto fail = [&]() {
        *abort_flag = 1;
        record_fault(DEV_TIMEOUT);
    };
    auto wwait = [&](uint64_t *bar, uint32_t parity) -> bool {
        return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort_flag, tlimit)) != 0;
    };
    auto stage = [&](int j) { return sbase + (uint32_t)((j % C::NST) * C::STAGE); };

    if (warp == 0) {
        // ---------------------------------------------------------------- TMA producer
        if (lane == 0) {
            int issued = 0;
            for (int j = 0; j < nb; ++j) {
                const int st = j % C::NST;
                if (!mbar_wait(&m->empty[st], (uint32_t)(((j / C::NST) & 1) ^ 1), abort_flag, tlimit)) {
                    fail();
                    break;
                }
                mbar_arrive_expect_tx(&m->full[st], (uint32_t)C::STAGE);
                const int row = seq_start + j * C::BETA, col = h * D;
#pragma unroll
                for (int d = 0; d < C::DB; ++d)
                    tma_load_2d(stage(j) + d * C::BOX, &p.tmap_k, col + 64 * d, row, &m->full[st]);
                tma_load_2d(stage(j) + C::DB * C::BOX, &p.tmap_v, col + 64 * vs, row, &m->full[st]);
                ++issued;
            }
            for (int j = (issued > C::NST ? issued - C::NST : 0); j < issued; ++j)
                mbar_wait(&m->full[j % C::NST], (uint32_t)((j / C::NST) & 1), nullptr, tlimit);
        }
        __syncwarp();
    } else if (warp == 1) {
        // ---------------------------------------------------------------- MMA issuer
        bool ok = true;
        for (int j = 0; ok && j < nb; ++j) {
            const int st = j % C::NST;
            if (!wwait(&m->full[st], (uint32_t)((j / C::NST) & 1))) {
                ok = false;
                break;
            }
            if (j == nb - 1 && tail_rows < C::BETA) {
                // This thread sees every block's barrier in order; it tells the epilogue
                // that the last block has landed and waits for its value rows past the
                // sequence end to be zeroed.
                if (lane == 0) mbar_arrive(&m->tail_landed);
                if (!wwait(&m->zeroed, 0u)) {
                    ok = false;
                    break;
                }
            }
            // accumulator j % 2 was last read by the epilogue for block j - 2
            if (j >= 2 && !wwait(&m->acc_free[j & 1], (uint32_t)(((j - 2) >> 1) & 1))) {
                ok = false;
                break;
            }
            tc_fence_after();
            if (lane == 0) {  // dKV_b^T[dims][own 64 value columns] = K_b^T V_b
                const uint64_t kd = desc_mnmajor_sw128(stage(j), C::BOX);
                const uint64_t vd = desc_mnmajor_sw128(stage(j) + C::DB * C::BOX, C::BOX);
#pragma unroll
                for (int ks = 0; ks < C::BETA / 16; ++ks)
                    mma_bf16_ss(tmem + 64 * (j & 1), desc_add(kd, ks * 2048), desc_add(vd, ks * 2048),
                                C::ID_KV, ks > 0 ? 1u : 0u);
                mma_commit(&m->empty[st]);
                mma_commit(&m->acc_full[j & 1]);
            }
            __syncwarp();
        }
        if (!ok) fail();
        if (lane == 0) {  // every issued MMA has finished before TMEM is freed
            mma_commit(&m->done);
            mbar_wait(&m->done, 0u, nullptr, tlimit);
        }
        __syncwarp();
    } else {
        // ---------------------------------------------------------------- epilogue
        const int t = threadIdx.x - 64;
        const int q = warp & 3;
        // row i of the accumulators: lane i for M = 128; lanes 0..15 of each 32-lane
        // quadrant for M = 64
        const int i = D == 128 ? 32 * q + lane : 16 * q + lane;
        const bool i_ok = D == 128 || lane < 16;
        float acc[64];  // state[i][64 vs .. 64 vs + 63]
#pragma unroll
        for (int x = 0; x < 64; ++x) acc[x] = 0.f;
        bool ok = true;
        for (int j = 0; j < nb; ++j) {
            if (j == nb - 1 && tail_rows < C::BETA) {
                // value rows past the sequence end must not enter K^T V
                if (!wwait(&m->tail_landed, 0u)) {
                    ok = false;
                    break;
                }
                const uint32_t v0 = stage(j) + C::DB * C::BOX;
                for (uint32_t a = v0 + tail_rows * 128 + t * 16; a < v0 + C::BOX; a += C::GROUP * 16)
                    st_shared_v4(a, 0u, 0u, 0u, 0u);
                fence_proxy_async_smem();
                mbar_arrive(&m->zeroed);
            }
            if (!wwait(&m->acc_full[j & 1], (uint32_t)((j >> 1) & 1))) {
                ok = false;
                break;
            }
            tc_fence_after();
            uint32_t a[32], c[32];
            const uint32_t tA = tmem + 64 * (j & 1) + ((uint32_t)(32 * q) << 16);
            tmem_ld32(tA, a);
            tmem_ld32(tA + 32, c);
            tmem_ld_wait();
            tc_fence_before();
            mbar_arrive(&m->acc_free[j & 1]);
#pragma unroll
            for (int x = 0; x < 32; ++x) {
                acc[x] += __uint_as_float(a[x]);
                acc[32 + x] += __uint_as_float(c[x]);
            }
        }
        if (ok && i_ok) {
            float4 *d4 = reinterpret_cast<float4 *>(p.state + (((size_t)sid * p.H + h) * D + i) * D + 64 * vs);
#pragma unroll
            for (int x = 0; x < 16; ++x)
                d4[x] = make_float4(acc[4 * x], acc[4 * x + 1], acc[4 * x + 2], acc[4 * x + 3]);
        }
        if (!ok) fail();
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, C::TMEM_COLS);
    }
}

// fp32 path: one CTA per (sequence, head); fp64 accumulation of every dot product.
template <int D>
__global__ void __launch_bounds__(256)
    chunk_state_simt_kernel(const float *__restrict__ k, const float *__restrict__ v,
                            float *__restrict__ state, int H, const __grid_constant__ SeqTable seqs) {
    constexpr int BETA = 64;
    extern __shared__ float sm[];
    float *sK = sm;                // [BETA][D]
    float *sV = sK + BETA * D;     // [BETA][D]
    float *sKV = sV + BETA * D;    // [D][D]
    const int tid = threadIdx.x;
    const int h = blockIdx.x % H, rank = blockIdx.x / H;
    int start, len, sid;
    seqs.get(rank, start, len, sid);
    for (int x = tid; x < D * D; x += 256) sKV[x] = 0.f;
    for (int p0 = 0; p0 < len; p0 += BETA) {
        const int nv = min(BETA, len - p0);
        __syncthreads();
        for (int x = tid; x < BETA * D; x += 256) {
            const int rr = x / D, d = x % D;
            const size_t g = ((size_t)(start + p0 + rr) * H + h) * D + d;
            sK[x] = rr < nv ? k[g] : 0.f;
            sV[x] = rr < nv ? v[g] : 0.f;
        }
        __syncthreads();
        for (int x = tid; x < D * D; x += 256) {
            const int i = x / D, j = x % D;
            double acc = (double)sKV[x];
            for (int c = 0; c < nv; ++c) acc = fma((double)sK[c * D + i], (double)sV[c * D + j], acc);
            sKV[x] = (float)acc;
        }
    }
    __syncthreads();
    float *dst = state + ((size_t)sid * H + h) * D * D;
    for (int x = tid; x < D * D; x += 256) dst[x] = sKV[x];
}

// out[s][h] = sum_{r < rank} gathered[r][s][h], summed in rank order; one CTA per (s, h).
__global__ void __launch_bounds__(256)
    state_prefix_kernel(const float4 *__restrict__ gathered, float4 *__restrict__ out, int rank,
                        size_t rank_stride4, int n4) {
    const float4 *src = gathered + (size_t)blockIdx.x * n4;
    float4 *dst = out + (size_t)blockIdx.x * n4;
    for (int i = threadIdx.x; i < n4; i += blockDim.x) {
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int r = 0; r < rank; ++r) {
            const float4 x = src[(size_t)r * rank_stride4 + i];
            acc.x += x.x;
            acc.y += x.y;
            acc.z += x.z;
            acc.w += x.w;
        }
        dst[i] = acc;
    }
}

}  // namespace la
