// Lightning-attention prefill, beta = 128 and D = 128, bf16: one CTA pair per
// (sequence, head), paired tcgen05 MMAs (cta_group::2).
//
// Same block algorithm as prefill_tc.cuh (MiniMax-01, "Scaling Foundation
// Models with Lightning Attention"; CSDN digest section 2.1, mizuki blog
// appendix "key concepts"): per block b of 128 tokens,
//     O_b = [(Q_b K_b^T) (.) M] V_b + Q_b KV,     KV += K_b^T V_b.
//
// Work split inside the pair (CTA rank c = 0 or 1): every MMA is an M = 128,
// N = 128 paired MMA issued by one thread of CTA 0.  Each CTA supplies half of
// the A rows and half of the B rows from its own shared memory and receives
// its half of the D rows, for all N columns, in its own TMEM:
//   S   = Q K^T      A: own 64 query rows    B: own 64 key rows      D: own rows x 128 keys
//   O   = P V        A: own 64 rows of P     B: own 64 value columns D: own rows x 128 columns
//   O  += Q snap     A: own 64 query rows    B: own 64 rows of KV^T  D: (the same O)
//   dKV^T = V^T K    A: own 64 value columns B: own 64 key dims      D: own 64 value cols x 128 dims
// so a CTA stages only its halves (64 KB per block instead of 80 KB for the
// unpaired kernel), three stages fit in shared memory, and each tensor-core
// operand byte is read once per pair instead of once per CTA.  Each CTA keeps
// its 64 columns of the fp32 state, transposed (KV^T[j][i]), in epilogue
// registers, and its output rows are complete (all 128 columns) inside the
// CTA, so the RMSNorm needs no exchange between the CTAs.
//
// The paired accumulators use the folded TMEM layout of an M = 64-per-CTA
// MMA: lanes 0..63 hold the 64 rows for columns [0, N/2), lanes 64..127 the
// same rows for columns [N/2, N), both in TMEM columns [0, N/2).
//
// Warps (320 threads per CTA):
//   warp 0      TMA producer (each CTA loads its own halves, completes its own barriers)
//   warp 1      CTA 0: TMEM owner and MMA issuer.  CTA 1: forwards each completed
//               stage of its own to CTA 0's stage barrier.
//   warps 2..5  group P: S -> causal mask -> bf16 P (shared memory, A operand of P V)
//   warps 6..9  group O: KV^T += dKV^T, bf16 snapshot, O -> (RMSNorm) -> bf16 store,
//               final fp32 state -> global store
// MMA issue order per block b: S_{b+1} (look-ahead), O_b = P_b V_b,
// O_b += Q_b snap(KV_{<b}), dKV_b^T = V_b^T K_b.  Signals to CTA 0's MMA thread
// are mbarrier arrivals (remote ones from CTA 1); the MMA thread's commits
// arrive on the barriers of both CTAs.  Every wait is
// bounded; on a timeout the CTA records DEV_TIMEOUT, drains its own copies
// and MMAs, frees TMEM and returns.
#pragma once

#include "prefill_tc.cuh"

namespace la {

struct PrefillPairParams {
    CUtensorMap tmap_q64;   // Q as [T][H*D], box 64 columns x 64 rows
    CUtensorMap tmap_k64;   // K, box 64 x 64
    CUtensorMap tmap_k128;  // K, box 64 x 128
    CUtensorMap tmap_v128;  // V, box 64 x 128
    __nv_bfloat16 *o;
    float *state;           // [S][H][D][D] or nullptr
    int H;
    int rmsnorm;
    unsigned long long timeout_ns;
    SeqTable seqs;
};

#ifndef LA_PAIR_PREFETCH
#define LA_PAIR_PREFETCH 0
#endif

struct PairCfg {
    static constexpr int BETA = 128, D = 128;
    // blocks beyond the TMA ring whose tiles are prefetched into L2
    static constexpr int PF = LA_PAIR_PREFETCH;
    static constexpr int HBOX = 64 * 128;               // 64 rows x 128 B
    static constexpr int FBOX = 128 * 128;              // 128 rows x 128 B
    // one stage, all tiles 128-byte swizzled:
    static constexpr int OFF_QH = 0;                    // own 64 query rows, dims [0,64) | [64,128)
    static constexpr int OFF_KK = 2 * HBOX;             // own 64 key rows, dims [0,64) | [64,128)
    static constexpr int OFF_KD = 4 * HBOX;             // 128 key rows, own 64 dims
    static constexpr int OFF_VC = 4 * HBOX + FBOX;      // 128 key rows, own 64 value columns
    static constexpr int STAGE = 4 * HBOX + 2 * FBOX;   // 64 KB
    static constexpr int NST = 3;
    static constexpr int OFF_P = NST * STAGE;           // own 64 rows of P, keys [0,64) | [64,128)
    static constexpr int OFF_SNAP = OFF_P + 2 * HBOX;   // own 64 rows of KV^T, dims [0,64) | [64,128)
    static constexpr int OFF_MISC = OFF_SNAP + 2 * HBOX;
    static constexpr int MISC = 2048;
    static constexpr int SMEM_BYTES = 1024 + OFF_MISC + MISC;
    static_assert(SMEM_BYTES <= 227 * 1024, "shared memory budget");
    // TMEM columns: S[2], O[2], dKV[2], 64 columns each (folded layout)
    static constexpr int TM_S = 0, TM_O = 128, TM_DKV = 256;
    static constexpr int TMEM_COLS = 512;
    static constexpr int GROUP = 128;
    static constexpr int THREADS = 64 + 2 * GROUP;
    static constexpr uint32_t ID_S = idesc_bf16_f32(128, 128, 0, 0);
    static constexpr uint32_t ID_PV = idesc_bf16_f32(128, 128, 0, 1);
    static constexpr uint32_t ID_QKV = idesc_bf16_f32(128, 128, 0, 0);
    static constexpr uint32_t ID_KV = idesc_bf16_f32(128, 128, 1, 1);
};

struct PairMisc {
    uint64_t full[PairCfg::NST];   // CTA 0: own bytes + CTA 1's forwarded arrival; CTA 1: own bytes
    uint64_t empty[PairCfg::NST];
    uint64_t s_full[2];
    uint64_t blk_full[2];          // both CTAs: O_b and dKV_b complete
    uint64_t o_free[2];            // used in CTA 0: arrivals from both CTAs
    uint64_t dkv_free[2];
    uint64_t p_ready;
    uint64_t p_free;               // both CTAs: P consumed by O = P V (MMA commit)
    uint64_t snap_ready;
    uint64_t drain;
    uint64_t ss_bar[2];            // group O: RMSNorm partial sums written (per block parity)
    uint32_t tmem_base;
    int abort_flag;
    float ss_x[2][2][64];          // RMSNorm partial sums [block parity][column half][row]
};

__global__ void __launch_bounds__(PairCfg::THREADS, 1)
    prefill_pair_kernel(const __grid_constant__ PrefillPairParams p) {
    using C = PairCfg;
    static_assert(sizeof(PairMisc) <= C::MISC, "misc area");
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    PairMisc *m = reinterpret_cast<PairMisc *>(smem + C::OFF_MISC);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t cta = cluster_ctarank();
    const int pr = blockIdx.x >> 1;
    const int h = pr % p.H;
    const int rank = pr / p.H;
    int seq_start, seq_len, sid;
    p.seqs.get(rank, seq_start, seq_len, sid);
    const int nb = (seq_len + C::BETA - 1) / C::BETA;
    const uint64_t tlimit = p.timeout_ns;
    volatile int *abort_flag = &m->abort_flag;

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::NST; ++s) {
            mbar_init(&m->full[s], cta == 0 ? 2 : 1);
            mbar_init(&m->empty[s], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&m->s_full[i], 1);
            mbar_init(&m->blk_full[i], 1);
            mbar_init(&m->o_free[i], 2 * C::GROUP);
            mbar_init(&m->dkv_free[i], 2 * C::GROUP);
        }
        mbar_init(&m->p_ready, 2 * C::GROUP);
        mbar_init(&m->p_free, 1);
        mbar_init(&m->snap_ready, 2 * C::GROUP);
        mbar_init(&m->drain, 1);
        mbar_init(&m->ss_bar[0], C::GROUP);
        mbar_init(&m->ss_bar[1], C::GROUP);
        m->abort_flag = 0;
        fence_mbarrier_init_cluster();
        tma_prefetch_desc(&p.tmap_q64);
        tma_prefetch_desc(&p.tmap_k64);
        tma_prefetch_desc(&p.tmap_k128);
        tma_prefetch_desc(&p.tmap_v128);
    }
    if (warp == 1) {
        tmem_alloc_pair(&m->tmem_base, C::TMEM_COLS);
        tmem_relinquish_pair();
    }
    tc_fence_before();
    __syncthreads();
    cluster_sync_all();
    tc_fence_after();
    const uint32_t tmem = m->tmem_base;

    auto fail = [&]() {
        *abort_flag = 1;
        record_fault(DEV_TIMEOUT);
    };
    auto stage_addr = [&](int st) { return sbase + (uint32_t)(st * C::STAGE); };
    // Bounded warp-uniform wait.  A CTA-scope poll suffices: remote producers
    // order their shared-memory writes with a cluster-scope release fence before
    // arriving, and MMA commits complete the barriers of both CTAs directly.
    auto wwait = [&](uint64_t *bar, uint32_t parity) -> bool {
        return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort_flag, tlimit)) != 0;
    };
    // Signals to CTA 0.  CTA 0's own threads arrive locally.  CTA 1's threads
    // publish their shared-memory writes (P, the state snapshot, a landed stage)
    // with a release fence restricted to shared memory and a relaxed remote
    // arrival; a full cluster-scope release would also wait for the thread's
    // outstanding global stores.  Signals that only free a TMEM buffer (the
    // tcgen05.ld has completed) publish nothing and use a plain relaxed arrival.
    auto arrive_leader = [&](uint64_t *bar) {
        if (cta == 0) {
            mbar_arrive(bar);
        } else {
            fence_release_smem_cluster();
            mbar_arrive_cluster_relaxed(cluster_addr(bar, 0));
        }
    };
    auto arrive_leader_free = [&](uint64_t *bar) {
        if (cta == 0)
            mbar_arrive(bar);
        else
            mbar_arrive_cluster_relaxed(cluster_addr(bar, 0));
    };

    if (warp == 0) {
        // ------------------------------------------------------------ producer (both CTAs)
        int issued = 0;
        if (lane == 0) {
            auto prefetch = [&](int j) {  // this CTA's tiles of block j, into L2
                const int row = seq_start + j * C::BETA, col = h * C::D;
                tma_prefetch_l2_2d(&p.tmap_q64, col, row + 64 * (int)cta);
                tma_prefetch_l2_2d(&p.tmap_q64, col + 64, row + 64 * (int)cta);
                tma_prefetch_l2_2d(&p.tmap_k64, col, row + 64 * (int)cta);
                tma_prefetch_l2_2d(&p.tmap_k64, col + 64, row + 64 * (int)cta);
                tma_prefetch_l2_2d(&p.tmap_k128, col + 64 * (int)cta, row);
                tma_prefetch_l2_2d(&p.tmap_v128, col + 64 * (int)cta, row);
            };
            if constexpr (C::PF > 0)
                for (int j = C::NST; j < C::NST + C::PF && j < nb; ++j) prefetch(j);
            for (int b = 0; b < nb; ++b) {
                const int st = b % C::NST;
                if (C::PF > 0 && b + C::NST + C::PF < nb) prefetch(b + C::NST + C::PF);
                if (!mbar_wait(&m->empty[st], (uint32_t)(((b / C::NST) & 1) ^ 1), abort_flag, tlimit)) {
                    fail();
                    break;
                }
                mbar_arrive_expect_tx(&m->full[st], (uint32_t)C::STAGE);
                const int row = seq_start + b * C::BETA;
                const uint32_t sa = stage_addr(st);
                const int col = h * C::D;
                tma_load_2d(sa + C::OFF_QH, &p.tmap_q64, col, row + 64 * (int)cta, &m->full[st]);
                tma_load_2d(sa + C::OFF_QH + C::HBOX, &p.tmap_q64, col + 64, row + 64 * (int)cta,
                            &m->full[st]);
                tma_load_2d(sa + C::OFF_KK, &p.tmap_k64, col, row + 64 * (int)cta, &m->full[st]);
                tma_load_2d(sa + C::OFF_KK + C::HBOX, &p.tmap_k64, col + 64, row + 64 * (int)cta,
                            &m->full[st]);
                tma_load_2d(sa + C::OFF_KD, &p.tmap_k128, col + 64 * (int)cta, row, &m->full[st]);
                tma_load_2d(sa + C::OFF_VC, &p.tmap_v128, col + 64 * (int)cta, row, &m->full[st]);
                ++issued;
            }
            // Drain: this CTA's last issued loads have landed before it exits (in CTA 0 the
            // barrier also needs CTA 1's forward; the wait is bounded either way).
            for (int b = (issued > C::NST ? issued - C::NST : 0); b < issued; ++b)
                mbar_wait(&m->full[b % C::NST], (uint32_t)((b / C::NST) & 1), nullptr, tlimit);
        }
        __syncwarp();
    } else if (warp == 1 && cta == 1) {
        // ------------------------------------------------------------ forwarder (CTA 1)
        if (lane == 0) {
            for (int b = 0; b < nb; ++b) {
                const int st = b % C::NST;
                if (!mbar_wait(&m->full[st], (uint32_t)((b / C::NST) & 1), abort_flag, tlimit)) {
                    fail();
                    break;
                }
                arrive_leader(&m->full[st]);
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer (CTA 0)
        bool any_issued = false;
        auto commit_both = [&](uint64_t *bar) {
            mma_commit_pair(smem_u32(bar));
            mma_commit_pair(cluster_addr(bar, 1));
        };
        auto stage_in = [&](int j) -> bool {
            const int st = j % C::NST;
            if (!wwait(&m->full[st], (uint32_t)((j / C::NST) & 1))) return false;
            if (lane == 0) {
                const uint32_t sa = stage_addr(st);
                const uint64_t qd = desc_kmajor_sw128(sa + C::OFF_QH);
                const uint64_t kd = desc_kmajor_sw128(sa + C::OFF_KK);
#pragma unroll
                for (int ks = 0; ks < C::D / 16; ++ks) {
                    const uint32_t off = (uint32_t)((ks >> 2) * C::HBOX + (ks & 3) * 32);
                    mma_bf16_ss_pair(tmem + C::TM_S + 64 * (j & 1), desc_add(qd, off),
                                     desc_add(kd, off), C::ID_S, ks > 0 ? 1u : 0u);
                }
                commit_both(&m->s_full[j & 1]);
            }
            any_issued = true;
            __syncwarp();
            return true;
        };

        // Per block b: S_{b+1} (look-ahead: its stage was loaded two blocks ago), then
        // O_b = P_b V_b, O_b += Q_b snap(KV_{<b}), dKV_b^T = V_b^T K_b.  While group P turns
        // S_{b+1} into P_{b+1} and group O turns dKV_b into the next snapshot, the tensor
        // pipe still holds queued work.
        bool ok = nb == 0 || stage_in(0);
        for (int b = 0; ok && b < nb; ++b) {
            const int st = b % C::NST;
            const uint32_t sa = stage_addr(st);
            const uint32_t dO = tmem + C::TM_O + 64 * (b & 1);
            const uint32_t dKV = tmem + C::TM_DKV + 64 * (b & 1);
            if (b + 1 < nb && !stage_in(b + 1)) {
                ok = false;
                break;
            }
            if (!wwait(&m->p_ready, (uint32_t)(b & 1))) {
                ok = false;
                break;
            }
            if (b >= 2 && (!wwait(&m->o_free[b & 1], (uint32_t)(((b - 2) >> 1) & 1)) ||
                           !wwait(&m->dkv_free[b & 1], (uint32_t)(((b - 2) >> 1) & 1)))) {
                ok = false;
                break;
            }
            tc_fence_after();
            const uint64_t vd = desc_mnmajor_sw128(sa + C::OFF_VC, C::FBOX);
            if (lane == 0) {  // O_b = P_b V_b
                const uint64_t pd = desc_kmajor_sw128(sbase + C::OFF_P);
#pragma unroll
                for (int ks = 0; ks < C::BETA / 16; ++ks)
                    mma_bf16_ss_pair(dO, desc_add(pd, (uint32_t)((ks >> 2) * C::HBOX + (ks & 3) * 32)),
                                     desc_add(vd, ks * 2048), C::ID_PV, ks > 0 ? 1u : 0u);
                commit_both(&m->p_free);
            }
            __syncwarp();
            if (b >= 1) {  // O_b += Q_b snap(KV_{<b})
                if (!wwait(&m->snap_ready, (uint32_t)((b - 1) & 1))) {
                    ok = false;
                    break;
                }
                if (lane == 0) {
                    const uint64_t qd = desc_kmajor_sw128(sa + C::OFF_QH);
                    const uint64_t sd = desc_kmajor_sw128(sbase + C::OFF_SNAP);
#pragma unroll
                    for (int ks = 0; ks < C::D / 16; ++ks) {
                        const uint32_t off = (uint32_t)((ks >> 2) * C::HBOX + (ks & 3) * 32);
                        mma_bf16_ss_pair(dO, desc_add(qd, off), desc_add(sd, off), C::ID_QKV, 1u);
                    }
                }
                __syncwarp();
            }
            if (lane == 0) {  // dKV_b^T = V_b^T K_b, then release the block
                const uint64_t kd = desc_mnmajor_sw128(sa + C::OFF_KD, C::FBOX);
#pragma unroll
                for (int ks = 0; ks < C::BETA / 16; ++ks)
                    mma_bf16_ss_pair(dKV, desc_add(vd, ks * 2048), desc_add(kd, ks * 2048), C::ID_KV,
                                     ks > 0 ? 1u : 0u);
                commit_both(&m->blk_full[b & 1]);
                commit_both(&m->empty[st]);
            }
            __syncwarp();
        }
        if (!ok) fail();
        if (any_issued && lane == 0) {  // every issued MMA has finished before TMEM is freed
            mma_commit_pair(smem_u32(&m->drain));
            mbar_wait(&m->drain, 0u, nullptr, tlimit);
        }
        __syncwarp();
    } else if (warp < 6) {
        // ------------------------------------------------------------ group P (both CTAs)
        const int q = warp & 3;
        const uint32_t lane_base = (uint32_t)(32 * q) << 16;
        const int r = 32 * (q & 1) + lane;     // own query row (0..63)
        const int kh = q >> 1;                 // key half held by this lane
        const int R = 64 * (int)cta + r;       // row within the block
        const uint32_t sP = sbase + C::OFF_P;
        bool ok = true;
        for (int b = 0; b < nb; ++b) {
            if (!wwait(&m->s_full[b & 1], (uint32_t)((b >> 1) & 1))) {
                ok = false;
                break;
            }
            tc_fence_after();
            uint32_t s0[32], s1[32];
            const uint32_t tS = tmem + C::TM_S + 64 * (b & 1) + lane_base;
            tmem_ld32(tS, s0);
            tmem_ld32(tS + 32, s1);
            tmem_ld_wait();
            uint32_t w[32];
#pragma unroll
            for (int u = 0; u < 32; ++u) {
                const uint32_t *s = u < 16 ? &s0[2 * u] : &s1[2 * (u - 16)];
                const int c0 = 64 * kh + 2 * u;
                const float x0 = c0 <= R ? __uint_as_float(s[0]) : 0.f;
                const float x1 = c0 + 1 <= R ? __uint_as_float(s[1]) : 0.f;
                w[u] = pack_bf16x2(x0, x1);
            }
            // the previous block's O = P V must have read P before it is overwritten
            if (b >= 1 && !wwait(&m->p_free, (uint32_t)((b - 1) & 1))) {
                ok = false;
                break;
            }
#pragma unroll
            for (int t = 0; t < 8; ++t)
                st_shared_v4(sP + kh * C::HBOX + r * 128 + ((uint32_t)(t ^ (r & 7)) << 4), w[4 * t],
                             w[4 * t + 1], w[4 * t + 2], w[4 * t + 3]);
            // V rows past the sequence end must not enter dKV^T: zero them in this CTA's slice.
            const int nv = min(C::BETA, seq_len - b * C::BETA);
            if (nv < C::BETA) {
                const uint32_t v0 = stage_addr(b % C::NST) + C::OFF_VC;
                for (uint32_t a = v0 + nv * 128 + (threadIdx.x - 64) * 16; a < v0 + C::FBOX;
                     a += C::GROUP * 16)
                    st_shared_v4(a, 0u, 0u, 0u, 0u);
            }
            fence_proxy_async_smem();
            tc_fence_before();
            arrive_leader(&m->p_ready);
        }
        if (!ok) fail();
    } else {
        // ------------------------------------------------------------ group O (both CTAs)
        const int q = warp & 3;
        const uint32_t lane_base = (uint32_t)(32 * q) << 16;
        const int r = 32 * (q & 1) + lane;     // own output row / own value column j
        const int half = q >> 1;               // column half (O) / dim half (state)
        const uint32_t sSnap = sbase + C::OFF_SNAP;
        float kv[64];                          // KV^T[64 c + r][64 half .. 64 half + 63]
#pragma unroll
        for (int t = 0; t < 64; ++t) kv[t] = 0.f;
        bool ok = true;
        for (int b = 0; b < nb; ++b) {
            // (1) state: KV^T += dKV_b^T, then the bf16 snapshot for O_{b+1} += Q_{b+1} KV
            if (!wwait(&m->blk_full[b & 1], (uint32_t)((b >> 1) & 1))) {
                ok = false;
                break;
            }
            tc_fence_after();
            {
                uint32_t a[32], c[32];
                const uint32_t tK = tmem + C::TM_DKV + 64 * (b & 1) + lane_base;
                tmem_ld32(tK, a);
                tmem_ld32(tK + 32, c);
                tmem_ld_wait();
                tc_fence_before();
                arrive_leader_free(&m->dkv_free[b & 1]);
#pragma unroll
                for (int t = 0; t < 32; ++t) {
                    kv[t] += __uint_as_float(a[t]);
                    kv[32 + t] += __uint_as_float(c[t]);
                }
            }
            if (b + 1 < nb) {
                // The snapshot buffer was last read by O_b += Q_b KV, issued before dKV_b and
                // so finished once blk_full(b) completed.
#pragma unroll
                for (int t = 0; t < 8; ++t)
                    st_shared_v4(sSnap + half * C::HBOX + r * 128 + ((uint32_t)(t ^ (r & 7)) << 4),
                                 pack_bf16x2(kv[8 * t + 0], kv[8 * t + 1]),
                                 pack_bf16x2(kv[8 * t + 2], kv[8 * t + 3]),
                                 pack_bf16x2(kv[8 * t + 4], kv[8 * t + 5]),
                                 pack_bf16x2(kv[8 * t + 6], kv[8 * t + 7]));
                fence_proxy_async_smem();
                arrive_leader(&m->snap_ready);
            }
            // (2) output block b (O_b completed with dKV_b)
            uint32_t a[32], c[32];
            const uint32_t tO = tmem + C::TM_O + 64 * (b & 1) + lane_base;
            tmem_ld32(tO, a);
            tmem_ld32(tO + 32, c);
            tmem_ld_wait();
            tc_fence_before();
            arrive_leader_free(&m->o_free[b & 1]);
            float scale = 1.0f;
            if (p.rmsnorm) {
                float ss = 0.f;
#pragma unroll
                for (int t = 0; t < 32; ++t) {
                    const float x = __uint_as_float(a[t]), y = __uint_as_float(c[t]);
                    ss = fmaf(x, x, ss);
                    ss = fmaf(y, y, ss);
                }
                // exchange with the lane holding the other column half (bounded wait)
                m->ss_x[b & 1][half][r] = ss;
                mbar_arrive(&m->ss_bar[b & 1]);
                if (!__all_sync(0xffffffffu, mbar_wait(&m->ss_bar[b & 1], (uint32_t)((b >> 1) & 1),
                                                       abort_flag, tlimit))) {
                    ok = false;
                    break;
                }
                const float other = m->ss_x[b & 1][half ^ 1][r];
                const float tot = half == 0 ? ss + other : other + ss;
                scale = rsqrtf(tot * (1.0f / C::D) + 1e-6f);
            }
            const int nv = min(C::BETA, seq_len - b * C::BETA);
            const int R = 64 * (int)cta + r;
            if (R < nv) {
                uint4 *dst = reinterpret_cast<uint4 *>(
                    p.o + ((size_t)(seq_start + b * C::BETA + R) * p.H + h) * C::D + 64 * half);
#pragma unroll
                for (int t = 0; t < 8; ++t) {
                    const uint32_t *src = t < 4 ? &a[8 * t] : &c[8 * (t - 4)];
                    dst[t] = make_uint4(
                        pack_bf16x2(__uint_as_float(src[0]) * scale, __uint_as_float(src[1]) * scale),
                        pack_bf16x2(__uint_as_float(src[2]) * scale, __uint_as_float(src[3]) * scale),
                        pack_bf16x2(__uint_as_float(src[4]) * scale, __uint_as_float(src[5]) * scale),
                        pack_bf16x2(__uint_as_float(src[6]) * scale, __uint_as_float(src[7]) * scale));
                }
            }
        }
        if (ok && p.state != nullptr) {  // final state K^T V (fp32), state[i][j] = KV^T[j][i]
            float *dst = p.state + ((size_t)sid * p.H + h) * C::D * C::D + 64 * (int)cta + r;
#pragma unroll
            for (int t = 0; t < 64; ++t) dst[(size_t)(64 * half + t) * C::D] = kv[t];
        }
        if (!ok) fail();
    }

    tc_fence_before();
    __syncthreads();
    cluster_sync_all();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc_pair(tmem, C::TMEM_COLS);
    }
}

}  // namespace la
