// Lightning-attention prefill, beta = 128 and D = 128, bf16: one CTA pair per
// (sequence, head), paired tcgen05 MMAs (cta_group::2).
//
// Block algorithm (MiniMax-01, "Scaling Foundation Models with Lightning
// Attention"; CSDN digest section 2.1, mizuki blog appendix "key concepts"): per
// block b of 128 tokens of one sequence and head,
//     O_b = [(Q_b K_b^T) (.) M] V_b + Q_b KV,     KV += K_b^T V_b,
// with the causal 0/1 mask M (j <= i), KV reset at the sequence start (or set to
// an initial state), and an optional RMSNorm of each output row.
//
// Products per block (CTA rank c = 0 or 1).  Every MMA is paired: M = 128 with
// 64 rows per CTA; each CTA supplies half of the B rows from its own shared
// memory and receives its 64 D rows, for all N columns, in its own TMEM:
//   F1 = [S_b | O_b] = Q_b [K_b ; snap_b]^T   N = 256, K = dims
//          A: own 64 query rows     B: own 64 key rows, then own 64 rows of KV^T
//   O_b += P_b V_b                           N = 128, K = keys
//          A: own 64 rows of P      B: own 64 value columns
//   dKV_b^T = V_b^T K_b                      N = 128, K = tokens
//          A: own 64 value columns  B: own 64 key dims
// F1 gives the intra-block scores and the inter-block term Q_b KV_{<b} in one
// product: both have Q_b as their A operand, so K_b and the bf16 snapshot of the
// state stack into one 128-row B tile.  An N = 256 paired MMA keeps the tensor
// pipe busy for about as long as one thread takes to issue a tcgen05.mma.  The
// accumulators use the folded layout of an M = 64-per-CTA MMA: lanes 0..63 hold
// the CTA's 64 rows for the N columns the even CTA supplies, lanes 64..127 the
// same rows for the odd CTA's columns.  So F1 leaves S in the first 64 TMEM
// columns of its region and O in the next 64, exactly where the N = 128 product
// P V accumulates.
//
// Schedule.  Two issuing threads: one issues dKV_0, dKV_1, ... as soon as each
// block's key dims and values have landed (the state chain runs ahead of F1), the
// other issues F1_0, then per block b: F1_{b+1}, P_b V_b.  The snapshot F1_{b+1}
// needs (from dKV_b) and the P_b that P_b V_b needs (from F1_b) are produced by
// the epilogue while the other products run.
//
// Warps (480 threads per CTA):
//   warp 0       TMA producer (both CTAs)
//   warp 1       TMEM owner (both CTAs); CTA 0: issuer of F1 and P V
//   warps 2..5   group P (S -> causal mask -> bf16 P in shared memory)
//   warps 6..9   group KV (KV^T += dKV^T in registers, bf16 snapshot into the key-row
//                slot of the next block, final state)
//   warps 10..13 group O (O -> optional RMSNorm -> bf16, TMA store; frees the value
//                slot of each block once P V has completed)
//   warp 14      CTA 0: issuer of dKV
// Each epilogue group has one warp per TMEM sub-partition (warp w reads lanes
// 32 (w mod 4) .. + 31).  Every wait is bounded; on a timeout the CTA records
// DEV_TIMEOUT, drains its own copies and MMAs, frees TMEM and returns.
#pragma once

#include "prefill_tc.cuh"

namespace la {

struct PrefillPairParams {
    CUtensorMap tmap_q64;   // Q as [T][H*D], box 64 columns x 64 rows
    CUtensorMap tmap_k64;   // K, box 64 x 64
    CUtensorMap tmap_k128;  // K, box 64 x 128
    CUtensorMap tmap_v128;  // V, box 64 x 128
    CUtensorMap tmap_o32;   // O, box 64 x 32 (stores)
    __nv_bfloat16 *o;
    float *state;           // [S][H][D][D] or nullptr: final states
    const float *state_in;  // [S][H][D][D] or nullptr: initial states (may alias state)
    int H;
    int rmsnorm;
    unsigned long long timeout_ns;
    SeqTable seqs;
};

struct PairCfg {
    static constexpr int BETA = 128, D = 128;
    static constexpr int HBOX = 64 * 128;               // 64 rows x 128 B
    static constexpr int FBOX = 128 * 128;              // 128 rows x 128 B
    // Shared-memory rings (128-byte swizzled tiles; a "half" is dims or columns
    // [0,64) | [64,128)), each slot released by the product that reads it last:
    //   Q : own 64 query rows, both dim halves (A of F1)                     f1_done
    //   KS: per dim half 128 rows: own 64 key rows (TMA), then own 64 rows of
    //       the snapshot KV^T (group KV) (B of F1)                           f1_done
    //   KD: 128 key rows x own 64 dims (B of dKV^T)                          dkv_done
    //   V : 128 value rows x own 64 columns (A of dKV^T, B of P V)           v_free
    //   P : own 64 rows of P, both key halves (A of P V)                     o_done
    // (a value tile is released once group O has seen P V complete; P V follows its
    // dKV in every schedule.  Its own release ring lets the value ring run deeper than
    // the three F1 regions, so that dKV, which feeds the snapshot chain, rarely waits
    // for a value tile.  One P buffer: group P stores P_b while F1_{b+1} runs.)
    static constexpr int NQ = 2, NKS = 2, NKD = 2, NV = 4, NPB = 1;
    static constexpr int NF = 3;                        // F1 TMEM regions (S | O)
    static constexpr int NDK = 2;                       // dKV TMEM buffers
    // A ring's slot of block x is tested free on the done barrier of block x, which
    // must not have been lapped (by block x + ring size) when the producer tests it.
    static_assert(NQ <= NF && NKS <= NF && NKD <= NDK && NPB <= NF, "release rings");
    // Group KV waits for the value tile of a partial last block one block before its dKV:
    // the wait is exact only if the slot's previous load fed a dKV it has seen complete.
    static_assert(NV >= 2, "value ring: group KV's tail wait");
    static constexpr int Q_BYTES = 2 * HBOX, KS_BYTES = 2 * FBOX, T_BYTES = FBOX;
    static constexpr int P_BYTES = 2 * HBOX;
    static constexpr int OST_BYTES = 32 * 128;          // one 32-row x 64-column O box
    static constexpr int OFF_Q = 0;
    static constexpr int OFF_KS = OFF_Q + NQ * Q_BYTES;
    static constexpr int OFF_KD = OFF_KS + NKS * KS_BYTES;
    static constexpr int OFF_V = OFF_KD + NKD * T_BYTES;
    static constexpr int OFF_P = OFF_V + NV * T_BYTES;
    static constexpr int OFF_OST = OFF_P + NPB * P_BYTES;
    static constexpr int OFF_MISC = OFF_OST + 4 * OST_BYTES;
    static constexpr int MISC = 2048;
    static constexpr int SMEM_BYTES = 1024 + OFF_MISC + MISC;
    static_assert(SMEM_BYTES <= 227 * 1024, "shared memory budget");
    // TMEM columns: F1 region f = [S (64) | O (64)] at 128 f, then the dKV buffers
    static constexpr int TM_F1 = 0, TM_DKV = 128 * NF;
    static_assert(TM_DKV + 64 * NDK <= 512, "TMEM columns");
    static constexpr int TMEM_COLS = 512;
    static constexpr int GROUP = 128;
    static constexpr int WARP_D = 14;                   // issuer of dKV (CTA 0)
    static constexpr int THREADS = 64 + 3 * GROUP + 32;
    static constexpr uint32_t ID_F1 = idesc_bf16_f32(128, 256, 0, 0);
    static constexpr uint32_t ID_PV = idesc_bf16_f32(128, 128, 0, 1);
    static constexpr uint32_t ID_KV = idesc_bf16_f32(128, 128, 1, 1);
};

// Every wait below is a parity wait on one phase x of a barrier.  Two rules make it
// exact: phase x - 1 is known complete when the wait starts, and phase x + 1 cannot
// complete before the wait returns (argued for each barrier where it is waited on).
struct PairMisc {
    // used in CTA 0: TMA completion (CTA 1's loads complete them directly)
    uint64_t full_q[PairCfg::NQ];
    uint64_t full_ks[PairCfg::NKS];
    uint64_t full_kd[PairCfg::NKD];
    uint64_t full_v[PairCfg::NV];
    uint64_t tail_v;               // CTA 1: its own value tile of a partial last block landed
    uint64_t tail_zeroed;          // used in CTA 0: value rows past the sequence end zeroed
    // MMA completion (each commit arrives in both CTAs)
    uint64_t f1_done[PairCfg::NF];   // F1_j complete (region j % NF)
    uint64_t dkv_done[PairCfg::NDK]; // dKV_j complete (buffer j % NDK)
    uint64_t o_done[PairCfg::NF];    // P_j V_j complete (region j % NF)
    // each CTA's own: its group O has seen P_j V_j complete, value slot j % NV is free
    uint64_t v_free[PairCfg::NV];
    // used in CTA 0: epilogue -> issuers (arrivals from both CTAs)
    uint64_t f1_free[PairCfg::NF];   // groups P and O have loaded S_j and O_j
    uint64_t dkv_free[PairCfg::NDK]; // group KV has loaded dKV_j
    uint64_t p_ready[PairCfg::NPB];  // P_j stored in buffer j % NPB
    uint64_t snap_ready[PairCfg::NKS];  // snapshot u (the state before block u) in slot u % NKS
    uint64_t drain;
    uint64_t done0;                // phase 0 completed at the start: a wait that always passes
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
    // a partial last block: its value rows past the sequence end are zeroed by group KV
    const bool tail = nb > 0 && seq_len < nb * C::BETA;
    const uint64_t tlimit = p.timeout_ns;
    volatile int *abort_flag = &m->abort_flag;

    if (threadIdx.x == 0) {
        constexpr uint32_t BOTH = 2 * C::GROUP;         // one group of both CTAs
        for (int s = 0; s < C::NQ; ++s) mbar_init(&m->full_q[s], 1);
        for (int s = 0; s < C::NKS; ++s) {
            mbar_init(&m->full_ks[s], 1);
            mbar_init(&m->snap_ready[s], BOTH);
        }
        for (int s = 0; s < C::NKD; ++s) mbar_init(&m->full_kd[s], 1);
        for (int s = 0; s < C::NV; ++s) {
            mbar_init(&m->full_v[s], 1);
            mbar_init(&m->v_free[s], 1);
        }
        for (int s = 0; s < C::NF; ++s) {
            mbar_init(&m->f1_done[s], 1);
            mbar_init(&m->o_done[s], 1);
            mbar_init(&m->f1_free[s], 2 * BOTH);        // groups P and O
        }
        for (int s = 0; s < C::NDK; ++s) {
            mbar_init(&m->dkv_done[s], 1);
            mbar_init(&m->dkv_free[s], BOTH);
        }
        for (int s = 0; s < C::NPB; ++s) mbar_init(&m->p_ready[s], BOTH);
        mbar_init(&m->tail_v, 1);
        mbar_init(&m->tail_zeroed, BOTH);
        mbar_init(&m->drain, 2);
        mbar_init(&m->done0, 1);
        mbar_arrive(&m->done0);
        m->abort_flag = 0;
        fence_mbarrier_init_cluster();
        tma_prefetch_desc(&p.tmap_q64);
        tma_prefetch_desc(&p.tmap_k64);
        tma_prefetch_desc(&p.tmap_k128);
        tma_prefetch_desc(&p.tmap_v128);
        tma_prefetch_desc(&p.tmap_o32);
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
    auto q_addr = [&](int j) { return sbase + (uint32_t)(C::OFF_Q + (j % C::NQ) * C::Q_BYTES); };
    auto ks_addr = [&](int j) { return sbase + (uint32_t)(C::OFF_KS + (j % C::NKS) * C::KS_BYTES); };
    auto kd_addr = [&](int j) { return sbase + (uint32_t)(C::OFF_KD + (j % C::NKD) * C::T_BYTES); };
    auto v_addr = [&](int j) { return sbase + (uint32_t)(C::OFF_V + (j % C::NV) * C::T_BYTES); };
    auto p_addr = [&](int j) { return sbase + (uint32_t)(C::OFF_P + (j % C::NPB) * C::P_BYTES); };
    // Bounded warp-uniform wait.  A CTA-scope poll suffices: remote producers
    // order their shared-memory writes with a cluster-scope release fence before
    // arriving, and MMA commits and TMA loads complete the barriers directly.
    auto wwait = [&](uint64_t *bar, uint32_t parity) -> bool {
        return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort_flag, tlimit)) != 0;
    };
    // Signals to CTA 0.  CTA 1's threads publish their shared-memory writes (P, the
    // snapshot, zeroed value rows) with a release fence restricted to shared memory
    // and a relaxed remote arrival; signals that only free a TMEM buffer publish
    // nothing and use a plain relaxed arrival.
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
    // Rows [nv, 128) of a 128-row value tile set to zero by one epilogue group (128 threads).
    auto zero_rows = [&](uint32_t tile, int nv, int gtid) {
        for (uint32_t a = tile + (uint32_t)nv * 128 + (uint32_t)gtid * 16; a < tile + C::FBOX;
             a += C::GROUP * 16)
            st_shared_v4(a, 0u, 0u, 0u, 0u);
    };

    if (warp == 0) {
        // ------------------------------------------------------------ producer (both CTAs)
        // One thread polls the four rings and refills whichever slot its reader has
        // released.  CTA 0 expects the bytes of both CTAs on its full barrier; CTA 1's
        // loads complete CTA 0's barrier directly.  The value tile of a partial last
        // block is the exception: CTA 1 loads it against its own tail barrier, so that
        // its group KV can zero the rows past the sequence end once they have landed.
        if (lane == 0) {
            const int col = h * C::D;
            const int own_rows = 64 * (int)cta, own_cols = col + 64 * (int)cta;
            int jq = 0, js = 0, jd = 0, jv = 0;
            // slot of block j free: block j - depth has released it
            auto freed = [&](uint64_t *ring, int nring, int j, int depth) {
                const int x = j - depth;
                return x < 0 || mbar_test(&ring[x % nring], (uint32_t)((x / nring) & 1));
            };
            uint64_t t0 = globaltimer_ns();
            uint32_t polls = 0;
            while (jq < nb || js < nb || jd < nb || jv < nb) {
                bool progressed = false;
                if (jd < nb && freed(m->dkv_done, C::NDK, jd, C::NKD)) {
                    uint64_t *fb = &m->full_kd[jd % C::NKD];
                    const uint32_t dst = kd_addr(jd);
                    const int row = seq_start + jd * C::BETA;
                    if (cta == 0) {
                        mbar_arrive_expect_tx(fb, (uint32_t)(2 * C::T_BYTES));
                        tma_load_2d(dst, &p.tmap_k128, own_cols, row, fb);
                    } else {
                        tma_load_2d_pairbar(dst, &p.tmap_k128, own_cols, row, cluster_addr(fb, 0));
                    }
                    ++jd;
                    progressed = true;
                }
                if (jv < nb && freed(m->v_free, C::NV, jv, C::NV)) {
                    uint64_t *fb = &m->full_v[jv % C::NV];
                    const uint32_t dst = v_addr(jv);
                    const int row = seq_start + jv * C::BETA;
                    const bool last_partial = tail && jv == nb - 1;
                    if (cta == 0) {
                        mbar_arrive_expect_tx(fb, (uint32_t)((last_partial ? 1 : 2) * C::T_BYTES));
                        tma_load_2d(dst, &p.tmap_v128, own_cols, row, fb);
                    } else if (last_partial) {
                        mbar_arrive_expect_tx(&m->tail_v, (uint32_t)C::T_BYTES);
                        tma_load_2d(dst, &p.tmap_v128, own_cols, row, &m->tail_v);
                    } else {
                        tma_load_2d_pairbar(dst, &p.tmap_v128, own_cols, row, cluster_addr(fb, 0));
                    }
                    ++jv;
                    progressed = true;
                }
                if (js < nb && freed(m->f1_done, C::NF, js, C::NKS)) {
                    uint64_t *fb = &m->full_ks[js % C::NKS];
                    const uint32_t dst = ks_addr(js);
                    const int row = seq_start + js * C::BETA + own_rows;
                    if (cta == 0) {
                        mbar_arrive_expect_tx(fb, (uint32_t)(4 * C::HBOX));
                        tma_load_2d(dst, &p.tmap_k64, col, row, fb);
                        tma_load_2d(dst + C::FBOX, &p.tmap_k64, col + 64, row, fb);
                    } else {
                        const uint32_t fr = cluster_addr(fb, 0);
                        tma_load_2d_pairbar(dst, &p.tmap_k64, col, row, fr);
                        tma_load_2d_pairbar(dst + C::FBOX, &p.tmap_k64, col + 64, row, fr);
                    }
                    ++js;
                    progressed = true;
                }
                if (jq < nb && freed(m->f1_done, C::NF, jq, C::NQ)) {
                    uint64_t *fb = &m->full_q[jq % C::NQ];
                    const uint32_t dst = q_addr(jq);
                    const int row = seq_start + jq * C::BETA + own_rows;
                    if (cta == 0) {
                        mbar_arrive_expect_tx(fb, (uint32_t)(2 * C::Q_BYTES));
                        tma_load_2d(dst, &p.tmap_q64, col, row, fb);
                        tma_load_2d(dst + C::HBOX, &p.tmap_q64, col + 64, row, fb);
                    } else {
                        const uint32_t fr = cluster_addr(fb, 0);
                        tma_load_2d_pairbar(dst, &p.tmap_q64, col, row, fr);
                        tma_load_2d_pairbar(dst + C::HBOX, &p.tmap_q64, col + 64, row, fr);
                    }
                    ++jq;
                    progressed = true;
                }
                if (progressed) {
                    t0 = globaltimer_ns();
                    polls = 0;
                } else if ((++polls & 31) == 0) {
                    if (*abort_flag) break;
                    if (globaltimer_ns() - t0 > tlimit) {
                        fail();
                        break;
                    }
                }
            }
            // Drain (CTA 0): the last loads of each ring have landed before the CTA
            // exits.  CTA 1's loads are tracked by CTA 0's barriers; on the normal path
            // every one of them was consumed by an MMA, and after an abort the CTAs
            // wait out any load still in flight before they exit.
            const uint64_t lim = tlimit < 10000000ull ? tlimit : 10000000ull;
            if (cta == 0) {
                for (int j = (jq > C::NQ ? jq - C::NQ : 0); j < jq; ++j)
                    mbar_wait(&m->full_q[j % C::NQ], (uint32_t)((j / C::NQ) & 1), nullptr, lim);
                for (int j = (js > C::NKS ? js - C::NKS : 0); j < js; ++j)
                    mbar_wait(&m->full_ks[j % C::NKS], (uint32_t)((j / C::NKS) & 1), nullptr, lim);
                for (int j = (jd > C::NKD ? jd - C::NKD : 0); j < jd; ++j)
                    mbar_wait(&m->full_kd[j % C::NKD], (uint32_t)((j / C::NKD) & 1), nullptr, lim);
                for (int j = (jv > C::NV ? jv - C::NV : 0); j < jv; ++j)
                    mbar_wait(&m->full_v[j % C::NV], (uint32_t)((j / C::NV) & 1), nullptr, lim);
            } else if (tail && jv == nb) {
                mbar_wait(&m->tail_v, 0u, nullptr, lim);
            }
        }
        __syncwarp();
    } else if (warp == 1 || warp == C::WARP_D) {
        if (cta == 0) {
            // -------------------------------------------------------- issuers (CTA 0)
            // Lane 0 alone waits and issues.  Before each product it probes every barrier
            // the product needs at once (one round trip to the barriers for all of them)
            // and falls back to a bounded wait on each only when one is not complete yet.
            // Unused slots name done0, whose phase 0 is always complete.
            auto ready = [&](uint64_t *b0, uint32_t p0, uint64_t *b1, uint32_t p1, uint64_t *b2,
                             uint32_t p2, uint64_t *b3, uint32_t p3) -> bool {
                if (mbar_test4(b0, p0, b1, p1, b2, p2, b3, p3)) return true;
                return mbar_wait(b0, p0, abort_flag, tlimit) && mbar_wait(b1, p1, abort_flag, tlimit) &&
                       mbar_wait(b2, p2, abort_flag, tlimit) && mbar_wait(b3, p3, abort_flag, tlimit);
            };
            uint64_t *const any = &m->done0;
            // dKV_j^T = V_j^T K_j into dKV buffer j % NDK.  Waits: key dims and values of
            // block j landed (their next phases need dKV_j itself); dKV_{j-NDK} loaded by
            // group KV (the next phase needs dKV_j); for a partial last block, the value
            // rows past the sequence end zeroed.
            auto dkv = [&](int j) -> bool {
                const bool last_tail = tail && j == nb - 1;
                if (!ready(&m->full_kd[j % C::NKD], (uint32_t)((j / C::NKD) & 1),
                           &m->full_v[j % C::NV], (uint32_t)((j / C::NV) & 1),
                           j >= C::NDK ? &m->dkv_free[j % C::NDK] : any,
                           j >= C::NDK ? (uint32_t)(((j - C::NDK) / C::NDK) & 1) : 0u,
                           last_tail ? &m->tail_zeroed : any, 0u))
                    return false;
                tc_fence_after();
                const uint64_t vd = desc_mnmajor_sw128(v_addr(j), C::FBOX);
                const uint64_t kd = desc_mnmajor_sw128(kd_addr(j), C::FBOX);
#pragma unroll
                for (int ks = 0; ks < C::BETA / 16; ++ks)
                    mma_bf16_ss_pair(tmem + C::TM_DKV + 64 * (j % C::NDK), desc_add(vd, ks * 2048),
                                     desc_add(kd, ks * 2048), C::ID_KV, ks > 0 ? 1u : 0u);
                mma_commit_pair_both(&m->dkv_done[j % C::NDK]);
                return true;
            };
            // F1_j = [S_j | O_j] = Q_j [K_j ; snap_j]^T into region j % NF.  Waits: query
            // and key rows landed and snapshot j written (their next phases need F1_j);
            // region j % NF loaded by groups P and O for block j - NF (the next phase needs
            // F1_j).
            auto f1 = [&](int j) -> bool {
                if (!ready(&m->full_q[j % C::NQ], (uint32_t)((j / C::NQ) & 1),
                           &m->full_ks[j % C::NKS], (uint32_t)((j / C::NKS) & 1),
                           &m->snap_ready[j % C::NKS], (uint32_t)((j / C::NKS) & 1),
                           j >= C::NF ? &m->f1_free[j % C::NF] : any,
                           j >= C::NF ? (uint32_t)(((j - C::NF) / C::NF) & 1) : 0u))
                    return false;
                tc_fence_after();
                const uint64_t qd = desc_kmajor_sw128(q_addr(j));
                const uint64_t bd = desc_kmajor_sw128(ks_addr(j));
#pragma unroll
                for (int ks = 0; ks < C::D / 16; ++ks)
                    mma_bf16_ss_pair(tmem + C::TM_F1 + 128 * (j % C::NF),
                                     desc_add(qd, (uint32_t)((ks >> 2) * C::HBOX + (ks & 3) * 32)),
                                     desc_add(bd, (uint32_t)((ks >> 2) * C::FBOX + (ks & 3) * 32)),
                                     C::ID_F1, ks > 0 ? 1u : 0u);
                mma_commit_pair_both(&m->f1_done[j % C::NF]);
                return true;
            };
            // O_j += P_j V_j onto the O half of region j % NF, issued after F1_j by this
            // thread.  Waits: P_j stored (the next phase needs o_done(j)).  The value tile
            // landed: the dKV issuer waited for it before dKV_j, whose completion group KV
            // saw before the snapshot F1_{j+1} waited for; and the next load into its slot
            // needs o_done(j).  It is waited for here all the same (one probe).
            auto pv = [&](int j) -> bool {
                if (!ready(&m->p_ready[j % C::NPB], (uint32_t)((j / C::NPB) & 1),
                           &m->full_v[j % C::NV], (uint32_t)((j / C::NV) & 1), any, 0u, any, 0u))
                    return false;
                tc_fence_after();
                const uint64_t pd = desc_kmajor_sw128(p_addr(j));
                const uint64_t vd = desc_mnmajor_sw128(v_addr(j), C::FBOX);
#pragma unroll
                for (int ks = 0; ks < C::BETA / 16; ++ks)
                    mma_bf16_ss_pair(tmem + C::TM_F1 + 128 * (j % C::NF) + 64,
                                     desc_add(pd, (uint32_t)((ks >> 2) * C::HBOX + (ks & 3) * 32)),
                                     desc_add(vd, ks * 2048), C::ID_PV, 1u);
                mma_commit_pair_both(&m->o_done[j % C::NF]);
                return true;
            };
            bool ok = true;
            if (lane == 0) {
                if (warp == C::WARP_D) {
                    for (int j = 0; ok && j < nb; ++j) ok = dkv(j);
                } else {
                    if (nb > 0) ok = f1(0);
                    for (int b = 0; ok && b < nb; ++b) {
                        if (b + 1 < nb && !f1(b + 1)) {
                            ok = false;
                            break;
                        }
                        if (!pv(b)) {
                            ok = false;
                            break;
                        }
                    }
                }
                if (!ok) fail();
                // every MMA of both issuers has finished before TMEM is freed
                mma_commit_pair(smem_u32(&m->drain));
                mbar_wait(&m->drain, 0u, nullptr, tlimit);
            }
            __syncwarp();
        }
    } else if (warp < 6) {
        // ------------------------------------------------------------ group P (both CTAs)
        const int q = warp & 3;
        const uint32_t lane_base = (uint32_t)(32 * q) << 16;
        const int r = 32 * (q & 1) + lane;     // own query row (0..63)
        const int kh = q >> 1;                 // key half held by this lane
        const int R = 64 * (int)cta + r;       // row within the block
        bool ok = true;
        for (int j = 0; j < nb; ++j) {
            // f1_done[j % NF] phase j / NF; the next phase (F1_{j+NF}) needs f1_free,
            // which needs this group's load below
            if (!wwait(&m->f1_done[j % C::NF], (uint32_t)((j / C::NF) & 1))) {
                ok = false;
                break;
            }
            tc_fence_after();
            uint32_t s0[32], s1[32];
            const uint32_t tS = tmem + C::TM_F1 + 128 * (j % C::NF) + lane_base;
            tmem_ld32(tS, s0);
            tmem_ld32(tS + 32, s1);
            tmem_ld_wait();
            tc_fence_before();
            arrive_leader_free(&m->f1_free[j % C::NF]);
            uint32_t w[32];
#pragma unroll
            for (int u = 0; u < 32; ++u) {
                const uint32_t *s = u < 16 ? &s0[2 * u] : &s1[2 * (u - 16)];
                const int c0 = 64 * kh + 2 * u;
                const float x0 = c0 <= R ? __uint_as_float(s[0]) : 0.f;
                const float x1 = c0 + 1 <= R ? __uint_as_float(s[1]) : 0.f;
                w[u] = pack_bf16x2(x0, x1);
            }
            // The P buffer was last read by P_{j-NPB} V: o_done phase (j - NPB) / NF.  Its
            // next phase (P V of block j - NPB + NF) needs P of a later block.
            const int pb = j - C::NPB;
            if (pb >= 0 && !wwait(&m->o_done[pb % C::NF], (uint32_t)((pb / C::NF) & 1))) {
                ok = false;
                break;
            }
            const uint32_t sP = p_addr(j);
#pragma unroll
            for (int t = 0; t < 8; ++t)
                st_shared_v4(sP + kh * C::HBOX + r * 128 + ((uint32_t)(t ^ (r & 7)) << 4), w[4 * t],
                             w[4 * t + 1], w[4 * t + 2], w[4 * t + 3]);
            fence_proxy_async_smem();
            arrive_leader(&m->p_ready[j % C::NPB]);
        }
        if (!ok) fail();
    } else if (warp < 10) {
        // ------------------------------------------------------------ group KV (both CTAs)
        const int q = warp & 3;
        const uint32_t lane_base = (uint32_t)(32 * q) << 16;
        const int r = 32 * (q & 1) + lane;     // own value column j (0..63)
        const int half = q >> 1;               // dim half of the state
        float kv[64];                          // KV^T[64 c + r][64 half .. 64 half + 63]
#pragma unroll
        for (int t = 0; t < 64; ++t) kv[t] = 0.f;
        bool ok = true;
        // snapshot u (the state before block u) into the snapshot rows of key-row slot u % NKS
        auto write_snap = [&](int u) {
            const uint32_t dst = ks_addr(u) + half * C::FBOX + C::HBOX;
#pragma unroll
            for (int t = 0; t < 8; ++t)
                st_shared_v4(dst + r * 128 + ((uint32_t)(t ^ (r & 7)) << 4),
                             pack_bf16x2(kv[8 * t + 0], kv[8 * t + 1]),
                             pack_bf16x2(kv[8 * t + 2], kv[8 * t + 3]),
                             pack_bf16x2(kv[8 * t + 4], kv[8 * t + 5]),
                             pack_bf16x2(kv[8 * t + 6], kv[8 * t + 7]));
            fence_proxy_async_smem();
            arrive_leader(&m->snap_ready[u % C::NKS]);
        };
        // The value rows past the end of a partial last block must not enter dKV^T (nor
        // P V): zero them in this CTA's value tile once it has landed.  Done one block
        // before that block's dKV (or first, for a one-block sequence), so that the dKV
        // issuer never waits for work that depends on products it has not issued.  CTA
        // 0's wait is exact: the slot's previous load (block nb - 1 - NV) fed
        // dKV_{nb-1-NV}, which this group has already seen complete.
        auto zero_tail = [&]() -> bool {
            const int b = nb - 1;
            const bool landed = cta == 0 ? wwait(&m->full_v[b % C::NV], (uint32_t)((b / C::NV) & 1))
                                         : wwait(&m->tail_v, 0u);
            if (!landed) return false;
            zero_rows(v_addr(b), seq_len - b * C::BETA, (int)threadIdx.x - 64 - C::GROUP);
            fence_proxy_async_smem();
            arrive_leader(&m->tail_zeroed);
            return true;
        };
        if (p.state_in != nullptr && (nb > 0 || p.state != nullptr)) {
            // KV^T[j][i] starts at the initial state X[i][j]
            const float *src = p.state_in + ((size_t)sid * p.H + h) * C::D * C::D + 64 * (int)cta + r;
#pragma unroll
            for (int t = 0; t < 64; ++t) kv[t] = src[(size_t)(64 * half + t) * C::D];
        }
        if (nb > 0) {
            write_snap(0);
            if (tail && nb == 1) ok = zero_tail();
        }
        for (int b = 0; ok && b < nb; ++b) {
            if (tail && nb >= 2 && b == nb - 2 && !zero_tail()) {
                ok = false;
                break;
            }
            // dkv_done[b % NDK] phase b / NDK; the next phase needs dkv_free from below
            if (!wwait(&m->dkv_done[b % C::NDK], (uint32_t)((b / C::NDK) & 1))) {
                ok = false;
                break;
            }
            tc_fence_after();
            const uint32_t tK = tmem + C::TM_DKV + 64 * (b % C::NDK) + lane_base;
            {
                uint32_t a[32];
                tmem_ld32(tK, a);
                tmem_ld_wait();
#pragma unroll
                for (int t = 0; t < 32; ++t) kv[t] += __uint_as_float(a[t]);
                tmem_ld32(tK + 32, a);
                tmem_ld_wait();
#pragma unroll
                for (int t = 0; t < 32; ++t) kv[32 + t] += __uint_as_float(a[t]);
            }
            tc_fence_before();
            arrive_leader_free(&m->dkv_free[b % C::NDK]);
            if (b + 1 < nb) {
                // slot (b+1) % NKS was last read by F1_{b+1-NKS}: f1_done phase
                // (b+1-NKS) / NF; its next phase needs snapshot b+1-NKS+NF, written later
                const int x = b + 1 - C::NKS;
                if (x >= 0 && !wwait(&m->f1_done[x % C::NF], (uint32_t)((x / C::NF) & 1))) {
                    ok = false;
                    break;
                }
                write_snap(b + 1);
            }
        }
        if (ok && p.state != nullptr) {  // final state (fp32), state[i][j] = KV^T[j][i]
            float *dst = p.state + ((size_t)sid * p.H + h) * C::D * C::D + 64 * (int)cta + r;
#pragma unroll
            for (int t = 0; t < 64; ++t) dst[(size_t)(64 * half + t) * C::D] = kv[t];
        }
        if (!ok) fail();
    } else if (warp < C::WARP_D) {
        // ------------------------------------------------------------ group O (both CTAs)
        const int q = warp & 3;
        const uint32_t lane_base = (uint32_t)(32 * q) << 16;
        const int r = 32 * (q & 1) + lane;     // own output row
        const int half = q >> 1;               // column half
        bool ok = true;
        for (int b = 0; b < nb; ++b) {
            // o_done[b % NF] phase b / NF; the next phase (P V of block b + NF) needs
            // F1_{b+NF}, which needs f1_free from the load below.  After a failed wait
            // the warp still meets the group's named barrier in every block (so no warp
            // of the group waits there for ever) but skips every other step.
            if (ok && !wwait(&m->o_done[b % C::NF], (uint32_t)((b / C::NF) & 1))) {
                ok = false;
                fail();
            }
            uint32_t a[32], c[32];
            if (ok) {
                // v_free[b % NV] phase b / NV; its next phase needs P V of block b + NV,
                // which reads the value tile the producer loads after this arrival
                if (q == 0 && lane == 0) mbar_arrive(&m->v_free[b % C::NV]);
                tc_fence_after();
                const uint32_t tO = tmem + C::TM_F1 + 128 * (b % C::NF) + 64 + lane_base;
                tmem_ld32(tO, a);
                tmem_ld32(tO + 32, c);
                tmem_ld_wait();
                tc_fence_before();
                arrive_leader_free(&m->f1_free[b % C::NF]);
            }
            float scale = 1.0f;
            if (p.rmsnorm) {
                float ss = 0.f;
                if (ok) {
                    float s4[4] = {0.f, 0.f, 0.f, 0.f};   // four chains: 16 dependent FMAs each
#pragma unroll
                    for (int t = 0; t < 32; t += 2) {
                        const float x0 = __uint_as_float(a[t]), x1 = __uint_as_float(a[t + 1]);
                        const float y0 = __uint_as_float(c[t]), y1 = __uint_as_float(c[t + 1]);
                        s4[0] = fmaf(x0, x0, s4[0]);
                        s4[1] = fmaf(x1, x1, s4[1]);
                        s4[2] = fmaf(y0, y0, s4[2]);
                        s4[3] = fmaf(y1, y1, s4[3]);
                    }
                    ss = (s4[0] + s4[1]) + (s4[2] + s4[3]);
                    // exchange with warp q ^ 2, which holds the other column half of the row
                    m->ss_x[b & 1][half][r] = ss;
                }
                // all four warps of the group, once per block.  Block b's buffer is next
                // written in block b + 2, after every warp has passed block b + 1's
                // barrier and so has read block b's partial sums: two buffers suffice.
                named_barrier(1, C::GROUP);
                if (ok) {
                    const float other = m->ss_x[b & 1][half ^ 1][r];
                    const float tot = half == 0 ? ss + other : other + ss;
                    scale = rsqrtf(tot * (1.0f / C::D) + 1e-6f);
                }
            }
            if (!ok) continue;
            const int nv = min(C::BETA, seq_len - b * C::BETA);
            const int R = 64 * (int)cta + r;
            const int R0 = 64 * (int)cta + 32 * (q & 1);     // first row of this warp's box
            if (R0 + 32 <= nv) {
                // the whole box lies inside the sequence: stage it (128-byte swizzle) and let
                // one lane issue a TMA store.  Register-to-global stores would wait in this
                // SM's memory pipe while HBM is saturated and hold up the MMA issue behind them.
                const uint32_t stage = sbase + C::OFF_OST + q * C::OST_BYTES;
                if (lane == 0) bulk_wait_read_all();   // the previous box has been read
                __syncwarp();
#pragma unroll
                for (int t = 0; t < 8; ++t) {
                    const uint32_t *src = t < 4 ? &a[8 * t] : &c[8 * (t - 4)];
                    st_shared_v4(stage + lane * 128 + ((uint32_t)(t ^ (lane & 7)) << 4),
                                 pack_bf16x2(__uint_as_float(src[0]) * scale, __uint_as_float(src[1]) * scale),
                                 pack_bf16x2(__uint_as_float(src[2]) * scale, __uint_as_float(src[3]) * scale),
                                 pack_bf16x2(__uint_as_float(src[4]) * scale, __uint_as_float(src[5]) * scale),
                                 pack_bf16x2(__uint_as_float(src[6]) * scale, __uint_as_float(src[7]) * scale));
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) {
                    tma_store_2d(&p.tmap_o32, stage, h * C::D + 64 * half, seq_start + b * C::BETA + R0);
                    bulk_commit_group();
                }
                __syncwarp();
            } else if (R < nv) {
                // the partial last block: plain stores of the rows inside the sequence
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
        if (lane == 0) bulk_wait_all();   // every O box stored before the CTA leaves
        __syncwarp();
        if (!ok) fail();
    }

    // After an abort, loads issued by CTA 1 against CTA 0's barriers may still be in
    // flight: wait 1 ms (bounded) before the CTAs leave, far beyond any TMA latency.
    __syncthreads();
    if (threadIdx.x == 0 && *abort_flag) {
        const uint64_t t1 = globaltimer_ns();
        while (globaltimer_ns() - t1 < 1000000ull) {
        }
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
