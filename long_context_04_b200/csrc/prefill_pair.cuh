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
// unpaired kernel) and each tensor-core operand byte is read once per pair
// instead of once per CTA.  The halves arrive through three TMA rings (key
// rows 2 deep, query rows 4 deep, key dims + value columns 2 deep), each slot
// released by the last MMA that reads it.  Each CTA keeps
// its 64 columns of the fp32 state, transposed (KV^T[j][i]), in epilogue
// registers, and its output rows are complete (all 128 columns) inside the
// CTA, so the RMSNorm needs no exchange between the CTAs.
//
// The paired accumulators use the folded TMEM layout of an M = 64-per-CTA
// MMA: lanes 0..63 hold the 64 rows for columns [0, N/2), lanes 64..127 the
// same rows for columns [N/2, N), both in TMEM columns [0, N/2).
//
// Warps (352 threads per CTA):
//   warp 0      TMA producer: each CTA loads its own halves; CTA 1's loads complete
//               CTA 0's ring barriers directly (the .cta_group::2 load form)
//   warp 1      CTA 0: TMEM owner and MMA issuer A: S_{b+1} (look-ahead), dKV_b^T = V_b^T K_b.
//               CTA 1: takes part in the TMEM allocation only.
//   warps 2..5  group P: S -> causal mask -> bf16 P (shared memory, A operand of P V)
//   warps 6..9  group O: KV^T += dKV^T, bf16 snapshot, O -> (RMSNorm) -> bf16 store,
//               final fp32 state -> global store
//   warp 10     CTA 0: MMA issuer B: O_b = Q_b snap(KV_{<b}), O_b += P_b V_b.
// Two issuing threads keep the tensor pipe fed; each has one commit per block
// (s_full and kv_done for A, o_done for B), and each commit arrives on the
// barriers of both CTAs.  Signals to the issuers are mbarrier arrivals (remote
// ones from CTA 1).  Every wait is bounded; on a timeout the CTA records
// DEV_TIMEOUT, drains its own copies and MMAs, frees TMEM and returns.
#pragma once

#include "prefill_tc.cuh"

namespace la {

struct PrefillPairParams {
    CUtensorMap tmap_q64;   // Q as [T][H*D], box 64 columns x 64 rows
    CUtensorMap tmap_k64;   // K, box 64 x 64
    CUtensorMap tmap_k128;  // K, box 64 x 128
    CUtensorMap tmap_v128;  // V, box 64 x 128
    __nv_bfloat16 *o;
    float *state;           // [S][H][D][D] or nullptr: final states
    const float *state_in;  // [S][H][D][D] or nullptr: initial states (may alias state)
    int H;
    int rmsnorm;
    unsigned long long timeout_ns;
    SeqTable seqs;
};

#ifndef LA_PAIR_S_AHEAD
#define LA_PAIR_S_AHEAD 1
#endif
#ifndef LA_PAIR_P_BUFS
#define LA_PAIR_P_BUFS 1
#endif
#ifndef LA_PAIR_KK_DEPTH
#define LA_PAIR_KK_DEPTH 2
#endif
#ifndef LA_PAIR_QH_DEPTH
#define LA_PAIR_QH_DEPTH 4
#endif
#ifndef LA_PAIR_KV_DEPTH
#define LA_PAIR_KV_DEPTH 2
#endif

struct PairCfg {
    static constexpr int BETA = 128, D = 128;
    static constexpr int HBOX = 64 * 128;               // 64 rows x 128 B
    static constexpr int FBOX = 128 * 128;              // 128 rows x 128 B
    // Three TMA rings, each released at the last use of its tiles (all tiles
    // 128-byte swizzled; a "half" is dims [0,64) | [64,128) of 64 rows):
    //   KK: own 64 key rows, both dim halves           (S = Q K^T)
    //   QH: own 64 query rows, both dim halves         (S, and O += Q snap)
    //   KV: 128 key rows x own 64 dims | 128 value rows x own 64 columns (P V, V^T K)
    static constexpr int NKK = LA_PAIR_KK_DEPTH, NQH = LA_PAIR_QH_DEPTH, NKV = LA_PAIR_KV_DEPTH;
    // ring of block-completion barriers; a ring's depth may not exceed the barrier
    // ring it waits on, or a phase could be lapped before its waiter sees it
    static constexpr int NDONE = 4;
    // S runs SAHEAD blocks ahead of the block whose P V consumes it, in a ring of
    // SAHEAD + 1 TMEM buffers (the extra one is being turned into P by group P)
    static constexpr int SAHEAD = LA_PAIR_S_AHEAD, NS = SAHEAD + 1;
    static_assert(NKK <= NS, "key-row slots are released by s_full[NS]");
    static_assert(NQH <= NDONE && NKV <= NDONE, "slot release ring");
    static constexpr int KK_BYTES = 2 * HBOX, QH_BYTES = 2 * HBOX, KV_BYTES = 2 * FBOX;
    static constexpr int OFF_KK = 0;
    static constexpr int OFF_QH = OFF_KK + NKK * KK_BYTES;
    static constexpr int OFF_KV = OFF_QH + NQH * QH_BYTES;
    static constexpr int KV_OFF_VC = FBOX;               // within a KV stage
    // P buffers (own 64 rows of P, keys [0,64) | [64,128)); P_b goes to buffer b % NPB
    static constexpr int NPB = LA_PAIR_P_BUFS, P_BYTES = 2 * HBOX;
    static_assert(NPB <= NDONE, "P buffers are released by o_done");
    static constexpr int OFF_P = OFF_KV + NKV * KV_BYTES;
    // two bf16 snapshots of the state (own 64 rows of KV^T, dims [0,64) | [64,128)):
    // the one for block b+1 is written while O_b = Q_b snap still reads the other
    static constexpr int SNAP_BYTES = 2 * HBOX;
    static constexpr int OFF_SNAP = OFF_P + NPB * P_BYTES;
    static constexpr int OFF_MISC = OFF_SNAP + 2 * SNAP_BYTES;
    static constexpr int MISC = 2048;
    static constexpr int SMEM_BYTES = 1024 + OFF_MISC + MISC;
    static_assert(SMEM_BYTES <= 227 * 1024, "shared memory budget");
    // TMEM columns: S[NS], O[2], dKV[2], 64 columns each (folded layout)
    static constexpr int TM_S = 0, TM_O = 64 * NS, TM_DKV = 64 * NS + 128;
    static_assert(TM_DKV + 128 <= 512, "TMEM columns");
    static constexpr int TMEM_COLS = 512;
    static constexpr int GROUP = 128;
    static constexpr int WARP_B = 10;                   // second MMA issuer (CTA 0)
    static constexpr int THREADS = 64 + 2 * GROUP + 32;
    static constexpr uint32_t ID_S = idesc_bf16_f32(128, 128, 0, 0);
    static constexpr uint32_t ID_PV = idesc_bf16_f32(128, 128, 0, 1);
    static constexpr uint32_t ID_QKV = idesc_bf16_f32(128, 128, 0, 0);
    static constexpr uint32_t ID_KV = idesc_bf16_f32(128, 128, 1, 1);
};

// Every wait below is a parity wait on one phase x of a barrier.  Two rules make
// it exact: phase x - 1 is known to be complete when the wait starts (the waiter
// saw it, or a chain of signals implies it), and phase x + 1 cannot complete
// before the wait returns.  This is why the S buffers, the P buffers and the
// snapshots have a barrier per buffer and the tail zeroing a single-phase barrier.
struct PairMisc {
    // Ring barriers.  "full" barriers are used in CTA 0 only: CTA 0's producer
    // expects the bytes of both CTAs and CTA 1's loads complete them directly.
    // A slot is free again once the MMAs reading it have completed: s_full[j % NS]
    // frees key-row slot j (S_j done), o_done[j % 4] the query slot (O_j done, which
    // follows S_j), o_done and kv_done[j % 4] together the K/V slot.  Every MMA
    // commit arrives on the barrier of both CTAs.
    uint64_t full_kk[PairCfg::NKK];
    uint64_t full_qh[PairCfg::NQH];
    uint64_t full_kv[PairCfg::NKV];
    uint64_t tail_kv;              // CTA 1: its own KV tiles of a partial last block landed
    uint64_t tail_zeroed;          // used in CTA 0: value rows past the sequence end zeroed
    uint64_t s_full[PairCfg::NS];  // S_j complete (buffer j % NS)
    uint64_t s_free[PairCfg::NS];  // used in CTA 0: group P of both CTAs has loaded S_j
    uint64_t kv_done[4];           // dKV_j complete (issuer A)
    uint64_t o_done[4];            // O_j complete (issuer B)
    uint64_t o_free[2];            // used in CTA 0: arrivals from both CTAs
    uint64_t dkv_free[2];
    uint64_t p_ready[PairCfg::NPB];  // used in CTA 0: P_j stored in buffer j % NPB
    uint64_t snap_ready[2];        // used in CTA 0: snapshot u (for block u) in buffer u % 2
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
    // a partial last block: its value rows past the sequence end are zeroed by group P
    const bool tail = nb > 0 && seq_len < nb * C::BETA;
    // Snapshot u of the state (bf16, buffer u % 2) feeds O_u = Q_u snap_u.  With an
    // initial state X the first one (u = 0) is X; without one, block 0 has no
    // inter-block term and the first snapshot is u = 1.
    const int u0 = p.state_in != nullptr ? 0 : 1;
    const uint64_t tlimit = p.timeout_ns;
    volatile int *abort_flag = &m->abort_flag;

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::NKK; ++s) mbar_init(&m->full_kk[s], 1);
        for (int s = 0; s < C::NQH; ++s) mbar_init(&m->full_qh[s], 1);
        for (int s = 0; s < C::NKV; ++s) mbar_init(&m->full_kv[s], 1);
        for (int s = 0; s < C::NS; ++s) {
            mbar_init(&m->s_full[s], 1);
            mbar_init(&m->s_free[s], 2 * C::GROUP);
        }
        for (int s = 0; s < C::NDONE; ++s) {
            mbar_init(&m->kv_done[s], 1);
            mbar_init(&m->o_done[s], 1);
        }
        mbar_init(&m->tail_kv, 1);
        mbar_init(&m->tail_zeroed, 2 * C::GROUP);
        for (int i = 0; i < 2; ++i) {
            mbar_init(&m->snap_ready[i], 2 * C::GROUP);
            mbar_init(&m->o_free[i], 2 * C::GROUP);
            mbar_init(&m->dkv_free[i], 2 * C::GROUP);
        }
        for (int i = 0; i < C::NPB; ++i) mbar_init(&m->p_ready[i], 2 * C::GROUP);
        mbar_init(&m->drain, 2);
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
    auto kk_addr = [&](int j) { return sbase + (uint32_t)(C::OFF_KK + (j % C::NKK) * C::KK_BYTES); };
    auto qh_addr = [&](int j) { return sbase + (uint32_t)(C::OFF_QH + (j % C::NQH) * C::QH_BYTES); };
    auto kv_addr = [&](int j) { return sbase + (uint32_t)(C::OFF_KV + (j % C::NKV) * C::KV_BYTES); };
    // Bounded warp-uniform wait.  A CTA-scope poll suffices: remote producers
    // order their shared-memory writes with a cluster-scope release fence before
    // arriving, and MMA commits and TMA loads complete the barriers directly.
    auto wwait = [&](uint64_t *bar, uint32_t parity) -> bool {
        return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort_flag, tlimit)) != 0;
    };
    // Signals to CTA 0.  CTA 0's own threads arrive locally.  CTA 1's threads
    // publish their shared-memory writes (P, the state snapshot, zeroed value
    // rows) with a release fence restricted to shared memory and a relaxed
    // remote arrival; a full cluster-scope release would also wait for the
    // thread's outstanding global stores.  Signals that only free a TMEM buffer
    // (the tcgen05.ld has completed) publish nothing and use a plain relaxed
    // arrival.
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
        // One thread polls the three rings and refills whichever slot the MMAs have
        // released.  CTA 0 expects the bytes of both CTAs on its full barrier; CTA 1's
        // loads complete CTA 0's barrier directly.  The KV tiles of a partial last
        // block are the exception: CTA 1 loads them against its own tail barrier, so
        // that its group P can zero the value rows past the sequence end once they
        // have landed, and CTA 0 expects only its own bytes for that block.
        if (lane == 0) {
            const int col = h * C::D;
            const int own_rows = 64 * (int)cta, own_cols = col + 64 * (int)cta;
            int jk = 0, jq = 0, jv = 0;
            // slot of block j free: block j - depth has released it
            auto freed = [&](uint64_t *ring, int nring, int j, int depth) {
                const int x = j - depth;
                return x < 0 || mbar_test(&ring[x % nring], (uint32_t)((x / nring) & 1));
            };
            uint64_t t0 = globaltimer_ns();
            uint32_t polls = 0;
            while (jk < nb || jq < nb || jv < nb) {
                bool progressed = false;
                if (jk < nb && freed(m->s_full, C::NS, jk, C::NKK)) {
                    uint64_t *fb = &m->full_kk[jk % C::NKK];
                    const uint32_t dst = kk_addr(jk);
                    const int row = seq_start + jk * C::BETA + own_rows;
                    if (cta == 0) {
                        mbar_arrive_expect_tx(fb, (uint32_t)(2 * C::KK_BYTES));
                        tma_load_2d(dst, &p.tmap_k64, col, row, fb);
                        tma_load_2d(dst + C::HBOX, &p.tmap_k64, col + 64, row, fb);
                    } else {
                        const uint32_t fr = cluster_addr(fb, 0);
                        tma_load_2d_pairbar(dst, &p.tmap_k64, col, row, fr);
                        tma_load_2d_pairbar(dst + C::HBOX, &p.tmap_k64, col + 64, row, fr);
                    }
                    ++jk;
                    progressed = true;
                }
                if (jq < nb && freed(m->o_done, C::NDONE, jq, C::NQH)) {
                    uint64_t *fb = &m->full_qh[jq % C::NQH];
                    const uint32_t dst = qh_addr(jq);
                    const int row = seq_start + jq * C::BETA + own_rows;
                    if (cta == 0) {
                        mbar_arrive_expect_tx(fb, (uint32_t)(2 * C::QH_BYTES));
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
                if (jv < nb && freed(m->kv_done, C::NDONE, jv, C::NKV) &&
                    freed(m->o_done, C::NDONE, jv, C::NKV)) {
                    uint64_t *fb = &m->full_kv[jv % C::NKV];
                    const uint32_t dst = kv_addr(jv);
                    const int row = seq_start + jv * C::BETA;
                    const bool last_partial = tail && jv == nb - 1;
                    if (cta == 0) {
                        mbar_arrive_expect_tx(fb, (uint32_t)((last_partial ? 1 : 2) * C::KV_BYTES));
                        tma_load_2d(dst, &p.tmap_k128, own_cols, row, fb);
                        tma_load_2d(dst + C::KV_OFF_VC, &p.tmap_v128, own_cols, row, fb);
                    } else if (last_partial) {
                        mbar_arrive_expect_tx(&m->tail_kv, (uint32_t)C::KV_BYTES);
                        tma_load_2d(dst, &p.tmap_k128, own_cols, row, &m->tail_kv);
                        tma_load_2d(dst + C::KV_OFF_VC, &p.tmap_v128, own_cols, row, &m->tail_kv);
                    } else {
                        const uint32_t fr = cluster_addr(fb, 0);
                        tma_load_2d_pairbar(dst, &p.tmap_k128, own_cols, row, fr);
                        tma_load_2d_pairbar(dst + C::KV_OFF_VC, &p.tmap_v128, own_cols, row, fr);
                    }
                    ++jv;
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
            if (cta == 0) {
                const uint64_t lim = tlimit < 10000000ull ? tlimit : 10000000ull;
                for (int j = (jk > C::NKK ? jk - C::NKK : 0); j < jk; ++j)
                    mbar_wait(&m->full_kk[j % C::NKK], (uint32_t)((j / C::NKK) & 1), nullptr, lim);
                for (int j = (jq > C::NQH ? jq - C::NQH : 0); j < jq; ++j)
                    mbar_wait(&m->full_qh[j % C::NQH], (uint32_t)((j / C::NQH) & 1), nullptr, lim);
                for (int j = (jv > C::NKV ? jv - C::NKV : 0); j < jv; ++j)
                    mbar_wait(&m->full_kv[j % C::NKV], (uint32_t)((j / C::NKV) & 1), nullptr, lim);
            } else if (tail && jv == nb) {
                mbar_wait(&m->tail_kv, 0u, nullptr, tlimit < 10000000ull ? tlimit : 10000000ull);
            }
        }
        __syncwarp();
    } else if (warp == 1 && cta == 0) {
        // ------------------------------------------------------------ issuer A (CTA 0): S, dKV
        // One thread issues tcgen05.mma at well under the tensor pipe's rate for these
        // M = 128 (64 rows per CTA), N = 128 paired MMAs, so the work is split between two
        // issuing warps: A issues the products that depend only on loads (S and dKV), B
        // those that wait on the epilogue warps (the inter-block term and P V).  A commit
        // covers the MMAs of its own thread only.
        auto stage_in = [&](int j) -> bool {  // S_j = Q_j K_j^T
            if (!wwait(&m->full_kk[j % C::NKK], (uint32_t)((j / C::NKK) & 1)) ||
                !wwait(&m->full_qh[j % C::NQH], (uint32_t)((j / C::NQH) & 1)))
                return false;
            // S buffer j % NS was last read by group P for block j - NS
            if (j >= C::NS && !wwait(&m->s_free[j % C::NS], (uint32_t)(((j - C::NS) / C::NS) & 1)))
                return false;
            tc_fence_after();
            if (lane == 0) {
                const uint64_t qd = desc_kmajor_sw128(qh_addr(j));
                const uint64_t kd = desc_kmajor_sw128(kk_addr(j));
#pragma unroll
                for (int ks = 0; ks < C::D / 16; ++ks) {
                    const uint32_t off = (uint32_t)((ks >> 2) * C::HBOX + (ks & 3) * 32);
                    mma_bf16_ss_pair(tmem + C::TM_S + 64 * (j % C::NS), desc_add(qd, off),
                                     desc_add(kd, off), C::ID_S, ks > 0 ? 1u : 0u);
                }
                mma_commit_pair_both(&m->s_full[j % C::NS]);
            }
            __syncwarp();
            return true;
        };
        // Per block b: dKV_b^T = V_b^T K_b, then S_{b+SAHEAD} (look-ahead, so that group P
        // has SAHEAD blocks' time to form P from it).  dKV_b goes first: the snapshot of
        // KV_{<b+1} that issuer B waits for is derived from it.
        bool ok = true;
        for (int j = 0; ok && j < C::SAHEAD && j < nb; ++j) ok = stage_in(j);
        for (int b = 0; ok && b < nb; ++b) {
            const uint32_t kva = kv_addr(b);
            // a partial last block: group P zeroes the value rows past the sequence end
            // before dKV_b may read them
            const bool zero_tail = tail && b == nb - 1;
            if ((zero_tail && !wwait(&m->tail_zeroed, 0u)) ||
                !wwait(&m->full_kv[b % C::NKV], (uint32_t)((b / C::NKV) & 1)) ||
                (b >= 2 && !wwait(&m->dkv_free[b & 1], (uint32_t)(((b - 2) >> 1) & 1)))) {
                ok = false;
                break;
            }
            tc_fence_after();
            if (lane == 0) {
                const uint64_t vd = desc_mnmajor_sw128(kva + C::KV_OFF_VC, C::FBOX);
                const uint64_t kd = desc_mnmajor_sw128(kva, C::FBOX);
#pragma unroll
                for (int ks = 0; ks < C::BETA / 16; ++ks)
                    mma_bf16_ss_pair(tmem + C::TM_DKV + 64 * (b & 1), desc_add(vd, ks * 2048),
                                     desc_add(kd, ks * 2048), C::ID_KV, ks > 0 ? 1u : 0u);
                mma_commit_pair_both(&m->kv_done[b % C::NDONE]);
            }
            __syncwarp();
            if (b + C::SAHEAD < nb && !stage_in(b + C::SAHEAD)) {
                ok = false;
                break;
            }
        }
        if (!ok) fail();
        if (lane == 0) {  // every MMA of both issuers has finished before TMEM is freed
            mma_commit_pair(smem_u32(&m->drain));
            mbar_wait(&m->drain, 0u, nullptr, tlimit);
        }
        __syncwarp();
    } else if (warp == 1) {
        // CTA 1's warp 1 only takes part in the TMEM allocation.
    } else if (warp == C::WARP_B) {
        if (cta == 0) {
            // -------------------------------------------------------- issuer B (CTA 0): O
            // Per block b: O_b = Q_b snap(KV_{<b}), then O_b += P_b V_b.
            bool ok = true;
            for (int b = 0; ok && b < nb; ++b) {
                const uint32_t dO = tmem + C::TM_O + 64 * (b & 1);
                // The query tile of block b must have landed: nothing else that this thread
                // waits for implies it (S_b was issued by the other thread, and the
                // snapshot does not depend on it).  Checked for every block, in order.
                if ((b >= 2 && !wwait(&m->o_free[b & 1], (uint32_t)(((b - 2) >> 1) & 1))) ||
                    !wwait(&m->full_qh[b % C::NQH], (uint32_t)((b / C::NQH) & 1))) {
                    ok = false;
                    break;
                }
                if (b >= u0) {
                    // snapshot b is the (b - u0)/2-th use of buffer b % 2
                    if (!wwait(&m->snap_ready[b & 1], (uint32_t)(((b - u0) >> 1) & 1))) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    if (lane == 0) {
                        const uint64_t qd = desc_kmajor_sw128(qh_addr(b));
                        const uint64_t sd = desc_kmajor_sw128(sbase + C::OFF_SNAP + (b & 1) * C::SNAP_BYTES);
#pragma unroll
                        for (int ks = 0; ks < C::D / 16; ++ks) {
                            const uint32_t off = (uint32_t)((ks >> 2) * C::HBOX + (ks & 3) * 32);
                            mma_bf16_ss_pair(dO, desc_add(qd, off), desc_add(sd, off), C::ID_QKV,
                                             ks > 0 ? 1u : 0u);
                        }
                    }
                    __syncwarp();
                }
                if (!wwait(&m->p_ready[b % C::NPB], (uint32_t)((b / C::NPB) & 1)) ||
                    !wwait(&m->full_kv[b % C::NKV], (uint32_t)((b / C::NKV) & 1))) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                if (lane == 0) {
                    const uint64_t pd = desc_kmajor_sw128(sbase + C::OFF_P + (b % C::NPB) * C::P_BYTES);
                    const uint64_t vd = desc_mnmajor_sw128(kv_addr(b) + C::KV_OFF_VC, C::FBOX);
#pragma unroll
                    for (int ks = 0; ks < C::BETA / 16; ++ks)
                        mma_bf16_ss_pair(dO, desc_add(pd, (uint32_t)((ks >> 2) * C::HBOX + (ks & 3) * 32)),
                                         desc_add(vd, ks * 2048), C::ID_PV, (b >= u0 || ks > 0) ? 1u : 0u);
                    mma_commit_pair_both(&m->o_done[b % C::NDONE]);
                }
                __syncwarp();
            }
            if (!ok) fail();
            if (lane == 0) {
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
        const uint32_t sP = sbase + C::OFF_P;
        bool ok = true;
        for (int b = 0; b < nb; ++b) {
            if (!wwait(&m->s_full[b % C::NS], (uint32_t)((b / C::NS) & 1))) {
                ok = false;
                break;
            }
            tc_fence_after();
            uint32_t s0[32], s1[32];
            const uint32_t tS = tmem + C::TM_S + 64 * (b % C::NS) + lane_base;
            tmem_ld32(tS, s0);
            tmem_ld32(tS + 32, s1);
            tmem_ld_wait();
            tc_fence_before();
            arrive_leader_free(&m->s_free[b % C::NS]);
            uint32_t w[32];
#pragma unroll
            for (int u = 0; u < 32; ++u) {
                const uint32_t *s = u < 16 ? &s0[2 * u] : &s1[2 * (u - 16)];
                const int c0 = 64 * kh + 2 * u;
                const float x0 = c0 <= R ? __uint_as_float(s[0]) : 0.f;
                const float x1 = c0 + 1 <= R ? __uint_as_float(s[1]) : 0.f;
                w[u] = pack_bf16x2(x0, x1);
            }
            // P buffer b % NPB was last read by O_{b-NPB} += P V; that must be complete
            const int pb = b - C::NPB;
            if (pb >= 0 && !wwait(&m->o_done[pb % C::NDONE], (uint32_t)((pb / C::NDONE) & 1))) {
                ok = false;
                break;
            }
#pragma unroll
            for (int t = 0; t < 8; ++t)
                st_shared_v4(sP + (b % C::NPB) * C::P_BYTES + kh * C::HBOX + r * 128 + ((uint32_t)(t ^ (r & 7)) << 4), w[4 * t],
                             w[4 * t + 1], w[4 * t + 2], w[4 * t + 3]);
            // V rows past the sequence end must not enter dKV^T: zero them in this CTA's
            // slice once its KV tiles of the block have landed.
            const int nv = min(C::BETA, seq_len - b * C::BETA);
            if (nv < C::BETA) {
                const bool landed = cta == 0 ? wwait(&m->full_kv[b % C::NKV], (uint32_t)((b / C::NKV) & 1))
                                             : wwait(&m->tail_kv, 0u);
                if (!landed) {
                    ok = false;
                    break;
                }
                const uint32_t v0 = kv_addr(b) + C::KV_OFF_VC;
                for (uint32_t a = v0 + nv * 128 + (threadIdx.x - 64) * 16; a < v0 + C::FBOX;
                     a += C::GROUP * 16)
                    st_shared_v4(a, 0u, 0u, 0u, 0u);
                fence_proxy_async_smem();
                arrive_leader(&m->tail_zeroed);
            }
            fence_proxy_async_smem();
            tc_fence_before();
            arrive_leader(&m->p_ready[b % C::NPB]);
        }
        if (!ok) fail();
    } else {
        // ------------------------------------------------------------ group O (both CTAs)
        const int q = warp & 3;
        const uint32_t lane_base = (uint32_t)(32 * q) << 16;
        const int r = 32 * (q & 1) + lane;     // own output row / own value column j
        const int half = q >> 1;               // column half (O) / dim half (state)
        float kv[64];                          // KV^T[64 c + r][64 half .. 64 half + 63]
#pragma unroll
        for (int t = 0; t < 64; ++t) kv[t] = 0.f;
        bool ok = true;
        // snapshot u of the state into buffer u % 2 (own 64 rows of KV^T, bf16, swizzled)
        auto write_snap = [&](int u) {
            const uint32_t sSnap = sbase + C::OFF_SNAP + (u & 1) * C::SNAP_BYTES;
#pragma unroll
            for (int t = 0; t < 8; ++t)
                st_shared_v4(sSnap + half * C::HBOX + r * 128 + ((uint32_t)(t ^ (r & 7)) << 4),
                             pack_bf16x2(kv[8 * t + 0], kv[8 * t + 1]),
                             pack_bf16x2(kv[8 * t + 2], kv[8 * t + 3]),
                             pack_bf16x2(kv[8 * t + 4], kv[8 * t + 5]),
                             pack_bf16x2(kv[8 * t + 6], kv[8 * t + 7]));
            fence_proxy_async_smem();
            arrive_leader(&m->snap_ready[u & 1]);
        };
        if (p.state_in != nullptr) {  // KV^T[j][i] starts at the initial state X[i][j]
            const float *src = p.state_in + ((size_t)sid * p.H + h) * C::D * C::D + 64 * (int)cta + r;
#pragma unroll
            for (int t = 0; t < 64; ++t) kv[t] = src[(size_t)(64 * half + t) * C::D];
            write_snap(0);
        }
        for (int b = 0; b < nb; ++b) {
            // (1) state: KV^T += dKV_b^T, then the bf16 snapshot for O_{b+1} += Q_{b+1} KV
            if (!wwait(&m->kv_done[b % C::NDONE], (uint32_t)((b / C::NDONE) & 1))) {
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
                // Snapshot b + 1 goes to buffer (b+1) & 1, last read by O_{b-1} = Q_{b-1}
                // snap_{b-1}, complete since o_done(b-1), which this group waited for in
                // the previous block.
                write_snap(b + 1);
            }
            // (2) output block b
            if (!wwait(&m->o_done[b % C::NDONE], (uint32_t)((b / C::NDONE) & 1))) {
                ok = false;
                break;
            }
            tc_fence_after();
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
