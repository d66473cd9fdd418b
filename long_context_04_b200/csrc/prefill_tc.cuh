// Lightning-attention prefill for bf16 inputs on sm_100a: TMA + tcgen05 + TMEM.
//
// Method (MiniMax-01, "Scaling Foundation Models with Lightning Attention";
// CSDN digest section 2.1, mizuki blog appendix "key concepts"): for every
// block b of BETA tokens of one sequence and one head,
//     O_b = [(Q_b K_b^T) (.) M] V_b + Q_b KV,     KV += K_b^T V_b,
// with the causal 0/1 mask M (j <= i) and KV reset at each sequence start,
// followed by an optional RMSNorm of each output row over the head dim.
//
// One CTA owns one work unit (sequence, head, 64-column slice of V/O).  With
// D = 128 the two slices of a (sequence, head) form a 2-CTA cluster: both
// compute S = Q_b K_b^T (the second reads Q/K from L2) and they exchange
// per-row sums of squares through distributed shared memory for the RMSNorm.
// The four block contractions run on the tensor cores with fp32 accumulators
// in TMEM.  The state update is split to keep the serial chain short: the MMA
// writes each block's increment dKV_b = K_b^T V_b into one of two TMEM
// buffers, and the epilogue keeps the running fp32 state KV in registers
// (one state row per thread), adds dKV_b, and writes the bf16 snapshot that
// the next block's Q_{b+1} KV product reads.  So the MMA never waits for a
// TMEM read before the next state update, and the whole state stays on chip
// for the entire sequence.
//
// Warp roles (480 threads):
//   warp 0      TMA producer: Q_b, K_b (D columns) and V_b (64 columns) into a
//               ring of NST shared-memory stages.
//   warp 1      TMEM owner and MMA issuer A: the scores S and dKV_b = K_b^T V_b
//               (lane 0 issues).
//   warp 14     MMA issuer B: O_b = P_b V_b and the inter-block term Q_b snap(KV_{<b})
//               (the warp first zeroes the V rows past a sequence end).
//   warps 2..5  group P: S_b -> causal mask -> bf16 P_b, written back into
//               the first BETA/2 columns of S_b's TMEM buffer, where the
//               O_b = P_b V_b product reads it as its A operand.
//   warps 6..9  group O: O_b -> (RMSNorm) -> bf16 global store.
//   warps 10..13 group KV: KV += dKV_b, bf16 snapshot of KV, final fp32 state.
// The state chain (group KV) and the output (group O) run on separate warps, so
// the next snapshot never waits behind an output store or the RMSNorm exchange.
// Per block b, issuer B: O_b = P_b V_b, then O_b += Q_b snap(KV_{<b}) on the same
// accumulator; issuer A, once P_b V_b has completed: dKV_b, then S_{b+2}.  Each
// issues 12 of the 24 MMAs of a block (at beta = 64) and releases the stage of
// block b after its last product that reads it.
// Every wait is bounded (see mbar_wait); on a timeout the CTA records
// DEV_TIMEOUT, drains its own copies and MMAs, frees TMEM and returns.
#pragma once

#include "la_device.cuh"
#include "../../include/lightning_attention.h"

namespace la {

// Sequences of one call.  Uniform batches (varlen = 0) use start = r * N and
// length N.  Packed batches list their sequences longest first, so that the
// hardware block scheduler, which starts CTAs in index order, hands out the
// longest chains first.
struct SeqTable {
    int varlen;
    int N;
    int seq_start[LA_MAX_VARLEN_SEQS];
    int seq_len[LA_MAX_VARLEN_SEQS];
    int seq_id[LA_MAX_VARLEN_SEQS];  // index of the sequence in the caller's order

    __device__ __forceinline__ void get(int r, int &start, int &len, int &sid) const {
        if (varlen) {
            start = seq_start[r];
            len = seq_len[r];
            sid = seq_id[r];
        } else {
            start = r * N;
            len = N;
            sid = r;
        }
    }
};

struct PrefillTcParams {
    CUtensorMap tmap_q;  // [T][H*D] bf16, box 64 x BETA, 128-byte swizzle
    CUtensorMap tmap_k;
    CUtensorMap tmap_v;
    __nv_bfloat16 *o;
    float *state;        // [S][H][D][D] or nullptr: final states
    const float *state_in;  // [S][H][D][D] or nullptr: initial states (may alias state)
    int H;
    int rmsnorm;
    unsigned long long timeout_ns;
    SeqTable seqs;
};

#ifndef LA_PREFETCH_BLOCKS
#define LA_PREFETCH_BLOCKS 0
#endif

template <int BETA, int D>
struct TcCfg {
    static constexpr int NVS = D / 64;          // CTAs per (sequence, head)
    static constexpr int DB = D / 64;           // 64-column tiles in Q or K
    static constexpr int BOX = BETA * 128;      // one 64-column tile of BETA rows (bytes)
    static constexpr int STAGE = (2 * DB + 1) * BOX;
    static constexpr int SNAP_BYTES = D * 128;  // D rows x 64 bf16
    static constexpr int SMEM_LIMIT = 227 * 1024;
    static constexpr int MISC = 2048;
    static constexpr int NST_FIT =
        (SMEM_LIMIT - 1024 - 2 * SNAP_BYTES - MISC) / STAGE;
    static constexpr int NST = NST_FIT > 4 ? 4 : NST_FIT;
    static_assert(NST >= 3, "shared memory budget: S runs two blocks ahead");
    // Blocks ahead of the TMA ring whose tiles are prefetched into L2, so that a
    // stage load is served from L2 rather than waiting on HBM.
    static constexpr int PF = LA_PREFETCH_BLOCKS;
    static constexpr int OFF_SNAP = NST * STAGE;              // two snapshot buffers
    static constexpr int OFF_MISC = OFF_SNAP + 2 * SNAP_BYTES;
    // At least 120 KB so that no two CTAs share an SM: each allocates all 512
    // TMEM columns, and a second resident CTA would block in tcgen05.alloc.
    static constexpr int SMEM_USED = 1024 + OFF_MISC + MISC;
    static constexpr int SMEM_BYTES = SMEM_USED < 120 * 1024 ? 120 * 1024 : SMEM_USED;
    static_assert(SMEM_USED <= SMEM_LIMIT, "shared memory budget");
    // TMEM columns: S[2] (BETA each; P overwrites the first BETA/2 of each),
    // O[2] (64 each), dKV[2] (64 each)
    static constexpr int TM_S = 0;
    static constexpr int TM_O = 2 * BETA;
    static constexpr int TM_DKV = 2 * BETA + 128;
    static constexpr int TMEM_COLS = 512;
    static_assert(TM_DKV + 128 <= TMEM_COLS, "TMEM budget");
    static constexpr int GROUP = 128;           // threads of one epilogue group
    static constexpr int THREADS = 64 + 3 * GROUP + 32;
    static constexpr int WARP_B = 14;           // issuer of P V and dKV
    static constexpr uint32_t ID_S = idesc_bf16_f32(BETA, BETA, 0, 0);
    static constexpr uint32_t ID_PV = idesc_bf16_f32(BETA, 64, 0, 1);
    static constexpr uint32_t ID_QKV = idesc_bf16_f32(BETA, 64, 0, 1);
    static constexpr uint32_t ID_KV = idesc_bf16_f32(D, 64, 1, 1);
};

// Barriers and small shared state, placed after the tiles.
template <int NST, int BETA>
struct TcMisc {
    uint64_t full[NST];
    uint64_t empty[NST];
    uint64_t s_full[2];
    uint64_t o_full[2];
    uint64_t o_free[2];
    uint64_t dkv_full[2];
    uint64_t dkv_free[2];
    uint64_t ss_full[2];
    uint64_t p_ready[2];     // P_b written over S_b in TMEM buffer b % 2
    uint64_t pv_done[2];     // P_b V_b complete (issuer B -> issuer A)
    uint64_t tail_zeroed;    // issuer B zeroed the value rows past the sequence end
    uint64_t snap_ready[2];  // snapshot u of the state is in buffer u % 2
    uint64_t drain;
    uint32_t tmem_base;
    int abort_flag;
    float ss_in[2][BETA];
};

template <int BETA, int D>
__global__ void __launch_bounds__(TcCfg<BETA, D>::THREADS, 1)
    prefill_tc_kernel(const __grid_constant__ PrefillTcParams p) {
    using C = TcCfg<BETA, D>;
    using Misc = TcMisc<C::NST, BETA>;
    static_assert(sizeof(Misc) <= C::MISC, "misc area");

    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    Misc *m = reinterpret_cast<Misc *>(smem + C::OFF_MISC);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int unit = blockIdx.x;
    const int vs = unit % C::NVS;
    const int rh = unit / C::NVS;
    const int h = rh % p.H;
    const int rank = rh / p.H;
    int seq_start, seq_len, sid;
    p.seqs.get(rank, seq_start, seq_len, sid);
    const int nb = (seq_len + BETA - 1) / BETA;
    // Snapshots u of the state feed O_u += Q_u snap_u.  With an initial state X the
    // first one (u = 0) is X itself; without one, block 0 has no inter-block term
    // and the first snapshot is u = 1.
    const int u0 = p.state_in != nullptr ? 0 : 1;
    const uint32_t partner = (uint32_t)(vs ^ 1);
    const uint64_t tlimit = p.timeout_ns;
    volatile int *abort_flag = &m->abort_flag;

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::NST; ++s) {
            mbar_init(&m->full[s], 1);
            mbar_init(&m->empty[s], 2);   // one commit from each issuer
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&m->s_full[i], 1);
            mbar_init(&m->o_full[i], 1);
            mbar_init(&m->o_free[i], C::GROUP);
            mbar_init(&m->dkv_full[i], 1);
            mbar_init(&m->dkv_free[i], C::GROUP);
            mbar_init(&m->ss_full[i], C::GROUP);
        }
        mbar_init(&m->p_ready[0], C::GROUP);
        mbar_init(&m->p_ready[1], C::GROUP);
        mbar_init(&m->pv_done[0], 1);
        mbar_init(&m->pv_done[1], 1);
        mbar_init(&m->tail_zeroed, 1);
        mbar_init(&m->snap_ready[0], C::GROUP);
        mbar_init(&m->snap_ready[1], C::GROUP);
        mbar_init(&m->drain, 2);   // one commit from each issuer
        m->abort_flag = 0;
        fence_mbarrier_init_cluster();
        tma_prefetch_desc(&p.tmap_q);
        tma_prefetch_desc(&p.tmap_k);
        tma_prefetch_desc(&p.tmap_v);
    }
    if (warp == 1) {
        tmem_alloc(&m->tmem_base, C::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    if constexpr (C::NVS > 1) cluster_sync_all();
    tc_fence_after();
    const uint32_t tmem = m->tmem_base;

    auto fail = [&]() {
        *abort_flag = 1;
        record_fault(DEV_TIMEOUT);
    };
    auto stage_addr = [&](int st) { return sbase + (uint32_t)(st * C::STAGE); };
    // Warp-uniform bounded wait: every lane polls (and so acquires), and the
    // warp proceeds only if all lanes saw the phase complete, so that the
    // warp-collective tcgen05 instructions after it stay converged.
    auto wwait = [&](uint64_t *bar, uint32_t parity) -> bool {
        return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort_flag, tlimit)) != 0;
    };

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        int issued = 0;
        if (lane == 0) {
            auto prefetch = [&](int j) {
                const int row = seq_start + j * BETA;
                for (int c = 0; c < C::DB; ++c) {
                    tma_prefetch_l2_2d(&p.tmap_q, h * D + 64 * c, row);
                    tma_prefetch_l2_2d(&p.tmap_k, h * D + 64 * c, row);
                }
                tma_prefetch_l2_2d(&p.tmap_v, h * D + 64 * vs, row);
            };
            if constexpr (C::PF > 0)
                for (int j = C::NST; j < C::NST + C::PF && j < nb; ++j) prefetch(j);
            for (int b = 0; b < nb; ++b) {
                if (C::PF > 0 && b + C::NST + C::PF < nb) prefetch(b + C::NST + C::PF);
                const int st = b % C::NST;
                const uint32_t ph = (uint32_t)((b / C::NST) & 1);
                if (!mbar_wait(&m->empty[st], ph ^ 1u, abort_flag, tlimit)) {
                    fail();
                    break;
                }
                mbar_arrive_expect_tx(&m->full[st], (uint32_t)C::STAGE);
                const int row = seq_start + b * BETA;
                const uint32_t sa = stage_addr(st);
                for (int c = 0; c < C::DB; ++c) {
                    tma_load_2d(sa + c * C::BOX, &p.tmap_q, h * D + 64 * c, row, &m->full[st]);
                    tma_load_2d(sa + (C::DB + c) * C::BOX, &p.tmap_k, h * D + 64 * c, row,
                                &m->full[st]);
                }
                tma_load_2d(sa + 2 * C::DB * C::BOX, &p.tmap_v, h * D + 64 * vs, row, &m->full[st]);
                ++issued;
            }
            // Drain: the last NST issued loads must have landed before the CTA exits.
            for (int b = (issued > C::NST ? issued - C::NST : 0); b < issued; ++b)
                mbar_wait(&m->full[b % C::NST], (uint32_t)((b / C::NST) & 1), nullptr, tlimit);
        }
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer

        // Wait for block j's tiles and issue S_j.
        auto stage_in = [&](int j) -> bool {
            const int st = j % C::NST;
            if (!wwait(&m->full[st], (uint32_t)((j / C::NST) & 1))) return false;
            tc_fence_after();
            if (lane == 0) {
                const uint32_t sa = stage_addr(st);
                const uint32_t dS = tmem + C::TM_S + BETA * (j & 1);
                const uint64_t qd = desc_kmajor_sw128(sa), kd = desc_kmajor_sw128(sa + C::DB * C::BOX);
#pragma unroll
                for (int ks = 0; ks < D / 16; ++ks) {
                    const uint32_t off = (uint32_t)((ks >> 2) * C::BOX + (ks & 3) * 32);
                    mma_bf16_ss(dS, desc_add(qd, off), desc_add(kd, off), C::ID_S, ks > 0 ? 1u : 0u);
                }
                mma_commit(&m->s_full[j & 1]);
            }
            __syncwarp();
            return true;
        };

        // Per block b (issuer A): once issuer B's P_b V_b has completed, dKV_b = K_b^T V_b;
        // the stage's use by A is released; then S_{b+2} = Q_{b+2} K_{b+2}^T into S_b's
        // buffer, whose P_b that P V has read.  The scores run two blocks ahead, so group P
        // turns S_{b+1} into P_{b+1} during block b.  P_b V_b completing also means that
        // issuer B zeroed the value rows past a sequence end (before P V) and that its
        // Q_{b-1} snap_{b-1} has completed (issued before P V): group KV then writes snapshot
        // b + 1 into that snapshot's buffer once dKV_b is done.
        bool ok = nb == 0 || stage_in(0);
        if (ok && nb > 1) ok = stage_in(1);
        for (int b = 0; ok && b < nb; ++b) {
            const int st = b % C::NST;
            const uint32_t sa = stage_addr(st);
            const uint32_t sV = sa + 2 * C::DB * C::BOX;
            const uint32_t dKV = tmem + C::TM_DKV + 64 * (b & 1);
            // pv_done[b % 2] phase b / 2: its next phase needs P_{b+2} V_{b+2}, issued after
            // Q_{b+1} snap_{b+1}, which waits for snapshot b + 1 from the dKV_b below.
            // dkv_free: group KV has loaded dKV_{b-2} from this buffer.
            // tail_zeroed (single phase): issuer B's zeroed value rows, published with a
            // release arrival, before dKV of a partial last block reads them
            const bool last_tail = b == nb - 1 && seq_len < nb * BETA;
            if (!wwait(&m->pv_done[b & 1], (uint32_t)((b >> 1) & 1)) ||
                (b >= 2 && !wwait(&m->dkv_free[b & 1], (uint32_t)(((b - 2) >> 1) & 1))) ||
                (last_tail && !wwait(&m->tail_zeroed, 0u))) {
                ok = false;
                break;
            }
            tc_fence_after();
            if (lane == 0) {
                const uint64_t vd = desc_mnmajor_sw128(sV, C::BOX);
                const uint64_t ktd = desc_mnmajor_sw128(sa + C::DB * C::BOX, C::BOX);
#pragma unroll
                for (int ks = 0; ks < BETA / 16; ++ks)
                    mma_bf16_ss(dKV, desc_add(ktd, ks * 2048), desc_add(vd, ks * 2048), C::ID_KV,
                                ks > 0 ? 1u : 0u);
                mma_commit(&m->dkv_full[b & 1]);
                mma_commit(&m->empty[st]);
            }
            __syncwarp();
            if (b + 2 < nb && !stage_in(b + 2)) {
                ok = false;
                break;
            }
        }
        if (!ok) fail();
        if (nb > 0 && lane == 0) {  // every issued MMA has finished before TMEM is freed
            mma_commit(&m->drain);
            mbar_wait(&m->drain, 0u, nullptr, tlimit);
        }
        __syncwarp();
    } else if (warp == C::WARP_B) {
        // ------------------------------------------------------------ MMA issuer B
        // Per block b: O_b = P_b V_b (initialising O_b), then, in order on the same
        // accumulator, O_b += Q_b snap(KV_{<b}).  The value rows past a sequence end are
        // zeroed first (no product before them reads V_b).
        bool ok = true;
        for (int b = 0; b < nb; ++b) {
            const int st = b % C::NST;
            const uint32_t sa = stage_addr(st);
            const uint32_t sV = sa + 2 * C::DB * C::BOX;
            const uint32_t dO = tmem + C::TM_O + 64 * (b & 1);
            // full[st] phase b / NST: its next phase needs both issuers' release of block b;
            // p_ready[b % 2] phase b / 2: its next phase needs S_{b+2}, which issuer A issues
            // only after this P V; o_free: group O has loaded O_{b-2} from this buffer
            if (!wwait(&m->full[st], (uint32_t)((b / C::NST) & 1)) ||
                !wwait(&m->p_ready[b & 1], (uint32_t)((b >> 1) & 1)) ||
                (b >= 2 && !wwait(&m->o_free[b & 1], (uint32_t)(((b - 2) >> 1) & 1)))) {
                ok = false;
                break;
            }
            const int nv = min(BETA, seq_len - b * BETA);
            if (nv < BETA) {
                for (uint32_t a = sV + nv * 128 + lane * 16; a < sV + C::BOX; a += 32 * 16)
                    st_shared_v4(a, 0u, 0u, 0u, 0u);
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(&m->tail_zeroed);   // for issuer A's dKV
            }
            __syncwarp();
            tc_fence_after();
            if (lane == 0) {
                // O_b = P_b V_b, P_b from TMEM: 16 keys = 8 packed columns per K-step
                const uint32_t tP = tmem + C::TM_S + BETA * (b & 1);
                const uint64_t vd = desc_mnmajor_sw128(sV, C::BOX);
#pragma unroll
                for (int ks = 0; ks < BETA / 16; ++ks)
                    mma_bf16_ts(dO, tP + 8 * ks, desc_add(vd, ks * 2048), C::ID_PV, ks > 0 ? 1u : 0u);
                mma_commit(&m->pv_done[b & 1]);
            }
            __syncwarp();
            if (b >= u0) {
                // Snapshot b, the (b - u0)/2-th use of buffer b % 2.  Its next phase needs
                // dKV_{b+1}, which issuer A issues only after P_{b+1} V_{b+1}, issued here
                // after this product.
                if (!wwait(&m->snap_ready[b & 1], (uint32_t)(((b - u0) >> 1) & 1))) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                if (lane == 0) {  // O_b += Q_b snap(KV_{<b})
                    const uint32_t sSnap = sbase + C::OFF_SNAP + C::SNAP_BYTES * (b & 1);
                    const uint64_t qd = desc_kmajor_sw128(sa), sd = desc_mnmajor_sw128(sSnap, C::BOX);
#pragma unroll
                    for (int ks = 0; ks < D / 16; ++ks)
                        mma_bf16_ss(dO, desc_add(qd, (uint32_t)((ks >> 2) * C::BOX + (ks & 3) * 32)),
                                    desc_add(sd, ks * 2048), C::ID_QKV, 1u);
                }
                __syncwarp();
            }
            if (lane == 0) {
                mma_commit(&m->o_full[b & 1]);
                mma_commit(&m->empty[st]);
            }
            __syncwarp();
        }
        if (!ok) fail();
        if (nb > 0 && lane == 0) {  // every issued MMA has finished before TMEM is freed
            mma_commit(&m->drain);
            mbar_wait(&m->drain, 0u, nullptr, tlimit);
        }
        __syncwarp();
    } else if (warp < 6) {
        // ------------------------------------------------------------ group P
        // S_b and P_b share a TMEM buffer: chunk cc reads S columns [64cc, 64cc+64)
        // and writes P columns [32cc, 32cc+32), which lie in S columns already read.
        // Issuer A issues S_{b+2} into the buffer only after it has seen O_b = P_b V_b
        // (issuer B) complete.
        const int q = warp & 3;                    // TMEM lane quadrant of this warp
        const uint32_t lane_base = (uint32_t)(32 * q) << 16;
        const int r = BETA == 128 ? 32 * q + lane : 16 * q + lane;   // query row in the block
        bool ok = true;
        for (int b = 0; b < nb; ++b) {
            if (!wwait(&m->s_full[b & 1], (uint32_t)((b >> 1) & 1))) {
                ok = false;
                break;
            }
            tc_fence_after();
            const uint32_t tS = tmem + C::TM_S + BETA * (b & 1) + lane_base;
#pragma unroll 1
            for (int cc = 0; cc < BETA / 64; ++cc) {
                uint32_t s0[32], s1[32], w[32];
                tmem_ld32(tS + 64 * cc, s0);
                tmem_ld32(tS + 64 * cc + 32, s1);
                tmem_ld_wait();
#pragma unroll
                for (int u = 0; u < 32; ++u) {
                    const uint32_t *s = u < 16 ? &s0[2 * u] : &s1[2 * (u - 16)];
                    const int c0 = 64 * cc + 2 * u;
                    const float x0 = c0 <= r ? __uint_as_float(s[0]) : 0.f;
                    const float x1 = c0 + 1 <= r ? __uint_as_float(s[1]) : 0.f;
                    w[u] = pack_bf16x2(x0, x1);
                }
                tmem_st32(tS + 32 * cc, w);
            }
            tmem_st_wait();
            tc_fence_before();
            mbar_arrive(&m->p_ready[b & 1]);
        }
        if (!ok) fail();
    } else if (warp < 10) {
        // ------------------------------------------------------------ group O
        const int q = warp & 3;
        const uint32_t lane_base = (uint32_t)(32 * q) << 16;
        const int r = BETA == 128 ? 32 * q + lane : 16 * q + lane;   // query row in the block
        const bool r_ok = BETA == 128 || lane < 16;
        const size_t o_col = (size_t)h * D + 64 * vs;
        bool ok = true;
        auto write_o = [&](int j) -> bool {  // read O_j out of TMEM, normalise, store
            if (!wwait(&m->o_full[j & 1], (uint32_t)((j >> 1) & 1))) return false;
            tc_fence_after();
            uint32_t a[32], c[32];
            const uint32_t tO = tmem + C::TM_O + 64 * (j & 1) + lane_base;
            tmem_ld32(tO, a);
            tmem_ld32(tO + 32, c);
            tmem_ld_wait();
            tc_fence_before();
            mbar_arrive(&m->o_free[j & 1]);
            float scale = 1.0f;
            if (p.rmsnorm) {
                float ss = 0.f;
#pragma unroll
                for (int t = 0; t < 32; ++t) {
                    const float x = __uint_as_float(a[t]), y = __uint_as_float(c[t]);
                    ss = fmaf(x, x, ss);
                    ss = fmaf(y, y, ss);
                }
                if constexpr (C::NVS > 1) {
                    if (r_ok) st_remote_f32(&m->ss_in[j & 1][r], partner, ss);
                    mbar_arrive_remote(&m->ss_full[j & 1], partner);
                    if (!__all_sync(0xffffffffu,
                                    mbar_wait<true>(&m->ss_full[j & 1], (uint32_t)((j >> 1) & 1),
                                                    abort_flag, tlimit)))
                        return false;
                    if (r_ok) ss = ss + m->ss_in[j & 1][r];
                }
                scale = rsqrtf(ss * (1.0f / D) + 1e-6f);
            }
            const int nv = min(BETA, seq_len - j * BETA);
            if (r_ok && r < nv) {
                uint4 *dst = reinterpret_cast<uint4 *>(
                    p.o + ((size_t)(seq_start + j * BETA + r) * p.H) * D + o_col);
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
            return true;
        };

        for (int b = 0; ok && b < nb; ++b) ok = write_o(b);
        if (!ok) fail();
    } else if (warp < C::WARP_B) {
        // ------------------------------------------------------------ group KV
        const int q = warp & 3;
        const uint32_t lane_base = (uint32_t)(32 * q) << 16;
        const int i = D == 128 ? 32 * q + lane : 16 * q + lane;      // state row
        const bool i_ok = D == 128 || lane < 16;
        float kv[64];                                              // KV[i][64 vs .. 64 vs + 63]
#pragma unroll
        for (int t = 0; t < 64; ++t) kv[t] = 0.f;
        bool ok = true;
        // snapshot u of KV into buffer u % 2 (bf16, 128-byte swizzled rows), then signal it
        auto write_snap = [&](int u) {
            const uint32_t sSnap = sbase + C::OFF_SNAP + C::SNAP_BYTES * (u & 1);
            if (i_ok) {
#pragma unroll
                for (int t = 0; t < 8; ++t) {
                    const uint32_t chunk = (uint32_t)(t ^ (i & 7));
                    st_shared_v4(sSnap + i * 128 + (chunk << 4), pack_bf16x2(kv[8 * t + 0], kv[8 * t + 1]),
                                 pack_bf16x2(kv[8 * t + 2], kv[8 * t + 3]),
                                 pack_bf16x2(kv[8 * t + 4], kv[8 * t + 5]),
                                 pack_bf16x2(kv[8 * t + 6], kv[8 * t + 7]));
                }
            }
            fence_proxy_async_smem();
            mbar_arrive(&m->snap_ready[u & 1]);
        };
        if (p.state_in != nullptr) {  // KV starts at the sequence's initial state
            if (i_ok) {
                const float4 *src = reinterpret_cast<const float4 *>(
                    p.state_in + (((size_t)sid * p.H + h) * D + i) * D + 64 * vs);
#pragma unroll
                for (int t = 0; t < 16; ++t) {
                    const float4 x = src[t];
                    kv[4 * t] = x.x;
                    kv[4 * t + 1] = x.y;
                    kv[4 * t + 2] = x.z;
                    kv[4 * t + 3] = x.w;
                }
            }
            write_snap(0);
        }

        for (int b = 0; b < nb; ++b) {
            // KV += dKV_b; the bf16 snapshot of KV_{<b+1} for O_{b+1} += Q_{b+1} KV.
            // dkv_full[b % 2] phase b / 2; its next phase (dKV_{b+2}) needs dkv_free below
            if (!wwait(&m->dkv_full[b & 1], (uint32_t)((b >> 1) & 1))) {
                ok = false;
                break;
            }
            tc_fence_after();
            {
                // one 32-column half at a time, to keep the state and one load in registers
                uint32_t a[32];
                const uint32_t tK = tmem + C::TM_DKV + 64 * (b & 1) + lane_base;
                tmem_ld32(tK, a);
                tmem_ld_wait();
#pragma unroll
                for (int t = 0; t < 32; ++t) kv[t] += __uint_as_float(a[t]);
                tmem_ld32(tK + 32, a);
                tmem_ld_wait();
                tc_fence_before();
                mbar_arrive(&m->dkv_free[b & 1]);
#pragma unroll
                for (int t = 0; t < 32; ++t) kv[32 + t] += __uint_as_float(a[t]);
            }
            if (b + 1 < nb) {
                // Buffer (b+1)&1 was last read by O_{b-1} += Q_{b-1} KV, which finished
                // before dKV_b (MMAs complete in issue order), so it is free here.
                write_snap(b + 1);
            }
        }
        if (ok && p.state != nullptr && i_ok) {  // final state K^T V of the sequence, fp32
            float4 *dst = reinterpret_cast<float4 *>(p.state + (((size_t)sid * p.H + h) * D + i) * D +
                                                     64 * vs);
#pragma unroll
            for (int t = 0; t < 16; ++t)
                dst[t] = make_float4(kv[4 * t], kv[4 * t + 1], kv[4 * t + 2], kv[4 * t + 3]);
        }
        if (!ok) fail();
    }

    tc_fence_before();
    __syncthreads();
    if constexpr (C::NVS > 1) cluster_sync_all();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, C::TMEM_COLS);
    }
}

}  // namespace la
