// liblightning.so: the C ABI declared in include/lightning_attention.h.
//
// Host side only: argument validation, the sequence table, TMA tensor maps and
// kernel launches.  Every step of the computation runs in the kernels of
// prefill_pair.cuh and prefill_tc.cuh (bf16, tcgen05), prefill_simt.cuh (fp32),
// chunk_state.cuh and decode.cuh.
#include <algorithm>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <numeric>
#include <vector>

#include "chunk_state.cuh"
#include "decode.cuh"
#include "prefill_simt.cuh"
#include "prefill_pair.cuh"
#include "prefill_tc.cuh"
#include "selftest.cuh"

namespace {

using la::PrefillTcParams;
using la::SeqTable;

constexpr unsigned long long kWaitLimitNs = 1000ull * 1000ull * 1000ull;  // 1 s per wait

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// cuTensorMapEncodeTiled, fetched through the runtime so that the library does
// not link libcuda directly.
using EncodeTiledFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                   const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                   const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

// [T][H*D] bf16 viewed as a 2-D tensor; boxes of 64 columns x beta rows, 128-B swizzle.
bool make_map(CUtensorMap *map, const void *base, long long T, int H, int D, int beta) {
    EncodeTiledFn fn = encode_fn();
    if (fn == nullptr) return false;
    cuuint64_t dims[2] = {(cuuint64_t)H * D, (cuuint64_t)T};
    cuuint64_t strides[1] = {(cuuint64_t)H * D * 2};
    cuuint32_t box[2] = {64, (cuuint32_t)beta};
    cuuint32_t estr[2] = {1, 1};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides,
              box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
           CUDA_SUCCESS;
}

// The sequence table of a call: B equal sequences of N tokens, or the packed
// boundaries cu_seqlens (host array, validated here), ordered longest first so
// that the block scheduler starts the longest chains first.
la_status build_seq_table(int B, int N, const int32_t *cu_seqlens, int num_seqs, SeqTable &seqs,
                          long long &T, int &S) {
    std::memset(&seqs, 0, sizeof seqs);
    T = 0;
    S = 0;
    if (cu_seqlens != nullptr) {
        if (B != 1) return LA_ERR_INVALID_ARG;
        if (num_seqs < 1) return LA_ERR_INVALID_ARG;
        if (num_seqs > LA_MAX_VARLEN_SEQS) return LA_ERR_UNSUPPORTED;
        if (cu_seqlens[0] != 0 || cu_seqlens[num_seqs] != N) return LA_ERR_INVALID_ARG;
        for (int s = 0; s < num_seqs; ++s)
            if (cu_seqlens[s + 1] < cu_seqlens[s]) return LA_ERR_INVALID_ARG;
        S = num_seqs;
        T = N;
        std::vector<int> order(S);
        std::iota(order.begin(), order.end(), 0);
        std::stable_sort(order.begin(), order.end(), [&](int a, int b) {
            return cu_seqlens[a + 1] - cu_seqlens[a] > cu_seqlens[b + 1] - cu_seqlens[b];
        });
        seqs.varlen = 1;
        for (int r = 0; r < S; ++r) {
            const int s = order[r];
            seqs.seq_start[r] = cu_seqlens[s];
            seqs.seq_len[r] = cu_seqlens[s + 1] - cu_seqlens[s];
            seqs.seq_id[r] = s;
        }
    } else {
        S = B;
        T = (long long)B * N;
        seqs.varlen = 0;
        seqs.N = N;
    }
    return LA_OK;
}

template <int BETA, int D>
la_status launch_tc(const PrefillTcParams &p, int units, cudaStream_t stream) {
    using C = la::TcCfg<BETA, D>;
    auto kern = la::prefill_tc_kernel<BETA, D>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES) !=
        cudaSuccess)
        return LA_ERR_CUDA;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)units);
    cfg.blockDim = dim3(C::THREADS);
    cfg.dynamicSmemBytes = C::SMEM_BYTES;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = C::NVS;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, p) == cudaSuccess ? LA_OK : LA_ERR_CUDA;
}

la_status launch_pair(const la::PrefillPairParams &p, int pairs, cudaStream_t stream) {
    using C = la::PairCfg;
    auto kern = la::prefill_pair_kernel;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES) !=
        cudaSuccess)
        return LA_ERR_CUDA;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(2 * pairs));
    cfg.blockDim = dim3(C::THREADS);
    cfg.dynamicSmemBytes = C::SMEM_BYTES;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, p) == cudaSuccess ? LA_OK : LA_ERR_CUDA;
}

template <int BETA, int D>
la_status launch_simt(const float *q, const float *k, const float *v, float *o, float *state,
                      const float *state_in, int H, int rmsnorm, const SeqTable &seqs, int S,
                      cudaStream_t stream) {
    using C = la::SimtCfg<BETA, D>;
    auto kern = la::prefill_simt_kernel<BETA, D>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES) !=
        cudaSuccess)
        return LA_ERR_CUDA;
    kern<<<S * H, C::THREADS, C::SMEM_BYTES, stream>>>(q, k, v, o, state, state_in, H, rmsnorm, seqs);
    return cudaGetLastError() == cudaSuccess ? LA_OK : LA_ERR_CUDA;
}

}  // namespace

extern "C" {

const char *la_status_string(la_status s) {
    switch (s) {
        case LA_OK: return "LA_OK";
        case LA_ERR_INVALID_ARG: return "LA_ERR_INVALID_ARG";
        case LA_ERR_UNSUPPORTED: return "LA_ERR_UNSUPPORTED";
        case LA_ERR_CUDA: return "LA_ERR_CUDA";
        case LA_ERR_DEVICE_TIMEOUT: return "LA_ERR_DEVICE_TIMEOUT";
        case LA_ERR_DEVICE_RANGE: return "LA_ERR_DEVICE_RANGE";
    }
    return "LA_ERR_UNKNOWN";
}

int la_version(void) { return 100; }

la_status la_prefill(const void *q, const void *k, const void *v, void *o, int B, int H, int N,
                     int D, int beta, const int32_t *cu_seqlens, int num_seqs, unsigned flags,
                     float *state_ws, void *stream_) {
    cudaStream_t stream = static_cast<cudaStream_t>(stream_);
    const unsigned known = LA_BF16 | LA_OUT_RMSNORM | LA_WRITE_STATE | LA_READ_STATE;
    if (flags & ~known) return LA_ERR_INVALID_ARG;
    if (H < 1 || N < 0 || B < 1) return LA_ERR_INVALID_ARG;
    // with no tokens (N == 0) the data pointers are never used and may be NULL
    if (N > 0 && (!q || !k || !v || !o)) return LA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o)) return LA_ERR_INVALID_ARG;
    const bool want_state = (flags & LA_WRITE_STATE) != 0;
    const bool read_state = (flags & LA_READ_STATE) != 0;
    if ((want_state || read_state) && (state_ws == nullptr || !aligned16(state_ws)))
        return LA_ERR_INVALID_ARG;
    if (D != 64 && D != 128) return LA_ERR_UNSUPPORTED;
    if (beta != 64 && beta != 128) return LA_ERR_UNSUPPORTED;

    // Sequence table (host-validated).
    SeqTable seqs;
    long long T = 0;
    int S = 0;
    if (la_status st = build_seq_table(B, N, cu_seqlens, num_seqs, seqs, T, S); st != LA_OK)
        return st;
    if (T >= (1ll << 31) || (long long)S * H * 2 >= (1ll << 31)) return LA_ERR_UNSUPPORTED;
    if (S == 0 || H == 0) return LA_OK;

    const int rms = (flags & LA_OUT_RMSNORM) ? 1 : 0;
    float *state = want_state ? state_ws : nullptr;
    const float *state_in = read_state ? state_ws : nullptr;
    if (T == 0) {
        // Every sequence is empty: its final state is its initial state, already in
        // place with LA_READ_STATE, else zero.
        if (want_state && !read_state) {
            la::state_zero_kernel<<<(unsigned)(S * H), 256, 0, stream>>>(
                reinterpret_cast<float4 *>(state_ws), D * D / 4);
            return cudaGetLastError() == cudaSuccess ? LA_OK : LA_ERR_CUDA;
        }
        return LA_OK;
    }

    if (flags & LA_BF16) {
        // Sequences of one token are decode steps: they go to the decode kernel (reading
        // their rows of the packed arrays in place), the rest to the prefill kernel.  A
        // one-token sequence would otherwise hold a whole prefill CTA (pair) for one row.
        la::OneTokenTable ot;
        ot.identity = 0;
        int n1 = 0;
        if (seqs.varlen) {
            int w = 0;
            for (int r = 0; r < S; ++r) {
                if (seqs.seq_len[r] == 1) {
                    ot.row[n1] = seqs.seq_start[r];
                    ot.sid[n1] = seqs.seq_id[r];
                    ++n1;
                } else {
                    seqs.seq_start[w] = seqs.seq_start[r];
                    seqs.seq_len[w] = seqs.seq_len[r];
                    seqs.seq_id[w] = seqs.seq_id[r];
                    ++w;
                }
            }
            S = w;
        } else if (N == 1) {
            ot.identity = 1;
            n1 = S;
            S = 0;
        }
        if (n1 > 0) {
            using bf = __nv_bfloat16;
            const bf *qb = static_cast<const bf *>(q), *kb = static_cast<const bf *>(k),
                     *vb = static_cast<const bf *>(v);
            bf *ob = static_cast<bf *>(o);
            float *ws = (want_state || read_state) ? state_ws : nullptr;
            if (D == 128)
                la::decode_rows_kernel<128, bf><<<(unsigned)(n1 * H), 256, 0, stream>>>(
                    qb, kb, vb, ob, ws, H, read_state ? 1 : 0, want_state ? 1 : 0, rms, ot);
            else
                la::decode_rows_kernel<64, bf><<<(unsigned)(n1 * H), 256, 0, stream>>>(
                    qb, kb, vb, ob, ws, H, read_state ? 1 : 0, want_state ? 1 : 0, rms, ot);
            if (cudaGetLastError() != cudaSuccess) return LA_ERR_CUDA;
        }
        if (S == 0) return LA_OK;
        const long long Tm = T;
        if (beta == 128 && D == 128) {
            // paired-CTA kernel: each CTA of a pair loads half of the rows / columns
            la::PrefillPairParams pp;
            std::memset(&pp, 0, sizeof pp);
            if (!make_map(&pp.tmap_q64, q, Tm, H, D, 64) || !make_map(&pp.tmap_k64, k, Tm, H, D, 64) ||
                !make_map(&pp.tmap_k128, k, Tm, H, D, 128) || !make_map(&pp.tmap_v128, v, Tm, H, D, 128) ||
                !make_map(&pp.tmap_o32, o, Tm, H, D, 32))
                return LA_ERR_CUDA;
            pp.o = static_cast<__nv_bfloat16 *>(o);
            pp.state = state;
            pp.state_in = state_in;
            pp.H = H;
            pp.rmsnorm = rms;
            pp.timeout_ns = kWaitLimitNs;
            pp.seqs = seqs;
            return launch_pair(pp, S * H, stream);
        }
        PrefillTcParams p;
        std::memset(&p, 0, sizeof p);
        if (!make_map(&p.tmap_q, q, Tm, H, D, beta) || !make_map(&p.tmap_k, k, Tm, H, D, beta) ||
            !make_map(&p.tmap_v, v, Tm, H, D, beta))
            return LA_ERR_CUDA;
        p.o = static_cast<__nv_bfloat16 *>(o);
        p.state = state;
        p.state_in = state_in;
        p.H = H;
        p.rmsnorm = rms;
        p.timeout_ns = kWaitLimitNs;
        p.seqs = seqs;
        const int units = S * H * (D / 64);
        if (beta == 64 && D == 128) return launch_tc<64, 128>(p, units, stream);
        if (beta == 128 && D == 64) return launch_tc<128, 64>(p, units, stream);
        return launch_tc<64, 64>(p, units, stream);
    }
    const float *qf = static_cast<const float *>(q), *kf = static_cast<const float *>(k),
                *vf = static_cast<const float *>(v);
    float *of = static_cast<float *>(o);
    if (beta == 128 && D == 128) return launch_simt<128, 128>(qf, kf, vf, of, state, state_in, H, rms, seqs, S, stream);
    if (beta == 64 && D == 128) return launch_simt<64, 128>(qf, kf, vf, of, state, state_in, H, rms, seqs, S, stream);
    if (beta == 128 && D == 64) return launch_simt<128, 64>(qf, kf, vf, of, state, state_in, H, rms, seqs, S, stream);
    return launch_simt<64, 64>(qf, kf, vf, of, state, state_in, H, rms, seqs, S, stream);
}

la_status la_chunk_state(const void *k, const void *v, int B, int H, int N, int D,
                         const int32_t *cu_seqlens, int num_seqs, unsigned flags, float *state_out,
                         void *stream_) {
    cudaStream_t stream = static_cast<cudaStream_t>(stream_);
    if (flags & ~(unsigned)LA_BF16) return LA_ERR_INVALID_ARG;
    if (H < 1 || N < 0 || B < 1) return LA_ERR_INVALID_ARG;
    if (N > 0 && (!k || !v)) return LA_ERR_INVALID_ARG;
    if (!state_out) return LA_ERR_INVALID_ARG;
    if (!aligned16(k) || !aligned16(v) || !aligned16(state_out)) return LA_ERR_INVALID_ARG;
    if (D != 64 && D != 128) return LA_ERR_UNSUPPORTED;
    SeqTable seqs;
    long long T = 0;
    int S = 0;
    if (la_status st = build_seq_table(B, N, cu_seqlens, num_seqs, seqs, T, S); st != LA_OK)
        return st;
    if (T >= (1ll << 31) || (long long)S * H * 2 >= (1ll << 31)) return LA_ERR_UNSUPPORTED;
    if (S == 0) return LA_OK;
    if (T == 0) {  // every sequence is empty: zero states
        la::state_zero_kernel<<<(unsigned)(S * H), 256, 0, stream>>>(
            reinterpret_cast<float4 *>(state_out), D * D / 4);
        return cudaGetLastError() == cudaSuccess ? LA_OK : LA_ERR_CUDA;
    }
    if (flags & LA_BF16) {
        la::ChunkStateParams p;
        std::memset(&p, 0, sizeof p);
        if (!make_map(&p.tmap_k, k, T, H, D, 128) || !make_map(&p.tmap_v, v, T, H, D, 128))
            return LA_ERR_CUDA;
        p.state = state_out;
        p.H = H;
        p.timeout_ns = kWaitLimitNs;
        p.seqs = seqs;
        auto launch = [&](auto kern, int smem, int threads, int nvs) -> la_status {
            if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) !=
                cudaSuccess)
                return LA_ERR_CUDA;
            kern<<<(unsigned)(S * H * nvs), threads, smem, stream>>>(p);
            return cudaGetLastError() == cudaSuccess ? LA_OK : LA_ERR_CUDA;
        };
        if (D == 128)
            return launch(la::chunk_state_tc_kernel<128>, la::ChunkCfg<128>::SMEM_BYTES,
                          la::ChunkCfg<128>::THREADS, la::ChunkCfg<128>::NVS);
        return launch(la::chunk_state_tc_kernel<64>, la::ChunkCfg<64>::SMEM_BYTES,
                      la::ChunkCfg<64>::THREADS, la::ChunkCfg<64>::NVS);
    }
    const float *kf = static_cast<const float *>(k), *vf = static_cast<const float *>(v);
    auto launch_simt_state = [&](auto kern, int Dv) -> la_status {
        const int smem = (2 * 64 * Dv + Dv * Dv) * 4;
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
            return LA_ERR_CUDA;
        kern<<<(unsigned)(S * H), 256, smem, stream>>>(kf, vf, state_out, H, seqs);
        return cudaGetLastError() == cudaSuccess ? LA_OK : LA_ERR_CUDA;
    };
    if (D == 128) return launch_simt_state(la::chunk_state_simt_kernel<128>, 128);
    return launch_simt_state(la::chunk_state_simt_kernel<64>, 64);
}

la_status la_state_prefix(const float *gathered, int R, int rank, int S, int H, int D, float *out,
                          void *stream_) {
    cudaStream_t stream = static_cast<cudaStream_t>(stream_);
    if (R < 1 || rank < 0 || rank > R || S < 0 || H < 1) return LA_ERR_INVALID_ARG;
    if (!gathered || !out || !aligned16(gathered) || !aligned16(out)) return LA_ERR_INVALID_ARG;
    if (D != 64 && D != 128) return LA_ERR_UNSUPPORTED;
    if ((long long)S * H >= (1ll << 31)) return LA_ERR_UNSUPPORTED;
    if (S == 0) return LA_OK;
    const int n4 = D * D / 4;
    la::state_prefix_kernel<<<(unsigned)(S * H), 256, 0, stream>>>(
        reinterpret_cast<const float4 *>(gathered), reinterpret_cast<float4 *>(out), rank,
        (size_t)S * H * n4, n4);
    return cudaGetLastError() == cudaSuccess ? LA_OK : LA_ERR_CUDA;
}

la_status la_selftest_wait(unsigned long long limit_ns, void *stream_) {
    cudaStream_t stream = static_cast<cudaStream_t>(stream_);
    if (limit_ns < 1000ull) limit_ns = 1000ull;
    if (limit_ns > kWaitLimitNs) limit_ns = kWaitLimitNs;
    la::selftest_wait_kernel<<<1, 32, 0, stream>>>(limit_ns);
    return cudaGetLastError() == cudaSuccess ? LA_OK : LA_ERR_CUDA;
}

la_status la_decode_step(const void *q, const void *k, const void *v, float *state, void *o, int B,
                         int H, int D, unsigned flags, void *stream_) {
    cudaStream_t stream = static_cast<cudaStream_t>(stream_);
    const unsigned known = LA_BF16 | LA_OUT_RMSNORM;
    if (flags & ~known) return LA_ERR_INVALID_ARG;
    if (B < 0 || H < 1) return LA_ERR_INVALID_ARG;
    if (!q || !k || !v || !o || !state) return LA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(state))
        return LA_ERR_INVALID_ARG;
    if (D != 64 && D != 128) return LA_ERR_UNSUPPORTED;
    if ((long long)B * H >= (1ll << 31)) return LA_ERR_UNSUPPORTED;
    if (B == 0) return LA_OK;
    const int rms = (flags & LA_OUT_RMSNORM) ? 1 : 0;
    const unsigned grid = (unsigned)(B * H);
    if (flags & LA_BF16) {
        using T = __nv_bfloat16;
        if (D == 128)
            la::decode_step_kernel<128, T><<<grid, 256, 0, stream>>>(
                (const T *)q, (const T *)k, (const T *)v, state, (T *)o, rms);
        else
            la::decode_step_kernel<64, T><<<grid, 256, 0, stream>>>(
                (const T *)q, (const T *)k, (const T *)v, state, (T *)o, rms);
    } else {
        if (D == 128)
            la::decode_step_kernel<128, float><<<grid, 256, 0, stream>>>(
                (const float *)q, (const float *)k, (const float *)v, state, (float *)o, rms);
        else
            la::decode_step_kernel<64, float><<<grid, 256, 0, stream>>>(
                (const float *)q, (const float *)k, (const float *)v, state, (float *)o, rms);
    }
    return cudaGetLastError() == cudaSuccess ? LA_OK : LA_ERR_CUDA;
}

la_status la_state_out(const float *state_ws, float *state_dst, int S, int H, int D,
                       const int32_t *seq_to_slot, int num_slots, void *stream_) {
    cudaStream_t stream = static_cast<cudaStream_t>(stream_);
    if (S < 0 || H < 1 || num_slots < 0) return LA_ERR_INVALID_ARG;
    if (!state_ws || !state_dst) return LA_ERR_INVALID_ARG;
    if (!aligned16(state_ws) || !aligned16(state_dst)) return LA_ERR_INVALID_ARG;
    if (D != 64 && D != 128) return LA_ERR_UNSUPPORTED;
    if (seq_to_slot == nullptr && S > num_slots) return LA_ERR_INVALID_ARG;
    if ((long long)S * H >= (1ll << 31)) return LA_ERR_UNSUPPORTED;
    if (S == 0) return LA_OK;
    la::state_copy_kernel<<<(unsigned)(S * H), 256, 0, stream>>>(
        reinterpret_cast<const float4 *>(state_ws), reinterpret_cast<float4 *>(state_dst),
        seq_to_slot, H, D * D / 4, num_slots);
    return cudaGetLastError() == cudaSuccess ? LA_OK : LA_ERR_CUDA;
}

la_status la_get_device_status(void *stream_) {
    cudaStream_t stream = static_cast<cudaStream_t>(stream_);
    if (cudaStreamSynchronize(stream) != cudaSuccess) return LA_ERR_CUDA;
    unsigned int word = 0, zero = 0;
    if (cudaMemcpyFromSymbol(&word, la::g_device_status, sizeof word) != cudaSuccess)
        return LA_ERR_CUDA;
    if (word != 0 && cudaMemcpyToSymbol(la::g_device_status, &zero, sizeof zero) != cudaSuccess)
        return LA_ERR_CUDA;
    if (word == la::DEV_TIMEOUT) return LA_ERR_DEVICE_TIMEOUT;
    if (word == la::DEV_RANGE) return LA_ERR_DEVICE_RANGE;
    return LA_OK;
}

}  // extern "C"
