/*
 * lightning_attention.h -- C ABI of the B200 (sm_100a) lightning-attention
 * library (liblightning.so).
 *
 * The method (MiniMax-01, "Scaling Foundation Models with Lightning
 * Attention"; CSDN digest section 2.1 and mizuki blog appendix "key concepts"):
 * causal linear attention in the NormAttention style, evaluated with the
 * right-product kernel trick and tiled into blocks of beta tokens.  Per packed
 * sequence s, head h, and block b of s:
 *
 *     O_b  = [(Q_b K_b^T) (.) M] V_b  +  Q_b KV          (M: causal, j <= i)
 *     KV  += K_b^T V_b                                   (KV = 0 at the start of s)
 *     y    = O / sqrt(mean_d O_d^2 + 1e-6)               (only with LA_OUT_RMSNORM)
 *
 * which equals O_i = sum_{j <= i in s} (q_i . k_j) v_j exactly in real
 * arithmetic.  Decode (jvyan.cn article, section 2 "compute optimisation":
 * length-1 and length>1 requests run as two kernels on two CUDA streams) is one
 * token per sequence: KV <- KV + k v^T, then o = q^T KV.
 *
 * Conventions for every entry point:
 *   - Layout: q, k, v, o are row-major [T][H][D] (T = B*N, or the packed total);
 *     states are row-major [S][H][D][D] fp32 with state[s][h][i][j] =
 *     sum_t k_t[i] v_t[j].
 *   - Device pointers unless stated otherwise.  The caller owns every buffer;
 *     the library allocates no device memory.
 *   - Work is enqueued on `stream` (a cudaStream_t; NULL = legacy default
 *     stream) and runs asynchronously.  No entry point synchronises except
 *     la_get_device_status.
 *   - Arguments are validated on the host before anything is launched; an
 *     invalid call returns LA_ERR_INVALID_ARG or LA_ERR_UNSUPPORTED and touches
 *     no memory.  Errors reported by the CUDA runtime at launch return
 *     LA_ERR_CUDA.  There is no fallback path: an unsupported shape is an
 *     error, never a slower kernel.
 *   - Faults found on the device (a wait that ran past its time limit, an
 *     out-of-range slot index) are recorded in a per-device status word and
 *     reported by la_get_device_status.
 *   - Device buffers must be 16-byte aligned; q, k, v, o of one call must not
 *     overlap o.
 */
#ifndef LIGHTNING_ATTENTION_H
#define LIGHTNING_ATTENTION_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    LA_OK = 0,
    LA_ERR_INVALID_ARG = 1,     /* null pointer, bad size, bad cu_seqlens, misaligned */
    LA_ERR_UNSUPPORTED = 2,     /* valid but not built: D or beta outside {64, 128}, ... */
    LA_ERR_CUDA = 3,            /* the CUDA runtime refused a launch or a query */
    LA_ERR_DEVICE_TIMEOUT = 4,  /* a kernel gave up waiting (see la_get_device_status) */
    LA_ERR_DEVICE_RANGE = 5     /* a kernel met an out-of-range index and skipped it */
} la_status;

/* Flags (bitwise OR). */
enum {
    LA_FP32 = 0,         /* q, k, v, o are fp32; CUDA-core arithmetic, fp64 accumulation */
    LA_BF16 = 1,         /* q, k, v, o are bf16; tensor-core bf16 products, fp32 accumulate */
    LA_OUT_RMSNORM = 2,  /* per-token, per-head RMSNorm over D of the output (eps 1e-6, unit weight) */
    LA_WRITE_STATE = 4,  /* la_prefill writes each sequence's final KV state to state_ws */
    LA_READ_STATE = 8    /* la_prefill starts each sequence from the KV state in state_ws */
};

/* Largest number of packed sequences one la_prefill call accepts. */
#define LA_MAX_VARLEN_SEQS 1024

/*
 * la_prefill -- causal lightning attention over a batch of sequences
 * (length > 1 path).
 *
 *   q, k, v   [T][H][D] inputs (bf16 with LA_BF16, fp32 otherwise), T = B*N.
 *   o         [T][H][D] output, same dtype.  Every row of every sequence is written.
 *             q, k, v and o may be NULL when there are no tokens (N == 0).
 *   B, N      without cu_seqlens: B sequences of N tokens each (B >= 1, N >= 0).
 *             With cu_seqlens: B must be 1 and N is the packed total T.
 *   H, D      heads (>= 1) and head dim; D in {64, 128}.
 *   beta      block size of the tiling, 64 or 128.  The result does not depend on
 *             beta beyond rounding.
 *   cu_seqlens HOST array of num_seqs+1 int32 entries, non-decreasing from 0 to N
 *             (data packing: sequences concatenated along the token axis, CSDN
 *             digest section 3.2).  The state is reset at every boundary;
 *             zero-length sequences are allowed.  NULL = B equal sequences.
 *             The array is read during the call only.  It is a host array on
 *             purpose, not a device one: the library validates it before the
 *             launch and passes the (longest-first) sequence table in the kernel
 *             parameters, so a call needs no device scratch and no synchronisation.
 *   num_seqs  entries of cu_seqlens minus one (1 .. LA_MAX_VARLEN_SEQS); ignored
 *             when cu_seqlens is NULL.
 *   flags     LA_BF16 or LA_FP32, optionally | LA_OUT_RMSNORM | LA_WRITE_STATE
 *             | LA_READ_STATE.
 *   state_ws  [S][H][D][D] fp32 (S = num_seqs or B), used when either state flag
 *             is set, otherwise ignored (may be NULL).
 *             LA_READ_STATE: on entry it holds each sequence's initial state X_s,
 *             and the sequence continues from it (chunked prefill, resume, and the
 *             per-chunk step of LASP+, mizuki blog section 5 and appendix "key
 *             concepts"): O_i = q_i^T X_s + sum_{j <= i in s} (q_i . k_j) v_j.
 *             Without it every sequence starts from 0.
 *             LA_WRITE_STATE: on exit it holds each sequence's final state,
 *             X_s + K_s^T V_s (X_s = 0 without LA_READ_STATE).  With both flags the
 *             update is in place: each (sequence, head) slice is read before it is
 *             overwritten, by the same threads.
 *   stream    cudaStream_t for the launch.
 *
 * With LA_BF16, the sequences of exactly one token are one decode step each (the
 * arithmetic of la_decode_step, from X_s or from 0): the call launches the decode
 * kernel for them, reading and writing their rows of q, k, v, o and their state
 * slices in place, and the prefill kernel for the other sequences, both on
 * `stream`.  (A mixed batch of one-token requests and longer chunks, jvyan.cn
 * article section 2, then needs one call and no gather.)
 *
 * Returns LA_OK once the work is enqueued.
 */
la_status la_prefill(const void *q, const void *k, const void *v, void *o,
                     int B, int H, int N, int D, int beta,
                     const int32_t *cu_seqlens, int num_seqs,
                     unsigned flags, float *state_ws, void *stream);

/*
 * la_chunk_state -- each sequence's state K_s^T V_s alone, without the attention
 * output: the local state of one chunk in LASP+, the sequence-parallel scheme the
 * pages name for lightning attention (mizuki blog, section 5 "pretraining" and
 * appendix "key concepts": local prefix sums of the chunk states, an all-gather,
 * then each chunk runs from the sum of the states before it).
 *
 *   k, v      [T][H][D] (bf16 with LA_BF16, else fp32), T = B*N; may be NULL when
 *             N == 0.
 *   B, N, H, D, cu_seqlens, num_seqs
 *             as for la_prefill (D in {64, 128}).
 *   flags     LA_BF16 or LA_FP32; no other bit.
 *   state_out [S][H][D][D] fp32: state_out[s][h][i][j] = sum_{t in s} k_t[i] v_t[j]
 *             (0 for an empty sequence).  Written, never read.
 *   stream    cudaStream_t for the launch.
 */
la_status la_chunk_state(const void *k, const void *v, int B, int H, int N, int D,
                         const int32_t *cu_seqlens, int num_seqs, unsigned flags,
                         float *state_out, void *stream);

/*
 * la_state_prefix -- the initial state of chunk `rank` in LASP+, from the chunk
 * states of all R ranks (as an all-gather lays them out):
 *     out[s][h] = sum_{r < rank} gathered[r][s][h]      (0 for rank 0),
 * summed in fp32 in ascending r, so every rank adds in the same order.
 *
 *   gathered  [R][S][H][D][D] fp32, rank-major.
 *   R         number of chunks (>= 1); rank in 0 .. R (rank = R gives the state
 *             after the whole sequence).
 *   out       [S][H][D][D] fp32; must not overlap gathered.
 */
la_status la_state_prefix(const float *gathered, int R, int rank, int S, int H, int D,
                          float *out, void *stream);

/*
 * la_selftest_wait -- exercise the device-side failure path.  Launches one small
 * kernel whose single wait (on a barrier that nothing completes) gives up after
 * limit_ns nanoseconds (clamped to 1 us .. 1 s), records LA_ERR_DEVICE_TIMEOUT in
 * the device status word and returns; nothing else is in flight.  The next
 * la_get_device_status on the stream reports LA_ERR_DEVICE_TIMEOUT and clears it;
 * the context stays usable.  This is not part of the method (the pages describe no
 * failure handling); it exists so that tests can check that bounded waits surface
 * as errors instead of hangs.
 */
la_status la_selftest_wait(unsigned long long limit_ns, void *stream);

/*
 * la_decode_step -- one token per sequence (length-1 path).
 *
 *   q, k, v   [B][H][D] the new token's projections (bf16 with LA_BF16, else fp32).
 *   state     [B][H][D][D] fp32, updated in place: KV <- KV + k v^T.
 *   o         [B][H][D] output o = q^T KV (after the update), optionally RMSNorm'ed
 *             with LA_OUT_RMSNORM; same dtype as q.
 *   B >= 0, H >= 1, D in {64, 128}.  B = 0 is a no-op.
 */
la_status la_decode_step(const void *q, const void *k, const void *v, float *state, void *o,
                         int B, int H, int D, unsigned flags, void *stream);

/*
 * la_state_out -- hand prefill states to decode: state_dst[slot(s)][h] =
 * state_ws[s][h] for s < S, where slot(s) = seq_to_slot[s], or s when
 * seq_to_slot is NULL.
 *
 *   state_ws    [S][H][D][D] fp32 source (as written by la_prefill).
 *   state_dst   [num_slots][H][D][D] fp32 destination (the decode batch state).
 *   num_slots   rows of state_dst.  Given explicitly, so that a slot index read on
 *               the device can be range-checked there.
 *   seq_to_slot DEVICE array of S int32 slot indices, or NULL (identity; then
 *               S <= num_slots is required).  A slot outside [0, num_slots) is
 *               skipped on the device and reported as LA_ERR_DEVICE_RANGE by
 *               la_get_device_status.
 *   The two buffers must not overlap.
 */
la_status la_state_out(const float *state_ws, float *state_dst, int S, int H, int D,
                       const int32_t *seq_to_slot, int num_slots, void *stream);

/* Human-readable name of a status code (static storage; never NULL). */
const char *la_status_string(la_status status);

/*
 * la_get_device_status -- synchronise `stream`, then return and clear the
 * current device's status word: LA_OK, LA_ERR_DEVICE_TIMEOUT or
 * LA_ERR_DEVICE_RANGE (the first recorded), or LA_ERR_CUDA if the stream
 * reports an error.  The word is per device, not per stream: it is shared by
 * every call on the device, so with prefill and decode on two streams a fault
 * recorded by either kernel is reported to (and cleared by) whichever
 * la_get_device_status call on that device comes first.
 */
la_status la_get_device_status(void *stream);

/* Library version: major * 10000 + minor * 100 + patch. */
int la_version(void);

#ifdef __cplusplus
}
#endif

#endif /* LIGHTNING_ATTENTION_H */
