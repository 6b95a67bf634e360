/*
 * kda.h -- C ABI of libkda.so: Kimi Delta Attention (KDA) on NVIDIA B200.
 *
 * The operation.  Per head, a fixed-size d_k x d_v fp32 state S is carried
 * through the sequence by the gated delta rule
 *
 *     S_t = (I - beta_t k_t k_t^T) Diag(exp g_t) S_{t-1} + beta_t k_t v_t^T
 *     o_t = S_t^T q_t
 *
 * with a scalar write strength beta_t in (0, 1) and a channel-wise log-decay
 * g_t (one value per key channel) bounded to [-5, 0].  Sources:
 *   - "T11E1: K3 tech report" podcast transcript (williamliu.ai): the KDA
 *     turn (recurrent state, learned write strength, channel-wise
 *     forgetting; decay bounded so chunk work stays in bf16 range on dense
 *     tensor cores) and the next turn (log-decay floor of -5 keeps the
 *     reciprocal scaling over a 16-token tile below the bf16 limit);
 *   - "Kimi K3 goes trillion-scale with sparse MoE efficiency" subtitles
 *     (podcast.do-not-panic.com), cue 14: delta-rule recurrence with a
 *     channel-wise forget gate, one fixed-size state, lower-bounded sigmoid
 *     decay, dense diagonal and off-diagonal tiles;
 *   - "177: Kimi K3 in Detail" episode notes (zjai.club), Deep dive 17 and 10:
 *     decoding reads a fixed per-request state that is rewritten in place
 *     for every token.
 * No output scale is applied (no 1/sqrt(d_k)); q and k are expected to be
 * L2-normalised by the caller.  Preconditions on values (g in [-5, 0],
 * beta in (0, 1), unit-norm keys) are documented, not checked or clamped.
 *
 * Conventions shared by every entry point:
 *   - All tensor pointers are DEVICE pointers, owned by the caller, 16-byte
 *     aligned, densely packed in the row-major layouts given per function.
 *     No entry point keeps a pointer after it returns.  Only the bf16
 *     prefill calls kda_chunk_fwd, kda_chunk_fwd_raw and kda_chunk_fwd_states
 *     take memory of their own, and only on the segment-scan path (see
 *     kda_chunk_fwd): stream-ordered workspace (cudaMallocAsync /
 *     cudaFreeAsync on `stream`).  kda_chunk_fwd_noalloc is kda_chunk_fwd
 *     without any allocation.
 *   - Calls are asynchronous on `stream` (0 = legacy default stream) and do
 *     no host synchronisation.  Asynchronous device errors surface at the
 *     caller's next synchronisation, as for any CUDA launch.
 *   - Return value: KDA_OK, or a negative kda_status.  Argument errors are
 *     detected on the host and return before anything is launched.
 *   - Inputs and outputs must not overlap, except that hT may equal h0.
 *   - Thread-safe: calls may come from several host threads, on several
 *     streams and devices at once.  A call runs on the current device.  The
 *     library's global state is a launch counter (atomic), one-time set-up
 *     per device (kernel shared-memory limits, the SM count, the memory
 *     pool's release threshold; idempotent, done by the first call on each
 *     device), one bounded-wait error word per device (kda_device_status)
 *     and the scratch array of kda_chunk_fwd_noalloc, whose segment-scan
 *     calls must be ordered with one another (see there).
 */
#ifndef KDA_H
#define KDA_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

struct CUstream_st;
typedef struct CUstream_st* kda_stream_t; /* identical to cudaStream_t */

typedef enum {
    KDA_OK = 0,
    KDA_ERR_INVALID_ARG = -1,  /* null/misaligned pointer, negative size   */
    KDA_ERR_UNSUPPORTED = -2,  /* valid but unsupported shape (dk, dv)      */
    KDA_ERR_CUDA = -3,         /* a CUDA launch or runtime call failed      */
    KDA_ERR_TIMEOUT = -4,      /* a bounded device wait expired (see below) */
    KDA_ERR_NO_MEMORY = -5     /* workspace allocation failed               */
} kda_status;

/*
 * kda_chunk_fwd -- chunked prefill, bf16 inputs and output, fp32 state.
 *
 *   q, k, g : bf16 [B][T][H][dk]        v, o : bf16 [B][T][H][dv]
 *   beta    : bf16 [B][T][H]
 *   h0      : fp32 [B][H][dk][dv], or NULL for a zero initial state
 *   hT      : fp32 [B][H][dk][dv], or NULL to skip; may equal h0
 *   B, T, H >= 0 (any of them 0: nothing to compute; with T == 0 and hT
 *   given, hT receives h0, or zeros).  Supported: dk == dv == 128.
 * o_t is written for every token; hT is S after the last token.  The work is
 * done in 16-token tiles on the tensor cores with an fp32 master state (the
 * "T11E1" transcript's log-decay-bound turn is what makes the diagonal tiles
 * dense).  Every MMA accumulates in fp32 and rounds each operand once, to
 * nearest: to tf32 for the products of decay-scaled keys (factors up to
 * e^80) and, on the cluster path (few heads), to fp16 for the three
 * state-sized products S^T W^T, S^T Qt^T and U^T Kb, for P U and for the
 * WY products T Kt and T V (tf32 for all of them on the one-SM path).  Both
 * keep a 10-bit significand, which keeps o within 1e-2 of the exact
 * recurrence where bf16 operands would not.  fp16's range is the cluster path's input contract:
 * h0 and v entries far below 65504 in magnitude (as unit-norm q and k
 * imply for the other operands); state entries below 2^-14 of absolute
 * size lose significand bits (absolute error up to 2^-24), negligible for
 * states of the order of 1e-3 or larger.  Returns KDA_ERR_UNSUPPORTED for
 * other dk/dv.
 *
 * Segment scan: with B*H <= 8 and T >= 4096 each sequence is cut into P
 * segments that run in parallel (P about SMs / (B*H), at least 256 tokens
 * each): a pass over all segments from a zero state and from the identity
 * (with v = 0) gives, per segment, the state it reaches from zero and its
 * transition matrix; a short chain over the segments gives each segment's
 * true start state; a last pass writes o.  This path takes 3 * B * P * H *
 * dk * dv * 4 bytes of stream-ordered workspace (at most 29,097,984 bytes
 * when the path is chosen by itself on a 148-SM B200) and returns KDA_ERR_NO_MEMORY if it
 * cannot.  The environment variable
 * KDA_PREFILL_VARIANT = fused | cluster | segmented forces one path
 * (measurement and tests; "segmented" needs T >= 512).
 */
int kda_chunk_fwd(const void* q, const void* k, const void* v, const void* g,
                  const void* beta, const float* h0, void* o, float* hT,
                  int B, int T, int H, int dk, int dv, kda_stream_t stream);

/*
 * kda_chunk_fwd_raw -- kda_chunk_fwd with the prologue fused in: q_raw and
 * k_raw are NOT normalised and z is the gate pre-activation.  Inside the
 * kernel, per token and head, q and k are L2-normalised over the dk channels
 * (in fp32; a zero vector stays zero) and the log-decay is g = -5 sigmoid(z)
 * (the lower-bounded sigmoid decay of the "Kimi K3 goes trillion-scale ..."
 * subtitles, cue 14, with the transcript's -5 floor), so no separate pass
 * writes normalised q, k or g.  Layouts, paths, results otherwise as
 * kda_chunk_fwd (z in the place of g).
 */
int kda_chunk_fwd_raw(const void* q_raw, const void* k_raw, const void* v, const void* z,
                      const void* beta, const float* h0, void* o, float* hT,
                      int B, int T, int H, int dk, int dv, kda_stream_t stream);

/*
 * kda_chunk_fwd_states -- kda_chunk_fwd that also writes intermediate states
 * (prefix-cache blocks): the fp32 state after every `state_every` tokens,
 *
 *   states : fp32 [B][H][T / state_every][dk][dv],  states[b][h][s] = S after
 *            token (s + 1) * state_every of sequence b, head h
 *
 * (floor division: a block that the sequence does not complete gets no
 * state; with T a multiple of state_every the last one equals hT).
 * state_every must be a positive multiple of 32 (the chunk of the state
 * recurrence), else KDA_ERR_INVALID_ARG; states may be NULL only when
 * T < state_every.  Same paths and arithmetic as kda_chunk_fwd (the states
 * are the fp32 master state, not a rounded copy).  The "177: Kimi K3 in
 * Detail" episode notes (Deep dive 10, 23) describe serving that keeps a
 * long shared prefix and adds a few thousand tokens per turn; a state
 * every block lets a later call resume from any block boundary.
 */
int kda_chunk_fwd_states(const void* q, const void* k, const void* v, const void* g,
                         const void* beta, const float* h0, void* o, float* hT,
                         float* states, int state_every,
                         int B, int T, int H, int dk, int dv, kda_stream_t stream);

/*
 * kda_chunk_transition -- the transition of each sequence as a whole,
 *
 *   M[b][h] = prod_{t = T..1} (I - beta_t k_t k_t^T) Diag(exp g_t)   (d_k x d_k)
 *
 * so that running the sequence from any start state S0 ends at
 * M S0 + (the state it reaches from zero).  Computed on the tensor cores as
 * the state reached from S = I with v = 0 (every state column evolves on its
 * own), no o written, with tf32 operands in every product (M decays towards
 * zero and keeps its relative accuracy there, which fp16 operands would
 * not).  q, k, g: bf16 [B][T][H][dk]; beta: bf16 [B][T][H];
 * M: fp32 [B][H][dk][dk] (T == 0: the identity).  Supported: dk == 128.
 * With kda_state_chain this joins segments of one sequence that were run
 * independently (for example one segment per GPU).
 */
int kda_chunk_transition(const void* q, const void* k, const void* g, const void* beta, float* M,
                         int B, int T, int H, int dk, kda_stream_t stream);

/*
 * kda_state_chain -- joins P consecutive segments of each sequence: with
 * M[b][p][h] a segment's transition (kda_chunk_transition) and N[b][p][h]
 * the state it reaches from zero (kda_chunk_fwd with h0 = NULL),
 *
 *   S_0 = h0[b][h] (or zero),   S_{p+1} = M_p S_p + N_p,
 *
 * writes S_start[b][p][h] = S_p (the true start state of segment p) and
 * hT[b][h] = S_P.  M, N, S_start: fp32 [B][P][H][dk][dv] (M's last two
 * dimensions are dk x dk, with dk == dv); h0, hT: fp32 [B][H][dk][dv], either
 * may be NULL; hT may equal h0.  fp32 arithmetic.  Supported: dk == dv == 128.
 */
int kda_state_chain(const float* M, const float* N, const float* h0, float* S_start, float* hT,
                    int B, int P, int H, int dk, int dv, kda_stream_t stream);

/*
 * kda_chunk_fwd_noalloc -- kda_chunk_fwd that allocates nothing: on the
 * segment-scan path its workspace is a fixed scratch array in the library's
 * device memory (one copy per device, 29,097,984 bytes: three fp32 state
 * arrays for up to 148 segment-heads, which covers every call that takes the
 * segment scan by itself).  Arguments, layouts, results and the choice of
 * path are those of kda_chunk_fwd (the same arithmetic, bit for bit).
 * Returns KDA_ERR_NO_MEMORY, before anything is launched, when the call
 * needs more scratch than that (possible only when the segment scan is
 * forced through KDA_PREFILL_VARIANT).  Calls that take the segment-scan
 * path share the one scratch of their device: order them (one stream, or
 * events between streams); the other paths use no scratch.
 */
int kda_chunk_fwd_noalloc(const void* q, const void* k, const void* v, const void* g,
                          const void* beta, const float* h0, void* o, float* hT,
                          int B, int T, int H, int dk, int dv, kda_stream_t stream);

/*
 * kda_chunk_fwd_f32 -- the same recurrence with fp32 inputs and fp32 output,
 * evaluated in fp32 arithmetic (for tolerance-critical callers).
 * Layouts as kda_chunk_fwd with every tensor fp32.
 * Supported: dk, dv in {32, 64, 128}.
 */
int kda_chunk_fwd_f32(const float* q, const float* k, const float* v,
                      const float* g, const float* beta, const float* h0,
                      float* o, float* hT,
                      int B, int T, int H, int dk, int dv, kda_stream_t stream);

/*
 * kda_decode_step -- one token for each of N requests, state updated IN PLACE
 * ("177: Kimi K3 in Detail", Deep dive 10: the state is a whiteboard that is
 * rewritten for every token).
 *
 *   q, k, g : bf16 [N][H][dk]     v, o : bf16 [N][H][dv]     beta : bf16 [N][H]
 *   state   : fp32 [N][H][dk][dv], read and overwritten with S_t
 *   N, H >= 0.  Supported: dk, dv in {32, 64, 128}.
 * The state layout is the one kda_chunk_fwd writes to hT, so a prefill's hT
 * is directly a decode state.
 */
int kda_decode_step(const void* q, const void* k, const void* v, const void* g,
                    const void* beta, float* state, void* o,
                    int N, int H, int dk, int dv, kda_stream_t stream);

/*
 * kda_decode_step_raw -- kda_decode_step with the same fused prologue as
 * kda_chunk_fwd_raw (q_raw, k_raw unnormalised; z the gate pre-activation).
 */
int kda_decode_step_raw(const void* q_raw, const void* k_raw, const void* v, const void* z,
                        const void* beta, float* state, void* o,
                        int N, int H, int dk, int dv, kda_stream_t stream);

/*
 * kda_chunk_bwd -- gradients of a kda_chunk_fwd call (training at the 8K-64K
 * pre-training lengths of the "T11E1: K3 tech report" transcript, the
 * context-length turn): with L = sum(dO * o) + sum(dhT * hT), the gradients
 * of L with respect to q, k, v, g, beta and h0.  The pages give the forward
 * only; the backward is its exact derivative (up to rounding).
 *
 *   q, k, g, v, beta, h0 : the forward's inputs (layouts of kda_chunk_fwd)
 *   dO   : bf16 [B][T][H][dv], the gradient of o
 *   dhT  : fp32 [B][H][dk][dv], the gradient of hT, or NULL (zero)
 *   dq, dk, dg : bf16 [B][T][H][dk]     dv : bf16 [B][T][H][dv]
 *   dbeta      : bf16 [B][T][H]         dh0 : fp32 [B][H][dk][dv], or NULL
 *   Supported: d_k == d_v == 128.  T == 0: dh0 receives dhT (or zeros).
 * Three launches on `stream`: per-chunk operands and the forward and reverse
 * state chains in fp32 (the gradient of the decay sums terms that nearly
 * cancel, and chunk-start states at tf32 precision would move it by about
 * 1e-2 of its scale), then the chunk-local gradients, whose five
 * state-sized products (W S0, Kb dS, dO S0^T, U dS^T, dU S0^T) run as tf32
 * tensor-core MMAs from the fp32 states and the rest in fp32.  The local
 * kernel's waits for its MMAs are bounded as the prefill's (a chunk whose
 * wait expired gets NaN gradients; kda_device_status reports it).  Stream-ordered
 * workspace of 209,408 bytes per 32-token chunk and head (about 6.5 KB per
 * token and head; KDA_ERR_NO_MEMORY if it cannot be had).  Outputs must not
 * overlap inputs or one another.
 */
int kda_chunk_bwd(const void* q, const void* k, const void* v, const void* g, const void* beta,
                  const float* h0, const void* dO, const float* dhT,
                  void* dq, void* dk, void* dv, void* dg, void* dbeta, float* dh0,
                  int B, int T, int H, int d_k, int d_v, kda_stream_t stream);

/*
 * kda_chunk_bwd_raw -- gradients of a kda_chunk_fwd_raw call: as
 * kda_chunk_bwd, with q_raw, k_raw and the gate pre-activation z in the
 * places of q, k and g, and dq_raw, dk_raw, dz returned for them.  The
 * prologue runs inside the kernels as in the raw forward (q, k normalised in
 * fp32, a zero vector staying zero with a zero gradient; g = -5 sigmoid(z),
 * g = 0 past the end), and its chain rule (dr = (dx - x (x . dx)) / |r|,
 * dz = -5 sigmoid(z) (1 - sigmoid(z)) dg) is applied to the outputs, so no
 * normalised tensor is written.  Layouts, workspace, errors as kda_chunk_bwd.
 */
int kda_chunk_bwd_raw(const void* q_raw, const void* k_raw, const void* v, const void* z, const void* beta,
                      const float* h0, const void* dO, const float* dhT,
                      void* dq_raw, void* dk_raw, void* dv, void* dz, void* dbeta, float* dh0,
                      int B, int T, int H, int d_k, int d_v, kda_stream_t stream);

/*
 * kda_verify_fwd -- K consecutive tokens of each of N requests from a start
 * state, keeping the state after EVERY token (speculative decoding: verify
 * K drafted tokens, then continue from the state after the last accepted
 * one).  The "177: Kimi K3 in Detail" episode notes (Deep dive 23) describe
 * the rollback this serves: keep a checkpoint and a short log per step, and
 * replay the accepted steps.
 *
 *   q, k, g : bf16 [N][K][H][dk]      v, o : bf16 [N][K][H][dv]
 *   beta    : bf16 [N][K][H]
 *   h0      : fp32 [N][H][dk][dv] start states, read only (NULL: zero)
 *   states  : fp32 [N][K][H][dk][dv]; states[n][t] = S after token t + 1
 *             of request n (all heads: one [H][dk][dv] block, the layout of
 *             a kda_decode_step state, so rolling back to an accepted
 *             prefix is one contiguous copy per request)
 *   1 <= K <= KDA_VERIFY_MAX_TOKENS (else KDA_ERR_UNSUPPORTED; K == 0 is a
 *   no-op).  Supported: dk, dv in {32, 64, 128}.
 * Every token is the exact arithmetic of kda_decode_step (fp32, CUDA
 * cores, the same operation order), so replaying the first j tokens from h0
 * with kda_decode_step reproduces states[n][j - 1] bit for bit.  Memory
 * bound: h0 read once, K states written.  o and states must not overlap
 * the inputs; h0 may not alias states.
 */
#define KDA_VERIFY_MAX_TOKENS 64
int kda_verify_fwd(const void* q, const void* k, const void* v, const void* g,
                   const void* beta, const float* h0, void* o, float* states,
                   int N, int K, int H, int dk, int dv, kda_stream_t stream);

/*
 * kda_device_status -- KDA_OK, or KDA_ERR_TIMEOUT if a kernel of this
 * library gave up on a bounded device-side wait since the last call (every
 * wait between the roles of a prefill kernel, and the backward's waits for
 * its tensor-core products, give up after 2 s).  The kernel then winds down
 * and fills the o rows and hT of the affected heads (backward: the dq, dk,
 * dv, dg and dbeta rows of the affected chunk) with NaN (intermediate
 * states, if asked for, are undefined), so a partial result never passes
 * for a real one.  Reads and clears the flag;
 * synchronises `stream`.  KDA_ERR_CUDA if a CUDA call fails.
 */
int kda_device_status(kda_stream_t stream);

/*
 * kda_selftest_bounded_wait -- launches a one-warp kernel whose device-side
 * wait can never be satisfied; the wait gives up after `limit_ns`
 * (1 <= limit_ns <= 1e9) and sets the status word that kda_device_status
 * reports as KDA_ERR_TIMEOUT.  Lets callers check, without any fault, that
 * an expired wait ends the kernel cleanly and leaves the context usable.
 * KDA_ERR_INVALID_ARG for a limit outside that range (nothing launched).
 */
int kda_selftest_bounded_wait(uint64_t limit_ns, kda_stream_t stream);

/* Human-readable name of a kda_status value (static storage). */
const char* kda_status_string(int status);

/* Number of kernels this library has launched in this process (all entry
 * points, all devices); lets callers count launches in a timed region. */
uint64_t kda_launch_count(void);

/*
 * kda_prefill_path -- which path a bf16 prefill call (kda_chunk_fwd and its
 * variants) of this shape takes on the current device: 0 = one SM per
 * (batch, head), 1 = a cluster of four SMs per head (when batch x heads x 4
 * fits in the device's SMs), 2 = the segment scan (batch x heads <= 8 and
 * T >= 4096), after any KDA_PREFILL_VARIANT override.  Launches nothing.
 * KDA_ERR_INVALID_ARG for negative sizes.
 */
int kda_prefill_path(int B, int T, int H);

/* ABI version: (major << 16) | minor. */
int kda_version(void);

#ifdef __cplusplus
}
#endif

#endif /* KDA_H */
