// KDA chunked prefill on the sm_100a tensor cores (tcgen05, kind::tf32,
// fp32 accumulation in tensor memory).
//
// The recurrence ("T11E1: K3 tech report" transcript, KDA turn; "Kimi K3 goes
// trillion-scale ..." subtitles, cue 14)
//     S_t = (I - b_t k_t k_t^T) Diag(exp g_t) S_{t-1} + b_t k_t v_t^T,  o_t = S_t^T q_t
// is evaluated exactly (up to rounding) in chunks of C = 32 tokens made of two
// 16-token tiles.  With Gam_r the running sum of g (per key channel) and
// gamma = exp(Gam), a chunk with start state S computes
//     A  = diag(b) strict_lower(G_kk),  P = lower_incl(G_qk)
//          (entries k_r . k_i exp(Gam_r - Gam_i) and q_r . k_i exp(Gam_r - Gam_i))
//     T  = (I + A)^-1 diag(b),   W = T Kt,   U' = T V
//     U  = U' - W S,   O = Qt S + P U,   S <- Diag(gamma_C) S + Kb^T U
// where Kt = K gamma and Qt = Q gamma are relative to the chunk start and
// Kb = K gamma_C / gamma.  The decayed products inside a 16-token tile use
// the tile start as reference: Kt_tile (<= 1) against Kh = K / gamma_tile
// (<= e^80).  The log-decay floor g >= -5 bounds that reciprocal scaling by
// e^{5*16}, inside the fp32/tf32 range, so the diagonal tiles are dense MMAs
// with no position-by-position path ("T11E1" transcript, log-decay-bound
// turn; subtitles, cue 14).  The block between the two tiles of a chunk uses
// the tile boundary as reference: Kb_tile0 (<= 1) against Kt_tile1 (<= 1).
//
// Three launch paths over this arithmetic (d_k = d_v = 128):
//   * prefill_tc_kernel, one SM per (batch, head), 512 threads in two roles:
//     chain warps 0-7 (thread (j, half) owns column j, rows [64 half, +64) of
//     the fp32 state S in registers; per chunk X = S^T [W | Qt]^T with the
//     tf32 copy of S^T in tensor memory as the A operand (M 128, N 64, K 128),
//     U^T = U'^T - X_W, S^T += U^T Kb (N 128, K 32), O^T += U^T P^T (N 32,
//     K 32), the decay/update of S and the bf16 store of o) and prep warps
//     8-15 (for the next chunk: TMA loads of q, k, v, g, the decay scaling,
//     the Gram MMA, the 32 x 32 unit-triangular solve, W^T = Kt^T T^T and
//     U'^T = V^T T^T (M 128, N 32, K 32), and the fill of the chain's
//     operand buffers).  The roles meet at named-barrier rendezvous.
//   * prefill_cluster_kernel, a cluster of four SMs per head when the heads
//     alone would leave most SMs idle: one chain CTA, three preparing CTAs
//     that push each prepared chunk into the chain CTA's shared memory over
//     DSMEM (description above the kernel).
//   * the segment scan for very few heads on long sequences: every sequence
//     cut into segments run in parallel by either kernel, joined through
//     their transitions (description above launch_segmented).
// Every MMA accumulates in fp32 and is issued by a whole converged warp with
// elect.sync.  The Gram product takes the decay-scaled keys (factors up to
// e^80) and is tf32 (kind::tf32) in both kernels, and so is every product of
// the one-SM kernel; operands are rounded to tf32 once, to nearest (ties away
// from zero), by an integer add-and-mask: bf16 operands would leave errors of
// a few percent of rms(o) on these products (the q.k diagonal times a large
// u); a 10-bit significand leaves a few tenths of a percent.  The cluster
// kernel's chain and WY products take fp16 instead (the same significand;
// see there).
// Shared-memory operands use the no-swizzle K-major layout; when the thread
// that produces a value owns the K index, the K-direction core-matrix stride
// is padded to 144 B so that a warp's scalar stores hit distinct banks.
#include <cuda.h>
#include <stdlib.h>
#include <string.h>

#include "kda_common.cuh"
#include "kda_tc.cuh"

namespace kda {

namespace pf {

constexpr int D = 128;         // d_k = d_v
constexpr int TILE = 16;
constexpr int C = 32;          // tokens per chunk (two tiles)
constexpr int NCH = 256;       // chain threads (warps 0-7)
constexpr int NPREP = 256;     // prep threads (warps 8-15)
constexpr int NT = NCH + NPREP;

constexpr uint32_t PAD_LBO = 144;            // padded K-direction core-matrix stride
constexpr uint32_t LBO = 128;                // dense K-direction core-matrix stride
constexpr uint32_t SBO_K128P = (D / 4) * PAD_LBO;   // 4608: K = 128, padded
constexpr uint32_t SBO_K32 = (C / 4) * LBO;         // 1024: K = 32, dense
constexpr uint32_t SBO_K32P = (C / 4) * PAD_LBO;    // 1152: K = 32, padded
// the same layouts for 16-bit elements (core matrices of 8 rows x 8 elements)
constexpr uint32_t H_SBO_K32 = (C / 8) * LBO;        // 512: K = 32, dense
constexpr uint32_t H_SBO_K32P = (C / 8) * PAD_LBO;   // 576: K = 32, padded

// shared memory map (bytes)
constexpr uint32_t RAW = 0;                                    // q, k, v, g rows of a chunk (bf16)
constexpr uint32_t RAW_T = C * D * 2;                          // one tensor
constexpr uint32_t BETA = RAW + 4 * RAW_T;                     // C fp32
constexpr uint32_t GEX = BETA + C * 4;                         // per tile gamma_16, 2 x 128 fp32
constexpr uint32_t GA = GEX + 2 * D * 4;                       // Gram A: Kh (32 rows), Kb tile 0 (16 rows)
constexpr uint32_t GB = GA + 6 * SBO_K128P;                    // Gram B: Kt (32 rows), Qt (32 rows);
                                                               // GA's padding rows 48-63 read GB
constexpr uint32_t WA = GB + 8 * SBO_K128P;                    // Kt^T: M 128 x K 32
constexpr uint32_t VA = WA + (D / 8) * SBO_K32;                // V^T:  M 128 x K 32
constexpr uint32_t TB = VA + (D / 8) * SBO_K32;                // T:    N 32 x K 32 (padded)
constexpr uint32_t B1 = TB + (C / 8) * SBO_K32P;               // [W | Qt]: N 64 x K 128 (padded)
constexpr uint32_t B2 = B1 + 8 * SBO_K128P;                    // Kb:   N 128 x K 32
constexpr uint32_t B3 = B2 + (D / 8) * SBO_K32;                // P:    N 32 x K 32 (padded)
constexpr uint32_t GAM = B3 + (C / 8) * SBO_K32P;              // gamma_C, 2 x 128 fp32 (by chunk parity)
constexpr int LD = C + 1;                                      // scratch row stride (floats)
constexpr uint32_t AMS = GAM + 2 * D * 4;                          // A (32 x 33 fp32)
constexpr uint32_t PMS = AMS + C * LD * 4;                     // P
constexpr uint32_t XMS = PMS + C * LD * 4;                     // diagonal-block inverses
constexpr uint32_t TMS = XMS + C * LD * 4;                     // T
constexpr uint32_t YMS = TMS + C * LD * 4;                     // A_10 X_00 (16 x 17)
constexpr uint32_t OST = YMS + TILE * (TILE + 1) * 4;           // o staging, 32 x 128 bf16
constexpr uint32_t NRM = OST + C * D * 2;                      // prologue: per-warp squared norms
constexpr uint32_t NRM_BYTES = 2 * 4 * 2 * TILE * 4;           // [tile][warp][q, k][token]
constexpr int LDT = C + 4;                                     // transposed-A row stride (16-byte rows)
constexpr uint32_t ATM = NRM + NRM_BYTES;                      // A^T of the diagonal blocks (32 x 36 fp32)
constexpr uint32_t SMEM_BYTES = ATM + C * LDT * 4;

static_assert(SMEM_BYTES <= 227 * 1024, "shared memory budget");
static_assert(OST % 16 == 0 && GA % 16 == 0 && GB % 16 == 0 && WA % 16 == 0 && VA % 16 == 0 && TB % 16 == 0 &&
              B1 % 16 == 0 && B2 % 16 == 0 && B3 % 16 == 0 && ATM % 16 == 0, "descriptor alignment");

// tensor memory columns (512 allocated)
constexpr uint32_t T_AS = 0;     // S^T (tf32), 128
constexpr uint32_t T_AU = 128;   // U^T (tf32), 32
constexpr uint32_t T_DX = 160;   // [(W S)^T | (Qt S + P U)^T], 64
constexpr uint32_t T_DKU = 224;  // (Kb^T U)^T, 128
constexpr uint32_t T_DG = 352;   // Gram (M = 64), 64
constexpr uint32_t T_DW = 416;   // W^T, 32
constexpr uint32_t T_DU = 448;   // U'^T, 2 x 32 (double-buffered)
constexpr uint32_t TMEM_COLS = 512;

// named barriers (0 is __syncthreads)
constexpr uint32_t BAR_FREE = 1, BAR_READY = 2, BAR_CHAIN = 3, BAR_PREP = 4;

constexpr uint64_t WAIT_NS = 2000000000ull;   // bounded waits: 2 s
// After an expired wait: how long a CTA lets a copy that was already issued
// land before it gives up its shared memory (an issued copy lands within
// microseconds; one that was never issued never does).
constexpr uint64_t DRAIN_NS = 20000000ull;    // 20 ms

// Launch flags (segment scan passes): treat v as zero, start from h0 = I
// (ignore h0), skip the o stores.
constexpr uint32_t SEG_V_ZERO = 1u, SEG_H0_EYE = 2u, SEG_NO_O = 4u;
// Fused prologue: q, k arrive unnormalised and the g tensor holds the gate
// pre-activation z; the kernel L2-normalises q and k per token and head (a
// zero vector stays zero) and takes g = -5 sigmoid(z) (g = 0 past the end).
constexpr uint32_t PROLOGUE = 8u;

}  // namespace pf

__device__ int g_prefill_status;   // set to KDA_ERR_TIMEOUT by a wait that expired

__device__ __forceinline__ void st_f32(unsigned char* base, uint32_t off, float v) {
    *reinterpret_cast<float*>(base + off) = v;
}
__device__ __forceinline__ void st_f32x2(unsigned char* base, uint32_t off, float a, float b) {
    *reinterpret_cast<float2*>(base + off) = make_float2(a, b);
}
__device__ __forceinline__ void st_f32x4(unsigned char* base, uint32_t off, float a, float b, float c, float d) {
    *reinterpret_cast<float4*>(base + off) = make_float4(a, b, c, d);
}
__device__ __forceinline__ void named_bar(uint32_t id, uint32_t count) {
    asm volatile("bar.sync %0, %1;" :: "r"(id), "r"(count) : "memory");
}

__device__ __forceinline__ void named_arrive(uint32_t id, uint32_t count) {
    asm volatile("bar.arrive %0, %1;" :: "r"(id), "r"(count) : "memory");
}

// State snapshots (prefix-cache blocks): with snap_every > 0 chunks, the fp32
// state after every snap_every * 32 tokens of the whole sequence is written
// to states[b][h][s][D][D], s = 0 .. T / (snap_every * 32) - 1 (a block that
// the sequence does not complete gets no snapshot).  gc is the index of the
// chunk just completed, counted from the start of the sequence.
__device__ __forceinline__ float* snapshot_slot(float* states, int snap_every, int gc, int T, int b, int H, int h)
{
    if (states == nullptr || snap_every <= 0 || (gc + 1) % snap_every != 0) return nullptr;
    const int s = (gc + 1) / snap_every - 1;
    const int n_snap = T / (snap_every * pf::C);
    if (s >= n_snap) return nullptr;
    return states + (((int64_t)b * H + h) * n_snap + s) * pf::D * pf::D;
}

// Prologue, part 1 (before the exponentials): a[] holds z and becomes
// g = -5 sigmoid(z) (0 for tokens t0 + rr >= Tl, which leaves the state
// alone); each warp writes the squared norms of q and k over its 32 channels
// for the 16 tokens of its tile to nrm[tile][warp][q, k][token].
__device__ __forceinline__ void prologue_gate_and_norms(float (&a)[pf::TILE], const float (&qr)[pf::TILE],
                                                        const float (&kr)[pf::TILE], int t0, int Tl,
                                                        float* nrm, int tau, int c)
{
    constexpr int TILE = pf::TILE;
    float nq[TILE], nk[TILE];
#pragma unroll
    for (int rr = 0; rr < TILE; ++rr) {
        a[rr] = (t0 + rr < Tl) ? -5.f / (1.f + __expf(-a[rr])) : 0.f;
        nq[rr] = qr[rr] * qr[rr];
        nk[rr] = kr[rr] * kr[rr];
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1)
#pragma unroll
        for (int rr = 0; rr < TILE; ++rr) {
            nq[rr] += __shfl_xor_sync(0xffffffffu, nq[rr], off);
            nk[rr] += __shfl_xor_sync(0xffffffffu, nk[rr], off);
        }
    if ((c & 31) == 0) {
        float* w = nrm + ((tau * 4 + (c >> 5)) * 2) * TILE;
#pragma unroll
        for (int rr = 0; rr < TILE; ++rr) {
            w[rr] = nq[rr];
            w[TILE + rr] = nk[rr];
        }
    }
}

// Prologue, part 2 (after a barrier): q, k of this thread's 16 tokens scaled
// to unit norm over the 128 channels (zero vectors stay zero).
__device__ __forceinline__ void prologue_normalise(float (&qr)[pf::TILE], float (&kr)[pf::TILE],
                                                   const float* nrm, int tau)
{
    constexpr int TILE = pf::TILE;
#pragma unroll
    for (int rr = 0; rr < TILE; ++rr) {
        float sq = 0.f, sk = 0.f;
#pragma unroll
        for (int w = 0; w < 4; ++w) {
            sq += nrm[((tau * 4 + w) * 2) * TILE + rr];
            sk += nrm[((tau * 4 + w) * 2) * TILE + TILE + rr];
        }
        qr[rr] *= sq > 0.f ? rsqrtf(sq) : 0.f;
        kr[rr] *= sk > 0.f ? rsqrtf(sk) : 0.f;
    }
}

// After a bounded wait expired anywhere in a CTA its o rows and hT are
// incomplete: fill them with NaN so that a caller who never reads
// kda_device_status cannot mistake a partial result for a real one.
// o_head points at token 0 of this head's segment, rows row_stride apart.
__device__ __forceinline__ void poison_head_outputs(__nv_bfloat16* o_head, int64_t row_stride, int Tl,
                                                    bool write_o, float* hT_head, int tid, int nthr)
{
    const float qnan = __int_as_float(0x7fc00000);
    if (write_o) {
        const __nv_bfloat16 nb = __float2bfloat16_rn(qnan);
        for (int64_t e = tid; e < (int64_t)Tl * pf::D; e += nthr)
            o_head[(e / pf::D) * row_stride + (e % pf::D)] = nb;
    }
    if (hT_head)
        for (int e = tid; e < pf::D * pf::D; e += nthr) hT_head[e] = qnan;
}

// A shared flag read once by lane 0 and broadcast: the same value in every
// lane, so a whole-warp MMA issue never diverges on it.
__device__ __forceinline__ bool warp_flag(const int& flag) {
    return __shfl_sync(0xffffffffu, *(const volatile int*)&flag, 0) != 0;
}

template <bool PRO>       // PRO: the fused prologue (launch flag PROLOGUE)
__global__ void __launch_bounds__(pf::NT, 1)
prefill_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_g,
                  const __nv_bfloat16* __restrict__ beta, const float* h0,
                  __nv_bfloat16* __restrict__ o, float* hT, int T, int H,
                  int seg_len, int n_seg, uint32_t flags, float* states, int snap_every,
                  uint64_t wait_ns)
{
    using namespace pf;
    using namespace tc;
    extern __shared__ __align__(1024) unsigned char sm[];
    __shared__ uint32_t s_taddr;
    __shared__ __align__(8) uint64_t s_bar[3];     // chain MMAs, prep MMAs, input loads
    __shared__ int s_abort;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    // grid.y = B * n_seg: sequence b, segment [ts, ts + Tl) of it (n_seg = 1: the whole sequence)
    const int h = blockIdx.x, bb = blockIdx.y;
    const int b = bb / n_seg;
    const int ts = (bb - b * n_seg) * seg_len;
    const int Tl = max(0, min(seg_len, T - ts));
    const int64_t head_off = (int64_t)bb * H + h;          // h0 / hT: [B * n_seg][H][D][D]
    const int64_t row_stride = (int64_t)H * D;            // elements between tokens
    const int64_t base = (((int64_t)b * T + ts) * H + h) * D;    // token ts of this head

    if (warp == 0) {
        tmem_alloc(smem_u32(&s_taddr), TMEM_COLS);
        tmem_relinquish();
    }
    if (tid == 0) {
        mbar_init(smem_u32(&s_bar[0]), 1);
        mbar_init(smem_u32(&s_bar[1]), 1);
        mbar_init(smem_u32(&s_bar[2]), 1);
        fence_mbar_init();
        s_abort = 0;
    }
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    const uint32_t tm = s_taddr;
    const int sp = warp & 3;                                   // TMEM sub-partition of this warp
    const uint32_t lane_base = (uint32_t)(32 * sp) << 16;
    const int n_chunks = (Tl + C - 1) / C;
    // A wait that expired sets s_abort; from then on both roles skip all MMA
    // work but keep the barrier protocol, so the CTA winds down without
    // further waits and reports KDA_ERR_TIMEOUT.
    auto expired = [&]() {
        s_abort = 1;
        atomicExch(&g_prefill_status, (int)KDA_ERR_TIMEOUT);
    };

    if (tid < NCH) {
        // =================================================== chain warpgroups ==
        // thread: state column j (tensor-memory lane), key rows [64 hh, 64 hh + 64)
        const int j = 32 * sp + lane;
        const int hh = warp >> 2;
        const uint32_t bar = smem_u32(&s_bar[0]);
        uint32_t phase = 0;
        // every thread waits on the MMA barrier itself (cheaper than a
        // hand-over through a named barrier)
        auto wait_mma = [&]() {
            if (!s_abort && !mbar_wait(bar, phase & 1u, wait_ns)) expired();
            ++phase;
            fence_after_sync();
        };
        uint32_t n_commit = 0;               // commits on `bar` issued by this (issuing) thread
        float S[D / 2];
        {
            const float* h0h = (h0 && !(flags & SEG_H0_EYE)) ? h0 + head_off * D * D : nullptr;
#pragma unroll
            for (int i = 0; i < D / 2; ++i)
                S[i] = (flags & SEG_H0_EYE) ? (64 * hh + i == j ? 1.f : 0.f)
                                            : (h0h ? h0h[(int64_t)(64 * hh + i) * D + j] : 0.f);
#pragma unroll
            for (int c0 = 0; c0 < D / 2; c0 += 32) {
                float t32[32];
#pragma unroll
                for (int i = 0; i < 32; ++i) t32[i] = to_tf32(S[c0 + i]);
                tmem_st32(tm + lane_base + T_AS + 64 * hh + c0, t32);
            }
            wait_st();
        }
        __nv_bfloat16* oh = o + base;
#pragma unroll 1
        for (int ch = 0; ch < n_chunks; ++ch) {
            fence_before_sync();
            named_bar(BAR_READY, NT);        // this chunk's operands are in place
            fence_after_sync();
            // X = S^T [W | Qt]^T  (one N = 64 MMA per K step; the issue loop is
            // unrolled with constant descriptor increments: the per-instruction
            // issue cost, not the math, bounds these small-N MMAs)
            if (warp == 0 && !warp_flag(s_abort)) {
                const uint32_t id = idesc_tf32(128, 2 * C, false, false);
                const uint64_t bd0 = sdesc(smem_u32(sm + B1), PAD_LBO, SBO_K128P);
#pragma unroll
                for (int ks = 0; ks < D / 8; ++ks)
                    mma_tf32_ts_w(tm + T_DX, tm + T_AS + ks * 8, bd0 + (uint64_t)((ks * 2 * PAD_LBO) >> 4),
                                  id, ks > 0 ? 1u : 0u);
                mma_commit_w(bar);
                ++n_commit;
            }
            wait_mma();
            {   // U = U' - W S  (this half: tokens [16 hh, 16 hh + 16))
                float x[16], up[16];
                tmem_ld16(tm + lane_base + T_DX + 16 * hh, x);
                tmem_ld16(tm + lane_base + T_DU + (ch & 1) * C + 16 * hh, up);
                wait_ld();
#pragma unroll
                for (int r = 0; r < 16; ++r) x[r] = to_tf32(up[r] - x[r]);
                tmem_st16(tm + lane_base + T_AU + 16 * hh, x);
                wait_st();
            }
            fence_before_sync();
            named_bar(BAR_CHAIN, NCH);
            fence_after_sync();
            if (warp == 0 && !warp_flag(s_abort)) {
                const uint32_t id2 = idesc_tf32(128, 128, false, false);
                const uint32_t id3 = idesc_tf32(128, 32, false, false);
                const uint64_t b20 = sdesc(smem_u32(sm + B2), LBO, SBO_K32);
                const uint64_t b30 = sdesc(smem_u32(sm + B3), PAD_LBO, SBO_K32P);
#pragma unroll
                for (int ks = 0; ks < C / 8; ++ks) {
                    mma_tf32_ts_w(tm + T_DKU, tm + T_AU + ks * 8, b20 + (uint64_t)((ks * 2 * LBO) >> 4),
                                  id2, ks > 0 ? 1u : 0u);
                    mma_tf32_ts_w(tm + T_DX + C, tm + T_AU + ks * 8, b30 + (uint64_t)((ks * 2 * PAD_LBO) >> 4),
                                  id3, 1u);
                }
                mma_commit_w(bar);
                ++n_commit;
            }
            wait_mma();
            // B1, B2, B3 are no longer read: the prep may fill the next chunk's
            // while the state update and the output store run
            if (ch + 1 < n_chunks) named_arrive(BAR_FREE, NT);
            {   // S <- Diag(gamma_C) S + Kb^T U ; refresh the tf32 copy; emit o
                const float4* gam4 = reinterpret_cast<const float4*>(sm + GAM + (ch & 1) * D * 4) + 16 * hh;
#pragma unroll
                for (int c0 = 0; c0 < D / 2; c0 += 16) {
                    float d[16];
                    tmem_ld16(tm + lane_base + T_DKU + 64 * hh + c0, d);
                    wait_ld();
#pragma unroll
                    for (int i4 = 0; i4 < 4; ++i4) {
                        const float4 gv = gam4[(c0 >> 2) + i4];
                        const float gg[4] = {gv.x, gv.y, gv.z, gv.w};
#pragma unroll
                        for (int u = 0; u < 4; ++u) {
                            const int i = c0 + i4 * 4 + u;
                            S[i] = fmaf(gg[u], S[i], d[i - c0]);
                            d[i - c0] = to_tf32(S[i]);
                        }
                    }
                    tmem_st16(tm + lane_base + T_AS + 64 * hh + c0, d);
                }
                if (float* snap = snapshot_slot(states, snap_every, ts / C + ch, T, b, H, h)) {
#pragma unroll
                    for (int i = 0; i < D / 2; ++i) snap[(int64_t)(64 * hh + i) * D + j] = S[i];
                }
                // o: this half's 16 tokens of column j into shared memory, then
                // whole rows to global memory in 16-byte vectors
                __nv_bfloat16* ost = reinterpret_cast<__nv_bfloat16*>(sm + OST);
                {
                    float ov[16];
                    tmem_ld16(tm + lane_base + T_DX + C + 16 * hh, ov);
                    wait_ld();
#pragma unroll
                    for (int r = 0; r < 16; ++r) ost[(16 * hh + r) * D + j] = __float2bfloat16_rn(ov[r]);
                }
                wait_st();
                named_bar(BAR_CHAIN, NCH);
                const int tb = ch * C;
#pragma unroll
                for (int m = 0; m < (C * D / 8) / NCH; ++m) {
                    const int vi = tid + m * NCH;
                    const int r = vi / (D / 8), cv = vi % (D / 8);
                    if (tb + r < Tl && !(flags & SEG_NO_O))
                        *reinterpret_cast<uint4*>(oh + (int64_t)(tb + r) * row_stride + cv * 8) =
                            *reinterpret_cast<const uint4*>(ost + r * D + cv * 8);
                }
                named_bar(BAR_CHAIN, NCH);   // staging read before the next chunk writes it
            }
        }
        if (hT && !s_abort) {
            float* hTh = hT + head_off * D * D;
#pragma unroll
            for (int i = 0; i < D / 2; ++i) hTh[(int64_t)(64 * hh + i) * D + j] = S[i];
        }
        // After an expired wait, the MMAs of the last commit may still run:
        // let them finish before tensor memory is released (the issuing thread
        // is also the waiting thread, so at most one commit is outstanding).
        if (tid == 0 && *(volatile int*)&s_abort && n_commit > 0)
            mbar_wait(bar, (n_commit - 1) & 1u, DRAIN_NS);
    } else {
        // ==================================================== prep warpgroups ==
        const int pt = tid - NCH;                  // 0..255
        const int pw = pt >> 5;                    // prep warp 0..7
        const uint32_t bar = smem_u32(&s_bar[1]);
        const uint32_t rbar = smem_u32(&s_bar[2]);
        uint32_t phase = 0, rphase = 0;
        uint32_t n_commit = 0, n_loads = 0;    // issued by pt == 0 (also the waiting thread)
        auto wait_mma = [&]() {
            if (!s_abort && !mbar_wait(bar, phase & 1u, wait_ns)) expired();
            ++phase;
            fence_after_sync();
        };
        auto prep_sync = [&]() { named_bar(BAR_PREP, NPREP); };
        // TMA: chunk ci's q, k, v, g rows (32 x 128 bf16 each; rows past T are zero);
        // none after an expired wait (the raw buffer may still be in use)
        // (with v = 0, the transition pass of the segment scan, v is not loaded)
        const bool load_v = !(flags & SEG_V_ZERO);
        auto issue_raw = [&](int ci) {
            if (pt == 0 && !*(volatile int*)&s_abort) {
                ++n_loads;
                mbar_arrive_expect_tx(rbar, (load_v ? 4 : 3) * RAW_T);
                tma_load_3d(smem_u32(sm + RAW + 0 * RAW_T), &tm_q, h * D, ts + ci * C, b, rbar);
                tma_load_3d(smem_u32(sm + RAW + 1 * RAW_T), &tm_k, h * D, ts + ci * C, b, rbar);
                if (load_v) tma_load_3d(smem_u32(sm + RAW + 2 * RAW_T), &tm_v, h * D, ts + ci * C, b, rbar);
                tma_load_3d(smem_u32(sm + RAW + 3 * RAW_T), &tm_g, h * D, ts + ci * C, b, rbar);
            }
        };
        if (n_chunks > 0) issue_raw(0);
        // beta one chunk ahead, kept as raw bf16 bits until it is stored (a
        // conversion right after the load would stall on the load)
        const __nv_bfloat16 bzero = __float2bfloat16_rn(0.f);
        __nv_bfloat16 beta_next = (pt < C && pt < Tl) ? beta[((int64_t)b * T + ts + pt) * H + h] : bzero;

        // decay-scaling slice of this thread: tile tau, key channel c
        const int tau = pt >> 7;
        const int c = pt & 127;
        float* am = reinterpret_cast<float*>(sm + AMS);
        float* pm = reinterpret_cast<float*>(sm + PMS);
        float* xm = reinterpret_cast<float*>(sm + XMS);
        float* tmx = reinterpret_cast<float*>(sm + TMS);
        float* ym = reinterpret_cast<float*>(sm + YMS);
        const float* bt = reinterpret_cast<const float*>(sm + BETA);
#pragma unroll 1
        for (int ch = 0; ch < n_chunks; ++ch) {
            // ---- inputs of this chunk (beta prefetched one chunk ahead)
            if (pt < C) {
                reinterpret_cast<float*>(sm + BETA)[pt] = to_f32(beta_next);
                const int tn = (ch + 1) * C + pt;
                beta_next = (tn < Tl) ? beta[((int64_t)b * T + ts + tn) * H + h] : bzero;
            }
            if (pt == 0 && !s_abort && !mbar_wait(rbar, rphase & 1u, wait_ns)) expired();
            ++rphase;
            __syncwarp();
            prep_sync();

            // ---- decay scaling (thread: 16 tokens of tile tau, channel c)
            float gam_c, fq, fk;                    // chunk-relative factors for the fill
            float vr[TILE];
            {
                const __nv_bfloat16* __restrict__ rq = reinterpret_cast<const __nv_bfloat16*>(sm + RAW + 0 * RAW_T);
                const __nv_bfloat16* __restrict__ rk = reinterpret_cast<const __nv_bfloat16*>(sm + RAW + 1 * RAW_T);
                const __nv_bfloat16* __restrict__ rv = reinterpret_cast<const __nv_bfloat16*>(sm + RAW + 2 * RAW_T);
                const __nv_bfloat16* __restrict__ rg = reinterpret_cast<const __nv_bfloat16*>(sm + RAW + 3 * RAW_T);
                // every shared-memory read of the slice first: later loads would
                // otherwise be ordered behind the operand stores
                float a[TILE], kr[TILE], qr[TILE];
#pragma unroll
                for (int rr = 0; rr < TILE; ++rr) {
                    const int idx = (tau * TILE + rr) * D + c;
                    kr[rr] = to_f32(rk[idx]);
                    qr[rr] = to_f32(rq[idx]);
                    vr[rr] = (flags & SEG_V_ZERO) ? 0.f : to_f32(rv[idx]);
                    a[rr] = to_f32(rg[idx]);
                }
                if constexpr (PRO) prologue_gate_and_norms(a, qr, kr, ch * C + tau * TILE, Tl,
                                                            reinterpret_cast<float*>(sm + NRM), tau, c);
                float e = 1.f;
#pragma unroll
                for (int rr = 0; rr < TILE; ++rr) {
                    a[rr] = __expf(a[rr]);
                    e *= a[rr];
                }
                float* gex = reinterpret_cast<float*>(sm + GEX);
                gex[tau * D + c] = e;
                prep_sync();
                if constexpr (PRO) prologue_normalise(qr, kr, reinterpret_cast<const float*>(sm + NRM), tau);
                const float oe = gex[(1 - tau) * D + c];
                const float f = tau ? oe : 1.f;          // chunk-relative factor of tile 1 rows
                gam_c = e * oe;
                fq = f;
                fk = tau ? e : oe;                       // Kb (chunk) from the stored Kh (tile 1) or Kb_0 (tile 0)
                // forward: Kt, Qt (tile-relative) for the Gram; Kt (chunk) for W
                float p = 1.f;
                float kc[4];
#pragma unroll
                for (int rr = 0; rr < TILE; ++rr) {
                    const int r = tau * TILE + rr;
                    p *= a[rr];
                    const float kt = kr[rr] * p;
                    const float qt = qr[rr] * p;
                    st_f32(sm, GB + off_kmajor(r, c, PAD_LBO, SBO_K128P), to_tf32(kt));
                    st_f32(sm, GB + off_kmajor(C + r, c, PAD_LBO, SBO_K128P), qt);   // full fp32: see below
                    kc[rr & 3] = to_tf32(kt * f);
                    if ((rr & 3) == 3)
                        st_f32x4(sm, WA + off_kmajor(c, r - 3, LBO, SBO_K32), kc[0], kc[1], kc[2], kc[3]);
                }
                // backward: Kb (tile-relative suffix) and Kh = Kb / gamma_tile
                const float inv = 1.f / e;
                float sgm = 1.f;
#pragma unroll
                for (int rr = TILE - 1; rr >= 0; --rr) {
                    const int r = tau * TILE + rr;
                    const float kb = kr[rr] * sgm;
                    // Qt (above), Kh and Kb_0 stay in full fp32: the operand fill
                    // rescales them into the chunk-relative Qt and Kb and rounds
                    // to tf32 once (rounding here too would round those twice);
                    // the Gram MMA reads the rows as tf32 (low mantissa bits
                    // ignored).
                    st_f32(sm, GA + off_kmajor(r, c, PAD_LBO, SBO_K128P), kb * inv);
                    if (tau == 0) st_f32(sm, GA + off_kmajor(C + rr, c, PAD_LBO, SBO_K128P), kb);
                    sgm *= a[rr];
                }
            }
            fence_smem_to_async();
            fence_before_sync();
            prep_sync();                     // raw buffer consumed, Gram operands written
            fence_after_sync();
            // ---- Gram: D_G = [Kh_0; Kh_1; Kb_0; pad] [Kt_0 Kt_1 | Qt_0 Qt_1]^T,
            // and the next chunk's inputs; V^T is written while the MMA runs
            if (pw == 0 && !warp_flag(s_abort)) {
                const uint32_t id = idesc_tf32(64, 64, false, false);
                const uint64_t ad0 = sdesc(smem_u32(sm + GA), PAD_LBO, SBO_K128P);
                const uint64_t bd0 = sdesc(smem_u32(sm + GB), PAD_LBO, SBO_K128P);
#pragma unroll
                for (int ks = 0; ks < D / 8; ++ks) {
                    const uint64_t step = (uint64_t)((ks * 2 * PAD_LBO) >> 4);
                    mma_tf32_ss_w(tm + T_DG, ad0 + step, bd0 + step, id, ks > 0 ? 1u : 0u);
                }
                mma_commit_w(bar);
                ++n_commit;
            }
            if (ch + 1 < n_chunks) issue_raw(ch + 1);
#pragma unroll
            for (int rr = 0; rr < TILE; rr += 4)
                st_f32x4(sm, VA + off_kmajor(c, tau * TILE + rr, LBO, SBO_K32),
                         to_tf32(vr[rr]), to_tf32(vr[rr + 1]), to_tf32(vr[rr + 2]), to_tf32(vr[rr + 3]));
            fence_smem_to_async();
            wait_mma();

            // ---- A and P (32 x 32) from the Gram (row m of D_G is lane
            // (m % 16) + 32 (m / 16)).  Sub-partition 0 holds the rows Kh_0
            // (columns Kt_0, Qt_0), 1 the rows Kh_1 (Kt_1, Qt_1), 2 the rows
            // Kb_0 (Kt_1, Qt_1: the blocks between the tiles).  Warps 0-2
            // take the A columns, warps 4-6 the P columns.  The warp that
            // holds a diagonal block of A also solves it, X = (I + A_tt)^-1,
            // column i per lane, right-looking, from A_tt^T in shared memory
            // (one 16-float column per step, read as four vectors).
            {
                const int spx = pw & 3;
                if (spx < 3) {
                    const bool is_p = pw >= 4;
                    const int colK = (spx == 0) ? 0 : TILE;
                    float gv[16];
                    tmem_ld16(tm + lane_base + T_DG + (is_p ? C : 0) + colK, gv);
                    wait_ld();
                    const int i = (spx == 1 ? TILE : 0) + lane;           // column of A / P
                    const int rbase = (spx == 0) ? 0 : TILE;              // rows covered
                    float* atm = reinterpret_cast<float*>(sm + ATM);
                    if (lane < TILE) {
                        if (is_p) {
#pragma unroll
                            for (int r = 0; r < TILE; ++r) {
                                const int rg = rbase + r;
                                pm[rg * LD + i] = (rg >= i) ? gv[r] : 0.f;
                            }
                            if (spx == 1) {                               // P_01 = 0
#pragma unroll
                                for (int r = 0; r < TILE; ++r) pm[r * LD + i] = 0.f;
                            }
                        } else if (spx == 2) {                            // A_10, all below the diagonal
#pragma unroll
                            for (int r = 0; r < TILE; ++r) am[(TILE + r) * LD + i] = bt[TILE + r] * gv[r];
                        } else {                                          // column i of A_tt into row i of A^T
#pragma unroll
                            for (int r = 0; r < TILE; r += 4) {
                                float e4[4];
#pragma unroll
                                for (int u = 0; u < 4; ++u) {
                                    const int rg = rbase + r + u;
                                    e4[u] = (rg > i) ? bt[rg] * gv[r + u] : 0.f;
                                }
                                *reinterpret_cast<float4*>(atm + i * LDT + rbase + r) =
                                    make_float4(e4[0], e4[1], e4[2], e4[3]);
                            }
                        }
                    }
                    if (!is_p && spx < 2) {
                        __syncwarp();
                        if (lane < TILE) {
                            const int off = spx * TILE;
                            float x[TILE];
#pragma unroll
                            for (int r = 0; r < TILE; ++r) x[r] = (r == lane) ? 1.f : 0.f;
#pragma unroll
                            for (int s2 = 0; s2 < TILE; ++s2) {
                                const float4* col = reinterpret_cast<const float4*>(atm + (off + s2) * LDT + off);
                                float a16[TILE];
#pragma unroll
                                for (int q4 = 0; q4 < TILE / 4; ++q4) {
                                    const float4 v4 = col[q4];
                                    a16[4 * q4] = v4.x; a16[4 * q4 + 1] = v4.y;
                                    a16[4 * q4 + 2] = v4.z; a16[4 * q4 + 3] = v4.w;
                                }
#pragma unroll
                                for (int r = s2 + 1; r < TILE; ++r) x[r] = fmaf(-a16[r], x[s2], x[r]);
                            }
                            const float bi = bt[off + lane];
#pragma unroll
                            for (int r = 0; r < TILE; ++r) {
                                xm[(off + r) * LD + off + lane] = x[r];
                                tmx[(off + r) * LD + off + lane] = x[r] * bi;     // T_tt = X_tt diag(b)
                                if (spx == 1) tmx[r * LD + off + lane] = 0.f;     // T_01 = 0
                            }
                        }
                    }
                }
            }
            prep_sync();
            // ---- off-diagonal block: T_10 = -X_11 (A_10 X_00) diag(b_0)
            {
                const int r = pt >> 4, i = pt & 15;
                float y = 0.f;
#pragma unroll
                for (int s2 = 0; s2 < TILE; ++s2) y = fmaf(am[(TILE + r) * LD + s2], xm[s2 * LD + i], y);
                ym[r * (TILE + 1) + i] = y;
            }
            prep_sync();
            {
                const int r = pt >> 4, i = pt & 15;
                float z = 0.f;
#pragma unroll
                for (int s2 = 0; s2 < TILE; ++s2) z = fmaf(xm[(TILE + r) * LD + TILE + s2], ym[s2 * (TILE + 1) + i], z);
                tmx[(TILE + r) * LD + i] = -z * bt[i];
            }
            prep_sync();
            // ---- T into the B operand of the W / U' products: element (n = r, k = i)
            {
                const int r = pt >> 3, i = (pt & 7) * 4;
                const float* row = tmx + r * LD + i;
                st_f32x4(sm, TB + off_kmajor(r, i, PAD_LBO, SBO_K32P),
                         to_tf32(row[0]), to_tf32(row[1]), to_tf32(row[2]), to_tf32(row[3]));
            }
            fence_smem_to_async();
            fence_before_sync();
            prep_sync();
            fence_after_sync();
            // ---- W^T = Kt^T T^T and U'^T = V^T T^T  (M 128, N 32, K 32)
            if (pw == 0 && !warp_flag(s_abort)) {
                const uint32_t id = idesc_tf32(128, 32, false, false);
                const uint64_t bd0 = sdesc(smem_u32(sm + TB), PAD_LBO, SBO_K32P);
                const uint64_t aw0 = sdesc(smem_u32(sm + WA), LBO, SBO_K32);
                const uint64_t av0 = sdesc(smem_u32(sm + VA), LBO, SBO_K32);
                const uint32_t du = tm + T_DU + (ch & 1) * C;
#pragma unroll
                for (int ks = 0; ks < C / 8; ++ks) {
                    const uint64_t bstep = (uint64_t)((ks * 2 * PAD_LBO) >> 4);
                    const uint64_t astep = (uint64_t)((ks * 2 * LBO) >> 4);
                    mma_tf32_ss_w(tm + T_DW, aw0 + astep, bd0 + bstep, id, ks > 0 ? 1u : 0u);
                    mma_tf32_ss_w(du, av0 + astep, bd0 + bstep, id, ks > 0 ? 1u : 0u);
                }
                mma_commit_w(bar);
                ++n_commit;
            }
            // operands of the fill that do not come from the W MMA, read now
            const float* gaf = reinterpret_cast<const float*>(sm + GA);
            const float* gbf = reinterpret_cast<const float*>(sm + GB);
            float qf[TILE], kf[TILE];
#pragma unroll
            for (int rr = 0; rr < TILE; ++rr) {
                const int r = tau * TILE + rr;
                qf[rr] = to_tf32(gbf[off_kmajor(C + r, c, PAD_LBO, SBO_K128P) >> 2] * fq);
                const int row = tau ? (TILE + rr) : (C + rr);
                kf[rr] = to_tf32(gaf[off_kmajor(row, c, PAD_LBO, SBO_K128P) >> 2] * fk);
            }
            float pf4[4];
            {
                const int r = pt >> 3, i = (pt & 7) * 4;
#pragma unroll
                for (int u = 0; u < 4; ++u) pf4[u] = to_tf32(pm[r * LD + i + u]);
            }
            wait_mma();
            float w[16];
            tmem_ld16(tm + lane_base + T_DW + 16 * tau, w);
            wait_ld();

            // ---- hand the chunk's operands to the chain
            if (ch > 0) {
                fence_before_sync();
                named_bar(BAR_FREE, NT);     // the chain no longer reads B1, B2, B3
                fence_after_sync();
            }
            {
                // W (key channel c = TMEM lane, tokens [16 tau, 16 tau + 16)): rows 0-31 of B1
#pragma unroll
                for (int r = 0; r < 16; ++r)
                    st_f32(sm, B1 + off_kmajor(16 * tau + r, c, PAD_LBO, SBO_K128P), to_tf32(w[r]));
                // Qt (chunk-relative): rows 32-63 of B1; Kb (chunk-relative): B2
#pragma unroll
                for (int rr = 0; rr < TILE; ++rr)
                    st_f32(sm, B1 + off_kmajor(C + tau * TILE + rr, c, PAD_LBO, SBO_K128P), qf[rr]);
#pragma unroll
                for (int rr = 0; rr < TILE; rr += 4)
                    st_f32x4(sm, B2 + off_kmajor(c, tau * TILE + rr, LBO, SBO_K32),
                             kf[rr], kf[rr + 1], kf[rr + 2], kf[rr + 3]);
                // P: element (n = r, k = i)
                {
                    const int r = pt >> 3, i = (pt & 7) * 4;
                    st_f32x4(sm, B3 + off_kmajor(r, i, PAD_LBO, SBO_K32P), pf4[0], pf4[1], pf4[2], pf4[3]);
                }
                if (tau == 0) reinterpret_cast<float*>(sm + GAM + (ch & 1) * D * 4)[c] = gam_c;
            }
            fence_smem_to_async();
            fence_before_sync();
            named_arrive(BAR_READY, NT);
        }
        // after an expired wait: the last MMAs and input load may still be in
        // flight; let them land before tensor and shared memory are released
        if (pt == 0 && *(volatile int*)&s_abort) {
            if (n_commit > 0) mbar_wait(bar, (n_commit - 1) & 1u, DRAIN_NS);
            if (n_loads > 0) mbar_wait(rbar, (n_loads - 1) & 1u, DRAIN_NS);
        }
    }

    fence_before_sync();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tm, TMEM_COLS);
    if (*(volatile int*)&s_abort)
        poison_head_outputs(o ? o + base : nullptr, row_stride, Tl, o && !(flags & SEG_NO_O),
                            hT ? hT + head_off * D * D : nullptr, tid, NT);
}

// ============================================================================
// Cluster variant for few heads (B * H small next to the SM count): each head
// gets a cluster of four CTAs on four SMs.  Role 0 (the CTA of cluster rank
// CHAIN_RANK) runs the chain; roles 1-3 prepare the chunks ch with
// ch % 3 == role - 1, each in its own SM, and push every prepared chunk (the
// chain's operands and U') into slot ch % 3 of the chain CTA's shared memory
// with a single bulk copy (shared::cta -> shared::cluster, no multicast).
// FULL[slot] (chain CTA) counts the copy's bytes and is armed by the chain CTA
// itself when it hands the slot back; EMPTY (the preparing CTA) is arrived on
// by the chain CTA once the chunk's MMAs are done and its decay applied.  o of
// a chunk is staged one chunk late, while the next chunk's first MMA runs, in
// one of two buffers (one in the tf32 instantiation), and written by a tensor
// store.  The arithmetic is the
// one of prefill_tc_kernel, except that the chain's three products
// (S^T [W | Qt]^T, Kb^T U, P U) and the preparers' WY products (T Kt, T V)
// take fp16 operands (kind::f16, K = 16 per MMA): fp16 keeps tf32's 10-bit
// significand, and these operands are bounded
// (|Qt|, |Kb|, |P| <= 1 for unit-norm q and k; S, W and U of the order of h0
// and v), far inside fp16's range (65504).  Half as many MMAs per chunk, and
// half the slot bytes for those operands.  fp16's range is the price: entries
// below 2^-14 lose significand bits (2^-24 absolute), so a state whose scale
// is itself tiny would lose relative accuracy.  The transition pass of the
// segment scan (state from I, v = 0, decaying towards zero, whose relative
// accuracy is tested) therefore runs the same kernel with tf32 operands.
namespace pc {
using namespace pf;
constexpr int NCW = 256;                                      // compute threads per CTA (both roles)
constexpr int NX = NCW + 32;                                  // compute warps + one helper warp (hand-overs)
constexpr int NTH = NCW + 64;                                 // plus an issuer warp and a remote-traffic warp
// named barriers (0 is __syncthreads): issuer hand-overs and compute-warp syncs
constexpr uint32_t NB_ASA = 1, NB_ASB = 2, NB_U = 3;                           // chain CTA
constexpr uint32_t NB_CW = 4;                                                  // compute-warp syncs
constexpr uint32_t NB_G = 5, NB_TB = 6, NB_STFREE = 7, NB_FILL = 8;              // preparing CTAs
constexpr int NPREPCTA = 3;                                   // preparing CTAs per cluster (= slots)
// Cluster rank of the chain CTA; the preparing CTAs follow it cyclically.
// A cluster of four occupies two TPCs (ranks 0-1 and 2-3).  With the chain on
// rank 0 the slots of some clusters streamed in too slowly (up to 20 % longer
// per chunk, depending on where the cluster was placed); with the chain on
// the second TPC every cluster kept pace (measured on the 8K workload).
constexpr uint32_t CHAIN_RANK = 2;
constexpr uint32_t OST_BYTES = C * D * 2;                      // o staging of one chunk (32 x 128 bf16)
constexpr uint32_t C_SLOT0 = 0;
// roles 1-3 (preparation): the fixed part of the layout
constexpr uint32_t P_RAW = 0;
constexpr uint32_t P_BETA = P_RAW + 4 * RAW_T;
constexpr uint32_t P_GEX = P_BETA + C * 4;
constexpr uint32_t P_GA = P_GEX + 2 * D * 4;
constexpr uint32_t P_GB = P_GA + 6 * SBO_K128P;
constexpr uint32_t P_WA = P_GB + 8 * SBO_K128P;
constexpr uint32_t P_VA = P_WA + (D / 8) * SBO_K32;
constexpr uint32_t P_TB = P_VA + (D / 8) * SBO_K32;
constexpr uint32_t P_ST = P_TB + (C / 8) * SBO_K32P;           // staging of one slot
constexpr int ATM_LD = 16;     // row stride (floats) of a transposed 16 x 16 diagonal block of A (16-byte rows)
static_assert(P_ST % 16 == 0 && P_GA % 16 == 0 && P_GB % 16 == 0 && P_WA % 16 == 0 && P_VA % 16 == 0 &&
              P_TB % 16 == 0, "alignment");
// The operands of the chain's three products, fp16 (H) or tf32, K-major:
// the slot layout (identical in role 0's slots and a preparer's staging) and
// everything that depends on its size.  fp16 is the default; the transition
// pass of the segment scan (state from I, v = 0) takes tf32, because its
// states shrink towards fp16's subnormal range while their relative accuracy
// is still wanted.
template <bool H> struct Chain {
    static constexpr int KSTEP = H ? 16 : 8;                             // K per MMA
    static constexpr uint32_t SBO_B1 = H ? (D / 8) * PAD_LBO : SBO_K128P;  // [W | Qt], K = 128, padded
    static constexpr uint32_t SBO_B23 = H ? (C / 8) * LBO : SBO_K32;       // Kb, P: K = 32, dense
    static constexpr uint32_t S_B1 = 0;                                  // [W | Qt]: N 64 x K 128
    static constexpr uint32_t S_B2 = S_B1 + 8 * SBO_B1;                  // Kb: N 128 x K 32
    static constexpr uint32_t S_B3 = S_B2 + (D / 8) * SBO_B23;           // P: N 32 x K 32
    static constexpr uint32_t S_GAM = S_B3 + (C / 8) * SBO_B23;          // gamma_C, 128 fp32
    static constexpr uint32_t S_UP = S_GAM + D * 4;                      // U' [32 tokens][128] fp32
    static constexpr uint32_t SLOT = S_UP + C * D * 4;                   // bytes per chunk
    // role 0: NPREPCTA slots, then NOST o staging buffers (two fit next to
    // fp16 slots, one next to tf32 slots)
    static constexpr int NOST = H ? 2 : 1;
    static constexpr uint32_t C_OST = NPREPCTA * SLOT;
    static constexpr uint32_t C_BYTES = C_OST + NOST * OST_BYTES;
    // roles 1-3: the staging of one slot, then the solve's scratch
    static constexpr uint32_t P_AMS = P_ST + SLOT;
    static constexpr uint32_t P_PMS = P_AMS + C * LD * 4;
    static constexpr uint32_t P_XMS = P_PMS + C * LD * 4;
    static constexpr uint32_t P_TMS = P_XMS + C * LD * 4;
    static constexpr uint32_t P_YMS = P_TMS + C * LD * 4;
    static constexpr uint32_t P_NRM = P_YMS + TILE * (TILE + 1) * 4;   // prologue: per-warp squared norms
    static constexpr uint32_t P_BYTES = P_NRM + NRM_BYTES;
    // A^T of the two diagonal blocks, used only between the Gram MMA and the
    // diagonal solve: it shares the bytes of YMS and NRM (YMS is written after
    // the solve, NRM is used before the Gram MMA), which keeps the tf32
    // layout inside the shared-memory budget
    static constexpr uint32_t P_ATM = P_YMS;
    static_assert(2 * TILE * ATM_LD * 4 <= TILE * (TILE + 1) * 4 + NRM_BYTES, "A^T fits YMS and NRM");
    static constexpr uint32_t SMEM_BYTES = P_BYTES > C_BYTES ? P_BYTES : C_BYTES;
    static_assert(SMEM_BYTES <= 227 * 1024, "shared memory budget");
    static_assert(SLOT % 16 == 0 && P_ATM % 16 == 0, "bulk copy size, vector rows");
    static_assert(C_OST % 128 == 0 && OST_BYTES % 128 == 0, "tensor store source alignment");
};
// tensor memory: role 0 uses 416 columns (512 allocated), roles 1-3 use 128
constexpr uint32_t CT_AS = 0, CT_AU = 128, CT_DX0 = 160, CT_DKU = 224, CT_DX1 = 352;
constexpr uint32_t PT_DG = 0, PT_DW = 64, PT_DU = 96;
}  // namespace pc

// PRO: the fused prologue (launch flag PROLOGUE); F16: fp16 chain operands
template <bool PRO, bool F16>
__global__ void __cluster_dims__(pc::NPREPCTA + 1, 1, 1) __launch_bounds__(pc::NTH, 1)
prefill_cluster_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                       const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_g,
                       const __grid_constant__ CUtensorMap tm_o,
                       const __nv_bfloat16* __restrict__ beta, const float* h0,
                       __nv_bfloat16* __restrict__ o, float* hT, int T, int H,
                       int seg_len, int n_seg, uint32_t flags, float* states, int snap_every,
                       uint64_t wait_ns)
{
    using namespace pc;
    using namespace tc;
    using CH = Chain<F16>;
    constexpr uint32_t S_B1 = CH::S_B1, S_B2 = CH::S_B2, S_B3 = CH::S_B3, S_GAM = CH::S_GAM, S_UP = CH::S_UP;
    constexpr uint32_t SLOT = CH::SLOT, C_OST = CH::C_OST;
    constexpr int NOST = CH::NOST;
    constexpr uint32_t P_AMS = CH::P_AMS, P_PMS = CH::P_PMS, P_XMS = CH::P_XMS, P_TMS = CH::P_TMS,
                       P_YMS = CH::P_YMS, P_NRM = CH::P_NRM, P_ATM = CH::P_ATM;
    // the chain's MMAs: kind::f16 or kind::tf32 by the operand type
    auto mma_chain = [](uint32_t d, uint32_t a_tmem, uint64_t b_desc, uint32_t id, uint32_t acc) {
        if constexpr (F16) mma_f16_ts_w(d, a_tmem, b_desc, id, acc);
        else mma_tf32_ts_w(d, a_tmem, b_desc, id, acc);
    };
    auto idesc_chain = [](int M, int N) -> uint32_t {
        if constexpr (F16) return idesc_f16(M, N);
        else return idesc_tf32(M, N, false, false);
    };
    extern __shared__ __align__(1024) unsigned char sm[];
    __shared__ uint32_t s_taddr;
    __shared__ __align__(8) uint64_t s_bar[8];   // role 0: FULL[0..2], X, KU0, KU1, o staged[0..1]; roles 1-3: EMPTY, MMA, input loads
    __shared__ int s_abort;
    __shared__ uint32_t s_odone;                 // role 0: chunks whose slot is consumed
    __shared__ uint32_t s_full;                  // role 0: chunks whose slot has landed (FULL observed)
    __shared__ uint32_t s_ofree;                 // role 0: chunks whose o store has read the staging
    __shared__ int s_last_armed[NPREPCTA];       // role 0: last chunk whose bytes FULL[slot] expects

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    // role: 0 = chain, 1..3 = preparing CTA (the cluster rank shifted by CHAIN_RANK)
    const uint32_t role = (cluster_ctarank() + 4u - CHAIN_RANK) & 3u;
    // grid.y = B * n_seg: sequence b, segment [ts, ts + Tl) of it (n_seg = 1: the whole sequence)
    const int h = blockIdx.x / (NPREPCTA + 1), bb = blockIdx.y;
    const int b = bb / n_seg;
    const int ts = (bb - b * n_seg) * seg_len;
    const int Tl = max(0, min(seg_len, T - ts));
    const int64_t head_off = (int64_t)bb * H + h;          // h0 / hT: [B * n_seg][H][D][D]
    const int n_chunks = (Tl + C - 1) / C;
    const uint32_t ncols = role == 0 ? 512u : 128u;
    const bool store_o = o != nullptr && !(flags & SEG_NO_O);    // o rows go out by tensor stores

    if (warp == 0) {
        tmem_alloc(smem_u32(&s_taddr), ncols);
        tmem_relinquish();
    }
    if (tid == 0) {
        for (int i = 0; i < 6; ++i) mbar_init(smem_u32(&s_bar[i]), 1);
        mbar_init(smem_u32(&s_bar[6]), NCW / 32);    // one arrive per compute warp
        mbar_init(smem_u32(&s_bar[7]), NCW / 32);
        fence_mbar_init();
        s_abort = 0;
        s_odone = 0;
        s_full = 0;
        s_ofree = 0;
        // role 0: FULL[s] expects the bytes of chunk s's push; later uses are
        // armed when the slot is released (the push itself carries no arrive)
        for (int i = 0; i < NPREPCTA; ++i) s_last_armed[i] = -1;
        if (role == 0)
            for (int i = 0; i < NPREPCTA && i < n_chunks; ++i) {
                mbar_arrive_expect_tx(smem_u32(&s_bar[i]), SLOT);
                s_last_armed[i] = i;
            }
    }
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    cluster_sync();                    // every CTA's barriers exist before any remote arrive
    const uint32_t tm = s_taddr;
    const int sp = warp & 3;
    const uint32_t lane_base = (uint32_t)(32 * sp) << 16;
    auto expired = [&]() {
        s_abort = 1;
        atomicExch(&g_prefill_status, (int)KDA_ERR_TIMEOUT);
    };

    if (role == 0) {
        // ========================================================= chain CTA ==
        const uint32_t mbar = smem_u32(&s_bar[3]);   // X of each chunk
        const uint32_t kbar0 = smem_u32(&s_bar[4]);  // Kb^T U, d_k columns [0, 64)
        const uint32_t kbar1 = smem_u32(&s_bar[5]);  // Kb^T U, d_k columns [64, 128), and P U
        if (warp == NCW / 32) {
            // ------------------------------------------------------ issuer warp --
            // Chunk ch: X = S^T [W | Qt]^T in two d_k halves (each as soon as
            // the compute warps have written that half of the tf32 state), then,
            // once U is in tensor memory, Kb^T U by d_k halves (one commit each,
            // so the next state update starts on the first half) and P U.
            // With fp16 operands (kind::f16, K = 16 per MMA) the state S^T and
            // U^T sit in tensor memory as packed pairs; either way an MMA reads
            // 8 tensor-memory columns of A and two K-adjacent core matrices of B.
            const uint32_t id1 = idesc_chain(128, 2 * C);
            const uint32_t id2 = idesc_chain(128, 64);
            const uint32_t id3 = idesc_chain(128, 32);
            constexpr int NKX = D / CH::KSTEP, NKU = C / CH::KSTEP;   // K steps of X and of Kb^T U, P U
            uint32_t n_x = 0, n_k0 = 0, n_k1 = 0;   // commits on mbar, kbar0, kbar1
#pragma unroll 1
            for (int ch = 0; ch < n_chunks; ++ch) {
                const int slot = ch % NPREPCTA;
                const uint32_t sb = C_SLOT0 + slot * SLOT;
                const uint32_t dx = (ch & 1) ? CT_DX1 : CT_DX0;
                const uint64_t bd0 = sdesc(smem_u32(sm + sb + S_B1), PAD_LBO, CH::SBO_B1);
                if (lane == 0 && !s_abort &&
                    !mbar_wait_cluster(smem_u32(&s_bar[slot]), (uint32_t)(ch / NPREPCTA) & 1u, wait_ns))
                    expired();
                __syncwarp();
                named_bar(NB_ASA, NX);
                fence_after_sync();
                if (!warp_flag(s_abort)) {
#pragma unroll
                    for (int ks = 0; ks < NKX / 2; ++ks)
                        mma_chain(tm + dx, tm + CT_AS + ks * 8, bd0 + (uint64_t)((ks * 2 * PAD_LBO) >> 4),
                                  id1, ks > 0 ? 1u : 0u);
                }
                __syncwarp();
                named_bar(NB_ASB, NX);
                fence_after_sync();
                if (!warp_flag(s_abort)) {
#pragma unroll
                    for (int ks = NKX / 2; ks < NKX; ++ks)
                        mma_chain(tm + dx, tm + CT_AS + ks * 8, bd0 + (uint64_t)((ks * 2 * PAD_LBO) >> 4),
                                  id1, 1u);
                    mma_commit_w(mbar);
                    ++n_x;
                }
                __syncwarp();
                named_bar(NB_U, NX);
                fence_after_sync();
                if (!warp_flag(s_abort)) {
                    // Kb rows [64, 128) start 8 core-matrix rows of SBO_K32 further
                    const uint64_t b20 = sdesc(smem_u32(sm + sb + S_B2), LBO, CH::SBO_B23);
                    const uint64_t b21 = sdesc(smem_u32(sm + sb + S_B2 + 8 * CH::SBO_B23), LBO, CH::SBO_B23);
                    const uint64_t b30 = sdesc(smem_u32(sm + sb + S_B3), LBO, CH::SBO_B23);
#pragma unroll
                    for (int ks = 0; ks < NKU; ++ks)
                        mma_chain(tm + CT_DKU, tm + CT_AU + ks * 8, b20 + (uint64_t)((ks * 2 * LBO) >> 4),
                                  id2, ks > 0 ? 1u : 0u);
                    mma_commit_w(kbar0);
                    ++n_k0;
#pragma unroll
                    for (int ks = 0; ks < NKU; ++ks)
                        mma_chain(tm + CT_DKU + 64, tm + CT_AU + ks * 8, b21 + (uint64_t)((ks * 2 * LBO) >> 4),
                                  id2, ks > 0 ? 1u : 0u);
#pragma unroll
                    for (int ks = 0; ks < NKU; ++ks)
                        mma_chain(tm + dx + C, tm + CT_AU + ks * 8, b30 + (uint64_t)((ks * 2 * LBO) >> 4),
                                  id3, 1u);
                    mma_commit_w(kbar1);
                    ++n_k1;
                }
                __syncwarp();
            }
            // after an expired wait: the last commit of each barrier (at most
            // one is outstanding: each is waited before the next is issued)
            // must complete before tensor memory is released
            if (lane == 0 && *(volatile int*)&s_abort) {
                if (n_x > 0) mbar_wait(mbar, (n_x - 1) & 1u, DRAIN_NS);
                if (n_k0 > 0) mbar_wait(kbar0, (n_k0 - 1) & 1u, DRAIN_NS);
                if (n_k1 > 0) mbar_wait(kbar1, (n_k1 - 1) & 1u, DRAIN_NS);
            }
            __syncwarp();
        } else if (warp == NCW / 32 + 1) {
            // ------------------------------------------------------ release warp --
            // Chunk ch: observe its slot's FULL phase (a cluster-scope acquire,
            // which costs a few hundred cycles) and publish that with a CTA
            // counter, so the compute warps, which read U' from the slot, pay
            // only a CTA-scope acquire on their path (publishing it from the
            // issuer, which waits on FULL too, put the release on the MMA path
            // and was slower).  Then, once chunk ch - 1's last MMAs are done (and
            // its decay applied), nothing reads its slot any more: hand it back
            // to its preparer.  A remote arrive is slow, so it stays off the
            // issuer's and the compute warps' path.  Completion comes from a
            // counter that the compute warps advance in order; a counter cannot
            // be misread by a reader that lags.
            // o of chunk cp, once the compute warps have staged it in buffer
            // cp % NOST: one tensor store (rows past T are clipped by the tensor
            // map), then the buffer is handed back as soon as the store has
            // read it (the compute warps refill it NOST chunks later).
            auto store_output = [&](int cp) {
                if (lane == 0) {
                    const uint32_t ob = (uint32_t)cp % NOST;
                    if (!s_abort && !mbar_wait(smem_u32(&s_bar[6 + ob]), ((uint32_t)cp / NOST) & 1u, wait_ns)) expired();
                    if (!*(volatile int*)&s_abort) {
                        tma_store_3d(&tm_o, h * D, ts + cp * C, b, smem_u32(sm + C_OST + ob * OST_BYTES));
                        bulk_commit();
                    }
                    bulk_wait_read_all();
                    counter_publish(smem_u32(&s_ofree), (uint32_t)cp + 1u);
                }
                __syncwarp();
            };
#pragma unroll 1
            for (int ch = 0; ch < n_chunks; ++ch) {
                if (lane == 0) {
                    if (!s_abort &&
                        !mbar_wait_cluster(smem_u32(&s_bar[ch % NPREPCTA]), (uint32_t)(ch / NPREPCTA) & 1u, wait_ns))
                        expired();
                    if (!*(volatile int*)&s_abort) counter_publish(smem_u32(&s_full), (uint32_t)ch + 1u);
                }
                __syncwarp();
                if (ch == 0) continue;
                if (lane == 0) {
                    if (!s_abort && !counter_wait(smem_u32(&s_odone), (uint32_t)ch, wait_ns)) expired();
                    // After an expired wait no slot is handed back (its previous
                    // bytes may still be on their way): the preparers then give up
                    // on their own bounded waits, and at most one push per slot is
                    // left to drain before the CTA exits.
                    if (!*(volatile int*)&s_abort) {
                        const int sl = (ch - 1) % NPREPCTA;
                        const int cn = ch - 1 + NPREPCTA;    // the chunk that will reuse this slot
                        if (cn < n_chunks) {
                            mbar_arrive_expect_tx(smem_u32(&s_bar[sl]), SLOT);
                            s_last_armed[sl] = cn;
                        }
                        mbar_arrive_remote_relaxed(map_to_rank(smem_u32(&s_bar[0]), (CHAIN_RANK + 1u + (uint32_t)sl) & 3u));
                    }
                }
                __syncwarp();
                if (store_o) store_output(ch - 1);
            }
            if (store_o && n_chunks > 0) store_output(n_chunks - 1);
            if (lane == 0) bulk_wait_all();   // every o store has landed (also after an expired wait)
            __syncwarp();
        } else {
            // ----------------------------------------------------- compute warps --
            // Per chunk ch: the state increment of chunk ch - 1 by d_k halves
            // (each half handed to the issuer as soon as it is in tensor
            // memory), the output of chunk ch - 1 (staged for a tensor store
            // while X of chunk ch is computed), then U = U' - W S, and the
            // decay S <- Diag(gamma_C) S while Kb^T U and P U run.  Chunk ch's
            // slot is then consumed and goes back to its preparer.
            const int j = 32 * sp + lane;                // dv row = TMEM lane
            const int hh = warp >> 2;                     // d_k columns [32 hh, +32) and [64 + 32 hh, +32)
            uint32_t phase = 0;
            // Every thread waits on the MMA barrier itself: a hand-over from one
            // polling thread through a named barrier costs a few hundred
            // cycles per wait on this path.
            auto wait_bar = [&](uint32_t bar, uint32_t parity) {
                if (!s_abort && !mbar_wait(bar, parity, wait_ns)) expired();
                fence_after_sync();
            };
            // S[32 q + i] holds d_k column 64 q + 32 hh + i of this thread's dv row.
            // The MMA copy of S^T: fp16 with two d_k columns per tensor-memory
            // column (d_k columns [64 q + 32 hh, +32) in packed columns
            // [32 q + 16 hh, +16) of CT_AS), or tf32 with one.
            float S[D / 2];
            auto put_state = [&](int q2) {
                if constexpr (F16) {
                    float hp[16];
#pragma unroll
                    for (int w = 0; w < 16; ++w) hp[w] = pack_f16x2(S[32 * q2 + 2 * w], S[32 * q2 + 2 * w + 1]);
                    tmem_st16(tm + lane_base + CT_AS + 32 * q2 + 16 * hh, hp);
                } else {
                    float t32[32];
#pragma unroll
                    for (int i = 0; i < 32; ++i) t32[i] = to_tf32(S[32 * q2 + i]);
                    tmem_st32(tm + lane_base + CT_AS + 64 * q2 + 32 * hh, t32);
                }
                wait_st();
            };
            {
                const float* h0h = (h0 && !(flags & SEG_H0_EYE)) ? h0 + head_off * D * D : nullptr;
#pragma unroll
                for (int q2 = 0; q2 < 2; ++q2) {
#pragma unroll
                    for (int i = 0; i < 32; ++i) {
                        const int row = 64 * q2 + 32 * hh + i;
                        S[32 * q2 + i] = (flags & SEG_H0_EYE) ? (row == j ? 1.f : 0.f)
                                                              : (h0h ? h0h[(int64_t)row * D + j] : 0.f);
                    }
                    put_state(q2);
                }
            }
            // S <- S + Kb^T U on d_k half q2 (the decay is already applied)
            auto state_half = [&](int q2) {
                float d[32];
                tmem_ld32(tm + lane_base + CT_DKU + 64 * q2 + 32 * hh, d);
                wait_ld();
#pragma unroll
                for (int i = 0; i < 32; ++i) S[32 * q2 + i] += d[i];
                put_state(q2);
            };
            // the fp32 state after chunk gc of the sequence, when it ends a snapshot block
            auto snapshot = [&](int gc) {
                if (float* snap = snapshot_slot(states, snap_every, gc, T, b, H, h)) {
#pragma unroll
                    for (int q2 = 0; q2 < 2; ++q2)
#pragma unroll
                        for (int i = 0; i < 32; ++i)
                            snap[(int64_t)(64 * q2 + 32 * hh + i) * D + j] = S[32 * q2 + i];
                }
            };
            // S <- Diag(gamma_C) S with gamma of the slot at sb
            auto decay = [&](uint32_t sb) {
                const float4* gam4 = reinterpret_cast<const float4*>(sm + sb + S_GAM);
#pragma unroll
                for (int q2 = 0; q2 < 2; ++q2)
#pragma unroll
                    for (int i4 = 0; i4 < 8; ++i4) {
                        const float4 gv = gam4[16 * q2 + 8 * hh + i4];
                        S[32 * q2 + 4 * i4 + 0] *= gv.x;
                        S[32 * q2 + 4 * i4 + 1] *= gv.y;
                        S[32 * q2 + 4 * i4 + 2] *= gv.z;
                        S[32 * q2 + 4 * i4 + 3] *= gv.w;
                    }
            };
            // o of chunk cp (X buffer cp & 1, complete since chunk cp's last
            // MMA wait): the tensor-memory load is issued early (its wait is
            // the next state half's), then the rows go to the staging buffer
            // and the release warp writes them with one tensor store, off the
            // compute warps' path (global stores from this SM are slow while
            // the slots stream in).
            float ov[16];
            auto load_output = [&](int cp) {
                const uint32_t dx = (cp & 1) ? CT_DX1 : CT_DX0;
                tmem_ld16(tm + lane_base + dx + C + 16 * hh, ov);
            };
            auto emit_output = [&](int cp) {
                if (!store_o) return;
                // the store of chunk cp - NOST has read buffer cp % NOST
                if (lane == 0 && cp >= NOST && !s_abort &&
                    !counter_wait(smem_u32(&s_ofree), (uint32_t)(cp - NOST + 1), wait_ns))
                    expired();
                __syncwarp();
                const uint32_t ob = (uint32_t)cp % NOST;
                __nv_bfloat16* ost = reinterpret_cast<__nv_bfloat16*>(sm + C_OST + ob * OST_BYTES);
#pragma unroll
                for (int r = 0; r < 16; ++r) ost[(16 * hh + r) * D + j] = __float2bfloat16_rn(ov[r]);
                fence_smem_to_async();
                __syncwarp();
                if (lane == 0) mbar_arrive(smem_u32(&s_bar[6 + ob]));
            };
            fence_before_sync();
            if (n_chunks > 0) {                       // the initial state for chunk 0
                named_arrive(NB_ASA, NX);
                named_arrive(NB_ASB, NX);
            }
#pragma unroll 1
            for (int ch = 0; ch < n_chunks; ++ch) {
                const int slot = ch % NPREPCTA;
                const uint32_t sb = C_SLOT0 + slot * SLOT;
                const uint32_t dx = (ch & 1) ? CT_DX1 : CT_DX0;
                if (ch > 0) {
                    state_half(0);
                    fence_before_sync();
                    named_arrive(NB_ASA, NX);
                    wait_bar(kbar1, (uint32_t)(ch - 1) & 1u);   // Kb^T U second half and P U of chunk ch - 1
                    if (tid == 0) counter_publish(smem_u32(&s_odone), (uint32_t)ch);
                    load_output(ch - 1);
                    state_half(1);                              // (its wait covers the o load)
                    fence_before_sync();
                    named_arrive(NB_ASB, NX);
                    snapshot(ts / C + ch - 1);                  // S after chunk ch - 1
                    emit_output(ch - 1);
                }
                // X of chunk ch (U' of this chunk is in the slot once its FULL
                // phase passed: the release warp publishes that as s_full)
                if (!s_abort && !counter_wait(smem_u32(&s_full), (uint32_t)ch + 1u, wait_ns)) expired();
                {   // U = U' - W S  (this thread: tokens [16 hh, 16 hh + 16)): fp16
                    // pairs into packed columns [8 hh, 8 hh + 8) of CT_AU, or tf32
                    // into columns [16 hh, 16 hh + 16).  U' is read before the
                    // wait for X, off the path from X to U.
                    const float* up = reinterpret_cast<const float*>(sm + sb + S_UP);
                    float upr[16];
#pragma unroll
                    for (int r = 0; r < 16; ++r) upr[r] = up[(16 * hh + r) * D + j];
                    wait_bar(mbar, phase & 1u);
                    ++phase;
                    float x[16];
                    tmem_ld16(tm + lane_base + dx + 16 * hh, x);
                    wait_ld();
                    if constexpr (F16) {
                        float hp[8];
#pragma unroll
                        for (int r = 0; r < 16; r += 2) hp[r >> 1] = pack_f16x2(upr[r] - x[r], upr[r + 1] - x[r + 1]);
                        tmem_st8(tm + lane_base + CT_AU + 8 * hh, hp);
                    } else {
#pragma unroll
                        for (int r = 0; r < 16; ++r) x[r] = to_tf32(upr[r] - x[r]);
                        tmem_st16(tm + lane_base + CT_AU + 16 * hh, x);
                    }
                    wait_st();
                }
                fence_before_sync();
                named_arrive(NB_U, NX);
                decay(sb);                            // while Kb^T U and P U run
                wait_bar(kbar0, (uint32_t)ch & 1u);   // Kb^T U, first d_k half, of chunk ch
            }
            if (n_chunks > 0) {
                state_half(0);
                wait_bar(kbar1, (uint32_t)(n_chunks - 1) & 1u);
                load_output(n_chunks - 1);
                state_half(1);
                snapshot(ts / C + n_chunks - 1);
                emit_output(n_chunks - 1);
            }
            if (hT && !s_abort) {
                float* hTh = hT + head_off * D * D;
#pragma unroll
                for (int q2 = 0; q2 < 2; ++q2)
#pragma unroll
                    for (int i = 0; i < 32; ++i) hTh[(int64_t)(64 * q2 + 32 * hh + i) * D + j] = S[32 * q2 + i];
            }
        }
    } else {
        // ================================================== preparing CTAs ==
        const int par = (int)role - 1;             // chunks ch with ch % NPREPCTA == par
        const uint32_t ebar = smem_u32(&s_bar[0]);
        const uint32_t mbar = smem_u32(&s_bar[1]);
        const uint32_t rbar = smem_u32(&s_bar[2]);
        unsigned char* st = sm + P_ST;
        if (warp == NCW / 32) {
            // ------------------------------------------------------ issuer warp --
            // MMAs and input loads: the compute warps hand over at named
            // barriers and never wait on an issue.
            uint32_t n_commit = 0, n_loads = 0;
            // no new load after an expired wait (the raw buffer may still be read)
            // (with v = 0, the transition pass of the segment scan, v is not loaded)
            const bool load_v = !(flags & SEG_V_ZERO);
            auto issue_raw = [&](int ci) {
                if (*(volatile int*)&s_abort) return;
                ++n_loads;
                mbar_arrive_expect_tx(rbar, (load_v ? 4 : 3) * RAW_T);
                tma_load_3d(smem_u32(sm + P_RAW + 0 * RAW_T), &tm_q, h * D, ts + ci * C, b, rbar);
                tma_load_3d(smem_u32(sm + P_RAW + 1 * RAW_T), &tm_k, h * D, ts + ci * C, b, rbar);
                if (load_v) tma_load_3d(smem_u32(sm + P_RAW + 2 * RAW_T), &tm_v, h * D, ts + ci * C, b, rbar);
                tma_load_3d(smem_u32(sm + P_RAW + 3 * RAW_T), &tm_g, h * D, ts + ci * C, b, rbar);
            };
            if (lane == 0 && par < n_chunks) issue_raw(par);
#pragma unroll 1
            for (int ch = par; ch < n_chunks; ch += NPREPCTA) {
                __syncwarp();
                named_bar(NB_G, NX);                  // Gram operands written, raw inputs consumed
                fence_after_sync();
                if (!warp_flag(s_abort)) {
                    const uint32_t id = idesc_tf32(64, 64, false, false);
                    const uint64_t ad0 = sdesc(smem_u32(sm + P_GA), PAD_LBO, SBO_K128P);
                    const uint64_t bd0 = sdesc(smem_u32(sm + P_GB), PAD_LBO, SBO_K128P);
#pragma unroll
                    for (int ks = 0; ks < D / 8; ++ks) {
                        const uint64_t step = (uint64_t)((ks * 2 * PAD_LBO) >> 4);
                        mma_tf32_ss_w(tm + PT_DG, ad0 + step, bd0 + step, id, ks > 0 ? 1u : 0u);
                    }
                    mma_commit_w(mbar);
                    ++n_commit;
                }
                if (lane == 0 && ch + NPREPCTA < n_chunks) issue_raw(ch + NPREPCTA);
                __syncwarp();
                named_bar(NB_TB, NX);                 // T, K~ f and V staged
                fence_after_sync();
                if (!warp_flag(s_abort)) {
                    // W^T = Kt^T T^T and U'^T = V^T T^T: fp16 operands with the
                    // fp16 chain (K = 16 per MMA), tf32 otherwise
                    const uint32_t id = F16 ? idesc_f16(128, 32) : idesc_tf32(128, 32, false, false);
                    const uint64_t bd0 = sdesc(smem_u32(sm + P_TB), PAD_LBO, F16 ? H_SBO_K32P : SBO_K32P);
                    const uint64_t aw0 = sdesc(smem_u32(sm + P_WA), LBO, F16 ? H_SBO_K32 : SBO_K32);
                    const uint64_t av0 = sdesc(smem_u32(sm + P_VA), LBO, F16 ? H_SBO_K32 : SBO_K32);
#pragma unroll
                    for (int ks = 0; ks < C / CH::KSTEP; ++ks) {
                        const uint64_t bstep = (uint64_t)((ks * 2 * PAD_LBO) >> 4);
                        const uint64_t astep = (uint64_t)((ks * 2 * LBO) >> 4);
                        if constexpr (F16) {
                            mma_f16_ss_w(tm + PT_DW, aw0 + astep, bd0 + bstep, id, ks > 0 ? 1u : 0u);
                            mma_f16_ss_w(tm + PT_DU, av0 + astep, bd0 + bstep, id, ks > 0 ? 1u : 0u);
                        } else {
                            mma_tf32_ss_w(tm + PT_DW, aw0 + astep, bd0 + bstep, id, ks > 0 ? 1u : 0u);
                            mma_tf32_ss_w(tm + PT_DU, av0 + astep, bd0 + bstep, id, ks > 0 ? 1u : 0u);
                        }
                    }
                    mma_commit_w(mbar);
                    ++n_commit;
                }
            }
            // after an expired wait: the last MMAs and input load may still be in flight
            if (lane == 0 && *(volatile int*)&s_abort) {
                if (n_commit > 0) mbar_wait(mbar, (n_commit - 1) & 1u, DRAIN_NS);
                if (n_loads > 0) mbar_wait(rbar, (n_loads - 1) & 1u, DRAIN_NS);
            }
            __syncwarp();
        } else if (warp == NCW / 32 + 1) {
            // --------------------------------------------------------- push warp --
            // Each prepared chunk goes to its slot in the chain CTA as one bulk
            // copy, once the chain has released the slot; then the staging is
            // handed back to the compute warps.
            uint32_t ephase = 0;
            const uint32_t full_remote = map_to_rank(smem_u32(&s_bar[par]), CHAIN_RANK);
            const uint32_t slot_remote = map_to_rank(smem_u32(sm + C_SLOT0 + par * SLOT), CHAIN_RANK);
#pragma unroll 1
            for (int ch = par; ch < n_chunks; ch += NPREPCTA) {
                named_bar(NB_FILL, NX);               // the staging holds chunk ch
                if (lane == 0) {
                    // the chain has released this slot (its previous use, chunk ch - NPREPCTA)
                    if (ch >= NPREPCTA && !s_abort && !mbar_wait_cluster(ebar, ephase & 1u, wait_ns)) expired();
                    if (ch >= NPREPCTA) ++ephase;
                    if (!s_abort) {                   // FULL was armed by the chain
                        bulk_copy_to_rank(slot_remote, smem_u32(st), SLOT, full_remote);
                        bulk_commit();
                    }
                    bulk_wait_read_all();             // the copy has read the staging
                }
                __syncwarp();
                if (ch + NPREPCTA < n_chunks) named_arrive(NB_STFREE, NX);
            }
        } else {
        // ---------------------------------------------------------- compute warps --
        const int pt = tid;
        const int pw = warp;
        uint32_t phase = 0, rphase = 0;
        auto prep_sync = [&]() { named_bar(NB_CW, NCW); };
        // every thread waits on the MMA barrier itself
        auto wait_mma = [&]() {
            if (!s_abort && !mbar_wait(mbar, phase & 1u, wait_ns)) expired();
            ++phase;
            fence_after_sync();
        };
        const __nv_bfloat16 bzero = __float2bfloat16_rn(0.f);
        __nv_bfloat16 beta_next = (pt < C && par * C + pt < Tl) ? beta[((int64_t)b * T + ts + par * C + pt) * H + h] : bzero;
        const int tau = pt >> 7;
        const int c = pt & 127;
        float* am = reinterpret_cast<float*>(sm + P_AMS);
        float* pm = reinterpret_cast<float*>(sm + P_PMS);
        float* xm = reinterpret_cast<float*>(sm + P_XMS);
        float* tmx = reinterpret_cast<float*>(sm + P_TMS);
        float* ym = reinterpret_cast<float*>(sm + P_YMS);
        const float* bt = reinterpret_cast<const float*>(sm + P_BETA);
#pragma unroll 1
        for (int ch = par; ch < n_chunks; ch += NPREPCTA) {
            if (pt < C) {
                reinterpret_cast<float*>(sm + P_BETA)[pt] = to_f32(beta_next);
                const int tn = (ch + NPREPCTA) * C + pt;
                beta_next = (tn < Tl) ? beta[((int64_t)b * T + ts + tn) * H + h] : bzero;
            }
            if (pt == 0 && !s_abort && !mbar_wait(rbar, rphase & 1u, wait_ns)) expired();
            ++rphase;
            __syncwarp();
            prep_sync();
            float gam_c, fq, fk;
            float vr[TILE];
            // fp16 instantiation: the chunk-relative Qt and Kb of this thread's
            // channel and tile, as fp16 pairs, kept in registers for the fill
            uint32_t qh[TILE / 2], kh[TILE / 2];
            {
                const __nv_bfloat16* __restrict__ rq = reinterpret_cast<const __nv_bfloat16*>(sm + P_RAW + 0 * RAW_T);
                const __nv_bfloat16* __restrict__ rk = reinterpret_cast<const __nv_bfloat16*>(sm + P_RAW + 1 * RAW_T);
                const __nv_bfloat16* __restrict__ rv = reinterpret_cast<const __nv_bfloat16*>(sm + P_RAW + 2 * RAW_T);
                const __nv_bfloat16* __restrict__ rg = reinterpret_cast<const __nv_bfloat16*>(sm + P_RAW + 3 * RAW_T);
                float a[TILE], kr[TILE], qr[TILE];
#pragma unroll
                for (int rr = 0; rr < TILE; ++rr) {
                    const int idx = (tau * TILE + rr) * D + c;
                    kr[rr] = to_f32(rk[idx]);
                    qr[rr] = to_f32(rq[idx]);
                    vr[rr] = (flags & SEG_V_ZERO) ? 0.f : to_f32(rv[idx]);
                    a[rr] = to_f32(rg[idx]);
                }
                if constexpr (PRO) prologue_gate_and_norms(a, qr, kr, ch * C + tau * TILE, Tl,
                                                            reinterpret_cast<float*>(sm + P_NRM), tau, c);
                float e = 1.f;
#pragma unroll
                for (int rr = 0; rr < TILE; ++rr) {
                    a[rr] = __expf(a[rr]);
                    e *= a[rr];
                }
                float* gex = reinterpret_cast<float*>(sm + P_GEX);
                gex[tau * D + c] = e;
                prep_sync();
                if constexpr (PRO) prologue_normalise(qr, kr, reinterpret_cast<const float*>(sm + P_NRM), tau);
                const float oe = gex[(1 - tau) * D + c];
                const float f = tau ? oe : 1.f;
                gam_c = e * oe;
                fq = f;
                fk = tau ? e : oe;
                float p = 1.f;
                float kc[8];
                float qprev = 0.f;
#pragma unroll
                for (int rr = 0; rr < TILE; ++rr) {
                    const int r = tau * TILE + rr;
                    p *= a[rr];
                    const float kt = kr[rr] * p;
                    const float qt = qr[rr] * p;
                    st_f32(sm, P_GB + off_kmajor(r, c, PAD_LBO, SBO_K128P), to_tf32(kt));
                    st_f32(sm, P_GB + off_kmajor(C + r, c, PAD_LBO, SBO_K128P), qt);   // full fp32: see below
                    if constexpr (F16) {
                        if (rr & 1) qh[rr >> 1] = __float_as_uint(pack_f16x2(qprev, qt * fq));
                        else qprev = qt * fq;
                    }
                    // Kt (chunk-relative) for W: fp16, 8 tokens per vector, or tf32, 4
                    if constexpr (F16) {
                        kc[rr & 7] = kt * f;
                        if ((rr & 7) == 7)
                            *reinterpret_cast<uint4*>(sm + P_WA + off16_kmajor(c, r - 7, LBO, H_SBO_K32)) =
                                make_uint4(__float_as_uint(pack_f16x2(kc[0], kc[1])),
                                           __float_as_uint(pack_f16x2(kc[2], kc[3])),
                                           __float_as_uint(pack_f16x2(kc[4], kc[5])),
                                           __float_as_uint(pack_f16x2(kc[6], kc[7])));
                    } else {
                        kc[rr & 3] = to_tf32(kt * f);
                        if ((rr & 3) == 3)
                            st_f32x4(sm, P_WA + off_kmajor(c, r - 3, LBO, SBO_K32), kc[0], kc[1], kc[2], kc[3]);
                    }
                }
                const float inv = 1.f / e;
                float sgm = 1.f;
                float knext = 0.f;
#pragma unroll
                for (int rr = TILE - 1; rr >= 0; --rr) {
                    const int r = tau * TILE + rr;
                    const float kb = kr[rr] * sgm;
                    // Qt (above), Kh and Kb_0 stay in full fp32: the operand fill
                    // rescales them into the chunk-relative Qt and Kb and rounds
                    // them once (rounding here too would round those twice);
                    // the Gram MMA reads the rows as tf32 (low mantissa bits
                    // ignored).  The fp16 instantiation forms the chunk-relative
                    // values here, from the same fp32 numbers the fill would read.
                    st_f32(sm, P_GA + off_kmajor(r, c, PAD_LBO, SBO_K128P), kb * inv);
                    if (tau == 0) st_f32(sm, P_GA + off_kmajor(C + rr, c, PAD_LBO, SBO_K128P), kb);
                    if constexpr (F16) {
                        const float kf = tau ? (kb * inv) * fk : kb * fk;
                        if (rr & 1) knext = kf;
                        else kh[rr >> 1] = __float_as_uint(pack_f16x2(kf, knext));
                    }
                    sgm *= a[rr];
                }
            }
            fence_smem_to_async();
            fence_before_sync();
            named_arrive(NB_G, NX);
            if constexpr (F16) {
#pragma unroll
                for (int rr = 0; rr < TILE; rr += 8)
                    *reinterpret_cast<uint4*>(sm + P_VA + off16_kmajor(c, tau * TILE + rr, LBO, H_SBO_K32)) =
                        make_uint4(__float_as_uint(pack_f16x2(vr[rr], vr[rr + 1])),
                                   __float_as_uint(pack_f16x2(vr[rr + 2], vr[rr + 3])),
                                   __float_as_uint(pack_f16x2(vr[rr + 4], vr[rr + 5])),
                                   __float_as_uint(pack_f16x2(vr[rr + 6], vr[rr + 7])));
            } else {
#pragma unroll
                for (int rr = 0; rr < TILE; rr += 4)
                    st_f32x4(sm, P_VA + off_kmajor(c, tau * TILE + rr, LBO, SBO_K32),
                             to_tf32(vr[rr]), to_tf32(vr[rr + 1]), to_tf32(vr[rr + 2]), to_tf32(vr[rr + 3]));
            }
            fence_smem_to_async();
            wait_mma();
            // A and P (32 x 32) from the Gram (row m of D_G is lane (m % 16) +
            // 32 (m / 16)).  Sub-partition 0 holds the rows Kh_0 (columns Kt_0,
            // Qt_0), 1 the rows Kh_1 (Kt_1, Qt_1), 2 the rows Kb_0 (Kt_1, Qt_1:
            // the block between the tiles).  Warps 0-2 take the A columns,
            // warps 4-6 the P columns.  The warp that holds a diagonal block of
            // A also solves it, X = (I + A_tt)^-1, column i per lane, forward
            // substitution, from A_tt^T in shared memory (one 16-float column
            // per step, read as four vectors), with no barrier in between.
            {
                const int spx = pw & 3;
                if (spx < 3) {
                    const bool is_p = pw >= 4;
                    const int colK = (spx == 0) ? 0 : TILE;
                    float gv[16];
                    tmem_ld16(tm + lane_base + PT_DG + (is_p ? C : 0) + colK, gv);
                    wait_ld();
                    const int i = (spx == 1 ? TILE : 0) + lane;           // column of A / P
                    const int rbase = (spx == 0) ? 0 : TILE;              // rows covered
                    float* atm = reinterpret_cast<float*>(sm + P_ATM) + spx * TILE * ATM_LD;
                    if (lane < TILE) {
                        if (is_p) {
#pragma unroll
                            for (int r = 0; r < TILE; ++r) {
                                const int rg = rbase + r;
                                pm[rg * LD + i] = (rg >= i) ? gv[r] : 0.f;
                            }
                            if (spx == 1) {                               // P_01 = 0
#pragma unroll
                                for (int r = 0; r < TILE; ++r) pm[r * LD + i] = 0.f;
                            }
                        } else if (spx == 2) {                            // A_10, all below the diagonal
#pragma unroll
                            for (int r = 0; r < TILE; ++r) am[(TILE + r) * LD + i] = bt[TILE + r] * gv[r];
                        } else {                                          // column i of A_tt into row i of A_tt^T
#pragma unroll
                            for (int r = 0; r < TILE; r += 4) {
                                float e4[4];
#pragma unroll
                                for (int u = 0; u < 4; ++u) {
                                    const int rg = rbase + r + u;
                                    e4[u] = (rg > i) ? bt[rg] * gv[r + u] : 0.f;
                                }
                                *reinterpret_cast<float4*>(atm + lane * ATM_LD + r) = make_float4(e4[0], e4[1], e4[2], e4[3]);
                            }
                        }
                    }
                    if (!is_p && spx < 2) {
                        __syncwarp();
                        if (lane < TILE) {
                            const int off = spx * TILE;
                            float x[TILE];
#pragma unroll
                            for (int r = 0; r < TILE; ++r) x[r] = (r == lane) ? 1.f : 0.f;
#pragma unroll
                            for (int s2 = 0; s2 < TILE; ++s2) {
                                const float4* col = reinterpret_cast<const float4*>(atm + s2 * ATM_LD);
                                float a16[TILE];
#pragma unroll
                                for (int q4 = 0; q4 < TILE / 4; ++q4) {
                                    const float4 v4 = col[q4];
                                    a16[4 * q4] = v4.x; a16[4 * q4 + 1] = v4.y;
                                    a16[4 * q4 + 2] = v4.z; a16[4 * q4 + 3] = v4.w;
                                }
#pragma unroll
                                for (int r = s2 + 1; r < TILE; ++r) x[r] = fmaf(-a16[r], x[s2], x[r]);
                            }
                            const float bi = bt[off + lane];
#pragma unroll
                            for (int r = 0; r < TILE; ++r) {
                                xm[(off + r) * LD + off + lane] = x[r];
                                tmx[(off + r) * LD + off + lane] = x[r] * bi;     // T_tt = X_tt diag(b)
                                if (spx == 1) tmx[r * LD + off + lane] = 0.f;     // T_01 = 0
                            }
                        }
                    }
                }
            }
            prep_sync();
            {
                const int r = pt >> 4, i = pt & 15;
                float y = 0.f;
#pragma unroll
                for (int s2 = 0; s2 < TILE; ++s2) y = fmaf(am[(TILE + r) * LD + s2], xm[s2 * LD + i], y);
                ym[r * (TILE + 1) + i] = y;
            }
            prep_sync();
            {
                const int r = pt >> 4, i = pt & 15;
                float z = 0.f;
#pragma unroll
                for (int s2 = 0; s2 < TILE; ++s2) z = fmaf(xm[(TILE + r) * LD + TILE + s2], ym[s2 * (TILE + 1) + i], z);
                tmx[(TILE + r) * LD + i] = -z * bt[i];
            }
            prep_sync();
            {   // T into the B operand of the WY products: element (n = r, k = i)
                const int r = pt >> 3, i = (pt & 7) * 4;
                const float* row = tmx + r * LD + i;
                if constexpr (F16)
                    *reinterpret_cast<uint2*>(sm + P_TB + off16_kmajor(r, i, PAD_LBO, H_SBO_K32P)) =
                        make_uint2(__float_as_uint(pack_f16x2(row[0], row[1])), __float_as_uint(pack_f16x2(row[2], row[3])));
                else
                    st_f32x4(sm, P_TB + off_kmajor(r, i, PAD_LBO, SBO_K32P),
                             to_tf32(row[0]), to_tf32(row[1]), to_tf32(row[2]), to_tf32(row[3]));
            }
            fence_smem_to_async();
            fence_before_sync();
            named_arrive(NB_TB, NX);
            float qf[TILE], kf[TILE];
            if constexpr (!F16) {
                const float* gaf = reinterpret_cast<const float*>(sm + P_GA);
                const float* gbf = reinterpret_cast<const float*>(sm + P_GB);
#pragma unroll
                for (int rr = 0; rr < TILE; ++rr) {
                    const int r = tau * TILE + rr;
                    qf[rr] = gbf[off_kmajor(C + r, c, PAD_LBO, SBO_K128P) >> 2] * fq;
                    const int row = tau ? (TILE + rr) : (C + rr);
                    kf[rr] = gaf[off_kmajor(row, c, PAD_LBO, SBO_K128P) >> 2] * fk;
                }
            }
            // P, element (n = r, k = i) (lane = row: no bank conflicts): fp16,
            // eight K-adjacent entries per thread (threads 0-127), or tf32, four
            uint4 pf4 = make_uint4(0u, 0u, 0u, 0u);
            if constexpr (F16) {
                if (pt < 4 * C) {
                    const int r = pt & 31, i = (pt >> 5) * 8;
                    const float* row = pm + r * LD + i;
                    pf4 = make_uint4(__float_as_uint(pack_f16x2(row[0], row[1])), __float_as_uint(pack_f16x2(row[2], row[3])),
                                     __float_as_uint(pack_f16x2(row[4], row[5])), __float_as_uint(pack_f16x2(row[6], row[7])));
                }
            } else {
                const int r = pt & 31, i = (pt >> 5) * 4;
                const float* row = pm + r * LD + i;
                pf4 = make_uint4(__float_as_uint(to_tf32(row[0])), __float_as_uint(to_tf32(row[1])),
                                 __float_as_uint(to_tf32(row[2])), __float_as_uint(to_tf32(row[3])));
            }
            // the previous chunk's bulk copy has finished reading the staging
            wait_mma();
            if (ch != par) named_bar(NB_STFREE, NX);  // the previous push has read the staging
            {
                float w[16], upv[16];
                tmem_ld16(tm + lane_base + PT_DW + 16 * tau, w);
                tmem_ld16(tm + lane_base + PT_DU + 16 * tau, upv);
                wait_ld();
                // [W | Qt] (element (token, d_k channel c)) and U' (fp32)
#pragma unroll
                for (int r = 0; r < 16; ++r) {
                    if constexpr (F16)
                        *reinterpret_cast<uint16_t*>(st + S_B1 + off16_kmajor(16 * tau + r, c, PAD_LBO, CH::SBO_B1)) =
                            to_f16_bits(w[r]);
                    else
                        st_f32(st, S_B1 + off_kmajor(16 * tau + r, c, PAD_LBO, CH::SBO_B1), to_tf32(w[r]));
                    reinterpret_cast<float*>(st + S_UP)[(16 * tau + r) * D + c] = upv[r];
                }
#pragma unroll
                for (int rr = 0; rr < TILE; ++rr) {
                    if constexpr (F16)
                        *reinterpret_cast<uint16_t*>(st + S_B1 + off16_kmajor(C + tau * TILE + rr, c, PAD_LBO, CH::SBO_B1)) =
                            (uint16_t)((rr & 1) ? (qh[rr >> 1] >> 16) : (qh[rr >> 1] & 0xffffu));
                    else
                        st_f32(st, S_B1 + off_kmajor(C + tau * TILE + rr, c, PAD_LBO, CH::SBO_B1), to_tf32(qf[rr]));
                }
                // Kb (element (d_k channel c, token)): 8 (fp16) or 4 (tf32) tokens per vector
                if constexpr (F16) {
#pragma unroll
                    for (int rr = 0; rr < TILE; rr += 8)
                        *reinterpret_cast<uint4*>(st + S_B2 + off16_kmajor(c, tau * TILE + rr, LBO, CH::SBO_B23)) =
                            make_uint4(kh[rr / 2], kh[rr / 2 + 1], kh[rr / 2 + 2], kh[rr / 2 + 3]);
                    if (pt < 4 * C) {
                        const int r = pt & 31, i = (pt >> 5) * 8;
                        *reinterpret_cast<uint4*>(st + S_B3 + off16_kmajor(r, i, LBO, CH::SBO_B23)) = pf4;
                    }
                } else {
#pragma unroll
                    for (int rr = 0; rr < TILE; rr += 4)
                        st_f32x4(st, S_B2 + off_kmajor(c, tau * TILE + rr, LBO, CH::SBO_B23),
                                 to_tf32(kf[rr]), to_tf32(kf[rr + 1]), to_tf32(kf[rr + 2]), to_tf32(kf[rr + 3]));
                    const int r = pt & 31, i = (pt >> 5) * 4;
                    *reinterpret_cast<uint4*>(st + S_B3 + off_kmajor(r, i, LBO, CH::SBO_B23)) = pf4;
                }
                if (tau == 0) reinterpret_cast<float*>(st + S_GAM)[c] = gam_c;
            }
            fence_smem_to_async();
            named_arrive(NB_FILL, NX);
        }
        }
    }

    fence_before_sync();
    __syncthreads();
    cluster_sync();                    // every push that will be issued has been issued
    if (role == 0 && tid == 0 && *(volatile int*)&s_abort) {
        // An expired wait let this CTA stop consuming slots: a push into a
        // slot may still be landing.  Let each slot's last expected push land
        // (or find that it was never sent) before the shared memory is given up.
        for (int sl = 0; sl < NPREPCTA; ++sl)
            if (s_last_armed[sl] >= 0)
                mbar_wait_cluster(smem_u32(&s_bar[sl]), (uint32_t)(s_last_armed[sl] / NPREPCTA) & 1u, DRAIN_NS);
    }
    __syncthreads();
    if (warp == 0) tmem_dealloc(tm, ncols);
    if (role == 0 && tid < NCW && *(volatile int*)&s_abort)
        poison_head_outputs(o ? o + ((int64_t)b * T + ts) * (int64_t)H * D + (int64_t)h * D : nullptr,
                            (int64_t)H * D, Tl, o && !(flags & SEG_NO_O),
                            hT ? hT + head_off * D * D : nullptr, tid, NCW);
}

static bool make_map(CUtensorMap* map, const void* base, int B, int T, int H)
{
    typedef CUresult (*encode_fn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
    // looked up once per process (thread-safe static initialisation): the
    // driver entry point is the same for every device
    static const encode_fn encode = []() -> encode_fn {
        void* fn = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            return nullptr;
        return (encode_fn)fn;
    }();
    if (!encode) return false;
    // [B][T][H * 128] bf16, box 128 x 32 x 1 (one head's 32 token rows)
    const cuuint64_t dims[3] = {(cuuint64_t)H * pf::D, (cuuint64_t)T, (cuuint64_t)B};
    const cuuint64_t strides[2] = {(cuuint64_t)H * pf::D * 2, (cuuint64_t)T * H * pf::D * 2};
    const cuuint32_t box[3] = {pf::D, pf::C, 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    return encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Dynamic shared memory of every prefill kernel, set once per device (the
// attribute applies to the current device only).
static cudaError_t segment_combine_attribute();
static DeviceFlags g_prefill_attr_done;

static cudaError_t set_prefill_attributes()
{
    return once_per_device(g_prefill_attr_done, [](int) {
        const cudaFuncAttribute a = cudaFuncAttributeMaxDynamicSharedMemorySize;
        cudaError_t e = cudaFuncSetAttribute(prefill_tc_kernel<false>, a, (int)pf::SMEM_BYTES);
        if (e == cudaSuccess) e = cudaFuncSetAttribute(prefill_tc_kernel<true>, a, (int)pf::SMEM_BYTES);
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(prefill_cluster_kernel<false, true>, a, (int)pc::Chain<true>::SMEM_BYTES);
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(prefill_cluster_kernel<true, true>, a, (int)pc::Chain<true>::SMEM_BYTES);
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(prefill_cluster_kernel<false, false>, a, (int)pc::Chain<false>::SMEM_BYTES);
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(prefill_cluster_kernel<true, false>, a, (int)pc::Chain<false>::SMEM_BYTES);
        if (e == cudaSuccess) e = segment_combine_attribute();
        return e;
    });
}

// SMs of the current device (148 on a B200 if the query fails).
static int64_t sm_count()
{
    const int n = current_sm_count();
    return n > 0 ? n : 148;
}

// Four SMs per head pay off while the heads alone leave most SMs idle:
// up to SMs / 4 heads (37 on a B200); larger batches use one SM per head.
static bool cluster_fits(int64_t heads) { return heads * (pc::NPREPCTA + 1) <= sm_count(); }

// Bounded waits give up after 2 s; KDA_WAIT_LIMIT_NS (0 .. 2e9 ns) shortens
// the limit for tests that make the prefill's own waits run out.  With 0 a
// wait checks its phase once, without blocking, and gives up if it has not
// completed: the first wait for an input load or for a chunk pushed by
// another SM then gives up, since neither can land in the few hundred cycles
// between its issue and the check.  The drain after an expired wait keeps
// its own 20 ms limit.
uint64_t bounded_wait_limit_ns()
{
    const char* env = getenv("KDA_WAIT_LIMIT_NS");
    if (!env || !*env) return pf::WAIT_NS;
    const unsigned long long v = strtoull(env, nullptr, 10);
    return v > pf::WAIT_NS ? pf::WAIT_NS : (uint64_t)v;
}
static uint64_t wait_limit_ns() { return bounded_wait_limit_ns(); }

// One launch of either variant over B * n_seg segment-sequences of length
// seg_len (n_seg = 1, seg_len = T: the plain prefill).
static cudaError_t launch_pass(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                               const CUtensorMap& mg, const void* beta, const float* h0, void* o, float* hT,
                               int B, int T, int H, int seg_len, int n_seg, uint32_t flags, bool cluster,
                               float* states, int snap_every, cudaStream_t stream)
{
    const bool pro = (flags & pf::PROLOGUE) != 0;
    if (cluster) {
        // o as a tensor map for the cluster variant's tensor stores
        CUtensorMap mo;
        memset(&mo, 0, sizeof(mo));
        if (o && !(flags & pf::SEG_NO_O) && T > 0 && !make_map(&mo, o, B, T, H)) return cudaErrorInvalidValue;
        dim3 grid((pc::NPREPCTA + 1) * H, B * n_seg);
        // fp16 chain operands, except for the transition pass (state from I)
        const bool h16 = !(flags & pf::SEG_H0_EYE);
        auto kern = h16 ? (pro ? prefill_cluster_kernel<true, true> : prefill_cluster_kernel<false, true>)
                        : (pro ? prefill_cluster_kernel<true, false> : prefill_cluster_kernel<false, false>);
        const uint32_t smem = h16 ? pc::Chain<true>::SMEM_BYTES : pc::Chain<false>::SMEM_BYTES;
        kern<<<grid, pc::NTH, smem, stream>>>(
            mq, mk, mv, mg, mo, (const __nv_bfloat16*)beta, h0, (__nv_bfloat16*)o, hT, T, H, seg_len, n_seg, flags,
            states, snap_every, wait_limit_ns());
    } else {
        dim3 grid(H, B * n_seg);
        auto kern = pro ? prefill_tc_kernel<true> : prefill_tc_kernel<false>;
        kern<<<grid, pf::NT, pf::SMEM_BYTES, stream>>>(
            mq, mk, mv, mg, (const __nv_bfloat16*)beta, h0, (__nv_bfloat16*)o, hT, T, H, seg_len, n_seg, flags,
            states, snap_every, wait_limit_ns());
    }
    return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// Segment scan (for very few heads on long sequences).  The sequence of each
// head is cut into n_seg segments of seg_len tokens (a multiple of the
// 32-token chunk).  The recurrence is affine in the state, so over a segment
// S_end = M_p S_start + N_p, with M_p the product of the segment's per-token
// transitions (I - b k k^T) Diag(exp g) and N_p the state the segment reaches
// from zero.  Pass 1 runs every segment at once twice: from S = 0 (giving
// N_p) and from S = I with v = 0 (giving M_p, since each state column evolves
// on its own).  Pass 2 chains S_{p+1} = M_p S_p + N_p over the segments.
// Pass 3 reruns every segment from its true S_p and writes o.
constexpr int SEG_MAX_HEADS = 8;      // B * H up to this: the segment scan
constexpr int SEG_MIN_CHUNKS = 8;     // chunks per segment at least
constexpr int SEG_MIN_T_CHUNKS = 128; // and a sequence of at least 128 chunks
constexpr int SEG_COLS = 16;          // state columns per combine CTA

// S_{p+1} = M_p S_p + N_p for the segments of one (b, h), in fp32 on CUDA
// cores (columns of S are independent: one CTA per group of 16 columns).
// Writes S_p, the start state of segment p, for pass 3, and the final state.
// M, N, S0: [B * n_seg][H][D][D]; h0, hT: [B][H][D][D] (either may be null;
// hT may equal h0).  M_p goes to shared memory with cp.async, one segment
// ahead (two buffers), rows padded to 132 floats (16-byte aligned; the 16
// rows a warp reads at one k fall on 16 banks pairwise).
constexpr int SEG_MLD = pf::D + 4;
constexpr uint32_t SEG_COMBINE_SMEM = (uint32_t)(pf::D * SEG_COLS + 2 * pf::D * SEG_MLD) * 4;

__device__ __forceinline__ void cp_async16(void* smem_dst, const void* gmem_src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;"
                 :: "r"(tc::smem_u32(smem_dst)), "l"(gmem_src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_1() { asm volatile("cp.async.wait_group 1;" ::: "memory"); }

__global__ void __launch_bounds__(256)
segment_combine_kernel(const float* __restrict__ M, const float* __restrict__ N, float* __restrict__ S0,
                       const float* h0, float* hT, int H, int n_seg)
{
    constexpr int D = pf::D;
    extern __shared__ __align__(16) float csm[];
    float (*s)[SEG_COLS] = reinterpret_cast<float (*)[SEG_COLS]>(csm);          // [D][SEG_COLS]
    float* mb = csm + D * SEG_COLS;                                              // 2 x [D][SEG_MLD]
    const int bh = blockIdx.y, b = bh / H, h = bh - b * H;
    const int tid = threadIdx.x;
    const int i = tid >> 1, jh = (tid & 1) * 8;              // row i, columns [col0, col0 + 8)
    const int col0 = blockIdx.x * SEG_COLS + jh;
    auto seg_base = [&](int p) { return ((int64_t)(b * n_seg + p) * H + h) * D * D; };
    auto load_m = [&](int p) {                               // M_p -> buffer p & 1 (16 x 16 B per thread)
        const float* src = M + seg_base(p);
        float* dst = mb + (p & 1) * D * SEG_MLD;
#pragma unroll
        for (int u = 0; u < (D * D / 4) / 256; ++u) {
            const int e = (u * 256 + tid) * 4;               // element of a row-major D x D matrix
            cp_async16(dst + (e / D) * SEG_MLD + (e % D), src + e);
        }
        cp_async_commit();
    };
    load_m(0);
    if (n_seg > 1) load_m(1); else cp_async_commit();
#pragma unroll
    for (int c = 0; c < 8; ++c) s[i][jh + c] = h0 ? h0[(int64_t)bh * D * D + (int64_t)i * D + col0 + c] : 0.f;
#pragma unroll 1
    for (int p = 0; p < n_seg; ++p) {
        const int64_t sp = seg_base(p) + (int64_t)i * D + col0;
        float acc[8];
#pragma unroll
        for (int c = 0; c < 8; ++c) acc[c] = N[sp + c];
        cp_async_wait_1();                                   // M_p has landed (M_{p+1} may be in flight)
        __syncthreads();                                     // ... for every thread; s holds S_p
#pragma unroll
        for (int c = 0; c < 8; ++c) S0[sp + c] = s[i][jh + c];
        const float* mrow = mb + (p & 1) * D * SEG_MLD + i * SEG_MLD;
#pragma unroll 8
        for (int k = 0; k < D; ++k) {
            const float m = mrow[k];
            const float4 a0 = *reinterpret_cast<const float4*>(&s[k][jh]);
            const float4 a1 = *reinterpret_cast<const float4*>(&s[k][jh + 4]);
            acc[0] = fmaf(m, a0.x, acc[0]); acc[1] = fmaf(m, a0.y, acc[1]);
            acc[2] = fmaf(m, a0.z, acc[2]); acc[3] = fmaf(m, a0.w, acc[3]);
            acc[4] = fmaf(m, a1.x, acc[4]); acc[5] = fmaf(m, a1.y, acc[5]);
            acc[6] = fmaf(m, a1.z, acc[6]); acc[7] = fmaf(m, a1.w, acc[7]);
        }
        __syncthreads();                                     // every read of S_p and of buffer p & 1 done
        if (p + 2 < n_seg) load_m(p + 2); else cp_async_commit();
#pragma unroll
        for (int c = 0; c < 8; ++c) s[i][jh + c] = acc[c];
    }
    __syncthreads();
    if (hT) {
#pragma unroll
        for (int c = 0; c < 8; ++c) hT[(int64_t)bh * D * D + (int64_t)i * D + col0 + c] = s[i][jh + c];
    }
}

static cudaError_t segment_combine_attribute()
{
    return cudaFuncSetAttribute(segment_combine_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)SEG_COMBINE_SMEM);
}

enum class PrefillPath { OneSm, Cluster, Segmented };

// KDA_PREFILL_VARIANT=fused|cluster|segmented overrides the choice (for
// measurement and tests).
static PrefillPath choose_path(int B, int T, int H)
{
    const int64_t heads = (int64_t)B * H;
    const int n_chunks = (T + pf::C - 1) / pf::C;
    const bool seg_ok = n_chunks >= 2 * SEG_MIN_CHUNKS;
    const char* env = getenv("KDA_PREFILL_VARIANT");
    if (env && strcmp(env, "cluster") == 0) return PrefillPath::Cluster;
    if (env && strcmp(env, "fused") == 0) return PrefillPath::OneSm;
    if (env && strcmp(env, "segmented") == 0 && seg_ok) return PrefillPath::Segmented;
    if (heads <= SEG_MAX_HEADS && n_chunks >= SEG_MIN_T_CHUNKS) return PrefillPath::Segmented;
    return cluster_fits(heads) ? PrefillPath::Cluster : PrefillPath::OneSm;
}

// Segments: about one wave of segment-heads, at least SEG_MIN_CHUNKS chunks
// each, at least two.
static void segment_plan(int B, int T, int H, int* seg_len, int* n_seg)
{
    const int64_t heads = (int64_t)B * H;
    const int n_chunks = (T + pf::C - 1) / pf::C;
    int64_t P = sm_count() / (heads > 0 ? heads : 1);
    P = P < (int64_t)(n_chunks / SEG_MIN_CHUNKS) ? P : (int64_t)(n_chunks / SEG_MIN_CHUNKS);
    if (P < 2) P = 2;
    const int seg_chunks = (int)((n_chunks + P - 1) / P);
    *seg_len = seg_chunks * pf::C;
    *n_seg = (T + *seg_len - 1) / *seg_len;
}

// Fixed scratch of the no-allocation entry point: the segment scan's three
// state arrays for up to 148 segment-heads, which covers every call that
// chooses the segment scan by itself (B * H * P <= 148).  One copy per device.
constexpr size_t NOALLOC_SCRATCH_BYTES = (size_t)3 * 148 * pf::D * pf::D * sizeof(float);
static __device__ __align__(256) unsigned char g_noalloc_scratch[NOALLOC_SCRATCH_BYTES];

static cudaError_t launch_segmented(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                                    const CUtensorMap& mg, const void* beta, const float* h0, void* o,
                                    float* hT, int B, int T, int H, bool no_alloc, float* states,
                                    int snap_every, uint32_t base_flags, cudaStream_t stream)
{
    int seg_len = 0, n_seg = 0;
    segment_plan(B, T, H, &seg_len, &n_seg);
    const size_t n_state = (size_t)B * n_seg * H * pf::D * pf::D;    // floats per array
    const size_t bytes = 3 * n_state * sizeof(float);
    float* ws = nullptr;
    cudaError_t e = cudaSuccess;
    if (no_alloc) {
        // nothing is launched when the fixed scratch is too small
        if (bytes > NOALLOC_SCRATCH_BYTES) return cudaErrorMemoryAllocation;
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);   // this device's copy
        if (e != cudaSuccess) return e;
        ws = static_cast<float*>(p);
    } else {
        keep_pool_memory();
        e = cudaMallocAsync(reinterpret_cast<void**>(&ws), bytes, stream);
        if (e != cudaSuccess) return e;
    }
    float* Mw = ws;
    float* Nw = ws + n_state;
    float* Sw = ws + 2 * n_state;
    const bool cl = cluster_fits((int64_t)B * n_seg * H);
    e = launch_pass(mq, mk, mv, mg, beta, nullptr, o, Nw, B, T, H, seg_len, n_seg, base_flags | pf::SEG_NO_O, cl,
                    nullptr, 0, stream);
    if (e == cudaSuccess)
        e = launch_pass(mq, mk, mv, mg, beta, nullptr, o, Mw, B, T, H, seg_len, n_seg,
                        base_flags | pf::SEG_V_ZERO | pf::SEG_H0_EYE | pf::SEG_NO_O, cl, nullptr, 0, stream);
    if (e == cudaSuccess) {
        segment_combine_kernel<<<dim3(pf::D / SEG_COLS, B * H), 256, SEG_COMBINE_SMEM, stream>>>(
            Mw, Nw, Sw, h0, hT, H, n_seg);
        e = cudaGetLastError();
    }
    if (e == cudaSuccess)
        e = launch_pass(mq, mk, mv, mg, beta, Sw, o, nullptr, B, T, H, seg_len, n_seg, base_flags, cl,
                        states, snap_every, stream);
    if (!no_alloc) {
        const cudaError_t ef = cudaFreeAsync(ws, stream);
        if (e == cudaSuccess) e = ef;
    }
    note_launches(4);
    return e;
}

// Which path a bf16 prefill of this shape takes on the current device
// (0 one SM per head, 1 cluster of four SMs per head, 2 segment scan).
int prefill_path_of(int B, int T, int H)
{
    return (int)choose_path(B, T, H);
}

cudaError_t prefill_tc_launch(const void* q, const void* k, const void* v, const void* g,
                              const void* beta, const float* h0, void* o, float* hT,
                              int B, int T, int H, bool no_alloc, float* states, int snap_every,
                              bool prologue, cudaStream_t stream)
{
    const uint32_t flags = prologue ? pf::PROLOGUE : 0u;
    {
        const cudaError_t e = set_prefill_attributes();
        if (e != cudaSuccess) return e;
    }
    CUtensorMap mq, mk, mv, mg;
    if (T > 0) {
        if (!make_map(&mq, q, B, T, H) || !make_map(&mk, k, B, T, H) ||
            !make_map(&mv, v, B, T, H) || !make_map(&mg, g, B, T, H))
            return cudaErrorInvalidValue;
    } else {   // no chunk, no load: the kernel only carries h0 to hT
        memset(&mq, 0, sizeof(mq)); memset(&mk, 0, sizeof(mk));
        memset(&mv, 0, sizeof(mv)); memset(&mg, 0, sizeof(mg));
    }
    const PrefillPath path = choose_path(B, T, H);
    if (path == PrefillPath::Segmented)
        return launch_segmented(mq, mk, mv, mg, beta, h0, o, hT, B, T, H, no_alloc, states, snap_every,
                                flags, stream);
    const cudaError_t e = launch_pass(mq, mk, mv, mg, beta, h0, o, hT, B, T, H, T, 1, flags,
                                      path == PrefillPath::Cluster, states, snap_every, stream);
    note_launches(1);
    return e;
}

// Transition of each whole sequence: M = prod_t (I - b_t k_t k_t^T) Diag(exp g_t)
// (d_k x d_k), as the state reached from S = I with v = 0 (each state column
// evolves on its own).  M: [B][H][D][D].  v is not read (its map reuses q's).
cudaError_t prefill_transition_launch(const void* q, const void* k, const void* g, const void* beta,
                                      float* M, int B, int T, int H, cudaStream_t stream)
{
    {
        const cudaError_t e = set_prefill_attributes();
        if (e != cudaSuccess) return e;
    }
    CUtensorMap mq, mk, mg;
    if (T > 0) {
        if (!make_map(&mq, q, B, T, H) || !make_map(&mk, k, B, T, H) || !make_map(&mg, g, B, T, H))
            return cudaErrorInvalidValue;
    } else {
        memset(&mq, 0, sizeof(mq)); memset(&mk, 0, sizeof(mk)); memset(&mg, 0, sizeof(mg));
    }
    const cudaError_t e = launch_pass(mq, mk, mq, mg, beta, nullptr, nullptr, M, B, T, H, T, 1,
                                      pf::SEG_V_ZERO | pf::SEG_H0_EYE | pf::SEG_NO_O,
                                      cluster_fits((int64_t)B * H), nullptr, 0, stream);
    note_launches(1);
    return e;
}

// S_{p+1} = M_p S_p + N_p over P consecutive segments of each (b, h):
// M, N, S_start: [B][P][H][D][D]; h0, hT: [B][H][D][D] (either may be null).
cudaError_t state_chain_launch(const float* M, const float* N, const float* h0, float* S_start, float* hT,
                               int B, int P, int H, cudaStream_t stream)
{
    {
        const cudaError_t e = set_prefill_attributes();
        if (e != cudaSuccess) return e;
    }
    segment_combine_kernel<<<dim3(pf::D / SEG_COLS, B * H), 256, SEG_COMBINE_SMEM, stream>>>(
        M, N, S_start, h0, hT, H, P);
    note_launches(1);
    return cudaGetLastError();
}

// Self-test of the bounded waits: one warp waits on an mbarrier that nothing
// completes, gives up after limit_ns and records KDA_ERR_TIMEOUT exactly as
// the prefill kernel does.  No fault, trap or unbounded wait is involved.
__global__ void bounded_wait_selftest_kernel(uint64_t limit_ns)
{
    __shared__ __align__(8) uint64_t bar;
    if (threadIdx.x == 0) {
        tc::mbar_init(tc::smem_u32(&bar), 1);
        tc::fence_mbar_init();
    }
    __syncwarp();
    if (threadIdx.x == 0 && !tc::mbar_wait(tc::smem_u32(&bar), 0, limit_ns))
        atomicExch(&g_prefill_status, (int)KDA_ERR_TIMEOUT);
}

cudaError_t bounded_wait_selftest_launch(uint64_t limit_ns, cudaStream_t stream)
{
    bounded_wait_selftest_kernel<<<1, 32, 0, stream>>>(limit_ns);
    note_launches(1);
    return cudaGetLastError();
}

// Reads and clears the timeout flag of the prefill kernels (blocking).
int prefill_device_status(cudaStream_t stream)
{
    int st = 0, zero = 0;
    if (cudaMemcpyFromSymbolAsync(&st, g_prefill_status, sizeof(int), 0,
                                  cudaMemcpyDeviceToHost, stream) != cudaSuccess)
        return KDA_ERR_CUDA;
    if (cudaMemcpyToSymbolAsync(g_prefill_status, &zero, sizeof(int), 0,
                                cudaMemcpyHostToDevice, stream) != cudaSuccess)
        return KDA_ERR_CUDA;
    if (cudaStreamSynchronize(stream) != cudaSuccess) return KDA_ERR_CUDA;
    return st;
}

}  // namespace kda
