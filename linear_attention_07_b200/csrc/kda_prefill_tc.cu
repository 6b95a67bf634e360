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
// One CTA of 256 threads per (batch, head), d_k = d_v = 128, two roles:
//   * chain warpgroup (warps 0-3): thread j owns column j of the fp32 state S
//     in registers.  Per chunk: X = S^T [W | Qt]^T (tf32 copy of S^T in tensor
//     memory as the A operand, M 128, N 64, K 128), U^T = U'^T - X_W into
//     tensor memory, S^T += U^T Kb (N 128, K 32) and O^T += U^T P^T (N 32,
//     K 32), then the decay/update of S and the bf16 store of o.
//   * prep warpgroup (warps 4-7): for the next chunk, the decay scaling
//     (two channels per thread), the Gram MMA Kh' [Kt | Qt]^T (M 64: rows
//     Kh of both tiles and Kb of tile 0), the 32x32 unit-triangular solve
//     (block-wise, all 128 threads), and W^T = Kt^T T^T, U'^T = V^T T^T
//     (M 128, N 32, K 32).  It then fills the chain's operand buffers.
// The two roles meet at two named-barrier rendezvous per chunk: "free" (the
// chain no longer reads the operand buffers) and "ready" (the next chunk's
// operands are in place).  Inputs of the next chunk are prefetched with
// cp.async while the current one is processed.
//
// All MMAs are tf32 with operands rounded to nearest (cvt.rna): bf16
// operands would leave errors of a few percent of rms(o) on these products
// (the q.k diagonal times a large u), tf32 leaves ~0.3%.
// Shared-memory operands use the no-swizzle K-major layout; when the thread
// that produces a value owns the K index, the K-direction core-matrix stride
// is padded to 144 B so that a warp's scalar stores hit distinct banks.
#include "kda_common.cuh"
#include "kda_tc.cuh"

namespace kda {

namespace pf {

constexpr int D = 128;         // d_k = d_v
constexpr int TILE = 16;
constexpr int C = 32;          // tokens per chunk (two tiles)
constexpr int NT = 256;        // threads per CTA: chain + prep warpgroups

constexpr uint32_t PAD_LBO = 144;            // padded K-direction core-matrix stride
constexpr uint32_t LBO = 128;                // dense K-direction core-matrix stride
constexpr uint32_t SBO_K128P = (D / 4) * PAD_LBO;   // 4608: K = 128, padded
constexpr uint32_t SBO_K32 = (C / 4) * LBO;         // 1024: K = 32, dense
constexpr uint32_t SBO_K32P = (C / 4) * PAD_LBO;    // 1152: K = 32, padded

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
constexpr uint32_t GAM = B3 + (C / 8) * SBO_K32P;              // gamma_C, 128 fp32
constexpr int LD = C + 1;                                      // scratch row stride (floats)
constexpr uint32_t AMS = GAM + D * 4;                          // A (32 x 33 fp32)
constexpr uint32_t PMS = AMS + C * LD * 4;                     // P
constexpr uint32_t XMS = PMS + C * LD * 4;                     // diagonal-block inverses
constexpr uint32_t TMS = XMS + C * LD * 4;                     // T
constexpr uint32_t YMS = TMS + C * LD * 4;                     // A_10 X_00 (16 x 17)
constexpr uint32_t OST = YMS + TILE * (TILE + 1) * 4;           // o staging, 32 x 128 bf16
constexpr uint32_t SMEM_BYTES = OST + C * D * 2;

static_assert(SMEM_BYTES <= 227 * 1024, "shared memory budget");
static_assert(OST % 16 == 0 && GA % 16 == 0 && GB % 16 == 0 && WA % 16 == 0 && VA % 16 == 0 && TB % 16 == 0 &&
              B1 % 16 == 0 && B2 % 16 == 0 && B3 % 16 == 0, "descriptor alignment");

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
// 16-byte asynchronous global->shared copy; src_bytes = 0 writes zeros
__device__ __forceinline__ void cp_async16(void* dst, const void* src, uint32_t src_bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;"
                 :: "r"(tc::smem_u32(dst)), "l"(src), "r"(src_bytes) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }

__global__ void __launch_bounds__(pf::NT, 1)
prefill_tc_kernel(const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k,
                  const __nv_bfloat16* __restrict__ v, const __nv_bfloat16* __restrict__ g,
                  const __nv_bfloat16* __restrict__ beta, const float* h0,
                  __nv_bfloat16* __restrict__ o, float* hT, int T, int H)
{
    using namespace pf;
    using namespace tc;
    extern __shared__ __align__(1024) unsigned char sm[];
    __shared__ uint32_t s_taddr;
    __shared__ __align__(8) uint64_t s_bar[2];     // [0] chain MMAs, [1] prep MMAs
    __shared__ int s_abort;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int h = blockIdx.x, b = blockIdx.y;
    const int64_t head_off = (int64_t)b * H + h;
    const int64_t row_stride = (int64_t)H * D;            // elements between tokens
    const int64_t base = ((int64_t)b * T * H + h) * D;    // token 0 of this head

    if (warp == 0) {
        tmem_alloc(smem_u32(&s_taddr), TMEM_COLS);
        tmem_relinquish();
    }
    if (tid == 0) {
        mbar_init(smem_u32(&s_bar[0]), 1);
        mbar_init(smem_u32(&s_bar[1]), 1);
        fence_mbar_init();
        s_abort = 0;
    }
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    const uint32_t tm = s_taddr;
    const uint32_t lane_base = (uint32_t)(32 * (warp & 3)) << 16;   // this warp's TMEM lanes
    const int n_chunks = (T + C - 1) / C;

    if (warp < 4) {
        // =================================================== chain warpgroup ==
        const int j = tid;
        const uint32_t bar = smem_u32(&s_bar[0]);
        uint32_t phase = 0;
        auto wait_mma = [&]() {
            const bool ok = mbar_wait(bar, phase & 1u, WAIT_NS);
            ++phase;
            if (!ok) {
                s_abort = 1;
                atomicExch(&g_prefill_status, (int)KDA_ERR_TIMEOUT);
            }
            fence_after_sync();
        };
        float S[D];
        {
            const float* h0h = h0 ? h0 + head_off * D * D : nullptr;
#pragma unroll
            for (int c = 0; c < D; ++c) S[c] = h0h ? h0h[(int64_t)c * D + j] : 0.f;
#pragma unroll
            for (int c0 = 0; c0 < D; c0 += 32) {
                float t32[32];
#pragma unroll
                for (int i = 0; i < 32; ++i) t32[i] = to_tf32(S[c0 + i]);
                tmem_st32(tm + lane_base + T_AS + c0, t32);
            }
            wait_st();
        }
        __nv_bfloat16* oh = o + base;
#pragma unroll 1
        for (int ch = 0; ch < n_chunks; ++ch) {
            fence_before_sync();
            named_bar(BAR_FREE, NT);
            named_bar(BAR_READY, NT);
            fence_after_sync();
            if (s_abort) break;
            // X = S^T [W | Qt]^T  (one N = 64 MMA per K step; the issue loop is
            // unrolled with constant descriptor increments: the per-instruction
            // issue cost, not the math, bounds these small-N MMAs)
            if (j == 0) {
                const uint32_t id = idesc_tf32(128, 2 * C, false, false);
                const uint64_t bd0 = sdesc(smem_u32(sm + B1), PAD_LBO, SBO_K128P);
#pragma unroll
                for (int ks = 0; ks < D / 8; ++ks)
                    mma_tf32_ts(tm + T_DX, tm + T_AS + ks * 8, bd0 + (uint64_t)((ks * 2 * PAD_LBO) >> 4),
                                id, ks > 0 ? 1u : 0u);
                mma_commit(bar);
            }
            __syncwarp();
            wait_mma();
            {   // U = U' - W S (thread j: 32 tokens)
                float x[16], up[16];
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    tmem_ld16(tm + lane_base + T_DX + half * 16, x);
                    tmem_ld16(tm + lane_base + T_DU + (ch & 1) * C + half * 16, up);
                    wait_ld();
#pragma unroll
                    for (int r = 0; r < 16; ++r) x[r] = to_tf32(up[r] - x[r]);
                    tmem_st16(tm + lane_base + T_AU + half * 16, x);
                }
                wait_st();
            }
            fence_before_sync();
            named_bar(BAR_CHAIN, 128);
            fence_after_sync();
            if (j == 0) {
                const uint32_t id2 = idesc_tf32(128, 128, false, false);
                const uint32_t id3 = idesc_tf32(128, 32, false, false);
                const uint64_t b20 = sdesc(smem_u32(sm + B2), LBO, SBO_K32);
                const uint64_t b30 = sdesc(smem_u32(sm + B3), PAD_LBO, SBO_K32P);
#pragma unroll
                for (int ks = 0; ks < C / 8; ++ks) {
                    mma_tf32_ts(tm + T_DKU, tm + T_AU + ks * 8, b20 + (uint64_t)((ks * 2 * LBO) >> 4),
                                id2, ks > 0 ? 1u : 0u);
                    mma_tf32_ts(tm + T_DX + C, tm + T_AU + ks * 8, b30 + (uint64_t)((ks * 2 * PAD_LBO) >> 4),
                                id3, 1u);
                }
                mma_commit(bar);
            }
            __syncwarp();
            wait_mma();
            {   // S <- Diag(gamma_C) S + Kb^T U ; refresh the tf32 copy; emit o
                const float4* gam4 = reinterpret_cast<const float4*>(sm + GAM);
#pragma unroll
                for (int c0 = 0; c0 < D; c0 += 32) {
                    float d[32];
                    tmem_ld32(tm + lane_base + T_DKU + c0, d);
                    wait_ld();
#pragma unroll
                    for (int i4 = 0; i4 < 8; ++i4) {
                        const float4 gv = gam4[(c0 >> 2) + i4];
                        const float gg[4] = {gv.x, gv.y, gv.z, gv.w};
#pragma unroll
                        for (int u = 0; u < 4; ++u) {
                            const int i = i4 * 4 + u;
                            S[c0 + i] = fmaf(gg[u], S[c0 + i], d[i]);
                            d[i] = to_tf32(S[c0 + i]);
                        }
                    }
                    tmem_st32(tm + lane_base + T_AS + c0, d);
                }
                // o: column j of the chunk's 32 x 128 tile into shared memory,
                // then whole rows to global memory in 16-byte vectors
                __nv_bfloat16* ost = reinterpret_cast<__nv_bfloat16*>(sm + OST);
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    float ov[16];
                    tmem_ld16(tm + lane_base + T_DX + C + half * 16, ov);
                    wait_ld();
#pragma unroll
                    for (int r = 0; r < 16; ++r) ost[(half * 16 + r) * D + j] = __float2bfloat16_rn(ov[r]);
                }
                wait_st();
                named_bar(BAR_CHAIN, 128);
                const int tb = ch * C;
#pragma unroll
                for (int m = 0; m < (C * D / 8) / 128; ++m) {
                    const int vi = j + m * 128;
                    const int r = vi / (D / 8), cv = vi % (D / 8);
                    if (tb + r < T)
                        *reinterpret_cast<uint4*>(oh + (int64_t)(tb + r) * row_stride + cv * 8) =
                            *reinterpret_cast<const uint4*>(ost + r * D + cv * 8);
                }
            }
        }
        if (hT && !s_abort) {
            float* hTh = hT + head_off * D * D;
#pragma unroll
            for (int c = 0; c < D; ++c) hTh[(int64_t)c * D + j] = S[c];
        }
    } else {
        // ==================================================== prep warpgroup ==
        const int pt = tid - 128;                  // 0..127
        const int sp = warp & 3;                   // TMEM sub-partition of this warp
        const uint32_t bar = smem_u32(&s_bar[1]);
        uint32_t phase = 0;
        auto wait_mma = [&]() {
            const bool ok = mbar_wait(bar, phase & 1u, WAIT_NS);
            ++phase;
            if (!ok) {
                s_abort = 1;
                atomicExch(&g_prefill_status, (int)KDA_ERR_TIMEOUT);
            }
            fence_after_sync();
        };
        auto prep_sync = [&]() { named_bar(BAR_PREP, 128); };
        auto issue_raw = [&](int ci) {   // cp.async of chunk ci's q, k, v, g rows
            const int tb = ci * C;
#pragma unroll
            for (int it = 0; it < (4 * C * (D / 8)) / 128; ++it) {
                const int idx = pt + it * 128;
                const int tensor = idx / (C * (D / 8));
                const int rem = idx % (C * (D / 8));
                const int r = rem / (D / 8), vec = rem % (D / 8);
                const bool in = tb + r < T;
                const __nv_bfloat16* src = (tensor == 0 ? q : tensor == 1 ? k : tensor == 2 ? v : g) + base;
                cp_async16(sm + RAW + tensor * RAW_T + (r * D + vec * 8) * 2,
                           in ? (const void*)(src + (int64_t)(tb + r) * row_stride + vec * 8)
                              : (const void*)src,
                           in ? 16u : 0u);
            }
            cp_async_commit();
        };
        if (n_chunks > 0) issue_raw(0);

        // this thread's decay-scaling slice: tile tau, channels c0, c0 + 1
        const int tau = pt >> 6;
        const int c0 = (pt & 63) * 2;
        float* am = reinterpret_cast<float*>(sm + AMS);
        float* pm = reinterpret_cast<float*>(sm + PMS);
        float* xm = reinterpret_cast<float*>(sm + XMS);
        float* tmx = reinterpret_cast<float*>(sm + TMS);
        float* ym = reinterpret_cast<float*>(sm + YMS);
        const float* bt = reinterpret_cast<const float*>(sm + BETA);
#pragma unroll 1
        for (int ch = 0; ch < n_chunks; ++ch) {
            const int t0 = ch * C;
            // ---- inputs of this chunk
            if (pt < C)
                reinterpret_cast<float*>(sm + BETA)[pt] =
                    (t0 + pt < T) ? to_f32(beta[((int64_t)b * T + t0 + pt) * H + h]) : 0.f;
            cp_async_wait_all();
            prep_sync();

            // ---- decay scaling (thread: 16 tokens of tile tau x 2 channels)
            float qtv[2][TILE], kbv[2][TILE];       // kept for the operand fill
            float gam_c0, gam_c1;
            {
                const __nv_bfloat162* rq = reinterpret_cast<const __nv_bfloat162*>(sm + RAW + 0 * RAW_T);
                const __nv_bfloat162* rk = reinterpret_cast<const __nv_bfloat162*>(sm + RAW + 1 * RAW_T);
                const __nv_bfloat162* rv = reinterpret_cast<const __nv_bfloat162*>(sm + RAW + 2 * RAW_T);
                const __nv_bfloat162* rg = reinterpret_cast<const __nv_bfloat162*>(sm + RAW + 3 * RAW_T);
                // all shared-memory reads of this slice first (independent of the
                // stores below, so they are not ordered behind them)
                __nv_bfloat162 Rq[TILE], Rk[TILE], Rv[TILE], Rg[TILE];
#pragma unroll
                for (int rr = 0; rr < TILE; ++rr) {
                    const int idx = ((tau * TILE + rr) * D + c0) >> 1;
                    Rq[rr] = rq[idx];
                    Rk[rr] = rk[idx];
                    Rv[rr] = rv[idx];
                    Rg[rr] = rg[idx];
                }
                float a0[TILE], a1[TILE];
                float e0 = 1.f, e1 = 1.f;
#pragma unroll
                for (int rr = 0; rr < TILE; ++rr) {
                    const float2 gg = __bfloat1622float2(Rg[rr]);
                    a0[rr] = __expf(gg.x);
                    a1[rr] = __expf(gg.y);
                    e0 *= a0[rr];
                    e1 *= a1[rr];
                }
                float* gex = reinterpret_cast<float*>(sm + GEX);
                gex[tau * D + c0] = e0;
                gex[tau * D + c0 + 1] = e1;
                prep_sync();
                const float o0 = gex[(1 - tau) * D + c0], o1 = gex[(1 - tau) * D + c0 + 1];
                // chunk-relative factors: tile 1 rows carry tile 0's decay
                const float f0 = tau ? o0 : 1.f, f1 = tau ? o1 : 1.f;
                gam_c0 = e0 * o0;
                gam_c1 = e1 * o1;
                // forward: Kt, Qt (tile-relative) for the Gram; Kt (chunk) for W;
                // Qt (chunk) kept for the state product's B operand
                float p0 = 1.f, p1 = 1.f;
                float kc0[4], kc1[4];
#pragma unroll
                for (int rr = 0; rr < TILE; ++rr) {
                    const int r = tau * TILE + rr;
                    p0 *= a0[rr];
                    p1 *= a1[rr];
                    const float2 kk = __bfloat1622float2(Rk[rr]);
                    const float2 qq = __bfloat1622float2(Rq[rr]);
                    const float kt0 = kk.x * p0, kt1 = kk.y * p1;
                    const float qt0 = qq.x * p0, qt1 = qq.y * p1;
                    st_f32x2(sm, GB + off_kmajor(r, c0, PAD_LBO, SBO_K128P), to_tf32(kt0), to_tf32(kt1));
                    st_f32x2(sm, GB + off_kmajor(C + r, c0, PAD_LBO, SBO_K128P), to_tf32(qt0), to_tf32(qt1));
                    qtv[0][rr] = to_tf32(qt0 * f0);
                    qtv[1][rr] = to_tf32(qt1 * f1);
                    kc0[rr & 3] = to_tf32(kt0 * f0);
                    kc1[rr & 3] = to_tf32(kt1 * f1);
                    if ((rr & 3) == 3) {
                        st_f32x4(sm, WA + off_kmajor(c0, r - 3, LBO, SBO_K32), kc0[0], kc0[1], kc0[2], kc0[3]);
                        st_f32x4(sm, WA + off_kmajor(c0 + 1, r - 3, LBO, SBO_K32), kc1[0], kc1[1], kc1[2], kc1[3]);
                    }
                }
                // backward: Kb (tile-relative suffix), Kh = Kb / gamma_tile,
                // Kb (chunk-relative) kept for the update's B operand
                const float i0 = 1.f / e0, i1 = 1.f / e1;
                const float h0f = tau ? 1.f : o0, h1f = tau ? 1.f : o1;   // tile 0 rows carry tile 1's decay
                float s0 = 1.f, s1 = 1.f;
#pragma unroll
                for (int rr = TILE - 1; rr >= 0; --rr) {
                    const int r = tau * TILE + rr;
                    const float2 kk = __bfloat1622float2(Rk[rr]);
                    const float kb0 = kk.x * s0, kb1 = kk.y * s1;
                    st_f32x2(sm, GA + off_kmajor(r, c0, PAD_LBO, SBO_K128P), to_tf32(kb0 * i0), to_tf32(kb1 * i1));
                    if (tau == 0)
                        st_f32x2(sm, GA + off_kmajor(C + rr, c0, PAD_LBO, SBO_K128P), to_tf32(kb0), to_tf32(kb1));
                    kbv[0][rr] = to_tf32(kb0 * h0f);
                    kbv[1][rr] = to_tf32(kb1 * h1f);
                    s0 *= a0[rr];
                    s1 *= a1[rr];
                }
                // V^T: thread's two value columns over its 16 tokens
#pragma unroll
                for (int rr = 0; rr < TILE; rr += 4) {
                    const int r = tau * TILE + rr;
                    float2 vv[4];
#pragma unroll
                    for (int u = 0; u < 4; ++u) vv[u] = __bfloat1622float2(Rv[rr + u]);
                    st_f32x4(sm, VA + off_kmajor(c0, r, LBO, SBO_K32),
                             to_tf32(vv[0].x), to_tf32(vv[1].x), to_tf32(vv[2].x), to_tf32(vv[3].x));
                    st_f32x4(sm, VA + off_kmajor(c0 + 1, r, LBO, SBO_K32),
                             to_tf32(vv[0].y), to_tf32(vv[1].y), to_tf32(vv[2].y), to_tf32(vv[3].y));
                }
            }
            fence_smem_to_async();
            fence_before_sync();
            prep_sync();                     // raw buffer consumed, operands written
            fence_after_sync();
            if (ch + 1 < n_chunks) issue_raw(ch + 1);

            // ---- Gram: D_G = [Kh_0; Kh_1; Kb_0; pad] [Kt_0 Kt_1 | Qt_0 Qt_1]^T
            if (pt == 0) {
                const uint32_t id = idesc_tf32(64, 64, false, false);
                const uint64_t ad0 = sdesc(smem_u32(sm + GA), PAD_LBO, SBO_K128P);
                const uint64_t bd0 = sdesc(smem_u32(sm + GB), PAD_LBO, SBO_K128P);
#pragma unroll
                for (int ks = 0; ks < D / 8; ++ks) {
                    const uint64_t step = (uint64_t)((ks * 2 * PAD_LBO) >> 4);
                    mma_tf32_ss(tm + T_DG, ad0 + step, bd0 + step, id, ks > 0 ? 1u : 0u);
                }
                mma_commit(bar);
            }
            __syncwarp();
            wait_mma();

            // ---- A and P (32 x 32) into scratch; row m of D_G is lane (m % 16) + 32 (m / 16)
            if (sp < 3) {
                // sp 0: rows Kh_0 (cols Kt_0, Qt_0); sp 1: rows Kh_1 (cols Kt_1, Qt_1);
                // sp 2: rows Kb_0 (cols Kt_1, Qt_1): the block between the tiles
                const int colK = (sp == 0) ? 0 : TILE;
                float gk[16], gq[16];
                tmem_ld16(tm + lane_base + T_DG + colK, gk);
                tmem_ld16(tm + lane_base + T_DG + C + colK, gq);
                wait_ld();
                if (lane < TILE) {
                    const int i = (sp == 1 ? TILE : 0) + lane;           // column of A / P
                    const int rbase = (sp == 0) ? 0 : TILE;              // rows covered
#pragma unroll
                    for (int r = 0; r < TILE; ++r) {
                        const int rg = rbase + r;
                        am[rg * LD + i] = (rg > i) ? bt[rg] * gk[r] : 0.f;
                        pm[rg * LD + i] = (rg >= i) ? gq[r] : 0.f;
                    }
                    if (sp == 1) {                                        // upper-right block is zero
#pragma unroll
                        for (int r = 0; r < TILE; ++r) {
                            am[r * LD + i] = 0.f;
                            pm[r * LD + i] = 0.f;
                        }
                    }
                }
            }
            prep_sync();
            // ---- diagonal blocks: X = (I + A_tt)^-1, column by column (right-looking)
            if (sp < 2 && lane < TILE) {
                const int off = sp * TILE;
                const int i = lane;
                float x[TILE];
#pragma unroll
                for (int r = 0; r < TILE; ++r) x[r] = (r == i) ? 1.f : 0.f;
#pragma unroll
                for (int s = 0; s < TILE; ++s) {
#pragma unroll
                    for (int r = s + 1; r < TILE; ++r)
                        x[r] = fmaf(-am[(off + r) * LD + off + s], x[s], x[r]);
                }
                const float bi = bt[off + i];
#pragma unroll
                for (int r = 0; r < TILE; ++r) {
                    xm[(off + r) * LD + off + i] = x[r];
                    tmx[(off + r) * LD + off + i] = x[r] * bi;            // T_tt = X_tt diag(b)
                    if (sp == 1) tmx[r * LD + off + i] = 0.f;            // T_01 = 0
                }
            }
            prep_sync();
            // ---- off-diagonal block: T_10 = -X_11 (A_10 X_00) diag(b_0)
            {
                const int r = pt >> 3, i = (pt & 7) * 2;
                float y0 = 0.f, y1 = 0.f;
#pragma unroll
                for (int s = 0; s < TILE; ++s) {
                    const float a = am[(TILE + r) * LD + s];
                    y0 = fmaf(a, xm[s * LD + i], y0);
                    y1 = fmaf(a, xm[s * LD + i + 1], y1);
                }
                ym[r * (TILE + 1) + i] = y0;
                ym[r * (TILE + 1) + i + 1] = y1;
            }
            prep_sync();
            {
                const int r = pt >> 3, i = (pt & 7) * 2;
                float z0 = 0.f, z1 = 0.f;
#pragma unroll
                for (int s = 0; s < TILE; ++s) {
                    const float x = xm[(TILE + r) * LD + TILE + s];
                    z0 = fmaf(x, ym[s * (TILE + 1) + i], z0);
                    z1 = fmaf(x, ym[s * (TILE + 1) + i + 1], z1);
                }
                tmx[(TILE + r) * LD + i] = -z0 * bt[i];
                tmx[(TILE + r) * LD + i + 1] = -z1 * bt[i + 1];
            }
            prep_sync();
            // ---- T into the B operand of the W / U' products: element (n = r, k = i)
            {
                const int r = pt >> 2, i = (pt & 3) * 8;
                const float* row = tmx + r * LD + i;
                st_f32x4(sm, TB + off_kmajor(r, i, PAD_LBO, SBO_K32P),
                         to_tf32(row[0]), to_tf32(row[1]), to_tf32(row[2]), to_tf32(row[3]));
                st_f32x4(sm, TB + off_kmajor(r, i + 4, PAD_LBO, SBO_K32P),
                         to_tf32(row[4]), to_tf32(row[5]), to_tf32(row[6]), to_tf32(row[7]));
            }
            fence_smem_to_async();
            fence_before_sync();
            prep_sync();
            fence_after_sync();
            // ---- W^T = Kt^T T^T and U'^T = V^T T^T  (M 128, N 32, K 32)
            if (pt == 0) {
                const uint32_t id = idesc_tf32(128, 32, false, false);
                const uint64_t bd0 = sdesc(smem_u32(sm + TB), PAD_LBO, SBO_K32P);
                const uint64_t aw0 = sdesc(smem_u32(sm + WA), LBO, SBO_K32);
                const uint64_t av0 = sdesc(smem_u32(sm + VA), LBO, SBO_K32);
                const uint32_t du = tm + T_DU + (ch & 1) * C;
#pragma unroll
                for (int ks = 0; ks < C / 8; ++ks) {
                    const uint64_t bstep = (uint64_t)((ks * 2 * PAD_LBO) >> 4);
                    const uint64_t astep = (uint64_t)((ks * 2 * LBO) >> 4);
                    mma_tf32_ss(tm + T_DW, aw0 + astep, bd0 + bstep, id, ks > 0 ? 1u : 0u);
                    mma_tf32_ss(du, av0 + astep, bd0 + bstep, id, ks > 0 ? 1u : 0u);
                }
                mma_commit(bar);
            }
            __syncwarp();
            wait_mma();

            // ---- hand the chunk's operands to the chain
            fence_before_sync();
            named_bar(BAR_FREE, NT);         // the chain no longer reads B1, B2, B3, GAM
            fence_after_sync();
            {
                // W (thread = key channel pt): rows 0-31 of B1
                float w[16];
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    tmem_ld16(tm + lane_base + T_DW + half * 16, w);
                    wait_ld();
#pragma unroll
                    for (int r = 0; r < 16; ++r)
                        st_f32(sm, B1 + off_kmajor(half * 16 + r, pt, PAD_LBO, SBO_K128P), to_tf32(w[r]));
                }
                // Qt (chunk-relative): rows 32-63 of B1; Kb (chunk-relative): B2
#pragma unroll
                for (int rr = 0; rr < TILE; ++rr) {
                    const int r = tau * TILE + rr;
                    st_f32x2(sm, B1 + off_kmajor(C + r, c0, PAD_LBO, SBO_K128P), qtv[0][rr], qtv[1][rr]);
                }
#pragma unroll
                for (int rr = 0; rr < TILE; rr += 4) {
                    const int r = tau * TILE + rr;
                    st_f32x4(sm, B2 + off_kmajor(c0, r, LBO, SBO_K32),
                             kbv[0][rr], kbv[0][rr + 1], kbv[0][rr + 2], kbv[0][rr + 3]);
                    st_f32x4(sm, B2 + off_kmajor(c0 + 1, r, LBO, SBO_K32),
                             kbv[1][rr], kbv[1][rr + 1], kbv[1][rr + 2], kbv[1][rr + 3]);
                }
                // P: element (n = r, k = i)
                {
                    const int r = pt >> 2, i = (pt & 3) * 8;
                    const float* row = pm + r * LD + i;
                    st_f32x4(sm, B3 + off_kmajor(r, i, PAD_LBO, SBO_K32P),
                             to_tf32(row[0]), to_tf32(row[1]), to_tf32(row[2]), to_tf32(row[3]));
                    st_f32x4(sm, B3 + off_kmajor(r, i + 4, PAD_LBO, SBO_K32P),
                             to_tf32(row[4]), to_tf32(row[5]), to_tf32(row[6]), to_tf32(row[7]));
                }
                if (tau == 0) {
                    float* gam = reinterpret_cast<float*>(sm + GAM);
                    gam[c0] = gam_c0;
                    gam[c0 + 1] = gam_c1;
                }
            }
            fence_smem_to_async();
            fence_before_sync();
            named_bar(BAR_READY, NT);
            fence_after_sync();
            if (s_abort) break;
        }
        cp_async_wait_all();
    }

    fence_before_sync();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tm, TMEM_COLS);
}

cudaError_t prefill_tc_launch(const void* q, const void* k, const void* v, const void* g,
                              const void* beta, const float* h0, void* o, float* hT,
                              int B, int T, int H, cudaStream_t stream)
{
    static bool attr_set = false;   // idempotent; races only repeat the same call
    if (!attr_set) {
        cudaError_t e = cudaFuncSetAttribute(prefill_tc_kernel,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)pf::SMEM_BYTES);
        if (e != cudaSuccess) return e;
        attr_set = true;
    }
    dim3 grid(H, B);
    prefill_tc_kernel<<<grid, pf::NT, pf::SMEM_BYTES, stream>>>(
        (const __nv_bfloat16*)q, (const __nv_bfloat16*)k, (const __nv_bfloat16*)v,
        (const __nv_bfloat16*)g, (const __nv_bfloat16*)beta, h0, (__nv_bfloat16*)o, hT, T, H);
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
