// KDA backward (training): the gradients of L = sum(dO * o) + sum(dhT * hT)
// with respect to q, k, v, g, beta and h0, for d_k = d_v = 128.
//
// The pages give the forward recurrence only ("T11E1: K3 tech report"
// transcript, the KDA turn; "Kimi K3 goes trillion-scale ..." subtitles, cue
// 14) and name 8K-64K pre-training lengths (transcript, the context-length
// turn); the backward is the derivative of the chunked forward taken chunk by
// chunk.  Per 32-token chunk with start state S0 (Gam the in-chunk running
// sum of g, gam = exp(Gam), gC = gam of the last token):
//     Kt = K gam, Qt = Q gam, Kb = K exp(Gam_C - Gam),
//     A  = diag(beta) strict_lower(Araw),  Araw_ri = sum_c k_rc k_ic exp(Gam_rc - Gam_ic),
//     P  = lower_incl(Praw),               Praw_ri = sum_c q_rc k_ic exp(Gam_rc - Gam_ic),
//     X  = (I + A)^-1,  Tm = X diag(beta),  W = Tm Kt,  U = Tm V - W S0,
//     O  = Qt S0 + P U,  S_C = Diag(gC) S0 + Kb^T U.
// Backward, with dS = dL/dS_C:
//     dU = P^T dO + Kb dS,   dS0 = Diag(gC) dS - W^T (Kb dS) + (Qt - P W)^T dO,
// and the chunk-local gradients of Tm, W, U, P, Kt, Qt, Kb, V and the decay.
// The decayed pair products (Araw, Praw and their gradients) are never formed
// with a chunk-relative 1/gam, which leaves fp32 after 17 tokens at the -5
// log-decay floor: a pair (r, i) inside one 16-token tile uses the tile start
// as reference (factors <= 1 and <= e^80), a pair across the two tiles the
// tile boundary (both factors <= 1) -- the bound of the transcript's
// log-decay-bound turn.
//
// Three launches, all fp32 arithmetic on CUDA cores:
//   1. bwd_prep_kernel   (one CTA per chunk): Araw, Praw, X, W, U' = Tm V,
//                         Z = Qt - P W, Kb, gC -> workspace;
//   2. bwd_chains_kernel (one CTA per (b, h, 32 state columns), two halves
//                         side by side): the forward state chain
//                         S <- Diag(gC) S + Kb^T (U' - W S), writing every
//                         chunk's start state, and the reverse chain
//                         dS <- Diag(gC) dS - W^T (Kb dS) + Z^T dO, writing every
//                         chunk's end gradient and dh0 (state columns are
//                         independent in both chains);
//   3. bwd_local_kernel  (one CTA per chunk): dq, dk, dv, dg, dbeta.
// The start states come from an fp32 chain rather than the tf32 forward
// kernel: dg sums terms that nearly cancel, and state errors at the tf32
// level (about 1e-3) move it by about 1e-2 of its scale.
#include "kda_common.cuh"
#include "kda_tc.cuh"

namespace kda {
namespace bw {

__device__ int g_bwd_status;     // set to KDA_ERR_TIMEOUT by a wait that expired
constexpr uint64_t DRAIN_NS = 20000000ull;   // after an expired wait: 20 ms for the MMAs in flight

constexpr int D = 128, C = 32, TILE = 16, NT = 256;
constexpr int LD = D + 1;        // odd row stride: conflict-free row and column walks
constexpr int L32 = C + 1;
constexpr int NS = 32;           // state columns per chain CTA
constexpr int JB = 16;           // state columns per block in the local kernel
constexpr int LJ = JB + 1;

// per-chunk record written by the prep kernel (floats)
constexpr int R_KB = 0, R_W = R_KB + C * D, R_UP = R_W + C * D, R_Z = R_UP + C * D, R_GC = R_Z + C * D,
              R_A = R_GC + D, R_P = R_A + C * C, R_X = R_P + C * C, R_FLOATS = R_X + C * C;
static_assert(R_FLOATS % 4 == 0, "records stay 16-byte aligned");

__device__ __forceinline__ float bf(const __nv_bfloat16 x) { return __bfloat162float(x); }

// Rows [t0, t0 + C) of one head of a [B][T][H][D] bf16 tensor into shared
// memory (row stride LD), zero past Tl.
template <int NTH = NT>
__device__ __forceinline__ void load_rows(float* dst, const __nv_bfloat16* __restrict__ src, int64_t row0,
                                          int64_t row_stride, int n_valid)
{
    for (int v = threadIdx.x; v < C * (D / 8); v += NTH) {
        const int r = v / (D / 8), c8 = (v % (D / 8)) * 8;
        float f[8];
        if (r < n_valid) {
            const uint4 u = *reinterpret_cast<const uint4*>(src + row0 + (int64_t)r * row_stride + c8);
            const __nv_bfloat162* p = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const float2 x = __bfloat1622float2(p[j]);
                f[2 * j] = x.x;
                f[2 * j + 1] = x.y;
            }
        } else {
#pragma unroll
            for (int j = 0; j < 8; ++j) f[j] = 0.f;
        }
#pragma unroll
        for (int j = 0; j < 8; ++j) dst[r * LD + c8 + j] = f[j];
    }
}

// Running sum of g over the chunk, per channel, in place.
__device__ __forceinline__ void running_sum(float* G)
{
    if (threadIdx.x < D) {
        float s = 0.f;
        for (int r = 0; r < C; ++r) {
            s += G[r * LD + threadIdx.x];
            G[r * LD + threadIdx.x] = s;
        }
    }
}

// The fused prologue on a chunk's rows in shared memory (row stride LD), as
// the raw forward applies it: q and k scaled to unit norm over the channels
// (rsqrt of the sum of squares; a zero row stays zero), the gate
// pre-activation z turned into g = -5 sigmoid(z) (g = 0 past the end of the
// sequence).  Any of the pointers may be null; the inverse norms are kept
// for the chain rule.
template <int NTH>
__device__ __forceinline__ void prologue_rows(float* sQ, float* invQ, float* sK, float* invK, float* sG, int n_valid)
{
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (int r = warp; r < C; r += NTH / 32) {
        float sq = 0.f, sk = 0.f;
#pragma unroll
        for (int j = 0; j < D / 32; ++j) {
            const int c = lane + 32 * j;
            if (sQ) sq = fmaf(sQ[r * LD + c], sQ[r * LD + c], sq);
            if (sK) sk = fmaf(sK[r * LD + c], sK[r * LD + c], sk);
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
            sq += __shfl_xor_sync(0xffffffffu, sq, off);
            sk += __shfl_xor_sync(0xffffffffu, sk, off);
        }
        const float iq = sq > 0.f ? rsqrtf(sq) : 0.f, ik = sk > 0.f ? rsqrtf(sk) : 0.f;
#pragma unroll
        for (int j = 0; j < D / 32; ++j) {
            const int c = lane + 32 * j;
            if (sQ) sQ[r * LD + c] *= iq;
            if (sK) sK[r * LD + c] *= ik;
            if (sG) sG[r * LD + c] = r < n_valid ? -5.f / (1.f + __expf(-sG[r * LD + c])) : 0.f;
        }
        if (lane == 0) {
            if (invQ) invQ[r] = iq;
            if (invK) invK[r] = ik;
        }
    }
}

// Reference of the tile-relative factors of row r: Gam before its tile.
__device__ __forceinline__ float tile_ref(const float* G, int r, int c)
{
    return r >= TILE ? G[(TILE - 1) * LD + c] : 0.f;
}

// Block GEMM on shared-memory operands, fp32 FMA, all NTH threads:
// out(m, n, sum_k a(m, k) b(k, n)) for an M x N result.  Thread (tm, tn)
// computes rows tm * TM .. + TM - 1 and columns tn + NC j: consecutive
// threads read consecutive columns of a row-major b (or one column each of
// a transposed one; odd row strides keep both conflict-free) and share the
// a values (broadcast).
template <int M, int N, int K, int TM, int TN, int NTH = NT, typename FA, typename FB, typename FO>
__device__ __forceinline__ void tgemm(FA a, FB b, FO out)
{
    constexpr int NC = N / TN, NR = M / TM;
    static_assert(NC * NR == NTH && NC * TN == N && NR * TM == M, "tile shape");
    const int t = threadIdx.x, tn = t % NC, tm = t / NC;
    float acc[TM][TN];
#pragma unroll
    for (int i = 0; i < TM; ++i)
#pragma unroll
        for (int j = 0; j < TN; ++j) acc[i][j] = 0.f;
#pragma unroll 4
    for (int k = 0; k < K; ++k) {
        float av[TM], bv[TN];
#pragma unroll
        for (int i = 0; i < TM; ++i) av[i] = a(tm * TM + i, k);
#pragma unroll
        for (int j = 0; j < TN; ++j) bv[j] = b(k, tn + NC * j);
#pragma unroll
        for (int i = 0; i < TM; ++i)
#pragma unroll
            for (int j = 0; j < TN; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
    }
#pragma unroll
    for (int i = 0; i < TM; ++i)
#pragma unroll
        for (int j = 0; j < TN; ++j) out(tm * TM + i, tn + NC * j, acc[i][j]);
}

// Block GEMM for a small output and a long K: a TM x TN register tile per
// thread over one of KS slices of K, the KS slices of a tile in KS
// consecutive lanes and summed with shuffles (every lane then writes TM TN /
// KS of the tile's outputs).  A slice takes four consecutive k out of every
// 4 KS, so the lanes of a slice group read k values four apart: with odd
// row strides the transposed reads of b fall on distinct banks.
template <int M, int N, int K, int TM, int TN, int KS, int NTH, typename FA, typename FB, typename FO>
__device__ __forceinline__ void tgemm_ks(FA a, FB b, FO out)
{
    constexpr int NC = N / TN, NR = M / TM;
    static_assert(NC * NR * KS == NTH && NC * TN == N && NR * TM == M, "tile shape");
    static_assert(K % (4 * KS) == 0 && (KS & (KS - 1)) == 0 && KS <= 32 && (TM * TN) % KS == 0, "K slices");
    const int t = threadIdx.x, ks = t % KS, tile = t / KS, tn = tile % NC, tm = tile / NC;
    float acc[TM][TN];
#pragma unroll
    for (int i = 0; i < TM; ++i)
#pragma unroll
        for (int j = 0; j < TN; ++j) acc[i][j] = 0.f;
#pragma unroll 2
    for (int q = 0; q < K / (4 * KS); ++q) {
#pragma unroll
        for (int r = 0; r < 4; ++r) {
            const int k = q * 4 * KS + 4 * ks + r;
            float av[TM], bv[TN];
#pragma unroll
            for (int i = 0; i < TM; ++i) av[i] = a(tm * TM + i, k);
#pragma unroll
            for (int j = 0; j < TN; ++j) bv[j] = b(k, tn + NC * j);
#pragma unroll
            for (int i = 0; i < TM; ++i)
#pragma unroll
                for (int j = 0; j < TN; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
        }
    }
#pragma unroll
    for (int off = 1; off < KS; off <<= 1)
#pragma unroll
        for (int i = 0; i < TM; ++i)
#pragma unroll
            for (int j = 0; j < TN; ++j) acc[i][j] += __shfl_xor_sync(0xffffffffu, acc[i][j], off);
#pragma unroll
    for (int e = 0; e < TM * TN; ++e)
        if (e % KS == ks) out(tm * TM + e / TN, tn + NC * (e % TN), acc[e / TN][e % TN]);
}

// ---------------------------------------------------------------- prep --

// Six [C][LD] arrays (buffers reused as their contents die) and three
// [C][L32] ones: 111,872 bytes, so two CTAs share an SM and overlap their
// serial phases (the triangular solve runs on one warp).
constexpr size_t PREP_SMEM = (size_t)(6 * C * LD + 3 * C * L32 + C) * sizeof(float);

template <bool RAW>    // RAW: q, k unnormalised and g the gate pre-activation (the fused prologue)
__global__ void __launch_bounds__(NT, 2)
bwd_prep_kernel(const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k,
                const __nv_bfloat16* __restrict__ v, const __nv_bfloat16* __restrict__ g,
                const __nv_bfloat16* __restrict__ beta, float* __restrict__ rec_all, int T, int H, int n_chunks)
{
    extern __shared__ __align__(16) float sm[];
    float* sK = sm;                // K, then V (from the pair products on)
    float* sQ = sK + C * LD;       // Q, then Kc in rows 0-15 (cross-tile pairs)
    float* sG = sQ + C * LD;       // G, the running sum of g
    float* s1 = sG + C * LD;       // Ka, then Kt
    float* s2 = s1 + C * LD;       // Qa, then U'
    float* s3 = s2 + C * LD;       // Kf, then W
    float* sA = s3 + C * LD;       // Araw
    float* sP = sA + C * L32;      // Praw (lower incl)
    float* sX = sP + C * L32;      // (I + A)^-1; Tm = X diag(beta) is formed on the fly
    float* sB = sX + C * L32;      // beta

    const int c_idx = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int t0 = c_idx * C;
    const int Tl = min(C, T - t0);
    const int tid = threadIdx.x;
    const int64_t rs = (int64_t)H * D;
    const int64_t row0 = ((int64_t)b * T + t0) * rs + (int64_t)h * D;
    float* rec = rec_all + (((int64_t)b * H + h) * n_chunks + c_idx) * R_FLOATS;
    auto Tm = [&](int r, int i) { return sX[r * L32 + i] * sB[i]; };

    load_rows(sK, k, row0, rs, Tl);
    load_rows(sQ, q, row0, rs, Tl);
    load_rows(sG, g, row0, rs, Tl);
    if (tid < C) sB[tid] = tid < Tl ? bf(beta[((int64_t)b * T + t0 + tid) * H + h]) : 0.f;
    __syncthreads();
    if constexpr (RAW) {
        prologue_rows<NT>(sQ, nullptr, sK, nullptr, sG, Tl);
        __syncthreads();
    }
    running_sum(sG);
    __syncthreads();
    // tile-relative operands of the pair products; Kb and gC go straight to the
    // record.  Each (r, c) is read and written by one thread, so Kc may take
    // the place of Q in rows 0-15.
    for (int e = tid; e < C * D; e += NT) {
        const int r = e / D, c = e % D;
        const float Gr = sG[r * LD + c], ref = tile_ref(sG, r, c);
        const float kk = sK[r * LD + c], qq = sQ[r * LD + c];
        const float a = __expf(Gr - ref);
        s1[r * LD + c] = kk * a;                                  // Ka
        s2[r * LD + c] = qq * a;                                  // Qa
        s3[r * LD + c] = kk * __expf(ref - Gr);                   // Kf (<= e^80)
        rec[R_KB + e] = kk * __expf(sG[(C - 1) * LD + c] - Gr);   // Kb
        if (r < TILE) sQ[r * LD + c] = kk * __expf(sG[(TILE - 1) * LD + c] - Gr);   // Kc (<= 1)
    }
    if (tid < D) rec[R_GC + tid] = __expf(sG[(C - 1) * LD + tid]);
    // V, read from global memory now and stored where K was once the pair
    // products are done
    constexpr int VPT = C * (D / 8) / NT;                     // 16-byte vectors per thread
    uint4 vr[VPT];
#pragma unroll
    for (int u = 0; u < VPT; ++u) {
        const int e = tid + u * NT, r = e / (D / 8), c8 = (e % (D / 8)) * 8;
        vr[u] = r < Tl ? *reinterpret_cast<const uint4*>(v + row0 + (int64_t)r * rs + c8) : make_uint4(0u, 0u, 0u, 0u);
    }
    __syncthreads();
    // Araw (strict lower) and Praw (lower incl) as block products: pairs inside
    // one tile from Ka / Qa against Kf (the full 32 x 32 product is finite:
    // the entries of mixed tiles, whose factors do not belong together, are
    // dropped), pairs across the tiles (rows of tile 1, columns of tile 0)
    // from Ka / Qa against Kc
    {
        auto same = [&](float* dst, const float* L, bool strict) {
            tgemm_ks<C, C, D, 4, 4, 4, NT>([&](int m, int kk) { return L[m * LD + kk]; },
                                 [&](int kk, int n) { return s3[n * LD + kk]; },
                                 [&](int m, int n, float x) {
                                     if (m / TILE == n / TILE) dst[m * L32 + n] = (n < m || (!strict && n == m)) ? x : 0.f;
                                     else if (n > m) dst[m * L32 + n] = 0.f;
                                 });
        };
        auto cross = [&](float* dst, const float* L) {
            tgemm<TILE, TILE, D, 1, 1>([&](int m, int kk) { return L[(TILE + m) * LD + kk]; },
                                       [&](int kk, int n) { return sQ[n * LD + kk]; },
                                       [&](int m, int n, float x) { dst[(TILE + m) * L32 + n] = x; });
        };
        same(sA, s1, true);
        same(sP, s2, false);
        cross(sA, s1);
        cross(sP, s2);
    }
#pragma unroll
    for (int u = 0; u < VPT; ++u) {
        const int e = tid + u * NT, r = e / (D / 8), c8 = (e % (D / 8)) * 8;
        const __nv_bfloat162* p2 = reinterpret_cast<const __nv_bfloat162*>(&vr[u]);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const float2 x = __bfloat1622float2(p2[j]);
            sK[r * LD + c8 + 2 * j] = x.x;
            sK[r * LD + c8 + 2 * j + 1] = x.y;
        }
    }
    __syncthreads();
    // Kt = K gam = Ka exp(ref) in place (Ka is no longer read); X = (I +
    // diag(beta) Araw)^-1 by forward substitution, one column per thread (four
    // partial sums per row keep the chain short)
    for (int e = tid; e < C * D; e += NT) {
        const int r = e / D, c = e % D;
        s1[r * LD + c] *= __expf(tile_ref(sG, r, c));
    }
    if (tid < C) {
        const int j = tid;
        float x[C];
#pragma unroll
        for (int r = 0; r < C; ++r) {
            float s4v[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int i = 0; i < r; ++i) s4v[i & 3] = fmaf(sA[r * L32 + i], x[i], s4v[i & 3]);
            const float s = (s4v[0] + s4v[1]) + (s4v[2] + s4v[3]);
            x[r] = (r == j) ? 1.f : (r > j ? -sB[r] * s : 0.f);
        }
#pragma unroll
        for (int r = 0; r < C; ++r) sX[r * L32 + j] = x[r];
    }
    __syncthreads();
    // W = Tm Kt -> s3 (Kf is no longer read)
    tgemm<C, D, C, 4, 4>([&](int m, int kk) { return Tm(m, kk); },
                         [&](int kk, int n) { return s1[kk * LD + n]; },
                         [&](int m, int n, float x) { s3[m * LD + n] = x; });
    __syncthreads();
    // Z = Qt - P W -> record, with Qt = Q gam = Qa exp(ref)
    tgemm<C, D, C, 4, 4>([&](int m, int kk) { return sP[m * L32 + kk]; },
                         [&](int kk, int n) { return s3[kk * LD + n]; },
                         [&](int m, int n, float x) {
                             rec[R_Z + m * D + n] = s2[m * LD + n] * __expf(tile_ref(sG, m, n)) - x;
                         });
    __syncthreads();
    // U' = Tm V -> s2 (Qa is no longer read)
    tgemm<C, D, C, 4, 4>([&](int m, int kk) { return Tm(m, kk); },
                         [&](int kk, int n) { return sK[kk * LD + n]; },
                         [&](int m, int n, float x) { s2[m * LD + n] = x; });
    __syncthreads();
    for (int e = tid; e < C * D; e += NT) {
        const int r = e / D, c = e % D;
        rec[R_W + e] = s3[r * LD + c];
        rec[R_UP + e] = s2[r * LD + c];
    }
    for (int e = tid; e < C * C; e += NT) {
        const int r = e / C, i = e % C;
        rec[R_A + e] = sA[r * L32 + i];
        rec[R_P + e] = sP[r * L32 + i];
        rec[R_X + e] = sX[r * L32 + i];
    }
}

// --------------------------------------------------------------- chains --
// Per (b, h, NS state columns), both chains in one CTA of 512 threads: the
// forward chain (threads 0-255) writes the start state of every chunk to
// S0_all[b][h][c]; the reverse chain (threads 256-511) writes the gradient at
// the end of every chunk to dS_all[b][h][c] and the start-state gradient to
// dh0.  The reverse chain needs only the per-chunk operands and dO, not the
// forward's states, so the two run side by side, each half with its own
// shared memory and named barrier.  Each operand buffer is refilled for the
// next chunk (cp.async) as soon as the step that reads it is done: step 1's
// operand after step 1, step 2's after step 2.

constexpr int CLD = D + 4;        // operand rows: 528 B, 16-byte aligned
constexpr int XLD = NS + 4;       // state / Y rows: 144 B
// one chain's shared memory: step-1 operand [C][CLD] (+ U' slice [C][XLD]
// forward), step-2 operands (Kb, or W and Z) [C][CLD] each (+ dO slice and gC),
// the state slice [D][XLD], Y [C][XLD] and step 1's partial sums over four K
// slices [4][C][XLD]
constexpr int FWD_FLOATS = 2 * C * CLD + 2 * C * XLD + D + D * XLD + C * XLD + 4 * C * XLD;
constexpr int REV_FLOATS = 3 * C * CLD + C * XLD + D + D * XLD + C * XLD + 4 * C * XLD;
constexpr size_t CHAIN_SMEM = (size_t)(FWD_FLOATS + REV_FLOATS) * sizeof(float);
constexpr int NT_CHAIN = 2 * NT;

__device__ __forceinline__ void cp_async16(void* dst, const void* src)
{
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;"
                 :: "r"((uint32_t)__cvta_generic_to_shared(dst)), "l"(src) : "memory");
}
// Bulk prefetch of `bytes` (a multiple of 16, 16-byte aligned start) into L2.
__device__ __forceinline__ void l2_prefetch(const void* p, uint32_t bytes)
{
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" :: "l"(p), "r"(bytes) : "memory");
}
__device__ __forceinline__ void cp_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_wait_1() { asm volatile("cp.async.wait_group 1;" ::: "memory"); }
__device__ __forceinline__ void half_sync(uint32_t id) { asm volatile("bar.sync %0, %1;" :: "r"(id), "r"(NT) : "memory"); }

// One chain over this CTA's state columns [j0, j0 + NS), run by NT threads
// (tid = 0 .. NT - 1) that synchronise on named barrier `bar`.
template <bool REV>
__device__ __forceinline__ void chain_run(float* sm, int tid, uint32_t bar, const float* __restrict__ rec_h,
                                          const __nv_bfloat16* __restrict__ dO, const float* S_init,
                                          float* __restrict__ S_all_h, float* out_last, int j0,
                                          int64_t bh, int b, int h, int T, int H, int n_chunks)
{
    float* o1 = sm;                                       // step 1: W (forward) or Kb (reverse)
    float* oU = o1 + C * CLD;                             // forward: U' slice [C][XLD]
    float* o2 = REV ? oU : oU + C * XLD;                  // step 2: Kb (forward) or W (reverse)
    float* oZ = o2 + C * CLD;                             // reverse: Z
    float* oS = REV ? oZ + C * CLD : o2 + C * CLD;        // reverse: dO slice (bf16 rows); forward: unused
    float* oG = REV ? oS + C * XLD : oS + C * XLD;        // gC [D]
    float* sXs = oG + D;                                  // state slice [D][XLD]
    float* sY = sXs + D * XLD;                            // [C][XLD]
    float* sYp = sY + C * XLD;                            // step-1 partial sums, 4 K slices [4][C][XLD]

    auto fill_rows = [&](float* dst, const float* src) {  // [C][D] fp32 record rows -> [C][CLD]
        for (int e = tid; e < C * (D / 4); e += NT) {
            const int row = e / (D / 4), c4 = (e % (D / 4)) * 4;
            cp_async16(dst + row * CLD + c4, src + row * D + c4);
        }
    };
    // step-1 operands of chunk c
    auto fetch1 = [&](int c) {
        const float* r = rec_h + (int64_t)c * R_FLOATS;
        fill_rows(o1, r + (REV ? R_KB : R_W));
        if (!REV)
            for (int e = tid; e < C * (NS / 4); e += NT) {
                const int row = e / (NS / 4), c4 = (e % (NS / 4)) * 4;
                cp_async16(oU + row * XLD + c4, r + R_UP + row * D + j0 + c4);
            }
        cp_commit();
    };
    // step-2 operands of chunk c
    auto fetch2 = [&](int c) {
        const float* r = rec_h + (int64_t)c * R_FLOATS;
        fill_rows(o2, r + (REV ? R_W : R_KB));
        if (REV) {
            fill_rows(oZ, r + R_Z);
            const int t0 = c * C;
            for (int e = tid; e < C * (NS / 8); e += NT) {
                const int row = e / (NS / 8), c8 = (e % (NS / 8)) * 8;
                __nv_bfloat16* d = reinterpret_cast<__nv_bfloat16*>(oS + row * XLD) + c8;
                if (t0 + row < T)
                    cp_async16(d, dO + (((int64_t)b * T + t0 + row) * H + h) * D + j0 + c8);
                else
                    *reinterpret_cast<uint4*>(d) = make_uint4(0u, 0u, 0u, 0u);
            }
        }
        for (int e = tid; e < D / 4; e += NT) cp_async16(oG + 4 * e, r + R_GC + 4 * e);
        cp_commit();
    };

    // state slice: thread (ig, cg) owns rows 4 ig .. 4 ig + 3, columns 4 cg .. 4 cg + 3
    // (float4 reads of its step-2 operand rows)
    const int ig = tid / (NS / 4), cg = tid % (NS / 4);
    float xr[4][4];
#pragma unroll
    for (int m = 0; m < 4; ++m) {
        const int i = 4 * ig + m;
        float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
        if (S_init) x = *reinterpret_cast<const float4*>(S_init + bh * D * D + (int64_t)i * D + j0 + 4 * cg);
        xr[m][0] = x.x; xr[m][1] = x.y; xr[m][2] = x.z; xr[m][3] = x.w;
        *reinterpret_cast<float4*>(sXs + i * XLD + 4 * cg) = x;
    }
    const int first = REV ? n_chunks - 1 : 0;
    const int step = REV ? -1 : 1;
    if (n_chunks > 0) {
        fetch1(first);
        fetch2(first);
    }
#pragma unroll 1
    for (int n = 0; n < n_chunks; ++n) {
        const int c = first + step * n;
        const bool more = n + 1 < n_chunks;
        // the state at this chunk boundary
        float* dst = S_all_h + (int64_t)c * D * D;
#pragma unroll
        for (int m = 0; m < 4; ++m)
            *reinterpret_cast<float4*>(dst + (int64_t)(4 * ig + m) * D + j0 + 4 * cg) =
                make_float4(xr[m][0], xr[m][1], xr[m][2], xr[m][3]);
        cp_wait_1();                         // step-1 operands of chunk c (step 2's may be in flight)
        half_sync(bar);
        {   // step 1, partial sums: thread (rows 4 r4 .. + 3, columns 4 cq .. + 3,
            // K slice [32 ks, 32 ks + 32)); a 4 x 4 register tile per slice
            // reads one float4 of X and four scalars of the operand per k
            const int cq = tid & 7, r4 = (tid >> 3) & 7, ks = tid >> 6;
            float acc[4][4];
#pragma unroll
            for (int m = 0; m < 4; ++m)
#pragma unroll
                for (int u = 0; u < 4; ++u) acc[m][u] = 0.f;
#pragma unroll 4
            for (int kk = 0; kk < 32; ++kk) {
                const int i = 32 * ks + kk;
                const float4 x = *reinterpret_cast<const float4*>(sXs + i * XLD + 4 * cq);
#pragma unroll
                for (int m = 0; m < 4; ++m) {
                    const float w = o1[(4 * r4 + m) * CLD + i];
                    acc[m][0] = fmaf(w, x.x, acc[m][0]); acc[m][1] = fmaf(w, x.y, acc[m][1]);
                    acc[m][2] = fmaf(w, x.z, acc[m][2]); acc[m][3] = fmaf(w, x.w, acc[m][3]);
                }
            }
#pragma unroll
            for (int m = 0; m < 4; ++m)
                *reinterpret_cast<float4*>(sYp + (ks * C + 4 * r4 + m) * XLD + 4 * cq) =
                    make_float4(acc[m][0], acc[m][1], acc[m][2], acc[m][3]);
        }
        half_sync(bar);                      // partial sums complete; the step-1 buffer is free
        {   // Y = U'_s - W X (forward) or Y = -(Kb X) (reverse); thread (r, cg)
            const int r = tid / (NS / 4);
            float4 y = *reinterpret_cast<const float4*>(sYp + r * XLD + 4 * cg);
#pragma unroll
            for (int k2 = 1; k2 < 4; ++k2) {
                const float4 p = *reinterpret_cast<const float4*>(sYp + (k2 * C + r) * XLD + 4 * cg);
                y = make_float4(y.x + p.x, y.y + p.y, y.z + p.z, y.w + p.w);
            }
            if (!REV) {
                const float4 u = *reinterpret_cast<const float4*>(oU + r * XLD + 4 * cg);
                y = make_float4(u.x - y.x, u.y - y.y, u.z - y.z, u.w - y.w);
            } else {
                y = make_float4(-y.x, -y.y, -y.z, -y.w);      // enters as -W^T (Kb dS)
            }
            *reinterpret_cast<float4*>(sY + r * XLD + 4 * cg) = y;
        }
        half_sync(bar);                      // Y complete
        if (more) fetch1(c + step); else cp_commit();
        cp_wait_1();                         // step-2 operands of chunk c
        half_sync(bar);
        {   // step 2: X = Diag(gC) X + Kb^T Y (forward) or X = Diag(gC) X + W^T Y + Z^T dO (reverse)
            float acc[4][4];
            {
                const float4 g4 = *reinterpret_cast<const float4*>(oG + 4 * ig);
                const float gcv[4] = {g4.x, g4.y, g4.z, g4.w};
#pragma unroll
                for (int m = 0; m < 4; ++m)
#pragma unroll
                    for (int u = 0; u < 4; ++u) acc[m][u] = gcv[m] * xr[m][u];
            }
#pragma unroll 4
            for (int r = 0; r < C; ++r) {
                const float4 y = *reinterpret_cast<const float4*>(sY + r * XLD + 4 * cg);
                const float4 b4 = *reinterpret_cast<const float4*>(o2 + r * CLD + 4 * ig);
                const float bb[4] = {b4.x, b4.y, b4.z, b4.w};
#pragma unroll
                for (int m = 0; m < 4; ++m) {
                    acc[m][0] = fmaf(bb[m], y.x, acc[m][0]); acc[m][1] = fmaf(bb[m], y.y, acc[m][1]);
                    acc[m][2] = fmaf(bb[m], y.z, acc[m][2]); acc[m][3] = fmaf(bb[m], y.w, acc[m][3]);
                }
            }
            if (REV) {
                const __nv_bfloat16* dOs = reinterpret_cast<const __nv_bfloat16*>(oS);
#pragma unroll 4
                for (int r = 0; r < C; ++r) {
                    const __nv_bfloat162* d2 = reinterpret_cast<const __nv_bfloat162*>(dOs + r * 2 * XLD + 4 * cg);
                    const float2 d01 = __bfloat1622float2(d2[0]), d23 = __bfloat1622float2(d2[1]);
                    const float4 z4 = *reinterpret_cast<const float4*>(oZ + r * CLD + 4 * ig);
                    const float z[4] = {z4.x, z4.y, z4.z, z4.w};
#pragma unroll
                    for (int m = 0; m < 4; ++m) {
                        acc[m][0] = fmaf(z[m], d01.x, acc[m][0]); acc[m][1] = fmaf(z[m], d01.y, acc[m][1]);
                        acc[m][2] = fmaf(z[m], d23.x, acc[m][2]); acc[m][3] = fmaf(z[m], d23.y, acc[m][3]);
                    }
                }
            }
#pragma unroll
            for (int m = 0; m < 4; ++m) {
#pragma unroll
                for (int u = 0; u < 4; ++u) xr[m][u] = acc[m][u];
                *reinterpret_cast<float4*>(sXs + (4 * ig + m) * XLD + 4 * cg) =
                    make_float4(acc[m][0], acc[m][1], acc[m][2], acc[m][3]);
            }
        }
        half_sync(bar);                      // state written; the step-2 buffers are free
        if (more) fetch2(c + step); else cp_commit();
    }
    if (out_last) {
#pragma unroll
        for (int m = 0; m < 4; ++m)
            *reinterpret_cast<float4*>(out_last + bh * D * D + (int64_t)(4 * ig + m) * D + j0 + 4 * cg) =
                make_float4(xr[m][0], xr[m][1], xr[m][2], xr[m][3]);
    }
}

__global__ void __launch_bounds__(NT_CHAIN, 1)
bwd_chains_kernel(const float* __restrict__ rec_all, const __nv_bfloat16* __restrict__ dO,
                  const float* h0, const float* dhT, float* __restrict__ S0_all, float* __restrict__ dS_all,
                  float* dh0, int T, int H, int n_chunks)
{
    extern __shared__ __align__(16) float sm[];
    const int s = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int64_t bh = (int64_t)b * H + h;
    const float* rec_h = rec_all + bh * n_chunks * R_FLOATS;
    if (threadIdx.x < NT)
        chain_run<false>(sm, threadIdx.x, 1, rec_h, dO, h0, S0_all + bh * n_chunks * D * D, nullptr,
                         s * NS, bh, b, h, T, H, n_chunks);
    else
        chain_run<true>(sm + FWD_FLOATS, threadIdx.x - NT, 2, rec_h, dO, dhT, dS_all + bh * n_chunks * D * D,
                        dh0, s * NS, bh, b, h, T, H, n_chunks);
}

// ---------------------------------------------------------- local grads --
// One CTA per chunk.  The state-sized products stream S0 and dS through
// shared memory twice: by rows (the K dimension of U = Tm V - W S0 and
// dU = P^T dO + Kb dS, accumulated over the rows), then by columns (the K
// dimension of dQt = dO S0^T, dKb = U dS^T and dW = -dU S0^T).  Every block
// product gives each thread a 4 x 4 tile of a 32 x 128 result.

constexpr int LOC_BIG = 11;    // K, Q, V, dO, G, W, U, dU, dKb, dQt, dW
constexpr int BLK = D * LJ > JB * LD ? D * LJ : JB * LD;    // one S0 or dS block (either shape)
constexpr size_t LOC_SMEM = (size_t)(LOC_BIG * C * LD + 2 * BLK + 6 * C * L32 + 4 * C + 2 * D) * sizeof(float);
constexpr int NL = 2 * NT;     // threads of the local kernel: 16 warps hide the shared-memory latency

__device__ __forceinline__ __nv_bfloat16 to_bf(float x) { return __float2bfloat16_rn(x); }

template <bool RAW>    // RAW: the fused prologue, and its chain rule on dq, dk, dg
__global__ void __launch_bounds__(NL, 1)
bwd_local_kernel(const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k,
                 const __nv_bfloat16* __restrict__ v, const __nv_bfloat16* __restrict__ g,
                 const __nv_bfloat16* __restrict__ beta, const __nv_bfloat16* __restrict__ dO,
                 const float* __restrict__ rec_all, const float* __restrict__ S0_all,
                 const float* __restrict__ dS_all,
                 __nv_bfloat16* __restrict__ dq, __nv_bfloat16* __restrict__ dk, __nv_bfloat16* __restrict__ dv,
                 __nv_bfloat16* __restrict__ dg, __nv_bfloat16* __restrict__ dbeta, int T, int H, int n_chunks,
                 uint64_t wait_ns)
{
    using namespace tc;
    extern __shared__ __align__(16) float sm[];
    __shared__ uint32_t s_taddr;
    __shared__ __align__(8) uint64_t s_mbar;
    __shared__ int s_abort;
    float* bK = sm;
    float* bQ = bK + C * LD;       // Kb during the state products, then Q
    float* bV = bQ + C * LD;       // V, then dGam
    float* bDO = bV + C * LD;      // dO, then dKt (from dW), then Kf
    float* bG = bDO + C * LD;      // Gam
    float* bW = bG + C * LD;       // W, then Kt, then Ka
    float* bU = bW + C * LD;       // U
    float* bDU = bU + C * LD;      // dU
    float* bDKB = bDU + C * LD;    // dKb -> dk
    float* bDQT = bDKB + C * LD;   // dQt (direct) -> dq
    float* bDW = bDQT + C * LD;    // dW, then Qa
    float* bS0 = bDW + C * LD;     // a block of S0 (rows: [JB][LD], columns: [D][LJ]), then Kc
    float* bDS = bS0 + BLK;        // the same block of dS
    float* sA = bDS + BLK;         // Araw
    float* sP = sA + C * L32;      // Praw (lower incl)
    float* sX = sP + C * L32;      // (I + A)^-1; Tm = X diag(beta) is formed on the fly
    float* sdP = sX + C * L32;     // dO U^T (masked to lower incl)
    float* sdUV = sdP + C * L32;   // dU V^T, then dX X^T
    float* sdT = sdUV + C * L32;   // dTm, then dX, then dA (unscaled), then dAr
    float* sB = sdT + C * L32;     // beta [C]
    float* sDB = sB + C;           // dbeta [C]
    float* sRS = sDB + C;          // sum_j dS_ij S0_ij [D]
    float* sKS = sRS + D;          // sum_r dKb_rc Kb_rc [D]
    float* sIQ = sKS + D;          // RAW: 1 / |q_raw| per token [C]
    float* sIK = sIQ + C;          // RAW: 1 / |k_raw| per token [C]

    const int c_idx = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int t0 = c_idx * C;
    const int Tl = min(C, T - t0);
    const int tid = threadIdx.x;
    const int64_t rs = (int64_t)H * D;
    const int64_t row0 = ((int64_t)b * T + t0) * rs + (int64_t)h * D;
    const int64_t bh = (int64_t)b * H + h;
    const float* rec = rec_all + (bh * n_chunks + c_idx) * R_FLOATS;
    const float* S0 = S0_all + (bh * n_chunks + c_idx) * D * D;
    const float* dS = dS_all + (bh * n_chunks + c_idx) * D * D;
    auto Tm = [&](int r, int i) { return sX[r * L32 + i] * sB[i]; };

    // tensor memory (the whole of it: one CTA per SM) and the MMA barrier
    if (tid < 32) {
        tmem_alloc(smem_u32(&s_taddr), 512);
        tmem_relinquish();
    }
    if (tid == 0) {
        mbar_init(smem_u32(&s_mbar), 1);
        fence_mbar_init();
        s_abort = 0;
    }
    fence_before_sync();
    __syncthreads();
    fence_after_sync();

    if (tid == 0) {                        // the chunk's states and record, on their way to L2
        l2_prefetch(S0, D * D * 4);
        l2_prefetch(dS, D * D * 4);
        l2_prefetch(rec, R_FLOATS * 4);
    }
    // ---- inputs, the prep record and the chunk's decay
    load_rows<NL>(bK, k, row0, rs, Tl);
    load_rows<NL>(bV, v, row0, rs, Tl);
    load_rows<NL>(bDO, dO, row0, rs, Tl);
    load_rows<NL>(bG, g, row0, rs, Tl);
    if (tid < C) {
        sB[tid] = tid < Tl ? bf(beta[((int64_t)b * T + t0 + tid) * H + h]) : 0.f;
        sDB[tid] = 0.f;
    }
    for (int e = tid; e < C * D; e += NL) {
        const int r = e / D, c = e % D;
        bW[r * LD + c] = rec[R_W + e];
    }
    for (int e = tid; e < C * C; e += NL) {
        const int r = e / C, i = e % C;
        sA[r * L32 + i] = rec[R_A + e];
        sP[r * L32 + i] = rec[R_P + e];
        sX[r * L32 + i] = rec[R_X + e];
    }
    __syncthreads();
    if constexpr (RAW) {
        prologue_rows<NL>(nullptr, nullptr, bK, sIK, bG, Tl);
        __syncthreads();
    }
    running_sum(bG);
    __syncthreads();
    for (int e = tid; e < C * D; e += NL) {                       // Kb = K exp(Gam_C - Gam)
        const int r = e / D, c = e % D;
        bQ[r * LD + c] = bK[r * LD + c] * __expf(bG[(C - 1) * LD + c] - bG[r * LD + c]);
    }
    // U = Tm V and dU = P^T dO, before the state terms
    tgemm<C, D, C, 2, 4, NL>([&](int m, int kk) { return Tm(m, kk); },
                         [&](int kk, int n) { return bV[kk * LD + n]; },
                         [&](int m, int n, float x) { bU[m * LD + n] = x; });
    tgemm<C, D, C, 2, 4, NL>([&](int m, int kk) { return sP[kk * L32 + m]; },
                         [&](int kk, int n) { return bDO[kk * LD + n]; },
                         [&](int m, int n, float x) { bDU[m * LD + n] = x; });
    __syncthreads();

    // ---- the five state-sized products on the tensor cores (tf32 operands,
    // fp32 sums), each as the transposed product with the 128-wide state
    // dimension as the MMA's M and the 32 tokens as N:
    //   phase A: (W S0)^T = S0^T W^T and (Kb dS)^T = dS^T Kb^T, A = S0^T, dS^T
    //            in tensor memory (lane = d_v row), B = W, Kb;
    //   phase B: dQt^T = S0 dO^T, dKb^T = dS U^T, (dU S0^T)^T = S0 dU^T,
    //            A = S0, dS in tensor memory (lane = d_k row), B = dO, U, dU.
    // B operands are K-major without swizzle, dense: element (n, k) at byte
    // (n / 8) * 4096 + (k / 4) * 128 + (n % 8) * 16 + (k % 4) * 4 (16 KB each),
    // in the space of dKb, dQt and dW, which are written only after phase B.
    // Tensor memory: A at columns 0-255 (phase A: S0^T, dS^T; phase B: S0, dS);
    // results at 256 (W S0), 288 (Kb dS), 320 (dQt), 352 (dKb), 384 (dU S0^T).
    const uint32_t tm = s_taddr;
    const int wp = tid >> 5, lane = tid & 31;
    const int spw = wp & 3, cg = wp >> 2;                 // sub-partition, column group 0..3
    const uint32_t lane_base = (uint32_t)(32 * spw) << 16;
    const int mrow = 32 * spw + lane;                      // tensor-memory lane of this thread
    float* bop = bDKB;                                     // B operands: 3 x 16 KB over dKb, dQt, dW
    const uint32_t idn = idesc_tf32(128, C, false, false);
    const uint32_t mbar = smem_u32(&s_mbar);
    uint32_t n_commit = 0;                                 // commits on s_mbar (issued by warp 0)
    auto expired = [&]() {
        s_abort = 1;
        atomicExch(&g_bwd_status, (int)KDA_ERR_TIMEOUT);
    };
    // a [C][LD] fp32 matrix into a B operand, rounded to tf32 (lanes: n % 8,
    // then k / 4, so a warp stores 512 contiguous bytes)
    auto put_b = [&](float* dst, const float* src) {
        for (int e = tid; e < C * (D / 4); e += NL) {
            const int n8 = e & 7, k4 = (e >> 3) & 31, ng = e >> 8;
            const float* x = src + (8 * ng + n8) * LD + 4 * k4;
            *reinterpret_cast<float4*>(reinterpret_cast<char*>(dst) + ng * 4096 + k4 * 128 + n8 * 16) =
                make_float4(to_tf32(x[0]), to_tf32(x[1]), to_tf32(x[2]), to_tf32(x[3]));
        }
    };
    auto issue = [&](uint32_t d_col, uint32_t a_col, const float* b) {
        const uint64_t b0 = sdesc(smem_u32(b), 128, 4096);
#pragma unroll
        for (int ks = 0; ks < D / 8; ++ks)
            mma_tf32_ts_w(tm + d_col, tm + a_col + ks * 8, b0 + (uint64_t)(ks * 16), idn, ks > 0 ? 1u : 0u);
    };
    auto wait_mma = [&](uint32_t parity) {
        if (!s_abort && !mbar_wait(mbar, parity, wait_ns)) expired();
        fence_after_sync();
    };

    // phase A
    put_b(bop, bW);
    put_b(bop + C * D, bQ);                                // Kb
    {
        float t32[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) t32[i] = to_tf32(S0[(int64_t)(32 * cg + i) * D + mrow]);
        tmem_st32(tm + lane_base + 32 * cg, t32);
#pragma unroll
        for (int i = 0; i < 32; ++i) t32[i] = to_tf32(dS[(int64_t)(32 * cg + i) * D + mrow]);
        tmem_st32(tm + lane_base + 128 + 32 * cg, t32);
        wait_st();
    }
    fence_smem_to_async();
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    if (wp == 0) {
        issue(256, 0, bop);
        issue(288, 128, bop + C * D);
        mma_commit_w(mbar);
        ++n_commit;
    }
    wait_mma(0);
    {   // U -= W S0, dU += Kb dS (this thread: d_v row mrow, tokens [8 cg, 8 cg + 8))
        float v8[8];
        tmem_ld8(tm + lane_base + 256 + 8 * cg, v8);
        wait_ld();
#pragma unroll
        for (int u = 0; u < 8; ++u) bU[(8 * cg + u) * LD + mrow] -= v8[u];
        tmem_ld8(tm + lane_base + 288 + 8 * cg, v8);
        wait_ld();
#pragma unroll
        for (int u = 0; u < 8; ++u) bDU[(8 * cg + u) * LD + mrow] += v8[u];
    }
    fence_before_sync();
    __syncthreads();
    fence_after_sync();

    // phase B
    put_b(bop, bDO);
    put_b(bop + C * D, bU);
    put_b(bop + 2 * C * D, bDU);
    {
        // S0 and dS rows (this thread: d_k row mrow, d_v columns [32 cg, 32 cg + 32)),
        // and this slice of sum_j dS_ij S0_ij
        const float4* s4 = reinterpret_cast<const float4*>(S0 + (int64_t)mrow * D + 32 * cg);
        const float4* d4 = reinterpret_cast<const float4*>(dS + (int64_t)mrow * D + 32 * cg);
        float rsum = 0.f;
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
            float t16[16], d16[16];
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4) {
                const float4 a4 = s4[4 * hf + q4], b4 = d4[4 * hf + q4];
                rsum = fmaf(a4.x, b4.x, fmaf(a4.y, b4.y, fmaf(a4.z, b4.z, fmaf(a4.w, b4.w, rsum))));
                t16[4 * q4] = to_tf32(a4.x); t16[4 * q4 + 1] = to_tf32(a4.y);
                t16[4 * q4 + 2] = to_tf32(a4.z); t16[4 * q4 + 3] = to_tf32(a4.w);
                d16[4 * q4] = to_tf32(b4.x); d16[4 * q4 + 1] = to_tf32(b4.y);
                d16[4 * q4 + 2] = to_tf32(b4.z); d16[4 * q4 + 3] = to_tf32(b4.w);
            }
            tmem_st16(tm + lane_base + 32 * cg + 16 * hf, t16);
            tmem_st16(tm + lane_base + 128 + 32 * cg + 16 * hf, d16);
        }
        wait_st();
        bDS[cg * D + mrow] = rsum;                         // partial sums, added below
    }
    fence_smem_to_async();
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    if (wp == 0 && !__any_sync(0xffffffffu, *(volatile int*)&s_abort != 0)) {
        issue(320, 0, bop);                                // dQt^T = S0 dO^T
        issue(352, 128, bop + C * D);                      // dKb^T = dS U^T
        issue(384, 0, bop + 2 * C * D);                    // (dU S0^T)^T = S0 dU^T
        mma_commit_w(mbar);
        ++n_commit;
    }
    wait_mma(1);
    {   // this thread: d_k row mrow, tokens [8 cg, 8 cg + 8)
        float v8[8];
        tmem_ld8(tm + lane_base + 320 + 8 * cg, v8);
        wait_ld();
#pragma unroll
        for (int u = 0; u < 8; ++u) bDQT[(8 * cg + u) * LD + mrow] = v8[u];
        tmem_ld8(tm + lane_base + 352 + 8 * cg, v8);
        wait_ld();
#pragma unroll
        for (int u = 0; u < 8; ++u) bDKB[(8 * cg + u) * LD + mrow] = v8[u];
        tmem_ld8(tm + lane_base + 384 + 8 * cg, v8);
        wait_ld();
#pragma unroll
        for (int u = 0; u < 8; ++u) bDW[(8 * cg + u) * LD + mrow] = -v8[u];
    }
    if (tid < D) sRS[tid] = bDS[tid] + bDS[D + tid] + bDS[2 * D + tid] + bDS[3 * D + tid];
    fence_before_sync();
    __syncthreads();

    // ---- products of the complete U and dU: dO U^T, dU V^T, dV = Tm^T dU
    tgemm_ks<C, C, D, 4, 4, 8, NL>([&](int m, int kk) { return bDO[m * LD + kk]; },
                         [&](int kk, int n) { return bU[n * LD + kk]; },
                         [&](int m, int n, float x) { sdP[m * L32 + n] = n <= m ? x : 0.f; });
    tgemm_ks<C, C, D, 4, 4, 8, NL>([&](int m, int kk) { return bDU[m * LD + kk]; },
                         [&](int kk, int n) { return bV[n * LD + kk]; },
                         [&](int m, int n, float x) { sdUV[m * L32 + n] = x; });
    tgemm<C, D, C, 2, 4, NL>([&](int m, int kk) { return Tm(kk, m); },
                         [&](int kk, int n) { return bDU[kk * LD + n]; },
                         [&](int m, int n, float x) {
                             if (m < Tl) dv[row0 + (int64_t)m * rs + n] = to_bf(x);
                         });
    __syncthreads();

    // ---- Q back in place of Kb; dGam from the direct terms; dq, dk partials
    load_rows<NL>(bQ, q, row0, rs, Tl);
    if constexpr (RAW) {
        __syncthreads();
        prologue_rows<NL>(bQ, sIQ, nullptr, nullptr, nullptr, Tl);
    }
    if (tid < D) {                                   // sum_r dKb_rc Kb_rc, before dKb is rescaled
        const int c = tid;
        const float gl = bG[(C - 1) * LD + c];
        float acc = 0.f;
        for (int r = 0; r < C; ++r)
            acc = fmaf(bDKB[r * LD + c], bK[r * LD + c] * __expf(gl - bG[r * LD + c]), acc);
        sKS[c] = acc;
    }
    __syncthreads();
    for (int e = tid; e < C * D; e += NL) {
        const int r = e / D, c = e % D;
        const float Gr = bG[r * LD + c];
        const float gam = __expf(Gr), kbf = __expf(bG[(C - 1) * LD + c] - Gr);
        const float kk = bK[r * LD + c], qq = bQ[r * LD + c];
        const float dqt = bDQT[r * LD + c], dkb = bDKB[r * LD + c];
        bV[r * LD + c] = dqt * qq * gam - dkb * kk * kbf;        // dGam (direct terms)
        bDQT[r * LD + c] = dqt * gam;
        bDKB[r * LD + c] = dkb * kbf;
        bW[r * LD + c] = kk * gam;                               // Kt
    }
    __syncthreads();
    // dTm = dW Kt^T + dU V^T;  dKt = Tm^T dW -> bDO
    tgemm_ks<C, C, D, 4, 4, 8, NL>([&](int m, int kk) { return bDW[m * LD + kk]; },
                         [&](int kk, int n) { return bW[n * LD + kk]; },
                         [&](int m, int n, float x) { sdT[m * L32 + n] = x + sdUV[m * L32 + n]; });
    tgemm<C, D, C, 2, 4, NL>([&](int m, int kk) { return Tm(kk, m); },
                         [&](int kk, int n) { return bDW[kk * LD + n]; },
                         [&](int m, int n, float x) { bDO[m * LD + n] = x; });
    __syncthreads();
    for (int e = tid; e < C * D; e += NL) {
        const int r = e / D, c = e % D;
        const float dkt = bDO[r * LD + c];
        bDKB[r * LD + c] += dkt * __expf(bG[r * LD + c]);
        bV[r * LD + c] += dkt * bW[r * LD + c];
    }
    // dbeta (columns: sum_r dTm_ri X_ri), then dX = dTm diag(beta)
    if (tid < C) {
        float acc = 0.f;
        for (int r = 0; r < C; ++r) acc = fmaf(sdT[r * L32 + tid], sX[r * L32 + tid], acc);
        sDB[tid] = acc;
    }
    __syncthreads();
    for (int e = tid; e < C * C; e += NL) {
        const int r = e / C, i = e % C;
        sdT[r * L32 + i] *= sB[i];
    }
    __syncthreads();
    // Y = dX X^T (in sdUV);  dA = -(X^T Y), strictly lower
    tgemm<C, C, C, 2, 1, NL>([&](int m, int kk) { return sdT[m * L32 + kk]; },
                         [&](int kk, int n) { return sX[n * L32 + kk]; },
                         [&](int m, int n, float x) { sdUV[m * L32 + n] = x; });
    __syncthreads();
    tgemm<C, C, C, 2, 1, NL>([&](int m, int kk) { return sX[kk * L32 + m]; },
                         [&](int kk, int n) { return sdUV[kk * L32 + n]; },
                         [&](int m, int n, float x) { sdT[m * L32 + n] = n < m ? -x : 0.f; });
    __syncthreads();
    // dbeta (rows: sum_i dA_ri Araw_ri), then dAr = diag(beta) dA
    if (tid < C) {
        float acc = sDB[tid];
        for (int i = 0; i < C; ++i) acc = fmaf(sdT[tid * L32 + i], sA[tid * L32 + i], acc);
        sDB[tid] = acc;
    }
    __syncthreads();
    for (int e = tid; e < C * C; e += NL) {
        const int r = e / C, i = e % C;
        sdT[r * L32 + i] *= sB[r];
    }
    // tile-relative operands: Ka -> bW, Qa -> bDW, Kf -> bDO, Kc -> bS0 (tile 0 rows)
    for (int e = tid; e < C * D; e += NL) {
        const int r = e / D, c = e % D;
        const float Gr = bG[r * LD + c], ref = tile_ref(bG, r, c);
        const float kk = bK[r * LD + c], a = __expf(Gr - ref);
        bW[r * LD + c] = kk * a;
        bDW[r * LD + c] = bQ[r * LD + c] * a;
        bDO[r * LD + c] = kk * __expf(ref - Gr);
        if (r < TILE) bS0[r * LD + c] = kk * __expf(bG[(TILE - 1) * LD + c] - Gr);
    }
    __syncthreads();
    // pair-product gradients: thread rows r0 .. r0 + RW - 1 (one tile), channels lane + 32 j
    {
        constexpr int RW = C / (NL / 32);        // rows per warp
        const int r0 = RW * (tid >> 5), lane = tid & 31;
        const int tau = r0 / TILE;
        const int i0 = tau * TILE;
        float rk[RW][4], rq[RW][4], ck_s[RW][4], ck_x[RW][4];
#pragma unroll
        for (int u = 0; u < RW; ++u)
#pragma unroll
            for (int j = 0; j < 4; ++j) rk[u][j] = rq[u][j] = ck_s[u][j] = ck_x[u][j] = 0.f;
        // same tile: row role over columns i, column role over rows rr, both in [i0, i0 + 16)
#pragma unroll 4
        for (int ii = 0; ii < TILE; ++ii) {
            const int i = i0 + ii;
            float kf[4], ka[4], qa[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int c = lane + 32 * j;
                kf[j] = bDO[i * LD + c];
                ka[j] = bW[i * LD + c];
                qa[j] = bDW[i * LD + c];
            }
#pragma unroll
            for (int u = 0; u < RW; ++u) {
                const float dar = sdT[(r0 + u) * L32 + i], dpr = sdP[(r0 + u) * L32 + i];   // (row r, col i)
                const float dac = sdT[i * L32 + r0 + u], dpc = sdP[i * L32 + r0 + u];       // (row i, col r)
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    rk[u][j] = fmaf(dar, kf[j], rk[u][j]);
                    rq[u][j] = fmaf(dpr, kf[j], rq[u][j]);
                    ck_s[u][j] = fmaf(dac, ka[j], fmaf(dpc, qa[j], ck_s[u][j]));
                }
            }
        }
        if (tau == 1) {       // rows of tile 1 against columns of tile 0 (row role)
#pragma unroll 4
            for (int i = 0; i < TILE; ++i) {
                float kc[4];
#pragma unroll
                for (int j = 0; j < 4; ++j) kc[j] = bS0[i * LD + lane + 32 * j];
#pragma unroll
                for (int u = 0; u < RW; ++u) {
                    const float dar = sdT[(r0 + u) * L32 + i], dpr = sdP[(r0 + u) * L32 + i];
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        rk[u][j] = fmaf(dar, kc[j], rk[u][j]);
                        rq[u][j] = fmaf(dpr, kc[j], rq[u][j]);
                    }
                }
            }
        } else {              // columns of tile 0 against rows of tile 1 (column role)
#pragma unroll 4
            for (int rr = TILE; rr < C; ++rr) {
                float ka[4], qa[4];
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    ka[j] = bW[rr * LD + lane + 32 * j];
                    qa[j] = bDW[rr * LD + lane + 32 * j];
                }
#pragma unroll
                for (int u = 0; u < RW; ++u) {
                    const float dac = sdT[rr * L32 + r0 + u], dpc = sdP[rr * L32 + r0 + u];
#pragma unroll
                    for (int j = 0; j < 4; ++j) ck_x[u][j] = fmaf(dac, ka[j], fmaf(dpc, qa[j], ck_x[u][j]));
                }
            }
        }
#pragma unroll
        for (int u = 0; u < RW; ++u) {
            const int r = r0 + u;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int c = lane + 32 * j;
                const float Gr = bG[r * LD + c], ref = tile_ref(bG, r, c);
                const float a = __expf(Gr - ref), bfac = __expf(ref - Gr);
                float colk = ck_s[u][j] * bfac;
                if (tau == 0) colk = fmaf(ck_x[u][j], __expf(bG[(TILE - 1) * LD + c] - Gr), colk);
                const float rowk = rk[u][j] * a, rowq = rq[u][j] * a;
                const float kk = bK[r * LD + c], qq = bQ[r * LD + c];
                bDKB[r * LD + c] += rowk + colk;
                bDQT[r * LD + c] += rowq;
                bV[r * LD + c] += kk * (rowk - colk) + qq * rowq;
            }
        }
    }
    __syncthreads();
    // the chunk's last token carries the terms of Gam_C; dg = reverse running sum
    if (tid < D) {
        const int c = tid;
        const float gl = bG[(C - 1) * LD + c];
        bV[(C - 1) * LD + c] += sKS[c] + sRS[c] * __expf(gl);
        float s = 0.f;
        for (int r = C - 1; r >= 0; --r) {
            s += bV[r * LD + c];
            bV[r * LD + c] = s;
        }
    }
    __syncthreads();
    if constexpr (RAW) {
        // the prologue's chain rule: for x = r / |r|, dr = (dx - x (x . dx)) / |r|
        // (zero where r = 0); for g = -5 sigmoid(z), dz = dg g (1 + g / 5),
        // with g the difference of the running sums
        const int warp = tid >> 5, lane = tid & 31;
        for (int r = warp; r < C; r += NL / 32) {
            float dotq = 0.f, dotk = 0.f;
#pragma unroll
            for (int j = 0; j < D / 32; ++j) {
                const int c = lane + 32 * j;
                dotq = fmaf(bQ[r * LD + c], bDQT[r * LD + c], dotq);
                dotk = fmaf(bK[r * LD + c], bDKB[r * LD + c], dotk);
            }
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) {
                dotq += __shfl_xor_sync(0xffffffffu, dotq, off);
                dotk += __shfl_xor_sync(0xffffffffu, dotk, off);
            }
#pragma unroll
            for (int j = 0; j < D / 32; ++j) {
                const int c = lane + 32 * j;
                bDQT[r * LD + c] = (bDQT[r * LD + c] - bQ[r * LD + c] * dotq) * sIQ[r];
                bDKB[r * LD + c] = (bDKB[r * LD + c] - bK[r * LD + c] * dotk) * sIK[r];
                const float gr = bG[r * LD + c] - (r > 0 ? bG[(r - 1) * LD + c] : 0.f);
                bV[r * LD + c] *= gr * (1.f + 0.2f * gr);
            }
        }
        __syncthreads();
    }
    for (int e = tid; e < C * D; e += NL) {
        const int r = e / D, c = e % D;
        if (r < Tl) {
            const int64_t o = row0 + (int64_t)r * rs + c;
            dq[o] = to_bf(bDQT[r * LD + c]);
            dk[o] = to_bf(bDKB[r * LD + c]);
            dg[o] = to_bf(bV[r * LD + c]);
        }
    }
    if (tid < Tl) dbeta[((int64_t)b * T + t0 + tid) * H + h] = to_bf(sDB[tid]);

    // After an expired wait the MMAs of the last commit may still run: let
    // them finish before tensor memory is released, and mark the chunk's
    // gradients as invalid (NaN) so a partial result never passes for one.
    const bool aborted = *(volatile int*)&s_abort != 0;
    if (tid == 0 && aborted && n_commit > 0) mbar_wait(mbar, (n_commit - 1) & 1u, DRAIN_NS);
    fence_before_sync();
    __syncthreads();
    if (tid < 32) tmem_dealloc(tm, 512);
    if (aborted) {
        const __nv_bfloat16 nan = __float2bfloat16_rn(__int_as_float(0x7fc00000));
        for (int e = tid; e < C * D; e += NL) {
            const int r = e / D, c = e % D;
            if (r < Tl) {
                const int64_t o = row0 + (int64_t)r * rs + c;
                dq[o] = nan;
                dk[o] = nan;
                dg[o] = nan;
                dv[o] = nan;
            }
        }
        if (tid < Tl) dbeta[((int64_t)b * T + t0 + tid) * H + h] = nan;
    }
}

}  // namespace bw

static DeviceFlags g_bwd_attr_done;

cudaError_t chunk_bwd_launch(const void* q, const void* k, const void* v, const void* g, const void* beta,
                             const float* h0, const void* dO, const float* dhT, void* dq, void* dk, void* dv,
                             void* dg, void* dbeta, float* dh0, int B, int T, int H, bool raw, cudaStream_t stream)
{
    using namespace bw;
    cudaError_t e = once_per_device(g_bwd_attr_done, [](int) {
        const cudaFuncAttribute a = cudaFuncAttributeMaxDynamicSharedMemorySize;
        cudaError_t r = cudaFuncSetAttribute(bwd_prep_kernel<false>, a, (int)PREP_SMEM);
        if (r == cudaSuccess) r = cudaFuncSetAttribute(bwd_prep_kernel<true>, a, (int)PREP_SMEM);
        if (r == cudaSuccess) r = cudaFuncSetAttribute(bwd_chains_kernel, a, (int)CHAIN_SMEM);
        if (r == cudaSuccess) r = cudaFuncSetAttribute(bwd_local_kernel<false>, a, (int)LOC_SMEM);
        if (r == cudaSuccess) r = cudaFuncSetAttribute(bwd_local_kernel<true>, a, (int)LOC_SMEM);
        return r;
    });
    if (e != cudaSuccess) return e;
    const size_t state_bytes = (size_t)D * D * sizeof(float);
    if (T == 0) {        // no token: the start-state gradient is the end-state gradient
        if (!dh0) return cudaSuccess;
        return dhT ? cudaMemcpyAsync(dh0, dhT, (size_t)B * H * state_bytes, cudaMemcpyDeviceToDevice, stream)
                   : cudaMemsetAsync(dh0, 0, (size_t)B * H * state_bytes, stream);
    }
    const int n_chunks = (T + C - 1) / C;
    const size_t units = (size_t)B * H * n_chunks;
    const size_t bytes = units * ((size_t)R_FLOATS * sizeof(float) + 2 * state_bytes);
    float* ws = nullptr;
    keep_pool_memory();
    e = cudaMallocAsync(reinterpret_cast<void**>(&ws), bytes, stream);
    if (e != cudaSuccess) return e;
    float* rec = ws;
    float* S0_all = rec + units * R_FLOATS;
    float* dS_all = S0_all + units * D * D;
    const dim3 grid_c((unsigned)n_chunks, (unsigned)H, (unsigned)B);
    const dim3 grid_s((unsigned)(D / NS), (unsigned)H, (unsigned)B);
    const __nv_bfloat16* bq = (const __nv_bfloat16*)q;
    const __nv_bfloat16* bk = (const __nv_bfloat16*)k;
    const __nv_bfloat16* bv = (const __nv_bfloat16*)v;
    const __nv_bfloat16* bg = (const __nv_bfloat16*)g;
    const __nv_bfloat16* bb = (const __nv_bfloat16*)beta;
    const __nv_bfloat16* bdo = (const __nv_bfloat16*)dO;
    (raw ? bwd_prep_kernel<true> : bwd_prep_kernel<false>)<<<grid_c, NT, PREP_SMEM, stream>>>(
        bq, bk, bv, bg, bb, rec, T, H, n_chunks);
    e = cudaGetLastError();
    if (e == cudaSuccess) {
        bwd_chains_kernel<<<grid_s, NT_CHAIN, CHAIN_SMEM, stream>>>(rec, bdo, h0, dhT, S0_all, dS_all, dh0, T, H,
                                                                      n_chunks);
        e = cudaGetLastError();
    }
    if (e == cudaSuccess) {
        (raw ? bwd_local_kernel<true> : bwd_local_kernel<false>)<<<grid_c, NL, LOC_SMEM, stream>>>(
            bq, bk, bv, bg, bb, bdo, rec, S0_all, dS_all, (__nv_bfloat16*)dq, (__nv_bfloat16*)dk,
            (__nv_bfloat16*)dv, (__nv_bfloat16*)dg, (__nv_bfloat16*)dbeta, T, H, n_chunks,
            bounded_wait_limit_ns());
        e = cudaGetLastError();
    }
    const cudaError_t ef = cudaFreeAsync(ws, stream);
    if (e == cudaSuccess) e = ef;
    note_launches(3);
    return e;
}

// Reads and clears the timeout flag of the backward kernels (blocking).
int bwd_device_status(cudaStream_t stream)
{
    int st = 0, zero = 0;
    if (cudaMemcpyFromSymbolAsync(&st, bw::g_bwd_status, sizeof(int), 0,
                                  cudaMemcpyDeviceToHost, stream) != cudaSuccess)
        return KDA_ERR_CUDA;
    if (cudaMemcpyToSymbolAsync(bw::g_bwd_status, &zero, sizeof(int), 0,
                                cudaMemcpyHostToDevice, stream) != cudaSuccess)
        return KDA_ERR_CUDA;
    if (cudaStreamSynchronize(stream) != cudaSuccess) return KDA_ERR_CUDA;
    return st;
}

}  // namespace kda
