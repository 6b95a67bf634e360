// Batched KDA decode step: one token for each (request, head), fp32 state
// updated in place.  HBM-bound: the whole d_k x d_v state is read once and
// written once per step ("177: Kimi K3 in Detail", Deep dive 17: decoding
// reads the whole fixed-size state for every new token; Deep dive 10: the
// state is rewritten in place for every token).
//
// Per (request, head), with a = exp(g) and D = Diag(a):
//   p = (D S)^T k,  r = (D S)^T q,  u = beta (v - p),
//   o = r + (q.k) u            (= S_new^T q),
//   S_new = D S + k u^T.
//
// One CTA of 256 threads per (request, head); the token's arithmetic is
// decode_token, shared with the multi-token verify kernel below.  Thread (rg, cg) owns columns
// 4cg..4cg+3 of rows rg, rg + RSTEP, ...: a warp reads whole 512-byte rows
// with float4 loads, so every state access is a fully coalesced 16-byte
// vector access.  All ROWS loads are issued before any arithmetic so that
// each thread has ROWS x 16 bytes in flight.  The two column reductions over
// d_k (p and r) go through one shared-memory pass.
//
// RAW (the fused prologue): q and k arrive unnormalised and g holds the gate
// pre-activation z; the step L2-normalises q and k (a zero vector stays
// zero) and takes g = -5 sigmoid(z) before the recurrence.
#include "kda_common.cuh"

namespace kda {

constexpr int kDecodeThreads = 256;

// Thread mapping of a decode CTA over one d_k x d_v state.
template <int DK, int DV>
struct DecodeMap {
    static constexpr int CG = DV / 4;                  // float4 column groups per row
    static constexpr int RSTEP = kDecodeThreads / CG;  // rows covered per block pass
    static constexpr int ROWS = DK / RSTEP;            // rows per thread
    static_assert(ROWS >= 1 && DK % RSTEP == 0, "unsupported decode shape");
};

template <int DK, int DV>
struct DecodeShared {
    float a[DK], k[DK], q[DK];
    float qk;
    float inv[2];                                     // RAW: 1 / |q|, 1 / |k|
    float4 red[2][DecodeMap<DK, DV>::RSTEP][DecodeMap<DK, DV>::CG];
};

// One token of one (request, head) on the state slice s[] held in registers
// (thread (rg, cg): rows rg + m RSTEP, columns 4 cg .. 4 cg + 3).  The
// pointers address this token's vectors: q, k, g [DK], v [DV], beta [1],
// o [DV].  The arithmetic and its order are fixed here, so the single-step
// kernel and the multi-token verify kernel give the same bits for the same
// token.  Starts by writing shared memory: a caller that runs several
// tokens synchronises the CTA between them.
template <int DK, int DV, bool RAW>
__device__ __forceinline__ void decode_token(float4 (&s)[DecodeMap<DK, DV>::ROWS],
                                             const __nv_bfloat16* __restrict__ q,
                                             const __nv_bfloat16* __restrict__ k,
                                             const __nv_bfloat16* __restrict__ v,
                                             const __nv_bfloat16* __restrict__ g,
                                             const __nv_bfloat16* __restrict__ beta,
                                             __nv_bfloat16* __restrict__ o,
                                             DecodeShared<DK, DV>& sh)
{
    using M = DecodeMap<DK, DV>;
    constexpr int CG = M::CG, RSTEP = M::RSTEP, ROWS = M::ROWS;
    const int tid = threadIdx.x;
    const int cg = tid % CG;
    const int rg = tid / CG;

    // small per-head vectors
    for (int i = tid; i < DK; i += kDecodeThreads) {
        const float gi = to_f32(g[i]);
        sh.a[i] = expf(RAW ? -5.f / (1.f + expf(-gi)) : gi);
        sh.k[i] = to_f32(k[i]);
        sh.q[i] = to_f32(q[i]);
    }
    if constexpr (RAW) {
        __syncthreads();
        if (tid < 32) {
            float nq = 0.f, nk = 0.f;
            for (int i = tid; i < DK; i += 32) {
                nq = fmaf(sh.q[i], sh.q[i], nq);
                nk = fmaf(sh.k[i], sh.k[i], nk);
            }
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) {
                nq += __shfl_xor_sync(0xffffffffu, nq, off);
                nk += __shfl_xor_sync(0xffffffffu, nk, off);
            }
            if (tid == 0) {
                sh.inv[0] = nq > 0.f ? rsqrtf(nq) : 0.f;
                sh.inv[1] = nk > 0.f ? rsqrtf(nk) : 0.f;
            }
        }
        __syncthreads();
        for (int i = tid; i < DK; i += kDecodeThreads) {
            sh.q[i] *= sh.inv[0];
            sh.k[i] *= sh.inv[1];
        }
    }
    const float b = to_f32(beta[0]);
    const __nv_bfloat162* v2 = reinterpret_cast<const __nv_bfloat162*>(v + 4 * cg);
    const float2 v01 = __bfloat1622float2(v2[0]);
    const float2 v23 = __bfloat1622float2(v2[1]);
    __syncthreads();
    if (tid < 32) {
        float acc = 0.f;
        for (int i = tid; i < DK; i += 32) acc = fmaf(sh.q[i], sh.k[i], acc);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
        if (tid == 0) sh.qk = acc;
    }

    // decay rows, then partial recall p = (DS)^T k and read r = (DS)^T q
    float4 p = make_float4(0.f, 0.f, 0.f, 0.f), r = p;
#pragma unroll
    for (int m = 0; m < ROWS; ++m) {
        const int i = rg + m * RSTEP;
        const float a = sh.a[i], ki = sh.k[i], qi = sh.q[i];
        s[m].x *= a; s[m].y *= a; s[m].z *= a; s[m].w *= a;
        p.x = fmaf(s[m].x, ki, p.x); p.y = fmaf(s[m].y, ki, p.y);
        p.z = fmaf(s[m].z, ki, p.z); p.w = fmaf(s[m].w, ki, p.w);
        r.x = fmaf(s[m].x, qi, r.x); r.y = fmaf(s[m].y, qi, r.y);
        r.z = fmaf(s[m].z, qi, r.z); r.w = fmaf(s[m].w, qi, r.w);
    }
    sh.red[0][rg][cg] = p;
    sh.red[1][rg][cg] = r;
    __syncthreads();
    float4 P = make_float4(0.f, 0.f, 0.f, 0.f), R = P;
#pragma unroll
    for (int w = 0; w < RSTEP; ++w) {
        const float4 a = sh.red[0][w][cg], c = sh.red[1][w][cg];
        P.x += a.x; P.y += a.y; P.z += a.z; P.w += a.w;
        R.x += c.x; R.y += c.y; R.z += c.z; R.w += c.w;
    }
    float4 u;
    u.x = b * (v01.x - P.x); u.y = b * (v01.y - P.y);
    u.z = b * (v23.x - P.z); u.w = b * (v23.y - P.w);
    if (rg == 0) {
        const float qk = sh.qk;
        __nv_bfloat162 o01 = __floats2bfloat162_rn(fmaf(qk, u.x, R.x), fmaf(qk, u.y, R.y));
        __nv_bfloat162 o23 = __floats2bfloat162_rn(fmaf(qk, u.z, R.z), fmaf(qk, u.w, R.w));
        __nv_bfloat162* o2 = reinterpret_cast<__nv_bfloat162*>(o + 4 * cg);
        o2[0] = o01;
        o2[1] = o23;
    }
    // write: S_new = D S + k u^T
#pragma unroll
    for (int m = 0; m < ROWS; ++m) {
        const float ki = sh.k[rg + m * RSTEP];
        s[m].x = fmaf(ki, u.x, s[m].x); s[m].y = fmaf(ki, u.y, s[m].y);
        s[m].z = fmaf(ki, u.z, s[m].z); s[m].w = fmaf(ki, u.w, s[m].w);
    }
}

template <int DK, int DV, bool RAW>
__global__ void __launch_bounds__(kDecodeThreads, 2)
decode_step_kernel(const __nv_bfloat16* __restrict__ q,
                   const __nv_bfloat16* __restrict__ k,
                   const __nv_bfloat16* __restrict__ v,
                   const __nv_bfloat16* __restrict__ g,
                   const __nv_bfloat16* __restrict__ beta,
                   float* __restrict__ state,
                   __nv_bfloat16* __restrict__ o)
{
    using M = DecodeMap<DK, DV>;
    __shared__ DecodeShared<DK, DV> sh;
    const int64_t nh = blockIdx.x;              // request * H + head
    const int tid = threadIdx.x;
    const int cg = tid % M::CG;
    const int rg = tid / M::CG;

    float4* S = reinterpret_cast<float4*>(state + nh * (int64_t)(DK * DV));
    float4 s[M::ROWS];
#pragma unroll
    for (int m = 0; m < M::ROWS; ++m) s[m] = __ldcs(S + (rg + m * M::RSTEP) * M::CG + cg);
    decode_token<DK, DV, RAW>(s, q + nh * DK, k + nh * DK, v + nh * DV, g + nh * DK, beta + nh,
                              o + nh * DV, sh);
#pragma unroll
    for (int m = 0; m < M::ROWS; ++m) __stcs(S + (rg + m * M::RSTEP) * M::CG + cg, s[m]);
}

// Multi-token verify (speculative decoding): K consecutive tokens of each
// (request, head) from the start state h0, which is read once and not
// modified; o is written for every token and the fp32 state after every
// token goes to states[n][t][h] (layout [N][K][H][DK][DV]: the states of
// one request after token t form one contiguous [H][DK][DV] block, the
// layout of a decode state).  Each token is decode_token, so replaying the
// first j tokens from h0 with the decode kernel gives states[n][j - 1]
// exactly ("177: Kimi K3 in Detail" episode notes, Deep dive 23: rollback
// keeps a checkpoint and replays the accepted steps).
template <int DK, int DV>
__global__ void __launch_bounds__(kDecodeThreads, 2)
verify_kernel(const __nv_bfloat16* __restrict__ q,
              const __nv_bfloat16* __restrict__ k,
              const __nv_bfloat16* __restrict__ v,
              const __nv_bfloat16* __restrict__ g,
              const __nv_bfloat16* __restrict__ beta,
              const float* __restrict__ h0,
              __nv_bfloat16* __restrict__ o,
              float* __restrict__ states, int K, int H)
{
    using M = DecodeMap<DK, DV>;
    __shared__ DecodeShared<DK, DV> sh;
    const int h = blockIdx.x, n = blockIdx.y;
    const int64_t nh = (int64_t)n * H + h;
    const int tid = threadIdx.x;
    const int cg = tid % M::CG;
    const int rg = tid / M::CG;

    float4 s[M::ROWS];
    if (h0) {
        const float4* S0 = reinterpret_cast<const float4*>(h0 + nh * (int64_t)(DK * DV));
#pragma unroll
        for (int m = 0; m < M::ROWS; ++m) s[m] = __ldg(S0 + (rg + m * M::RSTEP) * M::CG + cg);
    } else {
#pragma unroll
        for (int m = 0; m < M::ROWS; ++m) s[m] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll 1
    for (int t = 0; t < K; ++t) {
        const int64_t th = ((int64_t)n * K + t) * H + h;       // token t of request n, head h
        if (t > 0) __syncthreads();                           // previous token's shared reads done
        decode_token<DK, DV, false>(s, q + th * DK, k + th * DK, v + th * DV, g + th * DK, beta + th,
                                    o + th * DV, sh);
        float4* St = reinterpret_cast<float4*>(states + th * (int64_t)(DK * DV));
#pragma unroll
        for (int m = 0; m < M::ROWS; ++m) __stcs(St + (rg + m * M::RSTEP) * M::CG + cg, s[m]);
    }
}

template <int DK, int DV, bool RAW>
static cudaError_t launch_decode(const void* q, const void* k, const void* v,
                                 const void* g, const void* beta, float* state,
                                 void* o, int64_t NH, cudaStream_t stream)
{
    decode_step_kernel<DK, DV, RAW><<<(unsigned)NH, kDecodeThreads, 0, stream>>>(
        (const __nv_bfloat16*)q, (const __nv_bfloat16*)k, (const __nv_bfloat16*)v,
        (const __nv_bfloat16*)g, (const __nv_bfloat16*)beta, state, (__nv_bfloat16*)o);
    note_launches(1);
    return cudaGetLastError();
}

cudaError_t decode_step_launch(const void* q, const void* k, const void* v,
                               const void* g, const void* beta, float* state,
                               void* o, int64_t NH, int dk, int dv, bool raw,
                               cudaStream_t stream)
{
#define KDA_DEC(DK_, DV_) \
    if (dk == DK_ && dv == DV_) \
        return raw ? launch_decode<DK_, DV_, true>(q, k, v, g, beta, state, o, NH, stream) \
                   : launch_decode<DK_, DV_, false>(q, k, v, g, beta, state, o, NH, stream);
    KDA_DEC(32, 32) KDA_DEC(32, 64) KDA_DEC(32, 128)
    KDA_DEC(64, 32) KDA_DEC(64, 64) KDA_DEC(64, 128)
    KDA_DEC(128, 32) KDA_DEC(128, 64) KDA_DEC(128, 128)
#undef KDA_DEC
    return cudaErrorInvalidValue;
}

template <int DK, int DV>
static cudaError_t launch_verify(const void* q, const void* k, const void* v, const void* g,
                                 const void* beta, const float* h0, void* o, float* states,
                                 int N, int K, int H, cudaStream_t stream)
{
    verify_kernel<DK, DV><<<dim3((unsigned)H, (unsigned)N), kDecodeThreads, 0, stream>>>(
        (const __nv_bfloat16*)q, (const __nv_bfloat16*)k, (const __nv_bfloat16*)v,
        (const __nv_bfloat16*)g, (const __nv_bfloat16*)beta, h0, (__nv_bfloat16*)o, states, K, H);
    note_launches(1);
    return cudaGetLastError();
}

cudaError_t verify_launch(const void* q, const void* k, const void* v, const void* g,
                          const void* beta, const float* h0, void* o, float* states,
                          int N, int K, int H, int dk, int dv, cudaStream_t stream)
{
#define KDA_VER(DK_, DV_) \
    if (dk == DK_ && dv == DV_) return launch_verify<DK_, DV_>(q, k, v, g, beta, h0, o, states, N, K, H, stream);
    KDA_VER(32, 32) KDA_VER(32, 64) KDA_VER(32, 128)
    KDA_VER(64, 32) KDA_VER(64, 64) KDA_VER(64, 128)
    KDA_VER(128, 32) KDA_VER(128, 64) KDA_VER(128, 128)
#undef KDA_VER
    return cudaErrorInvalidValue;
}

}  // namespace kda
