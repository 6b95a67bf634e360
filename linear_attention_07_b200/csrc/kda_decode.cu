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
// One CTA of 256 threads per (request, head).  Thread (rg, cg) owns columns
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
    constexpr int CG = DV / 4;                  // float4 column groups per row
    constexpr int RSTEP = kDecodeThreads / CG;  // rows covered per block pass
    constexpr int ROWS = DK / RSTEP;            // rows per thread
    static_assert(ROWS >= 1 && DK % RSTEP == 0, "unsupported decode shape");

    __shared__ float s_a[DK], s_k[DK], s_q[DK];
    __shared__ float s_qk;
    __shared__ float s_inv[2];                  // RAW: 1 / |q|, 1 / |k|
    __shared__ float4 s_red[2][RSTEP][CG];

    const int64_t nh = blockIdx.x;              // request * H + head
    const int tid = threadIdx.x;
    const int cg = tid % CG;
    const int rg = tid / CG;

    float4* S = reinterpret_cast<float4*>(state + nh * (int64_t)(DK * DV));
    float4 s[ROWS];
#pragma unroll
    for (int m = 0; m < ROWS; ++m) s[m] = __ldcs(S + (rg + m * RSTEP) * CG + cg);

    // small per-head vectors
    for (int i = tid; i < DK; i += kDecodeThreads) {
        const float gi = to_f32(g[nh * DK + i]);
        s_a[i] = expf(RAW ? -5.f / (1.f + expf(-gi)) : gi);
        s_k[i] = to_f32(k[nh * DK + i]);
        s_q[i] = to_f32(q[nh * DK + i]);
    }
    if constexpr (RAW) {
        __syncthreads();
        if (tid < 32) {
            float nq = 0.f, nk = 0.f;
            for (int i = tid; i < DK; i += 32) {
                nq = fmaf(s_q[i], s_q[i], nq);
                nk = fmaf(s_k[i], s_k[i], nk);
            }
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) {
                nq += __shfl_xor_sync(0xffffffffu, nq, off);
                nk += __shfl_xor_sync(0xffffffffu, nk, off);
            }
            if (tid == 0) {
                s_inv[0] = nq > 0.f ? rsqrtf(nq) : 0.f;
                s_inv[1] = nk > 0.f ? rsqrtf(nk) : 0.f;
            }
        }
        __syncthreads();
        for (int i = tid; i < DK; i += kDecodeThreads) {
            s_q[i] *= s_inv[0];
            s_k[i] *= s_inv[1];
        }
    }
    const float b = to_f32(beta[nh]);
    const __nv_bfloat162* v2 = reinterpret_cast<const __nv_bfloat162*>(v + nh * DV + 4 * cg);
    const float2 v01 = __bfloat1622float2(v2[0]);
    const float2 v23 = __bfloat1622float2(v2[1]);
    __syncthreads();
    if (tid < 32) {
        float acc = 0.f;
        for (int i = tid; i < DK; i += 32) acc = fmaf(s_q[i], s_k[i], acc);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
        if (tid == 0) s_qk = acc;
    }

    // decay rows, then partial recall p = (DS)^T k and read r = (DS)^T q
    float4 p = make_float4(0.f, 0.f, 0.f, 0.f), r = p;
#pragma unroll
    for (int m = 0; m < ROWS; ++m) {
        const int i = rg + m * RSTEP;
        const float a = s_a[i], ki = s_k[i], qi = s_q[i];
        s[m].x *= a; s[m].y *= a; s[m].z *= a; s[m].w *= a;
        p.x = fmaf(s[m].x, ki, p.x); p.y = fmaf(s[m].y, ki, p.y);
        p.z = fmaf(s[m].z, ki, p.z); p.w = fmaf(s[m].w, ki, p.w);
        r.x = fmaf(s[m].x, qi, r.x); r.y = fmaf(s[m].y, qi, r.y);
        r.z = fmaf(s[m].z, qi, r.z); r.w = fmaf(s[m].w, qi, r.w);
    }
    s_red[0][rg][cg] = p;
    s_red[1][rg][cg] = r;
    __syncthreads();
    float4 P = make_float4(0.f, 0.f, 0.f, 0.f), R = P;
#pragma unroll
    for (int w = 0; w < RSTEP; ++w) {
        const float4 a = s_red[0][w][cg], c = s_red[1][w][cg];
        P.x += a.x; P.y += a.y; P.z += a.z; P.w += a.w;
        R.x += c.x; R.y += c.y; R.z += c.z; R.w += c.w;
    }
    float4 u;
    u.x = b * (v01.x - P.x); u.y = b * (v01.y - P.y);
    u.z = b * (v23.x - P.z); u.w = b * (v23.y - P.w);
    if (rg == 0) {
        const float qk = s_qk;
        __nv_bfloat162 o01 = __floats2bfloat162_rn(fmaf(qk, u.x, R.x), fmaf(qk, u.y, R.y));
        __nv_bfloat162 o23 = __floats2bfloat162_rn(fmaf(qk, u.z, R.z), fmaf(qk, u.w, R.w));
        __nv_bfloat162* o2 = reinterpret_cast<__nv_bfloat162*>(o + nh * DV + 4 * cg);
        o2[0] = o01;
        o2[1] = o23;
    }
    // write: S_new = D S + k u^T
#pragma unroll
    for (int m = 0; m < ROWS; ++m) {
        const float ki = s_k[rg + m * RSTEP];
        s[m].x = fmaf(ki, u.x, s[m].x); s[m].y = fmaf(ki, u.y, s[m].y);
        s[m].z = fmaf(ki, u.z, s[m].z); s[m].w = fmaf(ki, u.w, s[m].w);
        __stcs(S + (rg + m * RSTEP) * CG + cg, s[m]);
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

}  // namespace kda
