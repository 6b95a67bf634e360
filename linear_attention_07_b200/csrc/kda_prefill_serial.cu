// Token-serial KDA prefill on CUDA cores, fp32 arithmetic.
//
// This is the fp32 entry point's kernel (kda_chunk_fwd_f32): it evaluates
// the recurrence one token at a time in fp32, exactly in the order of its
// definition, so fp32 callers get fp32-level agreement with the fp64 result:
//   S <- Diag(exp g_t) S;  p = S^T k_t;  u = beta_t (v_t - p);
//   S <- S + k_t u^T;      o_t = S^T q_t = (decayed S)^T q_t + (q_t.k_t) u.
// ("T11E1: K3 tech report" transcript, KDA turn: learned write strength and
// channel-wise forgetting; "Kimi K3 goes trillion-scale ..." subtitles,
// cue 14: delta-rule recurrence with a channel-wise forget gate.)
//
// Grid (dv / 32, H, B): one CTA per (batch, head, 32-column slice of the
// state).  Columns of S evolve independently given the keys, so slices need
// no communication.  4 warps: lane = state column, warp w = rows
// [w*DK/4, (w+1)*DK/4), each thread keeps its DK/4 state entries in
// registers.  The two d_k reductions of a token (p and the read r) share
// one double-buffered shared-memory exchange, so each token costs one
// __syncthreads.  Inputs are staged per 16-token tile.
#include "kda_common.cuh"

namespace kda {

constexpr int kSerialThreads = 128;
constexpr int kSerialTile = 16;

template <int DK, typename Tin, typename Tout>
__global__ void __launch_bounds__(kSerialThreads)
prefill_serial_kernel(const Tin* __restrict__ q, const Tin* __restrict__ k,
                      const Tin* __restrict__ v, const Tin* __restrict__ g,
                      const Tin* __restrict__ beta, const float* h0,
                      Tout* __restrict__ o, float* hT, int T, int H, int DV)
{
    constexpr int RPW = DK / 4;   // state rows per warp
    __shared__ __align__(16) float s_a[kSerialTile][DK];
    __shared__ __align__(16) float s_k[kSerialTile][DK];
    __shared__ __align__(16) float s_q[kSerialTile][DK];
    __shared__ float s_v[kSerialTile][32];
    __shared__ float s_b[kSerialTile];
    __shared__ float s_qk[kSerialTile];
    __shared__ float2 s_red[2][4][32];

    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    const int h = blockIdx.y, b = blockIdx.z;
    const int j = blockIdx.x * 32 + lane;
    const int64_t state_off = ((int64_t)b * H + h) * DK * (int64_t)DV;

    float s[RPW];
#pragma unroll
    for (int m = 0; m < RPW; ++m)
        s[m] = h0 ? h0[state_off + (int64_t)(w * RPW + m) * DV + j] : 0.f;

    int buf = 0;
    for (int c0 = 0; c0 < T; c0 += kSerialTile) {
        const int n = min(kSerialTile, T - c0);
        __syncthreads();   // previous tile fully consumed
        for (int idx = threadIdx.x; idx < n * DK; idx += kSerialThreads) {
            const int t = idx / DK, i = idx % DK;
            const int64_t off = (((int64_t)b * T + c0 + t) * H + h) * DK + i;
            s_a[t][i] = expf(to_f32(g[off]));
            s_k[t][i] = to_f32(k[off]);
            s_q[t][i] = to_f32(q[off]);
        }
        for (int idx = threadIdx.x; idx < n * 32; idx += kSerialThreads) {
            const int t = idx / 32, jj = idx % 32;
            s_v[t][jj] = to_f32(v[(((int64_t)b * T + c0 + t) * H + h) * DV + blockIdx.x * 32 + jj]);
        }
        if (threadIdx.x < n)
            s_b[threadIdx.x] = to_f32(beta[((int64_t)b * T + c0 + threadIdx.x) * H + h]);
        __syncthreads();
        for (int t = w; t < n; t += 4) {          // q.k per token, one warp each
            float acc = 0.f;
            for (int i = lane; i < DK; i += 32) acc = fmaf(s_q[t][i], s_k[t][i], acc);
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
            if (lane == 0) s_qk[t] = acc;
        }
        __syncthreads();

        for (int t = 0; t < n; ++t) {
            const float* a = &s_a[t][w * RPW];
            const float* kk = &s_k[t][w * RPW];
            const float* qq = &s_q[t][w * RPW];
            float p = 0.f, r = 0.f;
#pragma unroll
            for (int m = 0; m < RPW; ++m) {
                s[m] *= a[m];
                p = fmaf(s[m], kk[m], p);
                r = fmaf(s[m], qq[m], r);
            }
            s_red[buf][w][lane] = make_float2(p, r);
            __syncthreads();
            float P = 0.f, R = 0.f;
#pragma unroll
            for (int w2 = 0; w2 < 4; ++w2) {
                const float2 x = s_red[buf][w2][lane];
                P += x.x;
                R += x.y;
            }
            buf ^= 1;
            const float u = s_b[t] * (s_v[t][lane] - P);
            if (w == 0)
                o[(((int64_t)b * T + c0 + t) * H + h) * DV + j] = from_f32<Tout>(fmaf(s_qk[t], u, R));
#pragma unroll
            for (int m = 0; m < RPW; ++m) s[m] = fmaf(kk[m], u, s[m]);
        }
    }
    if (hT) {
        __syncthreads();   // every CTA reads its own h0 slice only, before this
#pragma unroll
        for (int m = 0; m < RPW; ++m) hT[state_off + (int64_t)(w * RPW + m) * DV + j] = s[m];
    }
}

template <typename Tin, typename Tout>
cudaError_t prefill_serial_launch(const void* q, const void* k, const void* v,
                                  const void* g, const void* beta, const float* h0,
                                  void* o, float* hT, int B, int T, int H,
                                  int dk, int dv, cudaStream_t stream)
{
    dim3 grid(dv / 32, H, B);
#define KDA_SER(DK_)                                                                  \
    if (dk == DK_) {                                                                  \
        prefill_serial_kernel<DK_, Tin, Tout><<<grid, kSerialThreads, 0, stream>>>(   \
            (const Tin*)q, (const Tin*)k, (const Tin*)v, (const Tin*)g,               \
            (const Tin*)beta, h0, (Tout*)o, hT, T, H, dv);                            \
        note_launches(1);                                                             \
        return cudaGetLastError();                                                    \
    }
    KDA_SER(32) KDA_SER(64) KDA_SER(128)
#undef KDA_SER
    return cudaErrorInvalidValue;
}

template cudaError_t prefill_serial_launch<float, float>(
    const void*, const void*, const void*, const void*, const void*, const float*,
    void*, float*, int, int, int, int, int, cudaStream_t);
template cudaError_t prefill_serial_launch<__nv_bfloat16, __nv_bfloat16>(
    const void*, const void*, const void*, const void*, const void*, const float*,
    void*, float*, int, int, int, int, int, cudaStream_t);

}  // namespace kda
