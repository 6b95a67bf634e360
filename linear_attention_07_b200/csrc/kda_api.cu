// C ABI of libkda.so: host-side argument checks and kernel dispatch.
// Every argument error is detected here, before any launch.
#include <atomic>

#include "kda_common.cuh"

namespace kda {

static std::atomic<uint64_t> g_launches{0};
void note_launches(int n) { g_launches.fetch_add((uint64_t)n, std::memory_order_relaxed); }

static std::atomic<int> g_sm_count[MAX_DEVICES];

int current_sm_count()
{
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 0;
    const bool tracked = dev >= 0 && dev < MAX_DEVICES;
    if (tracked && (n = g_sm_count[dev].load(std::memory_order_relaxed)) > 0) return n;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) return 0;
    if (tracked) g_sm_count[dev].store(n, std::memory_order_relaxed);
    return n;
}

static DeviceFlags g_pool_done;

void keep_pool_memory()
{
    once_per_device(g_pool_done, [](int dev) {
        cudaMemPool_t pool;
        if (cudaDeviceGetDefaultMemPool(&pool, dev) == cudaSuccess) {
            uint64_t keep = UINT64_MAX;
            cudaMemPoolSetAttribute(pool, cudaMemPoolAttrReleaseThreshold, &keep);
        }
        return cudaSuccess;   // a pool that keeps nothing only costs speed
    });
}

cudaError_t decode_step_launch(const void* q, const void* k, const void* v,
                               const void* g, const void* beta, float* state,
                               void* o, int64_t NH, int dk, int dv, bool raw,
                               cudaStream_t stream);

cudaError_t verify_launch(const void* q, const void* k, const void* v, const void* g,
                          const void* beta, const float* h0, void* o, float* states,
                          int N, int K, int H, int dk, int dv, cudaStream_t stream);

cudaError_t chunk_bwd_launch(const void* q, const void* k, const void* v, const void* g, const void* beta,
                             const float* h0, const void* dO, const float* dhT, void* dq, void* dk, void* dv,
                             void* dg, void* dbeta, float* dh0, int B, int T, int H, bool raw,
                             cudaStream_t stream);

cudaError_t prefill_tc_launch(const void* q, const void* k, const void* v, const void* g,
                              const void* beta, const float* h0, void* o, float* hT,
                              int B, int T, int H, bool no_alloc, float* states, int snap_every,
                              bool prologue, cudaStream_t stream);
cudaError_t prefill_transition_launch(const void* q, const void* k, const void* g, const void* beta,
                                      float* M, int B, int T, int H, cudaStream_t stream);
cudaError_t state_chain_launch(const float* M, const float* N, const float* h0, float* S_start, float* hT,
                               int B, int P, int H, cudaStream_t stream);
int prefill_device_status(cudaStream_t stream);
int bwd_device_status(cudaStream_t stream);
int prefill_path_of(int B, int T, int H);
cudaError_t bounded_wait_selftest_launch(uint64_t limit_ns, cudaStream_t stream);

template <typename Tin, typename Tout>
cudaError_t prefill_serial_launch(const void* q, const void* k, const void* v,
                                  const void* g, const void* beta, const float* h0,
                                  void* o, float* hT, int B, int T, int H,
                                  int dk, int dv, cudaStream_t stream);

static bool dim_ok(int d) { return d == 32 || d == 64 || d == 128; }

static bool ptr_ok(const void* p) { return p != nullptr && aligned16(p); }
static bool opt_ptr_ok(const void* p) { return p == nullptr || aligned16(p); }

// Largest element count of any tensor must stay far below 2^62 bytes.
static bool sizes_ok(int64_t a, int64_t b, int64_t c, int64_t d)
{
    const int64_t lim = (int64_t)1 << 40;
    return a < lim && b < lim && c < lim && d < lim && a * b < lim && a * b * c < lim &&
           (double)a * (double)b * (double)c * (double)d < 4.0e18;
}

static int status_of(cudaError_t e)
{
    if (e == cudaSuccess) return KDA_OK;
    return e == cudaErrorMemoryAllocation ? KDA_ERR_NO_MEMORY : KDA_ERR_CUDA;
}

// Common checks of the two prefill entry points.
static int check_prefill(const void* q, const void* k, const void* v, const void* g,
                         const void* beta, const void* h0, const void* o,
                         const void* hT, int B, int T, int H, int dk, int dv)
{
    if (B < 0 || T < 0 || H < 0 || dk <= 0 || dv <= 0) return KDA_ERR_INVALID_ARG;
    if (!sizes_ok(B, T, H, dk > dv ? dk : dv)) return KDA_ERR_INVALID_ARG;
    if (H > 65535 || B > 65535) return KDA_ERR_UNSUPPORTED;
    if (!opt_ptr_ok(h0) || !opt_ptr_ok(hT)) return KDA_ERR_INVALID_ARG;
    if ((int64_t)B * T * H > 0) {
        if (!ptr_ok(q) || !ptr_ok(k) || !ptr_ok(v) || !ptr_ok(g) || !ptr_ok(o))
            return KDA_ERR_INVALID_ARG;
        // beta rows are [B][T][H] scalars: only element alignment is needed
        if (beta == nullptr) return KDA_ERR_INVALID_ARG;
    }
    return KDA_OK;
}

}  // namespace kda

using namespace kda;

extern "C" {

static int chunk_fwd_bf16(const void* q, const void* k, const void* v, const void* g,
                          const void* beta, const float* h0, void* o, float* hT,
                          int B, int T, int H, int dk, int dv, bool no_alloc,
                          float* states, int state_every, bool raw, kda_stream_t stream)
{
    int st = check_prefill(q, k, v, g, beta, h0, o, hT, B, T, H, dk, dv);
    if (st != KDA_OK) return st;
    if (!(dk == 128 && dv == 128)) return KDA_ERR_UNSUPPORTED;
    if ((reinterpret_cast<uintptr_t>(beta) & 1u) != 0) return KDA_ERR_INVALID_ARG;
    if ((int64_t)B * H == 0) return KDA_OK;
    if (T == 0 && hT == nullptr) return KDA_OK;
    return status_of(prefill_tc_launch(q, k, v, g, beta, h0, o, hT, B, T, H, no_alloc,
                                       states, state_every / 32, raw, (cudaStream_t)stream));
}

int kda_chunk_fwd(const void* q, const void* k, const void* v, const void* g,
                  const void* beta, const float* h0, void* o, float* hT,
                  int B, int T, int H, int dk, int dv, kda_stream_t stream)
{
    return chunk_fwd_bf16(q, k, v, g, beta, h0, o, hT, B, T, H, dk, dv, false, nullptr, 0, false, stream);
}

int kda_chunk_fwd_raw(const void* q_raw, const void* k_raw, const void* v, const void* z,
                      const void* beta, const float* h0, void* o, float* hT,
                      int B, int T, int H, int dk, int dv, kda_stream_t stream)
{
    return chunk_fwd_bf16(q_raw, k_raw, v, z, beta, h0, o, hT, B, T, H, dk, dv, false, nullptr, 0, true, stream);
}

int kda_chunk_fwd_states(const void* q, const void* k, const void* v, const void* g,
                         const void* beta, const float* h0, void* o, float* hT,
                         float* states, int state_every,
                         int B, int T, int H, int dk, int dv, kda_stream_t stream)
{
    if (state_every <= 0 || state_every % 32 != 0) return KDA_ERR_INVALID_ARG;
    const int64_t n_snap = T > 0 ? T / state_every : 0;
    if (n_snap > 0 && (states == nullptr || !aligned16(states))) return KDA_ERR_INVALID_ARG;
    return chunk_fwd_bf16(q, k, v, g, beta, h0, o, hT, B, T, H, dk, dv, false,
                          n_snap > 0 ? states : nullptr, state_every, false, stream);
}

int kda_chunk_transition(const void* q, const void* k, const void* g, const void* beta, float* M,
                         int B, int T, int H, int dk, kda_stream_t stream)
{
    // the checks of a prefill, with v and o absent and M in the place of hT
    int st = check_prefill(q, k, q, g, beta, nullptr, q, M, B, T, H, dk, dk);
    if (st != KDA_OK) return st;
    if (dk != 128) return KDA_ERR_UNSUPPORTED;
    if ((int64_t)B * H == 0) return KDA_OK;
    if (!ptr_ok(M)) return KDA_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(beta) & 1u) != 0) return KDA_ERR_INVALID_ARG;
    return status_of(prefill_transition_launch(q, k, g, beta, M, B, T, H, (cudaStream_t)stream));
}

int kda_state_chain(const float* M, const float* N, const float* h0, float* S_start, float* hT,
                    int B, int P, int H, int dk, int dv, kda_stream_t stream)
{
    if (B < 0 || P < 0 || H < 0) return KDA_ERR_INVALID_ARG;
    if (!(dk == 128 && dv == 128)) return KDA_ERR_UNSUPPORTED;
    if (B > 65535 || H > 65535) return KDA_ERR_UNSUPPORTED;
    if ((int64_t)B * P * H == 0) return KDA_OK;
    if (!ptr_ok(M) || !ptr_ok(N) || !ptr_ok(S_start) || !opt_ptr_ok(h0) || !opt_ptr_ok(hT))
        return KDA_ERR_INVALID_ARG;
    return status_of(state_chain_launch(M, N, h0, S_start, hT, B, P, H, (cudaStream_t)stream));
}

int kda_chunk_fwd_noalloc(const void* q, const void* k, const void* v, const void* g,
                          const void* beta, const float* h0, void* o, float* hT,
                          int B, int T, int H, int dk, int dv, kda_stream_t stream)
{
    return chunk_fwd_bf16(q, k, v, g, beta, h0, o, hT, B, T, H, dk, dv, true, nullptr, 0, false, stream);
}

int kda_chunk_fwd_f32(const float* q, const float* k, const float* v,
                      const float* g, const float* beta, const float* h0,
                      float* o, float* hT,
                      int B, int T, int H, int dk, int dv, kda_stream_t stream)
{
    int st = check_prefill(q, k, v, g, beta, h0, o, hT, B, T, H, dk, dv);
    if (st != KDA_OK) return st;
    if (!dim_ok(dk) || !dim_ok(dv)) return KDA_ERR_UNSUPPORTED;
    if ((reinterpret_cast<uintptr_t>(beta) & 3u) != 0) return KDA_ERR_INVALID_ARG;
    if ((int64_t)B * H == 0) return KDA_OK;
    if (T == 0 && hT == nullptr) return KDA_OK;
    return status_of(prefill_serial_launch<float, float>(
        q, k, v, g, beta, h0, o, hT, B, T, H, dk, dv, (cudaStream_t)stream));
}

static int decode_step_any(const void* q, const void* k, const void* v, const void* g,
                           const void* beta, float* state, void* o,
                           int N, int H, int dk, int dv, bool raw, kda_stream_t stream)
{
    if (N < 0 || H < 0 || dk <= 0 || dv <= 0) return KDA_ERR_INVALID_ARG;
    if (!dim_ok(dk) || !dim_ok(dv)) return KDA_ERR_UNSUPPORTED;
    const int64_t NH = (int64_t)N * H;
    if (NH == 0) return KDA_OK;
    if (NH > 0x7fffffffLL) return KDA_ERR_UNSUPPORTED;
    if (!ptr_ok(q) || !ptr_ok(k) || !ptr_ok(v) || !ptr_ok(g) || !ptr_ok(state) || !ptr_ok(o))
        return KDA_ERR_INVALID_ARG;
    if (beta == nullptr || (reinterpret_cast<uintptr_t>(beta) & 1u) != 0) return KDA_ERR_INVALID_ARG;
    return status_of(decode_step_launch(q, k, v, g, beta, state, o, NH, dk, dv, raw,
                                        (cudaStream_t)stream));
}

int kda_decode_step(const void* q, const void* k, const void* v, const void* g,
                    const void* beta, float* state, void* o,
                    int N, int H, int dk, int dv, kda_stream_t stream)
{
    return decode_step_any(q, k, v, g, beta, state, o, N, H, dk, dv, false, stream);
}

int kda_decode_step_raw(const void* q_raw, const void* k_raw, const void* v, const void* z,
                        const void* beta, float* state, void* o,
                        int N, int H, int dk, int dv, kda_stream_t stream)
{
    return decode_step_any(q_raw, k_raw, v, z, beta, state, o, N, H, dk, dv, true, stream);
}

static int chunk_bwd_any(const void* q, const void* k, const void* v, const void* g, const void* beta,
                         const float* h0, const void* dO, const float* dhT,
                         void* dq, void* dk, void* dv, void* dg, void* dbeta, float* dh0,
                         int B, int T, int H, int d_k, int d_v, bool raw, kda_stream_t stream)
{
    int st = check_prefill(q, k, v, g, beta, h0, dO, dhT, B, T, H, d_k, d_v);
    if (st != KDA_OK) return st;
    if (!(d_k == 128 && d_v == 128)) return KDA_ERR_UNSUPPORTED;
    if (!opt_ptr_ok(dh0)) return KDA_ERR_INVALID_ARG;
    if ((int64_t)B * T * H > 0) {
        if (!ptr_ok(dq) || !ptr_ok(dk) || !ptr_ok(dv) || !ptr_ok(dg) || dbeta == nullptr)
            return KDA_ERR_INVALID_ARG;
        if (((reinterpret_cast<uintptr_t>(beta) | reinterpret_cast<uintptr_t>(dbeta)) & 1u) != 0)
            return KDA_ERR_INVALID_ARG;
    }
    if ((int64_t)B * H == 0) return KDA_OK;
    if (T == 0 && dh0 == nullptr) return KDA_OK;
    return status_of(chunk_bwd_launch(q, k, v, g, beta, h0, dO, dhT, dq, dk, dv, dg, dbeta, dh0, B, T, H, raw,
                                      (cudaStream_t)stream));
}

int kda_chunk_bwd(const void* q, const void* k, const void* v, const void* g, const void* beta,
                  const float* h0, const void* dO, const float* dhT,
                  void* dq, void* dk, void* dv, void* dg, void* dbeta, float* dh0,
                  int B, int T, int H, int d_k, int d_v, kda_stream_t stream)
{
    return chunk_bwd_any(q, k, v, g, beta, h0, dO, dhT, dq, dk, dv, dg, dbeta, dh0, B, T, H, d_k, d_v, false,
                         stream);
}

int kda_chunk_bwd_raw(const void* q_raw, const void* k_raw, const void* v, const void* z, const void* beta,
                      const float* h0, const void* dO, const float* dhT,
                      void* dq_raw, void* dk_raw, void* dv, void* dz, void* dbeta, float* dh0,
                      int B, int T, int H, int d_k, int d_v, kda_stream_t stream)
{
    return chunk_bwd_any(q_raw, k_raw, v, z, beta, h0, dO, dhT, dq_raw, dk_raw, dv, dz, dbeta, dh0, B, T, H,
                         d_k, d_v, true, stream);
}

int kda_verify_fwd(const void* q, const void* k, const void* v, const void* g,
                   const void* beta, const float* h0, void* o, float* states,
                   int N, int K, int H, int dk, int dv, kda_stream_t stream)
{
    if (N < 0 || K < 0 || H < 0 || dk <= 0 || dv <= 0) return KDA_ERR_INVALID_ARG;
    if (!dim_ok(dk) || !dim_ok(dv)) return KDA_ERR_UNSUPPORTED;
    if (N > 65535 || H > 65535 || K > KDA_VERIFY_MAX_TOKENS) return KDA_ERR_UNSUPPORTED;
    if ((int64_t)N * K * H == 0) return KDA_OK;
    if (!ptr_ok(q) || !ptr_ok(k) || !ptr_ok(v) || !ptr_ok(g) || !ptr_ok(o) || !ptr_ok(states) ||
        !opt_ptr_ok(h0))
        return KDA_ERR_INVALID_ARG;
    if (beta == nullptr || (reinterpret_cast<uintptr_t>(beta) & 1u) != 0) return KDA_ERR_INVALID_ARG;
    return status_of(verify_launch(q, k, v, g, beta, h0, o, states, N, K, H, dk, dv,
                                   (cudaStream_t)stream));
}

const char* kda_status_string(int status)
{
    switch (status) {
        case KDA_OK: return "KDA_OK";
        case KDA_ERR_INVALID_ARG: return "KDA_ERR_INVALID_ARG";
        case KDA_ERR_UNSUPPORTED: return "KDA_ERR_UNSUPPORTED";
        case KDA_ERR_CUDA: return "KDA_ERR_CUDA";
        case KDA_ERR_TIMEOUT: return "KDA_ERR_TIMEOUT";
        case KDA_ERR_NO_MEMORY: return "KDA_ERR_NO_MEMORY";
        default: return "KDA_ERR_UNKNOWN";
    }
}

int kda_device_status(kda_stream_t stream)
{
    const int a = prefill_device_status((cudaStream_t)stream);
    const int b = bwd_device_status((cudaStream_t)stream);
    if (a == KDA_ERR_CUDA || b == KDA_ERR_CUDA) return KDA_ERR_CUDA;
    return a != KDA_OK ? a : b;
}

int kda_selftest_bounded_wait(uint64_t limit_ns, kda_stream_t stream)
{
    if (limit_ns == 0 || limit_ns > 1000000000ull) return KDA_ERR_INVALID_ARG;
    return status_of(bounded_wait_selftest_launch(limit_ns, (cudaStream_t)stream));
}

uint64_t kda_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

int kda_prefill_path(int B, int T, int H)
{
    if (B < 0 || T < 0 || H < 0) return KDA_ERR_INVALID_ARG;
    return prefill_path_of(B, T, H);
}

int kda_version(void) { return (1 << 16) | 0; }

}  // extern "C"
