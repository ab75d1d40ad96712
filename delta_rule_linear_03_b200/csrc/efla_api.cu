// efla_api.cu - the C ABI declared in include/efla.h: validation, scratch
// sizing and kernel dispatch.  Every step of the computation runs in the
// kernels included below; this file only checks arguments and launches.
#include <algorithm>
#include <atomic>
#include <cstdint>
#include <cstring>

#include <nvtx3/nvToolsExt.h>

#include "../../include/efla.h"
#include "efla_backward.cuh"
#include "efla_chunk_simt.cuh"
#include "efla_chunk_tc.cuh"
#include "efla_common.cuh"
#include "efla_decode.cuh"
#include "efla_gate.cuh"

using namespace efla;

namespace {

constexpr long long kMaxElems = (1LL << 46);  // sanity bound on any tensor's element count

// NVTX range around one C-ABI call (validation and launches), so a profiler
// timeline shows which library call enqueued which kernels.  Header-only
// NVTX: without an attached tool a push or pop is a test of a null pointer.
struct NvtxRange {
    explicit NvtxRange(const char *name) { nvtxRangePushA(name); }
    ~NvtxRange() { nvtxRangePop(); }
    NvtxRange(const NvtxRange &) = delete;
    NvtxRange &operator=(const NvtxRange &) = delete;
};

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool overlaps(const void *a, size_t na, const void *b, size_t nb) {
    if (!a || !b || na == 0 || nb == 0) return false;
    const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
    return x < y + nb && y < x + na;
}

size_t esize(efla_dtype_t dt) { return dt == EFLA_F32 ? 4 : 2; }

efla_status_t check_common(efla_dtype_t dtype, efla_mode_t mode) {
    if (dtype != EFLA_F32 && dtype != EFLA_BF16) return EFLA_ERR_DTYPE;
    if (mode != EFLA_MODE_EXACT && mode != EFLA_MODE_EULER) return EFLA_ERR_DTYPE;
    return EFLA_OK;
}

efla_status_t check_head(int d_k, int d_v) {
    if (d_k <= 0 || d_v <= 0) return EFLA_ERR_SHAPE;
    if (d_k != d_v) return EFLA_ERR_UNSUPPORTED;
    if (d_k != 32 && d_k != 64 && d_k != 128) return EFLA_ERR_UNSUPPORTED;
    return EFLA_OK;
}

efla_status_t launched() { return cudaGetLastError() == cudaSuccess ? EFLA_OK : EFLA_ERR_CUDA; }

int num_sms() {
    static std::atomic<int> cached[64];
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 148;
    if ((n = cached[dev & 63].load(std::memory_order_relaxed)) > 0) return n;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
    cached[dev & 63].store(n, std::memory_order_relaxed);
    return n;
}

template <typename T, int D>
efla_status_t launch_gate(const void *k, const float *beta, float *alpha, float *lambda, long rows, bool euler,
                          cudaStream_t st) {
    constexpr int UNROLL = 4;
    constexpr int RPW = 32 / (D / (16 / (int)sizeof(T)));
    const long rows_per_block = 8L * RPW * UNROLL;
    long blocks = (rows + rows_per_block - 1) / rows_per_block;
    const long cap = 8L * num_sms();
    if (blocks > cap) blocks = cap;
    gate_kernel<T, D, UNROLL><<<(unsigned)blocks, 256, 0, st>>>(static_cast<const T *>(k), beta, alpha, lambda,
                                                                rows, euler);
    return launched();
}

template <typename T, typename To, int D>
efla_status_t launch_decode(const void *q, const void *k, const void *v, const float *beta, float *S, void *o,
                            long bh, bool euler, cudaStream_t st) {
    decode_kernel<T, To, D, D><<<(unsigned)bh, 256, 0, st>>>(static_cast<const T *>(q), static_cast<const T *>(k),
                                                             static_cast<const T *>(v), beta, S,
                                                             static_cast<To *>(o), euler);
    return launched();
}

template <typename T, typename To, int D>
efla_status_t launch_chunk_simt(const void *q, const void *k, const void *v, const float *beta, const float *S0,
                                void *o, float *SL, long bh, int L, void *workspace, bool euler, cudaStream_t st) {
    const int nc = (L + kChunk - 1) / kChunk;
    const SimtScratch ws = SimtScratch::carve(static_cast<float *>(workspace), bh * nc, D);
    const size_t prep_smem = sizeof(PrepSmem<D>);
    const size_t state_smem = sizeof(StateSmem<D>);
    if (!ensure_smem<chunk_prep_kernel<T, D>>(prep_smem) || !ensure_smem<chunk_state_kernel<T, To, D>>(state_smem))
        return EFLA_ERR_CUDA;
    if ((long long)nc * bh > 0x7fffffffLL) return EFLA_ERR_SHAPE;
    chunk_prep_kernel<T, D><<<(unsigned)(nc * bh), 256, prep_smem, st>>>(
        static_cast<const T *>(q), static_cast<const T *>(k), static_cast<const T *>(v), beta, L, nc, ws, euler);
    if (launched() != EFLA_OK) return EFLA_ERR_CUDA;
    chunk_state_kernel<T, To, D><<<(unsigned)((D / StateSmem<D>::DVT) * bh), 256, state_smem, st>>>(
        static_cast<const T *>(q), static_cast<const T *>(k), S0, static_cast<To *>(o), SL, L, nc, ws);
    return launched();
}

size_t simt_workspace_bytes(long bh, int L, int d) {
    const long nc = (L + kChunk - 1) / kChunk;
    return SimtScratch::floats(bh * nc, d) * sizeof(float);
}

// Instantiate F<Tin, Tout, D>(args...) for the runtime (dtype, o_dtype, d).
#define EFLA_DISPATCH(F, dtype, odtype, d, ...)                                                   \
    do {                                                                                          \
        const bool bf_in_ = (dtype) == EFLA_BF16, bf_out_ = (odtype) == EFLA_BF16;                \
        if (!bf_in_ && !bf_out_) {                                                                \
            if ((d) == 32) return F<float, float, 32>(__VA_ARGS__);                               \
            if ((d) == 64) return F<float, float, 64>(__VA_ARGS__);                               \
            return F<float, float, 128>(__VA_ARGS__);                                             \
        }                                                                                         \
        if (!bf_in_ && bf_out_) {                                                                 \
            if ((d) == 32) return F<float, __nv_bfloat16, 32>(__VA_ARGS__);                       \
            if ((d) == 64) return F<float, __nv_bfloat16, 64>(__VA_ARGS__);                       \
            return F<float, __nv_bfloat16, 128>(__VA_ARGS__);                                     \
        }                                                                                         \
        if (bf_in_ && !bf_out_) {                                                                 \
            if ((d) == 32) return F<__nv_bfloat16, float, 32>(__VA_ARGS__);                       \
            if ((d) == 64) return F<__nv_bfloat16, float, 64>(__VA_ARGS__);                       \
            return F<__nv_bfloat16, float, 128>(__VA_ARGS__);                                     \
        }                                                                                         \
        if ((d) == 32) return F<__nv_bfloat16, __nv_bfloat16, 32>(__VA_ARGS__);                   \
        if ((d) == 64) return F<__nv_bfloat16, __nv_bfloat16, 64>(__VA_ARGS__);                   \
        return F<__nv_bfloat16, __nv_bfloat16, 128>(__VA_ARGS__);                                 \
    } while (0)

// One mbarrier that nobody arrives on, waited on with the prefill kernel's
// bounded wait: exercises the timeout path end to end.
__global__ void diag_wait_timeout_kernel(long long limit_cycles) {
    __shared__ uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        abort_flag = 0;
        efla::ptx::mbar_init(&bar, 1);
        efla::ptx::fence_mbar_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) efla::ptx::mbar_wait(&bar, 0, &abort_flag, limit_cycles);
}

}  // namespace

extern "C" {

efla_status_t efla_diag_wait_timeout(long long limit_cycles, efla_stream_t stream) {
    if (limit_cycles <= 0 || limit_cycles > 8000000000LL) return EFLA_ERR_SHAPE;
    diag_wait_timeout_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(limit_cycles);
    return launched();
}

const char *efla_status_string(efla_status_t s) {
    switch (s) {
        case EFLA_OK: return "EFLA_OK";
        case EFLA_ERR_NULL: return "EFLA_ERR_NULL: a required pointer is NULL";
        case EFLA_ERR_SHAPE: return "EFLA_ERR_SHAPE: invalid size";
        case EFLA_ERR_DTYPE: return "EFLA_ERR_DTYPE: unknown dtype or mode";
        case EFLA_ERR_ALIGN: return "EFLA_ERR_ALIGN: pointer not 16-byte aligned";
        case EFLA_ERR_UNSUPPORTED: return "EFLA_ERR_UNSUPPORTED: head size must be d_k == d_v in {32,64,128}";
        case EFLA_ERR_CUDA: return "EFLA_ERR_CUDA: CUDA call or kernel launch failed";
        case EFLA_ERR_TIMEOUT: return "EFLA_ERR_TIMEOUT: a device-side bounded wait gave up";
        case EFLA_ERR_WORKSPACE: return "EFLA_ERR_WORKSPACE: workspace missing or too small";
        case EFLA_ERR_ALIAS: return "EFLA_ERR_ALIAS: an output overlaps an input";
    }
    return "EFLA_ERR_UNKNOWN";
}

int efla_version(void) { return 100; }

efla_status_t efla_last_error(void) {
    if (cudaDeviceSynchronize() != cudaSuccess) return EFLA_ERR_CUDA;
    unsigned int w = 0;
    if (cudaMemcpyFromSymbol(&w, g_error_word, sizeof(w)) != cudaSuccess) return EFLA_ERR_CUDA;
    if (w) {
        const unsigned int zero = 0;
        if (cudaMemcpyToSymbol(g_error_word, &zero, sizeof(zero)) != cudaSuccess) return EFLA_ERR_CUDA;
        return EFLA_ERR_TIMEOUT;
    }
    return cudaGetLastError() == cudaSuccess ? EFLA_OK : EFLA_ERR_CUDA;
}

efla_status_t efla_gate(const void *k, efla_dtype_t dtype, efla_mode_t mode, const float *beta, float *alpha,
                        float *lambda, int B, int H, int L, int d_k, efla_stream_t stream) {
    NvtxRange nvtx_("efla_gate");
    efla_status_t s = check_common(dtype, mode);
    if (s != EFLA_OK) return s;
    if (B < 0 || H < 0 || L < 0 || d_k <= 0) return EFLA_ERR_SHAPE;
    if ((s = check_head(d_k, d_k)) != EFLA_OK) return s;
    const long long rows = (long long)B * H * L;
    if (rows * d_k > kMaxElems) return EFLA_ERR_SHAPE;
    if (rows == 0) return EFLA_OK;
    if (!k || !beta || !alpha) return EFLA_ERR_NULL;
    if (!aligned16(k) || !aligned16(beta) || !aligned16(alpha) || (lambda && !aligned16(lambda)))
        return EFLA_ERR_ALIGN;
    const size_t kb = rows * d_k * esize(dtype), rb = rows * sizeof(float);
    if (overlaps(alpha, rb, k, kb) || overlaps(alpha, rb, beta, rb) || overlaps(lambda, rb, k, kb) ||
        overlaps(lambda, rb, beta, rb) || overlaps(lambda, rb, alpha, rb))
        return EFLA_ERR_ALIAS;
    const bool eu = mode == EFLA_MODE_EULER;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (dtype == EFLA_F32) {
        switch (d_k) {
            case 32: return launch_gate<float, 32>(k, beta, alpha, lambda, rows, eu, st);
            case 64: return launch_gate<float, 64>(k, beta, alpha, lambda, rows, eu, st);
            default: return launch_gate<float, 128>(k, beta, alpha, lambda, rows, eu, st);
        }
    }
    switch (d_k) {
        case 32: return launch_gate<__nv_bfloat16, 32>(k, beta, alpha, lambda, rows, eu, st);
        case 64: return launch_gate<__nv_bfloat16, 64>(k, beta, alpha, lambda, rows, eu, st);
        default: return launch_gate<__nv_bfloat16, 128>(k, beta, alpha, lambda, rows, eu, st);
    }
}

size_t efla_chunk_fwd_workspace_size(efla_dtype_t dtype, int B, int H, int L, int d_k, int d_v) {
    if (check_common(dtype, EFLA_MODE_EXACT) != EFLA_OK || B <= 0 || H <= 0 || L <= 0) return 0;
    if (check_head(d_k, d_v) != EFLA_OK) return 0;
    if (tc_path_applies(dtype == EFLA_BF16, d_k, d_v)) return tc::workspace_bytes((long)B * H, L);
    return simt_workspace_bytes((long)B * H, L, d_k);
}

efla_status_t efla_chunk_fwd(const void *q, const void *k, const void *v, efla_dtype_t dtype, efla_mode_t mode,
                             const float *beta, const float *S0, void *o, efla_dtype_t o_dtype, float *S_L, int B,
                             int H, int L, int d_k, int d_v, void *workspace, size_t workspace_bytes,
                             efla_stream_t stream) {
    NvtxRange nvtx_("efla_chunk_fwd");
    efla_status_t s = check_common(dtype, mode);
    if (s != EFLA_OK) return s;
    if ((s = check_common(o_dtype, mode)) != EFLA_OK) return s;
    if (B < 0 || H < 0 || L < 0) return EFLA_ERR_SHAPE;
    if ((s = check_head(d_k, d_v)) != EFLA_OK) return s;
    const long long bh = (long long)B * H;
    if (bh * (long long)(L > 0 ? L : 1) * d_k > kMaxElems || bh > 0x7fffffffLL) return EFLA_ERR_SHAPE;
    if (bh == 0) return EFLA_OK;
    const size_t sbytes = (size_t)bh * d_k * d_v * sizeof(float);
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (L == 0) {  // empty sequence: the state passes through unchanged
        if (S_L) {
            if (!aligned16(S_L) || (S0 && !aligned16(S0))) return EFLA_ERR_ALIGN;
            if (S0 && S0 != S_L && overlaps(S0, sbytes, S_L, sbytes)) return EFLA_ERR_ALIAS;
            cudaError_t e = S0 ? (S0 == S_L ? cudaSuccess : cudaMemcpyAsync(S_L, S0, sbytes, cudaMemcpyDeviceToDevice, st))
                               : cudaMemsetAsync(S_L, 0, sbytes, st);
            return e == cudaSuccess ? EFLA_OK : EFLA_ERR_CUDA;
        }
        return EFLA_OK;
    }
    if (!q || !k || !v || !beta || !o) return EFLA_ERR_NULL;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(beta) || !aligned16(o) ||
        (S0 && !aligned16(S0)) || (S_L && !aligned16(S_L)) || (workspace && !aligned16(workspace)))
        return EFLA_ERR_ALIGN;
    const size_t xb = (size_t)bh * L * d_k * esize(dtype), bb = (size_t)bh * L * sizeof(float);
    const size_t ob = (size_t)bh * L * d_v * esize(o_dtype);
    if (overlaps(o, ob, q, xb) || overlaps(o, ob, k, xb) || overlaps(o, ob, v, xb) || overlaps(o, ob, beta, bb) ||
        overlaps(o, ob, S0, sbytes))
        return EFLA_ERR_ALIAS;
    if (S_L && (overlaps(S_L, sbytes, q, xb) || overlaps(S_L, sbytes, k, xb) || overlaps(S_L, sbytes, v, xb) ||
                overlaps(S_L, sbytes, beta, bb) || overlaps(S_L, sbytes, o, ob) ||
                (S0 && S0 != S_L && overlaps(S_L, sbytes, S0, sbytes))))
        return EFLA_ERR_ALIAS;
    const bool eu = mode == EFLA_MODE_EULER;
    const bool bf = dtype == EFLA_BF16;

    const bool tcp = tc_path_applies(bf, d_k, d_v);
    const size_t need = tcp ? tc::workspace_bytes(bh, L) : simt_workspace_bytes(bh, L, d_k);
    if (!workspace || workspace_bytes < need) return EFLA_ERR_WORKSPACE;
    if (overlaps(workspace, need, q, xb) || overlaps(workspace, need, k, xb) || overlaps(workspace, need, v, xb) ||
        overlaps(workspace, need, o, ob) || overlaps(workspace, need, beta, bb) ||
        overlaps(workspace, need, S0, sbytes) || overlaps(workspace, need, S_L, sbytes))
        return EFLA_ERR_ALIAS;
    if (tcp) return launch_chunk_tc(q, k, v, beta, S0, o, o_dtype == EFLA_BF16, S_L, bh, L, eu, workspace, st);
    EFLA_DISPATCH(launch_chunk_simt, dtype, o_dtype, d_k, q, k, v, beta, S0, o, S_L, bh, L, workspace, eu, st);
}

efla_status_t efla_decode_step(const void *q, const void *k, const void *v, efla_dtype_t dtype, efla_mode_t mode,
                               const float *beta, float *S, void *o, efla_dtype_t o_dtype, int B, int H, int d_k,
                               int d_v, efla_stream_t stream) {
    NvtxRange nvtx_("efla_decode_step");
    efla_status_t s = check_common(dtype, mode);
    if (s != EFLA_OK) return s;
    if ((s = check_common(o_dtype, mode)) != EFLA_OK) return s;
    if (B < 0 || H < 0) return EFLA_ERR_SHAPE;
    if ((s = check_head(d_k, d_v)) != EFLA_OK) return s;
    const long long bh = (long long)B * H;
    if (bh * d_k * d_v > kMaxElems || bh > 0x7fffffffLL) return EFLA_ERR_SHAPE;
    if (bh == 0) return EFLA_OK;
    if (!q || !k || !v || !beta || !S || !o) return EFLA_ERR_NULL;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(beta) || !aligned16(S) || !aligned16(o))
        return EFLA_ERR_ALIGN;
    const size_t xb = (size_t)bh * d_k * esize(dtype), bb = (size_t)bh * sizeof(float);
    const size_t ob = (size_t)bh * d_v * esize(o_dtype);
    const size_t sbytes = (size_t)bh * d_k * d_v * sizeof(float);
    if (overlaps(o, ob, q, xb) || overlaps(o, ob, k, xb) || overlaps(o, ob, v, xb) || overlaps(o, ob, beta, bb) ||
        overlaps(o, ob, S, sbytes) || overlaps(S, sbytes, q, xb) || overlaps(S, sbytes, k, xb) ||
        overlaps(S, sbytes, v, xb) || overlaps(S, sbytes, beta, bb))
        return EFLA_ERR_ALIAS;
    const bool eu = mode == EFLA_MODE_EULER;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    EFLA_DISPATCH(launch_decode, dtype, o_dtype, d_k, q, k, v, beta, S, o, bh, eu, st);
}

size_t efla_prefill_bwd_workspace_size(int B, int H, int L, int d_k, int d_v) {
    if (B <= 0 || H <= 0 || L <= 0 || check_head(d_k, d_v) != EFLA_OK) return 0;
    return (size_t)B * H * L * ((size_t)d_v + 1 + 4) * sizeof(float);  // e_t, one scalar, the gate (float4)
}

}  // extern "C"

namespace {
template <typename T, int D>
efla_status_t launch_bwd(const void *q, const void *k, const void *v, const float *beta, const float *S0,
                         const float *dO, const float *dSL, float *dq, float *dk, float *dv, float *dbeta, float *dS0,
                         long bh, int L, bool eu, void *ws, cudaStream_t st) {
    float4 *G = static_cast<float4 *>(ws);  // first: 16-byte aligned
    float *E = reinterpret_cast<float *>(G + (size_t)bh * L);
    float *Cg = E + (size_t)bh * L * D;
    const long rows = bh * L;
    const unsigned gblocks = (unsigned)std::min<long>((rows + 7) / 8, 148L * 16);
    efla::backward_gate_kernel<T, D><<<gblocks, 256, 0, st>>>(static_cast<const T *>(k), beta, G, rows, eu);
    if (cudaGetLastError() != cudaSuccess) return EFLA_ERR_CUDA;
    efla::backward_kernel<T, D, D><<<(unsigned)bh, 256, 0, st>>>(
        static_cast<const T *>(q), static_cast<const T *>(k), static_cast<const T *>(v), G, S0, dO, dSL, dq, dk, dv,
        dbeta, dS0, E, Cg, L);
    return cudaGetLastError() == cudaSuccess ? EFLA_OK : EFLA_ERR_CUDA;
}
}  // namespace

extern "C" {

efla_status_t efla_prefill_bwd(const void *q, const void *k, const void *v, efla_dtype_t dtype, efla_mode_t mode,
                               const float *beta, const float *S0, const float *dO, const float *dSL, float *dq,
                               float *dk, float *dv, float *dbeta, float *dS0, int B, int H, int L, int d_k, int d_v,
                               void *workspace, size_t workspace_bytes, efla_stream_t stream) {
    NvtxRange nvtx_("efla_prefill_bwd");
    efla_status_t s = check_common(dtype, mode);
    if (s != EFLA_OK) return s;
    if (B < 0 || H < 0 || L < 0) return EFLA_ERR_SHAPE;
    if ((s = check_head(d_k, d_v)) != EFLA_OK) return s;
    const long long bh = (long long)B * H;
    if (bh * (long long)(L > 0 ? L : 1) * d_k > kMaxElems || bh > 0x7fffffffLL) return EFLA_ERR_SHAPE;
    if (bh == 0) return EFLA_OK;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const size_t sbytes = (size_t)bh * d_k * d_v * sizeof(float);
    if (L == 0) {  // no tokens (per-token buffers may be NULL): dS0 = dSL
        if (!dS0) return EFLA_ERR_NULL;
        if (!aligned16(dS0) || (dSL && !aligned16(dSL))) return EFLA_ERR_ALIGN;
        if (dSL && overlaps(dS0, sbytes, dSL, sbytes)) return EFLA_ERR_ALIAS;
        if (dSL) return cudaMemcpyAsync(dS0, dSL, sbytes, cudaMemcpyDeviceToDevice, st) == cudaSuccess ? EFLA_OK
                                                                                                     : EFLA_ERR_CUDA;
        return cudaMemsetAsync(dS0, 0, sbytes, st) == cudaSuccess ? EFLA_OK : EFLA_ERR_CUDA;
    }
    if (!q || !k || !v || !beta || !dO || !dq || !dk || !dv || !dbeta || !dS0) return EFLA_ERR_NULL;
    const void *ins[] = {q, k, v, beta, S0, dO, dSL};
    const void *outs[] = {dq, dk, dv, dbeta, dS0};
    for (const void *p : ins)
        if (p && !aligned16(p)) return EFLA_ERR_ALIGN;
    for (const void *p : outs)
        if (!aligned16(p)) return EFLA_ERR_ALIGN;
    const size_t xb = (size_t)bh * L * d_k * esize(dtype), fb = (size_t)bh * L * d_k * sizeof(float);
    const size_t bb = (size_t)bh * L * sizeof(float);
    const size_t in_b[] = {xb, xb, xb, bb, sbytes, fb, sbytes};
    const size_t out_b[] = {fb, fb, fb, bb, sbytes};
    for (int i = 0; i < 5; ++i) {
        for (int j = 0; j < 7; ++j)
            if (ins[j] && overlaps(outs[i], out_b[i], ins[j], in_b[j])) return EFLA_ERR_ALIAS;
        for (int j = 0; j < i; ++j)
            if (overlaps(outs[i], out_b[i], outs[j], out_b[j])) return EFLA_ERR_ALIAS;
    }
    const size_t need = efla_prefill_bwd_workspace_size(B, H, L, d_k, d_v);
    if (!workspace || workspace_bytes < need) return EFLA_ERR_WORKSPACE;
    if (!aligned16(workspace)) return EFLA_ERR_ALIGN;
    const bool eu = mode == EFLA_MODE_EULER;
    const bool bf = dtype == EFLA_BF16;
#define EFLA_BWD(T, D) return launch_bwd<T, D>(q, k, v, beta, S0, dO, dSL, dq, dk, dv, dbeta, dS0, bh, L, eu, workspace, st)
    if (bf) {
        if (d_k == 32) EFLA_BWD(__nv_bfloat16, 32);
        if (d_k == 64) EFLA_BWD(__nv_bfloat16, 64);
        EFLA_BWD(__nv_bfloat16, 128);
    }
    if (d_k == 32) EFLA_BWD(float, 32);
    if (d_k == 64) EFLA_BWD(float, 64);
    EFLA_BWD(float, 128);
#undef EFLA_BWD
}

efla_status_t efla_state_affine(const float *SI, const float *SZ, const float *X, float *out, int B, int H, int d,
                                efla_stream_t stream) {
    NvtxRange nvtx_("efla_state_affine");
    if (B < 0 || H < 0) return EFLA_ERR_SHAPE;
    if (d != 32 && d != 64 && d != 128) return EFLA_ERR_UNSUPPORTED;
    const long long bh = (long long)B * H;
    if (bh * d * d > kMaxElems || bh > 0x7fffffffLL) return EFLA_ERR_SHAPE;
    if (bh == 0) return EFLA_OK;
    if (!SI || !SZ || !X || !out) return EFLA_ERR_NULL;
    if (!aligned16(SI) || !aligned16(SZ) || !aligned16(X) || !aligned16(out)) return EFLA_ERR_ALIGN;
    const size_t sb = (size_t)bh * d * d * sizeof(float);
    if (overlaps(out, sb, SI, sb) || overlaps(out, sb, SZ, sb) || overlaps(out, sb, X, sb)) return EFLA_ERR_ALIAS;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const dim3 grid((unsigned)bh, (unsigned)(d / 32));
    switch (d) {
        case 32: tc::affine_step_kernel<32><<<grid, 256, 0, st>>>(SI, SZ, X, out); break;
        case 64: tc::affine_step_kernel<64><<<grid, 256, 0, st>>>(SI, SZ, X, out); break;
        default: tc::affine_step_kernel<128><<<grid, 256, 0, st>>>(SI, SZ, X, out); break;
    }
    return cudaGetLastError() == cudaSuccess ? EFLA_OK : EFLA_ERR_CUDA;
}

}  // extern "C"

// ---------------------------------------------------------------------------
// No-allocation variant of the chunked prefill.
//
// For callers that cannot allocate device memory (an engine that owns every
// byte of GPU memory through its own pool, or a loop where cudaMalloc's
// implicit synchronisation is not acceptable): the CUDA-core chunked kernels
// run with their scratch in this fixed file-scope array instead of a
// caller-provided workspace.  Every GPU that loads the library holds it
// until the process exits; all calls on a device share it.
namespace {

static __device__ __align__(256) unsigned char g_noalloc_scratch[EFLA_NOALLOC_SCRATCH_BYTES];

// Device address of g_noalloc_scratch on the current device, looked up once
// per device.  Host code must not use the symbol itself as a pointer: on the
// host it is only a stand-in for the device variable.
void *noalloc_scratch_ptr() {
    static std::atomic<uintptr_t> cached[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
    uintptr_t p = cached[dev].load(std::memory_order_acquire);
    if (p) return reinterpret_cast<void *>(p);
    void *addr = nullptr;
    if (cudaGetSymbolAddress(&addr, g_noalloc_scratch) != cudaSuccess || !addr) return nullptr;
    cached[dev].store(reinterpret_cast<uintptr_t>(addr), std::memory_order_release);
    return addr;
}

}  // namespace

extern "C" {

size_t efla_chunk_fwd_workspace_size_simt(int B, int H, int L, int d_k, int d_v) {
    if (B <= 0 || H <= 0 || L <= 0 || check_head(d_k, d_v) != EFLA_OK) return 0;
    return simt_workspace_bytes((long)B * H, L, d_k);
}

efla_status_t efla_chunk_fwd_noalloc(const void *q, const void *k, const void *v, efla_dtype_t dtype,
                                     efla_mode_t mode, const float *beta, const float *S0, void *o,
                                     efla_dtype_t o_dtype, float *S_L, int B, int H, int L, int d_k, int d_v,
                                     efla_stream_t stream) {
    NvtxRange nvtx_("efla_chunk_fwd_noalloc");
    efla_status_t s = check_common(dtype, mode);
    if (s != EFLA_OK) return s;
    if ((s = check_common(o_dtype, mode)) != EFLA_OK) return s;
    if (B < 0 || H < 0 || L < 0) return EFLA_ERR_SHAPE;
    if ((s = check_head(d_k, d_v)) != EFLA_OK) return s;
    const long long bh = (long long)B * H;
    if (bh * (long long)(L > 0 ? L : 1) * d_k > kMaxElems || bh > 0x7fffffffLL) return EFLA_ERR_SHAPE;
    if (bh == 0 || L == 0)  // nothing uses scratch: the regular entry point handles these allocation-free
        return efla_chunk_fwd(q, k, v, dtype, mode, beta, S0, o, o_dtype, S_L, B, H, L, d_k, d_v, nullptr, 0,
                              stream);
    const size_t need = simt_workspace_bytes(bh, L, d_k);
    if (need > EFLA_NOALLOC_SCRATCH_BYTES) return EFLA_ERR_WORKSPACE;
    if (!q || !k || !v || !beta || !o) return EFLA_ERR_NULL;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(beta) || !aligned16(o) ||
        (S0 && !aligned16(S0)) || (S_L && !aligned16(S_L)))
        return EFLA_ERR_ALIGN;
    const size_t xb = (size_t)bh * L * d_k * esize(dtype), bb = (size_t)bh * L * sizeof(float);
    const size_t ob = (size_t)bh * L * d_v * esize(o_dtype);
    const size_t sbytes = (size_t)bh * d_k * d_v * sizeof(float);
    if (overlaps(o, ob, q, xb) || overlaps(o, ob, k, xb) || overlaps(o, ob, v, xb) || overlaps(o, ob, beta, bb) ||
        overlaps(o, ob, S0, sbytes))
        return EFLA_ERR_ALIAS;
    if (S_L && (overlaps(S_L, sbytes, q, xb) || overlaps(S_L, sbytes, k, xb) || overlaps(S_L, sbytes, v, xb) ||
                overlaps(S_L, sbytes, beta, bb) || overlaps(S_L, sbytes, o, ob) ||
                (S0 && S0 != S_L && overlaps(S_L, sbytes, S0, sbytes))))
        return EFLA_ERR_ALIAS;
    void *scratch = noalloc_scratch_ptr();
    if (!scratch) return EFLA_ERR_CUDA;
    const bool eu = mode == EFLA_MODE_EULER;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    EFLA_DISPATCH(launch_chunk_simt, dtype, o_dtype, d_k, q, k, v, beta, S0, o, S_L, bh, L, scratch, eu, st);
}

}  // extern "C"
