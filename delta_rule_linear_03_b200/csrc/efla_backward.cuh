// efla_backward.cuh - reverse-mode derivative of the prefill.
//
// The pages train with this mixer but print no backward; it follows from
// the recurrence of "Exact Flow Linear Attention" (papernotes.org summary,
// 关键设计 2; readout of the 整体框架 flowchart):
//   S_t = S_{t-1} + alpha_t k_t e_t^T,  e_t = v_t - S_{t-1}^T k_t,
//   o_t = S_t^T q_t,  alpha_t = gate(beta_t, ||k_t||^2).
// For the loss L = sum(dO * o) + sum(dS_L * S_L), backwards over t with
// H = dL/dS_t (its readout included: H += q_t do_t^T):
//   g = H^T k_t,  d alpha = g . e_t,  de = alpha g  (= dv_t),
//   dq_t = S_t do_t,  dk_t = alpha H e_t - S_{t-1} de + 2 d alpha (d alpha/d lambda) k_t,
//   dbeta_t = d alpha (d alpha/d beta),  H <- H - k_t de^T,  dS0 = H at the end.
//
// A parallel pre-pass stores alpha and its two derivatives per token.  Then
// one CTA of 256 threads per (b, h) keeps one d_k x d_v fp32 matrix in
// registers (the decode kernel's layout: thread (row group, column quad)
// holds RPT rows x 4 columns) and walks the sequence three times, the next
// token's vectors prefetched by cp.async into the other half of
// double-buffered shared memory:
//   1. forward:  S from S0; stores e_t and dq_t;
//   2. backward: H from dS_L; stores dv_t, alpha H e_t (into dk), dbeta_t and
//      2 d alpha (d alpha / d lambda), and dS0;
//   3. forward:  S from S0 again; dk_t -= S_{t-1} de_t, += the gate term.
// Exact fp32 arithmetic, serial over tokens: the plain first version of the
// backward (the tensor-core chunked form is not built).
#pragma once
#include "efla_common.cuh"

namespace efla {

// d alpha / d beta and d alpha / d lambda of gate_alpha.  With x = beta lambda:
// d alpha / d beta = e^{-x}; d alpha / d lambda = (x e^{-x} - (1 - e^{-x})) / lambda^2,
// summed as beta^2 sum_{n>=2} (-1)^{n+1} (n-1) x^{n-2} / n! for |x| < 0.05
// (the closed form cancels there).  Zero where the clamp lambda <= 1e-12 holds.
__device__ __forceinline__ void gate_alpha_grad(float beta, float lambda, bool euler, float &da_db, float &da_dl) {
    if (euler) {
        da_db = 1.f;
        da_dl = 0.f;
        return;
    }
    if (!(lambda > 1e-12f)) {
        da_db = expf(-beta * 1e-12f);
        da_dl = 0.f;
        return;
    }
    const float x = beta * lambda;
    da_db = expf(-x);
    if (fabsf(x) < 0.05f) {
        // -1/2 + 2x/3! - 3x^2/4! + 4x^3/5! - 5x^4/6! + 6x^5/7!
        const float s = -0.5f + x * (1.f / 3.f + x * (-1.f / 8.f + x * (1.f / 30.f + x * (-1.f / 144.f + x * (1.f / 840.f)))));
        da_dl = beta * beta * s;
    } else {
        da_dl = (x * expf(-x) + expm1f(-x)) / (lambda * lambda);
    }
}

// Per-token gate and its derivatives for the backward, all tokens in
// parallel: G[row] = (alpha, d alpha / d beta, d alpha / d lambda, 0).  One
// warp per key row.
template <typename T, int DK>
__global__ void __launch_bounds__(256) backward_gate_kernel(const T *__restrict__ k, const float *__restrict__ beta,
                                                            float4 *__restrict__ G, long rows, bool euler) {
    const int lane = threadIdx.x & 31;
    const long w0 = ((long)blockIdx.x * blockDim.x + threadIdx.x) >> 5, nw = ((long)gridDim.x * blockDim.x) >> 5;
    for (long r = w0; r < rows; r += nw) {
        float lam = 0.f;
#pragma unroll
        for (int i = lane; i < DK; i += 32) {
            const float x = to_f32(k[r * DK + i]);
            lam = fmaf(x, x, lam);
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) lam += __shfl_xor_sync(0xffffffffu, lam, o);
        if (lane == 0) {
            const float b = beta[r];
            float da_db, da_dl;
            gate_alpha_grad(b, lam, euler, da_db, da_dl);
            G[r] = make_float4(gate_alpha(b, lam, euler), da_db, da_dl, 0.f);
        }
    }
}

// 16 per-row partial sums spread over 32 lanes -> each even lane holds the
// full sum of row (lane >> 1) (reduce-scatter: 8 + 4 + 2 + 1 + 1 shuffles).
__device__ __forceinline__ float reduce_rows16(float (&v)[16], int lane) {
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const bool up = lane & 16;
        const float send = up ? v[i] : v[i + 8], keep = up ? v[i + 8] : v[i];
        v[i] = keep + __shfl_xor_sync(0xffffffffu, send, 16);
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const bool up = lane & 8;
        const float send = up ? v[i] : v[i + 4], keep = up ? v[i + 4] : v[i];
        v[i] = keep + __shfl_xor_sync(0xffffffffu, send, 8);
    }
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        const bool up = lane & 4;
        const float send = up ? v[i] : v[i + 2], keep = up ? v[i + 2] : v[i];
        v[i] = keep + __shfl_xor_sync(0xffffffffu, send, 4);
    }
    {
        const bool up = lane & 2;
        const float send = up ? v[0] : v[1], keep = up ? v[1] : v[0];
        v[0] = keep + __shfl_xor_sync(0xffffffffu, send, 2);
    }
    return v[0] + __shfl_xor_sync(0xffffffffu, v[0], 1);
}

// 4-byte-granular cp.async global -> shared (n_bytes a multiple of 16 here).
__device__ __forceinline__ void cp_async_bytes(void *dst, const void *src, int n_bytes, int tid, int nthreads) {
    for (int o = 16 * tid; o < n_bytes; o += 16 * nthreads)
        asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"((uint32_t)__cvta_generic_to_shared(
                         static_cast<char *>(dst) + o)),
                     "l"(static_cast<const char *>(src) + o)
                     : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() {
    asm volatile("cp.async.commit_group;\n\tcp.async.wait_group 0;" ::: "memory");
}

template <typename T, int DK, int DV>
__global__ void __launch_bounds__(256, 1)
    backward_kernel(const T *__restrict__ q, const T *__restrict__ k, const T *__restrict__ v,
                    const float4 *__restrict__ G, const float *__restrict__ S0, const float *__restrict__ dO,
                    const float *__restrict__ dSL, float *__restrict__ dq, float *__restrict__ dk,
                    float *__restrict__ dv, float *__restrict__ dbeta, float *__restrict__ dS0,
                    float *__restrict__ E, float *__restrict__ Cg, int L) {
    constexpr int CG = DV / 4;    // column quads
    constexpr int RG = 256 / CG;  // row groups
    constexpr int RPT = DK / RG;  // rows per thread
    static_assert(RPT >= 1 && RG * RPT == DK && (32 % CG) == 0, "state tile must cover d_k");
    constexpr bool kScatter = (RPT == 16 && CG == 32);  // reduce-scatter of the 16 row sums
    // double-buffered per-token vectors (raw input dtype for q, k, v)
    __shared__ __align__(16) T kb[2][DK], qb[2][DK], vb[2][DV];
    __shared__ __align__(16) float f1[2][DV], f2[2][DV], xk[2][DK];
    __shared__ __align__(16) float4 gb[2];
    __shared__ __align__(16) float red[RG][DV];
    __shared__ float cb[2];

    const long bh = blockIdx.x;
    const int t = threadIdx.x, lane = t & 31, cg = t % CG, rg = t / CG;
    const size_t S_off = (size_t)bh * DK * DV;
    auto rsum = [&](float x) {
#pragma unroll
        for (int o = CG / 2; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
        return x;
    };
    auto load_state = [&](const float *src, float4 (&m)[RPT]) {
#pragma unroll
        for (int i = 0; i < RPT; ++i)
            m[i] = src ? *(reinterpret_cast<const float4 *>(src + S_off + (size_t)(rg * RPT + i) * DV) + cg)
                       : make_float4(0.f, 0.f, 0.f, 0.f);
    };
    auto colsum = [&](const float4 &x) {  // sum over row groups of a per-thread column-quad partial
        *reinterpret_cast<float4 *>(&red[rg][4 * cg]) = x;
        __syncthreads();
        float4 s = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int g = 0; g < RG; ++g) {
            const float4 y = *reinterpret_cast<const float4 *>(&red[g][4 * cg]);
            s.x += y.x; s.y += y.y; s.z += y.z; s.w += y.w;
        }
        return s;
    };
    float4 m[RPT];

    // ---------------------------------------------------------------- pass 1: S forward; e_t, dq_t
    auto fetch1 = [&](int s, int b) {
        const size_t row = (size_t)bh * L + s;
        cp_async_bytes(kb[b], k + row * DK, DK * (int)sizeof(T), t, 256);
        cp_async_bytes(vb[b], v + row * DV, DV * (int)sizeof(T), t, 256);
        cp_async_bytes(f1[b], dO + row * DV, DV * 4, t, 256);
        cp_async_bytes(&gb[b], G + row, 16, t, 256);
    };
    load_state(S0, m);
    fetch1(0, 0);
    cp_async_wait_all();
    __syncthreads();
    for (int s = 0; s < L; ++s) {
        const int b = s & 1;
        const size_t row = (size_t)bh * L + s;
        if (s + 1 < L) fetch1(s + 1, b ^ 1);
        float4 r = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int i = 0; i < RPT; ++i) {
            const float kk = to_f32(kb[b][rg * RPT + i]);
            r.x = fmaf(m[i].x, kk, r.x); r.y = fmaf(m[i].y, kk, r.y);
            r.z = fmaf(m[i].z, kk, r.z); r.w = fmaf(m[i].w, kk, r.w);
        }
        const float4 rt = colsum(r);
        const float a = gb[b].x;
        const float4 e = make_float4(to_f32(vb[b][4 * cg]) - rt.x, to_f32(vb[b][4 * cg + 1]) - rt.y,
                                     to_f32(vb[b][4 * cg + 2]) - rt.z, to_f32(vb[b][4 * cg + 3]) - rt.w);
        if (rg == 0) *(reinterpret_cast<float4 *>(E + row * DV) + cg) = e;
        const float4 dd = *reinterpret_cast<const float4 *>(&f1[b][4 * cg]);
        float p[RPT];
#pragma unroll
        for (int i = 0; i < RPT; ++i) {
            const float kk = a * to_f32(kb[b][rg * RPT + i]);
            m[i].x = fmaf(kk, e.x, m[i].x); m[i].y = fmaf(kk, e.y, m[i].y);
            m[i].z = fmaf(kk, e.z, m[i].z); m[i].w = fmaf(kk, e.w, m[i].w);
            p[i] = m[i].x * dd.x + m[i].y * dd.y + m[i].z * dd.z + m[i].w * dd.w;
        }
        if constexpr (kScatter) {
            const float sv = reduce_rows16(p, lane);
            const int r_ = rg * RPT + (lane >> 1);
            if ((lane & 1) == 0) dq[row * DK + r_] = sv;
        } else {
#pragma unroll
            for (int i = 0; i < RPT; ++i) {
                const float sv = rsum(p[i]);
                const int r_ = rg * RPT + i;
                if (cg == 0) dq[row * DK + r_] = sv;
            }
        }
        cp_async_wait_all();
        __syncthreads();
    }

    // ---------------------------------------------------------------- pass 2: H backward
    auto fetch2 = [&](int s, int b) {
        const size_t row = (size_t)bh * L + s;
        cp_async_bytes(kb[b], k + row * DK, DK * (int)sizeof(T), t, 256);
        cp_async_bytes(qb[b], q + row * DK, DK * (int)sizeof(T), t, 256);
        cp_async_bytes(f1[b], dO + row * DV, DV * 4, t, 256);
        cp_async_bytes(f2[b], E + row * DV, DV * 4, t, 256);
        cp_async_bytes(&gb[b], G + row, 16, t, 256);
    };
    load_state(dSL, m);
    fetch2(L - 1, 0);
    cp_async_wait_all();
    __syncthreads();
    for (int s = L - 1, it = 0; s >= 0; --s, ++it) {
        const int b = it & 1;
        const size_t row = (size_t)bh * L + s;
        if (s > 0) fetch2(s - 1, b ^ 1);
        const float4 dd = *reinterpret_cast<const float4 *>(&f1[b][4 * cg]);
        float4 g = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int i = 0; i < RPT; ++i) {
            const float qq = to_f32(qb[b][rg * RPT + i]), kk = to_f32(kb[b][rg * RPT + i]);
            m[i].x = fmaf(qq, dd.x, m[i].x); m[i].y = fmaf(qq, dd.y, m[i].y);
            m[i].z = fmaf(qq, dd.z, m[i].z); m[i].w = fmaf(qq, dd.w, m[i].w);
            g.x = fmaf(m[i].x, kk, g.x); g.y = fmaf(m[i].y, kk, g.y);
            g.z = fmaf(m[i].z, kk, g.z); g.w = fmaf(m[i].w, kk, g.w);
        }
        const float4 gt = colsum(g);
        const float4 gg = gb[b];
        const float a = gg.x;
        const float4 e = *reinterpret_cast<const float4 *>(&f2[b][4 * cg]);
        const float dal = rsum(gt.x * e.x + gt.y * e.y + gt.z * e.z + gt.w * e.w);
        const float4 de = make_float4(a * gt.x, a * gt.y, a * gt.z, a * gt.w);
        if (rg == 0) *(reinterpret_cast<float4 *>(dv + row * DV) + cg) = de;
        float p[RPT];
#pragma unroll
        for (int i = 0; i < RPT; ++i) {
            p[i] = m[i].x * e.x + m[i].y * e.y + m[i].z * e.z + m[i].w * e.w;
            const float kk = to_f32(kb[b][rg * RPT + i]);
            m[i].x = fmaf(-kk, de.x, m[i].x); m[i].y = fmaf(-kk, de.y, m[i].y);
            m[i].z = fmaf(-kk, de.z, m[i].z); m[i].w = fmaf(-kk, de.w, m[i].w);
        }
        if constexpr (kScatter) {
            const float sv = reduce_rows16(p, lane);
            const int r_ = rg * RPT + (lane >> 1);
            if ((lane & 1) == 0) dk[row * DK + r_] = a * sv;
        } else {
#pragma unroll
            for (int i = 0; i < RPT; ++i) {
                const float sv = rsum(p[i]);
                const int r_ = rg * RPT + i;
                if (cg == 0) dk[row * DK + r_] = a * sv;
            }
        }
        if (t == 0) {
            dbeta[row] = dal * gg.y;
            Cg[row] = 2.f * dal * gg.z;
        }
        cp_async_wait_all();
        __syncthreads();
    }
#pragma unroll
    for (int i = 0; i < RPT; ++i)
        *(reinterpret_cast<float4 *>(dS0 + S_off + (size_t)(rg * RPT + i) * DV) + cg) = m[i];
    __syncthreads();  // dk, dv and Cg of pass 2 are read back below

    // ---------------------------------------------------------------- pass 3: S forward; dk_t
    auto fetch3 = [&](int s, int b) {
        const size_t row = (size_t)bh * L + s;
        cp_async_bytes(kb[b], k + row * DK, DK * (int)sizeof(T), t, 256);
        cp_async_bytes(xk[b], dk + row * DK, DK * 4, t, 256);
        cp_async_bytes(f1[b], dv + row * DV, DV * 4, t, 256);
        cp_async_bytes(f2[b], E + row * DV, DV * 4, t, 256);
        cp_async_bytes(&gb[b], G + row, 16, t, 256);
        if (t == 0) cb[b] = Cg[row];
    };
    load_state(S0, m);
    fetch3(0, 0);
    cp_async_wait_all();
    __syncthreads();
    for (int s = 0; s < L; ++s) {
        const int b = s & 1;
        const size_t row = (size_t)bh * L + s;
        if (s + 1 < L) fetch3(s + 1, b ^ 1);
        const float a = gb[b].x, c = cb[b];
        const float4 de = *reinterpret_cast<const float4 *>(&f1[b][4 * cg]);
        const float4 e = *reinterpret_cast<const float4 *>(&f2[b][4 * cg]);
        float p[RPT];
#pragma unroll
        for (int i = 0; i < RPT; ++i) {
            p[i] = m[i].x * de.x + m[i].y * de.y + m[i].z * de.z + m[i].w * de.w;
            const float kk = a * to_f32(kb[b][rg * RPT + i]);
            m[i].x = fmaf(kk, e.x, m[i].x); m[i].y = fmaf(kk, e.y, m[i].y);
            m[i].z = fmaf(kk, e.z, m[i].z); m[i].w = fmaf(kk, e.w, m[i].w);
        }
        if constexpr (kScatter) {
            const float sv = reduce_rows16(p, lane);
            const int r_ = rg * RPT + (lane >> 1);
            if ((lane & 1) == 0) dk[row * DK + r_] = xk[b][r_] - sv + c * to_f32(kb[b][r_]);
        } else {
#pragma unroll
            for (int i = 0; i < RPT; ++i) {
                const float sv = rsum(p[i]);
                const int r_ = rg * RPT + i;
                if (cg == 0) dk[row * DK + r_] = xk[b][r_] - sv + c * to_f32(kb[b][r_]);
            }
        }
        cp_async_wait_all();
        __syncthreads();
    }
}

}  // namespace efla
