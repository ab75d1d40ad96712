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
// One CTA of 256 threads per (b, h) keeps one d_k x d_v fp32 matrix in
// registers (the decode kernel's layout: thread (row group, column quad)
// holds RPT rows x 4 columns) and walks the sequence three times:
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

template <typename T, int DK, int DV>
__global__ void __launch_bounds__(256, 1)
    backward_kernel(const T *__restrict__ q, const T *__restrict__ k, const T *__restrict__ v,
                    const float *__restrict__ beta, const float *__restrict__ S0, const float *__restrict__ dO,
                    const float *__restrict__ dSL, float *__restrict__ dq, float *__restrict__ dk,
                    float *__restrict__ dv, float *__restrict__ dbeta, float *__restrict__ dS0,
                    float *__restrict__ E, float *__restrict__ Cg, int L, bool euler) {
    constexpr int CG = DV / 4;    // column quads
    constexpr int RG = 256 / CG;  // row groups
    constexpr int RPT = DK / RG;  // rows per thread
    static_assert(RPT >= 1 && RG * RPT == DK && (32 % CG) == 0, "state tile must cover d_k");
    __shared__ float ks[DK], qs[DK], xs[DK];
    __shared__ __align__(16) float vs[DV], ws[DV], es[DV];
    __shared__ __align__(16) float red[RG][DV];
    __shared__ float sc[4];

    const long bh = blockIdx.x;
    const int t = threadIdx.x, cg = t % CG, rg = t / CG;
    const size_t S_off = (size_t)bh * DK * DV;
    auto rsum = [&](float x) {  // sum over the CG threads holding one row
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
    // lambda and the gate of key row `row` (ks already in smem): warp 0
    auto gate = [&](size_t row) {
        if (t < 32) {
            float lam = 0.f;
            for (int i = t; i < DK; i += 32) lam = fmaf(ks[i], ks[i], lam);
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) lam += __shfl_xor_sync(0xffffffffu, lam, o);
            if (t == 0) {
                const float b = beta[row];
                float da_db, da_dl;
                gate_alpha_grad(b, lam, euler, da_db, da_dl);
                sc[0] = gate_alpha(b, lam, euler);
                sc[1] = da_db;
                sc[2] = da_dl;
            }
        }
    };
    float4 m[RPT];

    // ---------------------------------------------------------------- pass 1
    load_state(S0, m);
    for (int s = 0; s < L; ++s) {
        const size_t row = (size_t)bh * L + s;
        for (int i = t; i < DK; i += 256) ks[i] = to_f32(k[row * DK + i]);
        for (int j = t; j < DV; j += 256) {
            vs[j] = to_f32(v[row * DV + j]);
            ws[j] = dO[row * DV + j];
        }
        __syncthreads();
        gate(row);
        float4 r = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int i = 0; i < RPT; ++i) {
            const float kk = ks[rg * RPT + i];
            r.x = fmaf(m[i].x, kk, r.x); r.y = fmaf(m[i].y, kk, r.y);
            r.z = fmaf(m[i].z, kk, r.z); r.w = fmaf(m[i].w, kk, r.w);
        }
        *reinterpret_cast<float4 *>(&red[rg][4 * cg]) = r;
        __syncthreads();
        float4 rt = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int g = 0; g < RG; ++g) {
            const float4 x = *reinterpret_cast<const float4 *>(&red[g][4 * cg]);
            rt.x += x.x; rt.y += x.y; rt.z += x.z; rt.w += x.w;
        }
        const float a = sc[0];
        const float4 vv = *reinterpret_cast<const float4 *>(&vs[4 * cg]);
        const float4 e = make_float4(vv.x - rt.x, vv.y - rt.y, vv.z - rt.z, vv.w - rt.w);
        if (rg == 0) *(reinterpret_cast<float4 *>(E + row * DV) + cg) = e;
        const float4 dd = *reinterpret_cast<const float4 *>(&ws[4 * cg]);
#pragma unroll
        for (int i = 0; i < RPT; ++i) {
            const float kk = a * ks[rg * RPT + i];
            m[i].x = fmaf(kk, e.x, m[i].x); m[i].y = fmaf(kk, e.y, m[i].y);
            m[i].z = fmaf(kk, e.z, m[i].z); m[i].w = fmaf(kk, e.w, m[i].w);
            const float sd = rsum(m[i].x * dd.x + m[i].y * dd.y + m[i].z * dd.z + m[i].w * dd.w);
            if (cg == 0) dq[row * DK + rg * RPT + i] = sd;
        }
        __syncthreads();
    }

    // ---------------------------------------------------------------- pass 2
    load_state(dSL, m);
    for (int s = L - 1; s >= 0; --s) {
        const size_t row = (size_t)bh * L + s;
        for (int i = t; i < DK; i += 256) {
            ks[i] = to_f32(k[row * DK + i]);
            qs[i] = to_f32(q[row * DK + i]);
        }
        for (int j = t; j < DV; j += 256) {
            ws[j] = dO[row * DV + j];
            es[j] = E[row * DV + j];
        }
        __syncthreads();
        gate(row);
        const float4 dd = *reinterpret_cast<const float4 *>(&ws[4 * cg]);
        float4 g = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int i = 0; i < RPT; ++i) {
            const float qq = qs[rg * RPT + i], kk = ks[rg * RPT + i];
            m[i].x = fmaf(qq, dd.x, m[i].x); m[i].y = fmaf(qq, dd.y, m[i].y);
            m[i].z = fmaf(qq, dd.z, m[i].z); m[i].w = fmaf(qq, dd.w, m[i].w);
            g.x = fmaf(m[i].x, kk, g.x); g.y = fmaf(m[i].y, kk, g.y);
            g.z = fmaf(m[i].z, kk, g.z); g.w = fmaf(m[i].w, kk, g.w);
        }
        *reinterpret_cast<float4 *>(&red[rg][4 * cg]) = g;
        __syncthreads();
        float4 gt = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int gg = 0; gg < RG; ++gg) {
            const float4 x = *reinterpret_cast<const float4 *>(&red[gg][4 * cg]);
            gt.x += x.x; gt.y += x.y; gt.z += x.z; gt.w += x.w;
        }
        const float a = sc[0], da_db = sc[1], da_dl = sc[2];
        const float4 e = *reinterpret_cast<const float4 *>(&es[4 * cg]);
        const float dal = rsum(gt.x * e.x + gt.y * e.y + gt.z * e.z + gt.w * e.w);
        const float4 de = make_float4(a * gt.x, a * gt.y, a * gt.z, a * gt.w);
        if (rg == 0) *(reinterpret_cast<float4 *>(dv + row * DV) + cg) = de;
#pragma unroll
        for (int i = 0; i < RPT; ++i) {
            const float he = rsum(m[i].x * e.x + m[i].y * e.y + m[i].z * e.z + m[i].w * e.w);
            if (cg == 0) dk[row * DK + rg * RPT + i] = a * he;
            const float kk = ks[rg * RPT + i];
            m[i].x = fmaf(-kk, de.x, m[i].x); m[i].y = fmaf(-kk, de.y, m[i].y);
            m[i].z = fmaf(-kk, de.z, m[i].z); m[i].w = fmaf(-kk, de.w, m[i].w);
        }
        if (t == 0) {
            dbeta[row] = dal * da_db;
            Cg[row] = 2.f * dal * da_dl;
        }
        __syncthreads();
    }
#pragma unroll
    for (int i = 0; i < RPT; ++i)
        *(reinterpret_cast<float4 *>(dS0 + S_off + (size_t)(rg * RPT + i) * DV) + cg) = m[i];

    // ---------------------------------------------------------------- pass 3
    load_state(S0, m);
    for (int s = 0; s < L; ++s) {
        const size_t row = (size_t)bh * L + s;
        for (int i = t; i < DK; i += 256) {
            ks[i] = to_f32(k[row * DK + i]);
            xs[i] = dk[row * DK + i];
        }
        for (int j = t; j < DV; j += 256) {
            ws[j] = dv[row * DV + j];
            es[j] = E[row * DV + j];
        }
        if (t == 0) sc[3] = Cg[row];
        __syncthreads();
        gate(row);
        __syncthreads();
        const float a = sc[0], c = sc[3];
        const float4 de = *reinterpret_cast<const float4 *>(&ws[4 * cg]);
        const float4 e = *reinterpret_cast<const float4 *>(&es[4 * cg]);
#pragma unroll
        for (int i = 0; i < RPT; ++i) {
            const int r = rg * RPT + i;
            const float sde = rsum(m[i].x * de.x + m[i].y * de.y + m[i].z * de.z + m[i].w * de.w);
            if (cg == 0) dk[row * DK + r] = xs[r] - sde + c * ks[r];
            const float kk = a * ks[r];
            m[i].x = fmaf(kk, e.x, m[i].x); m[i].y = fmaf(kk, e.y, m[i].y);
            m[i].z = fmaf(kk, e.z, m[i].z); m[i].w = fmaf(kk, e.w, m[i].w);
        }
        __syncthreads();
    }
}

}  // namespace efla
