// efla_decode.cuh - one-token recurrent update of B*H fp32 states.
//
// Per (b,h) ("Exact Flow Linear Attention", papernotes.org summary,
// 关键设计 2 and the 整体框架 flowchart; sequential O(L d^2) decode of 整体框架):
//   lambda = k.k,  alpha = gate(beta, lambda)
//   r = S^T k,  p = S^T q                    (column reductions of the old S)
//   S <- S + alpha k (v - r)^T               (= (I - alpha k k^T) S + alpha k v^T)
//   o  = p + alpha (q.k) (v - r)             (= S_new^T q)
//
// HBM-bound: the d_k x d_v fp32 state is read once and written once
// (8 d^2 bytes per head-step).  One CTA of 256 threads per (b,h): thread
// (row group rg, column quad cg) holds RPT rows x 4 columns of S in
// registers, so the whole state is in flight after the first loads; the
// column reductions go through shared memory across row groups and the two
// dot products k.k and q.k are warp-shuffle reductions.
#pragma once
#include "efla_common.cuh"

namespace efla {

template <typename T, typename To, int DK, int DV>
__global__ void __launch_bounds__(256, 2) decode_kernel(const T *__restrict__ q, const T *__restrict__ k,
                                                        const T *__restrict__ v, const float *__restrict__ beta,
                                                        float *__restrict__ S, To *__restrict__ o, bool euler) {
    constexpr int CG = DV / 4;     // column quads
    constexpr int RG = 256 / CG;   // row groups
    constexpr int RPT = DK / RG;   // rows per thread
    static_assert(RPT >= 1 && RG * RPT == DK, "state tile must cover d_k");
    __shared__ float ks[DK], qs[DK];
    __shared__ __align__(16) float vs[DV];
    __shared__ __align__(16) float red_r[RG][DV];
    __shared__ __align__(16) float red_p[RG][DV];
    __shared__ float sc[2];

    const long bh = blockIdx.x;
    const int t = threadIdx.x;
    const int cg = t % CG, rg = t / CG;
    float *Sb = S + bh * (long)DK * DV;

    float4 s[RPT];
#pragma unroll
    for (int i = 0; i < RPT; ++i) s[i] = __ldcs(reinterpret_cast<const float4 *>(Sb + (long)(rg * RPT + i) * DV) + cg);

    for (int i = t; i < DK; i += 256) {
        ks[i] = to_f32(k[bh * DK + i]);
        qs[i] = to_f32(q[bh * DK + i]);
    }
    for (int j = t; j < DV; j += 256) vs[j] = to_f32(v[bh * DV + j]);
    __syncthreads();

    if (t < 32) {
        float lam = 0.f, qk = 0.f;
        for (int i = t; i < DK; i += 32) {
            lam = fmaf(ks[i], ks[i], lam);
            qk = fmaf(qs[i], ks[i], qk);
        }
        lam = warp_sum(lam);
        qk = warp_sum(qk);
        if (t == 0) {
            sc[0] = gate_alpha(beta[bh], lam, euler);
            sc[1] = qk;
        }
    }
    float4 r = make_float4(0.f, 0.f, 0.f, 0.f), p = r;
#pragma unroll
    for (int i = 0; i < RPT; ++i) {
        const float kk = ks[rg * RPT + i], qq = qs[rg * RPT + i];
        r.x = fmaf(s[i].x, kk, r.x); r.y = fmaf(s[i].y, kk, r.y);
        r.z = fmaf(s[i].z, kk, r.z); r.w = fmaf(s[i].w, kk, r.w);
        p.x = fmaf(s[i].x, qq, p.x); p.y = fmaf(s[i].y, qq, p.y);
        p.z = fmaf(s[i].z, qq, p.z); p.w = fmaf(s[i].w, qq, p.w);
    }
    *reinterpret_cast<float4 *>(&red_r[rg][4 * cg]) = r;
    *reinterpret_cast<float4 *>(&red_p[rg][4 * cg]) = p;
    __syncthreads();

    float4 rt = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int g = 0; g < RG; ++g) {
        const float4 x = *reinterpret_cast<const float4 *>(&red_r[g][4 * cg]);
        rt.x += x.x; rt.y += x.y; rt.z += x.z; rt.w += x.w;
    }
    const float a = sc[0];
    const float4 vv = *reinterpret_cast<const float4 *>(&vs[4 * cg]);
    // e_j = alpha (v_j - r_j): the rank-1 write direction
    const float4 e = make_float4(a * (vv.x - rt.x), a * (vv.y - rt.y), a * (vv.z - rt.z), a * (vv.w - rt.w));
#pragma unroll
    for (int i = 0; i < RPT; ++i) {
        const float kk = ks[rg * RPT + i];
        float4 x = s[i];
        x.x = fmaf(kk, e.x, x.x); x.y = fmaf(kk, e.y, x.y);
        x.z = fmaf(kk, e.z, x.z); x.w = fmaf(kk, e.w, x.w);
        __stcs(reinterpret_cast<float4 *>(Sb + (long)(rg * RPT + i) * DV) + cg, x);
    }
    if (rg == 0) {
        float4 pt = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int g = 0; g < RG; ++g) {
            const float4 x = *reinterpret_cast<const float4 *>(&red_p[g][4 * cg]);
            pt.x += x.x; pt.y += x.y; pt.z += x.z; pt.w += x.w;
        }
        const float qk = sc[1];
        const float4 out = make_float4(fmaf(qk, e.x, pt.x), fmaf(qk, e.y, pt.y), fmaf(qk, e.z, pt.z),
                                       fmaf(qk, e.w, pt.w));
        store4(o + bh * DV + 4 * cg, out);
    }
}

}  // namespace efla
