// efla_chunk_simt.cuh - exact-fp32 chunked prefill on the CUDA cores.
//
// This is the path for fp32 inputs (where bf16 or TF32 tensor-core operands
// would not meet a 1e-4 relative error bound) and for head sizes the
// tensor-core kernel does not take.  It evaluates the recurrence of "Exact
// Flow Linear Attention" (papernotes.org summary, 关键设计 2) chunk by
// chunk in the UT form of the chunk-parallel scheme that page cites
// (整体框架):
//
//   per chunk (rows t0..t0+n-1, C = 64, zero-padded past n):
//     alpha_r = gate(beta_r, ||k_r||^2)
//     A  = strictly-lower(diag(alpha) K K^T),   T = (I + A)^{-1}
//     T' = T diag(alpha);  W = T' K;  U = T' V;  M = lower-incl-diag(Q K^T)
//   then serially over chunks, per state column tile:
//     D = U - W S;   O = Q S + M D;   S <- S + K^T D
//
// Kernel 1 (chunk_prep_kernel) is independent per chunk and writes W, U, M
// to caller scratch; kernel 2 (chunk_state_kernel) walks the chunks of one
// (b,h) and one d_v tile with the fp32 state tile resident in shared memory.
#pragma once
#include "efla_common.cuh"

namespace efla {

constexpr int kChunk = 64;

// Scratch layout (fp32), per (bh, chunk g): W [C][D], U [C][D], M [C][C].
struct SimtScratch {
    float *W, *U, *M;
    __host__ __device__ static size_t floats(long n_chunks_total, int D) {
        return (size_t)n_chunks_total * (2 * (size_t)kChunk * D + (size_t)kChunk * kChunk);
    }
    __host__ __device__ static SimtScratch carve(float *base, long n_chunks_total, int D) {
        SimtScratch s;
        s.W = base;
        s.U = base + (size_t)n_chunks_total * kChunk * D;
        s.M = base + 2 * (size_t)n_chunks_total * kChunk * D;
        return s;
    }
};

template <int D>
struct PrepSmem {
    static constexpr int LD = D + 1;   // padded row stride of the C x D tiles
    static constexpr int LC = kChunk + 1;
    float K[kChunk * LD];
    float V[kChunk * LD];
    union {  // Q is dead once M = Q K^T is formed; A and T' come after it
        float Q[kChunk * LD];
        struct {
            float A[kChunk * LC];   // strictly-lower diag(alpha) K K^T
            float Tp[kChunk * LC];  // T' = (I + A)^{-1} diag(alpha)
        };
    };
    float alpha[kChunk];
};

template <typename Tin, int D>
__global__ void __launch_bounds__(256, 2) chunk_prep_kernel(const Tin *__restrict__ q, const Tin *__restrict__ k,
                                                            const Tin *__restrict__ v,
                                                            const float *__restrict__ beta, int L, int n_chunks,
                                                            SimtScratch ws, bool euler) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    PrepSmem<D> &sm = *reinterpret_cast<PrepSmem<D> *>(smem_raw);
    constexpr int LD = PrepSmem<D>::LD, LC = PrepSmem<D>::LC, C = kChunk;
    const int t = threadIdx.x;
    const unsigned q32 = blockIdx.x / (unsigned)n_chunks;  // 32-bit division: grid < 2^31
    const int chunk = (int)(blockIdx.x - q32 * (unsigned)n_chunks);
    const long bh = (long)q32;
    const int t0 = chunk * C;
    const int n = min(C, L - t0);
    const long row0 = bh * (long)L + t0;
    const long g = bh * n_chunks + chunk;

    // 1. load K, V, Q (widened to fp32), zero rows past n
    for (int e = t; e < C * (D / 4); e += 256) {
        const int r = e / (D / 4), c4 = (e % (D / 4)) * 4;
        float4 kk = make_float4(0.f, 0.f, 0.f, 0.f), vv = kk, qq = kk;
        if (r < n) {
            kk = load4(k + (row0 + r) * D + c4);
            vv = load4(v + (row0 + r) * D + c4);
            qq = load4(q + (row0 + r) * D + c4);
        }
        float *pk = &sm.K[r * LD + c4], *pv = &sm.V[r * LD + c4], *pq = &sm.Q[r * LD + c4];
        pk[0] = kk.x; pk[1] = kk.y; pk[2] = kk.z; pk[3] = kk.w;
        pv[0] = vv.x; pv[1] = vv.y; pv[2] = vv.z; pv[3] = vv.w;
        pq[0] = qq.x; pq[1] = qq.y; pq[2] = qq.z; pq[3] = qq.w;
    }
    __syncthreads();

    // 2. gate: 4 lanes per row
    {
        const int r = t >> 2, part = t & 3;
        float s = 0.f;
        for (int i = part; i < D; i += 4) s = fmaf(sm.K[r * LD + i], sm.K[r * LD + i], s);
        s += __shfl_xor_sync(0xffffffffu, s, 1);
        s += __shfl_xor_sync(0xffffffffu, s, 2);
        if (part == 0) sm.alpha[r] = (r < n) ? gate_alpha(beta[row0 + r], s, euler) : 0.f;
    }
    __syncthreads();

    // 3. A = strictly-lower(diag(alpha) K K^T); M = lower-incl-diag(Q K^T) -> scratch
    {
        const int tr = t >> 4, tc = t & 15;  // 4x4 register tile at rows 4tr.., cols 4tc..
        float g4[4][4] = {}, m4[4][4] = {};
        for (int i = 0; i < D; ++i) {
            float a[4], b[4], qa[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                a[u] = sm.K[(4 * tr + u) * LD + i];
                qa[u] = sm.Q[(4 * tr + u) * LD + i];
                b[u] = sm.K[(4 * tc + u) * LD + i];
            }
#pragma unroll
            for (int u = 0; u < 4; ++u)
#pragma unroll
                for (int w = 0; w < 4; ++w) {
                    g4[u][w] = fmaf(a[u], b[w], g4[u][w]);
                    m4[u][w] = fmaf(qa[u], b[w], m4[u][w]);
                }
        }
        float *Mg = ws.M + g * (size_t)C * C;
        __syncthreads();  // every thread has read Q: A may now overwrite it
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int r = 4 * tr + u;
            float4 mrow;
            float *mr = reinterpret_cast<float *>(&mrow);
#pragma unroll
            for (int w = 0; w < 4; ++w) {
                const int c = 4 * tc + w;
                sm.A[r * LC + c] = (c < r) ? sm.alpha[r] * g4[u][w] : 0.f;
                mr[w] = (c <= r) ? m4[u][w] : 0.f;
            }
            *reinterpret_cast<float4 *>(Mg + r * C + 4 * tc) = mrow;
        }
    }
    __syncthreads();

    // 4. T = (I + A)^{-1} by right-looking forward substitution: 4 adjacent
    //    lanes own one column c; lane part owns rows part + 4 s.  A is
    //    strictly lower, so updating every row with A[r][m] x_m is exact
    //    (A[r][m] = 0 for r <= m) and needs no branches.
    {
        const int c = t >> 2, part = t & 3, lane = t & 31;
        float acc[C / 4];
#pragma unroll
        for (int s = 0; s < C / 4; ++s) acc[s] = (part + 4 * s == c) ? 1.f : 0.f;
#pragma unroll
        for (int m = 0; m < C; ++m) {
            const float x = __shfl_sync(0xffffffffu, acc[m >> 2], (lane & ~3) | (m & 3));
#pragma unroll
            for (int s = 0; s < C / 4; ++s) acc[s] = fmaf(-sm.A[(part + 4 * s) * LC + m], x, acc[s]);
        }
        const float ac = sm.alpha[c];
#pragma unroll
        for (int s = 0; s < C / 4; ++s) sm.Tp[(part + 4 * s) * LC + c] = acc[s] * ac;
    }
    __syncthreads();

    // 5. W = T' K, U = T' V -> scratch.  Thread tile: 4 rows x (D/16) cols.
    {
        constexpr int CW = D / 16;
        const int tr = t >> 4, tc = t & 15;
        float w4[4][CW] = {}, u4[4][CW] = {};
        const int mmax = 4 * tr + 4;  // T' is lower triangular
        for (int m = 0; m < mmax; ++m) {
            float a[4];
#pragma unroll
            for (int uu = 0; uu < 4; ++uu) a[uu] = sm.Tp[(4 * tr + uu) * LC + m];
#pragma unroll
            for (int cc = 0; cc < CW; ++cc) {
                const float kk = sm.K[m * LD + tc + 16 * cc];
                const float vv = sm.V[m * LD + tc + 16 * cc];
#pragma unroll
                for (int uu = 0; uu < 4; ++uu) {
                    w4[uu][cc] = fmaf(a[uu], kk, w4[uu][cc]);
                    u4[uu][cc] = fmaf(a[uu], vv, u4[uu][cc]);
                }
            }
        }
        float *Wg = ws.W + g * (size_t)C * D, *Ug = ws.U + g * (size_t)C * D;
#pragma unroll
        for (int uu = 0; uu < 4; ++uu)
#pragma unroll
            for (int cc = 0; cc < CW; ++cc) {
                Wg[(4 * tr + uu) * D + tc + 16 * cc] = w4[uu][cc];
                Ug[(4 * tr + uu) * D + tc + 16 * cc] = u4[uu][cc];
            }
    }
}

template <int D>
struct StateSmem {
    static constexpr int DVT = 32;       // d_v columns per CTA
    static constexpr int LD = D + 1;
    static constexpr int LC = kChunk + 1;
    float W[kChunk * LD];
    float K[kChunk * LD];
    float Q[kChunk * LD];
    float M[kChunk * LC];
    __align__(16) float U[kChunk * DVT];
    __align__(16) float Dl[kChunk * DVT];
    __align__(16) float S[D * DVT];
};

// S0 and SL may be the same buffer (in-place state update), so neither is
// __restrict__.  That case is safe: each CTA reads and writes only its own
// d_v column slice of its own (b, h), and every read of S0 comes before the
// first __syncthreads of the chunk loop while SL is written after the last.
template <typename Tin, typename Tout, int D>
__global__ void __launch_bounds__(256, 1) chunk_state_kernel(const Tin *__restrict__ q, const Tin *__restrict__ k,
                                                             const float *S0, Tout *__restrict__ o,
                                                             float *SL, int L, int n_chunks,
                                                             SimtScratch ws) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    StateSmem<D> &sm = *reinterpret_cast<StateSmem<D> *>(smem_raw);
    constexpr int C = kChunk, DVT = StateSmem<D>::DVT, LD = StateSmem<D>::LD, LC = StateSmem<D>::LC;
    static_assert(D % DVT == 0, "d_v tile");
    const int t = threadIdx.x;
    const int j0 = (blockIdx.x % (D / DVT)) * DVT;
    const long bh = blockIdx.x / (D / DVT);

    // initial state tile
    for (int e = t; e < D * DVT; e += 256) {
        const int i = e / DVT, j = e % DVT;
        sm.S[e] = S0 ? S0[bh * (long)D * D + (long)i * D + j0 + j] : 0.f;
    }

    // The tiles of chunk n+1 (W, K, Q, this CTA's U columns, M) are loaded
    // into registers while chunk n computes, and moved to shared memory at the
    // top of the next iteration, so no chunk waits on a global-memory round trip.
    constexpr int NQ = C * (D / 4) / 256;   // float4s of a C x D tile per thread
    constexpr int NU = C * (DVT / 4) / 256;  // float4s of the C x DVT U tile per thread
    constexpr int NM = C * C / 256;          // floats of the C x C M tile per thread
    static_assert(NQ * 256 == C * (D / 4) && NU * 256 == C * (DVT / 4) && NM * 256 == C * C, "tile split");
    float4 rw[NQ], rk[NQ], rq[NQ], ru[NU];
    float rm[NM];
    auto fetch = [&](int chunk) {
        const int n = min(C, L - chunk * C);
        const long row0 = bh * (long)L + chunk * C;
        const long g = bh * n_chunks + chunk;
        const float *Wg = ws.W + g * (size_t)C * D;
        const float *Ug = ws.U + g * (size_t)C * D;
        const float *Mg = ws.M + g * (size_t)C * C;
#pragma unroll
        for (int x = 0; x < NQ; ++x) {
            const int e = t + 256 * x, r = e / (D / 4), c4 = (e % (D / 4)) * 4;
            rw[x] = *reinterpret_cast<const float4 *>(Wg + r * D + c4);
            rk[x] = rq[x] = make_float4(0.f, 0.f, 0.f, 0.f);
            if (r < n) {
                rk[x] = load4(k + (row0 + r) * D + c4);
                rq[x] = load4(q + (row0 + r) * D + c4);
            }
        }
#pragma unroll
        for (int x = 0; x < NU; ++x) {
            const int e = t + 256 * x, r = e / (DVT / 4), c4 = (e % (DVT / 4)) * 4;
            ru[x] = *reinterpret_cast<const float4 *>(Ug + r * D + j0 + c4);
        }
#pragma unroll
        for (int x = 0; x < NM; ++x) rm[x] = Mg[t + 256 * x];
    };
    auto stash = [&]() {
#pragma unroll
        for (int x = 0; x < NQ; ++x) {
            const int e = t + 256 * x, r = e / (D / 4), c4 = (e % (D / 4)) * 4;
            float *pw = &sm.W[r * LD + c4], *pk = &sm.K[r * LD + c4], *pq = &sm.Q[r * LD + c4];
            pw[0] = rw[x].x; pw[1] = rw[x].y; pw[2] = rw[x].z; pw[3] = rw[x].w;
            pk[0] = rk[x].x; pk[1] = rk[x].y; pk[2] = rk[x].z; pk[3] = rk[x].w;
            pq[0] = rq[x].x; pq[1] = rq[x].y; pq[2] = rq[x].z; pq[3] = rq[x].w;
        }
#pragma unroll
        for (int x = 0; x < NU; ++x) {
            const int e = t + 256 * x, r = e / (DVT / 4), c4 = (e % (DVT / 4)) * 4;
            *reinterpret_cast<float4 *>(&sm.U[r * DVT + c4]) = ru[x];
        }
#pragma unroll
        for (int x = 0; x < NM; ++x) {
            const int e = t + 256 * x;
            sm.M[(e / C) * LC + (e % C)] = rm[x];
        }
    };
    if (n_chunks > 0) fetch(0);

    for (int chunk = 0; chunk < n_chunks; ++chunk) {
        const int t0 = chunk * C;
        const int n = min(C, L - t0);
        const long row0 = bh * (long)L + t0;
        __syncthreads();  // previous chunk's readers are done with the tiles
        stash();
        if (chunk + 1 < n_chunks) fetch(chunk + 1);
        __syncthreads();

        // D = U - W S and O = Q S: thread owns rows {2 rp, 2 rp + 1}, cols 4 cq..
        const int rp = t >> 3, cq = t & 7;
        const int r0 = 2 * rp, r1 = r0 + 1;
        float d0[4] = {}, d1[4] = {}, o0[4] = {}, o1[4] = {};
        for (int i = 0; i < D; ++i) {
            const float4 s4 = *reinterpret_cast<const float4 *>(&sm.S[i * DVT + 4 * cq]);
            const float w0 = sm.W[r0 * LD + i], w1 = sm.W[r1 * LD + i];
            const float q0 = sm.Q[r0 * LD + i], q1 = sm.Q[r1 * LD + i];
            const float sv[4] = {s4.x, s4.y, s4.z, s4.w};
#pragma unroll
            for (int w = 0; w < 4; ++w) {
                d0[w] = fmaf(w0, sv[w], d0[w]);
                d1[w] = fmaf(w1, sv[w], d1[w]);
                o0[w] = fmaf(q0, sv[w], o0[w]);
                o1[w] = fmaf(q1, sv[w], o1[w]);
            }
        }
#pragma unroll
        for (int w = 0; w < 4; ++w) {
            sm.Dl[r0 * DVT + 4 * cq + w] = sm.U[r0 * DVT + 4 * cq + w] - d0[w];
            sm.Dl[r1 * DVT + 4 * cq + w] = sm.U[r1 * DVT + 4 * cq + w] - d1[w];
        }
        __syncthreads();

        // O += M D (M lower incl. diagonal), write rows < n
        for (int m = 0; m <= r1; ++m) {
            const float4 dm = *reinterpret_cast<const float4 *>(&sm.Dl[m * DVT + 4 * cq]);
            const float dv[4] = {dm.x, dm.y, dm.z, dm.w};
            const float ma = sm.M[r0 * LC + m], mb = sm.M[r1 * LC + m];
#pragma unroll
            for (int w = 0; w < 4; ++w) {
                o0[w] = fmaf(ma, dv[w], o0[w]);
                o1[w] = fmaf(mb, dv[w], o1[w]);
            }
        }
        if (r0 < n) store4(o + (row0 + r0) * D + j0 + 4 * cq, make_float4(o0[0], o0[1], o0[2], o0[3]));
        if (r1 < n) store4(o + (row0 + r1) * D + j0 + 4 * cq, make_float4(o1[0], o1[1], o1[2], o1[3]));

        // S += K^T D: thread owns rows 4 iq.. (d_k) x cols 4 jq.. (tile)
        for (int tile = t; tile < (D / 4) * (DVT / 4); tile += 256) {
            const int iq = tile / (DVT / 4), jq = tile % (DVT / 4);
            float acc[4][4] = {};
            for (int m = 0; m < C; ++m) {
                const float4 dm = *reinterpret_cast<const float4 *>(&sm.Dl[m * DVT + 4 * jq]);
                const float dv[4] = {dm.x, dm.y, dm.z, dm.w};
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const float kk = sm.K[m * LD + 4 * iq + u];
#pragma unroll
                    for (int w = 0; w < 4; ++w) acc[u][w] = fmaf(kk, dv[w], acc[u][w]);
                }
            }
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                float4 *sp = reinterpret_cast<float4 *>(&sm.S[(4 * iq + u) * DVT + 4 * jq]);
                float4 x = *sp;
                x.x += acc[u][0]; x.y += acc[u][1]; x.z += acc[u][2]; x.w += acc[u][3];
                *sp = x;
            }
        }
    }
    __syncthreads();
    if (SL)
        for (int e = t; e < D * DVT; e += 256) {
            const int i = e / DVT, j = e % DVT;
            SL[bh * (long)D * D + (long)i * D + j0 + j] = sm.S[e];
        }
}

}  // namespace efla
