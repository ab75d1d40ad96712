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
    // Row strides of 16-byte multiples (one 16-byte load reads four
    // consecutive elements of a row) that are not multiples of 32 words
    // (rows read together fall in different banks).
    static constexpr int LD = D + 4;
    static constexpr int LC = kChunk + 4;
    __align__(16) float K[kChunk * LD];
    __align__(16) float V[kChunk * LD];
    union {  // Q is dead once M = Q K^T is formed; A and T' come after it
        __align__(16) float Q[kChunk * LD];
        struct {
            __align__(16) float A[kChunk * LC];   // strictly-lower diag(alpha) K K^T
            __align__(16) float Tp[kChunk * LC];  // T' = (I + A)^{-1} diag(alpha)
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
        *reinterpret_cast<float4 *>(&sm.K[r * LD + c4]) = kk;
        *reinterpret_cast<float4 *>(&sm.V[r * LD + c4]) = vv;
        *reinterpret_cast<float4 *>(&sm.Q[r * LD + c4]) = qq;
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

    // 3. A = strictly-lower(diag(alpha) K K^T); M = lower-incl-diag(Q K^T) -> scratch.
    //    Thread: rows 4 tr + u, columns tc + 16 w (u, w < 4); four d_k indices
    //    per step, each row segment read by one 16-byte load.
    {
        const int tr = t >> 4, tc = t & 15;
        float g4[4][4] = {}, m4[4][4] = {};
#pragma unroll 2
        for (int i = 0; i < D; i += 4) {
            float4 a[4], qa[4], b[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                a[u] = *reinterpret_cast<const float4 *>(&sm.K[(4 * tr + u) * LD + i]);
                qa[u] = *reinterpret_cast<const float4 *>(&sm.Q[(4 * tr + u) * LD + i]);
                b[u] = *reinterpret_cast<const float4 *>(&sm.K[(tc + 16 * u) * LD + i]);
            }
#pragma unroll
            for (int u = 0; u < 4; ++u)
#pragma unroll
                for (int w = 0; w < 4; ++w) {
                    g4[u][w] = fmaf(a[u].x, b[w].x, fmaf(a[u].y, b[w].y, fmaf(a[u].z, b[w].z, fmaf(a[u].w, b[w].w, g4[u][w]))));
                    m4[u][w] = fmaf(qa[u].x, b[w].x, fmaf(qa[u].y, b[w].y, fmaf(qa[u].z, b[w].z, fmaf(qa[u].w, b[w].w, m4[u][w]))));
                }
        }
        float *Mg = ws.M + g * (size_t)C * C;
        __syncthreads();  // every thread has read Q: A may now overwrite it
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int r = 4 * tr + u;
#pragma unroll
            for (int w = 0; w < 4; ++w) {
                const int c = tc + 16 * w;
                sm.A[r * LC + c] = (c < r) ? sm.alpha[r] * g4[u][w] : 0.f;
                Mg[r * C + c] = (c <= r) ? m4[u][w] : 0.f;
            }
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

    // 5. W = T' K, U = T' V -> scratch.  Thread: rows 4 tr .., columns in
    //    groups of CW contiguous (CW = 4, or 2 at d = 32): group g starts at
    //    16 CW g + CW tc, so the 16 threads of a row read one contiguous
    //    segment.  Four chunk rows m per step (T' row segments by 16-byte
    //    loads); T' is lower triangular: m < 4 tr + 4.
    {
        constexpr int CW = D >= 64 ? 4 : 2, NG = D / (16 * CW), NCW = CW * NG;
        const int tr = t >> 4, tc = t & 15;
        float w4[4][NCW] = {}, u4[4][NCW] = {};
        auto col = [&](int c) { return 16 * CW * (c / CW) + CW * tc + (c % CW); };
        const int mmax = 4 * tr + 4;
        for (int m = 0; m < mmax; m += 4) {
            float4 a[4];
#pragma unroll
            for (int uu = 0; uu < 4; ++uu) a[uu] = *reinterpret_cast<const float4 *>(&sm.Tp[(4 * tr + uu) * LC + m]);
#pragma unroll
            for (int v4 = 0; v4 < 4; ++v4) {
                float kk[NCW], vv[NCW];
#pragma unroll
                for (int gg = 0; gg < NG; ++gg) {
                    const float *kr = &sm.K[(m + v4) * LD + col(CW * gg)];
                    const float *vr = &sm.V[(m + v4) * LD + col(CW * gg)];
                    if constexpr (CW == 4) {
                        const float4 k4 = *reinterpret_cast<const float4 *>(kr), v4v = *reinterpret_cast<const float4 *>(vr);
                        kk[4 * gg] = k4.x, kk[4 * gg + 1] = k4.y, kk[4 * gg + 2] = k4.z, kk[4 * gg + 3] = k4.w;
                        vv[4 * gg] = v4v.x, vv[4 * gg + 1] = v4v.y, vv[4 * gg + 2] = v4v.z, vv[4 * gg + 3] = v4v.w;
                    } else {
                        const float2 k2 = *reinterpret_cast<const float2 *>(kr), v2 = *reinterpret_cast<const float2 *>(vr);
                        kk[2 * gg] = k2.x, kk[2 * gg + 1] = k2.y, vv[2 * gg] = v2.x, vv[2 * gg + 1] = v2.y;
                    }
                }
#pragma unroll
                for (int uu = 0; uu < 4; ++uu) {
                    const float av = v4 == 0 ? a[uu].x : v4 == 1 ? a[uu].y : v4 == 2 ? a[uu].z : a[uu].w;
#pragma unroll
                    for (int c = 0; c < NCW; ++c) {
                        w4[uu][c] = fmaf(av, kk[c], w4[uu][c]);
                        u4[uu][c] = fmaf(av, vv[c], u4[uu][c]);
                    }
                }
            }
        }
        float *Wg = ws.W + g * (size_t)C * D, *Ug = ws.U + g * (size_t)C * D;
#pragma unroll
        for (int uu = 0; uu < 4; ++uu)
#pragma unroll
            for (int c = 0; c < NCW; ++c) {
                Wg[(4 * tr + uu) * D + col(c)] = w4[uu][c];
                Ug[(4 * tr + uu) * D + col(c)] = u4[uu][c];
            }
    }
}

template <int D>
struct StateSmem {
    static constexpr int DVT = 32;       // d_v columns per CTA
    // Row strides of 16-byte multiples, so a thread reads four consecutive
    // elements of a row with one 16-byte load, and not a multiple of 32
    // words, so the rows a warp reads at once fall in different banks.
    static constexpr int LD = D + 4;
    static constexpr int LC = kChunk + 4;
    __align__(16) float W[kChunk * LD];
    __align__(16) float K[kChunk * LD];
    __align__(16) float Q[kChunk * LD];
    __align__(16) float M[kChunk * LC];
    __align__(16) float U[kChunk * DVT];
    __align__(16) float Dl[kChunk * DVT];
    __align__(16) float S[D * DVT];
};

__device__ __forceinline__ void fma4(float (&acc)[4], float a, const float4 &b) {
    acc[0] = fmaf(a, b.x, acc[0]);
    acc[1] = fmaf(a, b.y, acc[1]);
    acc[2] = fmaf(a, b.z, acc[2]);
    acc[3] = fmaf(a, b.w, acc[3]);
}

// S0 and SL may be the same buffer (in-place state update), so neither is
// __restrict__.  That case is safe: each CTA reads and writes only its own
// d_v column slice of its own (b, h), and every read of S0 comes before the
// first __syncthreads of the chunk loop while SL is written after the last.
//
// Per chunk, with every contraction vectorised four elements at a time (one
// 16-byte load of a row segment feeds 16 FMAs):
//   D = U - W S,  O = Q S   thread: rows 2 rp, 2 rp + 1; columns 4 cq ..
//   O += M D                (M lower triangular: m up to the thread's rows)
//   S += K^T D              thread: d_k rows 4 iq ..; columns 4 jq ..
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
    // into registers while chunk n computes its last two products, and moved
    // to shared memory at the top of the next iteration, so no chunk waits on
    // a global-memory round trip.
    constexpr int NQ = C * (D / 4) / 256;   // float4s of a C x D tile per thread
    constexpr int NU = C * (DVT / 4) / 256;  // float4s of the C x DVT U tile per thread
    constexpr int NM = C * (C / 4) / 256;    // float4s of the C x C M tile per thread
    static_assert(NQ * 256 == C * (D / 4) && NU * 256 == C * (DVT / 4) && NM * 256 == C * (C / 4), "tile split");
    float4 rw[NQ], rk[NQ], rq[NQ], ru[NU], rm[NM];
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
        for (int x = 0; x < NM; ++x) {
            const int e = t + 256 * x, r = e / (C / 4), c4 = (e % (C / 4)) * 4;
            rm[x] = *reinterpret_cast<const float4 *>(Mg + r * C + c4);
        }
    };
    auto stash = [&]() {
#pragma unroll
        for (int x = 0; x < NQ; ++x) {
            const int e = t + 256 * x, r = e / (D / 4), c4 = (e % (D / 4)) * 4;
            *reinterpret_cast<float4 *>(&sm.W[r * LD + c4]) = rw[x];
            *reinterpret_cast<float4 *>(&sm.K[r * LD + c4]) = rk[x];
            *reinterpret_cast<float4 *>(&sm.Q[r * LD + c4]) = rq[x];
        }
#pragma unroll
        for (int x = 0; x < NU; ++x) {
            const int e = t + 256 * x, r = e / (DVT / 4), c4 = (e % (DVT / 4)) * 4;
            *reinterpret_cast<float4 *>(&sm.U[r * DVT + c4]) = ru[x];
        }
#pragma unroll
        for (int x = 0; x < NM; ++x) {
            const int e = t + 256 * x, r = e / (C / 4), c4 = (e % (C / 4)) * 4;
            *reinterpret_cast<float4 *>(&sm.M[r * LC + c4]) = rm[x];
        }
    };
    if (n_chunks > 0) fetch(0);

    const int rp = t >> 3, cq = t & 7;
    const int r0 = 2 * rp, r1 = r0 + 1;
    for (int chunk = 0; chunk < n_chunks; ++chunk) {
        const int t0 = chunk * C;
        const int n = min(C, L - t0);
        const long row0 = bh * (long)L + t0;
        __syncthreads();  // previous chunk's readers are done with the tiles
        stash();
        __syncthreads();

        // D = U - W S and O = Q S, four d_k indices per step
        float d0[4] = {}, d1[4] = {}, o0[4] = {}, o1[4] = {};
#pragma unroll 2
        for (int i = 0; i < D; i += 4) {
            const float4 w0 = *reinterpret_cast<const float4 *>(&sm.W[r0 * LD + i]);
            const float4 w1 = *reinterpret_cast<const float4 *>(&sm.W[r1 * LD + i]);
            const float4 q0 = *reinterpret_cast<const float4 *>(&sm.Q[r0 * LD + i]);
            const float4 q1 = *reinterpret_cast<const float4 *>(&sm.Q[r1 * LD + i]);
            const float4 s0 = *reinterpret_cast<const float4 *>(&sm.S[(i + 0) * DVT + 4 * cq]);
            const float4 s1 = *reinterpret_cast<const float4 *>(&sm.S[(i + 1) * DVT + 4 * cq]);
            const float4 s2 = *reinterpret_cast<const float4 *>(&sm.S[(i + 2) * DVT + 4 * cq]);
            const float4 s3 = *reinterpret_cast<const float4 *>(&sm.S[(i + 3) * DVT + 4 * cq]);
            fma4(d0, w0.x, s0); fma4(d0, w0.y, s1); fma4(d0, w0.z, s2); fma4(d0, w0.w, s3);
            fma4(d1, w1.x, s0); fma4(d1, w1.y, s1); fma4(d1, w1.z, s2); fma4(d1, w1.w, s3);
            fma4(o0, q0.x, s0); fma4(o0, q0.y, s1); fma4(o0, q0.z, s2); fma4(o0, q0.w, s3);
            fma4(o1, q1.x, s0); fma4(o1, q1.y, s1); fma4(o1, q1.z, s2); fma4(o1, q1.w, s3);
        }
        // the next chunk's tiles: issued here, so the registers they occupy are
        // free during the contraction above and the loads land during O += M D
        // and S += K^T D
        if (chunk + 1 < n_chunks) fetch(chunk + 1);
        {
            const float4 u0 = *reinterpret_cast<const float4 *>(&sm.U[r0 * DVT + 4 * cq]);
            const float4 u1 = *reinterpret_cast<const float4 *>(&sm.U[r1 * DVT + 4 * cq]);
            *reinterpret_cast<float4 *>(&sm.Dl[r0 * DVT + 4 * cq]) =
                make_float4(u0.x - d0[0], u0.y - d0[1], u0.z - d0[2], u0.w - d0[3]);
            *reinterpret_cast<float4 *>(&sm.Dl[r1 * DVT + 4 * cq]) =
                make_float4(u1.x - d1[0], u1.y - d1[1], u1.z - d1[2], u1.w - d1[3]);
        }
        __syncthreads();

        // O += M D (M lower incl. diagonal, zero above it), write rows < n
        for (int m = 0; m <= r1; m += 4) {
            const float4 ma = *reinterpret_cast<const float4 *>(&sm.M[r0 * LC + m]);
            const float4 mb = *reinterpret_cast<const float4 *>(&sm.M[r1 * LC + m]);
            const float4 e0 = *reinterpret_cast<const float4 *>(&sm.Dl[(m + 0) * DVT + 4 * cq]);
            const float4 e1 = *reinterpret_cast<const float4 *>(&sm.Dl[(m + 1) * DVT + 4 * cq]);
            const float4 e2 = *reinterpret_cast<const float4 *>(&sm.Dl[(m + 2) * DVT + 4 * cq]);
            const float4 e3 = *reinterpret_cast<const float4 *>(&sm.Dl[(m + 3) * DVT + 4 * cq]);
            fma4(o0, ma.x, e0); fma4(o0, ma.y, e1); fma4(o0, ma.z, e2); fma4(o0, ma.w, e3);
            fma4(o1, mb.x, e0); fma4(o1, mb.y, e1); fma4(o1, mb.z, e2); fma4(o1, mb.w, e3);
        }
        if (r0 < n) store4(o + (row0 + r0) * D + j0 + 4 * cq, make_float4(o0[0], o0[1], o0[2], o0[3]));
        if (r1 < n) store4(o + (row0 + r1) * D + j0 + 4 * cq, make_float4(o1[0], o1[1], o1[2], o1[3]));

        // S += K^T D: thread owns d_k rows 4 iq .. x columns 4 jq .. of the tile
        for (int tile = t; tile < (D / 4) * (DVT / 4); tile += 256) {
            const int iq = tile / (DVT / 4), jq = tile % (DVT / 4);
            float acc[4][4] = {};
#pragma unroll 4
            for (int m = 0; m < C; ++m) {
                const float4 km = *reinterpret_cast<const float4 *>(&sm.K[m * LD + 4 * iq]);
                const float4 dm = *reinterpret_cast<const float4 *>(&sm.Dl[m * DVT + 4 * jq]);
                fma4(acc[0], km.x, dm);
                fma4(acc[1], km.y, dm);
                fma4(acc[2], km.z, dm);
                fma4(acc[3], km.w, dm);
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
