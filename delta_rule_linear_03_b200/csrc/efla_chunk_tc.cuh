// efla_chunk_tc.cuh - fused chunked prefill on the 5th-generation tensor
// cores (tcgen05 + TMEM + TMA) for bf16 q/k/v, d_k = d_v = 128.
//
// Computes the recurrence of "Exact Flow Linear Attention" (papernotes.org
// summary of arXiv 2512.12602, 关键设计 2; readout of the 整体框架
// flowchart) chunk by chunk in the UT form of the chunk-parallel scheme that
// page cites (整体框架, "WY / UT"), with C = 64:
//
//   kernel chunk_T_kernel, one CTA per chunk, all chunks in parallel:
//   alpha = gate(beta, ||k||^2)                       (fp32, CUDA cores)
//   A  = strictly-lower(diag(alpha) K K^T)            (mma.sync bf16, fp32 acc.)
//   T  = (I + A)^{-1}                                 (CUDA cores + mma.sync TF32)
//   X  = [0; T diag(alpha)]                           (bf16 hi + lo, to scratch)
//   kernel chunk_tc_kernel, serial over the chunks of one (b, h, d_v half):
//   G  = [K; Q] K^T                                   (tcgen05, M=128 N=64 K=128)
//   [. ; W] = X K,   [0; U] = X V_tile                (tcgen05, N=128 and N=64)
//   Y += [Q; -W] S  ->  [Q S; U - W S] = [Q S; D]     (tcgen05, N=64 K=128)
//   S += K^T D                                        (tcgen05, N=64 K=64)
//   Y += [M; *] D   ->  O = Q S + M D,  M = lower-incl-diag(Q K^T)
//
// Every product is stacked to M = 128 rows so the accumulator of each
// tcgen05.mma occupies all 128 TMEM lanes, one row per lane.  (In the last
// product the lower 64 rows of the A operand are whatever follows M in shared
// memory: they only add into the D rows of Y, which are dead by then.)
//
// Precision: q, k, v are exact bf16 operands.  T diag(alpha), S, D and M are
// fp32 values fed to the bf16 tensor cores as a hi + lo pair of bf16
// (x = hi + lo to ~16 significant bits); only -W goes in as a single bf16.
// Accumulation is fp32 in TMEM and the state is kept in fp32.
//
// Everything S-independent and per-chunk that is not a tensor-core product
// (the gate and T) runs in the first kernel, so the serial kernel only moves
// T' in and keeps its tensor pipe and state chain busy.
// One CTA per (b, h, half of d_v): the 128 x 64 fp32 state tile lives in
// TMEM for the whole sequence.  Warp roles:
//   warps 0-1  "io":    T' image in (chunk n+1), O of chunk n-1 out to HBM
//   warps 2-3  "mw":    M and -W for chunk n+1 (S-independent)
//   warps 4-7  "state": D -> bf16 and S -> bf16 for chunk n (the serial chain)
//   warp 8     one thread issues every tcgen05.mma and commit
//   warp 9     one thread issues the TMA loads (2-stage K/Q/V ring)
// Every mbarrier wait is bounded; a wait that gives up sets the sticky
// device error word and an abort flag, every role then leaves its loop, the
// MMA thread drains its outstanding MMAs and the TMA thread its copies, and
// the CTA frees its TMEM before returning.
#pragma once
#include <cuda.h>

#include <mutex>

#include "../../include/efla.h"
#include "efla_common.cuh"
#include "efla_tc_ptx.cuh"

namespace efla {
namespace tc {

constexpr int C = 64, DK = 128, DVT = 64, NSPLIT = 2;
constexpr int kThreads = 320;
constexpr uint32_t SLOT = 8192;                 // one 64 x 64 bf16 swizzled box
constexpr uint32_t STAGE = 7 * SLOT;            // K0 Q0 W0 K1 Q1 W1 V
constexpr uint32_t SL_K0 = 0, SL_Q0 = 1, SL_W0 = 2, SL_V = 6;
constexpr uint32_t BOXSTRIDE = 3 * SLOT;        // K0->K1, Q0->Q1, W0->W1
constexpr int LDF = 64;                         // fp32 row stride of A and T
constexpr uint32_t OFF_M = 2 * STAGE;           // M hi/lo for chunk parity 0 and 1: 4 boxes
constexpr uint32_t OFF_Z0 = OFF_M + 4 * SLOT;   // zero box, then T' hi  ([0; T'hi] operand)
constexpr uint32_t OFF_THI = OFF_Z0 + SLOT;
constexpr uint32_t OFF_Z1 = OFF_THI + SLOT;     // zero box, then T' lo  ([0; T'lo] operand)
constexpr uint32_t OFF_TLO = OFF_Z1 + SLOT;
constexpr uint32_t OFF_SB = OFF_TLO + SLOT;     // S tile bf16 hi, then lo (MN-major B), 128 x 64 each
constexpr uint32_t OFF_DB = OFF_SB + 4 * SLOT;  // D bf16 hi, then lo (MN-major B), 64 x 64 each
constexpr uint32_t OFF_BAR = OFF_DB + 2 * SLOT;
constexpr uint32_t XBYTES = 2 * SLOT;           // T' hi and lo boxes of one chunk (workspace image)
constexpr uint32_t NBAR = 20;  // indices 0..19
constexpr uint32_t OFF_MISC = OFF_BAR + NBAR * 8;
constexpr uint32_t SMEM_BYTES = OFF_MISC + 16 + 1024;  // + slack to align the base to 1024 B
static_assert(SMEM_BYTES <= 232448, "shared memory per CTA");

// TMEM columns (fp32, 128 lanes)
// X K accumulates into two alternating buffers (YW, by chunk parity) so
// Y(n+1) can run while the -W readout of chunk n is still pending.
constexpr uint32_t T_S = 0, T_G = 64, T_YW = 128, T_YU = 384, TMEM_COLS = 512;

enum : int {
    B_FULL = 0,     // [2] TMA stage landed
    B_EMPTY = 2,    // [2] stage free again (commit after the last MMA reading it)
    B_GFULL = 4,    // G ready in TMEM
    B_GEMPTY = 5,   // G read out
    B_XFULL = 6,    // T' image of the next chunk in place
    B_YFULL = 7,    // [2] X K and X V of a chunk done (per X K buffer)
    B_A2FULL = 9,   // [2] -W and M written for chunk parity b
    B_SBFULL = 11,  // bf16 S tile written
    B_DFULL = 12,   // Y += [Q;-W] S done
    B_DELTA = 13,   // bf16 D written
    B_SFULL = 14,   // S += K^T D done
    B_DRAIN = 15,   // final drain of the MMA pipe
    B_OREAD = 16,   // [2] O of a chunk read out of Y buffer b
    B_OFULL = 18,   // [2] O += M D done for Y buffer b
};
// Barriers that complete once per chunk but can be waited on a chunk late
// come in pairs indexed by chunk parity: each then completes once per two
// chunks, so a parity wait can never see it two phases ahead.

constexpr uint32_t ID_G = ptx::idesc_bf16(128, 64, false, false);
constexpr uint32_t ID_YW = ptx::idesc_bf16(128, 128, false, true);
constexpr uint32_t ID_N64 = ptx::idesc_bf16(128, 64, false, true);
constexpr uint32_t ID_S = ptx::idesc_bf16(128, 64, true, true);

// Optional timeline trace (compile with -DEFLA_TRACE): threads of CTA 0
// store clock64() at their hand-off points into fixed slots
// g_efla_trace[chunk % 1024][event] (plain stores, no atomics, so tracing
// adds no round trip to the critical path).
#ifdef EFLA_TRACE
__device__ long long g_efla_trace[1024 * 64];
#define EFLA_TR(ev, chunk)                                                                   \
    do {                                                                                   \
        if (blockIdx.x == 0) g_efla_trace[((chunk) & 1023) * 64 + ((ev) & 63)] = clock64(); \
    } while (0)
#else
#define EFLA_TR(ev, chunk) \
    do {                   \
    } while (0)
#endif

__device__ __forceinline__ uint32_t f2tf32(float x) {
    uint32_t r;
    asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
    return r;
}
// D(16x8) += A(16x8, row) B(8x8, col), TF32 inputs, fp32 accumulation (warp-wide).
__device__ __forceinline__ void mma_tf32(float (&d)[4], const uint32_t (&a)[4], const uint32_t (&b)[2]) {
    asm volatile(
        "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}

__device__ __forceinline__ bool bar_any(uint32_t id, uint32_t n, bool v) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 p, %1, 0;\n\t"
        "bar.red.or.pred q, %2, %3, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)v), "r"(id), "r"(n)
        : "memory");
    return r != 0;
}

__device__ __forceinline__ void unpack8(const uint4 &u, float (&f)[8]) {
    const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&u);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float2 x = __bfloat1622float2(h[i]);
        f[2 * i] = x.x;
        f[2 * i + 1] = x.y;
    }
}

// A 64 x 64 fp32 matrix stored as two 32-row halves of 256-byte rows.  The
// 16-byte slots of row r are XOR-permuted by (r & 15), so row-per-thread
// float4 stores and same-column loads across rows hit distinct banks.
struct Split64 {
    float *lo, *hi;
    __device__ __forceinline__ float *row(int r) const { return (r < 32 ? lo : hi) + (r & 31) * LDF; }
    // element (r, c); for c % 4 == 0 this is the start of a contiguous float4
    __device__ __forceinline__ float *at(int r, int c) const {
        return row(r) + ((((c >> 2) ^ (r & 15)) << 2) | (c & 3));
    }
};

// T = (I + A)^{-1} for the strictly lower triangular 64 x 64 A.  First the
// four 16 x 16 diagonal blocks by right-looking forward substitution (one
// warp per block, one column per lane pair, fp32); then block rows I = 1..3:
//     R = A_{I,<I} T_{<I,<I},   T_{I,<I} = -T_II R,
// as 16 x 8 tiles on mma.sync (TF32 operands, fp32 accumulation).  TF32
// here costs nothing measurable: T then feeds bf16 hi/lo operands, and an
// emulation of the whole kernel gave the same error against the oracle
// with fp32 or TF32 block products.  128 threads (prep).
__device__ __forceinline__ void invert_unit_lower(const int p, const Split64 Af, const Split64 Tf, int n_trace = 0) {
    {
        const int w = p >> 5, l = p & 31, c = l & 15, h = l >> 4, base = 16 * w;
        float acc[8];
#pragma unroll
        for (int s = 0; s < 8; ++s) acc[s] = (2 * s + h == c) ? 1.f : 0.f;
#pragma unroll
        for (int m = 0; m < 16; ++m) {
            const float x = __shfl_sync(0xffffffffu, acc[m >> 1], ((m & 1) << 4) | c);
#pragma unroll
            for (int s = 0; s < 8; ++s) acc[s] = fmaf(-*Af.at(base + 2 * s + h, base + m), x, acc[s]);
        }
#pragma unroll
        for (int s = 0; s < 8; ++s) *Tf.at(base + 2 * s + h, base + c) = acc[s];
        if (l == 0) EFLA_TR(30 + w, n_trace);
    }
    ptx::named_bar(1, 128);
    // Block rows on the tensor cores through mma.sync m16n8k8 (TF32 inputs,
    // fp32 accumulation): warp w owns the 8-column tiles jt = w, w+4, ... of
    // block row I, so R's tile and the T tile computed from it stay inside
    // one warp.  R is parked in T's own slots between the two products.
    const int w = p >> 5, lane = p & 31, g = lane >> 2, t = lane & 3;
#pragma unroll 1
    for (int I = 1; I < 4; ++I) {
        const int r0 = 16 * I;
#pragma unroll 1
        for (int jt = w; jt < 2 * I; jt += 4) {
            const int c0 = 8 * jt;
            float acc[4] = {0.f, 0.f, 0.f, 0.f};
            // R tile = A[r0.., k] T[k, c0..] over k from the column's own block up to r0
#pragma unroll 1
            for (int k0 = 16 * (jt >> 1); k0 < r0; k0 += 8) {
                const uint32_t a[4] = {f2tf32(*Af.at(r0 + g, k0 + t)), f2tf32(*Af.at(r0 + g + 8, k0 + t)),
                                       f2tf32(*Af.at(r0 + g, k0 + t + 4)), f2tf32(*Af.at(r0 + g + 8, k0 + t + 4))};
                const uint32_t bb[2] = {f2tf32(*Tf.at(k0 + t, c0 + g)), f2tf32(*Tf.at(k0 + t + 4, c0 + g))};
                mma_tf32(acc, a, bb);
            }
            *Tf.at(r0 + g, c0 + 2 * t) = acc[0];
            *Tf.at(r0 + g, c0 + 2 * t + 1) = acc[1];
            *Tf.at(r0 + g + 8, c0 + 2 * t) = acc[2];
            *Tf.at(r0 + g + 8, c0 + 2 * t + 1) = acc[3];
            __syncwarp();
            uint32_t rb[2][2];
#pragma unroll
            for (int kk = 0; kk < 2; ++kk) {
                rb[kk][0] = f2tf32(*Tf.at(r0 + 8 * kk + t, c0 + g));
                rb[kk][1] = f2tf32(*Tf.at(r0 + 8 * kk + t + 4, c0 + g));
            }
            __syncwarp();
            float out[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int kk = 0; kk < 2; ++kk) {  // T tile = -T_II R tile
                const int k0 = r0 + 8 * kk;
                const uint32_t a[4] = {f2tf32(*Tf.at(r0 + g, k0 + t)), f2tf32(*Tf.at(r0 + g + 8, k0 + t)),
                                       f2tf32(*Tf.at(r0 + g, k0 + t + 4)), f2tf32(*Tf.at(r0 + g + 8, k0 + t + 4))};
                mma_tf32(out, a, rb[kk]);
            }
            *Tf.at(r0 + g, c0 + 2 * t) = -out[0];
            *Tf.at(r0 + g, c0 + 2 * t + 1) = -out[1];
            *Tf.at(r0 + g + 8, c0 + 2 * t) = -out[2];
            *Tf.at(r0 + g + 8, c0 + 2 * t + 1) = -out[3];
        }
        if (lane == 0) EFLA_TR(40 + 4 * I + w, n_trace);
        ptx::named_bar(1, 128);
    }
}

// One 64-value fp32 row (held as two 32-register halves) -> bf16 hi at
// `base` and lo at `base + lo_off`, row `row` of a 128-byte-swizzled tile.
__device__ __forceinline__ void write_split_row(unsigned char *base, uint32_t lo_off, int row, const uint32_t (&a)[32],
                                                const uint32_t (&b)[32]);

// bf16 hi + lo split of a pair of fp32 values (hi = rn(x), lo = rn(x - hi)).
__device__ __forceinline__ void split2(float x0, float x1, uint32_t &hi, uint32_t &lo) {
    uint32_t h, l;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(h) : "f"(x1), "f"(x0));  // x0 -> low half
    const float h0 = __uint_as_float(h << 16), h1 = __uint_as_float(h & 0xffff0000u);
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(l) : "f"(x1 - h1), "f"(x0 - h0));
    hi = h;
    lo = l;
}

__device__ __forceinline__ void write_split_row(unsigned char *base, uint32_t lo_off, int row, const uint32_t (&a)[32],
                                                const uint32_t (&b)[32]) {
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        uint32_t h4[4], l4[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int c0 = 8 * j + 2 * u;
            const float x0 = __uint_as_float(c0 < 32 ? a[c0] : b[c0 - 32]);
            const float x1 = __uint_as_float(c0 + 1 < 32 ? a[c0 + 1] : b[c0 + 1 - 32]);
            split2(x0, x1, h4[u], l4[u]);
        }
        *reinterpret_cast<uint4 *>(base + ptx::sw128_chunk(row, j)) = make_uint4(h4[0], h4[1], h4[2], h4[3]);
        *reinterpret_cast<uint4 *>(base + lo_off + ptx::sw128_chunk(row, j)) = make_uint4(l4[0], l4[1], l4[2], l4[3]);
    }
}

template <typename Tout>
__global__ void __launch_bounds__(kThreads, 1)
    chunk_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const unsigned char *__restrict__ xws,
                    const float *__restrict__ S0, Tout *__restrict__ o, float *__restrict__ SL, int L, int nc) {
    using namespace ptx;
    extern __shared__ unsigned char smem_raw[];
    unsigned char *sm =
        reinterpret_cast<unsigned char *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(sm);
    uint64_t *bar = reinterpret_cast<uint64_t *>(sm + OFF_BAR);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(sm + OFF_MISC);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + OFF_MISC + 4);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const long bh = blockIdx.x / NSPLIT;
    const int j0 = (blockIdx.x % NSPLIT) * DVT;

    if (threadIdx.x == 0) {
        *abort_flag = 0;
        mbar_init(&bar[B_FULL], 1);
        mbar_init(&bar[B_FULL + 1], 1);
        mbar_init(&bar[B_EMPTY], 1);
        mbar_init(&bar[B_EMPTY + 1], 1);
        mbar_init(&bar[B_GFULL], 1);
        mbar_init(&bar[B_GEMPTY], 64);
        mbar_init(&bar[B_XFULL], 64);
        mbar_init(&bar[B_YFULL], 1);
        mbar_init(&bar[B_YFULL + 1], 1);
        mbar_init(&bar[B_A2FULL], 64);
        mbar_init(&bar[B_A2FULL + 1], 64);
        mbar_init(&bar[B_SBFULL], 128);
        mbar_init(&bar[B_DFULL], 1);
        mbar_init(&bar[B_DELTA], 128);
        mbar_init(&bar[B_SFULL], 1);
        mbar_init(&bar[B_DRAIN], 1);
        mbar_init(&bar[B_OREAD], 64);
        mbar_init(&bar[B_OREAD + 1], 64);
        mbar_init(&bar[B_OFULL], 1);
        mbar_init(&bar[B_OFULL + 1], 1);
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(tmem_slot, TMEM_COLS);
        tmem_relinquish();
    }
    // constant zero boxes: rows 0-63 of the [0; T' hi] and [0; T' lo] operands
    for (int i = threadIdx.x; i < 2 * (int)SLOT / 16; i += kThreads) {
        const uint4 z = make_uint4(0u, 0u, 0u, 0u);
        *reinterpret_cast<uint4 *>(sm + (i < (int)SLOT / 16 ? OFF_Z0 : OFF_Z1 - SLOT) + 16 * i) = z;
    }
    fence_proxy_async();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp < 2) {
        // ------------------------------------------------------------ io (warps 0-1)
        // T' = T diag(alpha) of every chunk arrives precomputed from
        // chunk_T_kernel as hi and lo bf16 boxes, already in the swizzled
        // image the X operand descriptors read: copy it in (prefetched a
        // chunk ahead in registers).  Then read O of the previous chunk out
        // of TMEM lanes 0..63 and store it.
        const int p = threadIdx.x;  // TMEM lane / chunk row
        const uint32_t tl = tmem + ((uint32_t)(32 * warp) << 16);
        const uint4 *xsrc = reinterpret_cast<const uint4 *>(xws + (size_t)bh * nc * XBYTES);
        uint4 xr[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) xr[i] = __ldcs(xsrc + p + 64 * i);
        auto read_O = [&](int m) -> bool {
            const bool ok = mbar_wait(&bar[B_OFULL + (m & 1)], (m >> 1) & 1, abort_flag);
            if (bar_any(3, 64, !ok || *abort_flag)) return false;
            tc_fence_after();
            uint32_t oa[32], ob[32];
            tmem_ld32(tl + T_YU + 64 * (m & 1), oa);
            tmem_ld32(tl + T_YU + 64 * (m & 1) + 32, ob);
            tmem_ld_wait(oa);
            tmem_ld_wait(ob);
            tc_fence_before();
            mbar_arrive(&bar[B_OREAD + (m & 1)]);
            if (p == 0) EFLA_TR(14, m);
            if (m * C + p < L) {
                Tout *dst = o + ((size_t)bh * L + m * C + p) * DK + j0;
#pragma unroll
                for (int c = 0; c < 64; c += 4) {
                    const uint32_t *src = (c < 32) ? &oa[c] : &ob[c - 32];
                    store4(dst + c, make_float4(__uint_as_float(src[0]), __uint_as_float(src[1]),
                                                __uint_as_float(src[2]), __uint_as_float(src[3])));
                }
            }
            return true;
        };
        bool alive = true;
        for (int n = 0; n < nc && alive; ++n) {
            if (n > 0) {  // the [0; T'] boxes are free once Y(n-1) completed
                const bool ok = mbar_wait(&bar[B_YFULL + ((n - 1) & 1)], ((n - 1) >> 1) & 1, abort_flag);
                if (bar_any(3, 64, !ok || *abort_flag)) break;
            }
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const uint32_t bo = 16u * (uint32_t)(p + 64 * i);  // byte offset in the 16 KB image
                *reinterpret_cast<uint4 *>(sm + (bo < SLOT ? OFF_THI + bo : OFF_TLO + (bo - SLOT))) = xr[i];
            }
            fence_proxy_async();
            mbar_arrive(&bar[B_XFULL]);
            if (p == 0) EFLA_TR(5, n);
            if (n + 1 < nc) {
#pragma unroll
                for (int i = 0; i < 16; ++i) xr[i] = __ldcs(xsrc + (size_t)(n + 1) * (XBYTES / 16) + p + 64 * i);
            }
            if (n > 0) alive = read_O(n - 1);
        }
        if (alive && !*abort_flag) read_O(nc - 1);
    } else if (warp < 4) {
        // ------------------------------------------------------------ mw (warps 2-3)
        // M = lower(Q K^T) as hi/lo boxes and -W from X K; both live in TMEM
        // lanes 64..127, which these warps own.
        const int r = threadIdx.x - 64;  // chunk row
        const uint32_t tl = tmem + ((uint32_t)(32 * warp) << 16);
        for (int n = 0; n < nc; ++n) {
            unsigned char *st = sm + (n & 1) * STAGE;
            bool ok = mbar_wait(&bar[B_GFULL], n & 1, abort_flag);
            if (r == 0) EFLA_TR(2, n);
            if (bar_any(1, 64, !ok || *abort_flag)) break;
            tc_fence_after();
            {
                uint32_t ga[32], gb[32];
                tmem_ld32(tl + T_G, ga);
                tmem_ld32(tl + T_G + 32, gb);
                tmem_ld_wait(ga);
                tmem_ld_wait(gb);
                tc_fence_before();
                mbar_arrive(&bar[B_GEMPTY]);
                unsigned char *mhi = sm + OFF_M + (n & 1) * 2 * SLOT, *mlo = mhi + SLOT;
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    uint32_t h4[4], l4[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int c0 = 8 * j + 2 * e;
                        const float x0 = (c0 <= r) ? __uint_as_float(c0 < 32 ? ga[c0] : gb[c0 - 32]) : 0.f;
                        const float x1 =
                            (c0 + 1 <= r) ? __uint_as_float(c0 + 1 < 32 ? ga[c0 + 1] : gb[c0 + 1 - 32]) : 0.f;
                        split2(x0, x1, h4[e], l4[e]);
                    }
                    *reinterpret_cast<uint4 *>(mhi + sw128_chunk(r, j)) = make_uint4(h4[0], h4[1], h4[2], h4[3]);
                    *reinterpret_cast<uint4 *>(mlo + sw128_chunk(r, j)) = make_uint4(l4[0], l4[1], l4[2], l4[3]);
                }
            }
            if (r == 0) EFLA_TR(3, n);
            ok = mbar_wait(&bar[B_YFULL + (n & 1)], (n >> 1) & 1, abort_flag);
            if (r == 0) EFLA_TR(6, n);
            if (bar_any(1, 64, !ok || *abort_flag)) break;
            tc_fence_after();
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                uint32_t wa[32], wb[32];
                tmem_ld32(tl + T_YW + 128 * (n & 1) + 64 * h, wa);
                tmem_ld32(tl + T_YW + 128 * (n & 1) + 64 * h + 32, wb);
                tmem_ld_wait(wa);
                tmem_ld_wait(wb);
                unsigned char *wrow = st + SL_W0 * SLOT + h * BOXSTRIDE;
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    uint32_t w4[4];
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        const int c0 = 8 * j + 2 * u;
                        const float x0 = __uint_as_float(c0 < 32 ? wa[c0] : wb[c0 - 32]);
                        const float x1 = __uint_as_float(c0 + 1 < 32 ? wa[c0 + 1] : wb[c0 + 1 - 32]);
                        w4[u] = pack_bf16(-x0, -x1);
                    }
                    *reinterpret_cast<uint4 *>(wrow + sw128_chunk(r, j)) = make_uint4(w4[0], w4[1], w4[2], w4[3]);
                }
            }
            fence_proxy_async();
            tc_fence_before();
            mbar_arrive(&bar[B_A2FULL + (n & 1)]);
            if (r == 0) EFLA_TR(7, n);
        }
    } else if (warp < 8) {
        // ------------------------------------------------------------ state
        const int q = threadIdx.x - 128;  // TMEM lane / state row
        const uint32_t tl = tmem + ((uint32_t)(32 * (warp & 3)) << 16);
        {
            uint32_t ra[32], rb[32];
            const float *src = S0 ? S0 + ((size_t)bh * DK + q) * DK + j0 : nullptr;
#pragma unroll
            for (int c = 0; c < 64; c += 4) {
                const float4 v = src ? *reinterpret_cast<const float4 *>(src + c) : make_float4(0.f, 0.f, 0.f, 0.f);
                uint32_t *dst = (c < 32) ? &ra[c] : &rb[c - 32];
                dst[0] = __float_as_uint(v.x);
                dst[1] = __float_as_uint(v.y);
                dst[2] = __float_as_uint(v.z);
                dst[3] = __float_as_uint(v.w);
            }
            tmem_st32(tl + T_S, ra);
            tmem_st32(tl + T_S + 32, rb);
            tmem_st_wait();
            write_split_row(sm + OFF_SB, 2 * SLOT, q, ra, rb);
            fence_proxy_async();
            tc_fence_before();
            mbar_arrive(&bar[B_SBFULL]);
        }
        for (int n = 0; n < nc; ++n) {
            const int b = n & 1;
            bool ok = mbar_wait(&bar[B_DFULL], n & 1, abort_flag);
            if (q == 64) EFLA_TR(10, n);
            if (bar_any(2, 128, !ok || *abort_flag)) break;
            tc_fence_after();
            if (warp >= 6) {  // D rows (lanes 64..127) -> bf16 MN-major operand, row c = lane - 64
                const int c = q - 64;
                uint32_t da[32], db[32];
                tmem_ld32(tl + T_YU + 64 * b, da);
                tmem_ld32(tl + T_YU + 64 * b + 32, db);
                tmem_ld_wait(da);
                tmem_ld_wait(db);
                if (q == 64) EFLA_TR(15, n);
                write_split_row(sm + OFF_DB, SLOT, c, da, db);
                if (q == 64) EFLA_TR(16, n);
            }
            fence_proxy_async();
            if (q == 64) EFLA_TR(17, n);
            tc_fence_before();
            mbar_arrive(&bar[B_DELTA]);
            if (q == 64) EFLA_TR(11, n);
            ok = mbar_wait(&bar[B_SFULL], n & 1, abort_flag);
            if (q == 64) EFLA_TR(12, n);
            if (bar_any(2, 128, !ok || *abort_flag)) break;
            tc_fence_after();
            uint32_t sa[32], sb[32];
            tmem_ld32(tl + T_S, sa);
            tmem_ld32(tl + T_S + 32, sb);
            tmem_ld_wait(sa);
            tmem_ld_wait(sb);
            if (q == 64) EFLA_TR(24, n);
            write_split_row(sm + OFF_SB, 2 * SLOT, q, sa, sb);
            if (q == 64) EFLA_TR(25, n);
            fence_proxy_async();
            tc_fence_before();
            mbar_arrive(&bar[B_SBFULL]);
            if (q == 64) EFLA_TR(13, n);
            if (n == nc - 1 && SL) {
                float *dst = SL + ((size_t)bh * DK + q) * DK + j0;
#pragma unroll
                for (int c = 0; c < 64; c += 4) {
                    const uint32_t *src = (c < 32) ? &sa[c] : &sb[c - 32];
                    *reinterpret_cast<float4 *>(dst + c) = make_float4(
                        __uint_as_float(src[0]), __uint_as_float(src[1]), __uint_as_float(src[2]),
                        __uint_as_float(src[3]));
                }
            }
        }
    } else if (warp == 8) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            const uint32_t sba = sbase + OFF_SB, dba = sbase + OFF_DB;
            const uint32_t xhi = sbase + OFF_Z0, xlo = sbase + OFF_Z1;  // [0; T' hi], [0; T' lo]
            auto stage_addr = [&](int n) { return sbase + (uint32_t)(n & 1) * STAGE; };
            // Descriptors: the 14-bit start-address field holds addr >> 4, and
            // shared addresses stay below 256 KB, so the field never carries:
            // the descriptor of (addr + off) is desc(addr) + (off >> 4).  Each group
            // builds its base descriptors once; the unrolled k-steps add
            // compile-time offsets, keeping the single issuing thread ahead of
            // the tensor pipe.
            const uint64_t dX[2] = {sdesc_sw128(xhi, 16, 1024), sdesc_sw128(xlo, 16, 1024)};
            const uint64_t dSB = sdesc_sw128(sba, SLOT, 1024), dDB = sdesc_sw128(dba, SLOT, 1024);
            auto issue_G = [&](int n) {
                const uint64_t d0 = sdesc_sw128(stage_addr(n) + SL_K0 * SLOT, 16, 1024);
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    const uint64_t d = d0 + (((kk >> 2) * BOXSTRIDE + (kk & 3) * 32) >> 4);
                    mma_bf16(tmem + T_G, d, d, ID_G, kk > 0);
                }
                mma_commit(&bar[B_GFULL]);
            };
            auto issue_Y = [&](int n) {  // Y = X_hi [K | V] + X_lo [K | V]
                const uint32_t sa = stage_addr(n), yu = tmem + T_YU + 64 * (n & 1);
                const uint64_t dK = sdesc_sw128(sa + SL_K0 * SLOT, BOXSTRIDE, 1024);
                const uint64_t dV = sdesc_sw128(sa + SL_V * SLOT, SLOT, 1024);
#pragma unroll
                for (int part = 0; part < 2; ++part) {
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        mma_bf16(tmem + T_YW + 128 * (n & 1), dX[part] + ((kk * 32) >> 4), dK + ((kk * 2048) >> 4),
                                 ID_YW, part | kk);
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        mma_bf16(yu, dX[part] + ((kk * 32) >> 4), dV + ((kk * 2048) >> 4), ID_N64, part | kk);
                }
                mma_commit(&bar[B_YFULL + (n & 1)]);
            };
            auto issue_D = [&](int n) {  // Y += [Q; -W] (S_hi + S_lo)
                const uint32_t yu = tmem + T_YU + 64 * (n & 1);
                const uint64_t dA = sdesc_sw128(stage_addr(n) + SL_Q0 * SLOT, 16, 1024);
#pragma unroll
                for (int part = 0; part < 2; ++part)
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk)
                        mma_bf16(yu, dA + (((kk >> 2) * BOXSTRIDE + (kk & 3) * 32) >> 4),
                                 dSB + ((part * 2 * SLOT + kk * 2048) >> 4), ID_N64, 1);
                mma_commit(&bar[B_DFULL]);
            };
            auto issue_SO = [&](int n) {  // S += K^T (D_hi + D_lo);  Y += M_hi D_hi + M_hi D_lo + M_lo D_hi
                const uint32_t yu = tmem + T_YU + 64 * (n & 1);
                const uint64_t dKt = sdesc_sw128(stage_addr(n) + SL_K0 * SLOT, BOXSTRIDE, 1024);
                const uint64_t dM = sdesc_sw128(sbase + OFF_M + (n & 1) * 2 * SLOT, 16, 1024);
#pragma unroll
                for (int part = 0; part < 2; ++part)
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        mma_bf16(tmem + T_S, dKt + ((kk * 2048) >> 4), dDB + ((part * SLOT + kk * 2048) >> 4), ID_S, 1);
                mma_commit(&bar[B_SFULL]);  // the state chain waits only for S
#pragma unroll
                for (int part = 0; part < 3; ++part) {
                    const uint32_t moff = (part == 2) ? SLOT : 0, doff = (part == 1) ? SLOT : 0;
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        mma_bf16(yu, dM + ((moff + kk * 32) >> 4), dDB + ((doff + kk * 2048) >> 4), ID_N64, 1);
                }
                mma_commit(&bar[B_OFULL + (n & 1)]);
                mma_commit(&bar[B_EMPTY + (n & 1)]);
            };
            // Event-driven issue: each product goes out as soon as its inputs are
            // ready, the serial D / SO chain first, so Y(n+1) and G(n+2) fill the
            // gaps while the state warps read TMEM.  Ordering rules:
            //   D(n)  after -W/M of chunk n (a2) and the bf16 state (sb);
            //   SO(n) after the bf16 D (delta);
            //   Y(m)  after X(m), after O(m-2) left the Y buffer (oread[m%2]) and
            //         after D(m-2) was issued: D(m-2) waits for the -W readout
            //         of chunk m-2, the last reader of X K buffer m%2;
            //   G(m)  after its TMA stage landed, G(m-1) was read (gempty) and
            //         SO(m-2) was issued (so the commit that signals G(m)
            //         also covers every earlier reader of the buffers that
            //         chunk m's prep overwrites).
            int nD = 0, nS = 0, nY = 0, nG = 0;
            long long idle_since = clock64();
            while (nS < nc) {
                bool did = false;
                if (nD < nc && nD == nS && nD < nY && mbar_test(&bar[B_A2FULL + (nD & 1)], (nD >> 1) & 1) &&
                    mbar_test(&bar[B_SBFULL], nD & 1)) {
                    tc_fence_after();
                    EFLA_TR(20, nD); issue_D(nD++);
                    did = true;
                }
                if (nS < nD && mbar_test(&bar[B_DELTA], nS & 1)) {
                    tc_fence_after();
                    EFLA_TR(21, nS); issue_SO(nS++);
                    did = true;
                }
                if (nY < nc && nY < nG && nY <= nD + 1 && mbar_test(&bar[B_XFULL], nY & 1) &&
                    (nY < 2 || mbar_test(&bar[B_OREAD + (nY & 1)], ((nY - 2) >> 1) & 1))) {
                    tc_fence_after();
                    EFLA_TR(22, nY); issue_Y(nY++);
                    did = true;
                }
                if (nG < nc && nG <= nS + 1 && nG <= nY + 1 && mbar_test(&bar[B_FULL + (nG & 1)], (nG >> 1) & 1) &&
                    (nG == 0 || mbar_test(&bar[B_GEMPTY], (nG - 1) & 1))) {
                    tc_fence_after();
                    EFLA_TR(23, nG); issue_G(nG++);
                    did = true;
                }
                if (did) {
                    idle_since = clock64();
                } else if (*abort_flag) {
                    break;
                } else if (clock64() - idle_since > kWaitCycles) {
                    *abort_flag = 1;
                    raise_error(kErrTimeout);
                    break;
                }
            }
            // drain: wait (bounded, even after an abort) until every MMA issued has completed
            mma_commit(&bar[B_DRAIN]);
            int never = 0;
            mbar_wait(&bar[B_DRAIN], 0, &never);
        }
    } else {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            tma_prefetch(&tm_q);
            tma_prefetch(&tm_k);
            tma_prefetch(&tm_v);
            int last[2] = {-1, -1};
            for (int n = 0; n < nc; ++n) {
                const int s = n & 1;
                if (n >= 2 && !mbar_wait(&bar[B_EMPTY + s], ((n >> 1) - 1) & 1, abort_flag)) break;
                if (*abort_flag) break;
                unsigned char *st = sm + s * STAGE;
                uint64_t *fb = &bar[B_FULL + s];
                mbar_expect_tx(fb, 5 * SLOT);
                const int y = n * C, z = (int)bh;
                tma_load_3d(st + SL_K0 * SLOT, &tm_k, fb, 0, y, z);
                tma_load_3d(st + SL_K0 * SLOT + BOXSTRIDE, &tm_k, fb, 64, y, z);
                tma_load_3d(st + SL_Q0 * SLOT, &tm_q, fb, 0, y, z);
                tma_load_3d(st + SL_Q0 * SLOT + BOXSTRIDE, &tm_q, fb, 64, y, z);
                tma_load_3d(st + SL_V * SLOT, &tm_v, fb, j0, y, z);
                last[s] = n;
            }
            // drain: every copy this thread started has landed before the CTA exits
            int never = 0;
            for (int s = 0; s < 2; ++s)
                if (last[s] >= 0) mbar_wait(&bar[B_FULL + s], (last[s] >> 1) & 1, &never);
        }
    }
    __syncwarp();
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, TMEM_COLS);
    }
}

// ---------------------------------------------------------------- T' kernel
__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], const uint32_t (&a)[4], const uint32_t (&b)[2]) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}

constexpr int KLD = DK + 8;  // padded bf16 row stride of K: conflict-free mma.sync fragment loads
struct TPrepSmem {
    union {  // K is dead once K K^T is formed; T reuses its space (6 CTAs per SM instead of 4)
        __nv_bfloat16 K[C][KLD];
        float T[C * LDF];
    };
    float A[C * LDF];
    float alpha[C];
};

// Per chunk (rows past L zero): alpha = gate(beta, ||k||^2); A = strictly-lower
// (diag(alpha) K K^T) by mma.sync bf16 on the 20 lower 16 x 8 tiles;
// T = (I + A)^{-1}; writes T' = T diag(alpha) as bf16 hi and lo boxes in the
// 128-byte-swizzled image chunk_tc_kernel's descriptors read.  One CTA of 128
// threads per (b, h, chunk); independent chunks, so latency hides across CTAs.
__global__ void __launch_bounds__(128) chunk_T_kernel(const __nv_bfloat16 *__restrict__ k,
                                                      const float *__restrict__ beta,
                                                      unsigned char *__restrict__ xws, int L, int nc, int euler) {
    extern __shared__ __align__(16) unsigned char tsm_raw[];
    TPrepSmem &sm = *reinterpret_cast<TPrepSmem *>(tsm_raw);
    const int p = threadIdx.x, w = p >> 5, lane = p & 31, g = lane >> 2, t = lane & 3;
    const long gidx = blockIdx.x;
    const int chunk = (int)(gidx % nc);
    const long bh = gidx / nc;
    const int t0 = chunk * C, n = min(C, L - t0);
    const __nv_bfloat16 *kc = k + ((size_t)bh * L + t0) * DK;
    for (int e = p; e < C * (DK / 8); e += 128) {
        const int r = e / (DK / 8), c8 = (e % (DK / 8)) * 8;
        uint4 v = make_uint4(0u, 0u, 0u, 0u);
        if (r < n) v = __ldg(reinterpret_cast<const uint4 *>(kc + (size_t)r * DK + c8));
        *reinterpret_cast<uint4 *>(&sm.K[r][c8]) = v;
    }
    __syncthreads();
    {   // gate: two lanes per key row
        const int r = p >> 1, h = p & 1;
        float acc8[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            float f[8];
            unpack8(*reinterpret_cast<const uint4 *>(&sm.K[r][64 * h + 8 * j]), f);
#pragma unroll
            for (int e = 0; e < 8; ++e) acc8[e] = fmaf(f[e], f[e], acc8[e]);
        }
        float ss = ((acc8[0] + acc8[1]) + (acc8[2] + acc8[3])) + ((acc8[4] + acc8[5]) + (acc8[6] + acc8[7]));
        ss += __shfl_xor_sync(0xffffffffu, ss, 1);
        if (h == 0) sm.alpha[r] = (r < n) ? gate_alpha(beta[bh * (long)L + t0 + r], ss, euler != 0) : 0.f;
    }
    __syncthreads();
    const Split64 Af{sm.A, sm.A + 32 * LDF}, Tf{sm.T, sm.T + 32 * LDF};
    // the 20 tiles (row tile i of 16, column tile j of 8) on or below the diagonal blocks
    for (int tile = w; tile < 20; tile += 4) {
        int i = 0, j = tile;
        while (j >= 2 * i + 2) {
            j -= 2 * i + 2;
            ++i;
        }
        float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int k0 = 0; k0 < DK; k0 += 16) {
            const uint32_t a[4] = {*reinterpret_cast<const uint32_t *>(&sm.K[16 * i + g][k0 + 2 * t]),
                                   *reinterpret_cast<const uint32_t *>(&sm.K[16 * i + g + 8][k0 + 2 * t]),
                                   *reinterpret_cast<const uint32_t *>(&sm.K[16 * i + g][k0 + 2 * t + 8]),
                                   *reinterpret_cast<const uint32_t *>(&sm.K[16 * i + g + 8][k0 + 2 * t + 8])};
            const uint32_t b[2] = {*reinterpret_cast<const uint32_t *>(&sm.K[8 * j + g][k0 + 2 * t]),
                                   *reinterpret_cast<const uint32_t *>(&sm.K[8 * j + g][k0 + 2 * t + 8])};
            mma_bf16_16816(acc, a, b);
        }
        const int r0 = 16 * i + g, r1 = r0 + 8, c0 = 8 * j + 2 * t;
        *Af.at(r0, c0) = (c0 < r0) ? sm.alpha[r0] * acc[0] : 0.f;
        *Af.at(r0, c0 + 1) = (c0 + 1 < r0) ? sm.alpha[r0] * acc[1] : 0.f;
        *Af.at(r1, c0) = (c0 < r1) ? sm.alpha[r1] * acc[2] : 0.f;
        *Af.at(r1, c0 + 1) = (c0 + 1 < r1) ? sm.alpha[r1] * acc[3] : 0.f;
    }
    __syncthreads();
    invert_unit_lower(p, Af, Tf);
    unsigned char *dst = xws + (size_t)gidx * XBYTES;
#pragma unroll
    for (int ii = 0; ii < 4; ++ii) {
        const int e = p + 128 * ii, r = e >> 3, jj = e & 7;
        const float4 ta = *reinterpret_cast<const float4 *>(Tf.at(r, 8 * jj));
        const float4 tb = *reinterpret_cast<const float4 *>(Tf.at(r, 8 * jj + 4));
        const float tv[8] = {ta.x, ta.y, ta.z, ta.w, tb.x, tb.y, tb.z, tb.w};
        uint32_t h4[4], l4[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int c = 8 * jj + 2 * u;
            const float x0 = (c <= r) ? tv[2 * u] * sm.alpha[c] : 0.f;
            const float x1 = (c + 1 <= r) ? tv[2 * u + 1] * sm.alpha[c + 1] : 0.f;
            split2(x0, x1, h4[u], l4[u]);
        }
        *reinterpret_cast<uint4 *>(dst + ptx::sw128_chunk(r, jj)) = make_uint4(h4[0], h4[1], h4[2], h4[3]);
        *reinterpret_cast<uint4 *>(dst + SLOT + ptx::sw128_chunk(r, jj)) = make_uint4(l4[0], l4[1], l4[2], l4[3]);
    }
}

// ---------------------------------------------------------------- host side
typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

inline EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

// 3-D view [bh][L][128] of a bf16 [B][H][L][128] tensor, 64 x 64 boxes,
// 128-byte swizzle; rows past L read as zero.
inline bool make_map(CUtensorMap *m, const void *base, long bh, int L) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return false;
    const cuuint64_t dims[3] = {(cuuint64_t)DK, (cuuint64_t)L, (cuuint64_t)bh};
    const cuuint64_t strides[2] = {(cuuint64_t)DK * 2, (cuuint64_t)L * DK * 2};
    const cuuint32_t box[3] = {64, 64, 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Scratch of the tensor-core path: one T' image (hi + lo boxes) per chunk.
inline size_t workspace_bytes(long bh, int L) { return (size_t)bh * ((L + C - 1) / C) * XBYTES; }

template <typename Tout>
inline efla_status_t launch(const void *q, const void *k, const void *v, const float *beta, const float *S0,
                            void *o, float *SL, long bh, int L, bool euler, void *ws, cudaStream_t st) {
    CUtensorMap mq, mk, mv;
    if (!make_map(&mq, q, bh, L) || !make_map(&mk, k, bh, L) || !make_map(&mv, v, bh, L)) return EFLA_ERR_CUDA;
    if (!ensure_smem<chunk_tc_kernel<Tout>>(SMEM_BYTES) || !ensure_smem<chunk_T_kernel>(sizeof(TPrepSmem)))
        return EFLA_ERR_CUDA;
    const long grid = bh * NSPLIT;
    const int nc = (L + C - 1) / C;
    if (grid > 0x7fffffffL || bh * nc > 0x7fffffffL) return EFLA_ERR_SHAPE;
    unsigned char *xws = static_cast<unsigned char *>(ws);
    chunk_T_kernel<<<(unsigned)(bh * nc), 128, sizeof(TPrepSmem), st>>>(static_cast<const __nv_bfloat16 *>(k), beta,
                                                                        xws, L, nc, euler ? 1 : 0);
    if (cudaGetLastError() != cudaSuccess) return EFLA_ERR_CUDA;
    chunk_tc_kernel<Tout><<<(unsigned)grid, kThreads, SMEM_BYTES, st>>>(mq, mk, mv, xws, S0, static_cast<Tout *>(o),
                                                                         SL, L, nc);
    return cudaGetLastError() == cudaSuccess ? EFLA_OK : EFLA_ERR_CUDA;
}

}  // namespace tc

// The tensor-core kernel takes bf16 q/k/v with d_k = d_v = 128.
inline bool tc_path_applies(bool bf16, int d_k, int d_v) { return bf16 && d_k == 128 && d_v == 128; }

inline efla_status_t launch_chunk_tc(const void *q, const void *k, const void *v, const float *beta,
                                     const float *S0, void *o, bool o_bf16, float *SL, long bh, int L, bool euler,
                                     void *ws, cudaStream_t st) {
    return o_bf16 ? tc::launch<__nv_bfloat16>(q, k, v, beta, S0, o, SL, bh, L, euler, ws, st)
                  : tc::launch<float>(q, k, v, beta, S0, o, SL, bh, L, euler, ws, st);
}

}  // namespace efla
