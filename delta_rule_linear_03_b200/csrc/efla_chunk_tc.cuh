// efla_chunk_tc.cuh - fused chunked prefill on the 5th-generation tensor
// cores (tcgen05 + TMEM + TMA) for bf16 q/k/v, d_k = d_v = 128.
//
// Computes the recurrence of "Exact Flow Linear Attention" (papernotes.org
// summary of arXiv 2512.12602, 关键设计 2; readout of the 整体框架
// flowchart) chunk by chunk in the UT form of the chunk-parallel scheme that
// page cites (整体框架, "WY / UT"), with C = 64:
//
//   kernel chunk_prep_tc_kernel, one CTA per chunk, all chunks in parallel
//   (everything that does not depend on the state):
//   alpha = gate(beta, ||k||^2)                       (fp32, CUDA cores)
//   G  = [K; Q] K^T                                   (tcgen05, M=128 N=64 K=128)
//   A  = strictly-lower(diag(alpha) K K^T),  M = lower-incl-diag(Q K^T)   (from G)
//   T  = (I + A)^{-1},  T' = T diag(alpha)            (fp32 substitution on the
//                                                      diagonal blocks, 2 x 2 block
//                                                      inverse on TF32 mma.sync)
//   W  = T' K,  U = T' V                              (tcgen05, M=64 N=128,
//                                                      T' as bf16 hi + lo)
//   -> workspace: -W (bf16), M (bf16), U (fp32)
//   kernel chunk_tc_kernel, serial over the chunks of one (b, h, d_v half):
//   Y  = [Q; -W] S          ->  [Q S; -W S]           (tcgen05, M=128 N=128 K=128)
//   D  = U + (-W S)                                   (CUDA cores, TMEM -> smem)
//   S += K^T D                                        (tcgen05, M=128 N=128 K=64)
//   Y += [M; *] D           ->  O = Q S + M D         (tcgen05, M=128 N=128 K=64)
//
// Every product is stacked to M = 128 rows so the accumulator of each
// tcgen05.mma occupies all 128 TMEM lanes, one row per lane.  (In the last
// product the lower 64 rows of the A operand are whatever follows M in shared
// memory: they only add into the -W S rows of Y, which are dead by then.)
// The hi and lo halves of a split operand sit side by side as one N = 128
// operand, [S_hi | S_lo] and [D_hi | D_lo], so each product is half as many
// tcgen05.mma ops as with the halves issued one after the other (an N = 128
// op costs about a third more than an N = 64 one; an M = 64 op costs what an
// M = 128 op does).  The two 64-column halves of each accumulator are summed
// when read out; the state is kept as S = S_a + S_b, two fp32 accumulators
// that collect K^T D_hi and K^T D_lo.
//
// Precision: q, k, v are exact bf16 operands.  S, D and T' are fp32 values
// fed to the bf16 tensor cores as a hi + lo pair of bf16 (x = hi + lo to ~16
// significant bits); -W and M go in as single bf16 (M only reaches the
// output, not the state).  Accumulation is fp32 (TMEM or mma.sync registers)
// and the state is kept in fp32.
//
// The serial kernel holds only the state chain Y -> D -> S and the output
// product, so its tensor pipe is never busy with work the chain waits behind.
// One CTA per (b, h, half of d_v): the 128 x 64 fp32 state tile lives in
// TMEM for the whole sequence.  Warp roles:
//   warps 0-7  TMEM <-> registers <-> smem, each warp a 32-lane x 32-column
//              quarter-half: all 8 read S (-> bf16 hi/lo operand); warps
//              2,3,6,7 (lanes 64..127) form D; warps 0,1,4,5 (lanes 0..63)
//              read O out to HBM
//   warp 8     one thread issues every tcgen05.mma and commit
//   warp 9     one thread issues the TMA loads (2-stage ring: Q, K tiles and
//              the -W, M, U images of the workspace)
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
constexpr uint32_t SLOT = 8192;  // one 64 x 64 bf16 swizzled box
// Per-chunk workspace image written by chunk_prep_kernel:
//   [0, 16K)   -W, two boxes (d_k columns 0-63, 64-127), 128-byte swizzle
//   [16K, 24K) M box, 128-byte swizzle
//   [24K, 56K) U fp32, two d_v halves of 64 rows x 256 B; the 16-byte
//              chunk j of row r sits at position j ^ (r & 15)
constexpr uint32_t IMG_W = 0, IMG_M = 2 * SLOT, IMG_U = 3 * SLOT, PREP_BYTES = 7 * SLOT;
constexpr uint32_t UHALF = 2 * SLOT;
// Shared-memory stage (one chunk), in 8 KB slots: Q0 W0 Q1 W1 K0 K1 M U U.
// [Q0; W0] and [Q1; W1] are the two K-halves of the 128-row A operand [Q; -W].
constexpr uint32_t SL_Q0 = 0, SL_W0 = 1, SL_K0 = 4, SL_M = 6, SL_U = 7, NSLOTS = 9;
constexpr uint32_t STAGE = NSLOTS * SLOT;
// A stage lands in two parts with their own barriers: part A (Q, -W), read by
// Y = [Q; -W] S only, and part B (K, M, U), read until the end of the chunk;
// part A of chunk n+2 can then load as soon as Y of chunk n is done.
constexpr uint32_t TX_A = 4 * SLOT, TX_B = 5 * SLOT;
static_assert(TX_A + TX_B == STAGE, "stage parts");
constexpr int LDF = 64;                          // fp32 row stride of A and T (prep)
constexpr uint32_t OFF_SB = 2 * STAGE;           // S tile bf16 hi, then lo (MN-major B), 128 x 64 each
constexpr uint32_t OFF_DB = OFF_SB + 4 * SLOT;   // [2] D bf16 hi, then lo (MN-major B), 64 x 64 each
constexpr uint32_t OFF_OST = OFF_DB + 4 * SLOT;  // O tile staged for the TMA store (64 x 64, fp32 or bf16)
constexpr uint32_t OFF_BAR = OFF_OST + 2 * SLOT;
constexpr uint32_t NBAR = 20;
constexpr uint32_t OFF_MISC = OFF_BAR + NBAR * 8;
constexpr uint32_t SMEM_BYTES = OFF_MISC + 16 + 1024;  // + slack to align the base to 1024 B
static_assert(SMEM_BYTES <= 232448, "shared memory per CTA");

// TMEM columns (fp32, 128 lanes): the state tile [S_a | S_b], then two Y
// accumulators [Y S_hi | Y S_lo] (by chunk parity) so O of chunk n can wait
// in TMEM while Y(n+1) runs.
constexpr uint32_t T_S = 0, T_Y = 128, TMEM_COLS = 512;

enum : int {
    B_FULLA = 0,    // [2] stage part A landed (TMA transaction count)
    B_FULLB = 2,    // [2] stage part B landed
    B_EMPTYA = 4,   // [2] part A free again (commit after Y)
    B_EMPTYB = 6,   // [2] part B free again (commit after O)
    B_SBFULL = 8,   // bf16 S tile written (8 warps)
    B_DFULL = 9,    // Y = [Q; -W] S done
    B_DELTA = 10,   // bf16 D written (4 warps)
    B_SFULL = 11,   // S += K^T D done
    B_DRAIN = 12,   // final drain of the MMA pipe
    B_OREAD = 13,   // [2] O of a chunk read out of Y buffer b (4 warps)
    B_OFULL = 15,   // [2] O += M D done for Y buffer b
};
// Barriers that complete once per chunk but can be waited on a chunk late
// come in pairs indexed by chunk parity: each then completes once per two
// chunks, so a parity wait can never see it two phases ahead.

constexpr uint32_t ID_Y = ptx::idesc_bf16(128, 128, false, true);
constexpr uint32_t ID_S = ptx::idesc_bf16(128, 128, true, true);

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
// Launch timeline (globaltimer, ns): earliest CTA start and latest CTA end
// of each launch kind of a call: 0 prep (chunks from 0), 1 prep (a later
// chunk range), 2 pass A, 3 pass B or single pass, 4 segment chain.
__device__ unsigned long long g_efla_gt[8][2];
__device__ __forceinline__ unsigned long long efla_gtime() {
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}
#define EFLA_GT_BEGIN(kind) \
    do {                     \
        if (threadIdx.x == 0) atomicMin(&g_efla_gt[(kind)][0], efla_gtime()); \
    } while (0)
#define EFLA_GT_END(kind)    \
    do {                     \
        if (threadIdx.x == 0) atomicMax(&g_efla_gt[(kind)][1], efla_gtime()); \
    } while (0)
// Per-CTA times of the serial kernel (globaltimer, ns): [launch kind - 2]
// [job][CTA][0: past the grid dependency, 1: end]
__device__ unsigned long long g_efla_cta[2][16][64][2];
#define EFLA_CTA(kind, i)                                                                         \
    do {                                                                                        \
        if (threadIdx.x == 0 && blockIdx.x < 64) g_efla_cta[(kind) - 2][blockIdx.y][blockIdx.x][i] = efla_gtime(); \
    } while (0)
// the first paired-run job of the launch (blockIdx.y == 1), events 40-47
#define EFLA_TR2(ev, chunk)                                                                                   \
    do {                                                                                                      \
        if (blockIdx.x == 0 && blockIdx.y == 1) g_efla_trace[((chunk) & 1023) * 64 + ((ev) & 63)] = clock64(); \
    } while (0)
#else
#define EFLA_TR(ev, chunk) \
    do {                   \
    } while (0)
#define EFLA_TR2(ev, chunk) \
    do {                    \
    } while (0)
#define EFLA_GT_BEGIN(kind) \
    do {                    \
    } while (0)
#define EFLA_GT_END(kind) \
    do {                  \
    } while (0)
#define EFLA_CTA(kind, i) \
    do {                  \
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

// A 64 x 64 fp32 matrix of 256-byte rows whose 16-byte slots are XOR-permuted
// by (r & 15), so row-per-thread float4 stores and same-column loads across
// rows hit distinct banks.
struct Sw64 {
    float *p;
    // element (r, c); for c % 4 == 0 this is the start of a contiguous float4
    __device__ __forceinline__ float *at(int r, int c) const {
        return p + r * LDF + ((((c >> 2) ^ (r & 15)) << 2) | (c & 3));
    }
};

// Diagonal 16 x 16 blocks of A, laid out for the forward substitution:
// block b, column m, then its 16 rows r contiguous.
__device__ __forceinline__ int diag_index(int b, int m, int r) { return (b * 16 + m) * 16 + r; }

// One 16 x 8 tile product on mma.sync, acc += X[r0 + 0..15][k0 + 0..7] Y[k0 + 0..7][n0 + 0..7]
// (TF32 operands, fp32 accumulation; g = lane / 4, t = lane % 4 as in the
// m16n8k8 fragment layout).  xa(r, k) and yb(k, n) return TF32 bit patterns.
template <typename XA, typename YB>
__device__ __forceinline__ void tile_mma(float (&acc)[4], int g, int t, int r0, int k0, int n0, XA xa, YB yb) {
    const uint32_t a[4] = {xa(r0 + g, k0 + t), xa(r0 + g + 8, k0 + t), xa(r0 + g, k0 + t + 4),
                           xa(r0 + g + 8, k0 + t + 4)};
    const uint32_t b[2] = {yb(k0 + t, n0 + g), yb(k0 + t + 4, n0 + g)};
    mma_tf32(acc, a, b);
}

// T = (I + A)^{-1} for the strictly lower triangular 64 x 64 A, in place:
// AT holds A's blocks left of the diagonal (rounded to TF32) on entry and T's
// lower triangle (diagonal blocks included, zeros above them) on return; A's
// diagonal blocks come in their own copy Ad.
//   1. The four 16 x 16 diagonal blocks by forward substitution in fp32,
//      one column per lane (warps 0-1): step m takes T[m][c], final by then
//      in the lane's own registers, times column m of A.
//   2. The lower-left 16 x 16 block of each 32 x 32 diagonal block
//      (2 x 2 block inverse):  T21 = -T22 (A21 T11)      (warps 0-3)
//   3. The lower-left 32 x 32 block:  T_lower = -T2 (A21 T1), T1 and T2 the
//      32 x 32 diagonal blocks finished by 1 and 2         (warps 0-7)
// Products 2 and 3 run as 16 x 8 tiles on mma.sync with TF32 operands and
// fp32 accumulation, skipping the k-steps where T is zero.  TF32 here costs
// nothing measurable: T then feeds bf16 hi/lo operands, and an emulation of
// the whole computation gave the same error against the oracle with fp32
// or TF32 block products.  Each inner product A21 T is formed (and parked
// in Ad, free by then) before its result overwrites the A tile it read.
// NT = 256 threads call it together; it ends with all of them synchronised.
template <int NT>
__device__ __forceinline__ void invert_unit_lower(const int p, float *__restrict__ Ad, const Sw64 AT) {
    static_assert(NT == 256, "eight warps: one per 16 x 8 tile of the last step");
    const int w = p >> 5, lane = p & 31, g = lane >> 2, t = lane & 3;
    const auto at_tf32 = [&](int r, int c) { return f2tf32(*AT.at(r, c)); };        // T (fp32)
    const auto at_raw = [&](int r, int c) { return __float_as_uint(*AT.at(r, c)); };  // A (stored as TF32)
    // 1. diagonal blocks
    if (p < 64) {
        const int blk = p >> 4, c = p & 15, base = 16 * blk;
        float x[16];
#pragma unroll
        for (int r = 0; r < 16; ++r) x[r] = (r == c) ? 1.f : 0.f;
#pragma unroll
        for (int m = 0; m < 15; ++m) {
            const float4 *col = reinterpret_cast<const float4 *>(Ad + diag_index(blk, m, 0));
            float a[16];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const float4 v = col[q];
                a[4 * q] = v.x, a[4 * q + 1] = v.y, a[4 * q + 2] = v.z, a[4 * q + 3] = v.w;
            }
#pragma unroll
            for (int r = m + 1; r < 16; ++r) x[r] = fmaf(-a[r], x[m], x[r]);
        }
#pragma unroll
        for (int r = 0; r < 16; ++r) *AT.at(base + r, base + c) = x[r];
    }
    ptx::named_bar(1, NT);
    if (p == 0) EFLA_TR(55, 1023);
    // 2. T21 of the 32 x 32 block h (rows 32 h + 16 .., columns 32 h ..), column tile nt
    float *park2 = Ad + (w >> 1) * 256;  // R = A21 T11 of block h, 16 x 16 row-major
    if (p < 128) {
        const int base = 32 * (w >> 1), nt = w & 1;
        float acc[4] = {0.f, 0.f, 0.f, 0.f};
        for (int k0 = 8 * nt; k0 < 16; k0 += 8)  // T11[k][8 nt + j] = 0 for k < 8 nt
            tile_mma(acc, g, t, 16, k0, 8 * nt, [&](int r, int k) { return at_raw(base + r, base + k); },
                     [&](int k, int n) { return at_tf32(base + k, base + n); });
        *reinterpret_cast<float2 *>(park2 + g * 16 + 8 * nt + 2 * t) = make_float2(acc[0], acc[1]);
        *reinterpret_cast<float2 *>(park2 + (g + 8) * 16 + 8 * nt + 2 * t) = make_float2(acc[2], acc[3]);
    }
    ptx::named_bar(1, NT);
    if (p < 128) {
        const int base = 32 * (w >> 1), nt = w & 1;
        float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int k0 = 0; k0 < 16; k0 += 8)
            tile_mma(acc, g, t, 0, k0, 8 * nt, [&](int r, int k) { return at_tf32(base + 16 + r, base + 16 + k); },
                     [&](int k, int n) { return f2tf32(park2[k * 16 + n]); });
        *reinterpret_cast<float2 *>(AT.at(base + 16 + g, base + 8 * nt + 2 * t)) = make_float2(-acc[0], -acc[1]);
        *reinterpret_cast<float2 *>(AT.at(base + 16 + g + 8, base + 8 * nt + 2 * t)) = make_float2(-acc[2], -acc[3]);
    }
    ptx::named_bar(1, NT);
    if (p == 0) EFLA_TR(56, 1023);
    // 3. rows 32-63, columns 0-31: row tile mt, column tile nt per warp
    const int mt = w >> 2, nt = w & 3;
    {
        float acc[4] = {0.f, 0.f, 0.f, 0.f};
        for (int k0 = 8 * nt; k0 < 32; k0 += 8)  // T1[k][8 nt + j] = 0 for k < 8 nt
            tile_mma(acc, g, t, 32 + 16 * mt, k0, 8 * nt, at_raw, at_tf32);
        *reinterpret_cast<float2 *>(Ad + (16 * mt + g) * 32 + 8 * nt + 2 * t) = make_float2(acc[0], acc[1]);
        *reinterpret_cast<float2 *>(Ad + (16 * mt + g + 8) * 32 + 8 * nt + 2 * t) = make_float2(acc[2], acc[3]);
    }
    ptx::named_bar(1, NT);
    if (p == 0) EFLA_TR(57, 1023);
    {
        float acc[4] = {0.f, 0.f, 0.f, 0.f};
        for (int k0 = 0; k0 < 16 * (mt + 1); k0 += 8)  // T2[16 mt + i][k] = 0 for k >= 16 (mt + 1)
            tile_mma(acc, g, t, 16 * mt, k0, 8 * nt, [&](int r, int k) { return at_tf32(32 + r, 32 + k); },
                     [&](int k, int n) { return f2tf32(Ad[k * 32 + n]); });
        *reinterpret_cast<float2 *>(AT.at(32 + 16 * mt + g, 8 * nt + 2 * t)) = make_float2(-acc[0], -acc[1]);
        *reinterpret_cast<float2 *>(AT.at(32 + 16 * mt + g + 8, 8 * nt + 2 * t)) = make_float2(-acc[2], -acc[3]);
    }
    ptx::named_bar(1, NT);
    if (p == 0) EFLA_TR(58, 1023);
}

// bf16 hi + lo split of a pair of fp32 values (hi = rn(x), lo = rn(x - hi)).
__device__ __forceinline__ void split2(float x0, float x1, uint32_t &hi, uint32_t &lo) {
    uint32_t h, l;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(h) : "f"(x1), "f"(x0));  // x0 -> low half
    const float h0 = __uint_as_float(h << 16), h1 = __uint_as_float(h & 0xffff0000u);
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(l) : "f"(x1 - h1), "f"(x0 - h0));
    hi = h;
    lo = l;
}

// 32 fp32 values (columns 8 * chunk0 ..) of row `row` -> bf16 hi at `base`
// and lo at `base + lo_off`, in a 128-byte-swizzled tile of 64-column rows.
__device__ __forceinline__ void write_split32(unsigned char *base, uint32_t lo_off, int row, int chunk0,
                                              const float (&x)[32]) {
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        uint32_t h4[4], l4[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) split2(x[8 * j + 2 * u], x[8 * j + 2 * u + 1], h4[u], l4[u]);
        const uint32_t off = ptx::sw128_chunk(row, chunk0 + j);
        *reinterpret_cast<uint4 *>(base + off) = make_uint4(h4[0], h4[1], h4[2], h4[3]);
        *reinterpret_cast<uint4 *>(base + lo_off + off) = make_uint4(l4[0], l4[1], l4[2], l4[3]);
    }
}

__device__ __forceinline__ void as_float32(const uint32_t (&r)[32], float (&x)[32]) {
#pragma unroll
    for (int i = 0; i < 32; ++i) x[i] = __uint_as_float(r[i]);
}

// cp.async.bulk global -> shared, `bytes` (multiple of 16, both ends 16-byte
// aligned), completing as transaction bytes on `bar`.
__device__ __forceinline__ void bulk_load(void *dst, const void *src, uint32_t bytes, uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            ptx::smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(ptx::smem_u32(bar))
        : "memory");
}

// TMA tensor store of one box from shared memory (bulk async group of this thread).
__device__ __forceinline__ void tma_store_3d(const CUtensorMap *map, const void *src, int x, int y, int z) {
    asm volatile("cp.async.bulk.tensor.3d.global.shared::cta.bulk_group [%0, {%2, %3, %4}], [%1];" ::"l"(
                     reinterpret_cast<uint64_t>(map)),
                 "r"(ptx::smem_u32(src)), "r"(x), "r"(y), "r"(z)
                 : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// Wait until every committed bulk store of this thread has finished reading shared memory.
__device__ __forceinline__ void bulk_wait_read0() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }

// cp.async.bulk shared -> global of `bytes` (multiple of 16, both ends
// 16-byte aligned), in this thread's bulk async group.
__device__ __forceinline__ void bulk_store(void *dst, const void *src, uint32_t bytes) {
    asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(reinterpret_cast<uint64_t>(dst)),
                 "r"(ptx::smem_u32(src)), "r"(bytes)
                 : "memory");
}

// Bounded wait by a whole warp; the answer is warp-uniform (false when any lane gave up).
__device__ __forceinline__ bool warp_wait(uint64_t *bar, uint32_t parity, volatile int *abort) {
    return __all_sync(0xffffffffu, ptx::mbar_wait(bar, parity, abort));
}

// One arrival per warp (barriers counted in warps): every lane has finished
// its shared-memory writes (and fenced them for the async proxy) and its
// TMEM loads; the warp synchronises, then lane 0 arrives.  One arrival
// instead of 32 keeps the barrier's last arrival, the one the waiting MMA
// thread is woken by, from queueing behind the warp's other 31.
__device__ __forceinline__ void warp_arrive(uint64_t *bar) {
    __syncwarp();
    if ((threadIdx.x & 31) == 0) ptx::mbar_arrive(bar);
}

// One run of the serial kernel over a contiguous range of chunks, for every
// (b, h, d_v half) of the grid: the whole sequence, or one segment of it.
struct SegJob {
    int c0, nch;      // first chunk and number of chunks
    int s0_kind;      // initial state: 0 zero, 1 read from s0, 2 the identity
    int write_o;      // store the outputs of these chunks
    const float *s0;  // [B*H][d_k][d_v] fp32 (s0_kind 1)
    float *sl;        // final state, [B*H][d_k][d_v] fp32, or null
    int pair;         // run from zero and from the identity together (no outputs):
                      // final state from zero to sl, and the segment's map
                      // (final state from the identity minus sl) to sl2
    float *sl2;
};
constexpr int kMaxJobs = 16;
// The jobs of one launch (blockIdx.y picks the job) and the sequence's chunk count.
struct SegPlan {
    int nc, njobs;
    SegJob job[kMaxJobs];
};

// ---------------------------------------------------------------- paired runs
// Pass A of the segment-parallel prefill needs, for every middle segment,
// its final state from zero (S_Z) and from the identity (S_I), and no
// outputs.  Both runs read the same chunk data, and every state column
// evolves on its own, so one CTA per (b, h, half of d_v) carries both: its
// 128 state columns are [S_Z | S_I] over this d_v half.  That is half the
// CTAs of two separate runs, so twice as many segments fit one wave.  Per
// chunk (no Q, M or O):
//   Y  = [-W; -W] [S_hi | S_lo]            (tcgen05, M=128 N=256 K=128)
//   D  = U + Y_hi + Y_lo                   (both halves of the 128 columns)
//   S += K^T (D_hi + D_lo)                 (tcgen05, M=128 N=128 K=64, hi then lo)
// -W is stacked twice so that every row of Y sits in two TMEM lanes (i and
// 64 + i): an M = 128 product costs what an M = 64 one does, and all 32
// lanes of every read-out warp then carry a row (lanes 0-63 the run from
// zero, lanes 64-127 the run from the identity).
// Shared memory (offsets from the 1024-byte aligned base):
//   two stages of W0 W0 W1 W1 K0 K1 U (U: this d_v half, 64 rows x 256 B)
//   S bf16: hi box 0, hi box 1, lo box 0, lo box 1 (128 rows x 64 columns each)
//   D bf16: hi box 0, hi box 1, lo box 0, lo box 1 (64 rows x 64 columns each)
// The hi and lo halves of S sit side by side as one N = 256 operand of Y
// (as in the single run), and Y is read out as Y_hi + Y_lo.  The state
// update keeps one accumulator (D_hi, then D_lo): the S read-out of 128
// columns per row is the longest step here, and a second accumulator would
// add a load and an add per element to it.
// TMEM: S [0, 128) [run from zero | run from the identity], Y [256, 512) =
// [Y_hi | Y_lo], each half 128 columns [zero | identity].
constexpr uint32_t P2_STAGE = 8 * SLOT;
constexpr uint32_t P2_SB = 2 * P2_STAGE, P2_DB = P2_SB + 8 * SLOT, P2_BAR = P2_DB + 4 * SLOT;
static_assert(P2_BAR <= OFF_BAR, "paired runs keep their barriers inside the serial kernel's layout");
static_assert(P2_BAR + 128 + 1024 <= SMEM_BYTES, "paired runs fit the serial kernel's shared memory");
constexpr uint32_t T2_S = 0, T2_Y = 256, T2_COLS = 512;
constexpr uint32_t ID2_Y = ptx::idesc_bf16(128, 256, false, true);
constexpr uint32_t ID2_S = ptx::idesc_bf16(128, 128, true, true);
enum : int { P2_FULL = 0, P2_EMPTY = 2, P2_SBFULL = 4, P2_DFULL = 5, P2_DELTA = 6, P2_SFULL = 7, P2_DRAIN = 8 };

__device__ __forceinline__ void pair_run(unsigned char *sm, const CUtensorMap &tm_k, const unsigned char *ws,
                                         const SegJob &job, int nc, long bh, int half) {
    using namespace ptx;
    const uint32_t sbase = smem_u32(sm);
    uint64_t *bar = reinterpret_cast<uint64_t *>(sm + P2_BAR);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(sm + P2_BAR + 96);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + P2_BAR + 100);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int j0 = half * DVT, cb = job.c0, ncj = job.nch;
    const unsigned char *img = ws + (size_t)bh * nc * PREP_BYTES;

    if (threadIdx.x == 0) {
        *abort_flag = 0;
        for (int s = 0; s < 2; ++s) {
            mbar_init(&bar[P2_FULL + s], 1);
            mbar_init(&bar[P2_EMPTY + s], 1);
        }
        mbar_init(&bar[P2_SBFULL], 8);  // one arrival per converter warp
        mbar_init(&bar[P2_DFULL], 1);
        mbar_init(&bar[P2_DELTA], 8);
        mbar_init(&bar[P2_SFULL], 1);
        mbar_init(&bar[P2_DRAIN], 1);
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(tmem_slot, T2_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    asm volatile("griddepcontrol.wait;" ::: "memory");
    EFLA_CTA(2, 0);

    if (warp < 8) {
        // ------------------------------------------------------------ TMEM <-> smem warps
        // Warp w: TMEM lanes 32 (w % 4) .., columns 64 (w / 4) .. + 63 of each
        // 128-column tile, i.e. the run from zero (w < 4) or from the identity.
        const int quad = warp & 3, run = warp >> 2;
        const int row = 32 * quad + lane;           // state row (d_k)
        // D read-out: lanes 0-63 hold chunk rows 0-63 for the run from zero,
        // lanes 64-127 the same rows for the run from the identity; warp w
        // takes 32 of that run's 64 columns (32 (w / 4) ..)
        const int drun = quad >> 1, dcol = 32 * (warp >> 2);
        const int drow = 32 * (quad & 1) + lane;
        const uint32_t tl = tmem + ((uint32_t)(32 * quad) << 16);
        float x[32];
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {  // initial state: zero, or the identity columns j0 + 32 hh ..
#pragma unroll
            for (int c = 0; c < 32; ++c) x[c] = (run == 1 && row == j0 + 32 * hh + c) ? 1.f : 0.f;
            uint32_t r[32];
#pragma unroll
            for (int i = 0; i < 32; ++i) r[i] = __float_as_uint(x[i]);
            tmem_st32(tl + T2_S + 64 * run + 32 * hh, r);
            write_split32(sm + P2_SB + run * 2 * SLOT, 4 * SLOT, row, 4 * hh, x);
        }
        tmem_st_wait();
        fence_proxy_async();
        tc_fence_before();
        warp_arrive(&bar[P2_SBFULL]);
        bool fin = false;  // this warp reached the final states
        for (int n = 0; n < ncj; ++n) {
            const int s = n & 1;
            // D = U + Y for this warp's 64 columns (the same U for both runs)
            if (!warp_wait(&bar[P2_DFULL], n & 1, abort_flag)) break;
            if (!warp_wait(&bar[P2_FULL + s], (n >> 1) & 1, abort_flag)) break;
            if (threadIdx.x == 0) EFLA_TR2(41, n);
            tc_fence_after();
            const unsigned char *urow = sm + s * P2_STAGE + 6 * SLOT + drow * 256;
            {
                uint32_t r[32], r2[32];
                tmem_ld32(tl + T2_Y + 64 * drun + dcol, r);         // Y_hi
                tmem_ld32(tl + T2_Y + 128 + 64 * drun + dcol, r2);  // Y_lo
                tmem_ld_wait(r);
                tmem_ld_wait(r2);
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const float4 v = *reinterpret_cast<const float4 *>(
                        urow + (((uint32_t)(dcol / 4 + j) ^ (drow & 15)) << 4));
                    x[4 * j] = v.x + (__uint_as_float(r[4 * j]) + __uint_as_float(r2[4 * j]));
                    x[4 * j + 1] = v.y + (__uint_as_float(r[4 * j + 1]) + __uint_as_float(r2[4 * j + 1]));
                    x[4 * j + 2] = v.z + (__uint_as_float(r[4 * j + 2]) + __uint_as_float(r2[4 * j + 2]));
                    x[4 * j + 3] = v.w + (__uint_as_float(r[4 * j + 3]) + __uint_as_float(r2[4 * j + 3]));
                }
                write_split32(sm + P2_DB + drun * SLOT, 2 * SLOT, drow, dcol / 8, x);
            }
            fence_proxy_async();
            tc_fence_before();
            warp_arrive(&bar[P2_DELTA]);
            if (threadIdx.x == 0) EFLA_TR2(42, n);
            // S out of TMEM: the bf16 operand of the next chunk, or the final states
            if (!warp_wait(&bar[P2_SFULL], n & 1, abort_flag)) break;
            if (threadIdx.x == 0) EFLA_TR2(43, n);
            tc_fence_after();
            if (n == ncj - 1) {  // the final states are read after the loop
                fin = true;
                break;
            }
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                uint32_t r[32];
                tmem_ld32(tl + T2_S + 64 * run + 32 * hh, r);
                tmem_ld_wait(r);
                as_float32(r, x);
                write_split32(sm + P2_SB + run * 2 * SLOT, 4 * SLOT, row, 4 * hh, x);
            }
            fence_proxy_async();
            tc_fence_before();
            warp_arrive(&bar[P2_SBFULL]);
            if (threadIdx.x == 0) EFLA_TR2(44, n);
        }
        // Final states: S(0) to sl, and the segment's map M = S(I) - S(0) to
        // sl2 (the segment chain's operand).  Every converter warp reaches this
        // vote, also after a failed wait, so the named barrier below cannot
        // miss a warp; after a failure nobody writes.  The run-from-zero warps
        // park their rows in shared memory (the S operand tiles: every product
        // has completed by now) for the identity-run warps of the same lanes.
        if (!bar_any(4, 256, !fin || *abort_flag)) {
            float *park = reinterpret_cast<float *>(sm + P2_SB);  // 128 rows x 32 columns
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                uint32_t r[32];
                tmem_ld32(tl + T2_S + 64 * run + 32 * hh, r);
                tmem_ld_wait(r);
                as_float32(r, x);
                float *pk = park + row * 32;
                if (run == 0) {
                    float *d = job.sl + ((size_t)bh * DK + row) * DK + j0 + 32 * hh;
#pragma unroll
                    for (int c = 0; c < 32; c += 4) {
                        const float4 v = make_float4(x[c], x[c + 1], x[c + 2], x[c + 3]);
                        *reinterpret_cast<float4 *>(d + c) = v;
                        *reinterpret_cast<float4 *>(pk + c) = v;
                    }
                }
                named_bar(4, 256);  // the run-from-zero half-rows are parked
                if (run == 1) {
                    float *d = job.sl2 + ((size_t)bh * DK + row) * DK + j0 + 32 * hh;
#pragma unroll
                    for (int c = 0; c < 32; c += 4) {
                        const float4 z = *reinterpret_cast<const float4 *>(pk + c);
                        *reinterpret_cast<float4 *>(d + c) =
                            make_float4(x[c] - z.x, x[c + 1] - z.y, x[c + 2] - z.z, x[c + 3] - z.w);
                    }
                }
                named_bar(4, 256);  // read before the next half overwrites the park
            }
        }
    } else if (warp == 8) {
        // ------------------------------------------------------------ MMA issuer
        const bool leader = lane == 0;
        for (int n = 0; n < ncj; ++n) {
            const int s = n & 1;
            const uint32_t st = sbase + (uint32_t)s * P2_STAGE;
            if (!warp_wait(&bar[P2_FULL + s], (n >> 1) & 1, abort_flag)) break;
            if (!warp_wait(&bar[P2_SBFULL], n & 1, abort_flag)) break;
            tc_fence_after();
            if (leader) EFLA_TR2(40, n);
            if (leader) {  // Y = -W [S_hi | S_lo]: 8 k-steps over d_k
                const uint64_t dW = sdesc_sw128(st, 16, 1024);
                const uint64_t dS = sdesc_sw128(sbase + P2_SB, 2 * SLOT, 1024);
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    mma_bf16(tmem + T2_Y, dW + (((kk >> 2) * 2 * SLOT + (kk & 3) * 32) >> 4),
                             dS + ((kk * 2048) >> 4), ID2_Y, kk);
                mma_commit(&bar[P2_DFULL]);
            }
            __syncwarp();
            if (!warp_wait(&bar[P2_DELTA], n & 1, abort_flag)) break;
            tc_fence_after();
            if (leader) EFLA_TR2(45, n);
            if (leader) {  // S += K^T (D_hi + D_lo): 4 k-steps over the chunk, hi then lo
                const uint64_t dKt = sdesc_sw128(st + 4 * SLOT, SLOT, 1024);
                const uint64_t dD = sdesc_sw128(sbase + P2_DB, SLOT, 1024);
#pragma unroll
                for (int part = 0; part < 2; ++part)
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        mma_bf16(tmem + T2_S, dKt + ((kk * 2048) >> 4), dD + ((part * 2 * SLOT + kk * 2048) >> 4),
                                 ID2_S, 1);
                mma_commit(&bar[P2_SFULL]);
                mma_commit(&bar[P2_EMPTY + s]);
            }
            __syncwarp();
        }
        __syncwarp();
        if (leader) mma_commit(&bar[P2_DRAIN]);
        __syncwarp();
        int never = 0;
        mbar_wait(&bar[P2_DRAIN], 0, &never);
    } else {
        // ------------------------------------------------------------ loads
        const bool leader = lane == 0;
        if (leader) tma_prefetch(&tm_k);
        int last[2] = {-1, -1};
        for (int n = 0; n < ncj; ++n) {
            const int s = n & 1;
            unsigned char *st = sm + s * P2_STAGE;
            if (n >= 2 && !warp_wait(&bar[P2_EMPTY + s], ((n >> 1) - 1) & 1, abort_flag)) break;
            if (__any_sync(0xffffffffu, *abort_flag != 0)) break;
            if (leader) {
                uint64_t *fb = &bar[P2_FULL + s];
                const unsigned char *src = img + (size_t)(cb + n) * PREP_BYTES;
                mbar_expect_tx(fb, 8 * SLOT);
                bulk_load(st, src + IMG_W, SLOT, fb);  // [-W; -W] for each d_k half
                bulk_load(st + SLOT, src + IMG_W, SLOT, fb);
                bulk_load(st + 2 * SLOT, src + IMG_W + SLOT, SLOT, fb);
                bulk_load(st + 3 * SLOT, src + IMG_W + SLOT, SLOT, fb);
                tma_load_3d(st + 4 * SLOT, &tm_k, fb, 0, (cb + n) * C, (int)bh);
                tma_load_3d(st + 5 * SLOT, &tm_k, fb, 64, (cb + n) * C, (int)bh);
                bulk_load(st + 6 * SLOT, src + IMG_U + half * UHALF, UHALF, fb);
            }
            __syncwarp();
            last[s] = n;
        }
        int never = 0;
        for (int s = 0; s < 2; ++s)
            if (last[s] >= 0) mbar_wait(&bar[P2_FULL + s], (last[s] >> 1) & 1, &never);
    }
    __syncwarp();
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, T2_COLS);
    }
}

template <typename Tout>
__global__ void __launch_bounds__(kThreads, 1)
    chunk_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_o, const unsigned char *__restrict__ ws,
                    const __grid_constant__ SegPlan plan) {
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
    const int half = blockIdx.x % NSPLIT, j0 = half * DVT;
    const SegJob &job = plan.job[blockIdx.y];
    const int nc = plan.nc, cb = job.c0, ncj = job.nch;  // chunks cb .. cb + ncj - 1 of nc
    const int gt_kind = (plan.njobs > 1 && plan.job[1].pair) ? 2 : 3;
    EFLA_GT_BEGIN(gt_kind);
    if (job.pair) {
        pair_run(sm, tm_k, ws, job, nc, bh, half);
        EFLA_CTA(gt_kind, 1);
        EFLA_GT_END(gt_kind);
        return;
    }

    if (threadIdx.x == 0) {
        *abort_flag = 0;
        for (int s = 0; s < 2; ++s) {
            mbar_init(&bar[B_FULLA + s], 1);
            mbar_init(&bar[B_FULLB + s], 1);
            mbar_init(&bar[B_EMPTYA + s], 1);
            mbar_init(&bar[B_EMPTYB + s], 1);
            mbar_init(&bar[B_OREAD + s], 4);  // the 4 O warps
            mbar_init(&bar[B_OFULL + s], 1);
        }
        mbar_init(&bar[B_SBFULL], 8);  // one arrival per converter warp
        mbar_init(&bar[B_DFULL], 1);
        mbar_init(&bar[B_DELTA], 4);  // the 4 D warps
        mbar_init(&bar[B_SFULL], 1);
        mbar_init(&bar[B_DRAIN], 1);
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(tmem_slot, TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    // Launched as a programmatic dependent of the grid before it (the prep
    // kernel, or the segment chain): the prologue above overlaps that grid's
    // last wave; nothing it wrote is read before this wait returns.
    asm volatile("griddepcontrol.wait;" ::: "memory");
    EFLA_CTA(gt_kind, 0);

    if (warp < 8) {
        // ------------------------------------------------------------ TMEM <-> smem warps
        // Warp w owns TMEM lanes 32 (w % 4) .. + 31 and columns 32 (w / 4) .. + 31
        // of every 64-column tile.
        const int quad = warp & 3, cpart = warp >> 2, c0 = 32 * cpart;
        const int row = 32 * quad + lane;  // TMEM lane: state row, or chunk row (+64 for D)
        const uint32_t tl = tmem + ((uint32_t)(32 * quad) << 16);
        const bool dwarp = quad >= 2;  // lanes 64..127: the D rows of Y
        float x[32];
        {   // initial state: zero, given, or the identity (columns j0 + c0 .. of row `row`)
            const float *src = job.s0_kind == 1 ? job.s0 + ((size_t)bh * DK + row) * DK + j0 + c0 : nullptr;
#pragma unroll
            for (int c = 0; c < 32; c += 4) {
                const float4 v = src ? *reinterpret_cast<const float4 *>(src + c) : make_float4(0.f, 0.f, 0.f, 0.f);
                x[c] = v.x;
                x[c + 1] = v.y;
                x[c + 2] = v.z;
                x[c + 3] = v.w;
            }
            if (job.s0_kind == 2) {
#pragma unroll
                for (int c = 0; c < 32; ++c) x[c] = (row == j0 + c0 + c) ? 1.f : 0.f;
            }
            uint32_t r[32];
#pragma unroll
            for (int i = 0; i < 32; ++i) r[i] = __float_as_uint(x[i]);
            tmem_st32(tl + T_S + c0, r);  // S_a = S0
#pragma unroll
            for (int i = 0; i < 32; ++i) r[i] = 0u;
            tmem_st32(tl + T_S + 64 + c0, r);  // S_b = 0
            tmem_st_wait();
            write_split32(sm + OFF_SB, 2 * SLOT, row, 4 * cpart, x);
            fence_proxy_async();
            tc_fence_before();
            warp_arrive(&bar[B_SBFULL]);
        }
        // A state-row warp (quads 2, 3) leaves the loop on its own when a wait
        // fails: no barrier inside the loop ties it to the others.  The O
        // warps (quads 0, 1) share the staging tile through named barrier 3,
        // so they leave together, on the vote taken before it.  A failed wait
        // sets the abort flag, which makes every other wait give up at once.
        for (int n = 0; n < ncj; ++n) {
            const int b = n & 1;
            const uint32_t ty = T_Y + 128 * b + c0;
            if (dwarp) {
                // D = U + (-W S): TMEM lanes 64..127 of Y, plus U from the stage
                const int c = row - 64;
                // (the stage's own barrier too: U landed by the bulk copy is
                // visible to the threads that observe that barrier's phase)
                if (!warp_wait(&bar[B_FULLB + b], (n >> 1) & 1, abort_flag)) break;
                if (!warp_wait(&bar[B_DFULL], n & 1, abort_flag)) break;
                if (row == 64 && cpart == 0) EFLA_TR(28, n);
                tc_fence_after();
                uint32_t r[32], r2[32];
                tmem_ld32(tl + ty, r);        // -W S_hi
                tmem_ld32(tl + ty + 64, r2);  // -W S_lo
                const unsigned char *urow = sm + b * STAGE + SL_U * SLOT + c * 256;
                float u[32];
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const float4 v =
                        *reinterpret_cast<const float4 *>(urow + (((uint32_t)(8 * cpart + j) ^ (c & 15)) << 4));
                    u[4 * j] = v.x;
                    u[4 * j + 1] = v.y;
                    u[4 * j + 2] = v.z;
                    u[4 * j + 3] = v.w;
                }
                tmem_ld_wait(r);
                tmem_ld_wait(r2);
#pragma unroll
                for (int i = 0; i < 32; ++i) x[i] = u[i] + (__uint_as_float(r[i]) + __uint_as_float(r2[i]));
                write_split32(sm + OFF_DB + b * 2 * SLOT, SLOT, c, 4 * cpart, x);
                fence_proxy_async();
                tc_fence_before();
                warp_arrive(&bar[B_DELTA]);
                if (row == 64 && cpart == 0) EFLA_TR(11, n);
            }
            const bool ok = warp_wait(&bar[B_SFULL], n & 1, abort_flag);
            if (row == 64 && cpart == 0) EFLA_TR(12, n);
            if (!ok && dwarp) break;
            if (ok) {
                tc_fence_after();
                uint32_t r[32], r2[32];
                tmem_ld32(tl + T_S + c0, r);        // S_a
                tmem_ld32(tl + T_S + 64 + c0, r2);  // S_b
                tmem_ld_wait(r);
                tmem_ld_wait(r2);
                if (row == 64 && cpart == 0) EFLA_TR(30, n);
#pragma unroll
                for (int i = 0; i < 32; ++i) x[i] = __uint_as_float(r[i]) + __uint_as_float(r2[i]);
                write_split32(sm + OFF_SB, 2 * SLOT, row, 4 * cpart, x);
                if (row == 64 && cpart == 0) EFLA_TR(31, n);
                fence_proxy_async();
                tc_fence_before();
                warp_arrive(&bar[B_SBFULL]);
                if (row == 64 && cpart == 0) EFLA_TR(13, n);
            }
            if (ok && n == ncj - 1 && job.sl) {
                float *dst = job.sl + ((size_t)bh * DK + row) * DK + j0 + c0;
#pragma unroll
                for (int c = 0; c < 32; c += 4)
                    *reinterpret_cast<float4 *>(dst + c) = make_float4(x[c], x[c + 1], x[c + 2], x[c + 3]);
            }
            if (!dwarp) {
                // O = Q S + M D: TMEM lanes 0..63 of Y -> staging tile -> one TMA
                // store (rows past L are clipped by the tensor map).  The staging
                // tile is rewritten only after the previous store has read it.
                const bool storer = warp == 0 && lane == 0;
                const bool okO = ok && mbar_wait(&bar[B_OFULL + b], (n >> 1) & 1, abort_flag);
                if (storer) bulk_wait_read0();
                if (bar_any(3, 128, !okO || *abort_flag)) break;
                {
                    tc_fence_after();
                    uint32_t r[32], r2[32];
                    tmem_ld32(tl + ty, r);        // Q S_hi + M D_hi
                    tmem_ld32(tl + ty + 64, r2);  // Q S_lo + M D_lo
                    tmem_ld_wait(r);
                    tmem_ld_wait(r2);
                    tc_fence_before();
                    warp_arrive(&bar[B_OREAD + b]);
#pragma unroll
                    for (int i = 0; i < 32; ++i) r[i] = __float_as_uint(__uint_as_float(r[i]) + __uint_as_float(r2[i]));
                    if (row == 0 && cpart == 0) EFLA_TR(14, n);
                    // staging: 128-byte-swizzled boxes of 128-byte rows -- fp32: two
                    // 32-column boxes (one per column half c0); bf16: one 64-column box
                    if constexpr (sizeof(Tout) == 4) {
                        unsigned char *orow = sm + OFF_OST + cpart * SLOT + row * 128;
#pragma unroll
                        for (int i = 0; i < 8; ++i)
                            *reinterpret_cast<uint4 *>(orow + ((i ^ (row & 7)) << 4)) =
                                make_uint4(r[4 * i], r[4 * i + 1], r[4 * i + 2], r[4 * i + 3]);
                    } else {
                        unsigned char *orow = sm + OFF_OST + row * 128;
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            const float *f = reinterpret_cast<const float *>(&r[8 * i]);
                            *reinterpret_cast<uint4 *>(orow + (((4 * cpart + i) ^ (row & 7)) << 4)) =
                                make_uint4(ptx::pack_bf16(f[0], f[1]), ptx::pack_bf16(f[2], f[3]),
                                           ptx::pack_bf16(f[4], f[5]), ptx::pack_bf16(f[6], f[7]));
                        }
                    }
                    fence_proxy_async();
                    named_bar(3, 128);
                    if (storer && job.write_o) {
                        tma_store_3d(&tm_o, sm + OFF_OST, j0, (cb + n) * C, (int)bh);
                        if constexpr (sizeof(Tout) == 4)
                            tma_store_3d(&tm_o, sm + OFF_OST + SLOT, j0 + 32, (cb + n) * C, (int)bh);
                        bulk_commit();
                    }
                }
            }
        }
    } else if (warp == 8) {
        // ------------------------------------------------------------ MMA issuer
        // The whole warp runs the loop and waits (a lone lane waiting while
        // its 31 siblings sit at a convergence point notices completed
        // barrier phases late); lane 0 issues every tcgen05.mma and commit.
        // Descriptors: the 14-bit start-address field holds addr >> 4, and
        // shared addresses stay below 256 KB, so the field never carries: the
        // descriptor of (addr + off) is desc(addr) + (off >> 4).  Each product
        // builds its base descriptors once; the unrolled k-steps add
        // compile-time offsets, keeping the issuing lane ahead of the pipe.
        const bool leader = lane == 0;
        // N = 128 operands [S_hi | S_lo] (the lo tile 16 KB after hi) and
        // [D_hi | D_lo] (8 KB apart): the leading byte offset of the
        // MN-major descriptor steps from the first 64 columns to the second.
        const uint64_t dSB = sdesc_sw128(sbase + OFF_SB, 2 * SLOT, 1024);
        const uint64_t dDB = sdesc_sw128(sbase + OFF_DB, SLOT, 1024);
        // O += M (D_hi + D_lo) of chunk m: issued behind Y of chunk m+1, so it
        // runs while the state warps convert D of chunk m+1 (its readers then
        // wait a little longer, the state chain does not).
        auto issue_O = [&](int m) {
            const int b = m & 1;
            const uint64_t dM = sdesc_sw128(sbase + (uint32_t)b * STAGE + SL_M * SLOT, 16, 1024);
            const uint64_t dD = dDB + ((b * 2 * SLOT) >> 4);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
                mma_bf16(tmem + T_Y + 128 * b, dM + ((kk * 32) >> 4), dD + ((kk * 2048) >> 4), ID_Y, 1);
            mma_commit(&bar[B_OFULL + b]);
            mma_commit(&bar[B_EMPTYB + b]);
        };
        int n = 0;
        for (; n < ncj; ++n) {
            const int s = n & 1;
            const uint32_t sa = sbase + (uint32_t)s * STAGE, ty = tmem + T_Y + 128 * s;
            // Y = [Q; -W] (S_hi + S_lo) after: part A of the stage landed, O of
            // chunk n-2 left this Y buffer (both long done: waited while the
            // state warps still convert S), the bf16 state of chunk n written.
            if (!warp_wait(&bar[B_FULLA + s], (n >> 1) & 1, abort_flag)) break;
            if (n >= 2 && !warp_wait(&bar[B_OREAD + s], ((n - 2) >> 1) & 1, abort_flag)) break;
            if (leader) EFLA_TR(22, n);
            if (!warp_wait(&bar[B_SBFULL], n & 1, abort_flag)) break;
            tc_fence_after();
            if (leader) {
                EFLA_TR(20, n);
                const uint64_t dA = sdesc_sw128(sa + SL_Q0 * SLOT, 16, 1024);
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    mma_bf16(ty, dA + (((kk >> 2) * 2 * SLOT + (kk & 3) * 32) >> 4), dSB + ((kk * 2048) >> 4), ID_Y,
                             kk);
                mma_commit(&bar[B_DFULL]);
                mma_commit(&bar[B_EMPTYA + s]);
                EFLA_TR(24, n);
                if (n >= 1) issue_O(n - 1);
            }
            __syncwarp();
            // S += K^T (D_hi + D_lo) after part B landed (K) and D was written
            if (!warp_wait(&bar[B_FULLB + s], (n >> 1) & 1, abort_flag)) break;
            if (!warp_wait(&bar[B_DELTA], n & 1, abort_flag)) break;
            tc_fence_after();
            if (leader) {
                EFLA_TR(21, n);
                const uint64_t dKt = sdesc_sw128(sa + SL_K0 * SLOT, SLOT, 1024);
                const uint64_t dD = dDB + ((s * 2 * SLOT) >> 4);
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    mma_bf16(tmem + T_S, dKt + ((kk * 2048) >> 4), dD + ((kk * 2048) >> 4), ID_S, 1);
                mma_commit(&bar[B_SFULL]);
                EFLA_TR(25, n);
            }
            __syncwarp();
        }
        if (n == ncj && leader) issue_O(ncj - 1);
        __syncwarp();
        // drain: wait (bounded, even after an abort) until every MMA issued has completed
        if (leader) mma_commit(&bar[B_DRAIN]);
        __syncwarp();
        int never = 0;
        mbar_wait(&bar[B_DRAIN], 0, &never);
    } else {
        // ------------------------------------------------------------ TMA producer
        // Whole warp in the loop; lane 0 issues the copies.
        const bool leader = lane == 0;
        if (leader) {
            tma_prefetch(&tm_q);
            tma_prefetch(&tm_k);
        }
        const unsigned char *img = ws + (size_t)bh * nc * PREP_BYTES;
        int lastA[2] = {-1, -1}, lastB[2] = {-1, -1};  // last chunk loaded per stage and part
        for (int n = 0; n < ncj; ++n) {
            const int s = n & 1;
            unsigned char *st = sm + s * STAGE;
            const int y = (cb + n) * C, z = (int)bh;
            const unsigned char *src = img + (size_t)(cb + n) * PREP_BYTES;
            // part A: Q and -W, once Y of chunk n-2 no longer reads them
            if (n >= 2 && !warp_wait(&bar[B_EMPTYA + s], ((n >> 1) - 1) & 1, abort_flag)) break;
            if (__any_sync(0xffffffffu, *abort_flag != 0)) break;
            if (leader) {
                uint64_t *fb = &bar[B_FULLA + s];
                mbar_expect_tx(fb, TX_A);
                tma_load_3d(st + SL_Q0 * SLOT, &tm_q, fb, 0, y, z);
                tma_load_3d(st + (SL_Q0 + 2) * SLOT, &tm_q, fb, 64, y, z);
                bulk_load(st + SL_W0 * SLOT, src + IMG_W, SLOT, fb);
                bulk_load(st + (SL_W0 + 2) * SLOT, src + IMG_W + SLOT, SLOT, fb);
                EFLA_TR(27, n);
            }
            __syncwarp();
            lastA[s] = n;
            // part B: K, M and U, once chunk n-2 is finished with them
            if (n >= 2 && !warp_wait(&bar[B_EMPTYB + s], ((n >> 1) - 1) & 1, abort_flag)) break;
            if (__any_sync(0xffffffffu, *abort_flag != 0)) break;
            if (leader) {
                uint64_t *fb = &bar[B_FULLB + s];
                mbar_expect_tx(fb, TX_B);
                tma_load_3d(st + SL_K0 * SLOT, &tm_k, fb, 0, y, z);
                tma_load_3d(st + (SL_K0 + 1) * SLOT, &tm_k, fb, 64, y, z);
                bulk_load(st + SL_M * SLOT, src + IMG_M, SLOT, fb);
                bulk_load(st + SL_U * SLOT, src + IMG_U + half * UHALF, UHALF, fb);
            }
            __syncwarp();
            lastB[s] = n;
        }
        // drain: every copy this warp started has landed before the CTA exits
        // (a load is issued only after the previous one of its stage and part
        // was consumed, so the last one issued is the only one that can be pending)
        int never = 0;
        for (int s = 0; s < 2; ++s) {
            if (lastA[s] >= 0) mbar_wait(&bar[B_FULLA + s], (lastA[s] >> 1) & 1, &never);
            if (lastB[s] >= 0) mbar_wait(&bar[B_FULLB + s], (lastB[s] >> 1) & 1, &never);
        }
    }
    if (threadIdx.x == 0) bulk_wait_read0();  // the O stores this thread issued have read the staging tile
    __syncwarp();
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, TMEM_COLS);
    }
    EFLA_CTA(gt_kind, 1);
    EFLA_GT_END(gt_kind);
}

// ---------------------------------------------------------------- prep kernel
constexpr int kPrepThreads = 256;
constexpr int kCopyThread = 224;  // lane 0 of warp 7, idle during the diagonal solves
// Shared memory of one prep CTA (base aligned to 1024 B):
//   [0, 32K)   K0 Q0 K1 Q1 (64 x 64 bf16 boxes, 128-byte swizzle): [K; Q] is
//              the 128-row A operand of [K; Q] K^T per d_k half, K also its B;
//              V0 and V1 later land over Q0 and Q1; -W is staged over K0 and
//              K1, then U's second half over V0 and V1
//   [32K, 48K) A (fp32, Sw64), then T in place, then T' hi and lo boxes,
//              then U's first half
//   [48K, 52K) A's diagonal blocks (diag_index), then scratch of the solve
constexpr uint32_t P_KQ = 0, P_AT = 4 * SLOT, P_AD = 6 * SLOT, P_ALPHA = P_AD + 4096, P_BAR = P_ALPHA + 256;
constexpr uint32_t P_SMEM = P_BAR + 64 + 1024;  // + barriers, TMEM slot, abort flag; + alignment slack
constexpr uint32_t P_TMEM_COLS = 128;           // G (columns 0-63), then W, then U (0-127)
constexpr uint32_t ID_G = ptx::idesc_bf16(128, 64, false, false);  // [K; Q] K^T
// T' K and T' V: M = 64 (T' rows), N = 128, B MN-major.  An M = 64
// accumulator keeps row i in TMEM lane (i % 16) + 32 (i / 16), its N
// columns contiguous (the first 16 lanes of each warp's 32-lane quarter).
constexpr uint32_t ID_WU = ptx::idesc_bf16(64, 128, false, true);

// Byte offset of element (r, c) in a 64-column bf16 box with the 128-byte swizzle.
__device__ __forceinline__ uint32_t sw128_elem(int r, int c) {
    return (uint32_t)r * 128u + ((((uint32_t)c >> 3) ^ ((uint32_t)r & 7u)) << 4) + ((uint32_t)c & 7u) * 2u;
}

// Everything about one chunk that does not depend on the state, written as
// the workspace image chunk_tc_kernel reads (rows past L are zero):
//   alpha = gate(beta, ||k||^2)
//   G = [K; Q] K^T                      (tcgen05: A = [K; Q], B = K)
//   A = strictly-lower(diag(alpha) K K^T),  M = lower-incl-diag(Q K^T)  (bf16)
//   T = (I + A)^{-1},  T' = T diag(alpha)   (CUDA cores + mma.sync TF32)
//   W = T' K,  U = T' V                 (tcgen05, M = 64: A = T' as bf16 hi + lo, B = K / V)
//   -> -W (bf16), U (fp32)
// One 256-thread CTA per (b, h, chunk); thread 0 issues the TMA loads and the
// tcgen05 products, all eight warps share the TMEM read-outs and the solve.
__global__ void __launch_bounds__(kPrepThreads, 4) chunk_prep_tc_kernel(const __grid_constant__ CUtensorMap tm_q,
                                                                     const __grid_constant__ CUtensorMap tm_k,
                                                                     const __grid_constant__ CUtensorMap tm_v,
                                                                     const float *__restrict__ beta,
                                                                     unsigned char *__restrict__ ws, int L, int nc,
                                                                     int c_begin, int c_count, int euler) {
    using namespace ptx;
    extern __shared__ unsigned char psm_raw[];
    unsigned char *sm =
        reinterpret_cast<unsigned char *>((reinterpret_cast<uintptr_t>(psm_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(sm);
    float *alpha = reinterpret_cast<float *>(sm + P_ALPHA);
    float *Ad = reinterpret_cast<float *>(sm + P_AD);
    const Sw64 AT{reinterpret_cast<float *>(sm + P_AT)};
    // barriers 0: K, Q landed  1: V landed  2: G done  3: W done  4: U done  5: drain
    uint64_t *bar = reinterpret_cast<uint64_t *>(sm + P_BAR);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + P_BAR + 48);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(sm + P_BAR + 52);
    const int p = threadIdx.x, w = p >> 5, lane = p & 31;
    // chunks c_begin .. c_begin + c_count - 1 of every (b, h); 32-bit quotient
    // and remainder (grid < 2^31; a 64-bit division is a long instruction
    // sequence on the slow conversion pipe)
    const unsigned q32 = blockIdx.x / (unsigned)c_count;
    const int chunk = c_begin + (int)(blockIdx.x - q32 * (unsigned)c_count);
    const long bh = (long)q32;
    const long gidx = bh * nc + chunk;
    EFLA_GT_BEGIN(c_begin == 0 ? 0 : 1);
    const int t0 = chunk * C, n = min(C, L - t0);
    const size_t row0 = (size_t)bh * L + t0;
    if (p == 0) EFLA_TR(49, 1023);
    // the serial kernel may be scheduled once every prep CTA is running (it
    // waits for this grid's completion before reading the workspace)
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    if (p == 0) {
        *abort_flag = 0;
        for (int i = 0; i < 6; ++i) mbar_init(&bar[i], 1);
        fence_mbar_init();
        tma_prefetch(&tm_q);
        tma_prefetch(&tm_k);
        tma_prefetch(&tm_v);
        mbar_expect_tx(&bar[0], 4 * SLOT);
        tma_load_3d(sm + P_KQ, &tm_k, &bar[0], 0, t0, (int)bh);
        tma_load_3d(sm + P_KQ + SLOT, &tm_q, &bar[0], 0, t0, (int)bh);
        tma_load_3d(sm + P_KQ + 2 * SLOT, &tm_k, &bar[0], 64, t0, (int)bh);
        tma_load_3d(sm + P_KQ + 3 * SLOT, &tm_q, &bar[0], 64, t0, (int)bh);
    }
    if (w == 0) {
        tmem_alloc(tmem_slot, P_TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    // bounded wait by every thread; the answer is block-uniform
    auto wait_all = [&](int i, uint32_t parity) { return !__syncthreads_or(!mbar_wait(&bar[i], parity, abort_flag)); };
    bool issued_v = false, issued_mma = false;  // (copy thread / thread 0) for the drain after a failure
    // beta of the key row this thread gates (four lanes per row, lane 0 of
    // each four loads it), fetched while K and Q are still landing
    const float beta_r = ((p & 3) == 0 && (p >> 2) < n) ? beta[row0 + (p >> 2)] : 0.f;
    bool ok = wait_all(0, 0);
    if (p == 0) EFLA_TR(50, 1023);
    if (p == 0 && ok) {  // G = [K; Q] K^T: 8 k-steps over d_k
        tc_fence_after();
        const uint64_t d0 = sdesc_sw128(sbase + P_KQ, 16, 1024);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
            const uint64_t d = d0 + (((kk >> 2) * 2 * SLOT + (kk & 3) * 32) >> 4);
            mma_bf16(tmem, d, d, ID_G, kk > 0);
        }
        mma_commit(&bar[2]);
        issued_mma = true;
    }
    if (ok) {   // gate from the K tile: four lanes per key row; 16-byte chunk c of
                // row r sits in box c / 8 at position (c % 8) ^ (r % 8)
        const int r = p >> 2, h = p & 3;
        float acc8[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int c = 4 * h + j;
            float f[8];
            unpack8(*reinterpret_cast<const uint4 *>(sm + P_KQ + (c >> 3) * 2 * SLOT + sw128_chunk(r, c & 7)), f);
#pragma unroll
            for (int e = 0; e < 8; ++e) acc8[e] = fmaf(f[e], f[e], acc8[e]);
        }
        float ss = ((acc8[0] + acc8[1]) + (acc8[2] + acc8[3])) + ((acc8[4] + acc8[5]) + (acc8[6] + acc8[7]));
        ss += __shfl_xor_sync(0xffffffffu, ss, 1);
        ss += __shfl_xor_sync(0xffffffffu, ss, 2);
        if (h == 0) alpha[r] = (r < n) ? gate_alpha(beta_r, ss, euler != 0) : 0.f;
    }
    ok = ok && wait_all(2, 0);  // (also publishes alpha)
    if (p == 0) EFLA_TR(40, 1023);
    tc_fence_after();
    unsigned char *out = ws + (size_t)gidx * PREP_BYTES;
    const int quad = w & 3, cpart = w >> 2;
    if (ok) {
        // G read-out: lanes 0-63 hold K K^T rows (-> A and its diagonal-block
        // copy), lanes 64-127 Q K^T rows (-> M); warp (quad, cpart) takes
        // columns 32 cpart .. + 31
        uint32_t r32[32];
        tmem_ld32(tmem + ((uint32_t)(32 * quad) << 16) + 32 * cpart, r32);
        tmem_ld_wait(r32);
        if (quad < 2) {
            // row i (block b = i / 16) against the warp's two 16-column blocks
            // bj = 2 cpart, 2 cpart + 1: the diagonal block goes to Ad (its
            // strictly lower part, fp32, one column m at a time: diag_index
            // steps by 16 per column), blocks left of it to AT (only ever a TF32
            // operand: stored rounded, four columns at a time), blocks right of
            // it nowhere
            const int i = 32 * quad + lane, b = i >> 4, rl = i & 15;
            const float ai = alpha[i];
            float *adr = Ad + diag_index(b, 0, rl);
#pragma unroll
            for (int xb = 0; xb < 2; ++xb) {
                const int bj = 2 * cpart + xb;
                if (bj == b) {
#pragma unroll
                    for (int m = 0; m < 16; ++m) adr[16 * m] = (m < rl) ? ai * __uint_as_float(r32[16 * xb + m]) : 0.f;
                } else if (bj < b) {
#pragma unroll
                    for (int m = 0; m < 16; m += 4) {
                        const uint32_t *g = &r32[16 * xb + m];
                        *reinterpret_cast<float4 *>(AT.at(i, 16 * bj + m)) =
                            make_float4(__uint_as_float(f2tf32(ai * __uint_as_float(g[0]))),
                                        __uint_as_float(f2tf32(ai * __uint_as_float(g[1]))),
                                        __uint_as_float(f2tf32(ai * __uint_as_float(g[2]))),
                                        __uint_as_float(f2tf32(ai * __uint_as_float(g[3]))));
                    }
                }
            }
        } else {
            const int i = 32 * (quad - 2) + lane;
#pragma unroll
            for (int c8 = 0; c8 < 4; ++c8) {
                uint32_t v4[4];
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int x = 8 * c8 + 2 * u, j = 32 * cpart + x;
                    v4[u] = pack_bf16((j <= i) ? __uint_as_float(r32[x]) : 0.f,
                                      (j + 1 <= i) ? __uint_as_float(r32[x + 1]) : 0.f);
                }
                // staged in the Q0 box (free once G is done), stored by one bulk copy
                *reinterpret_cast<uint4 *>(sm + P_KQ + SLOT + sw128_elem(i, 32 * cpart + 8 * c8)) =
                    make_uint4(v4[0], v4[1], v4[2], v4[3]);
            }
        }
        fence_proxy_async();
    }
    tc_fence_before();
    __syncthreads();
    if (p == kCopyThread && ok) {
        // M out; then V over Q (Q0 once M has been read out of it), landing while T is solved
        bulk_store(out + IMG_M, sm + P_KQ + SLOT, SLOT);
        bulk_commit();
        bulk_wait_read0();
        mbar_expect_tx(&bar[1], 2 * SLOT);
        tma_load_3d(sm + P_KQ + SLOT, &tm_v, &bar[1], 0, t0, (int)bh);
        tma_load_3d(sm + P_KQ + 3 * SLOT, &tm_v, &bar[1], 64, t0, (int)bh);
        issued_v = true;
    }
    if (p == 0) EFLA_TR(51, 1023);
    if (ok) {
        invert_unit_lower<kPrepThreads>(p, Ad, AT);
        if (p == 0) EFLA_TR(52, 1023);
        // T' = T diag(alpha) (lower triangle) as 128-byte-swizzled bf16 hi and
        // lo boxes (rows i, 64 columns j: the K-major A operand), written over
        // T once every thread holds its part of T
        float tv[2][8];
#pragma unroll
        for (int it = 0; it < 2; ++it) {
            const int e = p + kPrepThreads * it, r = e >> 3, jj = e & 7;
            const float4 ta = *reinterpret_cast<const float4 *>(AT.at(r, 8 * jj));
            const float4 tb = *reinterpret_cast<const float4 *>(AT.at(r, 8 * jj + 4));
            tv[it][0] = ta.x, tv[it][1] = ta.y, tv[it][2] = ta.z, tv[it][3] = ta.w;
            tv[it][4] = tb.x, tv[it][5] = tb.y, tv[it][6] = tb.z, tv[it][7] = tb.w;
        }
        __syncthreads();
#pragma unroll
        for (int it = 0; it < 2; ++it) {
            const int e = p + kPrepThreads * it, r = e >> 3, jj = e & 7;
            uint32_t h4[4], l4[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int c = 8 * jj + 2 * u;
                split2((c <= r) ? tv[it][2 * u] * alpha[c] : 0.f, (c + 1 <= r) ? tv[it][2 * u + 1] * alpha[c + 1] : 0.f,
                       h4[u], l4[u]);
            }
            *reinterpret_cast<uint4 *>(sm + P_AT + sw128_chunk(r, jj)) = make_uint4(h4[0], h4[1], h4[2], h4[3]);
            *reinterpret_cast<uint4 *>(sm + P_AT + SLOT + sw128_chunk(r, jj)) = make_uint4(l4[0], l4[1], l4[2], l4[3]);
        }
        fence_proxy_async();
    }
    if (p == 0) EFLA_TR(53, 1023);
    ok = ok && wait_all(1, 0);  // (also orders the T' image before the products)
    // W = (T'_hi + T'_lo) K, then U = (T'_hi + T'_lo) V in the same columns:
    // 4 k-steps over the chunk, hi and lo; B = the K or V tile, MN-major
    // (d columns 0-63 and 64-127 two swizzled boxes apart)
    auto issue_wu = [&](uint32_t tile, int done) {
        tc_fence_after();
        const uint64_t dB = sdesc_sw128(sbase + P_KQ + tile, 2 * SLOT, 1024);
        const uint64_t dT = sdesc_sw128(sbase + P_AT, 16, 1024);
#pragma unroll
        for (int part = 0; part < 2; ++part)
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
                mma_bf16(tmem, dT + ((part * SLOT + kk * 32) >> 4), dB + ((kk * 2048) >> 4), ID_WU, part | kk);
        mma_commit(&bar[done]);
    };
    // row i of W / U sits in TMEM lane (i % 16) + 32 (i / 16): warp (quad,
    // cpart) lanes 0-15 hold rows 16 quad + lane, columns 64 cpart .. + 63
    // (= the bf16 box / fp32 half cpart of the image)
    const int wrow = 16 * quad + (lane & 15);
    const bool wlane = lane < 16;
    const uint32_t tq = tmem + ((uint32_t)(32 * quad) << 16) + 64 * cpart;
    if (p == 0 && ok) issue_wu(0, 3);
    ok = ok && wait_all(3, 0);
    if (p == 0) EFLA_TR(41, 1023);
    tc_fence_after();
    if (ok) {
#pragma unroll
        for (int h = 0; h < 2; ++h) {  // 32 columns at a time
            uint32_t r32[32];
            tmem_ld32(tq + 32 * h, r32);
            tmem_ld_wait(r32);
            if (wlane) {  // staged in the K box of the same d_k half (K is no longer read)
                unsigned char *dst = sm + P_KQ + cpart * 2 * SLOT + wrow * 128;
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    uint32_t v4[4];
#pragma unroll
                    for (int u = 0; u < 4; ++u)
                        v4[u] = pack_bf16(-__uint_as_float(r32[8 * c + 2 * u]), -__uint_as_float(r32[8 * c + 2 * u + 1]));
                    *reinterpret_cast<uint4 *>(dst + (((4 * h + c) ^ (wrow & 7)) << 4)) =
                        make_uint4(v4[0], v4[1], v4[2], v4[3]);
                }
            }
        }
    }
    fence_proxy_async();
    tc_fence_before();
    __syncthreads();
    if (p == 0 && ok) {
        bulk_store(out + IMG_W, sm + P_KQ, SLOT);
        bulk_store(out + IMG_W + SLOT, sm + P_KQ + 2 * SLOT, SLOT);
        bulk_commit();
        issue_wu(SLOT, 4);
        EFLA_TR(42, 1023);
    }
    ok = ok && wait_all(4, 0);
    if (p == 0) EFLA_TR(43, 1023);
    tc_fence_after();
    if (ok) {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            uint32_t r32[32];
            tmem_ld32(tq + 32 * h, r32);
            tmem_ld_wait(r32);
            if (wlane) {  // staged: half 0 over T', half 1 over V0 (rows 0-31) and V1 (rows 32-63),
                          // all free once U is done; the K boxes may still be in the W store
                unsigned char *dst = cpart ? sm + P_KQ + SLOT + (wrow >> 5) * 2 * SLOT + (wrow & 31) * 256
                                           : sm + P_AT + wrow * 256;
#pragma unroll
                for (int c = 0; c < 8; ++c)
                    *reinterpret_cast<uint4 *>(dst + (((8 * h + c) ^ (wrow & 15)) << 4)) =
                        make_uint4(r32[4 * c], r32[4 * c + 1], r32[4 * c + 2], r32[4 * c + 3]);
            }
        }
    }
    fence_proxy_async();
    __syncthreads();
    if (p == 0 && ok) {
        bulk_store(out + IMG_U, sm + P_AT, UHALF);
        bulk_store(out + IMG_U + UHALF, sm + P_KQ + SLOT, SLOT);
        bulk_store(out + IMG_U + UHALF + SLOT, sm + P_KQ + 3 * SLOT, SLOT);
        bulk_commit();
    }
    // shared memory stays valid until every bulk store has read it; the writes
    // themselves are published by the grid's completion (the serial kernel
    // reads them after griddepcontrol.wait)
    if (p == 0 || p == kCopyThread) bulk_wait_read0();
    if (p == 0) EFLA_TR(54, 1023);
    if (!ok) {
        // after a failed wait: every TMA load issued lands and every product
        // completes before the CTA exits (bounded waits that ignore the abort)
        int never = 0;
        if (p == 0) {
            mbar_wait(&bar[0], 0, &never);
            if (issued_mma) {
                mma_commit(&bar[5]);
                mbar_wait(&bar[5], 0, &never);
            }
        }
        if (p == kCopyThread && issued_v) mbar_wait(&bar[1], 0, &never);
    }
    tc_fence_before();
    __syncthreads();
    if (w == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, P_TMEM_COLS);
    }
    EFLA_GT_END(c_begin == 0 ? 0 : 1);
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

// 3-D view [bh][L][128] of a [B][H][L][128] tensor, boxes of bx columns x 64
// rows with the 128-byte swizzle; rows past L read as zero (loads) and are
// not written (stores).
inline bool make_map(CUtensorMap *m, const void *base, long bh, int L, CUtensorMapDataType dt, int esize,
                     unsigned bx) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return false;
    const cuuint64_t dims[3] = {(cuuint64_t)DK, (cuuint64_t)L, (cuuint64_t)bh};
    const cuuint64_t strides[2] = {(cuuint64_t)DK * esize, (cuuint64_t)L * DK * esize};
    const cuuint32_t box[3] = {bx, 64, 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    return enc(m, dt, 3, const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
               CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}
inline bool make_map_bf16_sw128(CUtensorMap *m, const void *base, long bh, int L) {
    return make_map(m, base, bh, L, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, 64);
}

// Scratch of the tensor-core path: one -W / M / U image per chunk.
// Number of SMs of the current device (looked up once per device).
inline int sm_count() {
    static int cached[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) dev = 0;
    if (!cached[dev]) {
        int n = 0;
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
        cached[dev] = n > 0 ? n : 148;
    }
    return cached[dev];
}

// Segment-parallel prefill for problems with too few heads to fill the GPU.
// The sequence splits into P segments; the state map of segment r is affine,
// S_out = M_r S_in + S_r, with S_r its final state from zero and M_r its final
// state from the identity minus S_r.  Pass A runs, in one launch, segment 0
// from the true S0 (with outputs) and every middle segment from 0 and from I
// (both runs in one CTA per d_v half, pair_run); a chain of small fp32
// products then gives every segment's true initial state,
// S_in(r+1) = M_r S_in(r) + S_r; pass B reruns segments 1..P-1 from those
// with outputs.  Serial latency drops from nc to about 2 nc / P chunks.
// P is the largest value in [3, 8] whose pass A (2 CTAs per segment and
// (b, h)) fits one wave, with at least kMinSegChunks chunks per segment;
// otherwise 1 (a single pass).
constexpr int kMinSegChunks = 16;
// The time of a paired-run chunk (pair_run) relative to a single run's, in
// per cent (clock64 traces: 4.29k cycles per paired-run chunk on the
// long-context prefill against 3.12k per single-run chunk on lm340m).
constexpr long kPairCost = 137;
inline int segments(long bh, int nc) {
    const long sms = sm_count();
    int best = 1;
    for (int p = 3; p <= 8; ++p)
        if (NSPLIT * bh * (p - 1) <= sms && nc / p >= kMinSegChunks) best = p;
    return best;
}
inline size_t state_bytes(long bh) { return (size_t)bh * DK * DK * sizeof(float); }

// Scratch of the tensor-core path: one -W / M / U image per chunk, then (when
// the prefill is segmented) 3P - 5 state buffers: S_in(1..P-1), the final
// states of the middle segments from zero, and from the identity.
inline size_t workspace_bytes(long bh, int L) {
    const int nc = (L + C - 1) / C, P = segments(bh, nc);
    return (size_t)bh * nc * PREP_BYTES + (P > 1 ? (size_t)(3 * P - 5) * state_bytes(bh) : 0);
}

// out = (SI - SZ) X + SZ for every (b, h), D x D fp32 matrices: one step of
// the segment chain.  CTA (bh, column block of 32) computes out[:, 32 cb ..];
// thread (ty, tx) four rows x four columns, the reduction in slabs of 32.
template <int D>
__global__ void __launch_bounds__(256) affine_step_kernel(const float *__restrict__ SI, const float *__restrict__ SZ,
                                                          const float *__restrict__ X, float *__restrict__ out) {
    static_assert(D % 32 == 0 && D <= 128, "D in {32, 64, 128}");
    __shared__ float Ms[D][33];
    __shared__ __align__(16) float Xs[32][36];
    const size_t base = (size_t)blockIdx.x * D * D;
    const int cb = 32 * blockIdx.y, tid = threadIdx.x, ty = tid >> 3, tx = tid & 7;
    const bool active = 4 * ty < D;
    float acc[4][4] = {};
    for (int k0 = 0; k0 < D; k0 += 32) {
        for (int e = tid; e < D * 32; e += 256) {
            const int r = e >> 5, c = e & 31;
            const size_t a = base + (size_t)r * D + k0 + c;
            Ms[r][c] = SI[a] - SZ[a];
        }
        for (int e = tid; e < 32 * 32; e += 256) {
            const int r = e >> 5, c = e & 31;
            Xs[r][c] = X[base + (size_t)(k0 + r) * D + cb + c];
        }
        __syncthreads();
        if (active) {
#pragma unroll 8
            for (int k = 0; k < 32; ++k) {
                const float4 b = *reinterpret_cast<const float4 *>(&Xs[k][4 * tx]);
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const float a = Ms[4 * ty + i][k];
                    acc[i][0] = fmaf(a, b.x, acc[i][0]);
                    acc[i][1] = fmaf(a, b.y, acc[i][1]);
                    acc[i][2] = fmaf(a, b.z, acc[i][2]);
                    acc[i][3] = fmaf(a, b.w, acc[i][3]);
                }
            }
        }
        __syncthreads();
    }
    if (!active) return;
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const size_t a = base + (size_t)(4 * ty + i) * D + cb + 4 * tx + j;
            out[a] = acc[i][j] + SZ[a];
        }
}

// The whole segment chain in one launch: for r = 1 .. steps,
//   X(r+1) = M(r) X(r) + SZ(r),
// with X(1) given, M(r) the segment maps written by the paired runs, and
// consecutive M, SZ and X states `stride` floats apart.  Column block j of
// X(r+1) needs only column block j of X(r), so CTA (bh, column block of 32)
// walks every step on its own, its X block resident in shared memory.  A
// step's whole M(r) (d x d) is loaded at once into shared memory, the next
// step's into registers while the current one is used, so each step waits
// for at most one memory round trip.  Thread (ty, tx) owns four rows x four
// columns.
template <int D>
__global__ void __launch_bounds__(256) affine_chain_kernel(const float *__restrict__ M, const float *__restrict__ SZ,
                                                           float *__restrict__ X, int steps, size_t stride) {
    static_assert(D % 32 == 0 && D <= 128, "D in {32, 64, 128}");
    constexpr int LM = D + 1;                 // row stride of M in shared memory (odd: column reads spread over banks)
    constexpr int NF = D * D / 4 / 256;       // float4s of one step's M per thread
    extern __shared__ __align__(16) float chain_sm[];
    float *Ms = chain_sm;                                          // D x LM
    float(*Xs)[36] = reinterpret_cast<float(*)[36]>(chain_sm + ((D * LM + 3) & ~3));  // D x 32 (+4)
    const size_t base = (size_t)blockIdx.x * D * D;
    const int cb = 32 * blockIdx.y, tid = threadIdx.x, ty = tid >> 3, tx = tid & 7;
    const bool active = 4 * ty < D;
    EFLA_GT_BEGIN(4);
    for (int e = tid; e < D * 32; e += 256) {
        const int r = e >> 5, c = e & 31;
        Xs[r][c] = X[base + (size_t)r * D + cb + c];
    }
    float4 mreg[NF];
    auto fetch = [&](int step) {
        const float4 *m = reinterpret_cast<const float4 *>(M + (size_t)step * stride + base);
#pragma unroll
        for (int x = 0; x < NF; ++x) mreg[x] = m[tid + 256 * x];
    };
    if (steps > 0) fetch(0);
    for (int step = 0; step < steps; ++step) {
        __syncthreads();  // the previous step is done with Ms (and, at step 0, Xs is written)
#pragma unroll
        for (int x = 0; x < NF; ++x) {
            const int e = 4 * (tid + 256 * x), r = e / D, c = e % D;
            float *d = Ms + r * LM + c;
            d[0] = mreg[x].x;
            d[1] = mreg[x].y;
            d[2] = mreg[x].z;
            d[3] = mreg[x].w;
        }
        if (step + 1 < steps) fetch(step + 1);
        // this step's SZ block of the thread, loaded during the product
        float szr[4][4];
        if (active) {
            const float *sz = SZ + (size_t)step * stride + base;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const float4 v = *reinterpret_cast<const float4 *>(sz + (size_t)(4 * ty + i) * D + cb + 4 * tx);
                szr[i][0] = v.x, szr[i][1] = v.y, szr[i][2] = v.z, szr[i][3] = v.w;
            }
        }
        __syncthreads();
        float acc[4][4] = {};
        if (active) {
#pragma unroll 8
            for (int k = 0; k < D; ++k) {
                const float4 b = *reinterpret_cast<const float4 *>(&Xs[k][4 * tx]);
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const float a = Ms[(4 * ty + i) * LM + k];
                    acc[i][0] = fmaf(a, b.x, acc[i][0]);
                    acc[i][1] = fmaf(a, b.y, acc[i][1]);
                    acc[i][2] = fmaf(a, b.z, acc[i][2]);
                    acc[i][3] = fmaf(a, b.w, acc[i][3]);
                }
            }
        }
        __syncthreads();  // every thread is done reading Xs of this step
        if (active) {
            float *out = X + (size_t)(step + 1) * stride + base;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int r = 4 * ty + i;
                const float4 y = make_float4(acc[i][0] + szr[i][0], acc[i][1] + szr[i][1], acc[i][2] + szr[i][2],
                                             acc[i][3] + szr[i][3]);
                *reinterpret_cast<float4 *>(out + (size_t)r * D + cb + 4 * tx) = y;
                *reinterpret_cast<float4 *>(&Xs[r][4 * tx]) = y;
            }
        }
    }
    EFLA_GT_END(4);
}
// Shared memory of affine_chain_kernel<D>.
template <int D>
constexpr size_t chain_smem_bytes() {
    return (size_t)(((D * (D + 1) + 3) & ~3) + D * 36) * sizeof(float);
}

template <typename Tout>
inline efla_status_t launch(const void *q, const void *k, const void *v, const float *beta, const float *S0,
                            void *o, float *SL, long bh, int L, bool euler, void *ws, cudaStream_t st) {
    CUtensorMap mq, mk, mo;
    const bool of32 = sizeof(Tout) == 4;
    if (!make_map_bf16_sw128(&mq, q, bh, L) || !make_map_bf16_sw128(&mk, k, bh, L) ||
        !make_map(&mo, o, bh, L, of32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16,
                  (int)sizeof(Tout), of32 ? 32u : 64u))
        return EFLA_ERR_CUDA;
    CUtensorMap mv;
    if (!make_map_bf16_sw128(&mv, v, bh, L)) return EFLA_ERR_CUDA;
    if (!ensure_smem<chunk_tc_kernel<Tout>>(SMEM_BYTES) || !ensure_smem<chunk_prep_tc_kernel>(P_SMEM) ||
        !ensure_smem<affine_chain_kernel<DK>>(chain_smem_bytes<DK>()))
        return EFLA_ERR_CUDA;
    const long grid = bh * NSPLIT;
    const int nc = (L + C - 1) / C;
    if (grid > 0x7fffffffL || bh * nc > 0x7fffffffL) return EFLA_ERR_SHAPE;
    unsigned char *img = static_cast<unsigned char *>(ws);
    const int P = segments(bh, nc);
    // Segment r covers chunks first(r) .. first(r + 1) - 1.  In pass A a
    // paired-run chunk costs kPairCost (per cent) of a single-run one, so
    // segment 0 (the only single run of pass A) gets that much more: pass A's
    // jobs then end together, and segments 1 .. P-1 split the rest evenly.
    const long seg0 = (long)nc * kPairCost / (kPairCost + 100L * (P - 1));
    auto first = [&](int r) {
        return r == 0 ? 0 : (int)(seg0 + (long)(r - 1) * (nc - seg0) / (P - 1));
    };
    // (A variant that prepared the last segment's images on a side stream,
    // on the SMs pass A leaves free, was measured slower: pass A's serial
    // chains lost more to the contention than the overlap saved.)
    chunk_prep_tc_kernel<<<(unsigned)(bh * nc), kPrepThreads, P_SMEM, st>>>(mq, mk, mv, beta, img, L, nc, 0, nc,
                                                                            euler ? 1 : 0);
    if (cudaGetLastError() != cudaSuccess) return EFLA_ERR_CUDA;
    auto run = [&](const SegPlan &plan) {
        // programmatic stream serialisation: the CTAs may start (and run
        // their prologue) before the previous grid has finished
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3((unsigned)grid, (unsigned)plan.njobs);
        cfg.blockDim = dim3(kThreads);
        cfg.dynamicSmemBytes = SMEM_BYTES;
        cfg.stream = st;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        const unsigned char *cimg = img;
        return cudaLaunchKernelEx(&cfg, chunk_tc_kernel<Tout>, mq, mk, mo, cimg, plan) == cudaSuccess;
    };
    SegPlan plan{};
    plan.nc = nc;
    if (P == 1) {
        plan.njobs = 1;
        plan.job[0] = SegJob{0, nc, S0 ? 1 : 0, 1, S0, SL, 0, nullptr};
        return run(plan) ? EFLA_OK : EFLA_ERR_CUDA;
    }
    float *sbuf = reinterpret_cast<float *>(img + (size_t)bh * nc * PREP_BYTES);
    const size_t sb = state_bytes(bh) / sizeof(float);
    auto Sin = [&](int r) { return sbuf + (size_t)(r - 1) * sb; };               // r = 1 .. P-1
    auto SZ = [&](int r) { return sbuf + (size_t)(P - 1 + r - 1) * sb; };         // r = 1 .. P-2
    auto SI = [&](int r) { return sbuf + (size_t)(2 * P - 3 + r - 1) * sb; };     // r = 1 .. P-2
    // pass A
    plan.njobs = 0;
    plan.job[plan.njobs++] = SegJob{0, first(1), S0 ? 1 : 0, 1, S0, Sin(1), 0, nullptr};
    for (int r = 1; r <= P - 2; ++r)
        plan.job[plan.njobs++] = SegJob{first(r), first(r + 1) - first(r), 0, 0, nullptr, SZ(r), 1, SI(r)};
    if (!run(plan)) return EFLA_ERR_CUDA;
    // the segment chain, one launch: Sin(r + 1) = M(r) Sin(r) + SZ(r), with
    // the paired runs' maps M(r) = S(I)(r) - S(0)(r) in the SI buffers
    // (an ordinary launch: as a programmatic dependent of pass A its first
    // CTAs were scheduled two to an SM on the SMs pass A leaves free, and the
    // chain took 40 instead of 23 µs)
    affine_chain_kernel<DK><<<dim3((unsigned)bh, DK / 32), 256, chain_smem_bytes<DK>(), st>>>(SI(1), SZ(1), Sin(1),
                                                                                           P - 2, sb);
    if (cudaGetLastError() != cudaSuccess) return EFLA_ERR_CUDA;
    // pass B
    plan.njobs = 0;
    for (int r = 1; r <= P - 1; ++r)
        plan.job[plan.njobs++] =
            SegJob{first(r), first(r + 1) - first(r), 1, 1, Sin(r), r == P - 1 ? SL : nullptr, 0, nullptr};
    return run(plan) ? EFLA_OK : EFLA_ERR_CUDA;
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
