// efla_gate.cuh - fused gate / key-normaliser kernel.
//
// For every key row: lambda = ||k||^2 (fp32 accumulation) and the exact-flow
// gate alpha ("Exact Flow Linear Attention", papernotes.org summary,
// 关键设计 2; numerics per 损失函数 / 训练策略, and the jsqmd.com blog's
// advice in section 6 to compile the soft gate into a CUDA kernel).
//
// HBM-bound: 2*d*esize + 12 bytes per row.  A group of G lanes covers one
// row with 16-byte vector loads (G = d*esize/16); each lane keeps UNROLL
// rows in flight; the group reduces with shuffles and its first lane writes
// alpha and lambda.  The grid is a grid-stride loop sized to the SM count.
#pragma once
#include "efla_common.cuh"

namespace efla {

template <typename T, int D, int UNROLL>
__global__ void __launch_bounds__(256) gate_kernel(const T *__restrict__ k, const float *__restrict__ beta,
                                                   float *__restrict__ alpha, float *__restrict__ lambda,
                                                   long rows, bool euler) {
    constexpr int VEC = 16 / sizeof(T);  // elements per 16-byte load
    constexpr int G = D / VEC;           // lanes per row
    static_assert(G >= 1 && G <= 32 && (32 % G) == 0, "row must map onto a lane group");
    constexpr int RPW = 32 / G;          // rows per warp per unrolled slot
    const int lane = threadIdx.x & 31;
    const int sub = lane / G;
    const int gl = lane % G;
    const long warp = ((long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const long nwarp = ((long)gridDim.x * blockDim.x) >> 5;

    for (long base = warp * (RPW * UNROLL); base < rows; base += nwarp * (RPW * UNROLL)) {
        uint4 raw[UNROLL];
        float bt[UNROLL];  // beta, loaded with the keys so its latency overlaps theirs
#pragma unroll
        for (int u = 0; u < UNROLL; ++u) {
            const long r = base + (long)u * RPW + sub;
            if (r < rows)
                raw[u] = __ldcs(reinterpret_cast<const uint4 *>(k + r * D) + gl);
            else
                raw[u] = make_uint4(0u, 0u, 0u, 0u);
            bt[u] = (gl == 0 && r < rows) ? __ldcs(beta + r) : 0.f;
        }
#pragma unroll
        for (int u = 0; u < UNROLL; ++u) {
            const long r = base + (long)u * RPW + sub;
            float s = 0.f;
            const T *e = reinterpret_cast<const T *>(&raw[u]);
#pragma unroll
            for (int i = 0; i < VEC; ++i) {
                const float x = to_f32(e[i]);
                s = fmaf(x, x, s);
            }
#pragma unroll
            for (int o = G / 2; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);  // stays in the group
            if (gl == 0 && r < rows) {
                alpha[r] = gate_alpha(bt[u], s, euler);
                if (lambda) lambda[r] = s;
            }
        }
    }
}

}  // namespace efla
