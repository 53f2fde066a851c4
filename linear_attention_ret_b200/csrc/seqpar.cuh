// Pieces of a sequence split into consecutive segments, each computed separately
// (on other GPUs, or later): the chunkwise recurrence ("RetNet retention
// mechanism" (aiqz.cc), section 块级循环; the gated page's cross_chunk state
// update) composes over segments as
//   S_in(0) = state_in,  S_in(r + 1) = D_r S_in(r) + U_r,
// with U_r the end state of segment r from a zero start and D_r its total decay
// (gamma^{N_r}, or exp of the sum of its gates). These kernels compute log2 D_r
// and the start states S_in(r) from the U_r; the end states come from the
// state-only pass of the tensor-core kernel (tc_chunk.cuh) or from the CUDA-core
// chunkwise kernel.
#pragma once

#include "common.cuh"

namespace ret {

// log2 of a segment's total decay per (b, h): N log2(gamma_h), or log2(e) times the
// sum of g[b, h, 0 .. N-1]. One block per (b, h).
template <bool GATED>
__global__ void __launch_bounds__(256) segment_log2_decay_kernel(const float* __restrict__ decay, float* __restrict__ out,
                                                                 int H, int N) {
    const int bh = blockIdx.x;
    if (!GATED) {
        if (threadIdx.x == 0) out[bh] = N == 0 ? 0.f : log2f(decay[bh % H]) * (float)N;
        return;
    }
    __shared__ float part[8];
    float s = 0.f;
    for (int n = threadIdx.x; n < N; n += blockDim.x) s += decay[(size_t)bh * N + n];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    if ((threadIdx.x & 31) == 0) part[threadIdx.x >> 5] = s;
    __syncthreads();
    if (threadIdx.x < 32) {
        s = threadIdx.x < (blockDim.x >> 5) ? part[threadIdx.x] : 0.f;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
        if (threadIdx.x == 0) out[bh] = s * kLog2e;
    }
}

// Start states of R segments: starts[r] = S_in(r) for r = 0 .. R-1 and, if end is not
// null, end = S_in(R), from seg_states[r] = U_r and seg_log2_decay[r] = log2 D_r.
// One thread per state element (each walks the R segments in order).
__global__ void __launch_bounds__(256)
state_prefix_kernel(const float* __restrict__ seg_states, const float* __restrict__ seg_log2_decay,
                    const float* __restrict__ state_in, float* __restrict__ starts, float* __restrict__ end, int R,
                    int BH, int per_bh) {
    const size_t n = (size_t)BH * per_bh;
    for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x) {
        const int bh = (int)(i / per_bh);
        float x = state_in ? state_in[i] : 0.f;
        for (int r = 0; r < R; ++r) {
            const float u = seg_states[(size_t)r * n + i];
            starts[(size_t)r * n + i] = x;
            x = fmaf(exp2f(seg_log2_decay[(size_t)r * BH + bh]), x, u);
        }
        if (end) end[i] = x;
    }
}

}  // namespace ret
