// Backward pass of chunkwise retention from a zero initial state, built from the
// forward kernels. With w_nm the decay weight of key m for query n (gamma^(n-m),
// or exp(G_n - G_m) for the gated form, "RetNet retention mechanism" (aiqz.cc)
// 保留机制初识 and the Gated RetNet page's parallel_gate_retention) and
// L = sum_n dO_n . O_n:
//   dQ_n = sum_{m<=n} w_nm (dO_n . v_m) k_m   = forward retention of (dO, V, K),
//   dK_m = sum_{n>=m} w_nm (dO_n . v_m) q_n   = time-reversed forward of (V, dO, Q),
//   dV_m = sum_{n>=m} w_nm (q_n . k_m) dO_n   = time-reversed forward of (K, Q, dO),
// and the decay gradient from a_t = q_t . dQ_t - k_t . dK_t = dL/dG_t:
//   gated: dg_t = sum_{u>=t} a_u (G is the cumulative sum of g);
//   fixed: dgamma_h = (1 / gamma_h) sum_{b, t} t a_t.
// Time reversal maps the decay between positions n >= m onto a forward decay: the
// same gamma, or the reversed gates shifted by one (g'_i = g_{N-i}, g'_0 = 0).
// The forward kernels take q/k widths up to 256, so a wider dv is contracted in
// pieces (retention is linear in the scores q . k) whose outputs are summed.
// This file holds the data-movement and reduction kernels of that composition.
#pragma once

#include "common.cuh"

namespace ret {

constexpr int kBwdThreads = 256;

// dst[bh, t, c] = src[bh, flip ? N-1-t : t, c0 + c] for c < w (a contiguous column
// slice, optionally time-reversed). src rows are d_src wide.
template <typename T>
__global__ void __launch_bounds__(kBwdThreads)
slice_flip_kernel(const T* __restrict__ src, T* __restrict__ dst, int N, int d_src, int c0, int w, bool flip,
                  size_t total) {
    for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < total; i += (size_t)gridDim.x * blockDim.x) {
        const int c = (int)(i % w);
        const size_t row = i / w;  // bh * N + t
        const int t = (int)(row % N);
        const size_t bh = row / N;
        const int ts = flip ? N - 1 - t : t;
        dst[i] = src[(bh * N + ts) * d_src + c0 + c];
    }
}

// out[bh, t, c] = sum_p parts[p][bh, flip ? N-1-t : t, c], summed in fp32.
template <typename T>
__global__ void __launch_bounds__(kBwdThreads)
sum_flip_kernel(const T* __restrict__ parts, int P, size_t part_elems, T* __restrict__ out, int N, int d, bool flip) {
    for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < part_elems;
         i += (size_t)gridDim.x * blockDim.x) {
        const int c = (int)(i % d);
        const size_t row = i / d;
        const int t = (int)(row % N);
        const size_t bh = row / N;
        const size_t src = (bh * N + (flip ? N - 1 - t : t)) * d + c;
        float s = 0.f;
        for (int p = 0; p < P; ++p) s += ld_elem(parts + (size_t)p * part_elems + src);
        st_elem(out + i, s);
    }
}

// Reversed, shifted gates: gf[bh, i] = g[bh, N - i] for i >= 1, gf[bh, 0] = 0.
__global__ void __launch_bounds__(kBwdThreads)
gate_flip_kernel(const float* __restrict__ g, float* __restrict__ gf, int N, size_t total) {
    for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < total; i += (size_t)gridDim.x * blockDim.x) {
        const int t = (int)(i % N);
        const size_t bh = i / N;
        gf[i] = t == 0 ? 0.f : g[bh * N + (N - t)];
    }
}

// Decay gradient from a_t = q_t . dQ_t - k_t . dK_t, one block per (b, h):
// gated: dg[bh, t] = sum_{u >= t} a_u; fixed: atomically adds (1/gamma_h) sum_t t a_t
// to dgamma[h] (zeroed by the caller). A warp computes each a_t; the block then scans
// from the end of the sequence in tiles of kBwdThreads tokens with a running carry.
template <typename T, bool GATED>
__global__ void __launch_bounds__(kBwdThreads)
decay_grad_kernel(const T* __restrict__ q, const T* __restrict__ dq, const T* __restrict__ k,
                  const T* __restrict__ dk, const float* __restrict__ decay, float* __restrict__ out, int H, int N,
                  int dk_dim) {
    __shared__ float a_s[kBwdThreads];
    __shared__ float warp_s[kBwdThreads / 32];
    const int bh = blockIdx.x;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const size_t base = (size_t)bh * N * dk_dim;
    float carry = 0.f;   // gated: sum of a_u over the tiles already scanned (later tokens)
    float weighted = 0.f;  // fixed: this thread's share of sum_t t a_t
    for (int tile_end = N; tile_end > 0; tile_end -= kBwdThreads) {
        const int tile0 = max(0, tile_end - kBwdThreads);
        const int len = tile_end - tile0;
        for (int j = warp; j < len; j += kBwdThreads / 32) {
            const size_t row = base + (size_t)(tile0 + j) * dk_dim;
            float s = 0.f;
            for (int c = lane; c < dk_dim; c += 32)
                s += ld_elem(q + row + c) * ld_elem(dq + row + c) - ld_elem(k + row + c) * ld_elem(dk + row + c);
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
            if (lane == 0) a_s[j] = s;
        }
        __syncthreads();
        const int j = threadIdx.x;
        const float a = j < len ? a_s[j] : 0.f;
        if (!GATED) {
            weighted += (float)(tile0 + j) * a;
        } else {
            // inclusive suffix sum inside the tile: reverse index r = len - 1 - j
            float x = a;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const float y = __shfl_down_sync(0xffffffffu, x, o);
                if (lane + o < 32) x += y;
            }
            if (lane == 0) warp_s[warp] = x;  // warp total (suffix sum at its first lane)
            __syncthreads();
            float later = 0.f;  // totals of the warps after this one
            for (int w2 = warp + 1; w2 < kBwdThreads / 32; ++w2) later += warp_s[w2];
            if (j < len) out[(size_t)bh * N + tile0 + j] = x + later + carry;
            float total = 0.f;
            for (int w2 = 0; w2 < kBwdThreads / 32; ++w2) total += warp_s[w2];
            carry += total;
        }
        __syncthreads();
    }
    if (!GATED) {
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) weighted += __shfl_xor_sync(0xffffffffu, weighted, o);
        if (lane == 0) warp_s[warp] = weighted;
        __syncthreads();
        if (threadIdx.x == 0) {
            float s = 0.f;
            for (int w2 = 0; w2 < kBwdThreads / 32; ++w2) s += warp_s[w2];
            atomicAdd(out + bh % H, s / decay[bh % H]);
        }
    }
}

}  // namespace ret
