// Recurrent (decode) step: "RetNet retention mechanism" (aiqz.cc), section
// 递归推理 (recurrent inference): S_n = gamma S_{n-1} + K_n^T V_n, R_n = Q_n S_n.
// Gated form (GATED, the chunk_gate_retention page's recurrent form): the decay of
// step n is exp(g_n) with g the step's log-decay per (b, h), S_n = e^{g_n} S_{n-1} + K_n^T V_n.
//
// The fp32 state [B, H, dk, dv] is read once and written once per step, so the
// kernel is bound by HBM bandwidth (0.5 flop per byte). Each thread owns four
// adjacent dv columns of one head and walks all dk rows: rows are 16-byte
// vectors, a warp touches 512 contiguous bytes per row, and the q.S reduction
// over dk stays inside the thread (no shuffles, no shared-memory reduction).
// Sixteen rows are in flight per thread to cover HBM latency; loads and stores
// use the streaming (evict-first) cache hint because the state is touched once.
#pragma once

#include "common.cuh"

namespace ret {

constexpr int kDecThreads = 128;
constexpr int kDecUnroll = 16;

// decay: gamma [H] (fixed), or g [B, H] natural-log step decays (GATED)
template <typename T, bool GATED>
__device__ __forceinline__ float step_decay(const float* decay, int bh, int H) {
    return GATED ? expf(decay[bh]) : decay[bh % H];
}

template <typename T, bool GATED>
__global__ void __launch_bounds__(kDecThreads)
recurrent_step_vec_kernel(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
                          const float* __restrict__ gamma, float* __restrict__ state, T* __restrict__ o,
                          int H, int dk, int dv) {
    extern __shared__ float qk_s[];  // q then k of this head, fp32
    const int bh = blockIdx.y;
    float* qs = qk_s;
    float* ks = qk_s + dk;
    for (int i = threadIdx.x; i < dk; i += blockDim.x) {
        qs[i] = ld_elem(q + (size_t)bh * dk + i);
        ks[i] = ld_elem(k + (size_t)bh * dk + i);
    }
    __syncthreads();
    const int cg = blockIdx.x * blockDim.x + threadIdx.x;  // column group: columns 4cg .. 4cg+3
    const int ngroups = dv >> 2;
    if (cg >= ngroups) return;
    const float gm = step_decay<T, GATED>(gamma, bh, H);
    const T* vp = v + (size_t)bh * dv + 4 * cg;
    const float v0 = ld_elem(vp), v1 = ld_elem(vp + 1), v2 = ld_elem(vp + 2), v3 = ld_elem(vp + 3);
    float4* S = reinterpret_cast<float4*>(state + (size_t)bh * dk * dv) + cg;
    float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
    int r = 0;
    for (; r + kDecUnroll <= dk; r += kDecUnroll) {
        float4 s[kDecUnroll];
#pragma unroll
        for (int u = 0; u < kDecUnroll; ++u) s[u] = __ldcs(S + (size_t)(r + u) * ngroups);
#pragma unroll
        for (int u = 0; u < kDecUnroll; ++u) {
            const float kr = ks[r + u], qr = qs[r + u];
            s[u].x = fmaf(gm, s[u].x, kr * v0);
            s[u].y = fmaf(gm, s[u].y, kr * v1);
            s[u].z = fmaf(gm, s[u].z, kr * v2);
            s[u].w = fmaf(gm, s[u].w, kr * v3);
            __stcs(S + (size_t)(r + u) * ngroups, s[u]);
            a0 = fmaf(qr, s[u].x, a0);
            a1 = fmaf(qr, s[u].y, a1);
            a2 = fmaf(qr, s[u].z, a2);
            a3 = fmaf(qr, s[u].w, a3);
        }
    }
    for (; r < dk; ++r) {
        float4 s = __ldcs(S + (size_t)r * ngroups);
        const float kr = ks[r], qr = qs[r];
        s.x = fmaf(gm, s.x, kr * v0);
        s.y = fmaf(gm, s.y, kr * v1);
        s.z = fmaf(gm, s.z, kr * v2);
        s.w = fmaf(gm, s.w, kr * v3);
        __stcs(S + (size_t)r * ngroups, s);
        a0 = fmaf(qr, s.x, a0);
        a1 = fmaf(qr, s.y, a1);
        a2 = fmaf(qr, s.z, a2);
        a3 = fmaf(qr, s.w, a3);
    }
    T* op = o + (size_t)bh * dv + 4 * cg;
    st_elem(op, a0);
    st_elem(op + 1, a1);
    st_elem(op + 2, a2);
    st_elem(op + 3, a3);
}

// Scalar variant for dv not a multiple of 4 or a state that is not 16-byte aligned.
template <typename T, bool GATED>
__global__ void __launch_bounds__(kDecThreads)
recurrent_step_scalar_kernel(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
                             const float* __restrict__ gamma, float* __restrict__ state, T* __restrict__ o,
                             int H, int dk, int dv) {
    extern __shared__ float qk_s[];
    const int bh = blockIdx.y;
    float* qs = qk_s;
    float* ks = qk_s + dk;
    for (int i = threadIdx.x; i < dk; i += blockDim.x) {
        qs[i] = ld_elem(q + (size_t)bh * dk + i);
        ks[i] = ld_elem(k + (size_t)bh * dk + i);
    }
    __syncthreads();
    const int c = blockIdx.x * blockDim.x + threadIdx.x;
    if (c >= dv) return;
    const float gm = step_decay<T, GATED>(gamma, bh, H);
    const float vc = ld_elem(v + (size_t)bh * dv + c);
    float* S = state + (size_t)bh * dk * dv + c;
    float acc = 0.f;
    for (int r = 0; r < dk; ++r) {
        const float s = fmaf(gm, S[(size_t)r * dv], ks[r] * vc);
        S[(size_t)r * dv] = s;
        acc = fmaf(qs[r], s, acc);
    }
    st_elem(o + (size_t)bh * dv + c, acc);
}

}  // namespace ret
