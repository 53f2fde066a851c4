// CUDA-core (FFMA) retention kernels: the parallel form and the chunkwise form
// (fixed per-head gamma or per-token gate). They serve fp32 inputs, where the
// 1e-5 accuracy target rules out bf16/TF32 tensor-core products, and every
// shape the tensor-core kernel does not take.
#pragma once

#include "common.cuh"

namespace ret {

// ============================================================== parallel form
// "RetNet retention mechanism" (aiqz.cc), section 并行训练 (parallel training):
// R = (Q K^T (.) D) V with D_nm = gamma^(n-m) for n >= m, else 0 (section 衰减矩阵).
// One CTA owns PQ query rows x PV value columns of one head and walks the key
// tiles up to the causal limit; scores never leave shared memory.
constexpr int kParQ = 32, kParK = 32, kParV = 64, kParD = 32, kParThreads = 256;

template <typename T>
__global__ void __launch_bounds__(kParThreads)
parallel_simt_kernel(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
                     const float* __restrict__ gamma, T* __restrict__ o, int H, int N, int dk, int dv) {
    __shared__ float Qs[kParQ][kParD + 1];
    __shared__ float Ks[kParK][kParD + 1];
    __shared__ float Vs[kParK][kParV];
    __shared__ float Ps[kParQ][kParK + 1];
    const int bh = blockIdx.z;
    const int n0 = blockIdx.x * kParQ;
    const int c0 = blockIdx.y * kParV;
    const int tid = threadIdx.x;
    const float lg = log2f(gamma[bh % H]);
    const T* Q = q + (size_t)bh * N * dk;
    const T* K = k + (size_t)bh * N * dk;
    const T* V = v + (size_t)bh * N * dv;
    T* O = o + (size_t)bh * N * dv;

    const int si = tid >> 3, sj0 = (tid & 7) * 4;  // score tile: row, 4 keys
    const int oi = tid >> 3, oc = tid & 7;          // output tile: row, columns oc + 8u
    float acc[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) acc[u] = 0.f;
    const int n_last = min(n0 + kParQ, N) - 1;

    for (int m0 = 0; m0 <= n_last; m0 += kParK) {
        float s[4] = {0.f, 0.f, 0.f, 0.f};
        for (int d0 = 0; d0 < dk; d0 += kParD) {
            for (int e = tid; e < kParQ * kParD; e += kParThreads) {
                const int r = e / kParD, c = e % kParD, d = d0 + c;
                const int n = n0 + r, m = m0 + r;
                Qs[r][c] = (n < N && d < dk) ? ld_elem(Q + (size_t)n * dk + d) : 0.f;
                Ks[r][c] = (m < N && d < dk) ? ld_elem(K + (size_t)m * dk + d) : 0.f;
            }
            __syncthreads();
#pragma unroll 8
            for (int c = 0; c < kParD; ++c) {
                const float a = Qs[si][c];
#pragma unroll
                for (int u = 0; u < 4; ++u) s[u] = fmaf(a, Ks[sj0 + u][c], s[u]);
            }
            __syncthreads();
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int n = n0 + si, m = m0 + sj0 + u;
            Ps[si][sj0 + u] = (m <= n && m < N) ? s[u] * pow_int_log2(lg, n - m) : 0.f;
        }
        for (int e = tid; e < kParK * kParV; e += kParThreads) {
            const int r = e / kParV, c = e % kParV, m = m0 + r, cc = c0 + c;
            Vs[r][c] = (m < N && cc < dv) ? ld_elem(V + (size_t)m * dv + cc) : 0.f;
        }
        __syncthreads();
#pragma unroll 4
        for (int j = 0; j < kParK; ++j) {
            const float p = Ps[oi][j];
#pragma unroll
            for (int u = 0; u < 8; ++u) acc[u] = fmaf(p, Vs[j][oc + 8 * u], acc[u]);
        }
        __syncthreads();
    }
    const int n = n0 + oi;
    if (n < N) {
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const int c = c0 + oc + 8 * u;
            if (c < dv) st_elem(O + (size_t)n * dv + c, acc[u]);
        }
    }
}

// ============================================================= chunkwise form
// "RetNet retention mechanism" (aiqz.cc), section 块级循环 (chunkwise recurrence),
// and for GATED the gated-RetNet chunk_gate_retention (pwwt.cn page):
//   O_[i] = (Q K^T (.) D) V + diag(r) Q S_[i-1]
//   S_[i] = decay * S_[i-1] + K^T diag(zeta) V
// fixed gamma: D_jm = gamma^(j-m), r_j = gamma^(j+1), zeta_m = gamma^(L-1-m), decay = gamma^L
// gated:       D_jm = exp(Gl_j-Gl_m), r_j = exp(Gl_j), zeta_m = exp(Gl_{L-1}-Gl_m), decay = exp(Gl_{L-1})
// One CTA owns one head and a 64-column slice of dv; its state slice [dk][64]
// stays in shared memory for the whole sequence.
constexpr int kCwV = 64, kCwC = 64, kCwD = 32, kCwThreads = 256;

__host__ __device__ constexpr size_t chunkwise_simt_smem_bytes(int dk) {
    return sizeof(float) * ((size_t)dk * kCwV + kCwC * (kCwC + 1) + kCwC * kCwV + 2 * kCwC * (kCwD + 1) + 3 * kCwC + 1);
}

template <typename T, bool GATED>
__global__ void __launch_bounds__(kCwThreads)
chunkwise_simt_kernel(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
                      const float* __restrict__ decay_in, const float* __restrict__ state_in,
                      float* __restrict__ state_out, T* __restrict__ o,
                      int H, int N, int dk, int dv, int chunk) {
    extern __shared__ float smem[];
    float* S = smem;                        // [dk][kCwV]
    float* A = S + (size_t)dk * kCwV;       // [kCwC][kCwC+1]
    float* Vt = A + kCwC * (kCwC + 1);      // [kCwC][kCwV]
    float* Qp = Vt + kCwC * kCwV;           // [kCwC][kCwD+1]
    float* Kp = Qp + kCwC * (kCwD + 1);     // [kCwC][kCwD+1]
    float* cum = Kp + kCwC * (kCwD + 1);    // gated: inclusive in-chunk cumsum of g, log2 units
    float* rr = cum + kCwC;                 // row factor of the cross term
    float* zz = rr + kCwC;                  // key weight of the state update
    float* dec = zz + kCwC;                 // [1] chunk decay of the state

    const int bh = blockIdx.y;
    const int c0 = blockIdx.x * kCwV;
    const int ncols = min(kCwV, dv - c0);
    const int tid = threadIdx.x;
    const T* Q = q + (size_t)bh * N * dk;
    const T* K = k + (size_t)bh * N * dk;
    const T* V = v + (size_t)bh * N * dv;
    T* O = o + (size_t)bh * N * dv;
    const float* G = GATED ? decay_in + (size_t)bh * N : nullptr;
    const float lg = GATED ? 0.f : log2f(decay_in[bh % H]);

    for (int e = tid; e < dk * kCwV; e += kCwThreads) {
        const int d = e / kCwV, c = e % kCwV;
        S[e] = (state_in != nullptr && c < ncols) ? state_in[((size_t)bh * dk + d) * dv + c0 + c] : 0.f;
    }

    const int Ce = min(chunk, kCwC);
    const int ai = tid >> 2, aj0 = (tid & 3) * 16;  // score / output row and column base
    for (int t0 = 0; t0 < N; t0 += Ce) {
        const int L = min(Ce, N - t0);
        __syncthreads();
        if (tid == 0) {
            if (GATED) {
                float acc = 0.f;
                for (int j = 0; j < L; ++j) { acc += G[t0 + j] * kLog2e; cum[j] = acc; }
                dec[0] = exp2f(cum[L - 1]);
            } else {
                dec[0] = pow_int_log2(lg, L);
            }
        }
        __syncthreads();
        for (int j = tid; j < L; j += kCwThreads) {
            if (GATED) {
                rr[j] = exp2f(cum[j]);
                zz[j] = exp2f(cum[L - 1] - cum[j]);
            } else {
                rr[j] = pow_int_log2(lg, j + 1);
                zz[j] = pow_int_log2(lg, L - 1 - j);
            }
        }
        // scores A = Q_[i] K_[i]^T, dk streamed in pieces
        float s[16];
#pragma unroll
        for (int u = 0; u < 16; ++u) s[u] = 0.f;
        for (int d0 = 0; d0 < dk; d0 += kCwD) {
            for (int e = tid; e < kCwC * kCwD; e += kCwThreads) {
                const int r = e / kCwD, c = e % kCwD, d = d0 + c;
                const bool ok = r < L && d < dk;
                Qp[r * (kCwD + 1) + c] = ok ? ld_elem(Q + (size_t)(t0 + r) * dk + d) : 0.f;
                Kp[r * (kCwD + 1) + c] = ok ? ld_elem(K + (size_t)(t0 + r) * dk + d) : 0.f;
            }
            __syncthreads();
#pragma unroll 4
            for (int c = 0; c < kCwD; ++c) {
                const float a = Qp[ai * (kCwD + 1) + c];
#pragma unroll
                for (int u = 0; u < 16; ++u) s[u] = fmaf(a, Kp[(aj0 + u) * (kCwD + 1) + c], s[u]);
            }
            __syncthreads();
        }
        // decay mask D (causal, generated here rather than loaded)
#pragma unroll
        for (int u = 0; u < 16; ++u) {
            const int j = ai, m = aj0 + u;
            float w = 0.f;
            if (m <= j && j < L) w = GATED ? exp2f(cum[j] - cum[m]) : pow_int_log2(lg, j - m);
            A[j * (kCwC + 1) + m] = s[u] * w;
        }
        for (int e = tid; e < kCwC * kCwV; e += kCwThreads) {
            const int r = e / kCwV, c = e % kCwV;
            Vt[e] = (r < L && c < ncols) ? ld_elem(V + (size_t)(t0 + r) * dv + c0 + c) : 0.f;
        }
        __syncthreads();
        // inner term (A V) and cross term r_j (Q S_[i-1]) for row ai, columns (tid&3) + 4u
        const int oc = tid & 3;
        float acc[16], cr[16];
#pragma unroll
        for (int u = 0; u < 16; ++u) { acc[u] = 0.f; cr[u] = 0.f; }
        for (int m = 0; m < L; ++m) {
            const float p = A[ai * (kCwC + 1) + m];
#pragma unroll
            for (int u = 0; u < 16; ++u) acc[u] = fmaf(p, Vt[m * kCwV + oc + 4 * u], acc[u]);
        }
        for (int d0 = 0; d0 < dk; d0 += kCwD) {
            __syncthreads();
            for (int e = tid; e < kCwC * kCwD; e += kCwThreads) {
                const int r = e / kCwD, c = e % kCwD, d = d0 + c;
                Qp[r * (kCwD + 1) + c] = (r < L && d < dk) ? ld_elem(Q + (size_t)(t0 + r) * dk + d) : 0.f;
            }
            __syncthreads();
            const int dlim = min(kCwD, dk - d0);
            for (int c = 0; c < dlim; ++c) {
                const float a = Qp[ai * (kCwD + 1) + c];
                const float* Srow = S + (size_t)(d0 + c) * kCwV;
#pragma unroll
                for (int u = 0; u < 16; ++u) cr[u] = fmaf(a, Srow[oc + 4 * u], cr[u]);
            }
        }
        if (ai < L) {
            const float r = rr[ai];
#pragma unroll
            for (int u = 0; u < 16; ++u) {
                const int c = oc + 4 * u;
                if (c < ncols) st_elem(O + (size_t)(t0 + ai) * dv + c0 + c, fmaf(r, cr[u], acc[u]));
            }
        }
        __syncthreads();
        // state update: S = decay S + K^T (zeta (.) V)
        for (int e = tid; e < L * kCwV; e += kCwThreads) Vt[e] *= zz[e / kCwV];
        const float decay = dec[0];
        const int sd = tid >> 3, sc = tid & 7;  // state piece: row sd, columns sc + 8u
        for (int d0 = 0; d0 < dk; d0 += kCwD) {
            __syncthreads();
            for (int e = tid; e < kCwC * kCwD; e += kCwThreads) {
                const int r = e / kCwD, c = e % kCwD, d = d0 + c;
                Kp[r * (kCwD + 1) + c] = (r < L && d < dk) ? ld_elem(K + (size_t)(t0 + r) * dk + d) : 0.f;
            }
            __syncthreads();
            if (d0 + sd < dk) {
                float sum[8];
#pragma unroll
                for (int u = 0; u < 8; ++u) sum[u] = 0.f;
                for (int m = 0; m < L; ++m) {
                    const float kk = Kp[m * (kCwD + 1) + sd];
#pragma unroll
                    for (int u = 0; u < 8; ++u) sum[u] = fmaf(kk, Vt[m * kCwV + sc + 8 * u], sum[u]);
                }
                float* Srow = S + (size_t)(d0 + sd) * kCwV;
#pragma unroll
                for (int u = 0; u < 8; ++u) Srow[sc + 8 * u] = fmaf(decay, Srow[sc + 8 * u], sum[u]);
            }
        }
    }
    __syncthreads();
    if (state_out != nullptr) {
        for (int e = tid; e < dk * kCwV; e += kCwThreads) {
            const int d = e / kCwV, c = e % kCwV;
            if (c < ncols) state_out[((size_t)bh * dk + d) * dv + c0 + c] = S[e];
        }
    }
}

}  // namespace ret
