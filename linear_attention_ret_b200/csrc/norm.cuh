// Multi-scale retention output epilogue: per-head RMSNorm without affine weights,
// times the swish of the gate projection ("Retentive Network (RetNet) 详解",
// section 3.2: multi-scale retention adds a gate and a normalisation to
// retention; the Gated RetNet page's GateRetention module: subln normalises
// each head over its dimension, g_proj feeds a swish gate):
//   y[b, n, h, :] = swish(gate[b, n, h, :]) * o[b, h, n, :] * rsqrt(mean_c o[b, h, n, c]^2 + eps),
//   swish(x) = x / (1 + e^-x).
// o is the retention output [B, H, N, dv]; gate and y are token-major
// [B, N, H, dv], the layout the module's projections use, so the transpose
// happens here on the way through.
//
// One pass over HBM: every row's O and gate are read once and y written once.
// A group of LPR lanes takes one row; each lane holds CH 16-byte chunks of O
// and of the gate in registers, so all of a row's loads are in flight before
// the sum of squares is reduced across the group with shuffles.
#pragma once

#include "common.cuh"

namespace ret {

constexpr int kNormThreads = 256;

template <typename T> struct Vec16;
template <> struct Vec16<float> {
    static constexpr int kE = 4;
    static __device__ __forceinline__ void unpack(const uint4& u, float* f) {
        f[0] = __uint_as_float(u.x); f[1] = __uint_as_float(u.y);
        f[2] = __uint_as_float(u.z); f[3] = __uint_as_float(u.w);
    }
    static __device__ __forceinline__ uint4 pack(const float* f) {
        return make_uint4(__float_as_uint(f[0]), __float_as_uint(f[1]), __float_as_uint(f[2]), __float_as_uint(f[3]));
    }
};
template <> struct Vec16<__nv_bfloat16> {
    static constexpr int kE = 8;
    static __device__ __forceinline__ void unpack(const uint4& u, float* f) {
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            __nv_bfloat162 b;
            memcpy(&b, &w[i], 4);
            const float2 x = __bfloat1622float2(b);
            f[2 * i] = x.x;
            f[2 * i + 1] = x.y;
        }
    }
    static __device__ __forceinline__ uint4 pack(const float* f) {
        uint32_t w[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const __nv_bfloat162 b = __floats2bfloat162_rn(f[2 * i], f[2 * i + 1]);
            memcpy(&w[i], &b, 4);
        }
        return make_uint4(w[0], w[1], w[2], w[3]);
    }
};

// swish(x) = x / (1 + e^-x) = x * rcp(1 + 2^(-x log2 e)) with the hardware ex2 and rcp
// (flush-to-zero forms; relative errors about 2^-22 and 1 ulp): five instructions. The
// flushes only touch e^-x below 2^-126 (where 1 + e^-x rounds to 1 anyway) and results
// below 2^-126 in magnitude (x < -87, where swish(x) is under 1e-36).
__device__ __forceinline__ float swish(float x) {
    float e, r;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(e) : "f"(-x * kLog2e));
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(1.f + e));
    return x * r;
}

// Source row of o and destination row of y for token-major row index r = (b N + n) H + h.
__device__ __forceinline__ void norm_rows(size_t r, int H, int N, size_t& o_row, size_t& y_row) {
    const int h = (int)(r % H);
    const size_t bn = r / H;
    const int n = (int)(bn % N);
    const size_t b = bn / N;
    o_row = (b * H + h) * N + n;
    y_row = r;
}

// Vector path: dv * sizeof(T) a multiple of 16 and all pointers 16-byte aligned.
// LPR lanes per row (a power of two dividing 32), CH chunks per lane.
template <typename T, int LPR, int CH>
__global__ void __launch_bounds__(kNormThreads)
norm_gate_vec_kernel(const T* __restrict__ o, const T* gate, T* y, int H, int N, int dv, float eps, size_t rows) {
    constexpr int kE = Vec16<T>::kE;
    constexpr int kRowsPerWarp = 32 / LPR;
    const int lane = threadIdx.x & 31, sub = lane % LPR;
    const int chunks = dv / kE;
    const float inv_dv = 1.f / (float)dv;
    const size_t warps = (size_t)gridDim.x * (kNormThreads / 32);
    for (size_t w = (size_t)blockIdx.x * (kNormThreads / 32) + (threadIdx.x >> 5); w * kRowsPerWarp < rows;
         w += warps) {
        const size_t r = w * kRowsPerWarp + lane / LPR;
        const bool live = r < rows;
        size_t o_row = 0, y_row = 0;
        if (live) norm_rows(r, H, N, o_row, y_row);
        const uint4* op = reinterpret_cast<const uint4*>(o + o_row * dv);
        const uint4* gp = reinterpret_cast<const uint4*>(gate + y_row * dv);
        uint4 ov[CH], gv[CH];
#pragma unroll
        for (int c = 0; c < CH; ++c) {
            const int idx = sub + c * LPR;
            if (live && idx < chunks) {
                ov[c] = __ldcs(op + idx);
                gv[c] = __ldcs(gp + idx);
            } else {
                ov[c] = make_uint4(0, 0, 0, 0);
                gv[c] = make_uint4(0, 0, 0, 0);
            }
        }
        float ss = 0.f;
#pragma unroll
        for (int c = 0; c < CH; ++c) {
            float f[kE];
            Vec16<T>::unpack(ov[c], f);
#pragma unroll
            for (int e = 0; e < kE; ++e) ss = fmaf(f[e], f[e], ss);
        }
#pragma unroll
        for (int off = LPR / 2; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
        const float inv_rms = rsqrtf(ss * inv_dv + eps);
        uint4* yp = reinterpret_cast<uint4*>(y + y_row * dv);
#pragma unroll
        for (int c = 0; c < CH; ++c) {
            const int idx = sub + c * LPR;
            if (live && idx < chunks) {
                float f[kE], g[kE];
                Vec16<T>::unpack(ov[c], f);
                Vec16<T>::unpack(gv[c], g);
#pragma unroll
                for (int e = 0; e < kE; ++e) f[e] = swish(g[e]) * (f[e] * inv_rms);
                yp[idx] = Vec16<T>::pack(f);
            }
        }
    }
}

// Any dv and alignment: one warp per row, two passes over the row (the second
// from L1/L2).
template <typename T>
__global__ void __launch_bounds__(kNormThreads)
norm_gate_scalar_kernel(const T* __restrict__ o, const T* gate, T* y, int H, int N, int dv, float eps, size_t rows) {
    const int lane = threadIdx.x & 31;
    const size_t warps = (size_t)gridDim.x * (kNormThreads / 32);
    for (size_t r = (size_t)blockIdx.x * (kNormThreads / 32) + (threadIdx.x >> 5); r < rows; r += warps) {
        size_t o_row, y_row;
        norm_rows(r, H, N, o_row, y_row);
        const T* op = o + o_row * dv;
        float ss = 0.f;
        for (int c = lane; c < dv; c += 32) {
            const float x = ld_elem(op + c);
            ss = fmaf(x, x, ss);
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
        const float inv_rms = rsqrtf(ss / (float)dv + eps);
        for (int c = lane; c < dv; c += 32)
            st_elem(y + y_row * dv + c, swish(ld_elem(gate + y_row * dv + c)) * (ld_elem(op + c) * inv_rms));
    }
}

}  // namespace ret
