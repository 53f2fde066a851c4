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
// This file holds the data-movement and reduction kernels of that composition:
// one warp per row, whole 16-byte chunks where rows allow it.
#pragma once

#include "common.cuh"

namespace ret {

constexpr int kBwdThreads = 256;
constexpr int kBwdWarps = kBwdThreads / 32;

// 16-byte chunks of a row: VEC when every row start and width is a whole number of
// chunks (checked by the caller), else element by element.
template <typename T, bool VEC>
struct RowIo {
    static constexpr int kE = VEC ? 16 / (int)sizeof(T) : 1;
};

// Rows one warp moves per iteration of the copy kernels (their loads all in flight
// before the stores).
constexpr int kCopyRows = 4;

// dst[bh, t, :w] = src[bh, flip ? N-1-t : t, c0 : c0+w] (a column slice, optionally
// time-reversed). src rows are d_src wide. A warp takes kCopyRows destination rows at a
// time, 64 chunks of each per pass.
template <typename T, bool VEC>
__global__ void __launch_bounds__(kBwdThreads)
slice_flip_kernel(const T* __restrict__ src, T* __restrict__ dst, int N, int d_src, int c0, int w, bool flip,
                  size_t rows) {
    const int lane = threadIdx.x & 31;
    const size_t nw = (size_t)gridDim.x * kBwdWarps;
    for (size_t r0 = ((size_t)blockIdx.x * kBwdWarps + (threadIdx.x >> 5)) * kCopyRows; r0 < rows;
         r0 += nw * kCopyRows) {
        if constexpr (VEC) {
            constexpr int kE = RowIo<T, true>::kE;
            const int cpr = w / kE;  // chunks per row
            for (int cb = 0; cb < cpr; cb += 64) {
                uint4 buf[kCopyRows][2];
#pragma unroll
                for (int i = 0; i < kCopyRows; ++i) {
                    const size_t r = r0 + i;
                    if (r >= rows) break;
                    const size_t bh = r / N;
                    const int t = (int)(r - bh * N);
                    const uint4* s = reinterpret_cast<const uint4*>(src + (bh * N + (flip ? N - 1 - t : t)) * d_src + c0);
#pragma unroll
                    for (int j = 0; j < 2; ++j) {
                        const int c = cb + lane + 32 * j;
                        if (c < cpr) buf[i][j] = __ldcs(s + c);
                    }
                }
#pragma unroll
                for (int i = 0; i < kCopyRows; ++i) {
                    const size_t r = r0 + i;
                    if (r >= rows) break;
                    uint4* d = reinterpret_cast<uint4*>(dst + r * w);
#pragma unroll
                    for (int j = 0; j < 2; ++j) {
                        const int c = cb + lane + 32 * j;
                        if (c < cpr) __stcs(d + c, buf[i][j]);
                    }
                }
            }
        } else {
            for (int i = 0; i < kCopyRows && r0 + i < rows; ++i) {
                const size_t r = r0 + i;
                const size_t bh = r / N;
                const int t = (int)(r - bh * N);
                const T* s = src + (bh * N + (flip ? N - 1 - t : t)) * d_src + c0;
                for (int c = lane; c < w; c += 32) dst[r * w + c] = s[c];
            }
        }
    }
}

// out[bh, t, :] = sum_p parts[p][bh, flip ? N-1-t : t, :], summed in fp32. One warp per row.
template <typename T, bool VEC>
__global__ void __launch_bounds__(kBwdThreads)
sum_flip_kernel(const T* __restrict__ parts, int P, size_t part_elems, T* __restrict__ out, int N, int d, bool flip,
                size_t rows) {
    const int lane = threadIdx.x & 31;
    for (size_t r = (size_t)blockIdx.x * kBwdWarps + (threadIdx.x >> 5); r < rows; r += (size_t)gridDim.x * kBwdWarps) {
        const size_t bh = r / N;
        const int t = (int)(r - bh * N);
        const T* s = parts + (bh * N + (flip ? N - 1 - t : t)) * d;
        T* o = out + r * d;
        if constexpr (VEC) {
            constexpr int kE = RowIo<T, true>::kE;
            for (int c = lane; c < d / kE; c += 32) {
                float acc[kE];
#pragma unroll
                for (int e = 0; e < kE; ++e) acc[e] = 0.f;
                for (int p = 0; p < P; ++p) {
                    const uint4 u = __ldcs(reinterpret_cast<const uint4*>(s + (size_t)p * part_elems) + c);
                    const T* x = reinterpret_cast<const T*>(&u);
#pragma unroll
                    for (int e = 0; e < kE; ++e) acc[e] += ld_elem(x + e);
                }
                uint4 u;
                T* y = reinterpret_cast<T*>(&u);
#pragma unroll
                for (int e = 0; e < kE; ++e) st_elem(y + e, acc[e]);
                reinterpret_cast<uint4*>(o)[c] = u;
            }
        } else {
            for (int c = lane; c < d; c += 32) {
                float acc = 0.f;
                for (int p = 0; p < P; ++p) acc += ld_elem(s + (size_t)p * part_elems + c);
                st_elem(o + c, acc);
            }
        }
    }
}

// Reversed, shifted gates: gf[bh, i] = g[bh, N - i] for i >= 1, gf[bh, 0] = 0.
__global__ void __launch_bounds__(kBwdThreads)
gate_flip_kernel(const float* __restrict__ g, float* __restrict__ gf, int N, size_t total) {
    for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < total; i += (size_t)gridDim.x * blockDim.x) {
        const size_t bh = i / N;
        const int t = (int)(i - bh * N);
        gf[i] = t == 0 ? 0.f : g[bh * N + (N - t)];
    }
}

// Tokens per block of the decay-gradient kernel.
constexpr int kGradTokens = 64;

// a_t = q_t . dQ_t - k_t . dK_t (= dL/dG_t) for a tile of kGradTokens tokens of one
// (b, h) (grid: token tiles x B*H; one warp per token).
// gated: out[bh, t] = a_t (the suffix sum follows in gate_grad_scan_kernel);
// fixed: adds (1/gamma_h) sum_t t a_t of the tile to dgamma[h] (zeroed by the caller).
template <typename T, bool VEC, bool GATED>
__global__ void __launch_bounds__(kBwdThreads)
decay_grad_kernel(const T* __restrict__ q, const T* __restrict__ dq, const T* __restrict__ k,
                  const T* __restrict__ dk, const float* __restrict__ decay, float* __restrict__ out, int H, int N,
                  int dk_dim) {
    __shared__ float warp_s[kBwdWarps];
    const int bh = blockIdx.y;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int t0 = blockIdx.x * kGradTokens;
    float weighted = 0.f;  // this warp's share of sum_t t a_t (fixed gamma)
    for (int j = warp; j < kGradTokens && t0 + j < N; j += kBwdWarps) {
        const int t = t0 + j;
        const size_t row = ((size_t)bh * N + t) * dk_dim;
        float s = 0.f;
        if constexpr (VEC) {
            constexpr int kE = RowIo<T, true>::kE;
            for (int c = lane; c < dk_dim / kE; c += 32) {
                const uint4 uq = __ldcs(reinterpret_cast<const uint4*>(q + row) + c);
                const uint4 udq = __ldcs(reinterpret_cast<const uint4*>(dq + row) + c);
                const uint4 uk = __ldcs(reinterpret_cast<const uint4*>(k + row) + c);
                const uint4 udk = __ldcs(reinterpret_cast<const uint4*>(dk + row) + c);
                const T* xq = reinterpret_cast<const T*>(&uq);
                const T* xdq = reinterpret_cast<const T*>(&udq);
                const T* xk = reinterpret_cast<const T*>(&uk);
                const T* xdk = reinterpret_cast<const T*>(&udk);
#pragma unroll
                for (int e = 0; e < kE; ++e)
                    s += ld_elem(xq + e) * ld_elem(xdq + e) - ld_elem(xk + e) * ld_elem(xdk + e);
            }
        } else {
            for (int c = lane; c < dk_dim; c += 32)
                s += ld_elem(q + row + c) * ld_elem(dq + row + c) - ld_elem(k + row + c) * ld_elem(dk + row + c);
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
        if (GATED) {
            if (lane == 0) out[(size_t)bh * N + t] = s;
        } else {
            weighted += (float)t * s;
        }
    }
    if (!GATED) {
        if (lane == 0) warp_s[warp] = weighted;
        __syncthreads();
        if (threadIdx.x == 0) {
            float s = 0.f;
            for (int w2 = 0; w2 < kBwdWarps; ++w2) s += warp_s[w2];
            atomicAdd(out + bh % H, s / decay[bh % H]);
        }
    }
}

// Dot product of two 16-byte chunks of T (8 bf16 or 4 fp32 values) in fp32. A bf16 value
// is the upper half of the fp32 value it stands for, so a 32-bit word holding two of them
// widens by a shift (the lower element) and a mask (the upper one).
template <typename T> struct Chunk16;
template <> struct Chunk16<__nv_bfloat16> {
    static __device__ __forceinline__ float dot(uint4 a, uint4 b) {
        const uint32_t x[4] = {a.x, a.y, a.z, a.w}, y[4] = {b.x, b.y, b.z, b.w};
        float s = 0.f;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            s = fmaf(__uint_as_float(x[i] << 16), __uint_as_float(y[i] << 16), s);
            s = fmaf(__uint_as_float(x[i] & 0xffff0000u), __uint_as_float(y[i] & 0xffff0000u), s);
        }
        return s;
    }
};
template <> struct Chunk16<float> {
    static __device__ __forceinline__ float dot(uint4 a, uint4 b) {
        float s = __uint_as_float(a.x) * __uint_as_float(b.x);
        s = fmaf(__uint_as_float(a.y), __uint_as_float(b.y), s);
        s = fmaf(__uint_as_float(a.z), __uint_as_float(b.z), s);
        return fmaf(__uint_as_float(a.w), __uint_as_float(b.w), s);
    }
};

// The same tile of a_t with more of the tile's loads in flight, for rows of C = dk_dim / kE
// 16-byte chunks with C a power of two (C = 1 << lc, at most 32): the tile's (token, chunk)
// pairs are spread over the block, C consecutive lanes per token, so no lane idles when
// C < 32, and each thread issues the loads of kFlatPer pairs before it uses any. Two pairs
// per thread with four blocks per SM kept in registers measured fastest (37.8 us for the
// 268 MB that the gated workload's shapes read, against 39-41 us with one or four pairs).
// gated: out[bh, t] = the tile's in-tile suffix sum s_t = sum_{u >= t in the tile} a_u and
// tile_tot[bh, tile] = the tile's total (gate_grad_carry_kernel then adds the later tiles');
// fixed: as decay_grad_kernel.
constexpr int kFlatPer = 2;
template <typename T, bool GATED>
__global__ void __launch_bounds__(kBwdThreads, 4)
decay_grad_flat_kernel(const T* __restrict__ q, const T* __restrict__ dq, const T* __restrict__ k,
                       const T* __restrict__ dk, const float* __restrict__ decay, float* __restrict__ out,
                       float* __restrict__ tile_tot, int H, int N, int lc) {
    __shared__ float a_s[kGradTokens];
    const int bh = blockIdx.y, t0 = blockIdx.x * kGradTokens;
    const int C = 1 << lc, items = kGradTokens << lc;
    const uint4* q4 = reinterpret_cast<const uint4*>(q);
    const uint4* dq4 = reinterpret_cast<const uint4*>(dq);
    const uint4* k4 = reinterpret_cast<const uint4*>(k);
    const uint4* dk4 = reinterpret_cast<const uint4*>(dk);
    for (int base = 0; base < items; base += kBwdThreads * kFlatPer) {
        uint4 uq[kFlatPer], udq[kFlatPer], uk[kFlatPer], udk[kFlatPer];
#pragma unroll
        for (int i = 0; i < kFlatPer; ++i) {
            const int idx = base + i * kBwdThreads + (int)threadIdx.x;
            const int j = idx >> lc;
            const bool ok = idx < items && t0 + j < N;
            const size_t off = (((size_t)bh * N + t0 + j) << lc) + (idx & (C - 1));
            const uint4 z = make_uint4(0u, 0u, 0u, 0u);
            uq[i] = ok ? __ldcs(q4 + off) : z;
            udq[i] = ok ? __ldcs(dq4 + off) : z;
            uk[i] = ok ? __ldcs(k4 + off) : z;
            udk[i] = ok ? __ldcs(dk4 + off) : z;
        }
        float part[kFlatPer];
#pragma unroll
        for (int i = 0; i < kFlatPer; ++i) part[i] = Chunk16<T>::dot(uq[i], udq[i]) - Chunk16<T>::dot(uk[i], udk[i]);
        for (int o = C >> 1; o > 0; o >>= 1) {
#pragma unroll
            for (int i = 0; i < kFlatPer; ++i) part[i] += __shfl_xor_sync(0xffffffffu, part[i], o);
        }
#pragma unroll
        for (int i = 0; i < kFlatPer; ++i) {
            const int idx = base + i * kBwdThreads + (int)threadIdx.x;
            if (idx < items && (idx & (C - 1)) == 0) a_s[idx >> lc] = t0 + (idx >> lc) < N ? part[i] : 0.f;
        }
    }
    __syncthreads();
    if (threadIdx.x >= 32) return;
    const int lane = threadIdx.x;  // warp 0: the tile's 64 values, two per lane
    const float x0 = a_s[2 * lane], x1 = a_s[2 * lane + 1];
    if constexpr (GATED) {
        const float run = x0 + x1;  // the lane's pair total
        float incl = run;           // suffix sum of the pair totals from this lane on
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const float y = __shfl_down_sync(0xffffffffu, incl, o);
            if (lane + o < 32) incl += y;
        }
        const float after = incl - run;  // every later pair of the tile
        const int t = t0 + 2 * lane;
        if (t < N) out[(size_t)bh * N + t] = run + after;
        if (t + 1 < N) out[(size_t)bh * N + t + 1] = x1 + after;
        if (lane == 0) tile_tot[(size_t)bh * gridDim.x + blockIdx.x] = incl;
    } else {
        float w = (float)(t0 + 2 * lane) * x0 + (float)(t0 + 2 * lane + 1) * x1;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) w += __shfl_xor_sync(0xffffffffu, w, o);
        if (lane == 0) atomicAdd(out + bh % H, w / decay[bh % H]);
    }
}

// dg[bh, t] += the totals of the tiles after t's tile (in place over the in-tile suffix sums
// of decay_grad_flat_kernel). Grid: (spans of kCarryTiles tiles, B*H). Each block sums the
// totals after its span, then walks its span's tiles from the last back.
constexpr int kCarryTiles = 16;
__global__ void __launch_bounds__(kBwdThreads)
gate_grad_carry_kernel(float* __restrict__ dg, const float* __restrict__ tile_tot, int N, int ntiles) {
    __shared__ float red[kBwdWarps];
    __shared__ float later_s[kCarryTiles];
    const int bh = blockIdx.y, tile0 = blockIdx.x * kCarryTiles;
    const float* tt = tile_tot + (size_t)bh * ntiles;
    float x = 0.f;
    for (int j = tile0 + kCarryTiles + (int)threadIdx.x; j < ntiles; j += kBwdThreads) x += tt[j];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (lane == 0) red[warp] = x;
    __syncthreads();
    if (threadIdx.x == 0) {
        float after = 0.f;
        for (int w2 = 0; w2 < kBwdWarps; ++w2) after += red[w2];
        for (int i = kCarryTiles - 1; i >= 0; --i) {
            later_s[i] = after;
            if (tile0 + i < ntiles) after += tt[tile0 + i];
        }
    }
    __syncthreads();
    float* row = dg + (size_t)bh * N;
    for (int e = threadIdx.x; e < kCarryTiles * kGradTokens; e += kBwdThreads) {
        const int t = tile0 * kGradTokens + e;
        if (t < N) row[t] += later_s[e / kGradTokens];
    }
}

// out[h] = sum_g rows[g, h]: the per-group dgamma rows of a host-buffer backward.
__global__ void __launch_bounds__(kBwdThreads)
sum_rows_kernel(const float* __restrict__ rows, int G, int H, float* __restrict__ out) {
    const int h = blockIdx.x * blockDim.x + threadIdx.x;
    if (h >= H) return;
    float s = 0.f;
    for (int g = 0; g < G; ++g) s += rows[(size_t)g * H + h];
    out[h] = s;
}

// In place: dg[bh, t] = sum_{u >= t} a[bh, u] (a suffix sum, since G_u includes g_t for
// every u >= t). One block of kScanThreads per (b, h): each thread owns kScanPer consecutive
// tokens of a span of kScanThreads * kScanPer (the whole row for N <= 16384), sums them from
// its last token back, and adds the totals of the later threads (a warp scan, then the warps'
// totals) and of the later spans (a running carry). All of a span's loads are in flight at once.
constexpr int kScanThreads = 1024, kScanPer = 16;
__global__ void __launch_bounds__(kScanThreads) gate_grad_scan_kernel(float* __restrict__ dg, int N) {
    __shared__ float warp_s[kScanThreads / 32];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    float* a = dg + (size_t)blockIdx.x * N;
    float carry = 0.f;
    for (int end = N; end > 0; end -= kScanThreads * kScanPer) {
        const int beg = max(0, end - kScanThreads * kScanPer);
        const int t0 = beg + threadIdx.x * kScanPer;
        float x[kScanPer];
#pragma unroll
        for (int i = 0; i < kScanPer; ++i) x[i] = t0 + i < end ? a[t0 + i] : 0.f;
        float run = 0.f;  // suffix sums inside the thread's tokens
#pragma unroll
        for (int i = kScanPer - 1; i >= 0; --i) {
            run += x[i];
            x[i] = run;
        }
        // inclusive suffix sum of the threads' totals inside the warp
        float incl = run;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const float y = __shfl_down_sync(0xffffffffu, incl, o);
            if (lane + o < 32) incl += y;
        }
        if (lane == 0) warp_s[warp] = incl;  // the warp's total
        __syncthreads();
        float later = 0.f, total = 0.f;
        for (int w2 = 0; w2 < kScanThreads / 32; ++w2) {
            if (w2 > warp) later += warp_s[w2];
            total += warp_s[w2];
        }
        const float after = incl - run + later + carry;  // every token after this thread's own
#pragma unroll
        for (int i = 0; i < kScanPer; ++i)
            if (t0 + i < end) a[t0 + i] = x[i] + after;
        carry += total;
        __syncthreads();
    }
}

}  // namespace ret
